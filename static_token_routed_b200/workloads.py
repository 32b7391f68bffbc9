"""Seeded synthetic inputs for the L³ (Large Lookup Layer) forward pass.

This module only draws random numbers and lays them out; it contains none of
the layer's arithmetic. It is the one module shared by the CUDA path's tests
and bench and by the CPU oracle's tests.

The pages ("L³: Large Lookup Layers", Tseng & De Sa) train on FineWeb-Edu
with a 180K-entry BPE tokenizer and an LZW allocation (papernotes.org note,
训练策略; kimjy99 review, Experiments). None of that is available here, so the
synthetic inputs below stand in for it with the same shapes:

* allocation D = {d_t}: Zipf weights r^-s over token rank r = t + 1, clipped
  to [1, k] and renormalised to sum exactly v (near-Zipf, heavy tokens at k and
  most at 1, as in Fig. 5 of the sciencestack page);
* token IDs: i.i.d. truncated Zipf over the same ranks, so frequent tokens are
  the heavily allocated ones;
* values: x ~ N(0, 1/d_in), W_K ~ N(0, 1/d_in), W_V ~ N(0, 1/d_emb),
  W_up ~ N(0, 1/d_emb), W_mix ~ N(0, 1/(d_up + d_in)), LayerNorm gamma = 1,
  beta = 0; rounded once to the working dtype.

Each tensor has its own random stream keyed by (seed, tensor tag, chunk), so
a tensor does not change when another one is added, and large tensors are
drawn in parallel chunks with a result that does not depend on thread count.
"""
from __future__ import annotations

import dataclasses
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

_CHUNK = 1 << 24  # elements per independent random stream of a large tensor

_TAGS = {"x": 1, "W_K": 2, "W_V": 3, "W_up": 4, "W_mix": 5, "ids": 6, "corpus": 7}


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and recipe of one synthetic L³ batch."""

    name: str
    vocab: int          # |tau|
    v: int              # embedding budget, sum of d_t
    k: int              # cap on d_t
    d_in: int
    d_emb: int
    d_up: int
    d_out: int
    n_tokens: int       # N
    dtype: str          # "bf16" or "fp32"
    alloc: str          # "zipf", "dense64" or "uniform"
    ids: str            # "zipf", "zipf_distinct", "uniform_first64" or "uniform"
    table_seed: int     # seed of the allocation and of the weight tables
    batch_seed: int     # seed of token IDs and x
    zipf_s: float = 1.1
    tied: bool = False  # W_V is W_K (one table serves as keys and values; d_in = d_emb)

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32


def _cfg2(**kw):
    base = dict(vocab=32000, v=128000, k=256, d_in=1024, d_emb=256, d_up=1024,
                d_out=1024, dtype="bf16", alloc="zipf", ids="zipf")
    base.update(kw)
    return base


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny_fp32", vocab=1000, v=4000, k=64, d_in=128, d_emb=128, d_up=128,
                 d_out=128, n_tokens=512, dtype="fp32", alloc="zipf", ids="zipf",
                 table_seed=0, batch_seed=0),
        Workload("small_bf16", n_tokens=16384, table_seed=1, batch_seed=1, **_cfg2()),
        Workload("paper_shaped", vocab=180000, v=710000, k=512, d_in=2048, d_emb=512,
                 d_up=2048, d_out=2048, n_tokens=65536, dtype="bf16", alloc="zipf",
                 ids="zipf", table_seed=2, batch_seed=2),
        # same tables and allocation as small_bf16; one token per ID group
        Workload("decode", n_tokens=256, table_seed=1, batch_seed=3,
                 **_cfg2(ids="zipf_distinct")),
        # IDs 0..63 hold d_t = 512 and take every token: large dense groups
        Workload("dense_stress", n_tokens=131072, table_seed=4, batch_seed=4,
                 **_cfg2(k=512, alloc="dense64", ids="uniform_first64")),
        # d_t = 4 for every ID, uniform IDs: every group is short
        Workload("uniform", n_tokens=131072, table_seed=4, batch_seed=4,
                 **_cfg2(alloc="uniform", ids="uniform")),
        # paper-shaped allocation and batch with one table for keys and values
        # (d_in = d_emb = 512)
        Workload("paper_tied", vocab=180000, v=710000, k=512, d_in=512, d_emb=512,
                 d_up=2048, d_out=2048, n_tokens=65536, dtype="bf16", alloc="zipf",
                 ids="zipf", table_seed=5, batch_seed=5, tied=True),
    ]
}


def with_tokens(w: Workload, n_tokens: int, batch_seed: int | None = None) -> Workload:
    """Same tables and allocation, a different batch size (and batch seed)."""
    return dataclasses.replace(
        w, n_tokens=n_tokens, batch_seed=w.batch_seed if batch_seed is None else batch_seed)


def _rng(seed: int, tag: str, chunk: int = 0) -> np.random.Generator:
    return np.random.default_rng([seed, _TAGS[tag], chunk])


def zipf_weights(vocab: int, s: float) -> np.ndarray:
    r = np.arange(1, vocab + 1, dtype=np.float64)
    return r ** (-s)


def zipf_allocation(vocab: int, v: int, k: int, s: float) -> np.ndarray:
    """d_t for t = 0..vocab-1: Zipf r^-s clipped to [1, k], summing exactly to v.

    lambda is bisected until sum(clip(lambda * w, 1, k)) >= v; the clipped
    values are floored and the missing rows go one each to the IDs with the
    largest fractional part (ties: lower rank), skipping IDs already at k.
    """
    if not (vocab <= v <= k * vocab):
        raise ValueError("need vocab <= v <= k * vocab")
    w = zipf_weights(vocab, s)

    def total(lam):
        return np.clip(lam * w, 1.0, k).sum()

    lo, hi = 0.0, float(k) / w[-1]
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if total(mid) >= v:
            hi = mid
        else:
            lo = mid
    c = np.clip(hi * w, 1.0, k)
    d = np.floor(c).astype(np.int64)
    frac = c - d
    rem = int(v - d.sum())
    if rem > 0:
        cand = np.nonzero(d < k)[0]
        order = cand[np.lexsort((cand, -frac[cand]))]
        d[order[:rem]] += 1
    elif rem < 0:
        cand = np.nonzero(d > 1)[0]
        order = cand[np.lexsort((cand, frac[cand]))]
        d[order[:-rem]] -= 1
    return d


def dense64_allocation(vocab: int, v: int, k: int) -> np.ndarray:
    """IDs 0..63 get k rows; the rest of v is spread as evenly as possible
    over the other IDs, extra rows going to the lowest IDs."""
    d = np.empty(vocab, dtype=np.int64)
    d[:64] = k
    rest = v - 64 * k
    m = vocab - 64
    base, extra = divmod(rest, m)
    d[64:] = base
    d[64:64 + extra] += 1
    return d


def uniform_allocation(vocab: int, v: int) -> np.ndarray:
    per = int(round(v / vocab))
    return np.full(vocab, per, dtype=np.int64)


def allocation(w: Workload) -> np.ndarray:
    if w.alloc == "zipf":
        d = zipf_allocation(w.vocab, w.v, w.k, w.zipf_s)
    elif w.alloc == "dense64":
        d = dense64_allocation(w.vocab, w.v, w.k)
    elif w.alloc == "uniform":
        d = uniform_allocation(w.vocab, w.v)
    else:
        raise ValueError(w.alloc)
    return d


def offsets_from_allocation(d: np.ndarray) -> np.ndarray:
    """Row offsets of the concatenated tables: offsets[t] = sum of d_i, i < t."""
    off = np.zeros(len(d) + 1, dtype=np.int64)
    np.cumsum(d, out=off[1:])
    return off.astype(np.int32)


def token_ids(w: Workload) -> np.ndarray:
    rng = _rng(w.batch_seed, "ids")
    n = w.n_tokens
    if w.ids == "zipf":
        p = zipf_weights(w.vocab, w.zipf_s)
        ids = rng.choice(w.vocab, size=n, p=p / p.sum())
    elif w.ids == "zipf_distinct":
        p = zipf_weights(w.vocab, w.zipf_s)
        ids = rng.choice(w.vocab, size=n, replace=False, p=p / p.sum())
    elif w.ids == "uniform_first64":
        ids = rng.integers(0, 64, size=n)
    elif w.ids == "uniform":
        ids = rng.integers(0, w.vocab, size=n)
    else:
        raise ValueError(w.ids)
    return ids.astype(np.int32)


def zipf_corpus(vocab: int, n: int, seed: int, s: float = 1.1, n_phrases: int = 50000,
                phrase_share: float = 0.5) -> np.ndarray:
    """A synthetic token stream standing in for a tokenised corpus (the pages'
    FineWeb-Edu text is not here): half of its items are single tokens drawn
    Zipf(s) over the vocabulary, half are phrases of 2-6 such tokens drawn
    Zipf(s) from a fixed phrase list, so frequent multi-token sequences recur
    as in text. int32 [n]."""
    rng = _rng(seed, "corpus")
    p_tok = zipf_weights(vocab, s)
    p_tok /= p_tok.sum()
    plen = rng.integers(2, 7, size=n_phrases)
    pstart = np.concatenate([[0], np.cumsum(plen)])
    ptoks = rng.choice(vocab, size=int(pstart[-1]), p=p_tok)
    p_phr = zipf_weights(n_phrases, s)
    p_phr /= p_phr.sum()
    out, have = [], 0
    while have < n:
        m = max(1024, (n - have) // 2)
        is_phr = rng.random(m) < phrase_share
        which = rng.choice(n_phrases, size=m, p=p_phr)
        single = rng.choice(vocab, size=m, p=p_tok)
        lens = np.where(is_phr, plen[which], 1)
        starts = np.where(is_phr, pstart[which], 0)
        item = np.repeat(np.arange(m), lens)
        offs = np.arange(int(lens.sum())) - np.repeat(np.cumsum(lens) - lens, lens)
        toks = np.where(is_phr[item], ptoks[np.minimum(starts[item] + offs, len(ptoks) - 1)],
                        single[item])
        out.append(toks)
        have += len(toks)
    return np.concatenate(out)[:n].astype(np.int32)


def normal_tensor(seed: int, tag: str, shape, std: float, dtype: torch.dtype,
                  threads: int = 8) -> torch.Tensor:
    """N(0, std^2) samples in `dtype` (rounded once, to nearest even)."""
    n = int(np.prod(shape))
    out = torch.empty(n, dtype=dtype)
    n_chunks = (n + _CHUNK - 1) // _CHUNK

    def work(c):
        lo, hi = c * _CHUNK, min(n, (c + 1) * _CHUNK)
        buf = _rng(seed, tag, c).standard_normal(hi - lo, dtype=np.float32)
        buf *= np.float32(std)
        out[lo:hi] = torch.from_numpy(buf).to(dtype)

    if n_chunks <= 1:
        for c in range(n_chunks):
            work(c)
    else:
        with ThreadPoolExecutor(min(threads, n_chunks)) as ex:
            list(ex.map(work, range(n_chunks)))
    return out.view(*shape)


@dataclasses.dataclass
class Tables:
    """Weights of one L³ layer, on the host."""

    offsets: torch.Tensor   # int32 [vocab + 1]
    W_K: torch.Tensor       # [v, d_in]
    W_V: torch.Tensor       # [v, d_emb]
    W_up: torch.Tensor      # [d_up, d_emb]
    ln_gamma: torch.Tensor  # [d_up]
    ln_beta: torch.Tensor   # [d_up]
    W_mix: torch.Tensor     # [d_out, d_up + d_in]; columns 0..d_up-1 act on the LN output


@dataclasses.dataclass
class Batch:
    ids: torch.Tensor       # int32 [N]
    x: torch.Tensor         # [N, d_in]


def make_tables(w: Workload) -> Tables:
    dt = w.torch_dtype
    s = w.table_seed
    off = torch.from_numpy(offsets_from_allocation(allocation(w)))
    W_K = normal_tensor(s, "W_K", (w.v, w.d_in), w.d_in ** -0.5, dt)
    if w.tied and w.d_in != w.d_emb:
        raise ValueError("a tied workload needs d_in == d_emb")
    return Tables(
        offsets=off,
        W_K=W_K,
        W_V=W_K if w.tied else normal_tensor(s, "W_V", (w.v, w.d_emb), w.d_emb ** -0.5, dt),
        W_up=normal_tensor(s, "W_up", (w.d_up, w.d_emb), w.d_emb ** -0.5, dt),
        ln_gamma=torch.ones(w.d_up, dtype=dt),
        ln_beta=torch.zeros(w.d_up, dtype=dt),
        W_mix=normal_tensor(s, "W_mix", (w.d_out, w.d_up + w.d_in),
                            (w.d_up + w.d_in) ** -0.5, dt),
    )


def make_batch(w: Workload) -> Batch:
    ids = torch.from_numpy(token_ids(w))
    x = normal_tensor(w.batch_seed, "x", (w.n_tokens, w.d_in), w.d_in ** -0.5, w.torch_dtype)
    return Batch(ids=ids, x=x)
