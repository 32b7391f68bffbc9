"""Pins that tie the CPU oracle to what the pages and the mathematics fix.

Each `pin_*` function runs the oracle (optionally a mutated build of it, given
by `lib_path`) and raises AssertionError when the oracle disagrees with an
independent statement of the same result. None of them retypes the oracle's
own loop: they use torch's attention / layer_norm routines, closed forms,
invariances, and a hand-derived worked example.

Pages: "L³: Large Lookup Layers" (Tseng & De Sa). kimjy99 review, Method:
the layer equation. kimjy99 review §2: applying L³ to a batch equals plain
attention with Q = B, K = W_K, V = W_V and a mask that admits only each token's
own rows. papernotes 整体框架: channel mixing only, no cross-token mixing.
sciencestack Fig. 3: the batch sort and its inverse.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch
import torch.nn.functional as F

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ----------------------------------------------------------------------------
# small random fp64 layers
# ----------------------------------------------------------------------------

def random_layer(seed: int, vocab=7, d_max=5, d_in=6, d_emb=5, d_up=4, d_out=3, n=11,
                 d_all=None, dtype=torch.float64):
    g = torch.Generator().manual_seed(seed)
    if d_all is None:
        d = torch.randint(1, d_max + 1, (vocab,), generator=g)
    else:
        d = torch.full((vocab,), d_all, dtype=torch.int64)
    offsets = torch.zeros(vocab + 1, dtype=torch.int32)
    offsets[1:] = torch.cumsum(d, 0).to(torch.int32)
    v = int(offsets[-1])
    ids = torch.randint(0, vocab, (n,), generator=g, dtype=torch.int32)

    def rn(*shape):
        return torch.randn(*shape, generator=g, dtype=torch.float64)

    layer = dict(
        ids=ids, offsets=offsets,
        x=rn(n, d_in), W_K=rn(v, d_in), W_V=rn(v, d_emb), W_up=rn(d_up, d_emb),
        ln_gamma=1.0 + 0.1 * rn(d_up), ln_beta=0.1 * rn(d_up), W_mix=rn(d_out, d_up + d_in),
    )
    for k in ("x", "W_K", "W_V", "W_up", "ln_gamma", "ln_beta", "W_mix"):
        layer[k] = layer[k].to(dtype)
    return layer


def run_oracle(layer, eps, lib_path=oracle.LIBRARY, select=None):
    return oracle.forward(layer["ids"], layer["offsets"], layer["x"], layer["W_K"],
                          layer["W_V"], layer["W_up"], layer["ln_gamma"], layer["ln_beta"],
                          layer["W_mix"], eps, select=select, lib_path=lib_path)


def masked_attention_reference(layer, eps):
    """The whole layer through torch's library routines, as the review's §2
    states it: attention of the batch (queries) over the full tables with a
    mask that admits only each token's rows, scale 1; then LayerNorm(W_up .),
    an explicit concat with x, and W_mix."""
    x = layer["x"].double()
    ids = layer["ids"].long()
    off = layer["offsets"].long()
    v = int(off[-1])
    rows = torch.arange(v)
    keep = (rows[None, :] >= off[ids][:, None]) & (rows[None, :] < off[ids + 1][:, None])
    a = F.scaled_dot_product_attention(x[None], layer["W_K"].double()[None],
                                       layer["W_V"].double()[None], attn_mask=keep[None],
                                       scale=1.0)[0]
    z = a @ layer["W_up"].double().T
    h = F.layer_norm(z, (z.shape[1],), layer["ln_gamma"].double(), layer["ln_beta"].double(),
                     eps=eps)
    return torch.cat([h, x], dim=1) @ layer["W_mix"].double().T


def rel_err(got, want):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    scale = max(float(np.sqrt(np.mean(want ** 2))), 1e-300)
    return float(np.max(np.abs(got - want))) / scale


# ----------------------------------------------------------------------------
# pins
# ----------------------------------------------------------------------------

def pin_masked_attention(lib_path=oracle.LIBRARY, seeds=range(6), eps=1e-5):
    """kimjy99 review §2: L³ over a batch == masked dense attention (Q=B, K=W_K,
    V=W_V), then the rest of the layer equation."""
    for seed in seeds:
        for shape in ({}, dict(vocab=3, d_max=9, d_in=4, d_emb=7, d_up=6, d_out=5, n=17)):
            layer = random_layer(seed, **shape)
            got = run_oracle(layer, eps, lib_path)
            want = masked_attention_reference(layer, eps).numpy()
            err = rel_err(got, want)
            assert err < 1e-12, f"masked-attention pin: seed {seed} rel err {err}"


def pin_worked_example(lib_path=oracle.LIBRARY):
    """Hand-derived worked example (tests/golden/worked_example_closed_form.json)."""
    with open(os.path.join(GOLDEN, "worked_example_closed_form.json")) as f:
        ex = json.load(f)
    inp = ex["inputs"]

    def val(v, eps):
        if isinstance(v, str):
            return float(eval(v, {"__builtins__": {}}, {"log": math.log, "sqrt": math.sqrt,
                                                         "eps": eps}))
        return float(v)

    def mat(rows, eps):
        return torch.tensor([[val(v, eps) for v in r] for r in rows], dtype=torch.float64)

    for eps in ex["eps_values"]:
        layer = dict(
            ids=torch.tensor(inp["ids"], dtype=torch.int32),
            offsets=torch.tensor(inp["offsets"], dtype=torch.int32),
            x=mat(inp["x"], eps), W_K=mat(inp["W_K"], eps), W_V=mat(inp["W_V"], eps),
            W_up=mat(inp["W_up"], eps),
            ln_gamma=torch.tensor(inp["ln_gamma"], dtype=torch.float64),
            ln_beta=torch.tensor(inp["ln_beta"], dtype=torch.float64),
            W_mix=mat(inp["W_mix"], eps))
        got = run_oracle(layer, eps, lib_path)
        want = mat(ex["expected_y"], eps).numpy()
        skip = set(ex["skip_rows_when_eps_is_zero"]) if eps == 0.0 else set()
        for r in range(want.shape[0]):
            if r in skip:
                continue
            np.testing.assert_allclose(got[r], want[r], rtol=1e-14, atol=1e-15,
                                       err_msg=f"worked example row {r}, eps {eps}")


def pin_single_row(lib_path=oracle.LIBRARY, eps=1e-5):
    """d_t = 1 for every ID: softmax over one logit is 1, so
    y = W_mix [LN(W_up V_t) ; x] whatever K_t and x are."""
    for seed in range(4):
        layer = random_layer(seed, vocab=9, d_all=1, n=13)
        got = run_oracle(layer, eps, lib_path)
        v_rows = layer["W_V"][layer["offsets"][layer["ids"].long()].long()]
        z = v_rows @ layer["W_up"].T
        h = F.layer_norm(z, (z.shape[1],), layer["ln_gamma"], layer["ln_beta"], eps=eps)
        want = (torch.cat([h, layer["x"]], 1) @ layer["W_mix"].T).numpy()
        assert rel_err(got, want) < 1e-12, "d_t = 1 closed form"


def pin_uniform_softmax(lib_path=oracle.LIBRARY, eps=1e-5):
    """x = 0 (all logits 0) or all rows of K_t equal: p is uniform, so a is the
    mean of the rows of V_t."""
    for seed in range(3):
        for case in ("x_zero", "equal_keys"):
            layer = random_layer(seed, vocab=4, d_max=6, n=9)
            if case == "x_zero":
                layer["x"] = torch.zeros_like(layer["x"])
            else:
                off = layer["offsets"].long()
                for t in range(len(off) - 1):
                    layer["W_K"][off[t]:off[t + 1]] = layer["W_K"][off[t]]
            off = layer["offsets"].long()
            ids = layer["ids"].long()
            a = torch.stack([layer["W_V"][off[t]:off[t + 1]].mean(0) for t in ids])
            z = a @ layer["W_up"].T
            h = F.layer_norm(z, (z.shape[1],), layer["ln_gamma"], layer["ln_beta"], eps=eps)
            want = (torch.cat([h, layer["x"]], 1) @ layer["W_mix"].T).numpy()
            got = run_oracle(layer, eps, lib_path)
            assert rel_err(got, want) < 1e-12, f"uniform softmax ({case})"


def pin_permutation(lib_path=oracle.LIBRARY, eps=1e-5):
    """papernotes 整体框架: no cross-token mixing, so y(pi X, pi T) = pi y(X, T)."""
    for seed in range(3):
        layer = random_layer(seed, n=19)
        y = run_oracle(layer, eps, lib_path)
        pi = torch.randperm(19, generator=torch.Generator().manual_seed(100 + seed))
        layer2 = dict(layer, ids=layer["ids"][pi], x=layer["x"][pi])
        y2 = run_oracle(layer2, eps, lib_path)
        assert np.array_equal(y2, y[pi.numpy()]), "permutation invariance"


def pin_layernorm_scale(lib_path=oracle.LIBRARY):
    """With eps = 0, LayerNorm is invariant to scaling its input: scaling W_up
    by 4 (exact in binary) leaves y bit-identical; by 3, equal to rounding."""
    for seed in range(3):
        layer = random_layer(seed)
        y = run_oracle(layer, 0.0, lib_path)
        for c, tol in ((4.0, 0.0), (3.0, 1e-12)):
            y2 = run_oracle(dict(layer, W_up=layer["W_up"] * c), 0.0, lib_path)
            assert rel_err(y2, y) <= tol, f"LayerNorm scale invariance (c={c})"
        # and LayerNorm itself matches torch's routine on the same z
        want = masked_attention_reference(layer, 0.0).numpy()
        assert rel_err(y, want) < 1e-12


def pin_plan(lib_path=oracle.LIBRARY):
    """sciencestack Fig. 3: sorting the batch by ID groups it into blocks.
    Checked against numpy's stable argsort and np.bincount."""
    rng = np.random.default_rng(5)
    for vocab, n in ((7, 1), (7, 40), (1000, 3000), (50, 0)):
        ids = rng.integers(0, vocab, size=n).astype(np.int32)
        d = rng.integers(1, 9, size=vocab)
        off = np.concatenate([[0], np.cumsum(d)]).astype(np.int32)
        p = oracle.plan(ids, off, lib_path=lib_path)
        want_perm = np.argsort(ids, kind="stable")
        assert np.array_equal(p["perm"], want_perm), "perm vs stable argsort"
        assert np.array_equal(p["sorted_ids"], ids[want_perm])
        inv = np.empty(n, dtype=np.int64)
        inv[want_perm] = np.arange(n)
        assert np.array_equal(p["inv_perm"], inv)
        counts = np.bincount(ids, minlength=vocab)
        present = np.nonzero(counts)[0]
        assert p["G"] == len(present)
        assert np.array_equal(p["group_ids"], present)
        assert np.array_equal(np.diff(p["group_tok_start"]), counts[present])
        assert p["group_tok_start"][0] == 0 and p["group_tok_start"][-1] == n
        assert np.array_equal(np.diff(p["seg_rows"]), d[present])
        assert p["seg_rows"][0] == 0


ALL_PINS = [pin_masked_attention, pin_worked_example, pin_single_row, pin_uniform_softmax,
            pin_permutation, pin_layernorm_scale, pin_plan]
