"""Shared helpers of the GPU parity tests: upload a seeded workload, run the
CUDA path through the C ABI, pick token samples, compare with the oracle."""
from __future__ import annotations

import functools

import numpy as np
import torch

import static_token_routed_b200 as l3
from static_token_routed_b200 import workloads as wl

EPS = 1e-5
# max |y_gpu - y_oracle| / RMS(y_oracle): bf16 and fp32 bars of the layer's
# parity contract
TOL = {"bf16": 2e-2, "fp32": 1e-4}


@functools.lru_cache(maxsize=2)
def host_workload(name: str, n_tokens: int | None = None, batch_seed: int | None = None):
    w = wl.WORKLOADS[name]
    if n_tokens is not None or batch_seed is not None:
        w = wl.with_tokens(w, n_tokens or w.n_tokens, batch_seed)
    return w, wl.make_tables(w), wl.make_batch(w)


def to_device(tables: wl.Tables, batch: wl.Batch, device="cuda"):
    dev = {k: getattr(tables, k).to(device) for k in
           ("offsets", "W_K", "W_up", "ln_gamma", "ln_beta", "W_mix")}
    # a tied workload passes one device table as keys and values
    dev["W_V"] = dev["W_K"] if tables.W_V is tables.W_K else tables.W_V.to(device)
    dev["ids"] = batch.ids.to(device)
    dev["x"] = batch.x.to(device)
    return dev


def dims_of(w: wl.Workload, eps=EPS):
    return l3.make_dims(w.vocab, w.v, w.k, w.d_in, w.d_emb, w.d_up, w.d_out, w.torch_dtype, eps)


def run_forward(w, dev, eps=EPS, y=None):
    plan = l3.l3_plan(dev["ids"], dev["offsets"], dims_of(w, eps))
    if y is None:
        y = torch.empty(dev["x"].shape[0], w.d_out, dtype=w.torch_dtype, device=dev["x"].device)
    l3.l3_forward(dev["x"], plan, dev["W_K"], dev["W_V"], dev["W_up"], dev["ln_gamma"],
                  dev["ln_beta"], dev["W_mix"], y)
    l3.l3_forward_status(plan)
    return y, plan


def sample_tokens(ids: np.ndarray, offsets: np.ndarray, n_sample: int, seed: int = 0):
    """A spread of token indices: members of the largest groups, of the
    groups with the largest and smallest d_t, singletons, first and last
    tokens, and uniform picks."""
    rng = np.random.default_rng(seed)
    n = len(ids)
    d = np.diff(offsets.astype(np.int64))[ids]
    cnt = np.bincount(ids, minlength=len(offsets) - 1)[ids]
    picks = {0, n - 1}
    for key in (cnt, d, -d, -cnt):
        order = np.argsort(-key, kind="stable")
        picks.update(order[: n_sample // 8].tolist())
    picks.update(rng.choice(n, size=min(n, n_sample), replace=False).tolist())
    picks = np.array(sorted(picks), dtype=np.int64)
    if len(picks) > n_sample:
        keep = np.concatenate([picks[:2], rng.choice(picks[2:], n_sample - 2, replace=False)])
        picks = np.unique(keep)
    return picks


def rel_max_err(got: np.ndarray, want: np.ndarray) -> float:
    rms = float(np.sqrt(np.mean(want ** 2)))
    return float(np.max(np.abs(got - want))) / rms


def bf16_half_ulp(v: np.ndarray) -> np.ndarray:
    """Half the bf16 spacing at |v| (8 significant bits): the largest error of
    rounding v itself to bf16."""
    e = np.floor(np.log2(np.maximum(np.abs(v), np.finfo(np.float64).tiny)))
    return 0.5 * np.exp2(e - 7)


def rounding_floor(want: np.ndarray) -> float:
    """max |bf16(want) - want| / RMS(want): the error of the exact result
    rounded once to bf16, which no bf16 output can beat."""
    rms = float(np.sqrt(np.mean(want ** 2)))
    rounded = torch.from_numpy(want).to(torch.bfloat16).double().numpy()
    return float(np.max(np.abs(rounded - want))) / rms


def within_bf16_bar(got: np.ndarray, want: np.ndarray, tol: float) -> bool:
    """Per element |got - want| <= tol * RMS(want) + bf16_half_ulp(want): the
    bar with the output's own final bf16 rounding excepted. Used where the
    exactly rounded result itself exceeds tol * RMS."""
    rms = float(np.sqrt(np.mean(want ** 2)))
    return bool(np.all(np.abs(got - want) <= tol * rms + bf16_half_ulp(want)))
