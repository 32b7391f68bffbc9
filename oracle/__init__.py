"""CPU oracle for the L³ (Large Lookup Layer) forward pass — test infrastructure.

Only `tests/`, `__graft_entry__.smoke()` and the CPU-baseline / reference leg
of `bench.py` may import this package. The CUDA library never calls it.

`l3_oracle.c` states the layer of "L³: Large Lookup Layers" (Tseng & De Sa;
kimjy99 review, Method, eq. L³; papernotes 整体框架) in fp64, token by token,
and the stable counting sort that groups a batch by token ID (sciencestack
page, Fig. 3). This module only compiles that file with gcc and marshals
arrays into it.

Parity pins (all under tests/, run without a GPU): masked dense attention
through torch's scaled_dot_product_attention (kimjy99 review §2), d_t = 1
closed form, uniform softmax cases, a hand-derived worked example in
tests/golden/, permutation invariance, LayerNorm scale invariance, and the
plan's sort against numpy's stable argsort. No function here is unpinned.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "l3_oracle.c")
LIBRARY = os.path.join(_HERE, "libl3_oracle.so")

F32, BF16, F64 = 0, 1, 2
_STATUS = {0: "ok", 1: "bad argument", 2: "token id out of range", 3: "bad offsets",
           4: "out of memory"}

_lock = threading.Lock()
_libs: dict[str, ctypes.CDLL] = {}


class OracleError(RuntimeError):
    pass


def compile_library(source: str = SOURCE, output: str = LIBRARY) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, no fast-math)."""
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", output, source, "-lm"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return output


def load(path: str = LIBRARY) -> ctypes.CDLL:
    with _lock:
        if path in _libs:
            return _libs[path]
        if path == LIBRARY and (not os.path.exists(path)
                                or os.path.getmtime(path) < os.path.getmtime(SOURCE)):
            compile_library()
        lib = ctypes.CDLL(path)
        p, i64, i32, d = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double
        lib.l3_oracle_forward.restype = i32
        lib.l3_oracle_forward.argtypes = [i64, p, i64, p, p, i64, i64, i64, i64, i64, i32,
                                          p, p, p, p, p, p, p, d, p, i32]
        lib.l3_oracle_plan.restype = i32
        lib.l3_oracle_plan.argtypes = [p, i64, p, i64, p, p, p, p, p, p, p]
        lib.l3_oracle_threads.restype = i32
        lib.l3_oracle_threads.argtypes = []
        _libs[path] = lib
        return lib


def threads(lib_path: str = LIBRARY) -> int:
    return int(load(lib_path).l3_oracle_threads())


def _as_host(t) -> tuple[np.ndarray, int]:
    """Contiguous host array plus dtype code; bf16 is passed as raw bits."""
    if isinstance(t, np.ndarray):
        t = torch.from_numpy(t)
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy(), BF16
    if t.dtype == torch.float32:
        return t.numpy(), F32
    if t.dtype == torch.float64:
        return t.numpy(), F64
    raise TypeError(f"unsupported dtype {t.dtype}")


def _i32(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        t = t.detach().cpu().numpy()
    return np.ascontiguousarray(t, dtype=np.int32)


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def forward(ids, offsets, x, W_K, W_V, W_up, ln_gamma, ln_beta, W_mix, eps: float,
            select=None, n_threads: int = 0, lib_path: str = LIBRARY) -> np.ndarray:
    """fp64 L³ output for the selected tokens (all tokens if select is None).

    All float tensors must share one dtype (bf16, fp32 or fp64); they are
    widened exactly to fp64 inside. Returns float64 [len(select), d_out].
    """
    lib = load(lib_path)
    ids_a = _i32(ids)
    off_a = _i32(offsets)
    arrs = [_as_host(t) for t in (x, W_K, W_V, W_up, ln_gamma, ln_beta, W_mix)]
    codes = {c for _, c in arrs}
    if len(codes) != 1:
        raise TypeError("all float inputs must share one dtype")
    dtype = codes.pop()
    n_tokens = ids_a.shape[0]
    d_in = int(x.shape[1])
    d_emb = int(W_V.shape[1])
    d_up = int(W_up.shape[0])
    d_out = int(W_mix.shape[0])
    vocab = off_a.shape[0] - 1
    if tuple(W_mix.shape) != (d_out, d_up + d_in) or int(W_up.shape[1]) != d_emb:
        raise ValueError("inconsistent shapes")
    sel = np.arange(n_tokens, dtype=np.int64) if select is None else \
        np.ascontiguousarray(select, dtype=np.int64)
    y = np.zeros((sel.shape[0], d_out), dtype=np.float64)
    st = lib.l3_oracle_forward(sel.shape[0], _ptr(sel), n_tokens, _ptr(ids_a), _ptr(off_a),
                               vocab, d_in, d_emb, d_up, d_out, dtype,
                               *[_ptr(a) for a, _ in arrs], float(eps), _ptr(y), n_threads)
    if st != 0:
        raise OracleError(_STATUS.get(st, str(st)))
    return y


def plan(ids, offsets, lib_path: str = LIBRARY) -> dict:
    """Stable counting-sort plan: perm, inv_perm, sorted_ids, group_ids,
    group_tok_start [G+1], seg_rows [G+1] (all int32) and G."""
    lib = load(lib_path)
    ids_a = _i32(ids)
    off_a = _i32(offsets)
    n = ids_a.shape[0]
    vocab = off_a.shape[0] - 1
    out = {k: np.zeros(n, dtype=np.int32) for k in ("perm", "inv_perm", "sorted_ids")}
    grp = {k: np.zeros(n + 1, dtype=np.int32) for k in ("group_ids", "group_tok_start",
                                                         "seg_rows")}
    G = ctypes.c_int64(0)
    st = lib.l3_oracle_plan(_ptr(ids_a), n, _ptr(off_a), vocab, _ptr(out["perm"]),
                            _ptr(out["inv_perm"]), _ptr(out["sorted_ids"]),
                            _ptr(grp["group_ids"]), _ptr(grp["group_tok_start"]),
                            _ptr(grp["seg_rows"]), ctypes.byref(G))
    if st != 0:
        raise OracleError(_STATUS.get(st, str(st)))
    g = int(G.value)
    out["G"] = g
    out["group_ids"] = grp["group_ids"][:g]
    out["group_tok_start"] = grp["group_tok_start"][:g + 1]
    out["seg_rows"] = grp["seg_rows"][:g + 1]
    return out
