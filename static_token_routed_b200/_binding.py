"""ctypes binding of libl3.so (include/l3.h). Argument marshalling only:
every step of the L³ forward pass runs in the library's CUDA kernels.

The functions keep the C names. Tensors are torch CUDA tensors; their data
pointers are passed through unchanged. `stream` defaults to torch's current
stream on the tensors' device.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIBRARY = os.path.join(_PKG, "libl3.so")

L3_BF16, L3_FP32 = 0, 1
STATUS = {0: "L3_OK", 1: "L3_ERR_INVALID_ARG", 2: "L3_ERR_TOKEN_RANGE", 3: "L3_ERR_BAD_OFFSETS",
          4: "L3_ERR_UNSUPPORTED", 5: "L3_ERR_CUDA", 6: "L3_ERR_TIMEOUT", 7: "L3_ERR_OOM"}

# every symbol include/l3.h declares
EXPORTED = ["l3_plan", "l3_plan_info", "l3_plan_export", "l3_forward", "l3_forward_status",
            "l3_plan_destroy", "l3_last_error", "l3_profile_enable", "l3_profile_read",
            "l3_sort_tokens_noalloc", "l3_plan_staged", "l3_stage_rows", "l3_lzw_allocate",
            "l3_lzw_allocate_device", "l3_check_bounded_wait", "l3_backward"]
L3_SORT_NOALLOC_MAX_TOKENS = 65536


class L3Error(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


class Dims(ctypes.Structure):
    _fields_ = [("vocab", ctypes.c_int64), ("v", ctypes.c_int64), ("k", ctypes.c_int64),
                ("d_in", ctypes.c_int64), ("d_emb", ctypes.c_int64), ("d_up", ctypes.c_int64),
                ("d_out", ctypes.c_int64), ("dtype", ctypes.c_int32), ("ln_eps", ctypes.c_float)]


class PlanInfo(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in ("n_tokens", "n_groups", "n_dense_groups",
                                               "n_dense_tiles", "n_tail_items", "unique_rows",
                                               "unique_rows_multi")]


class KernelTime(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 48), ("launches", ctypes.c_int64),
                ("total_ms", ctypes.c_double)]


_lib = None


def library() -> ctypes.CDLL:
    """Load libl3.so. Raises if it has not been built: there is no fallback."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIBRARY):
        raise RuntimeError(f"{LIBRARY} is missing; build it with "
                           "`python -m static_token_routed_b200.build`")
    lib = ctypes.CDLL(LIBRARY)
    p, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    lib.l3_plan.restype = i32
    lib.l3_plan.argtypes = [p, i64, p, ctypes.POINTER(Dims), p, ctypes.POINTER(p)]
    lib.l3_plan_staged.restype = i32
    lib.l3_plan_staged.argtypes = [p, i64, p, ctypes.POINTER(Dims), p, ctypes.POINTER(p)]
    lib.l3_stage_rows.restype = i32
    lib.l3_stage_rows.argtypes = [p, p, p, p, p, p]
    lib.l3_backward.restype = i32
    lib.l3_backward.argtypes = [p] * 17
    lib.l3_check_bounded_wait.restype = i32
    lib.l3_check_bounded_wait.argtypes = [p]
    lib.l3_lzw_allocate.restype = i32
    lib.l3_lzw_allocate.argtypes = [p, i64, i64, i64, i64, p, ctypes.POINTER(i64)]
    lib.l3_lzw_allocate_device.restype = i32
    lib.l3_lzw_allocate_device.argtypes = [p, i64, i64, i64, i64, p, ctypes.POINTER(i64), p]
    lib.l3_plan_info.restype = i32
    lib.l3_plan_info.argtypes = [p, ctypes.POINTER(PlanInfo)]
    lib.l3_plan_export.restype = i32
    lib.l3_plan_export.argtypes = [p, p, p, p, p, p, p, ctypes.POINTER(i64), p]
    lib.l3_forward.restype = i32
    lib.l3_forward.argtypes = [p, p, p, p, p, p, p, p, p, p]
    lib.l3_forward_status.restype = i32
    lib.l3_forward_status.argtypes = [p]
    lib.l3_plan_destroy.restype = None
    lib.l3_plan_destroy.argtypes = [p]
    lib.l3_last_error.restype = ctypes.c_char_p
    lib.l3_last_error.argtypes = []
    lib.l3_profile_enable.restype = None
    lib.l3_profile_enable.argtypes = [i32]
    lib.l3_profile_read.restype = i32
    lib.l3_profile_read.argtypes = [ctypes.POINTER(KernelTime), i32]
    lib.l3_sort_tokens_noalloc.restype = i32
    lib.l3_sort_tokens_noalloc.argtypes = [p, i64, i64, p, p, p, p]
    _lib = lib
    return lib


def l3_last_error() -> str:
    return library().l3_last_error().decode()


def _check(status: int):
    if status != 0:
        raise L3Error(status, l3_last_error())


def _stream(stream, device) -> int:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: torch.Tensor | None, name: str) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def make_dims(vocab, v, k, d_in, d_emb, d_up, d_out, dtype=torch.bfloat16, ln_eps=1e-5) -> Dims:
    code = L3_BF16 if dtype == torch.bfloat16 else L3_FP32
    return Dims(vocab, v, k, d_in, d_emb, d_up, d_out, code, ln_eps)


class Plan:
    """Owns an l3_plan_t; destroyed explicitly or when garbage collected."""

    def __init__(self, handle: int, dims: Dims, n_tokens: int, staged: bool = False):
        self.handle = handle
        self.dims = dims
        self.n_tokens = n_tokens
        self.staged = staged  # the forward reads staged tables of the batch's rows
        self.table_rows = l3_plan_info(self).unique_rows if staged else dims.v

    def info(self) -> PlanInfo:
        return l3_plan_info(self)

    def destroy(self):
        if self.handle:
            library().l3_plan_destroy(self.handle)
            self.handle = None

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.destroy()

    def __del__(self):
        try:
            self.destroy()
        except Exception:
            pass


def l3_plan(token_ids: torch.Tensor, offsets: torch.Tensor, dims: Dims, stream=None,
            staged: bool = False) -> Plan:
    """l3_plan, or l3_plan_staged when staged=True."""
    if token_ids.dtype != torch.int32 or offsets.dtype != torch.int32:
        raise TypeError("token_ids and offsets must be int32")
    out = ctypes.c_void_p()
    n = token_ids.numel()
    fn = library().l3_plan_staged if staged else library().l3_plan
    st = fn(_ptr(token_ids, "token_ids") if n else None, n, _ptr(offsets, "offsets"),
            ctypes.byref(dims), _stream(stream, offsets.device), ctypes.byref(out))
    _check(st)
    return Plan(out.value, dims, n, staged)


def l3_plan_staged(token_ids: torch.Tensor, offsets: torch.Tensor, dims: Dims,
                   stream=None) -> Plan:
    return l3_plan(token_ids, offsets, dims, stream, staged=True)


def _table_ptr(t: torch.Tensor, name: str) -> int:
    """A device tensor, or a pinned host tensor (read by the kernel through
    the device's mapping of it)."""
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if not (t.is_cuda or t.is_pinned()):
        raise ValueError(f"{name} must be a CUDA tensor or pinned host memory")
    return t.data_ptr()


def l3_stage_rows(plan: Plan, W_K: torch.Tensor, W_V: torch.Tensor, W_K_staged: torch.Tensor,
                  W_V_staged: torch.Tensor, stream=None) -> None:
    d = plan.dims
    for nm, t, shape in (("W_K", W_K, (d.v, d.d_in)), ("W_V", W_V, (d.v, d.d_emb)),
                         ("W_K_staged", W_K_staged, (plan.table_rows, d.d_in)),
                         ("W_V_staged", W_V_staged, (plan.table_rows, d.d_emb))):
        if tuple(t.shape) != shape:
            raise ValueError(f"{nm} has shape {tuple(t.shape)}, want {shape}")
    _check(library().l3_stage_rows(plan.handle, _table_ptr(W_K, "W_K"), _table_ptr(W_V, "W_V"),
                                   _ptr(W_K_staged, "W_K_staged"), _ptr(W_V_staged, "W_V_staged"),
                                   _stream(stream, W_K_staged.device)))


def l3_lzw_allocate(corpus, vocab: int, v: int, k: int) -> tuple[np.ndarray, int]:
    """d_t for every token ID (int32 [vocab]) and the number of codewords."""
    c = np.ascontiguousarray(np.asarray(corpus, dtype=np.int32))
    d = np.empty(int(vocab), dtype=np.int32)
    nw = ctypes.c_int64(0)
    _check(library().l3_lzw_allocate(c.ctypes.data if c.size else None, int(c.size), int(vocab),
                                     int(v), int(k), d.ctypes.data, ctypes.byref(nw)))
    return d, int(nw.value)


def l3_lzw_allocate_device(corpus, vocab: int, v: int, k: int, d_out: torch.Tensor | None = None,
                           stream=None) -> tuple[torch.Tensor, int]:
    """The LZW allocation with its codeword walk on the GPU: d_t as a device
    int32 tensor [vocab] (d_out, or a new one on the current device), and the
    number of codewords. The corpus is a host array."""
    c = np.ascontiguousarray(np.asarray(corpus, dtype=np.int32))
    if d_out is None:
        d_out = torch.empty(int(vocab), dtype=torch.int32, device="cuda")
    if d_out.dtype != torch.int32 or not d_out.is_cuda or d_out.numel() != int(vocab):
        raise ValueError("d_out must be a CUDA int32 tensor of vocab entries")
    nw = ctypes.c_int64(0)
    _check(library().l3_lzw_allocate_device(c.ctypes.data if c.size else None, int(c.size),
                                            int(vocab), int(v), int(k), d_out.data_ptr(),
                                            ctypes.byref(nw), _stream(stream, d_out.device)))
    return d_out, int(nw.value)


def l3_backward(x, plan: Plan, W_K, W_V, W_up, ln_gamma, ln_beta, W_mix, dy,
                stream=None) -> dict:
    """Gradients for dL/dy = dy after l3_forward on the same plan and inputs.
    Returns fp32 tensors: x, W_K, W_V (fresh zero buffers the library adds
    the batch's rows into; rows of IDs outside the batch stay zero), W_up,
    ln_gamma, ln_beta, W_mix."""
    d = plan.dims
    dev = x.device
    f32 = dict(dtype=torch.float32, device=dev)
    out = {"x": torch.empty(plan.n_tokens, d.d_in, **f32),
           "W_K": torch.zeros(d.v, d.d_in, **f32), "W_V": torch.zeros(d.v, d.d_emb, **f32),
           "W_up": torch.empty(d.d_up, d.d_emb, **f32), "ln_gamma": torch.empty(d.d_up, **f32),
           "ln_beta": torch.empty(d.d_up, **f32),
           "W_mix": torch.empty(d.d_out, d.d_up + d.d_in, **f32)}
    ins = [_ptr(t, nm) for t, nm in ((x, "x"), (None, "plan"), (W_K, "W_K"), (W_V, "W_V"),
                                     (W_up, "W_up"), (ln_gamma, "ln_gamma"),
                                     (ln_beta, "ln_beta"), (W_mix, "W_mix"), (dy, "dy"))]
    ins[1] = plan.handle
    outs = [out[k].data_ptr() for k in ("x", "W_K", "W_V", "W_up", "ln_gamma", "ln_beta",
                                        "W_mix")]
    _check(library().l3_backward(*ins, *outs, _stream(stream, dev)))
    return out


def l3_check_bounded_wait(stream=None, device=None) -> int:
    """Status of the device-side give-up check (L3_ERR_TIMEOUT = 6 expected)."""
    dev = device if device is not None else torch.cuda.current_device()
    return int(library().l3_check_bounded_wait(_stream(stream, torch.device("cuda", dev))))


def l3_plan_info(plan: Plan) -> PlanInfo:
    info = PlanInfo()
    _check(library().l3_plan_info(plan.handle, ctypes.byref(info)))
    return info


def l3_plan_export(plan: Plan, perm=None, inv_perm=None, sorted_ids=None, group_ids=None,
                   group_tok_start=None, seg_rows=None, stream=None, device=None) -> int:
    G = ctypes.c_int64(0)
    dev = device if device is not None else torch.cuda.current_device()
    _check(library().l3_plan_export(plan.handle, _ptr(perm, "perm"), _ptr(inv_perm, "inv_perm"),
                                    _ptr(sorted_ids, "sorted_ids"), _ptr(group_ids, "group_ids"),
                                    _ptr(group_tok_start, "group_tok_start"),
                                    _ptr(seg_rows, "seg_rows"), ctypes.byref(G),
                                    _stream(stream, dev)))
    return int(G.value)


def l3_forward(x: torch.Tensor, plan: Plan, W_K, W_V, W_up, ln_gamma, ln_beta, W_mix,
               y: torch.Tensor, stream=None):
    names = ("x", "W_K", "W_V", "W_up", "ln_gamma", "ln_beta", "W_mix", "y")
    tensors = (x, W_K, W_V, W_up, ln_gamma, ln_beta, W_mix, y)
    want = torch.bfloat16 if plan.dims.dtype == L3_BF16 else torch.float32
    for nm, t in zip(names, tensors):
        if t.dtype != want:
            raise TypeError(f"{nm} must be {want}")
    d = plan.dims
    rows = plan.table_rows
    shapes = {"x": (plan.n_tokens, d.d_in), "W_K": (rows, d.d_in), "W_V": (rows, d.d_emb),
              "W_up": (d.d_up, d.d_emb), "ln_gamma": (d.d_up,), "ln_beta": (d.d_up,),
              "W_mix": (d.d_out, d.d_up + d.d_in), "y": (plan.n_tokens, d.d_out)}
    for nm, t in zip(names, tensors):
        if tuple(t.shape) != shapes[nm]:
            raise ValueError(f"{nm} has shape {tuple(t.shape)}, want {shapes[nm]}")
    ptrs = [_ptr(t, nm) for nm, t in zip(names, tensors)]
    _check(library().l3_forward(ptrs[0], plan.handle, *ptrs[1:7], ptrs[7],
                                _stream(stream, x.device)))


def l3_forward_status(plan: Plan):
    _check(library().l3_forward_status(plan.handle))


def l3_plan_destroy(plan: Plan):
    plan.destroy()


def l3_profile_enable(enable=True):
    """True or 1: time every launch; 2: every launch but the plan's; False or 0: off."""
    library().l3_profile_enable(int(enable) if not isinstance(enable, bool) else (1 if enable else 0))


def l3_profile_read(max_entries: int = 64) -> dict:
    buf = (KernelTime * max_entries)()
    n = library().l3_profile_read(buf, max_entries)
    if n < 0:
        raise L3Error(5, "l3_profile_read failed")
    return {buf[i].name.decode(): (int(buf[i].launches), float(buf[i].total_ms))
            for i in range(min(n, max_entries))}


def l3_sort_tokens_noalloc(token_ids: torch.Tensor, vocab: int, perm: torch.Tensor,
                           inv_perm: torch.Tensor, sorted_ids: torch.Tensor, stream=None):
    """Stable sort by token ID into caller-owned buffers, with no device
    allocation inside the library (fixed scratch array; see include/l3.h)."""
    for nm, t in (("token_ids", token_ids), ("perm", perm), ("inv_perm", inv_perm),
                  ("sorted_ids", sorted_ids)):
        if t.dtype != torch.int32:
            raise TypeError(f"{nm} must be int32")
    n = token_ids.numel()
    _check(library().l3_sort_tokens_noalloc(
        _ptr(token_ids, "token_ids") if n else None, n, vocab,
        _ptr(perm, "perm") if n else None, _ptr(inv_perm, "inv_perm") if n else None,
        _ptr(sorted_ids, "sorted_ids") if n else None, _stream(stream, token_ids.device)))
