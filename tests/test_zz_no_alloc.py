"""The allocation-free sort entry point, through the C ABI.

l3_sort_tokens_noalloc serves callers that cannot allocate device memory
(an engine that has reserved nearly all of HBM, or a loop that cannot take
the synchronisation of cudaMalloc/cudaFree): its scratch is a fixed device
array inside libl3.so. Its outputs must equal the ones l3_plan produces for
the same IDs, bit for bit (integer work), on two calls in a row, since the
second call finds the first call's data in the shared array. This file is
collected last so that a failure here stops a `-x` run only after every
other test has run.
"""
import ctypes

import numpy as np
import pytest
import torch

import static_token_routed_b200 as l3

pytestmark = pytest.mark.gpu


def _plan_sort(ids: torch.Tensor, vocab: int):
    off = torch.arange(0, vocab + 1, dtype=torch.int32, device=ids.device)
    plan = l3.l3_plan(ids, off, l3.make_dims(vocab, vocab, 1, 16, 16, 16, 16))
    n = ids.numel()
    out = [torch.empty(n, dtype=torch.int32, device=ids.device) for _ in range(3)]
    l3.l3_plan_export(plan, perm=out[0], inv_perm=out[1], sorted_ids=out[2])
    torch.cuda.synchronize()
    plan.destroy()
    return out


def _noalloc_sort_via_c_abi(ids: torch.Tensor, vocab: int):
    lib = l3.library()
    n = ids.numel()
    out = [torch.full((n,), -1, dtype=torch.int32, device=ids.device) for _ in range(3)]
    stream = torch.cuda.current_stream().cuda_stream
    st = lib.l3_sort_tokens_noalloc(ctypes.c_void_p(ids.data_ptr()), n, vocab,
                                    ctypes.c_void_p(out[0].data_ptr()),
                                    ctypes.c_void_p(out[1].data_ptr()),
                                    ctypes.c_void_p(out[2].data_ptr()), ctypes.c_void_p(stream))
    assert st == 0, l3.l3_last_error()
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("vocab,n", [(180000, 65536), (32000, 3000)])
def test_noalloc_sort_matches_plan_twice(vocab, n):
    for call, seed in enumerate((11, 12)):   # two calls in a row, different batches
        rng = np.random.default_rng(seed + vocab)
        p = 1.0 / np.arange(1, vocab + 1) ** 1.1
        ids_np = rng.choice(vocab, size=n - call * 7, p=p / p.sum()).astype(np.int32)
        ids = torch.from_numpy(ids_np).cuda()
        want = _plan_sort(ids, vocab)
        got = _noalloc_sort_via_c_abi(ids, vocab)
        for name, g, w in zip(("perm", "inv_perm", "sorted_ids"), got, want):
            assert torch.equal(g, w), f"call {call}: {name} differs from l3_plan"


def test_noalloc_sort_rejects_oversize():
    lib = l3.library()
    st = lib.l3_sort_tokens_noalloc(None, l3.L3_SORT_NOALLOC_MAX_TOKENS + 1, 10, None, None, None,
                                    None)
    assert st == 1 and "65536" in l3.l3_last_error()
