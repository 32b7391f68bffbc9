"""The allocation-free sort entry point, through the C ABI.

l3_sort_tokens_noalloc serves callers that cannot allocate device memory
(an engine that has reserved nearly all of HBM, or a loop that cannot take
the synchronisation of cudaMalloc/cudaFree): its scratch is a fixed device
array inside libl3.so. Its outputs must equal, bit for bit (integer work),
both the oracle's stable counting sort and what l3_plan produces for the
same IDs, on two calls in a row, since the second call finds the first
call's data in the shared array. The cases cover one, two and three radix
passes of 9-bit digits (vocab <= 512, <= 262144, larger). This file is collected last so
that a failure here stops a `-x` run only after every other test has run.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
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


@pytest.mark.parametrize("vocab,n", [(300000, 65536), (180000, 65536), (32000, 3000), (200, 5000)])
def test_noalloc_sort_matches_plan_twice(vocab, n):
    for call, seed in enumerate((11, 12)):   # two calls in a row, different batches
        rng = np.random.default_rng(seed + vocab)
        p = 1.0 / np.arange(1, vocab + 1) ** 1.1
        ids_np = rng.choice(vocab, size=n - call * 7, p=p / p.sum()).astype(np.int32)
        ids = torch.from_numpy(ids_np).cuda()
        got = _noalloc_sort_via_c_abi(ids, vocab)
        ref = oracle.plan(ids_np, np.arange(vocab + 1, dtype=np.int32))
        for name, g in zip(("perm", "inv_perm", "sorted_ids"), got):
            assert np.array_equal(g.cpu().numpy(), ref[name]), \
                f"call {call}: {name} differs from the oracle"
        want = _plan_sort(ids, vocab)
        for name, g, w in zip(("perm", "inv_perm", "sorted_ids"), got, want):
            assert torch.equal(g, w), f"call {call}: {name} differs from l3_plan"


def test_noalloc_sort_rejects_overlap():
    lib = l3.library()
    ids = torch.zeros(64, dtype=torch.int32, device="cuda")
    out = torch.empty(64, dtype=torch.int32, device="cuda")
    p = lambda t, k=0: ctypes.c_void_p(t.data_ptr() + 4 * k)  # noqa: E731
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # the input as an output, and two outputs sharing half their range
    for args in ((p(ids), p(out), p(ids), p(ids)),
                 (p(ids), p(out), p(out, 32), p(torch.empty_like(out)))):
        st = lib.l3_sort_tokens_noalloc(args[0], 64, 10, *args[1:], stream)
        assert st == 1 and "overlap" in l3.l3_last_error()


def test_noalloc_sort_rejects_oversize():
    lib = l3.library()
    st = lib.l3_sort_tokens_noalloc(None, l3.L3_SORT_NOALLOC_MAX_TOKENS + 1, 10, None, None, None,
                                    None)
    assert st == 1 and "65536" in l3.l3_last_error()
