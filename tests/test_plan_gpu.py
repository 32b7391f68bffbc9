"""l3_plan on the GPU against the oracle's stable counting sort, bit for bit
(sciencestack Fig. 3: sort the batch by token ID; the stable reading makes
the plan unique)."""
import numpy as np
import pytest
import torch

import oracle
import static_token_routed_b200 as l3
from l3_cases import dims_of, host_workload
from static_token_routed_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def export(plan, n, dev="cuda"):
    bufs = {k: torch.full((n,), -7, dtype=torch.int32, device=dev)
            for k in ("perm", "inv_perm", "sorted_ids")}
    gbufs = {k: torch.full((n + 1,), -7, dtype=torch.int32, device=dev)
             for k in ("group_ids", "group_tok_start", "seg_rows")}
    G = l3.l3_plan_export(plan, **bufs, **gbufs)
    torch.cuda.synchronize()
    out = {k: v.cpu().numpy() for k, v in bufs.items()}
    out["group_ids"] = gbufs["group_ids"][:G].cpu().numpy()
    out["group_tok_start"] = gbufs["group_tok_start"][:G + 1].cpu().numpy()
    out["seg_rows"] = gbufs["seg_rows"][:G + 1].cpu().numpy()
    out["G"] = G
    return out


def check_plan(ids: np.ndarray, offsets: np.ndarray, dims):
    plan = l3.l3_plan(torch.from_numpy(ids).cuda(), torch.from_numpy(offsets).cuda(), dims)
    got = export(plan, len(ids))
    want = oracle.plan(ids, offsets)
    assert got["G"] == want["G"]
    for k in ("perm", "inv_perm", "sorted_ids", "group_ids", "group_tok_start", "seg_rows"):
        assert np.array_equal(got[k], want[k]), k
    info = plan.info()
    assert info.n_groups == want["G"] and info.unique_rows == want["seg_rows"][-1]
    plan.destroy()


@pytest.mark.parametrize("name", sorted(wl.WORKLOADS))
def test_plan_matches_oracle(name):
    w, t, b = host_workload(name)
    check_plan(b.ids.numpy(), t.offsets.numpy(), dims_of(w))


@pytest.mark.parametrize("vocab,n,seed", [(1, 5, 0), (2, 1, 1), (300, 4096, 2), (70000, 2049, 3),
                                          (1 << 20, 9000, 4), (5, 65537, 5)])
def test_plan_edge_shapes(vocab, n, seed):
    rng = np.random.default_rng(seed)
    ids = rng.integers(0, vocab, size=n).astype(np.int32)
    d = rng.integers(1, 4, size=vocab)
    off = np.concatenate([[0], np.cumsum(d)]).astype(np.int32)
    dims = l3.make_dims(vocab, int(off[-1]), 3, 16, 16, 16, 16)
    check_plan(ids, off, dims)


def test_all_tokens_one_id():
    ids = np.full(10000, 3, dtype=np.int32)
    off = np.arange(0, 11, dtype=np.int32) * 2
    check_plan(ids, off, l3.make_dims(10, 20, 2, 16, 16, 16, 16))


def test_empty_batch():
    off = torch.arange(0, 11, dtype=torch.int32, device="cuda")
    plan = l3.l3_plan(torch.empty(0, dtype=torch.int32, device="cuda"), off,
                      l3.make_dims(10, 10, 1, 16, 16, 16, 16))
    assert plan.info().n_groups == 0
    y = torch.empty(0, 16, dtype=torch.bfloat16, device="cuda")
    z = torch.zeros(16, 16, dtype=torch.bfloat16, device="cuda")
    # N = 0: nothing to do, but pointers are still checked
    l3.l3_forward(torch.empty(0, 16, dtype=torch.bfloat16, device="cuda"), plan,
                  torch.zeros(10, 16, dtype=torch.bfloat16, device="cuda"),
                  torch.zeros(10, 16, dtype=torch.bfloat16, device="cuda"), z,
                  torch.ones(16, dtype=torch.bfloat16, device="cuda"),
                  torch.zeros(16, dtype=torch.bfloat16, device="cuda"),
                  torch.zeros(16, 32, dtype=torch.bfloat16, device="cuda"), y)
    plan.destroy()


def test_token_out_of_range_is_reported():
    off = torch.arange(0, 11, dtype=torch.int32, device="cuda")
    ids = torch.tensor([0, 5, 10, 2], dtype=torch.int32, device="cuda")
    with pytest.raises(l3.L3Error) as e:
        l3.l3_plan(ids, off, l3.make_dims(10, 10, 1, 16, 16, 16, 16))
    assert e.value.status == 2
    ids = torch.tensor([0, -1], dtype=torch.int32, device="cuda")
    with pytest.raises(l3.L3Error) as e:
        l3.l3_plan(ids, off, l3.make_dims(10, 10, 1, 16, 16, 16, 16))
    assert e.value.status == 2


@pytest.mark.parametrize("bad", ["zero_row", "over_cap", "sum", "start"])
def test_bad_offsets_are_reported(bad):
    off = np.arange(0, 11, dtype=np.int32) * 2   # d_t = 2, v = 20
    k, v = 2, 20
    if bad == "zero_row":
        off[4] = off[3]
    elif bad == "over_cap":
        k = 1
    elif bad == "sum":
        v = 21
    elif bad == "start":
        off = off + 1
        v = 21
    ids = torch.tensor([1, 2, 3], dtype=torch.int32, device="cuda")
    with pytest.raises(l3.L3Error) as e:
        l3.l3_plan(ids, torch.from_numpy(off).cuda(), l3.make_dims(10, v, k, 16, 16, 16, 16))
    assert e.value.status == 3
