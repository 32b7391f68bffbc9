"""Staged (CPU-offloaded) tables: l3_plan_staged + l3_stage_rows + l3_forward
(papernotes note, 关键设计 / CPU offload: a token's rows follow from its ID,
so they can be fetched before the layer runs).

The staged forward does the same arithmetic on the same values as the forward
over resident tables, so y must be bitwise equal; it is also checked against
the oracle on sampled tokens.
"""
import numpy as np
import pytest
import torch

import oracle
import static_token_routed_b200 as l3
from l3_cases import EPS, TOL, dims_of, host_workload, rel_max_err, run_forward, to_device

pytestmark = pytest.mark.gpu


def staged_forward(w, t, b, dev, from_host: bool, fill=float("nan")):
    dims = dims_of(w)
    plan = l3.l3_plan_staged(dev["ids"], dev["offsets"], dims)
    rows = plan.info().unique_rows
    # staged rows the copy leaves alone (W_K of single-row groups) hold NaN:
    # the forward must never read them
    Ks = torch.full((rows, w.d_in), fill, dtype=w.torch_dtype, device="cuda")
    Vs = torch.full((rows, w.d_emb), fill, dtype=w.torch_dtype, device="cuda")
    if from_host:
        WK = t.W_K.pin_memory()
        WV = WK if t.W_V is t.W_K else t.W_V.pin_memory()
    else:
        WK, WV = dev["W_K"], dev["W_V"]
    l3.l3_stage_rows(plan, WK, WV, Ks, Vs)
    y = torch.empty(b.ids.numel(), w.d_out, dtype=w.torch_dtype, device="cuda")
    l3.l3_forward(dev["x"], plan, Ks, Vs, dev["W_up"], dev["ln_gamma"], dev["ln_beta"],
                  dev["W_mix"], y)
    l3.l3_forward_status(plan)
    return y, plan, Ks, Vs


@pytest.mark.parametrize("name,n_tokens", [("small_bf16", 4096), ("paper_shaped", 2048),
                                           ("tiny_fp32", None), ("paper_tied", 1024),
                                           ("dense_stress", 4096)])
def test_staged_forward_equals_resident(name, n_tokens):
    w, t, b = host_workload(name, n_tokens)
    dev = to_device(t, b)
    y_res, _ = run_forward(w, dev)
    y_host, plan, Ks, Vs = staged_forward(w, t, b, dev, from_host=True)
    assert torch.equal(y_host, y_res)
    y_dev, _, _, _ = staged_forward(w, t, b, dev, from_host=False)
    assert torch.equal(y_dev, y_res)
    # the staged tables hold each group's rows at seg_rows[g]
    G = plan.info().n_groups
    gid = torch.empty(b.ids.numel() + 1, dtype=torch.int32, device="cuda")
    seg = torch.empty_like(gid)
    l3.l3_plan_export(plan, group_ids=gid, seg_rows=seg)
    torch.cuda.synchronize()
    off = t.offsets.numpy()
    gid, seg = gid.cpu().numpy()[:G], seg.cpu().numpy()[:G + 1]
    pick = np.random.default_rng(0).choice(G, size=min(G, 64), replace=False)
    for g in pick:
        src, d = off[gid[g]], off[gid[g] + 1] - off[gid[g]]
        assert torch.equal(Vs[seg[g]:seg[g] + d].cpu(), t.W_V[src:src + d])
        if d > 1:
            assert torch.equal(Ks[seg[g]:seg[g] + d].cpu(), t.W_K[src:src + d])


def test_staged_forward_matches_oracle():
    w, t, b = host_workload("small_bf16", 2048)
    dev = to_device(t, b)
    y, _, _, _ = staged_forward(w, t, b, dev, from_host=True)
    want = oracle.forward(b.ids, t.offsets, b.x, t.W_K, t.W_V, t.W_up, t.ln_gamma, t.ln_beta,
                          t.W_mix, EPS)
    assert rel_max_err(y.double().cpu().numpy(), want) <= TOL["bf16"]


def test_stage_rows_needs_a_staged_plan():
    w, t, b = host_workload("small_bf16", 256)
    dev = to_device(t, b)
    plan = l3.l3_plan(dev["ids"], dev["offsets"], dims_of(w))
    # shapes the binding accepts for a plan over resident tables; the library
    # itself refuses to stage rows for it
    with pytest.raises(l3.L3Error):
        l3.l3_stage_rows(plan, dev["W_K"], dev["W_V"], torch.empty_like(dev["W_K"]),
                         torch.empty_like(dev["W_V"]))
