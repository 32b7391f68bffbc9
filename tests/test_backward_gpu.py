"""l3_backward on the GPU against the fp64 backward oracle (chain rule of
kimjy99 review, Method, eq. L³), gradient by gradient, on the same seeded
inputs: max |err| <= 1e-4 x RMS for the fp32 layer and 2e-2 x RMS for bf16
(the same bars as the forward)."""
import numpy as np
import pytest
import torch

import static_token_routed_b200 as l3
from l3_cases import EPS, TOL, dims_of, host_workload, rel_max_err, run_forward, to_device
from oracle import backward as bwd
from static_token_routed_b200 import workloads as wl

pytestmark = pytest.mark.gpu

NAMES = ("x", "W_K", "W_V", "W_up", "ln_gamma", "ln_beta", "W_mix")


def check(w, t, b, dims, tol, seed=0, names=NAMES):
    dev = to_device(t, b)
    plan = l3.l3_plan(dev["ids"], dev["offsets"], dims)
    y = torch.empty(b.ids.numel(), w.d_out, dtype=w.torch_dtype, device="cuda")
    l3.l3_forward(dev["x"], plan, dev["W_K"], dev["W_V"], dev["W_up"], dev["ln_gamma"],
                  dev["ln_beta"], dev["W_mix"], y)
    g = torch.Generator().manual_seed(seed)
    dy = torch.randn(b.ids.numel(), w.d_out, generator=g).to(w.torch_dtype)
    got = l3.l3_backward(dev["x"], plan, dev["W_K"], dev["W_V"], dev["W_up"], dev["ln_gamma"],
                         dev["ln_beta"], dev["W_mix"], dy.cuda())
    l3.l3_forward_status(plan)
    want = bwd.backward(b.ids, t.offsets, b.x, t.W_K, t.W_V, t.W_up, t.ln_gamma, t.ln_beta,
                        t.W_mix, EPS, dy)
    errs = {k: rel_max_err(got[k].double().cpu().numpy(), want[k]) for k in names}
    assert all(e <= tol for e in errs.values()), ", ".join(f"{k} {e:.3g}" for k, e in errs.items())
    # a second call gives the same bits, except dW_K / dW_V whose rows take
    # atomic adds from several units of a group
    again = l3.l3_backward(dev["x"], plan, dev["W_K"], dev["W_V"], dev["W_up"], dev["ln_gamma"],
                           dev["ln_beta"], dev["W_mix"], dy.cuda())
    for k in names:
        if k in ("W_K", "W_V"):
            assert rel_max_err(again[k].double().cpu().numpy(), want[k]) <= tol, k
        else:
            assert torch.equal(got[k], again[k]), k


def small_layer(vocab, rows, n, d_in, d_emb, d_up, d_out, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    off = torch.tensor([0] + list(rows), dtype=torch.int64).cumsum(0).to(torch.int32)
    v = int(off[-1])
    ids = torch.randint(0, vocab, (n,), generator=g, dtype=torch.int32)
    mk = lambda *s: (torch.randn(*s, generator=g) / s[-1] ** 0.5).to(dtype)
    t = wl.Tables(off, mk(v, d_in) * 4, mk(v, d_emb), mk(d_up, d_emb),
                  (1 + 0.1 * torch.randn(d_up, generator=g)).to(dtype),
                  (0.1 * torch.randn(d_up, generator=g)).to(dtype), mk(d_out, d_up + d_in))
    b = wl.Batch(ids, mk(n, d_in) * 4)
    dims = l3.make_dims(vocab, v, max(rows), d_in, d_emb, d_up, d_out, dtype, EPS)
    return t, b, dims


def test_backward_tiny_fp32():
    w, t, b = host_workload("tiny_fp32")
    check(w, t, b, dims_of(w), TOL["fp32"])


@pytest.mark.parametrize("vocab,rows,n,d_in,d_emb,d_up,d_out", [
    # dense groups of both sizes and short ones in one batch
    (6, (300, 96, 512, 256, 257, 33), 900, 64, 512, 64, 32),
    # groups of several 128-token tiles (units of one group share its rows)
    (3, (511, 260, 96), 1200, 128, 256, 64, 32),
    # many short groups, single rows among them
    (50, tuple(int(r) for r in np.random.default_rng(5).integers(1, 9, size=50)), 300, 128, 64,
     192, 80),
])
def test_backward_bf16(vocab, rows, n, d_in, d_emb, d_up, d_out):
    t, b, dims = small_layer(vocab, rows, n, d_in, d_emb, d_up, d_out, torch.bfloat16, vocab)
    w = wl.Workload("case", vocab, int(sum(rows)), max(rows), d_in, d_emb, d_up, d_out, n, "bf16",
                    "zipf", "zipf", 0, 0)
    check(w, t, b, dims, TOL["bf16"])


def test_backward_neighbour_rows_never_reach_a_group():
    """Static routing in the backward: the dense tiles' scores and g_p read
    K_t / V_t in blocks padded to 16 rows, which also cover the first rows of
    the next IDs. Here those IDs, absent from the batch, hold NaN, +-Inf and
    values past fp16's range in both tables: every gradient must stay finite
    and match the oracle."""
    vocab = 5
    rows = (300, 5, 200, 7, 40)   # IDs 1 and 3 are never in the batch
    off = torch.tensor([0] + list(rows), dtype=torch.int64).cumsum(0).to(torch.int32)
    v, d_in, d_emb, d_up, d_out = int(off[-1]), 256, 512, 64, 64
    g = torch.Generator().manual_seed(12)
    mk = lambda *s: (torch.randn(*s, generator=g) / s[-1] ** 0.5).to(torch.bfloat16)  # noqa: E731
    W_K, W_V = mk(v, d_in), mk(v, d_emb)
    poison = torch.tensor([float("nan"), float("inf"), float("-inf"), 1e6, -3e5],
                          dtype=torch.bfloat16)
    for t_id in (1, 3):
        for j, r in enumerate(range(int(off[t_id]), int(off[t_id + 1]))):
            W_K[r] = poison[j % 5]
            W_V[r] = poison[(j + 2) % 5]
    n = 700
    ids = torch.tensor([(0, 2, 4)[i % 3] for i in range(n)], dtype=torch.int32)
    ids = ids[torch.randperm(n, generator=g)].contiguous()
    t = wl.Tables(off, W_K, W_V, mk(d_up, d_emb),
                  (1 + 0.1 * torch.randn(d_up, generator=g)).to(torch.bfloat16),
                  (0.1 * torch.randn(d_up, generator=g)).to(torch.bfloat16), mk(d_out, d_up + d_in))
    b = wl.Batch(ids, mk(n, d_in) * 4)
    dims = l3.make_dims(vocab, v, max(rows), d_in, d_emb, d_up, d_out, torch.bfloat16, EPS)
    w = wl.Workload("case", vocab, v, max(rows), d_in, d_emb, d_up, d_out, n, "bf16", "zipf",
                    "zipf", 0, 0)
    check(w, t, b, dims, TOL["bf16"])


def test_backward_dense_dx_on_tensor_cores():
    """d_in a multiple of 256, so the dense tiles' dx = K_t^T g_s also runs on
    the tensor cores (besides their scores): d_t on and off multiples of 16,
    ragged 32-token chunks, a 512-row group. The attention gradients (x, W_K,
    W_V) are this case's subject; the GEMM-side ones are covered above."""
    vocab, rows, n, d_in, d_emb, d_up, d_out = 5, (512, 300, 257, 100, 37), 1100, 256, 256, 64, 32
    t, b, dims = small_layer(vocab, rows, n, d_in, d_emb, d_up, d_out, torch.bfloat16, vocab)
    w = wl.Workload("case", vocab, int(sum(rows)), max(rows), d_in, d_emb, d_up, d_out, n, "bf16",
                    "zipf", "zipf", 0, 0)
    check(w, t, b, dims, TOL["bf16"], names=("x", "W_K", "W_V"))


def test_backward_on_its_own_stream_then_replan():
    """Forward on one stream, backward on another, the plan destroyed right
    after and a new plan of the same size built and run at once on a third:
    the new plan may reuse the old one's device block only after the backward
    that reads it (a, h, the work lists) has finished, so the gradients still
    match the oracle."""
    vocab, rows, n, d_in, d_emb, d_up, d_out = 6, (300, 96, 512, 256, 257, 33), 900, 64, 512, 64, 32
    t, b, dims = small_layer(vocab, rows, n, d_in, d_emb, d_up, d_out, torch.bfloat16, 7)
    dev = to_device(t, b)
    g = torch.Generator().manual_seed(3)
    dy = torch.randn(n, d_out, generator=g).to(torch.bfloat16)
    dy_d = dy.cuda()
    s_fwd, s_bwd, s_next = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    for s in (s_fwd, s_bwd, s_next):
        s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s_fwd):
        plan = l3.l3_plan(dev["ids"], dev["offsets"], dims, s_fwd)
        y = torch.empty(n, d_out, dtype=torch.bfloat16, device="cuda")
        l3.l3_forward(dev["x"], plan, dev["W_K"], dev["W_V"], dev["W_up"], dev["ln_gamma"],
                      dev["ln_beta"], dev["W_mix"], y, s_fwd)
    s_bwd.wait_stream(s_fwd)
    with torch.cuda.stream(s_bwd):
        got = l3.l3_backward(dev["x"], plan, dev["W_K"], dev["W_V"], dev["W_up"],
                             dev["ln_gamma"], dev["ln_beta"], dev["W_mix"], dy_d, s_bwd)
    plan.destroy()  # no host wait before it: the backward may still be running
    # other IDs of the same count: same plan size, different sort and groups
    ids2 = torch.flip(dev["ids"], [0]).contiguous()
    with torch.cuda.stream(s_next):
        plan2 = l3.l3_plan(ids2, dev["offsets"], dims, s_next)
        y2 = torch.empty(n, d_out, dtype=torch.bfloat16, device="cuda")
        l3.l3_forward(dev["x"], plan2, dev["W_K"], dev["W_V"], dev["W_up"], dev["ln_gamma"],
                      dev["ln_beta"], dev["W_mix"], y2, s_next)
    l3.l3_forward_status(plan2)
    torch.cuda.synchronize()
    plan2.destroy()
    want = bwd.backward(b.ids, t.offsets, b.x, t.W_K, t.W_V, t.W_up, t.ln_gamma, t.ln_beta,
                        t.W_mix, EPS, dy)
    errs = {k: rel_max_err(got[k].double().cpu().numpy(), want[k]) for k in NAMES}
    assert all(e <= TOL["bf16"] for e in errs.values()), errs


def test_backward_paper_shaped_full_batch_sampled_dy():
    """The full paper-shaped batch (65,536 tokens: every dense tile, tail class
    and launch the bench's backward runs), with dL/dy nonzero on 384 sampled
    tokens only. The backward is linear in dL/dy and a token with zero dL/dy
    contributes nothing, so every gradient equals the oracle's backward over
    the sampled tokens alone: dx on those tokens (exactly zero elsewhere),
    dW_K / dW_V on every row, dW_up, dgamma, dbeta and dW_mix in full."""
    from l3_cases import host_workload, sample_tokens
    w, t, b = host_workload("paper_shaped")
    dev = to_device(t, b)
    dims = l3.make_dims(w.vocab, w.v, w.k, w.d_in, w.d_emb, w.d_up, w.d_out, w.torch_dtype, EPS)
    plan = l3.l3_plan(dev["ids"], dev["offsets"], dims)
    y = torch.empty(w.n_tokens, w.d_out, dtype=w.torch_dtype, device="cuda")
    l3.l3_forward(dev["x"], plan, dev["W_K"], dev["W_V"], dev["W_up"], dev["ln_gamma"],
                  dev["ln_beta"], dev["W_mix"], y)
    sel = sample_tokens(b.ids.numpy(), t.offsets.numpy(), 384, seed=3)
    g = torch.Generator().manual_seed(4)
    dy = torch.zeros(w.n_tokens, w.d_out, dtype=w.torch_dtype)
    dy[torch.from_numpy(sel)] = torch.randn(len(sel), w.d_out, generator=g).to(w.torch_dtype)
    got = l3.l3_backward(dev["x"], plan, dev["W_K"], dev["W_V"], dev["W_up"], dev["ln_gamma"],
                         dev["ln_beta"], dev["W_mix"], dy.cuda())
    l3.l3_forward_status(plan)
    plan.destroy()
    # the oracle on a compact table holding only the sampled tokens' IDs (the
    # full tables in fp64 would take tens of GB of host memory)
    ids_s = np.unique(b.ids.numpy()[sel])
    off = t.offsets.numpy().astype(np.int64)
    rows = np.concatenate([np.arange(off[i], off[i + 1]) for i in ids_s])
    compact = {int(i): j for j, i in enumerate(ids_s)}
    d_s = off[ids_s + 1] - off[ids_s]
    off_c = torch.from_numpy(np.concatenate([[0], np.cumsum(d_s)]).astype(np.int32))
    ids_c = torch.tensor([compact[int(i)] for i in b.ids.numpy()[sel]], dtype=torch.int32)
    rows_h = torch.from_numpy(rows)
    want = bwd.backward(ids_c, off_c, b.x[sel], t.W_K[rows_h], t.W_V[rows_h], t.W_up, t.ln_gamma,
                        t.ln_beta, t.W_mix, EPS, dy[torch.from_numpy(sel)])
    dx = got["x"]
    mask = torch.ones(w.n_tokens, dtype=torch.bool)
    mask[torch.from_numpy(sel)] = False
    assert torch.count_nonzero(dx[mask.cuda()]) == 0
    errs = {"x": rel_max_err(dx[torch.from_numpy(sel).cuda()].double().cpu().numpy(), want["x"])}
    for k in ("W_up", "ln_gamma", "ln_beta", "W_mix"):
        errs[k] = rel_max_err(got[k].double().cpu().numpy(), want[k])
    # dW_K / dW_V: the rows of the sampled tokens' IDs carry the gradient; every
    # other row must stay exactly zero
    for k in ("W_K", "W_V"):
        gk = got[k]
        rows_t = torch.from_numpy(rows).cuda()
        errs[k] = rel_max_err(gk[rows_t].double().cpu().numpy(), want[k])
        other = torch.ones(gk.shape[0], dtype=torch.bool, device="cuda")
        other[rows_t] = False
        assert torch.count_nonzero(gk[other]) == 0, k
    assert all(e <= TOL["bf16"] for e in errs.values()), errs
