"""Failure detection on the GPU without a fault: a bounded wait that can
never complete gives up, reports the timeout to the host, and the context
stays usable for the next forward (checked against the oracle)."""
import time

import pytest
import torch

import oracle
import static_token_routed_b200 as l3
from l3_cases import EPS, TOL, host_workload, rel_max_err, run_forward, to_device

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_the_context_stays_usable():
    t0 = time.perf_counter()
    st = l3.l3_check_bounded_wait()
    dt = time.perf_counter() - t0
    assert st == 6, (st, l3.l3_last_error())          # L3_ERR_TIMEOUT
    assert 1.5 < dt < 30.0, dt                          # the 2 s limit, not a hang
    w, t, b = host_workload("small_bf16", 512)
    y, _ = run_forward(w, to_device(t, b))
    torch.cuda.synchronize()
    want = oracle.forward(b.ids, t.offsets, b.x, t.W_K, t.W_V, t.W_up, t.ln_gamma, t.ln_beta,
                          t.W_mix, EPS)
    assert rel_max_err(y.double().cpu().numpy(), want) <= TOL["bf16"]
