"""The CPU oracle against what the pages and the mathematics fix (no GPU)."""
import json
import os

import numpy as np
import pytest
import torch
from hypothesis import given, settings, strategies as st

import oracle
import oracle_pins as pins
from static_token_routed_b200 import workloads as wl


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin()


def test_bf16_inputs_widen_exactly():
    """bf16 inputs are widened exactly: the oracle on bf16 tensors equals the
    oracle on the same values stored as fp64, bit for bit."""
    layer = pins.random_layer(3, dtype=torch.bfloat16)
    y16 = pins.run_oracle(layer, 1e-5)
    layer64 = {k: (v.double() if v.is_floating_point() else v) for k, v in layer.items()}
    assert np.array_equal(y16, pins.run_oracle(layer64, 1e-5))


def test_select_matches_full():
    layer = pins.random_layer(4, n=15)
    y = pins.run_oracle(layer, 1e-5)
    sel = np.array([14, 0, 7, 7])
    assert np.array_equal(pins.run_oracle(layer, 1e-5, select=sel), y[sel])


def test_out_of_range_id_is_an_error():
    layer = pins.random_layer(0)
    layer["ids"] = layer["ids"].clone()
    layer["ids"][3] = 7  # vocab is 7
    with pytest.raises(oracle.OracleError):
        pins.run_oracle(layer, 1e-5)
    with pytest.raises(oracle.OracleError):
        oracle.plan(layer["ids"], layer["offsets"])


@settings(max_examples=25, deadline=None)
@given(seed=st.integers(0, 10_000), vocab=st.integers(1, 6), d_max=st.integers(1, 8),
       d_in=st.integers(1, 7), d_emb=st.integers(1, 7), d_up=st.integers(2, 7),
       d_out=st.integers(1, 5), n=st.integers(1, 12))
def test_masked_attention_property(seed, vocab, d_max, d_in, d_emb, d_up, d_out, n):
    """Hypothesis sweep of the masked-dense-attention equivalence on tiny shapes."""
    layer = pins.random_layer(seed, vocab=vocab, d_max=d_max, d_in=d_in, d_emb=d_emb,
                              d_up=d_up, d_out=d_out, n=n)
    got = pins.run_oracle(layer, 1e-5)
    want = pins.masked_attention_reference(layer, 1e-5).numpy()
    assert pins.rel_err(got, want) < 1e-11


def test_regression_fixture():
    """Oracle outputs stored by tests/golden/make_oracle_regression.py (which
    calls only the oracle) for sampled tokens of the tiny fp32 workload."""
    path = os.path.join(pins.GOLDEN, "oracle_tiny_fp32_sample.json")
    with open(path) as f:
        fx = json.load(f)
    w = wl.WORKLOADS[fx["workload"]]
    t = wl.make_tables(w)
    b = wl.make_batch(w)
    y = oracle.forward(b.ids, t.offsets, b.x, t.W_K, t.W_V, t.W_up, t.ln_gamma, t.ln_beta,
                       t.W_mix, fx["eps"], select=fx["tokens"])
    np.testing.assert_allclose(y, np.array(fx["y"]), rtol=0, atol=1e-12)
