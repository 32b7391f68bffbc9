"""The error measures the parity tests use (CPU only)."""
import numpy as np
import torch

from l3_cases import bf16_half_ulp, rel_max_err, rounding_floor, within_bf16_bar


def test_half_ulp_matches_bf16_spacing():
    for v in [1.0, 1.5, 4.5, -3.0, 0.1, 1e-3, 123.0]:
        t = torch.tensor([v], dtype=torch.float64)
        up = torch.nextafter(t.to(torch.bfloat16), torch.tensor([np.inf], dtype=torch.bfloat16))
        lo = t.to(torch.bfloat16)
        spacing = abs(float(up.double()) - float(lo.double()))
        # at a power of two the spacing above is the one that applies to |v| >= it
        assert bf16_half_ulp(np.array([v]))[0] == spacing / 2, v


def test_exactly_rounded_result_meets_the_relaxed_bar():
    rng = np.random.default_rng(0)
    want = rng.standard_normal((64, 256)) * np.exp(rng.standard_normal((64, 1)))
    rounded = torch.from_numpy(want).to(torch.bfloat16).double().numpy()
    assert within_bf16_bar(rounded, want, 0.0)
    assert abs(rounding_floor(want) - rel_max_err(rounded, want)) < 1e-15
    # one element off by more than tol * RMS + half an ulp fails
    bad = rounded.copy()
    rms = np.sqrt(np.mean(want ** 2))
    bad[3, 7] = want[3, 7] + 0.02 * rms + 2 * bf16_half_ulp(want[3:4, 7:8])[0, 0]
    assert not within_bf16_bar(bad, want, 0.02)
