"""Pins of the backward oracle: torch autograd through the masked-attention
statement of the layer (kimjy99 review §2: L³ over a batch is attention of
the batch over the full tables with a per-token row mask), and central finite
differences of the forward oracle."""
import numpy as np
import pytest
import torch

import oracle
from oracle import backward as bwd
from oracle_pins import masked_attention_reference, random_layer, run_oracle

NAMES = ("x", "W_K", "W_V", "W_up", "ln_gamma", "ln_beta", "W_mix")


@pytest.mark.parametrize("seed", range(5))
def test_matches_autograd_of_masked_attention(seed):
    layer = random_layer(seed, vocab=6, d_max=5, n=13)
    eps = 1e-5
    g = torch.Generator().manual_seed(100 + seed)
    g_y = torch.randn(13, layer["W_mix"].shape[0], generator=g, dtype=torch.float64)
    leaves = {k: layer[k].clone().requires_grad_(True) for k in NAMES}
    y = masked_attention_reference(dict(layer, **leaves), eps)
    y.backward(g_y)
    got = bwd.backward(layer["ids"], layer["offsets"], *[layer[k] for k in NAMES], eps, g_y)
    for k in NAMES:
        want = leaves[k].grad.numpy()
        scale = max(1.0, np.abs(want).max())
        assert np.abs(got[k] - want).max() <= 1e-10 * scale, k


def test_matches_finite_differences_of_the_forward_oracle():
    layer = random_layer(7, vocab=5, d_max=4, d_in=4, d_emb=3, d_up=5, d_out=3, n=9)
    eps = 1e-3
    g_y = np.random.default_rng(1).standard_normal((9, 3))

    def loss(lay):
        return float((run_oracle(lay, eps) * g_y).sum())

    got = bwd.backward(layer["ids"], layer["offsets"], *[layer[k] for k in NAMES], eps, g_y)
    rng = np.random.default_rng(2)
    step = 1e-6
    for k in NAMES:
        flat = layer[k].reshape(-1)
        for idx in rng.choice(flat.numel(), size=min(6, flat.numel()), replace=False):
            plus = {kk: vv.clone() for kk, vv in layer.items()}
            minus = {kk: vv.clone() for kk, vv in layer.items()}
            plus[k].reshape(-1)[idx] += step
            minus[k].reshape(-1)[idx] -= step
            fd = (loss(plus) - loss(minus)) / (2 * step)
            an = got[k].reshape(-1)[idx]
            assert abs(fd - an) <= 1e-5 * max(1.0, abs(fd)), (k, idx, fd, an)


def test_rows_outside_the_batch_get_no_gradient():
    layer = random_layer(3, vocab=8, d_max=3, n=4)
    got = bwd.backward(layer["ids"], layer["offsets"], *[layer[k] for k in NAMES], 1e-5,
                       np.ones((4, layer["W_mix"].shape[0])))
    off = layer["offsets"].numpy()
    used = np.zeros(int(off[-1]), dtype=bool)
    for t in set(layer["ids"].tolist()):
        used[off[t]:off[t + 1]] = True
    assert not got["W_K"][~used].any() and not got["W_V"][~used].any()
