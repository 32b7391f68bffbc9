"""Oracle of the L³ layer's backward pass — test infrastructure.

Only `tests/` may import this module; the library never calls it.

The layer (kimjy99 review, Method, eq. L³), per token n with ID t and rows
K_t, V_t (the d_t-row slices of W_K, W_V):

    s = K_t x;  p = softmax(s);  a = V_t^T p;  z = W_up a;
    h = gamma * (z - mean z) / sqrt(var z + eps) + beta;  y = W_mix [h ; x]

Given dL/dy, this returns dL/dx and the gradients of every weight, in fp64,
token by token, by the chain rule written out step by step:

    dW_mix += g_y [h ; x]^T          g_h = W_mix[:, :d_up]^T g_y
                                     g_x = W_mix[:, d_up:]^T g_y
    dgamma += g_h * hhat             dbeta += g_h
    g_hhat = g_h * gamma
    g_z = (g_hhat - mean(g_hhat) - hhat * mean(g_hhat * hhat)) / sqrt(var z + eps)
    dW_up += g_z a^T                 g_a = W_up^T g_z
    g_p = V_t g_a                    dV_t += p g_a^T
    g_s = p * (g_p - p . g_p)
    dK_t += g_s x^T                  g_x += K_t^T g_s

(the LayerNorm and softmax derivatives are the textbook ones; the rest is
the product rule on the equation). Rows of W_K / W_V outside every K_t of
the batch get zero gradient. Plain numpy in fp64, one token at a time.
"""
from __future__ import annotations

import numpy as np
import torch


def _f64(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().to(torch.float64).cpu().numpy()
    return np.asarray(t, dtype=np.float64)


def backward(ids, offsets, x, W_K, W_V, W_up, ln_gamma, ln_beta, W_mix, eps: float, g_y) -> dict:
    ids = np.asarray(ids).astype(np.int64)
    off = np.asarray(offsets).astype(np.int64)
    x, W_K, W_V, W_up = _f64(x), _f64(W_K), _f64(W_V), _f64(W_up)
    gamma, W_mix, g_y = _f64(ln_gamma), _f64(W_mix), _f64(g_y)
    d_up = W_up.shape[0]
    grads = {"x": np.zeros_like(x), "W_K": np.zeros_like(W_K), "W_V": np.zeros_like(W_V),
             "W_up": np.zeros_like(W_up), "ln_gamma": np.zeros_like(gamma),
             "ln_beta": np.zeros_like(gamma), "W_mix": np.zeros_like(W_mix)}
    for n in range(len(ids)):
        r0, r1 = off[ids[n]], off[ids[n] + 1]
        K, V, xn = W_K[r0:r1], W_V[r0:r1], x[n]
        # forward of this token
        s = K @ xn
        e = np.exp(s - s.max())
        p = e / e.sum()
        a = V.T @ p
        z = W_up @ a
        mu = z.mean()
        rstd = 1.0 / np.sqrt(((z - mu) ** 2).mean() + eps)
        hhat = (z - mu) * rstd
        h = gamma * hhat + _f64(ln_beta)
        # backward
        gy = g_y[n]
        grads["W_mix"] += np.outer(gy, np.concatenate([h, xn]))
        g_h = W_mix[:, :d_up].T @ gy
        g_x = W_mix[:, d_up:].T @ gy
        grads["ln_gamma"] += g_h * hhat
        grads["ln_beta"] += g_h
        g_hhat = g_h * gamma
        g_z = (g_hhat - g_hhat.mean() - hhat * (g_hhat * hhat).mean()) * rstd
        grads["W_up"] += np.outer(g_z, a)
        g_a = W_up.T @ g_z
        g_p = V @ g_a
        grads["W_V"][r0:r1] += np.outer(p, g_a)
        g_s = p * (g_p - p @ g_p)
        grads["W_K"][r0:r1] += np.outer(g_s, xn)
        g_x = g_x + K.T @ g_s
        grads["x"][n] = g_x
    return grads
