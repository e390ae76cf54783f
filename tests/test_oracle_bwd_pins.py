"""Pins of the oracle's attention gradients against what mathematics fixes:
torch's fp64 autograd through its own scaled_dot_product_attention, central
finite differences of the oracle's forward, and closed forms / invariants."""
import math

import numpy as np
import pytest
import torch


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _mask(Lq, Lk, causal, wl, wr):
    m = np.zeros((Lq, Lk), dtype=bool)
    for i in range(Lq):
        pos = i + Lk - Lq
        for j in range(Lk):
            m[i, j] = ((not causal or j <= pos) and (wr < 0 or j <= pos + wr) and (wl < 0 or j >= pos - wl))
    return m


@pytest.mark.parametrize("Lq,Lk,causal,wl,wr", [(12, 12, False, -1, -1), (12, 12, True, -1, -1),
                                                 (16, 16, False, 3, 2), (9, 14, True, -1, -1),
                                                 (15, 15, True, 4, 0)])
def test_grads_match_torch_autograd_fp64(oracle, Lq, Lk, causal, wl, wr):
    B, H, d = 2, 2, 5
    q, k, v, do = _rand((B, H, Lq, d), 1), _rand((B, H, Lk, d), 2), _rand((B, H, Lk, d), 3), _rand((B, H, Lq, d), 4)
    scale = 0.41
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, scale, causal, wl, wr)
    qt, kt, vt = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    mask = torch.from_numpy(_mask(Lq, Lk, causal, wl, wr))
    out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale)
    out.backward(torch.from_numpy(do))
    assert np.abs(dq - qt.grad.numpy()).max() < 1e-12
    assert np.abs(dk - kt.grad.numpy()).max() < 1e-12
    assert np.abs(dv - vt.grad.numpy()).max() < 1e-12


def test_grads_match_finite_differences(oracle):
    """Central differences of L = sum(dO * O) through the oracle's forward."""
    Lq, Lk, d = 6, 7, 3
    q, k, v, do = _rand((1, 1, Lq, d), 5), _rand((1, 1, Lk, d), 6), _rand((1, 1, Lk, d), 7), _rand((1, 1, Lq, d), 8)
    scale, causal, wl, wr = 0.7, True, 3, 0
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, scale, causal, wl, wr)

    def loss(q_, k_, v_):
        o, _ = oracle.attn(q_, k_, v_, scale, causal, wl, wr)
        return float((o * do).sum())

    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": q, "k": k, "v": v}
            args_m = dict(args_p)
            args_p[name], args_m[name] = xp, xm
            fd = (loss(args_p["q"], args_p["k"], args_p["v"]) - loss(args_m["q"], args_m["k"], args_m["v"])) / (2 * h)
            assert abs(fd - g[idx]) < 1e-7, (name, idx, fd, g[idx])


def test_constant_v_gives_zero_score_gradients(oracle):
    """With every V row equal, O does not depend on the scores: dQ = dK = 0 and
    dV_j = sum_i P_ij dO_i (so sum_j dV_j = sum_i dO_i)."""
    q, k, do = _rand((1, 2, 20, 4), 9), _rand((1, 2, 20, 4), 10), _rand((1, 2, 20, 4), 11)
    v = np.broadcast_to(_rand((4,), 12), (1, 2, 20, 4)).copy()
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, 0.5, True)
    assert np.abs(dq).max() < 1e-13 and np.abs(dk).max() < 1e-13
    assert np.abs(dv.sum(axis=2) - do.sum(axis=2)).max() < 1e-12


def test_key_gradients_sum_to_zero(oracle):
    """Each softmax row's dS sums to zero, so sum_j dK_j = 0 per head."""
    q, k, v, do = _rand((2, 2, 30, 6), 13), _rand((2, 2, 30, 6), 14), _rand((2, 2, 30, 6), 15), _rand((2, 2, 30, 6), 16)
    _, dk, _ = oracle.attn_bwd(q, k, v, do, 0.3, False, 5, 5)
    assert np.abs(dk.sum(axis=2)).max() < 1e-12


def test_rows_without_keys_have_zero_gradient(oracle):
    q, k, v, do = _rand((1, 1, 10, 4), 17), _rand((1, 1, 6, 4), 18), _rand((1, 1, 6, 4), 19), _rand((1, 1, 10, 4), 20)
    dq, _, _ = oracle.attn_bwd(q, k, v, do, 0.5, True)
    assert np.all(dq[0, 0, :4] == 0.0)
