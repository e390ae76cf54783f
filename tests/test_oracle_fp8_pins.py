"""Pins of the oracle's FP8 functions (the FP8 forward reading of the
"FlashAttention 深度解析" §4 FlashAttention-3 note): the e4m3 codec against
torch's float8_e4m3fn conversion and the format's closed forms, the
per-head quantizer against the same conversion, the FP8 attention recurrence
against the exact definition when P is not rounded, closed forms when every
score is equal, and the rounding-error bound when it is; for the exact
running max (slack 0) and for reading R13's reference slack of 4."""
import math

import numpy as np
import pytest
import torch


def _rng(seed):
    return np.random.default_rng(seed)


def test_e4m3_decode_all_codes_match_torch(oracle):
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan) and nan.sum() == 2   # 0x7F and 0xFF
    assert np.array_equal(ours[~nan], ref[~nan])


def test_e4m3_closed_forms(oracle):
    v = oracle.e4m3_decode(np.array([0x7E, 0x01, 0x08, 0x38, 0x07, 0x80], np.uint8))
    assert list(v[:5]) == [448.0, 2.0 ** -9, 2.0 ** -6, 1.0, 7 * 2.0 ** -9]
    assert v[5] == 0.0 and math.copysign(1.0, v[5]) == -1.0
    # saturation above the largest finite value, NaN to 0x7F
    assert list(oracle.e4m3_encode(np.array([448.0, 460.0, 1e6, -1e6, np.nan]))) == [0x7E, 0x7E, 0x7E, 0xFE, 0x7F]


def test_e4m3_encode_matches_torch(oracle):
    r = _rng(1)
    x = np.concatenate([r.standard_normal(20000) * s for s in (1e-3, 0.05, 1.0, 30.0, 120.0)])
    # exact midpoints between neighbours (ties go to the even code) and subnormals
    vals = oracle.e4m3_decode(np.arange(0, 0x7E, dtype=np.uint8))
    mids = (vals[:-1] + vals[1:]) / 2
    x = np.concatenate([x, mids, -mids, np.arange(0, 40) * 2.0 ** -11])
    x = x[np.abs(x) < 464.0]          # torch turns magnitudes >= 480 into NaN instead of saturating
    x = x.astype(np.float32).astype(np.float64)   # both sides convert the same fp32 values
    ours = oracle.e4m3_encode(x)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_quantize_matches_torch_conversion(oracle):
    x = torch.from_numpy(_rng(2).standard_normal((2, 3, 50, 64)).astype(np.float32)).to(torch.bfloat16)
    x[1, 2] = 0.0                                   # an all-zero head: descale 1, codes 0
    codes, desc = oracle.quantize_fp8(x)
    xf = x.float()
    amax = xf.abs().amax(dim=(2, 3))
    inv = torch.where(amax > 0, torch.tensor(448.0) / amax, torch.ones_like(amax))
    want_desc = torch.where(amax > 0, amax / torch.tensor(448.0), torch.ones_like(amax))
    y = xf * inv[:, :, None, None]
    want = y.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(desc, want_desc.numpy())
    # values at 448 (the amax element) may round from just above 448: both saturate to 0x7E
    assert np.array_equal(codes, want)
    assert np.all(codes[1, 2] == 0) and desc[1, 2] == 1.0
    # the largest magnitude of each head maps to +-448
    dec = oracle.e4m3_decode(codes)
    assert np.allclose(np.abs(dec[0]).max(axis=(1, 2)), 448.0)


def _fp8_inputs(B, H, Lq, Lk, d, seed):
    r = _rng(seed)
    q8 = r.integers(0, 256, (B, H, Lq, d), dtype=np.uint8)
    k8 = r.integers(0, 256, (B, H, Lk, d), dtype=np.uint8)
    v8 = r.integers(0, 256, (B, H, Lk, d), dtype=np.uint8)
    for a in (q8, k8, v8):
        a[(a & 0x7F) == 0x7F] = 0x30               # no NaN codes
    qd = (r.random((B, H)) * 0.02 + 0.001).astype(np.float32)
    kd = (r.random((B, H)) * 0.02 + 0.001).astype(np.float32)
    vd = (r.random((B, H)) * 0.02 + 0.001).astype(np.float32)
    return q8, k8, v8, qd, kd, vd


@pytest.mark.parametrize("slack", [0.0, 4.0, 8.0])
@pytest.mark.parametrize("Lq,Lk,causal,wl,wr,bk", [(40, 40, False, -1, -1, 16), (37, 53, True, -1, -1, 8),
                                                   (64, 64, False, 9, 4, 128), (50, 30, True, 5, 0, 7)])
def test_fp8_recurrence_without_rounding_is_exact_attention(oracle, Lq, Lk, causal, wl, wr, bk, slack):
    """With P unrounded, the tiled FP8 recurrence (reference max with any
    slack, rescale, the 2^(8 - slack) factor, descales) is exact attention on
    the dequantized inputs: numerator and denominator share the reference."""
    q8, k8, v8, qd, kd, vd = _fp8_inputs(2, 2, Lq, Lk, 16, 3)
    # scores spread widely enough that the reference moves at several tiles
    q8 = oracle.e4m3_encode(oracle.e4m3_decode(q8) * 4.0)
    o, lse = oracle.attn_fp8(q8, k8, v8, qd, kd, vd, 0.25, causal, wl, wr, block_k=bk, quantize_p=False,
                             slack=slack)
    deq = lambda c, s: oracle.e4m3_decode(c) * s.astype(np.float64)[:, :, None, None]
    o_ref, lse_ref = oracle.attn(deq(q8, qd), deq(k8, kd), deq(v8, vd), 0.25, causal, wl, wr)
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(lse), fin)
    assert np.abs(o - o_ref).max() < 1e-12 * max(1.0, np.abs(o_ref).max())
    assert np.abs(lse[fin] - lse_ref[fin]).max() < 1e-10


@pytest.mark.parametrize("slack", [0.0, 4.0])
def test_fp8_equal_scores_give_exact_mean(oracle, slack):
    """All keys equal: every allowed p is exactly 2^(8 - slack) (an e4m3
    value), so even with rounding O is the plain mean of the allowed
    dequantized V rows."""
    q8, _, v8, qd, kd, vd = _fp8_inputs(1, 2, 20, 20, 16, 4)
    k8 = np.broadcast_to(q8[:, :, :1], (1, 2, 20, 16)).copy()
    o, lse = oracle.attn_fp8(q8, k8, v8, qd, kd, vd, 0.3, True, block_k=8, quantize_p=True, slack=slack)
    vdq = oracle.e4m3_decode(v8) * vd.astype(np.float64)[:, :, None, None]
    for i in range(20):
        assert np.abs(o[:, :, i] - vdq[:, :, : i + 1].mean(axis=2)).max() < 1e-13


@pytest.mark.parametrize("slack", [0.0, 4.0])
def test_fp8_rounding_error_within_bound(oracle, slack):
    """Rounding p (<= 2^8) to e4m3 changes each weight by at most 2^-4 of itself
    (3 mantissa bits, normal range) or 2^-10 absolute (subnormal range), so
    |O - O_unrounded| <= vd * max|v8| * (2^-4 + n * 2^-10 / l) per row."""
    q8, k8, v8, qd, kd, vd = _fp8_inputs(1, 2, 64, 64, 32, 5)
    o_q, lse = oracle.attn_fp8(q8, k8, v8, qd, kd, vd, 0.5, False, quantize_p=True, slack=slack)
    o_u, _ = oracle.attn_fp8(q8, k8, v8, qd, kd, vd, 0.5, False, quantize_p=False, slack=slack)
    vmax = np.abs(oracle.e4m3_decode(v8)).max(axis=(2, 3)) * vd
    # l >= 2^(8 - slack) (the element that set the reference contributes at least that); n = 64 keys
    bound = vmax[:, :, None] * (2.0 ** -4 + 64 * 2.0 ** -10 / 2.0 ** (8 - slack))
    err = np.abs(o_q - o_u).max(axis=3)
    assert np.all(err <= bound)
    assert err.max() > 0.0    # the rounding is really applied
