"""GPU parity of the FP8 path: the quantizer bit for bit, and attn_fwd_fp8
against the oracle's FP8 recurrence (same e4m3 inputs, P rounded the same
way) at the bf16 output bars, and against exact attention on the dequantized
inputs within the rounding bound of P.

Bound used against exact attention, per head: rounding p <= 2^8 to e4m3
moves each weight by at most 2^-4 of itself (normal range) or 2^-10
absolute (below it), and l >= 2^(8 - s) with s the reference slack of the
recurrence (reading R13), so |O - O_exact| <= vmax (2^-4 + n 2^(-18 + s))
with vmax the largest dequantized |v| and n the keys of the row; the bf16
output adds 2^-9 |O|.
"""
import numpy as np
import pytest
import torch

from io_aware_exact_34_b200 import synth
from tests._compare import BF16_O_MAXABS, BF16_O_RELL2, LSE_ABS, compare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fl():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from io_aware_exact_34_b200 import build
    build.build()
    from io_aware_exact_34_b200 import fattn
    return fattn


def _quantized(fl, q, k, v):
    qd_, kd_, vd_ = q.cuda(), k.cuda(), v.cuda()
    q8, qs = fl.attn_quantize_fp8(qd_)
    k8, ks = fl.attn_quantize_fp8(kd_)
    vt8, vs = fl.attn_quantize_fp8(vd_, transpose=True)
    return q8, k8, vt8, qs, ks, vs


@pytest.mark.parametrize("B,H,L,d", [(1, 2, 300, 128), (2, 1, 64, 64), (1, 1, 1, 128), (1, 3, 1000, 128)])
def test_quantize_bit_exact(fl, oracle, B, H, L, d):
    x = synth.random_qkv(B, H, L, L, d, "bf16", seed=L + d)[0]
    x[0, 0, 0, :8] = 0.0
    codes, desc = fl.attn_quantize_fp8(x.cuda())
    codes_t, desc_t = fl.attn_quantize_fp8(x.cuda(), transpose=True)
    torch.cuda.synchronize()
    ref_codes, ref_desc = oracle.quantize_fp8(x)
    assert np.array_equal(codes.cpu().numpy(), ref_codes)
    assert np.array_equal(desc.cpu().numpy(), ref_desc)
    ct = codes_t.cpu().numpy()
    ld = fl.attn_fp8_ld(L)
    assert ct.shape == (B, H, d, ld)
    assert np.array_equal(ct[..., :L], np.swapaxes(ref_codes, 2, 3))
    assert np.all(ct[..., L:] == 0)
    assert np.array_equal(desc_t.cpu().numpy(), ref_desc)


def test_quantize_zero_head(fl, oracle):
    x = torch.zeros((1, 2, 40, 128), dtype=torch.bfloat16)
    x[0, 1] = synth.random_qkv(1, 1, 40, 40, 128, "bf16", seed=9)[0][0, 0]
    codes, desc = fl.attn_quantize_fp8(x.cuda())
    torch.cuda.synchronize()
    ref_codes, ref_desc = oracle.quantize_fp8(x)
    assert np.array_equal(codes.cpu().numpy(), ref_codes) and desc[0, 0].item() == 1.0
    assert np.array_equal(desc.cpu().numpy(), ref_desc)


FP8_CASES = [
    # (B, H, Lq, Lk, causal, wl, wr)
    (1, 1, 128, 128, False, -1, -1),
    (1, 2, 256, 256, True, -1, -1),
    (2, 2, 300, 300, False, -1, -1),
    (1, 2, 200, 333, True, -1, -1),
    (1, 2, 333, 200, True, -1, -1),
    (1, 1, 640, 640, False, 130, 7),
    (1, 2, 1000, 1000, True, 257, 0),
    (1, 1, 1, 1, False, -1, -1),
    (1, 1, 7, 7, True, -1, -1),
    (1, 1, 1000, 1, True, -1, -1),
    (1, 1, 2048, 2048, True, -1, -1),
]


def _dequant(oracle, codes, desc):
    return oracle.e4m3_decode(codes) * desc.astype(np.float64)[:, :, None, None]


@pytest.mark.parametrize("B,H,Lq,Lk,causal,wl,wr", FP8_CASES)
def test_fp8_forward(fl, oracle, B, H, Lq, Lk, causal, wl, wr):
    d = 128
    q, k, v = synth.random_qkv(B, H, Lq, Lk, d, "bf16", seed=Lq * 13 + Lk)
    q8, k8, vt8, qs, ks, vs = _quantized(fl, q, k, v)
    counter = torch.zeros(1, dtype=torch.int64, device="cuda")
    scale = d ** -0.5
    o, lse = fl.attn_fwd_fp8(q8, k8, vt8, qs, ks, vs, scale=scale, causal=causal, window_left=wl,
                             window_right=wr, counter=counter)
    torch.cuda.synchronize()
    assert fl.fattn_device_status() == 0
    q8n, k8n = q8.cpu().numpy(), k8.cpu().numpy()
    v8n = np.ascontiguousarray(np.swapaxes(vt8.cpu().numpy()[..., :Lk], 2, 3))
    qsn, ksn, vsn = qs.cpu().numpy(), ks.cpu().numpy(), vs.cpu().numpy()
    o_gpu, lse_gpu = o.float().cpu().numpy(), lse.cpu().numpy()
    # the FP8 recurrence on the same codes: the bf16 bars
    o_ref, lse_ref = oracle.attn_fp8(q8n, k8n, v8n, qsn, ksn, vsn, scale, causal, wl, wr)
    compare(o_gpu, lse_gpu, o_ref, lse_ref, BF16_O_MAXABS, BF16_O_RELL2, LSE_ABS, label="fp8 vs fp8 oracle")
    # exact attention on the dequantized inputs: the rounding bound of P
    o_ex, lse_ex = oracle.attn(_dequant(oracle, q8n, qsn), _dequant(oracle, k8n, ksn), _dequant(oracle, v8n, vsn),
                               scale, causal, wl, wr)
    vmax = (np.abs(oracle.e4m3_decode(v8n)).max(axis=(2, 3)) * vsn)[:, :, None, None]
    # l >= 2^(8 - slack): the element that set the reference contributes at least that
    bound = vmax * (2.0 ** -4 + Lk * 2.0 ** (-18 + oracle.FP8_SLACK)) + 2.0 ** -9 * np.abs(o_ex) + 1e-6
    assert np.all(np.abs(o_gpu - o_ex) <= bound)
    fin = np.isfinite(lse_ex)
    assert np.array_equal(np.isfinite(lse_gpu), fin)
    c = fl.attn_count_blocks(Lq, Lk, causal, wl, wr)
    assert int(counter.item()) == B * H * c["visited"]


@pytest.mark.parametrize("causal,wl,wr", [(True, -1, -1), (False, 200, 200)])
def test_fp8_rescale_stress(fl, oracle, causal, wl, wr):
    """Scores spread over a wide range (Q scaled by 6 before quantizing): the
    reference max of the recurrence moves past its slack of 4 many times and
    O is rescaled in TMEM; against the oracle's FP8 recurrence on the same
    codes."""
    d, L = 128, 1024
    q, k, v = synth.random_qkv(1, 2, L, L, d, "bf16", seed=77 + max(wl, 0))
    q = (q.float() * 6.0).to(torch.bfloat16)
    q8, k8, vt8, qs, ks, vs = _quantized(fl, q, k, v)
    o, lse = fl.attn_fwd_fp8(q8, k8, vt8, qs, ks, vs, scale=d ** -0.5, causal=causal, window_left=wl,
                             window_right=wr)
    torch.cuda.synchronize()
    assert fl.fattn_device_status() == 0
    v8n = np.ascontiguousarray(np.swapaxes(vt8.cpu().numpy()[..., :L], 2, 3))
    o_ref, lse_ref = oracle.attn_fp8(q8.cpu().numpy(), k8.cpu().numpy(), v8n, qs.cpu().numpy(), ks.cpu().numpy(),
                                     vs.cpu().numpy(), d ** -0.5, causal, wl, wr)
    compare(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, BF16_O_MAXABS, BF16_O_RELL2, LSE_ABS,
            label=f"fp8 rescale stress {causal, wl, wr}")


def test_fp8_full_size_causal_4k_sampled_heads(fl, oracle):
    """The causal 4 x 16 x 4096 workload through the GPU quantizer and the FP8
    forward; two heads checked against the oracle's FP8 recurrence."""
    w = synth.WORKLOADS["causal_4k"]
    q, k, v = synth.make_inputs(w)
    q8, k8, vt8, qs, ks, vs = _quantized(fl, q, k, v)
    o, lse = fl.attn_fwd_fp8(q8, k8, vt8, qs, ks, vs, scale=w.scale, causal=True)
    torch.cuda.synchronize()
    for b, h in ((0, 0), (3, 15)):
        sl = (slice(b, b + 1), slice(h, h + 1))
        q8n, k8n = q8[sl].cpu().numpy(), k8[sl].cpu().numpy()
        v8n = np.ascontiguousarray(np.swapaxes(vt8[sl].cpu().numpy()[..., :w.Lk], 2, 3))
        o_ref, lse_ref = oracle.attn_fp8(q8n, k8n, v8n, qs[sl].cpu().numpy(), ks[sl].cpu().numpy(),
                                         vs[sl].cpu().numpy(), w.scale, True)
        compare(o[sl].float().cpu().numpy(), lse[sl].cpu().numpy(), o_ref, lse_ref, BF16_O_MAXABS, BF16_O_RELL2,
                LSE_ABS, label=f"fp8 causal_4k ({b},{h})")
        rq, _ = oracle.quantize_fp8(q[sl])
        assert np.array_equal(q8n, rq)
