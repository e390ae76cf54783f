"""GPU parity: the CUDA path through the C ABI against the fp64 CPU oracle on
the same seeded inputs.

Small shapes span several 128-row tiles and ragged tails and are compared
element by element; the full-size workloads are compared in full where the
oracle finishes in seconds (tiny fp32, causal 4 x 16 x 4096) and on
stratified row samples otherwise.
"""
import numpy as np
import pytest
import torch

from io_aware_exact_34_b200 import synth
from tests._compare import (BF16_O_MAXABS, BF16_O_RELL2, F32_O_MAXABS, LSE_ABS, compare)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fl():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from io_aware_exact_34_b200 import build
    build.build()
    from io_aware_exact_34_b200 import fattn
    return fattn


def _run_bf16(fl, q, k, v, scale, causal, wl, wr):
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o, lse = fl.attn_fwd(qd, kd, vd, scale=scale, causal=causal, window_left=wl, window_right=wr)
    torch.cuda.synchronize()
    return o.float().cpu().numpy(), lse.cpu().numpy()


# ------------------------------------------------------------------ fp32 path

def test_tiny_f32_config(fl, oracle):
    w = synth.WORKLOADS["tiny_f32"]
    q, k, v = synth.make_inputs(w)
    o, lse = fl.attn_fwd_f32(q.cuda(), k.cuda(), v.cuda(), scale=w.scale)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attn(q, k, v, w.scale)
    e = compare(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, F32_O_MAXABS, lse_abs=LSE_ABS, label="tiny_f32")
    assert e["lse_maxabs"] < 1e-5


F32_CASES = [
    (1, 2, 256, 256, 64, False, -1, -1),
    (2, 1, 100, 100, 128, True, -1, -1),
    (1, 2, 300, 300, 64, False, 37, 37),
    (1, 1, 129, 200, 128, True, -1, -1),
    (1, 1, 200, 129, 64, True, -1, -1),
    (1, 3, 65, 65, 128, False, 0, 0),
    (2, 2, 1, 77, 64, False, -1, -1),
]


@pytest.mark.parametrize("B,H,Lq,Lk,d,causal,wl,wr", F32_CASES)
def test_f32_grid(fl, oracle, B, H, Lq, Lk, d, causal, wl, wr):
    q, k, v = synth.random_qkv(B, H, Lq, Lk, d, "f32", seed=Lq * 7 + Lk)
    scale = d ** -0.5
    o, lse = fl.attn_fwd_f32(q.cuda(), k.cuda(), v.cuda(), scale=scale, causal=causal, window_left=wl,
                             window_right=wr)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attn(q, k, v, scale, causal, wl, wr)
    compare(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, F32_O_MAXABS, label="f32")


# ------------------------------------------------------------------ bf16 tensor-core path

BF16_CASES = [
    # (B, H, Lq, Lk, d, causal, wl, wr)
    (1, 1, 128, 128, 128, False, -1, -1),
    (1, 1, 256, 256, 128, False, -1, -1),
    (1, 2, 256, 256, 128, True, -1, -1),
    (2, 2, 512, 512, 128, True, -1, -1),
    (1, 1, 1, 1, 128, False, -1, -1),
    (1, 1, 7, 7, 128, True, -1, -1),
    (1, 1, 64, 64, 64, False, -1, -1),
    (1, 1, 127, 127, 128, True, -1, -1),
    (1, 1, 129, 129, 128, True, -1, -1),
    (1, 2, 255, 255, 64, False, -1, -1),
    (1, 1, 300, 300, 128, True, -1, -1),
    (1, 1, 300, 300, 64, True, -1, -1),
    (2, 3, 383, 383, 128, False, 63, 63),
    (1, 2, 700, 700, 128, False, 64, 64),
    (1, 2, 700, 700, 128, False, 65, 1),
    (1, 1, 700, 700, 128, True, 300, 0),
    (1, 1, 700, 700, 64, True, 1, 0),
    (1, 1, 600, 600, 128, False, 0, 0),
    (1, 1, 129, 300, 128, True, -1, -1),
    (1, 1, 300, 129, 128, True, -1, -1),
    (1, 1, 300, 129, 128, False, 7, 3),
    (1, 1, 1, 700, 128, False, -1, -1),
    (1, 1, 1000, 1000, 128, False, 300, 300),
    (3, 5, 1100, 1100, 64, True, 257, 0),
    (1, 1, 2048, 2048, 128, True, -1, -1),
]


@pytest.mark.parametrize("B,H,Lq,Lk,d,causal,wl,wr", BF16_CASES)
def test_bf16_grid(fl, oracle, B, H, Lq, Lk, d, causal, wl, wr):
    q, k, v = synth.random_qkv(B, H, Lq, Lk, d, "bf16", seed=Lq * 13 + Lk + d)
    scale = d ** -0.5
    o, lse = _run_bf16(fl, q, k, v, scale, causal, wl, wr)
    o_ref, lse_ref = oracle.attn(q, k, v, scale, causal, wl, wr)
    compare(o, lse, o_ref, lse_ref, BF16_O_MAXABS, BF16_O_RELL2, label=f"bf16 {B,H,Lq,Lk,d,causal,wl,wr}")


@pytest.mark.parametrize("d,causal,wl,wr", [(128, True, -1, -1), (64, True, -1, -1), (64, False, 300, 300),
                                             (64, True, 700, 0)])
def test_bf16_large_scores_stress_rescale(fl, oracle, d, causal, wl, wr):
    """Scores spread over a wide range (Q scaled by 6): the running-max
    reference moves many times and the accumulator rescale path runs (at
    d = 64 after the wait for the previous P.V product, P having columns of
    its own)."""
    q, k, v = synth.random_qkv(1, 4, 1024, 1024, d, "bf16", seed=99 + d + max(wl, 0))
    q = (q.float() * 6.0).to(torch.bfloat16)
    o, lse = _run_bf16(fl, q, k, v, d ** -0.5, causal, wl, wr)
    o_ref, lse_ref = oracle.attn(q, k, v, d ** -0.5, causal, wl, wr)
    compare(o, lse, o_ref, lse_ref, BF16_O_MAXABS, BF16_O_RELL2, label=f"rescale stress d={d} {causal,wl,wr}")


@pytest.mark.parametrize("d", [64, 128])
def test_many_short_items(fl, oracle, d):
    """Many work items per CTA (8 x 16 heads of 600 tokens, causal): every
    item boundary hands S, P and O of both tiles over to the next item."""
    q, k, v = synth.random_qkv(8, 16, 600, 600, d, "bf16", seed=400 + d)
    o, lse = _run_bf16(fl, q, k, v, d ** -0.5, True, -1, -1)
    o_ref, lse_ref = oracle.attn(q, k, v, d ** -0.5, True)
    compare(o, lse, o_ref, lse_ref, BF16_O_MAXABS, BF16_O_RELL2, label=f"short items d={d}")


def test_constant_v_rows(fl):
    """Every V row equal to c gives O = c (up to bf16 rounding of O)."""
    q, k, _ = synth.random_qkv(1, 2, 700, 700, 128, "bf16", seed=5)
    c = torch.randn(128).to(torch.bfloat16)
    v = c.view(1, 1, 1, 128).expand(1, 2, 700, 128).contiguous()
    for causal, wl, wr in [(False, -1, -1), (True, -1, -1), (False, 100, 100)]:
        o, _ = _run_bf16(fl, q, k, v, 128 ** -0.5, causal, wl, wr)
        assert np.abs(o - c.float().numpy()).max() <= 2 ** -8 * np.abs(c.float().numpy()).max() + 1e-6


def test_visited_tiles_counter(fl):
    """The kernel loads exactly the KV tiles of the closed-form range: its
    device counter equals the host count for every head."""
    cases = [(2, 3, 1000, 1000, True, -1, -1), (1, 2, 2000, 2000, False, 200, 200),
             (1, 1, 4096, 4096, True, 1000, 0), (1, 1, 300, 129, True, -1, -1)]
    for B, H, Lq, Lk, causal, wl, wr in cases:
        q, k, v = synth.random_qkv(B, H, Lq, Lk, 128, "bf16", seed=1)
        counter = torch.zeros(1, dtype=torch.int64, device="cuda")
        fl.attn_fwd_counted(q.cuda(), k.cuda(), v.cuda(), counter, causal=causal, window_left=wl, window_right=wr)
        torch.cuda.synchronize()
        want = fl.attn_count_blocks(Lq, Lk, causal, wl, wr, 128, 128)["visited"] * B * H
        assert int(counter.item()) == want


def test_outputs_stay_in_bounds(fl):
    """Guard regions filled with a NaN pattern around O and LSE stay intact
    (stands in for a memory checker) and rows of a ragged tail are written."""
    B, H, Lq, Lk, d = 1, 3, 333, 333, 128
    q, k, v = synth.random_qkv(B, H, Lq, Lk, d, "bf16", seed=3)
    n_o, n_l, g = B * H * Lq * d, B * H * Lq, 4096
    o_buf = torch.full((n_o + 2 * g,), float("nan"), dtype=torch.bfloat16, device="cuda")
    l_buf = torch.full((n_l + 2 * g,), float("nan"), dtype=torch.float32, device="cuda")
    o = o_buf[g:g + n_o].view(B, H, Lq, d)
    lse = l_buf[g:g + n_l].view(B, H, Lq)
    fl.attn_fwd(q.cuda(), k.cuda(), v.cuda(), o=o, lse=lse, causal=True)
    torch.cuda.synchronize()
    assert torch.isnan(o_buf[:g].float()).all() and torch.isnan(o_buf[g + n_o:].float()).all()
    assert torch.isnan(l_buf[:g]).all() and torch.isnan(l_buf[g + n_l:]).all()
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()


def test_no_device_status_error(fl):
    q, k, v = synth.random_qkv(1, 1, 256, 256, 128, "bf16", seed=4)
    fl.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True)
    assert fl.fattn_device_status() == 0


# ------------------------------------------------------------------ full-size workloads

@pytest.mark.parametrize("name", ["causal_4k", "causal_4k_d64"])
def test_causal_4k_full(fl, oracle, name):
    """Causal prefill 4 x 16 x 4096 at d = 128 and d = 64: every row against
    the oracle."""
    w = synth.WORKLOADS[name]
    q, k, v = synth.make_inputs(w)
    o, lse = _run_bf16(fl, q, k, v, w.scale, w.causal, w.window_left, w.window_right)
    o_ref, lse_ref = oracle.attn(q, k, v, w.scale, w.causal, w.window_left, w.window_right)
    compare(o, lse, o_ref, lse_ref, BF16_O_MAXABS, BF16_O_RELL2, label=name)


@pytest.mark.parametrize("name", ["window_bidir_32k", "window_causal_32k", "causal_64k_qscale",
                                  "window_bidir_32k_d64"])
def test_long_workloads_sampled(fl, oracle, name):
    """Sliding-window and long causal workloads at full size: the GPU runs
    the whole problem; the oracle checks one full head plus stratified rows of
    every other head (first / last rows, tile and window edges, random).  For
    the long causal workload with per-head query factors the full head is the
    one with the largest factor, whose scores spread widest (the factor is
    read back as the RMS of the head's Q, 8.4M draws)."""
    w = synth.WORKLOADS[name]
    q, k, v = synth.make_inputs(w)
    o, lse = _run_bf16(fl, q, k, v, w.scale, w.causal, w.window_left, w.window_right)
    head = w.H - 1
    if w.q_head_scale is not None:
        head = int(q.float().pow(2).mean(dim=(0, 2, 3)).argmax())
    rows = synth.sample_rows(w, n_random=24, seed=7, full_heads=[(0, head)])
    ro, rl = oracle.attn_rows(q, k, v, rows, w.scale, w.causal, w.window_left, w.window_right)
    r = rows.numpy()
    compare(o[r[:, 0], r[:, 1], r[:, 2]], lse[r[:, 0], r[:, 1], r[:, 2]], ro, rl,
            BF16_O_MAXABS, BF16_O_RELL2, label=name)


def test_window_bidir_visits_page_block_count(fl):
    """n = 32768, |i - j| <= 2048: 8176 of 65536 128x128 tiles per head."""
    w = synth.WORKLOADS["window_bidir_32k"]
    q, k, v = synth.make_inputs(w)
    counter = torch.zeros(1, dtype=torch.int64, device="cuda")
    fl.attn_fwd_counted(q.cuda(), k.cuda(), v.cuda(), counter, causal=w.causal,
                        window_left=w.window_left, window_right=w.window_right)
    torch.cuda.synchronize()
    assert int(counter.item()) == 8176 * w.B * w.H


# ------------------------------------------------------------------ decode

DEC_CASES = [
    # (B, H, Lk, d, S, with_seqlens)
    (2, 3, 1000, 128, 4, False),
    (3, 2, 4096, 128, 32, True),
    (2, 2, 777, 64, 5, True),
    (1, 4, 129, 128, 1, False),
    (2, 2, 64, 128, 64, False),
    (4, 1, 20000, 128, 0, True),
]


@pytest.mark.parametrize("B,H,Lk,d,S,with_seqlens", DEC_CASES)
def test_decode_grid(fl, oracle, B, H, Lk, d, S, with_seqlens):
    q, _, _ = synth.random_qkv(B, H, 1, 1, d, "bf16", seed=Lk)
    _, k, v = synth.random_qkv(B, H, 1, Lk, d, "bf16", seed=Lk + 1)
    seqlens = None
    if with_seqlens:
        g = torch.Generator().manual_seed(Lk)
        seqlens = torch.randint(0, Lk + 1, (B,), generator=g, dtype=torch.int32)
        seqlens[0] = Lk
        if B > 2:
            seqlens[-1] = 0
    o, lse = fl.attn_decode_splitkv(q.cuda(), k.cuda(), v.cuda(), scale=d ** -0.5, num_splits=S,
                                    seqlens_k=None if seqlens is None else seqlens.cuda())
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attn(q, k, v, d ** -0.5, seqlens_k=None if seqlens is None else seqlens.numpy())
    compare(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref[..., 0], BF16_O_MAXABS, BF16_O_RELL2,
            label="decode")


def test_decode_full_size_sampled(fl, oracle):
    """Decode 64 x 32 heads x 32768 keys, 32 splits: the GPU runs the whole
    batch; the oracle checks 48 (b, h) heads in full."""
    w = synth.WORKLOADS["decode_32k"]
    q, k, v = synth.make_inputs(w, device="cuda")
    o, lse = fl.attn_decode_splitkv(q, k, v, scale=w.scale, num_splits=w.num_splits)
    torch.cuda.synchronize()
    g = torch.Generator().manual_seed(11)
    heads = [(0, 0), (w.B - 1, w.H - 1)] + [tuple(x) for x in
                                           torch.stack([torch.randint(0, w.B, (46,), generator=g),
                                                        torch.randint(0, w.H, (46,), generator=g)], 1).tolist()]
    for b, h in heads:
        qs, ks, vs = (t[b:b + 1, h:h + 1].cpu() for t in (q, k, v))
        o_ref, lse_ref = oracle.attn(qs, ks, vs, w.scale)
        compare(o[b:b + 1, h:h + 1].float().cpu().numpy(), lse[b:b + 1, h:h + 1].cpu().numpy(),
                o_ref, lse_ref[..., 0], BF16_O_MAXABS, BF16_O_RELL2, label=f"decode_32k {b},{h}")


def test_output_base_16_not_32_byte_aligned(fl):
    # the epilogue writes 32-byte pieces of each O row when O's base allows it
    # and 16-byte pieces otherwise; both give the same bits
    from io_aware_exact_34_b200 import synth
    B, H, L, d = 1, 3, 300, 128
    q, k, v = (t.cuda() for t in synth.random_qkv(B, H, L, L, d, "bf16", seed=21))
    o_a, lse_a = fl.attn_fwd(q, k, v, causal=True)
    buf = torch.empty(B * H * L * d + 16, dtype=torch.bfloat16, device="cuda")
    base = buf.data_ptr() % 32
    off = ((16 - base) % 32) // 2  # elements to a 16-byte but not 32-byte boundary
    o_u = buf[off:off + B * H * L * d].view(B, H, L, d)
    assert o_u.data_ptr() % 32 == 16
    fl.attn_fwd(q, k, v, o=o_u, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o_a, o_u)
