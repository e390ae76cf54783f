"""GPU parity of the backward with recomputation (attn_bwd) against the
oracle's fp64 gradients on the same seeded bf16 inputs.

The GPU backward consumes the GPU forward's O and LSE, as a training step
would.  Tolerances (per gradient tensor, against the fp64 oracle): relative
L2 <= 1e-2 and max-abs <= 2e-2 times the tensor's largest magnitude.  Their
basis: P and dS are rounded to bf16 (unit roundoff 2^-9 = 1.95e-3) before each
enters a product once, D_i comes from the bf16-rounded O, and the outputs are
rounded to bf16 once; independent roundings add in quadrature along the sums,
so the relative error sits near a few units of 2^-9.  Gradients that vanish
structurally (keys no query attends) must be exactly zero; gradients that
vanish by cancellation are held to an fp32 residue bound (ZERO_RESIDUE).
"""
import numpy as np
import pytest
import torch

from io_aware_exact_34_b200 import synth

pytestmark = pytest.mark.gpu

GRAD_RELL2 = 1e-2
GRAD_MAXABS_REL = 2e-2
# Where the exact gradient is zero by cancellation, the residue of dP_ij - D_i
# (two fp32 dot products of length d over bf16 values of size ~1, summed in
# different orders: |error| <~ d * 2^-24 * sum |dO||v| ~ 1e-5) times scale * |k|.
ZERO_RESIDUE = 1e-5


@pytest.fixture(scope="module")
def fl():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from io_aware_exact_34_b200 import build
    build.build()
    from io_aware_exact_34_b200 import fattn
    return fattn


def _check_grad(got, ref, label):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (label, got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{label}: non-finite gradient"
    scale = float(np.abs(ref).max()) if ref.size else 0.0
    err = np.abs(got - ref)
    if scale == 0.0:
        # a gradient that is zero by cancellation (one key: P = 1, dP_i = D_i):
        # dP - D leaves the fp32 rounding residue of two dot products
        assert err.max() <= ZERO_RESIDUE, f"{label}: {err.max():.3e} where the gradient is 0"
        return {"maxabs": float(err.max()), "rell2": 0.0}
    rel = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
    mx = float(err.max())
    print(f"{label}: rel-L2 {rel:.2e}, max-abs {mx:.2e} (max |ref| {scale:.2e})")
    assert rel <= GRAD_RELL2, f"{label}: rel-L2 {rel:.3e} > {GRAD_RELL2:.0e}"
    assert mx <= GRAD_MAXABS_REL * scale, f"{label}: max-abs {mx:.3e} > {GRAD_MAXABS_REL:.0e} x {scale:.3e}"
    return {"maxabs": mx, "rell2": rel}


def _run(fl, q, k, v, do, scale, causal, wl, wr, counter=None):
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = fl.attn_fwd(qd, kd, vd, scale=scale, causal=causal, window_left=wl, window_right=wr)
    dq, dk, dv = fl.attn_bwd(qd, kd, vd, o, dod, lse, scale=scale, causal=causal, window_left=wl, window_right=wr,
                             counter=counter)
    torch.cuda.synchronize()
    assert fl.fattn_device_status() == 0
    return dq.float().cpu().numpy(), dk.float().cpu().numpy(), dv.float().cpu().numpy()


BWD_CASES = [
    # (B, H, Lq, Lk, d, causal, wl, wr)
    (1, 1, 128, 128, 128, False, -1, -1),
    (1, 2, 256, 256, 128, True, -1, -1),
    (2, 2, 384, 384, 128, False, -1, -1),
    (1, 1, 300, 300, 128, True, -1, -1),        # ragged last tile
    (1, 2, 300, 260, 128, True, -1, -1),        # Lq > Lk: leading rows without keys
    (1, 2, 200, 333, 128, True, -1, -1),        # Lq < Lk (bottom-right)
    (1, 1, 640, 640, 128, False, 130, 7),       # asymmetric window
    (1, 2, 1000, 1000, 128, True, 257, 0),      # causal left window
    (1, 1, 100, 1000, 128, True, 50, 0),        # keys no query sees: dK = dV = 0
    (1, 1, 2048, 2048, 128, True, -1, -1),      # 16 query tiles: both stages reused
    (1, 1, 513, 513, 64, False, 64, 64),        # d = 64
    (1, 2, 256, 256, 64, True, -1, -1),
    (1, 1, 1, 1, 128, False, -1, -1),           # one query, one key
    (2, 1, 7, 7, 64, True, -1, -1),
    (1, 1, 1000, 1, 128, True, -1, -1),         # a single key
    (1, 4, 5000, 5000, 128, True, -1, -1),      # heads scheduled in groups of 3: a partial last group
]


@pytest.mark.parametrize("B,H,Lq,Lk,d,causal,wl,wr", BWD_CASES)
def test_bwd_grid(fl, oracle, B, H, Lq, Lk, d, causal, wl, wr):
    seed = Lq * 31 + Lk * 7 + d
    q, k, v = synth.random_qkv(B, H, Lq, Lk, d, "bf16", seed=seed)
    do = synth.random_dout(B, H, Lq, d, "bf16", seed=seed)
    scale = d ** -0.5
    counter = torch.zeros(1, dtype=torch.int64, device="cuda")
    dq, dk, dv = _run(fl, q, k, v, do, scale, causal, wl, wr, counter=counter)
    rq, rk, rv = oracle.attn_bwd(q, k, v, do, scale, causal, wl, wr)
    label = f"{B}x{H}x{Lq}x{Lk} d{d} c{int(causal)} w({wl},{wr})"
    _check_grad(dq, rq, label + " dQ")
    _check_grad(dk, rk, label + " dK")
    _check_grad(dv, rv, label + " dV")
    assert int(counter.item()) == B * H * fl.attn_bwd_count_blocks(Lq, Lk, causal, wl, wr)


def test_bwd_unseen_keys_are_exact_zero(fl):
    """Keys outside every query's window get exactly zero dK and dV."""
    q, k, v = synth.random_qkv(1, 2, 100, 1000, 128, "bf16", seed=11)
    do = synth.random_dout(1, 2, 100, 128, "bf16", seed=11)
    _, dk, dv = _run(fl, q, k, v, do, 128 ** -0.5, True, 50, 0)
    # queries sit at key positions 900..999, so keys below 850 are never attended
    assert np.all(dk[:, :, :850] == 0.0) and np.all(dv[:, :, :850] == 0.0)
    assert np.abs(dv[:, :, 850:]).max() > 0.0


def test_bwd_full_size_causal_4k_sampled_heads(fl, oracle):
    """The causal 4 x 16 x 4096, d = 128 prefill workload: the whole backward
    runs on the GPU, two heads are compared in full with the oracle."""
    w = synth.WORKLOADS["causal_4k"]
    q, k, v = synth.make_inputs(w)
    do = synth.random_dout(w.B, w.H, w.Lq, w.d, "bf16", seed=w.seed)
    dq, dk, dv = _run(fl, q, k, v, do, w.scale, w.causal, w.window_left, w.window_right)
    for b, h in ((0, 0), (3, 15)):
        sl = (slice(b, b + 1), slice(h, h + 1))
        rq, rk, rv = oracle.attn_bwd(q[sl], k[sl], v[sl], do[sl], w.scale, w.causal, w.window_left, w.window_right)
        _check_grad(dq[sl], rq, f"causal_4k ({b},{h}) dQ")
        _check_grad(dk[sl], rk, f"causal_4k ({b},{h}) dK")
        _check_grad(dv[sl], rv, f"causal_4k ({b},{h}) dV")


def test_bwd_repeatable_dk_dv(fl):
    """dK and dV have a fixed summation order (tensor-memory accumulation over
    the query tiles in order): two runs agree bit for bit."""
    q, k, v = synth.random_qkv(1, 2, 700, 700, 128, "bf16", seed=5)
    do = synth.random_dout(1, 2, 700, 128, "bf16", seed=5)
    a = _run(fl, q, k, v, do, 128 ** -0.5, True, -1, -1)
    b = _run(fl, q, k, v, do, 128 ** -0.5, True, -1, -1)
    assert np.array_equal(a[1], b[1]) and np.array_equal(a[2], b[2])
