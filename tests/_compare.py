"""Comparison helpers for GPU-vs-oracle parity (tolerances stated per call)."""
import numpy as np

# Bars: fp32 path O max-abs 1e-5; bf16 paths O max-abs 2e-2 and relative L2
# 5e-3 against the fp64 oracle; LSE within 1e-3 absolute everywhere.
F32_O_MAXABS = 1e-5
BF16_O_MAXABS = 2e-2
BF16_O_RELL2 = 5e-3
LSE_ABS = 1e-3


def compare(o_gpu, lse_gpu, o_ref, lse_ref, o_maxabs, o_rell2=None, lse_abs=LSE_ABS, label=""):
    """Element-wise comparison; rows with LSE = -inf in the oracle must be
    exactly O = 0 and LSE = -inf on the GPU.  Returns a dict of the errors."""
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    assert o_gpu.shape == o_ref.shape, (o_gpu.shape, o_ref.shape)
    assert np.isfinite(o_gpu).all(), f"{label}: non-finite output"
    err = np.abs(o_gpu - o_ref)
    out = {"o_maxabs": float(err.max()) if err.size else 0.0}
    assert out["o_maxabs"] <= o_maxabs, f"{label}: O max-abs {out['o_maxabs']:.3e} > {o_maxabs:.1e}"
    if o_rell2 is not None:
        den = float(np.linalg.norm(o_ref))
        rel = float(np.linalg.norm(o_gpu - o_ref)) / den if den > 0 else float(np.linalg.norm(o_gpu))
        out["o_rell2"] = rel
        assert rel <= o_rell2, f"{label}: O rel-L2 {rel:.3e} > {o_rell2:.1e}"
    if lse_gpu is not None:
        lse_gpu = np.asarray(lse_gpu, dtype=np.float64)
        lse_ref = np.asarray(lse_ref, dtype=np.float64)
        empty = np.isneginf(lse_ref)
        assert np.array_equal(np.isneginf(lse_gpu), empty), f"{label}: empty-row pattern differs"
        if empty.any():
            assert np.all(o_gpu.reshape(lse_ref.shape + (-1,))[empty] == 0.0), f"{label}: empty rows not zero"
        full = ~empty
        lerr = float(np.abs(lse_gpu[full] - lse_ref[full]).max()) if full.any() else 0.0
        out["lse_maxabs"] = lerr
        assert lerr <= lse_abs, f"{label}: LSE max-abs {lerr:.3e} > {lse_abs:.1e}"
    return out
