"""Pins of the fp64 CPU oracle against what the pages and mathematics fix.

Each check is chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign or index, a transposed operand, an off-by-one window edge, a wrong
merge weight) fails at least one of them.  None of them compares the oracle
with itself, and none touches the CUDA library.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import naive_np

HERE = os.path.dirname(os.path.abspath(__file__))


def _rand(shape, seed, dtype=np.float64):
    rng = np.random.default_rng(seed)
    return rng.standard_normal(shape).astype(dtype)


def _sdpa_fp64(q, k, v, scale, mask):
    """torch's own scaled_dot_product_attention in float64 (a library routine)."""
    qt, kt, vt = (torch.from_numpy(np.ascontiguousarray(x)) for x in (q, k, v))
    mt = torch.from_numpy(mask)
    out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mt, scale=scale)
    return out.numpy()


MASK_CASES = [
    # (Lq, Lk, causal, wl, wr)
    (13, 13, False, -1, -1),
    (13, 13, True, -1, -1),
    (20, 20, False, 3, 3),
    (20, 20, True, 4, 0),
    (20, 20, False, 0, 5),
    (9, 17, True, -1, -1),      # Lq < Lk: bottom-right alignment
    (17, 17, False, 2, -1),
    (16, 16, False, -1, 2),
]


@pytest.mark.parametrize("Lq,Lk,causal,wl,wr", MASK_CASES)
def test_naive_matches_torch_sdpa_fp64(oracle, Lq, Lk, causal, wl, wr):
    """Pin: the oracle's softmax/contraction equals torch's fp64 SDPA given the
    band mask of the page (§4, §4.1, §7.1), built here as an explicit boolean matrix."""
    B, H, d = 2, 3, 8
    q = _rand((B, H, Lq, d), 1)
    k = _rand((B, H, Lk, d), 2)
    v = _rand((B, H, Lk, d), 3)
    scale = 0.37
    o, lse = oracle.attn(q, k, v, scale, causal, wl, wr)
    shift = Lk - Lq
    mask = np.zeros((Lq, Lk), dtype=bool)
    for i in range(Lq):
        for j in range(Lk):
            pos = i + shift
            ok = True
            if causal and j > pos:
                ok = False
            if wr >= 0 and j > pos + wr:
                ok = False
            if wl >= 0 and j < pos - wl:
                ok = False
            mask[i, j] = ok
    assert mask.any(axis=1).all(), "case chosen so every row has a key"
    ref = _sdpa_fp64(q, k, v, scale, mask)
    assert np.abs(o - ref).max() < 1e-13
    # LSE against scipy's logsumexp of the masked scores
    from scipy.special import logsumexp
    s = scale * np.einsum("bhid,bhjd->bhij", q, k)
    s = np.where(mask, s, -np.inf)
    assert np.abs(lse - logsumexp(s, axis=-1)).max() < 1e-12


def test_numpy_restatement_agrees(oracle):
    """Third restatement (whole-matrix NumPy) on a masked, ragged case."""
    q = _rand((1, 1, 37, 5), 4)
    k = _rand((1, 1, 41, 5), 5)
    v = _rand((1, 1, 41, 5), 6)
    for causal, wl, wr in [(False, -1, -1), (True, -1, -1), (True, 6, 0), (False, 4, 9)]:
        o, lse = oracle.attn(q, k, v, 0.5, causal, wl, wr)
        o2, lse2 = naive_np.attn_head(q[0, 0], k[0, 0], v[0, 0], 0.5, causal, wl, wr)
        assert np.abs(o[0, 0] - o2).max() < 1e-13
        assert np.abs(lse[0, 0] - lse2).max() < 1e-12


def test_bruteforce_tiny_enumeration(oracle):
    """P5: explicit enumeration with Python floats on tiny inputs (n <= 16, d <= 4)."""
    rng = np.random.default_rng(7)
    for (n, d, causal, wl, wr) in [(5, 3, False, -1, -1), (7, 2, True, -1, -1),
                                    (9, 4, False, 1, 2), (16, 4, True, 3, 0)]:
        q = rng.standard_normal((1, 1, n, d))
        k = rng.standard_normal((1, 1, n, d))
        v = rng.standard_normal((1, 1, n, d))
        scale = 1.0 / math.sqrt(d)
        o, lse = oracle.attn(q, k, v, scale, causal, wl, wr)
        for i in range(n):
            keys = [j for j in range(n)
                    if (not causal or j <= i) and (wr < 0 or j <= i + wr) and (wl < 0 or j >= i - wl)]
            scores = {j: scale * sum(q[0, 0, i, c] * k[0, 0, j, c] for c in range(d)) for j in keys}
            top = max(scores.values())
            weights = {j: math.exp(s - top) for j, s in scores.items()}
            z = sum(weights.values())
            for c in range(d):
                want = sum(weights[j] * v[0, 0, j, c] for j in keys) / z
                assert abs(o[0, 0, i, c] - want) < 1e-13
            assert abs(lse[0, 0, i] - (top + math.log(z))) < 1e-13


def test_diagonal_only_window_gives_v_and_score(oracle):
    """P5 closed form: wl = wr = 0 leaves only key i, so O_i = v_i and
    LSE_i = scale * q_i . k_i.  An exclusive window edge would leave rows empty."""
    q, k, v = _rand((1, 2, 11, 6), 8), _rand((1, 2, 11, 6), 9), _rand((1, 2, 11, 6), 10)
    o, lse = oracle.attn(q, k, v, 0.3, False, 0, 0)
    assert np.abs(o - v).max() < 1e-15
    assert np.abs(lse - 0.3 * (q * k).sum(-1)).max() < 1e-14


def test_two_key_window_closed_form(oracle):
    """wl = 1, wr = 0: row i > 0 attends keys {i-1, i}; softmax of two scores in
    closed form sigma(s_i - s_{i-1})."""
    q, k, v = _rand((1, 1, 9, 3), 11), _rand((1, 1, 9, 3), 12), _rand((1, 1, 9, 3), 13)
    o, _ = oracle.attn(q, k, v, 1.0, False, 1, 0)
    for i in range(1, 9):
        a = float(q[0, 0, i] @ k[0, 0, i - 1])
        b = float(q[0, 0, i] @ k[0, 0, i])
        w_b = 1.0 / (1.0 + math.exp(a - b))
        want = (1.0 - w_b) * v[0, 0, i - 1] + w_b * v[0, 0, i]
        assert np.abs(o[0, 0, i] - want).max() < 1e-14
    assert np.abs(o[0, 0, 0] - v[0, 0, 0]).max() < 1e-15


def test_single_key_row(oracle):
    """P9: Lk = 1 gives O = v_0 and LSE = scale * q . k_0 for every row."""
    q, k, v = _rand((2, 2, 5, 4), 14), _rand((2, 2, 1, 4), 15), _rand((2, 2, 1, 4), 16)
    o, lse = oracle.attn(q, k, v, 0.7)
    assert np.abs(o - v).max() < 1e-15
    assert np.abs(lse - 0.7 * np.einsum("bhid,bhd->bhi", q, k[:, :, 0])).max() < 1e-14


@pytest.mark.parametrize("causal,wl,wr", [(False, -1, -1), (True, -1, -1), (False, 3, 5), (True, 7, 0)])
def test_probability_rows_sum_to_one(oracle, causal, wl, wr):
    """P2: each softmax row sums to 1, and P @ V (numpy's matmul) is the oracle's O."""
    q, k, v = _rand((1, 1, 23, 6), 17), _rand((1, 1, 23, 6), 18), _rand((1, 1, 23, 6), 19)
    P = oracle.probs(q[0, 0], k[0, 0], 0.4, causal, wl, wr)
    assert np.abs(P.sum(axis=1) - 1.0).max() < 1e-14
    assert (P >= 0).all()
    o, _ = oracle.attn(q, k, v, 0.4, causal, wl, wr)
    assert np.abs(P @ v[0, 0] - o[0, 0]).max() < 1e-14


@pytest.mark.parametrize("causal,wl,wr", [(False, -1, -1), (True, -1, -1), (False, 2, 2), (True, 5, 0)])
def test_constant_v_gives_constant(oracle, causal, wl, wr):
    """P3: V rows all equal to c gives O = c for every mask (alpha / l bookkeeping)."""
    q, k = _rand((1, 2, 70, 8), 20), _rand((1, 2, 70, 8), 21)
    c = _rand((8,), 22)
    v = np.broadcast_to(c, (1, 2, 70, 8)).copy()
    for fn in ("naive", "tiled"):
        if fn == "naive":
            o, _ = oracle.attn(q, k, v, 0.5, causal, wl, wr)
        else:
            o, _, _ = oracle.attn_tiled(q, k, v, 0.5, causal, wl, wr, block_q=16, block_k=16)
        assert np.abs(o - c).max() < 1e-14


def test_wide_window_equals_plain_masks(oracle):
    """P4: a window >= n is no window (causal stays causal, full stays full)."""
    q, k, v = _rand((1, 1, 30, 4), 23), _rand((1, 1, 30, 4), 24), _rand((1, 1, 30, 4), 25)
    oc, lc = oracle.attn(q, k, v, 0.5, True)
    ow, lw = oracle.attn(q, k, v, 0.5, True, 30, 0)
    assert np.array_equal(oc, ow) and np.array_equal(lc, lw)
    of, lf = oracle.attn(q, k, v, 0.5, False)
    ob, lb = oracle.attn(q, k, v, 0.5, False, 40, 40)
    assert np.array_equal(of, ob) and np.array_equal(lf, lb)


TILED_CASES = [
    # (Lq, Lk, causal, wl, wr, block_q, block_k)
    (256, 256, False, -1, -1, 64, 64),      # the tiny exact-check shape, block 64
    (256, 256, True, -1, -1, 64, 64),
    (200, 200, False, 37, 37, 64, 64),
    (200, 200, True, 50, 0, 32, 48),        # block sizes that differ and do not divide n
    (130, 170, True, -1, -1, 64, 32),       # Lq != Lk
    (96, 96, False, 0, 0, 16, 16),
]


@pytest.mark.parametrize("Lq,Lk,causal,wl,wr,bq,bk", TILED_CASES)
def test_tiled_recurrence_equals_naive(oracle, Lq, Lk, causal, wl, wr, bq, bk):
    """P1: the page's tiled online softmax (§3.2, §5.3) reaches the exact result."""
    q, k, v = _rand((1, 2, Lq, 16), 26), _rand((1, 2, Lk, 16), 27), _rand((1, 2, Lk, 16), 28)
    o, lse = oracle.attn(q, k, v, 0.25, causal, wl, wr)
    ot, lt, _ = oracle.attn_tiled(q, k, v, 0.25, causal, wl, wr, block_q=bq, block_k=bk)
    assert np.abs(o - ot).max() < 1e-12
    assert np.abs(lse - lt).max() < 1e-12


def test_tiled_with_block_equal_n_is_standard_softmax(oracle):
    """§3.2: with block_size equal to the sequence length the recurrence is
    plain softmax attention; compared against torch's fp64 softmax."""
    q, k, v = _rand((1, 1, 64, 8), 29), _rand((1, 1, 64, 8), 30), _rand((1, 1, 64, 8), 31)
    ot, lt, visited = oracle.attn_tiled(q, k, v, 0.35, block_q=64, block_k=64)
    assert visited == 1
    s = torch.from_numpy(0.35 * q[0, 0] @ k[0, 0].T)
    ref = torch.softmax(s, dim=-1).numpy() @ v[0, 0]
    assert np.abs(ot[0, 0] - ref).max() < 1e-14
    assert np.abs(lt[0, 0] - torch.logsumexp(s, -1).numpy()).max() < 1e-13


@pytest.mark.parametrize("Lq,Lk,causal,wl,wr,bq,bk", TILED_CASES)
def test_skipped_blocks_are_exact(oracle, Lq, Lk, causal, wl, wr, bq, bk):
    """P6 (§5.5): skipping out-of-band blocks gives the result of visiting and
    masking them, and visits exactly the tiles that hold an allowed pair."""
    q, k, v = _rand((1, 1, Lq, 8), 32), _rand((1, 1, Lk, 8), 33), _rand((1, 1, Lk, 8), 34)
    o1, l1, n_skip = oracle.attn_tiled(q, k, v, 0.5, causal, wl, wr, bq, bk, skip=True)
    o2, l2, n_all = oracle.attn_tiled(q, k, v, 0.5, causal, wl, wr, bq, bk, skip=False)
    assert np.abs(o1 - o2).max() < 1e-15
    assert np.abs(l1 - l2).max() < 1e-15
    counts = oracle.count_blocks(Lq, Lk, causal, wl, wr, bq, bk)
    assert n_all == counts["total"]
    assert n_skip == counts["visited"]


def test_nan_guard_reading_r7(oracle):
    """Reading R7: with the page's literal update order a row whose first
    visited block is fully masked for it gives NaN; the m_safe guard removes it
    and agrees with the definition (n = 256, d = 16, w = 100, block 64)."""
    q, k, v = _rand((1, 1, 256, 16), 35), _rand((1, 1, 256, 16), 36), _rand((1, 1, 256, 16), 37)
    o_lit, _, _ = oracle.attn_tiled(q, k, v, 0.25, False, 100, 100, 64, 64, nan_guard=False)
    assert np.isnan(o_lit).any(axis=-1).sum() > 0
    o_g, l_g, _ = oracle.attn_tiled(q, k, v, 0.25, False, 100, 100, 64, 64, nan_guard=True)
    o, l = oracle.attn(q, k, v, 0.25, False, 100, 100)
    assert not np.isnan(o_g).any()
    assert np.abs(o_g - o).max() < 1e-12 and np.abs(l_g - l).max() < 1e-12


def test_rows_without_keys(oracle):
    """A causal query with Lq > Lk (bottom-right alignment) before the first key
    has no allowed key: O = 0 and LSE = -inf, in every routine."""
    q, k, v = _rand((1, 1, 10, 4), 38), _rand((1, 1, 6, 4), 39), _rand((1, 1, 6, 4), 40)
    o, lse = oracle.attn(q, k, v, 0.5, True)
    assert np.all(o[0, 0, :4] == 0) and np.all(np.isneginf(lse[0, 0, :4]))
    assert np.isfinite(lse[0, 0, 4:]).all()
    ot, lt, _ = oracle.attn_tiled(q, k, v, 0.5, True, -1, -1, 4, 4)
    assert np.abs(ot - o).max() < 1e-13
    assert np.all(np.isneginf(lt[0, 0, :4]))


def test_bf16_inputs_are_widened_exactly(oracle):
    """bf16 and fp32 inputs holding the same values give identical results."""
    q = torch.randn(1, 2, 33, 16, dtype=torch.float32).to(torch.bfloat16)
    k = torch.randn(1, 2, 40, 16, dtype=torch.float32).to(torch.bfloat16)
    v = torch.randn(1, 2, 40, 16, dtype=torch.float32).to(torch.bfloat16)
    o1, l1 = oracle.attn(q, k, v, 0.25, True)
    o2, l2 = oracle.attn(q.double(), k.double(), v.double(), 0.25, True)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_rows_routine_matches_full(oracle):
    q, k, v = _rand((2, 3, 50, 8), 41), _rand((2, 3, 50, 8), 42), _rand((2, 3, 50, 8), 43)
    o, lse = oracle.attn(q, k, v, 0.5, False, 9, 3)
    rows = np.array([(1, 2, 0), (0, 0, 49), (1, 0, 17), (0, 2, 33), (1, 2, 49)])
    ro, rl = oracle.attn_rows(q, k, v, rows, 0.5, False, 9, 3)
    for t, (b, h, i) in enumerate(rows):
        assert np.array_equal(ro[t], o[b, h, i]) and rl[t] == lse[b, h, i]


@pytest.mark.parametrize("S", [1, 2, 7, 32, 1000])
def test_decode_split_merge_equals_naive(oracle, S):
    """P8 (reading R5): split-KV partials merged through their LSE equal exact
    attention of the single query, also with per-sequence lengths and splits
    that are empty."""
    B, H, Lk, d = 3, 2, 1000, 8
    q, k, v = _rand((B, H, 1, d), 44), _rand((B, H, Lk, d), 45), _rand((B, H, Lk, d), 46)
    seqlens = np.array([1000, 517, 3], dtype=np.int32)
    o, lse = oracle.decode_splitmerge(q, k, v, 0.3, S, seqlens)
    o_ref, lse_ref = oracle.attn(q, k, v, 0.3, seqlens_k=seqlens)
    assert np.abs(o - o_ref).max() < 1e-12
    assert np.abs(lse - lse_ref[:, :, 0]).max() < 1e-12


def test_merge_weights_pin(oracle):
    """The merge of two halves equals softmax over the union: a split at the
    middle of two keys with known scores gives the closed-form sigmoid weight."""
    q = np.array([[[[1.0, 0.0]]]])
    k = np.array([[[[2.0, 0.0], [-1.0, 0.0]]]])
    v = np.array([[[[1.0, 3.0], [5.0, -2.0]]]])
    o, lse = oracle.decode_splitmerge(q, k, v, 1.0, 2)
    w0 = 1.0 / (1.0 + math.exp(-3.0))
    assert np.abs(o[0, 0, 0] - (w0 * v[0, 0, 0] + (1 - w0) * v[0, 0, 1])).max() < 1e-15
    assert abs(lse[0, 0] - math.log(math.exp(2.0) + math.exp(-1.0))) < 1e-15


# ---- pair / block counts ([P2] §5.4) -------------------------------------------------------

def _pairs_closed_form(n, causal, wl, wr):
    """In-band pair count of an n x n band, summed row by row in closed form."""
    right = 0 if causal else wr
    total = 0
    for i in range(n):
        lo = 0 if wl < 0 else max(0, i - wl)
        hi = n - 1 if right < 0 else min(n - 1, i + right)
        total += max(0, hi - lo + 1)
    return total


@pytest.mark.parametrize("n,causal,wl,wr,B", [
    (300, False, -1, -1, 64), (300, True, -1, -1, 64), (1000, False, 100, 100, 128),
    (1000, True, 257, 0, 128), (777, False, 0, 0, 64), (640, False, 130, 7, 128),
])
def test_counts_against_closed_forms(oracle, n, causal, wl, wr, B):
    c = oracle.count_blocks(n, n, causal, wl, wr, B, B)
    assert c["pairs"] == _pairs_closed_form(n, causal, wl, wr)
    nb = -(-n // B)
    assert c["total"] == nb * nb
    if causal and wl < 0:
        assert c["pairs"] == n * (n + 1) // 2
        assert c["visited"] == nb * (nb + 1) // 2
    if not causal and wl < 0 and wr < 0:
        assert c["visited"] == nb * nb
    if not causal and wl == wr and wl >= 0:
        w = wl
        assert c["pairs"] == n * (2 * w + 1) - w * (w + 1)


def test_page_band_example(oracle):
    """The worked example of §1 / §5.4 (n = 32768, w = 2048, B = 128): the
    exact counts meet the figures the page prints."""
    with open(os.path.join(HERE, "golden", "p2_band_example.json")) as f:
        g = json.load(f)
    n, w, B, pr = g["n"], g["w"], g["block"], g["printed"]
    assert abs(n * n - pr["n_squared_approx"]) / pr["n_squared_approx"] < 0.01
    assert abs(n * w - pr["n_times_w_approx"]) / pr["n_times_w_approx"] < 0.01
    assert abs((n * w) / (n * n) - pr["compute_ratio_approx"]) < 1e-12
    c = oracle.count_blocks(n, n, False, w, w, B, B)
    assert c["total"] == pr["full_block_pairs"] == pr["q_blocks"] ** 2
    # exact band: n(2w + 1) - w(w + 1) pairs, between the page's n*w and n*(2w+1)
    assert c["pairs"] == n * (2 * w + 1) - w * (w + 1) == 130054144
    # the page's 2w/B + 2 blocks per Q block is an upper bound; interior Q blocks visit 2w/B + 1
    assert c["visited"] <= pr["window_block_pairs_approx"]
    assert c["visited"] == 8176
    assert pr["full_block_pairs"] / c["visited"] >= pr["reduction_approx"]
    one = oracle.count_blocks(n, n, False, w, w, B, B)
    assert one == c
