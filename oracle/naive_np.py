"""NumPy fp64 restatement of exact masked attention, for tiny shapes.

TEST INFRASTRUCTURE ONLY (see ``oracle.py``).  A third, independent statement
of the definition in the sliding-window FlashAttention prefill page
(m.xxqk.cn/news/265020) §2 and §4: the whole score matrix is formed, masked
with -inf outside the band, soft-maxed row by row and multiplied by V.
Window bounds are inclusive and, for Lq != Lk, query i sits at key position
i + Lk - Lq.  Rows with no allowed key give O = 0 and LSE = -inf.
"""
from __future__ import annotations

import numpy as np


def band_mask(Lq, Lk, causal=False, window_left=-1, window_right=-1, len_k=None):
    """Boolean [Lq, Lk] matrix, True where query i may attend key j."""
    i = np.arange(Lq)[:, None] + (Lk - Lq)
    j = np.arange(Lk)[None, :]
    ok = np.ones((Lq, Lk), dtype=bool)
    if len_k is not None:
        ok &= j < len_k
    if causal:
        ok &= j <= i
    if window_right >= 0:
        ok &= j <= i + window_right
    if window_left >= 0:
        ok &= j >= i - window_left
    return ok


def attn_head(q, k, v, scale, causal=False, window_left=-1, window_right=-1, len_k=None):
    """q: [Lq, d], k, v: [Lk, d] float64 -> (O [Lq, d], LSE [Lq])."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    ok = band_mask(q.shape[0], k.shape[0], causal, window_left, window_right, len_k)
    s = np.where(ok, scale * (q @ k.T), -np.inf)
    row_max = s.max(axis=1, keepdims=True)
    empty = ~ok.any(axis=1)
    row_max[empty] = 0.0
    e = np.where(ok, np.exp(s - row_max), 0.0)
    z = e.sum(axis=1, keepdims=True)
    z_safe = np.where(empty[:, None], 1.0, z)
    o = (e @ v) / z_safe
    lse = np.where(empty, -np.inf, row_max[:, 0] + np.log(z_safe[:, 0]))
    return o, lse
