"""Seeded synthetic workloads (shapes, value distributions and seeds).

This module only draws random inputs; it holds none of the attention
arithmetic, so both the CUDA path and the CPU oracle can take their inputs
from it.  Every draw is fp32 from a seeded ``torch.Generator`` (Q first, then
K, then V, then any per-head factors); bf16 workloads are then rounded to
bf16 by round-to-nearest-even and both sides see the rounded values.

The workloads follow the sliding-window FlashAttention prefill page
(m.xxqk.cn/news/265020): n from 4K to 64K, windows of 2048 / 4096, head
dim 64 / 128, and the flash-decoding shape of "算子与编译器：FlashAttention
与长上下文" §4 (one query against a long cached K/V).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "prefill" or "decode"
    B: int
    H: int
    Lq: int
    Lk: int
    d: int
    dtype: str           # "f32" or "bf16"
    causal: bool = False
    window_left: int = -1
    window_right: int = -1
    seed: int = 0
    q_head_scale: Optional[tuple] = None   # (lo, hi): per-head U(lo, hi) factor on Q
    num_splits: int = 0                    # decode only

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def describe(self) -> dict:
        out = {"workload": self.name, "B": self.B, "H": self.H, "Lq": self.Lq, "Lk": self.Lk,
               "d": self.d, "dtype": self.dtype}
        if self.kind == "prefill":
            out.update(causal=self.causal, window_left=self.window_left,
                       window_right=self.window_right)
        else:
            out.update(num_splits=self.num_splits)
        if self.q_head_scale:
            out["q_head_scale"] = list(self.q_head_scale)
        return out


WORKLOADS = {
    # tiny exact check: fp32, full attention, block size 64 in the tiled oracle
    "tiny_f32": Workload("tiny_f32", "prefill", 1, 1, 256, 256, 64, "f32", seed=1),
    # causal prefill 4 x 16 x 4096, d = 128
    "causal_4k": Workload("causal_4k", "prefill", 4, 16, 4096, 4096, 128, "bf16",
                          causal=True, seed=2),
    # the same causal prefill at head dim 64
    "causal_4k_d64": Workload("causal_4k_d64", "prefill", 4, 16, 4096, 4096, 64, "bf16",
                              causal=True, seed=8),
    # sliding window n = 32768, bidirectional |i - j| <= 2048
    "window_bidir_32k": Workload("window_bidir_32k", "prefill", 1, 32, 32768, 32768, 128,
                                 "bf16", window_left=2048, window_right=2048, seed=3),
    # the same bidirectional window at head dim 64
    "window_bidir_32k_d64": Workload("window_bidir_32k_d64", "prefill", 1, 32, 32768, 32768, 64,
                                     "bf16", window_left=2048, window_right=2048, seed=9),
    # sliding window n = 32768, causal left window j in [i - 4096, i]
    "window_causal_32k": Workload("window_causal_32k", "prefill", 1, 32, 32768, 32768, 128,
                                  "bf16", causal=True, window_left=4096, window_right=0, seed=3),
    # long full-causal prefill, per-head query scale U(0.5, 2)
    "causal_64k_qscale": Workload("causal_64k_qscale", "prefill", 1, 16, 65536, 65536, 128,
                                  "bf16", causal=True, seed=4, q_head_scale=(0.5, 2.0)),
    # flash-decoding shape: 64 x 32 heads, 32768 cached keys, 32 splits
    "decode_32k": Workload("decode_32k", "decode", 64, 32, 1, 32768, 128, "bf16",
                           seed=5, num_splits=32),
}


def _torch_dtype(name: str):
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def _draw(shape, g, dev, dt):
    """fp32 N(0, 1) draw of ``shape`` rounded to ``dt``; large draws go in
    slices along the batch axis so the fp32 staging stays small."""
    out = torch.empty(shape, dtype=dt, device=dev)
    for b in range(shape[0]):
        out[b].copy_(torch.randn(shape[1:], generator=g, device=dev, dtype=torch.float32))
    return out


def make_inputs(w: Workload, device="cpu", seed: Optional[int] = None):
    """Draw (q, k, v) for workload ``w``: layout [B, H, L, d], contiguous.

    CPU draws use a CPU generator; ``device="cuda..."`` draws on the GPU with a
    seeded CUDA generator (used for the multi-GB decode cache).  Draw order:
    Q (fp32), K, V, then the per-head Q factors; Q is multiplied by its head
    factor in fp32 before it is rounded.
    """
    seed = w.seed if seed is None else seed
    dev = torch.device(device)
    g = torch.Generator(device=dev.type)
    g.manual_seed(seed)
    dt = _torch_dtype(w.dtype)
    q = _draw((w.B, w.H, w.Lq, w.d), g, dev, torch.float32)
    k = _draw((w.B, w.H, w.Lk, w.d), g, dev, dt)
    v = _draw((w.B, w.H, w.Lk, w.d), g, dev, dt)
    if w.q_head_scale is not None:
        lo, hi = w.q_head_scale
        u = torch.rand((w.H,), generator=g, device=dev, dtype=torch.float32) * (hi - lo) + lo
        q.mul_(u.view(1, w.H, 1, 1))
    q = q.to(dt)
    return q, k, v


def random_qkv(B, H, Lq, Lk, d, dtype="bf16", seed=0, device="cpu"):
    """Plain i.i.d. N(0, 1) draws of a given shape (test grids)."""
    w = Workload("adhoc", "prefill", B, H, Lq, Lk, d, dtype, seed=seed)
    return make_inputs(w, device=device)


def random_dout(B, H, Lq, d, dtype="bf16", seed=0, device="cpu"):
    """Upstream gradient dO for the backward: i.i.d. N(0, 1), [B, H, Lq, d],
    from its own generator (seed offset so it never equals a Q draw)."""
    dev = torch.device(device)
    g = torch.Generator(device=dev.type)
    g.manual_seed(1_000_003 + seed)
    return _draw((B, H, Lq, d), g, dev, _torch_dtype(dtype))


def varlen_lengths(n_seqs: int, lo: int, hi: int, seed: int):
    """Sequence lengths drawn uniformly from [lo, hi] (a length mix for packed
    batches of requests)."""
    g = torch.Generator().manual_seed(seed)
    return torch.randint(lo, hi + 1, (n_seqs,), generator=g).tolist()


def make_varlen_inputs(lens_q, lens_k, H: int, d: int, seed: int, device="cpu"):
    """Packed token-major inputs: q [sum(lens_q), H, d], k and v
    [sum(lens_k), H, d] (bf16, from fp32 N(0, 1) draws, Q then K then V) and
    the int32 offsets cu_seqlens_q / cu_seqlens_k [n + 1]."""
    dev = torch.device(device)
    g = torch.Generator(device=dev.type)
    g.manual_seed(seed)
    tq, tk = int(sum(lens_q)), int(sum(lens_k))
    q = torch.randn((tq, H, d), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    k = torch.randn((tk, H, d), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    v = torch.randn((tk, H, d), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    cu_q = torch.tensor([0] + list(_cumsum(lens_q)), dtype=torch.int32, device=dev)
    cu_k = torch.tensor([0] + list(_cumsum(lens_k)), dtype=torch.int32, device=dev)
    return q, k, v, cu_q, cu_k


def _cumsum(xs):
    total = 0
    for x in xs:
        total += int(x)
        yield total


def scatter_to_pages(k, v, page_size: int, seed: int, extra_pages: int = 0):
    """Place a contiguous cache k, v [B, H, L, d] (L a multiple of page_size)
    into a pool of pages [num_pages, page_size, H, d] in a seeded random page
    order; returns (k_pages, v_pages, block_table int32 [B, L / page_size]).
    extra_pages unused pages are added to the pool.  Pure data movement."""
    B, H, L, d = k.shape
    assert L % page_size == 0
    per_seq = L // page_size
    num_pages = B * per_seq + extra_pages
    g = torch.Generator().manual_seed(seed)
    perm = torch.randperm(num_pages, generator=g)[: B * per_seq].view(B, per_seq)
    kp = torch.zeros((num_pages, page_size, H, d), dtype=k.dtype, device=k.device)
    vp = torch.zeros_like(kp)
    # [B, H, per_seq, page_size, d] -> [B, per_seq, page_size, H, d]
    kk = k.view(B, H, per_seq, page_size, d).permute(0, 2, 3, 1, 4)
    vv = v.view(B, H, per_seq, page_size, d).permute(0, 2, 3, 1, 4)
    idx = perm.to(k.device).reshape(-1)
    kp[idx] = kk.reshape(B * per_seq, page_size, H, d)
    vp[idx] = vv.reshape(B * per_seq, page_size, H, d)
    return kp, vp, perm.to(torch.int32).to(k.device).contiguous()


def make_paged_inputs(B: int, H: int, L: int, d: int, page_size: int, seed: int, device="cuda"):
    """A decode batch over a paged cache: q [B, H, 1, d], page pools
    [B * L / page_size, page_size, H, d] drawn directly (fp32 N(0, 1) rounded
    to bf16, pool by pool), a seeded random block table [B, L / page_size]
    (a permutation of the pool) and full lengths L."""
    dev = torch.device(device)
    g = torch.Generator(device=dev.type)
    g.manual_seed(seed)
    per_seq = L // page_size
    num_pages = B * per_seq
    q = torch.randn((B, H, 1, d), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    kp = _draw((num_pages, page_size, H, d), g, dev, torch.bfloat16)
    vp = _draw((num_pages, page_size, H, d), g, dev, torch.bfloat16)
    gc = torch.Generator().manual_seed(seed)
    table = torch.randperm(num_pages, generator=gc).view(B, per_seq).to(torch.int32).to(dev)
    seqlens = torch.full((B,), L, dtype=torch.int32, device=dev)
    return q, kp, vp, table, seqlens


def sample_rows(w: Workload, n_random: int, seed: int = 0, full_heads=()):
    """Stratified (b, h, i) row sample: first / last rows, rows at 128-block
    and window edges, plus ``n_random`` uniform rows per head; every row of the
    heads listed in ``full_heads`` (pairs (b, h)).  Returns an int tensor [n, 3].
    """
    g = torch.Generator().manual_seed(seed)
    rows = set()
    Lq = w.Lq
    edges = {0, 1, Lq - 1, Lq - 2, 127, 128, 129, 255, 256}
    for wsz in (w.window_left, w.window_right):
        if wsz and wsz > 0:
            edges |= {wsz - 1, wsz, wsz + 1, Lq - wsz - 1, Lq - wsz}
    edges = {e for e in edges if 0 <= e < Lq}
    for b in range(w.B):
        for h in range(w.H):
            for e in edges:
                rows.add((b, h, e))
            if n_random > 0:
                for i in torch.randint(0, Lq, (n_random,), generator=g).tolist():
                    rows.add((b, h, i))
    for (b, h) in full_heads:
        for i in range(Lq):
            rows.add((b, h, i))
    return torch.tensor(sorted(rows), dtype=torch.int32)
