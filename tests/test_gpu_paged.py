"""Paged-KV split decode (attn_decode_paged) against the fp64 oracle: a
contiguous cache is scattered into randomly ordered pages, the GPU reads it
through the block table, the oracle reads the contiguous copy."""
import numpy as np
import pytest
import torch

from io_aware_exact_34_b200 import synth
from tests._compare import BF16_O_MAXABS, BF16_O_RELL2, compare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fl():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from io_aware_exact_34_b200 import build
    build.build()
    from io_aware_exact_34_b200 import fattn
    return fattn


@pytest.mark.parametrize("B,H,L,d,page,S", [
    (3, 2, 1024, 128, 16, 4), (2, 3, 4096, 128, 256, 8), (4, 2, 512, 64, 64, 0), (2, 2, 2048, 128, 128, 1),
])
def test_paged_decode_matches_oracle(fl, oracle, B, H, L, d, page, S):
    q, _, _ = synth.random_qkv(B, H, 1, 1, d, "bf16", seed=L + page)
    _, k, v = synth.random_qkv(B, H, 1, L, d, "bf16", seed=L + page + 1)
    g = torch.Generator().manual_seed(L)
    seqlens = torch.randint(1, L + 1, (B,), generator=g, dtype=torch.int32)
    seqlens[0] = L
    kp, vp, table = synth.scatter_to_pages(k.cuda(), v.cuda(), page, seed=page, extra_pages=5)
    o, lse = fl.attn_decode_paged(q.cuda(), kp, vp, table, seqlens.cuda(), num_splits=S)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attn(q, k, v, d ** -0.5, seqlens_k=seqlens.numpy())
    compare(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref[..., 0], BF16_O_MAXABS, BF16_O_RELL2,
            label=f"paged {B},{H},{L},{d},{page}")


def test_paged_equals_contiguous_decode(fl):
    """Same inputs through the contiguous and the paged entry points: the
    split layout is identical, so the outputs agree to the last bit."""
    B, H, L, d = 4, 4, 8192, 128
    q, _, _ = synth.random_qkv(B, H, 1, 1, d, "bf16", seed=5)
    _, k, v = synth.random_qkv(B, H, 1, L, d, "bf16", seed=6)
    seqlens = torch.tensor([8192, 100, 4097, 1], dtype=torch.int32).cuda()
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o1, l1 = fl.attn_decode_splitkv(qd, kd, vd, seqlens_k=seqlens, num_splits=8)
    kp, vp, table = synth.scatter_to_pages(kd, vd, 256, seed=3)
    o2, l2 = fl.attn_decode_paged(qd, kp, vp, table, seqlens, num_splits=8)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
