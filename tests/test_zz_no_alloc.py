"""The decode entry point for callers that cannot allocate device memory.

attn_decode_splitkv_noalloc keeps its split partials in a scratch array that
is part of the library, so a caller that only owns its inputs and outputs (a
plugin handed buffers by its host application, a service under a fixed memory
budget) can run split-KV decode without a workspace.  These checks call it
through the C ABI and compare it with attn_decode_splitkv, which takes a
caller workspace, bit for bit on calls in a row with different shapes (a call
must not depend on what the one before left in the shared scratch), and with
the fp64 oracle.  The file sorts last so that a run stopping at the first
failure has run every other test.
"""
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


def _inputs(B, H, Lk, d, seed):
    q, _, _ = synth.random_qkv(B, H, 1, 1, d, "bf16", seed=seed)
    _, k, v = synth.random_qkv(B, H, 1, Lk, d, "bf16", seed=seed + 1)
    g = torch.Generator().manual_seed(seed)
    seqlens = torch.randint(0, Lk + 1, (B,), generator=g, dtype=torch.int32)
    seqlens[0] = Lk
    seqlens[-1] = 0
    return q.cuda(), k.cuda(), v.cuda(), seqlens.cuda()


def test_noalloc_decode_matches_workspace_decode(fl):
    # Both entry points run the same split and merge kernels with the same
    # split count, so their outputs must be identical bit for bit; a partial
    # left in the shared scratch by the previous call would show up here.
    # num_splits = 0 lets both pick the split count themselves.
    for B, H, Lk, d, S, seed in [(6, 8, 5000, 128, 16, 21), (3, 4, 700, 64, 5, 22), (4, 8, 3000, 128, 0, 23)]:
        q, k, v, seqlens = _inputs(B, H, Lk, d, seed)
        o_ref, lse_ref = fl.attn_decode_splitkv(q, k, v, seqlens_k=seqlens, num_splits=S)
        o, lse = fl.attn_decode_splitkv_noalloc(q, k, v, seqlens_k=seqlens, num_splits=S)
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref)
        assert torch.equal(lse, lse_ref)


def test_noalloc_decode_matches_oracle(fl, oracle):
    # the same check against the fp64 oracle directly, at the bars of the
    # other decode tests
    B, H, Lk, d = 3, 4, 2500, 128
    q, k, v, seqlens = _inputs(B, H, Lk, d, 31)
    o, lse = fl.attn_decode_splitkv_noalloc(q, k, v, seqlens_k=seqlens, num_splits=0)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attn(q.cpu(), k.cpu(), v.cpu(), d ** -0.5, seqlens_k=seqlens.cpu().numpy())
    compare(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref[..., 0], BF16_O_MAXABS, BF16_O_RELL2,
            label="noalloc decode")


def test_noalloc_rejects_more_than_its_scratch(fl):
    # 16 x 32 heads x 64 splits x 129 floats x 4 B = 16.9 MB > 16 MiB of scratch;
    # the tensors are full size, so the call would be valid with a workspace
    B, H, Lk, d, S = 16, 32, 8192, 128, 64
    need = fl.attn_decode_workspace_bytes(B, H, Lk, d, S)
    assert need > (16 << 20)
    q = torch.zeros((B, H, 1, d), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((B, H, Lk, d), dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    status = fl.lib.attn_decode_splitkv_noalloc(q.data_ptr(), kv.data_ptr(), kv.data_ptr(), o.data_ptr(), None,
                                                None, B, H, Lk, d, 0.1, S, None)
    assert status == fl.FATTN_ERR_WORKSPACE
    o2, _ = fl.attn_decode_splitkv_noalloc(q, kv, kv, num_splits=8)   # fits: 2.1 MB
    torch.cuda.synchronize()
    assert torch.all(o2 == 0)
