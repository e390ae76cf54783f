"""The Python binding refuses tensors whose shapes disagree before any kernel
is launched: the kernels index every buffer from (B, H, Lq, Lk, d), so a
short output or workspace would otherwise be written past its end."""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fl():
    from io_aware_exact_34_b200 import fattn
    return fattn


def _bf(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16, device="cuda")


def _f(*shape):
    return torch.zeros(shape, dtype=torch.float32, device="cuda")


def test_fwd_rejects_mismatched_shapes(fl):
    q, k, v = _bf(1, 2, 64, 128), _bf(1, 2, 96, 128), _bf(1, 2, 96, 128)
    with pytest.raises(ValueError, match="o:"):
        fl.attn_fwd(q, k, v, o=_bf(1, 2, 63, 128))
    with pytest.raises(ValueError, match="v:"):
        fl.attn_fwd(q, k, _bf(1, 2, 95, 128))
    with pytest.raises(ValueError, match="k:"):
        fl.attn_fwd(q, _bf(1, 1, 96, 128), v)
    with pytest.raises(ValueError, match="lse:"):
        fl.attn_fwd(q, k, v, lse=_f(1, 2, 32))
    with pytest.raises(ValueError, match="counter:"):
        fl.attn_fwd_counted(q, k, v, torch.zeros(1, dtype=torch.int32, device="cuda"))


def test_varlen_rejects_mismatched_shapes(fl):
    q, k = _bf(40, 2, 128), _bf(50, 2, 128)
    cq = torch.tensor([0, 10, 40], dtype=torch.int32, device="cuda")
    ck = torch.tensor([0, 20, 50], dtype=torch.int32, device="cuda")
    with pytest.raises(ValueError, match="cu_seqlens_k:"):
        fl.attn_fwd_varlen(q, k, k, cq, ck[:2], 30)
    with pytest.raises(ValueError, match="lse:"):
        fl.attn_fwd_varlen(q, k, k, cq, ck, 30, lse=_f(2, 39))


def test_decode_rejects_mismatched_shapes(fl):
    q, kc = _bf(2, 2, 1, 128), _bf(2, 2, 300, 128)
    with pytest.raises(ValueError, match="decode takes one query"):
        fl.attn_decode_splitkv(_bf(2, 2, 2, 128), kc, kc)
    with pytest.raises(ValueError, match="lse:"):
        fl.attn_decode_splitkv(q, kc, kc, lse=_f(2, 1))
    with pytest.raises(ValueError, match="seqlens_k:"):
        fl.attn_decode_splitkv_noalloc(q, kc, kc, seqlens_k=torch.ones(3, dtype=torch.int32, device="cuda"))
    pages = _bf(8, 64, 2, 128)
    bt = torch.zeros((2, 4), dtype=torch.int32, device="cuda")
    sk = torch.ones(2, dtype=torch.int32, device="cuda")
    with pytest.raises(ValueError, match="block_table:"):
        fl.attn_decode_paged(q, pages, pages, bt[:1], sk)
    with pytest.raises(ValueError, match="v_pages:"):
        fl.attn_decode_paged(q, pages, _bf(8, 32, 2, 128), bt, sk)


def test_bwd_and_fp8_reject_mismatched_shapes(fl):
    q, k = _bf(1, 2, 64, 128), _bf(1, 2, 96, 128)
    lse = _f(1, 2, 64)
    with pytest.raises(ValueError, match="dk:"):
        fl.attn_bwd(q, k, k, q, q, lse, dk=_bf(1, 2, 64, 128))
    with pytest.raises(ValueError, match="dout:"):
        fl.attn_bwd(q, k, k, q, _bf(1, 2, 65, 128), lse)
    with pytest.raises(ValueError, match="codes:"):
        fl.attn_quantize_fp8(q, transpose=True, codes=torch.zeros((1, 2, 128, 64), dtype=torch.uint8,
                                                                     device="cuda")[..., :48].contiguous())
    q8 = torch.zeros((1, 2, 64, 128), dtype=torch.uint8, device="cuda")
    k8 = torch.zeros((1, 2, 96, 128), dtype=torch.uint8, device="cuda")
    vt8 = torch.zeros((1, 2, 128, fl.attn_fp8_ld(96)), dtype=torch.uint8, device="cuda")
    ds = _f(1, 2)
    with pytest.raises(ValueError, match="k_descale:"):
        fl.attn_fwd_fp8(q8, k8, vt8, ds, _f(2, 1), ds)
