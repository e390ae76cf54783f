"""Python binding of libfattn: argument marshalling over the C ABI only.

Every function here takes torch tensors, checks their dtype / device / layout,
passes raw pointers, sizes and the current CUDA stream to the library of the
same name, and raises ``FattnError`` on a non-zero status.  All arithmetic runs
in the library's CUDA kernels; there is no fallback of any kind.  If the
shared library is missing, importing this module fails.
"""
from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfattn.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"libfattn.so is not built ({_LIB_PATH}); run "
                      "`python -m io_aware_exact_34_b200.build`")
lib = ctypes.CDLL(_LIB_PATH)

_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
_llp = ctypes.POINTER(ctypes.c_longlong)
lib.attn_fwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _i, _i, _i, _vp]
lib.attn_fwd.restype = _i
lib.attn_fwd_host.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _i, _i, _i, _vp, ctypes.c_size_t, _vp]
lib.attn_fwd_host.restype = _i
lib.attn_fwd_host_workspace_bytes.argtypes = [_i, _i, _i, _i, _i]
lib.attn_fwd_host_workspace_bytes.restype = ctypes.c_size_t
lib.attn_fwd_counted.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _i, _i, _i, _vp, _vp]
lib.attn_fwd_counted.restype = _i
lib.attn_fwd_varlen.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _i, _i, _vp]
lib.attn_fwd_varlen.restype = _i
lib.attn_fwd_varlen_counted.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _i, _i,
                                        _vp, _vp]
lib.attn_fwd_varlen_counted.restype = _i
lib.attn_fwd_f32.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _i, _i, _i, _vp]
lib.attn_fwd_f32.restype = _i
lib.attn_decode_splitkv.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _vp, _sz, _vp]
lib.attn_decode_splitkv.restype = _i
lib.attn_decode_splitkv_noalloc.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _vp]
lib.attn_decode_splitkv_noalloc.restype = _i
lib.attn_decode_paged.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _vp, _vp, _vp, _i, _i, _i, _f, _i, _vp, _sz, _vp]
lib.attn_decode_paged.restype = _i
lib.attn_decode_auto_splits.argtypes = [_i, _i, _i, _i]
lib.attn_decode_auto_splits.restype = _i
lib.attn_decode_workspace_bytes.argtypes = [_i, _i, _i, _i, _i]
lib.attn_decode_workspace_bytes.restype = _sz
lib.attn_count_blocks.argtypes = [_i, _i, _i, _i, _i, _i, _i, _llp, _llp, _llp, _llp]
lib.attn_count_blocks.restype = _i
lib.attn_bwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _i, _i, _i, _vp, _sz, _vp]
lib.attn_bwd.restype = _i
lib.attn_bwd_counted.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _i, _i, _i, _vp,
                                 _sz, _vp, _vp]
lib.attn_bwd_counted.restype = _i
lib.attn_bwd_workspace_bytes.argtypes = [_i, _i, _i, _i]
lib.attn_bwd_workspace_bytes.restype = _sz
lib.attn_bwd_count_blocks.argtypes = [_i, _i, _i, _i, _i, _i, _i, _llp]
lib.attn_bwd_count_blocks.restype = _i
lib.attn_fwd_fp8.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _i, _i, _i, _vp]
lib.attn_fwd_fp8.restype = _i
lib.attn_fwd_fp8_counted.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _i, _i, _i, _vp,
                                     _vp]
lib.attn_fwd_fp8_counted.restype = _i
lib.attn_fp8_ld.argtypes = [_i]
lib.attn_fp8_ld.restype = _i
lib.attn_quantize_fp8.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _i, _vp]
lib.attn_quantize_fp8.restype = _i
lib.fattn_status_string.argtypes = [_i]
lib.fattn_status_string.restype = ctypes.c_char_p
lib.fattn_device_status.argtypes = [_vp]
lib.fattn_device_status.restype = _i
lib.fattn_debug_inject_stall.argtypes = [_i]
lib.fattn_debug_inject_stall.restype = _i

FATTN_OK = 0
FATTN_ERR_INVALID_ARG = -1
FATTN_ERR_UNSUPPORTED = -2
FATTN_ERR_MISALIGNED = -3
FATTN_ERR_WORKSPACE = -4
FATTN_ERR_CUDA = -5
FATTN_ERR_TIMEOUT = -6
FATTN_ERR_NO_DEVICE = -7


class FattnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {lib.fattn_status_string(status).decode()}")


def _check(status: int, where: str) -> None:
    if status != FATTN_OK:
        raise FattnError(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _want(t, dtype, ndim, name, shape=None, device=None):
    """Every pointer the library receives comes from a tensor checked here:
    dtype, rank, contiguity, CUDA residency and, where given, the exact shape
    and the device of the first input (the kernels trust all of these)."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype or t.dim() != ndim or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous {dtype} CUDA tensor with {ndim} dims, got "
                         f"{t.dtype} {tuple(t.shape)} on {t.device}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if device is not None and t.device != device:
        raise ValueError(f"{name}: on {t.device}, expected {device}")


def _want_counter(counter, device):
    if counter is not None:
        if not isinstance(counter, torch.Tensor) or counter.dtype not in (torch.int64, torch.uint64) \
                or counter.numel() != 1 or not counter.is_cuda or counter.device != device:
            raise ValueError(f"counter: expected a one-element int64 tensor on {device}")


def _want_workspace(ws, device):
    if ws is not None:
        if not isinstance(ws, torch.Tensor) or not ws.is_cuda or ws.device != device or not ws.is_contiguous():
            raise ValueError(f"workspace: expected a contiguous CUDA tensor on {device}")


def attn_fwd(q, k, v, o=None, lse=None, scale=None, causal=False, window_left=-1, window_right=-1,
             need_lse=True, counter=None):
    """bf16 prefill forward.  q: [B,H,Lq,d], k, v: [B,H,Lk,d] -> (o, lse).
    ``counter`` (optional, a zeroed one-element int64 CUDA tensor) receives the
    number of KV tiles visited."""
    _want(q, torch.bfloat16, 4, "q")
    B, H, Lq, d = q.shape
    dev = q.device
    _want(k, torch.bfloat16, 4, "k", device=dev)
    Lk = k.shape[2]
    _want(k, torch.bfloat16, 4, "k", shape=(B, H, Lk, d))  # same batch, heads and head dim as q
    _want(v, torch.bfloat16, 4, "v", shape=(B, H, Lk, d), device=dev)
    _want_counter(counter, dev)
    if o is None:
        o = torch.empty_like(q)
    _want(o, torch.bfloat16, 4, "o", shape=(B, H, Lq, d), device=dev)
    if lse is None and need_lse:
        lse = torch.empty((B, H, Lq), dtype=torch.float32, device=dev)
    if lse is not None:
        _want(lse, torch.float32, 3, "lse", shape=(B, H, Lq), device=dev)
    scale = (1.0 / d ** 0.5) if scale is None else scale
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Lq, Lk, d, scale, int(bool(causal)),
            int(window_left), int(window_right))
    if counter is None:
        _check(lib.attn_fwd(*args, _stream()), "attn_fwd")
    else:
        _check(lib.attn_fwd_counted(*args, _ptr(counter), _stream()), "attn_fwd_counted")
    return o, lse


def attn_fwd_counted(q, k, v, counter, o=None, lse=None, scale=None, causal=False, window_left=-1,
                     window_right=-1):
    """attn_fwd that adds the number of KV tiles visited to ``counter``
    (a zeroed uint64/int64 CUDA tensor with one element)."""
    return attn_fwd(q, k, v, o, lse, scale, causal, window_left, window_right, counter=counter)


def attn_fwd_host_workspace_bytes(B, H, Lq, Lk, d) -> int:
    return lib.attn_fwd_host_workspace_bytes(B, H, Lq, Lk, d)


def _want_host(t, dtype, ndim, name, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype or t.dim() != ndim or t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous {dtype} host tensor with {ndim} dims, got "
                         f"{t.dtype} {tuple(t.shape)} on {t.device}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")


def attn_fwd_host(q, k, v, o=None, lse=None, scale=None, causal=False, window_left=-1, window_right=-1,
                  need_lse=True, workspace=None):
    """attn_fwd on host tensors (pin them for the copies to overlap the
    kernels): q [B,H,Lq,d], k, v [B,H,Lk,d] bf16 on the CPU -> (o, lse) on the
    CPU.  The device workspace is allocated here unless given (a uint8 CUDA
    tensor of attn_fwd_host_workspace_bytes).  Returns once the results are in
    o and lse (the current stream is synchronised)."""
    _want_host(q, torch.bfloat16, 4, "q")
    B, H, Lq, d = q.shape
    Lk = k.shape[2] if k.dim() == 4 else -1
    _want_host(k, torch.bfloat16, 4, "k", shape=(B, H, Lk, d))
    _want_host(v, torch.bfloat16, 4, "v", shape=(B, H, Lk, d))
    if o is None:
        o = torch.empty_like(q, pin_memory=True)
    _want_host(o, torch.bfloat16, 4, "o", shape=(B, H, Lq, d))
    if lse is None and need_lse:
        lse = torch.empty((B, H, Lq), dtype=torch.float32, pin_memory=True)
    if lse is not None:
        _want_host(lse, torch.float32, 3, "lse", shape=(B, H, Lq))
    dev = torch.device("cuda", torch.cuda.current_device())
    need = attn_fwd_host_workspace_bytes(B, H, Lq, Lk, d)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    _want_workspace(workspace, dev)
    scale = (1.0 / d ** 0.5) if scale is None else scale
    _check(lib.attn_fwd_host(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Lq, Lk, d, scale,
                             int(bool(causal)), int(window_left), int(window_right), _ptr(workspace),
                             workspace.numel() * workspace.element_size(), _stream()), "attn_fwd_host")
    torch.cuda.current_stream().synchronize()
    return o, lse


def attn_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, o=None, lse=None, scale=None,
                    causal=False, window_left=-1, window_right=-1, counter=None):
    """Packed variable-length prefill.  q: [total_q, H, d], k, v: [total_k, H, d]
    bf16; cu_seqlens_*: int32 [num_seqs + 1] on the device -> (o, lse [H, total_q])."""
    _want(q, torch.bfloat16, 3, "q")
    _want(k, torch.bfloat16, 3, "k")
    _want(v, torch.bfloat16, 3, "v")
    _want(cu_seqlens_q, torch.int32, 1, "cu_seqlens_q")
    _want(cu_seqlens_k, torch.int32, 1, "cu_seqlens_k")
    total_q, H, d = q.shape
    dev = q.device
    total_k = k.shape[0]
    nseq = cu_seqlens_q.numel() - 1
    _want(k, torch.bfloat16, 3, "k", shape=(total_k, H, d), device=dev)
    _want(v, torch.bfloat16, 3, "v", shape=(total_k, H, d), device=dev)
    _want(cu_seqlens_q, torch.int32, 1, "cu_seqlens_q", device=dev)
    _want(cu_seqlens_k, torch.int32, 1, "cu_seqlens_k", shape=(nseq + 1,), device=dev)
    _want_counter(counter, dev)
    if o is None:
        o = torch.empty_like(q)
    _want(o, torch.bfloat16, 3, "o", shape=(total_q, H, d), device=dev)
    if lse is None:
        lse = torch.empty((H, total_q), dtype=torch.float32, device=dev)
    _want(lse, torch.float32, 2, "lse", shape=(H, total_q), device=dev)
    scale = (1.0 / d ** 0.5) if scale is None else scale
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), nseq, H, total_q,
            total_k, int(max_seqlen_q), d, scale, int(bool(causal)), int(window_left), int(window_right))
    if counter is None:
        _check(lib.attn_fwd_varlen(*args, _stream()), "attn_fwd_varlen")
    else:
        _check(lib.attn_fwd_varlen_counted(*args, _ptr(counter), _stream()), "attn_fwd_varlen_counted")
    return o, lse


def attn_fwd_f32(q, k, v, o=None, lse=None, scale=None, causal=False, window_left=-1, window_right=-1):
    """fp32 prefill forward on the CUDA cores.  Same arguments as attn_fwd."""
    _want(q, torch.float32, 4, "q")
    _want(k, torch.float32, 4, "k")
    _want(v, torch.float32, 4, "v")
    B, H, Lq, d = q.shape
    dev = q.device
    Lk = k.shape[2]
    _want(k, torch.float32, 4, "k", shape=(B, H, Lk, d), device=dev)
    _want(v, torch.float32, 4, "v", shape=(B, H, Lk, d), device=dev)
    if o is None:
        o = torch.empty_like(q)
    _want(o, torch.float32, 4, "o", shape=(B, H, Lq, d), device=dev)
    if lse is None:
        lse = torch.empty((B, H, Lq), dtype=torch.float32, device=dev)
    _want(lse, torch.float32, 3, "lse", shape=(B, H, Lq), device=dev)
    scale = (1.0 / d ** 0.5) if scale is None else scale
    _check(lib.attn_fwd_f32(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Lq, Lk, d, scale,
                            int(bool(causal)), int(window_left), int(window_right), _stream()), "attn_fwd_f32")
    return o, lse


def attn_decode_auto_splits(B, H, Lk, d) -> int:
    return lib.attn_decode_auto_splits(B, H, Lk, d)


def attn_decode_workspace_bytes(B, H, Lk, d, num_splits=0) -> int:
    return lib.attn_decode_workspace_bytes(B, H, Lk, d, num_splits)


def attn_decode_splitkv(q, k_cache, v_cache, o=None, lse=None, seqlens_k=None, scale=None,
                        num_splits=0, workspace=None):
    """Split-KV decode.  q: [B,H,1,d], caches [B,H,Lk,d] -> (o [B,H,1,d], lse [B,H])."""
    _want(q, torch.bfloat16, 4, "q")
    _want(k_cache, torch.bfloat16, 4, "k_cache")
    _want(v_cache, torch.bfloat16, 4, "v_cache")
    B, H, Lq, d = q.shape
    dev = q.device
    if Lq != 1:
        raise ValueError(f"q: decode takes one query per head, got Lq={Lq}")
    Lk = k_cache.shape[2]
    _want(k_cache, torch.bfloat16, 4, "k_cache", shape=(B, H, Lk, d), device=dev)
    _want(v_cache, torch.bfloat16, 4, "v_cache", shape=(B, H, Lk, d), device=dev)
    if o is None:
        o = torch.empty_like(q)
    _want(o, torch.bfloat16, 4, "o", shape=(B, H, 1, d), device=dev)
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=dev)
    _want(lse, torch.float32, 2, "lse", shape=(B, H), device=dev)
    if seqlens_k is not None:
        _want(seqlens_k, torch.int32, 1, "seqlens_k", shape=(B,), device=dev)
    S = num_splits if num_splits > 0 else attn_decode_auto_splits(B, H, Lk, d)
    need = attn_decode_workspace_bytes(B, H, Lk, d, S)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    _want_workspace(workspace, dev)
    scale = (1.0 / d ** 0.5) if scale is None else scale
    _check(lib.attn_decode_splitkv(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(o), _ptr(lse),
                                   _ptr(seqlens_k), B, H, Lk, d, scale, S, _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream()),
           "attn_decode_splitkv")
    return o, lse


def attn_decode_splitkv_noalloc(q, k_cache, v_cache, o=None, lse=None, seqlens_k=None, scale=None,
                                num_splits=0):
    """Split-KV decode whose split partials live in the library's own static
    scratch (for callers that cannot allocate device memory); o and lse are
    still the caller's.  Same results as attn_decode_splitkv."""
    _want(q, torch.bfloat16, 4, "q")
    _want(k_cache, torch.bfloat16, 4, "k_cache")
    _want(v_cache, torch.bfloat16, 4, "v_cache")
    B, H, Lq, d = q.shape
    dev = q.device
    if Lq != 1:
        raise ValueError(f"q: decode takes one query per head, got Lq={Lq}")
    Lk = k_cache.shape[2]
    _want(k_cache, torch.bfloat16, 4, "k_cache", shape=(B, H, Lk, d), device=dev)
    _want(v_cache, torch.bfloat16, 4, "v_cache", shape=(B, H, Lk, d), device=dev)
    if o is None:
        o = torch.empty_like(q)
    _want(o, torch.bfloat16, 4, "o", shape=(B, H, 1, d), device=dev)
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=dev)
    _want(lse, torch.float32, 2, "lse", shape=(B, H), device=dev)
    if seqlens_k is not None:
        _want(seqlens_k, torch.int32, 1, "seqlens_k", shape=(B,), device=dev)
    scale = (1.0 / d ** 0.5) if scale is None else scale
    _check(lib.attn_decode_splitkv_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(o), _ptr(lse),
                                           _ptr(seqlens_k), B, H, Lk, d, scale, int(num_splits), _stream()),
           "attn_decode_splitkv_noalloc")
    return o, lse


def attn_decode_paged(q, k_pages, v_pages, block_table, seqlens_k, o=None, lse=None, scale=None, num_splits=0,
                      workspace=None):
    """Split-KV decode over a paged cache.  q: [B,H,1,d]; k_pages, v_pages:
    [num_pages, page_size, H, d] bf16; block_table: int32 [B, max_pages];
    seqlens_k: int32 [B] -> (o [B,H,1,d], lse [B,H])."""
    _want(q, torch.bfloat16, 4, "q")
    _want(k_pages, torch.bfloat16, 4, "k_pages")
    _want(v_pages, torch.bfloat16, 4, "v_pages")
    _want(block_table, torch.int32, 2, "block_table")
    _want(seqlens_k, torch.int32, 1, "seqlens_k")
    B, H, Lq, d = q.shape
    dev = q.device
    if Lq != 1:
        raise ValueError(f"q: decode takes one query per head, got Lq={Lq}")
    num_pages, page_size = k_pages.shape[0], k_pages.shape[1]
    max_pages = block_table.shape[1]
    Lk = max_pages * page_size
    _want(k_pages, torch.bfloat16, 4, "k_pages", shape=(num_pages, page_size, H, d), device=dev)
    _want(v_pages, torch.bfloat16, 4, "v_pages", shape=(num_pages, page_size, H, d), device=dev)
    _want(block_table, torch.int32, 2, "block_table", shape=(B, max_pages), device=dev)
    _want(seqlens_k, torch.int32, 1, "seqlens_k", shape=(B,), device=dev)
    if o is None:
        o = torch.empty_like(q)
    _want(o, torch.bfloat16, 4, "o", shape=(B, H, 1, d), device=dev)
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=dev)
    _want(lse, torch.float32, 2, "lse", shape=(B, H), device=dev)
    S = num_splits if num_splits > 0 else attn_decode_auto_splits(B, H, Lk, d)
    if workspace is None:
        workspace = torch.empty(attn_decode_workspace_bytes(B, H, Lk, d, S), dtype=torch.uint8, device=dev)
    _want_workspace(workspace, dev)
    scale = (1.0 / d ** 0.5) if scale is None else scale
    _check(lib.attn_decode_paged(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table), max_pages, page_size,
                                 num_pages, _ptr(o), _ptr(lse), _ptr(seqlens_k), B, H, d, scale, S, _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream()), "attn_decode_paged")
    return o, lse


def attn_fp8_ld(Lk) -> int:
    return lib.attn_fp8_ld(Lk)


def attn_quantize_fp8(x, transpose=False, codes=None, descale=None):
    """bf16 [B,H,L,d] -> (e4m3 codes as uint8 [B,H,L,d], or [B,H,d,ld] when
    transposed; fp32 descale [B,H])."""
    _want(x, torch.bfloat16, 4, "x")
    B, H, L, d = x.shape
    dev = x.device
    shape = (B, H, d, attn_fp8_ld(L)) if transpose else (B, H, L, d)
    if codes is None:
        codes = torch.empty(shape, dtype=torch.uint8, device=dev)
    _want(codes, torch.uint8, 4, "codes", shape=shape, device=dev)
    if descale is None:
        descale = torch.empty((B, H), dtype=torch.float32, device=dev)
    _want(descale, torch.float32, 2, "descale", shape=(B, H), device=dev)
    _check(lib.attn_quantize_fp8(_ptr(x), _ptr(codes), _ptr(descale), B, H, L, d, int(bool(transpose)), _stream()),
           "attn_quantize_fp8")
    return codes, descale


def attn_fwd_fp8(q8, k8, vt8, q_descale, k_descale, v_descale, o=None, lse=None, scale=None, causal=False,
                 window_left=-1, window_right=-1, counter=None):
    """FP8 prefill forward.  q8: [B,H,Lq,128], k8: [B,H,Lk,128] and vt8:
    [B,H,128,ld] uint8 e4m3 codes; descales fp32 [B,H] -> (o bf16, lse fp32)."""
    for t, name in ((q8, "q8"), (k8, "k8"), (vt8, "vt8")):
        _want(t, torch.uint8, 4, name)
    for t, name in ((q_descale, "q_descale"), (k_descale, "k_descale"), (v_descale, "v_descale")):
        _want(t, torch.float32, 2, name)
    B, H, Lq, d = q8.shape
    dev = q8.device
    Lk = k8.shape[2]
    _want(k8, torch.uint8, 4, "k8", shape=(B, H, Lk, d), device=dev)
    _want(vt8, torch.uint8, 4, "vt8", shape=(B, H, d, attn_fp8_ld(Lk)), device=dev)
    for t, name in ((q_descale, "q_descale"), (k_descale, "k_descale"), (v_descale, "v_descale")):
        _want(t, torch.float32, 2, name, shape=(B, H), device=dev)
    _want_counter(counter, dev)
    if o is None:
        o = torch.empty((B, H, Lq, d), dtype=torch.bfloat16, device=dev)
    _want(o, torch.bfloat16, 4, "o", shape=(B, H, Lq, d), device=dev)
    if lse is None:
        lse = torch.empty((B, H, Lq), dtype=torch.float32, device=dev)
    _want(lse, torch.float32, 3, "lse", shape=(B, H, Lq), device=dev)
    scale = (1.0 / d ** 0.5) if scale is None else scale
    args = (_ptr(q8), _ptr(k8), _ptr(vt8), _ptr(q_descale), _ptr(k_descale), _ptr(v_descale), _ptr(o), _ptr(lse),
            B, H, Lq, Lk, d, scale, int(bool(causal)), int(window_left), int(window_right))
    if counter is None:
        _check(lib.attn_fwd_fp8(*args, _stream()), "attn_fwd_fp8")
    else:
        _check(lib.attn_fwd_fp8_counted(*args, _ptr(counter), _stream()), "attn_fwd_fp8_counted")
    return o, lse


def attn_bwd_workspace_bytes(B, H, Lq, d) -> int:
    return lib.attn_bwd_workspace_bytes(B, H, Lq, d)


def attn_bwd(q, k, v, o, dout, lse, scale=None, causal=False, window_left=-1, window_right=-1, dq=None, dk=None,
             dv=None, workspace=None, counter=None):
    """Attention backward with recomputation.  q, o, dout: [B,H,Lq,d], k, v:
    [B,H,Lk,d] bf16; lse: fp32 [B,H,Lq] from attn_fwd -> (dq, dk, dv) bf16.
    ``counter`` (optional, a zeroed one-element int64 CUDA tensor) receives the
    number of (key tile, query tile) pairs computed."""
    for t, name in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout")):
        _want(t, torch.bfloat16, 4, name)
    _want(lse, torch.float32, 3, "lse")
    B, H, Lq, d = q.shape
    dev = q.device
    Lk = k.shape[2]
    for t, name, shp in ((k, "k", (B, H, Lk, d)), (v, "v", (B, H, Lk, d)), (o, "o", (B, H, Lq, d)),
                         (dout, "dout", (B, H, Lq, d))):
        _want(t, torch.bfloat16, 4, name, shape=shp, device=dev)
    _want(lse, torch.float32, 3, "lse", shape=(B, H, Lq), device=dev)
    _want_counter(counter, dev)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for t, name, shp in ((dq, "dq", (B, H, Lq, d)), (dk, "dk", (B, H, Lk, d)), (dv, "dv", (B, H, Lk, d))):
        _want(t, torch.bfloat16, 4, name, shape=shp, device=dev)
    if workspace is None:
        workspace = torch.empty(attn_bwd_workspace_bytes(B, H, Lq, d), dtype=torch.uint8, device=dev)
    _want_workspace(workspace, dev)
    scale = (1.0 / d ** 0.5) if scale is None else scale
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv), B, H, Lq, Lk, d,
            scale, int(bool(causal)), int(window_left), int(window_right), _ptr(workspace),
            workspace.numel() * workspace.element_size())
    if counter is None:
        _check(lib.attn_bwd(*args, _stream()), "attn_bwd")
    else:
        _check(lib.attn_bwd_counted(*args, _ptr(counter), _stream()), "attn_bwd_counted")
    return dq, dk, dv


def attn_bwd_count_blocks(Lq, Lk, causal=False, window_left=-1, window_right=-1, block_q=128, block_k=128) -> int:
    """Host-side: (query tile, key tile) pairs the backward visits per head."""
    out = ctypes.c_longlong(0)
    _check(lib.attn_bwd_count_blocks(Lq, Lk, int(bool(causal)), window_left, window_right, block_q, block_k,
                                     ctypes.byref(out)), "attn_bwd_count_blocks")
    return out.value


def attn_count_blocks(Lq, Lk, causal=False, window_left=-1, window_right=-1, block_q=128, block_k=128):
    """Host-side block accounting -> dict(visited, total, partial, pairs)."""
    out = [ctypes.c_longlong(0) for _ in range(4)]
    _check(lib.attn_count_blocks(Lq, Lk, int(bool(causal)), window_left, window_right, block_q, block_k,
                                 *[ctypes.byref(x) for x in out]), "attn_count_blocks")
    return dict(visited=out[0].value, total=out[1].value, partial=out[2].value, pairs=out[3].value)


def fattn_device_status() -> int:
    return lib.fattn_device_status(_stream())


def fattn_debug_inject_stall(on: bool = True) -> None:
    """Test hook: the next prefill launch lets its bounded waits run out."""
    _check(lib.fattn_debug_inject_stall(int(bool(on))), "fattn_debug_inject_stall")


def status_string(status: int) -> str:
    return lib.fattn_status_string(status).decode()
