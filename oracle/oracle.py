"""ctypes front end of the fp64 CPU oracle (``oracle.cpp``).

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU-baseline leg may import this module; the library's product path never does.
It imports nothing from the CUDA package and shares no code with it.

Inputs are numpy arrays (float64, float32, or bfloat16 given as raw uint16
bit patterns) or CPU torch tensors of dtype float64 / float32 / bfloat16; every
element is widened exactly to double inside the oracle.  Outputs are float64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

DT_F64, DT_F32, DT_BF16 = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` next to its source (g++, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["g++", "-O2", "-std=c++17", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            vp, dp, ip, i, d = (ctypes.c_void_p, ctypes.POINTER(ctypes.c_double),
                                ctypes.POINTER(ctypes.c_int), ctypes.c_int, ctypes.c_double)
            llp = ctypes.POINTER(ctypes.c_longlong)
            lib.oracle_attn_naive.argtypes = [vp, vp, vp, i, dp, dp, i, i, i, i, i, d, i, i, i, ip]
            lib.oracle_attn_rows.argtypes = [vp, vp, vp, i, ip, i, dp, dp, i, i, i, i, i, d, i, i, i, ip]
            lib.oracle_attn_probs.argtypes = [vp, vp, i, dp, i, i, i, d, i, i, i]
            lib.oracle_attn_tiled.argtypes = [vp, vp, vp, i, dp, dp, i, i, i, i, i, d, i, i, i, i, i, i, i, llp]
            lib.oracle_decode_splitmerge.argtypes = [vp, vp, vp, i, dp, dp, i, i, i, i, d, ip, i]
            lib.oracle_count_blocks.argtypes = [i, i, i, i, i, i, i, llp, llp, llp, llp]
            lib.oracle_attn_bwd.argtypes = [vp, vp, vp, vp, i, dp, dp, dp, i, i, i, i, i, d, i, i, i]
            u8p = ctypes.POINTER(ctypes.c_uint8)
            fp = ctypes.POINTER(ctypes.c_float)
            ll = ctypes.c_longlong
            lib.oracle_e4m3_decode.argtypes = [u8p, ll, dp]
            lib.oracle_e4m3_encode.argtypes = [dp, ll, u8p]
            lib.oracle_quantize_fp8.argtypes = [vp, i, ll, ll, u8p, fp]
            lib.oracle_attn_fp8.argtypes = [u8p, u8p, u8p, fp, fp, fp, dp, dp, i, i, i, i, i, d, i, i, i, i, i, d]
            lib.oracle_num_threads.restype = ctypes.c_int
            lib.oracle_set_num_threads.argtypes = [i]
            _lib = lib
    return _lib


def _as_array(x):
    """Return (contiguous numpy array, dtype code) without changing any value."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                return x.view(torch.int16).numpy().view(np.uint16), DT_BF16
            if x.dtype == torch.float32:
                return x.numpy(), DT_F32
            if x.dtype == torch.float64:
                return x.numpy(), DT_F64
            raise TypeError(f"oracle: unsupported tensor dtype {x.dtype}")
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    if x.dtype == np.float64:
        return x, DT_F64
    if x.dtype == np.float32:
        return x, DT_F32
    if x.dtype == np.uint16:
        return x, DT_BF16
    raise TypeError(f"oracle: unsupported array dtype {x.dtype}")


def _same_kind(*arrays):
    conv = [_as_array(a) for a in arrays]
    kinds = {c[1] for c in conv}
    if len(kinds) != 1:
        raise TypeError("oracle: q, k and v must share one element type")
    return [c[0] for c in conv], conv[0][1]


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _dptr(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _seqlens(seqlens_k):
    if seqlens_k is None:
        return None, None
    arr = np.ascontiguousarray(np.asarray(seqlens_k, dtype=np.int32))
    return arr, arr.ctypes.data_as(ctypes.POINTER(ctypes.c_int))


def num_threads() -> int:
    return _load().oracle_num_threads()


def set_num_threads(n: int) -> None:
    _load().oracle_set_num_threads(int(n))


def attn(q, k, v, scale, causal=False, window_left=-1, window_right=-1, seqlens_k=None):
    """Exact masked attention of every row.  q: [B,H,Lq,d]; k, v: [B,H,Lk,d].

    Returns (O [B,H,Lq,d] float64, LSE [B,H,Lq] float64)."""
    (qa, ka, va), dt = _same_kind(q, k, v)
    B, H, Lq, d = qa.shape
    Lk = ka.shape[2]
    o = np.empty((B, H, Lq, d), np.float64)
    lse = np.empty((B, H, Lq), np.float64)
    keep, sl = _seqlens(seqlens_k)
    _load().oracle_attn_naive(_ptr(qa), _ptr(ka), _ptr(va), dt, _dptr(o), _dptr(lse),
                              B, H, Lq, Lk, d, float(scale), int(bool(causal)),
                              int(window_left), int(window_right), sl)
    del keep
    return o, lse


def attn_rows(q, k, v, rows, scale, causal=False, window_left=-1, window_right=-1, seqlens_k=None):
    """Exact attention of the listed rows.  rows: int array [n, 3] of (b, h, i).

    Returns (O [n, d] float64, LSE [n] float64)."""
    (qa, ka, va), dt = _same_kind(q, k, v)
    B, H, Lq, d = qa.shape
    Lk = ka.shape[2]
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int32).reshape(-1, 3))
    n = r.shape[0]
    o = np.empty((n, d), np.float64)
    lse = np.empty((n,), np.float64)
    keep, sl = _seqlens(seqlens_k)
    _load().oracle_attn_rows(_ptr(qa), _ptr(ka), _ptr(va), dt,
                             r.ctypes.data_as(ctypes.POINTER(ctypes.c_int)), n,
                             _dptr(o), _dptr(lse), B, H, Lq, Lk, d, float(scale),
                             int(bool(causal)), int(window_left), int(window_right), sl)
    del keep
    return o, lse


def probs(q, k, scale, causal=False, window_left=-1, window_right=-1):
    """Softmax probability matrix of one head.  q: [Lq, d], k: [Lk, d] -> P [Lq, Lk]."""
    (qa, ka), dt = _same_kind(q, k)
    Lq, d = qa.shape
    Lk = ka.shape[0]
    P = np.empty((Lq, Lk), np.float64)
    _load().oracle_attn_probs(_ptr(qa), _ptr(ka), dt, _dptr(P), Lq, Lk, d, float(scale),
                              int(bool(causal)), int(window_left), int(window_right))
    return P


def attn_tiled(q, k, v, scale, causal=False, window_left=-1, window_right=-1,
               block_q=64, block_k=64, skip=True, nan_guard=True):
    """The tiled online-softmax recurrence (with block skip / break).

    Returns (O, LSE, visited_block_pairs)."""
    (qa, ka, va), dt = _same_kind(q, k, v)
    B, H, Lq, d = qa.shape
    Lk = ka.shape[2]
    o = np.empty((B, H, Lq, d), np.float64)
    lse = np.empty((B, H, Lq), np.float64)
    visited = ctypes.c_longlong(0)
    _load().oracle_attn_tiled(_ptr(qa), _ptr(ka), _ptr(va), dt, _dptr(o), _dptr(lse),
                              B, H, Lq, Lk, d, float(scale), int(bool(causal)),
                              int(window_left), int(window_right), int(block_q), int(block_k),
                              int(bool(skip)), int(bool(nan_guard)), ctypes.byref(visited))
    return o, lse, visited.value


def decode_splitmerge(q, k, v, scale, num_splits, seqlens_k=None):
    """Split-KV decode by exact partials and the LSE merge.  q: [B,H,1,d].

    Returns (O [B,H,1,d] float64, LSE [B,H] float64)."""
    (qa, ka, va), dt = _same_kind(q, k, v)
    B, H, one, d = qa.shape
    assert one == 1
    Lk = ka.shape[2]
    o = np.empty((B, H, 1, d), np.float64)
    lse = np.empty((B, H), np.float64)
    keep, sl = _seqlens(seqlens_k)
    _load().oracle_decode_splitmerge(_ptr(qa), _ptr(ka), _ptr(va), dt, _dptr(o), _dptr(lse),
                                     B, H, Lk, d, float(scale), sl, int(num_splits))
    del keep
    return o, lse


def attn_bwd(q, k, v, do, scale, causal=False, window_left=-1, window_right=-1):
    """Gradients (dQ, dK, dV) of L = sum(dO * O) for exact masked attention,
    fp64.  q, do: [B,H,Lq,d]; k, v: [B,H,Lk,d]."""
    (qa, ka, va, da), dt = _same_kind(q, k, v, do)
    B, H, Lq, d = qa.shape
    Lk = ka.shape[2]
    dq = np.empty((B, H, Lq, d), np.float64)
    dk = np.empty((B, H, Lk, d), np.float64)
    dv = np.empty((B, H, Lk, d), np.float64)
    _load().oracle_attn_bwd(_ptr(qa), _ptr(ka), _ptr(va), _ptr(da), dt, _dptr(dq), _dptr(dk), _dptr(dv),
                            B, H, Lq, Lk, d, float(scale), int(bool(causal)), int(window_left),
                            int(window_right))
    return dq, dk, dv


def _u8(a):
    a = np.ascontiguousarray(a, dtype=np.uint8)
    return a, a.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8))


def _f32(a):
    a = np.ascontiguousarray(a, dtype=np.float32)
    return a, a.ctypes.data_as(ctypes.POINTER(ctypes.c_float))


def e4m3_decode(codes):
    """Values (float64) of e4m3 codes (uint8 array)."""
    c, cp = _u8(codes)
    out = np.empty(c.shape, np.float64)
    _load().oracle_e4m3_decode(cp, c.size, _dptr(out))
    return out


def e4m3_encode(x):
    """Nearest e4m3 codes (ties to even, saturating at 448) of float64 values."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, np.uint8)
    _load().oracle_e4m3_encode(_dptr(x), x.size, out.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)))
    return out


def quantize_fp8(x):
    """Per-(b,h) FP8 quantization of x [B,H,L,d] -> (codes uint8 [B,H,L,d],
    descale float32 [B,H])."""
    xa, dt = _as_array(x)
    B, H, L, d = xa.shape
    codes = np.empty((B, H, L, d), np.uint8)
    desc = np.empty((B, H), np.float32)
    _load().oracle_quantize_fp8(_ptr(xa), dt, B * H, L * d, codes.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)),
                                desc.ctypes.data_as(ctypes.POINTER(ctypes.c_float)))
    return codes, desc


# Reading R13: the FP8 recurrence keeps a reference max that moves only when a
# tile's max passes it by more than FP8_SLACK (log2 units), and rounds
# p = 2^(x - m + 8 - FP8_SLACK) <= 2^8 to e4m3.
FP8_SLACK = 4.0


def attn_fp8(q8, k8, v8, qd, kd, vd, scale, causal=False, window_left=-1, window_right=-1, block_k=128,
             quantize_p=True, slack=FP8_SLACK):
    """FP8 forward by its steps (e4m3 codes [B,H,L,d], per-(b,h) descales) ->
    (O [B,H,Lq,d] float64, LSE [B,H,Lq] float64).  ``slack`` = 0 takes the exact
    running max."""
    (q8, qp), (k8, kp), (v8, vp) = _u8(q8), _u8(k8), _u8(v8)
    (qd, qdp), (kd, kdp), (vd, vdp) = _f32(qd), _f32(kd), _f32(vd)
    B, H, Lq, d = q8.shape
    Lk = k8.shape[2]
    o = np.empty((B, H, Lq, d), np.float64)
    lse = np.empty((B, H, Lq), np.float64)
    _load().oracle_attn_fp8(qp, kp, vp, qdp, kdp, vdp, _dptr(o), _dptr(lse), B, H, Lq, Lk, d, float(scale),
                            int(bool(causal)), int(window_left), int(window_right), int(block_k),
                            int(bool(quantize_p)), float(slack))
    return o, lse


def count_blocks(Lq, Lk, causal, window_left, window_right, block_q, block_k):
    """Brute-force mask enumeration -> dict(pairs, visited, total, partial)."""
    out = [ctypes.c_longlong(0) for _ in range(4)]
    _load().oracle_count_blocks(int(Lq), int(Lk), int(bool(causal)), int(window_left),
                                int(window_right), int(block_q), int(block_k),
                                *[ctypes.byref(x) for x in out])
    return dict(pairs=out[0].value, visited=out[1].value, total=out[2].value, partial=out[3].value)
