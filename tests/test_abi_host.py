"""Host-side tests of the C ABI: the library loads without a GPU, exports
every function ``include/fattn.h`` declares, rejects bad arguments before any
CUDA call, and its tile scheduler matches brute-force mask enumeration."""
import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def fl():
    from io_aware_exact_34_b200 import build
    build.build()
    from io_aware_exact_34_b200 import fattn
    return fattn


def _declared_functions():
    with open(os.path.join(ROOT, "include", "fattn.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_\s\*]*?\b([A-Za-z_][A-Za-z0-9_]*)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if n not in ("defined",)))


def test_header_symbols_are_exported(fl):
    names = _declared_functions()
    assert {"attn_fwd", "attn_fwd_f32", "attn_decode_splitkv", "attn_count_blocks"} <= set(names)
    lib = ctypes.CDLL(fl._LIB_PATH)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in fattn.h but not exported"


def test_status_strings(fl):
    for code in range(-7, 1):
        assert fl.status_string(code).startswith("FATTN_")
    assert "unknown" in fl.status_string(123)


FAKE = 0x10000  # never dereferenced: every call below fails validation first


def _fwd(fl, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=None, B=1, H=1, Lq=8, Lk=8, d=128, scale=0.1,
         causal=0, wl=-1, wr=-1, fn="attn_fwd"):
    return getattr(fl.lib, fn)(q, k, v, o, lse, B, H, Lq, Lk, d, scale, causal, wl, wr, None)


@pytest.mark.parametrize("fn", ["attn_fwd", "attn_fwd_f32"])
def test_prefill_argument_checks(fl, fn):
    assert _fwd(fl, q=None, fn=fn) == fl.FATTN_ERR_INVALID_ARG
    assert _fwd(fl, o=None, fn=fn) == fl.FATTN_ERR_INVALID_ARG
    assert _fwd(fl, B=0, fn=fn) == fl.FATTN_ERR_INVALID_ARG
    assert _fwd(fl, Lq=0, fn=fn) == fl.FATTN_ERR_INVALID_ARG
    assert _fwd(fl, Lk=-3, fn=fn) == fl.FATTN_ERR_INVALID_ARG
    assert _fwd(fl, scale=0.0, fn=fn) == fl.FATTN_ERR_INVALID_ARG
    assert _fwd(fl, scale=-1.0, fn=fn) == fl.FATTN_ERR_INVALID_ARG
    assert _fwd(fl, scale=float("inf"), fn=fn) == fl.FATTN_ERR_INVALID_ARG
    assert _fwd(fl, scale=float("nan"), fn=fn) == fl.FATTN_ERR_INVALID_ARG
    assert _fwd(fl, d=96, fn=fn) == fl.FATTN_ERR_UNSUPPORTED
    assert _fwd(fl, d=256, fn=fn) == fl.FATTN_ERR_UNSUPPORTED
    assert _fwd(fl, q=FAKE + 8, fn=fn) == fl.FATTN_ERR_MISALIGNED
    assert _fwd(fl, o=FAKE + 2, fn=fn) == fl.FATTN_ERR_MISALIGNED
    assert _fwd(fl, lse=FAKE + 2, fn=fn) == fl.FATTN_ERR_MISALIGNED


def test_counted_needs_counter(fl):
    r = fl.lib.attn_fwd_counted(FAKE, FAKE, FAKE, FAKE, None, 1, 1, 8, 8, 128, 0.1, 0, -1, -1, None, None)
    assert r == fl.FATTN_ERR_INVALID_ARG
    r = fl.lib.attn_fwd_counted(FAKE, FAKE, FAKE, FAKE, None, 1, 1, 8, 8, 128, 0.1, 0, -1, -1, FAKE + 4, None)
    assert r == fl.FATTN_ERR_MISALIGNED


def _dec(fl, q=FAKE, k=FAKE, v=FAKE, o=FAKE, B=2, H=2, Lk=64, d=128, S=4, ws=FAKE, ws_bytes=1 << 20,
         scale=0.1, seqlens=None):
    return fl.lib.attn_decode_splitkv(q, k, v, o, None, seqlens, B, H, Lk, d, scale, S, ws, ws_bytes, None)


def test_decode_argument_checks(fl):
    need = fl.attn_decode_workspace_bytes(2, 2, 64, 128, 4)
    assert need == 2 * 2 * 4 * 129 * 4
    assert _dec(fl, k=None) == fl.FATTN_ERR_INVALID_ARG
    assert _dec(fl, S=-1) == fl.FATTN_ERR_INVALID_ARG
    assert _dec(fl, S=65) == fl.FATTN_ERR_INVALID_ARG            # more splits than keys
    assert _dec(fl, d=80) == fl.FATTN_ERR_UNSUPPORTED
    assert _dec(fl, v=FAKE + 4) == fl.FATTN_ERR_MISALIGNED
    assert _dec(fl, seqlens=FAKE + 2) == fl.FATTN_ERR_MISALIGNED
    assert _dec(fl, ws=None) == fl.FATTN_ERR_WORKSPACE
    assert _dec(fl, ws_bytes=need - 1) == fl.FATTN_ERR_WORKSPACE
    assert _dec(fl, ws=FAKE + 4, ws_bytes=need) == fl.FATTN_ERR_MISALIGNED
    assert fl.attn_decode_workspace_bytes(0, 1, 1, 128, 1) == 0


def test_auto_splits(fl):
    assert fl.attn_decode_auto_splits(64, 32, 32768, 128) == 32
    assert fl.attn_decode_auto_splits(1, 1, 100, 128) == 1
    assert fl.attn_decode_auto_splits(1, 1, 1 << 20, 64) == 64
    assert fl.attn_decode_workspace_bytes(64, 32, 32768, 128, 0) == 64 * 32 * 32 * 129 * 4


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU path")
def test_valid_call_without_gpu_reports_no_device(fl):
    assert _fwd(fl) == fl.FATTN_ERR_NO_DEVICE
    assert _fwd(fl, fn="attn_fwd_f32", d=64) == fl.FATTN_ERR_NO_DEVICE
    need = fl.attn_decode_workspace_bytes(2, 2, 64, 128, 4)
    assert _dec(fl, ws_bytes=need) == fl.FATTN_ERR_NO_DEVICE


SCHED_CASES = [
    # (Lq, Lk, causal, wl, wr, bq, bk)
    (4096, 4096, True, -1, -1, 128, 128),
    (300, 300, True, -1, -1, 128, 128),
    (1000, 1000, False, 100, 100, 128, 128),
    (1000, 1000, True, 257, 0, 128, 128),
    (777, 777, False, 0, 0, 128, 128),
    (640, 640, False, 130, 7, 128, 128),
    (129, 300, True, -1, -1, 128, 128),    # Lq < Lk (bottom-right)
    (300, 129, True, -1, -1, 128, 128),    # Lq > Lk: leading rows without keys
    (300, 129, False, 5, 3, 128, 128),
    (1, 1000, False, -1, -1, 128, 128),
    (1000, 1, True, -1, -1, 128, 128),
    (256, 256, False, -1, -1, 64, 64),
    (257, 333, True, 40, 0, 32, 64),
    (513, 513, False, 64, 64, 64, 128),
]


@pytest.mark.parametrize("Lq,Lk,causal,wl,wr,bq,bk", SCHED_CASES)
def test_scheduler_matches_bruteforce(fl, oracle, Lq, Lk, causal, wl, wr, bq, bk):
    """The library's closed-form KV tile ranges (§5.4, §7.3) visit exactly the
    tiles that hold an allowed pair; partial tiles and pair counts agree with
    the oracle's brute-force enumeration."""
    got = fl.attn_count_blocks(Lq, Lk, causal, wl, wr, bq, bk)
    want = oracle.count_blocks(Lq, Lk, causal, wl, wr, bq, bk)
    assert got == want


def test_scheduler_page_example(fl):
    """n = 32768, w = 2048, B = 128 (sliding-window page §5.4): 8176 of 65536."""
    c = fl.attn_count_blocks(32768, 32768, False, 2048, 2048, 128, 128)
    assert (c["visited"], c["total"], c["partial"]) == (8176, 65536, 480)
    c = fl.attn_count_blocks(32768, 32768, True, 4096, 0, 128, 128)
    assert (c["visited"], c["partial"]) == (7920, 480)
    c = fl.attn_count_blocks(4096, 4096, True, -1, -1, 128, 128)
    assert (c["visited"], c["partial"]) == (528, 32)
    c = fl.attn_count_blocks(65536, 65536, True, -1, -1, 128, 128)
    assert (c["visited"], c["partial"]) == (131328, 512)


def test_varlen_argument_checks(fl):
    f = fl.lib.attn_fwd_varlen
    args = lambda **kw: dict(dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=None, cq=FAKE, ck=FAKE, n=2, H=2, tq=100,
                                  tk=100, mx=64, d=128, scale=0.1), **kw)
    def call(**kw):
        a = args(**kw)
        return f(a["q"], a["k"], a["v"], a["o"], a["lse"], a["cq"], a["ck"], a["n"], a["H"], a["tq"], a["tk"], a["mx"],
                 a["d"], a["scale"], 1, -1, -1, None)
    assert call(cq=None) == fl.FATTN_ERR_INVALID_ARG
    assert call(n=0) == fl.FATTN_ERR_INVALID_ARG
    assert call(mx=0) == fl.FATTN_ERR_INVALID_ARG
    assert call(tq=0) == fl.FATTN_ERR_INVALID_ARG
    assert call(d=80) == fl.FATTN_ERR_UNSUPPORTED
    assert call(ck=FAKE + 2) == fl.FATTN_ERR_MISALIGNED
    assert call(k=FAKE + 8) == fl.FATTN_ERR_MISALIGNED


def test_paged_decode_argument_checks(fl):
    def call(page=16, table=FAKE, sl=FAKE, ws=FAKE, ws_bytes=1 << 20, d=128, S=1):
        return fl.lib.attn_decode_paged(FAKE, FAKE, FAKE, table, 4, page, 4, FAKE, None, sl, 1, 1, d, 0.1, S, ws,
                                        ws_bytes, None)
    assert call(page=24) == fl.FATTN_ERR_INVALID_ARG      # not a power of two
    assert call(page=8) == fl.FATTN_ERR_INVALID_ARG       # below 16
    assert call(table=None) == fl.FATTN_ERR_INVALID_ARG
    assert call(sl=None) == fl.FATTN_ERR_INVALID_ARG      # lengths are required
    assert call(d=96) == fl.FATTN_ERR_UNSUPPORTED
    assert call(table=FAKE + 2) == fl.FATTN_ERR_MISALIGNED
    assert call(ws=None) == fl.FATTN_ERR_WORKSPACE


def _bwd(fl, q=FAKE, k=FAKE, v=FAKE, o=FAKE, do=FAKE, lse=FAKE, dq=FAKE, dk=FAKE, dv=FAKE, B=1, H=2, Lq=300, Lk=260,
         d=128, scale=0.1, ws=FAKE, ws_bytes=None):
    if ws_bytes is None:
        ws_bytes = fl.attn_bwd_workspace_bytes(B, H, Lq, d) if B > 0 and Lq > 0 else 0
    return fl.lib.attn_bwd(q, k, v, o, do, lse, dq, dk, dv, B, H, Lq, Lk, d, scale, 1, -1, -1, ws, ws_bytes, None)


def test_bwd_argument_checks(fl):
    need = fl.attn_bwd_workspace_bytes(1, 2, 300, 128)
    assert need == 1 * 2 * 384 * 130 * 4
    assert fl.attn_bwd_workspace_bytes(1, 1, 1, 96) == 0
    assert _bwd(fl, lse=None) == fl.FATTN_ERR_INVALID_ARG
    assert _bwd(fl, do=None) == fl.FATTN_ERR_INVALID_ARG
    assert _bwd(fl, dq=None) == fl.FATTN_ERR_INVALID_ARG
    assert _bwd(fl, dk=None) == fl.FATTN_ERR_INVALID_ARG
    assert _bwd(fl, o=None) == fl.FATTN_ERR_INVALID_ARG
    assert _bwd(fl, B=0) == fl.FATTN_ERR_INVALID_ARG
    assert _bwd(fl, scale=0.0) == fl.FATTN_ERR_INVALID_ARG
    assert _bwd(fl, d=96, ws_bytes=1 << 30) == fl.FATTN_ERR_UNSUPPORTED
    assert _bwd(fl, do=FAKE + 8) == fl.FATTN_ERR_MISALIGNED
    assert _bwd(fl, dv=FAKE + 2) == fl.FATTN_ERR_MISALIGNED
    assert _bwd(fl, lse=FAKE + 2) == fl.FATTN_ERR_MISALIGNED
    assert _bwd(fl, ws=None) == fl.FATTN_ERR_WORKSPACE
    assert _bwd(fl, ws_bytes=need - 1) == fl.FATTN_ERR_WORKSPACE
    assert _bwd(fl, ws=FAKE + 4) == fl.FATTN_ERR_MISALIGNED
    r = fl.lib.attn_bwd_counted(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 300, 260, 128, 0.1, 1, -1,
                                -1, FAKE, need, None, None)
    assert r == fl.FATTN_ERR_INVALID_ARG


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU path")
def test_bwd_valid_call_without_gpu_reports_no_device(fl):
    assert _bwd(fl) == fl.FATTN_ERR_NO_DEVICE


@pytest.mark.parametrize("Lq,Lk,causal,wl,wr,bq,bk", SCHED_CASES)
def test_bwd_scheduler_matches_bruteforce(fl, oracle, Lq, Lk, causal, wl, wr, bq, bk):
    """Walking the query tiles of each key tile (the backward's order) visits
    exactly the tiles with an allowed pair: the oracle's brute-force count."""
    got = fl.attn_bwd_count_blocks(Lq, Lk, causal, wl, wr, bq, bk)
    assert got == oracle.count_blocks(Lq, Lk, causal, wl, wr, bq, bk)["visited"]


def test_fp8_argument_checks(fl):
    def fwd(d=128, qd=FAKE, kd=FAKE, vd=FAKE, q=FAKE, Lk=300):
        return fl.lib.attn_fwd_fp8(q, FAKE, FAKE, qd, kd, vd, FAKE, None, 1, 2, 300, Lk, d, 0.1, 1, -1, -1, None)
    assert fwd(d=64) == fl.FATTN_ERR_UNSUPPORTED
    assert fwd(qd=None) == fl.FATTN_ERR_INVALID_ARG
    assert fwd(vd=FAKE + 2) == fl.FATTN_ERR_MISALIGNED
    assert fwd(q=FAKE + 8) == fl.FATTN_ERR_MISALIGNED
    assert fwd(Lk=0) == fl.FATTN_ERR_INVALID_ARG
    assert [fl.attn_fp8_ld(n) for n in (1, 16, 17, 300, 4096, 0)] == [16, 16, 32, 304, 4096, 0]
    q = fl.lib.attn_quantize_fp8
    assert q(FAKE, FAKE, FAKE, 1, 1, 10, 96, 0, None) == fl.FATTN_ERR_UNSUPPORTED
    assert q(None, FAKE, FAKE, 1, 1, 10, 128, 0, None) == fl.FATTN_ERR_INVALID_ARG
    assert q(FAKE, FAKE, FAKE + 2, 1, 1, 10, 128, 0, None) == fl.FATTN_ERR_MISALIGNED
    assert q(FAKE, FAKE, FAKE, 1, 70000, 10, 128, 0, None) == fl.FATTN_ERR_UNSUPPORTED
    if not torch.cuda.is_available():
        assert fwd() == fl.FATTN_ERR_NO_DEVICE
        assert q(FAKE, FAKE, FAKE, 1, 1, 10, 128, 1, None) == fl.FATTN_ERR_NO_DEVICE


def test_host_prefill_argument_checks(fl):
    lib = fl.lib
    ws_need = fl.attn_fwd_host_workspace_bytes(2, 3, 300, 300, 128)
    assert ws_need > 0
    # invalid sizes give no workspace size
    assert fl.attn_fwd_host_workspace_bytes(2, 3, 300, 300, 96) == 0
    assert fl.attn_fwd_host_workspace_bytes(0, 3, 300, 300, 128) == 0
    # two chunk buffers, each holding at least one head's Q, K, V, O and LSE
    per_head = (300 * 128 * 2) * 4 + 300 * 4
    assert ws_need >= 2 * per_head
    # more heads never need less workspace; the chunk size is capped, so many heads need no more than a few
    assert fl.attn_fwd_host_workspace_bytes(64, 16, 4096, 4096, 128) >= fl.attn_fwd_host_workspace_bytes(1, 1, 4096, 4096, 128)
    assert fl.attn_fwd_host_workspace_bytes(64, 16, 4096, 4096, 128) == fl.attn_fwd_host_workspace_bytes(128, 16, 4096, 4096, 128)

    def call(q=FAKE, k=FAKE, v=FAKE, o=FAKE, d=128, scale=0.1, ws=FAKE * 16, ws_bytes=None):
        return lib.attn_fwd_host(q, k, v, o, None, 2, 3, 300, 300, d, scale, 1, -1, -1, ws,
                                 ws_need if ws_bytes is None else ws_bytes, None)

    assert call(q=None) == fl.FATTN_ERR_INVALID_ARG
    assert call(o=None) == fl.FATTN_ERR_INVALID_ARG
    assert call(scale=0.0) == fl.FATTN_ERR_INVALID_ARG
    assert call(d=96) == fl.FATTN_ERR_UNSUPPORTED
    assert call(ws=None) == fl.FATTN_ERR_WORKSPACE
    assert call(ws=FAKE * 16 + 16) == fl.FATTN_ERR_WORKSPACE  # not 256-byte aligned
    assert call(ws_bytes=ws_need - 1) == fl.FATTN_ERR_WORKSPACE
