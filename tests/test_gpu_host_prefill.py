"""attn_fwd_host: the prefill on host buffers, its copies overlapped with the
kernels in chunks of heads.  Each head is an independent problem, so the
results must equal attn_fwd's on the same data bit for bit, whatever the
chunking; one small case is also checked against the fp64 oracle."""
import numpy as np
import pytest
import torch

from io_aware_exact_34_b200 import synth
from tests._compare import BF16_O_MAXABS, BF16_O_RELL2, compare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fl():
    from io_aware_exact_34_b200 import build
    build.build()
    from io_aware_exact_34_b200 import fattn
    return fattn


def _device_reference(fl, q, k, v, **kw):
    o, lse = fl.attn_fwd(q.cuda(), k.cuda(), v.cuda(), **kw)
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu()


@pytest.mark.parametrize("B,H,Lq,Lk,d,causal,wl,wr,pinned", [
    (1, 2, 300, 300, 128, True, -1, -1, True),      # one chunk
    (4, 16, 4096, 4096, 128, True, -1, -1, True),   # the causal_4k shape: several chunks, ragged last one
    (3, 5, 1000, 1500, 64, False, 200, 100, True),  # d = 64, window, Lq != Lk
    (2, 7, 2500, 2500, 128, True, -1, -1, False),   # pageable host memory: copies serialised, same results
])
def test_host_prefill_matches_device_prefill(fl, B, H, Lq, Lk, d, causal, wl, wr, pinned):
    q, k, v = synth.random_qkv(B, H, Lq, Lk, d, "bf16", seed=B * 100 + H)
    if pinned:
        q, k, v = q.pin_memory(), k.pin_memory(), v.pin_memory()
    o, lse = fl.attn_fwd_host(q, k, v, causal=causal, window_left=wl, window_right=wr)
    o_ref, lse_ref = _device_reference(fl, q, k, v, causal=causal, window_left=wl, window_right=wr)
    assert torch.equal(o, o_ref)
    assert torch.equal(lse, lse_ref)


def test_host_prefill_without_lse_and_caller_workspace(fl):
    B, H, L, d = 2, 24, 2048, 128
    q, k, v = (t.pin_memory() for t in synth.random_qkv(B, H, L, L, d, "bf16", seed=5))
    ws = torch.empty(fl.attn_fwd_host_workspace_bytes(B, H, L, L, d), dtype=torch.uint8, device="cuda")
    o = torch.full((B, H, L, d), float("nan"), dtype=torch.bfloat16).pin_memory()
    o2, lse = fl.attn_fwd_host(q, k, v, o=o, causal=True, need_lse=False, workspace=ws)
    assert lse is None and o2 is o
    o_ref, _ = _device_reference(fl, q, k, v, causal=True)
    assert torch.equal(o, o_ref)
    # the same workspace again, back to back
    o3, _ = fl.attn_fwd_host(q, k, v, causal=True, need_lse=False, workspace=ws)
    assert torch.equal(o3, o_ref)


def test_host_prefill_against_oracle(fl, oracle):
    q, k, v = synth.random_qkv(2, 3, 257, 257, 128, "bf16", seed=9)
    o, lse = fl.attn_fwd_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), causal=True)
    o_ref, lse_ref = oracle.attn(q, k, v, 128 ** -0.5, True)
    compare(o.float().numpy(), lse.numpy(), o_ref, lse_ref, BF16_O_MAXABS, BF16_O_RELL2, label="host prefill")


def test_host_prefill_rejects_device_tensors(fl):
    q = torch.zeros(1, 1, 8, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError, match="host tensor"):
        fl.attn_fwd_host(q, q, q)


def test_host_prefill_from_two_threads(fl):
    # the library serialises the threads' enqueues on its own streams; each
    # thread gets its own results
    import threading
    cases = [synth.random_qkv(1, 6, 700, 700, 128, "bf16", seed=s) for s in (11, 12)]
    cases = [tuple(t.pin_memory() for t in c) for c in cases]
    refs = [_device_reference(fl, *c, causal=True) for c in cases]
    dev = torch.cuda.current_device()
    results = [None, None]
    errors = []

    def work(n):
        try:
            torch.cuda.set_device(dev)
            for _ in range(3):
                results[n] = fl.attn_fwd_host(*cases[n], causal=True)
                assert torch.equal(results[n][0], refs[n][0]) and torch.equal(results[n][1], refs[n][1])
        except Exception as e:  # reported in the main thread
            errors.append(e)

    threads = [threading.Thread(target=work, args=(n,)) for n in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=120)
    assert not errors, errors
    assert all(r is not None for r in results)
