"""Packed variable-length prefill (attn_fwd_varlen) against the fp64 oracle.

Each sequence of the packed batch is cut out and given to the dense oracle
([1, H, L, d]); the GPU computes the whole batch in one launch."""
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


def _check_varlen(fl, oracle, lens_q, lens_k, H, d, causal, wl, wr, seed, max_q=None):
    q, k, v, cu_q, cu_k = synth.make_varlen_inputs(lens_q, lens_k, H, d, seed)
    counter = torch.zeros(1, dtype=torch.int64, device="cuda")
    o, lse = fl.attn_fwd_varlen(q.cuda(), k.cuda(), v.cuda(), cu_q.cuda(), cu_k.cuda(), max_q or max(lens_q),
                                causal=causal, window_left=wl, window_right=wr, counter=counter)
    torch.cuda.synchronize()
    o, lse = o.float().cpu().numpy(), lse.cpu().numpy()
    scale = d ** -0.5
    want_tiles = 0
    for b in range(len(lens_q)):
        qs, qe = int(cu_q[b]), int(cu_q[b + 1])
        ks, ke = int(cu_k[b]), int(cu_k[b + 1])
        if qe == qs:
            continue
        # re-layout [L, H, d] -> [1, H, L, d] for the dense oracle
        qb = q[qs:qe].permute(1, 0, 2).unsqueeze(0).contiguous()
        kb = k[ks:ke].permute(1, 0, 2).unsqueeze(0).contiguous()
        vb = v[ks:ke].permute(1, 0, 2).unsqueeze(0).contiguous()
        if ke == ks:
            o_ref = np.zeros((1, H, qe - qs, d))
            lse_ref = np.full((1, H, qe - qs), -np.inf)
        else:
            o_ref, lse_ref = oracle.attn(qb, kb, vb, scale, causal, wl, wr)
            want_tiles += fl.attn_count_blocks(qe - qs, ke - ks, causal, wl, wr, 128, 128)["visited"] * H
        got_o = np.transpose(o[qs:qe], (1, 0, 2))[None]
        got_l = lse[:, qs:qe][None]
        compare(got_o, got_l, o_ref, lse_ref, BF16_O_MAXABS, BF16_O_RELL2, label=f"seq {b} ({qe - qs}x{ke - ks})")
    assert int(counter.item()) == want_tiles


@pytest.mark.parametrize("causal,wl,wr", [(True, -1, -1), (False, -1, -1), (False, 100, 100), (True, 300, 0)])
def test_varlen_mixed_lengths(fl, oracle, causal, wl, wr):
    lens = [1, 127, 128, 129, 300, 1000, 37, 700]
    _check_varlen(fl, oracle, lens, lens, 3, 128, causal, wl, wr, seed=31)


def test_varlen_query_shorter_than_keys(fl, oracle):
    # chunked-prefill shape: new query tokens attend to a longer history (bottom-right)
    _check_varlen(fl, oracle, [64, 200, 1, 300], [500, 200, 90, 1000], 2, 128, True, -1, -1, seed=32)


def test_varlen_head_dim_64_and_empty_sequences(fl, oracle):
    _check_varlen(fl, oracle, [250, 0, 513, 7], [250, 0, 513, 7], 4, 64, True, -1, -1, seed=33)


def test_varlen_large_mix(fl, oracle):
    lens = synth.varlen_lengths(12, 256, 3000, seed=34)
    _check_varlen(fl, oracle, lens, lens, 4, 128, True, -1, -1, seed=35)


def test_varlen_max_seqlen_above_every_length(fl, oracle):
    # pair indices no sequence reaches: the compacted work order skips them
    lens = [900, 130, 0, 2000, 256, 257]
    _check_varlen(fl, oracle, lens, lens, 2, 128, True, -1, -1, seed=36, max_q=5000)


@pytest.mark.parametrize("n_short", [2045, 2046])
def test_varlen_many_sequences(fl, oracle, n_short):
    # 2048 sequences take the compacted work order built in shared memory;
    # 2049 exceed its table and take the dense order.  Both must give the
    # same per-sequence results; a few long sequences give several pair indices.
    g = np.random.default_rng(37)
    lens = [int(x) for x in g.integers(0, 100, n_short)] + [1500, 777, 2100]
    g.shuffle(lens)
    _check_varlen(fl, oracle, lens, lens, 1, 64, True, -1, -1, seed=38)


def test_varlen_concurrent_streams(fl):
    # launches in flight together on two streams draw different work counters
    # and give the same bits as when run one at a time
    lens_a = synth.varlen_lengths(9, 100, 1500, seed=41)
    lens_b = synth.varlen_lengths(13, 50, 900, seed=42)
    ins = []
    for lens, seed in ((lens_a, 43), (lens_b, 44)):
        q, k, v, cq, ck = synth.make_varlen_inputs(lens, lens, 4, 128, seed)
        ins.append((q.cuda(), k.cuda(), v.cuda(), cq.cuda(), ck.cuda(), max(lens)))
    refs = []
    for q, k, v, cq, ck, m in ins:
        o, lse = fl.attn_fwd_varlen(q, k, v, cq, ck, m, causal=True)
        torch.cuda.synchronize()
        refs.append((o.clone(), lse.clone()))
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = []
    for it in range(6):
        for (q, k, v, cq, ck, m), s in zip(ins, streams):
            with torch.cuda.stream(s):
                outs.append(fl.attn_fwd_varlen(q, k, v, cq, ck, m, causal=True))
    torch.cuda.synchronize()
    for n, (o, lse) in enumerate(outs):
        assert torch.equal(o, refs[n % 2][0]) and torch.equal(lse, refs[n % 2][1]), f"launch {n}"
