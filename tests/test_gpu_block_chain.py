"""Chains of residual blocks with the next block's first RMS_norm + SiLU moved
into the previous block's conv2 epilogue ("Cosmos3 Wan VAE", §10.4: in a
stage of residual blocks, block k+1 begins with SiLU(RMS_norm(y_k))).

Block k's conv2 writes y_k and, from the same accumulator row, a0_{k+1} =
SiLU(RMS_norm(bf16(y_k); g1 of block k+1)); block k+1 takes a0_{k+1} and
skips its own first norm.  Checked against the fp64 oracle block by block
(each block's oracle input is the chain's own bf16 y_{k-1}), against the
unfused chain, and chunk-streamed against the whole sequence."""
import pytest
import torch

import oracle
from tests.parity import assert_close_bf16, ncthw_np, to_dev
from tests.test_gpu_block_sc import _block, _oracle_args, block_sc_case
from video_vae_causal_implicit_b200 import cc3d, synth

pytestmark = pytest.mark.gpu


def _chain_cases(spec, n, t, h, w, seed):
    return [block_sc_case(ci, co, t, h, w, n=n, seed=seed + 100 * i, shortcut=ci != co)
            for i, (ci, co) in enumerate(spec)]


def _empty(n, t, h, w, c):
    return torch.empty((n, t, h, w, c), dtype=torch.bfloat16, device="cuda")


def _run_fused(blocks, x, n, t, h, w, c1_out=None, c2_out=None):
    """The chain with the fused hand-over; returns the y's and a0's.
    c1_out / c2_out: per-block cache outputs (or None)."""
    ys, a0s = [], [None]
    xin, a_in = x, None
    for i, b in enumerate(blocks):
        nxt = blocks[i + 1] if i + 1 < len(blocks) else None
        y = _empty(n, t, h, w, b.c_out)
        a_next = _empty(n, t, h, w, b.c_out) if nxt else None
        b.forward(xin, y, a0_in=a_in, g_next=nxt.g1 if nxt else None, a0_next=a_next,
                  cache1_out=c1_out[i] if c1_out else None,
                  cache2_out=c2_out[i] if c2_out else None)
        ys.append(y)
        a0s.append(a_next)
        xin, a_in = y, a_next
    return ys, a0s


CHAINS = [
    # (n, t, h, w, [(c_in, c_out), ...]): a shortcut block then two identity
    # blocks at 192 channels; a batch of two 64-channel blocks; 384-channel
    # blocks, which hand over through a norm pass after conv2
    (1, 3, 20, 24, [(96, 192), (192, 192), (192, 192)]),
    (2, 2, 16, 20, [(64, 64), (64, 64)]),
    (1, 2, 12, 16, [(192, 384), (384, 384)]),
]


@pytest.mark.parametrize("n,t,h,w,spec", CHAINS)
def test_fused_chain_matches_oracle(n, t, h, w, spec):
    cases = _chain_cases(spec, n, t, h, w, seed=7 * spec[0][1])
    blocks = [_block(c, n, h, w, t) for c in cases]
    x = to_dev(synth.ndhwc(cases[0]["x"]))
    ys, a0s = _run_fused(blocks, x, n, t, h, w)
    # the unfused chain: every block runs its own first norm
    yu, xin = [], x
    for b in blocks:
        y = _empty(n, t, h, w, b.c_out)
        b.forward(xin, y)
        yu.append(y)
        xin = y
    cc3d.sync_status()
    # block 0 is the same computation either way (its conv2 also writes a0_1)
    assert torch.equal(ys[0].cpu(), yu[0].cpu())
    xin = synth.ncthw_view(x.cpu())
    for i, c in enumerate(cases):
        args, kw = _oracle_args(c)
        what = f"chain block {i} {spec[i][0]}->{spec[i][1]} n{n} {t}x{h}x{w}"
        if a0s[i] is not None:
            # the hand-over: SiLU(RMS_norm(y_{i-1}; g1 of block i)) from the
            # bf16 block output
            ref_a0 = oracle.rms_norm(xin.double().numpy(), args[2], None, silu=True)
            assert_close_bf16(ncthw_np(a0s[i]), ref_a0, what + " a0")
        ref = oracle.resblock(xin, *args, **kw)
        assert_close_bf16(ncthw_np(ys[i]), ref, what)
        assert_close_bf16(ncthw_np(yu[i]), ref, what + " unfused")
        xin = synth.ncthw_view(ys[i].cpu())


@pytest.mark.parametrize("own_history", [True, False])
def test_streamed_fused_chain_equals_whole_bitwise(own_history):
    """Chunks of 1, 2 and 2 frames with every block's caches carried.  The
    next block's conv1 history (a0 frames) is written either by that block's
    conv1 from a0_in (own_history) or by the previous block's conv2 epilogue
    through a0_next_cache_*; both equal the whole-sequence chain bit for bit,
    caches included."""
    n, t, h, w = 1, 5, 16, 20
    spec = [(64, 96), (96, 96), (96, 96)]
    cases = _chain_cases(spec, n, t, h, w, seed=41)
    blocks = [_block(c, n, h, w, t) for c in cases]
    x = to_dev(synth.ndhwc(cases[0]["x"]))
    nb = len(blocks)
    cache = lambda c: torch.zeros((n, 2, h, w, c), dtype=torch.bfloat16, device="cuda")  # noqa: E731
    ref_c1 = [cache(ci) for ci, _ in spec]
    ref_c2 = [cache(co) for _, co in spec]
    whole, _ = _run_fused(blocks, x, n, t, h, w, ref_c1, ref_c2)
    c1 = [[cache(ci), cache(ci)] for ci, _ in spec]
    c2 = [[cache(co), cache(co)] for _, co in spec]
    outs = [[] for _ in blocks]
    f0 = 0
    for s, tc in enumerate([1, 2, 2]):
        cur, new = s % 2, (s + 1) % 2
        xin, a_in = x[:, f0:f0 + tc].contiguous(), None
        for i, b in enumerate(blocks):
            nxt = i + 1 < nb
            y = _empty(n, tc, h, w, b.c_out)
            a_next = _empty(n, tc, h, w, b.c_out) if nxt else None
            writes_next = nxt and not own_history
            b.forward(xin, y, cache1_in=c1[i][cur], cache2_in=c2[i][cur],
                      cache1_out=c1[i][new] if (i == 0 or own_history) else None,
                      cache2_out=c2[i][new], a0_in=a_in,
                      g_next=blocks[i + 1].g1 if nxt else None, a0_next=a_next,
                      a0_next_cache_in=c1[i + 1][cur] if writes_next else None,
                      a0_next_cache_out=c1[i + 1][new] if writes_next else None)
            outs[i].append(y)
            xin, a_in = y, a_next
        f0 += tc
    cc3d.sync_status()
    for i in range(nb):
        assert torch.equal(torch.cat(outs[i], dim=1).cpu(), whole[i].cpu()), f"block {i}"
    # the carried caches after the last chunk (three chunks: the ones written
    # last are index 1) against the whole sequence's
    for i in range(nb):
        assert torch.equal(c1[i][1].cpu(), ref_c1[i].cpu()), f"cache1 of block {i}"
        assert torch.equal(c2[i][1].cpu(), ref_c2[i].cpu()), f"cache2 of block {i}"


def test_hand_over_cache_is_last_two_frames():
    """a0_next_cache_out = the last two frames of concat(a0_next_cache_in,
    a0_next) for chunks of one and three frames."""
    n, h, w = 1, 12, 16
    spec = [(64, 64), (64, 64)]
    for tc in (1, 3):
        cases = _chain_cases(spec, n, tc, h, w, seed=90 + tc)
        b0, b1 = (_block(c, n, h, w, tc) for c in cases)
        x = to_dev(synth.ndhwc(cases[0]["x"]))
        hist = to_dev(synth.ndhwc(synth.normal((n, 64, 2, h, w), 77 + tc)))
        y, a = _empty(n, tc, h, w, 64), _empty(n, tc, h, w, 64)
        hout = torch.empty_like(hist)
        b0.forward(x, y, g_next=b1.g1, a0_next=a, a0_next_cache_in=hist, a0_next_cache_out=hout)
        cc3d.sync_status()
        full = torch.cat([hist.cpu(), a.cpu()], dim=1)
        assert torch.equal(hout.cpu(), full[:, -2:])
        b0.close()
        b1.close()


def test_fused_chain_refusals():
    n, t, h, w = 1, 2, 8, 8
    cases = _chain_cases([(64, 64), (64, 64)], n, t, h, w, seed=5)
    b0, b1 = (_block(c, n, h, w, t) for c in cases)
    x = to_dev(synth.ndhwc(cases[0]["x"]))
    y, a = _empty(n, t, h, w, 64), _empty(n, t, h, w, 64)
    fused = cc3d.cc3d_resblock_forward_fused
    ptr = lambda q: q.data_ptr()  # noqa: E731
    nul = None
    # a0_next without g_next, g_next without a0_next, a history without both
    assert fused(b0.handle, ptr(x), nul, t, nul, nul, ptr(y), nul, nul, nul, ptr(a), nul, nul,
                 nul) == cc3d.ERR_INVALID_ARG
    assert fused(b0.handle, ptr(x), nul, t, nul, nul, ptr(y), nul, nul, ptr(b1.g1), nul, nul,
                 nul, nul) == cc3d.ERR_INVALID_ARG
    assert fused(b0.handle, ptr(x), nul, t, nul, nul, ptr(y), nul, nul, nul, nul, nul, ptr(a),
                 nul) == cc3d.ERR_INVALID_ARG
    # a0_next over x, over y: refused before anything is launched
    before = cc3d.cc3d_launch_count()
    assert fused(b0.handle, ptr(x), nul, t, nul, nul, ptr(y), nul, nul, ptr(b1.g1), ptr(x), nul,
                 nul, nul) == cc3d.ERR_ALIAS
    assert fused(b0.handle, ptr(x), nul, t, nul, nul, ptr(y), nul, nul, ptr(b1.g1), ptr(y), nul,
                 nul, nul) == cc3d.ERR_ALIAS
    # the hand-over history written over its own input, a cache that is not
    # 16-byte aligned: refused before anything runs as well
    hist = torch.empty((n, 2, h, w, 64), dtype=torch.bfloat16, device="cuda")
    assert fused(b0.handle, ptr(x), nul, t, nul, nul, ptr(y), nul, nul, ptr(b1.g1), ptr(a),
                 ptr(hist), ptr(hist), nul) == cc3d.ERR_ALIAS
    assert fused(b0.handle, ptr(x), nul, t, nul, ptr(hist) + 2, ptr(y), nul, nul, ptr(b1.g1),
                 ptr(a), nul, nul, nul) == cc3d.ERR_ALIGNMENT
    assert cc3d.cc3d_launch_count() == before
    cc3d.sync_status()
    for b in (b0, b1):
        b.close()


@pytest.mark.parametrize("c", [384, 640])
def test_wide_hand_over_is_the_norm_pass(c):
    """Above 256 channels the hand-over is the stand-alone norm over y: a0_next
    and its history equal rms_silu(y) bit for bit (that kernel is pinned to
    the oracle on its own)."""
    n, t, h, w = 1, 2, 6, 10
    cases = _chain_cases([(c, c), (c, c)], n, t, h, w, seed=c)
    b0, b1 = (_block(cs, n, h, w, t) for cs in cases)
    x = to_dev(synth.ndhwc(cases[0]["x"]))
    y, a, ref = _empty(n, t, h, w, c), _empty(n, t, h, w, c), _empty(n, t, h, w, c)
    hist = to_dev(synth.ndhwc(synth.normal((n, c, 2, h, w), c + 1)))
    hout, ref_hout = torch.empty_like(hist), torch.empty_like(hist)
    b0.forward(x, y, g_next=b1.g1, a0_next=a, a0_next_cache_in=hist, a0_next_cache_out=hout)
    cc3d.rms_silu(y, b1.g1, ref, cache_in=hist, cache_out=ref_hout)
    cc3d.sync_status()
    assert torch.equal(a.cpu(), ref.cpu())
    assert torch.equal(hout.cpu(), ref_hout.cpu())
    b0.close()
    b1.close()
