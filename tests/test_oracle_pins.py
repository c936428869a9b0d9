"""Pins for the fp64 CPU oracle (no GPU).

The oracle is checked against things other than itself:
  * a library special case: torch's float64 conv3d on an explicitly padded
    input (zero frames or the cache in front of t, spatial zeros);
  * a second brute force written here: explicit padded copy, then a dense
    3-D correlation with numpy windows;
  * the per-temporal-slice algebra of the "cache-aware video decoder
    lowering" summary (one Conv2D per kernel time slice, summed, bias once);
  * k_t = 1 reducing to a per-frame Conv2D;
  * the impulse response (pins orientation and the causal time shift);
  * the invariants the pages state: causality, chunked streaming with a
    2-frame cache equal to whole-sequence evaluation, bias added once,
    linearity in x;
  * closed forms for RMS_norm, SiLU and bf16 rounding;
  * a hand-worked example under tests/golden/.
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from video_vae_causal_implicit_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rnd(shape, seed, scale=1.0):
    g = np.random.default_rng(seed)
    return g.standard_normal(shape) * scale


def torch_causal_conv3d(x, w, b, cache=None, pad=(1, 1), stride_t=1):
    """Library special case: F.pad + conv3d (temporal stride stride_t) in
    float64."""
    x = torch.from_numpy(np.ascontiguousarray(x))
    w = torch.from_numpy(np.ascontiguousarray(w))
    kt = w.shape[2]
    if cache is not None:
        xt = torch.cat([torch.from_numpy(np.ascontiguousarray(cache)), x], dim=2)
        xt = F.pad(xt, (pad[1], pad[1], pad[0], pad[0], 0, 0))
    else:
        xt = F.pad(x, (pad[1], pad[1], pad[0], pad[0], kt - 1, 0))
    bb = torch.from_numpy(np.asarray(b)) if b is not None else None
    return F.conv3d(xt, w, bb, stride=(stride_t, 1, 1)).numpy()


def numpy_padded_correlation(x, w, b, cache=None):
    """Brute force 2: materialise the padded input, then correlate."""
    N, Ci, T, H, W = x.shape
    Co, _, KT, KH, KW = w.shape
    front = cache if cache is not None else np.zeros((N, Ci, KT - 1, H, W))
    xt = np.concatenate([front, x], axis=2)
    xt = np.pad(xt, ((0, 0), (0, 0), (0, 0), (KH // 2, KH // 2), (KW // 2, KW // 2)))
    y = np.zeros((N, Co, T, H, W))
    for t in range(T):
        for h in range(H):
            for ww in range(W):
                patch = xt[:, :, t:t + KT, h:h + KH, ww:ww + KW]  # N,Ci,KT,KH,KW
                y[:, :, t, h, ww] = np.einsum("nijkl,oijkl->no", patch, w)
    return y + (0 if b is None else np.asarray(b)[None, :, None, None, None])


def per_slice_conv2d(x, w, b):
    """Per-temporal-slice lowering: for each kernel time slice kt, one Conv2D
    over the frames it reads (tau = t + kt - 2; frames before 0 are zero and
    contribute nothing), summed over kt; bias once at the end."""
    N, Ci, T, H, W = x.shape
    Co, _, KT, KH, KW = w.shape
    y = torch.zeros((N, Co, T, H, W), dtype=torch.float64)
    xt = torch.from_numpy(x)
    for kt in range(KT):
        shift = KT - 1 - kt  # output t reads frame t - shift
        if shift >= T:
            continue
        frames = xt[:, :, : T - shift]  # frames 0 .. T-shift-1 feed outputs shift .. T-1
        batch = frames.permute(0, 2, 1, 3, 4).reshape(-1, Ci, H, W)
        out = F.conv2d(batch, torch.from_numpy(w[:, :, kt]), padding=(KH // 2, KW // 2))
        out = out.reshape(N, T - shift, Co, H, W).permute(0, 2, 1, 3, 4)
        y[:, :, shift:] += out
    return (y + torch.from_numpy(np.asarray(b))[None, :, None, None, None]).numpy()


SHAPES = [
    (1, 3, 4, 2, 5, 6),
    (2, 4, 3, 3, 4, 3),
    (1, 8, 8, 4, 6, 6),
    (1, 2, 5, 1, 1, 1),
    (1, 5, 2, 6, 3, 7),
]


@pytest.mark.parametrize("N,Ci,Co,T,H,W", SHAPES)
def test_conv_matches_torch_fp64(N, Ci, Co, T, H, W):
    x = rnd((N, Ci, T, H, W), 1)
    w = rnd((Co, Ci, 3, 3, 3), 2, 0.3)
    b = rnd((Co,), 3, 0.1)
    y = oracle.causal_conv3d(x, w, b)
    ref = torch_causal_conv3d(x, w, b)
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("N,Ci,Co,T,H,W", SHAPES[:3])
def test_conv_with_cache_matches_torch_fp64(N, Ci, Co, T, H, W):
    x = rnd((N, Ci, T, H, W), 4)
    cache = rnd((N, Ci, 2, H, W), 5)
    w = rnd((Co, Ci, 3, 3, 3), 6, 0.3)
    b = rnd((Co,), 7, 0.1)
    y = oracle.causal_conv3d(x, w, b, cache=cache)
    np.testing.assert_allclose(y, torch_causal_conv3d(x, w, b, cache=cache), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(y, numpy_padded_correlation(x, w, b, cache), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("N,Ci,Co,T,H,W", SHAPES)
def test_conv_matches_padded_copy_and_per_slice(N, Ci, Co, T, H, W):
    x = rnd((N, Ci, T, H, W), 8)
    w = rnd((Co, Ci, 3, 3, 3), 9, 0.3)
    b = rnd((Co,), 10, 0.1)
    y = oracle.causal_conv3d(x, w, b)
    np.testing.assert_allclose(y, numpy_padded_correlation(x, w, b), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(y, per_slice_conv2d(x, w, b), rtol=1e-12, atol=1e-12)


def test_kt1_is_per_frame_conv2d():
    x = rnd((1, 4, 3, 5, 6), 11)
    w = rnd((6, 4, 1, 3, 3), 12, 0.3)
    b = rnd((6,), 13)
    y = oracle.causal_conv3d(x, w, b)
    for t in range(3):
        ref = F.conv2d(torch.from_numpy(x[:, :, t]), torch.from_numpy(w[:, :, 0]),
                       torch.from_numpy(b), padding=1).numpy()
        np.testing.assert_allclose(y[:, :, t], ref, rtol=1e-12, atol=1e-12)


def test_impulse_response_pins_orientation_and_causal_shift():
    Ci, Co, T, H, W = 2, 3, 5, 5, 5
    w = rnd((Co, Ci, 3, 3, 3), 14)
    b = rnd((Co,), 15)
    ci, t0, h0, w0 = 1, 1, 2, 2
    x = np.zeros((1, Ci, T, H, W))
    x[0, ci, t0, h0, w0] = 1.0
    y = oracle.causal_conv3d(x, w, None)
    yb = oracle.causal_conv3d(x, w, b)
    np.testing.assert_allclose(yb - y, np.broadcast_to(b[None, :, None, None, None], y.shape),
                               rtol=0, atol=1e-15)
    for kt in range(3):
        for kh in range(3):
            for kw in range(3):
                # y[t] reads frame t + kt - 2, so the impulse at t0 reaches
                # output t0 + 2 - kt; rows/cols likewise with pad 1.
                t, h, ww = t0 + 2 - kt, h0 + 1 - kh, w0 + 1 - kw
                if t < T:
                    np.testing.assert_array_equal(y[0, :, t, h, ww], w[:, ci, kt, kh, kw])
    # nothing before t0, nothing beyond t0 + 2
    assert np.all(y[0, :, :t0] == 0.0)
    assert np.all(y[0, :, t0 + 3:] == 0.0)


def test_causality_future_frames_do_not_leak():
    x = rnd((1, 3, 6, 4, 5), 16)
    w = rnd((4, 3, 3, 3, 3), 17)
    b = rnd((4,), 18)
    y = oracle.causal_conv3d(x, w, b)
    for t0 in range(6):
        x2 = x.copy()
        x2[:, :, t0] += rnd((1, 3, 4, 5), 100 + t0)
        y2 = oracle.causal_conv3d(x2, w, b)
        np.testing.assert_array_equal(y2[:, :, :t0], y[:, :, :t0])
        assert np.any(y2[:, :, t0] != y[:, :, t0])


@pytest.mark.parametrize("chunk", [1, 2, 3])
def test_streaming_equals_whole_sequence_bitwise(chunk):
    T = 7
    x = rnd((1, 3, T, 4, 5), 19)
    w = rnd((4, 3, 3, 3, 3), 20)
    b = rnd((4,), 21)
    whole = oracle.causal_conv3d(x, w, b)
    cache = None
    outs = []
    for s in range(0, T, chunk):
        xc = x[:, :, s:s + chunk]
        outs.append(oracle.causal_conv3d(xc, w, b, cache=cache))
        # next cache: last 2 frames of concat(cache or zeros, chunk)
        prev = cache if cache is not None else np.zeros((1, 3, 2, 4, 5))
        cache = np.ascontiguousarray(np.concatenate([prev, xc], axis=2)[:, :, -2:])
    np.testing.assert_array_equal(np.concatenate(outs, axis=2), whole)


# ---- temporal stride (the downsample path's time_conv, stride (2,1,1)) ----------

@pytest.mark.parametrize("T,k,cached", [(6, (3, 3, 3), False), (7, (3, 1, 1), False),
                                        (5, (3, 1, 1), True), (4, (1, 3, 3), False)])
def test_strided_conv_matches_torch_fp64(T, k, cached):
    x = rnd((2, 3, T, 4, 5), 40)
    w = rnd((4, 3) + k, 41, 0.3)
    b = rnd((4,), 42, 0.1)
    cache = rnd((2, 3, k[0] - 1, 4, 5), 43) if cached else None
    pad = (k[1] // 2, k[2] // 2)
    y = oracle.causal_conv3d(x, w, b, cache=cache, pad=pad, stride_t=2)
    assert y.shape[2] == (T + 1) // 2
    ref = torch_causal_conv3d(x, w, b, cache=cache, pad=pad, stride_t=2)
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_strided_conv_is_unit_stride_at_even_frames_bitwise():
    """Output frame t of the stride-2 conv reads the same padded frames
    2t .. 2t+kt-1 as output frame 2t of the unit-stride conv."""
    x = rnd((1, 4, 9, 5, 4), 44)
    w = rnd((3, 4, 3, 3, 3), 45, 0.3)
    b = rnd((3,), 46, 0.1)
    for cache in (None, rnd((1, 4, 2, 5, 4), 47)):
        y2 = oracle.causal_conv3d(x, w, b, cache=cache, stride_t=2)
        y1 = oracle.causal_conv3d(x, w, b, cache=cache)
        np.testing.assert_array_equal(y2, y1[:, :, ::2])


@pytest.mark.parametrize("chunk", [2, 4])
def test_strided_streaming_even_chunks_equals_whole_bitwise(chunk):
    """Chunks of an even number of frames, carrying the last 2 input frames,
    give the whole-sequence stride-2 output."""
    T = 8
    x = rnd((1, 3, T, 4, 5), 48)
    w = rnd((4, 3, 3, 1, 1), 49, 0.3)
    b = rnd((4,), 50, 0.1)
    whole = oracle.causal_conv3d(x, w, b, pad=(0, 0), stride_t=2)
    cache = None
    outs = []
    for s0 in range(0, T, chunk):
        xc = x[:, :, s0:s0 + chunk]
        outs.append(oracle.causal_conv3d(xc, w, b, cache=cache, pad=(0, 0), stride_t=2))
        prev = cache if cache is not None else np.zeros((1, 3, 2, 4, 5))
        cache = np.ascontiguousarray(np.concatenate([prev, xc], axis=2)[:, :, -2:])
    np.testing.assert_array_equal(np.concatenate(outs, axis=2), whole)


def test_strided_points_equal_full_bitwise():
    x = rnd((1, 3, 7, 4, 5), 51)
    w = rnd((2, 3, 3, 3, 3), 52, 0.3)
    b = rnd((2,), 53, 0.1)
    full = oracle.causal_conv3d(x, w, b, stride_t=2)
    pts = [(0, t, h, ww) for t in range(4) for h in range(4) for ww in (0, 4)]
    got = oracle.causal_conv3d_points(x, w, b, None, pts, stride_t=2)
    for p, (n, t, h, ww) in enumerate(pts):
        np.testing.assert_array_equal(got[p], full[n, :, t, h, ww])


def test_zero_cache_equals_no_cache_bitwise():
    x = rnd((1, 3, 3, 4, 4), 22)
    w = rnd((2, 3, 3, 3, 3), 23)
    b = rnd((2,), 24)
    np.testing.assert_array_equal(oracle.causal_conv3d(x, w, b),
                                  oracle.causal_conv3d(x, w, b, cache=np.zeros((1, 3, 2, 4, 4))))


def test_bias_added_once_and_linearity():
    x1 = rnd((1, 3, 4, 4, 5), 25)
    x2 = rnd((1, 3, 4, 4, 5), 26)
    w = rnd((4, 3, 3, 3, 3), 27)
    b = rnd((4,), 28)
    y0 = oracle.causal_conv3d(np.zeros_like(x1), w, b)
    np.testing.assert_array_equal(y0, np.broadcast_to(b[None, :, None, None, None], y0.shape))
    f = lambda x: oracle.causal_conv3d(x, w, b) - y0  # noqa: E731
    a, c = 0.7, -1.9
    np.testing.assert_allclose(f(a * x1 + c * x2), a * f(x1) + c * f(x2), rtol=1e-12, atol=1e-12)
    # bias twice (once per temporal slice) would break this:
    np.testing.assert_allclose(oracle.causal_conv3d(x1, w, None) + b[None, :, None, None, None],
                               oracle.causal_conv3d(x1, w, b), rtol=0, atol=1e-13)


def test_points_equal_full_conv_bitwise():
    x = rnd((2, 3, 4, 5, 6), 29)
    cache = rnd((2, 3, 2, 5, 6), 30)
    w = rnd((4, 3, 3, 3, 3), 31)
    b = rnd((4,), 32)
    y = oracle.causal_conv3d(x, w, b, cache=cache)
    pts = np.array([[0, 0, 0, 0], [1, 3, 4, 5], [0, 1, 2, 3], [1, 0, 4, 0], [0, 2, 0, 5]])
    yp = oracle.causal_conv3d_points(x, w, b, cache, pts)
    for k, (n, t, h, ww) in enumerate(pts):
        np.testing.assert_array_equal(yp[k], y[n, :, t, h, ww])


def test_strided_bf16_view_reads_channels_last():
    """The oracle reads a channels-last bf16 buffer through a permuted view
    exactly as it reads the same values in NCTHW float64."""
    case = synth.conv_case(4, 5, 3, 4, 6)
    x_cl = synth.ndhwc(case["x"])
    y_view = oracle.causal_conv3d(synth.ncthw_view(x_cl), case["w"], case["b"].double().numpy())
    y_f64 = oracle.causal_conv3d(case["x"].double().numpy(), case["w"].double().numpy(),
                                 case["b"].double().numpy())
    np.testing.assert_array_equal(y_view, y_f64)


# ---- RMS_norm, SiLU, bf16 rounding -------------------------------------------

def test_rms_norm_closed_forms():
    C = 6
    g = np.linspace(0.5, 1.5, C)
    x = rnd((1, C, 2, 3, 4), 33)
    r = oracle.rms_norm(x, g)
    # || r / gamma ||_2 = sqrt(C) at every voxel
    nrm = np.sqrt(((r / g[None, :, None, None, None]) ** 2).sum(axis=1))
    np.testing.assert_allclose(nrm, math.sqrt(C), rtol=1e-13)
    # invariant to positive scaling of the channel vector
    np.testing.assert_allclose(oracle.rms_norm(3.7 * x, g), r, rtol=1e-13, atol=1e-15)
    # one-hot v = a e_k  ->  r = sqrt(C) gamma_k e_k (sign of a)
    oh = np.zeros((1, C, 1, 1, 1))
    oh[0, 2] = -4.0
    ro = oracle.rms_norm(oh, g)[0, :, 0, 0, 0]
    exp = np.zeros(C)
    exp[2] = -math.sqrt(C) * g[2]
    np.testing.assert_allclose(ro, exp, rtol=1e-15, atol=0)
    # zero vector -> 0 (denominator floored at 1e-12), SiLU(0) = 0
    z = oracle.rms_norm(np.zeros((1, C, 1, 1, 1)), g, silu=True)
    assert np.all(z == 0.0)
    # beta is added after the scale
    beta = np.arange(C) * 0.25
    np.testing.assert_allclose(oracle.rms_norm(x, g, beta), r + beta[None, :, None, None, None],
                               rtol=1e-14, atol=1e-14)


def test_rms_norm_matches_torch_normalize():
    C = 8
    x = rnd((2, C, 3, 2, 2), 34)
    g = rnd((C,), 35)
    ref = F.normalize(torch.from_numpy(x), dim=1).numpy() * math.sqrt(C) * g[None, :, None, None, None]
    np.testing.assert_allclose(oracle.rms_norm(x, g), ref, rtol=1e-13, atol=1e-14)
    ref_silu = F.silu(torch.from_numpy(ref)).numpy()
    np.testing.assert_allclose(oracle.rms_norm(x, g, silu=True), ref_silu, rtol=1e-13, atol=1e-14)


def test_silu_closed_forms():
    assert oracle.silu(0.0) == 0.0
    assert abs(oracle.silu(1.0) - 1.0 / (1.0 + math.exp(-1.0))) < 1e-16
    for z in (-7.5, -1.0, -1e-3, 0.25, 3.0, 20.0):
        assert abs((oracle.silu(z) - oracle.silu(-z)) - z) < 1e-14 * max(1.0, abs(z))
    assert abs(oracle.silu(-40.0)) < 1e-15


def test_round_bf16_ties_and_library_case():
    r = oracle.round_bf16
    assert r(1.0) == 1.0
    assert r(1.0 + 2.0 ** -8) == 1.0                      # tie -> even (mantissa 0)
    assert r(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6      # tie -> even (mantissa 2)
    assert r(1.0 + 2.0 ** -8 + 2.0 ** -30) == 1.0 + 2.0 ** -7
    assert r(-3.0) == -3.0
    assert r(2.0 ** -140) == 0.0
    assert r(2.0 ** -133) == 2.0 ** -133
    assert math.isinf(r(3.5e38))
    # library special case: torch's fp32 -> bf16 cast is RNE too
    v = torch.randn(4096, dtype=torch.float64, generator=torch.Generator().manual_seed(5)) * 10
    v32 = v.float()
    ref = v32.to(torch.bfloat16).double().numpy()
    got = oracle.round_bf16_array(v32.double().numpy())
    np.testing.assert_array_equal(got, ref)


# ---- residual block -----------------------------------------------------------

def _block_small(C=8, T=4, H=5, W=6, seed=0):
    return synth.block_case(C, T, H, W, seed_base=seed)


def _np(t):
    return t.double().numpy()


def test_block_is_composition_of_pinned_parts():
    c = _block_small()
    y, a0, a1 = oracle.resblock(c["x"], c["w1"], _np(c["b1"]), _np(c["g1"]), c["w2"], _np(c["b2"]),
                                _np(c["g2"]), return_acts=True)
    # rebuild with torch fp64 ops: normalize*sqrt(C)*gamma, silu, bf16 RNE, conv
    x = c["x"].double()
    C = x.shape[1]

    def rs(v, g):
        return F.silu(F.normalize(v, dim=1) * math.sqrt(C) * g.double()[None, :, None, None, None])

    a0_ref = rs(x, c["g1"]).float().to(torch.bfloat16).double()
    # double->float->bf16 can double-round; compare with tolerance of 1 bf16 ulp
    np.testing.assert_allclose(a0, a0_ref.numpy(), rtol=2 ** -7, atol=1e-30)
    a0t = torch.from_numpy(a0)
    # conv1's output h1 is a bf16 activation (the default reading)
    h1 = torch.from_numpy(oracle.round_bf16_array(
        torch_causal_conv3d(a0t.numpy(), _np(c["w1"]), _np(c["b1"]))))
    a1_ref = rs(h1, c["g2"]).numpy()
    np.testing.assert_allclose(a1, oracle.round_bf16_array(a1_ref), rtol=0, atol=0)
    y_ref = torch_causal_conv3d(a1, _np(c["w2"]), _np(c["b2"])) + x.numpy()
    np.testing.assert_allclose(y, y_ref, rtol=1e-12, atol=1e-12)


def test_block_identity_when_conv2_is_zero():
    c = _block_small(seed=3)
    y = oracle.resblock(c["x"], c["w1"], _np(c["b1"]), _np(c["g1"]), torch.zeros_like(c["w2"]),
                        np.zeros(8), _np(c["g2"]))
    np.testing.assert_array_equal(y, _np(c["x"]))


def test_block_points_equal_full_block_bitwise():
    c = _block_small(C=6, T=4, H=5, W=5, seed=7)
    cache1 = synth.normal((1, 6, 2, 5, 5), 90)
    cache2 = synth.normal((1, 6, 2, 5, 5), 91)
    args = (c["x"], c["w1"], _np(c["b1"]), _np(c["g1"]), c["w2"], _np(c["b2"]), _np(c["g2"]))
    for c1, c2 in ((None, None), (cache1, cache2)):
        y = oracle.resblock(*args, cache1=c1, cache2=c2)
        pts = np.array([[0, 0, 0, 0], [0, 3, 4, 4], [0, 1, 2, 3], [0, 2, 0, 4], [0, 0, 4, 1]])
        yp = oracle.resblock_points(*args, pts, cache1=c1, cache2=c2)
        for k, (n, t, h, w) in enumerate(pts):
            np.testing.assert_array_equal(yp[k], y[n, :, t, h, w])


def test_block_streaming_equals_whole():
    """Chunked block with per-conv 2-frame caches (a0 history for conv1, a1
    history for conv2) equals the whole-sequence block, bitwise."""
    C, T, H, W = 4, 5, 4, 4
    c = _block_small(C=C, T=T, H=H, W=W, seed=11)
    args = (_np(c["w1"]), _np(c["b1"]), _np(c["g1"]), _np(c["w2"]), _np(c["b2"]), _np(c["g2"]))
    x = _np(c["x"])
    whole, a0, a1 = oracle.resblock(x, *args[:3], *args[3:], return_acts=True)
    outs = []
    c1 = c2 = None
    for s in range(T):
        xc = np.ascontiguousarray(x[:, :, s:s + 1])
        outs.append(oracle.resblock(xc, *args, cache1=c1, cache2=c2))
        c1 = np.ascontiguousarray(a0[:, :, max(0, s - 1):s + 1]) if s >= 1 else np.concatenate(
            [np.zeros((1, C, 1, H, W)), a0[:, :, :1]], axis=2)
        c2 = np.ascontiguousarray(a1[:, :, max(0, s - 1):s + 1]) if s >= 1 else np.concatenate(
            [np.zeros((1, C, 1, H, W)), a1[:, :, :1]], axis=2)
    np.testing.assert_array_equal(np.concatenate(outs, axis=2), whole)


# ---- channel-changing block: the 1x1x1 conv_shortcut ---------------------------

def _block_sc(Cin=6, Cout=10, T=4, H=5, W=5, seed=20):
    c = synth.block_case(Cin, T, H, W, seed_base=seed)
    return {
        "x": c["x"],
        "w1": synth.kaiming_uniform(Cout, Cin, (3, 3, 3), seed + 31),
        "b1": synth.uniform((Cout,), -0.1, 0.1, seed + 32),
        "g1": c["g1"],
        "w2": synth.kaiming_uniform(Cout, Cout, (3, 3, 3), seed + 33),
        "b2": synth.uniform((Cout,), -0.1, 0.1, seed + 34),
        "g2": synth.uniform((Cout,), 0.5, 1.5, seed + 35),
        "wsc": synth.kaiming_uniform(Cout, Cin, (1, 1, 1), seed + 36),
        "bsc": synth.uniform((Cout,), -0.1, 0.1, seed + 37),
    }


def _sc_args(c):
    return (c["x"], c["w1"], _np(c["b1"]), _np(c["g1"]), c["w2"], _np(c["b2"]), _np(c["g2"]))


def test_shortcut_block_matches_torch_composition():
    """C_in != C_out: y = conv2(a1) + b2 + conv_1x1x1(x; wsc) + bsc, rebuilt
    with torch fp64 ops (normalize * sqrt(C) * gamma, silu, conv3d); with
    round_h1 conv1's output is rounded to bf16 before its RMS_norm."""
    c = _block_sc()
    x = c["x"].double()

    def rs(v, g):
        C = v.shape[1]
        return F.silu(F.normalize(v, dim=1) * math.sqrt(C) * g.double()[None, :, None, None, None])

    for round_h1 in (False, True):
        y, a0, a1 = oracle.resblock(*_sc_args(c), return_acts=True, w_sc=c["wsc"],
                                    b_sc=_np(c["bsc"]), round_h1=round_h1)
        a0_ref = rs(x, c["g1"]).float().to(torch.bfloat16).double()
        np.testing.assert_allclose(a0, a0_ref.numpy(), rtol=2 ** -7, atol=1e-30)
        h1 = torch_causal_conv3d(a0, _np(c["w1"]), _np(c["b1"]))
        if round_h1:
            h1 = oracle.round_bf16_array(h1)
        a1_ref = rs(torch.from_numpy(h1), c["g2"]).numpy()
        np.testing.assert_allclose(a1, oracle.round_bf16_array(a1_ref), rtol=0, atol=0)
        sc = F.conv3d(x, c["wsc"].double(), c["bsc"].double()).numpy()
        y_ref = torch_causal_conv3d(a1, _np(c["w2"]), _np(c["b2"])) + sc
        np.testing.assert_allclose(y, y_ref, rtol=1e-12, atol=1e-12)


def test_identity_shortcut_weights_give_the_identity_block_bitwise():
    """C_in == C_out with wsc = I and bsc = 0 is the identity shortcut."""
    c = _block_small(C=6, seed=21)
    eye = torch.eye(6, dtype=torch.float64).reshape(6, 6, 1, 1, 1)
    args = (c["x"], c["w1"], _np(c["b1"]), _np(c["g1"]), c["w2"], _np(c["b2"]), _np(c["g2"]))
    y_id = oracle.resblock(*args)
    y_sc = oracle.resblock(*args, w_sc=eye, b_sc=np.zeros(6))
    np.testing.assert_array_equal(y_sc, y_id)


def test_shortcut_block_points_equal_full_bitwise():
    c = _block_sc(seed=22)
    cache1 = synth.normal((1, 6, 2, 5, 5), 92)
    cache2 = synth.normal((1, 10, 2, 5, 5), 93)
    kw = dict(w_sc=c["wsc"], b_sc=_np(c["bsc"]))
    for c1, c2, rh in ((None, None, False), (cache1, cache2, True)):
        y = oracle.resblock(*_sc_args(c), cache1=c1, cache2=c2, round_h1=rh, **kw)
        pts = np.array([[0, 0, 0, 0], [0, 3, 4, 4], [0, 1, 2, 3], [0, 2, 0, 4]])
        yp = oracle.resblock_points(*_sc_args(c), pts, cache1=c1, cache2=c2, round_h1=rh, **kw)
        for k, (n, t, h, w) in enumerate(pts):
            np.testing.assert_array_equal(yp[k], y[n, :, t, h, w])


def test_shortcut_block_streaming_equals_whole():
    Cin, Cout, T, H, W = 4, 6, 4, 4, 4
    c = _block_sc(Cin, Cout, T, H, W, seed=23)
    x = _np(c["x"])
    rest = _sc_args(c)[1:]
    kw = dict(w_sc=c["wsc"], b_sc=_np(c["bsc"]))
    whole, a0, a1 = oracle.resblock(x, *rest, return_acts=True, **kw)
    outs, c1, c2 = [], None, None
    for s in range(T):
        xc = np.ascontiguousarray(x[:, :, s:s + 1])
        outs.append(oracle.resblock(xc, *rest, cache1=c1, cache2=c2, **kw))
        pad0 = np.zeros((1, Cin, 1, H, W))
        pad1 = np.zeros((1, Cout, 1, H, W))
        c1 = np.ascontiguousarray(a0[:, :, s - 1:s + 1]) if s >= 1 else np.concatenate(
            [pad0, a0[:, :, :1]], axis=2)
        c2 = np.ascontiguousarray(a1[:, :, s - 1:s + 1]) if s >= 1 else np.concatenate(
            [pad1, a1[:, :, :1]], axis=2)
    np.testing.assert_array_equal(np.concatenate(outs, axis=2), whole)


# ---- the downsample path's per-frame stride-2 Conv2d ----------------------------

def torch_conv2d_frames(x, w, b, stride, pad):
    """Library special case: frames to the batch, F.pad, F.conv2d (fp64)."""
    x = torch.from_numpy(np.ascontiguousarray(x))
    N, C, T, H, W = x.shape
    xf = x.permute(0, 2, 1, 3, 4).reshape(N * T, C, H, W)
    yf = F.conv2d(F.pad(xf, pad), torch.from_numpy(w), torch.from_numpy(b), stride=stride)
    Co, Ho, Wo = yf.shape[1:]
    return yf.reshape(N, T, Co, Ho, Wo).permute(0, 2, 1, 3, 4).numpy()


@pytest.mark.parametrize("stride,pad", [((2, 2), (0, 1, 0, 1)), ((2, 2), (1, 1, 1, 1)),
                                        ((2, 2), (1, 0, 1, 0)), ((1, 1), (1, 1, 1, 1))])
def test_conv2d_frames_matches_torch(stride, pad):
    x = rnd((2, 3, 3, 9, 10), 60)
    w = rnd((5, 3, 3, 3), 61, 0.3)
    b = rnd((5,), 62)
    y = oracle.conv2d_frames(x, w, b, stride=stride, pad=pad)
    ref = torch_conv2d_frames(x, w, b, stride, pad)
    assert y.shape == ref.shape
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_conv2d_frames_stride1_is_the_kt1_causal_conv_bitwise():
    x = rnd((1, 4, 3, 6, 7), 63)
    w = rnd((2, 4, 3, 3), 64)
    b = rnd((2,), 65)
    y = oracle.conv2d_frames(x, w, b, stride=(1, 1), pad=(1, 1, 1, 1))
    ref = oracle.causal_conv3d(x, w.reshape(2, 4, 1, 3, 3), b, pad=(1, 1))
    np.testing.assert_array_equal(y, ref)


def test_conv2d_frames_impulse_pins_stride_and_padding_side():
    """A one-hot input reaches output (i, j) through tap (kh, kw) exactly
    when 2i + kh - top = h0 and 2j + kw - left = w0."""
    C, T, H, W = 2, 2, 8, 9
    h0, w0, ci0, t0 = 4, 5, 1, 1
    x = np.zeros((1, C, T, H, W))
    x[0, ci0, t0, h0, w0] = 1.0
    w = rnd((3, C, 3, 3), 66)
    for pad in ((0, 1, 0, 1), (1, 0, 1, 0)):
        left, _, top, _ = pad
        y = oracle.conv2d_frames(x, w, None, stride=(2, 2), pad=pad)
        want = np.zeros_like(y)
        for i in range(y.shape[3]):
            for j in range(y.shape[4]):
                for kh in range(3):
                    for kw in range(3):
                        if 2 * i + kh - top == h0 and 2 * j + kw - left == w0:
                            want[0, :, t0, i, j] += w[:, ci0, kh, kw]
        np.testing.assert_array_equal(y, want)


def test_conv2d_frames_halves_the_pages_frame():
    """ZeroPad2d(0, 1, 0, 1) + 3x3 stride 2 maps 480 x 832 to 240 x 416."""
    y = oracle.conv2d_frames(np.ones((1, 1, 1, 480, 832)), np.ones((1, 1, 3, 3)), None)
    assert y.shape == (1, 1, 1, 240, 416)
    assert y[0, 0, 0, 0, 0] == 9.0 and y[0, 0, 0, -1, -1] == 4.0


# ---- FP8 E4M3 quantiser and the conv on E4M3 operands --------------------------

def _e4m3_values():
    codes = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn)
    v = codes.to(torch.float64).numpy()
    return v[np.isfinite(v)]


def test_e4m3_fixes_every_e4m3_value():
    vals = _e4m3_values()
    assert len(vals) == 254 and vals.max() == 448.0 and vals.min() == -448.0
    got = np.array([oracle.round_e4m3(v) for v in vals])
    np.testing.assert_array_equal(got, vals)


def test_e4m3_matches_torch_cast_on_values_and_midpoints():
    """Single rounding from float32: every E4M3 value, every midpoint
    between neighbours (the ties), and seeded values across the range."""
    pos = np.unique(np.abs(_e4m3_values()))
    mids = (pos[:-1] + pos[1:]) / 2
    g = np.random.default_rng(70)
    rand = np.concatenate([g.uniform(-460, 460, 3000), g.standard_normal(3000) * 0.01,
                           g.standard_normal(3000)])
    v32 = torch.from_numpy(np.concatenate([pos, -pos, mids, -mids, rand])).float()
    ref = v32.to(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.round_e4m3(float(v)) for v in v32.double().numpy()])
    np.testing.assert_array_equal(got, ref)


def test_e4m3_special_cases():
    assert oracle.round_e4m3(1.0625) == 1.0      # tie -> even mantissa
    assert oracle.round_e4m3(1.1875) == 1.25     # tie -> even mantissa
    assert oracle.round_e4m3(2.0 ** -10) == 0.0  # half the smallest subnormal
    assert oracle.round_e4m3(3 * 2.0 ** -11) == 2.0 ** -9
    assert oracle.round_e4m3(500.0) == 448.0 and oracle.round_e4m3(-1e9) == -448.0  # clamp
    assert oracle.round_e4m3(-1.3) == -oracle.round_e4m3(1.3)


def test_e4m3_quantiser_with_f32_quotient_matches_torch():
    """quotient="f32": the float32 division x / s followed by one rounding to
    E4M3 equals torch's float32 division and float8_e4m3fn cast (saturated
    to +-448 first), code for code, across scales and values; the f64
    quotient gives the same codes away from rounding boundaries."""
    g = np.random.default_rng(73)
    x = np.concatenate([g.standard_normal(4000) * 3, g.uniform(-2000, 2000, 1000),
                        g.standard_normal(1000) * 1e-3]).astype(np.float32)
    for s in (0.0137, 0.5, 1.0, 3.7, 448.0 / 7.3):
        got = oracle.quantize_e4m3(x, s, quotient="f32")
        q = (torch.from_numpy(x) / torch.tensor(s, dtype=torch.float32)).clamp(-448, 448)
        ref = q.to(torch.float8_e4m3fn).to(torch.float64).numpy()
        np.testing.assert_array_equal(got, ref)
        got64 = oracle.quantize_e4m3(x, s, quotient="f64")
        assert np.mean(got64 == got) > 0.99


def test_fp8_conv_on_representable_operands_is_the_plain_conv():
    """Unit scales and operands already in E4M3: quantisation is exact, so
    the FP8 conv is the plain conv bit for bit."""
    vals = _e4m3_values()
    g = np.random.default_rng(71)
    small = vals[np.abs(vals) <= 4]
    x = g.choice(small, size=(1, 3, 3, 5, 6))
    w = g.choice(small, size=(4, 3, 3, 3, 3))
    b = rnd((4,), 72)
    y = oracle.causal_conv3d_fp8(x, w, b, 1.0, np.ones(4))
    np.testing.assert_array_equal(y, oracle.causal_conv3d(x, w, b))


def test_fp8_conv_scales_multiply_the_contraction():
    """y = s_x * s_w[co] * conv(q_x, q_w) + b equals the conv of the
    dequantised operands, and stays close to the unquantised conv."""
    g = np.random.default_rng(73)
    x = g.standard_normal((1, 4, 3, 5, 5))
    w = g.standard_normal((3, 4, 3, 3, 3)) * 0.2
    b = rnd((3,), 74)
    s_x = np.abs(x).max() / 448
    s_w = np.abs(w).reshape(3, -1).max(axis=1) / 448
    y = oracle.causal_conv3d_fp8(x, w, b, s_x, s_w)
    xd = s_x * oracle.quantize_e4m3(x, s_x)
    wd = s_w.reshape(-1, 1, 1, 1, 1) * oracle.quantize_e4m3(w, s_w.reshape(-1, 1, 1, 1, 1))
    np.testing.assert_allclose(y, oracle.causal_conv3d(xd, wd, b), rtol=1e-12, atol=1e-12)
    ref = oracle.causal_conv3d(x, w, b)
    assert np.abs(y - ref).max() < 0.1 * np.abs(ref).max()


# ---- hand-worked example --------------------------------------------------------

def _read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, val = line.split("=")
            vals[key.strip()] = [float(v) for v in val.split()]
    return vals


def test_golden_hand_worked_ones():
    g = _read_golden("causal_ones_T3_H2_W3.txt")
    T, H, W = 3, 2, 3
    x = np.ones((1, 1, T, H, W))
    w = np.ones((1, 1, 3, 3, 3))
    y = oracle.causal_conv3d(x, w, np.array([0.5]))
    np.testing.assert_array_equal(y.reshape(-1), np.array(g["y"]))


def test_golden_hand_worked_ramp_kernel():
    g = _read_golden("causal_timeramp_T4.txt")
    x = np.array(g["x"]).reshape(1, 1, 4, 1, 1)
    w = np.zeros((1, 1, 3, 3, 3))
    w[0, 0, :, 1, 1] = g["w_t"]
    y = oracle.causal_conv3d(x, w, np.array(g["b"]))
    np.testing.assert_array_equal(y.reshape(-1), np.array(g["y"]))
