"""The oracle's pins catch plausible mistakes.  Each case plants one bug in a
copy of the oracle's C source (an off-by-one causal shift, a flipped
kernel, a transposed weight index, bias counted twice, a wrong cache frame,
a missing sqrt(C), truncation instead of round-to-nearest-even, a
transposed shortcut weight, a wrong E4M3 mantissa width, padding on the
wrong side of the downsample conv), builds that copy as a separate module,
and checks that the library-based pins reject it -- while the unmodified
copy passes the same checks.  CPU only; the mutants never leave the test's
temporary directory."""
import importlib.util
import math
import os
import shutil
import sys

import numpy as np
import pytest
import torch
import torch.nn.functional as F

HERE = os.path.dirname(os.path.abspath(__file__))
ORACLE_DIR = os.path.join(os.path.dirname(HERE), "oracle")

MUTANTS = {
    "causal shift off by one": ("int tau = stride_t * t + kt - (KT - 1);",
                                "int tau = stride_t * t + kt - KT;"),
    "kernel flipped (convolution, not correlation)": ("int hh = h + kh - pad_h;",
                                                      "int hh = h - kh + pad_h;"),
    "weight taps transposed": ("acc += orc_get(wt, co, ci, kt, kh, kw) * xv;",
                               "acc += orc_get(wt, co, ci, kt, kw, kh) * xv;"),
    "bias counted twice": ("if (bias) acc += bias[co]; /* bias once, after all taps */",
                           "if (bias) acc += 2.0 * bias[co];"),
    "wrong cache frame": (": orc_get(cache, n, ci, tau + (KT - 1), hh, ww);",
                          ": orc_get(cache, n, ci, tau + (KT - 2) < 0 ? 0 : tau + (KT - 2), hh, ww);"),
    "RMS without sqrt(C)": ("double scale = sqrt((double)C);", "double scale = 1.0;"),
    "bf16 truncation": ("r = nearbyint(ldexp(m, 8));", "r = floor(ldexp(m, 8));"),
    "shortcut weight transposed": (
        "sc += orc_get(wsc, c, ci, 0, 0, 0) * orc_get(x, n, ci, t, h, w);",
        "sc += orc_get(wsc, ci % Cout, c % Cin, 0, 0, 0) * orc_get(x, n, ci, t, h, w);"),
    "E4M3 with 2 mantissa bits": ("r = ldexp(nearbyint(ldexp(m, 4)), e - 4);",
                                  "r = ldexp(nearbyint(ldexp(m, 3)), e - 3);"),
    "downsample padded before the frame": ("const int r = sh * i + kh - pad_t;",
                                           "const int r = sh * i + kh - pad_b;"),
}


def _load_copy(tmp, name, mutation):
    d = os.path.join(tmp, name)
    os.makedirs(d)
    shutil.copy(os.path.join(ORACLE_DIR, "__init__.py"), d)
    src = open(os.path.join(ORACLE_DIR, "cc3d_oracle.c")).read()
    if mutation is not None:
        old, new = mutation
        assert src.count(old) == 1, f"mutation site not found: {old}"
        src = src.replace(old, new)
    with open(os.path.join(d, "cc3d_oracle.c"), "w") as fh:
        fh.write(src)
    spec = importlib.util.spec_from_file_location(name, os.path.join(d, "__init__.py"),
                                                  submodule_search_locations=[d])
    mod = importlib.util.module_from_spec(spec)
    sys.modules[name] = mod
    spec.loader.exec_module(mod)
    mod.build(force=True)
    return mod


def _rnd(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def _torch_conv(x, w, b, cache=None, pad=(1, 1), stride_t=1):
    xt = torch.from_numpy(x)
    kt = w.shape[2]
    front = torch.from_numpy(cache) if cache is not None else torch.zeros(
        x.shape[0], x.shape[1], kt - 1, *x.shape[3:], dtype=torch.float64)
    xt = F.pad(torch.cat([front, xt], dim=2), (pad[1], pad[1], pad[0], pad[0], 0, 0))
    return F.conv3d(xt, torch.from_numpy(w), torch.from_numpy(b), stride=(stride_t, 1, 1)).numpy()


def _rs(v, g):
    C = v.shape[1]
    return F.silu(F.normalize(v, dim=1) * math.sqrt(C) * g[None, :, None, None, None])


def _failures(mod):
    """Names of the library-based pins `mod` fails."""
    fails = []
    x, w, b = _rnd((1, 3, 4, 5, 6), 1), _rnd((4, 3, 3, 3, 3), 2, 0.3), _rnd((4,), 3)
    cache = _rnd((1, 3, 2, 5, 6), 4)
    for st in (1, 2):
        for c in (None, cache):
            got = mod.causal_conv3d(x, w, b, cache=c, stride_t=st)
            if not np.allclose(got, _torch_conv(x, w, b, c, stride_t=st), rtol=1e-12, atol=1e-12):
                fails.append(f"conv stride {st} cache {c is not None}")
    g = np.abs(_rnd((3,), 5)) + 0.5
    got = mod.rms_norm(x, g, silu=True)
    if not np.allclose(got, _rs(torch.from_numpy(x), torch.from_numpy(g)).numpy(), rtol=1e-12,
                       atol=1e-12):
        fails.append("rms")
    v32 = torch.from_numpy(_rnd((500,), 6, 10.0)).float()
    if not np.array_equal(mod.round_bf16_array(v32.double().numpy()),
                          v32.to(torch.bfloat16).double().numpy()):
        fails.append("bf16")
    if not np.array_equal(np.array([mod.round_e4m3(float(v)) for v in v32.double().numpy()]),
                          v32.clamp(-448, 448).to(torch.float8_e4m3fn).double().numpy()):
        fails.append("e4m3")
    # the channel-changing block's shortcut, against a torch composition
    # (rounding off, so that only the arithmetic is compared)
    xb = _rnd((1, 4, 3, 4, 4), 7)
    w1, w2, wsc = _rnd((6, 4, 3, 3, 3), 8, 0.2), _rnd((6, 6, 3, 3, 3), 9, 0.2), _rnd((6, 4, 1, 1, 1), 10)
    b1, b2, bsc = _rnd((6,), 11), _rnd((6,), 12), _rnd((6,), 13)
    g1, g2 = np.abs(_rnd((4,), 14)) + 0.5, np.abs(_rnd((6,), 15)) + 0.5
    y = mod.resblock(xb, w1, b1, g1, w2, b2, g2, round_bf16=False, round_h1=False, w_sc=wsc,
                     b_sc=bsc)
    a0 = _rs(torch.from_numpy(xb), torch.from_numpy(g1)).numpy()
    a1 = _rs(torch.from_numpy(_torch_conv(a0, w1, b1)), torch.from_numpy(g2)).numpy()
    ref = _torch_conv(a1, w2, b2) + F.conv3d(torch.from_numpy(xb), torch.from_numpy(wsc),
                                              torch.from_numpy(bsc)).numpy()
    if not np.allclose(y, ref, rtol=1e-11, atol=1e-11):
        fails.append("shortcut block")
    # the downsample path's spatial step
    xf = _rnd((1, 3, 2, 9, 10), 16)
    w2d = _rnd((4, 3, 3, 3), 17)
    got = mod.conv2d_frames(xf, w2d, b[:4], stride=(2, 2), pad=(0, 1, 0, 1))
    xx = torch.from_numpy(xf).permute(0, 2, 1, 3, 4).reshape(2, 3, 9, 10)
    ref = F.conv2d(F.pad(xx, (0, 1, 0, 1)), torch.from_numpy(w2d), torch.from_numpy(b[:4]),
                   stride=2)
    ref = ref.reshape(1, 2, 4, *ref.shape[2:]).permute(0, 2, 1, 3, 4).numpy()
    if got.shape != ref.shape or not np.allclose(got, ref, rtol=1e-12, atol=1e-12):
        fails.append("downsample")
    return fails


@pytest.fixture(scope="module")
def tmp(tmp_path_factory):
    return str(tmp_path_factory.mktemp("oracle_mutants"))


def test_unmodified_copy_passes_every_check(tmp):
    assert _failures(_load_copy(tmp, "oracle_copy_clean", None)) == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(tmp, name):
    mod = _load_copy(tmp, "oracle_mut_" + str(sorted(MUTANTS).index(name)), MUTANTS[name])
    assert _failures(mod), f"no pin caught: {name}"
