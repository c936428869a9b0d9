"""fp64 CPU oracle for the Wan-style causal Conv3D and residual block.

TEST INFRASTRUCTURE ONLY.  Nothing in the product library imports this
package; only the tests, the smoke check and the benchmark's CPU-baseline leg
use it.  It shares no code with the CUDA library.

The arithmetic lives in ``cc3d_oracle.c`` (plain C, fp64, OpenMP).  This
module compiles it with gcc on first use (or from ``build()``) and marshals
numpy / torch CPU arrays into it.  All tensors use the pages' logical layout
[B, C, T, H, W] ("Cosmos3 Wan VAE -- engine size vs context memory",
§10.1); a caller holding channels-last data passes a permuted view and the
strides carry the layout.

Functions (each cites the passage it follows in the C source):
  causal_conv3d         -- §10.3 WanCausalConv3d, bias once
  causal_conv3d_points  -- the same definition at chosen output voxels
  rms_norm              -- §10.2 WanRMS_norm (+ optional SiLU, §10.4)
  resblock              -- §10.4 WanResidualBlock: identity shortcut, or the
                           1x1x1 conv_shortcut when C_in != C_out
  resblock_points       -- the same definition at chosen output voxels
  conv2d_frames         -- §10.5 the downsample path's per-frame ZeroPad2d +
                           stride-2 Conv2d
  round_bf16            -- bfloat16 round-to-nearest-even of one double
  round_e4m3 / quantize_e4m3 / causal_conv3d_fp8
                        -- FP8 E4M3 quantiser and the causal conv on E4M3
                           operands with per-tensor / per-channel scales
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "cc3d_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libcc3d_oracle.so")

_lock = threading.Lock()
_lib = None

F64, F32, BF16 = 0, 1, 2


class _Tensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int),
                ("stride", ctypes.c_longlong * 5)]


def build(force: bool = False) -> str:
    """Compile the oracle into oracle/_build/libcc3d_oracle.so."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
           "-Wall", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.POINTER
            T = P(_Tensor)
            dp = P(ctypes.c_double)
            ip = P(ctypes.c_int)
            i = ctypes.c_int
            lib.orc_causal_conv3d.argtypes = [T, T, i, i, i, i, i, T, i, i, i, i, i, i, dp, dp]
            lib.orc_causal_conv3d_points.argtypes = [T, T, i, i, i, i, i, T, i, i, i, i, i, i, dp,
                                                     i, ip, dp]
            lib.orc_causal_conv3d_s.argtypes = [T, T, i, i, i, i, i, T, i, i, i, i, i, i, i, dp,
                                                dp]
            lib.orc_causal_conv3d_points_s.argtypes = [T, T, i, i, i, i, i, T, i, i, i, i, i, i, i,
                                                       dp, i, ip, dp]
            lib.orc_rms_norm.argtypes = [T, i, i, i, i, i, dp, dp, i, dp]
            lib.orc_resblock.argtypes = [T, T, T, i, i, i, i, i, T, dp, dp, T, dp, dp, i, dp, dp, dp]
            lib.orc_resblock_points.argtypes = [T, T, T, i, i, i, i, i, T, dp, dp, T, dp, dp, i,
                                                i, ip, dp]
            lib.orc_resblock2.argtypes = [T, T, T, i, i, i, i, i, i, T, dp, dp, T, dp, dp, T, dp,
                                          i, i, dp, dp, dp]
            lib.orc_resblock2_points.argtypes = [T, T, T, i, i, i, i, i, i, T, dp, dp, T, dp, dp,
                                                 T, dp, i, i, i, ip, dp]
            lib.orc_conv2d_frames.argtypes = [T, i, i, i, i, i, T, i, i, i, i, i, i, i, i, i,
                                              dp, dp]
            lib.orc_round_e4m3.argtypes = [ctypes.c_double]
            lib.orc_round_e4m3.restype = ctypes.c_double
            lib.orc_round_e4m3_array.argtypes = [dp, ctypes.c_longlong]
            lib.orc_round_e4m3_array.restype = None
            lib.orc_round_bf16.argtypes = [ctypes.c_double]
            lib.orc_round_bf16.restype = ctypes.c_double
            lib.orc_silu.argtypes = [ctypes.c_double]
            lib.orc_silu.restype = ctypes.c_double
            for name in ("orc_causal_conv3d", "orc_causal_conv3d_points", "orc_causal_conv3d_s",
                         "orc_causal_conv3d_points_s", "orc_rms_norm", "orc_resblock",
                         "orc_resblock_points", "orc_resblock2", "orc_resblock2_points",
                         "orc_conv2d_frames"):
                getattr(lib, name).restype = ctypes.c_int
            _lib = lib
    return _lib


def _view(a, keep):
    """Describe a 5-D array (numpy, or torch CPU tensor of float64/float32/
    bfloat16) as an oracle tensor.  Logical dims are (n, c, t, h, w); the
    array's own strides carry the memory layout."""
    if a is None:
        return None
    try:
        import torch
    except ImportError:  # pragma: no cover
        torch = None
    if torch is not None and isinstance(a, torch.Tensor):
        assert a.device.type == "cpu", "oracle inputs live in host memory"
        assert a.dim() == 5
        if a.dtype == torch.bfloat16:
            dt = BF16
        elif a.dtype == torch.float32:
            dt = F32
        elif a.dtype == torch.float64:
            dt = F64
        else:
            raise TypeError(f"unsupported dtype {a.dtype}")
        keep.append(a)
        st = _Tensor()
        st.data = a.data_ptr()
        st.dtype = dt
        for k in range(5):
            st.stride[k] = a.stride(k)
        return st
    a = np.asarray(a)
    assert a.ndim == 5
    if a.dtype == np.float64:
        dt = F64
    elif a.dtype == np.float32:
        dt = F32
    elif a.dtype == np.uint16:
        dt = BF16
    else:
        raise TypeError(f"unsupported dtype {a.dtype}")
    keep.append(a)
    st = _Tensor()
    st.data = a.ctypes.data
    st.dtype = dt
    for k in range(5):
        st.stride[k] = a.strides[k] // a.itemsize
    return st


def _ptr(st):
    return ctypes.byref(st) if st is not None else None


def _dvec(v, keep):
    if v is None:
        return None
    v = np.ascontiguousarray(np.asarray(v, dtype=np.float64).reshape(-1))
    keep.append(v)
    return v.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _shape5(a):
    return tuple(int(s) for s in a.shape)


def causal_conv3d(x, weight, bias=None, cache=None, pad=(1, 1), stride_t=1):
    """y[n,co,t,h,w] = b[co] + sum_{ci,kt,kh,kw} W[co,ci,kt,kh,kw] *
    xt[n,ci,s*t+kt,h+kh-pad_h,w+kw-pad_w], xt = concat(cache or zeros, x) on
    t, s = stride_t.  x: [N,Cin,T,H,W]; weight: [Cout,Cin,KT,KH,KW]; cache:
    [N,Cin,KT-1,H,W] or None.  Returns float64 [N,Cout,(T-1)//s+1,H,W]."""
    lib = _load()
    keep = []
    N, Cin, T, H, W = _shape5(x)
    Cout, Cin2, KT, KH, KW = _shape5(weight)
    assert Cin2 == Cin
    if cache is not None:
        assert _shape5(cache) == (N, Cin, KT - 1, H, W)
    tx, tc, tw = _view(x, keep), _view(cache, keep), _view(weight, keep)
    Tout = (T - 1) // stride_t + 1
    y = np.empty((N, Cout, Tout, H, W), dtype=np.float64)
    rc = lib.orc_causal_conv3d_s(_ptr(tx), _ptr(tc), N, Cin, T, H, W, _ptr(tw), Cout, KT, KH, KW,
                                 pad[0], pad[1], stride_t, _dvec(bias, keep),
                                 y.ctypes.data_as(ctypes.POINTER(ctypes.c_double)))
    if rc != 0:
        raise ValueError(f"orc_causal_conv3d_s failed ({rc})")
    return y


def _pts(points, keep):
    p = np.ascontiguousarray(np.asarray(points, dtype=np.int32).reshape(-1, 4))
    keep.append(p)
    return p.shape[0], p.ctypes.data_as(ctypes.POINTER(ctypes.c_int))


def causal_conv3d_points(x, weight, bias, cache, points, pad=(1, 1), stride_t=1):
    """The causal Conv3D (temporal stride stride_t) at the output voxels in
    ``points`` (rows n,t,h,w; t an output frame).  Returns float64 [P, Cout]."""
    lib = _load()
    keep = []
    N, Cin, T, H, W = _shape5(x)
    Cout, _, KT, KH, KW = _shape5(weight)
    tx, tc, tw = _view(x, keep), _view(cache, keep), _view(weight, keep)
    P, pp = _pts(points, keep)
    y = np.empty((P, Cout), dtype=np.float64)
    rc = lib.orc_causal_conv3d_points_s(_ptr(tx), _ptr(tc), N, Cin, T, H, W, _ptr(tw), Cout, KT,
                                        KH, KW, pad[0], pad[1], stride_t, _dvec(bias, keep), P,
                                        pp, y.ctypes.data_as(ctypes.POINTER(ctypes.c_double)))
    if rc != 0:
        raise ValueError(f"orc_causal_conv3d_points_s failed ({rc})")
    return y


def rms_norm(x, gamma, beta=None, silu=False):
    """Channel RMS_norm over C (+ SiLU).  Returns float64 [N,C,T,H,W]."""
    lib = _load()
    keep = []
    N, C, T, H, W = _shape5(x)
    tx = _view(x, keep)
    y = np.empty((N, C, T, H, W), dtype=np.float64)
    rc = lib.orc_rms_norm(_ptr(tx), N, C, T, H, W, _dvec(gamma, keep), _dvec(beta, keep),
                          1 if silu else 0, y.ctypes.data_as(ctypes.POINTER(ctypes.c_double)))
    if rc != 0:
        raise ValueError(f"orc_rms_norm failed ({rc})")
    return y


def resblock(x, w1, b1, g1, w2, b2, g2, cache1=None, cache2=None, round_bf16=True,
             return_acts=False, w_sc=None, b_sc=None, round_h1=True):
    """WanResidualBlock from C_in = x's channels to C_out = w1's output
    channels.  The shortcut is x itself (w_sc None, C_in == C_out) or the
    1x1x1 conv_shortcut w_sc [C_out, C_in, 1, 1, 1] + b_sc.  round_bf16
    rounds a0 and a1 to bf16; round_h1 rounds conv1's output h1 to bf16
    before its RMS_norm.  Both are on by default: in every block the page's
    module hands a0, h1 and a1 on as bf16 activations ("Cosmos3 Wan VAE",
    §10.4 WanResidualBlock, run in bf16).  Returns y float64
    [N, C_out, T, H, W] (and a0, a1 when return_acts)."""
    lib = _load()
    keep = []
    N, Cin, T, H, W = _shape5(x)
    Cout = _shape5(w1)[0]
    tx, t1, t2 = _view(x, keep), _view(cache1, keep), _view(cache2, keep)
    tw1, tw2, tsc = _view(w1, keep), _view(w2, keep), _view(w_sc, keep)
    y = np.empty((N, Cout, T, H, W), dtype=np.float64)
    a0 = np.empty((N, Cin, T, H, W), dtype=np.float64) if return_acts else None
    a1 = np.empty((N, Cout, T, H, W), dtype=np.float64) if return_acts else None
    dp = ctypes.POINTER(ctypes.c_double)
    rc = lib.orc_resblock2(_ptr(tx), _ptr(t1), _ptr(t2), N, Cin, Cout, T, H, W,
                           _ptr(tw1), _dvec(b1, keep), _dvec(g1, keep),
                           _ptr(tw2), _dvec(b2, keep), _dvec(g2, keep),
                           _ptr(tsc), _dvec(b_sc, keep),
                           1 if round_bf16 else 0, 1 if round_h1 else 0, y.ctypes.data_as(dp),
                           a0.ctypes.data_as(dp) if a0 is not None else None,
                           a1.ctypes.data_as(dp) if a1 is not None else None)
    if rc != 0:
        raise ValueError(f"orc_resblock2 failed ({rc})")
    return (y, a0, a1) if return_acts else y


def resblock_points(x, w1, b1, g1, w2, b2, g2, points, cache1=None, cache2=None,
                    round_bf16=True, w_sc=None, b_sc=None, round_h1=True):
    """The residual block at chosen output voxels.  Returns float64 [P, C_out]."""
    lib = _load()
    keep = []
    N, Cin, T, H, W = _shape5(x)
    Cout = _shape5(w1)[0]
    tx, t1, t2 = _view(x, keep), _view(cache1, keep), _view(cache2, keep)
    tw1, tw2, tsc = _view(w1, keep), _view(w2, keep), _view(w_sc, keep)
    P, pp = _pts(points, keep)
    y = np.empty((P, Cout), dtype=np.float64)
    rc = lib.orc_resblock2_points(_ptr(tx), _ptr(t1), _ptr(t2), N, Cin, Cout, T, H, W,
                                  _ptr(tw1), _dvec(b1, keep), _dvec(g1, keep),
                                  _ptr(tw2), _dvec(b2, keep), _dvec(g2, keep),
                                  _ptr(tsc), _dvec(b_sc, keep),
                                  1 if round_bf16 else 0, 1 if round_h1 else 0, P, pp,
                                  y.ctypes.data_as(ctypes.POINTER(ctypes.c_double)))
    if rc != 0:
        raise ValueError(f"orc_resblock2_points failed ({rc})")
    return y


def conv2d_frames(x, weight, bias=None, stride=(2, 2), pad=(0, 1, 0, 1)):
    """Per-frame ZeroPad2d(pad = (left, right, top, bottom)) + Conv2d with
    `stride` (the downsample path's spatial step).  x: [N, Cin, T, H, W];
    weight: [Cout, Cin, KH, KW].  Returns float64 [N, Cout, T, Ho, Wo],
    Ho = (H + top + bottom - KH) // stride[0] + 1 (likewise Wo)."""
    lib = _load()
    keep = []
    N, Cin, T, H, W = _shape5(x)
    Cout, Cin2, KH, KW = (int(s) for s in weight.shape)
    assert Cin2 == Cin
    l, r, t, b = pad
    Ho = (H + t + b - KH) // stride[0] + 1
    Wo = (W + l + r - KW) // stride[1] + 1
    w5 = weight.reshape(Cout, Cin, 1, KH, KW)
    tx, tw = _view(x, keep), _view(w5, keep)
    y = np.empty((N, Cout, T, Ho, Wo), dtype=np.float64)
    rc = lib.orc_conv2d_frames(_ptr(tx), N, Cin, T, H, W, _ptr(tw), Cout, KH, KW, stride[0],
                               stride[1], l, r, t, b, _dvec(bias, keep),
                               y.ctypes.data_as(ctypes.POINTER(ctypes.c_double)))
    if rc != 0:
        raise ValueError(f"orc_conv2d_frames failed ({rc})")
    return y


def round_e4m3(v: float) -> float:
    """FP8 E4M3 (e4m3fn) round-to-nearest-even of one double, clamped to
    +-448."""
    return _load().orc_round_e4m3(float(v))


def quantize_e4m3(a, scale, quotient="f64"):
    """E4M3 codes of a / scale, returned as their float64 values (so that
    a ~= scale * quantize_e4m3(a, scale)); scale broadcasts against a.
    quotient "f64" divides in float64; "f32" divides the float32 values of
    a and scale in float32 (one correctly rounded IEEE division), the
    precision in which a GPU kernel that quantises in fp32 takes the same
    rounding decision.  Each code is round_e4m3 of its quotient."""
    lib = _load()
    if quotient == "f32":
        v = (np.asarray(a, dtype=np.float32) / np.asarray(scale, dtype=np.float32)).astype(
            np.float64)
    elif quotient == "f64":
        v = np.asarray(a, dtype=np.float64) / np.asarray(scale, dtype=np.float64)
    else:
        raise ValueError(quotient)
    out = np.ascontiguousarray(v, dtype=np.float64).copy()
    lib.orc_round_e4m3_array(out.ctypes.data_as(ctypes.POINTER(ctypes.c_double)), out.size)
    return out


def causal_conv3d_fp8(x, weight, bias, s_x, s_w, cache=None, pad=(1, 1), quotient="f64",
                      stride_t=1):
    """The causal Conv3D on E4M3 operands: x is quantised with the
    per-tensor scale s_x (cache too), weight with the per-output-channel
    scales s_w [Cout]; y = s_x * s_w[co] * conv(q_x, q_w) + b[co], the
    contraction exact in float64.  quotient: as for quantize_e4m3.
    Returns float64 [N, Cout, (T-1)//stride_t+1, H, W]."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(weight, dtype=np.float64)
    s_w = np.asarray(s_w, dtype=np.float64).reshape(-1)
    qx = quantize_e4m3(x, s_x, quotient)
    qw = quantize_e4m3(w, s_w.reshape(-1, 1, 1, 1, 1), quotient)
    qc = (quantize_e4m3(np.asarray(cache, dtype=np.float64), s_x, quotient)
          if cache is not None else None)
    y = causal_conv3d(qx, qw, None, cache=qc, pad=pad, stride_t=stride_t)
    y *= float(s_x) * s_w.reshape(1, -1, 1, 1, 1)
    if bias is not None:
        y += np.asarray(bias, dtype=np.float64).reshape(1, -1, 1, 1, 1)
    return y


def round_bf16(v: float) -> float:
    return _load().orc_round_bf16(float(v))


def silu(z: float) -> float:
    return _load().orc_silu(float(z))


def round_bf16_array(a):
    """Elementwise bfloat16 RNE of a float64 array (loops over round_bf16;
    meant for small arrays)."""
    lib = _load()
    a = np.asarray(a, dtype=np.float64)
    out = np.empty_like(a)
    flat_in, flat_out = a.reshape(-1), out.reshape(-1)
    for k in range(flat_in.size):
        flat_out[k] = lib.orc_round_bf16(float(flat_in[k]))
    return out
