"""ctypes binding of libcc3d.so (the C ABI in include/cc3d.h).

Argument marshalling only: every step of the computation runs in the CUDA
library.  The raw entry points keep the C names (``cc3d_plan_create``,
``cc3d_forward``, ``rmsnorm_silu``, ``cc3d_block_create``,
``cc3d_resblock_forward``, ...).  ``Plan`` and ``Block`` wrap them for
torch tensors: they pass ``data_ptr()`` and the current CUDA stream, nothing
else.  Loading fails loudly when the library is missing -- there is no CPU
path.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libcc3d.so")

(OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_ALIGNMENT, ERR_ALIAS, ERR_OOM, ERR_CUDA, ERR_TIMEOUT,
 ERR_TOO_LARGE) = range(9)
BF16, FP32, FP8_E4M3 = 0, 1, 2
EPI_BIAS, EPI_BIAS_RESIDUAL, EPI_BIAS_RMS_SILU, EPI_BIAS_RMS = 0, 1, 2, 3
VARIANT_NONE, VARIANT_UMMA, VARIANT_THIN, VARIANT_FP32 = 0, 1, 2, 3

_STATUS_NAMES = {0: "CC3D_OK", 1: "CC3D_ERR_INVALID_ARG", 2: "CC3D_ERR_UNSUPPORTED",
                 3: "CC3D_ERR_ALIGNMENT", 4: "CC3D_ERR_ALIAS", 5: "CC3D_ERR_OOM",
                 6: "CC3D_ERR_CUDA", 7: "CC3D_ERR_TIMEOUT", 8: "CC3D_ERR_TOO_LARGE"}


class Cc3dError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__(f"{where}: {_STATUS_NAMES.get(status, status)} "
                         f"({lib().cc3d_status_string(status).decode()})")


class Desc(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "n", "c_in", "c_out", "h", "w", "max_t", "kt", "kh", "kw", "pad_h", "pad_w",
        "stride_t", "stride_h", "stride_w", "dil_t", "dil_h", "dil_w", "groups", "dtype")] + [
        ("weight", ctypes.c_void_p), ("bias", ctypes.c_void_p), ("epi", ctypes.c_int),
        ("gamma", ctypes.c_void_p), ("beta", ctypes.c_void_p), ("w_scale", ctypes.c_void_p),
        ("x_scale", ctypes.c_float)]


class Stats(ctypes.Structure):
    _fields_ = [("calls", ctypes.c_uint64), ("rejected", ctypes.c_uint64),
                ("tiles", ctypes.c_uint64), ("variant", ctypes.c_int), ("tile_h", ctypes.c_int),
                ("tile_w", ctypes.c_int), ("n_tile", ctypes.c_int), ("k_chunk", ctypes.c_int),
                ("k_split", ctypes.c_int), ("mma_ctas", ctypes.c_int),
                ("w_resident", ctypes.c_int), ("row_ctas", ctypes.c_int),
                ("one_frame_mma_ctas", ctypes.c_int), ("one_frame_n_tile", ctypes.c_int),
                ("second_tile_calls", ctypes.c_uint64)]


class HostCall(ctypes.Structure):
    _fields_ = [("x_host", ctypes.c_void_p), ("t", ctypes.c_int), ("cache_in", ctypes.c_void_p),
                ("cache_out", ctypes.c_void_p), ("residual", ctypes.c_void_p),
                ("y_host", ctypes.c_void_p)]


# name -> (restype, argtypes)
_VP, _I = ctypes.c_void_p, ctypes.c_int
SIGNATURES = {
    "cc3d_plan_create": (_I, [ctypes.POINTER(Desc), ctypes.POINTER(_VP)]),
    "cc3d_plan_destroy": (_I, [_VP]),
    "cc3d_forward": (_I, [_VP, _VP, _I, _VP, _VP, _VP, _VP, _VP, _VP, _VP]),
    "cc3d_forward_host": (_I, [_VP, ctypes.POINTER(HostCall), _I, _VP]),
    "rmsnorm_silu": (_I, [_VP, _VP, _VP, _I, _I, _I, _I, _I, _VP, _VP, _VP, _VP]),
    "rms_norm": (_I, [_VP, _VP, _VP, _I, _I, _I, _I, _I, _VP, _VP, _VP, _VP]),
    "cc3d_quantize_e4m3": (_I, [_VP, ctypes.c_size_t, ctypes.c_float, _VP, _VP]),
    "cc3d_block_create": (_I, [_I, _I, _I, _I, _I, _VP, _VP, _VP, _VP, _VP, _VP,
                               ctypes.POINTER(_VP)]),
    "cc3d_block_create2": (_I, [_I, _I, _I, _I, _I, _I, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP,
                                ctypes.POINTER(_VP)]),
    "cc3d_block_destroy": (_I, [_VP]),
    "cc3d_resblock_forward": (_I, [_VP, _VP, _I, _VP, _VP, _VP, _VP, _VP, _VP]),
    "cc3d_resblock_forward_fused": (_I, [_VP, _VP, _VP, _I, _VP, _VP, _VP, _VP, _VP, _VP, _VP,
                                         _VP, _VP, _VP]),
    "cc3d_sync_status": (_I, [_VP]),
    "cc3d_get_stats": (_I, [_VP, ctypes.POINTER(Stats)]),
    "cc3d_status_string": (ctypes.c_char_p, [_I]),
    "cc3d_launch_count": (ctypes.c_uint64, []),
    "cc3d_forward_noalloc": (_I, [ctypes.POINTER(Desc), _VP, _I, _VP, _VP, _VP, _VP, _VP, _VP,
                                  _VP]),
}

_lib = None


def lib():
    """Load libcc3d.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m video_vae_causal_implicit_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def check(status, where):
    if status != OK:
        raise Cc3dError(status, where)


# Raw C entry points, same names as the header.
def cc3d_plan_create(desc, out):
    return lib().cc3d_plan_create(ctypes.byref(desc), ctypes.byref(out))


def cc3d_plan_destroy(plan):
    return lib().cc3d_plan_destroy(plan)


def cc3d_forward(plan, x, t, cache_in, y, cache_out, residual, next_cache_in, next_cache_out,
                 stream):
    return lib().cc3d_forward(plan, x, t, cache_in, y, cache_out, residual, next_cache_in,
                              next_cache_out, stream)


def cc3d_forward_host(plan, calls, ncalls, stream):
    return lib().cc3d_forward_host(plan, calls, ncalls, stream)


def rmsnorm_silu(x, gamma, beta, n, t, h, w, c, y, cache_in, cache_out, stream):
    return lib().rmsnorm_silu(x, gamma, beta, n, t, h, w, c, y, cache_in, cache_out, stream)


def rms_norm(x, gamma, beta, n, t, h, w, c, y, cache_in, cache_out, stream):
    return lib().rms_norm(x, gamma, beta, n, t, h, w, c, y, cache_in, cache_out, stream)


def cc3d_block_create(n, c, h, w, max_t, w1, b1, g1, w2, b2, g2, out):
    return lib().cc3d_block_create(n, c, h, w, max_t, w1, b1, g1, w2, b2, g2, ctypes.byref(out))


def cc3d_block_create2(n, c_in, c_out, h, w, max_t, w1, b1, g1, w2, b2, g2, w_sc, b_sc, out):
    return lib().cc3d_block_create2(n, c_in, c_out, h, w, max_t, w1, b1, g1, w2, b2, g2, w_sc,
                                    b_sc, ctypes.byref(out))


def cc3d_block_destroy(block):
    return lib().cc3d_block_destroy(block)


def cc3d_resblock_forward(block, x, t, cache1_in, cache2_in, y, cache1_out, cache2_out, stream):
    return lib().cc3d_resblock_forward(block, x, t, cache1_in, cache2_in, y, cache1_out,
                                       cache2_out, stream)


def cc3d_resblock_forward_fused(block, x, a0_in, t, cache1_in, cache2_in, y, cache1_out,
                                cache2_out, g_next, a0_next, a0_next_cache_in, a0_next_cache_out,
                                stream):
    return lib().cc3d_resblock_forward_fused(block, x, a0_in, t, cache1_in, cache2_in, y,
                                             cache1_out, cache2_out, g_next, a0_next,
                                             a0_next_cache_in, a0_next_cache_out, stream)


def cc3d_sync_status(stream):
    return lib().cc3d_sync_status(stream)


def cc3d_get_stats(plan, out):
    return lib().cc3d_get_stats(plan, ctypes.byref(out))


def cc3d_status_string(status):
    return lib().cc3d_status_string(status).decode()


def cc3d_launch_count():
    return int(lib().cc3d_launch_count())


def cc3d_forward_noalloc(desc, x, t, cache_in, y, cache_out, residual, next_cache_in,
                         next_cache_out, stream):
    """The conv without a plan and without device allocation (scratch is a
    fixed array inside the library; see include/cc3d.h)."""
    return lib().cc3d_forward_noalloc(ctypes.byref(desc), x, t, cache_in, y, cache_out, residual,
                                      next_cache_in, next_cache_out, stream)


# ---- torch conveniences (pointers + current stream only) --------------------------

def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


class Plan:
    """A causal conv plan.  ``weight`` is [C_out, C_in, kt, kh, kw] on the
    device (bf16, or fp32 for dtype=FP32); bias/gamma/beta fp32 [C_out]."""

    def __init__(self, weight, bias=None, *, n=1, h, w, max_t, epi=EPI_BIAS, gamma=None,
                 beta=None, dtype=BF16, pad=None, stride_t=1, stride_hw=1, w_scale=None,
                 x_scale=0.0):
        co, ci, kt, kh, kw = (int(s) for s in weight.shape)
        d = Desc()
        d.n, d.c_in, d.c_out, d.h, d.w, d.max_t = n, ci, co, h, w, max_t
        d.kt, d.kh, d.kw = kt, kh, kw
        d.pad_h, d.pad_w = pad if pad is not None else (kh // 2, kw // 2)
        d.stride_t = stride_t
        d.stride_h = d.stride_w = stride_hw
        d.dil_t = d.dil_h = d.dil_w = 1
        d.groups = 1
        d.dtype = dtype
        weight = weight.contiguous()
        d.weight = weight.data_ptr()
        d.bias = bias.data_ptr() if bias is not None else None
        d.epi = epi
        d.gamma = gamma.data_ptr() if gamma is not None else None
        d.beta = beta.data_ptr() if beta is not None else None
        d.w_scale = w_scale.data_ptr() if w_scale is not None else None
        d.x_scale = float(x_scale)
        self.desc = d
        self.handle = ctypes.c_void_p()
        check(cc3d_plan_create(d, self.handle), "cc3d_plan_create")

    def forward(self, x, y, t=None, cache_in=None, cache_out=None, residual=None,
                next_cache_in=None, next_cache_out=None, stream=None):
        t = int(x.shape[1]) if t is None else t
        check(cc3d_forward(self.handle, _ptr(x), t, _ptr(cache_in), _ptr(y), _ptr(cache_out),
                           _ptr(residual), _ptr(next_cache_in), _ptr(next_cache_out),
                           _stream(stream)), "cc3d_forward")
        return y

    def forward_host(self, calls, stream=None):
        """cc3d_forward_host: ``calls`` is a list of dicts with x_host and
        y_host (host tensors, pinned for overlap) and optionally t,
        cache_in, cache_out, residual (device tensors)."""
        arr = (HostCall * len(calls))()
        for i, c in enumerate(calls):
            arr[i].x_host = c["x_host"].data_ptr()
            arr[i].t = int(c.get("t", c["x_host"].shape[1]))
            for k in ("cache_in", "cache_out", "residual"):
                v = c.get(k)
                setattr(arr[i], k, v.data_ptr() if v is not None else None)
            arr[i].y_host = c["y_host"].data_ptr()
        check(cc3d_forward_host(self.handle, arr, len(calls), _stream(stream)),
              "cc3d_forward_host")

    def stats(self):
        s = Stats()
        check(cc3d_get_stats(self.handle, s), "cc3d_get_stats")
        return s

    def close(self):
        if self.handle:
            cc3d_plan_destroy(self.handle)
            self.handle = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class Block:
    """Residual block, 3x3x3 convs, from C_in = w1.shape[1] to C_out =
    w1.shape[0] channels; w_sc [C_out, C_in, 1, 1, 1] (+ b_sc) is the
    1x1x1 conv_shortcut (None: the identity shortcut, C_in == C_out).

    In a chain of blocks, ``forward(..., g_next=next_block.g1, a0_next=A)``
    also writes the next block's first activation SiLU(RMS_norm(y; g_next))
    to A (from this block's conv2 epilogue), and the next block takes it as
    ``forward(y, ..., a0_in=A)``, skipping its own first norm."""

    def __init__(self, w1, b1, g1, w2, b2, g2, *, n=1, h, w, max_t, w_sc=None, b_sc=None):
        self.c_out, self.c_in = int(w1.shape[0]), int(w1.shape[1])
        self.c = self.c_out
        keep = [None if t is None else t.contiguous() for t in (w1, b1, g1, w2, b2, g2, w_sc, b_sc)]
        self.g1 = keep[2].float().contiguous()  # (the previous block's g_next)
        self.handle = ctypes.c_void_p()
        check(cc3d_block_create2(n, self.c_in, self.c_out, h, w, max_t,
                                 *(_ptr(t) for t in keep), self.handle),
              "cc3d_block_create2")

    def forward(self, x, y, t=None, cache1_in=None, cache2_in=None, cache1_out=None,
                cache2_out=None, stream=None, a0_in=None, g_next=None, a0_next=None,
                a0_next_cache_in=None, a0_next_cache_out=None):
        t = int(x.shape[1]) if t is None else t
        if a0_in is None and g_next is None and a0_next is None:
            check(cc3d_resblock_forward(self.handle, _ptr(x), t, _ptr(cache1_in),
                                        _ptr(cache2_in), _ptr(y), _ptr(cache1_out),
                                        _ptr(cache2_out), _stream(stream)),
                  "cc3d_resblock_forward")
            return y
        check(cc3d_resblock_forward_fused(self.handle, _ptr(x), _ptr(a0_in), t, _ptr(cache1_in),
                                          _ptr(cache2_in), _ptr(y), _ptr(cache1_out),
                                          _ptr(cache2_out), _ptr(g_next), _ptr(a0_next),
                                          _ptr(a0_next_cache_in), _ptr(a0_next_cache_out),
                                          _stream(stream)),
              "cc3d_resblock_forward_fused")
        return y

    def close(self):
        if self.handle:
            cc3d_block_destroy(self.handle)
            self.handle = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def rms_silu(x, gamma, y, beta=None, cache_in=None, cache_out=None, stream=None):
    n, t, h, w, c = (int(s) for s in x.shape)
    check(rmsnorm_silu(_ptr(x), _ptr(gamma), _ptr(beta), n, t, h, w, c, _ptr(y), _ptr(cache_in),
                       _ptr(cache_out), _stream(stream)), "rmsnorm_silu")
    return y


def rms(x, gamma, y, beta=None, cache_in=None, cache_out=None, stream=None):
    """The RMS_norm alone (no SiLU)."""
    n, t, h, w, c = (int(s) for s in x.shape)
    check(rms_norm(_ptr(x), _ptr(gamma), _ptr(beta), n, t, h, w, c, _ptr(y), _ptr(cache_in),
                   _ptr(cache_out), _stream(stream)), "rms_norm")
    return y


def quantize_e4m3(x, scale, q, stream=None):
    """q (uint8, same element count as the bf16 tensor x) = E4M3(x / scale)."""
    check(lib().cc3d_quantize_e4m3(_ptr(x), x.numel(), float(scale), _ptr(q), _stream(stream)),
          "cc3d_quantize_e4m3")
    return q


def sync_status(stream=None):
    check(cc3d_sync_status(_stream(stream)), "cc3d_sync_status")
