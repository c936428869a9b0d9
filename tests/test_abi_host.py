"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/cc3d.h declares, and refuses bad descriptors and
arguments before touching the device."""
import ctypes
import os
import re
import subprocess

import pytest

from video_vae_causal_implicit_b200 import build as cbuild
from video_vae_causal_implicit_b200 import cc3d

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "cc3d.h")


@pytest.fixture(scope="module")
def lib():
    cbuild.build()
    return cc3d.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b([a-z_0-9]+)\s*\(", src, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "while")))


def test_header_declares_the_abi():
    names = declared_functions()
    for need in ("cc3d_plan_create", "cc3d_plan_destroy", "cc3d_forward", "rmsnorm_silu",
                 "cc3d_block_create", "cc3d_block_create2", "cc3d_block_destroy",
                 "cc3d_resblock_forward", "cc3d_resblock_forward_fused",
                 "cc3d_sync_status", "cc3d_get_stats", "cc3d_status_string",
                 "cc3d_launch_count"):
        assert need in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", cc3d.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(line.split()[-1] for line in out.splitlines() if " T " in line)
    for name in declared_functions():
        assert name in exported, name
        assert getattr(lib, name) is not None
    # and the binding knows every one of them
    assert set(declared_functions()) <= set(cc3d.SIGNATURES)


def test_forward_host_refuses_bad_calls_on_the_host(lib):
    # no plan, no calls: refused before any CUDA call
    assert cc3d.cc3d_forward_host(None, None, 0, None) == cc3d.ERR_INVALID_ARG
    arr = (cc3d.HostCall * 1)()
    assert cc3d.cc3d_forward_host(None, arr, 1, None) == cc3d.ERR_INVALID_ARG


def test_status_strings(lib):
    for s in range(8):
        assert cc3d.cc3d_status_string(s)
    assert cc3d.cc3d_status_string(99) == "unknown status"


def _desc(**kw):
    d = cc3d.Desc()
    vals = dict(n=1, c_in=64, c_out=64, h=8, w=8, max_t=4, kt=3, kh=3, kw=3, pad_h=1, pad_w=1,
                stride_t=1, stride_h=1, stride_w=1, dil_t=1, dil_h=1, dil_w=1, groups=1,
                dtype=cc3d.BF16, epi=cc3d.EPI_BIAS)
    vals.update(kw)
    for k, v in vals.items():
        setattr(d, k, v)
    d.weight = kw.get("weight", 0x1000)
    return d


@pytest.mark.parametrize("field,value", [("stride_t", 3), ("stride_h", 2), ("groups", 2),
                                         ("dil_t", 2), ("kh", 2), ("pad_h", 0), ("c_out", 40),
                                         ("c_in", 20), ("kt", 5)])
def test_unsupported_descriptors_refused(lib, field, value):
    out = ctypes.c_void_p()
    assert cc3d.cc3d_plan_create(_desc(**{field: value}), out) == cc3d.ERR_UNSUPPORTED
    assert not out.value


@pytest.mark.parametrize("kw", [dict(dtype=cc3d.FP32), dict(c_in=3),
                                dict(c_in=3, kh=1, kw=1, pad_h=0, pad_w=0)])
def test_temporal_stride_only_on_the_tensor_core_path(lib, kw):
    """Stride 2 in time is a bf16 tensor-core descriptor; the fp32 and the
    thin (c_in <= 8) variants refuse it before any device query."""
    out = ctypes.c_void_p()
    assert cc3d.cc3d_plan_create(_desc(stride_t=2, **kw), out) == cc3d.ERR_UNSUPPORTED
    assert not out.value


@pytest.mark.parametrize("kw", [dict(pad_h=1, pad_w=1), dict(kt=3), dict(h=9), dict(w=7),
                                dict(stride_t=2), dict(dtype=cc3d.FP32), dict(c_in=3),
                                dict(epi=cc3d.EPI_BIAS_RMS_SILU, gamma=0x2000),
                                dict(stride_w=1)])
def test_spatial_stride_two_only_for_the_downsample_conv(lib, kw):
    """Stride 2 in H and W is the downsample path's 3x3 conv (kt = 1, no
    leading pad, even frame, bf16 tensor-core channels, no RMS epilogue);
    anything else with it is refused before any device query."""
    base = dict(kt=1, kh=3, kw=3, pad_h=0, pad_w=0, stride_h=2, stride_w=2, h=8, w=8)
    base.update(kw)
    out = ctypes.c_void_p()
    assert cc3d.cc3d_plan_create(_desc(**base), out) == cc3d.ERR_UNSUPPORTED
    assert not out.value


@pytest.mark.parametrize("field,value", [("n", 0), ("h", 0), ("max_t", 0), ("epi", 7)])
def test_invalid_descriptors_refused(lib, field, value):
    out = ctypes.c_void_p()
    assert cc3d.cc3d_plan_create(_desc(**{field: value}), out) == cc3d.ERR_INVALID_ARG


def test_null_weight_and_rms_without_gamma_refused(lib):
    out = ctypes.c_void_p()
    d = _desc()
    d.weight = None
    assert cc3d.cc3d_plan_create(d, out) == cc3d.ERR_INVALID_ARG
    assert cc3d.cc3d_plan_create(_desc(epi=cc3d.EPI_BIAS_RMS_SILU), out) == cc3d.ERR_INVALID_ARG
    assert cc3d.cc3d_plan_create(_desc(epi=cc3d.EPI_BIAS_RMS_SILU, c_out=384, gamma=1),
                                 out) in (cc3d.ERR_UNSUPPORTED, cc3d.ERR_INVALID_ARG)


def test_rmsnorm_argument_checks(lib):
    p = ctypes.c_void_p(0x1000)
    assert cc3d.rmsnorm_silu(None, p, None, 1, 1, 1, 1, 8, p, None, None, None) == \
        cc3d.ERR_INVALID_ARG
    assert cc3d.rmsnorm_silu(p, p, None, 1, 1, 1, 1, 12, p, None, None, None) == \
        cc3d.ERR_UNSUPPORTED
    assert cc3d.rmsnorm_silu(ctypes.c_void_p(0x1008), p, None, 1, 1, 1, 1, 8, p, None, None,
                             None) == cc3d.ERR_ALIGNMENT
    # cache_out overlapping y
    assert cc3d.rmsnorm_silu(ctypes.c_void_p(0x10000), p, None, 1, 1, 4, 4, 8,
                             ctypes.c_void_p(0x20000), None, ctypes.c_void_p(0x20000),
                             None) == cc3d.ERR_ALIAS


def test_forward_and_block_null_handles(lib):
    assert cc3d.cc3d_forward(None, None, 1, None, None, None, None, None, None, None) == \
        cc3d.ERR_INVALID_ARG
    assert cc3d.cc3d_resblock_forward(None, None, 1, None, None, None, None, None, None) == \
        cc3d.ERR_INVALID_ARG
    assert cc3d.cc3d_resblock_forward_fused(None, None, None, 1, None, None, None, None, None,
                                            None, None, None, None, None) == cc3d.ERR_INVALID_ARG
    assert cc3d.cc3d_plan_destroy(None) == cc3d.ERR_INVALID_ARG
    assert cc3d.cc3d_block_destroy(None) == cc3d.ERR_INVALID_ARG
    out = ctypes.c_void_p()
    p = ctypes.c_void_p(0x1000)
    assert cc3d.cc3d_block_create(1, 40, 8, 8, 2, p, p, p, p, p, p, out) == cc3d.ERR_UNSUPPORTED
    assert cc3d.cc3d_block_create(1, 64, 8, 8, 0, p, p, p, p, p, p, out) == cc3d.ERR_INVALID_ARG


def test_channel_changing_block_validation(lib):
    out = ctypes.c_void_p()
    p = ctypes.c_void_p(0x1000)
    # c_in != c_out needs the conv_shortcut; a shortcut bias needs its weights
    assert cc3d.cc3d_block_create2(1, 64, 128, 8, 8, 2, p, p, p, p, p, p, None, None, out) == \
        cc3d.ERR_INVALID_ARG
    assert cc3d.cc3d_block_create2(1, 64, 64, 8, 8, 2, p, p, p, p, p, p, None, p, out) == \
        cc3d.ERR_INVALID_ARG
    assert cc3d.cc3d_block_create2(1, 64, 128, 8, 8, 2, p, p, None, p, p, p, p, p, out) == \
        cc3d.ERR_INVALID_ARG
    # channel counts no kernel covers
    assert cc3d.cc3d_block_create2(1, 48, 64, 8, 8, 2, p, p, p, p, p, p, p, p, out) == \
        cc3d.ERR_UNSUPPORTED
    assert cc3d.cc3d_block_create2(1, 64, 2048, 8, 8, 2, p, p, p, p, p, p, p, p, out) == \
        cc3d.ERR_UNSUPPORTED
    assert not out.value


def test_no_gpu_means_unsupported_not_a_fallback(lib):
    """A valid descriptor on a machine without an sm_100 GPU is refused:
    there is no CPU path to fall back to."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("GPU present")
    out = ctypes.c_void_p()
    assert cc3d.cc3d_plan_create(_desc(), out) == cc3d.ERR_UNSUPPORTED
    assert cc3d.cc3d_launch_count() == 0

def test_noalloc_validation_before_any_device_work(lib):
    """cc3d_forward_noalloc refuses bad calls on the host, before touching
    its scratch or the GPU (so these run without one)."""
    p = ctypes.c_void_p(0x10000)
    odd = ctypes.c_void_p(0x10008)
    f = cc3d.cc3d_forward_noalloc
    assert f(_desc(), None, 1, None, p, None, None, None, None, None) == cc3d.ERR_INVALID_ARG
    assert f(_desc(), p, 5, None, p, None, None, None, None, None) == cc3d.ERR_INVALID_ARG  # t > max_t
    assert f(_desc(epi=cc3d.EPI_BIAS_RESIDUAL), p, 1, None, p, None, None, None, None,
             None) == cc3d.ERR_INVALID_ARG  # residual epilogue without a residual
    assert f(_desc(stride_h=2, stride_w=2), p, 1, None, p, None, None, None, None, None) == \
        cc3d.ERR_UNSUPPORTED
    assert f(_desc(c_in=48), p, 1, None, p, None, None, None, None, None) == cc3d.ERR_UNSUPPORTED
    assert f(_desc(dtype=cc3d.FP32), p, 1, None, p, None, None, None, None, None) == \
        cc3d.ERR_UNSUPPORTED
    assert f(_desc(c_in=1024, c_out=1024), p, 1, None, p, None, None, None, None, None) == \
        cc3d.ERR_TOO_LARGE  # 56 MB of weights against an 8 MiB scratch
    assert f(_desc(), odd, 1, None, p, None, None, None, None, None) == cc3d.ERR_ALIGNMENT
