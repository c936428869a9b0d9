"""Shared helpers of the parity tests: error metrics and device plumbing.

The tolerance is the one fixed for bf16 operands with fp32 accumulation:
max|d| <= 2e-2 * max|y_ref| and sum|d| / sum|y_ref| <= 2e-3; fp32 plans
must match within 1e-4 relative on both measures.
"""
import numpy as np
import torch

BF16_MAX_REL = 2e-2
BF16_MEAN_REL = 2e-3
FP32_REL = 1e-4


def errors(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    d = np.abs(got - ref)
    max_rel = d.max() / max(np.abs(ref).max(), 1e-30)
    mean_rel = d.sum() / max(np.abs(ref).sum(), 1e-30)
    return float(max_rel), float(mean_rel)


def assert_close_bf16(got, ref, what=""):
    max_rel, mean_rel = errors(got, ref)
    assert np.all(np.isfinite(np.asarray(got, dtype=np.float64))), f"{what}: non-finite output"
    assert max_rel <= BF16_MAX_REL, f"{what}: max|d|/max|ref| = {max_rel:.3e}"
    assert mean_rel <= BF16_MEAN_REL, f"{what}: sum|d|/sum|ref| = {mean_rel:.3e}"
    return max_rel, mean_rel


def assert_close_fp32(got, ref, what=""):
    max_rel, mean_rel = errors(got, ref)
    assert max_rel <= FP32_REL and mean_rel <= FP32_REL, \
        f"{what}: max {max_rel:.3e} mean {mean_rel:.3e}"
    return max_rel, mean_rel


def to_dev(t):
    return t.contiguous().cuda()


def ncthw_np(y_ndhwc):
    """float64 NCTHW numpy copy of a device/host NDHWC tensor."""
    return y_ndhwc.detach().float().cpu().permute(0, 4, 1, 2, 3).double().numpy()


def gather_points(y_ndhwc_cpu, pts):
    p = torch.as_tensor(pts, dtype=torch.long)
    return y_ndhwc_cpu[p[:, 0], p[:, 1], p[:, 2], p[:, 3]].double().numpy()
