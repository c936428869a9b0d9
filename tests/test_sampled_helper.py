"""The sampled-parity helper used by the full-size GPU tests, checked on
the CPU: fed the oracle's own whole-sequence output it passes, and a
single wrong voxel at a sampled pixel makes it fail."""
import numpy as np
import pytest
import torch

import oracle
from tests.sampled import (border_pixels, check_frames, check_voxels, random_voxels,
                           sample_frame_points)
from video_vae_causal_implicit_b200 import synth


def _case():
    case = synth.conv_case(6, 5, 6, 7, 9, seed_base=40)
    x = synth.ndhwc(case["x"])
    y = oracle.causal_conv3d(synth.ncthw_view(x), case["w"], case["b"].double().numpy())
    y = torch.from_numpy(y).permute(0, 2, 3, 4, 1).contiguous()  # NDHWC, float64
    return x, y, case


def test_helper_accepts_the_oracle_output():
    x, y, case = _case()
    check_frames(x, y, case["w"], case["b"], [0, 1, 2, 5], 6, 7, "helper")


def test_helper_rejects_a_wrong_voxel():
    x, y, case = _case()
    hw = sample_frame_points(7, 9, 6, 7 + 2)  # the pixels frame index 2 samples
    y[0, 2, hw[-1, 0], hw[-1, 1], 3] += 10.0
    with pytest.raises(AssertionError):
        check_frames(x, y, case["w"], case["b"], [0, 1, 2, 5], 6, 7, "helper")


def test_voxel_helper_accepts_the_oracle_and_rejects_a_wrong_voxel():
    x, y, case = _case()
    pts = random_voxels(6, 7, 9, 40, 3)
    pts[0] = border_pixels(7, 9)
    check_voxels(x, y, case["w"], case["b"], pts, "voxels")
    f = max(pts)
    y[0, f, pts[f][0, 0], pts[f][0, 1], 1] += 10.0
    with pytest.raises(AssertionError):
        check_voxels(x, y, case["w"], case["b"], pts, "voxels")


def test_border_pixels_are_the_frame_edge():
    b = border_pixels(5, 7)
    assert len(b) == 2 * 7 + 2 * 3
    assert all(i in (0, 4) or j in (0, 6) for i, j in b)
