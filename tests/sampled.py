"""Sampled parity for full-size causal convs (test helper).

The oracle computes chosen output voxels of frame f from input frames
f-2 .. f only, so each checked frame needs just those frames copied to the
host: output frame f of the whole sequence is output frame (f - s) of the
sub-sequence that starts at s = max(0, f - 2) (before frame 0 the causal
zero padding, before s > 0 nothing the output reads).  This keeps the host
copy at three frames however long the sequence is."""
import numpy as np
import torch

import oracle
from tests.parity import assert_close_bf16
from video_vae_causal_implicit_b200 import synth


def sample_frame_points(h, w, count, seed):
    """The four corners, the centre and `count` seeded pixels: rows (h, w)."""
    g = torch.Generator().manual_seed(seed)
    rand = torch.stack([torch.randint(0, h, (count,), generator=g),
                        torch.randint(0, w, (count,), generator=g)], dim=1).numpy()
    fixed = np.array([[0, 0], [0, w - 1], [h - 1, 0], [h - 1, w - 1], [h // 2, w // 2]])
    return np.concatenate([fixed, rand]).astype(np.int32)


def border_pixels(h, w):
    """Every pixel of the frame's first and last rows and columns (where the
    spatial zero padding enters): rows (h, w)."""
    rows = [(i, j) for i in (0, h - 1) for j in range(w)]
    rows += [(i, j) for j in (0, w - 1) for i in range(1, h - 1)]
    return np.unique(np.array(rows, dtype=np.int32), axis=0)


def all_pixels(h, w):
    hh, ww = np.meshgrid(np.arange(h), np.arange(w), indexing="ij")
    return np.stack([hh.reshape(-1), ww.reshape(-1)], axis=1).astype(np.int32)


def random_voxels(t, h, w, count, seed):
    """`count` seeded output voxels over every frame: {frame: pixels}."""
    g = torch.Generator().manual_seed(seed)
    tt = torch.randint(0, t, (count,), generator=g).numpy()
    hh = torch.randint(0, h, (count,), generator=g).numpy()
    ww = torch.randint(0, w, (count,), generator=g).numpy()
    out = {}
    for f in np.unique(tt):
        sel = tt == f
        out[int(f)] = np.stack([hh[sel], ww[sel]], axis=1).astype(np.int32)
    return out


def check_voxels(x, y, weight, bias, pixels_by_frame, what, pad=(1, 1)):
    """Compare y (NDHWC, any device) with the oracle at the given pixels of
    the given output frames of batch 0: {frame: int32 rows (h, w)}.  Only
    the three input frames each output frame reads are copied to the host;
    the compared outputs are gathered on y's device."""
    got, ref = [], []
    for f, hw in sorted(pixels_by_frame.items()):
        s = max(0, f - 2)
        x_sub = x[:1, s:f + 1].cpu()
        pts = np.concatenate([np.zeros((len(hw), 1), np.int32),
                              np.full((len(hw), 1), f - s, np.int32), hw], axis=1)
        ref.append(oracle.causal_conv3d_points(synth.ncthw_view(x_sub), weight,
                                               bias.double().numpy(), None, pts, pad=pad))
        ih = torch.as_tensor(hw[:, 0], dtype=torch.long, device=y.device)
        iw = torch.as_tensor(hw[:, 1], dtype=torch.long, device=y.device)
        got.append(y[0, f][ih, iw].double().cpu().numpy())
    return assert_close_bf16(np.concatenate(got), np.concatenate(ref), what)


def check_frames(x, y, weight, bias, frames, count, seed, what, pad=(1, 1)):
    """Compare y (NDHWC, any device) with the oracle at sampled pixels of
    the given output frames of batch 0; x is the NDHWC input sequence,
    weight [Co, Ci, 3, kh, kw] and bias [Co] CPU tensors."""
    _, T, H, W, _ = x.shape
    got, ref = [], []
    for k, f in enumerate(frames):
        s = max(0, f - 2)
        x_sub = x[:1, s:f + 1].cpu()
        hw = sample_frame_points(H, W, count, seed + k)
        pts = np.concatenate([np.zeros((len(hw), 1), np.int32),
                              np.full((len(hw), 1), f - s, np.int32), hw], axis=1)
        ref.append(oracle.causal_conv3d_points(synth.ncthw_view(x_sub), weight,
                                               bias.double().numpy(), None, pts, pad=pad))
        yf = y[0, f].cpu()
        got.append(yf[torch.as_tensor(hw[:, 0], dtype=torch.long),
                      torch.as_tensor(hw[:, 1], dtype=torch.long)].double().numpy())
    return assert_close_bf16(np.concatenate(got), np.concatenate(ref), what)
