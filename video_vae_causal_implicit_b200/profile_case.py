"""Run one named workload a few times, for profiler captures (ncu).

    python -m video_vae_causal_implicit_b200.profile_case --case NAME [--reps R]

Cases (seeded synthetic inputs, generated on the device):
  c2      384 -> 384 causal conv, whole sequence, x[1,384,5,30,52]
  c2s     the same as 5 one-frame chunks with a 2-frame cache, planned for
          one-frame calls (max_t = 1)
  c2c     the 5 one-frame chunks with the whole-sequence plan (max_t = 5), as
          in the benchmark step
  c3a     3 -> 96 causal conv on x[1,3,17,480,832]
  c3b     96 -> 96 causal conv on x[1,96,17,480,832]
  c4      the residual block on x[1,192,9,240,416]
  c4s     the residual block on a 3-frame slice x[1,192,3,240,416]
  c5big   384 -> 384, one frame of 360 x 640 with a 2-frame cache
  tc192   the downsample path's time_conv: 192 -> 192, kernel (3, 1, 1),
          stride 2 in time, x[1,192,17,120,208] (9 output frames)
  tc384   the same at 384 channels on x[1,384,9,60,104] (5 output frames)
  ds96    the downsample path's per-frame ZeroPad2d(0,1,0,1) + 3x3 stride-2
          conv, 96 channels, x[1,96,17,480,832] -> 240 x 416
  blk96   the encoder's channel-changing block 96 -> 192 (conv_shortcut fused
          into conv2) on x[1,96,17,240,416]
  blk384  a 384-channel residual block on x[1,384,5,60,104] (conv1's RMS_norm
          + SiLU in its epilogue, each 192-channel half of a row on one CTA
          of a two-CTA cluster)
  c2f8    the 384 -> 384 conv of c2 on FP8 E4M3 operands
  c4chain two c4 blocks in a row, the first one's conv2 epilogue also
          writing the second one's SiLU(RMS_norm(y)) (launches: rmsnorm,
          conv1, conv2 with the hand-over; conv1, conv2)
Prints nothing but a final "ok"; timing comes from the profiler.
"""
from __future__ import annotations

import argparse

import torch

from . import cc3d, synth


def _rand(shape, dev, seed=0):
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    return torch.randn(shape, generator=g, device=dev).to(torch.bfloat16)


def build_case(name, dev):
    if name in ("c2", "c2s", "c2c"):
        c, T, H, W = 384, 5, 30, 52
    elif name == "c3a":
        c, T, H, W = 3, 17, 480, 832
    elif name == "c3b":
        c, T, H, W = 96, 17, 480, 832
    elif name in ("c4", "c4s", "c4chain"):
        c, T, H, W = 192, (3 if name == "c4s" else 9), 240, 416
    elif name == "c5big":
        c, T, H, W = 384, 1, 360, 640
    elif name == "tc192":
        c, T, H, W = 192, 17, 120, 208
    elif name == "tc384":
        c, T, H, W = 384, 9, 60, 104
    elif name == "ds96":
        c, T, H, W = 96, 17, 480, 832
    elif name == "blk96":
        c, T, H, W = 96, 17, 240, 416
    elif name == "blk384":
        c, T, H, W = 384, 5, 60, 104
    elif name == "c2f8":
        c, T, H, W = 384, 5, 30, 52
    else:
        raise SystemExit(f"unknown case {name}")
    x = _rand((1, T, H, W, c), dev)
    if name in ("c4", "c4s"):
        w1 = synth.kaiming_uniform(c, c, (3, 3, 3), 1).to(dev)
        w2 = synth.kaiming_uniform(c, c, (3, 3, 3), 4).to(dev)
        b1 = synth.uniform((c,), -0.1, 0.1, 2).to(dev)
        b2 = synth.uniform((c,), -0.1, 0.1, 5).to(dev)
        g1 = synth.uniform((c,), 0.5, 1.5, 3).to(dev)
        g2 = synth.uniform((c,), 0.5, 1.5, 6).to(dev)
        blk = cc3d.Block(w1, b1, g1, w2, b2, g2, h=H, w=W, max_t=T)
        y = torch.empty_like(x)
        return lambda: blk.forward(x, y), [blk]
    if name == "c4chain":
        blks = []
        for s in (0, 10):
            blks.append(cc3d.Block(synth.kaiming_uniform(c, c, (3, 3, 3), 1 + s).to(dev),
                                   synth.uniform((c,), -0.1, 0.1, 2 + s).to(dev),
                                   synth.uniform((c,), 0.5, 1.5, 3 + s).to(dev),
                                   synth.kaiming_uniform(c, c, (3, 3, 3), 4 + s).to(dev),
                                   synth.uniform((c,), -0.1, 0.1, 5 + s).to(dev),
                                   synth.uniform((c,), 0.5, 1.5, 6 + s).to(dev),
                                   h=H, w=W, max_t=T))
        y0, y1, a1 = torch.empty_like(x), torch.empty_like(x), torch.empty_like(x)

        def run():
            blks[0].forward(x, y0, g_next=blks[1].g1, a0_next=a1)
            blks[1].forward(y0, y1, a0_in=a1)
        return run, blks
    if name == "ds96":
        wt = synth.kaiming_uniform(c, c, (1, 3, 3), 1).to(dev)
        b = synth.uniform((c,), -0.1, 0.1, 2).to(dev)
        plan = cc3d.Plan(wt, b, h=H, w=W, max_t=T, pad=(0, 0), stride_hw=2)
        y = torch.empty((1, T, H // 2, W // 2, c), dtype=torch.bfloat16, device=dev)
        return (lambda: plan.forward(x, y)), [plan]
    if name == "blk96":
        co = 192
        wts = dict(w1=synth.kaiming_uniform(co, c, (3, 3, 3), 1),
                   b1=synth.uniform((co,), -0.1, 0.1, 2), g1=synth.uniform((c,), 0.5, 1.5, 3),
                   w2=synth.kaiming_uniform(co, co, (3, 3, 3), 4),
                   b2=synth.uniform((co,), -0.1, 0.1, 5), g2=synth.uniform((co,), 0.5, 1.5, 6),
                   w_sc=synth.kaiming_uniform(co, c, (1, 1, 1), 7),
                   b_sc=synth.uniform((co,), -0.1, 0.1, 8))
        blk = cc3d.Block(**{k: v.to(dev) for k, v in wts.items()}, h=H, w=W, max_t=T)
        y = torch.empty((1, T, H, W, co), dtype=torch.bfloat16, device=dev)
        return (lambda: blk.forward(x, y)), [blk]
    if name == "blk384":
        wts = dict(w1=synth.kaiming_uniform(c, c, (3, 3, 3), 1),
                   b1=synth.uniform((c,), -0.1, 0.1, 2), g1=synth.uniform((c,), 0.5, 1.5, 3),
                   w2=synth.kaiming_uniform(c, c, (3, 3, 3), 4),
                   b2=synth.uniform((c,), -0.1, 0.1, 5), g2=synth.uniform((c,), 0.5, 1.5, 6))
        blk = cc3d.Block(**{k: v.to(dev) for k, v in wts.items()}, h=H, w=W, max_t=T)
        y = torch.empty_like(x)
        return (lambda: blk.forward(x, y)), [blk]
    if name == "c2f8":
        wt = synth.kaiming_uniform(c, c, (3, 3, 3), 1).to(dev)
        s_w = (wt.float().abs().reshape(c, -1).amax(dim=1) / 448.0).contiguous()
        s_x = float(x.float().abs().max()) / 448.0
        plan = cc3d.Plan(wt, synth.uniform((c,), -0.1, 0.1, 2).to(dev), h=H, w=W, max_t=T,
                         dtype=cc3d.FP8_E4M3, w_scale=s_w, x_scale=s_x)
        xq = torch.empty(x.shape, dtype=torch.uint8, device=dev)
        cc3d.quantize_e4m3(x, s_x, xq)
        y = torch.empty_like(x)
        return (lambda: plan.forward(xq, y)), [plan, xq]
    if name in ("tc192", "tc384"):
        wt = synth.kaiming_uniform(c, c, (3, 1, 1), 1).to(dev)
        b = synth.uniform((c,), -0.1, 0.1, 2).to(dev)
        plan = cc3d.Plan(wt, b, h=H, w=W, max_t=T, stride_t=2)
        y = torch.empty((1, (T - 1) // 2 + 1, H, W, c), dtype=torch.bfloat16, device=dev)
        return (lambda: plan.forward(x, y)), [plan]
    cout = 96 if name == "c3a" else c
    wt = synth.kaiming_uniform(cout, c, (3, 3, 3), 1).to(dev)
    b = synth.uniform((cout,), -0.1, 0.1, 2).to(dev)
    if name in ("c2s", "c2c"):
        plan = cc3d.Plan(wt, b, h=H, w=W, max_t=1 if name == "c2s" else T)
        ys = [torch.empty((1, 1, H, W, cout), dtype=torch.bfloat16, device=dev) for _ in range(T)]
        cb = [torch.empty((1, 2, H, W, c), dtype=torch.bfloat16, device=dev) for _ in range(2)]

        def run():
            cache = None
            for k in range(T):
                plan.forward(x[:, k:k + 1], ys[k], t=1, cache_in=cache, cache_out=cb[k % 2])
                cache = cb[k % 2]
        return run, [plan]
    plan = cc3d.Plan(wt, b, h=H, w=W, max_t=T)
    y = torch.empty((1, T, H, W, cout), dtype=torch.bfloat16, device=dev)
    cache = _rand((1, 2, H, W, c), dev, 9) if name == "c5big" else None
    return (lambda: plan.forward(x, y, cache_in=cache)), [plan]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--case", required=True)
    ap.add_argument("--reps", type=int, default=3)
    args = ap.parse_args()
    dev = torch.device("cuda", 0)
    run, keep = build_case(args.case, dev)
    for _ in range(args.reps):
        run()
    torch.cuda.synchronize()
    cc3d.sync_status()
    del keep
    print("ok")


if __name__ == "__main__":
    main()
