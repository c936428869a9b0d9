"""Failure detection without a GPU fault: every device-side wait in the
kernels is bounded.  A child process runs with a 1 microsecond wait limit
(CC3D_WAIT_LIMIT_US=1), so the pipelines' first real waits run out; the
kernels must record the timeout, drain their own in-flight copies and
MMAs, free tensor memory and return.  The limit governs every entry point,
cc3d_forward_noalloc included, and every kind of wait, the exchange between
the two CTAs that share a wide RMS row included.  The host then sees CC3D_ERR_TIMEOUT
from cc3d_sync_status (once: reading clears it) and the CUDA context stays
usable."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import json, sys, torch
sys.path.insert(0, %r)
from video_vae_causal_implicit_b200 import cc3d, synth
dev = torch.device('cuda', 0)
out = {}
# tensor-core conv, one CTA per tile (not a CTA pair: a pair's drain at
# exit covers the loads its leader armed, which a 1 us limit can outrun)
case = synth.conv_case(96, 96, 2, 30, 52)
plan = cc3d.Plan(case['w'].to(dev), case['b'].to(dev), h=30, w=52, max_t=2)
assert plan.stats().mma_ctas == 1
x = synth.ndhwc(case['x']).to(dev)
y = torch.empty((1, 2, 30, 52, 96), dtype=torch.bfloat16, device=dev)
cache_out = torch.empty((1, 2, 30, 52, 96), dtype=torch.bfloat16, device=dev)
plan.forward(x, y, cache_out=cache_out)
out['umma_first'] = cc3d.cc3d_sync_status(cc3d._stream())
out['umma_second'] = cc3d.cc3d_sync_status(cc3d._stream())
# the same conv through the entry point without device allocation
d = plan.desc
wkeep = case['w'].to(dev)
d.weight = wkeep.data_ptr()
bkeep = case['b'].to(dev)
d.bias = bkeep.data_ptr()
import ctypes
out['noalloc_call'] = cc3d.cc3d_forward_noalloc(d, ctypes.c_void_p(x.data_ptr()), 2, None,
                                                ctypes.c_void_p(y.data_ptr()), None, None, None,
                                                None, cc3d._stream())
out['noalloc_first'] = cc3d.cc3d_sync_status(cc3d._stream())
# an RMS row split over a cluster of two CTAs: each runs its own pipeline,
# and the exchange of the rows' partial sums of squares is bounded too
cw = synth.conv_case(64, 320, 2, 16, 20)
gw = synth.uniform((320,), 0.5, 1.5, 3).to(dev)
pw = cc3d.Plan(cw['w'].to(dev), cw['b'].to(dev), h=16, w=20, max_t=2,
               epi=cc3d.EPI_BIAS_RMS_SILU, gamma=gw)
assert pw.stats().row_ctas == 2
xw = synth.ndhwc(cw['x']).to(dev)
yw = torch.empty((1, 2, 16, 20, 320), dtype=torch.bfloat16, device=dev)
pw.forward(xw, yw)
out['row_split_first'] = cc3d.cc3d_sync_status(cc3d._stream())
# thin first-layer conv
c3 = synth.conv_case(3, 96, 3, 48, 64, x_dist='uniform')
p3 = cc3d.Plan(c3['w'].to(dev), c3['b'].to(dev), h=48, w=64, max_t=3)
x3 = synth.ndhwc(c3['x']).to(dev)
y3 = torch.empty((1, 3, 48, 64, 96), dtype=torch.bfloat16, device=dev)
p3.forward(x3, y3)
out['thin_first'] = cc3d.cc3d_sync_status(cc3d._stream())
# the context still works
torch.cuda.synchronize()
z = (torch.arange(1024, device=dev, dtype=torch.float32) * 2).sum().item()
out['torch_after'] = z
print('RESULT ' + json.dumps(out))
""" % ROOT


def test_bounded_waits_report_timeout_and_leave_context_usable():
    env = dict(os.environ, CC3D_WAIT_LIMIT_US="1")
    proc = subprocess.run([sys.executable, "-c", CHILD], env=env, capture_output=True, text=True,
                          timeout=300)
    assert proc.returncode == 0, proc.stderr[-3000:]
    line = [l for l in proc.stdout.splitlines() if l.startswith("RESULT ")][-1]
    res = json.loads(line[len("RESULT "):])
    TIMEOUT, OK = 7, 0
    assert res["umma_first"] == TIMEOUT
    assert res["umma_second"] == OK          # reading the status clears it
    assert res["noalloc_call"] == OK         # the limit reaches this entry point too
    assert res["noalloc_first"] == TIMEOUT
    assert res["row_split_first"] == TIMEOUT
    assert res["thin_first"] == TIMEOUT
    assert res["torch_after"] == float(sum(range(1024)) * 2)
