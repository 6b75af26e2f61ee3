"""PA_NVTX=1 wraps every launch in an NVTX range (a host-side annotation for
profilers): the results must not change.  The variable is read once per
process, so the annotated run is a child process."""
import os
import subprocess
import sys

import pytest
import torch

import block_sparse_attention_pa_b200 as pa
from block_sparse_attention_pa_b200 import build, synth

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys, torch
sys.path.insert(0, sys.argv[1])
import block_sparse_attention_pa_b200 as pa
from block_sparse_attention_pa_b200 import synth
w = synth.small_workload(seqlen=1024, heads=8, kv_heads=2, head_dim=128, groups=1, gamma=0.9, seed=21)
x = synth.make_inputs(w, device="cuda")
o, m = pa.prefill(x["q"], x["k"], x["v"], 1, pa.DYNAMIC, 0.9)
torch.cuda.synchronize()
assert pa.device_status() == 0
torch.save({"o": o.cpu(), "cnt": m.cnt.cpu(), "rank": m.rank.cpu()}, sys.argv[2])
"""


def test_nvtx_ranges_leave_results_unchanged(tmp_path):
    build.build()
    out = tmp_path / "nvtx.pt"
    env = dict(os.environ, PA_NVTX="1")
    r = subprocess.run([sys.executable, "-c", CHILD, ROOT, str(out)], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    got = torch.load(out)
    w = synth.small_workload(seqlen=1024, heads=8, kv_heads=2, head_dim=128, groups=1, gamma=0.9, seed=21)
    x = synth.make_inputs(w, device="cuda")
    o, m = pa.prefill(x["q"], x["k"], x["v"], 1, pa.DYNAMIC, 0.9)
    torch.cuda.synchronize()
    assert pa.device_status() == 0
    assert torch.equal(got["o"], o.cpu()) and torch.equal(got["cnt"], m.cnt.cpu())
    assert torch.equal(got["rank"], m.rank.cpu())
