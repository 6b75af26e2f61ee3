"""Failure detection without faulting the GPU: bounded waits that run out and
lists/counts/scores that the kernels' own checks catch are reported through
the device status word, and the context stays usable afterwards."""
import ctypes

import numpy as np
import pytest
import torch

import block_sparse_attention_pa_b200 as pa
from block_sparse_attention_pa_b200 import build, synth


@pytest.fixture(scope="module")
def L():
    build.build()
    return pa.lib()


def test_selftest_rejects_bad_timeout(L):
    assert L.pa_selftest_wait_timeout(0, None) == 1
    assert L.pa_selftest_wait_timeout(2_000_000, None) == 1


def small():
    w = synth.small_workload(seqlen=512, heads=4, kv_heads=2, head_dim=64, groups=1, gamma=0.9)
    x = synth.make_inputs(w, device="cuda")
    return w, x["q"], x["k"], x["v"]


def healthy_run():
    w, q, k, v = small()
    o, _ = pa.prefill(q, k, v, 1, pa.DYNAMIC, 0.9)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all()
    assert pa.device_status() == 0


@pytest.mark.gpu
def test_wait_timeout_is_reported_and_context_survives(L):
    assert pa.device_status(clear=True) == 0
    pa.selftest_wait_timeout(2000)          # a wait nothing completes, bounded at 2 ms
    assert pa.device_status(clear=False) == 5  # PA_ERR_TIMEOUT
    assert pa.device_status(clear=True) == 5   # read and clear
    assert pa.device_status() == 0
    healthy_run()


@pytest.mark.gpu
def test_out_of_range_list_entry_and_count_are_flagged(L):
    w, q, k, v = small()
    qp, kp = pa.pool_heads(q, k, 1)
    scores = pa.block_scores(qp, kp, 4, 2)
    mask = pa.build_mask(scores, q, k, 1, pa.DYNAMIC, 0.9)
    torch.cuda.synchronize()
    assert pa.device_status() == 0
    rank = mask.rank.clone()
    qb = 3
    rank[0, 0, qb * (qb + 1) // 2] = qb + 5       # the first entry: a block after the query block
    o = pa.block_sparse_attn(q, k, v, rank, mask.cnt, 1)
    torch.cuda.synchronize()
    assert pa.device_status() == 6                 # PA_ERR_DEVICE_BOUNDS
    cnt = mask.cnt.clone()
    cnt[0, 1, 2] = 99                              # more blocks than the row has
    pa.block_sparse_attn(q, k, v, mask.rank, cnt, 1)
    torch.cuda.synchronize()
    assert pa.device_status() == 6
    healthy_run()


@pytest.mark.gpu
def test_non_finite_score_is_flagged(L):
    w, q, k, v = small()
    qp, kp = pa.pool_heads(q, k, 1)
    scores = pa.block_scores(qp, kp, 4, 2)
    scores[0, 0, 3 * 4 // 2 + 1] = float("nan")
    pa.build_mask(scores, q, k, 1, pa.DYNAMIC, 0.9)
    torch.cuda.synchronize()
    assert pa.device_status() == 7                 # PA_ERR_DEVICE_NONFINITE
    healthy_run()
