"""GPU parity of BLASST's running-max block skip inside the block-sparse
attention kernel (pa_block_sparse_attn_skip, pa_prefill with
pa_budget.skip_threshold), against the oracle's o7 on the same seeded inputs.

Acceptance:
  decisions  the kernel's skipped blocks equal the oracle's fp64 decisions,
             except for blocks whose margin lies within 1e-3 (log2 units) of
             the threshold, where the fp32 logits of the tensor core may
             decide either way
  O, LSE     against the oracle run with the kernel's own decisions:
             max-abs <= 2e-2, mean-abs <= 2e-3; |LSE| < 1e-3
  lambda = 0 and a threshold that skips nothing: bit-identical to the plain
             kernel (the skip variant changes no arithmetic of a kept block)
Inputs: the seeded generator with a strong attention sink (sink_logit), so
that blocks are both skipped and kept.
"""
import numpy as np
import pytest
import torch

import oracle
import block_sparse_attention_pa_b200 as pa
from block_sparse_attention_pa_b200 import build, synth

pytestmark = pytest.mark.gpu

MARGIN = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    pa.lib()
    assert pa.device_status() == 0


CASES = [
    # name,                N,    H, Hkv, d,   G, mode,               gamma, frac, lam,  B
    ("all_d64_lam0.5",     1024, 4, 2,  64,  1, pa.ALL,             0.0,   0,    0.5,  1),
    ("all_d128_lam0.1",    768,  4, 2,  128, 1, pa.ALL,             0.0,   0,    0.1,  1),
    ("dyn_d128_lam0.3",    1024, 8, 2,  128, 2, pa.DYNAMIC,         0.95,  0,    0.3,  1),
    ("fixed_odd_heads",    896,  6, 2,  64,  2, pa.FIXED_FRACTION,  0.0,   600,  0.5,  1),
    ("batch2_lam0.05",     640,  4, 2,  64,  1, pa.ALL,             0.0,   0,    0.05, 2),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_skip_parity(case):
    name, N, H, Hkv, d, G, mode, gamma, frac, lam, B = case
    w = synth.small_workload(seqlen=N, heads=H, kv_heads=Hkv, head_dim=d, groups=G, gamma=gamma, batch=B,
                             needles=8, seed=500 + CASES.index(case), sink_logit=4.0)
    x = synth.make_inputs(w)
    qc, kc, vc = x["q"], x["k"], x["v"]
    q, k, v = qc.cuda(), kc.cuda(), vc.cuda()
    nb = N // 128
    qp, kp = pa.pool_heads(q, k, G)
    scores = pa.block_scores(qp, kp, H, Hkv)
    mask = pa.build_mask(scores, q, k, G, mode, gamma, frac)
    o, lse, skipped = pa.block_sparse_attn(q, k, v, mask.rank, mask.cnt, G, return_lse=True, skip_threshold=lam,
                                           return_skipped=True)
    torch.cuda.synchronize()
    assert pa.device_status() == 0

    rank, cnt = mask.rank.cpu().numpy(), mask.cnt.cpu().numpy()
    items = [(b, h, qb) for b in range(B) for h in range(H) for qb in range(nb)]
    sg = skipped.cpu().numpy()
    _, _, own, gap = oracle.sparse_attn_skip(qc, kc, vc, rank, cnt, G, items, lam)
    differ = sg != own
    assert np.all(np.abs(gap[differ]) < MARGIN), gap[differ]
    first = np.isinf(gap)
    assert not np.any(sg[first]), "the first visited block of a row was skipped"
    assert np.all(sg[np.isnan(gap)] == 0), "a block that was not visited is marked"
    n_after_first = int(np.isfinite(gap).sum())
    assert 0 < int(sg.sum()) < n_after_first, (int(sg.sum()), n_after_first)  # both outcomes occur

    oref, lref, _, _ = oracle.sparse_attn_skip(qc, kc, vc, rank, cnt, G, items, lam, skip_in=sg)
    og = o.float().cpu().numpy()
    lg = lse.cpu().numpy()
    ogi = np.stack([og[b, qb * 128:(qb + 1) * 128, h] for (b, h, qb) in items])
    lgi = np.stack([lg[b, h, qb * 128:(qb + 1) * 128] for (b, h, qb) in items])
    diff = np.abs(ogi - oref)
    assert diff.max() <= 2e-2 and diff.mean() <= 2e-3, (diff.max(), diff.mean())
    assert np.abs(lgi - lref).max() < 1e-3


def test_skip_threshold_one_keeps_only_rising_blocks():
    """lambda = 1: a block is kept only if it raises some row's running max;
    on the strong-sink inputs that leaves the first block of every row (the
    sink block) and hardly anything else, and O is the oracle's o7 with the
    kernel's decisions."""
    w = synth.small_workload(seqlen=640, heads=4, kv_heads=2, head_dim=64, groups=1, gamma=0.0, batch=2,
                             needles=8, seed=504, sink_logit=4.0)
    x = synth.make_inputs(w)
    qc, kc, vc = x["q"], x["k"], x["v"]
    q, k, v = qc.cuda(), kc.cuda(), vc.cuda()
    qp, kp = pa.pool_heads(q, k, 1)
    mask = pa.build_mask(pa.block_scores(qp, kp, 4, 2), q, k, 1, pa.ALL)
    o, skipped = pa.block_sparse_attn(q, k, v, mask.rank, mask.cnt, 1, skip_threshold=1.0, return_skipped=True)
    torch.cuda.synchronize()
    assert pa.device_status() == 0
    items = [(b, h, qb) for b in range(2) for h in range(4) for qb in range(5)]
    rank, cnt = mask.rank.cpu().numpy(), mask.cnt.cpu().numpy()
    sg = skipped.cpu().numpy()
    _, _, own, gap = oracle.sparse_attn_skip(qc, kc, vc, rank, cnt, 1, items, 1.0)
    assert np.all(np.abs(gap[sg != own]) < MARGIN)
    oref, _, _, _ = oracle.sparse_attn_skip(qc, kc, vc, rank, cnt, 1, items, 1.0, skip_in=sg)
    og = o.float().cpu().numpy()
    diff = np.abs(np.stack([og[b, qb * 128:(qb + 1) * 128, h] for (b, h, qb) in items]) - oref)
    assert diff.max() <= 2e-2 and diff.mean() <= 2e-3, (diff.max(), diff.mean())


def test_skip_off_is_the_plain_kernel():
    """lambda = 0 and a lambda too small to skip anything give the plain
    kernel's output bit for bit; pa_prefill with skip_threshold equals the
    stages."""
    w = synth.small_workload(seqlen=1024, heads=8, kv_heads=2, head_dim=128, groups=1, gamma=0.95, needles=8,
                             seed=600, sink_logit=4.0)
    x = synth.make_inputs(w, device="cuda")
    q, k, v = x["q"], x["k"], x["v"]
    qp, kp = pa.pool_heads(q, k, 1)
    mask = pa.build_mask(pa.block_scores(qp, kp, 8, 2), q, k, 1, pa.ALL)
    plain, lse0 = pa.block_sparse_attn(q, k, v, mask.rank, mask.cnt, 1, return_lse=True)
    o0, l0, s0 = pa.block_sparse_attn(q, k, v, mask.rank, mask.cnt, 1, return_lse=True, skip_threshold=0.0,
                                      return_skipped=True)
    o1, l1, s1 = pa.block_sparse_attn(q, k, v, mask.rank, mask.cnt, 1, return_lse=True, skip_threshold=1e-30,
                                      return_skipped=True)
    torch.cuda.synchronize()
    assert pa.device_status() == 0
    assert int(s0.sum()) == 0 and int(s1.sum()) == 0
    assert torch.equal(o0, plain) and torch.equal(o1, plain)
    assert torch.equal(l0, lse0) and torch.equal(l1, lse0)
    # pa_prefill with the skip equals the stages
    lam = 0.4
    o_pf, m_pf = pa.prefill(q, k, v, 1, pa.ALL, skip_threshold=lam)
    o_st = pa.block_sparse_attn(q, k, v, m_pf.rank, m_pf.cnt, 1, skip_threshold=lam)
    torch.cuda.synchronize()
    assert torch.equal(o_pf, o_st)
    assert not torch.equal(o_pf, plain)
