"""GPU parity of the non-causal mode (pa_shape.non_causal = 1: every query
attends every key; rows of block scores and ranked lists hold all nb blocks)
against the oracle run with causal = False on the same seeded inputs.

Acceptance is that of the causal path: proxies bit-exact; scores within
1e-3 * max(|ref|, 1); rank, cnt and budget bit-exact given the GPU's scores
and masses; head mass within 2e-5 + 2e-3 * ref; O within max-abs 2e-2 and
mean-abs 2e-3 against o5 with the GPU's mask; with every block selected, O
against the oracle's dense non-causal attention.
"""
import numpy as np
import pytest
import torch

import oracle
import block_sparse_attention_pa_b200 as pa
from block_sparse_attention_pa_b200 import build, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    pa.lib()
    assert pa.device_status() == 0


CASES = [
    # name,              N,    H, Hkv, d,   G, mode,              gamma, frac, r, B
    ("dyn_d64",          1024, 8, 2,  64,  1, pa.DYNAMIC,         0.9,  0,    1, 1),
    ("fixed_g2_d128",    640,  4, 2,  128, 2, pa.FIXED_FRACTION,  0.0,  400,  1, 1),
    ("dyn_stride4_g4",   1152, 8, 2,  128, 4, pa.DYNAMIC,         0.8,  0,    4, 1),
    ("single_block",     128,  4, 2,  64,  1, pa.DYNAMIC,         0.9,  0,    1, 1),
    ("batch2_gqa",       512,  6, 2,  64,  2, pa.DYNAMIC,         0.95, 0,    2, 2),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_noncausal_stage_parity(case):
    name, N, H, Hkv, d, G, mode, gamma, frac, r, B = case
    w = synth.small_workload(seqlen=N, heads=H, kv_heads=Hkv, head_dim=d, groups=G, gamma=gamma, batch=B,
                             needles=8, seed=800 + CASES.index(case))
    x = synth.make_inputs(w)
    qc, kc, vc = x["q"], x["k"], x["v"]
    q, k, v = qc.cuda(), kc.cuda(), vc.cuda()
    nb = N // 128
    qp, kp = pa.pool_heads(q, k, G, score_stride=r, causal=False)
    scores = pa.block_scores(qp, kp, H, Hkv, score_stride=r, causal=False)
    mask = pa.build_mask(scores, q, k, G, mode, gamma, frac, causal=False)
    o, lse = pa.block_sparse_attn(q, k, v, mask.rank, mask.cnt, G, return_lse=True, causal=False)
    torch.cuda.synchronize()
    assert pa.device_status() == 0
    assert scores.shape == (B, G, nb * nb)

    _, _, qpb, kpb = oracle.pool(qc, kc, G)
    assert torch.equal(qp.cpu().view(torch.int16), qpb[:, :, r - 1::r].contiguous().view(torch.int16))
    sref = oracle.block_scores(qpb, kpb, stride=r, causal=False)
    sg = scores.double().cpu().numpy()
    assert np.all(np.abs(sg - sref) <= 1e-3 * np.maximum(np.abs(sref), 1.0))

    rank_ref = oracle.rank(scores.cpu().numpy(), nb, causal=False)
    assert np.array_equal(mask.rank.cpu().numpy(), rank_ref)
    mg = mask.mass.cpu().numpy() if mask.mass is not None else None
    bud_ref, cnt_ref = oracle.budget(rank_ref, mg, H, G, nb, mode, float(np.float32(gamma)), frac, causal=False)
    assert np.array_equal(mask.cnt.cpu().numpy(), cnt_ref)
    assert np.array_equal(mask.budget.cpu().numpy(), bud_ref)
    if mode == pa.DYNAMIC:
        mref = oracle.head_mass(qc, kc, causal=False)
        assert np.all(np.abs(mg - mref) <= 2e-5 + 2e-3 * mref)

    items = [(b, h, qb) for b in range(B) for h in range(H) for qb in range(nb)]
    oref, lref = oracle.sparse_attn(qc, kc, vc, mask.rank.cpu().numpy(), mask.cnt.cpu().numpy(), G, items,
                                    causal=False)
    og = o.float().cpu().numpy()
    lg = lse.cpu().numpy()
    ogi = np.stack([og[b, qb * 128:(qb + 1) * 128, h] for (b, h, qb) in items])
    lgi = np.stack([lg[b, h, qb * 128:(qb + 1) * 128] for (b, h, qb) in items])
    diff = np.abs(ogi - oref)
    assert diff.max() <= 2e-2 and diff.mean() <= 2e-3, (diff.max(), diff.mean())
    assert np.abs(lgi - lref).max() < 1e-3


def test_noncausal_all_is_dense_and_prefill_equals_stages():
    w = synth.small_workload(seqlen=768, heads=4, kv_heads=2, head_dim=128, groups=1, gamma=0.9, needles=8, seed=900)
    x = synth.make_inputs(w)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    od, md = pa.prefill(q, k, v, 1, pa.ALL, causal=False)
    torch.cuda.synchronize()
    assert pa.device_status() == 0
    assert (md.cnt == 6).all()
    rows = [(0, h, i) for h in range(4) for i in (0, 1, 127, 128, 500, 767)]
    ref, _ = oracle.dense_attn(x["q"], x["k"], x["v"], rows, causal=False)
    got = np.stack([od[0, i, h].float().cpu().numpy() for (_, h, i) in rows])
    diff = np.abs(got - ref)
    assert diff.max() <= 2e-2 and diff.mean() <= 2e-3
    # the causal result differs (row 0 sees only key 0 there)
    oc, _ = pa.prefill(q, k, v, 1, pa.ALL)
    assert not torch.equal(oc, od)
    # pa_prefill equals the stages, with the block skip too
    o1, m1 = pa.prefill(q, k, v, 1, pa.DYNAMIC, 0.9, causal=False, skip_threshold=0.3)
    qp, kp = pa.pool_heads(q, k, 1, causal=False)
    m2 = pa.build_mask(pa.block_scores(qp, kp, 4, 2, causal=False), q, k, 1, pa.DYNAMIC, 0.9, causal=False)
    o2 = pa.block_sparse_attn(q, k, v, m2.rank, m2.cnt, 1, skip_threshold=0.3, causal=False)
    torch.cuda.synchronize()
    assert torch.equal(m1.rank, m2.rank) and torch.equal(m1.cnt, m2.cnt)
    assert torch.equal(o1, o2)


def test_noncausal_skip_matches_o7():
    w = synth.small_workload(seqlen=1024, heads=4, kv_heads=2, head_dim=64, groups=1, gamma=0.0, needles=8,
                             seed=901, sink_logit=4.0)
    x = synth.make_inputs(w)
    qc, kc, vc = x["q"], x["k"], x["v"]
    q, k, v = qc.cuda(), kc.cuda(), vc.cuda()
    nb = 8
    qp, kp = pa.pool_heads(q, k, 1, causal=False)
    mask = pa.build_mask(pa.block_scores(qp, kp, 4, 2, causal=False), q, k, 1, pa.ALL, causal=False)
    o, skipped = pa.block_sparse_attn(q, k, v, mask.rank, mask.cnt, 1, skip_threshold=0.01, return_skipped=True,
                                      causal=False)
    torch.cuda.synchronize()
    assert pa.device_status() == 0
    rank, cnt = mask.rank.cpu().numpy(), mask.cnt.cpu().numpy()
    items = [(0, h, qb) for h in range(4) for qb in range(nb)]
    sg = skipped.cpu().numpy()
    _, _, own, gap = oracle.sparse_attn_skip(qc, kc, vc, rank, cnt, 1, items, 0.01, causal=False)
    assert np.all(np.abs(gap[sg != own]) < 1e-3)
    assert 0 < int(sg.sum()) < int(np.isfinite(gap).sum())
    oref, _, _, _ = oracle.sparse_attn_skip(qc, kc, vc, rank, cnt, 1, items, 0.01, skip_in=sg, causal=False)
    og = o.float().cpu().numpy()
    diff = np.abs(np.stack([og[0, qb * 128:(qb + 1) * 128, h] for (_, h, qb) in items]) - oref)
    assert diff.max() <= 2e-2 and diff.mean() <= 2e-3
