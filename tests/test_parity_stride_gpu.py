"""GPU parity of the query-row stride of the proxy block scores (the
sequence-level skip: only rows i = r-1 (mod r) of each block are scored),
through pa_pool_heads_strided, pa_block_scores_strided and pa_prefill with
pa_budget.score_stride, against the CPU oracle on the same seeded inputs.

Acceptance is that of the unstrided path:
  q proxy       bit-exact on the scored rows (compact [B, G, N/r, d])
  k proxy       bit-exact (complete)
  block scores  |gpu - ref| <= 1e-3 * max(|ref|, 1) against the oracle's
                strided scores from the same bf16 proxies
  rank/cnt/budget  bit-exact given the GPU's fp32 scores and masses
  O             max-abs <= 2e-2, mean-abs <= 2e-3 with the GPU's mask
Small cases span several A tiles with a ragged last one (nb not a multiple
of r); the full-size cases sample tiles and items as the unstrided ones do.
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


def compare_scores(gpu, ref):
    err = np.abs(gpu - ref)
    lim = 1e-3 * np.maximum(np.abs(ref), 1.0)
    assert np.all(err <= lim), f"score error {err.max()} (worst ratio {(err / lim).max():.3f})"


def expand_rows(qp_compact, N, r):
    """Compact scored rows -> a [B, G, N, d] proxy with row t at t*r + r-1
    (the other rows are never read by the strided oracle)."""
    B, G, _, d = qp_compact.shape
    full = torch.zeros(B, G, N, d, dtype=qp_compact.dtype)
    full[:, :, r - 1::r] = qp_compact
    return full


CASES = [
    # name,              N,    H, Hkv, d,  G, r, mode,              gamma, frac, B
    ("r2_ragged_d64",    640,  8, 2,  64, 1, 2, pa.DYNAMIC,         0.9,  0,   1),
    ("r4_ragged_d128",   1408, 4, 2, 128, 2, 4, pa.DYNAMIC,         0.9,  0,   1),
    ("r8_two_tiles",     2048, 4, 1, 128, 1, 8, pa.FIXED_FRACTION,  0.0,  300, 1),
    ("r8_ragged_g4",     1152, 8, 4,  64, 4, 8, pa.DYNAMIC,         0.95, 0,   1),
    ("r4_single_block",  128,  4, 2, 128, 1, 4, pa.DYNAMIC,         0.9,  0,   1),
    ("r2_batch2",        768,  4, 2,  64, 2, 2, pa.DYNAMIC,         0.95, 0,   2),
    ("r4_mha_g_eq_h",    512,  4, 4,  64, 4, 4, pa.ALL,             0.0,  0,   1),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_strided_stage_parity(case):
    name, N, H, Hkv, d, G, r, mode, gamma, frac, B = case
    w = synth.small_workload(seqlen=N, heads=H, kv_heads=Hkv, head_dim=d, groups=G, gamma=gamma, batch=B,
                             needles=8, seed=300 + CASES.index(case))
    x = synth.make_inputs(w)
    qc, kc, vc = x["q"], x["k"], x["v"]
    q, k, v = qc.cuda(), kc.cuda(), vc.cuda()
    nb = N // 128

    qp, kp = pa.pool_heads(q, k, G, score_stride=r)
    scores = pa.block_scores(qp, kp, H, Hkv, score_stride=r)
    mask = pa.build_mask(scores, q, k, G, mode, gamma, frac)
    o = pa.block_sparse_attn(q, k, v, mask.rank, mask.cnt, G)
    torch.cuda.synchronize()
    assert pa.device_status() == 0
    assert tuple(qp.shape) == (B, G, N // r, d)

    # proxies: bit-exact (scored q rows only)
    _, _, qpb, kpb = oracle.pool(qc, kc, G)
    assert torch.equal(qp.cpu().view(torch.int16), qpb[:, :, r - 1::r].contiguous().view(torch.int16))
    assert torch.equal(kp.cpu().view(torch.int16), kpb.view(torch.int16))

    # scores: the oracle's strided scores from the same bf16 proxies
    sg = scores.cpu().numpy()
    compare_scores(sg, oracle.block_scores(qpb, kpb, stride=r))
    # and the stride really skips rows: some tile differs from the every-row scores
    if nb > 1:
        assert np.any(sg != pa.block_scores(*pa.pool_heads(q, k, G), H, Hkv).cpu().numpy())

    # rank / budget: bit-exact given the GPU's scores and masses
    rank_ref = oracle.rank(sg, nb)
    assert np.array_equal(mask.rank.cpu().numpy(), rank_ref)
    mg = mask.mass.cpu().numpy() if mask.mass is not None else None
    bud_ref, cnt_ref = oracle.budget(rank_ref, mg, H, G, nb, mode, float(np.float32(gamma)), frac)
    assert np.array_equal(mask.cnt.cpu().numpy(), cnt_ref)
    assert np.array_equal(mask.budget.cpu().numpy(), bud_ref)

    # attention with the GPU's mask
    items = [(b, h, qb) for b in range(B) for h in range(H) for qb in range(nb)]
    oref, _ = oracle.sparse_attn(qc, kc, vc, mask.rank.cpu().numpy(), mask.cnt.cpu().numpy(), G, items)
    og = o.float().cpu().numpy()
    ogi = np.stack([og[b, qb * 128:(qb + 1) * 128, h] for (b, h, qb) in items])
    diff = np.abs(ogi - oref)
    assert diff.max() <= 2e-2 and diff.mean() <= 2e-3, (diff.max(), diff.mean())


@pytest.mark.parametrize("r", [2, 4, 8])
def test_strided_prefill_equals_stages(r):
    w = synth.small_workload(seqlen=1024, heads=8, kv_heads=2, head_dim=128, groups=2, gamma=0.9, needles=8,
                             seed=400 + r)
    x = synth.make_inputs(w, device="cuda")
    q, k, v = x["q"], x["k"], x["v"]
    o1, m1 = pa.prefill(q, k, v, 2, pa.DYNAMIC, 0.9, score_stride=r)
    qp, kp = pa.pool_heads(q, k, 2, score_stride=r)
    scores = pa.block_scores(qp, kp, 8, 2, score_stride=r)
    m2 = pa.build_mask(scores, q, k, 2, pa.DYNAMIC, 0.9)
    o2 = pa.block_sparse_attn(q, k, v, m2.rank, m2.cnt, 2)
    torch.cuda.synchronize()
    assert pa.device_status() == 0
    assert torch.equal(m1.rank, m2.rank) and torch.equal(m1.cnt, m2.cnt) and torch.equal(m1.budget, m2.budget)
    assert torch.equal(o1, o2)


FULL = [
    # workload,        G, r, mode,        gamma
    ("llama8b_n128k",  4, 4, pa.DYNAMIC,  0.95),
    ("qwen7b_n64k",    4, 2, pa.DYNAMIC,  0.9),
]


@pytest.mark.parametrize("case", FULL, ids=[f"{c[0]}_G{c[1]}_r{c[2]}" for c in FULL])
def test_strided_full_size(case):
    name, G, r, mode, gamma = case
    w = synth.WORKLOADS[name]
    B, N, H, Hkv, d = w.batch, w.seqlen, w.num_q_heads, w.num_kv_heads, w.head_dim
    nb = N // 128
    rng = np.random.default_rng(11)
    x = synth.make_inputs(w, device="cuda")
    q, k, v = x["q"], x["k"], x["v"]

    qp, kp = pa.pool_heads(q, k, G, score_stride=r)
    scores = pa.block_scores(qp, kp, H, Hkv, score_stride=r)
    mask = pa.build_mask(scores, q, k, G, mode, gamma)
    o = pa.block_sparse_attn(q, k, v, mask.rank, mask.cnt, G)
    torch.cuda.synchronize()
    assert pa.device_status() == 0
    qc, kc, vc = q.cpu(), k.cpu(), v.cpu()

    # q proxy: bit-exact on sampled scored rows (oracle pools the matching tokens)
    rows = np.sort(rng.choice(N // r, size=1024, replace=False))
    tok = torch.from_numpy(rows * r + r - 1)
    _, _, qpb, kpb = oracle.pool(qc[:, tok].contiguous(), kc[:, tok].contiguous(), G)
    assert torch.equal(qp[:, :, torch.from_numpy(rows)].cpu().view(torch.int16), qpb.view(torch.int16))

    # scores: sampled tiles, with the diagonal, the sink and the last block
    qfull = expand_rows(qp.cpu(), N, r)
    kpc = kp.cpu()
    tiles = [(0, g, qb, kb) for g in range(G) for qb, kb in
             [(nb - 1, nb - 1), (nb - 1, 0), (0, 0), (1, 0), (1, 1), (r - 1, r - 1), (r, r - 1)]]
    for _ in range(40):
        qb = int(rng.integers(nb))
        tiles.append((0, int(rng.integers(G)), qb, int(rng.integers(qb + 1))))
    ref = oracle.block_score_tiles(qfull, kpc, tiles, stride=r)
    sg = scores.cpu().numpy()
    got = np.array([sg[b, g, qb * (qb + 1) // 2 + kb] for (b, g, qb, kb) in tiles], np.float64)
    compare_scores(got, ref)

    # masks: complete and bit-exact given the GPU's scores and masses
    rank_ref = oracle.rank(sg, nb)
    assert np.array_equal(mask.rank.cpu().numpy(), rank_ref)
    mg = mask.mass.cpu().numpy()
    bud_ref, cnt_ref = oracle.budget(rank_ref, mg, H, G, nb, mode, float(np.float32(gamma)), 0)
    assert np.array_equal(mask.cnt.cpu().numpy(), cnt_ref)
    assert np.array_equal(mask.budget.cpu().numpy(), bud_ref)

    # attention: sampled items
    items = [(0, 0, 0), (0, H - 1, nb - 1), (0, int(rng.integers(H)), int(rng.integers(nb)))]
    oref, _ = oracle.sparse_attn(qc, kc, vc, mask.rank.cpu().numpy(), mask.cnt.cpu().numpy(), G, items)
    og = torch.stack([o[b, qb * 128:(qb + 1) * 128, h] for (b, h, qb) in items]).float().cpu().numpy()
    diff = np.abs(og - oref)
    assert diff.max() <= 2e-2 and diff.mean() <= 2e-3, (diff.max(), diff.mean())
