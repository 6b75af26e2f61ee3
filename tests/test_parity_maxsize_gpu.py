"""The largest supported sequence: N = 524288 tokens (nb = 4096 blocks, the
limit of the attention kernel's per-head block bitmaps and of the budget
kernel's four list entries per thread), two heads on one KV head.  Complete,
bit-exact masks given the GPU's scores and masses; sampled scores and
attention items against the oracle, including the last query block (4096
blocks in its list) and the first."""
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


@pytest.mark.parametrize("mode,gamma,frac", [(pa.DYNAMIC, 0.3, 0), (pa.FIXED_FRACTION, 0.0, 8)],
                         ids=["dynamic", "fixed"])
def test_max_sequence(mode, gamma, frac):
    w = synth.small_workload(seqlen=524288, heads=2, kv_heads=1, head_dim=128, groups=1, gamma=gamma,
                             needles=512, seed=1300)
    x = synth.make_inputs(w, device="cuda")
    q, k, v = x["q"], x["k"], x["v"]
    N, H, nb = 524288, 2, 4096
    qp, kp = pa.pool_heads(q, k, 1)
    scores = pa.block_scores(qp, kp, H, 1)
    mask = pa.build_mask(scores, q, k, 1, mode, gamma, frac)
    o = pa.block_sparse_attn(q, k, v, mask.rank, mask.cnt, 1)
    torch.cuda.synchronize()
    assert pa.device_status() == 0

    sg = scores.cpu().numpy()
    rank_ref = oracle.rank(sg, nb)
    assert np.array_equal(mask.rank.cpu().numpy(), rank_ref)
    mg = mask.mass.cpu().numpy() if mask.mass is not None else None
    bud_ref, cnt_ref = oracle.budget(rank_ref, mg, H, 1, nb, mode, float(np.float32(gamma)), frac)
    assert np.array_equal(mask.cnt.cpu().numpy(), cnt_ref)
    assert np.array_equal(mask.budget.cpu().numpy(), bud_ref)

    rng = np.random.default_rng(5)
    qpc, kpc = qp.cpu(), kp.cpu()
    tiles = [(0, 0, nb - 1, nb - 1), (0, 0, nb - 1, 0), (0, 0, 0, 0), (0, 0, 4095, 2048)]
    for _ in range(12):
        qb = int(rng.integers(nb))
        tiles.append((0, 0, qb, int(rng.integers(qb + 1))))
    ref = oracle.block_score_tiles(qpc, kpc, tiles)
    got = np.array([sg[0, 0, qb * (qb + 1) // 2 + kb] for (_, _, qb, kb) in tiles], np.float64)
    assert np.all(np.abs(got - ref) <= 1e-3 * np.maximum(np.abs(ref), 1.0))

    items = [(0, 0, 0), (0, 1, nb - 1), (0, 0, 2047)]
    oref, _ = oracle.sparse_attn(q.cpu(), k.cpu(), v.cpu(), mask.rank.cpu().numpy(), mask.cnt.cpu().numpy(), 1,
                                 items)
    og = torch.stack([o[b, qb * 128:(qb + 1) * 128, h] for (b, h, qb) in items]).float().cpu().numpy()
    diff = np.abs(og - oref)
    assert diff.max() <= 2e-2 and diff.mean() <= 2e-3, (diff.max(), diff.mean())
