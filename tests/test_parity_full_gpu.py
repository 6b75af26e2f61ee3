"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark times (the same C-ABI stages), against the CPU oracle on what it can
compute one by one:

  pool           bit-exact on a random sample of tokens (every group)
  block scores   sampled tiles, including the diagonal and the sink column
  rank/cnt/budget  complete and bit-exact (oracle fed the GPU's fp32 scores/masses)
  head mass      rows sum to one for every head; oracle on sampled heads
  attention O    sampled (b, h, qb) items, always including qb = 0, 1, nb-1
"""
import numpy as np
import pytest
import torch

import oracle
import block_sparse_attention_pa_b200 as pa
from block_sparse_attention_pa_b200 import build, synth

pytestmark = pytest.mark.gpu

FULL = [
    # workload,        G,  mode,              gamma, frac
    ("llama8b_n32k",   1, pa.DYNAMIC,         0.95, 0),
    ("llama8b_n128k",  1, pa.DYNAMIC,         0.95, 0),
    ("llama8b_n128k",  4, pa.DYNAMIC,         0.95, 0),
    ("qwen7b_n64k",    4, pa.DYNAMIC,         0.9,  0),
    ("llama8b_n256k",  1, pa.DYNAMIC,         0.8,  0),
    ("llama8b_n256k",  1, pa.FIXED_FRACTION,  0.0,  50),
]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    pa.lib()


@pytest.mark.parametrize("case", FULL, ids=[f"{c[0]}_G{c[1]}_{['dyn', 'fixed', 'all'][c[2]]}" for c in FULL])
def test_full_size(case):
    name, G, mode, gamma, frac = case
    w = synth.WORKLOADS[name]
    B, N, H, Hkv, d = w.batch, w.seqlen, w.num_q_heads, w.num_kv_heads, w.head_dim
    nb = N // 128
    T = nb * (nb + 1) // 2
    rng = np.random.default_rng(7)
    x = synth.make_inputs(w, device="cuda")
    q, k, v = x["q"], x["k"], x["v"]

    qp, kp = pa.pool_heads(q, k, G)
    scores = pa.block_scores(qp, kp, H, Hkv)
    mask = pa.build_mask(scores, q, k, G, mode, gamma, frac)
    o = pa.block_sparse_attn(q, k, v, mask.rank, mask.cnt, G)
    torch.cuda.synchronize()
    assert pa.device_status() == 0

    qc, kc, vc = q.cpu(), k.cpu(), v.cpu()

    # pool: bit-exact on sampled tokens
    tok = np.sort(rng.choice(N, size=min(N, 2048), replace=False))
    tok_t = torch.from_numpy(tok)
    _, _, qpb, kpb = oracle.pool(qc[:, tok_t].contiguous(), kc[:, tok_t].contiguous(), G)
    assert torch.equal(qp[:, :, tok_t].cpu().view(torch.int16), qpb.view(torch.int16))
    assert torch.equal(kp[:, :, tok_t].cpu().view(torch.int16), kpb.view(torch.int16))

    # scores: sampled tiles from the GPU's (verified) proxies
    qpc, kpc = qp.cpu(), kp.cpu()
    tiles = [(0, g, qb, kb) for g in range(G) for qb, kb in
             [(nb - 1, nb - 1), (nb - 1, 0), (0, 0), (1, 0), (1, 1)]]
    for _ in range(48):
        qb = int(rng.integers(nb))
        tiles.append((int(rng.integers(B)), int(rng.integers(G)), qb, int(rng.integers(qb + 1))))
    ref = oracle.block_score_tiles(qpc, kpc, tiles)
    sg = scores.cpu().numpy()
    got = np.array([sg[b, g, qb * (qb + 1) // 2 + kb] for (b, g, qb, kb) in tiles], np.float64)
    assert np.all(np.abs(got - ref) <= 1e-3 * np.maximum(np.abs(ref), 1.0))

    # rank / budget / counts: complete, bit-exact
    rank_ref = oracle.rank(sg, nb)
    assert np.array_equal(mask.rank.cpu().numpy(), rank_ref)
    mg = mask.mass.cpu().numpy() if mask.mass is not None else None
    bud_ref, cnt_ref = oracle.budget(rank_ref, mg, H, G, nb, mode, float(np.float32(gamma)), frac)
    assert np.array_equal(mask.cnt.cpu().numpy(), cnt_ref)
    assert np.array_equal(mask.budget.cpu().numpy(), bud_ref)

    # head mass: every head sums to one; two heads against the oracle
    if mode == pa.DYNAMIC:
        np.testing.assert_allclose(mg.sum(-1), 1.0, atol=1e-4)
        hs = [0, H - 1]
        kvs = [h * Hkv // H for h in hs]
        mref = oracle.head_mass(qc[:, :, hs].contiguous(), kc[:, :, kvs].contiguous())  # one head per KV head
        assert np.all(np.abs(mg[:, hs] - mref) <= 2e-5 + 2e-3 * mref)

    # attention: sampled items
    items = [(0, 0, 0), (0, H - 1, 1), (0, int(rng.integers(H)), nb - 1)]
    for _ in range(3):
        items.append((int(rng.integers(B)), int(rng.integers(H)), int(rng.integers(nb))))
    oref, _ = oracle.sparse_attn(qc, kc, vc, mask.rank.cpu().numpy(), mask.cnt.cpu().numpy(), G, items)
    og = torch.stack([o[b, qb * 128:(qb + 1) * 128, h] for (b, h, qb) in items]).float().cpu().numpy()
    diff = np.abs(og - oref)
    assert diff.max() <= 2e-2 and diff.mean() <= 2e-3, (diff.max(), diff.mean())
