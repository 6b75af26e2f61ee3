"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark times (the same C-ABI stages), against the CPU oracle on what it can
compute one by one.  The cases are the five configs of the method's
Llama-3.1-8B / Qwen2.5-7B prefill workloads: 32K; 128K at G = 1, G = 4 and
with every block (the dense run the benchmark divides by); the Qwen 64K layer
at G = 4; and the 256K sweep (gamma 0.8, 0.9, 0.95, 0.99 and fixed 5, 10,
25 %).  Sweep points of one workload share one input draw.

  pool           complete and bit-exact against the oracle's own proxies
  block scores   complete rows (every tile) of sampled query blocks, always
                 including 0, 1, nb/2 and nb-1, against the oracle's scores of
                 its own proxies
  rank/cnt/budget  complete and bit-exact with the oracle fed the GPU's fp32
                 scores and masses
  end to end     the sampled rows ranked from the oracle's own scores, and
                 the budgets of sampled heads from the oracle's own head
                 masses: every disagreement a near tie or near threshold
                 (tests/mask_compare.py), the counts logged
  head mass      every head sums to one; sampled heads against the oracle
  attention O    four query blocks of every head, always 0, 1 and nb-1 plus
                 one drawn at random, against the oracle run with the GPU's
                 mask
"""
import numpy as np
import pytest
import torch

import oracle
import block_sparse_attention_pa_b200 as pa
from block_sparse_attention_pa_b200 import build, synth

from mask_compare import check_budgets, compare_lists, log_counts

pytestmark = pytest.mark.gpu

FULL = [
    # workload,        G,  mode,              gamma, frac
    ("llama8b_n32k",   1, pa.DYNAMIC,         0.95, 0),
    ("llama8b_n128k",  1, pa.DYNAMIC,         0.95, 0),
    ("llama8b_n128k",  4, pa.DYNAMIC,         0.95, 0),
    ("llama8b_n128k",  1, pa.ALL,             0.0,  0),
    ("qwen7b_n64k",    4, pa.DYNAMIC,         0.9,  0),
    ("llama8b_n256k",  1, pa.DYNAMIC,         0.8,  0),
    ("llama8b_n256k",  1, pa.DYNAMIC,         0.9,  0),
    ("llama8b_n256k",  1, pa.DYNAMIC,         0.95, 0),
    ("llama8b_n256k",  1, pa.DYNAMIC,         0.99, 0),
    ("llama8b_n256k",  1, pa.FIXED_FRACTION,  0.0,  50),
    ("llama8b_n256k",  1, pa.FIXED_FRACTION,  0.0,  100),
    ("llama8b_n256k",  1, pa.FIXED_FRACTION,  0.0,  250),
]


def _id(c):
    tag = {pa.DYNAMIC: f"g{c[3]}", pa.FIXED_FRACTION: f"fixed{c[4]}", pa.ALL: "all"}[c[2]]
    return f"{c[0]}_G{c[1]}_{tag}"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    pa.lib()
    yield
    _cache.clear()


# One workload's inputs (device and host copies) and what the oracle computes
# from them independently of the budget, shared by that workload's cases.
_cache = {}


def _workload(name):
    if name not in _cache:
        _cache.clear()
        torch.cuda.empty_cache()
        w = synth.WORKLOADS[name]
        x = synth.make_inputs(w, device="cuda")
        _cache[name] = dict(w=w, q=x["q"], k=x["k"], v=x["v"], qc=x["q"].cpu(), kc=x["k"].cpu(),
                            vc=x["v"].cpu(), per_g={})
    return _cache[name]


def _oracle_side(dat, G):
    """The oracle's own proxies (every token), its block scores of complete
    sampled rows, and its head masses of sampled heads."""
    if G in dat["per_g"]:
        return dat["per_g"][G]
    w = dat["w"]
    B, H, Hkv, nb = w.batch, w.num_q_heads, w.num_kv_heads, w.nb
    rng = np.random.default_rng(11 + G)
    _, _, qpb, kpb = oracle.pool(dat["qc"], dat["kc"], G)
    qbs = sorted({0, 1, nb // 2, nb - 1} | {int(x) for x in rng.integers(2, nb - 1, size=3)})
    rows = [(b, g, qb) for b in range(B) for g in range(G) for qb in qbs]
    tiles = [(b, g, qb, kb) for (b, g, qb) in rows for kb in range(qb + 1)]
    s_tiles = oracle.block_score_tiles(qpb, kpb, tiles)
    heads = sorted({0, H - 1} | {int(x) for x in rng.choice(np.arange(1, H - 1), size=2, replace=False)})
    kvs = [h * Hkv // H for h in heads]
    mass = oracle.head_mass(dat["qc"][:, :, heads].contiguous(), dat["kc"][:, :, kvs].contiguous())
    out = dict(qpb=qpb, kpb=kpb, rows=rows, tiles=tiles, s_tiles=s_tiles, heads=heads, mass=mass)
    dat["per_g"][G] = out
    return out


@pytest.mark.parametrize("case", FULL, ids=[_id(c) for c in FULL])
def test_full_size(case):
    name, G, mode, gamma, frac = case
    dat = _workload(name)
    w = dat["w"]
    B, N, H, Hkv, d = w.batch, w.seqlen, w.num_q_heads, w.num_kv_heads, w.head_dim
    nb = N // 128
    T = nb * (nb + 1) // 2
    rng = np.random.default_rng(7)
    q, k, v = dat["q"], dat["k"], dat["v"]
    g32 = float(np.float32(gamma))

    qp, kp = pa.pool_heads(q, k, G)
    scores = pa.block_scores(qp, kp, H, Hkv)
    mask = pa.build_mask(scores, q, k, G, mode, gamma, frac)
    o = pa.block_sparse_attn(q, k, v, mask.rank, mask.cnt, G)
    torch.cuda.synchronize()
    assert pa.device_status() == 0

    ora = _oracle_side(dat, G)
    # pool: every token, bit-exact
    assert torch.equal(qp.cpu().view(torch.int16), ora["qpb"].view(torch.int16))
    assert torch.equal(kp.cpu().view(torch.int16), ora["kpb"].view(torch.int16))

    # scores: complete sampled rows from the oracle's own proxies
    sg = scores.cpu().numpy()
    got = np.array([sg[b, g, qb * (qb + 1) // 2 + kb] for (b, g, qb, kb) in ora["tiles"]], np.float64)
    ref = ora["s_tiles"]
    assert np.all(np.abs(got - ref) <= 1e-3 * np.maximum(np.abs(ref), 1.0))

    # rank / budget / counts: complete, bit-exact given the GPU's scores and masses
    rank_g = mask.rank.cpu().numpy()
    rank_ref = oracle.rank(sg, nb)
    assert np.array_equal(rank_g, rank_ref)
    mg = mask.mass.cpu().numpy() if mask.mass is not None else None
    bud_g, cnt_g = mask.budget.cpu().numpy(), mask.cnt.cpu().numpy()
    bud_ref, cnt_ref = oracle.budget(rank_ref, mg, H, G, nb, mode, g32, frac)
    assert np.array_equal(cnt_g, cnt_ref)
    assert np.array_equal(bud_g, bud_ref)

    # end to end: the sampled rows ranked from the oracle's own scores, the
    # sampled heads' budgets from the oracle's own masses
    s_own = sg.astype(np.float64)
    for (b, g, qb, kb), s in zip(ora["tiles"], ref):
        s_own[b, g, qb * (qb + 1) // 2 + kb] = s
    rank_own = oracle.rank(s_own, nb)
    nrows, npos, tot = compare_lists(rank_g, rank_own, s_own, ora["rows"], nb)
    nbud = 0
    heads = [(0, h) for h in ora["heads"]]
    if mode == pa.DYNAMIC:
        m_own = mg.astype(np.float64)
        m_own[:, ora["heads"]] = ora["mass"]
        bud_own, _ = oracle.budget(rank_own, m_own, H, G, nb, mode, g32, frac)
        nbud = check_budgets(bud_g, rank_g, bud_own, m_own, heads, H, G, nb, g32)
    log_counts({"test": "full_size_e2e_mask", "case": _id(case), "rows": len(ora["rows"]),
                "rows_differing": nrows, "positions_differing": npos, "positions": tot,
                "heads": len(heads), "budgets_differing": nbud,
                "budgets": bud_g[0, ora["heads"]].tolist(), "density": float(cnt_g.sum()) / (B * H * T)})
    assert npos <= max(4, tot // 100)

    # head mass: every head sums to one; sampled heads against the oracle
    if mode == pa.DYNAMIC:
        np.testing.assert_allclose(mg.sum(-1), 1.0, atol=1e-4)
        assert np.all(np.abs(mg[:, ora["heads"]] - ora["mass"]) <= 2e-5 + 2e-3 * ora["mass"])

    # attention: four query blocks of every head (0, 1, nb-1 and one at random)
    items = []
    for h in range(H):
        extra = int(rng.integers(2, nb - 1))
        items += [(0, h, qb) for qb in (0, 1, extra, nb - 1)]
    oref, _ = oracle.sparse_attn(dat["qc"], dat["kc"], dat["vc"], rank_g, cnt_g, G, items)
    og = torch.stack([o[b, qb * 128:(qb + 1) * 128, h] for (b, h, qb) in items]).float().cpu().numpy()
    diff = np.abs(og - oref)
    log_counts({"test": "full_size_o", "case": _id(case), "items": len(items),
                "max_abs": float(diff.max()), "mean_abs": float(diff.mean())})
    assert diff.max() <= 2e-2 and diff.mean() <= 2e-3, (diff.max(), diff.mean())
