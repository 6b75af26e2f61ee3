"""GPU parity: every stage of the CUDA path against the CPU oracle on the same
seeded bf16 inputs, called through the C ABI (libpa.so).

Acceptance (stated with the method's configs):
  pool          bit-exact (both take the fp64 mean and round it once to bf16)
  block scores  |gpu - ref| <= 1e-3 * max(|ref|, 1)
  rank, budget, cnt   bit-exact when the oracle is fed the GPU's fp32 scores
                and masses (ties to the lower block index)
  head mass     |gpu - ref| <= 2e-5 + 2e-3 * ref: the GPU's logits are fp32
                sums of bf16 products (about 1e-6 relative error), its
                exponentials ex2.approx (about 2^-22), and a mass adds up to
                16K keys' probabilities in fp32
  O             max-abs <= 2e-2 and mean-abs <= 2e-3 against the fp64 oracle
                run with the GPU's mask
"""
import numpy as np
import pytest
import torch

import oracle
import block_sparse_attention_pa_b200 as pa
from block_sparse_attention_pa_b200 import build, synth

pytestmark = pytest.mark.gpu

O_MAX_ABS, O_MEAN_ABS = 2e-2, 2e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    pa.lib()
    assert pa.device_status() == 0


def to_cpu(x):
    return {k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


def check_status():
    assert pa.device_status(clear=True) == 0


def run_stages(q, k, v, G, mode, gamma=0.9, frac=0):
    """Pool -> scores -> mask -> attention through the separate entry points."""
    qp, kp = pa.pool_heads(q, k, G)
    scores = pa.block_scores(qp, kp, q.shape[2], k.shape[2])
    mask = pa.build_mask(scores, q, k, G, mode, gamma, frac)
    o, lse = pa.block_sparse_attn(q, k, v, mask.rank, mask.cnt, G, return_lse=True)
    torch.cuda.synchronize()
    check_status()
    return qp, kp, scores, mask, o, lse


def compare_scores(gpu, ref):
    gpu = gpu.double().cpu().numpy()
    err = np.abs(gpu - ref)
    lim = 1e-3 * np.maximum(np.abs(ref), 1.0)
    assert np.all(err <= lim), f"score error {err.max()} (worst ratio {(err / lim).max():.3f})"


def compare_o(o_gpu, o_ref):
    diff = np.abs(o_gpu - o_ref)
    assert diff.max() <= O_MAX_ABS, diff.max()
    assert diff.mean() <= O_MEAN_ABS, diff.mean()


CASES = [
    # name,               N,    H, Hkv, d,  G, mode,        gamma, frac, B
    ("tiny_gqa_c0",       1024, 8, 2,  64, 1, pa.DYNAMIC,   0.95, 0,   1),
    ("mha_g_eq_h_d128",   384,  4, 4, 128, 4, pa.DYNAMIC,   0.9,  0,   1),
    ("gqa_g2_fixed",      640,  6, 2, 128, 2, pa.FIXED_FRACTION, 0, 300, 1),
    ("mqa_all",           512,  4, 1,  64, 1, pa.ALL,       0,    0,   1),
    ("single_block",      128,  4, 2, 128, 1, pa.DYNAMIC,   0.9,  0,   1),
    ("odd_heads_per_grp", 768, 14, 2, 128, 2, pa.DYNAMIC,   0.8,  0,   1),
    ("batch2",            512,  4, 2,  64, 2, pa.DYNAMIC,   0.95, 0,   2),
    ("gamma_one",         512,  4, 2, 128, 1, pa.DYNAMIC,   1.0,  0,   1),
    # paired heads (one KV head) that follow different lists: G = H under GQA
    ("gqa_g_eq_h_pairs",  768,  8, 2,  64, 8, pa.DYNAMIC,   0.9,  0,   1),
    ("gqa_g4_pairs_d128", 640,  8, 2, 128, 4, pa.FIXED_FRACTION, 0, 400, 1),
    # odd head counts per KV head: the lone units of query blocks qb and qb-1
    # share a CTA (odd and even nb, a single block, MHA where every unit is lone)
    ("lone_single_block", 128,  3, 1,  64, 1, pa.DYNAMIC,   0.9,  0,   1),
    ("lone_mha_nb3",      384,  2, 2, 128, 2, pa.DYNAMIC,   0.9,  0,   1),
    ("lone_g5_nb6_b2",    768, 10, 2,  64, 2, pa.FIXED_FRACTION, 0, 500, 2),
]


# The labelled extra generator with the direction weight in logit units: the
# per-head dynamic budgets differ, so the two heads of a CTA keep different
# prefixes of their list on most query blocks.
LOGIT_CASES = [
    # name,               N,    H, Hkv, d,  G, mode,        gamma, frac, B
    ("logit_gqa_d128",    2048, 8, 2, 128, 1, pa.DYNAMIC,   0.95, 0,   1),
    ("logit_g2_d64",      1536, 6, 2,  64, 2, pa.DYNAMIC,   0.9,  0,   1),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_stage_parity(case):
    check_case(case, seed=100 + CASES.index(case), needles=8)


@pytest.mark.parametrize("case", LOGIT_CASES, ids=[c[0] for c in LOGIT_CASES])
def test_stage_parity_logit_units(case):
    cnt = check_case(case, seed=300 + LOGIT_CASES.index(case), needles=24, logit_units=True)
    # the budgets really differ between the heads that share a CTA
    assert (cnt[:, 0::2] != cnt[:, 1::2]).any()


def check_case(case, seed, needles, logit_units=False):
    name, N, H, Hkv, d, G, mode, gamma, frac, B = case
    w = synth.small_workload(seqlen=N, heads=H, kv_heads=Hkv, head_dim=d, groups=G, gamma=gamma, batch=B,
                             needles=needles, seed=seed, logit_units=logit_units)
    x = synth.make_inputs(w)
    qc, kc, vc = x["q"], x["k"], x["v"]
    q, k, v = qc.cuda(), kc.cuda(), vc.cuda()
    qp, kp, scores, mask, o, lse = run_stages(q, k, v, G, mode, gamma, frac)
    nb = N // 128

    # pool: bit-exact
    _, _, qpb, kpb = oracle.pool(qc, kc, G)
    assert torch.equal(qp.cpu().view(torch.int16), qpb.view(torch.int16))
    assert torch.equal(kp.cpu().view(torch.int16), kpb.view(torch.int16))

    # scores vs fp64 oracle from the same bf16 proxies
    compare_scores(scores, oracle.block_scores(qpb, kpb))

    # rank/budget: bit-exact given the GPU's own scores and masses
    sg = scores.cpu().numpy()
    rank_ref = oracle.rank(sg, nb)
    assert np.array_equal(mask.rank.cpu().numpy(), rank_ref)
    mass_g = mask.mass.cpu().numpy() if mask.mass is not None else None
    bud_ref, cnt_ref = oracle.budget(rank_ref, mass_g, H, G, nb, mode, float(np.float32(gamma)), frac)
    assert np.array_equal(mask.cnt.cpu().numpy(), cnt_ref)
    assert np.array_equal(mask.budget.cpu().numpy(), bud_ref)

    # head mass vs fp64 oracle
    if mode == pa.DYNAMIC:
        mref = oracle.head_mass(qc, kc)
        err = np.abs(mass_g - mref)
        assert np.all(err <= 2e-5 + 2e-3 * mref), err.max()
        np.testing.assert_allclose(mass_g.sum(-1), 1.0, atol=1e-4)

    # attention vs fp64 oracle with the GPU's mask
    items = [(b, h, qb) for b in range(B) for h in range(H) for qb in range(nb)]
    oref, lref = oracle.sparse_attn(qc, kc, vc, mask.rank.cpu().numpy(), mask.cnt.cpu().numpy(), G, items)
    og = o.float().cpu().numpy()
    lg = lse.cpu().numpy()
    ogi = np.stack([og[b, qb * 128:(qb + 1) * 128, h] for (b, h, qb) in items])
    lgi = np.stack([lg[b, h, qb * 128:(qb + 1) * 128] for (b, h, qb) in items])
    compare_o(ogi, oref)
    assert np.abs(lgi - lref).max() < 1e-3
    return mask.cnt.cpu().numpy()


def test_prefill_equals_stages_and_dense_all():
    w = synth.WORKLOADS["tiny_gqa_n1024"]
    x = synth.make_inputs(w)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    G = w.num_groups
    o1, m1 = pa.prefill(q, k, v, G, pa.DYNAMIC, w.gamma)
    *_, mask, o2, _ = run_stages(q, k, v, G, pa.DYNAMIC, w.gamma)
    torch.cuda.synchronize()
    check_status()
    assert torch.equal(m1.rank, mask.rank) and torch.equal(m1.cnt, mask.cnt)
    assert torch.equal(o1, o2)
    # budget = all: the same kernel is dense causal attention
    od, _ = pa.prefill(q, k, v, G, pa.ALL)
    torch.cuda.synchronize()
    rows = [(0, h, i) for h in range(w.num_q_heads) for i in (0, 1, 127, 128, 500, 1023)]
    ref, _ = oracle.dense_attn(x["q"], x["k"], x["v"], rows)
    got = np.stack([od[0, i, h].float().cpu().numpy() for (_, h, i) in rows])
    compare_o(got, ref)


def test_strided_packed_qkv():
    """q, k, v as views of one packed [B, N, H + 2 Hkv, d] buffer; o strided too."""
    w = synth.small_workload(seqlen=512, heads=4, kv_heads=2, head_dim=128, groups=1, gamma=0.9)
    x = synth.make_inputs(w)
    packed = torch.cat([x["q"], x["k"], x["v"]], dim=2).cuda()
    q, k, v = packed[:, :, :4], packed[:, :, 4:6], packed[:, :, 6:8]
    o_buf = torch.zeros(1, 512, 8, 128, dtype=torch.bfloat16, device="cuda")
    o = o_buf[:, :, 2:6]
    qp, kp = pa.pool_heads(q, k, 1)
    scores = pa.block_scores(qp, kp, 4, 2)
    mask = pa.build_mask(scores, q, k, 1, pa.DYNAMIC, 0.9)
    pa.block_sparse_attn(q, k, v, mask.rank, mask.cnt, 1, out=o)
    torch.cuda.synchronize()
    check_status()
    qc, kc, vc = x["q"], x["k"], x["v"]
    ref_mask = pa.build_mask(scores, qc.cuda(), kc.cuda(), 1, pa.DYNAMIC, 0.9)
    assert torch.equal(ref_mask.cnt, mask.cnt)
    items = [(0, h, qb) for h in range(4) for qb in range(4)]
    oref, _ = oracle.sparse_attn(qc, kc, vc, mask.rank.cpu().numpy(), mask.cnt.cpu().numpy(), 1, items)
    og = o.float().cpu().numpy()
    compare_o(np.stack([og[0, qb * 128:(qb + 1) * 128, h] for (_, h, qb) in items]), oref)
    # the untouched heads of the output buffer stay zero
    assert o_buf[:, :, :2].abs().max().item() == 0 and o_buf[:, :, 6:].abs().max().item() == 0


def pairs_by_head(cnt, b, hk, nh, qtop, nb, causal=True):
    """The kernel's choice for the CTAs of query blocks qtop and qtop - 1 of
    one KV head (a scheduling model, not method arithmetic): True when each
    CTA takes one head at both query blocks, False when heads are paired by
    their counts per query block."""
    if qtop == 0:
        return False
    pairs = lone = 0
    for qx in (qtop, qtop - 1):
        c = np.clip(cnt[b, hk:hk + nh, qx], 0, qx + 1 if causal else nb)
        order = sorted(range(nh), key=lambda y: (c[y], y))
        for r, y in enumerate(order):
            if nh % 2 and r == nh - 1:
                lone = max(lone, int(c[y]))
            elif r % 2:
                pairs += int(c[y])
    top = np.clip(cnt[b, hk:hk + nh, qtop], 0, qtop + 1 if causal else nb)
    low = np.clip(cnt[b, hk:hk + nh, qtop - 1], 0, qtop if causal else nb)
    by_head = int(np.maximum(top, low).sum())
    return 50 * by_head < 49 * (pairs + lone)


PAIRING_CASES = [
    # name,               N,    H, Hkv, d,  B, G, causal
    ("nh4_nb10",          1280, 8, 2, 128, 1, 1, True),
    ("nh3_nb9_odd",       1152, 6, 2,  64, 1, 1, True),
    ("nh5_nb8_b2",        1024, 10, 2, 64, 2, 1, True),
    # the heads of a KV head in two proxy groups (two lists per KV head)
    ("nh4_g4_two_lists",  1280, 8, 2, 128, 1, 4, True),
    # non-causal rows: every block of the row can be listed
    ("nh4_noncausal",     1152, 8, 2,  64, 1, 1, False),
]


@pytest.mark.parametrize("case", PAIRING_CASES, ids=[c[0] for c in PAIRING_CASES])
def test_attention_under_both_head_pairings(case):
    """Counts crafted on a real ranking so that, in one launch, some pairs of
    query blocks have heads with very different budgets (the CTAs take one
    head at both query blocks) and others equal budgets (heads paired by
    count): O and LSE of every (batch, head, query block) against the oracle
    with the same lists."""
    name, N, H, Hkv, d, B, G, causal = case
    w = synth.small_workload(seqlen=N, heads=H, kv_heads=Hkv, head_dim=d, groups=G, gamma=0.9, batch=B,
                             needles=8, seed=500 + PAIRING_CASES.index(case))
    x = synth.make_inputs(w)
    qc, kc, vc = x["q"], x["k"], x["v"]
    q, k, v = qc.cuda(), kc.cuda(), vc.cuda()
    qp, kp = pa.pool_heads(q, k, G)
    mask = pa.build_mask(pa.block_scores(qp, kp, H, Hkv, causal=causal), q, k, G, pa.ALL, causal=causal)
    rank = mask.rank.cpu().numpy()
    nb = N // 128
    rng = np.random.default_rng(7)
    cnt = np.zeros((B, H, nb), np.int32)
    for b in range(B):
        for qb in range(nb):
            n = qb + 1 if causal else nb
            pair_index = (nb - 1 - qb) // 2
            if pair_index % 2 == 0:   # budgets spread evenly from n/nh to n over the heads of a KV head
                nh = H // Hkv
                cnt[b, :, qb] = np.maximum(1, (n * (np.arange(H) % nh + 1)) // nh)
            else:                     # equal budgets across heads
                cnt[b, :, qb] = max(1, int(rng.integers(1, n + 1)))
    modes = set()
    for b in range(B):
        for kv in range(Hkv):
            hk, nh = kv * (H // Hkv), H // Hkv
            for qtop in range(nb - 1, 0, -2):
                modes.add(pairs_by_head(cnt, b, hk, nh, qtop, nb, causal))
    assert modes == {True, False}, modes
    cnt_t = torch.from_numpy(cnt).cuda()
    o, lse = pa.block_sparse_attn(q, k, v, mask.rank, cnt_t, G, return_lse=True, causal=causal)
    torch.cuda.synchronize()
    check_status()
    items = [(b, h, qb) for b in range(B) for h in range(H) for qb in range(nb)]
    oref, lref = oracle.sparse_attn(qc, kc, vc, rank, cnt, G, items, causal=causal)
    og = o.float().cpu().numpy()
    lg = lse.cpu().numpy()
    ogi = np.stack([og[b, qb * 128:(qb + 1) * 128, h] for (b, h, qb) in items])
    lgi = np.stack([lg[b, h, qb * 128:(qb + 1) * 128] for (b, h, qb) in items])
    compare_o(ogi, oref)
    assert np.abs(lgi - lref).max() < 1e-3
