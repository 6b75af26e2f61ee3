"""Pins for the CPU oracle, against facts fixed by the pages and by mathematics
(closed forms, library routines on special cases, brute force on tiny inputs),
never against the oracle itself.  No GPU."""
import itertools
import math

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from block_sparse_attention_pa_b200 import synth


def bf16(a):
    return torch.as_tensor(np.asarray(a, np.float32)).to(torch.bfloat16)


def bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def bf16_value(b):
    return float(np.array([int(b) << 16], np.uint32).view(np.float32)[0])


# ----------------------------------------------------------- bf16 rounding
def test_bf16_rne_exact_and_midpoints():
    """Every finite bf16 value maps to itself; the exact midpoint of two
    neighbours goes to the one with an even last mantissa bit; points just off
    the midpoint go to the nearer neighbour (IEEE roundTiesToEven)."""
    f = oracle.f64_to_bf16_bits
    for b in list(range(0x0000, 0x7F7F, 7)) + [0x0001, 0x007F, 0x0080, 0x3F80, 0x7F7E]:
        v, w = bf16_value(b), bf16_value(b + 1)
        assert f(v) == b and f(-v) == (b | 0x8000)
        mid = (v + w) / 2.0
        even = b if b % 2 == 0 else b + 1
        assert f(mid) == even
        assert f(-mid) == (even | 0x8000)
        assert f(mid - (w - v) * 2.0 ** -20) == b
        assert f(mid + (w - v) * 2.0 ** -20) == b + 1
    # beyond the largest finite bf16 by half a spacing -> inf
    big = bf16_value(0x7F7F)
    assert f(big + (big - bf16_value(0x7F7E)) / 2) == 0x7F80
    assert f(0.0) == 0 and f(-0.0) == 0x8000


def test_bf16_rne_matches_torch_from_float32():
    """On float32 inputs (exact in fp64) the oracle's rounding agrees with
    torch's float32 -> bfloat16 conversion (round to nearest even)."""
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(3000).astype(np.float32) * 10.0 ** rng.integers(-30, 30, 3000),
                        rng.standard_normal(1000).astype(np.float32)]).astype(np.float32)
    ref = bits(torch.from_numpy(x).to(torch.bfloat16))
    got = np.array([oracle.f64_to_bf16_bits(float(v)) for v in x], np.uint16)
    np.testing.assert_array_equal(got, ref)


# ------------------------------------------------------------------- pool
def test_pool_closed_form():
    """H=4 heads with constant values 1,2,3,4; Hkv=2 KV heads with 10, 20.
    G=1: Qp=2.5, Kp=mean(10,10,20,20)=15.  G=2: Qp=(1.5, 3.5), Kp=(10, 20)."""
    N, d = 128, 8
    q = torch.empty(1, N, 4, d)
    for h in range(4):
        q[:, :, h] = h + 1
    k = torch.empty(1, N, 2, d)
    k[:, :, 0], k[:, :, 1] = 10.0, 20.0
    q, k = q.bfloat16(), k.bfloat16()
    qp, kp, qpb, kpb = oracle.pool(q, k, 1)
    assert np.all(qp == 2.5) and np.all(kp == 15.0)
    qp, kp, qpb, kpb = oracle.pool(q, k, 2)
    assert np.all(qp[0, 0] == 1.5) and np.all(qp[0, 1] == 3.5)
    assert np.all(kp[0, 0] == 10.0) and np.all(kp[0, 1] == 20.0)
    assert torch.equal(qpb.float(), torch.from_numpy(qp).float())


def test_pool_one_head_per_group_is_identity():
    """G = H: each proxy is its own head, bit for bit (Q), and the KV head of that
    q head (K)."""
    w = synth.small_workload(seqlen=256, heads=4, kv_heads=2, head_dim=64, groups=4)
    x = synth.make_inputs(w)
    q, k = x["q"], x["k"]
    _, _, qpb, kpb = oracle.pool(q, k, 4)
    for h in range(4):
        assert torch.equal(qpb[0, h], q[0, :, h])
        assert torch.equal(kpb[0, h], k[0, :, h * 2 // 4])


def test_pool_matches_numpy_mean_and_head_permutation():
    w = synth.small_workload(seqlen=256, heads=8, kv_heads=4, head_dim=64, groups=2)
    x = synth.make_inputs(w)
    q, k = x["q"], x["k"]
    qp, kp, qpb, kpb = oracle.pool(q, k, 2)
    qn = q.double().numpy()
    kn = k.double().numpy()
    for g in range(2):
        heads = list(range(4 * g, 4 * g + 4))
        np.testing.assert_allclose(qp[0, g], qn[0][:, heads].mean(axis=1), rtol=1e-15, atol=0)
        kvs = [h * 4 // 8 for h in heads]
        np.testing.assert_allclose(kp[0, g], kn[0][:, kvs].mean(axis=1), rtol=1e-15, atol=0)
    # the bf16 proxies are the mean rounded to nearest even: where the mean of
    # the four bf16 values is exact in fp32 (almost everywhere), torch's
    # fp32 -> bf16 conversion is an independent reference
    qmean = np.stack([qn[0][:, list(range(4 * g, 4 * g + 4))].mean(axis=1) for g in range(2)])
    exact = qmean.astype(np.float32).astype(np.float64) == qmean
    assert exact.mean() > 0.9
    ref = torch.from_numpy(qmean.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy()
    got = qpb[0].view(torch.int16).numpy()
    assert np.array_equal(got[exact], ref[exact])
    # permuting the heads inside each group leaves the proxies unchanged
    perm = [3, 1, 0, 2, 7, 6, 4, 5]
    qp2, _, qpb2, _ = oracle.pool(q[:, :, perm].contiguous(), k, 2)
    assert np.array_equal(qp, qp2) and torch.equal(qpb, qpb2)


def test_pool_strided_input_equals_contiguous():
    w = synth.small_workload(seqlen=256, heads=4, kv_heads=2, head_dim=64)
    x = synth.make_inputs(w)
    packed = torch.cat([x["q"], x["k"], x["v"]], dim=2)  # [B, N, H+2Hkv, d]
    q, k = packed[:, :, :4], packed[:, :, 4:6]
    assert not q.is_contiguous()
    a = oracle.pool(q, k, 1)
    b = oracle.pool(x["q"], x["k"], 1)
    assert torch.equal(a[2], b[2]) and torch.equal(a[3], b[3])


# ----------------------------------------------------------------- scores
def brute_block_max(qh, kh, scale):
    """Per-head causal block maxima of scale * q k^T by numpy (fp64)."""
    N = qh.shape[0]
    nb = N // 128
    s = (qh @ kh.T) * scale
    s[np.triu_indices(N, 1)] = -np.inf
    out = []
    for qb in range(nb):
        for kb in range(qb + 1):
            out.append(s[qb * 128:(qb + 1) * 128, kb * 128:(kb + 1) * 128].max())
    return np.array(out)


def test_scores_one_head_per_group_equal_per_head_scores():
    """Check (b): MHA with G = H, so each proxy is one head; the proxy block
    scores equal each head's own causal block maxima."""
    w = synth.small_workload(seqlen=384, heads=3, kv_heads=3, head_dim=64, groups=3)
    x = synth.make_inputs(w)
    q, k = x["q"], x["k"]
    _, _, qpb, kpb = oracle.pool(q, k, 3)
    sc = oracle.block_scores(qpb, kpb)
    for h in range(3):
        ref = brute_block_max(q[0, :, h].double().numpy(), k[0, :, h].double().numpy(), 1 / 8.0)
        np.testing.assert_allclose(sc[0, h], ref, rtol=1e-13, atol=1e-13)


def test_scores_planted_pair_and_causal_mask():
    """All-zero proxies except one query row i and key rows j: the tile holding
    (i, j) scores a*b/sqrt(d); a larger product placed above the diagonal
    (j > i, same block) must not count; every other tile scores 0."""
    N, d = 512, 64
    qp = torch.zeros(1, 1, N, d)
    kp = torch.zeros(1, 1, N, d)
    qp[0, 0, 300, 5] = 2.0          # row 300 -> qb 2
    kp[0, 0, 140, 5] = 3.0          # key 140 -> kb 1: score 6/8 at (2, 1)
    kp[0, 0, 310, 5] = 16.0         # key 310 > 300 in the diagonal tile: masked
    sc = oracle.block_scores(qp.bfloat16(), kp.bfloat16())[0, 0]
    tri = lambda qb: qb * (qb + 1) // 2
    assert sc[tri(2) + 1] == pytest.approx(6.0 / 8.0)
    assert sc[tri(2) + 2] == 0.0
    # row 310 > key 310? no: row 311+ sees key 310 only if qp is nonzero there; it is zero
    mask = np.ones_like(sc, bool)
    mask[tri(2) + 1] = False
    assert np.all(sc[mask] == 0.0)
    # negative products: max keeps the largest (least negative) valid entry
    qp2 = torch.zeros(1, 1, 256, d)
    qp2[0, 0, :, 0] = -1.0
    kp2 = torch.zeros(1, 1, 256, d)
    kp2[0, 0, :, 0] = torch.linspace(1, 2, 256)
    sc2 = oracle.block_scores(qp2.bfloat16(), kp2.bfloat16())[0, 0]
    kv = kp2.bfloat16().double()[0, 0, :, 0].numpy()
    assert sc2[0] == pytest.approx(-kv[0] / 8)       # tile (0,0): smallest key
    assert sc2[1] == pytest.approx(-kv[0] / 8)       # tile (1,0)
    assert sc2[2] == pytest.approx(-kv[128] / 8)     # tile (1,1)


@pytest.mark.parametrize("r", [2, 4, 8])
def test_strided_scores_planted_rows(r):
    """Query-row stride r: only rows i = r-1 (mod r) are scored.  A product
    planted on a scored row sets its tile's score; a larger one planted on a
    skipped row of another tile leaves that tile at 0; in the diagonal tile a
    key at j = i counts and a key at j = i + 1 does not."""
    N, d = 512, 64
    tri = lambda qb: qb * (qb + 1) // 2
    qp = torch.zeros(1, 1, N, d)
    kp = torch.zeros(1, 1, N, d)
    i_on = 2 * 128 + 5 * r + (r - 1)        # scored row of qb 2
    i_off = 3 * 128 + 7 * r                  # skipped row of qb 3 (i_off mod r == 0)
    qp[0, 0, i_on, 3] = 2.0
    kp[0, 0, 130, 3] = 3.0                   # kb 1: tile (2, 1) = 6/8; tile (3, 1) sees it through no scored row
    qp[0, 0, i_off, 9] = 4.0
    kp[0, 0, 20, 9] = 4.0                    # kb 0: 16/8 only through the skipped row
    sc = oracle.block_scores(qp.bfloat16(), kp.bfloat16(), stride=r)[0, 0]
    assert sc[tri(2) + 1] == pytest.approx(6.0 / 8.0)
    assert sc[tri(3) + 0] == 0.0
    rest = np.ones_like(sc, bool)
    rest[tri(2) + 1] = False
    assert np.all(sc[rest] == 0.0)
    # diagonal tile: key j = i_on counts, j = i_on + 1 does not
    kp2 = torch.zeros(1, 1, N, d)
    kp2[0, 0, i_on, 3] = 1.0
    kp2[0, 0, i_on + 1, 3] = 8.0
    sc2 = oracle.block_scores(qp.bfloat16(), kp2.bfloat16(), stride=r)[0, 0]
    assert sc2[tri(2) + 2] == pytest.approx(2.0 / 8.0)
    # stride 1 sees the skipped row's product
    sc1 = oracle.block_scores(qp.bfloat16(), kp.bfloat16(), stride=1)[0, 0]
    assert sc1[tri(3) + 0] == pytest.approx(16.0 / 8.0)


@pytest.mark.parametrize("r", [2, 4, 8])
def test_strided_scores_equal_full_scores_of_window_copies(r):
    """Replacing every query row by the scored row of its window (the last of
    each r rows) gives a proxy whose every-row scores equal the strided
    scores of the original: each copy sees a subset of the keys the scored row
    sees.  Scores also shrink as the stride doubles (the scored rows of 2r are
    a subset of those of r)."""
    w = synth.small_workload(seqlen=640, heads=4, kv_heads=2, head_dim=64, groups=2)
    x = synth.make_inputs(w)
    _, _, qpb, kpb = oracle.pool(x["q"], x["k"], 2)
    N = qpb.shape[2]
    src = (np.arange(N) // r) * r + (r - 1)
    dup = qpb[:, :, torch.as_tensor(src)].contiguous()
    strided = oracle.block_scores(qpb, kpb, stride=r)
    full_dup = oracle.block_scores(dup, kpb, stride=1)
    assert np.array_equal(strided, full_dup)
    full = oracle.block_scores(qpb, kpb, stride=1)
    assert np.all(strided <= full)
    if r < 8:
        assert np.all(oracle.block_scores(qpb, kpb, stride=2 * r) <= strided)
    assert np.any(strided < full)


def test_score_tiles_equal_full_scores():
    w = synth.small_workload(seqlen=384, heads=4, kv_heads=2, head_dim=64, groups=2)
    x = synth.make_inputs(w)
    _, _, qpb, kpb = oracle.pool(x["q"], x["k"], 2)
    sc = oracle.block_scores(qpb, kpb)
    tiles = [(0, 1, 2, 0), (0, 0, 1, 1), (0, 1, 0, 0)]
    got = oracle.block_score_tiles(qpb, kpb, tiles)
    tri = lambda qb: qb * (qb + 1) // 2
    for (b, g, qb, kb), v in zip(tiles, got):
        assert v == sc[b, g, tri(qb) + kb]


# ------------------------------------------------------------------- mass
def test_mass_rows_sum_to_one_and_match_scipy_softmax():
    """Check (d) and a library pin: mass from scipy.special.softmax rows."""
    w = synth.small_workload(seqlen=384, heads=4, kv_heads=2, head_dim=64)
    x = synth.make_inputs(w)
    q, k = x["q"], x["k"]
    mass, dev = oracle.head_mass(q, k, with_rowsum=True)
    assert np.all(dev < 1e-12)
    np.testing.assert_allclose(mass.sum(-1), 1.0, atol=1e-12)
    N = 384
    for h in range(4):
        qh = q[0, N - 128:, h].double().numpy()
        kh = k[0, :, h * 2 // 4].double().numpy()
        z = qh @ kh.T / 8.0
        rows = np.arange(N - 128, N)
        z[np.arange(N)[None, :] > rows[:, None]] = -np.inf
        p = scipy.special.softmax(z, axis=1)
        ref = p.reshape(128, 3, 128).sum(-1).mean(0)
        np.testing.assert_allclose(mass[0, h], ref, rtol=1e-12, atol=1e-15)


def test_mass_single_block_is_one():
    w = synth.small_workload(seqlen=128, heads=2, kv_heads=1, head_dim=64)
    x = synth.make_inputs(w)
    mass = oracle.head_mass(x["q"], x["k"])
    np.testing.assert_allclose(mass, 1.0, atol=1e-13)


# ------------------------------------------------------------------- rank
def brute_rank_row(row, qb):
    """The unique order of blocks 1..qb-1 in which every neighbour pair is
    (higher score first) or (equal score, lower index first), found by
    enumerating permutations."""
    rest = list(range(1, qb))
    for perm in itertools.permutations(rest):
        ok = all(row[a] > row[b] or (row[a] == row[b] and a < b) for a, b in zip(perm, perm[1:]))
        if ok:
            return [0, qb] + list(perm)
    raise AssertionError


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_rank_brute_force_with_ties(seed):
    nb = 8
    rng = np.random.default_rng(seed)
    T = nb * (nb + 1) // 2
    scores = rng.integers(0, 4, size=(1, 2, T)).astype(np.float64) * 0.5 - 0.7  # many ties
    r = oracle.rank(scores, nb)
    for g in range(2):
        for qb in range(nb):
            row = scores[0, g, qb * (qb + 1) // 2: qb * (qb + 1) // 2 + qb + 1]
            got = list(r[0, g, qb * (qb + 1) // 2: qb * (qb + 1) // 2 + qb + 1])
            exp = [0] if qb == 0 else brute_rank_row(row, qb)
            assert got == exp


def test_rank_treats_float32_scores_exactly():
    """Scores that differ only in the last float32 bit keep their order."""
    nb = 4
    a = np.float32(1.0)
    b = np.nextafter(a, np.float32(2.0))
    s = np.zeros((1, 1, 10), np.float32)
    s[0, 0, 6:10] = [0.0, a, b, 5.0]  # row qb=3: blocks 0..3
    r = oracle.rank(s, nb)
    assert list(r[0, 0, 6:10]) == [0, 3, 2, 1]


# ----------------------------------------------------------------- budget
def fx(m):
    return int(np.rint(m * 2.0 ** 40))


def brute_budget(list_last, mass_h, gamma, nb):
    F = 1 if nb == 1 else 2
    g = fx(gamma)
    for k in range(F, nb + 1):
        if sum(fx(mass_h[b]) for b in list_last[:k]) >= g:
            return k
    return nb


@pytest.mark.parametrize("seed", range(4))
def test_budget_brute_force_and_invariants(seed):
    rng = np.random.default_rng(seed)
    nb, H, G = 9, 4, 2
    T = nb * (nb + 1) // 2
    scores = rng.standard_normal((1, G, T))
    r = oracle.rank(scores, nb)
    mass = rng.dirichlet(np.ones(nb) * 0.3, size=(1, H))
    for gamma in [0.05, 0.5, 0.8, 0.95, 0.999, 1.0]:
        bud, cnt = oracle.budget(r, mass, H, G, nb, oracle.DYNAMIC, gamma)
        for h in range(H):
            g = h * G // H
            last = list(r[0, g, T - nb:])
            k = brute_budget(last, mass[0, h], gamma, nb)
            assert bud[0, h] == k
            # invariants: prefix reaches gamma; one block fewer does not (unless at |F|)
            pre = lambda n: sum(fx(mass[0, h][b]) for b in last[:n])
            if k < nb or pre(nb) >= fx(gamma):
                assert pre(k) >= fx(gamma)
            if k > 2:
                assert pre(k - 1) < fx(gamma)
            assert cnt[0, h, nb - 1] == k
            for qb in range(nb):
                exp = min(max(-(-k * (qb + 1) // nb), 1 if qb == 0 else 2), qb + 1)
                assert cnt[0, h, qb] == exp


def test_budget_nested_in_gamma():
    rng = np.random.default_rng(5)
    nb, H = 16, 2
    T = nb * (nb + 1) // 2
    r = oracle.rank(rng.standard_normal((1, 1, T)), nb)
    mass = rng.dirichlet(np.ones(nb), size=(1, H))
    prev = None
    for gamma in np.linspace(0.01, 1.0, 25):
        bud, cnt = oracle.budget(r, mass, H, 1, nb, oracle.DYNAMIC, float(gamma))
        if prev is not None:
            assert np.all(cnt >= prev)
        prev = cnt


def test_budget_is_find_blocks_when_ranking_follows_mass():
    """XAttention's find_blocks: the smallest block set whose mass reaches the
    threshold.  When the shared ranking orders blocks by this head's own mass,
    the oracle's prefix rule gives the size of the smallest such set among all
    subsets that contain the forced sink and diagonal blocks (brute force over
    all subsets)."""
    rng = np.random.default_rng(11)
    nb = 8
    T = nb * (nb + 1) // 2
    for trial in range(6):
        m = rng.dirichlet(np.ones(nb) * 0.5)
        scores = np.zeros((1, 1, T))
        scores[0, 0, T - nb:] = m  # last row ranked by the head's mass
        r = oracle.rank(scores, nb)
        for gamma in [0.3, 0.6, 0.9]:
            bud, _ = oracle.budget(r, m[None, None], 1, 1, nb, oracle.DYNAMIC, gamma)
            best = nb
            others = list(range(1, nb - 1))
            for size in range(0, nb - 1):
                for sub in itertools.combinations(others, size):
                    s = [0, nb - 1] + list(sub)
                    if sum(fx(m[b]) for b in s) >= fx(gamma):
                        best = min(best, len(s))
            assert bud[0, 0] == best


def test_fixed_and_all_counts_closed_form():
    nb, H = 10, 3
    T = nb * (nb + 1) // 2
    r = oracle.rank(np.zeros((1, 1, T)), nb)
    bud, cnt = oracle.budget(r, None, H, 1, nb, oracle.FIXED_FRACTION, frac_permille=250)
    for qb in range(nb):
        assert cnt[0, 0, qb] == min(max(math.ceil(250 * (qb + 1) / 1000), 1 if qb == 0 else 2), qb + 1)
    assert bud[0, 0] == 3
    bud, cnt = oracle.budget(r, None, H, 1, nb, oracle.ALL)
    assert np.all(cnt[0] == np.arange(1, nb + 1)) and np.all(bud == nb)


# -------------------------------------------------------------- attention
def sdpa_reference(q, k, v, mask=None):
    """torch scaled_dot_product_attention in fp64 on [B, N, H, d] tensors (GQA
    by repeating KV heads); causal unless an explicit boolean mask [N, N] or
    [H, N, N] is given."""
    B, N, H, d = q.shape
    rep = H // k.shape[2]
    qq = q.double().permute(0, 2, 1, 3)
    kk = k.double().repeat_interleave(rep, dim=2).permute(0, 2, 1, 3)
    vv = v.double().repeat_interleave(rep, dim=2).permute(0, 2, 1, 3)
    if mask is None:
        o = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, is_causal=True)
    else:
        o = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, attn_mask=mask)
    return o.permute(0, 2, 1, 3)


def test_dense_matches_torch_sdpa():
    w = synth.small_workload(seqlen=256, heads=4, kv_heads=2, head_dim=64)
    x = synth.make_inputs(w)
    q, k, v = x["q"], x["k"], x["v"]
    rows = [(0, h, i) for h in range(4) for i in [0, 1, 127, 128, 200, 255]]
    o, lse = oracle.dense_attn(q, k, v, rows)
    ref = sdpa_reference(q, k, v)
    for (b, h, i), oo in zip(rows, o):
        np.testing.assert_allclose(oo, ref[b, i, h].numpy(), rtol=1e-12, atol=1e-12)
    # lse against torch.logsumexp
    for (b, h, i), l in zip(rows, lse):
        z = (q[b, i, h].double() @ k[b, :i + 1, h * 2 // 4].double().T) / 8.0
        assert l == pytest.approx(torch.logsumexp(z, 0).item(), abs=1e-12)


def test_sparse_all_equals_dense():
    """Check (a): with the budget covering every causal block, block-sparse
    attention is dense causal softmax attention."""
    w = synth.small_workload(seqlen=384, heads=4, kv_heads=2, head_dim=64)
    x = synth.make_inputs(w)
    q, k, v = x["q"], x["k"], x["v"]
    m = oracle.prefill_masks(q, k, 1, mode=oracle.ALL)
    items = [(0, h, qb) for h in range(4) for qb in range(3)]
    o, lse = oracle.sparse_attn(q, k, v, m["rank"], m["cnt"], 1, items)
    rows = [(0, h, qb * 128 + i) for (_, h, qb) in items for i in range(128)]
    od, lsed = oracle.dense_attn(q, k, v, rows)
    np.testing.assert_allclose(o.reshape(-1, 64), od, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse.reshape(-1), lsed, rtol=0, atol=1e-12)


def test_sparse_matches_sdpa_with_block_mask():
    """Block-sparse attention equals torch SDPA (fp64) under the explicit
    token mask built from the selected blocks and causality."""
    w = synth.small_workload(seqlen=512, heads=4, kv_heads=2, head_dim=64, groups=2)
    x = synth.make_inputs(w)
    q, k, v = x["q"], x["k"], x["v"]
    m = oracle.prefill_masks(q, k, 2, mode=oracle.FIXED_FRACTION, frac_permille=500)
    nb = 4
    mask = torch.zeros(4, 512, 512, dtype=torch.bool)
    for h in range(4):
        g = h * 2 // 4
        for qb in range(nb):
            sel = m["rank"][0, g, qb * (qb + 1) // 2: qb * (qb + 1) // 2 + m["cnt"][0, h, qb]]
            for kb in sel:
                mask[h, qb * 128:(qb + 1) * 128, kb * 128:(kb + 1) * 128] = True
    mask &= torch.ones(512, 512, dtype=torch.bool).tril()[None]
    ref = sdpa_reference(q, k, v, mask=mask[None])
    items = [(0, h, qb) for h in range(4) for qb in range(nb)]
    o, _ = oracle.sparse_attn(q, k, v, m["rank"], m["cnt"], 2, items)
    for (b, h, qb), oo in zip(items, o):
        np.testing.assert_allclose(oo, ref[0, qb * 128:(qb + 1) * 128, h].numpy(), rtol=1e-12, atol=1e-12)
    # a head that keeps fewer blocks really attends to fewer keys
    assert (m["cnt"][0, :, 3] < 4).all()


def test_attention_head_dim_one_textbook_softmax():
    """d = 1, N = 128: O_i = sum_j softmax(q_i k_j)_j v_j over j <= i, written
    with numpy exp."""
    N = 128
    rng = np.random.default_rng(3)
    q = bf16(rng.standard_normal((1, N, 1, 1)))
    k = bf16(rng.standard_normal((1, N, 1, 1)))
    v = bf16(rng.standard_normal((1, N, 1, 1)))
    m = oracle.prefill_masks(q, k, 1, mode=oracle.ALL)
    o, _ = oracle.sparse_attn(q, k, v, m["rank"], m["cnt"], 1, [(0, 0, 0)])
    qd, kd, vd = (t.double().numpy().reshape(N) for t in (q, k, v))
    for i in range(N):
        z = qd[i] * kd[:i + 1]
        p = np.exp(z - z.max())
        p /= p.sum()
        assert o[0, i, 0] == pytest.approx(float(p @ vd[:i + 1]), abs=1e-13)


# ------------------------------------------------ o7 running-max block skip
def _skip_inputs(N=512, d=16, seed=21, scales=(1.0, 0.25, 3.0, 0.5)):
    """One head, random bf16 q, k, v; K of block kb scaled by scales[kb] so
    that some blocks sit far below the running max and some do not."""
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(1, N, 1, d, generator=g)
    k = torch.randn(1, N, 1, d, generator=g)
    v = torch.randn(1, N, 1, d, generator=g)
    for kb, s in enumerate(scales):
        k[:, kb * 128:(kb + 1) * 128] *= s
    return q.bfloat16(), k.bfloat16(), v.bfloat16()


def _full_lists(nb, shuffle_seed=None):
    """Every causal block listed, each row's list in a shuffled order."""
    T = nb * (nb + 1) // 2
    rank = np.zeros((1, 1, T), np.int32)
    rng = np.random.default_rng(shuffle_seed)
    for qb in range(nb):
        lst = np.arange(qb + 1)
        if shuffle_seed is not None:
            rng.shuffle(lst)
        rank[0, 0, qb * (qb + 1) // 2: qb * (qb + 1) // 2 + qb + 1] = lst
    cnt = np.array([[[qb + 1 for qb in range(nb)]]], np.int32)
    return rank, cnt


def brute_skip(q, k, v, qb, blocks, lam, scale):
    """numpy: the query block's logits against the listed blocks in ascending
    order, each row's running max, the block decisions, and the softmax over
    the keys of the blocks kept."""
    qf = q[0, :, 0].double().numpy()
    kf = k[0, :, 0].double().numpy()
    vf = v[0, :, 0].double().numpy()
    rows = np.arange(qb * 128, qb * 128 + 128)
    z = scale * qf[rows] @ kf.T
    z[np.arange(128)[:, None] + qb * 128 < np.arange(kf.shape[0])[None, :]] = -np.inf
    run = np.full(128, -np.inf)
    keep = []
    for t, kb in enumerate(sorted(blocks)):
        tile_max = z[:, kb * 128:(kb + 1) * 128].max(axis=1)
        skip = t > 0 and lam > 0 and np.max(tile_max - run) < np.log(lam)
        run = np.maximum(run, tile_max)
        keep.append((kb, not skip))
    cols = np.concatenate([np.arange(kb * 128, kb * 128 + 128) for kb, kp in keep if kp])
    zz = z[:, cols]
    p = np.exp(zz - zz.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    return p @ vf[cols], {kb: not kp for kb, kp in keep}


@pytest.mark.parametrize("lam", [0.02, 0.2, 0.6])
def test_skip_brute_force(lam):
    """o7 against a numpy restatement on a tiny case (decisions and O)."""
    q, k, v = _skip_inputs()
    nb = 4
    rank, cnt = _full_lists(nb, shuffle_seed=1)
    items = [(0, 0, qb) for qb in range(nb)]
    out, _, skip, gap = oracle.sparse_attn_skip(q, k, v, rank, cnt, 1, items, lam)
    scale = 1 / 4.0
    for n, (_, _, qb) in enumerate(items):
        ref, dec = brute_skip(q, k, v, qb, list(range(qb + 1)), lam, scale)
        np.testing.assert_allclose(out[n], ref, rtol=1e-10, atol=1e-12)
        for kb, sk in dec.items():
            assert skip[0, 0, qb * (qb + 1) // 2 + kb] == sk
            assert abs(gap[0, 0, qb * (qb + 1) // 2 + kb]) > 1e-9  # no decision on a knife edge


def test_skip_sweep_skips_some_and_nests():
    """The decisions are nested in lambda, and the sweep above both skips and
    keeps later blocks (so the brute-force pin is not vacuous)."""
    q, k, v = _skip_inputs()
    rank, cnt = _full_lists(4)
    items = [(0, 0, qb) for qb in range(4)]
    prev = None
    counts = []
    for lam in (0.0, 0.02, 0.2, 0.6, 1.0):
        _, _, skip, _ = oracle.sparse_attn_skip(q, k, v, rank, cnt, 1, items, lam)
        if prev is not None:
            assert np.all(skip >= prev)
        prev = skip
        counts.append(int(skip.sum()))
    assert counts[0] == 0 and counts[-1] > counts[1] and counts[-1] < 6


def test_skip_planted_running_max():
    """Logits 0 (block 0), 8 (block 1), 4 (blocks 2, 3) for every row of query
    block 3; lambda = e^-2.  Block 1 raises the running max to 8, so blocks 2
    and 3 (4 - 8 < -2) are skipped though they lie far above block 0; the
    output is the softmax over blocks 0 and 1 alone (o5 with the list [0, 1]),
    and the margins are (4 - 8 + 2) log2(e)."""
    N, d = 512, 16
    q = torch.zeros(1, N, 1, d)
    q[..., 0] = 2.0
    k = torch.zeros(1, N, 1, d)
    k[:, 128:256, 0, 0] = 16.0
    k[:, 256:512, 0, 0] = 8.0
    v = torch.randn(1, N, 1, d, generator=torch.Generator().manual_seed(3))
    q, k, v = q.bfloat16(), k.bfloat16(), v.bfloat16()
    rank, cnt = _full_lists(4, shuffle_seed=2)
    out, _, skip, gap = oracle.sparse_attn_skip(q, k, v, rank, cnt, 1, [(0, 0, 3)], math.exp(-2.0))
    assert list(skip[0, 0, 6:10]) == [0, 0, 1, 1]
    np.testing.assert_allclose(gap[0, 0, 8:10], (4 - 8 + 2) / math.log(2), rtol=1e-12)
    assert gap[0, 0, 7] == pytest.approx((8 - 0 + 2) / math.log(2))
    r2 = rank.copy()
    r2[0, 0, 6:10] = [0, 1, 2, 3]
    c2 = cnt.copy()
    c2[0, 0, 3] = 2
    ref, _ = oracle.sparse_attn(q, k, v, r2, c2, 1, [(0, 0, 3)])
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-14)


def test_skip_zero_threshold_and_given_decisions():
    """lambda = 0 skips nothing and equals o5; decisions passed in are the
    ones applied (none skipped -> o5; the oracle's own -> its own output)."""
    w = synth.small_workload(seqlen=512, heads=4, kv_heads=2, head_dim=64, groups=2, gamma=0.9)
    x = synth.make_inputs(w)
    m = oracle.prefill_masks(x["q"], x["k"], 2, mode=oracle.FIXED_FRACTION, frac_permille=700)
    items = [(0, h, qb) for h in range(4) for qb in range(4)]
    ref, lref = oracle.sparse_attn(x["q"], x["k"], x["v"], m["rank"], m["cnt"], 2, items)
    o0, l0, s0, _ = oracle.sparse_attn_skip(x["q"], x["k"], x["v"], m["rank"], m["cnt"], 2, items, 0.0)
    assert s0.sum() == 0
    np.testing.assert_allclose(o0, ref, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(l0, lref, rtol=1e-12)
    # a case with skips: decisions passed in replace the oracle's own
    q, k, v = _skip_inputs()
    rank, cnt = _full_lists(4, shuffle_seed=4)
    items = [(0, 0, qb) for qb in range(4)]
    ref, _ = oracle.sparse_attn(q, k, v, rank, cnt, 1, items)
    o1, _, s1, _ = oracle.sparse_attn_skip(q, k, v, rank, cnt, 1, items, 0.6)
    assert s1.sum() > 0
    o2, _, _, _ = oracle.sparse_attn_skip(q, k, v, rank, cnt, 1, items, 0.6, skip_in=np.zeros_like(s1))
    np.testing.assert_allclose(o2, ref, rtol=1e-11, atol=1e-13)
    o3, _, _, _ = oracle.sparse_attn_skip(q, k, v, rank, cnt, 1, items, 0.0, skip_in=s1)
    np.testing.assert_array_equal(o3, o1)


# ------------------------------------------- o8 XAttention antidiagonal estimate
def _antidiag_numpy(q, k, h, S, causal=True):
    """numpy: the token-level score map of head h, each S x S sub-block summed
    along its antidiagonal (row offset S-1-t, column offset t), divided by
    sqrt(d) * S; strided rows softmax-normalised over sub-blocks on or below
    the diagonal; block estimates = mean over a block's strided rows."""
    B, N, H, d = q.shape
    Hkv = k.shape[2]
    qf = q[0, :, h].double().numpy()
    kf = k[0, :, h * Hkv // H].double().numpy()
    Z = qf @ kf.T
    n = N // S
    A = np.zeros((n, n))
    for t in range(S):
        A += Z[np.arange(n)[:, None] * S + S - 1 - t, np.arange(n)[None, :] * S + t]
    A /= math.sqrt(d) * S
    if causal:
        A[np.triu_indices(n, 1)] = -np.inf
    P = scipy.special.softmax(A, axis=1)
    rpb = 128 // S
    nb = N // 128
    out = []
    for qb in range(nb):
        rows = P[qb * rpb:(qb + 1) * rpb]
        out.extend(rows[:, kb * rpb:(kb + 1) * rpb].sum() / rpb for kb in range(qb + 1 if causal else nb))
    return np.array(out)


@pytest.mark.parametrize("S", [2, 4, 8, 16])
def test_xattn_mass_is_the_antidiagonal_sum_softmax(S):
    """o8 against the full score map summed along each sub-block's antidiagonal."""
    w = synth.small_workload(seqlen=512, heads=4, kv_heads=2, head_dim=32, groups=1)
    x = synth.make_inputs(w)
    mass = oracle.xattn_mass(x["q"], x["k"], S)
    for h in range(4):
        np.testing.assert_allclose(mass[0, h], _antidiag_numpy(x["q"], x["k"], h, S), rtol=1e-10, atol=1e-13)
    # every query block's estimates sum to one
    nb = 4
    for qb in range(nb):
        np.testing.assert_allclose(mass[0, :, qb * (qb + 1) // 2: qb * (qb + 1) // 2 + qb + 1].sum(-1), 1.0,
                                   atol=1e-12)


@pytest.mark.parametrize("S", [4, 16])
def test_xattn_noncausal_is_the_unmasked_antidiagonal_softmax(S):
    """Non-causal o8: every strided column, rows of all nb blocks summing to one;
    S = 1 on the last block equals o3's non-causal mass."""
    w = synth.small_workload(seqlen=384, heads=2, kv_heads=1, head_dim=32, groups=1)
    x = synth.make_inputs(w)
    mass = oracle.xattn_mass(x["q"], x["k"], S, causal=False)
    for h in range(2):
        np.testing.assert_allclose(mass[0, h], _antidiag_numpy(x["q"], x["k"], h, S, causal=False),
                                   rtol=1e-10, atol=1e-13)
    np.testing.assert_allclose(mass.reshape(1, 2, 3, 3).sum(-1), 1.0, atol=1e-12)
    m1 = oracle.xattn_mass(x["q"], x["k"], 1, causal=False)
    np.testing.assert_allclose(m1[:, :, 6:9], oracle.head_mass(x["q"], x["k"], causal=False), rtol=1e-12,
                               atol=1e-15)
    rank, cnt = oracle.find_blocks(mass, 3, 0.99, causal=False)
    for h in range(2):
        for qb in range(3):
            v = mass[0, h, qb * 3:(qb + 1) * 3]
            assert list(rank[0, h, qb * 3:(qb + 1) * 3]) == sorted(range(3), key=lambda kb: (-v[kb], kb))


def test_xattn_stride_one_is_the_exact_mass():
    """S = 1: strided rows are tokens, the antidiagonal is one entry, and the
    last block's estimates are o3's exact softmax mass."""
    w = synth.small_workload(seqlen=384, heads=4, kv_heads=2, head_dim=64, groups=1)
    x = synth.make_inputs(w)
    mass = oracle.xattn_mass(x["q"], x["k"], 1)
    exact = oracle.head_mass(x["q"], x["k"])
    np.testing.assert_allclose(mass[:, :, 3:6], exact, rtol=1e-12, atol=1e-15)


def test_find_blocks_brute_force():
    """The smallest number of blocks whose estimates reach tau (over all
    subsets) equals the prefix length; the prefix is ordered by (estimate
    desc, index asc) and reaches tau while one block fewer does not.  A sum
    that lands exactly on tau counts as reaching it (the equation's >=)."""
    exact = np.array([[[1.0, 0.25, 0.75, 0.125, 0.5, 0.375]]])  # qb 2: 0.125 + 0.5 + 0.375
    _, c = oracle.find_blocks(exact, 3, 0.875)
    assert list(c[0, 0]) == [1, 2, 2]
    rng = np.random.default_rng(8)
    nb = 5
    T = nb * (nb + 1) // 2
    for trial in range(30):
        m = np.zeros((1, 2, T))
        for qb in range(nb):
            v = rng.dirichlet(np.ones(qb + 1) * 0.5)
            if trial % 3 == 0 and qb >= 2:
                v[1] = v[2]  # a tie
            m[0, :, qb * (qb + 1) // 2: qb * (qb + 1) // 2 + qb + 1] = v
        tau = float(rng.choice([0.3, 0.5, 0.8, 0.95]))
        rank, cnt = oracle.find_blocks(m, nb, tau)
        for h in range(2):
            for qb in range(nb):
                v = m[0, h, qb * (qb + 1) // 2: qb * (qb + 1) // 2 + qb + 1]
                lst = rank[0, h, qb * (qb + 1) // 2: qb * (qb + 1) // 2 + qb + 1]
                assert sorted(lst) == list(range(qb + 1))
                assert all((v[a] > v[b_]) or (v[a] == v[b_] and a < b_) for a, b_ in zip(lst, lst[1:]))
                best = min(len(s) for r in range(1, qb + 2) for s in itertools.combinations(range(qb + 1), r)
                           if v[list(s)].sum() >= tau - 1e-12) if v.sum() >= tau - 1e-12 else qb + 1
                assert cnt[0, h, qb] == best


# --------------------------------------------------------- non-causal mode
def test_noncausal_dense_and_sparse_all_match_sdpa():
    """Non-causal: o6 equals torch SDPA without a mask (fp64, GQA), and o5 with
    every block selected equals o6."""
    w = synth.small_workload(seqlen=384, heads=4, kv_heads=2, head_dim=64)
    x = synth.make_inputs(w)
    q, k, v = x["q"], x["k"], x["v"]
    N = 384
    ref = sdpa_reference(q, k, v, mask=torch.ones(N, N, dtype=torch.bool))
    rows = [(0, h, i) for h in range(4) for i in (0, 5, 127, 200, 383)]
    od, lsed = oracle.dense_attn(q, k, v, rows, causal=False)
    for (b, h, i), oo in zip(rows, od):
        np.testing.assert_allclose(oo, ref[b, i, h].numpy(), rtol=1e-12, atol=1e-12)
    for (b, h, i), l in zip(rows, lsed):
        z = (q[b, i, h].double() @ k[b, :, h * 2 // 4].double().T) / 8.0
        assert l == pytest.approx(torch.logsumexp(z, 0).item(), abs=1e-12)
    m = oracle.prefill_masks(q, k, 1, mode=oracle.ALL, causal=False)
    assert list(m["cnt"][0, 0]) == [3, 3, 3]
    items = [(0, h, qb) for h in range(4) for qb in range(3)]
    o, lse = oracle.sparse_attn(q, k, v, m["rank"], m["cnt"], 1, items, causal=False)
    rows2 = [(0, h, qb * 128 + i) for (_, h, qb) in items for i in range(128)]
    od2, lsed2 = oracle.dense_attn(q, k, v, rows2, causal=False)
    np.testing.assert_allclose(o.reshape(-1, 64), od2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse.reshape(-1), lsed2, rtol=0, atol=1e-12)


def test_noncausal_sparse_matches_sdpa_with_block_mask():
    w = synth.small_workload(seqlen=512, heads=4, kv_heads=2, head_dim=64, groups=2)
    x = synth.make_inputs(w)
    q, k, v = x["q"], x["k"], x["v"]
    m = oracle.prefill_masks(q, k, 2, mode=oracle.FIXED_FRACTION, frac_permille=500, causal=False)
    nb = 4
    assert (m["cnt"] == 2).all()  # ceil(0.5 * 4)
    mask = torch.zeros(4, 512, 512, dtype=torch.bool)
    for h in range(4):
        g = h * 2 // 4
        for qb in range(nb):
            for kb in m["rank"][0, g, qb * nb: qb * nb + m["cnt"][0, h, qb]]:
                mask[h, qb * 128:(qb + 1) * 128, kb * 128:(kb + 1) * 128] = True
    ref = sdpa_reference(q, k, v, mask=mask[None])
    items = [(0, h, qb) for h in range(4) for qb in range(nb)]
    o, _ = oracle.sparse_attn(q, k, v, m["rank"], m["cnt"], 2, items, causal=False)
    for (b, h, qb), oo in zip(items, o):
        np.testing.assert_allclose(oo, ref[0, qb * 128:(qb + 1) * 128, h].numpy(), rtol=1e-12, atol=1e-12)


def test_noncausal_scores_mass_rank_budget():
    """Non-causal scores equal per-head unmasked numpy block maxima (G = H);
    head mass rows equal scipy softmax over all keys; lists are [0, qb, rest by
    score] over all nb blocks; counts are clamp(k_h, |F|, nb) and the fixed
    fraction ceil(p nb / 1000)."""
    w = synth.small_workload(seqlen=512, heads=3, kv_heads=3, head_dim=64, groups=3)
    x = synth.make_inputs(w)
    q, k = x["q"], x["k"]
    nb = 4
    _, _, qpb, kpb = oracle.pool(q, k, 3)
    sc = oracle.block_scores(qpb, kpb, causal=False)
    for h in range(3):
        s = (q[0, :, h].double().numpy() @ k[0, :, h].double().numpy().T) / 8.0
        ref = [s[a * 128:(a + 1) * 128, c * 128:(c + 1) * 128].max() for a in range(nb) for c in range(nb)]
        np.testing.assert_allclose(sc[0, h], ref, rtol=1e-13, atol=1e-13)
    mass = oracle.head_mass(q, k, causal=False)
    for h in range(3):
        z = (q[0, 384:, h].double().numpy() @ k[0, :, h].double().numpy().T) / 8.0
        p = scipy.special.softmax(z, axis=1)
        np.testing.assert_allclose(mass[0, h], p.reshape(128, nb, 128).sum(2).mean(0), rtol=1e-12, atol=1e-15)
    r = oracle.rank(sc, nb, causal=False)
    for h in range(3):
        for qb in range(nb):
            lst = list(r[0, h, qb * nb:(qb + 1) * nb])
            rest = sorted((kb for kb in range(1, nb) if kb != qb), key=lambda kb: (-sc[0, h, qb * nb + kb], kb))
            assert lst == ([0] + ([qb] if qb else []) + rest)
    bud, cnt = oracle.budget(r, mass, 3, 3, nb, oracle.DYNAMIC, 0.9, causal=False)
    for h in range(3):
        lst = r[0, h, (nb - 1) * nb:]
        cum = np.cumsum([int(np.rint(mass[0, h, kb] * 2.0 ** 40)) for kb in lst])
        kh = next(t + 1 for t in range(nb) if t + 1 >= 2 and cum[t] >= int(np.rint(0.9 * 2.0 ** 40)))
        assert bud[0, h] == kh
        assert list(cnt[0, h]) == [max(kh, 1)] + [max(kh, 2)] * (nb - 1)
    _, cf = oracle.budget(r, None, 3, 3, nb, oracle.FIXED_FRACTION, 0, 300, causal=False)
    assert (cf == 2).all()  # ceil(0.3 * 4) = 2


def _post_softmax_block_max(qp, kp, scale):
    """The reading the oracle does not take: a per-row causal softmax of the
    proxy logits before the 128 x 128 max-pool (numpy, fp64)."""
    N = qp.shape[0]
    z = scale * (qp @ kp.T)
    z[np.triu_indices(N, 1)] = -np.inf
    p = np.exp(z - z.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    nb = N // 128
    return np.array([p[qb * 128:(qb + 1) * 128, kb * 128:(kb + 1) * 128].max()
                     for qb in range(nb) for kb in range(qb + 1)])


def test_rank_invariant_under_positive_scale():
    """Proxy scores are pre-softmax scaled logits, so any positive factor on
    them (a different softmax scale, or pooling by sum instead of mean) scales
    every block maximum by that factor and leaves the ranked lists unchanged.
    Powers of two keep the scaling exact, so lists must match entry for entry.
    The same change of scale reorders the lists of the post-softmax reading,
    which is what makes the test able to tell the two readings apart."""
    w = synth.small_workload(seqlen=1024, heads=4, kv_heads=2, head_dim=64, needles=8, seed=17)
    x = synth.make_inputs(w)
    _, _, qpb, kpb = oracle.pool(x["q"], x["k"], 1)
    nb = 8
    base = oracle.block_scores(qpb, kpb)
    ranked = oracle.rank(base, nb)
    for c in (2.0 ** -7, 2.0 ** -3, 2.0 ** 4):
        sc = oracle.block_scores(qpb, kpb, scale=c)
        np.testing.assert_array_equal(sc, base * (c * 8.0))
        np.testing.assert_array_equal(oracle.rank(sc, nb), ranked)
    # group sum instead of group mean (4 heads: a factor of 4 on both proxies)
    sc = oracle.block_scores((qpb.float() * 4).bfloat16(), (kpb.float() * 4).bfloat16())
    np.testing.assert_array_equal(oracle.rank(sc, nb), ranked)
    # the post-softmax reading is not invariant on the same input
    q0 = qpb[0, 0].double().numpy()
    k0 = kpb[0, 0].double().numpy()
    lists = [oracle.rank(_post_softmax_block_max(q0, k0, c)[None, None], nb)
             for c in (2.0 ** -7, 1 / 8.0, 2.0 ** 4)]
    assert any(not np.array_equal(lists[0], l) for l in lists[1:])


@pytest.mark.parametrize("S", [2, 4])
@pytest.mark.parametrize("causal", [True, False])
def test_xattn_mass_uniform_closed_form(S, causal):
    """With every query zero all antidiagonal sums are 0, so each strided row's
    softmax is uniform over its valid strided columns (c <= R when causal, all
    N/S otherwise).  Block kb's estimate for query block qb is then the mean
    over qb's 128/S strided rows R of (valid columns of kb) / (valid columns),
    an exact rational worked out here without the oracle's loops."""
    from fractions import Fraction
    N, d = 512, 16
    nb, per = N // 128, 128 // S
    q = torch.zeros(1, N, 1, d).bfloat16()
    k = (torch.randn(1, N, 1, d, generator=torch.Generator().manual_seed(3))).bfloat16()
    got = oracle.xattn_mass(q, k, S, causal=causal)[0, 0]
    for qb in range(nb):
        for kb in range(qb + 1 if causal else nb):
            est = Fraction(0)
            for i in range(per):
                R = qb * per + i
                valid = R + 1 if causal else N // S
                inside = (min(R, (kb + 1) * per - 1) - kb * per + 1) if causal else per
                est += Fraction(max(inside, 0), valid)
            est /= per
            at = (qb * (qb + 1) // 2 if causal else qb * nb) + kb
            assert got[at] == pytest.approx(float(est), rel=1e-12, abs=1e-15), (qb, kb)
