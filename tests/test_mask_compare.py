"""The end-to-end mask comparison rules (tests/mask_compare.py) on the CPU:
lists ranked from fp32-rounded oracle scores pass as near ties of the fp64
ranking, while a planted swap of two blocks that are not tied, a dropped
block or a budget one block off (away from the threshold) fails."""
import numpy as np
import pytest

import oracle
from block_sparse_attention_pa_b200 import synth

from mask_compare import check_budgets, compare_lists


@pytest.fixture(scope="module")
def own():
    w = synth.small_workload(seqlen=2048, heads=4, kv_heads=2, head_dim=64, groups=2, gamma=0.9,
                             needles=8, seed=5, logit_units=True)
    x = synth.make_inputs(w)
    ref = oracle.prefill_masks(x["q"], x["k"], 2, oracle.DYNAMIC, 0.9)
    return w, ref


def test_fp32_rounded_scores_are_near_ties(own):
    w, ref = own
    nb = w.nb
    r32 = oracle.rank(ref["scores"].astype(np.float32), nb)
    rows = [(0, g, qb) for g in range(2) for qb in range(nb)]
    nrows, npos, tot = compare_lists(r32, ref["rank"], ref["scores"], rows, nb)
    assert tot == 2 * nb * (nb + 1) // 2 and npos <= tot // 100


def test_planted_swap_is_caught(own):
    w, ref = own
    nb = w.nb
    bad = ref["rank"].copy()
    qb = nb - 1
    o = qb * (qb + 1) // 2
    s = ref["scores"][0, 0, o:o + qb + 1]
    lst = bad[0, 0, o:o + qb + 1]
    # swap the best ranked free block with the worst one (far from a tie)
    assert abs(s[lst[2]] - s[lst[-1]]) > 1e-2
    lst[2], lst[-1] = lst[-1], lst[2]
    with pytest.raises(AssertionError):
        compare_lists(bad, ref["rank"], ref["scores"], [(0, 0, qb)], nb)
    dropped = ref["rank"].copy()
    dropped[0, 0, o + 2] = dropped[0, 0, o + 3]  # a block listed twice, another missing
    with pytest.raises(AssertionError):
        compare_lists(dropped, ref["rank"], ref["scores"], [(0, 0, qb)], nb)


def test_budget_rules(own):
    w, ref = own
    nb, H = w.nb, 4
    heads = [(0, h) for h in range(H)]
    assert check_budgets(ref["budget"], ref["rank"], ref["budget"], ref["mass"], heads, H, 2, nb, 0.9) == 0
    # one block more or less than the minimal prefix, away from the threshold, fails
    last = ref["rank"][0, 0, (nb - 1) * nb // 2:]
    cum = np.concatenate([[0.0], np.cumsum(ref["mass"][0, 0][last])])
    k = int(ref["budget"][0, 0])
    tried = 0
    for kk in (k - 1, k + 1):
        if 2 <= kk <= nb and abs(cum[min(kk, k)] - 0.9) > 1e-3:
            bad = ref["budget"].copy()
            bad[0, 0] = kk
            with pytest.raises(AssertionError):
                check_budgets(bad, ref["rank"], ref["budget"], ref["mass"], heads[:1], H, 2, nb, 0.9)
            tried += 1
    assert tried >= 1
