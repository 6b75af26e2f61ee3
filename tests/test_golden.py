"""The oracle against hand-derived worked examples in tests/golden (each file
names the page passage it follows).  No GPU."""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def load(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def test_golden_pool():
    g = load("pool_closed_form.json")
    N, d = g["seqlen"], g["head_dim"]
    H, Hkv = len(g["q_head_values"]), len(g["kv_head_values"])
    q = torch.empty(1, N, H, d)
    k = torch.empty(1, N, Hkv, d)
    for h, val in enumerate(g["q_head_values"]):
        q[:, :, h] = val
    for h, val in enumerate(g["kv_head_values"]):
        k[:, :, h] = val
    for case in g["cases"]:
        qp, kp, _, _ = oracle.pool(q.bfloat16(), k.bfloat16(), case["groups"])
        for gi in range(case["groups"]):
            assert np.all(qp[0, gi] == case["qp"][gi])
            assert np.all(kp[0, gi] == case["kp"][gi])


def test_golden_rank():
    g = load("rank_worked_example.json")
    qb = g["qb"]
    nb = qb + 1
    T = nb * (nb + 1) // 2
    s = np.zeros((1, 1, T))
    s[0, 0, T - nb:] = g["row_scores"]
    r = oracle.rank(s, nb)
    assert list(r[0, 0, T - nb:]) == g["list"]


def test_golden_budget():
    g = load("budget_worked_example.json")
    nb = g["nb"]
    T = nb * (nb + 1) // 2
    # scores that produce the given last-row list
    lst = g["last_row_list"]
    s = np.zeros((1, 1, T))
    for pos, kb in enumerate(lst[2:]):
        s[0, 0, T - nb + kb] = 100.0 - pos
    r = oracle.rank(s, nb)
    assert list(r[0, 0, T - nb:]) == lst
    mass = np.array(g["mass"])[None, None]
    for case in g["dynamic"]:
        bud, cnt = oracle.budget(r, mass, 1, 1, nb, oracle.DYNAMIC, case["gamma"])
        assert bud[0, 0] == case["k"]
        if "cnt" in case:
            assert list(cnt[0, 0]) == case["cnt"]
    _, cnt = oracle.budget(r, None, 1, 1, nb, oracle.FIXED_FRACTION, frac_permille=g["fixed_permille"])
    assert list(cnt[0, 0]) == g["fixed_cnt"]
    _, cnt = oracle.budget(r, None, 1, 1, nb, oracle.ALL)
    assert list(cnt[0, 0]) == g["all_cnt"]


def test_golden_uniform_attention():
    g = load("uniform_attention.json")
    N = g["seqlen"]
    q = torch.zeros(1, N, 1, 1).bfloat16()
    k = torch.randn(1, N, 1, 1, generator=torch.Generator().manual_seed(0)).bfloat16()
    v = torch.arange(N, dtype=torch.float32).reshape(1, N, 1, 1).bfloat16()
    m = oracle.prefill_masks(q, k, 1, mode=oracle.ALL)
    o, lse = oracle.sparse_attn(q, k, v, m["rank"], m["cnt"], 1, [(0, 0, 0)])
    for i, oi, li in zip(g["rows"], g["o"], g["lse"]):
        assert o[0, i, 0] == pytest.approx(oi, abs=1e-12)
        assert lse[0, i] == pytest.approx(li, abs=1e-12)
        assert li == pytest.approx(math.log(i + 1), abs=1e-15)
