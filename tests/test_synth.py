"""The seeded input generator and its labelled extra with the direction weight
in logit units (the recipe in block_sparse_attention_pa_b200/synth.py).  The
generator holds none of the method's arithmetic; these tests pin what it
draws, and that the logit-unit extra is the variant whose per-head dynamic
budgets differ (the reason it exists)."""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_pa_b200 import synth


def test_same_seed_same_tensors_and_sink():
    w = synth.small_workload(seqlen=512, heads=4, kv_heads=2, head_dim=64, needles=8, seed=3)
    a, b = synth.make_inputs(w), synth.make_inputs(w)
    for n in ("q", "k", "v"):
        assert a[n].dtype == torch.bfloat16 and torch.equal(a[n], b[n])
    c = synth.make_inputs(w, seed=4)
    assert not torch.equal(a["q"], c["q"])
    # the sink row is four times the size of the other key rows on average
    kn = a["k"].float().norm(dim=-1)[0]            # [N, Hkv]
    assert (kn[0] > 3.0 * kn[1:].mean(dim=0)).all()


@pytest.mark.parametrize("d", [64, 128])
def test_logit_units_scale_the_direction(d):
    """With the same seed the two recipes draw the same noise, so logit minus
    literal is (w - 2) s_h u on every q row and (w - 2) u on every needle row of
    K, with w = 2 d^(1/4); everything else is unchanged."""
    base = synth.small_workload(seqlen=512, heads=4, kv_heads=2, head_dim=d, needles=8, seed=5)
    lit = synth.make_inputs(base)
    log = synth.make_inputs(base.replace(logit_units=True))
    assert torch.equal(lit["v"], log["v"])
    wu = 2.0 * d ** 0.25
    s = lit["s"]
    dq = log["q"].float() - lit["q"].float()          # [1, N, H, d]
    step = dq[0].mean(dim=0)                          # [H, d]: (w - 2) s_h u
    for h in range(4):
        u_h = step[h] / ((wu - 2.0) * s[h])
        assert abs(u_h.norm().item() - 1.0) < 0.02
        # every token row carries the same shift, up to bf16 rounding of both sides
        dev = (dq[0, :, h] - step[h]).abs().max().item()
        assert dev < 0.05 * (wu - 2.0) * s[h].item()
    dk = log["k"].float() - lit["k"].float()          # [1, N, Hkv, d]
    moved = dk[0].abs().amax(dim=(1, 2)) > 0
    needles = set(lit["needles"].tolist())
    assert set(torch.nonzero(moved).ravel().tolist()) == needles
    kstep = dk[0, sorted(needles)].mean(dim=0)        # [Hkv, d]: (w - 2) u
    assert ((kstep.norm(dim=-1) / (wu - 2.0)) - 1.0).abs().max().item() < 0.02


def test_logit_units_make_per_head_budgets_differ():
    """The literal recipe gives nearly uniform attention (every head keeps
    almost every block at gamma 0.95); in logit units the sharper heads need
    fewer blocks, the sharpest the fewest."""
    base = synth.small_workload(seqlen=4096, heads=8, kv_heads=2, head_dim=64, needles=32, gamma=0.95, seed=11)
    budgets = {}
    for logit in (False, True):
        x = synth.make_inputs(base.replace(logit_units=logit))
        m = oracle.prefill_masks(x["q"], x["k"], 1, oracle.DYNAMIC, 0.95)
        budgets[logit] = np.asarray(m["budget"]).ravel()
        s = x["s"].numpy()
    nb = base.nb
    assert (budgets[False] >= nb - 2).all() and len(set(budgets[False].tolist())) == 1
    assert budgets[True].max() - budgets[True].min() >= 5
    assert int(np.argmin(budgets[True])) == int(np.argmax(s))


def test_per_group_directions_are_shared_within_a_group_only():
    """The Qwen-shaped recipe draws one direction per GQA group: the mean q row
    of a head points along its group's u_g (shared by the group's heads, scaled
    by s_h), and the groups' directions differ."""
    w = synth.small_workload(seqlen=2048, heads=8, kv_heads=4, head_dim=64, needles=0, seed=9, per_group=True)
    x = synth.make_inputs(w)
    mean = x["q"].float()[0].mean(dim=0)                 # [H, d]: 2 s_h u_{g(h)} + noise of size ~0.5/sqrt(N)
    dirs = mean / mean.norm(dim=-1, keepdim=True)
    cos = dirs @ dirs.T
    for a in range(8):
        for b in range(8):
            same = a * 4 // 8 == b * 4 // 8
            assert (cos[a, b] > 0.99) if same else (abs(cos[a, b]) < 0.6), (a, b, float(cos[a, b]))
    # the norm of each head's mean is 2 s_h
    assert torch.allclose(mean.norm(dim=-1), 2.0 * x["s"], rtol=0.03)
    # no needles were asked for: K carries no direction apart from the sink scaling
    assert x["needles"].numel() == 0
