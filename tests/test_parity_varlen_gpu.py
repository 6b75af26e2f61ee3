"""GPU parity of the packed variable-length batch (pa_prefill_varlen): every
sequence equals pa_prefill run on that sequence alone (output bit for bit,
masks equal), and attention of sampled items against the oracle on the
sequence's own tokens with the GPU's mask."""
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
    # name,           cu_seqlens,                          H, Hkv, d,  G, mode,               gamma, frac, r, causal
    ("dyn_d64",       [0, 384, 1408, 1536, 2560],          8, 2,  64, 2, pa.DYNAMIC,          0.9,  0,    1, True),
    ("fixed_d128",    [0, 1024, 1152, 2176],               4, 2, 128, 1, pa.FIXED_FRACTION,   0.0,  300,  1, True),
    ("noncausal_r2",  [0, 640, 1024, 2048],                8, 2, 128, 2, pa.DYNAMIC,          0.95, 0,    2, False),
    ("single_seq",    [0, 1024],                           4, 1,  64, 1, pa.DYNAMIC,          0.9,  0,    1, True),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_varlen_equals_per_sequence(case):
    name, cu, H, Hkv, d, G, mode, gamma, frac, r, causal = case
    total = cu[-1]
    w = synth.small_workload(seqlen=total, heads=H, kv_heads=Hkv, head_dim=d, groups=G, gamma=gamma, needles=8,
                             seed=1100 + CASES.index(case))
    x = synth.make_inputs(w)
    qc, kc, vc = x["q"], x["k"], x["v"]
    q, k, v = qc.cuda(), kc.cuda(), vc.cuda()
    o, vm = pa.prefill_varlen(q, k, v, cu, G, mode, gamma, frac, score_stride=r, causal=causal)
    torch.cuda.synchronize()
    assert pa.device_status() == 0
    rng = np.random.default_rng(3)
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        qs, ks, vs = (t[:, a:b].contiguous() for t in (q, k, v))
        o1, m1 = pa.prefill(qs, ks, vs, G, mode, gamma, frac, score_stride=r, causal=causal)
        torch.cuda.synchronize()
        assert torch.equal(o[:, a:b], o1)
        mv = vm.views[s]
        assert torch.equal(mv.rank, m1.rank) and torch.equal(mv.cnt, m1.cnt) and torch.equal(mv.budget, m1.budget)
        if mode == pa.DYNAMIC:
            assert torch.equal(mv.mass, m1.mass)
        nb = (b - a) // 128
        items = [(0, int(rng.integers(H)), int(rng.integers(nb))) for _ in range(3)] + [(0, H - 1, nb - 1)]
        oref, _ = oracle.sparse_attn(qc[:, a:b].contiguous(), kc[:, a:b].contiguous(), vc[:, a:b].contiguous(),
                                     mv.rank.cpu().numpy(), mv.cnt.cpu().numpy(), G, items, causal=causal)
        og = torch.stack([o[0, a + qb * 128:a + (qb + 1) * 128, h] for (_, h, qb) in items]).float().cpu().numpy()
        diff = np.abs(og - oref)
        assert diff.max() <= 2e-2 and diff.mean() <= 2e-3, (diff.max(), diff.mean())
