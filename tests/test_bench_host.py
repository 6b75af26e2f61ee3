"""The benchmark's multi-rank host logic on CPU (gloo, world size 2): the job
time is the max over ranks and `value` counts every rank's layer; the
reference arm prints only on rank 0."""
import json
import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        t = bench.max_over_ranks(10.0 + 5.0 * rank, torch.device("cpu"))
        # one rank's rejected clock record makes every rank measure again
        again = bench.agree_any(rank == 1, torch.device("cpu"), True)
        dist.barrier()
        out[rank] = (t, again)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    port = 29500 + os.getpid() % 1000
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
        assert out[0] == out[1] == (15.0, True)


def test_single_process_and_per_layer():
    assert bench.max_over_ranks(3.5, torch.device("cpu")) == 3.5
    assert bench.per_layer(100.0, 4) == 25.0


@pytest.mark.parametrize("rank,expect_line", [(0, True), (1, False)])
def test_reference_arm_prints_on_rank0_only(rank, expect_line):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        "tiny_gqa_n1024", "--steps", "1", "--warmup", "0", "--gpus", "2"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    if expect_line:
        d = json.loads(lines[-1])
        assert d["impl"] == "reference" and d["unit"] == "ms/layer" and d["e2e"]["h2d_bytes_per_step"] == 0
        assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    else:
        assert lines == []


def test_selected_blocks_matches_loops():
    """The bench's selection map (used to compare two estimates) against plain
    loops over the ranked lists and counts."""
    import types
    import numpy as np
    import torch
    rng = np.random.default_rng(3)
    B, H, G, nb = 2, 4, 2, 6
    T = nb * (nb + 1) // 2
    rank = np.zeros((B, G, T), np.int32)
    for b in range(B):
        for g in range(G):
            for qb in range(nb):
                rank[b, g, qb * (qb + 1) // 2: qb * (qb + 1) // 2 + qb + 1] = rng.permutation(qb + 1)
    cnt = np.stack([[[int(rng.integers(1, qb + 2)) for qb in range(nb)] for _ in range(H)] for _ in range(B)])
    pipe = types.SimpleNamespace(B=B, H=H, G=G, nb=nb, T=T,
                                 mask=types.SimpleNamespace(rank=torch.from_numpy(rank),
                                                            cnt=torch.from_numpy(cnt.astype(np.int32))))
    got = bench.selected_blocks(pipe).numpy()
    ref = np.zeros((B, H, T), bool)
    for b in range(B):
        for h in range(H):
            g = h * G // H
            for qb in range(nb):
                s = qb * (qb + 1) // 2
                for kb in rank[b, g, s:s + cnt[b, h, qb]]:
                    ref[b, h, s + kb] = True
    assert np.array_equal(got, ref)


def test_gen_logit_is_a_labelled_extra(monkeypatch):
    """--gen logit keeps the workload's shape but switches the generator to the
    logit-unit recipe and renames the workload, so a bench line can never be
    mistaken for the literal configuration."""
    monkeypatch.setattr(sys, "argv", ["bench.py", "--workload", "llama8b_n32k", "--gen", "logit"])
    w = bench.resolve_workload(bench.parse_args())
    base = bench.synth.WORKLOADS["llama8b_n32k"]
    assert w.logit_units and w.name == "llama8b_n32k_logit"
    assert (w.seqlen, w.num_q_heads, w.num_kv_heads, w.head_dim, w.gamma) == \
        (base.seqlen, base.num_q_heads, base.num_kv_heads, base.head_dim, base.gamma)
    monkeypatch.setattr(sys, "argv", ["bench.py", "--workload", "llama8b_n32k"])
    assert bench.resolve_workload(bench.parse_args()) == base


def test_traffic_only_for_the_profiled_kernel_and_workload(tmp_path):
    """roofline.traffic comes from committed ncu counters only while the
    attention sources hash to what was profiled, and only for the exact
    workload and budget of the capture; anything else reports null.  (The
    committed profiles/counters.json is a record of an earlier kernel version,
    so the bench reports null for today's; the rule is checked on a copy that
    carries today's hash.)"""
    with open(os.path.join(ROOT, "profiles", "counters.json")) as f:
        rec = json.load(f)["attn_kernel"]
    fresh = dict(rec, source_sha256=bench.sources_sha256(bench.ATTN_SOURCES))
    p = tmp_path / "counters.json"
    p.write_text(json.dumps({"attn_kernel": fresh}))
    ctr = bench.counters_for("attn_kernel", bench.ATTN_SOURCES, path=str(p))
    assert ctr is not None
    w = bench.synth.WORKLOADS[ctr["workload"]]
    mode = {"dynamic": 0, "fixed": 1, "all": 2}[ctr["mode"]]
    got = bench.traffic_for(ctr, w, ctr["groups"], mode, ctr.get("gamma", 0.95))
    assert got == float(ctr["dram_bytes"]) == float(ctr["dram_bytes_read"] + ctr["dram_bytes_write"])
    assert bench.traffic_for(ctr, w, ctr["groups"] + 3, mode, ctr.get("gamma", 0.95)) is None
    assert bench.traffic_for(ctr, w, ctr["groups"], mode, 0.5) is None
    other = bench.synth.WORKLOADS["llama8b_n32k"]
    assert bench.traffic_for(ctr, other, ctr["groups"], mode, ctr.get("gamma", 0.95)) is None
    assert bench.traffic_for(ctr, w, ctr["groups"], mode, ctr.get("gamma", 0.95), stride=4) is None
    # a changed kernel source invalidates the counters
    assert bench.counters_for("attn_kernel", bench.ATTN_SOURCES[:1], path=str(p)) is None
    assert bench.traffic_for(None, w, ctr["groups"], mode, 0.95) is None
    # the committed record no longer matches today's sources: the bench reports null
    if rec["source_sha256"] != fresh["source_sha256"]:
        assert bench.counters_for("attn_kernel", bench.ATTN_SOURCES) is None


def test_clock_records_that_force_a_second_measurement():
    ok = {"sm_mhz": 1695.0, "sm_max_mhz": 1965.0, "samples": 20, "reasons": ["sw_power_cap"]}
    assert not bench.clocks_rejected(ok)
    assert not bench.clocks_rejected(None)
    for r in ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"):
        assert bench.clocks_rejected(dict(ok, reasons=["sw_power_cap", r]))
    # a clock held low with no power-cap reason reads as a leftover lock
    assert bench.clocks_rejected(dict(ok, sm_mhz=1200.0, reasons=[]))
    assert not bench.clocks_rejected(dict(ok, sm_mhz=1200.0))
    assert not bench.clocks_rejected(dict(ok, sm_mhz=1900.0, reasons=[]))
    assert bench.agree_any(True, "cpu", False) and not bench.agree_any(False, "cpu", False)


def test_cpu_sample_uses_every_thread_and_both_arms_share_config():
    """The CPU-baseline leg and the reference arm take the same oracle sample,
    whose stages keep every oracle thread busy, and print the same config."""
    import argparse
    import oracle
    from block_sparse_attention_pa_b200 import synth
    w = synth.small_workload(seqlen=1024, heads=8, kv_heads=2, head_dim=64)
    x = synth.make_inputs(w)
    ms, det, used, sample = bench.oracle_estimate(x, w, 1, 0, 0.95, 0, seed=0)
    threads = oracle.num_threads()
    assert ms > 0 and set(det) == {"pool_s", "scores_s", "mass_s", "rank_s", "budget_s", "attn_s"}
    assert used["attn"] == min(threads, 8 * 8 * 128) and used["pool"] == min(threads, 1024)
    args = argparse.Namespace(non_causal=False, estimator="proxy", score_stride=1, skip_threshold=0.0, tau=0.9,
                              xattn_stride=8)
    cfg = bench.line_config(args, w, 1, 0, 0.95, 0, 1)
    assert cfg["parallelism"] == "replicas x1" and cfg["causal"] is True and cfg["workload"] == w.name
