"""Seeded synthetic inputs for block-sparse prefill attention.

This module only draws random tensors; it holds none of the method's
arithmetic (no pooling, scoring, ranking, budget or attention).  Both the CUDA
path and the CPU oracle consume the tensors it returns, so a parity test feeds
the two sides byte-identical bf16 inputs.

Recipe (shapes follow the Llama-3.1-8B / Qwen2.5-7B long-context prefill
workloads on the ProxyAttn pages, "5. Experiments"; there is no dataset here):

* ``Q, K, V = 0.5 * N(0, 1)`` in the ``[B, N, heads, d]`` layout.
* A unit direction ``u`` (``u = z / |z|`` with ``z ~ N(0, I_d)``) is shared by
  every head, or one ``u_g`` per GQA group (one per KV head) when
  ``per_group_direction`` is set.
* ``Q[:, :, h] += 2.0 * s_h * u_{dir(h)}`` where ``s_h = 1`` or, with
  ``per_head_sharpness``, ``s_h ~ U[0.5, 3]``.
* ``n_needles`` positions are drawn without replacement from ``[1, N)`` and
  ``K[:, pos, kvh] += 2.0 * u_{dir(kvh)}`` for every KV head.
* ``K[:, 0] *= 4`` (an attention sink).
* Optional, a labelled extra that never replaces a workload below
  (``logit_units``): the direction weight 2.0 on Q and on the needles becomes
  ``w = 2 d^(1/4)``, so a needle lifts the scaled logit of head h by
  ``w^2 s_h / sqrt(d) = 4 s_h`` instead of ``4 s_h / sqrt(d)`` (about 0.35 s_h
  at d = 128).  Attention is then concentrated enough that the per-head
  dynamic budgets differ.
* Optional, for the running-max block skip only (``sink_logit`` > 0, a
  labelled extra, never one of the five workloads below): ``K[:, 0, kvh] +=
  (sink_logit * sqrt(d) / 2) * u_{dir(kvh)}``, which lifts the sink's scaled
  logit of head h by about ``s_h * sink_logit`` above the other keys, the way
  trained models concentrate attention on their first token.
* Everything is drawn in fp32 with a seeded ``torch.Generator`` on ``device``
  and cast to bf16 (round to nearest even).  A given (workload, seed, device
  type) always yields the same tensors.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    seqlen: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    num_groups: int
    gamma: float
    n_needles: int
    per_head_sharpness: bool
    per_group_direction: bool
    seed: int
    sink_logit: float = 0.0
    logit_units: bool = False

    @property
    def nb(self) -> int:
        return self.seqlen // 128

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads: a tiny GQA layer, then Llama-3.1-8B and Qwen2.5-7B shaped
# prefill layers from 32K to 256K tokens.
WORKLOADS = {
    "tiny_gqa_n1024": Workload("tiny_gqa_n1024", 1, 1024, 8, 2, 64, 1, 0.95, 16, False, False, 1234),
    "llama8b_n32k": Workload("llama8b_n32k", 1, 32768, 32, 8, 128, 1, 0.95, 64, True, False, 1235),
    "llama8b_n128k": Workload("llama8b_n128k", 1, 131072, 32, 8, 128, 1, 0.95, 256, True, False, 1236),
    "qwen7b_n64k": Workload("qwen7b_n64k", 1, 65536, 28, 4, 128, 4, 0.9, 0, True, True, 1237),
    "llama8b_n256k": Workload("llama8b_n256k", 1, 262144, 32, 8, 128, 1, 0.95, 512, True, False, 1238),
}

# Labelled extra for the running-max block skip: the 128K Llama shape with a
# strong attention sink (see ``sink_logit`` above).
EXTRA_WORKLOADS = {
    "llama8b_n128k_sink": Workload("llama8b_n128k_sink", 1, 131072, 32, 8, 128, 1, 0.95, 256, True, False, 1239,
                                   sink_logit=4.0),
}


def make_inputs(w: Workload, device="cpu", seed: int | None = None):
    """Return ``dict(q, k, v, s, needles)``; q/k/v are bf16 ``[B, N, heads, d]``."""
    B, N, H, Hkv, d = w.batch, w.seqlen, w.num_q_heads, w.num_kv_heads, w.head_dim
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed if seed is None else seed)
    f32 = dict(device=dev, dtype=torch.float32)

    n_dirs = Hkv if w.per_group_direction else 1
    u = torch.randn(n_dirs, d, generator=g, **f32)
    u = u / u.norm(dim=-1, keepdim=True)
    q = torch.randn(B, N, H, d, generator=g, **f32).mul_(0.5)
    k = torch.randn(B, N, Hkv, d, generator=g, **f32).mul_(0.5)
    v = torch.randn(B, N, Hkv, d, generator=g, **f32).mul_(0.5)
    if w.per_head_sharpness:
        s = torch.rand(H, generator=g, **f32) * 2.5 + 0.5
    else:
        s = torch.ones(H, **f32)
    # direction index of each q head / kv head (GQA group = q heads of one kv head)
    q_dir = (torch.arange(H, device=dev) * Hkv // H) if n_dirs > 1 else torch.zeros(H, dtype=torch.long, device=dev)
    kv_dir = torch.arange(Hkv, device=dev) if n_dirs > 1 else torch.zeros(Hkv, dtype=torch.long, device=dev)
    wu = 2.0 * d ** 0.25 if w.logit_units else 2.0  # direction weight
    q += (wu * s[:, None] * u[q_dir])[None, None]
    n_needles = min(w.n_needles, max(N - 1, 0))
    if n_needles > 0:
        needles = torch.randperm(N - 1, generator=g, device=dev)[:n_needles] + 1
        k[:, needles] += (wu * u[kv_dir])[None, None]
    else:
        needles = torch.zeros(0, dtype=torch.long, device=dev)
    k[:, 0] *= 4.0
    if w.sink_logit > 0.0:
        k[:, 0] += (w.sink_logit * d ** 0.5 / 2.0 * u[kv_dir])[None]
    return dict(
        q=q.to(torch.bfloat16),
        k=k.to(torch.bfloat16),
        v=v.to(torch.bfloat16),
        s=s,
        needles=needles,
    )


def small_workload(seqlen=512, heads=4, kv_heads=2, head_dim=64, groups=1, gamma=0.9,
                   needles=8, batch=1, seed=7, sharp=True, per_group=False, sink_logit=0.0,
                   logit_units=False) -> Workload:
    """A small custom workload for parity tests (sizes the oracle finishes in seconds)."""
    return Workload(f"custom_n{seqlen}_h{heads}_kv{kv_heads}_d{head_dim}_g{groups}",
                    batch, seqlen, heads, kv_heads, head_dim, groups, gamma, needles,
                    sharp, per_group, seed, sink_logit, logit_units)
