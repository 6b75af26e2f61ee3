"""pa_build_mask_noalloc: the mask builder for callers that cannot give the
library any device scratch memory (for example a plugin hook that receives
no workspace pointer, or a runtime that reserved all device memory up front and
forbids further cudaMalloc calls).  Its scratch lives in a fixed array inside
libpa.so instead.

The test calls the entry point through the C ABI and checks it against
pa_build_mask (which takes a caller workspace) on two calls in a row with
different inputs, the larger shape first: every scratch byte the second call
reads then still holds the first call's (non-zero) statistics, so a tile the
second call failed to write would show.  This file is collected last on
purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import block_sparse_attention_pa_b200 as pa
from block_sparse_attention_pa_b200 import build, synth


def _noalloc():
    build.build()
    L = pa.lib()
    f = L.pa_build_mask_noalloc
    P = ctypes.POINTER
    f.argtypes = [P(pa.Shape), P(pa.Budget), ctypes.c_void_p, ctypes.c_void_p, pa.Strides, ctypes.c_void_p,
                  pa.Strides, P(pa.MaskBufs), ctypes.c_void_p]
    f.restype = ctypes.c_int
    return f


def test_noalloc_rejects_shapes_beyond_its_scratch():
    """No GPU needed: the size check happens before anything is launched."""
    f = _noalloc()
    st = pa.Strides(0, 32 * 128, 128)
    bufs = pa.MaskBufs(256, 256, 256, 256)
    shape = pa.Shape(1, 131072, 32, 8, 128, 128, 1)  # 32 heads x 1024 blocks > 16384
    r = f(ctypes.byref(shape), ctypes.byref(pa.make_budget(pa.DYNAMIC, 0.9)), 256, 256, st, 256, st,
          ctypes.byref(bufs), None)
    assert r == 2
    assert b"16384" in pa.lib().pa_last_error()


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_twice():
    f = _noalloc()
    for call, (seed, N, H, Hkv, d, G, gamma) in enumerate([(12, 2048, 8, 2, 128, 2, 0.9),
                                                            (11, 1024, 8, 2, 64, 1, 0.95)]):
        w = synth.small_workload(seqlen=N, heads=H, kv_heads=Hkv, head_dim=d, groups=G, gamma=gamma, seed=seed)
        x = synth.make_inputs(w, device="cuda")
        q, k = x["q"], x["k"]
        qp, kp = pa.pool_heads(q, k, G)
        scores = pa.block_scores(qp, kp, H, Hkv)
        ref = pa.build_mask(scores, q, k, G, pa.DYNAMIC, gamma)

        shape = pa.make_shape(q, k, G)
        budget = pa.make_budget(pa.DYNAMIC, gamma)
        got = pa.Mask.empty(shape, q.device, True)
        bufs = got.bufs()
        r = f(ctypes.byref(shape), ctypes.byref(budget), scores.data_ptr(), q.data_ptr(), pa._strides(q),
              k.data_ptr(), pa._strides(k), ctypes.byref(bufs), pa._stream(q.device))
        assert r == 0, pa.lib().pa_last_error()
        torch.cuda.synchronize()
        assert pa.device_status() == 0

        # integer outputs bit-exact; masses within the head-mass tolerance of the parity tests
        assert torch.equal(got.rank, ref.rank), f"call {call}: rank"
        assert torch.equal(got.cnt, ref.cnt), f"call {call}: cnt"
        assert torch.equal(got.budget, ref.budget), f"call {call}: budget"
        mg, mr = got.mass.cpu().numpy(), ref.mass.cpu().numpy()
        assert np.all(np.abs(mg - mr) <= 2e-5 + 2e-3 * np.abs(mr)), f"call {call}: mass"


@pytest.mark.gpu
def test_noalloc_under_cuda_graph_capture():
    """After one eager call on the device (which looks up the scratch address),
    the entry point records into a CUDA graph: capture it on a side stream,
    replay the graph on new inputs copied into the captured buffers, and
    compare with an eager call on the same inputs bit for bit."""
    f = _noalloc()
    G, gamma = 2, 0.9
    w = synth.small_workload(seqlen=1536, heads=8, kv_heads=2, head_dim=128, groups=G, gamma=gamma, seed=21)
    x = synth.make_inputs(w, device="cuda")
    q, k = x["q"].clone(), x["k"].clone()
    shape = pa.make_shape(q, k, G)
    budget = pa.make_budget(pa.DYNAMIC, gamma)

    def call(scores, out, stream):
        bufs = out.bufs()
        r = f(ctypes.byref(shape), ctypes.byref(budget), scores.data_ptr(), q.data_ptr(), pa._strides(q),
              k.data_ptr(), pa._strides(k), ctypes.byref(bufs), stream)
        assert r == 0, pa.lib().pa_last_error()

    qp, kp = pa.pool_heads(q, k, G)
    scores = pa.block_scores(qp, kp, 8, 2)
    warm = pa.Mask.empty(shape, q.device, True)
    call(scores, warm, pa._stream(q.device))
    torch.cuda.synchronize()

    captured = pa.Mask.empty(shape, q.device, True)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            call(scores, captured, side.cuda_stream)
    torch.cuda.synchronize()

    # new inputs into the captured buffers, then replay
    x2 = synth.make_inputs(synth.small_workload(seqlen=1536, heads=8, kv_heads=2, head_dim=128, groups=G,
                                                gamma=gamma, seed=22), device="cuda")
    q.copy_(x2["q"])
    k.copy_(x2["k"])
    qp2, kp2 = pa.pool_heads(q, k, G)
    scores.copy_(pa.block_scores(qp2, kp2, 8, 2))
    g.replay()
    torch.cuda.synchronize()
    eager = pa.Mask.empty(shape, q.device, True)
    call(scores, eager, pa._stream(q.device))
    torch.cuda.synchronize()
    assert pa.device_status() == 0
    assert torch.equal(captured.rank, eager.rank)
    assert torch.equal(captured.cnt, eager.cnt)
    assert torch.equal(captured.budget, eager.budget)
    assert torch.equal(captured.mass, eager.mass)
    del g
