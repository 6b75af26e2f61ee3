"""GPU parity of head pooling on inputs far from the synthetic workloads:
random bf16 bit patterns over a wide exponent range (sums that are not exact
even in fp64, so the result depends on the order of the additions), subnormals,
signed zeros, values whose sum overflows fp32, and groups whose size is not a
power of two (the mean is then a true division).  The kernel sums in fp64 in
ascending head order like the oracle, so the result must equal the oracle's
mean rounded once to bf16, bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import block_sparse_attention_pa_b200 as pa
from block_sparse_attention_pa_b200 import build

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    pa.lib()
    assert pa.device_status() == 0


def wide_bf16(rng, shape, emax):
    """bf16 tensors from random bit patterns with biased exponent <= emax
    (finite values; exponent 0 gives subnormals and zeros)."""
    bits = rng.integers(0, 65536, size=shape, dtype=np.int64)
    e = ((bits >> 7) & 0xFF) % (emax + 1)
    out = ((bits & 0x807F) | (e << 7)).astype(np.uint16)
    return torch.from_numpy(out.view(np.int16)).view(torch.bfloat16)


def same_bits(a, b):
    return torch.equal(a.cpu().contiguous().view(torch.int16), b.contiguous().view(torch.int16))


@pytest.mark.parametrize("N,H,Hkv,d,G,emax", [
    (256, 8, 2, 64, 1, 0x90),    # 8 heads per group, wide exponents
    (384, 28, 4, 128, 4, 0x90),  # 7 heads per group (true division)
    (128, 6, 3, 128, 2, 0x7F),   # 3 heads per group, |x| < 2
    (256, 12, 4, 128, 1, 0xFE),  # full finite range: fp32 sums overflow
])
def test_pool_bit_exact_wide_range(N, H, Hkv, d, G, emax):
    rng = np.random.default_rng(N * 131 + H * 7 + G)
    q = wide_bf16(rng, (1, N, H, d), emax)
    k = wide_bf16(rng, (1, N, Hkv, d), emax)
    q[0, :4, 0, :8] = torch.tensor([0.0, -0.0, 1e-40, -3e-39, 5e-41, 0.0, 1.0, -2.0]).bfloat16()
    q[0, 4, :, 0] = -0.0                   # an all-negative-zero group sums to +0
    k[0, 5, :, :8] = 9.0e-41               # a subnormal row of k
    qp, kp = pa.pool_heads(q.cuda(), k.cuda(), G)
    torch.cuda.synchronize()
    assert pa.device_status(clear=True) == 0
    _, _, qpb, kpb = oracle.pool(q, k, G)
    assert same_bits(qp, qpb)
    assert same_bits(kp, kpb)


def test_pool_sum_overflowing_fp32():
    """Two copies of the largest finite bf16 overflow an fp32 sum but not an
    fp64 one; their mean is the value itself."""
    big = torch.finfo(torch.bfloat16).max
    q = torch.full((1, 128, 2, 128), big, dtype=torch.bfloat16)
    k = torch.full((1, 128, 2, 128), -big, dtype=torch.bfloat16)
    qp, kp = pa.pool_heads(q.cuda(), k.cuda(), 1)
    torch.cuda.synchronize()
    assert pa.device_status(clear=True) == 0
    assert torch.equal(qp.cpu(), q[:, :, :1].permute(0, 2, 1, 3).reshape(qp.shape))
    assert torch.equal(kp.cpu(), k[:, :, :1].permute(0, 2, 1, 3).reshape(kp.shape))


@pytest.mark.parametrize("r", [2, 4])
def test_pool_strided_bit_exact_wide_range(r):
    """With a query-row stride r the q proxy holds rows r-1, 2r-1, ... of the
    full proxy; the k proxy is complete."""
    rng = np.random.default_rng(77 + r)
    q = wide_bf16(rng, (1, 512, 8, 128), 0x90)
    k = wide_bf16(rng, (1, 512, 2, 128), 0x90)
    qp, kp = pa.pool_heads(q.cuda(), k.cuda(), 2, score_stride=r)
    torch.cuda.synchronize()
    assert pa.device_status(clear=True) == 0
    _, _, qpb, kpb = oracle.pool(q, k, 2)
    assert same_bits(qp, qpb[:, :, r - 1::r])
    assert same_bits(kp, kpb)


def test_pool_batch_beyond_one_launch():
    """More sequences than one launch's grid holds along the batch axis
    (65535): the rest go to a second launch with offset pointers.  With one q
    head per group the q proxy of a row is that head's row and the k proxy the
    row of the KV head it reads, so the whole output is known exactly."""
    B, N, H, Hkv, d = 65537, 128, 2, 1, 64
    gen = torch.Generator(device="cuda")
    gen.manual_seed(5)
    q = torch.randn(B, N, H, d, device="cuda", dtype=torch.bfloat16, generator=gen)
    k = torch.randn(B, N, Hkv, d, device="cuda", dtype=torch.bfloat16, generator=gen)
    qp, kp = pa.pool_heads(q, k, H)
    torch.cuda.synchronize()
    assert pa.device_status(clear=True) == 0
    assert torch.equal(qp, q.permute(0, 2, 1, 3))
    assert torch.equal(kp, k.permute(0, 2, 1, 3).expand(B, H, N, d))
    del q, k, qp, kp
    torch.cuda.empty_cache()
