// pool.cuh -- head pooling (ProxyAttn blog, "4. ProxyAttn method", Step 1
// "Head Pooling"): the proxy of group g is the mean of the group's q heads,
// and of the KV heads those q heads read.
//
// HBM-bound: every byte of q and k is read once and the proxies are written
// once.  One thread owns 8 consecutive head-dim elements (one 16-byte vector)
// of one (batch, token, group); a warp therefore reads whole 128-byte lines of
// each head row.  Sums run in fp64 over ascending heads and the quotient is
// rounded once to bf16, so the result equals the exact-mean definition bit for
// bit whenever the sum of the group's bf16 values is exact in fp64 (always,
// unless the values span more than ~2^40 in magnitude).
//
// With a query-row stride r only the q rows i = r-1 (mod r) are pooled (the
// only rows the strided block scores read), into row i/r of a [B][G][N/r][d]
// q proxy; the k proxy is always complete.
#pragma once
#include "sm100.cuh"

namespace pa {

struct PoolParams {
    const __nv_bfloat16 *q;
    const __nv_bfloat16 *k;
    __nv_bfloat16 *qp;
    __nv_bfloat16 *kp;
    int64_t qsb, qss, qsh, ksb, kss, ksh;
    int B, N, H, Hkv, G, d;
    int stride;  // query-row stride r (1: every row)
};

// The 8 bf16 values of v as fp64 (exact).
__device__ __forceinline__ void to_f64x8(double (&x)[8], const uint4 &v) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = static_cast<double>(__uint_as_float(w[i] << 16));
        x[2 * i + 1] = static_cast<double>(__uint_as_float(w[i] & 0xFFFF0000u));
    }
}

__device__ __forceinline__ void add_bf16x8(double (&acc)[8], const uint4 &v) {
    double x[8];
    to_f64x8(x, v);
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] += x[j];
}

// sum / n rounded to bf16.  When n is a power of two, sum * (1/n) is exact and
// therefore the same IEEE result as the (slow) fp64 division.
__device__ __forceinline__ uint4 mean_to_bf16x8(const double (&acc)[8], int n) {
    const bool pow2 = (n & (n - 1)) == 0;
    const double inv = 1.0 / static_cast<double>(n);
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const double m0 = pow2 ? acc[2 * i] * inv : acc[2 * i] / n;
        const double m1 = pow2 ? acc[2 * i + 1] * inv : acc[2 * i + 1] / n;
        const __nv_bfloat16 lo = __double2bfloat16(m0);
        const __nv_bfloat16 hi = __double2bfloat16(m1);
        w[i] = static_cast<uint32_t>(__bfloat16_as_ushort(lo)) |
               (static_cast<uint32_t>(__bfloat16_as_ushort(hi)) << 16);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

template <int D>
__global__ void __launch_bounds__(256, 3) pool_heads_kernel(PoolParams p) {
    constexpr int TPR = D / 8;  // threads per (token, group) row
    // grid (tokens * TPR / 256, G, B): no runtime division in the index math
    const uint32_t t = blockIdx.x * blockDim.x + threadIdx.x;
    const int i = static_cast<int>(t / TPR);
    if (i >= p.N) return;
    const int c = static_cast<int>(t % TPR) * 8;
    const int g = static_cast<int>(blockIdx.y);
    const int b = static_cast<int>(blockIdx.z);

    const int hpg = p.H / p.G;
    const int h0 = g * hpg;
    const __nv_bfloat16 *qrow = p.q + b * p.qsb + i * p.qss + c;
    const __nv_bfloat16 *krow = p.k + b * p.ksb + i * p.kss + c;
    const bool doq = (i % p.stride) == p.stride - 1;

    double aq[8], ak[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) aq[j] = ak[j] = 0.0;

    // The q heads first, in blocks of 4, software-pipelined: the next block's
    // 16-byte loads are in flight while this block is added (adds in ascending
    // head order).  Then the k proxy: for every q head h of the group in
    // ascending order it adds the row of its KV head v(h) = h * Hkv / H; v(h)
    // does not decrease with h, so each KV row is converted to fp64 once and
    // added once per q head reading it, which is the same sequence of
    // additions.  The group's distinct KV rows are loaded up to 4 per pass
    // (small blocks keep the kernel at 80 registers, three CTAs per SM).
    constexpr int KB = 4;  // KV rows loaded per pass
    const int hend = h0 + hpg;
    const int v_lo = static_cast<int>(static_cast<int64_t>(h0) * p.Hkv / p.H);
    const int v_hi = static_cast<int>(static_cast<int64_t>(hend - 1) * p.Hkv / p.H);
    if (doq) {
        constexpr int QB = 4;
        uint4 qa[QB], qb2[QB];
        auto load_blk = [&](uint4 (&dst)[QB], int t0) {
#pragma unroll
            for (int t = 0; t < QB; ++t)
                if (t0 + t < hpg) dst[t] = __ldg(reinterpret_cast<const uint4 *>(qrow + (h0 + t0 + t) * p.qsh));
        };
        auto add_blk = [&](const uint4 (&src)[QB], int t0) {
#pragma unroll
            for (int t = 0; t < QB; ++t)
                if (t0 + t < hpg) add_bf16x8(aq, src[t]);
        };
        load_blk(qa, 0);
        for (int t0 = 0; t0 < hpg; t0 += 2 * QB) {
            if (t0 + QB < hpg) load_blk(qb2, t0 + QB);
            add_blk(qa, t0);
            if (t0 + QB >= hpg) break;
            if (t0 + 2 * QB < hpg) load_blk(qa, t0 + 2 * QB);
            add_blk(qb2, t0 + QB);
        }
    }
    for (int v0 = v_lo; v0 <= v_hi; v0 += KB) {
        const int nv = min(KB, v_hi - v0 + 1);
        uint4 kvv[KB];
#pragma unroll
        for (int t = 0; t < KB; ++t)
            if (t < nv) kvv[t] = __ldg(reinterpret_cast<const uint4 *>(krow + (v0 + t) * p.ksh));
#pragma unroll
        for (int t = 0; t < KB; ++t) {
            if (t < nv) {
                const int v = v0 + t;
                // q heads reading KV head v: [ceil(v H / Hkv), ceil((v+1) H / Hkv)) within the group
                const int a = max(h0, static_cast<int>((static_cast<int64_t>(v) * p.H + p.Hkv - 1) / p.Hkv));
                const int z = min(hend, static_cast<int>((static_cast<int64_t>(v + 1) * p.H + p.Hkv - 1) / p.Hkv));
                double x[8];
                to_f64x8(x, kvv[t]);
                for (int r = a; r < z; ++r) {
#pragma unroll
                    for (int j = 0; j < 8; ++j) ak[j] += x[j];
                }
            }
        }
    }
    const int64_t o = ((static_cast<int64_t>(b) * p.G + g) * p.N + i) * D + c;
    *reinterpret_cast<uint4 *>(p.kp + o) = mean_to_bf16x8(ak, hpg);
    if (doq) {
        const int nq = p.N / p.stride;
        const int64_t oq = ((static_cast<int64_t>(b) * p.G + g) * nq + i / p.stride) * D + c;
        *reinterpret_cast<uint4 *>(p.qp + oq) = mean_to_bf16x8(aq, hpg);
    }
}

}  // namespace pa
