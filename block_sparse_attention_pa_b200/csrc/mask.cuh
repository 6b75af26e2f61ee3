// mask.cuh -- from block scores and last-block partial softmax statistics to
// the block-sparse mask (ProxyAttn blog, "4. ProxyAttn method": Step 1 "Block
// Ranking" and Step 2 "dynamic budget"; the threshold rule is XAttention's
// find_blocks, XAttention blog 2.2).
//
//   mass_combine_kernel  exact softmax normalisation across all KV blocks of
//                        each last-block row, then mass[kb] = mean over rows
//   rank_kernel          per (b, g, qb): [0, qb, then blocks 1..qb-1 by
//                        (score desc, index asc)] via a bitonic sort of
//                        64-bit keys in shared memory
//   budget_kernel        per (b, h): fixed-point prefix scan of the head's
//                        masses along the last row's list -> k_h, then the
//                        per-row counts
#pragma once
#include <cooperative_groups.h>

#include "sm100.cuh"

namespace pa {

// ------------------------------------------------------------ mass combine
// partial: [B*H][nb][128] (m, l) with m the log2-domain row max of a tile and
// l the sum of exp2(x - m) over its valid entries (m = -inf, l = 0 for a tile
// with no valid entry in the row).
//
// One cluster of kMcCta CTAs per (b, h); CTA c owns the key blocks
// [c*nb/kMcCta, (c+1)*nb/kMcCta).  Each CTA reduces its blocks to a per-row
// (M, L); after a cluster barrier every CTA combines the kMcCta partial
// statistics of each row in CTA order through distributed shared memory (the
// same fixed order in every CTA, so all hold identical normalisers and the
// result is deterministic), then writes mass[kb] for its own blocks.
constexpr int kMcCta = 8;
constexpr int kMcThreads = 512;

// (M, L) <- (M, L) merged with the tile statistics v[0..n), in log2 domain
template <int n>
__device__ __forceinline__ void online_merge(float &M, float &L, const float2 (&v)[n]) {
    float mx = M;
#pragma unroll
    for (int j = 0; j < n; ++j) mx = fmaxf(mx, v[j].x);
    if (mx == -INFINITY) return;  // nothing valid so far
    float l = (M == -INFINITY) ? 0.0f : L * exp2f(M - mx);
#pragma unroll
    for (int j = 0; j < n; ++j) l += (v[j].x == -INFINITY) ? 0.0f : v[j].y * exp2f(v[j].x - mx);
    M = mx;
    L = l;
}

__global__ void __cluster_dims__(kMcCta, 1, 1) __launch_bounds__(kMcThreads)
    mass_combine_kernel(const float2 *__restrict__ partial, float *__restrict__ mass, int nb) {
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    __shared__ float sM[4][128], sL[4][128];  // per quarter, then [0] = this CTA's (M, L)
    __shared__ float gM[128], gI[128];         // row max and 1/L over all blocks
    const long long bh = blockIdx.x / kMcCta;
    const int c = static_cast<int>(cluster.block_rank());
    const int lo = static_cast<int>(static_cast<long long>(c) * nb / kMcCta);
    const int hi = static_cast<int>(static_cast<long long>(c + 1) * nb / kMcCta);
    const float2 *part = partial + bh * nb * 128;
    const int tid = threadIdx.x;
    const int r = tid & 127, qt = tid >> 7;  // row, quarter of the CTA's blocks

    float M = -INFINITY, L = 0.0f;
    int kb = lo + qt;
    for (; kb + 12 < hi; kb += 16) {  // four independent loads per merge
        float2 v[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) v[j] = part[static_cast<long long>(kb + 4 * j) * 128 + r];
        online_merge<4>(M, L, v);
    }
    for (; kb < hi; kb += 4) {
        float2 v[1] = {part[static_cast<long long>(kb) * 128 + r]};
        online_merge<1>(M, L, v);
    }
    sM[qt][r] = M;
    sL[qt][r] = L;
    __syncthreads();
    if (tid < 128) {
        float2 v[3] = {make_float2(sM[1][r], sL[1][r]), make_float2(sM[2][r], sL[2][r]),
                       make_float2(sM[3][r], sL[3][r])};
        float m0 = sM[0][r], l0 = sL[0][r];
        online_merge<3>(m0, l0, v);
        sM[0][r] = m0;
        sL[0][r] = l0;
    }
    cluster.sync();  // every CTA's (M, L) visible cluster-wide
    if (tid < 128) {
        float Mx = -INFINITY, Lx = 0.0f;
#pragma unroll 1
        for (int cc = 0; cc < kMcCta; ++cc) {
            const float *rM = cluster.map_shared_rank(&sM[0][0], cc);
            const float *rL = cluster.map_shared_rank(&sL[0][0], cc);
            float2 v[1] = {make_float2(rM[r], rL[r])};
            online_merge<1>(Mx, Lx, v);
        }
        gM[r] = Mx;
        gI[r] = 1.0f / Lx;
    }
    cluster.sync();  // remote reads done before any CTA exits; gM/gI visible

    const int warp = tid >> 5, lane = tid & 31;
    float Mr[4], Ir[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        Mr[j] = gM[lane + 32 * j];
        Ir[j] = gI[lane + 32 * j];
    }
    for (int b = lo + warp; b < hi; b += kMcThreads / 32) {
        float s = 0.0f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 v = part[static_cast<long long>(b) * 128 + lane + 32 * j];
            s += (v.x == -INFINITY) ? 0.0f : v.y * exp2f(v.x - Mr[j]) * Ir[j];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) mass[bh * nb + b] = s * (1.0f / 128.0f);
    }
}

// ------------------------------------------------------------------- rank
__device__ __forceinline__ uint32_t score_desc_key(float f) {
    const uint32_t u = __float_as_uint(f + 0.0f);  // -0 and +0 compare equal
    const uint32_t ord = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return ~ord;  // larger score -> smaller key
}

// One CTA per (b, g, qb); dynamic smem holds P = pow2 >= n keys.  Causal
// rows hold blocks 0..qb at qb(qb+1)/2; non-causal rows all nb blocks at
// qb*nb.  The sorted blocks are the row's blocks other than 0 and qb: the
// i-th of them is i+1, or i+2 once i+1 reaches qb.
__global__ void __launch_bounds__(256) rank_kernel(const float *__restrict__ scores, int32_t *__restrict__ rank,
                                                   int nb, int causal) {
    extern __shared__ unsigned long long keys[];
    const long long bg = blockIdx.x / nb;
    const int qb = nb - 1 - static_cast<int>(blockIdx.x % nb);  // long rows first
    const long long T = causal ? static_cast<long long>(nb) * (nb + 1) / 2 : static_cast<long long>(nb) * nb;
    const long long row0 = bg * T + (causal ? static_cast<long long>(qb) * (qb + 1) / 2 : static_cast<long long>(qb) * nb);
    const float *srow = scores + row0;
    int32_t *out = rank + row0;
    const int lead = qb > 0 ? 2 : 1;
    const int n = (causal ? qb + 1 : nb) - lead;
    int P = 1;
    while (P < n) P <<= 1;
    for (int i = threadIdx.x; i < P; i += blockDim.x) {
        unsigned long long key = ~0ull;
        if (i < n) {
            const int kb = i + 1 + ((qb > 0 && i + 1 >= qb) ? 1 : 0);
            float s = srow[kb];
            if (!isfinite(s)) {
                flag_status(kStNonFinite);
                s = -INFINITY;
            }
            key = (static_cast<unsigned long long>(score_desc_key(s)) << 32) | static_cast<uint32_t>(kb);
        }
        keys[i] = key;
    }
    __syncthreads();
    for (int k = 2; k <= P; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = threadIdx.x; i < P; i += blockDim.x) {
                const int ixj = i ^ j;
                if (ixj > i) {
                    const unsigned long long a = keys[i], c = keys[ixj];
                    const bool up = (i & k) == 0;
                    if ((a > c) == up) {
                        keys[i] = c;
                        keys[ixj] = a;
                    }
                }
            }
            __syncthreads();
        }
    }
    if (threadIdx.x == 0) {
        out[0] = 0;
        if (qb > 0) out[1] = qb;
    }
    for (int i = threadIdx.x; i < n; i += blockDim.x) out[lead + i] = static_cast<int32_t>(keys[i] & 0xFFFFFFFFu);
}

// ----------------------------------------------------------------- budget
struct BudgetParams {
    int B, H, G, nb;
    int mode;            // 0 dynamic, 1 fixed fraction, 2 all
    int causal;          // 0: every row holds all nb blocks
    float gamma;
    int frac_permille;
    const int32_t *rank;
    const float *mass;   // [B][H][nb]
    int32_t *cnt;        // [B][H][nb]
    int32_t *budget;     // [B][H]
};

__device__ __forceinline__ int forced_blocks(int qb) { return qb == 0 ? 1 : 2; }

// One CTA of 1024 threads per (b, h); nb <= 4096 -> at most 4 list entries per thread.
__global__ void __launch_bounds__(1024) budget_kernel(BudgetParams p) {
    __shared__ long long warp_sums[32];
    __shared__ int kmin;
    const int bh = blockIdx.x;
    const int b = bh / p.H, h = bh % p.H;
    const int nb = p.nb;
    int k = nb;
    if (p.mode == 0) {
        const int g = static_cast<int>(static_cast<long long>(h) * p.G / p.H);
        const long long T = p.causal ? static_cast<long long>(nb) * (nb + 1) / 2 : static_cast<long long>(nb) * nb;
        const int32_t *last = p.rank + (static_cast<long long>(b) * p.G + g) * T +
                              (p.causal ? static_cast<long long>(nb - 1) * nb / 2 : static_cast<long long>(nb - 1) * nb);
        const float *m = p.mass + static_cast<long long>(bh) * nb;
        const long long gfx = __double2ll_rn(static_cast<double>(p.gamma) * 1099511627776.0);
        const int F = forced_blocks(nb - 1);
        const int per = (nb + blockDim.x - 1) / blockDim.x;
        const int t0 = threadIdx.x * per;
        long long v[4];
        long long local = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            v[j] = 0;
            const int t = t0 + j;
            if (j < per && t < nb) {
                int kb = last[t];
                if (kb < 0 || kb >= nb) {
                    flag_status(kStBounds);
                    kb = 0;
                }
                const float mk = m[kb];
                if (!isfinite(mk)) flag_status(kStNonFinite);
                v[j] = __float2ll_rn(mk * 1099511627776.0f);  // exact scaling by 2^40
                local += v[j];
            }
        }
        // block-wide exclusive scan of the per-thread sums
        const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
        long long incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) warp_sums[warp] = incl;
        if (threadIdx.x == 0) kmin = nb;
        __syncthreads();
        if (warp == 0) {
            long long ws = (lane < static_cast<int>(blockDim.x >> 5)) ? warp_sums[lane] : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const long long y = __shfl_up_sync(0xffffffffu, ws, o);
                if (lane >= o) ws += y;
            }
            warp_sums[lane] = ws;  // inclusive over warps
        }
        __syncthreads();
        long long run = (incl - local) + (warp > 0 ? warp_sums[warp - 1] : 0);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int t = t0 + j;
            if (j < per && t < nb) {
                run += v[j];
                if (t + 1 >= F && run >= gfx) {
                    atomicMin(&kmin, t + 1);
                    break;
                }
            }
        }
        __syncthreads();
        k = kmin;
    }
    int32_t *c = p.cnt + static_cast<long long>(bh) * nb;
    for (int qb = threadIdx.x; qb < nb; qb += blockDim.x) {
        // a causal row holds qb+1 blocks and takes its share of the last row's
        // budget; a non-causal row holds nb blocks and takes the budget itself
        const long long len = p.causal ? qb + 1 : nb;
        long long want;
        if (p.mode == 0)
            want = p.causal ? (static_cast<long long>(k) * (qb + 1) + nb - 1) / nb : k;
        else if (p.mode == 1)
            want = (static_cast<long long>(p.frac_permille) * len + 999) / 1000;
        else
            want = len;
        const long long lo = forced_blocks(qb), hi = len;
        const int val = static_cast<int>(want < lo ? lo : (want > hi ? hi : want));
        c[qb] = val;
        if (qb == nb - 1) p.budget[bh] = val;
    }
}

}  // namespace pa
