// tile_gemm.cuh -- 128x128 QK^T tiles on the tcgen05 tensor core, reduced in
// the epilogue so that no token-level score reaches memory.
//
//   MODE_SCORES  (ProxyAttn blog, "4. ProxyAttn method", Step 1 "Score
//                Estimation": the QK product of the proxy heads fused with
//                block-level max pooling).  For every causal tile (qb, kb<=qb)
//                of every proxy group: score = max over the tile's valid
//                entries of (q_p . k_p)/sqrt(d).  With a query-row stride r
//                (the sequence-level skip of "5. Experiments", read as scoring
//                every r-th query row) the A operand holds only the scored
//                rows, so one 128-row A tile spans r query blocks of 128/r
//                scored rows each and the tensor work drops by r.
//   MODE_MASS    (Step 2, budget from the last query block).  For every head,
//                the last query block against every key block: per row, the
//                max m and sum l of exp2 of the log2-scaled logits over the
//                tile (the inputs of an exact softmax combine).
//
// Persistent, warp-specialised CTA (one per SM, 320 threads):
//   warp 0     TMA producer: the unit's A tile (double-buffered) and a ring of
//              B stages of two 128-row key tiles, 128-byte swizzle.
//   warp 1     allocates 512 TMEM columns (two fp32 128x256 accumulators) and
//              issues tcgen05.mma (M=128, N=256, K=16: two key tiles per
//              instruction, so each wait of the issuing thread covers twice
//              the tensor work) from one thread.
//   warps 2-9  epilogue: warps 2-5 take the first key tile of each pair, warps
//              6-9 the second; each thread owns one accumulator row (TMEM
//              lane) of its tile, reads it with tcgen05.ld and reduces it.
// A unit is a run of up to `chunk` consecutive tiles sharing one A tile.
#pragma once
#include "sm100.cuh"

namespace pa {

enum { MODE_SCORES = 0, MODE_MASS = 1 };

constexpr int kTileThreads = 320;  // producer, MMA issuer, eight epilogue warps

struct TileParams {
    int B, nb, NH;         // NH: proxy groups (scores) or q heads (mass)
    int H, Hkv;            // mass: q head -> KV head
    int chunk;             // tiles per unit (a multiple of stride)
    int stride;            // scores: query-row stride r in {1,2,4,8}; mass: 1
    int causal;            // 1: keys j <= i only (triangular rows); 0: every key (square rows)
    long long units_per_bh;
    long long num_units;
    float scale;           // scores: 1/sqrt(d); mass: scale*log2(e)
    float *scores;         // [B][G][T]
    float2 *partial;       // [B][H][nb][128] (m, l)
    uint64_t timeout_ns;
};

struct Unit {
    int b, bh_head, qb, kb0, kb1;  // tiles kb0 .. kb1-1; scores: qb is the A tile (query blocks qb*r ..)
};

// Scores: A tile m covers query blocks m*r .. m*r+r-1 and so key tiles
// 0 .. min(r(m+1), nb)-1, split into units of C tiles: ceil((m+1)/Cr) units
// with Cr = C/r.  Within one (b, g) the A tiles m = Cr*a + t (t < Cr) own a+1
// units each, so the units before A tile Cr*a number Cr*a(a+1)/2.
__device__ __forceinline__ Unit decode_unit(const TileParams &p, long long u, int mode) {
    Unit r;
    const long long bh = u / p.units_per_bh;
    long long w = u - bh * p.units_per_bh;
    r.b = static_cast<int>(bh / p.NH);
    r.bh_head = static_cast<int>(bh % p.NH);
    const int C = p.chunk;
    if (mode == MODE_SCORES && !p.causal) {
        // non-causal: every A tile owns ceil(nb / C) units over all key tiles
        const long long upr = (p.nb + C - 1) / C;
        r.qb = static_cast<int>(w / upr);
        r.kb0 = static_cast<int>(w % upr) * C;
        r.kb1 = min(r.kb0 + C, p.nb);
    } else if (mode == MODE_SCORES) {
        const int Cr = C / p.stride;
        long long a = static_cast<long long>((sqrt(1.0 + 8.0 * static_cast<double>(w) / Cr) - 1.0) * 0.5);
        while (a > 0 && static_cast<long long>(Cr) * a * (a + 1) / 2 > w) --a;
        while (static_cast<long long>(Cr) * (a + 1) * (a + 2) / 2 <= w) ++a;
        const long long rem = w - static_cast<long long>(Cr) * a * (a + 1) / 2;
        const int t = static_cast<int>(rem / (a + 1));
        const int c = static_cast<int>(rem % (a + 1));
        r.qb = static_cast<int>(Cr * a + t);
        r.kb0 = c * C;
        r.kb1 = min(r.kb0 + C, min(p.stride * (r.qb + 1), p.nb));
    } else {
        r.qb = p.nb - 1;
        r.kb0 = static_cast<int>(w) * C;
        r.kb1 = min(r.kb0 + C, p.nb);
    }
    return r;
}

// Order-preserving float <-> uint32 map (for an integer atomicMax on scores).
__device__ __forceinline__ uint32_t f2ord(float f) {
    const uint32_t u = __float_as_uint(f + 0.0f);  // -0 -> +0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float ord2f(uint32_t o) {
    return __uint_as_float((o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o);
}

// Shared memory: A (the unit's 128-row Q tile) double-buffered, then a ring
// of B stages that each hold two consecutive 128-row K tiles as one 256-row
// K-major operand (per 64-column chunk: 256 rows x 128 B, 128-byte swizzle).
template <int D>
struct TileSmem {
    static constexpr int TILE_BYTES = 128 * D * 2;
    static constexpr int PAIR_BYTES = 2 * TILE_BYTES;
    static constexpr int STAGES = (D == 128) ? 2 : 4;
    static constexpr int BYTES = 2 * TILE_BYTES + STAGES * PAIR_BYTES + 1024 /*align*/ + 512 /*barriers*/;
};

// Tiles of a unit are processed in pairs (kb, kb+1) with one N=256 MMA per K
// step; a unit with an odd tile count ends with a single N=128 tile.
__device__ __forceinline__ int pairs_of(const Unit &un) { return (un.kb1 - un.kb0 + 1) >> 1; }

template <int D, int MODE>
__global__ void __launch_bounds__(kTileThreads, 1)
    tile_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     TileParams p) {
    using S = TileSmem<D>;
    constexpr int TB = S::TILE_BYTES;
    constexpr int PB = S::PAIR_BYTES;
    constexpr int NST = S::STAGES;
    constexpr int KSTEPS = D / 16;
    constexpr uint32_t IDESC256 = idesc_bf16_f32(128, 256, false, false);
    constexpr uint32_t IDESC128 = idesc_bf16_f32(128, 128, false, false);

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;                       // [2][TB]
    uint8_t *sB = smem + 2 * TB;              // [NST][PB]
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + 2 * TB + NST * PB);
    uint64_t *a_full = bars;                  // 2
    uint64_t *a_empty = bars + 2;             // 2
    uint64_t *acc_full = bars + 4;            // 2
    uint64_t *acc_empty = bars + 6;           // 2
    uint64_t *drain = bars + 8;               // 1
    uint64_t *b_full = bars + 9;              // NST
    uint64_t *b_empty = bars + 9 + NST;       // NST
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 9 + 2 * NST);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    uint32_t *red_max = tmem_slot + 2;        // [16] per-(tile, query block) cross-warp max (ring)
    uint32_t *red_cnt = tmem_slot + 18;       // [16]

    const uint32_t warp = warp_id(), lane = lane_id();
    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&a_full[i], 1);
            mbar_init(&a_empty[i], 1);
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], 256);
        }
        for (int i = 0; i < NST; ++i) {
            mbar_init(&b_full[i], 1);
            mbar_init(&b_empty[i], 1);
        }
        for (int i = 0; i < 16; ++i) red_max[i] = red_cnt[i] = 0;
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);  // two 128x256 fp32 accumulators
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const WaitCtl wc{abort_flag, p.timeout_ns};

    if (warp == 0) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            long long pair = 0;
            int local = 0;
            bool ok = true;
            for (long long u = blockIdx.x; u < p.num_units && ok && !*abort_flag; u += gridDim.x) {
                const Unit un = decode_unit(p, u, MODE);
                const int a = local & 1;
                if (local >= 2 && !mbar_wait(&a_empty[a], ((local >> 1) - 1) & 1, wc)) break;
                ++local;
                mbar_arrive_expect_tx(&a_full[a], TB);
#pragma unroll
                for (int cc = 0; cc < D / 64; ++cc) {
                    if (MODE == MODE_SCORES)
                        tma_load_4d(sA + a * TB + cc * 16384, &tmA, &a_full[a], cc * 64, un.qb * 128, un.bh_head, un.b);
                    else
                        tma_load_4d(sA + a * TB + cc * 16384, &tmA, &a_full[a], cc * 64, un.bh_head, un.qb * 128, un.b);
                }
                const int kvh = (MODE == MODE_MASS)
                                    ? static_cast<int>(static_cast<long long>(un.bh_head) * p.Hkv / p.H) : 0;
                for (int kb = un.kb0; kb < un.kb1; kb += 2, ++pair) {
                    const int s = static_cast<int>(pair % NST);
                    const int nt = min(2, un.kb1 - kb);
                    if (pair >= NST && !mbar_wait(&b_empty[s], ((pair / NST) - 1) & 1, wc)) { ok = false; break; }
                    mbar_arrive_expect_tx(&b_full[s], nt * TB);
                    for (int j = 0; j < nt; ++j) {
#pragma unroll
                        for (int cc = 0; cc < D / 64; ++cc) {
                            // chunk cc of the 256-row operand: rows 128 j .. 128 j + 127
                            uint8_t *dst = sB + s * PB + cc * (2 * 16384) + j * 16384;
                            if (MODE == MODE_SCORES)
                                tma_load_4d(dst, &tmB, &b_full[s], cc * 64, (kb + j) * 128, un.bh_head, un.b);
                            else
                                tma_load_4d(dst, &tmB, &b_full[s], cc * 64, kvh, (kb + j) * 128, un.b);
                        }
                    }
                }
            }
            // Let in-flight copies land before the CTA can exit.
            for (long long t = (pair > NST ? pair - NST : 0); t < pair; ++t)
                mbar_wait_drain(&b_full[t % NST], (t / NST) & 1, p.timeout_ns);
            for (int l = (local > 2 ? local - 2 : 0); l < local; ++l)
                mbar_wait_drain(&a_full[l & 1], (l >> 1) & 1, p.timeout_ns);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint64_t da0 = sdesc_sw128(smem_u32(sA), 16, 1024);
            const uint64_t db0 = sdesc_sw128(smem_u32(sB), 16, 1024);
            long long pair = 0;
            int local = 0;
            bool ok = true;
            for (long long u = blockIdx.x; u < p.num_units && ok; u += gridDim.x, ++local) {
                const Unit un = decode_unit(p, u, MODE);
                const int a = local & 1;
                if (!mbar_wait(&a_full[a], (local >> 1) & 1, wc)) break;
                const uint64_t da = da0 + static_cast<uint64_t>((a * TB) >> 4);
                for (int kb = un.kb0; kb < un.kb1; kb += 2, ++pair) {
                    const int s = static_cast<int>(pair % NST);
                    const int acc = static_cast<int>(pair & 1);
                    if (!mbar_wait(&b_full[s], (pair / NST) & 1, wc)) { ok = false; break; }
                    if (pair >= 2 && !mbar_wait(&acc_empty[acc], ((pair >> 1) - 1) & 1, wc)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t db = db0 + static_cast<uint64_t>((s * PB) >> 4);
                    const uint32_t idesc = (un.kb1 - kb >= 2) ? IDESC256 : IDESC128;
#pragma unroll
                    for (int kk = 0; kk < KSTEPS; ++kk) {
                        const uint64_t oa = static_cast<uint64_t>(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
                        const uint64_t ob = static_cast<uint64_t>(((kk >> 2) * 32768 + (kk & 3) * 32) >> 4);
                        umma_ss(tmem + acc * 256, da + oa, db + ob, idesc, kk > 0 ? 1u : 0u);
                    }
                    umma_commit(&b_empty[s]);
                    umma_commit(&acc_full[acc]);
                }
                if (ok) umma_commit(&a_empty[a]);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------ epilogue
        // Warps 2..9: warp w reduces TMEM lanes 32 (w & 3) .. +31 of tile (w - 2) / 4
        // of each key-tile pair, so two warps per SMSP share a pair.
        const int q4 = static_cast<int>(warp & 3);
        const int jt = static_cast<int>(warp - 2) >> 2;
        const int row = q4 * 32 + static_cast<int>(lane);
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
        // A row -> (query block within the A tile, token offset inside that block)
        const int rows_per_qb = 128 / p.stride;
        const int qsub = row / rows_per_qb;
        const int toff = (row % rows_per_qb) * p.stride + p.stride - 1;
        const int span = min(rows_per_qb, 32);  // lanes of a warp that share a query block
        const int wpq = rows_per_qb / 32;       // warps that share a query block (0: part of one warp)
        long long pair = 0;
        bool ok = true;
        for (long long u = blockIdx.x; u < p.num_units && ok; u += gridDim.x) {
            const Unit un = decode_unit(p, u, MODE);
            const int qbw = (MODE == MODE_SCORES) ? un.qb * p.stride + qsub : un.qb;  // this row's query block
            for (int kb0 = un.kb0; kb0 < un.kb1; kb0 += 2, ++pair) {
                const int acc = static_cast<int>(pair & 1);
                const int nt = min(2, un.kb1 - kb0);
                if (!warp_wait(&acc_full[acc], (pair >> 1) & 1, wc)) { ok = false; break; }
                tc_fence_after();
                if (jt >= nt) {  // a unit's odd last tile: nothing for this warp
                    tc_fence_before();
                    mbar_arrive(&acc_empty[acc]);
                    continue;
                }
                const int kb = kb0 + jt;
                const long long tj = pair * 2 + jt;  // a distinct index per tile (reduction ring slot)
                const bool diag = p.causal && (kb == qbw);
                uint32_t r[128];
                tmem_ld128(lane_base + acc * 256 + jt * 128, r);
                // this tile is in registers: hand its TMEM back to the MMA warp
                tc_fence_before();
                mbar_arrive(&acc_empty[acc]);
                if (diag) {
#pragma unroll
                    for (int c = 0; c < 128; ++c)
                        if (c > toff) r[c] = 0xFF800000u;  // -inf above the diagonal (j > i)
                }
                float m8[16];
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const uint32_t *v = r + 8 * c;
                    m8[c] = fmax3(fmax3(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2])),
                                  fmax3(__uint_as_float(v[3]), __uint_as_float(v[4]), __uint_as_float(v[5])),
                                  fmaxf(__uint_as_float(v[6]), __uint_as_float(v[7])));
                }
                const float mx = fmax3(fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]),
                                             fmax3(m8[6], m8[7], m8[8])),
                                       fmax3(m8[9], m8[10], m8[11]), fmax3(m8[12], m8[13], fmaxf(m8[14], m8[15])));
                if (MODE == MODE_SCORES) {
                    float w = mx * p.scale;
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1)
                        if (o < span) w = fmaxf(w, __shfl_xor_sync(0xffffffffu, w, o));
                    // tiles above this query block's diagonal, and A rows past the last
                    // block (zero-filled), give no score
                    const bool valid = (!p.causal || kb <= qbw) && qbw < p.nb;
                    if (valid && (static_cast<int>(lane) & (span - 1)) == 0) {
                        const long long T = p.causal ? static_cast<long long>(p.nb) * (p.nb + 1) / 2
                                                     : static_cast<long long>(p.nb) * p.nb;
                        const long long idx = (static_cast<long long>(un.b) * p.NH + un.bh_head) * T +
                                              (p.causal ? static_cast<long long>(qbw) * (qbw + 1) / 2
                                                        : static_cast<long long>(qbw) * p.nb) + kb;
                        if (wpq <= 1) {
                            p.scores[idx] = w;
                        } else {
                            const int slot = static_cast<int>(tj & 7) * 2 + (qsub & 1);
                            atomicMax(&red_max[slot], f2ord(w));
                            __threadfence_block();
                            if (atomicAdd(&red_cnt[slot], 1u) == static_cast<uint32_t>(wpq - 1)) {
                                const uint32_t best = atomicExch(&red_max[slot], 0u);
                                atomicExch(&red_cnt[slot], 0u);
                                p.scores[idx] = ord2f(best);
                            }
                        }
                    }
                } else {
                    // log2-domain row max and sum of exp2 over the valid entries
                    const float m = mx * p.scale;
                    float acc8[8];
#pragma unroll
                    for (int c = 0; c < 8; ++c) acc8[c] = 0.0f;
#pragma unroll
                    for (int c = 0; c < 128; ++c) acc8[c & 7] += ex2(fmaf(__uint_as_float(r[c]), p.scale, -m));
                    const float lsum = ((acc8[0] + acc8[1]) + (acc8[2] + acc8[3])) + ((acc8[4] + acc8[5]) + (acc8[6] + acc8[7]));
                    const long long idx = ((static_cast<long long>(un.b) * p.H + un.bh_head) * p.nb + kb) * 128 + row;
                    p.partial[idx] = make_float2(m, lsum);
                }
            }
        }
    }

    // ---------------------------------------------------------- teardown
    if (warp == 1) {
        // every MMA (and commit) this CTA issued has completed before TMEM is released
        if (lane == 0) {
            umma_commit(drain);
            mbar_wait_drain(drain, 0, p.timeout_ns);
        }
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace pa
