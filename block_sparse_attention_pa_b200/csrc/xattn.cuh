// xattn.cuh -- XAttention's antidiagonal block estimate and its threshold
// selection (XAttention blog, 2.1 "importance prediction" and 2.2 "threshold
// block selection"), as a second estimator that feeds the same block-sparse
// attention kernel.
//
// For head h and stride S, strided query row R stands for tokens R*S ..
// R*S+S-1 and strided key column c for tokens c*S .. c*S+S-1; the antidiagonal
// sum of that S x S sub-block of the score map is
//     z[R][c] = sum_{t<S} q[R*S + S-1-t] . k[c*S + t],
// a plain product of a reshaped Q (rows of S*d features, token offsets taken
// from S-1 down to 0) and a reshaped K (offsets 0 up to S-1).  Each strided row
// is softmax-normalised (scale 1/(sqrt(d) S), sub-blocks on or below the
// diagonal); the estimate of KV block kb for query block qb is the mean over
// qb's 128/S strided rows of the probability in kb's 128/S columns.
//
//   xattn_gemm_kernel   tcgen05 GEMM, M = 128 strided rows, N = 256 strided
//                       columns, K = S*d streamed in 64-wide chunks by TMA
//                       through 5-D tensor maps that view the token axis as
//                       (token / S, token mod S).  The epilogue reduces each
//                       128-column half to per-row softmax partials: the max
//                       m (log2 units) and, per KV block, sum 2^(x - m).
//   xattn_select_kernel one CTA per (b, h, qb): combines the partials of the
//                       query block's strided rows into the block estimates,
//                       sorts them (estimate desc, index asc) and finds the
//                       shortest prefix whose estimates reach tau in 2^-40
//                       fixed point (find_blocks).
#pragma once

#include "sm100.cuh"

namespace pa {

struct XattnParams {
    int B, H, Hkv, nb;
    int rows;               // strided rows (= strided columns) per head: N / S
    int nchunk;             // 128-column chunks per strided row: ceil(rows / 128)
    long long units_per_bh; // output tiles per (b, h)
    long long num_units;
    float c2;               // log2(e) / (sqrt(d) * S)
    int causal;             // 0: every strided column of every row (square rows of estimates)
    float *part_s;          // [B][H][rows][nb]   sum of 2^(x - m) over the block's valid columns
    float *part_m;          // [B][H][nchunk][rows]  row max of the 128-column chunk (log2 units)
    uint64_t timeout_ns;
};

// Output tiles of one (b, h): strided-row tile mt covers rows 128 mt ..
// 128 mt + 127 and needs column tiles 0 .. floor(mt / 2) (256 columns each,
// on or below the diagonal).  Row tiles 2a and 2a+1 own a+1 column tiles
// each, so the tiles before row tile 2a number a(a+1).
struct XUnit {
    int b, h, mt, nt;
};

__device__ __forceinline__ XUnit xattn_decode(const XattnParams &p, long long u) {
    XUnit x;
    const long long bh = u / p.units_per_bh;
    const long long w = u - bh * p.units_per_bh;
    x.b = static_cast<int>(bh / p.H);
    x.h = static_cast<int>(bh % p.H);
    if (!p.causal) {  // every row tile needs every column tile
        const long long ntn = (p.rows + 255) / 256;
        x.mt = static_cast<int>(w / ntn);
        x.nt = static_cast<int>(w % ntn);
        return x;
    }
    long long a = static_cast<long long>((sqrt(1.0 + 4.0 * static_cast<double>(w)) - 1.0) * 0.5);
    while (a > 0 && a * (a + 1) > w) --a;
    while ((a + 1) * (a + 2) <= w) ++a;
    const long long rem = w - a * (a + 1);
    x.mt = static_cast<int>(2 * a + (rem >= a + 1 ? 1 : 0));
    x.nt = static_cast<int>(rem >= a + 1 ? rem - (a + 1) : rem);
    return x;
}

template <int D, int S>
struct XattnSmem {
    static constexpr int A_BYTES = 128 * 64 * 2;   // one 64-wide K chunk of 128 rows
    static constexpr int B_BYTES = 256 * 64 * 2;   // one 64-wide K chunk of 256 columns
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int STAGES = 4;
    static constexpr int KCHUNKS = S * D / 64;
    static constexpr int BYTES = STAGES * STAGE + 1024 /*align*/ + 256 /*barriers*/;
};

template <int D, int S>
__global__ void __launch_bounds__(192, 1)
    xattn_gemm_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const XattnParams p) {
    using SM = XattnSmem<D, S>;
    constexpr int NST = SM::STAGES;
    constexpr int KC = SM::KCHUNKS;
    constexpr int CPT = D / 64;        // 64-wide chunks per token
    constexpr int CPB = 128 / S;       // strided columns (and rows) per 128-token block
    constexpr uint32_t IDESC = idesc_bf16_f32(128, 256, false, false);

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + NST * SM::STAGE);
    uint64_t *full = bars;                 // NST
    uint64_t *empty = bars + NST;          // NST
    uint64_t *acc_full = bars + 2 * NST;   // 2
    uint64_t *acc_empty = bars + 2 * NST + 2;  // 2
    uint64_t *drain = bars + 2 * NST + 4;  // 1
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * NST + 5);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const uint32_t warp = warp_id(), lane = lane_id();
    if (threadIdx.x == 0) {
        for (int i = 0; i < NST; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], 128);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
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
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            long long it = 0;
            bool ok = true;
            for (long long u = blockIdx.x; u < p.num_units && ok && !*abort_flag; u += gridDim.x) {
                const XUnit x = xattn_decode(p, u);
                const int kvh = static_cast<int>(static_cast<long long>(x.h) * p.Hkv / p.H);
                for (int kc = 0; kc < KC; ++kc, ++it) {
                    const int s = static_cast<int>(it % NST);
                    if (it >= NST && !mbar_wait(&empty[s], ((it / NST) - 1) & 1, wc)) { ok = false; break; }
                    const int t = kc / CPT;             // token offset inside the S-token group
                    const int c0 = (kc % CPT) * 64;     // feature offset inside the token
                    uint8_t *st = smem + s * SM::STAGE;
                    mbar_arrive_expect_tx(&full[s], SM::STAGE);
                    // A: rows R = 128 mt .., token R*S + S-1-t; B: columns c = 256 nt .., token c*S + t
                    tma_load_5d(st, &tmQ, &full[s], c0, x.h, S - 1 - t, x.mt * 128, x.b);
                    tma_load_5d(st + SM::A_BYTES, &tmK, &full[s], c0, kvh, t, x.nt * 256, x.b);
                }
            }
            for (long long t2 = (it > NST ? it - NST : 0); t2 < it; ++t2)
                mbar_wait_drain(&full[t2 % NST], (t2 / NST) & 1, p.timeout_ns);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint64_t da0 = sdesc_sw128(smem_u32(smem), 16, 1024);
            const uint64_t db0 = sdesc_sw128(smem_u32(smem + SM::A_BYTES), 16, 1024);
            long long it = 0;
            long long local = 0;
            bool ok = true;
            for (long long u = blockIdx.x; u < p.num_units && ok; u += gridDim.x, ++local) {
                const int acc = static_cast<int>(local & 1);
                if (local >= 2 && !mbar_wait(&acc_empty[acc], ((local >> 1) - 1) & 1, wc)) break;
                tc_fence_after();
                for (int kc = 0; kc < KC; ++kc, ++it) {
                    const int s = static_cast<int>(it % NST);
                    if (!mbar_wait(&full[s], (it / NST) & 1, wc)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t off = static_cast<uint64_t>((s * SM::STAGE) >> 4);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_ss(tmem + acc * 256, da0 + off + static_cast<uint64_t>(kk * 2),
                                db0 + off + static_cast<uint64_t>(kk * 2), IDESC, (kc > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&empty[s]);
                }
                if (ok) umma_commit(&acc_full[acc]);
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------- epilogue
        const int q4 = static_cast<int>(warp & 3);
        const int row = q4 * 32 + static_cast<int>(lane);
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
        long long local = 0;
        for (long long u = blockIdx.x; u < p.num_units; u += gridDim.x, ++local) {
            const XUnit x = xattn_decode(p, u);
            const int acc = static_cast<int>(local & 1);
            if (!warp_wait(&acc_full[acc], (local >> 1) & 1, wc)) break;
            tc_fence_after();
            const int R = x.mt * 128 + row;            // this thread's strided row
            const int qb = R / CPB;                    // its query block
            const long long bh = static_cast<long long>(x.b) * p.H + x.h;
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                uint32_t r[128];
                __syncwarp();  // the TMEM load below is warp-collective
                tmem_ld128(lane_base + acc * 256 + half * 128, r);
                if (half == 1) {
                    tc_fence_before();
                    mbar_arrive(&acc_empty[acc]);  // the accumulator is in registers
                }
                const int C0 = x.nt * 256 + half * 128;  // first strided column of this chunk
                // past the last row or column, or (causal) above the diagonal
                if (R >= p.rows || C0 >= p.rows || (p.causal && C0 > R)) continue;
                // columns C0 + j with j <= lim are valid: on or below the diagonal (causal) and
                // inside the sequence (the columns past it are TMA zero fill)
                const int lim = min(p.causal ? R - C0 : 127, p.rows - 1 - C0);
#pragma unroll
                for (int j = 0; j < 128; ++j)
                    if (j > lim) r[j] = 0xFF800000u;     // -inf
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
                const float m2 = mx * p.c2;
                const int ch = C0 / 128;
                p.part_m[(bh * p.nchunk + ch) * p.rows + R] = m2;
                // the chunk's S block sums of this row are adjacent in part_s
                float sums[S];
#pragma unroll
                for (int kbl = 0; kbl < S; ++kbl) {
                    float acc4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
                    for (int j = 0; j < CPB; ++j)
                        acc4[j & 3] += ex2(fmaf(__uint_as_float(r[kbl * CPB + j]), p.c2, -m2));
                    sums[kbl] = (acc4[0] + acc4[1]) + (acc4[2] + acc4[3]);
                }
                float *dst = p.part_s + (bh * p.rows + R) * p.nb + ch * S;
                const int nvalid = min(S, (p.causal ? qb + 1 : p.nb) - ch * S);
                if (nvalid == S && (p.nb & 3) == 0) {  // 16-byte aligned whole chunk
#pragma unroll
                    for (int v = 0; v < S / 4; ++v)
                        reinterpret_cast<float4 *>(dst)[v] =
                            make_float4(sums[4 * v], sums[4 * v + 1], sums[4 * v + 2], sums[4 * v + 3]);
                } else {
#pragma unroll
                    for (int kbl = 0; kbl < S; ++kbl)
                        if (kbl < nvalid) dst[kbl] = sums[kbl];
                }
            }
        }
    }

    // ---------------------------------------------------------- teardown
    if (warp == 1) {
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

// ------------------------------------------------------------ selection
struct XselParams {
    int B, H, nb, rows, nchunk;  // the stride S is the kernel's template argument
    int causal;
    float tau;
    const float *part_s;  // as XattnParams
    const float *part_m;
    float *mass;          // [B][H][T] block estimates, or nullptr
    int32_t *rank;        // [B][H][T] blocks by (estimate desc, index asc)
    int32_t *cnt;         // [B][H][nb] shortest prefix reaching tau
};

// Order-preserving map of a float to a key that sorts larger values first.
__device__ __forceinline__ uint32_t xsel_desc_key(float f) {
    const uint32_t u = __float_as_uint(f + 0.0f);
    const uint32_t ord = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return ~ord;
}
__device__ __forceinline__ float xsel_key_value(uint32_t key) {
    const uint32_t ord = ~key;
    return __uint_as_float((ord & 0x80000000u) ? (ord & 0x7FFFFFFFu) : ~ord);
}

// Ascending bitonic sort of the 256*E keys in shared memory by a CTA of 256
// threads.  Thread t holds keys t*E .. t*E+E-1 in registers: a compare-exchange
// stage whose partner index differs by j < E stays in the thread, one with
// E <= j < 32E is a warp shuffle, and only the stages with j >= 32E go through
// shared memory (6 of the 55 stages for 1024 keys).  The result is the unique
// ascending order of the keys (they are distinct), back in shared memory.
// the in-thread stage with partner distance J < E (J a compile-time constant,
// so the key array stays in registers)
template <int E, int J>
__device__ __forceinline__ void bitonic_stage_in_thread(unsigned long long (&v)[E], int k, int tid) {
#pragma unroll
    for (int e = 0; e < E; ++e) {
        if ((e & J) == 0) {
            const int i = tid * E + e;
            const unsigned long long a = v[e], c = v[e ^ J];
            if ((a > c) == ((i & k) == 0)) {
                v[e] = c;
                v[e ^ J] = a;
            }
        }
    }
}

template <int E>
__device__ __forceinline__ void bitonic_sort_256(unsigned long long *keys) {
    constexpr int PP = 256 * E;
    const int tid = static_cast<int>(threadIdx.x);
    unsigned long long v[E];
#pragma unroll
    for (int e = 0; e < E; ++e) v[e] = keys[tid * E + e];
    for (int k = 2; k <= PP; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            if (j >= 32 * E) {
                __syncthreads();  // every thread has read the previous stage's keys
#pragma unroll
                for (int e = 0; e < E; ++e) keys[tid * E + e] = v[e];
                __syncthreads();
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const int i = tid * E + e, l = i ^ j;
                    const unsigned long long w = keys[l];
                    const bool keep_min = (i < l) == ((i & k) == 0);
                    v[e] = keep_min ? (v[e] < w ? v[e] : w) : (v[e] < w ? w : v[e]);
                }
            } else if (j >= E) {
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const int i = tid * E + e, l = i ^ j;
                    const unsigned long long w = __shfl_xor_sync(0xffffffffu, v[e], j / E);
                    const bool keep_min = (i < l) == ((i & k) == 0);
                    v[e] = keep_min ? (v[e] < w ? v[e] : w) : (v[e] < w ? w : v[e]);
                }
            } else if (j == 4) {
                if constexpr (E > 4) bitonic_stage_in_thread<E, 4>(v, k, tid);
            } else if (j == 2) {
                if constexpr (E > 2) bitonic_stage_in_thread<E, 2>(v, k, tid);
            } else {
                if constexpr (E > 1) bitonic_stage_in_thread<E, 1>(v, k, tid);
            }
        }
    }
    __syncthreads();
#pragma unroll
    for (int e = 0; e < E; ++e) keys[tid * E + e] = v[e];
    __syncthreads();
}

// The sort of 1024 or 2048 keys: a stable LSD radix sort of the upper 32
// bits, the descending-estimate code, four bits per pass, with the lower 32
// bits, the block index, carried along.  Thread t holds entries t*E ..
// t*E+E-1 (the keys start in block-index order).  A pass:
//   1. each thread counts its keys per digit in two packed words (4 bits per
//      digit, E <= 8 keys) and writes the 16 counts to cnt[digit][thread];
//   2. one exclusive scan over cnt in (digit, thread) order gives each
//      thread the first output position of its keys of each digit;
//   3. each thread scatters its keys, in its own order, to those positions.
// Positions follow (digit, thread, key) order, so the pass is stable, and a
// stable LSD sort leaves equal estimates in index order: the result is the
// ascending order of the whole 64-bit keys, as the bitonic network produces.
// A pass whose digit is the same for every key would not move any and is
// skipped.  Shorter rows keep the bitonic network, which is faster there.
constexpr int kXselRadixBits = 4;
constexpr int kXselDigits = 1 << kXselRadixBits;

// Shared memory the selection kernel needs beyond its P keys for the sort:
// the per-(digit, thread) counts and the eight warps' scan totals.
__host__ __device__ constexpr size_t xsel_sort_temp_bytes(int P) {
    return (P == 1024 || P == 2048) ? (kXselDigits * 256 + 8) * sizeof(uint32_t) : 0;
}

// count field of digit d in the packed pair (lo: digits 0-7, hi: 8-15)
__device__ __forceinline__ uint32_t xsel_field(uint32_t lo, uint32_t hi, uint32_t d) {
    return ((d < 8 ? lo : hi) >> (4 * (d & 7))) & 15u;
}

template <int E>
__device__ __forceinline__ void radix_sort_keys(unsigned long long *keys, void *temp) {
    static_assert(E <= 8, "4-bit packed counts hold at most 15 keys per digit");
    constexpr int P = 256 * E;
    uint32_t *cnt = reinterpret_cast<uint32_t *>(temp);  // [kXselDigits][256]
    uint32_t *wsum = cnt + kXselDigits * 256;           // [8]
    const int tid = static_cast<int>(threadIdx.x);
    const int lane = tid & 31, warp = tid >> 5;
    uint32_t k[E], v[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const unsigned long long x = keys[tid * E + e];
        k[e] = static_cast<uint32_t>(x >> 32);
        v[e] = static_cast<uint32_t>(x);
    }
    for (int shift = 0; shift < 32; shift += kXselRadixBits) {
        // a pass that would not move any key is skipped (the whole CTA agrees)
        const uint32_t ref = static_cast<uint32_t>(keys[0] >> (32 + shift)) & (kXselDigits - 1);
        bool same = true;
#pragma unroll
        for (int e = 0; e < E; ++e) same = same && ((k[e] >> shift) & (kXselDigits - 1)) == ref;
        if (__syncthreads_and(same)) continue;
        // 1. this thread's counts per digit
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const uint32_t d = (k[e] >> shift) & (kXselDigits - 1);
            if (d < 8) lo += 1u << (4 * d); else hi += 1u << (4 * (d - 8));
        }
#pragma unroll
        for (int d = 0; d < kXselDigits; ++d) cnt[d * 256 + tid] = xsel_field(lo, hi, d);
        __syncthreads();
        // 2. exclusive scan of the 4096 counts in (digit, thread) order: thread
        // t scans the 16 consecutive counts at 16t, the warps' totals are
        // scanned through shared memory
        uint32_t c[kXselDigits];
        uint32_t run = 0;
#pragma unroll
        for (int x = 0; x < kXselDigits; ++x) {
            c[x] = run;
            run += cnt[tid * kXselDigits + x];
        }
        uint32_t incl = run;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) wsum[warp] = incl;
        __syncthreads();
        uint32_t base = incl - run;
        for (int w = 0; w < warp; ++w) base += wsum[w];
#pragma unroll
        for (int x = 0; x < kXselDigits; ++x) cnt[tid * kXselDigits + x] = base + c[x];
        __syncthreads();
        // 3. scatter: the first free position of each digit of this thread
        uint32_t seen_lo = 0, seen_hi = 0;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const uint32_t d = (k[e] >> shift) & (kXselDigits - 1);
            const uint32_t pos = cnt[d * 256 + tid] + xsel_field(seen_lo, seen_hi, d);
            if (d < 8) seen_lo += 1u << (4 * d); else seen_hi += 1u << (4 * (d - 8));
            keys[pos] = (static_cast<unsigned long long>(k[e]) << 32) | v[e];
        }
        __syncthreads();
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const unsigned long long x = keys[tid * E + e];
            k[e] = static_cast<uint32_t>(x >> 32);
            v[e] = static_cast<uint32_t>(x);
        }
        __syncthreads();  // every thread has read its keys before the next pass writes
    }
    (void)P;
}

// One CTA of 256 threads per (b, h, qb), long rows first; dynamic shared
// memory holds max(P, 256) 64-bit sort keys, P >= qb+1 a power of two,
// followed (P = 1024, 2048) by the radix sort's temporary storage.
template <int S>
__global__ void __launch_bounds__(256) xattn_select_kernel(XselParams p) {
    extern __shared__ unsigned long long keys[];
    __shared__ float red[256];
    __shared__ float rowM[32], rowI[32];
    __shared__ long long warp_sums[8];
    __shared__ int kmin;
    const long long bh = blockIdx.x / p.nb;
    const int qb = p.nb - 1 - static_cast<int>(blockIdx.x % p.nb);
    const int tid = threadIdx.x;
    constexpr int CPB = 128 / S;        // strided rows of the query block (<= 32); compile-time, so
                                        // the loops over them unroll and their loads overlap
    const int R0 = qb * CPB;
    const int cq = p.causal ? R0 / 128 : p.nchunk - 1;  // the rows' last 128-column chunk
    const int n = p.causal ? qb + 1 : p.nb;              // blocks of the row
    const long long T = p.causal ? static_cast<long long>(p.nb) * (p.nb + 1) / 2 : static_cast<long long>(p.nb) * p.nb;
    const long long row_at = p.causal ? static_cast<long long>(qb) * (qb + 1) / 2 : static_cast<long long>(qb) * p.nb;
    // part_s rows of this query block: row x's block sums at ps[x * nb + kb] (contiguous in kb)
    const float *ps = p.part_s + (bh * p.rows + R0) * static_cast<long long>(p.nb);
    const float *pm = p.part_m + bh * p.nchunk * static_cast<long long>(p.rows) + R0;
    const long long rs = p.rows;

    // 1. each strided row's max over its chunks (slots threads per row)
    constexpr int slots = 256 / CPB;
    const int r = tid / slots, sl = tid % slots;
    float M = -INFINITY;
#pragma unroll 4
    for (int ch = sl; ch <= cq; ch += slots) M = fmaxf(M, pm[ch * rs + r]);
    red[tid] = M;
    __syncthreads();
    if (tid < CPB) {
        float m = -INFINITY;
        for (int x = 0; x < slots; ++x) m = fmaxf(m, red[tid * slots + x]);
        rowM[tid] = m;
    }
    __syncthreads();
    // 2. each row's softmax denominator over the blocks 0..qb (consecutive
    // threads read consecutive blocks of one row)
    const float Mr = rowM[r];
    const float *psr = ps + static_cast<long long>(r) * p.nb;
    float L = 0.0f;
#pragma unroll 4
    for (int kb = sl; kb < n; kb += slots) L += exp2f(pm[(kb / S) * rs + r] - Mr) * psr[kb];
    red[tid] = L;
    __syncthreads();
    if (tid < CPB) {
        float l = 0.0f;
        for (int x = 0; x < slots; ++x) l += red[tid * slots + x];
        rowI[tid] = 1.0f / l;
    }
    __syncthreads();
    // 3. block estimates -> sort keys (padded with the largest key to at least 256)
    int P = 256;
    while (P < n) P <<= 1;
    for (int kb = tid; kb < P; kb += blockDim.x) {
        unsigned long long key = ~0ull;
        if (kb < n) {
            float e = 0.0f;
            const float *mcol = pm + (kb / S) * rs;
#pragma unroll
            for (int x = 0; x < CPB; ++x)
                e += exp2f(mcol[x] - rowM[x]) * ps[static_cast<long long>(x) * p.nb + kb] * rowI[x];
            e *= 1.0f / static_cast<float>(CPB);
            if (!isfinite(e)) {
                flag_status(kStNonFinite);
                e = 0.0f;
            }
            if (p.mass) p.mass[bh * T + row_at + kb] = e;
            key = (static_cast<unsigned long long>(xsel_desc_key(e)) << 32) | static_cast<uint32_t>(kb);
        }
        keys[kb] = key;
    }
    if (tid == 0) kmin = n;
    __syncthreads();
    if (P == 256) {
        bitonic_sort_256<1>(keys);
    } else if (P == 512) {
        bitonic_sort_256<2>(keys);
    } else if (P == 1024) {
        radix_sort_keys<4>(keys, keys + P);
    } else if (P == 2048) {
        radix_sort_keys<8>(keys, keys + P);
    } else {
        for (int k = 2; k <= P; k <<= 1) {
            for (int j = k >> 1; j > 0; j >>= 1) {
                for (int i = tid; i < P; i += blockDim.x) {
                    const int ixj = i ^ j;
                    if (ixj > i) {
                        const unsigned long long a = keys[i], c = keys[ixj];
                        if ((a > c) == ((i & k) == 0)) {
                            keys[i] = c;
                            keys[ixj] = a;
                        }
                    }
                }
                __syncthreads();
            }
        }
    }
    // 4. ranked list and the shortest prefix reaching tau (2^-40 fixed point)
    int32_t *out = p.rank + bh * T + row_at;
    for (int i = tid; i < n; i += blockDim.x) out[i] = static_cast<int32_t>(keys[i] & 0xFFFFFFFFu);
    const long long tfx = __double2ll_rn(static_cast<double>(p.tau) * 1099511627776.0);
    const int per = (n + 255) / 256;    // <= 16 entries per thread
    const int t0 = tid * per;
    long long local = 0;
    for (int j = 0; j < per; ++j)
        if (t0 + j < n) local += __float2ll_rn(xsel_key_value(static_cast<uint32_t>(keys[t0 + j] >> 32)) * 1099511627776.0f);
    const int lane = tid & 31, warp = tid >> 5;
    long long incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    long long run = incl - local;
    for (int w = 0; w < warp; ++w) run += warp_sums[w];
    for (int j = 0; j < per; ++j) {
        const int t = t0 + j;
        if (t < n) {
            run += __float2ll_rn(xsel_key_value(static_cast<uint32_t>(keys[t] >> 32)) * 1099511627776.0f);
            if (run >= tfx) {
                atomicMin(&kmin, t + 1);
                break;
            }
        }
    }
    __syncthreads();
    if (tid == 0) p.cnt[bh * p.nb + qb] = kmin;
}

}  // namespace pa
