// attn.cuh -- causal block-sparse FlashAttention on tcgen05 (ProxyAttn blog:
// the block-sparse mask "fed to FlashAttention", end of "4. ProxyAttn
// method"; the attention formula of "2. Background").
//
// One CTA computes two (q head, query block) items of one KV head, one per
// slot: two heads at one query block, or one head at two adjacent query
// blocks (the work decode below chooses from the counts).  The item of slot t
// visits the first cnt entries of its row of its proxy group's ranked list;
// a K/V tile is loaded once for both slots whenever either needs it, so the
// pairing aims at two items that share most of their tiles.
//
// Warp roles (384 threads = three warpgroups, one CTA per SM, all 512 TMEM
// columns).  At the start the third warpgroup hands registers to the two
// softmax warpgroups (setmaxnreg: 2 x 128 x 208 + 128 x 88 = 384 x 168):
//   warps 0-3  softmax of slot 0, warps 4-7 softmax of slot 1 (below)
//   warp 8     TMA producer: the two Q tiles (issued before the CTA's setup
//              barrier, so the copy overlaps the setup), then K and V tiles of the
//              listed blocks into rings (128-byte swizzle).  V of tile i and K
//              of tile i+1 share one barrier and one release, since the MMA
//              thread needs both at the same point (PV(i), then QK(i+1)).
//   warp 9     TMEM owner and single-thread tcgen05.mma issuer:
//                S_t = Q_t K^T   (M=128, N=128, K=16 steps; A, B K-major smem)
//                O_t += P_t V    (M=128, N=d,   A = P_t read from TMEM,
//                                 B = V, MN-major smem)
//              in ping-pong order  PV_0(i), QK_0(i+1), PV_1(i), QK_1(i+1), so
//              the tensor core computes one slot's products while the other
//              slot's softmax runs.
//   softmax    one thread per query row (TMEM lane).  S is read from TMEM once; row max,
//              then exp2/row sum/bf16 pack of P, written back over S; online
//              softmax with the running max raised only when it grows by more
//              than 2^8 (then O is rescaled in TMEM, after the tile's P is
//              stored and before it is handed over), final O/l and LSE.
// TMEM columns: S_0 [0,128)  S_1 [128,256)  O_0 [256,384)  O_1 [384,512);
// P_t (bf16 pairs) overwrites the first 64 columns of S_t.
//
// SKIP = true adds BLASST's running-max block skip (BLASST introduction and
// 3.1): a visited block after the first whose row maxima all lie below the
// rows' running maxima (over the blocks visited before, in ascending order)
// by more than -log2(lambda) is dropped -- no exponentials, no P, no PV, and
// no V load: K runs ahead on a ring of its own, and the producer loads V of a
// tile only once a head that visits it has kept it.  The four warps of a head
// take the block-level decision by a bounded vote in shared memory; the
// producer reads it from a tagged slot per head, the MMA warp after the
// head's p_full barrier.
#pragma once
#include "sm100.cuh"

namespace pa {

constexpr int kMaxHeads = 128;

// 12 warps: 0-7 softmax (two warpgroups), 8 producer, 9 MMA, 10-11 idle.
constexpr int kAttnThreads = 384;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kRegsLaunch = 168;   // 65536 / 384, rounded down to a multiple of 8
constexpr int kRegsSoftmax = 208;
constexpr int kRegsAux = 88;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsAux <= kAttnThreads * kRegsLaunch,
              "setmaxnreg split exceeds the registers the CTA is launched with");

struct AttnParams {
    int B, N, H, Hkv, G, nb;
    int units_per_kv;          // max head units (CTAs) of one KV head per (b, qb): the grid stride
    const int32_t *rank;       // [B][G][T]
    const int32_t *cnt;        // [B][H][nb]
    float scale_log2;          // softmax_scale * log2(e)
    __nv_bfloat16 *o;
    int64_t osb, oss, osh;
    float *lse;                // [B][H][N] or nullptr
    int causal;                // 1: keys j <= i, rows at qb(qb+1)/2; 0: every key, rows at qb*nb
    float skip_log2;           // SKIP: log2(lambda) (lambda in (0, 1])
    uint8_t *skipped;          // SKIP: [B][H][T], 1 written for every skipped block, or nullptr
    uint64_t timeout_ns;
    int16_t kv_units[kMaxHeads];  // head units of KV head kv: ceil(its q heads / 2)
};

// Smallest block index >= from whose bit is set in (a | b), or -1; words
// bitmap words are in range.
__device__ __forceinline__ int next_block(const uint32_t *a, const uint32_t *b, int from, int words) {
    int w = from >> 5;
    if (w >= words) return -1;
    uint32_t m = (a[w] | b[w]) & (0xFFFFFFFFu << (from & 31));
    while (m == 0u) {
        if (++w >= words) return -1;
        m = a[w] | b[w];
    }
    return (w << 5) + __ffs(static_cast<int>(m)) - 1;
}

// Block-level vote of the four warps of one head: true when every row of the
// query block votes yes.  Each warp publishes (tile << 1 | its vote) in its
// own slot; lanes 0-3 poll the four slots until all carry this tile's tag.
// The poll is bounded like every other wait: on a timeout (or the CTA's abort
// flag) `ok` is false for the whole warp.
__device__ __forceinline__ bool head_vote_all(volatile uint32_t *slots, int q4, uint32_t tile, bool vote,
                                              const WaitCtl &w, bool &ok) {
    const uint32_t lane = lane_id();
    const bool wv = __all_sync(0xffffffffu, vote);
    if (lane == 0) {
        slots[q4] = (tile << 1) | (wv ? 1u : 0u);
        __threadfence_block();
    }
    __syncwarp();
    bool yes = true, good = true;
    if (lane < 4) {
        const uint64_t t0 = globaltimer();
        for (uint32_t it = 0;; ++it) {
            const uint32_t v = slots[lane];
            if ((v >> 1) == tile) {
                yes = (v & 1u) != 0u;
                break;
            }
            if ((it & 31u) == 31u) {
                if (*w.abort) { good = false; break; }
                if (globaltimer() - t0 > w.timeout_ns || it > (1u << 30)) {
                    *w.abort = 1;
                    flag_status(kStTimeout);
                    good = false;
                    break;
                }
            }
        }
    }
    ok = __all_sync(0xffffffffu, good);
    return __all_sync(0xffffffffu, yes);
}

template <int D>
struct AttnSmem {
    static constexpr int TB = 128 * D * 2;
    static constexpr int KS = (D == 128) ? 2 : 4;
    static constexpr int BYTES = (2 + 2 * KS) * TB + 1024 + 512 + 1024;  // + two 4096-bit block bitmaps
};

template <int D, bool SKIP>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
    using SM = AttnSmem<D>;
    constexpr int TB = SM::TB;
    constexpr int KS = SM::KS;
    constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, 128, false, false);
    constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, false, true);

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem;                      // [2][TB]
    uint8_t *sK = smem + 2 * TB;             // [KS][TB]
    uint8_t *sV = smem + (2 + KS) * TB;      // [KS][TB]
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + (2 + 2 * KS) * TB);
    // Without SKIP, k_full[g % KS] / k_empty[g % KS] carry load group g: K(0)
    // for g = 0, then V(g-1) with K(g) (the MMA thread needs both at the same
    // point, PV(g-1) then QK(g)), the last group V alone; v_full / v_empty are
    // unused.  With SKIP, K and V have rings of their own (below).
    uint64_t *q_full = bars;                 // 1
    uint64_t *s_full = bars + 1;             // 2
    uint64_t *p_full = bars + 3;             // 2
    uint64_t *drain = bars + 5;              // 1: every MMA of the CTA has completed
    uint64_t *k_full = bars + 6;             // KS
    uint64_t *k_empty = bars + 6 + KS;       // KS
    uint64_t *v_full = bars + 6 + 2 * KS;    // KS
    uint64_t *v_empty = bars + 6 + 3 * KS;   // KS
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 6 + 4 * KS);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    volatile uint32_t *vote = tmem_slot + 4;        // SKIP: [2 heads][4 warps] tagged votes
    volatile uint32_t *skip_flag = tmem_slot + 12;  // SKIP: [2 heads][2 tile parities]
    volatile uint32_t *dec = tmem_slot + 16;        // SKIP: [2 heads][2 tile parities] (block << 1 | skipped)
    uint32_t *bm = reinterpret_cast<uint32_t *>(smem + (2 + 2 * KS) * TB + 512);  // [2][128] block bitmaps

    // ------------------------------------------------------------ work item
    // Grid order: (batch, KV head) outermost, then query blocks from the
    // longest down, then the head units of that KV head.  The CTAs resident at
    // one time therefore share one KV head, whose K/V then stays in L2.
    const int U = p.units_per_kv;
    const int j = static_cast<int>(blockIdx.x % U);
    long long rest = blockIdx.x / U;
    const int qb_grid = p.nb - 1 - static_cast<int>(rest % p.nb);
    rest /= p.nb;
    const int kv_of_cta = static_cast<int>(rest % p.Hkv);
    const int b = static_cast<int>(rest / p.Hkv);
    if (j >= p.kv_units[kv_of_cta]) return;  // this KV head has fewer units (whole CTA, before any sync)
    const int kvh = kv_of_cta;
    const int hk = static_cast<int>((static_cast<long long>(kvh) * p.H + p.Hkv - 1) / p.Hkv);
    const int nh = static_cast<int>((static_cast<long long>(kvh + 1) * p.H + p.Hkv - 1) / p.Hkv) - hk;
    // The CTAs of query blocks qtop and qtop - 1 (qtop at an even distance from
    // the last block) sit next to each other in the grid and split the 2 * nh
    // (head, query block) items of this KV head between them in one of two ways:
    //
    // by count: per query block, the heads ranked by (cnt, head), unit j taking
    //   ranks 2j and 2j+1.  Heads of one proxy group visit prefixes of the same
    //   list, so a pair with close counts shares most of its K/V tiles and both
    //   heads are busy on them.  An odd head count leaves the last unit of a
    //   query block one head; such lone units of the two query blocks share the
    //   CTA of qtop (slot 0 at qtop, slot 1 at qtop - 1), and the lone unit at
    //   qtop - 1 has no work.
    // by head: each CTA takes one head at qtop (slot 0) and qtop - 1 (slot 1):
    //   two rows of one ranking with nearly equal budgets, whose lists overlap
    //   in most blocks even when the heads of the KV head have very different
    //   budgets (where pairs by count leave many tiles to one slot alone).
    //
    // Both CTAs choose the same way from the counts of both query blocks: by
    // head when the sum over heads of the larger of a head's two counts, plus
    // 2 % for the blocks only one of the two rows keeps, is below the tiles of
    // the pairs by count (the larger count of each pair, and the larger of the
    // two lone heads' counts).  With the block skip every unit is one head at
    // qtop and qtop - 1 (one unit per head, units_per_kv = the heads of a KV
    // head): a tile saves time only when both slots skip it, and one head's
    // decisions on the blocks of two adjacent rows agree far more often than
    // two heads' decisions do.  qbt[t] is slot t's query block.
    const bool upper = ((p.nb - 1 - qb_grid) & 1) == 0;
    const int qtop = upper ? qb_grid : qb_grid + 1;
    __shared__ int pair_heads[2];
    __shared__ int pair_cost[3];  // by count (pairs), by head, by count (the lone heads)
    bool by_head = SKIP;
    if constexpr (!SKIP) {
        if (qtop > 0) {  // uniform over the CTA
            if (threadIdx.x < 3) pair_cost[threadIdx.x] = 0;
            __syncthreads();
            if (static_cast<int>(threadIdx.x) < nh) {
                const int me = static_cast<int>(threadIdx.x);
                int c_me[2];
                for (int t = 0; t < 2; ++t) {
                    const int qx = qtop - t;
                    const int len = p.causal ? qx + 1 : p.nb;
                    const int32_t *cq = p.cnt + (static_cast<long long>(b) * p.H + hk) * p.nb + qx;
                    c_me[t] = min(max(static_cast<int>(cq[static_cast<long long>(me) * p.nb]), 0), len);
                    int r = 0;
                    for (int y = 0; y < nh; ++y) {
                        const int c_y = min(max(static_cast<int>(cq[static_cast<long long>(y) * p.nb]), 0), len);
                        r += (c_y < c_me[t] || (c_y == c_me[t] && y < me)) ? 1 : 0;
                    }
                    if ((nh & 1) != 0 && r == nh - 1)
                        atomicMax(&pair_cost[2], c_me[t]);
                    else if ((r & 1) != 0)
                        atomicAdd(&pair_cost[0], c_me[t]);
                }
                atomicAdd(&pair_cost[1], max(c_me[0], c_me[1]));
            }
            __syncthreads();
            by_head = 50LL * pair_cost[1] < 49LL * (static_cast<long long>(pair_cost[0]) + pair_cost[2]);
        }
    }
    int qb = qb_grid;  // slot 0's query block
    bool lone_pair;    // slot 1 takes query block qb - 1
    if (by_head) {
        const int x = SKIP ? (upper ? j : nh) : (upper ? 0 : static_cast<int>(p.kv_units[kvh])) + j;
        if (x >= nh) return;  // no head left for this CTA (the whole CTA returns)
        qb = qtop;
        lone_pair = qtop > 0;
        if (threadIdx.x == 0) {
            pair_heads[0] = hk + x;
            pair_heads[1] = lone_pair ? hk + x : -1;
        }
    } else {
        const bool lone = (nh & 1) != 0 && j == (nh >> 1);
        if (lone && !upper) return;  // taken by the CTA of qtop (the whole CTA returns)
        lone_pair = lone && qb > 0;
        for (int t = 0; t < (lone_pair ? 2 : 1); ++t) {
            const int qx = qb - t;
            if (static_cast<int>(threadIdx.x) < nh) {
                const int32_t *cq = p.cnt + (static_cast<long long>(b) * p.H + hk) * p.nb + qx;
                const int me = static_cast<int>(threadIdx.x);
                const int32_t c_me = cq[static_cast<long long>(me) * p.nb];
                int r = 0;
                for (int y = 0; y < nh; ++y) {
                    const int32_t c_y = cq[static_cast<long long>(y) * p.nb];
                    r += (c_y < c_me || (c_y == c_me && y < me)) ? 1 : 0;
                }
                if (lone) {
                    if (r == nh - 1) pair_heads[t] = hk + me;  // the lone head of query block qx
                } else if ((r >> 1) == j) {
                    pair_heads[r & 1] = hk + me;
                }
            }
        }
        if (threadIdx.x == 0 && 2 * j + 1 >= nh && !lone_pair) pair_heads[1] = -1;  // one head, one slot
    }
    // The selected blocks of each head as a bitmap over 0..qb: head t takes the
    // first c[t] entries of its list.  Every role then visits them in
    // ascending block order (the result does not depend on the order), so the
    // CTAs resident at one time sweep K/V in step.
    for (int w = threadIdx.x; w < 256; w += blockDim.x) bm[w] = 0u;
    __syncthreads();
    // the roles below re-read the pair from shared memory where they need it
    // (cheaper than keeping two registers live through every role)
    const volatile int *pair = pair_heads;
    const int h0 = pair[0];
    const int h1 = pair[1];
    const int qbt[2] = {qb, lone_pair ? qb - 1 : qb};
    const long long T = p.causal ? static_cast<long long>(p.nb) * (p.nb + 1) / 2 : static_cast<long long>(p.nb) * p.nb;
    auto row_off_of = [&](int x) -> long long {
        return p.causal ? static_cast<long long>(x) * (x + 1) / 2 : static_cast<long long>(x) * p.nb;
    };
    const int row_len = p.causal ? qb + 1 : p.nb;  // blocks in slot 0's list (slot 1's is no longer)
    const int row_len1 = p.causal ? qbt[1] + 1 : p.nb;
    const int32_t *list0 =
        p.rank + (static_cast<long long>(b) * p.G + static_cast<long long>(h0) * p.G / p.H) * T + row_off_of(qbt[0]);
    const int32_t *list1 =
        p.rank + (static_cast<long long>(b) * p.G + static_cast<long long>(h1 >= 0 ? h1 : h0) * p.G / p.H) * T +
        row_off_of(qbt[1]);
    int craw[2];
    craw[0] = p.cnt[(static_cast<long long>(b) * p.H + h0) * p.nb + qbt[0]];
    craw[1] = (h1 >= 0) ? p.cnt[(static_cast<long long>(b) * p.H + h1) * p.nb + qbt[1]] : 0;
    int c[2];
    c[0] = min(max(craw[0], 0), row_len);
    c[1] = min(max(craw[1], 0), row_len1);
    const int ntiles = (h1 >= 0) ? 2 : 1;
    const int words = (row_len + 31) >> 5;  // bitmap words covering both slots' blocks

    const uint32_t warp = warp_id(), lane = lane_id();
    if (warp == kProducerWarp && lane == 0) {
        // The barriers, then the two Q tiles at once: their copy overlaps the
        // bitmap build, the TMEM allocation and the CTA barrier below.  No other
        // thread touches a barrier before that CTA barrier.
        mbar_init(q_full, 1);
        for (int t = 0; t < 2; ++t) {
            mbar_init(&s_full[t], 1);
            mbar_init(&p_full[t], 128);
        }
        mbar_init(drain, 1);
        for (int s = 0; s < KS; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        *abort_flag = 0;
        for (int x = 0; x < 8; ++x) vote[x] = 0xFFFFFFFFu;  // a tag no tile carries
        for (int x = 0; x < 4; ++x) skip_flag[x] = 0u;
        for (int x = 0; x < 4; ++x) dec[x] = 0xFFFFFFFFu;  // a tag no block carries
        fence_mbar_init();
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        mbar_arrive_expect_tx(q_full, ntiles * TB);
#pragma unroll
        for (int cc = 0; cc < D / 64; ++cc) {
            tma_load_4d(sQ + cc * 16384, &tmQ, q_full, cc * 64, h0, qbt[0] * 128, b);
            if (h1 >= 0) tma_load_4d(sQ + TB + cc * 16384, &tmQ, q_full, cc * 64, h1, qbt[1] * 128, b);
        }
    }

    for (int x = threadIdx.x; x < c[0] + c[1]; x += blockDim.x) {
        const int t = (x < c[0]) ? 0 : 1;
        const int kb = t ? list1[x - c[0]] : list0[x];
        if (kb < 0 || kb >= (t ? row_len1 : row_len)) {
            flag_status(kStBounds);
            continue;
        }
        atomicOr(&bm[t * 128 + (kb >> 5)], 1u << (kb & 31));
    }

    if (threadIdx.x == 0 && (c[0] != craw[0] || (h1 >= 0 && c[1] != craw[1]))) flag_status(kStBounds);
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const WaitCtl wc{abort_flag, p.timeout_ns};

    if (warp >= 8) {
      // warpgroup 2 (producer, MMA issuer, two idle warps) hands registers to
      // the softmax warpgroups; the branch is uniform per warpgroup
      reg_release<kRegsAux>();
      if (warp == kProducerWarp) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {  // (the Q tiles are already on their way)
          if constexpr (SKIP) {
            // K runs KS tiles ahead.  V of a tile is loaded only once a head that
            // visits it has kept it (its decision slot carries the block's tag with
            // the skip bit clear); a tile every visiting head skips loads no V.  A
            // head decides at most one tile ahead of this loop (its next S needs a
            // K this loop loads after the decision), so two slots per head suffice.
            int nk = 0, nvl = 0;  // K and V copies issued
            int kbk = next_block(bm, bm + 128, 0, words);
            for (; kbk >= 0 && nk < KS; kbk = next_block(bm, bm + 128, kbk + 1, words), ++nk) {
                mbar_arrive_expect_tx(&k_full[nk], TB);
#pragma unroll
                for (int cc = 0; cc < D / 64; ++cc)
                    tma_load_4d(sK + nk * TB + cc * 16384, &tmK, &k_full[nk], cc * 64, kvh, kbk * 128, b);
            }
            int seen_t[2] = {0, 0};  // tiles of each head passed so far
            for (int kb = next_block(bm, bm + 128, 0, words); kb >= 0; kb = next_block(bm, bm + 128, kb + 1, words)) {
                const bool f0 = ((bm[kb >> 5] >> (kb & 31)) & 1u) != 0u;
                const bool f1 = ((bm[128 + (kb >> 5)] >> (kb & 31)) & 1u) != 0u;
                bool d0 = !f0, d1 = !f1, keep = false, good = true;
                const uint64_t t0 = globaltimer();
                for (uint32_t it = 0; !keep && !(d0 && d1); ++it) {
                    if (!d0) {
                        const uint32_t v = dec[seen_t[0] & 1];
                        if ((v >> 1) == static_cast<uint32_t>(kb)) { d0 = true; keep = keep || (v & 1u) == 0u; }
                    }
                    if (!d1) {
                        const uint32_t v = dec[2 + (seen_t[1] & 1)];
                        if ((v >> 1) == static_cast<uint32_t>(kb)) { d1 = true; keep = keep || (v & 1u) == 0u; }
                    }
                    if ((it & 31u) == 31u) {
                        if (*wc.abort) { good = false; break; }
                        if (globaltimer() - t0 > wc.timeout_ns || it > (1u << 30)) {
                            *wc.abort = 1;
                            flag_status(kStTimeout);
                            good = false;
                            break;
                        }
                    }
                }
                if (!good) break;
                seen_t[0] += f0 ? 1 : 0;
                seen_t[1] += f1 ? 1 : 0;
                if (keep) {
                    const int sv = nvl % KS;
                    if (nvl >= KS && !mbar_wait(&v_empty[sv], ((nvl / KS) - 1) & 1, wc)) break;
                    mbar_arrive_expect_tx(&v_full[sv], TB);
#pragma unroll
                    for (int cc = 0; cc < D / 64; ++cc)
                        tma_load_4d(sV + sv * TB + cc * 16384, &tmV, &v_full[sv], cc * 64, kvh, kb * 128, b);
                    ++nvl;
                }
                if (kbk >= 0) {
                    const int sk = nk % KS;
                    if (!mbar_wait(&k_empty[sk], ((nk / KS) - 1) & 1, wc)) break;
                    mbar_arrive_expect_tx(&k_full[sk], TB);
#pragma unroll
                    for (int cc = 0; cc < D / 64; ++cc)
                        tma_load_4d(sK + sk * TB + cc * 16384, &tmK, &k_full[sk], cc * 64, kvh, kbk * 128, b);
                    ++nk;
                    kbk = next_block(bm, bm + 128, kbk + 1, words);
                }
            }
            // teardown: let every copy in flight land before the CTA exits
            mbar_wait_drain(q_full, 0, p.timeout_ns);
            for (int x = max(nk - KS, 0); x < nk; ++x) mbar_wait_drain(&k_full[x % KS], (x / KS) & 1, p.timeout_ns);
            for (int x = max(nvl - KS, 0); x < nvl; ++x) mbar_wait_drain(&v_full[x % KS], (x / KS) & 1, p.timeout_ns);
          } else {
            // group 0 = K(0); group g >= 1 = V(g-1) and K(g); the last group V(n-1) alone.
            // Group g uses barrier slot g % KS, K slot g % KS and V slot (g-1) % KS, which
            // group g - KS released.
            int kb = next_block(bm, bm + 128, 0, words);
            int kb_v = -1;
            int issued = 0;
            for (int g = 0; kb >= 0 || kb_v >= 0; ++g) {
                const int s = g % KS;
                if (g >= KS && !mbar_wait(&k_empty[s], ((g / KS) - 1) & 1, wc)) break;
                mbar_arrive_expect_tx(&k_full[s], (kb >= 0 ? TB : 0) + (kb_v >= 0 ? TB : 0));
                if (kb_v >= 0) {
                    const int sv = (g + KS - 1) % KS;
#pragma unroll
                    for (int cc = 0; cc < D / 64; ++cc)
                        tma_load_4d(sV + sv * TB + cc * 16384, &tmV, &k_full[s], cc * 64, kvh, kb_v * 128, b);
                }
                if (kb >= 0) {
#pragma unroll
                    for (int cc = 0; cc < D / 64; ++cc)
                        tma_load_4d(sK + s * TB + cc * 16384, &tmK, &k_full[s], cc * 64, kvh, kb * 128, b);
                }
                issued = g + 1;
                kb_v = kb;
                if (kb >= 0) kb = next_block(bm, bm + 128, kb + 1, words);
            }
            // teardown: let every copy in flight land before the CTA exits
            mbar_wait_drain(q_full, 0, p.timeout_ns);
            for (int g = max(issued - KS, 0); g < issued; ++g)
                mbar_wait_drain(&k_full[g % KS], (g / KS) & 1, p.timeout_ns);
          }
        }
    } else if (warp == kMmaWarp) {
        // ---------------------------------------------------------- MMA issuer
        const int kb_first = next_block(bm, bm + 128, 0, words);
        if (lane == 0 && kb_first >= 0) {
            // smem descriptors precomputed once; a K step only moves the start
            // address (+32 B within a 128-byte swizzle row, +16 KB per 64-column
            // chunk; +2 KB per 16 keys of V)
            const uint64_t dq[2] = {sdesc_sw128(smem_u32(sQ), 16, 1024), sdesc_sw128(smem_u32(sQ + TB), 16, 1024)};
            const uint64_t dk0 = sdesc_sw128(smem_u32(sK), 16, 1024);
            const uint64_t dv0 = sdesc_sw128(smem_u32(sV), 16384, 1024);
            auto issue_qk = [&](int t, int s) {
                const uint64_t a = t ? dq[1] : dq[0];
                const uint64_t bk = dk0 + static_cast<uint64_t>((s * TB) >> 4);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t off = static_cast<uint64_t>(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
                    if (kk == 0)
                        umma_ss_c<false>(tmem + t * 128, a + off, bk + off, IDESC_QK);
                    else
                        umma_ss_c<true>(tmem + t * 128, a + off, bk + off, IDESC_QK);
                }
                umma_commit(&s_full[t]);
            };
            auto issue_pv = [&](int t, int s, bool accumulate) {
                const uint64_t bv = dv0 + static_cast<uint64_t>((s * TB) >> 4);
                const uint32_t acc0 = accumulate ? 1u : 0u;
                umma_ts(tmem + 256 + t * 128, tmem + t * 128, bv, IDESC_PV, acc0);
#pragma unroll
                for (int kk = 1; kk < 8; ++kk)  // 128 keys, 16 per step
                    umma_ts_c<true>(tmem + 256 + t * 128, tmem + t * 128 + kk * 8, bv + static_cast<uint64_t>(kk * 128),
                                    IDESC_PV);
            };
            // Visit cursor: the bitmap word holding the current block, of both
            // heads, stays in registers, so shared memory is read once per 32
            // blocks instead of on every step (shared-memory reads of this
            // thread queue behind the tensor core's operand reads).
            int cw = kb_first >> 5;
            uint32_t w0 = bm[cw], w1 = bm[128 + cw];
            // next visited block after kb (a block of word cw) and its per-head flags; -1 past the row
            auto next_visit = [&](int kb, uint32_t &f0, uint32_t &f1) -> int {
                const int sh = (kb & 31) + 1;
                uint32_t m = sh < 32 ? (w0 | w1) & (0xFFFFFFFFu << sh) : 0u;
                while (m == 0u) {
                    if (++cw >= words) return -1;
                    w0 = bm[cw];
                    w1 = bm[128 + cw];
                    m = w0 | w1;
                }
                const int bit = __ffs(static_cast<int>(m)) - 1;
                f0 = (w0 >> bit) & 1u;
                f1 = (w1 >> bit) & 1u;
                return (cw << 5) + bit;
            };
            uint32_t c0 = (w0 >> (kb_first & 31)) & 1u, c1 = (w1 >> (kb_first & 31)) & 1u;  // heads active at kb
            int seen0 = 0, seen1 = 0;  // tiles of each head whose P was handed over
            int pv0 = 0, pv1 = 0;      // SKIP: PV products issued for each head
            bool ok = mbar_wait(q_full, 0, wc) && mbar_wait(&k_full[0], 0, wc);
            if (ok) {
                tc_fence_after();
                if (c0) issue_qk(0, 0);
                if (c1) issue_qk(1, 0);
                umma_commit(&k_empty[0]);
            }
            int i = 0;
            int nvl = 0;  // SKIP: V tiles loaded (tiles some head kept), the V ring's counter
            for (int kb = kb_first; kb >= 0 && ok; ++i) {
                const int s1 = (i + 1) % KS;
                uint32_t n0 = 0u, n1 = 0u;  // heads active at kb_next
                const int kb_next = next_visit(kb, n0, n1);
                const bool has_next = kb_next >= 0;
                if constexpr (SKIP) {
                    // K(i+1) now; V(i) only once a head has kept tile i
                    if (has_next && !mbar_wait(&k_full[s1], ((i + 1) / KS) & 1, wc)) break;
                    tc_fence_after();
                    const int sv = nvl % KS;
                    bool v_in = false;
                    for (int t = 0; t < 2; ++t) {
                        if (t ? c1 : c0) {
                            int &seen = t ? seen1 : seen0;
                            int &pv = t ? pv1 : pv0;
                            if (!mbar_wait(&p_full[t], seen & 1, wc)) { ok = false; break; }
                            tc_fence_after();
                            const bool skipped = skip_flag[t * 2 + (seen & 1)] != 0u;
                            ++seen;
                            if (!skipped) {
                                if (!v_in) {
                                    if (!mbar_wait(&v_full[sv], (nvl / KS) & 1, wc)) { ok = false; break; }
                                    tc_fence_after();
                                    v_in = true;
                                }
                                issue_pv(t, sv, pv > 0);
                                ++pv;
                            }
                        }
                        if (has_next && (t ? n1 : n0)) issue_qk(t, s1);
                    }
                    if (!ok) break;
                    if (v_in) {
                        umma_commit(&v_empty[sv]);
                        ++nvl;
                    }
                    if (has_next) umma_commit(&k_empty[s1]);
                    kb = kb_next;
                    c0 = n0;
                    c1 = n1;
                    continue;
                }
                const int s = i % KS;
                // load group i+1: V(i) and, with a next tile, K(i+1)
                if (!mbar_wait(&k_full[s1], ((i + 1) / KS) & 1, wc)) break;
                tc_fence_after();
                for (int t = 0; t < 2; ++t) {
                    if (t ? c1 : c0) {
                        int &seen = t ? seen1 : seen0;
                        if (!mbar_wait(&p_full[t], seen & 1, wc)) { ok = false; break; }
                        tc_fence_after();
                        issue_pv(t, s, seen > 0);  // without skipping every tile has its PV
                        ++seen;
                    }
                    if (has_next && (t ? n1 : n0)) issue_qk(t, s1);
                }
                if (!ok) break;
                umma_commit(&k_empty[s1]);  // load group i+1 consumed
                kb = kb_next;
                c0 = n0;
                c1 = n1;
            }
        }
        if (lane == 0) {
            umma_commit(drain);
            mbar_wait_drain(drain, 0, p.timeout_ns);
        }
        __syncwarp();
      }
    } else {
        reg_acquire<kRegsSoftmax>();
        // ---------------------------------------------------------- softmax
        const int t = static_cast<int>(warp >> 2);
        const int h = (t && pair[1] >= 0) ? pair[1] : pair[0];  // an unpaired unit's second warpgroup has no blocks
        const int qbs = qbt[t];  // this slot's query block
        const long long skip_base = (static_cast<long long>(b) * p.H + h) * T + row_off_of(qbs);
        const uint32_t *bmt = bm + t * 128;
        const int q4 = static_cast<int>(warp & 3);
        const int row = q4 * 32 + static_cast<int>(lane);
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
        const uint32_t s_addr = lane_base + t * 128;
        const uint32_t o_addr = lane_base + 256 + t * 128;
        float m = -INFINITY, l = 0.0f;
        float mtrue = -INFINITY;  // SKIP: exact running max (log2 units) of the tiles visited
        bool ok = true;
        uint32_t s[128];
        int i = 0;    // tiles of this head so far
        int npv = 0;  // of them, tiles whose PV product was issued
        for (int kb = next_block(bmt, bmt, 0, words); kb >= 0; kb = next_block(bmt, bmt, kb + 1, words), ++i) {
            if (!warp_wait(&s_full[t], i & 1, wc)) { ok = false; break; }
            tc_fence_after();
            const bool masked = p.causal && kb == qbs;  // the causal diagonal tile: same for the whole warpgroup
            tmem_ld128(s_addr, s);
            if (masked) {
#pragma unroll
                for (int j = 0; j < 128; ++j)
                    if (j > row) s[j] = 0xFF800000u;  // -inf: causal mask of the diagonal tile
            }
            // row max of the tile: a tree of three-input maxima
            float mx[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const uint32_t *v = s + 8 * j;
                mx[j] = fmax3(fmax3(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2])),
                              fmax3(__uint_as_float(v[3]), __uint_as_float(v[4]), __uint_as_float(v[5])),
                              fmaxf(__uint_as_float(v[6]), __uint_as_float(v[7])));
            }
            const float mt = p.scale_log2 *
                fmax3(fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmax3(mx[6], mx[7], mx[8])),
                      fmax3(mx[9], mx[10], mx[11]), fmax3(mx[12], mx[13], fmaxf(mx[14], mx[15])));
            if constexpr (SKIP) {
                bool skip = false;
                if (i > 0) {
                    bool vote_ok = true;
                    skip = head_vote_all(vote + t * 4, q4, static_cast<uint32_t>(i), mt < mtrue + p.skip_log2, wc,
                                         vote_ok);
                    if (!vote_ok) { ok = false; break; }
                }
                mtrue = fmaxf(mtrue, mt);
                if (row == 0) {
                    skip_flag[t * 2 + (i & 1)] = skip ? 1u : 0u;
                    dec[t * 2 + (i & 1)] = (static_cast<uint32_t>(kb) << 1) | (skip ? 1u : 0u);
                }
                if (skip) {
                    // nothing of this tile enters O or l; S is free for the next QK
                    if (row == 0 && p.skipped) p.skipped[skip_base + kb] = 1;
                    tc_fence_before();
                    mbar_arrive(&p_full[t]);
                    continue;
                }
            }
            // The running max is raised only when it grows by more than 2^8; then O
            // (in TMEM) and l scale by alpha = 2^(m - m_new).  O is scaled after this
            // tile's P is stored, when the S registers are dead, and before P is
            // handed over, so before this tile's PV adds into O.
            const float m_new = fmaxf(m, mt);
            bool rescale = false;
            float alpha = 1.0f;
            if (i > 0) {
                const bool need = m_new > m + 8.0f;
                if (__any_sync(0xffffffffu, need)) {
                    rescale = true;
                    alpha = (m == -INFINITY) ? 0.0f : ex2(m - m_new);
                    m = m_new;
                }
            } else {
                m = m_new;
            }
            // P = 2^(x - m) as bf16 pairs written over the first 64 columns of S.
            // Each column pair takes one packed FMA for x = s * scale - m and
            // one packed add into four partial row sums.
            const float negm = (m == -INFINITY) ? 0.0f : -m;
            const float2 c2 = make_float2(p.scale_log2, p.scale_log2);
            const float2 nm = make_float2(negm, negm);
            float2 acc[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[j] = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t pk[32];
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) {
                    const int j = half * 32 + jj;
                    const float2 x =
                        __ffma2_rn(make_float2(__uint_as_float(s[2 * j]), __uint_as_float(s[2 * j + 1])), c2, nm);
                    const float2 e = make_float2(ex2(x.x), ex2(x.y));
                    acc[j & 3] = __fadd2_rn(acc[j & 3], e);
                    pk[jj] = pack_bf16x2(e.x, e.y);
                }
                tmem_st32(s_addr + half * 32, pk);
            }
            l = l * alpha + (((acc[0].x + acc[0].y) + (acc[1].x + acc[1].y)) +
                             ((acc[2].x + acc[2].y) + (acc[3].x + acc[3].y)));
            if (rescale) {
                // (this tile's S was committed after the head's last PV was issued,
                // and a commit covers every earlier MMA, so that PV is complete)
                tc_fence_after();
#pragma unroll
                for (int ch = 0; ch < D / 32; ++ch) {
                    uint32_t o[32];
                    tmem_ld32(o_addr + ch * 32, o);
#pragma unroll
                    for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
                    tmem_st32(o_addr + ch * 32, o);
                }
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&p_full[t]);
            if constexpr (SKIP) ++npv;
        }
        // epilogue: O / l -> bf16 -> global; LSE
        const int ct = SKIP ? npv : i;
        if (ct > 0 && ok && warp_wait(drain, 0, wc)) {
            tc_fence_after();
            const float inv = (l > 0.0f) ? 1.0f / l : 0.0f;
            __nv_bfloat16 *orow = p.o + b * p.osb + static_cast<int64_t>(qbs * 128 + row) * p.oss + h * p.osh;
#pragma unroll
            for (int ch = 0; ch < D / 32; ++ch) {
                uint32_t r[32];
                tmem_ld32(o_addr + ch * 32, r);
                uint32_t w[16];
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    w[j] = pack_bf16x2(__uint_as_float(r[2 * j]) * inv, __uint_as_float(r[2 * j + 1]) * inv);
                uint4 *dst = reinterpret_cast<uint4 *>(orow + ch * 32);
                dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
                dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
                dst[2] = make_uint4(w[8], w[9], w[10], w[11]);
                dst[3] = make_uint4(w[12], w[13], w[14], w[15]);
            }
            if (p.lse)
                p.lse[(static_cast<long long>(b) * p.H + h) * p.N + qbs * 128 + row] =
                    (m + log2f(l)) * 0.69314718055994531f;
        }
    }

    // -------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

}  // namespace pa
