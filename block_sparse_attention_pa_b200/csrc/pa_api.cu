// pa_api.cu -- the C ABI of libpa.so (declared in include/pa.h): argument
// validation, TMA descriptor construction, workspace carving and kernel
// launches.  Every step of the method runs in the kernels of this library;
// the host code only checks arguments and launches.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>

#include <nvtx3/nvToolsExt.h>

#include "pa.h"
#include "attn.cuh"
#include "mask.cuh"
#include "pool.cuh"
#include "tile_gemm.cuh"
#include "xattn.cuh"

namespace {

thread_local std::string g_last_error;

pa_status fail(pa_status s, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return s;
}

pa_status ok() {
    g_last_error.clear();
    return PA_OK;
}

#define PA_CUDA(call)                                                                       \
    do {                                                                                    \
        cudaError_t e_ = (call);                                                            \
        if (e_ != cudaSuccess) return fail(PA_ERR_CUDA, "%s: %s", #call, cudaGetErrorString(e_)); \
    } while (0)

constexpr int kBlk = 128;
constexpr int kMaxNb = 4096;
constexpr int kScoreChunk = 16;  // tiles per score/mass work unit

// NVTX ranges around every launch (and around pa_prefill and
// pa_prefill_varlen as a whole) when PA_NVTX=1, for profilers that group
// kernels by range; off by default (read once, at the first call).
bool nvtx_on() {
    static const bool v = [] {
        const char *e = getenv("PA_NVTX");
        return e && e[0] == '1';
    }();
    return v;
}

struct Trace {
    bool on;
    explicit Trace(const char *name) : on(nvtx_on()) {
        if (on) nvtxRangePushA(name);
    }
    ~Trace() {
        if (on) nvtxRangePop();
    }
    Trace(const Trace &) = delete;
    Trace &operator=(const Trace &) = delete;
};

uint64_t wait_timeout_ns() {
    static uint64_t v = [] {
        const char *e = getenv("PA_WAIT_TIMEOUT_MS");
        double ms = e ? atof(e) : 2000.0;
        if (!(ms > 0.0)) ms = 2000.0;
        return static_cast<uint64_t>(ms * 1e6);
    }();
    return v;
}

// ------------------------------------------------------------- validation
pa_status check_shape(const pa_shape *s) {
    if (!s) return fail(PA_ERR_INVALID_ARG, "shape is NULL");
    if (s->batch < 1 || s->seqlen < 1 || s->num_q_heads < 1 || s->num_kv_heads < 1 || s->num_groups < 1)
        return fail(PA_ERR_INVALID_ARG, "shape fields must be positive");
    if (s->block != kBlk) return fail(PA_ERR_UNSUPPORTED, "block must be 128 (got %d)", s->block);
    if (s->head_dim != 64 && s->head_dim != 128)
        return fail(PA_ERR_UNSUPPORTED, "head_dim must be 64 or 128 (got %d)", s->head_dim);
    if (s->seqlen % kBlk) return fail(PA_ERR_UNSUPPORTED, "seqlen %d is not a multiple of 128", s->seqlen);
    if (s->seqlen / kBlk > kMaxNb) return fail(PA_ERR_UNSUPPORTED, "seqlen %d exceeds %d", s->seqlen, kMaxNb * kBlk);
    if (s->num_q_heads > pa::kMaxHeads) return fail(PA_ERR_UNSUPPORTED, "more than %d q heads", pa::kMaxHeads);
    if (s->num_q_heads % s->num_kv_heads)
        return fail(PA_ERR_UNSUPPORTED, "num_q_heads %d not a multiple of num_kv_heads %d", s->num_q_heads,
                    s->num_kv_heads);
    if (s->num_q_heads % s->num_groups)
        return fail(PA_ERR_UNSUPPORTED, "num_q_heads %d not a multiple of num_groups %d", s->num_q_heads,
                    s->num_groups);
    if (s->non_causal != 0 && s->non_causal != 1)
        return fail(PA_ERR_INVALID_ARG, "non_causal must be 0 or 1 (got %d)", s->non_causal);
    return PA_OK;
}

bool causal_of(const pa_shape *s) { return s->non_causal == 0; }

// Entries of one (b, g) set of block scores or ranked lists.
size_t rows_total(const pa_shape *s) {
    const size_t nb = s->seqlen / kBlk;
    return causal_of(s) ? nb * (nb + 1) / 2 : nb * nb;
}

// Query-row stride of the block scores: 1, 2, 4 or 8.
pa_status check_stride(int r) {
    if (r != 1 && r != 2 && r != 4 && r != 8)
        return fail(PA_ERR_INVALID_ARG, "score_stride must be 1, 2, 4 or 8 (got %d)", r);
    return PA_OK;
}

// pa_budget.score_stride with 0 (a zero-initialised struct) read as 1.
int stride_of(const pa_budget *bu) { return (bu && bu->score_stride > 0) ? bu->score_stride : 1; }

pa_status check_skip(float lambda) {
    if (!(lambda >= 0.0f && lambda <= 1.0f))
        return fail(PA_ERR_INVALID_ARG, "skip_threshold must be in [0, 1] (got %g)", static_cast<double>(lambda));
    return PA_OK;
}

pa_status check_budget(const pa_budget *bu) {
    if (!bu) return fail(PA_ERR_INVALID_ARG, "budget is NULL");
    if (check_skip(bu->skip_threshold)) return PA_ERR_INVALID_ARG;
    if (bu->score_stride != 0 && check_stride(bu->score_stride)) return PA_ERR_INVALID_ARG;
    if (bu->mode == PA_BUDGET_DYNAMIC) {
        if (!(bu->gamma > 0.0f && bu->gamma <= 1.0f))
            return fail(PA_ERR_INVALID_ARG, "gamma must be in (0, 1] (got %g)", static_cast<double>(bu->gamma));
    } else if (bu->mode == PA_BUDGET_FIXED_FRACTION) {
        if (bu->frac_permille < 1 || bu->frac_permille > 1000)
            return fail(PA_ERR_INVALID_ARG, "frac_permille must be in 1..1000 (got %d)", bu->frac_permille);
    } else if (bu->mode != PA_BUDGET_ALL) {
        return fail(PA_ERR_INVALID_ARG, "unknown budget mode %d", bu->mode);
    }
    return PA_OK;
}

pa_status check_ptr(const void *p, const char *name, size_t align = 16) {
    if (!p) return fail(PA_ERR_INVALID_ARG, "%s is NULL", name);
    if (reinterpret_cast<uintptr_t>(p) % align)
        return fail(PA_ERR_INVALID_ARG, "%s is not %zu-byte aligned", name, align);
    return PA_OK;
}

pa_status check_tensor(const void *p, pa_strides st, const char *name) {
    pa_status s = check_ptr(p, name);
    if (s) return s;
    if (st.b < 0 || st.s <= 0 || st.h <= 0 || st.b % 8 || st.s % 8 || st.h % 8)
        return fail(PA_ERR_INVALID_ARG, "%s strides (%lld, %lld, %lld) must be positive multiples of 8 elements", name,
                    static_cast<long long>(st.b), static_cast<long long>(st.s), static_cast<long long>(st.h));
    return PA_OK;
}

// ------------------------------------------------------------ tensor maps
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// A bf16 tensor of 4 dims (innermost first) with byte strides of dims 1..3,
// box 64 x b1 x b2 x 1, 128-byte swizzle.
pa_status make_map(CUtensorMap *m, const void *base, const cuuint64_t dims[4], const cuuint64_t strides[3],
                   cuuint32_t box1, cuuint32_t box2, const char *name) {
    auto fn = encode_fn();
    if (!fn) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    const cuuint32_t box[4] = {64, box1, box2, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled(%s) failed: %d", name, static_cast<int>(r));
    return PA_OK;
}

// [B][N][heads][d] with element strides -> dims (d, heads, N, B), box 64x1x128x1
pa_status map_bnhd(CUtensorMap *m, const void *base, int B, int N, int heads, int d, pa_strides st,
                   const char *name) {
    const int64_t sb = (B == 1) ? st.s * N : st.b;
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(heads),
                                static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(B)};
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(st.h) * 2, static_cast<cuuint64_t>(st.s) * 2,
                                   static_cast<cuuint64_t>(sb) * 2};
    return make_map(m, base, dims, strides, 1, 128, name);
}

// contiguous [B][G][N][d] proxies -> dims (d, N, G, B), box 64x128x1x1
pa_status map_proxy(CUtensorMap *m, const void *base, int B, int G, int N, int d, const char *name) {
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                                static_cast<cuuint64_t>(G), static_cast<cuuint64_t>(B)};
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(N) * d * 2,
                                   static_cast<cuuint64_t>(G) * N * d * 2};
    return make_map(m, base, dims, strides, 128, 1, name);
}

// [B][N][heads][d] with element strides, the token axis split as (token mod S,
// token / S) -> dims (d, heads, S, N/S, B), box 64 x 1 x 1 x rows x 1.
pa_status map_bnhd_split(CUtensorMap *m, const void *base, int B, int N, int heads, int d, int S, pa_strides st,
                         cuuint32_t rows, const char *name) {
    auto fn = encode_fn();
    if (!fn) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    const int64_t sb = (B == 1) ? st.s * N : st.b;
    const cuuint64_t dims[5] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(heads),
                                static_cast<cuuint64_t>(S), static_cast<cuuint64_t>(N / S),
                                static_cast<cuuint64_t>(B)};
    const cuuint64_t strides[4] = {static_cast<cuuint64_t>(st.h) * 2, static_cast<cuuint64_t>(st.s) * 2,
                                   static_cast<cuuint64_t>(st.s) * S * 2, static_cast<cuuint64_t>(sb) * 2};
    const cuuint32_t box[5] = {64, 1, 1, rows, 1};
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled(%s) failed: %d", name, static_cast<int>(r));
    return PA_OK;
}

int num_sms() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

// ------------------------------------------------------------- workspace
struct WsLayout {
    size_t qp, kp, scores, partial, total;
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

WsLayout ws_layout(const pa_shape *s, const pa_budget *bu) {
    const size_t B = s->batch, G = s->num_groups, N = s->seqlen, d = s->head_dim, H = s->num_q_heads;
    const size_t nb = N / kBlk, T = rows_total(s);
    WsLayout w;
    w.partial = 0;
    const size_t part = (bu && bu->mode == PA_BUDGET_DYNAMIC) ? align256(B * H * nb * 128 * sizeof(float2)) : 0;
    w.qp = part;
    w.kp = w.qp + align256(B * G * (N / stride_of(bu)) * d * 2);  // strided q proxy: scored rows only
    w.scores = w.kp + align256(B * G * N * d * 2);
    w.total = w.scores + align256(B * G * T * sizeof(float));
    return w;
}

size_t mask_ws_bytes(const pa_shape *s, const pa_budget *bu) {
    return ws_layout(s, bu).qp;  // the partial-softmax statistics come first
}

// XAttention partials: part_s [B][H][N/S][nb] then part_m [B][H][nchunk][N/S].
struct XWsLayout {
    size_t part_s, part_m, total;
};

XWsLayout xattn_ws_layout(const pa_shape *s, int S) {
    const size_t B = s->batch, H = s->num_q_heads, N = s->seqlen, nb = N / kBlk;
    const size_t rows = N / S, nchunk = (rows + 127) / 128;
    XWsLayout w;
    w.part_s = 0;
    w.part_m = align256(B * H * nb * rows * sizeof(float));
    w.total = w.part_m + align256(B * H * nchunk * rows * sizeof(float));
    return w;
}

pa_status check_xstride(int S) {
    if (S != 4 && S != 8 && S != 16) return fail(PA_ERR_INVALID_ARG, "stride must be 4, 8 or 16 (got %d)", S);
    return PA_OK;
}

// ------------------------------------------------------------- launches
pa_status launch_pool(const pa_shape *s, int stride, const void *q, pa_strides qs, const void *k, pa_strides ks,
                      void *qp, void *kp, cudaStream_t st) {
    Trace tr_("pa.pool_heads");
    pa::PoolParams p;
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.k = static_cast<const __nv_bfloat16 *>(k);
    p.qp = static_cast<__nv_bfloat16 *>(qp);
    p.kp = static_cast<__nv_bfloat16 *>(kp);
    p.qsb = qs.b; p.qss = qs.s; p.qsh = qs.h;
    p.ksb = ks.b; p.kss = ks.s; p.ksh = ks.h;
    p.B = s->batch; p.N = s->seqlen; p.H = s->num_q_heads; p.Hkv = s->num_kv_heads;
    p.G = s->num_groups; p.d = s->head_dim;
    p.stride = stride;
    // one thread per 8 head-dim elements of one (batch, token, group): x over
    // tokens, y over groups, z over the batch (in launches of at most 65535
    // sequences, the grid's z limit)
    const int B = p.B;
    constexpr int kMaxZ = 65535;
    for (int b0 = 0; b0 < B; b0 += kMaxZ) {
        pa::PoolParams pc = p;
        pc.B = std::min(kMaxZ, B - b0);
        pc.q = p.q + static_cast<int64_t>(b0) * p.qsb;
        pc.k = p.k + static_cast<int64_t>(b0) * p.ksb;
        pc.qp = p.qp + static_cast<int64_t>(b0) * p.G * (p.N / stride) * p.d;
        pc.kp = p.kp + static_cast<int64_t>(b0) * p.G * p.N * p.d;
        const dim3 grid(static_cast<unsigned>((static_cast<long long>(p.N) * (p.d / 8) + 255) / 256),
                        static_cast<unsigned>(p.G), static_cast<unsigned>(pc.B));
        if (p.d == 128) pa::pool_heads_kernel<128><<<grid, 256, 0, st>>>(pc);
        else pa::pool_heads_kernel<64><<<grid, 256, 0, st>>>(pc);
    }
    PA_CUDA(cudaGetLastError());
    return PA_OK;
}

template <int D, int MODE>
pa_status launch_tile_gemm_t(const CUtensorMap &a, const CUtensorMap &b, const pa::TileParams &p, cudaStream_t st) {
    auto kern = pa::tile_gemm_kernel<D, MODE>;
    const int smem = pa::TileSmem<D>::BYTES;
    PA_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    const long long grid = std::min<long long>(p.num_units, num_sms());
    if (grid <= 0) return PA_OK;
    kern<<<static_cast<unsigned>(grid), pa::kTileThreads, smem, st>>>(a, b, p);
    PA_CUDA(cudaGetLastError());
    return PA_OK;
}

pa_status launch_scores(const pa_shape *s, int stride, const void *qp, const void *kp, float *scores,
                        cudaStream_t st) {
    Trace tr_("pa.block_scores");
    const int B = s->batch, G = s->num_groups, N = s->seqlen, d = s->head_dim, nb = N / kBlk;
    CUtensorMap ma, mb;
    pa_status r = map_proxy(&ma, qp, B, G, N / stride, d, "q_proxy");
    if (r) return r;
    if ((r = map_proxy(&mb, kp, B, G, N, d, "k_proxy"))) return r;
    pa::TileParams p{};
    p.B = B; p.nb = nb; p.NH = G; p.H = s->num_q_heads; p.Hkv = s->num_kv_heads;
    p.chunk = kScoreChunk;
    p.stride = stride;
    p.causal = causal_of(s) ? 1 : 0;
    // causal: A tile m (query blocks m*r .. m*r+r-1) owns ceil((m+1) / (chunk/r))
    // units; non-causal: every A tile owns ceil(nb / chunk)
    const int cr = kScoreChunk / stride;
    const int a_tiles = (nb + stride - 1) / stride;
    long long per = 0;
    if (p.causal)
        for (int m = 0; m < a_tiles; ++m) per += (m + cr) / cr;
    else
        per = static_cast<long long>(a_tiles) * ((nb + kScoreChunk - 1) / kScoreChunk);
    p.units_per_bh = per;
    p.num_units = per * B * G;
    p.scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(d)));
    p.scores = scores;
    p.partial = nullptr;
    p.timeout_ns = wait_timeout_ns();
    return d == 128 ? launch_tile_gemm_t<128, pa::MODE_SCORES>(ma, mb, p, st)
                    : launch_tile_gemm_t<64, pa::MODE_SCORES>(ma, mb, p, st);
}

pa_status launch_mass(const pa_shape *s, const void *q, pa_strides qs, const void *k, pa_strides ks, float2 *partial,
                      float *mass, cudaStream_t st) {
    Trace tr_("pa.head_mass");
    const int B = s->batch, H = s->num_q_heads, Hkv = s->num_kv_heads, N = s->seqlen, d = s->head_dim;
    const int nb = N / kBlk;
    CUtensorMap ma, mb;
    pa_status r = map_bnhd(&ma, q, B, N, H, d, qs, "q");
    if (r) return r;
    if ((r = map_bnhd(&mb, k, B, N, Hkv, d, ks, "k"))) return r;
    pa::TileParams p{};
    p.B = B; p.nb = nb; p.NH = H; p.H = H; p.Hkv = Hkv;
    p.chunk = kScoreChunk;
    p.stride = 1;
    p.causal = causal_of(s) ? 1 : 0;
    p.units_per_bh = (nb + kScoreChunk - 1) / kScoreChunk;
    p.num_units = p.units_per_bh * B * H;
    p.scale = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(d)));
    p.scores = nullptr;
    p.partial = partial;
    p.timeout_ns = wait_timeout_ns();
    r = d == 128 ? launch_tile_gemm_t<128, pa::MODE_MASS>(ma, mb, p, st)
                 : launch_tile_gemm_t<64, pa::MODE_MASS>(ma, mb, p, st);
    if (r) return r;
    pa::mass_combine_kernel<<<B * H * pa::kMcCta, pa::kMcThreads, 0, st>>>(partial, mass, nb);
    PA_CUDA(cudaGetLastError());
    return PA_OK;
}

pa_status launch_rank(const pa_shape *s, const float *scores, int32_t *rank, cudaStream_t st) {
    Trace tr_("pa.rank");
    const int nb = s->seqlen / kBlk;
    int P = 1;
    while (P < nb - 1) P <<= 1;
    const int smem = P * 8;
    PA_CUDA(cudaFuncSetAttribute(pa::rank_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, std::max(smem, 1)));
    const long long grid = static_cast<long long>(s->batch) * s->num_groups * nb;
    pa::rank_kernel<<<static_cast<unsigned>(grid), 256, smem, st>>>(scores, rank, nb, causal_of(s) ? 1 : 0);
    PA_CUDA(cudaGetLastError());
    return PA_OK;
}

pa_status launch_budget(const pa_shape *s, const pa_budget *bu, const int32_t *rank, const float *mass, int32_t *cnt,
                        int32_t *budget, cudaStream_t st) {
    Trace tr_("pa.budget");
    pa::BudgetParams p;
    p.B = s->batch; p.H = s->num_q_heads; p.G = s->num_groups; p.nb = s->seqlen / kBlk;
    p.mode = bu->mode; p.gamma = bu->gamma; p.frac_permille = bu->frac_permille;
    p.causal = causal_of(s) ? 1 : 0;
    p.rank = rank; p.mass = mass; p.cnt = cnt; p.budget = budget;
    pa::budget_kernel<<<s->batch * s->num_q_heads, 1024, 0, st>>>(p);
    PA_CUDA(cudaGetLastError());
    return PA_OK;
}

template <int D, int S>
pa_status launch_xattn_gemm_t(const CUtensorMap &mq, const CUtensorMap &mk, const pa::XattnParams &p,
                              cudaStream_t st) {
    auto kern = pa::xattn_gemm_kernel<D, S>;
    const int smem = pa::XattnSmem<D, S>::BYTES;
    PA_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    const long long grid = std::min<long long>(p.num_units, num_sms());
    if (grid <= 0) return PA_OK;
    kern<<<static_cast<unsigned>(grid), 192, smem, st>>>(mq, mk, p);
    PA_CUDA(cudaGetLastError());
    return PA_OK;
}

template <int D>
pa_status launch_xattn_gemm_d(int S, const CUtensorMap &mq, const CUtensorMap &mk, const pa::XattnParams &p,
                              cudaStream_t st) {
    if (S == 4) return launch_xattn_gemm_t<D, 4>(mq, mk, p, st);
    if (S == 8) return launch_xattn_gemm_t<D, 8>(mq, mk, p, st);
    return launch_xattn_gemm_t<D, 16>(mq, mk, p, st);
}

pa_status launch_xattn(const pa_shape *s, int S, float tau, const void *q, pa_strides qs, const void *k,
                       pa_strides ks, int32_t *rank, int32_t *cnt, float *mass, void *ws, cudaStream_t st) {
    Trace tr_("pa.xattn_mask");
    const int B = s->batch, H = s->num_q_heads, Hkv = s->num_kv_heads, N = s->seqlen, d = s->head_dim;
    const int nb = N / kBlk, rows = N / S;
    CUtensorMap mq, mk;
    pa_status r = map_bnhd_split(&mq, q, B, N, H, d, S, qs, 128, "q");
    if (r) return r;
    if ((r = map_bnhd_split(&mk, k, B, N, Hkv, d, S, ks, 256, "k"))) return r;
    const XWsLayout w = xattn_ws_layout(s, S);
    uint8_t *base = static_cast<uint8_t *>(ws);
    pa::XattnParams p{};
    p.B = B; p.H = H; p.Hkv = Hkv; p.nb = nb;
    p.rows = rows;
    p.nchunk = (rows + 127) / 128;
    const int mtiles = (rows + 127) / 128;
    p.causal = causal_of(s) ? 1 : 0;
    long long per = 0;
    if (p.causal) {
        for (int mt = 0; mt < mtiles; ++mt) per += mt / 2 + 1;
    } else {
        per = static_cast<long long>(mtiles) * ((rows + 255) / 256);
    }
    p.units_per_bh = per;
    p.num_units = per * B * H;
    p.c2 = static_cast<float>(1.4426950408889634 / (std::sqrt(static_cast<double>(d)) * S));
    p.part_s = reinterpret_cast<float *>(base + w.part_s);
    p.part_m = reinterpret_cast<float *>(base + w.part_m);
    p.timeout_ns = wait_timeout_ns();
    r = d == 128 ? launch_xattn_gemm_d<128>(S, mq, mk, p, st) : launch_xattn_gemm_d<64>(S, mq, mk, p, st);
    if (r) return r;
    pa::XselParams sp{};
    sp.B = B; sp.H = H; sp.nb = nb; sp.rows = rows; sp.nchunk = p.nchunk;
    sp.causal = p.causal;
    sp.tau = tau;
    sp.part_s = p.part_s;
    sp.part_m = p.part_m;
    sp.mass = mass;
    sp.rank = rank;
    sp.cnt = cnt;
    int P = 256;  // the selection sorts at least 256 keys
    while (P < nb) P <<= 1;
    auto sel = S == 4 ? pa::xattn_select_kernel<4> : S == 8 ? pa::xattn_select_kernel<8> : pa::xattn_select_kernel<16>;
    const int smem = P * 8 + static_cast<int>((pa::xsel_sort_temp_bytes(P) + 15) / 16 * 16);
    PA_CUDA(cudaFuncSetAttribute(sel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    const long long grid = static_cast<long long>(B) * H * nb;
    sel<<<static_cast<unsigned>(grid), 256, smem, st>>>(sp);
    PA_CUDA(cudaGetLastError());
    return PA_OK;
}

// Head units of every KV head: its q heads h with h * Hkv / H == kv share one
// K/V stream.  Without the block skip ceil(heads / 2) units per query block: the
// kernel's CTAs of two adjacent query blocks pair the heads by row count per
// query block (a head left over at both forms one unit of two query blocks) or
// take one head at both query blocks each; with the skip one head per unit
// (its CTA takes two query blocks).  Returns the largest count.
int build_units(const pa_shape *s, int16_t *kv_units, bool one_head_per_unit) {
    const int H = s->num_q_heads, Hkv = s->num_kv_heads;
    int most = 0;
    for (int kv = 0; kv < Hkv; ++kv) {
        const long long first = (static_cast<long long>(kv) * H + Hkv - 1) / Hkv;
        const long long next = (static_cast<long long>(kv + 1) * H + Hkv - 1) / Hkv;
        const int units = static_cast<int>(one_head_per_unit ? next - first : (next - first + 1) / 2);
        kv_units[kv] = static_cast<int16_t>(units);
        most = std::max(most, units);
    }
    return most;
}

template <int D, bool SKIP>
pa_status launch_attn_t(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv, const pa::AttnParams &p,
                        cudaStream_t st) {
    auto kern = pa::attn_kernel<D, SKIP>;
    const int smem = pa::AttnSmem<D>::BYTES;
    PA_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    // The kernel's warpgroups re-split the registers it is launched with; the
    // split only adds up if every thread starts with kRegsLaunch registers.
    cudaFuncAttributes fa;
    PA_CUDA(cudaFuncGetAttributes(&fa, kern));
    if (fa.numRegs != pa::kRegsLaunch)
        return fail(PA_ERR_CUDA, "attn_kernel built with %d registers per thread, expected %d", fa.numRegs,
                    pa::kRegsLaunch);
    const long long grid = static_cast<long long>(p.units_per_kv) * p.Hkv * p.B * p.nb;
    kern<<<static_cast<unsigned>(grid), pa::kAttnThreads, smem, st>>>(mq, mk, mv, p);
    PA_CUDA(cudaGetLastError());
    return PA_OK;
}

// skip_threshold: BLASST's lambda in [0, 1] (0: no skipping, the plain kernel)
pa_status launch_attn(const pa_shape *s, const void *q, pa_strides qs, const void *k, pa_strides ks, const void *v,
                      pa_strides vs, const int32_t *rank, const int32_t *cnt, float scale, void *o, pa_strides os,
                      float *lse, float skip_threshold, uint8_t *skipped, cudaStream_t st) {
    Trace tr_("pa.block_sparse_attn");
    const int B = s->batch, H = s->num_q_heads, Hkv = s->num_kv_heads, N = s->seqlen, d = s->head_dim;
    CUtensorMap mq, mk, mv;
    pa_status r = map_bnhd(&mq, q, B, N, H, d, qs, "q");
    if (r) return r;
    if ((r = map_bnhd(&mk, k, B, N, Hkv, d, ks, "k"))) return r;
    if ((r = map_bnhd(&mv, v, B, N, Hkv, d, vs, "v"))) return r;
    pa::AttnParams p{};
    p.B = B; p.N = N; p.H = H; p.Hkv = Hkv; p.G = s->num_groups; p.nb = N / kBlk;
    const bool skip = skip_threshold > 0.0f;
    p.units_per_kv = build_units(s, p.kv_units, skip);
    p.rank = rank; p.cnt = cnt;
    p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
    p.o = static_cast<__nv_bfloat16 *>(o);
    p.osb = os.b; p.oss = os.s; p.osh = os.h;
    p.lse = lse;
    p.causal = causal_of(s) ? 1 : 0;
    p.timeout_ns = wait_timeout_ns();
    p.skip_log2 = skip ? static_cast<float>(std::log2(static_cast<double>(skip_threshold))) : -INFINITY;
    p.skipped = skip ? skipped : nullptr;
    if (skip)
        return d == 128 ? launch_attn_t<128, true>(mq, mk, mv, p, st) : launch_attn_t<64, true>(mq, mk, mv, p, st);
    return d == 128 ? launch_attn_t<128, false>(mq, mk, mv, p, st) : launch_attn_t<64, false>(mq, mk, mv, p, st);
}

pa_status check_mask(const pa_mask *m, const pa_budget *bu, bool need_rank_cnt) {
    if (!m) return fail(PA_ERR_INVALID_ARG, "mask is NULL");
    pa_status r;
    if (need_rank_cnt) {
        if ((r = check_ptr(m->rank, "mask.rank", 4))) return r;
        if ((r = check_ptr(m->cnt, "mask.cnt", 4))) return r;
    }
    if ((r = check_ptr(m->budget, "mask.budget", 4))) return r;
    if (bu->mode == PA_BUDGET_DYNAMIC && (r = check_ptr(m->mass, "mask.mass", 4))) return r;
    return PA_OK;
}

}  // namespace

// ===================================================================== C ABI
extern "C" {

int32_t pa_abi_version(void) { return PA_ABI_VERSION; }

const char *pa_last_error(void) { return g_last_error.c_str(); }

const char *pa_status_string(pa_status s) {
    switch (s) {
        case PA_OK: return "ok";
        case PA_ERR_INVALID_ARG: return "invalid argument";
        case PA_ERR_UNSUPPORTED: return "unsupported shape";
        case PA_ERR_WORKSPACE: return "workspace too small";
        case PA_ERR_CUDA: return "CUDA error";
        case PA_ERR_TIMEOUT: return "device wait timed out";
        case PA_ERR_DEVICE_BOUNDS: return "block index out of range on device";
        case PA_ERR_DEVICE_NONFINITE: return "non-finite block score or mass on device";
    }
    return "unknown status";
}

size_t pa_workspace_size(const pa_shape *shape, const pa_budget *budget) {
    if (check_shape(shape) || check_budget(budget)) return 0;
    return ws_layout(shape, budget).total;
}

pa_status pa_pool_heads_strided(const pa_shape *shape, int32_t score_stride, const void *q, pa_strides qs,
                                const void *k, pa_strides ks, void *q_proxy, void *k_proxy, pa_stream_t stream) {
    pa_status r;
    if ((r = check_shape(shape)) || (r = check_stride(score_stride))) return r;
    if ((r = check_tensor(q, qs, "q")) || (r = check_tensor(k, ks, "k"))) return r;
    if ((r = check_ptr(q_proxy, "q_proxy")) || (r = check_ptr(k_proxy, "k_proxy"))) return r;
    if ((r = launch_pool(shape, score_stride, q, qs, k, ks, q_proxy, k_proxy, reinterpret_cast<cudaStream_t>(stream))))
        return r;
    return ok();
}

pa_status pa_pool_heads(const pa_shape *shape, const void *q, pa_strides qs, const void *k, pa_strides ks,
                        void *q_proxy, void *k_proxy, pa_stream_t stream) {
    return pa_pool_heads_strided(shape, 1, q, qs, k, ks, q_proxy, k_proxy, stream);
}

pa_status pa_block_scores_strided(const pa_shape *shape, int32_t score_stride, const void *q_proxy,
                                  const void *k_proxy, float *scores, pa_stream_t stream) {
    pa_status r;
    if ((r = check_shape(shape)) || (r = check_stride(score_stride))) return r;
    if ((r = check_ptr(q_proxy, "q_proxy")) || (r = check_ptr(k_proxy, "k_proxy"))) return r;
    if ((r = check_ptr(scores, "scores", 4))) return r;
    if ((r = launch_scores(shape, score_stride, q_proxy, k_proxy, scores, reinterpret_cast<cudaStream_t>(stream))))
        return r;
    return ok();
}

pa_status pa_block_scores(const pa_shape *shape, const void *q_proxy, const void *k_proxy, float *scores,
                          pa_stream_t stream) {
    return pa_block_scores_strided(shape, 1, q_proxy, k_proxy, scores, stream);
}

pa_status pa_build_mask(const pa_shape *shape, const pa_budget *budget, const float *scores, const void *q,
                        pa_strides qs, const void *k, pa_strides ks, const pa_mask *out, void *ws, size_t ws_bytes,
                        pa_stream_t stream) {
    pa_status r;
    if ((r = check_shape(shape)) || (r = check_budget(budget))) return r;
    if ((r = check_ptr(scores, "scores", 4))) return r;
    if ((r = check_mask(out, budget, true))) return r;
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (budget->mode == PA_BUDGET_DYNAMIC) {
        if ((r = check_tensor(q, qs, "q")) || (r = check_tensor(k, ks, "k"))) return r;
        const size_t need = mask_ws_bytes(shape, budget);
        if (!ws || ws_bytes < need)
            return fail(PA_ERR_WORKSPACE, "workspace of %zu bytes is smaller than the %zu needed", ws_bytes, need);
        if ((r = check_ptr(ws, "workspace", 256))) return r;
        if ((r = launch_mass(shape, q, qs, k, ks, static_cast<float2 *>(ws), out->mass, st))) return r;
    }
    if ((r = launch_rank(shape, scores, out->rank, st))) return r;
    if ((r = launch_budget(shape, budget, out->rank, out->mass, out->cnt, out->budget, st))) return r;
    return ok();
}

pa_status pa_block_sparse_attn_skip(const pa_shape *shape, const void *q, pa_strides qs, const void *k,
                                    pa_strides ks, const void *v, pa_strides vs, const int32_t *rank,
                                    const int32_t *cnt, float softmax_scale, float skip_threshold, void *o,
                                    pa_strides os, float *lse, uint8_t *skipped, pa_stream_t stream) {
    pa_status r;
    if ((r = check_shape(shape)) || (r = check_skip(skip_threshold))) return r;
    if ((r = check_tensor(q, qs, "q")) || (r = check_tensor(k, ks, "k")) || (r = check_tensor(v, vs, "v")) ||
        (r = check_tensor(o, os, "o")))
        return r;
    if ((r = check_ptr(rank, "rank", 4)) || (r = check_ptr(cnt, "cnt", 4))) return r;
    if (lse && (r = check_ptr(lse, "lse", 4))) return r;
    if (!(softmax_scale > 0.0f) || !std::isfinite(softmax_scale))
        return fail(PA_ERR_INVALID_ARG, "softmax_scale must be positive and finite");
    if ((r = launch_attn(shape, q, qs, k, ks, v, vs, rank, cnt, softmax_scale, o, os, lse, skip_threshold, skipped,
                         reinterpret_cast<cudaStream_t>(stream))))
        return r;
    return ok();
}

pa_status pa_block_sparse_attn(const pa_shape *shape, const void *q, pa_strides qs, const void *k, pa_strides ks,
                               const void *v, pa_strides vs, const int32_t *rank, const int32_t *cnt,
                               float softmax_scale, void *o, pa_strides os, float *lse, pa_stream_t stream) {
    pa_status r;
    if ((r = check_shape(shape))) return r;
    if ((r = check_tensor(q, qs, "q")) || (r = check_tensor(k, ks, "k")) || (r = check_tensor(v, vs, "v")) ||
        (r = check_tensor(o, os, "o")))
        return r;
    if ((r = check_ptr(rank, "rank", 4)) || (r = check_ptr(cnt, "cnt", 4))) return r;
    if (lse && (r = check_ptr(lse, "lse", 4))) return r;
    if (!(softmax_scale > 0.0f) || !std::isfinite(softmax_scale))
        return fail(PA_ERR_INVALID_ARG, "softmax_scale must be positive and finite");
    if ((r = launch_attn(shape, q, qs, k, ks, v, vs, rank, cnt, softmax_scale, o, os, lse, 0.0f, nullptr,
                         reinterpret_cast<cudaStream_t>(stream))))
        return r;
    return ok();
}

}  // extern "C"

namespace {

// The launches of pa_prefill for one already-validated problem.
pa_status run_prefill(const pa_shape *shape, const pa_budget *budget, const void *q, pa_strides qs, const void *k,
                      pa_strides ks, const void *v, pa_strides vs, void *o, pa_strides os, const pa_mask *mask_out,
                      void *ws, cudaStream_t st) {
    pa_status r;
    const WsLayout w = ws_layout(shape, budget);
    uint8_t *base = static_cast<uint8_t *>(ws);
    void *qp = base + w.qp;
    void *kp = base + w.kp;
    float *scores = reinterpret_cast<float *>(base + w.scores);
    const int stride = stride_of(budget);
    if ((r = launch_pool(shape, stride, q, qs, k, ks, qp, kp, st))) return r;
    if ((r = launch_scores(shape, stride, qp, kp, scores, st))) return r;
    if (budget->mode == PA_BUDGET_DYNAMIC &&
        (r = launch_mass(shape, q, qs, k, ks, reinterpret_cast<float2 *>(base + w.partial), mask_out->mass, st)))
        return r;
    if ((r = launch_rank(shape, scores, mask_out->rank, st))) return r;
    if ((r = launch_budget(shape, budget, mask_out->rank, mask_out->mass, mask_out->cnt, mask_out->budget, st)))
        return r;
    const float scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(shape->head_dim)));
    if ((r = launch_attn(shape, q, qs, k, ks, v, vs, mask_out->rank, mask_out->cnt, scale, o, os, nullptr,
                         budget->skip_threshold, nullptr, st)))
        return r;
    return PA_OK;
}

// Validates a packed variable-length batch; fills the longest sequence.
pa_status check_varlen(const pa_shape *shape, int32_t num_seqs, const int32_t *cu, int32_t *max_len) {
    pa_status r;
    if ((r = check_shape(shape))) return r;
    if (shape->batch != 1) return fail(PA_ERR_INVALID_ARG, "a packed batch needs shape->batch = 1 (got %d)", shape->batch);
    if (num_seqs < 1) return fail(PA_ERR_INVALID_ARG, "num_seqs must be >= 1 (got %d)", num_seqs);
    if (!cu) return fail(PA_ERR_INVALID_ARG, "cu_seqlens is NULL");
    if (cu[0] != 0) return fail(PA_ERR_INVALID_ARG, "cu_seqlens[0] must be 0 (got %d)", cu[0]);
    int32_t mx = 0;
    for (int s = 0; s < num_seqs; ++s) {
        const int64_t len = static_cast<int64_t>(cu[s + 1]) - cu[s];
        if (len <= 0 || len % kBlk)
            return fail(PA_ERR_UNSUPPORTED, "sequence %d has %lld tokens: lengths must be positive multiples of 128", s,
                        static_cast<long long>(len));
        if (len / kBlk > kMaxNb)
            return fail(PA_ERR_UNSUPPORTED, "sequence %d has %lld tokens, more than %d", s, static_cast<long long>(len),
                        kMaxNb * kBlk);
        mx = std::max<int32_t>(mx, static_cast<int32_t>(len));
    }
    if (cu[num_seqs] != shape->seqlen)
        return fail(PA_ERR_INVALID_ARG, "cu_seqlens[num_seqs] = %d differs from shape->seqlen = %d", cu[num_seqs],
                    shape->seqlen);
    *max_len = mx;
    return PA_OK;
}

}  // namespace

extern "C" {

pa_status pa_prefill(const pa_shape *shape, const pa_budget *budget, const void *q, pa_strides qs, const void *k,
                     pa_strides ks, const void *v, pa_strides vs, void *o, pa_strides os, const pa_mask *mask_out,
                     void *ws, size_t ws_bytes, pa_stream_t stream) {
    pa_status r;
    if ((r = check_shape(shape)) || (r = check_budget(budget))) return r;
    if ((r = check_tensor(q, qs, "q")) || (r = check_tensor(k, ks, "k")) || (r = check_tensor(v, vs, "v")) ||
        (r = check_tensor(o, os, "o")))
        return r;
    if ((r = check_mask(mask_out, budget, true))) return r;
    const WsLayout w = ws_layout(shape, budget);
    if (!ws || ws_bytes < w.total)
        return fail(PA_ERR_WORKSPACE, "workspace of %zu bytes is smaller than the %zu needed", ws_bytes, w.total);
    if ((r = check_ptr(ws, "workspace", 256))) return r;
    Trace tr_("pa.prefill");
    if ((r = run_prefill(shape, budget, q, qs, k, ks, v, vs, o, os, mask_out, ws,
                         reinterpret_cast<cudaStream_t>(stream))))
        return r;
    return ok();
}

size_t pa_workspace_size_varlen(const pa_shape *shape, const pa_budget *budget, int32_t num_seqs,
                                const int32_t *cu_seqlens) {
    int32_t mx = 0;
    if (check_varlen(shape, num_seqs, cu_seqlens, &mx) || check_budget(budget)) return 0;
    pa_shape one = *shape;
    one.seqlen = mx;
    return ws_layout(&one, budget).total;
}

pa_status pa_prefill_varlen(const pa_shape *shape, const pa_budget *budget, int32_t num_seqs,
                            const int32_t *cu_seqlens, const void *q, pa_strides qs, const void *k, pa_strides ks,
                            const void *v, pa_strides vs, void *o, pa_strides os, const pa_mask *mask_out, void *ws,
                            size_t ws_bytes, pa_stream_t stream) {
    pa_status r;
    int32_t mx = 0;
    if ((r = check_varlen(shape, num_seqs, cu_seqlens, &mx)) || (r = check_budget(budget))) return r;
    if ((r = check_tensor(q, qs, "q")) || (r = check_tensor(k, ks, "k")) || (r = check_tensor(v, vs, "v")) ||
        (r = check_tensor(o, os, "o")))
        return r;
    if ((r = check_mask(mask_out, budget, true))) return r;
    pa_shape longest = *shape;
    longest.seqlen = mx;
    const size_t need = ws_layout(&longest, budget).total;
    if (!ws || ws_bytes < need)
        return fail(PA_ERR_WORKSPACE, "workspace of %zu bytes is smaller than the %zu needed", ws_bytes, need);
    if ((r = check_ptr(ws, "workspace", 256))) return r;
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int G = shape->num_groups, H = shape->num_q_heads;
    Trace tr_("pa.prefill_varlen");
    int64_t rows_off = 0, blk_off = 0;  // sums of T_s and nb_s over the sequences before
    for (int s = 0; s < num_seqs; ++s) {
        pa_shape one = *shape;
        one.seqlen = cu_seqlens[s + 1] - cu_seqlens[s];
        const int64_t nb = one.seqlen / kBlk;
        const int64_t T = static_cast<int64_t>(rows_total(&one));
        const int64_t t0 = cu_seqlens[s];
        pa_mask m;
        m.rank = mask_out->rank + G * rows_off;
        m.cnt = mask_out->cnt + H * blk_off;
        m.budget = mask_out->budget + static_cast<int64_t>(H) * s;
        m.mass = mask_out->mass ? mask_out->mass + H * blk_off : nullptr;
        const auto *qb = static_cast<const __nv_bfloat16 *>(q) + t0 * qs.s;
        const auto *kb = static_cast<const __nv_bfloat16 *>(k) + t0 * ks.s;
        const auto *vb = static_cast<const __nv_bfloat16 *>(v) + t0 * vs.s;
        auto *ob = static_cast<__nv_bfloat16 *>(o) + t0 * os.s;
        if ((r = run_prefill(&one, budget, qb, qs, kb, ks, vb, vs, ob, os, &m, ws, st))) return r;
        rows_off += T;
        blk_off += nb;
    }
    return ok();
}

pa_status pa_get_device_status(pa_stream_t stream, int clear) {
    PA_CUDA(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)));
    unsigned v = 0;
    PA_CUDA(cudaMemcpyFromSymbol(&v, pa::g_status, sizeof v));
    if (clear) {
        const unsigned zero = 0;
        PA_CUDA(cudaMemcpyToSymbol(pa::g_status, &zero, sizeof zero));
    }
    g_last_error.clear();
    return static_cast<pa_status>(v);
}

}  // extern "C"

// ================================================================ XAttention
extern "C" {

size_t pa_xattn_workspace_size(const pa_shape *shape, int32_t stride) {
    if (check_shape(shape) || check_xstride(stride)) return 0;
    return xattn_ws_layout(shape, stride).total;
}

pa_status pa_xattn_mask(const pa_shape *shape, int32_t stride, float tau, const void *q, pa_strides qs,
                        const void *k, pa_strides ks, int32_t *rank, int32_t *cnt, float *mass, void *ws,
                        size_t ws_bytes, pa_stream_t stream) {
    pa_status r;
    if ((r = check_shape(shape)) || (r = check_xstride(stride))) return r;
    if (!(tau > 0.0f && tau <= 1.0f))
        return fail(PA_ERR_INVALID_ARG, "tau must be in (0, 1] (got %g)", static_cast<double>(tau));
    if ((r = check_tensor(q, qs, "q")) || (r = check_tensor(k, ks, "k"))) return r;
    if ((r = check_ptr(rank, "rank", 4)) || (r = check_ptr(cnt, "cnt", 4))) return r;
    if (mass && (r = check_ptr(mass, "mass", 4))) return r;
    const size_t need = xattn_ws_layout(shape, stride).total;
    if (!ws || ws_bytes < need)
        return fail(PA_ERR_WORKSPACE, "workspace of %zu bytes is smaller than the %zu needed", ws_bytes, need);
    if ((r = check_ptr(ws, "workspace", 256))) return r;
    if ((r = launch_xattn(shape, stride, tau, q, qs, k, ks, rank, cnt, mass, ws,
                          reinterpret_cast<cudaStream_t>(stream))))
        return r;
    return ok();
}

}  // extern "C"

// ======================================================== no-allocation mask
// pa_build_mask_noalloc keeps its scratch (the per-tile softmax statistics of
// the last query block) in this file-scope device array instead of a
// caller-provided workspace.  Every GPU that loads the library holds these
// bytes until the process exits; every call on a device shares them.
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;

// Device address of g_noalloc_scratch on the current device.  The host-side
// name of the array is only a stand-in, so the address is looked up once per
// device with cudaGetSymbolAddress (with that device current) and cached.
pa_status noalloc_scratch(void **out) {
    static std::mutex mu;
    static void *addr[kMaxDevices] = {};
    int dev = 0;
    PA_CUDA(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) return fail(PA_ERR_UNSUPPORTED, "device ordinal %d >= %d", dev, kMaxDevices);
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p)
            return fail(PA_ERR_CUDA, "cudaGetSymbolAddress(scratch) failed: %s", cudaGetErrorString(e));
        addr[dev] = p;
    }
    *out = addr[dev];
    return PA_OK;
}

}  // namespace

extern "C" PA_API pa_status pa_build_mask_noalloc(const pa_shape *shape, const pa_budget *budget,
                                                  const float *scores, const void *q, pa_strides qs,
                                                  const void *k, pa_strides ks, const pa_mask *out,
                                                  pa_stream_t stream) {
    pa_status r;
    if ((r = check_shape(shape)) || (r = check_budget(budget))) return r;
    if ((r = check_ptr(scores, "scores", 4))) return r;
    if ((r = check_mask(out, budget, true))) return r;
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (budget->mode == PA_BUDGET_DYNAMIC) {
        if ((r = check_tensor(q, qs, "q")) || (r = check_tensor(k, ks, "k"))) return r;
        const size_t need = mask_ws_bytes(shape, budget);
        if (need > kNoAllocScratchBytes)
            return fail(PA_ERR_UNSUPPORTED,
                        "pa_build_mask_noalloc: this shape needs %zu bytes of scratch but the built-in scratch holds "
                        "%zu (batch * q_heads * seqlen/128 must be <= %zu); use pa_build_mask with a workspace",
                        need, kNoAllocScratchBytes, kNoAllocScratchBytes / (128 * sizeof(float2)));
        void *scratch = nullptr;
        if ((r = noalloc_scratch(&scratch))) return r;
        // every byte of the scratch that is read is written first in this call: nothing to clear
        if ((r = launch_mass(shape, q, qs, k, ks, static_cast<float2 *>(scratch), out->mass, st))) return r;
    }
    if ((r = launch_rank(shape, scores, out->rank, st))) return r;
    if ((r = launch_budget(shape, budget, out->rank, out->mass, out->cnt, out->budget, st))) return r;
    return ok();
}

// ========================================================== wait self-test
namespace pa {
// One warp waits on an mbarrier that nothing ever completes; the bounded wait
// gives up after timeout_ns, records PA_ERR_TIMEOUT and the kernel returns.
__global__ void selftest_wait_timeout_kernel(uint64_t timeout_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    const WaitCtl wc{&abort_flag, timeout_ns};
    (void)warp_wait(&bar, 0, wc);
}
}  // namespace pa

extern "C" PA_API pa_status pa_selftest_wait_timeout(uint32_t timeout_us, pa_stream_t stream) {
    if (timeout_us < 1 || timeout_us > 1000000)
        return fail(PA_ERR_INVALID_ARG, "timeout_us must be in 1..1000000 (got %u)", timeout_us);
    pa::selftest_wait_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        static_cast<uint64_t>(timeout_us) * 1000u);
    PA_CUDA(cudaGetLastError());
    return ok();
}
