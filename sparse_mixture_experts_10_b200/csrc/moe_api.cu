// moe_api.cu -- host side of the C ABI declared in include/moe.h.
//
// Validates arguments on the host, carves the caller's workspace, encodes the
// TMA tensor maps and enqueues the stages of the layer on the caller's stream:
//   route    fused router (N <= 32) or router GEMM + top-k kernel
//   scan     counting-sort scan over chunk histograms
//   permute  stable scatter of token rows into expert segments
//   up       grouped GEMM + GELU / SwiGLU epilogue  -> h
//   down     grouped GEMM + gate-weight epilogue    -> z (one row per slot)
//   combine  y[t] = sum_j z[t, j] in slot order
//   stats    optional per-batch statistics
// No call synchronises the stream or allocates memory (moe_get_device_status
// excepted, which synchronises the device).
#include "../../include/moe.h"
#include "moe_backward.cuh"
#include "moe_common.cuh"
#include "moe_decode_fused.cuh"
#include "moe_gemm_simt.cuh"
#include "moe_gemm_decode.cuh"
#include "moe_gemm_tc.cuh"
#include "moe_route.cuh"
#include "moe_router_tc.cuh"

#include <algorithm>
#include <cmath>
#include <atomic>
#include <mutex>

using namespace moe;

namespace {

std::atomic<int64_t> g_launches{0};
constexpr uint64_t kTimeoutNs = 1000000000ull;  // bounded waits give up after 1 s
constexpr int kMaxDevices = 64;
constexpr size_t kSmallRouterSmemMax = 200 * 1024;
constexpr int64_t kRerouteSmem = 160 * 1024;   // reroute_kernel: loads + two staged batches
constexpr int64_t kRowdotMaxT = 2048;  // below this the chunked router has too few blocks
constexpr int64_t kDecodeMaxT = 64;    // up to this many tokens the expert GEMMs stream weights (decode path)
constexpr int kDecodeMaxGrid = 256;    // decode GEMMs: most persistent CTAs (stream-K buffers are sized for it)

struct DeviceInfo {
    int sms = 0;
    int pair_clusters = 0;   // 2-CTA clusters of the pair GEMM that can be resident at once
    bool attrs = false;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }
int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

struct Plan {
    int64_t T;
    int D, H, N, K, act, dtype, has_bias, es;
    bool small_router;   // chunked fused router (W_g staged in shared memory)
    bool rowdot_router;  // one block per token (few tokens, N <= 32)
    int np;       // padded expert count of the fused router (8, 16, 32)
    int vpl;      // values per lane of the top-k kernel
    int n_chunks;
    int aux_blocks;
    int64_t rows_cap;
    bool tc_router;    // bf16, N <= 256: router, top-k, statistics and scan in one tensor-core kernel
    bool few_router;   // bf16, T <= 64, N <= 32: one block per token instead
    bool simt_router;  // bf16, N <= 32, more tokens: SIMT router with W_g in shared memory
    int chunk_tokens;  // tokens per dispatch chunk (32; the tensor-core router's 128-token tile; 1 token)
    int rnp, rkm;      // tensor-core router: padded expert count, top-k list length
    bool decode;  // few tokens: weight-streaming expert GEMMs
    int nt;       // decode: padded token tile (16, 32 or 64)
    int route_splits;  // few-token router: W_g slabs per token
    int dec_cap;       // decode GEMMs: CTAs the stream-K partials and tickets are sized for
    int n_shared;      // 1: a shared expert (dense FFN over every token) is added after the routed sum
    int capacity;      // assignments each expert accepts (rows served in order)
    bool reroute;      // refused assignments go to the next candidate (reroute_kernel) instead of being dropped
    int rr_batch;      // reroute_kernel: tokens per batch (selections staged, two buffers)
    int rr_vbatch;     // reroute_kernel: tokens whose selection values are staged at a time
    bool fused_decode; // few tokens, N <= 32, no shared expert: the whole layer in one cooperative kernel
    bool given_routing;
    int slab_rows, n_slabs;   // fused decode: W_g rows per routing slab, slabs
    // Counters region (zeroed on every call), 32-bit words: [0] router ticket,
    // [1] statistics ticket, [2] number of live experts, [64, 128) per-token
    // tickets of the few-token router; from byte 512 the stream-K tile tickets
    // of the decode up- and down-projections and of the shared expert's two
    // decode GEMMs (dec_cap each); then the routers' per-expert probability
    // and gate-weight sums (u64, N each).  Words 4, 8 and 9 count
    // the fused decode kernel's grid barrier arrivals, word 7 the cooperative
    // SIMT router's, word 10 is the scan's ticket after a reroute.
    size_t counters_bytes;
    size_t stat_sums;  // offset inside the counters region of the routers' fixed-point sums [2][N] (u64)
    size_t counters, logits, idx, w, counts, offsets, row_offsets, live, chunk_counts, chunk_base,
        perm_slot, slot_row, x_perm, h, z, wgt, aux_p, aux_i, aux_c, route_part, dec_part, shared_tbl, h_s, s_out,
        fd_slab, fd_tokp, total;
};

// given_routing: the (token, slot) -> expert assignments and weights are inputs
// (expert parallelism's received rows), so no router runs and the dispatch
// tables come from chunk histograms of the given indices.
int make_plan(const moe_config *c, int64_t T, Plan *p, bool given_routing = false) {
    if (!c || !p) return MOE_ERR_INVALID_ARG;
    const int64_t D = c->DModel, H = c->DHidden, N = c->NExperts, K = c->TopK;
    if (D <= 0 || H <= 0 || N <= 0 || K <= 0 || T < 0) return MOE_ERR_INVALID_ARG;
    if (N > 1024 || K > N || K > 32) return MOE_ERR_INVALID_ARG;
    if (c->act != MOE_ACT_GELU && c->act != MOE_ACT_SWIGLU) return MOE_ERR_INVALID_ARG;
    if (c->dtype != MOE_F32 && c->dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
    if (c->has_bias && c->act != MOE_ACT_GELU) return MOE_ERR_UNSUPPORTED;
    if (c->n_shared != 0 && c->n_shared != 1) return MOE_ERR_INVALID_ARG;
    if (!(c->capacity_factor >= 0.0f) || c->capacity_factor > 1.0e6f) return MOE_ERR_INVALID_ARG;   // NaN too
    if (c->overflow != MOE_OVERFLOW_DROP && c->overflow != MOE_OVERFLOW_REROUTE) return MOE_ERR_INVALID_ARG;
    const int es = c->dtype == MOE_F32 ? 4 : 2;
    const int vec = 16 / es;
    if (D % vec || H % vec) return MOE_ERR_INVALID_ARG;
    // index arithmetic inside kernels uses 32-bit rows and slot ids
    if (T * K + N * (int64_t)kRowAlign >= (int64_t)1 << 31) return MOE_ERR_UNSUPPORTED;
    if (N * 2 * H >= (int64_t)1 << 31 || N * D >= (int64_t)1 << 31) return MOE_ERR_UNSUPPORTED;

    p->T = T;
    p->D = (int)D; p->H = (int)H; p->N = (int)N; p->K = (int)K;
    p->act = c->act; p->dtype = c->dtype; p->has_bias = c->has_bias ? 1 : 0; p->es = es;
    p->n_shared = c->n_shared;
    // C = ceil(cf T K / N) in double; no limit without a capacity factor
    if (c->capacity_factor > 0.0f) {
        const double cap = std::ceil((double)c->capacity_factor * (double)T * (double)K / (double)N);
        p->capacity = cap >= (double)INT32_MAX ? INT32_MAX : (int)cap;
    } else {
        p->capacity = INT32_MAX;
    }
    p->reroute = c->capacity_factor > 0.0f && c->overflow == MOE_OVERFLOW_REROUTE;
    p->rr_batch = (int)std::min<int64_t>(1024, std::max<int64_t>(1, (kRerouteSmem / 4 - N * 8 - 32) / (2 * K * 4)));
    p->rr_vbatch = (int)std::max<int64_t>(1, std::min<int64_t>(p->rr_batch,
        (kRerouteSmem - N * 8 - 32 - (int64_t)2 * p->rr_batch * K * 4) / (N * 4)));
    p->np = N <= 8 ? 8 : N <= 16 ? 16 : 32;
    const bool fits = N <= 32 && (size_t)p->np * D * es + 256 <= kSmallRouterSmemMax;
    p->rowdot_router = N <= 32 && (T < kRowdotMaxT || !fits);
    p->small_router = fits && !p->rowdot_router;
    const int need = (int)cdiv(N, 32);
    p->vpl = need <= 1 ? 1 : need <= 2 ? 2 : need <= 4 ? 4 : need <= 8 ? 8 : need <= 16 ? 16 : 32;
    p->decode = c->dtype == MOE_BF16 && T <= kDecodeMaxT;
    p->nt = T <= 16 ? 16 : T <= 32 ? 32 : 64;
    p->tc_router = c->dtype == MOE_BF16 && N <= 256;
    p->few_router = p->tc_router && T <= kDecodeMaxT && N <= 32;
    const size_t simt_bytes = p->np == 8    ? rtc::SimtShape<8>::smem_bytes((int)D)
                              : p->np == 16 ? rtc::SimtShape<16>::smem_bytes((int)D)
                                            : rtc::SimtShape<32>::smem_bytes((int)D);
    p->simt_router = p->tc_router && !p->few_router && N <= 32 && simt_bytes <= kSmallRouterSmemMax;
    p->given_routing = given_routing;
    if (given_routing) p->tc_router = p->few_router = p->simt_router = p->rowdot_router = p->small_router = false;
    p->chunk_tokens = p->few_router ? 1 : p->simt_router ? rtc::kSimtChunk : p->tc_router ? rtc::BM : kChunk;
    p->rnp = N <= 16 ? 16 : N <= 32 ? 32 : N <= 64 ? 64 : N <= 128 ? 128 : 256;
    p->rkm = K <= 8 ? 8 : 32;
    p->n_chunks = (int)cdiv(T, p->chunk_tokens);
    p->aux_blocks = (int)cdiv(T, kAuxTokens);
    p->rows_cap = cdiv(T * K + N * (kRowAlign - 1), kRowAlign) * kRowAlign;

    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align256(off + bytes);
        return o;
    };
    p->route_splits = p->few_router ? (int)std::min<int64_t>(rtc::kFewMaxSplits, std::max<int64_t>(1, cdiv(D, 256))) : 1;
    p->dec_cap = p->decode ? kDecodeMaxGrid : 0;
    p->stat_sums = (512 + (size_t)4 * p->dec_cap * 4 + 7) / 8 * 8;
    p->counters_bytes = align256(p->stat_sums + (size_t)2 * N * 8);
    p->counters = take(p->counters_bytes);
    p->logits = take((size_t)T * N * 4);
    p->idx = take((size_t)T * K * 4);
    p->w = take((size_t)T * K * 4);
    p->counts = take((size_t)N * 4);
    p->offsets = take((size_t)(N + 1) * 4);
    p->row_offsets = take((size_t)(N + 1) * 4);
    p->live = take((size_t)N * 4);
    const int64_t max_chunks = std::max<int64_t>(p->n_chunks, 1);
    p->chunk_counts = take((size_t)max_chunks * N * 4);
    p->chunk_base = take((size_t)max_chunks * N * 4);
    p->perm_slot = take((size_t)p->rows_cap * 4);
    p->slot_row = take((size_t)T * K * 4);
    p->x_perm = take((size_t)p->rows_cap * D * es);
    p->h = take((size_t)p->rows_cap * H * es);
    // z rows: slot order (T*K rows) for decode and fp32 layers; the permuted
    // row order (rows_cap rows) for bf16 prefill layers, whose down projection
    // writes it with bulk tensor stores
    p->z = take((size_t)(p->dtype == MOE_BF16 && !p->decode ? p->rows_cap : T * K) * D * 4);
    p->wgt = take((N <= 32 && !(p->tc_router && !p->few_router && !p->simt_router)) ? 0 : (size_t)N * D * es);
    p->aux_p = take((size_t)p->aux_blocks * N * 4);
    p->aux_i = take((size_t)p->aux_blocks * N * 4);
    p->aux_c = take((size_t)p->aux_blocks * N * 4);
    p->route_part = take(p->few_router ? (size_t)T * p->route_splits * 32 * 4 : 0);
    p->dec_part = take(p->decode ? (size_t)p->dec_cap * 2 * dec::BM * p->nt * 4 : 0);
    // shared expert: its one-group dispatch table for the decode GEMMs (live = {0},
    // one live group, count T, first row 0), its hidden rows and its fp32 output
    p->shared_tbl = take(16);
    // fused decode: routing slabs of W_g rows (a multiple of 8 rows each, at most
    // 32 slabs) and each token's full softmax
    p->fused_decode = p->decode && N <= dfu::kMaxN && !p->n_shared && T <= dfu::kMaxT && !given_routing && !p->reroute;
    p->slab_rows = (int)(cdiv(cdiv(D, dfu::kMaxSlabs), 8) * 8);
    p->n_slabs = (int)cdiv(D, p->slab_rows);
    p->fd_slab = take(p->fused_decode ? (size_t)p->n_slabs * T * 32 * 4 : 0);
    p->fd_tokp = take(p->fused_decode ? (size_t)T * 32 * 4 : 0);
    p->h_s = take(p->n_shared ? (size_t)std::max<int64_t>(T, 1) * H * es : 0);
    p->s_out = take(p->n_shared ? (size_t)T * D * 4 : 0);
    p->total = off;
    return MOE_OK;
}

bool aligned16(const void *ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

#define MOE_TRY(expr)                  \
    do {                               \
        const int _rc = (expr);        \
        if (_rc != MOE_OK) return _rc; \
    } while (0)

// Lets a kernel use as much dynamic shared memory as the per-block limit leaves
// next to its static shared memory.
template <typename K>
int allow_smem(K *kernel) {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess) return MOE_ERR_CUDA;
    const int limit = 227 * 1024 - (int)fa.sharedSizeBytes;
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, limit) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

int device_info(DeviceInfo **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceInfo &d = g_dev[dev];
    if (d.sms == 0) {
        if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return MOE_ERR_CUDA;
    }
    if (!d.attrs) {
        MOE_TRY(allow_smem(reroute_kernel<1>));
        MOE_TRY(allow_smem(reroute_kernel<2>));
        MOE_TRY(allow_smem(reroute_kernel<4>));
        MOE_TRY(allow_smem(reroute_kernel<8>));
        MOE_TRY(allow_smem(reroute_kernel<16>));
        MOE_TRY(allow_smem(reroute_kernel<32>));
        MOE_TRY(allow_smem(tc::grouped_gemm_tc_kernel<256, tc::EPI_GELU>));
        MOE_TRY(allow_smem(tc::grouped_gemm_tc_kernel<256, tc::EPI_SWIGLU>));
        MOE_TRY(allow_smem(tc::grouped_gemm_tc_kernel<256, tc::EPI_SCATTER>));
        MOE_TRY(allow_smem(tc::grouped_gemm_tc_kernel<256, tc::EPI_LOGITS>));
        MOE_TRY(allow_smem(tc::grouped_gemm_tc2_kernel<tc::EPI_GELU>));
        MOE_TRY(allow_smem(tc::grouped_gemm_tc2_kernel<tc::EPI_SWIGLU>));
        MOE_TRY(allow_smem(tc::grouped_gemm_tc2_kernel<tc::EPI_SCATTER>));
        MOE_TRY(allow_smem(tc::grouped_gemm_tc2_kernel<tc::EPI_LOGITS>));
        MOE_TRY(allow_smem(tc::grouped_gemm_tc_kernel<128, tc::EPI_GELU>));
        MOE_TRY(allow_smem(tc::grouped_gemm_tc_kernel<128, tc::EPI_SWIGLU>));
        MOE_TRY(allow_smem(tc::grouped_gemm_tc_kernel<128, tc::EPI_SCATTER>));
        MOE_TRY(allow_smem(router_small_kernel<float, 8>));
        MOE_TRY(allow_smem(router_small_kernel<float, 16>));
        MOE_TRY(allow_smem(router_small_kernel<float, 32>));
        MOE_TRY(allow_smem(router_small_kernel<__nv_bfloat16, 8>));
        MOE_TRY(allow_smem(router_small_kernel<__nv_bfloat16, 16>));
        MOE_TRY(allow_smem(router_small_kernel<__nv_bfloat16, 32>));
        MOE_TRY(allow_smem(aux_partial_kernel));
        MOE_TRY(allow_smem(aux_partials_kernel));
#define MOE_FUSED_ATTR(NT)                                                  \
    MOE_TRY(allow_smem(dfu::decode_layer_kernel<NT, dec::EPI_SWIGLU>)); \
    MOE_TRY(allow_smem(dfu::decode_layer_kernel<NT, dec::EPI_GELU>))
        MOE_FUSED_ATTR(16);
        MOE_FUSED_ATTR(32);
        MOE_FUSED_ATTR(64);
#undef MOE_FUSED_ATTR
        MOE_TRY(allow_smem(rtc::router_simt_kernel<8, false>));
        MOE_TRY(allow_smem(rtc::router_simt_kernel<16, false>));
        MOE_TRY(allow_smem(rtc::router_simt_kernel<32, false>));
        MOE_TRY(allow_smem(rtc::router_simt_kernel<8, true>));
        MOE_TRY(allow_smem(rtc::router_simt_kernel<16, true>));
        MOE_TRY(allow_smem(rtc::router_simt_kernel<32, true>));
#define MOE_RTC_ATTR(NP)                                                                                     \
    MOE_TRY(allow_smem(rtc::router_tc_kernel<NP, 8>)); \
    MOE_TRY(allow_smem(rtc::router_tc_kernel<NP, 32>))
        MOE_RTC_ATTR(16);
        MOE_RTC_ATTR(32);
        MOE_RTC_ATTR(64);
        MOE_RTC_ATTR(128);
        MOE_RTC_ATTR(256);
#undef MOE_RTC_ATTR
#define MOE_DEC_ATTR(NT)                                                                                          \
    MOE_TRY(allow_smem(dec::decode_gemm_kernel<NT, dec::EPI_GELU>)); \
    MOE_TRY(allow_smem(dec::decode_gemm_kernel<NT, dec::EPI_SWIGLU>)); \
    MOE_TRY(allow_smem(dec::decode_gemm_kernel<NT, dec::EPI_SCATTER>))
        MOE_DEC_ATTR(16);
        MOE_DEC_ATTR(32);
        MOE_DEC_ATTR(64);
#undef MOE_DEC_ATTR
        // Clusters need both CTAs in one GPC, so fewer than sms / 2 pairs may fit
        // at once; the persistent pair GEMM is launched with no more than fit
        // (at the largest shared-memory size it uses).
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(2 * (d.sms / 2)));
        cfg.blockDim = dim3(tc::kThreads);
        cfg.dynamicSmemBytes = tc::Shape2::smem_bytes(1024);
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, (const void *)tc::grouped_gemm_tc2_kernel<tc::EPI_GELU>, &cfg) !=
            cudaSuccess)
            return MOE_ERR_CUDA;
        d.pair_clusters = n > 0 ? std::min(n, d.sms / 2) : d.sms / 2;
        d.attrs = true;
    }
    *out = &d;
    return MOE_OK;
}

int check_launch() {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// Launch with programmatic stream serialisation: the kernel may be launched
// while the previous kernel of the stream is still running; it calls
// pdl_enter() before its first global access, which waits for that kernel's
// completion.  Captured into a CUDA graph this is a programmatic edge.
template <typename... KArgs, typename... Args>
int launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// Zeroes `bytes` (a multiple of 16) at the 16-byte aligned p; with tbl, also
// writes the shared expert's one-group table {0, 1, T, 0} there.
int launch_zero(void *p, size_t bytes, int sms, cudaStream_t s, int *tbl = nullptr, int tbl_T = 0) {
    const int64_t n16 = (int64_t)(bytes / 16);
    if (n16 == 0 && !tbl) return MOE_OK;
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(cdiv(n16, 256), (int64_t)sms * 8));
    return launch_pdl(zero_kernel, dim3(grid), dim3(256), 0, s, static_cast<uint4 *>(p), n16, tbl, tbl_T);
}


// --------------------------------------------------------------- TMA tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    });
    return fn;
}

// 2-D bf16 matrix [rows, cols] row-major; box of box_rows x 64 columns, 128-byte swizzle.
int make_map(CUtensorMap *m, const void *base, int64_t rows, int64_t cols, int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return MOE_ERR_CUDA;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1u, 1u};
    const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

// 2-D bf16 matrix [rows, cols] row-major as the destination of the epilogue's
// bulk stores: boxes of 32 rows x 16 columns, no swizzle.
int make_store_map(CUtensorMap *m, void *base, int64_t rows, int64_t cols) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return MOE_ERR_CUDA;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {16u, 32u};
    const cuuint32_t estr[2] = {1u, 1u};
    const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

// 2-D fp32 matrix [rows, cols] row-major as the destination of the down
// projection's bulk stores: boxes of 32 rows x 8 columns, no swizzle.
int make_store_map_f32(CUtensorMap *m, void *base, int64_t rows, int64_t cols) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return MOE_ERR_CUDA;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 4};
    const cuuint32_t box[2] = {8u, 32u};
    const cuuint32_t estr[2] = {1u, 1u};
    const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

// O: destination map of bf16 outputs (EPI_GELU, EPI_SWIGLU); other epilogues
// store directly and get A in its place (unused).
template <int BN, int EPI>
int launch_tc(const CUtensorMap &A, const CUtensorMap &B, const CUtensorMap &O, const tc::Params &p,
              int64_t tiles_upper, int sms, cudaStream_t s) {
    const int grid = (int)std::min<int64_t>(std::max<int64_t>(tiles_upper, 1), sms);
    const size_t smem = tc::Shape<BN>::smem_bytes(p.num_groups);
    return launch_pdl(tc::grouped_gemm_tc_kernel<BN, EPI>, dim3(grid), dim3(tc::kThreads), smem, s, A, B, O, p);
}

// Pair (2-CTA cluster) version for 256-column tiles: 256-row units per cluster.
template <int EPI>
int launch_tc2(const CUtensorMap &A, const CUtensorMap &B, const CUtensorMap &O, const tc::Params &p,
               int64_t units_upper, int pair_clusters, cudaStream_t s) {
    const int64_t clusters = std::min<int64_t>(std::max<int64_t>(units_upper, 1), pair_clusters);
    const size_t smem = tc::Shape2::smem_bytes(p.num_groups);
    return launch_pdl(tc::grouped_gemm_tc2_kernel<EPI>, dim3((unsigned)(2 * clusters)), dim3(tc::kThreads), smem, s, A,
                      B, O, p);
}

template <int EPI>
int launch_simt(const simt::Params &p, int64_t rows, int n_blocks, cudaStream_t s) {
    const dim3 grid((unsigned)cdiv(std::max<int64_t>(rows, 1), simt::TM), (unsigned)std::max(n_blocks, 1));
    simt::grouped_gemm_simt_kernel<EPI><<<grid, 256, 0, s>>>(p);
    return check_launch();
}

struct Bufs {
    char *ws;
    const Plan *p;
    template <typename T>
    T *at(size_t off) const { return reinterpret_cast<T *>(ws + off); }
};

// ---------------------------------------------------------------- stages
// route: logits (always written to `logits`), top-k, chunk histograms.
template <int NP, int KM>
int launch_rtc(const CUtensorMap &mx, const CUtensorMap &mw, const rtc::Params &p, int grid, cudaStream_t s) {
    return launch_pdl(rtc::router_tc_kernel<NP, KM>, dim3(grid), dim3(rtc::kThreads), rtc::Shape<NP>::kSmem, s, mx, mw,
                      p);
}

// Tensor-core router: scores, top-k, statistics partials and (in the last CTA)
// the dispatch tables and the finished statistics.
// y_zero: the fp32 output to clear (SIMT router only; see stage_permute), else null.
int stage_route_tc(const Plan &P, const Bufs &b, const void *x, const moe_weights *w, float *logits, int *idx,
                   float *tw, int *counts_out, const moe_aux *aux, float *y_zero, cudaStream_t s) {
    const int T = (int)P.T, D = P.D, N = P.N;
    rtc::Params p{};
    p.T = T;
    p.D = D;
    p.N = N;
    p.K = P.K;
    p.np = P.rnp;
    p.bg = w->b_g;
    p.bsel = w->b_sel;
    p.logits = logits;
    p.topk_idx = idx;
    p.topk_w = tw;
    p.tile_counts = b.at<int>(P.chunk_counts);
    p.sum_p = reinterpret_cast<unsigned long long *>(b.ws + P.counters + P.stat_sums);
    p.sum_imp = p.sum_p + N;
    p.ticket = b.at<unsigned>(P.counters);
    p.chunk_base = b.at<int>(P.chunk_base);
    p.counts = b.at<int>(P.counts);
    p.offsets = b.at<int>(P.offsets);
    p.row_offsets = b.at<int>(P.row_offsets);
    p.perm_slot = b.at<int>(P.perm_slot);
    p.live = b.at<int>(P.live);
    p.n_live = b.at<int>(P.counters) + 2;
    p.counts_out = counts_out;
    p.capacity = P.reroute ? INT32_MAX : P.capacity;   // a reroute's tables come from the scan after it
    if (aux) {
        p.aux_counts = aux->counts;
        p.aux_importance = aux->importance;
        p.aux_p_mean = aux->p_mean;
        p.aux_scalars = aux->scalars;
    }
    p.y_zero = P.simt_router ? y_zero : nullptr;
    p.timeout_ns = kTimeoutNs;
    if (P.few_router) {
        const __nv_bfloat16 *xb = static_cast<const __nv_bfloat16 *>(x);
        const __nv_bfloat16 *wg = static_cast<const __nv_bfloat16 *>(w->W_g);
        const int S = P.route_splits;
        const int rows = (int)cdiv(D, S);
        return launch_pdl(rtc::router_few_kernel, dim3((unsigned)T, (unsigned)S), dim3(256), 0, s, xb, wg, p,
                          b.at<float>(P.route_part), b.at<unsigned>(P.counters) + 64, rows);
    }
    if (P.simt_router) {
        const __nv_bfloat16 *xb = static_cast<const __nv_bfloat16 *>(x);
        const __nv_bfloat16 *wg = static_cast<const __nv_bfloat16 *>(w->W_g);
        const unsigned grid = (unsigned)P.n_chunks;
#define MOE_SIMT(NP) \
    return launch_pdl(rtc::router_simt_kernel<NP, false>, dim3(grid), dim3(256), rtc::SimtShape<NP>::smem_bytes(D), s, xb, \
                      wg, p)
        if (P.np == 8) MOE_SIMT(8);
        if (P.np == 16) MOE_SIMT(16);
        MOE_SIMT(32);
#undef MOE_SIMT
    }
    __nv_bfloat16 *wgt = b.at<__nv_bfloat16>(P.wgt);
    MOE_TRY(launch_pdl(transpose_kernel<__nv_bfloat16>, dim3((unsigned)cdiv(N, 32), (unsigned)cdiv(D, 32)), dim3(32, 8),
                       0, s, static_cast<const __nv_bfloat16 *>(w->W_g), D, N, wgt));
    CUtensorMap mx, mw;
    MOE_TRY(make_map(&mx, x, T, D, rtc::BM));
    MOE_TRY(make_map(&mw, wgt, N, D, P.rnp));
    const int grid = P.n_chunks;
#define MOE_RTC(NP)                                                                        \
    return P.rkm == 8 ? launch_rtc<NP, 8>(mx, mw, p, grid, s) : launch_rtc<NP, 32>(mx, mw, p, grid, s)
    switch (P.rnp) {
        case 16: MOE_RTC(16);
        case 32: MOE_RTC(32);
        case 64: MOE_RTC(64);
        case 128: MOE_RTC(128);
        default: MOE_RTC(256);
    }
#undef MOE_RTC
}

// The SIMT router with the dispatch in the same cooperative launch (every chunk's
// block resident at once): routing, the y clear, a grid barrier, then each
// block scatters its own chunk.  Sets *done = false, launching nothing, when
// the blocks would not all be resident; the caller then runs the router and
// the permute kernel instead.
template <int NP>
int launch_simt_dispatch(const Plan &P, const rtc::Params &p, const __nv_bfloat16 *xb, const __nv_bfloat16 *wg,
                         const DeviceInfo &dev, cudaStream_t s, bool *done) {
    const size_t smem = rtc::SimtShape<NP>::smem_bytes(P.D);
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, rtc::router_simt_kernel<NP, true>, 256, smem) !=
        cudaSuccess)
        return MOE_ERR_CUDA;
    if ((int64_t)per_sm * dev.sms < P.n_chunks) {
        *done = false;
        return MOE_OK;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)P.n_chunks);
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, rtc::router_simt_kernel<NP, true>, xb, wg, p);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    *done = true;
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int stage_route_simt_dispatch(const Plan &P, const Bufs &b, const void *x, const moe_weights *w, moe_aux *aux,
                              float *y_zero, const DeviceInfo &dev, cudaStream_t s, bool *done) {
    rtc::Params p{};
    p.T = (int)P.T;
    p.D = P.D;
    p.N = P.N;
    p.K = P.K;
    p.np = P.rnp;
    p.bg = w->b_g;
    p.bsel = w->b_sel;
    p.logits = b.at<float>(P.logits);
    p.topk_idx = b.at<int>(P.idx);
    p.topk_w = b.at<float>(P.w);
    p.tile_counts = b.at<int>(P.chunk_counts);
    p.sum_p = reinterpret_cast<unsigned long long *>(b.ws + P.counters + P.stat_sums);
    p.sum_imp = p.sum_p + P.N;
    p.ticket = b.at<unsigned>(P.counters);
    p.chunk_base = b.at<int>(P.chunk_base);
    p.counts = b.at<int>(P.counts);
    p.offsets = b.at<int>(P.offsets);
    p.row_offsets = b.at<int>(P.row_offsets);
    p.perm_slot = b.at<int>(P.perm_slot);
    p.live = b.at<int>(P.live);
    p.n_live = b.at<int>(P.counters) + 2;
    p.capacity = P.capacity;
    if (aux) {
        p.aux_counts = aux->counts;
        p.aux_importance = aux->importance;
        p.aux_p_mean = aux->p_mean;
        p.aux_scalars = aux->scalars;
    }
    p.y_zero = y_zero;
    p.x_perm = b.at<__nv_bfloat16>(P.x_perm);
    p.slot_row = b.at<int>(P.slot_row);
    p.grid_bar = b.at<unsigned>(P.counters) + 7;
    p.timeout_ns = kTimeoutNs;
    const __nv_bfloat16 *xb = static_cast<const __nv_bfloat16 *>(x);
    const __nv_bfloat16 *wg = static_cast<const __nv_bfloat16 *>(w->W_g);
    if (P.np == 8) return launch_simt_dispatch<8>(P, p, xb, wg, dev, s, done);
    if (P.np == 16) return launch_simt_dispatch<16>(P, p, xb, wg, dev, s, done);
    return launch_simt_dispatch<32>(P, p, xb, wg, dev, s, done);
}

int stage_route(const Plan &P, const Bufs &b, const void *x, const moe_weights *w, float *logits, int *idx,
                float *tw, const DeviceInfo &dev, cudaStream_t s) {
    const int T = (int)P.T, D = P.D, N = P.N, K = P.K;
    int *cc = b.at<int>(P.chunk_counts);
    if (P.rowdot_router) {
        if (cudaMemsetAsync(cc, 0, (size_t)P.n_chunks * N * 4, s) != cudaSuccess) return MOE_ERR_CUDA;
        if (P.dtype == MOE_F32)
            router_rowdot_kernel<float><<<T, 1024, 0, s>>>(static_cast<const float *>(x), T, D, N, K,
                                                           static_cast<const float *>(w->W_g), w->b_g, w->b_sel,
                                                           logits, idx, tw, cc);
        else
            router_rowdot_kernel<__nv_bfloat16><<<T, 1024, 0, s>>>(static_cast<const __nv_bfloat16 *>(x), T, D, N, K,
                                                                   static_cast<const __nv_bfloat16 *>(w->W_g), w->b_g,
                                                                   w->b_sel, logits, idx, tw, cc);
        return check_launch();
    }
    if (P.small_router) {
        const size_t smem = (size_t)P.np * D * P.es + (size_t)P.np * 4;
#define MOE_ROUTER(TIN, NP)                                                                                     \
    router_small_kernel<TIN, NP><<<P.n_chunks, 256, smem, s>>>(static_cast<const TIN *>(x), T, D, N, K,        \
                                                               static_cast<const TIN *>(w->W_g), w->b_g, w->b_sel, \
                                                               logits, idx, tw, cc)
        if (P.dtype == MOE_F32) {
            if (P.np == 8) MOE_ROUTER(float, 8);
            else if (P.np == 16) MOE_ROUTER(float, 16);
            else MOE_ROUTER(float, 32);
        } else {
            if (P.np == 8) MOE_ROUTER(__nv_bfloat16, 8);
            else if (P.np == 16) MOE_ROUTER(__nv_bfloat16, 16);
            else MOE_ROUTER(__nv_bfloat16, 32);
        }
#undef MOE_ROUTER
        return check_launch();
    }
    // scores by GEMM: logits = x W_g + b_g
    if (P.dtype == MOE_BF16) {
        __nv_bfloat16 *wgt = b.at<__nv_bfloat16>(P.wgt);
        transpose_kernel<__nv_bfloat16><<<dim3((unsigned)cdiv(N, 32), (unsigned)cdiv(D, 32)), dim3(32, 8), 0, s>>>(
            static_cast<const __nv_bfloat16 *>(w->W_g), D, N, wgt);
        MOE_TRY(check_launch());
        CUtensorMap ma, mb;
        MOE_TRY(make_map(&ma, x, T, D, tc::BM));
        MOE_TRY(make_map(&mb, wgt, N, D, 128));
        tc::Params p{};
        p.num_groups = 1;
        p.row_offsets = nullptr;
        p.dense_rows = T;
        p.n_tiles = (int)cdiv(N, 256);
        p.num_k_blocks = (int)cdiv(D, tc::BK);
        p.b_group_rows = 0;
        p.n_valid = N;
        p.out = logits;
        p.ldo = N;
        p.bias = w->b_g;
        p.timeout_ns = kTimeoutNs;
        MOE_TRY((launch_tc2<tc::EPI_LOGITS>(ma, mb, ma, p, cdiv(T, 2 * tc::BM) * p.n_tiles, dev.pair_clusters, s)));
    } else {
        float *wgt = b.at<float>(P.wgt);
        transpose_kernel<float><<<dim3((unsigned)cdiv(N, 32), (unsigned)cdiv(D, 32)), dim3(32, 8), 0, s>>>(
            static_cast<const float *>(w->W_g), D, N, wgt);
        MOE_TRY(check_launch());
        simt::Params p{};
        p.A = static_cast<const float *>(x);
        p.lda = D;
        p.B = wgt;
        p.ldb = D;
        p.K = D;
        p.num_groups = 1;
        p.dense_rows = T;
        p.b_group_rows = 0;
        p.n_valid = N;
        p.out = logits;
        p.ldo = N;
        p.bias = w->b_g;
        MOE_TRY(launch_simt<simt::EPI_LOGITS>(p, T, (int)cdiv(N, simt::TN), s));
    }
    const size_t hs = (size_t)N * 4;
#define MOE_TOPK(V) topk_kernel<V><<<P.n_chunks, 256, hs, s>>>(logits, T, N, K, w->b_sel, idx, tw, cc)
    switch (P.vpl) {
        case 1: MOE_TOPK(1); break;
        case 2: MOE_TOPK(2); break;
        case 4: MOE_TOPK(4); break;
        case 8: MOE_TOPK(8); break;
        case 16: MOE_TOPK(16); break;
        default: MOE_TOPK(32); break;
    }
#undef MOE_TOPK
    return check_launch();
}

// The reroute ("MoE(Mixture of Experts)", design notes on the capacity
// factor): the statistics first when no router kernel took them (they describe
// the router's choice), then the sequential reroute over idx, then the chunk
// histograms and the capacity scan of the rerouted assignments.
int stage_scan(const Plan &P, const Bufs &b, int *counts_out, cudaStream_t s, int counter_word = 0);
int stage_reroute(const Plan &P, const Bufs &b, const moe_weights *w, cudaStream_t s) {
    const int N = P.N, K = P.K, B = P.rr_batch;
    const int VB = P.rr_vbatch;
    const size_t smem = (size_t)2 * ((N + 3) & ~3) * 4 + (size_t)2 * B * K * 4 + (size_t)VB * N * 4;
    if (smem > (size_t)kRerouteSmem) return MOE_ERR_UNSUPPORTED;
    const int npl = (N + 31) / 32;
    auto go = [&](auto kernel) {
        kernel<<<1, kRerouteThreads, smem, s>>>(b.at<float>(P.logits), w->b_sel, b.at<int>(P.idx), P.T, N, K,
                                                P.capacity, B, VB);
    };
    if (npl <= 1) go(reroute_kernel<1>);
    else if (npl <= 2) go(reroute_kernel<2>);
    else if (npl <= 4) go(reroute_kernel<4>);
    else if (npl <= 8) go(reroute_kernel<8>);
    else if (npl <= 16) go(reroute_kernel<16>);
    else go(reroute_kernel<32>);
    MOE_TRY(check_launch());
    hist_kernel<<<P.n_chunks, 256, (size_t)N * 4, s>>>(b.at<int>(P.idx), P.T * K, P.chunk_tokens * K, N, 1,
                                                      b.at<int>(P.chunk_counts));
    MOE_TRY(check_launch());
    return stage_scan(P, b, nullptr, s, 10);   // word 0 may hold the router's spent ticket
}

int stage_scan(const Plan &P, const Bufs &b, int *counts_out, cudaStream_t s, int counter_word) {
    scan_kernel<<<(unsigned)cdiv(P.N, 32), 1024, 0, s>>>(
        b.at<int>(P.chunk_counts), P.n_chunks, P.N, P.T * P.K, P.capacity, b.at<int>(P.chunk_base), b.at<int>(P.counts),
        b.at<int>(P.offsets), b.at<int>(P.row_offsets), b.at<int>(P.perm_slot), counts_out,
        b.at<unsigned>(P.counters) + counter_word, b.at<int>(P.live), b.at<int>(P.counters) + 2);
    return check_launch();
}

// y_zero: the fp32 output to clear on the way (when the combine folds into the
// down projection), else null.
int stage_permute(const Plan &P, const Bufs &b, const void *x, float *y_zero, const DeviceInfo &dev,
                  cudaStream_t s) {
    const size_t smem = (size_t)(3 * P.N + 1 + P.chunk_tokens * P.K) * 4;
    // enough blocks to keep every SM copying with many rows in flight: split each
    // chunk's rows over up to eight blocks, aiming at eight blocks per SM
    const int split = (int)std::max<int64_t>(1, std::min<int64_t>(8, cdiv(8 * dev.sms, P.n_chunks)));
    const dim3 grid((unsigned)P.n_chunks, (unsigned)split);
    if (P.dtype == MOE_F32)
        return launch_pdl(permute_kernel<float>, grid, dim3(256), smem, s, static_cast<const float *>(x), (int)P.T, P.D,
                          P.K, P.N, P.chunk_tokens, P.capacity, (const int *)b.at<int>(P.idx),
                          (const int *)b.at<int>(P.chunk_base),
                          (const int *)b.at<int>(P.row_offsets), b.at<int>(P.perm_slot), b.at<int>(P.slot_row),
                          b.at<float>(P.x_perm), y_zero, (const int *)nullptr);
    return launch_pdl(permute_kernel<__nv_bfloat16>, grid, dim3(256), smem, s, static_cast<const __nv_bfloat16 *>(x),
                      (int)P.T, P.D, P.K, P.N, P.chunk_tokens, P.capacity, (const int *)b.at<int>(P.idx),
                      (const int *)b.at<int>(P.chunk_base), (const int *)b.at<int>(P.row_offsets),
                      b.at<int>(P.perm_slot), b.at<int>(P.slot_row), b.at<__nv_bfloat16>(P.x_perm), y_zero,
                      (const int *)b.at<int>(P.counts));
}

// Expert GEMMs for few tokens (decode path): weight rows are the MMA's M
// operand, each expert's token rows (at most T <= 64) its narrow N operand.
template <int NT, int EPI>
int launch_dec(const CUtensorMap &W, const CUtensorMap &X, const dec::Params &p, int64_t items_upper, int sms,
               cudaStream_t s) {
    // stream-K spreads any number of tiles over every SM (up to the CTAs its
    // partial buffer is sized for); whole tiles need no more CTAs than tiles
    const int grid = p.split_cap > 0 ? std::min(sms, p.split_cap)
                                     : (int)std::min<int64_t>(std::max<int64_t>(items_upper, 1), sms);
    return launch_pdl(dec::decode_gemm_kernel<NT, EPI>, dim3(grid), dim3(dec::kThreads), dec::Shape<NT, EPI>::kSmem, s, W,
                      X, p);
}

template <int EPI>
int launch_dec_nt(int nt, const CUtensorMap &W, const CUtensorMap &X, const dec::Params &p, int64_t items_upper,
                  int sms, cudaStream_t s) {
    if (nt == 16) return launch_dec<16, EPI>(W, X, p, items_upper, sms, s);
    if (nt == 32) return launch_dec<32, EPI>(W, X, p, items_upper, sms, s);
    return launch_dec<64, EPI>(W, X, p, items_upper, sms, s);
}

int stage_up_decode(const Plan &P, const Bufs &b, const moe_weights *w, const DeviceInfo &dev, cudaStream_t s) {
    const int D = P.D, H = P.H, N = P.N;
    const bool swiglu = P.act == MOE_ACT_SWIGLU;
    CUtensorMap mw, mx;
    MOE_TRY(make_map(&mw, w->W1, (int64_t)N * (swiglu ? 2 * H : H), D, swiglu ? 64 : 128));
    MOE_TRY(make_map(&mx, b.ws + P.x_perm, P.rows_cap, D, P.nt));
    dec::Params p{};
    p.row_offsets = b.at<int>(P.row_offsets);
    p.counts = b.at<int>(P.counts);
    p.live = b.at<int>(P.live);
    p.n_live = b.at<int>(P.counters) + 2;
    p.tiles_per_group = (int)cdiv(H, swiglu ? 64 : 128);
    p.num_k_blocks = (int)cdiv(D, dec::BK);
    p.w_group_rows = swiglu ? 2 * H : H;
    p.w_up_offset = H;
    p.n_valid = H;
    p.out = b.ws + P.h;
    p.ldo = H;
    p.bias = swiglu ? nullptr : w->b1;
    p.split_cap = P.dec_cap;
    p.part = b.at<float>(P.dec_part);
    p.tickets = b.at<unsigned>(P.counters) + 128;
    p.timeout_ns = kTimeoutNs;
    const int64_t upper = std::min<int64_t>(N, P.T * P.K) * p.tiles_per_group;
    if (swiglu) return launch_dec_nt<dec::EPI_SWIGLU>(P.nt, mw, mx, p, upper, dev.sms, s);
    return launch_dec_nt<dec::EPI_GELU>(P.nt, mw, mx, p, upper, dev.sms, s);
}

int stage_down_decode(const Plan &P, const Bufs &b, const moe_weights *w, const DeviceInfo &dev, cudaStream_t s) {
    const int D = P.D, H = P.H, N = P.N;
    CUtensorMap mw, mx;
    MOE_TRY(make_map(&mw, w->W2, (int64_t)N * D, H, 128));
    MOE_TRY(make_map(&mx, b.ws + P.h, P.rows_cap, H, P.nt));
    dec::Params p{};
    p.row_offsets = b.at<int>(P.row_offsets);
    p.counts = b.at<int>(P.counts);
    p.live = b.at<int>(P.live);
    p.n_live = b.at<int>(P.counters) + 2;
    p.tiles_per_group = (int)cdiv(D, 128);
    p.num_k_blocks = (int)cdiv(H, dec::BK);
    p.w_group_rows = D;
    p.n_valid = D;
    p.out = b.ws + P.z;
    p.ldo = D;
    p.bias = P.act == MOE_ACT_SWIGLU ? nullptr : w->b2;
    p.perm_slot = b.at<int>(P.perm_slot);
    p.gate_w = b.at<float>(P.w);
    p.split_cap = P.dec_cap;
    p.part = b.at<float>(P.dec_part);
    p.tickets = b.at<unsigned>(P.counters) + 128 + P.dec_cap;
    p.timeout_ns = kTimeoutNs;
    const int64_t upper = std::min<int64_t>(N, P.T * P.K) * p.tiles_per_group;
    return launch_dec_nt<dec::EPI_SCATTER>(P.nt, mw, mx, p, upper, dev.sms, s);
}

// True when the grouped GEMM would have too few 256-wide tiles to fill the
// GPU: the row tiles are estimated from the routed rows (at least T*K/128),
// since the per-expert counts live on the device.
bool narrow_tiles(const Plan &P, int64_t n_tiles_256, const DeviceInfo &dev) {
    const int64_t m_tiles_min = std::max<int64_t>(1, cdiv(P.T * P.K, tc::BM));
    return m_tiles_min * n_tiles_256 < (int64_t)dev.sms;
}

// Whether the experts' odd last 128-row blocks go to a 1-CTA tail kernel beside
// the pair kernel instead of half-empty pair tiles.  The half-empty tiles cost
// about 64 rows per expert (half the experts have an odd block count), a share
// 64 N / (T K) of the rows; the tail kernel's tiles are less efficient (B not
// shared by a pair) and partly run after the pair kernel, which measured slower
// at 2.3% (6 experts x 2731 rows) and 6% (8 x 1024) and faster at 12.5%
// (256 x 512).
bool tail_split(const Plan &P) { return 64.0 * P.N > 0.1 * (double)(P.T * P.K); }

// With the tail split, the SMs are divided between the two kernels from the
// start so that both walk the experts at about the same pace (the tail tiles
// then find their expert's weights still in L2): the tail kernel's share is
// its expected work, about N/2 odd blocks of 128 rows at 1.3 times a pair
// tile's cost per SM, against the pair units of the rest.
int tail_sms(const Plan &P, const DeviceInfo &dev) {
    const double blocks = (double)(P.T * P.K) / 128.0 + 0.5 * P.N;
    const double tails = 0.5 * P.N, pairs = std::max(1.0, (blocks - tails) / 2.0);
    const double share = 1.3 * tails / (2.0 * pairs + 1.3 * tails);
    const int n = (int)(share * dev.sms + 0.5) & ~1;
    return std::max(2, std::min(dev.sms / 2, n));
}

int stage_up(const Plan &P, const Bufs &b, const moe_weights *w, const DeviceInfo &dev, cudaStream_t s) {
    if (P.decode) return stage_up_decode(P, b, w, dev, s);
    const int D = P.D, H = P.H, N = P.N;
    const bool swiglu = P.act == MOE_ACT_SWIGLU;
    if (P.dtype == MOE_BF16) {
        const int bn = narrow_tiles(P, swiglu ? cdiv(H, 128) : cdiv(H, 256), dev) ? 128 : 256;
        const int out_cols = swiglu ? bn / 2 : bn;  // h columns per tile
        CUtensorMap ma, mb;
        MOE_TRY(make_map(&ma, b.ws + P.x_perm, P.rows_cap, D, tc::BM));
        MOE_TRY(make_map(&mb, w->W1, (int64_t)N * (swiglu ? 2 * H : H), D, bn == 256 ? 128 : (swiglu ? bn / 2 : bn)));
        tc::Params p{};
        p.num_groups = N;
        p.row_offsets = b.at<int>(P.row_offsets);
        p.n_tiles = (int)cdiv(H, out_cols);
        p.num_k_blocks = (int)cdiv(D, tc::BK);
        p.b_group_rows = swiglu ? 2 * H : H;
        p.b_up_offset = H;
        p.n_valid = H;
        p.out = b.ws + P.h;
        p.ldo = H;
        p.bias = swiglu ? nullptr : w->b1;
        p.timeout_ns = kTimeoutNs;
        CUtensorMap mo;
        MOE_TRY(make_store_map(&mo, b.ws + P.h, P.rows_cap, H));
        const int64_t upper = (P.rows_cap / tc::BM) * p.n_tiles;
        if (bn == 128) {
            if (swiglu) return launch_tc<128, tc::EPI_SWIGLU>(ma, mb, mo, p, upper, dev.sms, s);
            return launch_tc<128, tc::EPI_GELU>(ma, mb, mo, p, upper, dev.sms, s);
        }
        // 256-row pair tiles for each expert's pairs of 128-row blocks, then
        // 128-row tiles on one CTA for the experts' odd last blocks
        const int64_t units = (P.rows_cap / (2 * tc::BM) + N) * p.n_tiles;
        if (!tail_split(P)) {
            if (swiglu) return launch_tc2<tc::EPI_SWIGLU>(ma, mb, mo, p, units, dev.pair_clusters, s);
            return launch_tc2<tc::EPI_GELU>(ma, mb, mo, p, units, dev.pair_clusters, s);
        }
        p.tail_mode = 1;
        const int tsm = tail_sms(P, dev);
        const int pcl = std::max(1, dev.pair_clusters - tsm / 2);
        if (swiglu) MOE_TRY(launch_tc2<tc::EPI_SWIGLU>(ma, mb, mo, p, units, pcl, s));
        else MOE_TRY(launch_tc2<tc::EPI_GELU>(ma, mb, mo, p, units, pcl, s));
        // the tail tiles are 128 x 256 (SwiGLU: 128 gate + 128 up rows of W1,
        // the pair kernel's B box; GELU: one 256-row box)
        tc::Params pt = p;
        pt.tail_mode = 2;
        CUtensorMap mbt = mb;
        if (!swiglu) MOE_TRY(make_map(&mbt, w->W1, (int64_t)N * H, D, 256));
        if (swiglu) return launch_tc<256, tc::EPI_SWIGLU>(ma, mbt, mo, pt, (int64_t)N * pt.n_tiles, tsm, s);
        return launch_tc<256, tc::EPI_GELU>(ma, mbt, mo, pt, (int64_t)N * pt.n_tiles, tsm, s);
    }
    simt::Params p{};
    p.A = b.at<float>(P.x_perm);
    p.lda = D;
    p.B = static_cast<const float *>(w->W1);
    p.ldb = D;
    p.K = D;
    p.num_groups = N;
    p.row_offsets = b.at<int>(P.row_offsets);
    p.b_group_rows = swiglu ? 2 * H : H;
    p.b_up_offset = H;
    p.n_valid = H;
    p.out = b.at<float>(P.h);
    p.ldo = H;
    p.bias = swiglu ? nullptr : w->b1;
    if (swiglu) return launch_simt<simt::EPI_SWIGLU>(p, P.rows_cap, (int)cdiv(H, simt::TN / 2), s);
    return launch_simt<simt::EPI_GELU>(p, P.rows_cap, (int)cdiv(H, simt::TN), s);
}

// The combine folds into the down projection (fp32 reductions into y) for bf16
// prefill layers with K <= 2 and an fp32 y: at most two additions per element
// onto +0, so the result is the same in any order.
bool combine_in_down(const Plan &P, int y_dtype) {
    return P.dtype == MOE_BF16 && !P.decode && P.K <= 2 && y_dtype == MOE_F32 && !P.n_shared;
}

int stage_down(const Plan &P, const Bufs &b, const moe_weights *w, void *y, int y_dtype, const DeviceInfo &dev,
               cudaStream_t s) {
    if (P.decode) return stage_down_decode(P, b, w, dev, s);
    const int D = P.D, H = P.H, N = P.N;
    const float *bias = P.act == MOE_ACT_SWIGLU ? nullptr : w->b2;
    if (P.dtype == MOE_BF16) {
        const int bn = narrow_tiles(P, cdiv(D, 256), dev) ? 128 : 256;
        CUtensorMap ma, mb;
        MOE_TRY(make_map(&ma, b.ws + P.h, P.rows_cap, H, tc::BM));
        MOE_TRY(make_map(&mb, w->W2, (int64_t)N * D, H, 128));
        tc::Params p{};
        p.num_groups = N;
        p.row_offsets = b.at<int>(P.row_offsets);
        p.n_tiles = (int)cdiv(D, bn);
        p.num_k_blocks = (int)cdiv(H, tc::BK);
        p.b_group_rows = D;
        p.n_valid = D;
        p.out = b.ws + P.z;
        p.ldo = D;
        p.bias = bias;
        p.perm_slot = b.at<int>(P.perm_slot);
        p.gate_w = b.at<float>(P.w);
        p.slot_limit = P.T * P.K;
        p.timeout_ns = kTimeoutNs;
        CUtensorMap mo = ma;   // unused unless z is written by rows
        if (combine_in_down(P, y_dtype)) {   // y was cleared by the router or the permute kernel
            p.out = y;
            p.accum_k = P.K;
        } else {
            MOE_TRY(make_store_map_f32(&mo, b.ws + P.z, P.rows_cap, D));
            p.scatter_rows = 1;
        }
        const int64_t upper = (P.rows_cap / tc::BM) * p.n_tiles;
        if (bn == 128) return launch_tc<128, tc::EPI_SCATTER>(ma, mb, mo, p, upper, dev.sms, s);
        // pair tiles, then the odd last blocks on one CTA (as in the up projection)
        if (!tail_split(P))
            return launch_tc2<tc::EPI_SCATTER>(ma, mb, mo, p, (P.rows_cap / (2 * tc::BM) + N) * p.n_tiles,
                                               dev.pair_clusters, s);
        p.tail_mode = 1;
        const int tsm = tail_sms(P, dev);
        MOE_TRY(launch_tc2<tc::EPI_SCATTER>(ma, mb, mo, p, (P.rows_cap / (2 * tc::BM) + N) * p.n_tiles,
                                            std::max(1, dev.pair_clusters - tsm / 2), s));
        tc::Params pt = p;
        pt.tail_mode = 2;
        CUtensorMap mbt;
        MOE_TRY(make_map(&mbt, w->W2, (int64_t)N * D, H, 256));
        return launch_tc<256, tc::EPI_SCATTER>(ma, mbt, mo, pt, (int64_t)N * pt.n_tiles, tsm, s);
    }
    simt::Params p{};
    p.A = b.at<float>(P.h);
    p.lda = H;
    p.B = static_cast<const float *>(w->W2);
    p.ldb = H;
    p.K = H;
    p.num_groups = N;
    p.row_offsets = b.at<int>(P.row_offsets);
    p.b_group_rows = D;
    p.n_valid = D;
    p.out = b.at<float>(P.z);
    p.ldo = D;
    p.bias = bias;
    p.perm_slot = b.at<int>(P.perm_slot);
    p.gate_w = b.at<float>(P.w);
    return launch_simt<simt::EPI_SCATTER>(p, P.rows_cap, (int)cdiv(D, simt::TN), s);
}

// ---------------------------------------------------------------- shared expert
// A dense FFN over every token: the grouped GEMMs in dense mode (one group,
// the token rows of x as the A operand, no dispatch) for prefill, the
// weight-streaming GEMMs with a one-group table for few tokens.  Its fp32
// output s_out is added by the combine after the routed sum.
int stage_shared_up(const Plan &P, const Bufs &b, const void *x, const moe_weights *w, const DeviceInfo &dev,
                    cudaStream_t s) {
    const int D = P.D, H = P.H;
    const bool swiglu = P.act == MOE_ACT_SWIGLU;
    const int rows1 = swiglu ? 2 * H : H;
    const float *bias = swiglu ? nullptr : w->sb1;
    if (P.dtype == MOE_F32) {
        simt::Params p{};
        p.A = static_cast<const float *>(x);
        p.lda = D;
        p.B = static_cast<const float *>(w->S1);
        p.ldb = D;
        p.K = D;
        p.num_groups = 1;
        p.row_offsets = nullptr;
        p.dense_rows = (int)P.T;
        p.b_group_rows = rows1;
        p.b_up_offset = H;
        p.n_valid = H;
        p.out = b.at<float>(P.h_s);
        p.ldo = H;
        p.bias = bias;
        if (swiglu) return launch_simt<simt::EPI_SWIGLU>(p, P.T, (int)cdiv(H, simt::TN / 2), s);
        return launch_simt<simt::EPI_GELU>(p, P.T, (int)cdiv(H, simt::TN), s);
    }
    if (P.decode) {
        CUtensorMap mw, mx;
        MOE_TRY(make_map(&mw, w->S1, rows1, D, swiglu ? 64 : 128));
        MOE_TRY(make_map(&mx, x, P.T, D, P.nt));
        dec::Params p{};
        int *tbl = b.at<int>(P.shared_tbl);
        p.live = tbl;
        p.n_live = tbl + 1;
        p.counts = tbl + 2;
        p.row_offsets = tbl + 3;
        p.tiles_per_group = (int)cdiv(H, swiglu ? 64 : 128);
        p.num_k_blocks = (int)cdiv(D, dec::BK);
        p.w_group_rows = rows1;
        p.w_up_offset = H;
        p.n_valid = H;
        p.out = b.ws + P.h_s;
        p.ldo = H;
        p.bias = bias;
        p.split_cap = P.dec_cap;
        p.part = b.at<float>(P.dec_part);
        p.tickets = b.at<unsigned>(P.counters) + 128 + 2 * P.dec_cap;
        p.timeout_ns = kTimeoutNs;
        if (swiglu) return launch_dec_nt<dec::EPI_SWIGLU>(P.nt, mw, mx, p, p.tiles_per_group, dev.sms, s);
        return launch_dec_nt<dec::EPI_GELU>(P.nt, mw, mx, p, p.tiles_per_group, dev.sms, s);
    }
    const int bn = narrow_tiles(P, swiglu ? cdiv(H, 128) : cdiv(H, 256), dev) ? 128 : 256;
    const int out_cols = swiglu ? bn / 2 : bn;
    CUtensorMap ma, mb, mo;
    MOE_TRY(make_map(&ma, x, P.T, D, tc::BM));
    MOE_TRY(make_map(&mb, w->S1, rows1, D, bn == 256 ? 128 : (swiglu ? bn / 2 : bn)));
    MOE_TRY(make_store_map(&mo, b.ws + P.h_s, P.T, H));
    tc::Params p{};
    p.num_groups = 1;
    p.row_offsets = nullptr;
    p.dense_rows = (int)P.T;
    p.n_tiles = (int)cdiv(H, out_cols);
    p.num_k_blocks = (int)cdiv(D, tc::BK);
    p.b_group_rows = rows1;
    p.b_up_offset = H;
    p.n_valid = H;
    p.out = b.ws + P.h_s;
    p.ldo = H;
    p.bias = bias;
    p.timeout_ns = kTimeoutNs;
    if (bn == 128) {
        const int64_t upper = cdiv(P.T, tc::BM) * p.n_tiles;
        if (swiglu) return launch_tc<128, tc::EPI_SWIGLU>(ma, mb, mo, p, upper, dev.sms, s);
        return launch_tc<128, tc::EPI_GELU>(ma, mb, mo, p, upper, dev.sms, s);
    }
    const int64_t units = cdiv(P.T, 2 * tc::BM) * p.n_tiles;
    if (swiglu) return launch_tc2<tc::EPI_SWIGLU>(ma, mb, mo, p, units, dev.pair_clusters, s);
    return launch_tc2<tc::EPI_GELU>(ma, mb, mo, p, units, dev.pair_clusters, s);
}

int stage_shared_down(const Plan &P, const Bufs &b, const moe_weights *w, const DeviceInfo &dev, cudaStream_t s) {
    const int D = P.D, H = P.H;
    const float *bias = P.act == MOE_ACT_SWIGLU ? nullptr : w->sb2;
    if (P.dtype == MOE_F32) {
        simt::Params p{};
        p.A = b.at<float>(P.h_s);
        p.lda = H;
        p.B = static_cast<const float *>(w->S2);
        p.ldb = H;
        p.K = H;
        p.num_groups = 1;
        p.row_offsets = nullptr;
        p.dense_rows = (int)P.T;
        p.b_group_rows = D;
        p.n_valid = D;
        p.out = b.at<float>(P.s_out);
        p.ldo = D;
        p.bias = bias;
        p.perm_slot = nullptr;   // row r is token r, weight 1
        p.gate_w = nullptr;
        return launch_simt<simt::EPI_SCATTER>(p, P.T, (int)cdiv(D, simt::TN), s);
    }
    if (P.decode) {
        CUtensorMap mw, mx;
        MOE_TRY(make_map(&mw, w->S2, D, H, 128));
        MOE_TRY(make_map(&mx, b.ws + P.h_s, P.T, H, P.nt));
        dec::Params p{};
        int *tbl = b.at<int>(P.shared_tbl);
        p.live = tbl;
        p.n_live = tbl + 1;
        p.counts = tbl + 2;
        p.row_offsets = tbl + 3;
        p.tiles_per_group = (int)cdiv(D, 128);
        p.num_k_blocks = (int)cdiv(H, dec::BK);
        p.w_group_rows = D;
        p.n_valid = D;
        p.out = b.ws + P.s_out;
        p.ldo = D;
        p.bias = bias;
        p.perm_slot = nullptr;   // row j is token j, weight 1
        p.gate_w = nullptr;
        p.split_cap = P.dec_cap;
        p.part = b.at<float>(P.dec_part);
        p.tickets = b.at<unsigned>(P.counters) + 128 + 3 * P.dec_cap;
        p.timeout_ns = kTimeoutNs;
        return launch_dec_nt<dec::EPI_SCATTER>(P.nt, mw, mx, p, p.tiles_per_group, dev.sms, s);
    }
    const int bn = narrow_tiles(P, cdiv(D, 256), dev) ? 128 : 256;
    CUtensorMap ma, mb, mo;
    MOE_TRY(make_map(&ma, b.ws + P.h_s, P.T, H, tc::BM));
    MOE_TRY(make_map(&mb, w->S2, D, H, 128));
    MOE_TRY(make_store_map_f32(&mo, b.ws + P.s_out, P.T, D));
    tc::Params p{};
    p.num_groups = 1;
    p.row_offsets = nullptr;
    p.dense_rows = (int)P.T;
    p.n_tiles = (int)cdiv(D, bn);
    p.num_k_blocks = (int)cdiv(H, tc::BK);
    p.b_group_rows = D;
    p.n_valid = D;
    p.out = b.ws + P.s_out;
    p.ldo = D;
    p.bias = bias;
    p.perm_slot = nullptr;   // dense rows: row r is token r, weight 1
    p.gate_w = nullptr;
    p.scatter_rows = 1;
    p.timeout_ns = kTimeoutNs;
    if (bn == 128) return launch_tc<128, tc::EPI_SCATTER>(ma, mb, mo, p, cdiv(P.T, tc::BM) * p.n_tiles, dev.sms, s);
    return launch_tc2<tc::EPI_SCATTER>(ma, mb, mo, p, cdiv(P.T, 2 * tc::BM) * p.n_tiles, dev.pair_clusters, s);
}

int stage_combine(const Plan &P, const Bufs &b, void *y, int y_dtype, const DeviceInfo &dev, cudaStream_t s) {
    const int64_t nq = P.T * (P.D / 4);
    const int grid = (int)std::min<int64_t>(cdiv(nq, 256), (int64_t)dev.sms * 8);
    // bf16 prefill layers keep z in the permuted row order (see stage_down); every
    // layer marks the slots the capacity limit dropped with slot_row -1
    const int *slot_row = b.at<int>(P.slot_row);
    const int z_by_row = P.dtype == MOE_BF16 && !P.decode ? 1 : 0;
    const float *shared = P.n_shared ? b.at<float>(P.s_out) : nullptr;
    const int64_t z_rows = z_by_row ? (int64_t)P.rows_cap : P.T * P.K;
    if (y_dtype == MOE_F32)
        return launch_pdl(combine_kernel<float>, dim3(grid), dim3(256), 0, s, (const float *)b.at<float>(P.z), z_rows,
                          P.T, P.D, P.K, slot_row, z_by_row, shared, static_cast<float *>(y));
    return launch_pdl(combine_kernel<__nv_bfloat16>, dim3(grid), dim3(256), 0, s, (const float *)b.at<float>(P.z),
                      z_rows, P.T, P.D, P.K, slot_row, z_by_row, shared, static_cast<__nv_bfloat16 *>(y));
}

int stage_aux(const Plan &P, const Bufs &b, const float *logits, const int *idx, const float *tw, moe_aux *aux,
              cudaStream_t s) {
    const int N = P.N;
    AuxOut out{aux->counts, aux->importance, aux->p_mean, aux->scalars};
    unsigned *counter = b.at<unsigned>(P.counters) + 1;
    if (N <= 32) {
        const unsigned grid = (unsigned)cdiv(P.T, 256);
#define MOE_AUX(NP)                                                                                        \
    aux_small_kernel<NP><<<grid, 256, 0, s>>>(logits, idx, tw, (int)P.T, N, P.K, b.at<float>(P.aux_p),     \
                                              b.at<float>(P.aux_i), b.at<int>(P.aux_c), counter, out)
        if (N <= 8) MOE_AUX(8);
        else if (N <= 16) MOE_AUX(16);
        else MOE_AUX(32);
#undef MOE_AUX
        return check_launch();
    }
    aux_partial_kernel<<<P.aux_blocks, 256, (size_t)24 * N * 4, s>>>(logits, idx, tw, (int)P.T, N, P.K,
                                                                     b.at<float>(P.aux_p), b.at<float>(P.aux_i),
                                                                     b.at<int>(P.aux_c), counter, out);
    return check_launch();
}

int zero_counters(const Plan &P, const Bufs &b, cudaStream_t s) {
    DeviceInfo *dev = nullptr;
    MOE_TRY(device_info(&dev));
    return launch_zero(b.ws + P.counters, P.counters_bytes, dev->sms, s,
                       P.n_shared ? b.at<int>(P.shared_tbl) : nullptr, (int)P.T);
}

int zero_aux(const Plan &P, moe_aux *aux, cudaStream_t s) {
    if (!aux) return MOE_OK;
    if (aux->counts && cudaMemsetAsync(aux->counts, 0, (size_t)P.N * 4, s) != cudaSuccess) return MOE_ERR_CUDA;
    if (aux->importance && cudaMemsetAsync(aux->importance, 0, (size_t)P.N * 4, s) != cudaSuccess) return MOE_ERR_CUDA;
    if (aux->p_mean && cudaMemsetAsync(aux->p_mean, 0, (size_t)P.N * 4, s) != cudaSuccess) return MOE_ERR_CUDA;
    if (aux->scalars && cudaMemsetAsync(aux->scalars, 0, 16, s) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
}

// ---------------------------------------------------------------- fused decode
// Whether the fused decode kernel is launched with programmatic serialization
// besides the cooperative attribute (cleared if the runtime refuses the pair).
std::atomic<bool> g_fused_pdl{true};

// Routing scratch of the fused decode kernel, in its ring: R1 x rows and the
// W_g slab; R2 (every token's slab sums for few tokens, after R3's arrays) the slabs' scores of one token; R3 top-k experts,
// ranks, gate weights and full softmax.
size_t fused_scratch(int T, int slab_rows, int n_slabs) {
    const size_t r1 = ((size_t)T * slab_rows + (size_t)slab_rows * 32) * 4;
    const size_t r2 = (size_t)n_slabs * 32 * 4;
    const size_t r3 = ((size_t)3 * dfu::kMaxSlots + (size_t)T * 32) * 4;
    // R2 in every CTA for few tokens: the slab sums of all tokens after R3's arrays
    const size_t r2a = T <= dfu::kAllR2T ? ((size_t)3 * dfu::kMaxSlots + (size_t)dfu::kMaxT * 32) * 4 +
                                               (size_t)n_slabs * T * 32 * 4
                                         : 0;
    return std::max(std::max(r1, r2a), std::max(r2, r3));
}

template <int NT, int EPI>
int launch_fused(const CUtensorMap &mw1, const CUtensorMap &mxp, const CUtensorMap &mw2, const CUtensorMap &mh,
                 const dfu::Params &p, int grid, cudaStream_t s) {
    using S = dfu::Shape<NT, EPI>;
    // routing scratch (R1-R3) lives in the ring before the expert phases use it
    if (fused_scratch(p.T, p.slab_rows, p.n_slabs) > S::kRingBytes) return MOE_ERR_UNSUPPORTED;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(dfu::kThreads);
    cfg.dynamicSmemBytes = S::kSmem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;   // every CTA resident: the grid barriers need it
    attr[0].val.cooperative = 1;
    // and launched while the counters are being cleared (its pdl_enter waits for that)
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = g_fused_pdl ? 2 : 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, dfu::decode_layer_kernel<NT, EPI>, mw1, mxp, mw2, mh, p);
    if (e != cudaSuccess && cfg.numAttrs == 2) {   // the runtime refused the pair: cooperative alone
        (void)cudaGetLastError();
        g_fused_pdl = false;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, dfu::decode_layer_kernel<NT, EPI>, mw1, mxp, mw2, mh, p);
    }
    g_launches.fetch_add(1, std::memory_order_relaxed);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

template <int EPI>
int launch_fused_nt(int nt, const CUtensorMap &mw1, const CUtensorMap &mxp, const CUtensorMap &mw2,
                    const CUtensorMap &mh, const dfu::Params &p, int grid, cudaStream_t s) {
    if (nt == 16) return launch_fused<16, EPI>(mw1, mxp, mw2, mh, p, grid, s);
    if (nt == 32) return launch_fused<32, EPI>(mw1, mxp, mw2, mh, p, grid, s);
    return launch_fused<64, EPI>(mw1, mxp, mw2, mh, p, grid, s);
}

// Whether the fused kernel's routing scratch fits its ring for this layer.
template <int EPI>
bool fused_fits_nt(int nt, size_t scratch) {
    if (nt == 16) return scratch <= dfu::Shape<16, EPI>::kRingBytes;
    if (nt == 32) return scratch <= dfu::Shape<32, EPI>::kRingBytes;
    return scratch <= dfu::Shape<64, EPI>::kRingBytes;
}
bool fused_fits(const Plan &P) {
    const size_t scratch = fused_scratch((int)P.T, P.slab_rows, P.n_slabs);
    return P.act == MOE_ACT_SWIGLU ? fused_fits_nt<dec::EPI_SWIGLU>(P.nt, scratch)
                                   : fused_fits_nt<dec::EPI_GELU>(P.nt, scratch);
}

// The whole layer for few tokens in one cooperative kernel (moe_decode_fused.cuh).
int stage_decode_fused(const Plan &P, const Bufs &b, const void *x, const moe_weights *w, void *y, int y_dtype,
                       moe_aux *aux, const DeviceInfo &dev, cudaStream_t s) {
    const int D = P.D, H = P.H, N = P.N;
    const bool swiglu = P.act == MOE_ACT_SWIGLU;
    const int grid = dev.sms;
    CUtensorMap mw1, mxp, mw2, mh;
    MOE_TRY(make_map(&mw1, w->W1, (int64_t)N * (swiglu ? 2 * H : H), D, swiglu ? 64 : 128));
    MOE_TRY(make_map(&mxp, b.ws + P.x_perm, P.rows_cap, D, P.nt));
    MOE_TRY(make_map(&mw2, w->W2, (int64_t)N * D, H, 128));
    MOE_TRY(make_map(&mh, b.ws + P.h, P.rows_cap, H, P.nt));
    dfu::Params p{};
    p.T = (int)P.T;
    p.D = D;
    p.H = H;
    p.N = N;
    p.K = P.K;
    p.capacity = P.capacity;
    p.slab_rows = P.slab_rows;
    p.n_slabs = P.n_slabs;
    p.x = static_cast<const __nv_bfloat16 *>(x);
    p.Wg = static_cast<const __nv_bfloat16 *>(w->W_g);
    p.bg = w->b_g;
    p.bsel = w->b_sel;
    p.b1 = swiglu ? nullptr : w->b1;
    p.b2 = swiglu ? nullptr : w->b2;
    p.logits = b.at<float>(P.logits);
    p.topk_idx = b.at<int>(P.idx);
    p.topk_w = b.at<float>(P.w);
    p.counts = b.at<int>(P.counts);
    p.offsets = b.at<int>(P.offsets);
    p.row_offsets = b.at<int>(P.row_offsets);
    p.perm_slot = b.at<int>(P.perm_slot);
    p.slot_row = b.at<int>(P.slot_row);
    p.live = b.at<int>(P.live);
    p.n_live = b.at<int>(P.counters) + 2;
    p.x_perm = b.at<__nv_bfloat16>(P.x_perm);
    p.h = b.at<__nv_bfloat16>(P.h);
    p.z = b.at<float>(P.z);
    p.slab = b.at<float>(P.fd_slab);
    p.tok_p = b.at<float>(P.fd_tokp);
    unsigned *ctr = b.at<unsigned>(P.counters);
    p.bar = ctr + 4;
    p.bar4 = ctr + 8;
    p.tk_up = ctr + 128;
    p.tk_down = ctr + 128 + P.dec_cap;
    p.bar5 = ctr + 9;
    p.part = b.at<float>(P.dec_part);
    p.split_cap = P.dec_cap;
    p.y = y;
    p.y_bf16 = y_dtype == MOE_BF16 ? 1 : 0;
    if (aux) {
        p.aux_counts = aux->counts;
        p.aux_importance = aux->importance;
        p.aux_p_mean = aux->p_mean;
        p.aux_scalars = aux->scalars;
    }
    p.timeout_ns = kTimeoutNs;
    if (swiglu) return launch_fused_nt<dec::EPI_SWIGLU>(P.nt, mw1, mxp, mw2, mh, p, grid, s);
    return launch_fused_nt<dec::EPI_GELU>(P.nt, mw1, mxp, mw2, mh, p, grid, s);
}

int check_weights(const Plan &P, const moe_weights *w, bool need_experts) {
    if (!w || (!w->W_g && !P.given_routing)) return MOE_ERR_INVALID_ARG;   // given routing needs no router
    if (!need_experts) return MOE_OK;
    if (!w->W1 || !w->W2) return MOE_ERR_INVALID_ARG;
    if (P.has_bias && (!w->b1 || !w->b2)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(w->W1) || !aligned16(w->W2)) return MOE_ERR_INVALID_ARG;
    if (P.n_shared) {
        if (!w->S1 || !w->S2 || !aligned16(w->S1) || !aligned16(w->S2)) return MOE_ERR_INVALID_ARG;
        if (P.has_bias && (!w->sb1 || !w->sb2)) return MOE_ERR_INVALID_ARG;
    }
    return MOE_OK;
}

int forward_impl(const moe_config *cfg, const void *x, int64_t T, const moe_weights *w, void *y, int32_t y_dtype,
                 moe_aux *aux, void *ws, size_t ws_bytes, cudaStream_t s, void *const *ev,
                 const int *given_idx = nullptr, const float *given_w = nullptr) {
    Plan P;
    MOE_TRY(make_plan(cfg, T, &P, given_idx != nullptr));
    MOE_TRY(check_weights(P, w, true));
    if (y_dtype != MOE_F32 && y_dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!x || !y || !aligned16(x) || !aligned16(y))) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u))) return MOE_ERR_INVALID_ARG;
    if (T > 0 && ws_bytes < P.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    // Under stream capture the events become external event-record nodes, so
    // that a replayed graph records them (and they can be timed).
    unsigned rec_flags = cudaEventRecordDefault;
    if (ev) {
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) return MOE_ERR_CUDA;
        if (cs == cudaStreamCaptureStatusActive) rec_flags = cudaEventRecordExternal;
    }
    auto rec = [&](int i) -> int {
        if (!ev || !ev[i]) return MOE_OK;
        return cudaEventRecordWithFlags(static_cast<cudaEvent_t>(ev[i]), s, rec_flags) == cudaSuccess ? MOE_OK
                                                                                                      : MOE_ERR_CUDA;
    };
    if (T == 0) {
        for (int i = 0; i <= MOE_N_STAGES; ++i) MOE_TRY(rec(i));
        return zero_aux(P, aux, s);
    }
    DeviceInfo *dev = nullptr;
    MOE_TRY(device_info(&dev));
    Bufs b{static_cast<char *>(ws), &P};
    float *logits = b.at<float>(P.logits);
    int *idx = b.at<int>(P.idx);
    float *tw = b.at<float>(P.w);
    // the down projection adds into y when the combine folds into it; y is then
    // cleared on the way, by the SIMT router or else by the permute kernel
    float *y_zero = combine_in_down(P, y_dtype) ? static_cast<float *>(y) : nullptr;
    MOE_TRY(rec(0));
    MOE_TRY(zero_counters(P, b, s));
    // few tokens: the whole layer in one cooperative kernel when the device can
    // hold one CTA per token and W_g allows the routing's 16-byte loads
    if (P.fused_decode && dev->sms >= (int)P.T && dev->sms >= P.n_slabs && dev->sms <= P.dec_cap &&
        aligned16(w->W_g) && fused_fits(P)) {
        for (int i = 1; i <= 3; ++i) MOE_TRY(rec(i));
        MOE_TRY(stage_decode_fused(P, b, x, w, y, y_dtype, aux, *dev, s));
        for (int i = 4; i <= MOE_N_STAGES; ++i) MOE_TRY(rec(i));
        return MOE_OK;
    }
    if (P.given_routing) {
        // the assignments are inputs: into the workspace, then chunk histograms and the scan
        if (cudaMemcpyAsync(idx, given_idx, (size_t)P.T * P.K * 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess ||
            cudaMemcpyAsync(tw, given_w, (size_t)P.T * P.K * 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
            return MOE_ERR_CUDA;
        hist_kernel<<<P.n_chunks, 256, (size_t)P.N * 4, s>>>(idx, P.T * P.K, P.chunk_tokens * P.K, P.N, 1,
                                                              b.at<int>(P.chunk_counts));
        MOE_TRY(check_launch());
        MOE_TRY(rec(1));
        MOE_TRY(stage_scan(P, b, nullptr, s));
    } else if (P.tc_router) {
        // the SIMT router takes the dispatch into its own (cooperative) launch when it can
        bool dispatched = false;
        if (P.simt_router && !P.reroute)
            MOE_TRY(stage_route_simt_dispatch(P, b, x, w, aux, y_zero, *dev, s, &dispatched));
        if (dispatched) {
            MOE_TRY(rec(1));
            MOE_TRY(rec(2));
            goto experts;
        }
        MOE_TRY(stage_route_tc(P, b, x, w, logits, idx, tw, nullptr, aux, y_zero, s));
        MOE_TRY(rec(1));
        if (P.reroute) MOE_TRY(stage_reroute(P, b, w, s));
    } else {
        MOE_TRY(stage_route(P, b, x, w, logits, idx, tw, *dev, s));
        MOE_TRY(rec(1));
        if (P.reroute) {
            if (aux) MOE_TRY(stage_aux(P, b, logits, idx, tw, aux, s));   // before idx is rerouted
            MOE_TRY(stage_reroute(P, b, w, s));
        } else {
            MOE_TRY(stage_scan(P, b, nullptr, s));
        }
    }
    MOE_TRY(rec(2));
    MOE_TRY(stage_permute(P, b, x, P.simt_router ? nullptr : y_zero, *dev, s));
experts:
    MOE_TRY(rec(3));
    MOE_TRY(stage_up(P, b, w, *dev, s));
    if (P.n_shared) MOE_TRY(stage_shared_up(P, b, x, w, *dev, s));
    MOE_TRY(rec(4));
    MOE_TRY(stage_down(P, b, w, y, y_dtype, *dev, s));
    if (P.n_shared) MOE_TRY(stage_shared_down(P, b, w, *dev, s));
    MOE_TRY(rec(5));
    if (!combine_in_down(P, y_dtype)) MOE_TRY(stage_combine(P, b, y, y_dtype, *dev, s));
    MOE_TRY(rec(6));
    if (aux && !P.tc_router && !P.given_routing && !P.reroute) MOE_TRY(stage_aux(P, b, logits, idx, tw, aux, s));
    MOE_TRY(rec(7));
    return MOE_OK;
}

}  // namespace

// ===================================================================== C ABI
extern "C" {

size_t moe_workspace_size(const moe_config *cfg, int64_t T) {
    Plan P;
    if (make_plan(cfg, T, &P) != MOE_OK) return 0;
    return P.total;
}

int moe_get_workspace_layout(const moe_config *cfg, int64_t T, moe_workspace_layout *out) {
    if (!out) return MOE_ERR_INVALID_ARG;
    Plan P;
    MOE_TRY(make_plan(cfg, T, &P));
    out->total = P.total;
    out->logits = P.logits;
    out->topk_idx = P.idx;
    out->topk_w = P.w;
    out->counts = P.counts;
    out->offsets = P.offsets;
    out->row_offsets = P.row_offsets;
    out->perm_slot = P.perm_slot;
    out->slot_row = P.slot_row;
    out->x_perm = P.x_perm;
    out->h = P.h;
    out->z = P.z;
    out->rows_cap = P.rows_cap;
    out->row_align = kRowAlign;
    return MOE_OK;
}

int moe_route(const moe_config *cfg, const void *x, int64_t T, const moe_weights *w, float *logits, int32_t *topk_idx,
              float *topk_w, int32_t *counts, void *ws, size_t ws_bytes, moe_stream_t stream) {
    Plan P;
    MOE_TRY(make_plan(cfg, T, &P));
    MOE_TRY(check_weights(P, w, false));
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (T == 0) {
        if (counts && cudaMemsetAsync(counts, 0, (size_t)P.N * 4, s) != cudaSuccess) return MOE_ERR_CUDA;
        return MOE_OK;
    }
    if (!x || !aligned16(x) || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return MOE_ERR_INVALID_ARG;
    if (ws_bytes < P.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    DeviceInfo *dev = nullptr;
    MOE_TRY(device_info(&dev));
    Bufs b{static_cast<char *>(ws), &P};
    float *lg = logits ? logits : b.at<float>(P.logits);
    MOE_TRY(zero_counters(P, b, s));
    if (P.tc_router) return stage_route_tc(P, b, x, w, lg, topk_idx, topk_w, counts, nullptr, nullptr, s);
    MOE_TRY(stage_route(P, b, x, w, lg, topk_idx, topk_w, *dev, s));
    if (counts) MOE_TRY(stage_scan(P, b, counts, s));
    return MOE_OK;
}

int moe_forward(const moe_config *cfg, const void *x, int64_t T, const moe_weights *w, void *y, int32_t y_dtype,
                moe_aux *aux, void *ws, size_t ws_bytes, moe_stream_t stream) {
    return forward_impl(cfg, x, T, w, y, y_dtype, aux, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream), nullptr);
}

int moe_forward_timed(const moe_config *cfg, const void *x, int64_t T, const moe_weights *w, void *y, int32_t y_dtype,
                      moe_aux *aux, void *ws, size_t ws_bytes, moe_stream_t stream, void *const *stage_events) {
    if (!stage_events) return MOE_ERR_INVALID_ARG;
    return forward_impl(cfg, x, T, w, y, y_dtype, aux, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream),
                        stage_events);
}

int moe_aux_stats(const moe_config *cfg, int64_t T, const float *logits, const int32_t *topk_idx, const float *topk_w,
                  moe_aux *out, void *ws, size_t ws_bytes, moe_stream_t stream) {
    Plan P;
    MOE_TRY(make_plan(cfg, T, &P));
    if (!out) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (T == 0) return zero_aux(P, out, s);
    if (!logits || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return MOE_ERR_INVALID_ARG;
    if (ws_bytes < P.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    DeviceInfo *dev = nullptr;
    MOE_TRY(device_info(&dev));
    Bufs b{static_cast<char *>(ws), &P};
    MOE_TRY(zero_counters(P, b, s));
    return stage_aux(P, b, logits, topk_idx, topk_w, out, s);
}

int moe_aux_partials(const moe_config *cfg, int64_t T, const float *logits, const int32_t *topk_idx,
                     const float *topk_w, int64_t *partials, moe_stream_t stream) {
    Plan P;
    MOE_TRY(make_plan(cfg, T, &P));
    if (!partials) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!logits || !topk_idx || !topk_w)) return MOE_ERR_INVALID_ARG;
    if (T > INT32_MAX) return MOE_ERR_UNSUPPORTED;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const size_t bytes = (size_t)(3 * P.N + 1) * 8;
    if (cudaMemsetAsync(partials, 0, bytes, s) != cudaSuccess) return MOE_ERR_CUDA;
    if (T == 0) return MOE_OK;
    DeviceInfo *dev = nullptr;
    MOE_TRY(device_info(&dev));
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(cdiv(T, 8), (int64_t)dev->sms * 4));
    aux_partials_kernel<<<grid, 256, (size_t)3 * P.N * 8, s>>>(logits, topk_idx, topk_w, (int)T, P.N, P.K,
                                                                reinterpret_cast<unsigned long long *>(partials));
    return check_launch();
}

int moe_aux_finalize(const moe_config *cfg, const int64_t *partials, moe_aux *out, moe_stream_t stream) {
    Plan P;
    MOE_TRY(make_plan(cfg, 0, &P));
    if (!partials || !out) return MOE_ERR_INVALID_ARG;
    AuxOut o{out->counts, out->importance, out->p_mean, out->scalars};
    aux_finalize_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        P.N, P.K, reinterpret_cast<const long long *>(partials), o);
    return check_launch();
}

int moe_aux_finalize_host(const moe_config *cfg, const int64_t *partials, int32_t *counts, float *importance,
                          float *p_mean, float *scalars) {
    Plan P;
    MOE_TRY(make_plan(cfg, 0, &P));
    if (!partials) return MOE_ERR_INVALID_ARG;
    if (partials[3 * P.N] < 0) return MOE_ERR_INVALID_ARG;
    for (int e = 0; e < 3 * P.N; ++e)
        if (partials[e] < 0) return MOE_ERR_INVALID_ARG;
    aux_finalize_partials(P.N, P.K, reinterpret_cast<const long long *>(partials), counts, importance, p_mean,
                          scalars);
    return MOE_OK;
}

// ---------------------------------------------------------------- expert parallelism
namespace {
struct EpPlan {
    Plan P;          // the routing of this rank's tokens
    int R, epr, n_chunks;
    size_t cc, cb, offsets, rowoff, live, perm, total;
};

int make_ep_plan(const moe_config *cfg, int32_t n_ranks, int64_t T, EpPlan *e) {
    MOE_TRY(make_plan(cfg, T, &e->P));
    const int N = e->P.N;
    if (n_ranks < 1 || n_ranks > N || N % n_ranks) return MOE_ERR_INVALID_ARG;
    if (e->P.n_shared || cfg->capacity_factor > 0.0f) return MOE_ERR_UNSUPPORTED;
    e->R = n_ranks;
    e->epr = N / n_ranks;
    e->n_chunks = (int)std::max<int64_t>(1, cdiv(T, kChunk));
    size_t off = align256(e->P.total);
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align256(off + bytes);
        return o;
    };
    e->cc = take((size_t)e->n_chunks * n_ranks * 4);
    e->cb = take((size_t)e->n_chunks * n_ranks * 4);
    e->offsets = take((size_t)(n_ranks + 1) * 4);
    e->rowoff = take((size_t)(n_ranks + 1) * 4);
    e->live = take((size_t)n_ranks * 4);
    e->perm = take((size_t)(cdiv(T * e->P.K + (int64_t)n_ranks * (kRowAlign - 1), kRowAlign) * kRowAlign) * 4);
    e->total = off;
    return MOE_OK;
}
}  // namespace

size_t moe_ep_workspace_size(const moe_config *cfg, int32_t n_ranks, int64_t T) {
    EpPlan e;
    if (make_ep_plan(cfg, n_ranks, T, &e) != MOE_OK) return 0;
    return e.total;
}

int moe_ep_dispatch(const moe_config *cfg, int32_t n_ranks, const void *x, int64_t T, const moe_weights *w,
                    void *send_x, int32_t *send_expert, float *send_w, int32_t *send_counts, int32_t *send_pos,
                    moe_aux *aux, void *ws, size_t ws_bytes, moe_stream_t stream) {
    EpPlan e;
    MOE_TRY(make_ep_plan(cfg, n_ranks, T, &e));
    const Plan &P = e.P;
    MOE_TRY(check_weights(P, w, false));
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (!send_counts) return MOE_ERR_INVALID_ARG;
    if (T == 0) {
        if (cudaMemsetAsync(send_counts, 0, (size_t)n_ranks * 4, s) != cudaSuccess) return MOE_ERR_CUDA;
        return zero_aux(P, aux, s);
    }
    if (!x || !aligned16(x) || !send_x || !aligned16(send_x) || !send_expert || !send_w || !send_pos)
        return MOE_ERR_INVALID_ARG;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return MOE_ERR_INVALID_ARG;
    if (ws_bytes < e.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    DeviceInfo *dev = nullptr;
    MOE_TRY(device_info(&dev));
    Bufs b{static_cast<char *>(ws), &P};
    float *logits = b.at<float>(P.logits);
    int *idx = b.at<int>(P.idx);
    float *tw = b.at<float>(P.w);
    MOE_TRY(zero_counters(P, b, s));
    if (P.tc_router) {
        MOE_TRY(stage_route_tc(P, b, x, w, logits, idx, tw, nullptr, aux, nullptr, s));
    } else {
        MOE_TRY(stage_route(P, b, x, w, logits, idx, tw, *dev, s));
        if (aux) MOE_TRY(stage_aux(P, b, logits, idx, tw, aux, s));
    }
    // group the (token, slot) pairs by the rank holding their expert: chunk
    // histograms, the scan (send counts and offsets), the packing
    const int R = e.R;
    int *cc = b.at<int>(e.cc), *cb = b.at<int>(e.cb), *offs = b.at<int>(e.offsets);
    unsigned *ctr = b.at<unsigned>(P.counters);
    hist_kernel<<<e.n_chunks, 256, (size_t)R * 4, s>>>(idx, T * P.K, kChunk * P.K, R, e.epr, cc);
    MOE_TRY(check_launch());
    scan_kernel<<<(unsigned)cdiv(R, 32), 1024, 0, s>>>(cc, e.n_chunks, R, T * P.K, INT32_MAX, cb, send_counts, offs,
                                                       b.at<int>(e.rowoff), b.at<int>(e.perm), nullptr, ctr + 5,
                                                       b.at<int>(e.live), reinterpret_cast<int *>(ctr) + 6);
    MOE_TRY(check_launch());
    const size_t smem = (size_t)(R + kChunk * P.K) * 4;
    if (P.dtype == MOE_F32)
        ep_pack_kernel<float><<<e.n_chunks, 256, smem, s>>>(static_cast<const float *>(x), (int)T, P.D, P.K, R, e.epr,
                                                             kChunk, idx, tw, cb, offs, static_cast<float *>(send_x),
                                                             send_expert, send_w, send_pos);
    else
        ep_pack_kernel<__nv_bfloat16><<<e.n_chunks, 256, smem, s>>>(
            static_cast<const __nv_bfloat16 *>(x), (int)T, P.D, P.K, R, e.epr, kChunk, idx, tw, cb, offs,
            static_cast<__nv_bfloat16 *>(send_x), send_expert, send_w, send_pos);
    return check_launch();
}

size_t moe_ep_experts_workspace_size(const moe_config *cfg_local, int64_t M) {
    Plan P;
    if (make_plan(cfg_local, M, &P, true) != MOE_OK || P.K != 1) return 0;
    return P.total;
}

int moe_ep_experts(const moe_config *cfg_local, const void *recv_x, int64_t M, const int32_t *recv_expert,
                   const float *recv_w, const moe_weights *w_local, float *z_out, void *ws, size_t ws_bytes,
                   moe_stream_t stream) {
    if (!cfg_local || cfg_local->TopK != 1 || cfg_local->n_shared || cfg_local->capacity_factor > 0.0f)
        return MOE_ERR_INVALID_ARG;
    if (M > 0 && (!recv_expert || !recv_w)) return MOE_ERR_INVALID_ARG;
    return forward_impl(cfg_local, recv_x, M, w_local, z_out, MOE_F32, nullptr, ws, ws_bytes,
                        reinterpret_cast<cudaStream_t>(stream), nullptr, recv_expert, recv_w);
}

int moe_ep_combine(const moe_config *cfg, const float *z_back, int64_t T, const int32_t *send_pos, void *y,
                   int32_t y_dtype, moe_stream_t stream) {
    Plan P;
    MOE_TRY(make_plan(cfg, T, &P));
    if (y_dtype != MOE_F32 && y_dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!z_back || !send_pos || !y || !aligned16(z_back) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
    DeviceInfo *dev = nullptr;
    MOE_TRY(device_info(&dev));
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int64_t nq = T * (P.D / 4);
    const int grid = (int)std::min<int64_t>(cdiv(nq, 256), (int64_t)dev->sms * 8);
    if (y_dtype == MOE_F32)
        return launch_pdl(combine_kernel<float>, dim3(grid), dim3(256), 0, s, z_back, T * P.K, T, P.D, P.K,
                          (const int *)send_pos, 1, (const float *)nullptr, static_cast<float *>(y));
    return launch_pdl(combine_kernel<__nv_bfloat16>, dim3(grid), dim3(256), 0, s, z_back, T * P.K, T, P.D, P.K,
                      (const int *)send_pos, 1, (const float *)nullptr, static_cast<__nv_bfloat16 *>(y));
}

// ---------------------------------------------------------------- backward
}  // extern "C"

namespace {
struct BwdPlan {
    Plan P;
    int rows1;
    size_t g, pre, dhr, h, dA, gw, dxp, dw, ds, dxr, part, f, dimp, total;
};

int make_bwd_plan(const moe_config *cfg, int64_t T, BwdPlan *b) {
    MOE_TRY(make_plan(cfg, T, &b->P));
    const Plan &P = b->P;
    if (P.n_shared || cfg->capacity_factor > 0.0f) return MOE_ERR_UNSUPPORTED;
    b->rows1 = P.act == MOE_ACT_SWIGLU ? 2 * P.H : P.H;
    size_t off = align256(P.total);
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align256(off + bytes);
        return o;
    };
    const size_t R = (size_t)P.rows_cap;
    b->g = take(R * P.D * 4);
    b->pre = take(R * b->rows1 * 4);
    b->dhr = take(R * P.H * 4);
    b->h = take(R * P.H * 4);
    b->dA = take(R * b->rows1 * 4);
    b->gw = take(R * P.D * 4);
    b->dxp = take(R * P.D * 4);
    b->dw = take(R * 4);
    b->ds = take((size_t)T * P.N * 4);
    b->dxr = take((size_t)T * P.D * 4);
    b->part = take((size_t)(3 * P.N + 1) * 8);
    b->f = take((size_t)P.N * 4);
    b->dimp = take((size_t)P.N * 4);
    b->total = off;
    return MOE_OK;
}

template <typename TA, typename TB>
int launch_gemm_strided(const bwd::GemmParams<TA, TB> &p, int64_t m_extent, cudaStream_t s) {
    if (m_extent <= 0 || p.N <= 0) return MOE_OK;
    const dim3 grid((unsigned)cdiv(m_extent, bwd::TM), (unsigned)cdiv(p.N, bwd::TN),
                    (unsigned)(p.mode == bwd::KGRP ? p.groups : 1));
    bwd::gemm_strided_kernel<TA, TB><<<grid, 256, 0, s>>>(p);
    return check_launch();
}

// The backward GEMMs for one element type of x and the weights (float or bf16).
template <typename DT>
int backward_gemms(const BwdPlan &B, const Bufs &b, const void *x, const moe_weights *w, moe_grads *gr, int phase,
                   cudaStream_t s) {
    const Plan &P = B.P;
    const int D = P.D, H = P.H, N = P.N, R1 = B.rows1;
    const DT *xp = b.at<DT>(P.x_perm);
    const DT *W1 = static_cast<const DT *>(w->W1);
    const DT *W2 = static_cast<const DT *>(w->W2);
    const DT *Wg = static_cast<const DT *>(w->W_g);
    const int *ro = b.at<int>(P.row_offsets), *cn = b.at<int>(P.counts);
    if (phase == 0) {
        // pre = W1 x (per permuted row), dhr = W2^T dy
        bwd::GemmParams<DT, DT> g1{};
        g1.A = xp; g1.a_sm = D; g1.a_sk = 1;
        g1.B = W1; g1.b_sn = D; g1.b_sk = 1; g1.b_group = (int64_t)R1 * D;
        g1.C = b.at<float>(B.pre); g1.c_sm = R1; g1.c_sn = 1;
        g1.N = R1; g1.K = D; g1.row_offsets = ro; g1.counts = cn; g1.groups = N; g1.mode = bwd::ROWS;
        MOE_TRY(launch_gemm_strided(g1, P.rows_cap, s));
        bwd::GemmParams<float, DT> g2{};
        g2.A = b.at<float>(B.g); g2.a_sm = D; g2.a_sk = 1;
        g2.B = W2; g2.b_sn = 1; g2.b_sk = H; g2.b_group = (int64_t)D * H;
        g2.C = b.at<float>(B.dhr); g2.c_sm = H; g2.c_sn = 1;
        g2.N = H; g2.K = D; g2.row_offsets = ro; g2.counts = cn; g2.groups = N; g2.mode = bwd::ROWS;
        return launch_gemm_strided(g2, P.rows_cap, s);
    }
    // dx_perm = W1^T da; dxr = W_g ds; dW2 = sum w dy h^T; dW1 = sum da x^T; dW_g = sum x ds^T
    bwd::GemmParams<float, DT> g3{};
    g3.A = b.at<float>(B.dA); g3.a_sm = R1; g3.a_sk = 1;
    g3.B = W1; g3.b_sn = 1; g3.b_sk = D; g3.b_group = (int64_t)R1 * D;
    g3.C = b.at<float>(B.dxp); g3.c_sm = D; g3.c_sn = 1;
    g3.N = D; g3.K = R1; g3.row_offsets = ro; g3.counts = cn; g3.groups = N; g3.mode = bwd::ROWS;
    MOE_TRY(launch_gemm_strided(g3, P.rows_cap, s));
    bwd::GemmParams<float, DT> g6{};
    g6.A = b.at<float>(B.ds); g6.a_sm = N; g6.a_sk = 1;
    g6.B = Wg; g6.b_sn = N; g6.b_sk = 1;
    g6.C = b.at<float>(B.dxr); g6.c_sm = D; g6.c_sn = 1;
    g6.M = (int)P.T; g6.N = D; g6.K = N; g6.mode = bwd::DENSE;
    MOE_TRY(launch_gemm_strided(g6, P.T, s));
    bwd::GemmParams<float, float> g4{};
    g4.A = b.at<float>(B.gw); g4.a_sm = 1; g4.a_sk = D;
    g4.B = b.at<float>(B.h); g4.b_sn = 1; g4.b_sk = H;
    g4.C = gr->dW2; g4.c_sm = H; g4.c_sn = 1; g4.c_group = (int64_t)D * H;
    g4.M = D; g4.N = H; g4.row_offsets = ro; g4.counts = cn; g4.groups = N; g4.mode = bwd::KGRP;
    MOE_TRY(launch_gemm_strided(g4, D, s));
    bwd::GemmParams<float, DT> g5{};
    g5.A = b.at<float>(B.dA); g5.a_sm = 1; g5.a_sk = R1;
    g5.B = xp; g5.b_sn = 1; g5.b_sk = D;
    g5.C = gr->dW1; g5.c_sm = D; g5.c_sn = 1; g5.c_group = (int64_t)R1 * D;
    g5.M = R1; g5.N = D; g5.row_offsets = ro; g5.counts = cn; g5.groups = N; g5.mode = bwd::KGRP;
    MOE_TRY(launch_gemm_strided(g5, R1, s));
    bwd::GemmParams<DT, float> g7{};
    g7.A = static_cast<const DT *>(x); g7.a_sm = 1; g7.a_sk = D;
    g7.B = b.at<float>(B.ds); g7.b_sn = 1; g7.b_sk = N;
    g7.C = gr->dW_g; g7.c_sm = N; g7.c_sn = 1;
    g7.M = D; g7.N = N; g7.K = (int)P.T; g7.mode = bwd::DENSE;
    return launch_gemm_strided(g7, D, s);
}
}  // namespace

extern "C" {

size_t moe_backward_workspace_size(const moe_config *cfg, int64_t T) {
    BwdPlan B;
    if (make_bwd_plan(cfg, T, &B) != MOE_OK) return 0;
    return B.total;
}

int moe_backward(const moe_config *cfg, const void *x, int64_t T, const moe_weights *w, const float *dy,
                 float alpha_switch, float alpha_importance, moe_grads *gr, void *ws, size_t ws_bytes,
                 moe_stream_t stream) {
    BwdPlan B;
    MOE_TRY(make_bwd_plan(cfg, T, &B));
    const Plan &P = B.P;
    MOE_TRY(check_weights(P, w, true));
    if (!gr || !gr->dx || !gr->dW_g || !gr->dW1 || !gr->dW2) return MOE_ERR_INVALID_ARG;
    if (P.has_bias && (!gr->db1 || !gr->db2)) return MOE_ERR_INVALID_ARG;
    if (!(alpha_switch == alpha_switch) || !(alpha_importance == alpha_importance)) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int D = P.D, H = P.H, N = P.N, K = P.K, R1 = B.rows1;
    if (T == 0) {
        const size_t zs[] = {(size_t)D * N * 4, (size_t)N * R1 * D * 4, (size_t)N * D * H * 4};
        void *zp[] = {gr->dW_g, gr->dW1, gr->dW2};
        for (int i = 0; i < 3; ++i)
            if (cudaMemsetAsync(zp[i], 0, zs[i], s) != cudaSuccess) return MOE_ERR_CUDA;
        if (gr->db_g && cudaMemsetAsync(gr->db_g, 0, (size_t)N * 4, s) != cudaSuccess) return MOE_ERR_CUDA;
        if (P.has_bias && (cudaMemsetAsync(gr->db1, 0, (size_t)N * H * 4, s) != cudaSuccess ||
                           cudaMemsetAsync(gr->db2, 0, (size_t)N * D * 4, s) != cudaSuccess))
            return MOE_ERR_CUDA;
        return MOE_OK;
    }
    if (!x || !aligned16(x) || !dy || !aligned16(dy) || !aligned16(gr->dx)) return MOE_ERR_INVALID_ARG;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return MOE_ERR_INVALID_ARG;
    if (ws_bytes < B.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    DeviceInfo *dev = nullptr;
    MOE_TRY(device_info(&dev));
    Bufs b{static_cast<char *>(ws), &P};
    float *logits = b.at<float>(P.logits);
    int *idx = b.at<int>(P.idx);
    float *tw = b.at<float>(P.w);
    // the forward's routing and dispatch
    MOE_TRY(zero_counters(P, b, s));
    if (P.tc_router) {
        MOE_TRY(stage_route_tc(P, b, x, w, logits, idx, tw, nullptr, nullptr, nullptr, s));
    } else {
        MOE_TRY(stage_route(P, b, x, w, logits, idx, tw, *dev, s));
        MOE_TRY(stage_scan(P, b, nullptr, s));
    }
    MOE_TRY(stage_permute(P, b, x, nullptr, *dev, s));
    const int grid_ew = (int)std::min<int64_t>(cdiv(P.rows_cap * (D / 4), 256), (int64_t)dev->sms * 8);
    const int *row_end = b.at<int>(P.row_offsets) + N;   // rows past it are outside every segment
    bwd::gather_rows_kernel<<<grid_ew, 256, 0, s>>>(dy, P.rows_cap, D, K, b.at<int>(P.perm_slot), row_end,
                                                    b.at<float>(B.g));
    MOE_TRY(check_launch());
    if (P.dtype == MOE_F32) MOE_TRY(backward_gemms<float>(B, b, x, w, gr, 0, s));
    else MOE_TRY(backward_gemms<__nv_bfloat16>(B, b, x, w, gr, 0, s));
    const bool swiglu = P.act == MOE_ACT_SWIGLU;
    bwd::act_backward_kernel<<<(unsigned)cdiv(P.rows_cap * 32, 256), 256, 0, s>>>(
        b.at<float>(B.pre), b.at<float>(B.dhr), b.at<float>(B.g), P.rows_cap, D, H, swiglu ? 1 : 0,
        b.at<int>(P.perm_slot), row_end, idx, tw, swiglu ? nullptr : w->b1, swiglu ? nullptr : w->b2, b.at<float>(B.h),
        b.at<float>(B.dA), b.at<float>(B.gw), b.at<float>(B.dw));
    MOE_TRY(check_launch());
    // the auxiliary losses' batch quantities, then the router scores' gradient
    unsigned long long *part = b.at<unsigned long long>(B.part);
    if (cudaMemsetAsync(part, 0, (size_t)(3 * N + 1) * 8, s) != cudaSuccess) return MOE_ERR_CUDA;
    aux_partials_kernel<<<(int)std::max<int64_t>(1, std::min<int64_t>(cdiv(T, 8), (int64_t)dev->sms * 4)), 256,
                          (size_t)3 * N * 8, s>>>(logits, idx, tw, (int)T, N, K, part);
    MOE_TRY(check_launch());
    bwd::aux_grad_prep_kernel<<<1, 32, 0, s>>>(N, K, reinterpret_cast<const long long *>(part), b.at<float>(B.f),
                                               b.at<float>(B.dimp));
    MOE_TRY(check_launch());
    bwd::router_backward_kernel<<<(unsigned)cdiv(T * 32, 256), 256, 0, s>>>(
        logits, idx, tw, b.at<int>(P.slot_row), b.at<float>(B.dw), b.at<float>(B.f), b.at<float>(B.dimp), (int)T, N,
        K, alpha_switch, alpha_importance, b.at<float>(B.ds));
    MOE_TRY(check_launch());
    if (P.dtype == MOE_F32) MOE_TRY(backward_gemms<float>(B, b, x, w, gr, 1, s));
    else MOE_TRY(backward_gemms<__nv_bfloat16>(B, b, x, w, gr, 1, s));
    // dx[t] = sum_j dx_perm[row of (t, j)] in slot order + W_g ds[t]
    const int grid_c = (int)std::min<int64_t>(cdiv(T * (D / 4), 256), (int64_t)dev->sms * 8);
    combine_kernel<float><<<grid_c, 256, 0, s>>>(b.at<float>(B.dxp), (int64_t)P.rows_cap, T, D, K, b.at<int>(P.slot_row), 1,
                                                 b.at<float>(B.dxr), gr->dx);
    MOE_TRY(check_launch());
    // bias gradients: column sums over each expert's rows (row order), over the tokens for b_g
    if (P.has_bias) {
        bwd::column_sums_kernel<<<dim3((unsigned)cdiv(D, 256), (unsigned)N), 256, 0, s>>>(
            b.at<float>(B.gw), D, D, b.at<int>(P.row_offsets), b.at<int>(P.counts), 0, gr->db2);
        MOE_TRY(check_launch());
        bwd::column_sums_kernel<<<dim3((unsigned)cdiv(H, 256), (unsigned)N), 256, 0, s>>>(
            b.at<float>(B.dA), R1, H, b.at<int>(P.row_offsets), b.at<int>(P.counts), 0, gr->db1);
        MOE_TRY(check_launch());
    }
    if (gr->db_g) {
        bwd::column_sums_kernel<<<dim3((unsigned)cdiv(N, 256), 1), 256, 0, s>>>(b.at<float>(B.ds), N, N, nullptr,
                                                                                 nullptr, T, gr->db_g);
        MOE_TRY(check_launch());
    }
    return MOE_OK;
}

int64_t moe_total_params(const moe_config *c) {
    Plan P;
    if (make_plan(c, 0, &P) != MOE_OK) return -1;
    const int64_t D = P.D, H = P.H, N = P.N;
    const int64_t ex = P.act == MOE_ACT_SWIGLU ? 3 * D * H : 2 * D * H + (P.has_bias ? H + D : 0);
    return D * N + (N + P.n_shared) * ex;
}

int64_t moe_active_params(const moe_config *c) {
    Plan P;
    if (make_plan(c, 0, &P) != MOE_OK) return -1;
    const int64_t D = P.D, H = P.H, N = P.N, K = P.K;
    const int64_t ex = P.act == MOE_ACT_SWIGLU ? 3 * D * H : 2 * D * H + (P.has_bias ? H + D : 0);
    return D * N + (K + P.n_shared) * ex;
}

int moe_get_device_status(void) {
    if (cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_status, sizeof v) != cudaSuccess) return MOE_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_status, &zero, sizeof zero) != cudaSuccess) return MOE_ERR_CUDA;
    return v;
}

int64_t moe_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char *moe_error_string(int code) {
    switch (code) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
        case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
        case MOE_ERR_CUDA: return "CUDA runtime error";
        case MOE_ERR_DEVICE_TIMEOUT: return "a kernel's bounded wait ran out";
        case MOE_ERR_DEVICE_BOUNDS: return "a kernel found an index out of range";
        default: return "unknown error";
    }
}

// ---------------------------------------------------------------- statistics without a workspace
// moe_aux_stats_noalloc keeps its scratch in one fixed array inside the library
// instead of a caller-provided workspace: a 256-byte block of counters that
// must be zero when the kernels start (cleared on every call), then the three
// per-block partial arrays of the statistics kernels.  Every call on a device
// uses the same array, so two calls whose kernels overlap (other streams,
// other host threads) corrupt each other's results.
}  // extern "C"

namespace {
__device__ __align__(256) unsigned char g_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];

constexpr int kNoallocMaxDevices = 64;
std::mutex g_noalloc_mutex;
void *g_noalloc_ptr[kNoallocMaxDevices];

// Device address of g_noalloc_scratch on the current device, looked up once per
// device (the first call on it) with that device current.
int noalloc_scratch(char **out) {
    int d = -1;
    if (cudaGetDevice(&d) != cudaSuccess) return MOE_ERR_CUDA;
    if (d < 0 || d >= kNoallocMaxDevices) return MOE_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_ptr[d]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return MOE_ERR_CUDA;
        g_noalloc_ptr[d] = ptr;
    }
    *out = static_cast<char *>(g_noalloc_ptr[d]);
    return MOE_OK;
}
}  // namespace

extern "C" {

int moe_aux_stats_noalloc(const moe_config *cfg, int64_t T, const float *logits, const int32_t *topk_idx,
                          const float *topk_w, moe_aux *out, moe_stream_t stream) {
    Plan P;
    MOE_TRY(make_plan(cfg, T, &P));
    if (!out) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!logits || !topk_idx || !topk_w)) return MOE_ERR_INVALID_ARG;
    // the same kernels as moe_aux_stats, with their scratch moved into the fixed array
    const size_t part = align256((size_t)P.aux_blocks * P.N * 4);
    if (256 + 3 * part > (size_t)MOE_NOALLOC_SCRATCH_BYTES) return MOE_ERR_WORKSPACE_TOO_SMALL;
    char *scratch = nullptr;
    MOE_TRY(noalloc_scratch(&scratch));
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (T == 0) return zero_aux(P, out, s);
    DeviceInfo *dev = nullptr;
    MOE_TRY(device_info(&dev));
    Plan Q = P;
    Q.n_shared = 0;   // nothing outside the fixed array is written
    Q.counters = 0;
    Q.counters_bytes = 256;
    Q.aux_p = 256;
    Q.aux_i = 256 + part;
    Q.aux_c = 256 + 2 * part;
    Q.total = 256 + 3 * part;
    Bufs b{scratch, &Q};
    MOE_TRY(zero_counters(Q, b, s));
    return stage_aux(Q, b, logits, topk_idx, topk_w, out, s);
}

int moe_selftest_wait_timeout(int64_t timeout_ns, moe_stream_t stream) {
    if (timeout_ns <= 0 || timeout_ns > 10000000000ll) return MOE_ERR_INVALID_ARG;
    wait_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>((uint64_t)timeout_ns);
    return check_launch();
}

}  // extern "C"
