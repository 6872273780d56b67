// moe_decode_fused.cuh -- the whole layer for a few tokens in one persistent,
// cooperative kernel.
//
// With a handful of tokens the layer's time is the time it takes to stream the
// live experts' weights from HBM (the Transformers-v5 MoE article's remark that
// small batches want another strategy than grouped_mm; its gpt-oss decode
// estimate).  Separate launches for routing, dispatch, the two expert GEMMs
// and the combine leave that stream idle across every kernel boundary and
// every dependent table load, so one kernel runs all of it, with grid-wide
// barriers where a step needs every CTA's results:
//   R1  slab scores: CTAs 0..S-1 each multiply a slab of W_g rows (staged in
//       shared memory) with the same columns of every token
//   --- barrier 1
//   R2  CTA t finishes token t: the slab sums in slab order (+ b_g), the K
//       best experts, the gate weights over them ("MoE(Mixture of Experts)",
//       section (2); Shazeer article, gating section), the full softmax
//   --- barrier 2
//   R3  every CTA builds the same dispatch tables in shared memory from the
//       top-k (stable counting sort by expert; capacity applied); CTA 0 writes
//       them and the statistics to the workspace; the kept (token, slot) rows
//       are copied to x_perm, spread over the CTAs
//   --- barrier 3 (x_perm complete): only the token-row loads wait for it
//   U   up projection: swap-AB tcgen05 tiles (128 weight rows x the expert's
//       token rows, moe_gemm_decode.cuh), stream-K over live experts x tiles x
//       K blocks, GELU / SwiGLU epilogue -> h
//   --- barrier 4 (h complete): only the hidden-row loads wait for it, so the
//       down projection's weight tiles stream in while the up projection ends
//   D   down projection + gate scale -> z (one row per slot)
//   --- barrier 5 (z complete), epilogue warps only
//   C   the combine, shared by all CTAs: y[t] = the kept slots' z rows of token
//       t in slot order, with many loads in flight per thread
// The cooperative launch keeps every CTA resident, so the barriers cannot wait
// on a CTA that never runs; every wait is still bounded by time (status word
// MOE_STATUS_TIMEOUT on expiry, then the CTA drains and returns).
#pragma once

#include "moe_common.cuh"
#include "moe_gemm_decode.cuh"
#include "moe_route.cuh"

namespace moe {
namespace dfu {

constexpr int BM = dec::BM;   // weight rows per tile
constexpr int BK = dec::BK;
constexpr int kThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue; all six route first
constexpr int kEpiWarps = 4;
constexpr int kMaxT = 64;
constexpr int kMaxN = 32;
constexpr int kMaxSlots = kMaxT * 32;   // T * K
constexpr int kMaxSlabs = 32;

struct Params {
    int T, D, H, N, K, capacity;
    int slab_rows, n_slabs;        // R1: W_g rows per slab (a multiple of 8), slabs
    const __nv_bfloat16 *x;        // [T, D]
    const __nv_bfloat16 *Wg;       // [D, N]
    const float *bg, *bsel;        // [N] or nullptr
    const float *b1, *b2;          // GELU expert biases or nullptr
    float *logits;                 // [T, N]
    int *topk_idx;                 // [T, K]
    float *topk_w;                 // [T, K]
    int *counts, *offsets, *row_offsets, *perm_slot, *slot_row, *live, *n_live;
    __nv_bfloat16 *x_perm, *h;     // [rows_cap, D], [rows_cap, H]
    float *z;                      // [T * K, D], slot rows
    float *slab;                   // [n_slabs][T][32]
    float *tok_p;                  // [T][32] full softmax of each token
    unsigned *bar;                 // arrivals of grid barriers 1-3 (zero at launch)
    unsigned *bar4;                // arrivals of grid barrier 4 (zero at launch): a counter of its own,
                                   // since CTAs without up-projection work arrive there before barrier 3
    unsigned *tk_up, *tk_down;     // stream-K tile tickets [split_cap] (zero at launch)
    unsigned *bar5;                // arrivals of grid barrier 5 (z complete, zero at launch)
    float *part;                   // stream-K partials [split_cap][2][BM][NT]
    int split_cap;
    void *y;                       // [T, D]
    int y_bf16;
    int *aux_counts;
    float *aux_importance, *aux_p_mean, *aux_scalars;
    uint64_t timeout_ns;
};

template <int NT, int EPI_UP>
struct Shape {
    static constexpr uint32_t kABytes = BM * BK * 2;
    static constexpr uint32_t kBBytes = NT * BK * 2;
    static constexpr uint32_t kStageBytes = kABytes + kBBytes;
    static constexpr uint32_t kEpiBytes = EPI_UP == dec::EPI_SWIGLU ? (64 * NT * 4 + NT * 64 * 2) : NT * 128 * 2;
    static constexpr uint32_t kTableBytes = 2 * kMaxSlots * 2 + 8 * 40 * 4;
    static constexpr int kStages0 =
        (int)((220 * 1024 - 1024 - kEpiBytes - kTableBytes - 256) / kStageBytes);
    static constexpr int kStages = kStages0 > 16 ? 16 : kStages0;   // as many weight tiles in flight as fit
    static constexpr uint32_t kRingBytes = kStages * kStageBytes;
    static constexpr uint32_t kTmemCols = 2 * NT < 32 ? 32 : 2 * NT;
    static constexpr size_t kSmem = 1024 + (size_t)kRingBytes + kEpiBytes + kTableBytes + (2 * kStages + 6) * 8 + 64;
};

// ------------------------------------------------------------------ grid barrier
__device__ __forceinline__ void grid_arrive(unsigned *bar) {
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(bar) : "memory");
}
// Until at least `target` arrivals, for at most timeout_ns (then status, false).
__device__ __forceinline__ bool grid_wait(const unsigned *bar, unsigned target, uint64_t timeout_ns) {
    if (dec::ld_acquire_u32(bar) >= target) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (dec::ld_acquire_u32(bar) >= target) return true;
        if (globaltimer_ns() - t0 > timeout_ns) {
            set_status(kStatusTimeout);
            return false;
        }
    }
}
// Generic-proxy global writes before / after async-proxy (TMA) accesses.
__device__ __forceinline__ void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

// Every thread: the CTA's writes so far are released, the whole grid arrives,
// every CTA waits for all arrivals of barrier number `k` (1-based).
__device__ __forceinline__ bool grid_sync_all(const Params &p, unsigned k, int *s_flag) {
    __syncthreads();
    if (threadIdx.x == 0) {
        fence_proxy_async_global();
        grid_arrive(p.bar);
        *s_flag = grid_wait(p.bar, k * gridDim.x, p.timeout_ns) ? 1 : 0;
    }
    __syncthreads();
    return *s_flag != 0;
}

// Tables the routing leaves in every CTA's shared memory.
struct Tables {
    int16_t *row;   // [T*K] permuted row of each slot, -1 if dropped
    int16_t *ent;   // [kept total] slots grouped by expert (kept only), slot order inside an expert
    int *cnt;       // [32] routed
    int *kept;      // [32]
    int *rowoff;    // [33] padded segment starts (multiples of 128)
    int *koff;      // [33] exclusive scan of kept
    int *live;      // [32]
    int *nlive;     // [1]
};

// ------------------------------------------------------------------ routing phases
template <int NT, int EPI_UP>
__device__ __forceinline__ void route_r1(const Params &p, uint8_t *scratch) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int T = p.T, N = p.N, D = p.D, R = p.slab_rows;
    const int c = blockIdx.x;
    const int d0 = c * R, nd = min(D, d0 + R) - d0;
    if (nd <= 0) return;
    float *xs = reinterpret_cast<float *>(scratch);            // [T][R]
    float *ws = xs + (size_t)T * R;                            // [R][32]
    // 16-byte loads: slab rows start at multiples of 8 elements and D, N * 8 are multiples of 8
    const int xv = nd / 8;
    for (int i = tid; i < T * xv; i += kThreads) {
        const int t = i / xv, v = i - t * xv;
        const uint4 q = __ldg(reinterpret_cast<const uint4 *>(p.x + (size_t)t * D + d0) + v);
        float f[8];
        Vec16<__nv_bfloat16>::unpack(q, f);
#pragma unroll
        for (int k = 0; k < 8; ++k) xs[t * R + v * 8 + k] = f[k];
    }
    const int wtot = nd * N;   // W_g slab is contiguous: rows d0.., N experts each
    for (int i = tid * 8; i < wtot; i += kThreads * 8) {
        float f[8];
        if (i + 8 <= wtot && ((d0 * N) % 8) == 0) {
            Vec16<__nv_bfloat16>::unpack(__ldg(reinterpret_cast<const uint4 *>(p.Wg + (size_t)d0 * N + i)), f);
        } else {
#pragma unroll
            for (int k = 0; k < 8; ++k) f[k] = i + k < wtot ? __bfloat162float(p.Wg[(size_t)d0 * N + i + k]) : 0.f;
        }
#pragma unroll
        for (int k = 0; k < 8; ++k)
            if (i + k < wtot) {
                const int dd = (i + k) / N, e = (i + k) - dd * N;
                ws[dd * 32 + e] = f[k];
            }
    }
    __syncthreads();
    // partial scores of the slab: warp w takes tokens w, w + 6, ...; lane = expert;
    // four running sums over the slab rows (k mod 4), added in a fixed order
    for (int t = warp; t < T; t += kThreads / 32) {
        const float *xr = xs + (size_t)t * R;
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
        int k = 0;
        for (; k + 4 <= nd; k += 4) {
            a0 = fmaf(xr[k], ws[k * 32 + lane], a0);
            a1 = fmaf(xr[k + 1], ws[(k + 1) * 32 + lane], a1);
            a2 = fmaf(xr[k + 2], ws[(k + 2) * 32 + lane], a2);
            a3 = fmaf(xr[k + 3], ws[(k + 3) * 32 + lane], a3);
        }
        for (; k < nd; ++k) a0 = fmaf(xr[k], ws[k * 32 + lane], a0);
        const float v = (a0 + a1) + (a2 + a3);
        p.slab[((size_t)c * T + t) * 32 + lane] = lane < N ? v : 0.f;   // lanes past N hold no expert
    }
}

// R2 for token t by one warp: the slabs' scores sl[c * ld + lane] (c < n_slabs)
// added in slab order, bias, NaN ranked as -inf, the top k (ties to the lower
// index) on the selection values, gate weights, the full softmax.  With out the
// results go to the workspace (logits, topk_idx, topk_w, tok_p); with s_idx the
// selected experts also go there (shared memory, read by R3).
__device__ __forceinline__ void r2_token(const Params &p, int t, const float *sl, int ld, bool out, int *s_idx) {
    const int lane = threadIdx.x & 31;
    const int N = p.N, K = p.K;
    const bool live = lane < N;
    float s = 0.f;
    for (int c = 0; c < p.n_slabs; ++c) s += sl[c * ld + lane];   // slab order
    if (live) {
        if (p.bg) s += __ldg(p.bg + lane);
        if (s != s) {
            set_status(kStatusNanLogit);
            s = -INFINITY;
        }
        if (out) p.logits[(size_t)t * N + lane] = s;
    } else {
        s = -INFINITY;
    }
    int slot_e;
    float slot_w;
    if (segment_topk<32>(sel_value(p.bsel, s, lane, live), s, lane, !live, K, lane, lane, slot_e, slot_w)) {
        if (out) {
            p.topk_idx[(size_t)t * K + lane] = slot_e;
            p.topk_w[(size_t)t * K + lane] = slot_w;
        }
        if (s_idx) s_idx[t * K + lane] = slot_e;
    }
    float mx = s;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float ex = (live && mx != -INFINITY) ? expf(s - mx) : 0.f;
    float zs = ex;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) zs += __shfl_xor_sync(0xffffffffu, zs, o);
    if (out) p.tok_p[(size_t)t * 32 + lane] = zs > 0.f ? ex / zs : 0.f;
}

// R2 for token t = blockIdx.x: every thread of the CTA loads the slabs' scores
// into shared memory at once (one round trip), warp 0 finishes the token.
__device__ __forceinline__ void route_r2(const Params &p, uint8_t *scratch) {
    const int tid = threadIdx.x;
    const int t = blockIdx.x;
    float *sl = reinterpret_cast<float *>(scratch);   // [n_slabs][32]
    for (int i = tid; i < p.n_slabs * 32; i += kThreads)
        sl[i] = __ldcg(p.slab + ((size_t)(i >> 5) * p.T + t) * 32 + (i & 31));
    __syncthreads();
    if (tid < 32) r2_token(p, t, sl, 32, true, nullptr);
}

// R2 for every token in every CTA (few tokens): all slabs' scores loaded at once,
// each warp finishes tokens warp, warp + 6, ...; the selected experts land in
// R3's index array, CTA 0 also writes the workspace.  Replaces R2 and the grid
// barrier after it: every CTA derives the same tables from the same sums.
constexpr int kAllR2T = 12;   // up to two tokens per warp
__device__ __forceinline__ int r2_all_offset() { return (3 * kMaxSlots + kMaxT * 32) * 4; }
__device__ __forceinline__ void route_r2_all(const Params &p, uint8_t *scratch) {
    const int tid = threadIdx.x, warp = tid >> 5;
    int *s_idx = reinterpret_cast<int *>(scratch);                          // R3's index array
    float *sl = reinterpret_cast<float *>(scratch + r2_all_offset());       // [n_slabs][T][32]
    const int n = p.n_slabs * p.T * 32;
    for (int i = tid; i < n; i += kThreads) sl[i] = __ldcg(p.slab + i);
    __syncthreads();
    for (int t = warp; t < p.T; t += kThreads / 32) r2_token(p, t, sl + t * 32, p.T * 32, blockIdx.x == 0, s_idx);
    __syncthreads();
}

// CTA 0 after R3: the workspace tables (moe_get_workspace_layout) and the
// statistics of the router's choice, by threads tid < nth of the CTA that sync()
// brings together; s_idx holds the T*K selected experts, stat has room for
// 64 + T*K + 32*T floats.
template <class Sync>
__device__ __forceinline__ void r3_publish(const Params &p, const Tables &tb, const int *s_idx, float *stat, int tid,
                                           int nth, Sync sync) {
    const int warp = tid >> 5, lane = tid & 31;
    const int N = p.N, TK = p.T * p.K;
    // the workspace tables (moe_get_workspace_layout) and the statistics
    for (int e = tid; e < N; e += nth) {
        p.counts[e] = tb.kept[e];
        p.offsets[e] = tb.koff[e];
        p.row_offsets[e] = tb.rowoff[e];
    }
    if (tid == 0) {
        p.offsets[N] = tb.koff[N - 1] + tb.kept[N - 1];
        p.row_offsets[N] = tb.rowoff[N - 1] + (tb.kept[N - 1] + kRowAlign - 1) / kRowAlign * kRowAlign;
        *p.n_live = *tb.nlive;
    }
    for (int i = tid; i < *tb.nlive; i += nth) p.live[i] = tb.live[i];
    for (int i = tid; i < TK; i += nth) {
        const int r = tb.row[i];
        p.slot_row[i] = r;
        if (r >= 0) p.perm_slot[r] = i;
    }
    for (int e = warp; e < N; e += (nth >> 5)) {
        const int start = tb.rowoff[e] + tb.kept[e];
        const int end = tb.rowoff[e] + (tb.kept[e] + kRowAlign - 1) / kRowAlign * kRowAlign;
        for (int r = start + lane; r < end; r += 32) p.perm_slot[r] = -1;
    }
    // statistics of the router's choice: fixed orders (tokens ascending, slots
    // ascending), from the gate weights and the full softmax loaded at once
    float *f_im = stat, *f_pm = stat + 32;   // [32] each
    float *s_w = stat + 64;                  // [T*K]
    float *s_tp = s_w + TK;                  // [T][32]
    for (int i = tid; i < TK; i += nth) s_w[i] = __ldcg(p.topk_w + i);
    for (int i = tid; i < p.T * 32; i += nth) s_tp[i] = __ldcg(p.tok_p + i);
    sync();
    if (tid < 32) {
        const int e = tid;
        float im = 0.f, pm = 0.f;
        if (e < N) {
            for (int i = 0; i < TK; ++i)
                if (s_idx[i] == e) im += s_w[i];
            for (int t = 0; t < p.T; ++t) pm += s_tp[t * 32 + e];
            pm /= (float)p.T;
        }
        f_im[e] = im;
        f_pm[e] = pm;
        if (e < N) {
            if (p.aux_counts) p.aux_counts[e] = tb.cnt[e];
            if (p.aux_importance) p.aux_importance[e] = im;
            if (p.aux_p_mean) p.aux_p_mean[e] = pm;
        }
    }
    sync();
    if (tid == 0 && p.aux_scalars) {
        const double tk = (double)p.T * (double)p.K;
        double sw = 0.0, ss = 0.0, mi = 0.0, mc = 0.0;
        for (int e = 0; e < N; ++e) {
            const double f = tb.cnt[e] / tk;
            sw += f * f_pm[e];
            ss += f * f;
            mi += f_im[e];
            mc += tb.cnt[e];
        }
        mi /= N;
        mc /= N;
        double vi = 0.0, vc = 0.0;
        for (int e = 0; e < N; ++e) {
            vi += (f_im[e] - mi) * (f_im[e] - mi);
            vc += (tb.cnt[e] - mc) * (tb.cnt[e] - mc);
        }
        vi /= N;
        vc /= N;
        p.aux_scalars[0] = (float)(N * sw);
        p.aux_scalars[1] = (float)(N * ss);
        p.aux_scalars[2] = mi == 0.0 ? 0.f : (float)(vi / (mi * mi));
        p.aux_scalars[3] = mc == 0.0 ? 0.f : (float)(vc / (mc * mc));
    }
}

// The kept slots' token rows into x_perm, one slot per CTA at a time, by threads
// tid < nth that sync() brings together; then the CTA releases x_perm to the grid
// (barrier 3 is waited on only by the producers, before their first token-row
// load).
template <class Sync>
__device__ __forceinline__ void r3_copy_rows(const Params &p, const Tables &tb, int tid, int nth, Sync sync) {
    const int nv = p.D / 8, TK = p.T * p.K;
    for (int i = blockIdx.x; i < TK; i += gridDim.x) {
        const int r = tb.row[i];
        if (r < 0) continue;
        const uint4 *src = reinterpret_cast<const uint4 *>(p.x + (size_t)(i / p.K) * p.D);
        uint4 *dst = reinterpret_cast<uint4 *>(p.x_perm + (size_t)r * p.D);
        for (int v = tid; v < nv; v += nth) dst[v] = __ldg(src + v);
    }
    sync();
    if (tid == 0) {
        fence_proxy_async_global();
        grid_arrive(p.bar);
    }
}

// R3: the dispatch tables from the top-k, in every CTA.  scratch holds the
// top-k indices and each slot's position inside its expert while they are built.
// With publish false, CTA 0 leaves the workspace tables and the statistics to
// the caller (r3_publish); with copy_rows false, the x_perm copies and the
// arrival at barrier 3 are left to the caller too (r3_copy_rows).
__device__ __forceinline__ void route_r3(const Params &p, const Tables &tb, uint8_t *scratch, bool idx_ready,
                                         bool publish = true, bool copy_rows = true) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int N = p.N, TK = p.T * p.K;
    int *s_idx = reinterpret_cast<int *>(scratch);   // filled by route_r2_all when idx_ready
    int *s_pos = s_idx + kMaxSlots;
    for (int i = tid; !idx_ready && i < TK; i += kThreads) {
        int e = __ldcg(p.topk_idx + i);
        if (e < 0 || e >= N) {
            set_status(kStatusBounds);
            e = -1;
        }
        s_idx[i] = e;
    }
    __syncthreads();
    if (warp == 0) {
        // stable rank of every slot inside its expert (slot order = token, then selection)
        tb.cnt[lane] = 0;
        __syncwarp();
        for (int base = 0; base < TK; base += 32) {
            const int i = base + lane;
            const int e = i < TK ? s_idx[i] : -1;
            const unsigned peers = __match_any_sync(0xffffffffu, e);
            const int rank = __popc(peers & lanemask_lt());
            const int run = e >= 0 ? tb.cnt[e] : 0;
            __syncwarp();
            if (e >= 0 && lane == __ffs(peers) - 1) tb.cnt[e] = run + __popc(peers);
            __syncwarp();
            if (i < TK) s_pos[i] = e >= 0 ? run + rank : -1;
        }
        const int c = lane < N ? tb.cnt[lane] : 0;
        const int kp = min(c, p.capacity);
        const int pad = (kp + kRowAlign - 1) / kRowAlign * kRowAlign;
        int ik = kp, ip = pad;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int a = __shfl_up_sync(0xffffffffu, ik, o), b = __shfl_up_sync(0xffffffffu, ip, o);
            if (lane >= o) { ik += a; ip += b; }
        }
        tb.kept[lane] = kp;
        tb.koff[lane] = ik - kp;
        tb.rowoff[lane] = ip - pad;
        if (lane == 31) {
            tb.koff[32] = ik;
            tb.rowoff[32] = ip;
        }
        const unsigned m = __ballot_sync(0xffffffffu, kp > 0);
        if (kp > 0) tb.live[__popc(m & lanemask_lt())] = lane;
        if (lane == 0) *tb.nlive = __popc(m);
    }
    __syncthreads();
    for (int i = tid; i < TK; i += kThreads) {
        const int e = s_idx[i], pos = s_pos[i];
        const bool keep = e >= 0 && pos < tb.kept[e];
        tb.row[i] = (int16_t)(keep ? tb.rowoff[e] + pos : -1);
        if (keep) tb.ent[tb.koff[e] + pos] = (int16_t)i;
    }
    __syncthreads();
    if (copy_rows) r3_copy_rows(p, tb, tid, kThreads, [] { __syncthreads(); });
    if (publish && blockIdx.x == 0)
        r3_publish(p, tb, s_idx, reinterpret_cast<float *>(s_pos), tid, kThreads, [] { __syncthreads(); });
}

// ------------------------------------------------------------------ the expert phases
// One phase's share of work for this CTA: stream-K unit range or whole tiles.
struct PhaseWork {
    dec::Work wk;
    int tiles, nkb, tpg;
    bool stream_k;
    int64_t u_begin, u_end, u_step;
    __device__ __forceinline__ void init(int n_live, int tiles_per_group, int num_k_blocks, int split_cap) {
        tpg = tiles_per_group;
        nkb = num_k_blocks;
        tiles = n_live * tpg;
        wk = dec::Work{(int64_t)tiles * nkb, (int)gridDim.x, nkb};
        const int waves = (tiles + (int)gridDim.x - 1) / (int)gridDim.x;
        stream_k = split_cap >= (int)gridDim.x && wk.W >= 4 * (int64_t)gridDim.x &&
                   10 * tiles < 9 * waves * (int)gridDim.x;
        u_begin = stream_k ? wk.begin(blockIdx.x) : (int64_t)blockIdx.x * nkb;
        u_end = stream_k ? wk.begin(blockIdx.x + 1) : wk.W;
        u_step = (int64_t)gridDim.x * nkb;
    }
    __device__ __forceinline__ dec::Piece piece(int64_t u) const { return dec::Piece(u, stream_k ? u_end : u + nkb, nkb); }
    __device__ __forceinline__ int64_t next(int64_t u, const dec::Piece &pc) const {
        return stream_k ? u + (pc.k1 - pc.k0) : u + u_step;
    }
};

template <int NT, int EPI_UP>
__global__ void __launch_bounds__(kThreads, 1)
    decode_layer_kernel(const __grid_constant__ CUtensorMap tmW1, const __grid_constant__ CUtensorMap tmXp,
                        const __grid_constant__ CUtensorMap tmW2, const __grid_constant__ CUtensorMap tmH,
                        const Params p) {
    pdl_enter();
    using S = Shape<NT, EPI_UP>;
    constexpr int kStages = S::kStages;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = smem + kStages * S::kABytes;
    uint8_t *sE = smem + S::kRingBytes;
    uint8_t *sT = sE + S::kEpiBytes;
    Tables tb;
    tb.row = reinterpret_cast<int16_t *>(sT);
    tb.ent = tb.row + kMaxSlots;
    tb.cnt = reinterpret_cast<int *>(tb.ent + kMaxSlots);
    tb.kept = tb.cnt + 40;
    tb.rowoff = tb.kept + 40;
    tb.koff = tb.rowoff + 40;
    tb.live = tb.koff + 40;
    tb.nlive = tb.live + 40;
    int *s_flag = tb.nlive + 40;   // [2]
    uint64_t *full = reinterpret_cast<uint64_t *>(sT + S::kTableBytes);
    uint64_t *empty = full + kStages;
    uint64_t *tfull = empty + kStages;
    uint64_t *tempty = tfull + 2;
    uint64_t *drain = tempty + 2;
    uint64_t *epib = drain + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(epib + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp == 0 && lane == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], kEpiWarps);
        }
        mbar_init(drain, 1);
        mbar_init(epib, kEpiWarps * 32);
        fence_mbar_init();
        tma_prefetch_desc(&tmW1);
        tma_prefetch_desc(&tmXp);
        tma_prefetch_desc(&tmW2);
        tma_prefetch_desc(&tmH);
    }
    if (warp == 1) tmem_alloc(tmem_slot, S::kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    // ---------------------------------------------------------------- routing
    bool ok = true;
    if ((int)blockIdx.x < p.n_slabs) route_r1<NT, EPI_UP>(p, smem);
    ok = grid_sync_all(p, 1, s_flag);
    const bool r2_all = p.T <= kAllR2T;
    if (r2_all) {
        if (ok) route_r2_all(p, smem);
    } else {
        if (ok && (int)blockIdx.x < p.T) route_r2(p, smem);
        if (ok) ok = grid_sync_all(p, 2, s_flag);
    }
    // CTA 0's workspace tables and statistics: done by its epilogue warps while
    // they wait for their first accumulator (so that CTA 0's weight stream
    // starts with everyone else's) when the selection and the scratch fit the
    // epilogue staging area, which is idle until then
    const int TK = p.T * p.K;
    const bool defer = (size_t)(2 * TK + 64 + 32 * p.T) * 4 <= S::kEpiBytes;
    // with at most 8 rows to copy, the x_perm copies (CTAs 0 .. TK - 1) and the
    // arrival at barrier 3 go to the epilogue warps too, so that no producer
    // starts late (decode1 0.4 to 1.4 us faster on two boxes); with more rows
    // the copies take longer in 128 threads and barrier 3 comes later (decode8
    // 1.5 us slower), so they stay here
    const bool defer_copy = TK <= 8;
    if (ok) {
        route_r3(p, tb, smem, r2_all, !defer, !defer_copy);
        if (defer && blockIdx.x == 0)
            for (int i = threadIdx.x; i < TK; i += kThreads) reinterpret_cast<int *>(sE)[i] = reinterpret_cast<const int *>(smem)[i];
    }
    __syncthreads();

    const bool swiglu = EPI_UP == dec::EPI_SWIGLU;
    const int D = p.D, H = p.H;
    PhaseWork wu, wd;
    wu.init(ok ? *tb.nlive : 0, (H + (swiglu ? 64 : 128) - 1) / (swiglu ? 64 : 128), (D + BK - 1) / BK, p.split_cap);
    wd.init(ok ? *tb.nlive : 0, (D + BM - 1) / BM, (H + BK - 1) / BK, p.split_cap);

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0 && ok) {
            int stage = 0;
            uint32_t phase = 0;
            IssuedSlots iss;
            // weight rows of a piece: the first row of its 128-row tile (SwiGLU up: gate and up halves)
            auto a_rows = [&](int ph, const PhaseWork &w, const dec::Piece &pc, int &wrow, int &wrow2) {
                const int g = tb.live[pc.tile / w.tpg];
                const int mt = pc.tile % w.tpg;
                wrow2 = 0;
                if (ph == 0 && swiglu) {
                    wrow = g * 2 * H + mt * (BM / 2);
                    wrow2 = wrow + H;
                } else if (ph == 0) {
                    wrow = g * H + mt * BM;
                } else {
                    wrow = g * D + mt * BM;
                }
            };
            for (int ph = 0; ph < 2 && ok; ++ph) {
                const PhaseWork &w = ph == 0 ? wu : wd;
                const CUtensorMap *mW = ph == 0 ? &tmW1 : &tmW2;
                const CUtensorMap *mB = ph == 0 ? &tmXp : &tmH;
                const unsigned *bar = ph == 0 ? p.bar : p.bar4;
                // barrier 3 is the third arrival on p.bar (the second without barrier 2)
                const unsigned target = (ph == 0 ? (r2_all ? 2u : 3u) : 1u) * gridDim.x;
                bool ready = false;
                int ndef = 0;
                int def_stage[kStages], def_col[kStages], def_row[kStages];
                auto flush = [&]() {
                    fence_proxy_async_global();
                    for (int q = 0; q < ndef; ++q)
                        tma_load_2d(mB, &full[def_stage[q]], sB + def_stage[q] * S::kBBytes, def_col[q], def_row[q]);
                    ndef = 0;
                };
                for (int64_t u = w.u_begin; u < w.u_end && ok;) {
                    const dec::Piece pc = w.piece(u);
                    u = w.next(u, pc);
                    const int trow = tb.rowoff[tb.live[pc.tile / w.tpg]];
                    int wrow, wrow2;
                    a_rows(ph, w, pc, wrow, wrow2);
                    for (int kb = pc.k0; kb < pc.k1; ++kb) {
                        if (!ready && ndef == kStages) {   // the ring holds only deferred stages: wait for the data
                            if (!grid_wait(bar, target, p.timeout_ns)) {
                                ok = false;
                                break;
                            }
                            ready = true;
                            flush();
                        }
                        if (!mbar_wait(&empty[stage], phase ^ 1, p.timeout_ns)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&full[stage], S::kStageBytes);
                        if (ph == 0 && swiglu) {
                            tma_load_2d(mW, &full[stage], sA + stage * S::kABytes, kb * BK, wrow);
                            tma_load_2d(mW, &full[stage], sA + stage * S::kABytes + (BM / 2) * BK * 2, kb * BK, wrow2);
                        } else {
                            tma_load_2d(mW, &full[stage], sA + stage * S::kABytes, kb * BK, wrow);
                        }
                        if (!ready && dec::ld_acquire_u32(bar) >= target) {
                            ready = true;
                            flush();
                        }
                        if (ready) {
                            tma_load_2d(mB, &full[stage], sB + stage * S::kBBytes, kb * BK, trow);
                        } else {
                            def_stage[ndef] = stage;
                            def_col[ndef] = kb * BK;
                            def_row[ndef] = trow;
                            ++ndef;
                        }
                        iss.note(stage, phase);
                        if (++stage == kStages) {
                            stage = 0;
                            phase ^= 1;
                        }
                    }
                }
                if (ok && ndef > 0) {
                    if (grid_wait(bar, target, p.timeout_ns)) flush();
                    else ok = false;
                }
            }
            if (!ok) iss.drain(full, p.timeout_ns);   // copies in flight land before the CTA leaves
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && ok) {
            constexpr uint32_t idesc = idesc_bf16_f32(BM, NT);
            int stage = 0;
            uint32_t phase = 0;
            int local = 0;
            bool mok = true;
            for (int ph = 0; ph < 2 && mok; ++ph) {
                const PhaseWork &w = ph == 0 ? wu : wd;
                for (int64_t u = w.u_begin; u < w.u_end && mok; ++local) {
                    const dec::Piece pc = w.piece(u);
                    u = w.next(u, pc);
                    const int a = local & 1;
                    const uint32_t aph = (local >> 1) & 1;
                    if (!mbar_wait(&tempty[a], aph ^ 1, p.timeout_ns)) {
                        mok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + a * NT;
                    for (int kb = pc.k0; kb < pc.k1; ++kb) {
                        if (!mbar_wait(&full[stage], phase, p.timeout_ns)) {
                            mok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint64_t adesc = smem_desc_sw128(smem_u32(sA + stage * S::kABytes));
                        const uint64_t bdesc = smem_desc_sw128(smem_u32(sB + stage * S::kBBytes));
#pragma unroll
                        for (int k = 0; k < BK / 16; ++k)
                            tc_mma_bf16(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, (kb != pc.k0 || k != 0) ? 1u : 0u);
                        tc_commit(&empty[stage]);
                        if (++stage == kStages) {
                            stage = 0;
                            phase ^= 1;
                        }
                    }
                    if (mok) tc_commit(&tfull[a]);
                }
            }
            if (!mok) {
                tc_commit(drain);
                mbar_wait(drain, 0, p.timeout_ns);
            }
        }
    } else if (ok) {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;
        const int L = q * 32 + lane;        // TMEM lane = weight row within the tile
        const int et = threadIdx.x - 64;    // 0..127
        // the x_perm copies and the arrival at barrier 3, then (CTA 0) the tables and
        // the statistics, while the producer already streams weight tiles
        auto epi_sync = [] { asm volatile("bar.sync 1, 128;" ::: "memory"); };
        if (defer_copy) r3_copy_rows(p, tb, et, 128, epi_sync);
        if (defer && blockIdx.x == 0) {
            r3_publish(p, tb, reinterpret_cast<const int *>(sE), reinterpret_cast<float *>(sE) + TK, et, 128, epi_sync);
            epi_sync();   // sE is the staging area again from here on
        }
        dec::EpiBarrier eb{epib, 0u, p.timeout_ns};
        int local = 0;
        bool eok = true;
        for (int ph = 0; ph < 2 && eok; ++ph) {
            const PhaseWork &w = ph == 0 ? wu : wd;
            unsigned *tickets = ph == 0 ? p.tk_up : p.tk_down;
            for (int64_t u = w.u_begin; u < w.u_end; ++local) {
                const int64_t u_piece = u;
                const dec::Piece pc = w.piece(u);
                u = w.next(u, pc);
                const int tile = pc.tile;
                const int a = local & 1;
                const uint32_t aph = (local >> 1) & 1;
                const int g = tb.live[tile / w.tpg];
                const int mt = tile % w.tpg;
                const int cnt = tb.kept[g];
                const int trow = tb.rowoff[g];
                const int kbase = tb.koff[g];
                const bool cut = pc.k1 - pc.k0 < w.nkb;
                const int64_t ts = (int64_t)tile * w.nkb;
                const int c_first = cut ? w.wk.cta_of(ts) : 0, c_last = cut ? w.wk.cta_of(ts + w.nkb - 1) : 0;
                if (!__all_sync(0xffffffffu, mbar_wait(&tfull[a], aph, p.timeout_ns))) {
                    eok = false;
                    break;
                }
                tc_fence_after();
                float acc[NT];
                dec::tmem_ld_row<NT>(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + a * NT, acc);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[a]);   // accumulator is in registers now
                if (cut) {
                    // publish this piece's partial row and take the tile's ticket; the
                    // last piece to arrive adds all of the tile's pieces in piece order
                    const int my_slot = (u_piece == w.u_begin && w.u_begin >= ts) ? 0 : 1;
                    float *mine = p.part + ((int64_t)(blockIdx.x * 2 + my_slot) * BM + L) * NT;
#pragma unroll
                    for (int j = 0; j < NT; j += 4)
                        __stcg(reinterpret_cast<float4 *>(mine + j), make_float4(acc[j], acc[j + 1], acc[j + 2], acc[j + 3]));
                    if (!eb.sync()) { eok = false; break; }
                    if (et == 0) s_flag[1] = ticket_arrive(tickets + c_first) == (unsigned)(c_last - c_first);
                    if (!eb.sync()) { eok = false; break; }
                    if (!s_flag[1]) continue;
                    // pieces added from the last CTA's down to the first's; the loads of
                    // GC pieces are issued together (one round trip per group)
                    constexpr int GC = NT >= 64 ? 1 : 64 / NT;
                    float sum[NT];
                    for (int c0 = c_last; c0 >= c_first; c0 -= GC) {
                        float v[GC][NT];
#pragma unroll
                        for (int gi = 0; gi < GC; ++gi) {
                            const int c = c0 - gi;
                            if (c < c_first) continue;
                            if (c == (int)blockIdx.x) {
#pragma unroll
                                for (int j = 0; j < NT; ++j) v[gi][j] = acc[j];
                            } else {
                                const float *src =
                                    p.part + ((int64_t)(c * 2 + (w.wk.begin(c) >= ts ? 0 : 1)) * BM + L) * NT;
#pragma unroll
                                for (int j = 0; j < NT; j += 4) {
                                    const float4 q4 = __ldcg(reinterpret_cast<const float4 *>(src + j));
                                    v[gi][j] = q4.x; v[gi][j + 1] = q4.y; v[gi][j + 2] = q4.z; v[gi][j + 3] = q4.w;
                                }
                            }
                        }
#pragma unroll
                        for (int gi = 0; gi < GC; ++gi) {
                            const int c = c0 - gi;
                            if (c < c_first) continue;
#pragma unroll
                            for (int j = 0; j < NT; ++j) sum[j] = c == c_last ? v[gi][j] : v[gi][j] + sum[j];
                        }
                    }
#pragma unroll
                    for (int j = 0; j < NT; ++j) acc[j] = sum[j];
                }
                if (ph == 0) {
                    // ---- up projection epilogue -> h rows of the expert's kept tokens
                    __nv_bfloat16 *hout = p.h;
                    if (EPI_UP == dec::EPI_GELU) {
                        __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(sE);   // [NT][128]
                        const int f = mt * BM + L;
                        const float b = (p.b1 && f < H) ? __ldg(p.b1 + (int64_t)g * H + f) : 0.f;
#pragma unroll
                        for (int j = 0; j < NT; j += 2) {
                            const uint32_t hv = tc::gelu_erf_bf16x2(acc[j] + b, acc[j + 1] + b);
                            o[j * 128 + L] = __ushort_as_bfloat16(static_cast<unsigned short>(hv & 0xffffu));
                            o[(j + 1) * 128 + L] = __ushort_as_bfloat16(static_cast<unsigned short>(hv >> 16));
                        }
                        if (!eb.sync()) { eok = false; break; }
                        const int f0 = mt * BM;
                        for (int v = et; v < NT * 16; v += 128) {
                            const int j = v >> 4, c = (v & 15) * 8;
                            if (j < cnt) {
                                __nv_bfloat16 *dst = hout + (int64_t)(trow + j) * H + f0 + c;
                                const __nv_bfloat16 *src = o + j * 128 + c;
                                if (f0 + c + 8 <= H) {
                                    *reinterpret_cast<uint4 *>(dst) = *reinterpret_cast<const uint4 *>(src);
                                } else {
                                    for (int k = 0; k < 8; ++k)
                                        if (f0 + c + k < H) dst[k] = src[k];
                                }
                            }
                        }
                        if (!eb.sync()) { eok = false; break; }
                    } else {
                        float *up = reinterpret_cast<float *>(sE);                                  // [NT][64]
                        __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(sE + 64 * NT * 4);     // [NT][64]
                        if (L >= 64) {
#pragma unroll
                            for (int j = 0; j < NT; ++j) up[j * 64 + (L - 64)] = acc[j];
                        }
                        if (!eb.sync()) { eok = false; break; }
                        if (L < 64) {
#pragma unroll
                            for (int j = 0; j < NT; j += 2) {
                                const uint32_t hv =
                                    tc::swiglu_bf16x2(acc[j], acc[j + 1], up[j * 64 + L], up[(j + 1) * 64 + L]);
                                o[j * 64 + L] = __ushort_as_bfloat16(static_cast<unsigned short>(hv & 0xffffu));
                                o[(j + 1) * 64 + L] = __ushort_as_bfloat16(static_cast<unsigned short>(hv >> 16));
                            }
                        }
                        if (!eb.sync()) { eok = false; break; }
                        const int f0 = mt * (BM / 2);
                        for (int v = et; v < NT * 8; v += 128) {
                            const int j = v >> 3, c = (v & 7) * 8;
                            if (j < cnt) {
                                __nv_bfloat16 *dst = hout + (int64_t)(trow + j) * H + f0 + c;
                                const __nv_bfloat16 *src = o + j * 64 + c;
                                if (f0 + c + 8 <= H) {
                                    *reinterpret_cast<uint4 *>(dst) = *reinterpret_cast<const uint4 *>(src);
                                } else {
                                    for (int k = 0; k < 8; ++k)
                                        if (f0 + c + k < H) dst[k] = src[k];
                                }
                            }
                        }
                        if (!eb.sync()) { eok = false; break; }
                    }
                } else {
                    // ---- down projection epilogue: z[slot, d] = w[slot] (acc + b2[d])
                    const int d = mt * BM + L;
                    if (d < D) {
                        const float b = p.b2 ? __ldg(p.b2 + (int64_t)g * D + d) : 0.f;
#pragma unroll
                        for (int j = 0; j < NT; ++j) {
                            if (j < cnt) {
                                const int slot = tb.ent[kbase + j];
                                __stcg(p.z + (int64_t)slot * D + d, __ldcg(p.topk_w + slot) * (acc[j] + b));
                            }
                        }
                    }
                }
            }
            if (ph == 0 && eok) {
                // h written by this CTA: release it to the grid (barrier 4)
                if (!eb.sync()) { eok = false; break; }
                if (et == 0) {
                    __threadfence();
                    fence_proxy_async_global();
                    grid_arrive(p.bar4);
                }
            }
        }
        // ---- the combine: once every CTA's z rows are written (barrier 5), the epilogue
        // threads of all CTAs share y: y[t, d] = z[t K, d] + ... + z[t K + K - 1, d] in slot
        // order over the kept slots; two outputs per thread and four slots each have their
        // loads in flight together
        if (eok && eb.sync()) {
            if (et == 0) {
                __threadfence();
                grid_arrive(p.bar5);
                s_flag[1] = grid_wait(p.bar5, gridDim.x, p.timeout_ns) ? 1 : 0;
            }
            if (eb.sync() && s_flag[1]) {
                // compact code: this runs once per launch, so its instructions are fetched cold
                const int K = p.K;
                const int O = p.T * D;
                const int stride = (int)gridDim.x * 128;
                for (int o0 = (int)blockIdx.x * 128 + et; o0 < O; o0 += 2 * stride) {
                    float acc[2] = {0.f, 0.f};
                    bool any[2] = {false, false};
                    for (int j0 = 0; j0 < K; j0 += 4) {
                        float v[2][4];
                        bool h[2][4];
#pragma unroll
                        for (int q = 0; q < 2; ++q) {
                            const int o = o0 + q * stride;
                            const int t = o < O ? o / D : 0;
                            const float *zt = p.z + (size_t)t * K * D + (o - t * D);
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                const int j = j0 + u;
                                h[q][u] = o < O && j < K && tb.row[t * K + j] >= 0;   // dropped by the capacity
                                v[q][u] = h[q][u] ? __ldcg(zt + (size_t)j * D) : 0.f;
                            }
                        }
#pragma unroll
                        for (int q = 0; q < 2; ++q)
#pragma unroll
                            for (int u = 0; u < 4; ++u)
                                if (h[q][u]) {
                                    acc[q] = any[q] ? acc[q] + v[q][u] : v[q][u];
                                    any[q] = true;
                                }
                    }
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const int o = o0 + q * stride;
                        if (o >= O) continue;
                        if (p.y_bf16) static_cast<__nv_bfloat16 *>(p.y)[o] = __float2bfloat16_rn(acc[q]);
                        else static_cast<float *>(p.y)[o] = acc[q];
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, S::kTmemCols);
    }
}

}  // namespace dfu
}  // namespace moe
