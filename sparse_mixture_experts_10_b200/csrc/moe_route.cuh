// moe_route.cuh -- routing, dispatch, combine and statistics kernels.
//
// Routing follows the page "MoE(Mixture of Experts)" (sharin-2a1.pages.dev/
// parts/moe), section (2) Route: scores = x W_g, a stable descending sort of
// the expert indices (equal scores: lower index first), the first TopK kept,
// and a softmax over only those scores shifted by the best one.  This is
// softmax(KeepTopK(x W_g, k)) of the Shazeer article (qiita), gating section,
// in its noise-free inference form.
//
// Dispatch groups the (token, slot) pairs by expert with a stable counting
// sort: per-chunk histograms (written by the router), a scan over chunks and
// experts, then a scatter of token rows into expert-contiguous segments, each
// starting on a multiple of kRowAlign rows so that every 128-row tensor-core
// tile lies inside one expert.  This is the "sort and group by expert id" step
// of the grouped_mm backend (Transformers-v5 MoE article, section 2).
#pragma once

#include "moe_common.cuh"

namespace moe {

constexpr int kChunk = 32;       // tokens per router / permute block (counting-sort chunk)
constexpr int kRowAlign = 128;   // expert segment alignment in the permuted buffers
constexpr int kAuxTokens = 64;   // tokens per statistics block

__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// (taken, value, index) ordering of the top-k selection: an untaken entry beats
// a taken one; then the larger value; then the lower expert index.  NaN never
// reaches this comparison (it is ranked as -inf beforehand).
__device__ __forceinline__ bool beats(float v, int e, bool t, float ov, int oe, bool ot) {
    if (t != ot) return !t;
    return v > ov || (v == ov && e < oe);
}

// Reduce-scatter of 32 per-lane partial sums: afterwards lane l holds, in a[0],
// the warp-wide sum of entry l.  Each step halves the entries a lane keeps.
template <int C>
__device__ __forceinline__ void reduce_scatter_step(float (&a)[32], int lane) {
    constexpr int H = C / 2;
    const bool upper = (lane & H) != 0;
#pragma unroll
    for (int i = 0; i < H; ++i) {
        const float send = upper ? a[i] : a[i + H];
        const float keep = upper ? a[i + H] : a[i];
        a[i] = keep + __shfl_xor_sync(0xffffffffu, send, H);
    }
}

__device__ __forceinline__ void reduce_scatter32(float (&a)[32], int lane) {
    reduce_scatter_step<32>(a, lane);
    reduce_scatter_step<16>(a, lane);
    reduce_scatter_step<8>(a, lane);
    reduce_scatter_step<4>(a, lane);
    reduce_scatter_step<2>(a, lane);
}

template <typename T>
struct Vec16;  // 16 bytes of T widened to float
template <>
struct Vec16<float> {
    static constexpr int n = 4;
    __device__ __forceinline__ static void unpack(const uint4 v, float (&f)[8]) {
        f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y); f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
    }
    __device__ __forceinline__ static void load(const float *p, float (&f)[8]) {
        unpack(*reinterpret_cast<const uint4 *>(p), f);
    }
};
template <>
struct Vec16<__nv_bfloat16> {
    static constexpr int n = 8;
    __device__ __forceinline__ static void unpack(const uint4 v, float (&f)[8]) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    __device__ __forceinline__ static void load(const __nv_bfloat16 *p, float (&f)[8]) {
        unpack(*reinterpret_cast<const uint4 *>(p), f);
    }
};

// Top-k over one segment of NP lanes, each holding one expert: its selection
// value v (the score, plus a selection-only bias when one is given) and its raw
// score.  The K best by (v, lower index on ties) are kept; the gate weights
// are the softmax over the kept experts' raw scores, shifted by the largest of
// them -- softmax(KeepTopK(.)) of the Shazeer article's gating section with the
// kept set chosen on v.  Without a selection bias v == raw and the shift is
// slot 0's score.  Lane r of the segment (r < K) returns slot r.  Returns true
// for lanes that hold a slot.
template <int NP>
__device__ __forceinline__ bool segment_topk(float v, float raw, int e, bool taken, int K, int seg_lane, int lane,
                                             int &slot_e, float &slot_w) {
    float my_raw = -INFINITY;
    int my_e = 0;
    for (int r = 0; r < K; ++r) {
        float cv = v, cr = raw;
        int ce = e;
        bool ct = taken;
#pragma unroll
        for (int o = NP / 2; o >= 1; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, cv, o);
            const float orw = __shfl_xor_sync(0xffffffffu, cr, o);
            const int oe = __shfl_xor_sync(0xffffffffu, ce, o);
            const bool ot = __shfl_xor_sync(0xffffffffu, (int)ct, o) != 0;
            if (beats(ov, oe, ot, cv, ce, ct)) { cv = ov; cr = orw; ce = oe; ct = ot; }
        }
        if (e == ce) taken = true;
        if (seg_lane == r) { my_raw = cr; my_e = ce; }
    }
    float m = seg_lane < K ? my_raw : -INFINITY;
#pragma unroll
    for (int o = NP / 2; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float ex = seg_lane < K ? expf(my_raw - m) : 0.f;
    float sum = 0.f;
    const int seg_base = lane - seg_lane;
    for (int q = 0; q < K; ++q) sum += __shfl_sync(0xffffffffu, ex, seg_base + q);  // slot order
    slot_e = my_e;
    slot_w = ex / sum;
    return seg_lane < K;
}

// The selection value of a score: score + selection-only bias (fp32), or the
// score itself.
__device__ __forceinline__ float sel_value(const float *bsel, float s, int e, bool valid) {
    return (bsel && valid) ? s + __ldg(bsel + e) : s;
}

// ---------------------------------------------------------------------------
// Fused router for N <= 32 experts: scores, top-k, softmax, chunk histogram.
// One block per chunk of kChunk tokens; W_g is staged transposed ([NP][D],
// zero rows for experts N..NP-1) in shared memory; each warp handles 32/NP
// tokens at a time, each lane a strided set of 16-byte slices of D; a
// reduce-scatter leaves lane l with the score of (token l/NP, expert l%NP).
// ---------------------------------------------------------------------------
template <typename Tin, int NP>
__global__ void __launch_bounds__(256) router_small_kernel(const Tin *__restrict__ x, int T, int D, int N, int K,
                                                           const Tin *__restrict__ Wg, const float *__restrict__ bg,
                                                           const float *__restrict__ bsel,
                                                           float *__restrict__ logits, int *__restrict__ topk_idx,
                                                           float *__restrict__ topk_w, int *__restrict__ chunk_counts) {
    constexpr int TPW = 32 / NP;
    constexpr int VEC = Vec16<Tin>::n;
    constexpr int U = 4;  // 16-byte vectors in flight per token and lane
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Tin *WgT = reinterpret_cast<Tin *>(smem_raw);
    int *hist = reinterpret_cast<int *>(smem_raw + (size_t)NP * D * sizeof(Tin));

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // one router row d per thread: contiguous global reads, consecutive shared addresses per expert row
    for (int d = tid; d < D; d += blockDim.x) {
#pragma unroll
        for (int e = 0; e < NP; ++e) WgT[(size_t)e * D + d] = e < N ? Wg[(size_t)d * N + e] : Tin(0.f);
    }
    if (tid < NP) hist[tid] = 0;
    __syncthreads();

    const int t_begin = blockIdx.x * kChunk;
    const int nvec = D / VEC;
    const int seg_lane = lane % NP;
    for (int g = warp * TPW; g < kChunk; g += 8 * TPW) {
        const int t0 = t_begin + g;
        float a[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) a[i] = 0.f;
        for (int v0 = lane; v0 < nvec; v0 += 32 * U) {
            uint4 xr[TPW][U];
#pragma unroll
            for (int tt = 0; tt < TPW; ++tt)
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int v = v0 + 32 * u;
                    xr[tt][u] = (t0 + tt < T && v < nvec)
                                    ? __ldg(reinterpret_cast<const uint4 *>(x + (size_t)(t0 + tt) * D) + v)
                                    : make_uint4(0u, 0u, 0u, 0u);
                }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int v = v0 + 32 * u;
                if (v >= nvec) break;
                float xf[TPW][8];
#pragma unroll
                for (int tt = 0; tt < TPW; ++tt) Vec16<Tin>::unpack(xr[tt][u], xf[tt]);
#pragma unroll
                for (int e = 0; e < NP; ++e) {
                    float wf[8];
                    Vec16<Tin>::load(WgT + (size_t)e * D + (size_t)v * VEC, wf);
#pragma unroll
                    for (int tt = 0; tt < TPW; ++tt)
#pragma unroll
                        for (int q = 0; q < VEC; ++q) a[tt * NP + e] = fmaf(xf[tt][q], wf[q], a[tt * NP + e]);
                }
            }
        }
        reduce_scatter32(a, lane);
        const int e = seg_lane;
        const int t = t0 + lane / NP;
        const bool valid_e = e < N;
        float s = a[0];
        if (valid_e && bg) s += bg[e];
        if (logits && t < T && valid_e) logits[(size_t)t * N + e] = s;
        if (s != s) {
            if (valid_e && t < T) set_status(kStatusNanLogit);
            s = -INFINITY;
        }
        int slot_e;
        float slot_w;
        const bool has_slot =
            segment_topk<NP>(sel_value(bsel, s, e, valid_e), s, e, !valid_e, K, seg_lane, lane, slot_e, slot_w);
        if (has_slot && t < T) {
            topk_idx[(size_t)t * K + seg_lane] = slot_e;
            topk_w[(size_t)t * K + seg_lane] = slot_w;
            atomicAdd(&hist[slot_e], 1);
        }
    }
    __syncthreads();
    if (tid < N) chunk_counts[(size_t)blockIdx.x * N + tid] = hist[tid];
}

// ---------------------------------------------------------------------------
// Router for few tokens (N <= 32): one block per token, lane = expert, each of
// the 32 warps accumulates a strided share of the D rows of W_g (one coalesced
// row read per step, no staging), the warps' partial sums are added in warp
// order, then warp 0 selects the top k.  Chunk histograms are built with
// integer atomics on a zeroed array (order-independent).
// ---------------------------------------------------------------------------
template <typename Tin>
__global__ void __launch_bounds__(1024) router_rowdot_kernel(const Tin *__restrict__ x, int T, int D, int N, int K,
                                                             const Tin *__restrict__ Wg, const float *__restrict__ bg,
                                                             const float *__restrict__ bsel,
                                                             float *__restrict__ logits, int *__restrict__ topk_idx,
                                                             float *__restrict__ topk_w, int *__restrict__ chunk_counts) {
    __shared__ float part[32][33];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x;
    const Tin *xt = x + (size_t)t * D;
    // warp w takes rows w, w+32, ...; eight rows' loads are issued before their FMAs
    constexpr int R = 8;
    float acc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r] = 0.f;
    const bool live = lane < N;
    for (int d0 = warp; d0 < D; d0 += 32 * R) {
        float xv[R], wv[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int d = d0 + 32 * r;
            xv[r] = d < D ? to_f32(__ldg(xt + d)) : 0.f;
            wv[r] = (d < D && live) ? to_f32(__ldg(Wg + (size_t)d * N + lane)) : 0.f;
        }
#pragma unroll
        for (int r = 0; r < R; ++r) acc[r] = fmaf(xv[r], wv[r], acc[r]);
    }
    float tot = 0.f;
#pragma unroll
    for (int r = 0; r < R; ++r) tot += acc[r];
    part[warp][lane] = tot;
    __syncthreads();
    if (warp != 0) return;
    float s = 0.f;
    for (int w = 0; w < 32; ++w) s += part[w][lane];
    if (live && bg) s += bg[lane];
    if (logits && live) logits[(size_t)t * N + lane] = s;
    if (s != s) {
        if (live) set_status(kStatusNanLogit);
        s = -INFINITY;
    }
    int slot_e;
    float slot_w;
    if (segment_topk<32>(sel_value(bsel, s, lane, live), s, lane, !live, K, lane, lane, slot_e, slot_w)) {
        topk_idx[(size_t)t * K + lane] = slot_e;
        topk_w[(size_t)t * K + lane] = slot_w;
        atomicAdd(&chunk_counts[(size_t)(t / kChunk) * N + slot_e], 1);
    }
}

// ---------------------------------------------------------------------------
// Top-k + softmax from precomputed fp32 scores [T, N] (N <= 32 * VPL), with the
// chunk histogram.  One warp per token; lane l holds experts l, l+32, ...
// ---------------------------------------------------------------------------
template <int VPL>
__global__ void __launch_bounds__(256) topk_kernel(const float *__restrict__ logits, int T, int N, int K,
                                                   const float *__restrict__ bsel,
                                                   int *__restrict__ topk_idx, float *__restrict__ topk_w,
                                                   int *__restrict__ chunk_counts) {
    extern __shared__ int hist_s[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int e = tid; e < N; e += blockDim.x) hist_s[e] = 0;
    __syncthreads();
    for (int tl = warp; tl < kChunk; tl += 8) {
        const int t = blockIdx.x * kChunk + tl;
        if (t >= T) break;
        float v[VPL], raw[VPL];   // selection values (score + selection bias) and raw scores
        uint32_t taken = 0;
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            const int e = lane + 32 * i;
            if (e < N) {
                raw[i] = logits[(size_t)t * N + e];
                if (raw[i] != raw[i]) {
                    set_status(kStatusNanLogit);
                    raw[i] = -INFINITY;
                }
                v[i] = sel_value(bsel, raw[i], e, true);
            } else {
                v[i] = raw[i] = -INFINITY;
                taken |= 1u << i;
            }
        }
        float my_raw = -INFINITY;
        int my_e = 0;
        for (int r = 0; r < K; ++r) {
            // best untaken entry of this lane (lower index first on ties)
            float cv = -INFINITY, cr = -INFINITY;
            int ce = 0x7fffffff;
            bool ct = true;
#pragma unroll
            for (int i = 0; i < VPL; ++i) {
                const bool ti = (taken >> i) & 1u;
                if (beats(v[i], lane + 32 * i, ti, cv, ce, ct)) { cv = v[i]; cr = raw[i]; ce = lane + 32 * i; ct = ti; }
            }
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, cv, o);
                const float orw = __shfl_xor_sync(0xffffffffu, cr, o);
                const int oe = __shfl_xor_sync(0xffffffffu, ce, o);
                const bool ot = __shfl_xor_sync(0xffffffffu, (int)ct, o) != 0;
                if (beats(ov, oe, ot, cv, ce, ct)) { cv = ov; cr = orw; ce = oe; ct = ot; }
            }
            if ((ce & 31) == lane) taken |= 1u << (ce >> 5);
            if (lane == r) { my_raw = cr; my_e = ce; }
        }
        // shift by the largest kept raw score (slot 0's without a selection bias)
        float best0 = lane < K ? my_raw : -INFINITY;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) best0 = fmaxf(best0, __shfl_xor_sync(0xffffffffu, best0, o));
        const float ex = lane < K ? expf(my_raw - best0) : 0.f;
        float sum = 0.f;
        for (int m = 0; m < K; ++m) sum += __shfl_sync(0xffffffffu, ex, m);
        if (lane < K) {
            topk_idx[(size_t)t * K + lane] = my_e;
            topk_w[(size_t)t * K + lane] = ex / sum;
            atomicAdd(&hist_s[my_e], 1);
        }
    }
    __syncthreads();
    for (int e = tid; e < N; e += blockDim.x) chunk_counts[(size_t)blockIdx.x * N + e] = hist_s[e];
}

// ---------------------------------------------------------------------------
// Chunk histograms of given assignments: chunk c holds entries
// [c * per_chunk, (c + 1) * per_chunk) of idx; bucket = idx / div (div = 1:
// experts; div = experts per rank: destination ranks).  Integer shared-memory
// atomics, so the counts do not depend on scheduling.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) hist_kernel(const int *__restrict__ idx, int64_t n_entries, int per_chunk,
                                                   int n_buckets, int div, int *__restrict__ chunk_counts) {
    extern __shared__ int s_hist[];
    for (int b = threadIdx.x; b < n_buckets; b += blockDim.x) s_hist[b] = 0;
    __syncthreads();
    const int64_t f0 = (int64_t)blockIdx.x * per_chunk;
    const int64_t f1 = min(n_entries, f0 + per_chunk);
    for (int64_t f = f0 + threadIdx.x; f < f1; f += blockDim.x) {
        const int e = idx[f];
        const int b = e / div;
        if (e < 0 || b >= n_buckets) {
            set_status(kStatusBounds);
            continue;
        }
        atomicAdd(&s_hist[b], 1);
    }
    __syncthreads();
    for (int b = threadIdx.x; b < n_buckets; b += blockDim.x) chunk_counts[(size_t)blockIdx.x * n_buckets + b] = s_hist[b];
}

// ---------------------------------------------------------------------------
// Reroute, the capacity's other overflow policy ("MoE(Mixture of Experts)",
// design notes on the capacity factor: what overflows is dropped or passed to
// the next candidate).  Rows are served in token order: row t offers each of
// its K selected experts its slot, accepted while the expert holds fewer than
// C; each refused slot, in slot order, goes to the best-ranked expert (larger
// selection value logit + b_sel in fp32, ties to the lower index; NaN ranked as
// -inf) that row t does not hold yet and that still holds fewer than C.  The
// new expert is written over idx[t, j]; a slot with no such expert keeps its
// (full) selected expert, so the capacity scan that follows drops it, and
// every accepted slot lands within the first C of its expert.
//
// The order of service makes this sequential in t.  One CTA, the per-expert
// loads in shared memory, tokens staged in batches (two buffers):
//   * a batch in which no expert would pass C (its histogram added to the
//     loads) is accepted whole by all threads -- the common case while the
//     experts fill;
//   * otherwise warp 0 walks it, vbatch tokens at a time whose selection
//     values all threads stage first (only such batches need them): 32/K
//     tokens per step, each lane one (token, slot), its place = the
//     expert's load + the earlier lanes with the same expert (match.any); the
//     tokens before the first refused slot are accepted, the refusing token
//     takes the per-token step: its free candidates are read into registers
//     once (NPL per lane) and each refused slot takes the best of them by a
//     warp arg-max, in slot order.
// ---------------------------------------------------------------------------
constexpr int kRerouteThreads = 1024;

// The selections of tokens [t0, t0 + rows) into shared memory (eight loads in
// flight per thread).
__device__ __forceinline__ void reroute_stage_idx(const int *__restrict__ idx, int64_t t0, int rows, int N, int K,
                                                  int *sidx) {
    const int n = rows * K;
    for (int i0 = threadIdx.x; i0 < n; i0 += 8 * kRerouteThreads) {
        int v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = i0 + u * kRerouteThreads;
            v[u] = i < n ? idx[t0 * K + i] : 0;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = i0 + u * kRerouteThreads;
            if (i >= n) continue;
            int e = v[u];
            if ((unsigned)e >= (unsigned)N) {   // not an expert: counted against expert 0, flagged
                set_status(kStatusBounds);
                e = 0;
            }
            sidx[i] = e;
        }
    }
}

// The selection values (logit + b_sel in fp32, NaN ranked as -inf) of tokens
// [t0, t0 + rows) into shared memory, eight loads in flight per thread.
__device__ __forceinline__ void reroute_stage_values(const float *__restrict__ logits, const float *__restrict__ bsel,
                                                     int64_t t0, int rows, int N, float *sv) {
    const int n = rows * N;
    const float *src = logits + t0 * N;
    for (int i0 = threadIdx.x; i0 < n; i0 += 8 * kRerouteThreads) {
        float v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = i0 + u * kRerouteThreads;
            v[u] = i < n ? src[i] : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = i0 + u * kRerouteThreads;
            if (i >= n) continue;
            float x = v[u];
            if (bsel) x += __ldg(bsel + i % N);
            sv[i] = x != x ? -INFINITY : x;
        }
    }
}

// Warp 0's walk over one batch (see above).
template <int NPL>
__device__ __forceinline__ void reroute_walk(int *load, const int *bidx, const float *bv, int *__restrict__ idx,
                                             int64_t t0, int rows, int N, int K, int C) {
    const int lane = threadIdx.x & 31;
    const unsigned FULL = 0xffffffffu;
    const int G = 32 / K;   // tokens per step of the fast path
    int lt = 0;
    while (lt < rows) {
        const int g = min(G, rows - lt);
        const bool act = lane < g * K;
        const int tl = lane / K, j = lane - tl * K;
        const int e = act ? bidx[(lt + tl) * K + j] : -1 - lane;   // inactive lanes: distinct keys
        const unsigned peers = __match_any_sync(FULL, e);
        const int pos = act ? load[e] + __popc(peers & lanemask_lt()) : 0;
        const unsigned refused = __ballot_sync(FULL, act && pos >= C);
        const int good = refused ? (__ffs(refused) - 1) / K : g;   // tokens accepted as they are
        const unsigned accm = __ballot_sync(FULL, act && tl < good);
        const unsigned pa = peers & accm;
        if (((accm >> lane) & 1u) && (pa >> lane) == 1u) load[e] += __popc(pa);   // last lane of its expert
        __syncwarp();
        lt += good;
        if (good == g) continue;
        // the refusing token, alone: accept what fits, reroute the rest in slot order
        const int64_t t = t0 + lt;
        const int ej = lane < K ? bidx[lt * K + lane] : -1;
        const bool room = lane < K && load[ej] < C;
        if (room) load[ej] += 1;   // a token's K experts are distinct
        __syncwarp();
        unsigned todo = __ballot_sync(FULL, lane < K && !room);
        uint32_t held = 0;         // bit i: expert lane + 32 i is one of the token's
        for (int jj = 0; jj < K; ++jj) {
            const int h = __shfl_sync(FULL, ej, jj);
            if ((h & 31) == lane) held |= 1u << (h >> 5);
        }
        // this lane's free candidates, read once: value, or unavailable
        const float *vrow = bv + (size_t)lt * N;
        float cv[NPL];
        bool ca[NPL];
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
            const int c = lane + 32 * i;
            const bool in = c < N;
            const int ld = in ? load[c] : C;
            cv[i] = in ? vrow[c] : 0.f;
            ca[i] = in && ld < C && !((held >> i) & 1u);
        }
        while (todo) {
            const int js = __ffs(todo) - 1;
            todo &= todo - 1;
            float best_v = -INFINITY;
            int best_e = -1;
#pragma unroll
            for (int i = 0; i < NPL; ++i)
                if (ca[i] && (best_e < 0 || cv[i] > best_v)) {   // ascending experts: ties keep the lower index
                    best_v = cv[i];
                    best_e = lane + 32 * i;
                }
#pragma unroll
            for (int o = 16; o; o >>= 1) {
                const float ov = __shfl_xor_sync(FULL, best_v, o);
                const int oe = __shfl_xor_sync(FULL, best_e, o);
                if (oe >= 0 && (best_e < 0 || ov > best_v || (ov == best_v && oe < best_e))) {
                    best_v = ov;
                    best_e = oe;
                }
            }
            if (best_e < 0) break;   // no expert left with room: the remaining refused slots are dropped
            if (lane == 0) {
                load[best_e] += 1;
                idx[t * K + js] = best_e;
            }
            if ((best_e & 31) == lane) {
#pragma unroll
                for (int i = 0; i < NPL; ++i)
                    if ((best_e >> 5) == i) ca[i] = false;
            }
        }
        __syncwarp();
        lt += 1;
    }
}

template <int NPL>
__global__ void __launch_bounds__(kRerouteThreads, 1)
    reroute_kernel(const float *__restrict__ logits, const float *__restrict__ bsel, int *__restrict__ idx,
                   int64_t T, int N, int K, int C, int batch, int vbatch) {
    extern __shared__ __align__(16) unsigned char rr_smem[];
    const int npad = (N + 3) & ~3;
    int *load = reinterpret_cast<int *>(rr_smem);                        // [N]
    int *hist = load + npad;                                             // [N] the batch's histogram
    int *sidx = hist + npad;                                             // [2][batch * K]
    float *sv = reinterpret_cast<float *>(sidx + 2 * batch * K);         // [vbatch * N]
    const int tid = threadIdx.x, warp = tid >> 5;
    for (int e = tid; e < N; e += kRerouteThreads) load[e] = 0;
    const int nb = (int)((T + batch - 1) / batch);
    auto rows_of = [&](int bi) {
        const int64_t t0 = (int64_t)bi * batch;
        return (int)(T - t0 < (int64_t)batch ? T - t0 : (int64_t)batch);
    };
    reroute_stage_idx(idx, 0, rows_of(0), N, K, sidx);
    __syncthreads();
    for (int bi = 0; bi < nb; ++bi) {
        const int cur = bi & 1;
        const int *bidx = sidx + cur * batch * K;
        const int64_t t0 = (int64_t)bi * batch;
        const int rows = rows_of(bi);
        // the whole batch at once when no expert would pass C
        for (int e = tid; e < N; e += kRerouteThreads) hist[e] = 0;
        __syncthreads();
        for (int i = tid; i < rows * K; i += kRerouteThreads) atomicAdd(&hist[bidx[i]], 1);
        __syncthreads();
        bool over = false;
        for (int e = tid; e < N; e += kRerouteThreads) over |= load[e] + hist[e] > C;
        over = __syncthreads_or(over);
        if (!over) {
            for (int e = tid; e < N; e += kRerouteThreads) load[e] += hist[e];
        } else {
            // warp 0 walks the batch, vbatch tokens at a time with their values staged by all
            for (int s0 = 0; s0 < rows; s0 += vbatch) {
                const int vr = min(vbatch, rows - s0);
                reroute_stage_values(logits, bsel, t0 + s0, vr, N, sv);
                __syncthreads();
                if (warp == 0) reroute_walk<NPL>(load, bidx + s0 * K, sv, idx, t0 + s0, vr, N, K, C);
                __syncthreads();
            }
        }
        if (bi + 1 < nb) reroute_stage_idx(idx, t0 + batch, rows_of(bi + 1), N, K, sidx + (cur ^ 1) * batch * K);
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// Expert-parallel dispatch: the (token, slot) pairs of a chunk, grouped by the
// rank that holds their expert (bucket = expert / experts_per_rank) in stable
// (token, slot) order, packed without padding at
// offsets[r] + chunk_base[c, r] + rank inside the chunk.  Writes the token row,
// the expert's index on its rank and the gate weight of every pair, and the
// pair's position in the send buffer (send_pos, read by the combine).
// ---------------------------------------------------------------------------
template <typename Tin>
__global__ void __launch_bounds__(256) ep_pack_kernel(const Tin *__restrict__ x, int T, int D, int K, int R, int epr,
                                                      int chunk_tokens, const int *__restrict__ topk_idx,
                                                      const float *__restrict__ topk_w,
                                                      const int *__restrict__ chunk_base,
                                                      const int *__restrict__ offsets, Tin *__restrict__ send_x,
                                                      int *__restrict__ send_expert, float *__restrict__ send_w,
                                                      int *__restrict__ send_pos) {
    extern __shared__ int s_ep[];
    int *s_run = s_ep;          // [R]
    int *s_dest = s_ep + R;     // [chunk_tokens * K]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c = blockIdx.x;
    const int t_begin = c * chunk_tokens, t_end = min(T, t_begin + chunk_tokens);
    const int n_entries = (t_end - t_begin) * K;
    const int64_t f0 = (int64_t)t_begin * K;
    for (int r = tid; r < R; r += blockDim.x) s_run[r] = offsets[r] + chunk_base[(size_t)c * R + r];
    __syncthreads();
    if (warp == 0) {
        for (int base = 0; base < n_entries; base += 32) {
            const int f = base + lane;
            const int e = f < n_entries ? topk_idx[f0 + f] : -1;
            int r = e >= 0 ? e / epr : -1;
            if (f < n_entries && (e < 0 || r >= R)) {
                set_status(kStatusBounds);
                r = -1;
            }
            const unsigned peers = __match_any_sync(0xffffffffu, r);
            const int rank = __popc(peers & lanemask_lt());
            const int base_pos = r >= 0 ? s_run[r] : 0;
            __syncwarp();
            if (r >= 0 && lane == __ffs(peers) - 1) s_run[r] = base_pos + __popc(peers);
            __syncwarp();
            if (f < n_entries) {
                const int dest = r >= 0 ? base_pos + rank : -1;
                s_dest[f] = dest;
                send_pos[f0 + f] = dest;
                if (dest >= 0) {
                    send_expert[dest] = e - r * epr;
                    send_w[dest] = topk_w[f0 + f];
                }
            }
        }
    }
    __syncthreads();
    constexpr int VEC = 16 / sizeof(Tin);
    const int nvec = D / VEC;
    for (int f = warp; f < n_entries; f += blockDim.x / 32) {
        const int dest = s_dest[f];
        if (dest < 0) continue;
        const uint4 *src = reinterpret_cast<const uint4 *>(x + (int64_t)(t_begin + f / K) * D);
        uint4 *dst = reinterpret_cast<uint4 *>(send_x + (int64_t)dest * D);
        for (int v = lane; v < nvec; v += 32) dst[v] = __ldg(src + v);
    }
}

// ---------------------------------------------------------------------------
// Scan: per expert, the exclusive prefix of the chunk histograms (chunk_base);
// then, in the last block to finish, the per-expert counts, their exclusive
// scan (offsets) and the padded segment starts (row_offsets, multiples of
// kRowAlign); padding rows get slot -1.  Grid: ceil(N/32) blocks of 32 warps,
// warp w of block b owns expert 32b + w; each lane loads 16 consecutive chunk
// counts at once.  *counter must be 0 at launch.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) scan_kernel(const int *__restrict__ chunk_counts, int n_chunks, int N,
                                                    int64_t expect_total, int capacity, int *__restrict__ chunk_base,
                                                    int *__restrict__ counts, int *__restrict__ offsets,
                                                    int *__restrict__ row_offsets, int *__restrict__ perm_slot,
                                                    int *__restrict__ counts_out, unsigned *__restrict__ counter,
                                                    int *__restrict__ live, int *__restrict__ n_live) {
    constexpr int CPL = 16;
    __shared__ int s_cnt[1024];
    __shared__ int s_row[1025];
    __shared__ bool s_last;
    __shared__ int s_routed;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int e = blockIdx.x * 32 + warp;
    if (e < N) {
        int carry = 0;
        for (int c0 = 0; c0 < n_chunks; c0 += 32 * CPL) {
            const int cb = c0 + lane * CPL;
            int v[CPL];
#pragma unroll
            for (int i = 0; i < CPL; ++i) v[i] = cb + i < n_chunks ? chunk_counts[(size_t)(cb + i) * N + e] : 0;
            int run = 0;
#pragma unroll
            for (int i = 0; i < CPL; ++i) run += v[i];
            int incl = run;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += n;
            }
            int base = carry + incl - run;
#pragma unroll
            for (int i = 0; i < CPL; ++i) {
                if (cb + i < n_chunks) chunk_base[(size_t)(cb + i) * N + e] = base;
                base += v[i];
            }
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) counts[e] = carry;
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        s_last = atomicAdd(counter, 1u) == gridDim.x - 1;
        s_routed = 0;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    int routed = 0;
    for (int i = tid; i < N; i += blockDim.x) {
        const int c = __ldcg(counts + i);
        if (counts_out) counts_out[i] = c;          // the router's choice
        routed += c;
        s_cnt[i] = min(c, capacity);                // rows each expert accepts
        counts[i] = s_cnt[i];
    }
    routed = __reduce_add_sync(0xffffffffu, routed);
    if (lane == 0 && routed) atomicAdd(&s_routed, routed);
    __syncthreads();
    if (warp == 0) {
        int carry = 0, pcarry = 0;
        for (int e0 = 0; e0 < N; e0 += 32) {
            const int ee = e0 + lane;
            const int c = ee < N ? s_cnt[ee] : 0;
            const int pc = (c + kRowAlign - 1) / kRowAlign * kRowAlign;
            int ic = c, ip = pc;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n1 = __shfl_up_sync(0xffffffffu, ic, o);
                const int n2 = __shfl_up_sync(0xffffffffu, ip, o);
                if (lane >= o) { ic += n1; ip += n2; }
            }
            if (ee < N) {
                offsets[ee] = carry + ic - c;
                row_offsets[ee] = pcarry + ip - pc;
                s_row[ee] = pcarry + ip - pc;
            }
            carry += __shfl_sync(0xffffffffu, ic, 31);
            pcarry += __shfl_sync(0xffffffffu, ip, 31);
        }
        if (lane == 0) {
            offsets[N] = carry;
            row_offsets[N] = pcarry;
            s_row[N] = pcarry;
            if ((int64_t)s_routed != expect_total) set_status(kStatusBounds);
        }
        // ascending list of the experts that received tokens
        int nl = 0;
        for (int e0 = 0; e0 < N; e0 += 32) {
            const int ee = e0 + lane;
            const bool has = ee < N && s_cnt[ee] > 0;
            const unsigned m = __ballot_sync(0xffffffffu, has);
            if (has) live[nl + __popc(m & lanemask_lt())] = ee;
            nl += __popc(m);
        }
        if (lane == 0) *n_live = nl;
    }
    __syncthreads();
    for (int ee = warp; ee < N; ee += 32) {
        const int start = s_row[ee] + s_cnt[ee], end = s_row[ee + 1];
        for (int r = start + lane; r < end; r += 32) perm_slot[r] = -1;
    }
}

// ---------------------------------------------------------------------------
// Permute: stable rank of every (token, slot) entry of a chunk inside its
// expert (ascending token, then slot), its permuted row, the two index maps,
// and the copy of the token row into the expert-contiguous buffer.
// ---------------------------------------------------------------------------
// Grid: (chunks, split).  Every block of a chunk ranks the chunk's entries
// (cheap, identical results); block (c, 0) writes the index maps and block
// (c, s) copies the entries f with f % split == s.  With counts (the rows each
// expert keeps), the blocks also clear the padding rows of every segment
// (rows counts[e] .. the next 128-row boundary), spread over all blocks: the
// grouped GEMMs compute those rows too, and zero operands draw less power on
// the tensor cores than stale data (measured: up and down projections 2.6%
// faster at the DeepSeek-V3 shape under the power cap).
template <typename Tin>
__global__ void __launch_bounds__(256) permute_kernel(const Tin *__restrict__ x, int T, int D, int K, int N,
                                                      int chunk_tokens, int capacity, const int *__restrict__ topk_idx,
                                                      const int *__restrict__ chunk_base,
                                                      const int *__restrict__ row_offsets, int *__restrict__ perm_slot,
                                                      int *__restrict__ slot_row, Tin *__restrict__ x_perm,
                                                      float *__restrict__ y_zero, const int *__restrict__ counts) {
    pdl_enter();
    extern __shared__ int s_perm[];
    int *s_run = s_perm;            // [N] next position inside each expert's assignments
    int *s_row0 = s_perm + N;       // [N] first row of each expert's segment
    int *s_pad = s_perm + 2 * N;    // [N + 1] padding rows before each expert (exclusive prefix)
    int *s_dest = s_perm + 3 * N + 1;   // [chunk_tokens * K]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c = blockIdx.x;
    const bool writer = blockIdx.y == 0;
    const int t_begin = c * chunk_tokens;
    const int t_end = min(T, t_begin + chunk_tokens);
    const int n_entries = (t_end - t_begin) * K;
    const int64_t f0 = (int64_t)t_begin * K;
    const int n_tok = t_end - t_begin;
    constexpr int VEC = 16 / sizeof(Tin);
    const int nvec = D / VEC;
    // loads that do not wait for the ranking go out first: the chunk's expert
    // indices (all threads, into s_dest, one round trip) and each warp's first
    // token's first 128 slices
    for (int f = tid; f < n_entries; f += blockDim.x) s_dest[f] = topk_idx[f0 + f];
    const int tt_first = blockIdx.y + gridDim.y * warp;
    constexpr int kInFlight = 4;    // 16-byte slices per lane in flight
    uint4 pre[kInFlight];
    if (tt_first < n_tok) {
        const uint4 *src = reinterpret_cast<const uint4 *>(x + (int64_t)(t_begin + tt_first) * D);
#pragma unroll
        for (int u = 0; u < kInFlight; ++u)
            if (lane + 32 * u < nvec) pre[u] = __ldg(src + lane + 32 * u);
    }
    for (int e = tid; e < N; e += blockDim.x) {
        s_run[e] = chunk_base[(size_t)c * N + e];
        s_row0[e] = row_offsets[e];
    }
    __syncthreads();
    if (counts && warp == 1) {   // padding rows per expert, exclusive prefix
        int carry = 0;
        for (int e0 = 0; e0 < N; e0 += 32) {
            const int e = e0 + lane;
            const int pad = e < N ? (e + 1 < N ? s_row0[e + 1] : row_offsets[N]) - s_row0[e] - counts[e] : 0;
            int incl = pad;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            if (e < N) s_pad[e] = carry + incl - pad;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) s_pad[N] = carry;
    }
    if (warp == 0) {
        for (int base = 0; base < n_entries; base += 32) {
            const int f = base + lane;
            int e = f < n_entries ? s_dest[f] : -1;   // overwritten by its destination below
            if (f < n_entries && (e < 0 || e >= N)) {
                set_status(kStatusBounds);
                e = -1;
            }
            const unsigned peers = __match_any_sync(0xffffffffu, e);
            const int rank = __popc(peers & lanemask_lt());
            const int leader = __ffs(peers) - 1;
            const int base_row = e >= 0 ? s_run[e] : 0;
            __syncwarp();
            if (e >= 0 && lane == leader) s_run[e] = base_row + __popc(peers);
            __syncwarp();
            if (f < n_entries) {
                // the assignment's position among its expert's: accepted below the capacity
                const int pos = base_row + rank;
                int dest = (e >= 0 && pos < capacity) ? s_row0[e] + pos : -1;
                // bounds-check build: the row lies inside its expert's padded segment
                if (dest >= 0 && !MOE_BOUNDS(pos >= 0 && dest < (e + 1 < N ? s_row0[e + 1] : row_offsets[N])))
                    dest = -1;
                s_dest[f] = dest;
                if (writer) {
                    if (dest >= 0) perm_slot[dest] = (int)(f0 + f);
                    slot_row[f0 + f] = dest;
                }
            }
        }
    }
    __syncthreads();
    // one token per warp at a time: each 16-byte slice of its row is loaded
    // once (four in flight per lane) and written to all K of its rows; when
    // y_zero is given the warp also clears the token's fp32 output row, which
    // the down projection then accumulates into
    for (int tt = tt_first; tt < n_tok; tt += 8 * gridDim.y) {
        const uint4 *src = reinterpret_cast<const uint4 *>(x + (int64_t)(t_begin + tt) * D);
        const int *dest = s_dest + tt * K;
        for (int v0 = lane; v0 < nvec; v0 += 32 * kInFlight) {
            uint4 r[kInFlight];
            const bool prefetched = tt == tt_first && v0 == lane;
#pragma unroll
            for (int u = 0; u < kInFlight; ++u)
                if (v0 + 32 * u < nvec) r[u] = prefetched ? pre[u] : __ldg(src + v0 + 32 * u);
            for (int j = 0; j < K; ++j) {
                const int d = dest[j];
                if (d < 0) continue;
                uint4 *dst = reinterpret_cast<uint4 *>(x_perm + (int64_t)d * D);
#pragma unroll
                for (int u = 0; u < kInFlight; ++u)
                    if (v0 + 32 * u < nvec) dst[v0 + 32 * u] = r[u];
            }
        }
        if (y_zero) {
            uint4 *yr = reinterpret_cast<uint4 *>(y_zero + (int64_t)(t_begin + tt) * D);
            for (int v = lane; v < D / 4; v += 32) yr[v] = make_uint4(0u, 0u, 0u, 0u);
        }
    }
    if (counts) {
        // padding row q (of s_pad[N]) is cleared by block q mod (blocks); its expert by
        // binary search over the prefix
        const int G = gridDim.x * gridDim.y, gi = blockIdx.y * gridDim.x + blockIdx.x;
        for (int q = gi; q < s_pad[N]; q += G) {
            int lo = 0, hi = N - 1;   // the last e with s_pad[e] <= q
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (s_pad[mid] <= q) lo = mid;
                else hi = mid - 1;
            }
            const int64_t row = (int64_t)s_row0[lo] + counts[lo] + (q - s_pad[lo]);
            if (!MOE_BOUNDS(counts[lo] >= 0 && row < row_offsets[N])) continue;
            uint4 *dst = reinterpret_cast<uint4 *>(x_perm + row * D);
            for (int v = tid; v < nvec; v += blockDim.x) dst[v] = make_uint4(0u, 0u, 0u, 0u);
        }
    }
}

// Zero n16 16-byte words at p (a memset that takes part in programmatic
// dependent launch); with tbl, also write the shared expert's one-group
// dispatch table there: live = {0}, one live group, count T, first row 0.
__global__ void __launch_bounds__(256) zero_kernel(uint4 *__restrict__ p, int64_t n16, int *__restrict__ tbl,
                                                   int tbl_T) {
    pdl_enter();
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n16; i += (int64_t)gridDim.x * blockDim.x)
        p[i] = make_uint4(0u, 0u, 0u, 0u);
    if (tbl && blockIdx.x == 0 && threadIdx.x == 0) {
        tbl[0] = 0;
        tbl[1] = 1;
        tbl[2] = tbl_T;
        tbl[3] = 0;
    }
}

// ---------------------------------------------------------------------------
// Combine: y[t] = z[t, 0] + z[t, 1] + ... + z[t, K-1], left to right (slot
// order), no atomics ("MoE(Mixture of Experts)", section (2), Forward, which
// adds the weighted expert outputs of a row in selection order); then, with a
// shared expert, + s[t] (its output, added after the routed sum).
// ---------------------------------------------------------------------------
// slot_row: the permuted row of each slot, -1 for a slot dropped by the
// capacity limit (it adds nothing); z_by_row: z rows are permuted rows (bf16
// prefill) rather than slots; z_rows: the rows z holds (checked in the
// bounds-check build).
template <typename Tout>
__global__ void __launch_bounds__(256) combine_kernel(const float *__restrict__ z, int64_t z_rows, int64_t T, int D,
                                                      int K, const int *__restrict__ slot_row, int z_by_row,
                                                      const float *__restrict__ shared, Tout *__restrict__ y) {
    pdl_enter();
    const int64_t nq = T * (D / 4);
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < nq; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = i / (D / 4);
        const int d = (int)(i - t * (D / 4)) * 4;
        // z row of slot (t, j): its permuted row or t*K + j; -1 when the slot was dropped
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        bool first = true;
        for (int j = 0; j < K; ++j) {
            const int rr = __ldg(slot_row + t * K + j);
            if (rr < 0) continue;
            const int64_t r = z_by_row ? (int64_t)rr : t * K + j;
            if (!MOE_BOUNDS(r < z_rows)) continue;
            const float4 v = *reinterpret_cast<const float4 *>(z + r * D + d);
            if (first) {
                acc = v;
                first = false;
            } else {
                acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
            }
        }
        if (shared) {
            const float4 v = *reinterpret_cast<const float4 *>(shared + t * D + d);
            acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
        }
        if constexpr (sizeof(Tout) == 4) {
            *reinterpret_cast<float4 *>(y + t * D + d) = acc;
        } else {
            uint2 o;
            o.x = pack_bf16x2(acc.x, acc.y);
            o.y = pack_bf16x2(acc.z, acc.w);
            *reinterpret_cast<uint2 *>(y + t * D + d) = o;
        }
    }
}

// ---------------------------------------------------------------------------
// Statistics.  Each block reduces a fixed range of tokens to partial sums per
// expert (full-softmax probabilities, gate weights, counts) in a fixed order;
// the last block to finish adds the partials block by block, also in a fixed
// order, and computes the scalars in double precision:
//   f_e = counts_e / (T K); switch = N sum f_e P_e; simple = N sum f_e^2;
//   CV^2 = population variance / mean^2 (0 when the mean is 0).
// No float atomics anywhere, so the results do not depend on scheduling.
// ---------------------------------------------------------------------------
struct AuxOut {
    int *counts;
    float *importance;
    float *p_mean;
    float *scalars;
};

__device__ void aux_finalize_block(const float *__restrict__ part_p, const float *__restrict__ part_imp,
                                   const int *__restrict__ part_cnt, int nblk, int T, int N, int K, AuxOut out) {
    __shared__ float f_p[1024], f_i[1024];
    __shared__ int f_c[1024];
    __shared__ float q_p[1024], q_i[1024];
    __shared__ int q_c[1024];
    const int nt = blockDim.x, tid = threadIdx.x;
    int Q = 1;
    while (Q * 2 * N <= nt && Q * 2 <= 32) Q *= 2;   // threads per expert
    for (int e0 = 0; e0 < N; e0 += nt / Q) {
        const int e = e0 + tid / Q, q = tid % Q;
        float p = 0.f, im = 0.f;
        int c = 0;
        if (tid / Q < nt / Q && e < N) {
#pragma unroll 16
            for (int bb = q; bb < nblk; bb += Q) {
                p += __ldcg(part_p + (size_t)bb * N + e);
                im += __ldcg(part_imp + (size_t)bb * N + e);
                c += __ldcg(part_cnt + (size_t)bb * N + e);
            }
        }
        q_p[tid] = p;
        q_i[tid] = im;
        q_c[tid] = c;
        __syncthreads();
        if (q == 0 && tid / Q < nt / Q && e < N) {
            float sp = 0.f, si = 0.f;
            int sc = 0;
            for (int j = 0; j < Q; ++j) { sp += q_p[tid + j]; si += q_i[tid + j]; sc += q_c[tid + j]; }
            f_p[e] = T > 0 ? sp / (float)T : 0.f;
            f_i[e] = si;
            f_c[e] = sc;
        }
        __syncthreads();
    }
    for (int e = tid; e < N; e += nt) {
        if (out.counts) out.counts[e] = f_c[e];
        if (out.importance) out.importance[e] = f_i[e];
        if (out.p_mean) out.p_mean[e] = f_p[e];
    }
    if (tid == 0 && out.scalars) {
        double sw = 0.0, ss = 0.0, mi = 0.0, mc = 0.0;
        const double tk = (double)T * (double)K;
        const double inv_tk = tk > 0 ? 1.0 / tk : 0.0;
        const double inv_n = 1.0 / N;
        for (int e = 0; e < N; ++e) {
            const double f = f_c[e] * inv_tk;
            sw += f * f_p[e];
            ss += f * f;
            mi += f_i[e];
            mc += f_c[e];
        }
        mi *= inv_n;
        mc *= inv_n;
        double vi = 0.0, vc = 0.0;
        for (int e = 0; e < N; ++e) {
            vi += (f_i[e] - mi) * (f_i[e] - mi);
            vc += (f_c[e] - mc) * (f_c[e] - mc);
        }
        vi *= inv_n;
        vc *= inv_n;
        out.scalars[0] = (float)(N * sw);
        out.scalars[1] = (float)(N * ss);
        out.scalars[2] = mi == 0.0 ? 0.f : (float)(vi / (mi * mi));
        out.scalars[3] = mc == 0.0 ? 0.f : (float)(vc / (mc * mc));
    }
}

// Returns true in every thread of the block that finished last (*counter must
// start at 0 for the launch).
__device__ __forceinline__ bool last_block_done(unsigned *counter) {
    __shared__ bool s_last;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(counter, 1u) == gridDim.x - 1;
    __syncthreads();
    if (s_last) __threadfence();
    return s_last;
}

// N <= NP <= 32: one thread per token, 256 tokens per block.
template <int NP>
__global__ void __launch_bounds__(256) aux_small_kernel(const float *__restrict__ logits,
                                                        const int *__restrict__ topk_idx,
                                                        const float *__restrict__ topk_w, int T, int N, int K,
                                                        float *__restrict__ part_p, float *__restrict__ part_imp,
                                                        int *__restrict__ part_cnt, unsigned *__restrict__ counter,
                                                        AuxOut out) {
    __shared__ float w_p[8][NP], w_i[8][NP];
    __shared__ int w_c[8][NP];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int t = blockIdx.x * 256 + tid;
    float p[NP], im[NP];
    int c[NP];
#pragma unroll
    for (int e = 0; e < NP; ++e) { p[e] = 0.f; im[e] = 0.f; c[e] = 0; }
    if (t < T) {
        float s[NP];
        float mx = -INFINITY;
#pragma unroll
        for (int e = 0; e < NP; ++e) {
            s[e] = e < N ? logits[(size_t)t * N + e] : -INFINITY;
            mx = fmaxf(mx, s[e]);
        }
        float z = 0.f;
#pragma unroll
        for (int e = 0; e < NP; ++e) {
            s[e] = e < N ? expf(s[e] - mx) : 0.f;
            z += s[e];
        }
        const float inv_z = 1.0f / z;
#pragma unroll
        for (int e = 0; e < NP; ++e) p[e] = s[e] * inv_z;
        for (int j = 0; j < K; ++j) {
            const int ej = topk_idx[(size_t)t * K + j];
            const float wj = topk_w[(size_t)t * K + j];
            if (ej < 0 || ej >= N) set_status(kStatusBounds);
#pragma unroll
            for (int e = 0; e < NP; ++e)
                if (e == ej) { im[e] += wj; c[e] += 1; }
        }
    }
#pragma unroll
    for (int e = 0; e < NP; ++e) {
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            p[e] += __shfl_xor_sync(0xffffffffu, p[e], o);
            im[e] += __shfl_xor_sync(0xffffffffu, im[e], o);
            c[e] += __shfl_xor_sync(0xffffffffu, c[e], o);
        }
    }
    if (lane == 0) {
#pragma unroll
        for (int e = 0; e < NP; ++e) { w_p[warp][e] = p[e]; w_i[warp][e] = im[e]; w_c[warp][e] = c[e]; }
    }
    __syncthreads();
    if (tid < N) {
        float sp = 0.f, si = 0.f;
        int sc = 0;
        for (int w = 0; w < 8; ++w) { sp += w_p[w][tid]; si += w_i[w][tid]; sc += w_c[w][tid]; }
        part_p[(size_t)blockIdx.x * N + tid] = sp;
        part_imp[(size_t)blockIdx.x * N + tid] = si;
        part_cnt[(size_t)blockIdx.x * N + tid] = sc;
    }
    if (last_block_done(counter)) aux_finalize_block(part_p, part_imp, part_cnt, gridDim.x, T, N, K, out);
}

// Any N: one warp per token (lane holds experts lane, lane+32, ...), kAuxTokens
// tokens per block, warp-private shared rows accumulated in token order and
// added in warp order.
__global__ void __launch_bounds__(256) aux_partial_kernel(const float *__restrict__ logits,
                                                          const int *__restrict__ topk_idx,
                                                          const float *__restrict__ topk_w, int T, int N, int K,
                                                          float *__restrict__ part_p, float *__restrict__ part_imp,
                                                          int *__restrict__ part_cnt, unsigned *__restrict__ counter,
                                                          AuxOut out) {
    extern __shared__ float s_aux[];
    float *acc_p = s_aux;                                     // [8][N]
    float *acc_i = s_aux + 8 * N;                             // [8][N]
    int *acc_c = reinterpret_cast<int *>(s_aux + 16 * N);     // [8][N]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int i = tid; i < 8 * N; i += blockDim.x) { acc_p[i] = 0.f; acc_i[i] = 0.f; acc_c[i] = 0; }
    __syncthreads();
    const int t_begin = blockIdx.x * kAuxTokens;
    const int t_end = min(T, t_begin + kAuxTokens);
    for (int t = t_begin + warp; t < t_end; t += 8) {
        const float *s = logits + (size_t)t * N;
        float mx = -INFINITY;
        for (int e = lane; e < N; e += 32) mx = fmaxf(mx, s[e]);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        float zsum = 0.f;
        for (int e = lane; e < N; e += 32) zsum += expf(s[e] - mx);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) zsum += __shfl_xor_sync(0xffffffffu, zsum, o);
        for (int e = lane; e < N; e += 32) acc_p[warp * N + e] += expf(s[e] - mx) / zsum;
        if (lane == 0) {
            for (int j = 0; j < K; ++j) {
                const int e = topk_idx[(size_t)t * K + j];
                if (e < 0 || e >= N) {
                    set_status(kStatusBounds);
                    continue;
                }
                acc_i[warp * N + e] += topk_w[(size_t)t * K + j];
                acc_c[warp * N + e] += 1;
            }
        }
        __syncwarp();
    }
    __syncthreads();
    for (int e = tid; e < N; e += blockDim.x) {
        float p = 0.f, im = 0.f;
        int c = 0;
        for (int w = 0; w < 8; ++w) { p += acc_p[w * N + e]; im += acc_i[w * N + e]; c += acc_c[w * N + e]; }
        part_p[(size_t)blockIdx.x * N + e] = p;
        part_imp[(size_t)blockIdx.x * N + e] = im;
        part_cnt[(size_t)blockIdx.x * N + e] = c;
    }
    if (last_block_done(counter)) aux_finalize_block(part_p, part_imp, part_cnt, gridDim.x, T, N, K, out);
}

// ---------------------------------------------------------------------------
// Statistics as exact integer sums, for data parallelism.  Under token-sharded
// data parallelism the layer's losses are defined over the global batch (the
// Shazeer article's Importance(X) and Load(X) sum over the batch X; the chapter
// "MoE(Mixture of Experts)", section (3), takes f_e over all routed tokens), so
// each rank's partial sums are added across ranks and then finalised.  Here
// every partial is an integer: per expert the routed slots, the gate weights
// and the full-softmax probabilities, each term rounded to 2^-32 fixed point.
// Integer additions give the same bits in any order -- inside the kernel (its
// atomics), across ranks (an all-reduce of int64) -- so every rank finalises
// the same numbers.
//   part[0, N)    counts
//   part[N, 2N)   sum of round(w * 2^32) over the slots routed to e
//   part[2N, 3N)  sum over tokens of round(softmax(scores)_e * 2^32)
//   part[3N]      tokens
// ---------------------------------------------------------------------------
constexpr double kFixScale = 4294967296.0;

// part must be zero at launch.  One warp per token; per-block sums in shared
// memory (integer atomics), then one global integer atomic per nonzero entry.
__global__ void __launch_bounds__(256) aux_partials_kernel(const float *__restrict__ logits,
                                                           const int *__restrict__ topk_idx,
                                                           const float *__restrict__ topk_w, int T, int N, int K,
                                                           unsigned long long *__restrict__ part) {
    extern __shared__ unsigned long long s_fx[];   // [3N]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int i = tid; i < 3 * N; i += blockDim.x) s_fx[i] = 0ull;
    __syncthreads();
    for (int t = blockIdx.x * 8 + warp; t < T; t += gridDim.x * 8) {
        const float *row = logits + (size_t)t * N;
        float mx = -INFINITY;
        for (int e = lane; e < N; e += 32) {
            const float v = row[e];
            mx = fmaxf(mx, v != v ? -INFINITY : v);
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        float z = 0.f;
        for (int e = lane; e < N; e += 32) {
            const float v = row[e];
            z += (v != v || mx == -INFINITY) ? 0.f : expf(v - mx);
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
        for (int e = lane; e < N; e += 32) {
            const float v = row[e];
            const float pe = (v != v || mx == -INFINITY) ? 0.f : expf(v - mx) / z;
            const unsigned long long q = __double2ull_rn((double)pe * kFixScale);
            if (q) atomicAdd(&s_fx[2 * N + e], q);
        }
        for (int j = lane; j < K; j += 32) {
            const int e = topk_idx[(size_t)t * K + j];
            if (e < 0 || e >= N) {
                set_status(kStatusBounds);
                continue;
            }
            atomicAdd(&s_fx[e], 1ull);
            atomicAdd(&s_fx[N + e], __double2ull_rn((double)topk_w[(size_t)t * K + j] * kFixScale));
        }
    }
    __syncthreads();
    for (int i = tid; i < 3 * N; i += blockDim.x)
        if (s_fx[i]) atomicAdd(part + i, s_fx[i]);
    if (blockIdx.x == 0 && tid == 0) atomicAdd(part + 3 * N, (unsigned long long)T);
}

// The statistics from summed partials (the layout above).  Shared by the device
// kernel and the host entry point, so both give the same bits:
//   counts_e, importance_e = fixed / 2^32, p_mean_e = fixed / 2^32 / T,
//   f_e = counts_e / (T K); switch = N sum_e f_e P_e; simple = N sum_e f_e^2;
//   CV^2 = population variance / mean^2 (0 when the mean is 0); sums over e in
// ascending order, in double precision.  All zero when T = 0.
__host__ __device__ inline void aux_finalize_partials(int N, int K, const long long *part, int *counts,
                                                      float *importance, float *p_mean, float *scalars) {
    const long long T = part[3 * N];
    const double tk = (double)T * (double)K;
    double sw = 0.0, ss = 0.0, si = 0.0, sc = 0.0;
    for (int e = 0; e < N; ++e) {
        const double c = (double)part[e];
        const double im = (double)part[N + e] / kFixScale;
        const double pm = T > 0 ? (double)part[2 * N + e] / kFixScale / (double)T : 0.0;
        if (counts) counts[e] = (int)part[e];
        if (importance) importance[e] = (float)im;
        if (p_mean) p_mean[e] = (float)pm;
        const double f = tk > 0 ? c / tk : 0.0;
        sw += f * pm;
        ss += f * f;
        si += im;
        sc += c;
    }
    const double mi = si / N, mc = sc / N;
    double vi = 0.0, vc = 0.0;
    for (int e = 0; e < N; ++e) {
        const double im = (double)part[N + e] / kFixScale, c = (double)part[e];
        vi += (im - mi) * (im - mi);
        vc += (c - mc) * (c - mc);
    }
    vi /= N;
    vc /= N;
    if (scalars) {
        scalars[0] = (float)(N * sw);
        scalars[1] = (float)(N * ss);
        scalars[2] = mi == 0.0 ? 0.f : (float)(vi / (mi * mi));
        scalars[3] = mc == 0.0 ? 0.f : (float)(vc / (mc * mc));
    }
}

__global__ void aux_finalize_kernel(int N, int K, const long long *__restrict__ part, AuxOut out) {
    if (blockIdx.x == 0 && threadIdx.x == 0)
        aux_finalize_partials(N, K, part, out.counts, out.importance, out.p_mean, out.scalars);
}

// W_g [D, N] -> W_g^T [N, D] (the K-major operand layout of the router GEMM).
template <typename Tin>
__global__ void transpose_kernel(const Tin *__restrict__ src, int R, int C, Tin *__restrict__ dst) {
    pdl_enter();
    __shared__ Tin tile[32][33];
    const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {
        const int r = r0 + i, c = c0 + threadIdx.x;
        if (r < R && c < C) tile[i][threadIdx.x] = src[(size_t)r * C + c];
    }
    __syncthreads();
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {
        const int c = c0 + i, r = r0 + threadIdx.x;
        if (r < R && c < C) dst[(size_t)c * R + r] = tile[threadIdx.x][i];
    }
}

// Bounded-wait self-test: one thread waits on a barrier nothing completes.
__global__ void wait_selftest_kernel(uint64_t timeout_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        mbar_wait(&bar, 0, timeout_ns);
    }
}

}  // namespace moe
