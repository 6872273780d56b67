// moe_router_tc.cuh -- routers for bf16 layers with N <= 256 (tensor cores) and
// for few tokens (N <= 32), each with top-k, statistics and the dispatch scan
// in one launch.
//
// Routing follows "MoE(Mixture of Experts)", section (2), Route: scores x W_g
// (+ b_g), the K best experts of a stable descending sort (equal scores keep
// ascending expert index), and the softmax over only the kept scores shifted
// by the best one -- softmax(KeepTopK(H, k)) of the Shazeer article (qiita),
// gating section, inference form.  Statistics follow the Shazeer article's
// load-balancing section and the Switch-style loss: per expert the mean of the
// full N-way softmax, the importance (sum of gate weights) and the counts.
//
// router_tc_kernel   one CTA per tile of 128 tokens: tcgen05.mma computes the
//   128 x N logits (fp32 accumulation of exact bf16 products, operands staged by
//   TMA); each of 128 epilogue threads owns one token (one TMEM lane), keeps the
//   K best (value, index) pairs in a static insertion network, computes the
//   gate weights and its full-softmax probabilities; the tile's per-expert
//   probability sums are reduced in a fixed order (lanes, then warps), its
//   counts and gate-weight sums with shared-memory atomics on integers (gate
//   weights in 2^-32 fixed point), which are exact and order-independent.
// router_few_kernel  few tokens (T <= 64, N <= 32): several blocks per token,
//   each over a slab of W_g rows with lane = expert (coalesced row loads); the
//   block completing a token adds the slabs in order and selects the top k;
//   the token's probabilities, gate weights and counts are its partials.
// In both, the last block to finish (atomic ticket) turns the per-tile (or
// per-token) partials into the dispatch tables -- per tile and expert the first
// row of its tokens inside the expert's segment, per-expert counts and offsets,
// segment starts padded to 128 rows, padding slots -1, the ascending list of
// experts with tokens -- and the statistics, scalars in double precision.  No
// float atomics anywhere: results do not depend on scheduling.
#pragma once

#include "moe_common.cuh"
#include "moe_route.cuh"

namespace moe {
namespace rtc {

constexpr int BM = 128;   // tokens per tile (= dispatch chunk)
constexpr int BK = 64;
constexpr int kThreads = 192;   // warp 0 TMA, warp 1 MMA, warps 2..5 one token per thread
constexpr double kImpScale = 4294967296.0;   // gate weights summed in 2^-32 fixed point

struct Params {
    int T, D, N, K, np;                  // np: N rounded up to the MMA width
    const float *bg;                     // [N] or nullptr
    const float *bsel;                   // [N] or nullptr: selection-only bias (changes the kept set only)
    float *logits;                       // [T, N]
    int *topk_idx;                       // [T, K]
    float *topk_w;                       // [T, K]
    int *tile_counts;                    // [tiles, N]
    unsigned long long *sum_p;           // [N] full-softmax probability sums, 2^-32 fixed point (zero at launch)
    unsigned long long *sum_imp;         // [N] gate-weight sums, 2^-32 fixed point (zero at launch)
    unsigned *ticket;                    // zero at launch
    // dispatch tables (written by the last block)
    int *chunk_base;                     // [tiles, N] first row (relative to the expert's segment) of the tile's tokens
    int *counts;                         // [N]
    int *offsets;                        // [N+1]
    int *row_offsets;                    // [N+1]
    int *perm_slot;                      // padding rows -> -1
    int *live;                           // [N]
    int *n_live;
    int *counts_out;                     // [N] or nullptr (moe_route)
    int capacity;                        // rows each expert accepts (assignments beyond are dropped)
    // statistics (each may be nullptr)
    int *aux_counts;
    float *aux_importance, *aux_p_mean, *aux_scalars;
    // SIMT router: the layer's fp32 output [T, D] to clear (each block its chunk's
    // rows) for the down projection's reductions, or nullptr
    float *y_zero;
    // SIMT router with the dispatch (cooperative launch): the kept rows' copies,
    // the slot -> row map, the arrivals of its grid barrier (zero at launch)
    __nv_bfloat16 *x_perm;
    int *slot_row;
    unsigned *grid_bar;
    uint64_t timeout_ns;
};

// Scratch of the finalisation (shared memory, up to 256 experts, 256 threads).
// 16-byte aligned size: barriers and 8-byte words are placed right after it.
struct __align__(16) FinalScratch {
    int cnt[256];
    float pm[256];
    float im[256];
    int row[257];
    int q_cnt[256];
};

// Executed by every thread of the last block.  The blocks have added their
// probability and gate-weight sums into sum_p / sum_imp (integer sums, exact
// and order-independent) and written their per-expert token counts per tile.
// The [tiles, N] count matrix is loaded into cnt_smem (cap ints of the
// kernel's shared memory, no longer used by then) in one coalesced pass when
// it fits; per expert e, Q threads then take contiguous tile ranges for the
// totals and the exclusive scan that gives each tile's first row.
// At most 256 threads work (the scratch arrays' size); larger blocks' other
// threads only take part in the barriers.
__device__ __forceinline__ void finalize_tables(const Params &p, int ntiles, FinalScratch &f, int *cnt_smem, int cap) {
    const int N = p.N, tid = threadIdx.x;
    const int nt = blockDim.x < 256 ? (int)blockDim.x : 256;
    const bool worker = tid < nt;
    const int warp = tid >> 5, lane = tid & 31;
    const bool in_smem = cnt_smem != nullptr && (int64_t)ntiles * N <= cap;
    if (in_smem) {
        // 16-byte loads, eight in flight per thread (the matrix starts 16-byte aligned)
        const int total = ntiles * N;
        const int total4 = total / 4;
        const int4 *src4 = reinterpret_cast<const int4 *>(p.tile_counts);
        int4 *dst4 = reinterpret_cast<int4 *>(cnt_smem);
        for (int i0 = tid; worker && i0 < total4; i0 += 8 * nt) {
            int4 v[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) v[k] = i0 + k * nt < total4 ? __ldcg(src4 + i0 + k * nt) : make_int4(0, 0, 0, 0);
#pragma unroll
            for (int k = 0; k < 8; ++k)
                if (i0 + k * nt < total4) dst4[i0 + k * nt] = v[k];
        }
        for (int i = total4 * 4 + tid; worker && i < total; i += nt) cnt_smem[i] = __ldcg(p.tile_counts + i);
        __syncthreads();
    }
    // one pointer for both cases (generic loads reach shared or global memory), so the
    // loops below hold no per-element choice between two kinds of load
    const int *cm = in_smem ? cnt_smem : p.tile_counts;
    auto count_at = [&](int c, int e) -> int { return cm[(int64_t)c * N + e]; };
    int Q = nt / N;
    Q = Q < 1 ? 1 : (Q > 32 ? 32 : Q);
    const int epp = nt / Q;                       // experts per pass
    const int R = (ntiles + Q - 1) / Q;           // tiles per thread
    for (int e0 = 0; e0 < N; e0 += epp) {
        const int e = e0 + tid / Q, q = tid % Q;
        const bool act = worker && tid < epp * Q && e < N;
        const int c0 = q * R, c1 = min(ntiles, c0 + R);
        int cnt = 0;
        if (act) {
#pragma unroll 8
            for (int c = c0; c < c1; ++c) cnt += count_at(c, e);
        }
        if (worker) f.q_cnt[tid] = cnt;
        __syncthreads();
        int base = 0;
        if (act) {
            for (int j = 0; j < q; ++j) base += f.q_cnt[tid - q + j];   // tiles before this range
            if (q == 0) {
                int tc = 0;
                for (int j = 0; j < Q; ++j) tc += f.q_cnt[tid + j];
                f.cnt[e] = tc;
                f.pm[e] = p.T > 0 ? (float)((double)__ldcg(p.sum_p + e) / kImpScale / (double)p.T) : 0.f;
                f.im[e] = (float)((double)__ldcg(p.sum_imp + e) / kImpScale);
            }
            // eight tiles' counts read together, then the running base written
            for (int cb = c0; cb < c1; cb += 8) {
                int v[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) v[k] = cb + k < c1 ? count_at(cb + k, e) : 0;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    if (cb + k < c1) p.chunk_base[(int64_t)(cb + k) * N + e] = base;
                    base += v[k];
                }
            }
        }
        __syncthreads();
    }
    // the dispatch tables hold each expert's accepted rows, min(count, capacity);
    // the statistics and moe_route's counts the router's own choice
    for (int e = tid; e < N; e += nt) {
        p.counts[e] = min(f.cnt[e], p.capacity);
        if (p.counts_out) p.counts_out[e] = f.cnt[e];
        if (p.aux_counts) p.aux_counts[e] = f.cnt[e];
        if (p.aux_p_mean) p.aux_p_mean[e] = f.pm[e];
        if (p.aux_importance) p.aux_importance[e] = f.im[e];
    }
    if (warp == 0) {
        int carry = 0, pcarry = 0, nl = 0;
        int routed = 0;
        for (int e0 = 0; e0 < N; e0 += 32) {
            const int e = e0 + lane;
            routed += e < N ? f.cnt[e] : 0;
            const int c = e < N ? min(f.cnt[e], p.capacity) : 0;
            const int pc = (c + kRowAlign - 1) / kRowAlign * kRowAlign;
            int ic = c, ip = pc;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n1 = __shfl_up_sync(0xffffffffu, ic, o);
                const int n2 = __shfl_up_sync(0xffffffffu, ip, o);
                if (lane >= o) { ic += n1; ip += n2; }
            }
            if (e < N) {
                p.offsets[e] = carry + ic - c;
                p.row_offsets[e] = pcarry + ip - pc;
                f.row[e] = pcarry + ip - pc;
            }
            const unsigned m = __ballot_sync(0xffffffffu, c > 0);
            if (c > 0) p.live[nl + __popc(m & lanemask_lt())] = e;
            nl += __popc(m);
            carry += __shfl_sync(0xffffffffu, ic, 31);
            pcarry += __shfl_sync(0xffffffffu, ip, 31);
        }
        if (lane == 0) {
            p.offsets[N] = carry;
            p.row_offsets[N] = pcarry;
            f.row[N] = pcarry;
            *p.n_live = nl;
        }
        routed = __reduce_add_sync(0xffffffffu, routed);
        if (lane == 0) {
            if ((int64_t)routed != (int64_t)p.T * p.K) set_status(kStatusBounds);
        }
    } else if (warp == 1 && p.aux_scalars) {
        // f_e = counts_e / (T K); switch = N sum f P; simple = N sum f^2;
        // CV^2 = popvar / mean^2; lanes take experts lane, lane+32, ...; xor tree in double
        const double tk = (double)p.T * (double)p.K;
        const double inv_tk = tk > 0 ? 1.0 / tk : 0.0;
        double sw = 0.0, ss = 0.0, si = 0.0, sc = 0.0;
        for (int e = lane; e < N; e += 32) {
            const double fe = f.cnt[e] * inv_tk;
            sw += fe * f.pm[e];
            ss += fe * fe;
            si += f.im[e];
            sc += f.cnt[e];
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            sw += __shfl_xor_sync(0xffffffffu, sw, o);
            ss += __shfl_xor_sync(0xffffffffu, ss, o);
            si += __shfl_xor_sync(0xffffffffu, si, o);
            sc += __shfl_xor_sync(0xffffffffu, sc, o);
        }
        const double mi = si / N, mc = sc / N;
        double vi = 0.0, vc = 0.0;
        for (int e = lane; e < N; e += 32) {
            vi += (f.im[e] - mi) * (f.im[e] - mi);
            vc += (f.cnt[e] - mc) * (f.cnt[e] - mc);
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            vi += __shfl_xor_sync(0xffffffffu, vi, o);
            vc += __shfl_xor_sync(0xffffffffu, vc, o);
        }
        vi /= N;
        vc /= N;
        if (lane == 0) {
            p.aux_scalars[0] = (float)(N * sw);
            p.aux_scalars[1] = (float)(N * ss);
            p.aux_scalars[2] = mi == 0.0 ? 0.f : (float)(vi / (mi * mi));
            p.aux_scalars[3] = mc == 0.0 ? 0.f : (float)(vc / (mc * mc));
        }
    }
    __syncthreads();
    for (int e = warp; worker && e < N; e += nt / 32) {
        const int start = f.row[e] + min(f.cnt[e], p.capacity), end = f.row[e + 1];
        for (int rr = start + lane; rr < end; rr += 32) p.perm_slot[rr] = -1;
    }
}

// True in every thread of the block that finished last.
// The barrier orders the block's stores before thread 0's acquire-release
// ticket, whose release covers them; in the last block the acquire, followed
// by the second barrier, lets its other threads read what the other blocks
// wrote.
__device__ __forceinline__ bool last_block(unsigned *ticket, int *s_flag) {
    __syncthreads();
    if (threadIdx.x == 0) *s_flag = ticket_arrive(ticket) == gridDim.x - 1;
    __syncthreads();
    return *s_flag != 0;
}

template <int NP>
struct Shape {
    static constexpr uint32_t kABytes = BM * BK * 2;
    static constexpr uint32_t kBBytes = NP * BK * 2;
    static constexpr uint32_t kStageBytes = kABytes + kBBytes;
    static constexpr int kStages0 = (160 * 1024) / (int)kStageBytes;
    static constexpr int kStages = kStages0 > 8 ? 8 : kStages0;
    static constexpr uint32_t kTmemCols = NP <= 32 ? 32 : NP <= 64 ? 64 : NP <= 128 ? 128 : 256;
    // the epilogue's score tile [BM][NP + 1] and 1/z per row reuse the ring
    static_assert((size_t)BM * (NP + 1) * 4 + BM * 4 <= (size_t)kStages * kStageBytes, "score tile exceeds the ring");
    // ring + per-warp probability rows + tile counters + finalisation scratch + barriers
    static constexpr size_t kSmem = 1024 + (size_t)kStages * kStageBytes + 4 * 256 * 4 + 256 * 4 + 256 * 8 +
                                    sizeof(FinalScratch) + (2 * kStages + 2) * 8 + 64;
};

// Columns [c, c+32) (or [c, c+16)) of this thread's TMEM lane as floats.
__device__ __forceinline__ void ld_cols32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    tmem_ld_32x32b_x32(taddr, r);
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void ld_cols16(uint32_t taddr, float (&v)[32]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
#pragma unroll
    for (int i = 16; i < 32; ++i) v[i] = 0.f;
}

// The logit of expert e from its accumulator: bias added, NaN ranked as -inf (flagged).
__device__ __forceinline__ float score(const float *bg, float acc, int e) {
    float s = acc + (bg ? __ldg(bg + e) : 0.f);
    if (s != s) {
        set_status(kStatusNanLogit);
        s = -INFINITY;
    }
    return s;
}

template <int NP, int KM>
__global__ void __launch_bounds__(kThreads, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                     const Params p) {
    pdl_enter();
    using S = Shape<NP>;
    constexpr int kStages = S::kStages;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = align_smem_1024(smem_raw);
    uint8_t *sA = smem;
    uint8_t *sB = smem + kStages * S::kABytes;
    float *s_wp = reinterpret_cast<float *>(sB + kStages * S::kBBytes);                  // [256] (of [4][256])
    int *s_cnt = reinterpret_cast<int *>(s_wp + 4 * 256);                                 // [256]
    unsigned long long *s_imp = reinterpret_cast<unsigned long long *>(s_cnt + 256);      // [256]
    FinalScratch *fs = reinterpret_cast<FinalScratch *>(s_imp + 256);
    uint64_t *full = reinterpret_cast<uint64_t *>(fs + 1);
    uint64_t *empty = full + kStages;
    uint64_t *tfull = empty + kStages;
    uint64_t *drain = tfull + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    int *s_flag = reinterpret_cast<int *>(tmem_slot + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tile = blockIdx.x;
    const int nkb = (p.D + BK - 1) / BK;
    for (int e = threadIdx.x; e < 256; e += blockDim.x) {
        s_cnt[e] = 0;
        s_imp[e] = 0ull;
    }
    if (warp == 0 && lane == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(tfull, 1);
        mbar_init(drain, 1);
        fence_mbar_init();
        tma_prefetch_desc(&tmX);
        tma_prefetch_desc(&tmW);
    }
    if (warp == 1) tmem_alloc(tmem_slot, S::kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            IssuedSlots iss;
            for (int kb = 0; kb < nkb; ++kb) {
                if (!mbar_wait(&empty[stage], phase ^ 1, p.timeout_ns)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(&full[stage], S::kStageBytes);
                tma_load_2d(&tmX, &full[stage], sA + stage * S::kABytes, kb * BK, tile * BM);
                tma_load_2d(&tmW, &full[stage], sB + stage * S::kBBytes, kb * BK, 0);
                iss.note(stage, phase);
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1;
                }
            }
            if (!ok) iss.drain(full, p.timeout_ns);   // copies in flight land before the CTA leaves
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(BM, NP);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int kb = 0; kb < nkb; ++kb) {
                if (!mbar_wait(&full[stage], phase, p.timeout_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t adesc = smem_desc_sw128(smem_u32(sA + stage * S::kABytes));
                const uint64_t bdesc = smem_desc_sw128(smem_u32(sB + stage * S::kBBytes));
#pragma unroll
                for (int k = 0; k < BK / 16; ++k)
                    tc_mma_bf16(tmem_base, adesc + 2 * k, bdesc + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
                tc_commit(&empty[stage]);
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1;
                }
            }
            if (ok) tc_commit(tfull);
            else {
                tc_commit(drain);
                mbar_wait(drain, 0, p.timeout_ns);
            }
        }
    } else {
        // ------------------------------------------------------------ one token per thread
        // warp w may only read TMEM lanes 32*(w%4)..+31, which fixes the rows it owns.
        // The scores go through a padded [BM][NP + 1] fp32 tile in the ring (free once
        // the MMAs are complete): coalesced logits rows, conflict-free row scans for the
        // top-k, and per-expert column sums over the tile's tokens in token order.
        const int ew = warp & 3;
        const int r = ew * 32 + lane;            // row of the tile = TMEM lane
        const int t = tile * BM + r;
        const bool live_row = t < p.T;
        constexpr int LD = NP + 1;
        float *S = reinterpret_cast<float *>(smem);   // [BM][LD]
        float *inv_z_s = S + BM * LD;                  // [BM]
        const bool have = __all_sync(0xffffffffu, mbar_wait(tfull, 0, p.timeout_ns));   // warp-uniform
        tc_fence_after();
        float smax = -INFINITY;
        if (have) {
            const uint32_t tlane = tmem_base + (static_cast<uint32_t>(ew * 32) << 16);
            float *row = S + r * LD;
            bool nan_seen = false;
#pragma unroll 1
            for (int c = 0; c < NP; c += 32) {
                float v[32];
                if (NP - c >= 32) ld_cols32(tlane + c, v);
                else ld_cols16(tlane + c, v);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int e = c + i;
                    if (e < p.N && (NP - c >= 32 || i < 16)) {
                        float sc = v[i] + (p.bg ? __ldg(p.bg + e) : 0.f);
                        nan_seen |= sc != sc;
                        sc = sc != sc ? -INFINITY : sc;   // NaN ranked as -inf (flagged below)
                        row[e] = sc;
                        smax = fmaxf(smax, sc);
                    }
                }
            }
            if (nan_seen) set_status(kStatusNanLogit);
            __syncwarp();
            // logits: this warp's 32 rows, each stored by the whole warp (coalesced)
            for (int rr = 0; rr < 32; ++rr) {
                const int tt = tile * BM + ew * 32 + rr;
                if (tt >= p.T) break;
                const float *src = S + (ew * 32 + rr) * LD;
                for (int e = lane; e < p.N; e += 32) p.logits[(int64_t)tt * p.N + e] = src[e];
            }
            // top-K of the selection values, best first (larger value, then lower index):
            // each expert as one 64-bit key, the value's order-preserving bits above the
            // complemented index, entering the sorted key list with all positions compared
            // at once (selects only); the raw scores are read back for the kept experts
            unsigned long long tk[KM];
#pragma unroll
            for (int j = 0; j < KM; ++j) tk[j] = 0ull;   // below every real key (NaN became -inf)
            for (int e = 0; e < p.N; ++e) {
                const float sv = p.bsel ? row[e] + __ldg(p.bsel + e) : row[e];
                const uint32_t u = __float_as_uint(sv);
                const uint32_t o = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
                const unsigned long long k = ((unsigned long long)o << 32) | (uint32_t)~e;
                bool b[KM];
#pragma unroll
                for (int j = 0; j < KM; ++j) b[j] = k > tk[j];
#pragma unroll
                for (int j = KM - 1; j >= 0; --j) {
                    const unsigned long long nk = (j > 0 && b[j - 1]) ? tk[j - 1] : k;
                    tk[j] = b[j] ? nk : tk[j];
                }
            }
            float tr[KM];
            int te[KM];
#pragma unroll
            for (int j = 0; j < KM; ++j) {
                te[j] = (int)~(uint32_t)tk[j];
                tr[j] = j < p.K ? row[te[j]] : -INFINITY;
            }
            // gate weights: softmax over the K kept raw scores, shifted by their largest
            // (slot 0's without a selection bias), slot order
            float kmax = -INFINITY;
#pragma unroll
            for (int j = 0; j < KM; ++j)
                if (j < p.K) kmax = fmaxf(kmax, tr[j]);
            float ex[KM];
            float sum = 0.f;
#pragma unroll
            for (int j = 0; j < KM; ++j) {
                ex[j] = j < p.K ? expf(tr[j] - kmax) : 0.f;
                sum += ex[j];
            }
            const float inv = 1.0f / sum;
#pragma unroll
            for (int j = 0; j < KM; ++j) {
                if (j < p.K && live_row) {
                    const float wj = ex[j] * inv;
                    p.topk_idx[(int64_t)t * p.K + j] = te[j];
                    p.topk_w[(int64_t)t * p.K + j] = wj;
                    atomicAdd(&s_cnt[te[j]], 1);
                    atomicAdd(&s_imp[te[j]], (unsigned long long)__double2ull_rn((double)wj * kImpScale));
                }
            }
            // the full softmax of the raw scores: exponentials in place, the normaliser
            float z = 0.f;
            for (int e = 0; e < p.N; ++e) {
                const float x = expf(row[e] - smax);
                row[e] = x;
                z += x;
            }
            inv_z_s[r] = live_row ? 1.0f / z : 0.f;
        }
        // per-expert probability sums over the tile's tokens, rows ascending (the four
        // epilogue warps meet on named barrier 1)
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (__all_sync(0xffffffffu, have)) {
            const int et = threadIdx.x - 64;
            for (int e = et; e < p.N; e += 128) {
                float ps = 0.f;
                for (int rr = 0; rr < BM; ++rr) ps = fmaf(S[rr * LD + e], inv_z_s[rr], ps);
                s_wp[e] = ps;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    for (int e = threadIdx.x; e < p.N; e += blockDim.x) {
        atomicAdd(p.sum_p + e, __double2ull_rn((double)s_wp[e] * kImpScale));
        atomicAdd(p.sum_imp + e, s_imp[e]);
        p.tile_counts[(int64_t)tile * p.N + e] = s_cnt[e];
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, S::kTmemCols);
    }
    if (last_block(p.ticket, s_flag))
        finalize_tables(p, gridDim.x, *fs, reinterpret_cast<int *>(smem),
                        (int)(kStages * (S::kABytes + S::kBBytes) / 4));
}

// ---------------------------------------------------------------------------
// N <= 32 experts (bf16): SIMT router.  One block of 256 threads per chunk of
// kSimtChunk tokens.  W_g is staged transposed ([NP][D], rows N..NP-1 zero) in
// shared memory; each warp takes 32/NP tokens at a time, one segment of NP
// lanes per token, each lane a strided set of 16-byte slices of its token's x
// row (four in flight) against all NP experts; a reduce-scatter inside the
// segment leaves lane l with the score of (token l/NP, expert l%NP).
// Per token: logits, the top k (ties to the lower index), renormalised gate
// weights and the full-softmax probabilities.  Each lane accumulates, for its
// expert and in token order, probabilities, counts and 2^-32 fixed-point gate
// weights; lanes of the same expert, then warps, are added in fixed order into
// the chunk's partials, and the last block builds the tables.
// ---------------------------------------------------------------------------
constexpr int kSimtChunk = 32;

// Reduce-scatter over a segment of NP lanes (aligned at a multiple of NP):
// afterwards lane seg_lane holds, in a[0], the segment's sum of entry seg_lane.
template <int NP>
__device__ __forceinline__ void reduce_scatter_seg(float (&a)[NP], int seg_lane) {
#pragma unroll
    for (int C = NP; C >= 2; C /= 2) {
        const int H = C / 2;
        const bool upper = (seg_lane & H) != 0;
#pragma unroll
        for (int i = 0; i < H; ++i) {
            const float send = upper ? a[i] : a[i + H];
            const float keep = upper ? a[i + H] : a[i];
            a[i] = keep + __shfl_xor_sync(0xffffffffu, send, H);
        }
    }
}

// Shared memory of the SIMT router: W_g transposed ([NP][D] bf16), per-warp
// partials, finalisation scratch.
template <int NP>
struct SimtShape {
    __host__ __device__ static constexpr size_t w_bytes(int D) { return ((size_t)NP * D * 2 + 15) / 16 * 16; }
    static size_t smem_bytes(int D) { return w_bytes(D) + 256 * (4 + 4 + 8) + sizeof(FinalScratch) + 16; }
};

// acc + x.lo * w.lo + x.hi * w.hi for two bf16 pairs, with sm_100's mixed
// fp32 += bf16 x bf16 FMA: the products are exact and each step rounds as an
// fp32 FMA of the widened values would, without widening them first.
__device__ __forceinline__ float fma_bf16x2_acc(uint32_t x, uint32_t w, float acc) {
    asm("{\n\t.reg .b16 xl, xh, wl, wh;\n\tmov.b32 {xl, xh}, %1;\n\tmov.b32 {wl, wh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, xl, wl, %0;\n\tfma.rn.f32.bf16 %0, xh, wh, %0;\n\t}"
        : "+f"(acc)
        : "r"(x), "r"(w));
    return acc;
}

// ---------------------------------------------------------------------------
// The dispatch inside the SIMT router (DISPATCH = true): after a grid barrier
// (the launch is cooperative, every block resident), every block adds up the
// chunk counts of all blocks -- per expert its total and the tokens of the
// chunks before its own, one warp per expert -- and scatters its own chunk's
// (token, slot) pairs into the expert segments (stable, capacity applied);
// block 0 writes the tables and the statistics.  This replaces the last
// block's serial table build and the separate permute launch.
// ---------------------------------------------------------------------------
__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned *ptr) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ptr) : "memory");
    return v;
}

__device__ void simt_dispatch_chunk(const Params &p, const __nv_bfloat16 *__restrict__ x, int n_chunks, int *sm) {
    const int N = p.N, K = p.K, T = p.T, D = p.D;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c = blockIdx.x;
    int *s_tot = sm, *s_base = sm + 32, *s_kept = sm + 64, *s_row = sm + 96;   // s_row [33]
    int *s_run = sm + 136, *s_dest = sm + 176;                                 // s_dest [chunk * K]
    for (int e = warp; e < N; e += blockDim.x / 32) {
        int tot = 0, base = 0;
        for (int c0 = 0; c0 < n_chunks; c0 += 256) {   // eight chunk counts in flight per lane
            int v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int cc = c0 + lane + 32 * u;
                v[u] = cc < n_chunks ? __ldcg(p.tile_counts + (int64_t)cc * N + e) : 0;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                tot += v[u];
                if (c0 + lane + 32 * u < c) base += v[u];
            }
        }
        tot = __reduce_add_sync(0xffffffffu, tot);
        base = __reduce_add_sync(0xffffffffu, base);
        if (lane == 0) {
            s_tot[e] = tot;
            s_base[e] = base;
        }
    }
    __syncthreads();
    if (warp == 0) {
        const int cnt = lane < N ? s_tot[lane] : 0;
        const int kp = min(cnt, p.capacity);
        const int pad = (kp + kRowAlign - 1) / kRowAlign * kRowAlign;
        int ik = kp, ip = pad;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int a = __shfl_up_sync(0xffffffffu, ik, o), b = __shfl_up_sync(0xffffffffu, ip, o);
            if (lane >= o) { ik += a; ip += b; }
        }
        s_kept[lane] = kp;
        s_row[lane] = ip - pad;
        if (lane == 31) s_row[32] = ip;
        s_run[lane] = lane < N ? s_base[lane] : 0;
        if (c == 0) {
            if (lane < N) {
                p.counts[lane] = kp;
                p.offsets[lane] = ik - kp;
                p.row_offsets[lane] = ip - pad;
                const float im = (float)((double)__ldcg(p.sum_imp + lane) / kImpScale);
                const float pm = T > 0 ? (float)((double)__ldcg(p.sum_p + lane) / kImpScale / (double)T) : 0.f;
                if (p.aux_counts) p.aux_counts[lane] = cnt;
                if (p.aux_importance) p.aux_importance[lane] = im;
                if (p.aux_p_mean) p.aux_p_mean[lane] = pm;
            }
            const unsigned m = __ballot_sync(0xffffffffu, kp > 0);
            if (kp > 0) p.live[__popc(m & lanemask_lt())] = lane;
            const int routed = __reduce_add_sync(0xffffffffu, cnt);
            if (lane == N - 1) {
                p.offsets[N] = ik;
                p.row_offsets[N] = ip;
            }
            if (lane == 0) {
                *p.n_live = __popc(m);
                if ((int64_t)routed != (int64_t)T * K) set_status(kStatusBounds);
            }
        }
    } else if (warp == 1 && c == 0 && p.aux_scalars) {
        // f_e = counts / (T K); switch = N sum f P; simple = N sum f^2; CV^2 = popvar / mean^2
        const double tk = (double)T * (double)K;
        double sw = 0.0, ss = 0.0, si = 0.0, sc = 0.0, im = 0.0, cn = 0.0;
        if (lane < N) {
            cn = s_tot[lane];
            im = (double)__ldcg(p.sum_imp + lane) / kImpScale;
            const double pm = T > 0 ? (double)__ldcg(p.sum_p + lane) / kImpScale / (double)T : 0.0;
            const double fe = tk > 0 ? cn / tk : 0.0;
            sw = fe * (double)(float)pm;
            ss = fe * fe;
            si = (double)(float)im;
            sc = cn;
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            sw += __shfl_xor_sync(0xffffffffu, sw, o);
            ss += __shfl_xor_sync(0xffffffffu, ss, o);
            si += __shfl_xor_sync(0xffffffffu, si, o);
            sc += __shfl_xor_sync(0xffffffffu, sc, o);
        }
        const double mi = si / N, mc = sc / N;
        double vi = lane < N ? ((double)(float)im - mi) * ((double)(float)im - mi) : 0.0;
        double vc = lane < N ? (cn - mc) * (cn - mc) : 0.0;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            vi += __shfl_xor_sync(0xffffffffu, vi, o);
            vc += __shfl_xor_sync(0xffffffffu, vc, o);
        }
        vi /= N;
        vc /= N;
        if (lane == 0) {
            p.aux_scalars[0] = (float)(N * sw);
            p.aux_scalars[1] = (float)(N * ss);
            p.aux_scalars[2] = mi == 0.0 ? 0.f : (float)(vi / (mi * mi));
            p.aux_scalars[3] = mc == 0.0 ? 0.f : (float)(vc / (mc * mc));
        }
    }
    __syncthreads();
    if (c == 0) {   // padding rows of every segment
        for (int e = warp; e < N; e += blockDim.x / 32) {
            const int start = s_row[e] + s_kept[e], end = s_row[e + 1];
            for (int r = start + lane; r < end; r += 32) p.perm_slot[r] = -1;
        }
    }
    // this chunk's (token, slot) pairs: stable rank inside each expert, then the copies
    const int t_begin = c * kSimtChunk, t_end = min(T, t_begin + kSimtChunk);
    const int n_entries = (t_end - t_begin) * K;
    const int64_t f0 = (int64_t)t_begin * K;
    // the chunk's expert indices in one round trip (into s_dest, overwritten below)
    for (int f = tid; f < n_entries; f += blockDim.x) s_dest[f] = __ldcg(p.topk_idx + f0 + f);
    __syncthreads();
    if (warp == 0) {
        for (int base = 0; base < n_entries; base += 32) {
            const int f = base + lane;
            int e = f < n_entries ? s_dest[f] : -1;
            if (f < n_entries && (e < 0 || e >= N)) {
                set_status(kStatusBounds);
                e = -1;
            }
            const unsigned peers = __match_any_sync(0xffffffffu, e);
            const int rank = __popc(peers & lanemask_lt());
            const int run = e >= 0 ? s_run[e] : 0;
            __syncwarp();
            if (e >= 0 && lane == __ffs(peers) - 1) s_run[e] = run + __popc(peers);
            __syncwarp();
            if (f < n_entries) {
                const int pos = run + rank;
                const int dest = (e >= 0 && pos < s_kept[e]) ? s_row[e] + pos : -1;
                s_dest[f] = dest;
                if (dest >= 0) p.perm_slot[dest] = (int)(f0 + f);
                p.slot_row[f0 + f] = dest;
            }
        }
    }
    __syncthreads();
    // the copies: a warp takes four of its tokens at a time (tt, tt + W, tt + 2W,
    // tt + 3W for W warps), their slices' loads in flight together
    const int nvec = D / 8;
    const int W = blockDim.x / 32, n_tok = t_end - t_begin;
    for (int tt = warp; tt < n_tok; tt += 4 * W) {
        for (int v0 = lane; v0 < nvec; v0 += 128) {
            uint4 r[4][4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int tq = tt + q * W;
                const uint4 *src = reinterpret_cast<const uint4 *>(x + (int64_t)(t_begin + tq) * D);
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    if (tq < n_tok && v0 + 32 * u < nvec) r[q][u] = __ldg(src + v0 + 32 * u);
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int tq = tt + q * W;
                if (tq >= n_tok) break;
                for (int j = 0; j < K; ++j) {
                    const int d = s_dest[tq * K + j];
                    if (d < 0) continue;
                    uint4 *dst = reinterpret_cast<uint4 *>(p.x_perm + (int64_t)d * D);
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        if (v0 + 32 * u < nvec) dst[v0 + 32 * u] = r[q][u];
                }
            }
        }
    }
}

template <int NP, bool DISPATCH>
__global__ void __launch_bounds__(256, NP == 8 ? 2 : 1) router_simt_kernel(const __nv_bfloat16 *__restrict__ x,
                                                                          const __nv_bfloat16 *__restrict__ Wg,
                                                                          const Params p) {
    pdl_enter();
    constexpr int TPW = 32 / NP;
    constexpr int kSimtU = 8;   // 16-byte slices of x in flight per lane
    using WT = __nv_bfloat16;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const int D = p.D, N = p.N, K = p.K, T = p.T;
    WT *WgT = reinterpret_cast<WT *>(smem_raw);
    float *s_p = reinterpret_cast<float *>(smem_raw + SimtShape<NP>::w_bytes(D));   // [8][32]
    int *s_c = reinterpret_cast<int *>(s_p + 256);                                        // [8][32]
    unsigned long long *s_i = reinterpret_cast<unsigned long long *>(s_c + 256);          // [8][32]
    FinalScratch *fs = reinterpret_cast<FinalScratch *>(s_i + 256);
    int *s_flag = reinterpret_cast<int *>(fs + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // W_g [D][N] -> WgT [NP][D]: 16-byte reads of the flat matrix, eight in
    // flight per thread, (d, e) advanced per element
    for (int i = tid; i < (NP - N) * D; i += blockDim.x) WgT[(size_t)N * D + i] = WT(0.f);
    const int total = D * N;
    if ((reinterpret_cast<uintptr_t>(Wg) & 15) == 0) {
        for (int i_base = tid * 8; i_base < total; i_base += blockDim.x * 8 * 8) {
            uint4 v[8];
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const int i0 = i_base + r * blockDim.x * 8;
                if (i0 + 8 <= total) {
                    v[r] = __ldg(reinterpret_cast<const uint4 *>(Wg + i0));
                } else {
                    __nv_bfloat16 t8[8];
#pragma unroll
                    for (int k = 0; k < 8; ++k) t8[k] = i0 + k < total ? Wg[i0 + k] : __float2bfloat16(0.f);
                    v[r] = *reinterpret_cast<const uint4 *>(t8);
                }
            }
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const int i0 = i_base + r * blockDim.x * 8;
                if (i0 >= total) break;
                const __nv_bfloat16 *t8 = reinterpret_cast<const __nv_bfloat16 *>(&v[r]);
                int d = i0 / N, e = i0 - d * N;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    if (i0 + k < total) WgT[(size_t)e * D + d] = WT(t8[k]);
                    if (++e == N) { e = 0; ++d; }
                }
            }
        }
    } else {
        for (int i = tid; i < total; i += blockDim.x) {
            const int d = i / N, e = i - d * N;
            WgT[(size_t)e * D + d] = WT(Wg[i]);
        }
    }
    __syncthreads();

    const int t_begin = blockIdx.x * kSimtChunk;
    const int nvec = D / 8;
    const int seg_lane = lane % NP, seg_base = lane - seg_lane;
    const int e = seg_lane;
    const bool valid_e = e < N;
    float acc_p = 0.f;
    int acc_c = 0;
    unsigned long long acc_i = 0ull;
    for (int g = warp * TPW; g < kSimtChunk; g += 8 * TPW) {
        const int t0 = t_begin + g;
        const int t = t0 + lane / NP;
        const uint4 *xrow = reinterpret_cast<const uint4 *>(x + (int64_t)t * D);
        float a[NP];
#pragma unroll
        for (int i = 0; i < NP; ++i) a[i] = 0.f;
        for (int v0 = seg_lane; v0 < nvec; v0 += NP * kSimtU) {
            uint4 xr[kSimtU];
#pragma unroll
            for (int u = 0; u < kSimtU; ++u) {
                const int v = v0 + NP * u;
                xr[u] = (t < T && v < nvec) ? __ldg(xrow + v) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < kSimtU; ++u) {
                const int v = v0 + NP * u;
                if (v >= nvec) break;
                {
                    const uint32_t xw[4] = {xr[u].x, xr[u].y, xr[u].z, xr[u].w};
#pragma unroll
                    for (int ee = 0; ee < NP; ++ee) {
                        const uint4 w4 = *reinterpret_cast<const uint4 *>(WgT + (size_t)ee * D + (size_t)v * 8);
                        a[ee] = fma_bf16x2_acc(xw[0], w4.x, a[ee]);
                        a[ee] = fma_bf16x2_acc(xw[1], w4.y, a[ee]);
                        a[ee] = fma_bf16x2_acc(xw[2], w4.z, a[ee]);
                        a[ee] = fma_bf16x2_acc(xw[3], w4.w, a[ee]);
                    }
                }
            }
        }
        reduce_scatter_seg<NP>(a, seg_lane);
        const bool tok = t < T;
        float s = a[0];
        if (valid_e && p.bg) s += p.bg[e];
        if (tok && valid_e) p.logits[(int64_t)t * N + e] = s;
        if (s != s) {
            if (valid_e && tok) set_status(kStatusNanLogit);
            s = -INFINITY;
        }
        int slot_e;
        float slot_w;
        const bool has = segment_topk<NP>(sel_value(p.bsel, s, e, valid_e), s, e, !valid_e, K, seg_lane, lane, slot_e,
                                          slot_w);
        if (has && tok) {
            p.topk_idx[(int64_t)t * K + seg_lane] = slot_e;
            p.topk_w[(int64_t)t * K + seg_lane] = slot_w;
        }
        // the token's full softmax (segment of NP lanes); its counts and gate weights per expert
        float mx = valid_e ? s : -INFINITY;
#pragma unroll
        for (int o = NP / 2; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        const float ex = valid_e ? expf(s - mx) : 0.f;
        float z = ex;
#pragma unroll
        for (int o = NP / 2; o >= 1; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
        if (tok && valid_e) acc_p += ex / z;
        for (int j = 0; j < K; ++j) {
            const int ej = __shfl_sync(0xffffffffu, slot_e, seg_base + j);
            const float wj = __shfl_sync(0xffffffffu, slot_w, seg_base + j);
            if (tok && valid_e && ej == e) {
                ++acc_c;
                acc_i += __double2ull_rn((double)wj * kImpScale);
            }
        }
    }
    // lanes e, e+NP, ... hold the same expert: fixed xor tree, then warps in order
#pragma unroll
    for (int o = NP; o < 32; o <<= 1) {
        acc_p += __shfl_xor_sync(0xffffffffu, acc_p, o);
        acc_c += __shfl_xor_sync(0xffffffffu, acc_c, o);
        acc_i += __shfl_xor_sync(0xffffffffu, acc_i, o);
    }
    if (lane < NP) {
        s_p[warp * 32 + lane] = acc_p;
        s_c[warp * 32 + lane] = acc_c;
        s_i[warp * 32 + lane] = acc_i;
    }
    __syncthreads();
    if (tid < N) {
        float ps = 0.f;
        int cs = 0;
        unsigned long long is = 0ull;
        for (int w = 0; w < 8; ++w) {
            ps += s_p[w * 32 + tid];
            cs += s_c[w * 32 + tid];
            is += s_i[w * 32 + tid];
        }
        p.tile_counts[(int64_t)blockIdx.x * N + tid] = cs;
        atomicAdd(p.sum_p + tid, __double2ull_rn((double)ps * kImpScale));
        atomicAdd(p.sum_imp + tid, is);
    }
    if (DISPATCH) {
        // the chunk's partials are written: arrive, clear this chunk's rows of y
        // while the others arrive, wait (bounded), then dispatch
        __syncthreads();
        if (tid == 0) asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(p.grid_bar) : "memory");
        if (p.y_zero) {
            const int64_t t0 = (int64_t)blockIdx.x * kSimtChunk;
            const int64_t t1 = t0 + kSimtChunk < T ? t0 + kSimtChunk : (int64_t)T;
            const int64_t n16 = (t1 - t0) * (D / 4);
            uint4 *yb = reinterpret_cast<uint4 *>(p.y_zero + t0 * D);
            for (int64_t i = tid; i < n16; i += blockDim.x) yb[i] = make_uint4(0u, 0u, 0u, 0u);
        }
        if (tid == 0) {
            bool ok = ld_acquire_gpu(p.grid_bar) >= gridDim.x;
            const uint64_t t0 = globaltimer_ns();
            while (!ok) {
#pragma unroll 1
                for (int i = 0; i < 32 && !ok; ++i) ok = ld_acquire_gpu(p.grid_bar) >= gridDim.x;
                if (!ok && globaltimer_ns() - t0 > p.timeout_ns) {
                    set_status(kStatusTimeout);
                    break;
                }
            }
            *s_flag = ok ? 1 : 0;
        }
        __syncthreads();
        if (*s_flag) simt_dispatch_chunk(p, x, gridDim.x, reinterpret_cast<int *>(fs));
        return;
    }
    const bool last = last_block(p.ticket, s_flag);
    if (last)
        finalize_tables(p, gridDim.x, *fs, reinterpret_cast<int *>(smem_raw),
                        (int)(SimtShape<NP>::w_bytes(D) / 4));
    // this chunk's output rows are cleared after the ticket, so that neither the
    // ticket's release nor the tables wait for these stores: they drain while
    // the last block builds the tables (the down projection, which adds into y,
    // starts only after this kernel has completed)
    if (p.y_zero) {
        const int64_t t0 = (int64_t)blockIdx.x * kSimtChunk;
        const int64_t t1 = t0 + kSimtChunk < T ? t0 + kSimtChunk : (int64_t)T;
        const int64_t n16 = (t1 - t0) * (D / 4);
        uint4 *yb = reinterpret_cast<uint4 *>(p.y_zero + t0 * D);
        for (int64_t i = tid; i < n16; i += blockDim.x) yb[i] = make_uint4(0u, 0u, 0u, 0u);
    }
}

// ---------------------------------------------------------------------------
// Few tokens (T <= 64, N <= 32): grid (T, S).  Block (t, s) takes the rows
// [s*rows, (s+1)*rows) of W_g; lane e of every warp owns expert e, so each
// warp-wide load reads one contiguous W_g row, and warp w takes the slab's rows
// w, w+8, ... with kFewUnroll rows in flight.  The block adds its warps' sums
// in warp order and publishes the slab's scores; the block that completes a
// token (an atomic ticket per token) adds the S slabs in slab order, selects
// the top k and writes the token's partials (full-softmax probabilities, gate
// weights, counts: one-token "tiles"); the last token's block builds the
// tables.  Every sum has a fixed order, so results do not depend on scheduling.
// ---------------------------------------------------------------------------
constexpr int kFewUnroll = 16;
constexpr int kFewMaxSplits = 16;
constexpr int kFewMaxT = 64;   // tokens (tiles) the few-token router handles

__global__ void __launch_bounds__(256) router_few_kernel(const __nv_bfloat16 *__restrict__ x,
                                                          const __nv_bfloat16 *__restrict__ Wg, const Params p,
                                                          float *__restrict__ slab_scores,   // [T][S][32]
                                                          unsigned *__restrict__ token_ticket, int rows) {
    pdl_enter();
    __shared__ float part[8][32];
    __shared__ FinalScratch fs;
    __shared__ __align__(16) int s_cnt[kFewMaxT * 32];   // the count matrix in the finalisation (16-byte loads)
    __shared__ int s_flag;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int t = blockIdx.x, sl = blockIdx.y, S = gridDim.y, N = p.N, D = p.D;
    const bool live = lane < N;
    const int d_begin = sl * rows, d_end = min(D, d_begin + rows);
    const __nv_bfloat16 *xt = x + (int64_t)t * D;
    float acc = 0.f;
    for (int d0 = d_begin + warp; d0 < d_end; d0 += 8 * kFewUnroll) {
        float wv[kFewUnroll], xv[kFewUnroll];
#pragma unroll
        for (int u = 0; u < kFewUnroll; ++u) {
            const int d = d0 + 8 * u;
            const bool in = d < d_end;
            xv[u] = in ? __bfloat162float(xt[d]) : 0.f;
            wv[u] = (in && live) ? __bfloat162float(Wg[(int64_t)d * N + lane]) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < kFewUnroll; ++u) acc = fmaf(xv[u], wv[u], acc);
    }
    part[warp][lane] = acc;
    __syncthreads();
    if (warp == 0) {
        float v = 0.f;
        for (int w = 0; w < 8; ++w) v += part[w][lane];
        slab_scores[((int64_t)t * S + sl) * 32 + lane] = v;
    }
    __syncthreads();
    if (tid == 0) s_flag = ticket_arrive(token_ticket + t) == (unsigned)(S - 1);
    __syncthreads();
    if (!s_flag) return;   // block-uniform: another slab completes this token
    if (warp == 0) {
        float s = 0.f;
        for (int j = 0; j < S; ++j) s += __ldcg(slab_scores + ((int64_t)t * S + j) * 32 + lane);
        s = live ? score(p.bg, s, lane) : -INFINITY;
        if (live) p.logits[(int64_t)t * N + lane] = s;
        int slot_e;
        float slot_w;
        const bool has = segment_topk<32>(sel_value(p.bsel, s, lane, live), s, lane, !live, p.K, lane, lane, slot_e,
                                          slot_w);
        if (has) {
            p.topk_idx[(int64_t)t * p.K + lane] = slot_e;
            p.topk_w[(int64_t)t * p.K + lane] = slot_w;
        }
        // full softmax of the token; its counts and gate weights per expert
        float mx = s;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        const float ex = live ? expf(s - mx) : 0.f;
        float z = ex;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
        int cnt = 0;
        unsigned long long im = 0;
        for (int j = 0; j < p.K; ++j) {
            const int ej = __shfl_sync(0xffffffffu, slot_e, j);
            const float wj = __shfl_sync(0xffffffffu, slot_w, j);
            if (ej == lane) {
                ++cnt;
                im += __double2ull_rn((double)wj * kImpScale);
            }
        }
        if (live) {
            p.tile_counts[(int64_t)t * N + lane] = cnt;
            atomicAdd(p.sum_p + lane, __double2ull_rn((double)(ex / z) * kImpScale));
            if (im) atomicAdd(p.sum_imp + lane, im);
        }
    }
    if (last_block(p.ticket, &s_flag)) finalize_tables(p, gridDim.x, fs, s_cnt, kFewMaxT * 32);
}

}  // namespace rtc
}  // namespace moe
