// moe_gemm_decode.cuh -- expert GEMMs for few tokens, weight-streaming bound.
//
// With a handful of tokens per expert (decode), the work is reading each live
// expert's weights once from HBM; only the selected experts are touched (the
// Shazeer article's conditional computation; the Transformers-v5 article's
// remark that small batches want a different strategy than grouped_mm).  Here
// the weight rows are the 128-row operand of tcgen05.mma and the expert's
// tokens (at most NT, padded) are the narrow N operand:
//     acc[f, j] = sum_k W[e][f, k] * X[row_offsets[e] + j, k]
// so no tensor-core work is spent on padding rows of tokens, and every CTA
// streams 128 whole weight rows per item.
//
// The work is (live expert, tile of 128 weight rows) tiles, expert-major, each
// of num_k_blocks 64-wide K blocks.  When whole tiles dealt round-robin would
// leave the last wave less than 90% full (e.g. 180 tiles on 148 SMs) and
// split_cap > 0, the tiles x K blocks units are cut into gridDim.x equal
// contiguous ranges, one per persistent CTA (stream-K): every SM streams the
// same number of weight bytes whatever the number of tiles.  A CTA's range is a sequence of pieces (a tile and a K
// range); a tile cut between CTAs has its pieces' fp32 partials written to
// the workspace, and the CTA that finishes its last piece (an atomic ticket per
// tile) adds them in piece order and runs the epilogue, so the result does not
// depend on which CTA finishes when.  Without split_cap the tiles go whole to
// the CTAs round-robin.  One CTA per SM, 192 threads:
//   warp 0      TMA producer: weight tile (16 KB per 64-wide K slice) and the
//               expert's token tile into a kStages-deep ring.
//   warp 1      TMEM allocation; one thread issues 128 x NT x 16 MMAs into one
//               of two TMEM accumulators.
//   warps 2..5  epilogue, warp w owning TMEM lanes (weight rows) 32*(w%4)...:
//     EPI_GELU     h[j, f] = bf16(gelu(acc + b1[f]))   via a shared [NT][128] tile
//     EPI_SWIGLU   rows 0..63 gate, 64..127 the matching up rows of the packed
//                  gate_up weight; h[j, f] = bf16(silu(g) * u)   via shared memory
//     EPI_SCATTER  z[slot(j), d] = w[slot(j)] * (acc + b2[d]), 128-byte rows
// All waits are bounded as in the prefill GEMM.
#pragma once

#include "moe_common.cuh"
#include "moe_gemm_tc.cuh"

namespace moe {
namespace dec {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int kEpiWarps = 4;
constexpr int kThreads = 64 + 32 * kEpiWarps;

enum { EPI_GELU = 0, EPI_SWIGLU = 1, EPI_SCATTER = 2 };

struct Params {
    const int *row_offsets;   // [N+1] token segment starts in the permuted buffers
    const int *counts;        // [N] tokens per expert
    const int *live;          // [N] experts with at least one token, ascending
    const int *n_live;        // number of entries of live
    int tiles_per_group;      // weight-row tiles per expert
    int num_k_blocks;
    int w_group_rows;         // weight rows per expert in the 2-D view
    int w_up_offset;          // SwiGLU: first up row inside an expert (= H)
    int n_valid;              // output features per expert
    void *out;                // h [rows, H] (token rows) or z [T*K, D] (slot rows)
    int64_t ldo;
    const float *bias;        // [N, n_valid] or nullptr
    const int *perm_slot;     // EPI_SCATTER (nullptr: row j is token j, weight 1)
    const float *gate_w;      // EPI_SCATTER
    // stream-K (split_cap == 0: whole tiles round-robin)
    int split_cap;            // CTAs the partial buffer and the tickets are sized for (>= gridDim.x)
    float *part;              // [split_cap][2][BM][NT] fp32: each CTA's first and last cut piece
    unsigned *tickets;        // [split_cap] zero at launch, indexed by the CTA holding a tile's first piece
    uint64_t timeout_ns;
};

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned *ptr) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ptr) : "memory");
    return v;
}

// One CTA's share of the tiles x K-block units and the pieces it is cut into.
struct Work {
    int64_t W;     // units in all
    int G, nkb;    // CTAs, K blocks per tile
    __device__ __forceinline__ int64_t begin(int c) const { return (int64_t)c * W / G; }
    // CTA whose range holds unit u: the largest c with begin(c) <= u
    __device__ __forceinline__ int cta_of(int64_t u) const { return (int)(((u + 1) * G - 1) / W); }
};

// Piece of a CTA's range starting at unit u (< end): its tile and K blocks.
struct Piece {
    int tile, k0, k1;
    __device__ __forceinline__ Piece(int64_t u, int64_t end, int nkb) {
        tile = (int)(u / nkb);
        k0 = (int)(u - (int64_t)tile * nkb);
        const int64_t rest = (int64_t)k0 + (end - u);
        k1 = rest < nkb ? (int)rest : nkb;
    }
};

template <int NT, int EPI>
struct Shape {
    static constexpr uint32_t kABytes = BM * BK * 2;
    static constexpr uint32_t kBBytes = NT * BK * 2;
    static constexpr uint32_t kStageBytes = kABytes + kBBytes;
    static constexpr uint32_t kEpiBytes = EPI == EPI_SWIGLU ? (64 * NT * 4 + NT * 64 * 2)
                                        : EPI == EPI_GELU   ? NT * 128 * 2
                                                            : 0;
    static constexpr int kStages0 = (200 * 1024 - (int)kEpiBytes) / (int)kStageBytes;
    static constexpr int kStages = kStages0 > 8 ? 8 : kStages0;
    static constexpr uint32_t kTmemCols = 2 * NT < 32 ? 32 : 2 * NT;
    static constexpr size_t kSmem = 1024 + (size_t)kStages * kStageBytes + kEpiBytes + (2 * kStages + 6) * 8 + 32;
};

__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t *r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

// All NT accumulator columns of this thread's TMEM lane.
template <int NT>
__device__ __forceinline__ void tmem_ld_row(uint32_t taddr, float (&acc)[NT]) {
    uint32_t r[NT];
    if constexpr (NT == 16) {
        tmem_ld_32x32b_x16(taddr, r);
    } else {
#pragma unroll
        for (int c = 0; c < NT; c += 32) {
            uint32_t q[32];
            tmem_ld_32x32b_x32(taddr + c, q);
#pragma unroll
            for (int i = 0; i < 32; ++i) r[c + i] = q[i];
        }
    }
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < NT; ++i) acc[i] = __uint_as_float(r[i]);
}

// Barrier among the epilogue threads built on an mbarrier (every epilogue
// thread arrives), so that its wait is bounded like every other wait: a warp
// that gives up leaves the loop and the others give up too instead of waiting
// forever.
struct EpiBarrier {
    uint64_t *bar;
    uint32_t phase;
    uint64_t timeout_ns;
    __device__ __forceinline__ bool sync() {
        mbar_arrive(bar);
        const bool ok = __all_sync(0xffffffffu, mbar_wait(bar, phase, timeout_ns));
        phase ^= 1;
        return ok;
    }
};


template <int NT, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    decode_gemm_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                       const Params p) {
    pdl_enter();
    using S = Shape<NT, EPI>;
    constexpr int kStages = S::kStages;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = smem + kStages * S::kABytes;
    uint8_t *sE = sB + kStages * S::kBBytes;
    uint64_t *full = reinterpret_cast<uint64_t *>(sE + S::kEpiBytes);
    uint64_t *empty = full + kStages;
    uint64_t *tfull = empty + kStages;
    uint64_t *tempty = tfull + 2;
    uint64_t *drain = tempty + 2;
    uint64_t *epib = drain + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(epib + 1);
    int *s_last = reinterpret_cast<int *>(tmem_slot + 1);

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
        tma_prefetch_desc(&tmW);
        tma_prefetch_desc(&tmX);
    }
    if (warp == 1) tmem_alloc(tmem_slot, S::kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int tiles = *p.n_live * p.tiles_per_group;
    const int nkb = p.num_k_blocks;
    const Work wk{(int64_t)tiles * nkb, (int)gridDim.x, nkb};
    // stream-K when whole tiles round-robin would leave more than a tenth of
    // the CTA-tile slots of the last wave empty; it needs at least 4 units per
    // CTA, so that every CTA's range is non-empty and every piece of a cut
    // tile exists
    const int waves = (tiles + (int)gridDim.x - 1) / (int)gridDim.x;
    const bool stream_k = p.split_cap >= (int)gridDim.x && wk.W >= 4 * (int64_t)gridDim.x &&
                          10 * tiles < 9 * waves * (int)gridDim.x;
    // stream-K: this CTA's unit range; otherwise whole tiles blockIdx.x, +gridDim.x, ...
    const int64_t u_begin = stream_k ? wk.begin(blockIdx.x) : (int64_t)blockIdx.x * nkb;
    const int64_t u_end = stream_k ? wk.begin(blockIdx.x + 1) : wk.W;
    const int64_t u_step = (int64_t)gridDim.x * nkb;   // whole tiles: on to this CTA's next tile

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            IssuedSlots iss;
            for (int64_t u = u_begin; u < u_end && ok;) {
                const Piece pc(u, stream_k ? u_end : u + nkb, nkb);
                u = stream_k ? u + (pc.k1 - pc.k0) : u + u_step;
                const int tile = pc.tile, k0 = pc.k0, k1 = pc.k1;
                const int g = p.live[tile / p.tiles_per_group];
                const int mt = tile % p.tiles_per_group;
                const int trow = p.row_offsets[g];
                int wrow, wrow2 = 0;
                if (EPI == EPI_SWIGLU) {
                    wrow = g * p.w_group_rows + mt * (BM / 2);
                    wrow2 = wrow + p.w_up_offset;
                } else {
                    wrow = g * p.w_group_rows + mt * BM;
                }
                for (int kb = k0; kb < k1; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[stage], S::kStageBytes);
                    if (EPI == EPI_SWIGLU) {
                        tma_load_2d(&tmW, &full[stage], sA + stage * S::kABytes, kb * BK, wrow);
                        tma_load_2d(&tmW, &full[stage], sA + stage * S::kABytes + (BM / 2) * BK * 2, kb * BK, wrow2);
                    } else {
                        tma_load_2d(&tmW, &full[stage], sA + stage * S::kABytes, kb * BK, wrow);
                    }
                    tma_load_2d(&tmX, &full[stage], sB + stage * S::kBBytes, kb * BK, trow);
                    iss.note(stage, phase);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            if (!ok) iss.drain(full, p.timeout_ns);   // copies in flight land before the CTA leaves
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(BM, NT);
            int stage = 0;
            uint32_t phase = 0;
            int local = 0;
            bool ok = true;
            for (int64_t u = u_begin; u < u_end && ok; ++local) {
                const Piece pc(u, stream_k ? u_end : u + nkb, nkb);
                u = stream_k ? u + (pc.k1 - pc.k0) : u + u_step;
                const int k0 = pc.k0, k1 = pc.k1;
                const int a = local & 1;
                const uint32_t aph = (local >> 1) & 1;
                if (!mbar_wait(&tempty[a], aph ^ 1, p.timeout_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + a * NT;
                for (int kb = k0; kb < k1; ++kb) {
                    if (!mbar_wait(&full[stage], phase, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t adesc = smem_desc_sw128(smem_u32(sA + stage * S::kABytes));
                    const uint64_t bdesc = smem_desc_sw128(smem_u32(sB + stage * S::kBBytes));
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        tc_mma_bf16(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, (kb != k0 || k != 0) ? 1u : 0u);
                    tc_commit(&empty[stage]);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (ok) tc_commit(&tfull[a]);
            }
            if (!ok) {
                tc_commit(drain);
                mbar_wait(drain, 0, p.timeout_ns);
            }
        }
    } else {
        const int q = warp & 3;
        const int L = q * 32 + lane;                 // TMEM lane = weight row within the tile
        const int et = threadIdx.x - 64;             // 0..127 inside the epilogue warps
        EpiBarrier eb{epib, 0u, p.timeout_ns};
        int local = 0;
        for (int64_t u = u_begin; u < u_end; ++local) {
            const int64_t u_piece = u;
            const Piece pc(u, stream_k ? u_end : u + nkb, nkb);
            u = stream_k ? u + (pc.k1 - pc.k0) : u + u_step;
            const int tile = pc.tile;
            const int a = local & 1;
            const uint32_t aph = (local >> 1) & 1;
            const int g = p.live[tile / p.tiles_per_group];
            const int mt = tile % p.tiles_per_group;
            const int cnt = p.counts[g];
            const int trow = p.row_offsets[g];
            // A cut tile's pieces belong to CTAs c_first..c_last and are added as
            // a right fold in piece order, p_first + (... + (p_last-1 + p_last)),
            // whichever piece does it.  A piece is slot 0 of its CTA when the
            // CTA's range starts inside the tile (its first piece), else slot 1.
            const bool cut = pc.k1 - pc.k0 < nkb;
            const int64_t ts = (int64_t)tile * nkb;
            const int c_first = cut ? wk.cta_of(ts) : 0, c_last = cut ? wk.cta_of(ts + nkb - 1) : 0;
            // While this piece's MMAs run: if it is the tile's first piece and
            // every other piece is already published, it will be the one to add
            // them up, so the others' sum is loaded now.
            constexpr int NR = NT <= 32 ? NT : 4;   // (64 token columns: no room in registers)
            float rest[NR];
            bool have_rest = false;
            if (NT <= 32 && cut && c_first == (int)blockIdx.x) {
                if (et == 0) *s_last = ld_acquire_u32(p.tickets + c_first) == (unsigned)(c_last - c_first);
                if (!eb.sync()) break;
                have_rest = *s_last != 0;
                if (have_rest) {
                    for (int c = c_last; c > c_first; --c) {
                        const float *src = p.part + ((int64_t)(c * 2 + (wk.begin(c) >= ts ? 0 : 1)) * BM + L) * NT;
#pragma unroll
                        for (int j = 0; j < NR; j += 4) {
                            const float4 v = __ldcg(reinterpret_cast<const float4 *>(src + j));
                            if (c == c_last) {
                                rest[j] = v.x; rest[j + 1] = v.y; rest[j + 2] = v.z; rest[j + 3] = v.w;
                            } else {
                                rest[j] = v.x + rest[j]; rest[j + 1] = v.y + rest[j + 1];
                                rest[j + 2] = v.z + rest[j + 2]; rest[j + 3] = v.w + rest[j + 3];
                            }
                        }
                    }
                }
                // the flag is read by all before the next item's writer may change it
                if (!eb.sync()) break;
            }
            // warp-uniform decision: the TMEM loads below are warp-collective
            if (!__all_sync(0xffffffffu, mbar_wait(&tfull[a], aph, p.timeout_ns))) break;
            tc_fence_after();
            float acc[NT];
            tmem_ld_row<NT>(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + a * NT, acc);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[a]);   // accumulator is in registers now

            if (have_rest) {
#pragma unroll
                for (int j = 0; j < NR; ++j) acc[j] = acc[j] + rest[j];
            } else if (cut) {
                // publish this piece's partial row and take the tile's ticket;
                // the last piece to arrive adds all of the tile's pieces
                const int my_slot = (u_piece == u_begin && u_begin >= ts) ? 0 : 1;
                float *mine = p.part + ((int64_t)(blockIdx.x * 2 + my_slot) * BM + L) * NT;
#pragma unroll
                for (int j = 0; j < NT; j += 4)
                    __stcg(reinterpret_cast<float4 *>(mine + j), make_float4(acc[j], acc[j + 1], acc[j + 2], acc[j + 3]));
                // the barrier orders every epilogue thread's stores before the
                // ticket thread's acquire-release ticket, whose release covers
                // them; in the last piece its acquire, followed by the barrier,
                // lets the other threads read the earlier pieces
                if (!eb.sync()) break;
                if (et == 0) *s_last = ticket_arrive(p.tickets + c_first) == (unsigned)(c_last - c_first);
                if (!eb.sync()) break;
                if (!*s_last) continue;
                float sum[NT];
                for (int c = c_last; c >= c_first; --c) {
                    if (c == (int)blockIdx.x) {
#pragma unroll
                        for (int j = 0; j < NT; ++j) sum[j] = c == c_last ? acc[j] : acc[j] + sum[j];
                    } else {
                        const float *src = p.part + ((int64_t)(c * 2 + (wk.begin(c) >= ts ? 0 : 1)) * BM + L) * NT;
#pragma unroll
                        for (int j = 0; j < NT; j += 4) {
                            const float4 v = __ldcg(reinterpret_cast<const float4 *>(src + j));
                            if (c == c_last) {
                                sum[j] = v.x; sum[j + 1] = v.y; sum[j + 2] = v.z; sum[j + 3] = v.w;
                            } else {
                                sum[j] = v.x + sum[j]; sum[j + 1] = v.y + sum[j + 1];
                                sum[j + 2] = v.z + sum[j + 2]; sum[j + 3] = v.w + sum[j + 3];
                            }
                        }
                    }
                }
#pragma unroll
                for (int j = 0; j < NT; ++j) acc[j] = sum[j];
            }

            if (EPI == EPI_SCATTER) {
                const int d = mt * BM + L;
                if (d < p.n_valid) {
                    const float b = p.bias ? __ldg(p.bias + (int64_t)g * p.n_valid + d) : 0.f;
                    float *z = static_cast<float *>(p.out);
#pragma unroll
                    for (int j = 0; j < NT; ++j) {
                        if (j < cnt) {   // no perm_slot (shared expert): row j is token j, weight 1
                            const int slot = p.perm_slot ? p.perm_slot[trow + j] : trow + j;
                            const float gw = p.perm_slot ? p.gate_w[slot] : 1.f;
                            z[(int64_t)slot * p.ldo + d] = gw * (acc[j] + b);
                        }
                    }
                }
            } else if (EPI == EPI_GELU) {
                __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(sE);   // [NT][128]
                const int f = mt * BM + L;
                const float b = (p.bias && f < p.n_valid) ? __ldg(p.bias + (int64_t)g * p.n_valid + f) : 0.f;
#pragma unroll
                for (int j = 0; j < NT; j += 2) {
                    const uint32_t hv = tc::gelu_erf_bf16x2(acc[j] + b, acc[j + 1] + b);
                    o[j * 128 + L] = __ushort_as_bfloat16(static_cast<unsigned short>(hv & 0xffffu));
                    o[(j + 1) * 128 + L] = __ushort_as_bfloat16(static_cast<unsigned short>(hv >> 16));
                }
                if (!eb.sync()) break;
                __nv_bfloat16 *h = static_cast<__nv_bfloat16 *>(p.out);
                const int f0 = mt * BM;
                for (int v = et; v < NT * 16; v += 128) {   // 16 x 16-byte pieces per token row
                    const int j = v >> 4, c = (v & 15) * 8;
                    if (j < cnt) {
                        __nv_bfloat16 *dst = h + (int64_t)(trow + j) * p.ldo + f0 + c;
                        const uint4 val = *reinterpret_cast<const uint4 *>(o + j * 128 + c);
                        if (f0 + c + 8 <= p.n_valid) {
                            *reinterpret_cast<uint4 *>(dst) = val;
                        } else {
                            const __nv_bfloat16 *src = o + j * 128 + c;
                            for (int k = 0; k < 8; ++k)
                                if (f0 + c + k < p.n_valid) dst[k] = src[k];
                        }
                    }
                }
                if (!eb.sync()) break;
            } else {  // EPI_SWIGLU
                float *up = reinterpret_cast<float *>(sE);                                   // [NT][64]
                __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(sE + 64 * NT * 4);      // [NT][64]
                if (L >= 64) {
#pragma unroll
                    for (int j = 0; j < NT; ++j) up[j * 64 + (L - 64)] = acc[j];
                }
                if (!eb.sync()) break;
                if (L < 64) {
#pragma unroll
                    for (int j = 0; j < NT; j += 2) {
                        const uint32_t hv = tc::swiglu_bf16x2(acc[j], acc[j + 1], up[j * 64 + L], up[(j + 1) * 64 + L]);
                        o[j * 64 + L] = __ushort_as_bfloat16(static_cast<unsigned short>(hv & 0xffffu));
                        o[(j + 1) * 64 + L] = __ushort_as_bfloat16(static_cast<unsigned short>(hv >> 16));
                    }
                }
                if (!eb.sync()) break;
                __nv_bfloat16 *h = static_cast<__nv_bfloat16 *>(p.out);
                const int f0 = mt * (BM / 2);
                for (int v = et; v < NT * 8; v += 128) {    // 8 x 16-byte pieces per token row
                    const int j = v >> 3, c = (v & 7) * 8;
                    if (j < cnt) {
                        __nv_bfloat16 *dst = h + (int64_t)(trow + j) * p.ldo + f0 + c;
                        const uint4 val = *reinterpret_cast<const uint4 *>(o + j * 64 + c);
                        if (f0 + c + 8 <= p.n_valid) {
                            *reinterpret_cast<uint4 *>(dst) = val;
                        } else {
                            const __nv_bfloat16 *src = o + j * 64 + c;
                            for (int k = 0; k < 8; ++k)
                                if (f0 + c + k < p.n_valid) dst[k] = src[k];
                        }
                    }
                }
                if (!eb.sync()) break;
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

}  // namespace dec
}  // namespace moe
