// moe_gemm_tc.cuh -- grouped GEMM on the sm_100a tensor cores (tcgen05 + TMEM).
//
// C[r, n] = sum_k A[r, k] * B[g * b_group_rows + n, k], bf16 x bf16 -> fp32,
// for every 128-row tile r of an expert segment g of the permuted activations
// (or of a plain row-major matrix, "dense" mode with one group).  Both operands
// are K-major; A rows are tokens, B rows are output features of expert g
// (weights stored out x in).  This evaluates each selected expert only on the
// rows routed to it -- the "conditional computation" of the Shazeer article
// (qiita, layer formula section): unselected experts are skipped, not
// multiplied by zero -- as one grouped GEMM, the grouped_mm backend idea of the
// Transformers-v5 MoE article, section 2.
//
// Kernel structure (one persistent CTA per SM, 320 threads):
//   warp 0      TMA producer: 64-wide K slices of A (128 rows) and B (BN rows)
//               into a kStages-deep shared-memory ring (128-byte swizzle).
//   warp 1      allocates 2*BN TMEM columns; one thread issues
//               tcgen05.mma (128 x BN x 16) into one of two TMEM accumulators
//               and commits ring slots / finished accumulators to mbarriers.
//   warps 2..9  epilogue: tcgen05.ld of the accumulator (warp w reads TMEM
//               lanes 32*(w%4)..+31, half of the columns each), fused
//               activation / scaling, stores to global memory.
// The two accumulators let the epilogue of tile i overlap the MMAs of tile
// i+1.  Tiles are ordered expert by expert and, inside an expert, by column
// tile then row tile, so concurrently running CTAs share the same weight
// columns in L2.
//
// Epilogues:
//   EPI_GELU     h = bf16(gelu_erf(acc + b1[g, n]))           (GPT-2 expert, first linear)
//   EPI_SWIGLU   B tile = 128 gate rows + 128 up rows (two TMA boxes of the
//                packed gate_up weight); h = bf16(silu(gate) * up)
//   EPI_SCATTER  z[slot(r), n] = w[slot(r)] * (acc + b2[g, n]), fp32, rows
//                with slot -1 (padding) skipped      (down projection)
//   EPI_LOGITS   out[r, n] = acc + b_g[n], fp32, rows < dense_rows   (router)
//
// Every wait is bounded (mbar_wait); on expiry the waiting role stops issuing
// work, the status word records MOE_STATUS_TIMEOUT and the CTA drains and
// returns.
#pragma once

#include "moe_common.cuh"

namespace moe {
namespace tc {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;

enum { EPI_GELU = 0, EPI_SWIGLU = 1, EPI_SCATTER = 2, EPI_LOGITS = 3 };

struct Params {
    int num_groups;           // G
    const int *row_offsets;   // [G+1] segment starts (multiples of BM) or nullptr for dense mode
    int dense_rows;           // dense mode: valid rows of A / out
    int n_tiles;              // output column tiles per group
    int num_k_blocks;         // ceil(K / BK)
    int b_group_rows;         // rows of B per group in its 2-D view
    int b_up_offset;          // SwiGLU: first up row inside a group (= H)
    int n_valid;              // valid output columns per group
    void *out;                // output base
    int64_t ldo;              // output row stride (elements)
    const float *bias;        // [G, n_valid] or nullptr
    const int *perm_slot;     // EPI_SCATTER: slot of each permuted row (-1 = padding)
    const float *gate_w;      // EPI_SCATTER: gate weight of each slot
    uint64_t timeout_ns;
};

template <int BN>
struct Shape {
    static constexpr int kStages = BN == 256 ? 4 : 6;   // 192 KB of ring either way
    static constexpr uint32_t kABytes = BM * BK * 2;
    static constexpr uint32_t kBBytes = BN * BK * 2;
    static constexpr uint32_t kTmemCols = 2 * BN;
    static constexpr size_t kBarrierBytes = (2 * kStages + 5) * 8 + 16;
    // ring + alignment slack + barriers + tmem slot; the group table follows
    static size_t smem_bytes(int groups) {
        return 1024 + kStages * (size_t)(kABytes + kBBytes) + kBarrierBytes + 4 * (size_t)(groups + 1) + 16;
    }
};

struct TileCoord {
    int g, row0, nt;
};

__device__ __forceinline__ TileCoord decode_tile(int i, const int *s_rowoff, int G, int n_tiles, int dense_mtiles) {
    TileCoord c;
    if (s_rowoff == nullptr) {
        c.g = 0;
        c.nt = i / dense_mtiles;
        c.row0 = (i - c.nt * dense_mtiles) * BM;
        return c;
    }
    int lo = 0, hi = G - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if ((s_rowoff[mid] / BM) * n_tiles <= i) lo = mid;
        else hi = mid - 1;
    }
    const int mt0 = s_rowoff[lo] / BM;
    const int mtn = s_rowoff[lo + 1] / BM - mt0;
    const int local = i - mt0 * n_tiles;
    c.g = lo;
    c.nt = local / mtn;
    c.row0 = (mt0 + local - c.nt * mtn) * BM;
    return c;
}

// GELU(v) = v Phi(v) = 0.5 v (1 + erf(v / sqrt 2)), exact-erf form, with erfc
// from Abramowitz & Stegun, Handbook of Mathematical Functions, formula 7.1.26
// (absolute error of erf at most 1.5e-7, far below the bf16 rounding of h):
//   erfc(z) ~ (a1 t + a2 t^2 + a3 t^3 + a4 t^4 + a5 t^5) exp(-z^2), t = 1 / (1 + p z), z >= 0.
// For v < 0, 1 + erf(v / sqrt 2) = erfc(|v| / sqrt 2) is used directly (no cancellation).
__device__ __forceinline__ float gelu_erf(float v) {
    const float z = fabsf(v) * 0.70710678118654752f;
    const float t = __fdividef(1.0f, fmaf(0.3275911f, z, 1.0f));
    float poly = fmaf(t, 1.061405429f, -1.453152027f);
    poly = fmaf(t, poly, 1.421413741f);
    poly = fmaf(t, poly, -0.284496736f);
    poly = fmaf(t, poly, 0.254829592f);
    const float q = poly * t * __expf(-z * z);
    return 0.5f * v * (v >= 0.f ? 2.0f - q : q);
}
__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + __expf(-g)); }

template <int BN, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                           const Params p) {
    using S = Shape<BN>;
    constexpr int kStages = S::kStages;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = smem + kStages * S::kABytes;
    uint64_t *full = reinterpret_cast<uint64_t *>(sB + kStages * S::kBBytes);
    uint64_t *empty = full + kStages;
    uint64_t *tfull = empty + kStages;
    uint64_t *tempty = tfull + 2;
    uint64_t *drain = tempty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    int *s_rowoff = reinterpret_cast<int *>(tmem_slot + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = p.num_groups;
    if (p.row_offsets)
        for (int i = threadIdx.x; i <= G; i += blockDim.x) s_rowoff[i] = p.row_offsets[i];
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
        fence_mbar_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) tmem_alloc(tmem_slot, S::kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int *rowoff = p.row_offsets ? s_rowoff : nullptr;
    const int dense_mtiles = (p.dense_rows + BM - 1) / BM;
    const int m_tiles = rowoff ? s_rowoff[G] / BM : dense_mtiles;
    const int total = m_tiles * p.n_tiles;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int i = blockIdx.x; i < total && ok; i += gridDim.x) {
                const TileCoord c = decode_tile(i, rowoff, G, p.n_tiles, dense_mtiles);
                int brow, brow2 = 0;
                if (EPI == EPI_SWIGLU) {
                    brow = c.g * p.b_group_rows + c.nt * (BN / 2);
                    brow2 = brow + p.b_up_offset;
                } else {
                    brow = c.g * p.b_group_rows + c.nt * BN;
                }
                for (int kb = 0; kb < p.num_k_blocks; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[stage], S::kABytes + S::kBBytes);
                    tma_load_2d(&tmA, &full[stage], sA + stage * S::kABytes, kb * BK, c.row0);
                    if (EPI == EPI_SWIGLU) {
                        tma_load_2d(&tmB, &full[stage], sB + stage * S::kBBytes, kb * BK, brow);
                        tma_load_2d(&tmB, &full[stage], sB + stage * S::kBBytes + (BN / 2) * BK * 2, kb * BK, brow2);
                    } else {
                        tma_load_2d(&tmB, &full[stage], sB + stage * S::kBBytes, kb * BK, brow);
                    }
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            if (!ok) {
                // let copies already in flight land before the CTA leaves
                const uint64_t t0 = globaltimer_ns();
                while (globaltimer_ns() - t0 < 1000000ull) {
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(BM, BN);
            int stage = 0;
            uint32_t phase = 0;
            int local = 0;
            bool ok = true;
            for (int i = blockIdx.x; i < total && ok; i += gridDim.x, ++local) {
                const int a = local & 1;
                const uint32_t aph = (local >> 1) & 1;
                if (!mbar_wait(&tempty[a], aph ^ 1, p.timeout_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + a * BN;
                for (int kb = 0; kb < p.num_k_blocks; ++kb) {
                    if (!mbar_wait(&full[stage], phase, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t adesc = smem_desc_sw128(smem_u32(sA + stage * S::kABytes));
                    const uint64_t bdesc = smem_desc_sw128(smem_u32(sB + stage * S::kBBytes));
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        tc_mma_bf16(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
                    tc_commit(&empty[stage]);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (ok) tc_commit(&tfull[a]);
            }
            if (!ok) {
                // wait (bounded) for the MMAs already issued before TMEM is freed
                tc_commit(drain);
                mbar_wait(drain, 0, p.timeout_ns);
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int ew = warp - 2;
        const int q = warp & 3;
        const int half = ew >> 2;
        const int r_in_tile = q * 32 + lane;
        int local = 0;
        for (int i = blockIdx.x; i < total; i += gridDim.x, ++local) {
            const int a = local & 1;
            const uint32_t aph = (local >> 1) & 1;
            const TileCoord c = decode_tile(i, rowoff, G, p.n_tiles, dense_mtiles);
            if (!mbar_wait(&tfull[a], aph, p.timeout_ns)) break;
            tc_fence_after();
            const int row = c.row0 + r_in_tile;
            const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + a * BN;

            if (EPI == EPI_SWIGLU) {
                constexpr int kOutCols = BN / 2;             // h columns per tile
                constexpr int kPerHalf = kOutCols / 2;       // per epilogue warp
                __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(p.out);
#pragma unroll 1
                for (int cc = 0; cc < kPerHalf; cc += 32) {
                    const int col = half * kPerHalf + cc;
                    uint32_t rg[32], ru[32];
                    tmem_ld_32x32b_x32(tbase + col, rg);
                    tmem_ld_32x32b_x32(tbase + kOutCols + col, ru);
                    tmem_ld_wait();
                    const int n0 = c.nt * kOutCols + col;
                    uint32_t pk[16];
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        const float h0 = silu_f(__uint_as_float(rg[2 * k])) * __uint_as_float(ru[2 * k]);
                        const float h1 = silu_f(__uint_as_float(rg[2 * k + 1])) * __uint_as_float(ru[2 * k + 1]);
                        pk[k] = pack_bf16x2(h0, h1);
                    }
                    __nv_bfloat16 *dst = out + (int64_t)row * p.ldo + n0;
                    if (n0 + 32 <= p.n_valid) {
#pragma unroll
                        for (int v = 0; v < 4; ++v)
                            reinterpret_cast<uint4 *>(dst)[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
                    } else {
#pragma unroll
                        for (int k = 0; k < 32; ++k)
                            if (n0 + k < p.n_valid)
                                dst[k] = __ushort_as_bfloat16(static_cast<unsigned short>((pk[k >> 1] >> ((k & 1) * 16)) & 0xffffu));
                    }
                }
            } else {
                constexpr int kPerHalf = BN / 2;
                int slot = -1;
                float gw = 0.f;
                if (EPI == EPI_SCATTER) {
                    slot = p.perm_slot[row];
                    if (slot >= 0) gw = p.gate_w[slot];
                }
#pragma unroll 1
                for (int cc = 0; cc < kPerHalf; cc += 32) {
                    const int col = half * kPerHalf + cc;
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(tbase + col, r);
                    tmem_ld_wait();
                    const int n0 = c.nt * BN + col;
                    if (n0 >= p.n_valid) continue;
                    const bool full_chunk = n0 + 32 <= p.n_valid;
                    float v[32];
#pragma unroll
                    for (int k = 0; k < 32; ++k) v[k] = __uint_as_float(r[k]);
                    if (p.bias) {
                        const float *bias = p.bias + (int64_t)c.g * p.n_valid + n0;
                        if (full_chunk) {
#pragma unroll
                            for (int u = 0; u < 8; ++u) {
                                const float4 b4 = __ldg(reinterpret_cast<const float4 *>(bias) + u);
                                v[4 * u] += b4.x; v[4 * u + 1] += b4.y; v[4 * u + 2] += b4.z; v[4 * u + 3] += b4.w;
                            }
                        } else {
#pragma unroll
                            for (int k = 0; k < 32; ++k)
                                if (n0 + k < p.n_valid) v[k] += __ldg(bias + k);
                        }
                    }
                    if (EPI == EPI_GELU) {
                        __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(p.out) + (int64_t)row * p.ldo + n0;
                        uint32_t pk[16];
#pragma unroll
                        for (int k = 0; k < 16; ++k) pk[k] = pack_bf16x2(gelu_erf(v[2 * k]), gelu_erf(v[2 * k + 1]));
                        if (full_chunk) {
#pragma unroll
                            for (int u = 0; u < 4; ++u)
                                reinterpret_cast<uint4 *>(dst)[u] = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
                        } else {
#pragma unroll
                            for (int k = 0; k < 32; ++k)
                                if (n0 + k < p.n_valid)
                                    dst[k] = __ushort_as_bfloat16(static_cast<unsigned short>((pk[k >> 1] >> ((k & 1) * 16)) & 0xffffu));
                        }
                    } else if (EPI == EPI_SCATTER) {
                        if (slot >= 0) {
                            float *dst = static_cast<float *>(p.out) + (int64_t)slot * p.ldo + n0;
                            if (full_chunk) {
#pragma unroll
                                for (int u = 0; u < 8; ++u)
                                    reinterpret_cast<float4 *>(dst)[u] =
                                        make_float4(gw * v[4 * u], gw * v[4 * u + 1], gw * v[4 * u + 2], gw * v[4 * u + 3]);
                            } else {
#pragma unroll
                                for (int k = 0; k < 32; ++k)
                                    if (n0 + k < p.n_valid) dst[k] = gw * v[k];
                            }
                        }
                    } else {  // EPI_LOGITS
                        if (row < p.dense_rows) {
                            float *dst = static_cast<float *>(p.out) + (int64_t)row * p.ldo + n0;
#pragma unroll
                            for (int k = 0; k < 32; ++k)
                                if (n0 + k < p.n_valid) dst[k] = v[k];
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[a]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, S::kTmemCols);
    }
}

}  // namespace tc
}  // namespace moe
