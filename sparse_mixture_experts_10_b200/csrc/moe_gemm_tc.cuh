// moe_gemm_tc.cuh -- grouped GEMM on the sm_100a tensor cores (tcgen05 + TMEM).
//
// C[r, n] = sum_k A[r, k] * B[g * b_group_rows + n, k], bf16 x bf16 -> fp32,
// for every row tile r of an expert segment g of the permuted activations
// (or of a plain row-major matrix, "dense" mode with one group).  Both operands
// are K-major; A rows are tokens, B rows are output features of expert g
// (weights stored out x in).  This evaluates each selected expert only on the
// rows routed to it -- the "conditional computation" of the Shazeer article
// (qiita, layer formula section): unselected experts are skipped, not
// multiplied by zero -- as one grouped GEMM, the grouped_mm backend idea of the
// Transformers-v5 MoE article, section 2.
//
// Two kernels share the epilogue:
//
// grouped_gemm_tc_kernel<BN, EPI>  one CTA per tile of 128 rows x BN columns,
//   persistent, 576 threads:
//   warp 0      TMA producer: 64-wide K slices of A (128 rows) and B (BN rows)
//               into a shared-memory ring (128-byte swizzle).
//   warp 1      allocates 2*BN TMEM columns; one thread issues
//               tcgen05.mma.cta_group::1 (128 x BN x 16) into one of two TMEM
//               accumulators and commits ring slots / accumulators to mbarriers.
//   warps 2..17 epilogue: tcgen05.ld of the accumulator (warp w reads TMEM
//               lanes 32*(w%4)..+31 and a quarter of the columns), fused
//               activation / scaling, stores to global memory.
//
// grouped_gemm_tc2_kernel<EPI>  a cluster of two CTAs (one per SM of a pair)
//   per tile of 256 rows x 256 columns: each CTA loads its own 128 rows of A
//   and its own 128 rows of B (no multicast), the leader CTA issues
//   tcgen05.mma.cta_group::2 (256 x 256 x 16), which reads both CTAs' shared
//   memory and accumulates into both CTAs' TMEM; ring slots and finished
//   accumulators are committed to the barriers of both CTAs; the epilogue of
//   each CTA reads its own TMEM and releases the accumulator on the leader's
//   barrier.  Per SM, a 64-wide K slice then moves 32 KB for 4 MFLOP (instead
//   of 48 KB), and the ring holds 6 slices instead of 4.
//
// The two accumulators let the epilogue of tile i overlap the MMAs of tile
// i+1.  Tiles are ordered expert by expert and, inside an expert, by column
// tile then row tile, so concurrently running CTAs share the same weight
// columns in L2.
//
// Epilogues:
//   EPI_GELU     h = bf16(gelu_erf(acc + b1[g, n]))           (GPT-2 expert, first linear)
//   EPI_SWIGLU   B tile = 128 gate rows + 128 up rows of the packed gate_up
//                weight; h = bf16(silu(gate) * up)
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
constexpr int kEpiWarps = 16;                  // four per TMEM lane quadrant
constexpr int kEpiGroups = kEpiWarps / 4;      // column groups of a tile
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
    const int *perm_slot;     // EPI_SCATTER: slot of each permuted row (-1 = padding); nullptr: row = slot, weight 1
    const float *gate_w;      // EPI_SCATTER: gate weight of each slot
    // EPI_SCATTER with accum_k > 0: out is y [T, ldo] fp32 (zeroed before the
    // launch) and each row's scaled result is added into row slot / accum_k with
    // fp32 reductions; with accum_k <= 2 every element receives at most two
    // additions onto +0, whose result does not depend on their order.
    int accum_k;
    // EPI_SCATTER with scatter_rows: out is z [rows, ldo] fp32 in the permuted
    // row order (written by bulk tensor stores through tmO); otherwise z rows
    // are indexed by slot.
    int scatter_rows;
    // Row tiles of a group whose padded segment holds an odd number of 128-row
    // blocks: the pair kernel's last 256-row unit would be half past the
    // segment.  tail_mode 1 (pair kernel): leave each such group's last block
    // out; tail_mode 2 (1-CTA kernel): compute only those blocks, one 128-row
    // tile per group.  0: every row tile.
    // The tail kernel is launched right behind the pair kernel and runs beside
    // it: the pair kernel lets its dependent launch only after its own
    // programmatic wait (so everything before it is complete and visible),
    // the tail kernel starts without waiting, takes SMs as the pair CTAs
    // finish, and waits for the pair kernel only before it exits (so the next
    // kernel, which waits for the tail kernel, sees both).
    int tail_mode;
    uint64_t timeout_ns;
    int64_t slot_limit;       // EPI_SCATTER: entries of gate_w (checked in the bounds-check build when > 0)
};

__device__ __forceinline__ void red_add_v4(float *ptr, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(ptr), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}

// bf16 output staging for the bulk tensor stores: 32 rows x 16 columns per
// epilogue warp.
constexpr uint32_t kOutStageWarpBytes = 32 * 16 * 2;
constexpr uint32_t kOutStageBytes = kEpiWarps * kOutStageWarpBytes;

template <int BN>
struct Shape {
    static constexpr int kStages = BN == 256 ? 4 : 6;   // 192 KB of ring either way
    static constexpr uint32_t kABytes = BM * BK * 2;
    static constexpr uint32_t kBBytes = BN * BK * 2;
    static constexpr uint32_t kTmemCols = 2 * BN;
    static constexpr size_t kBarrierBytes = (2 * kStages + 5) * 8 + 16;
    // ring + alignment slack + output staging + barriers + tmem slot; the group
    // table and the tail-tile table follow
    static size_t smem_bytes(int groups) {
        return 1024 + kStages * (size_t)(kABytes + kBBytes) + kOutStageBytes + kBarrierBytes +
               8 * (size_t)(groups + 1) + 16;
    }
};

// Pair kernel: per CTA, 128 rows of A and 128 rows of B per K slice.
struct Shape2 {
    static constexpr int kStages = 6;
    static constexpr uint32_t kABytes = BM * BK * 2;
    static constexpr uint32_t kBBytes = 128 * BK * 2;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr size_t kBarrierBytes = (2 * kStages + 5) * 8 + 16;
    // ring + slack + output staging + barriers + tmem slot; group table and 256-row unit table follow
    static size_t smem_bytes(int groups) {
        return 1024 + kStages * (size_t)(kABytes + kBBytes) + kOutStageBytes + kBarrierBytes +
               8 * (size_t)(groups + 1) + 16;
    }
};

struct TileCoord {
    int g, row0, nt;
};

// Bounds-check build: a group table's segments start on 128-row blocks and
// do not decrease.
__device__ __forceinline__ bool group_table_ok(const int *s_rowoff, int G) {
    bool ok = s_rowoff[0] >= 0 && s_rowoff[0] % BM == 0;
    for (int g = 0; g < G; ++g) ok = ok && s_rowoff[g + 1] >= s_rowoff[g] && s_rowoff[g + 1] % BM == 0;
    return ok;
}

// Tile i of 128-row tiles: group, first row and column tile.
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

// Tile i of the tail tiles (tail_mode 2): s_tcum[g] = number of groups before
// g whose segment has an odd number of 128-row blocks; each such group has one
// tile per column tile, its last 128 rows.
__device__ __forceinline__ TileCoord decode_tail_tile(int i, const int *s_rowoff, const int *s_tcum, int G,
                                                      int n_tiles) {
    int lo = 0, hi = G - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_tcum[mid] * n_tiles <= i) lo = mid;
        else hi = mid - 1;
    }
    TileCoord c;
    c.g = lo;
    c.nt = i - s_tcum[lo] * n_tiles;
    c.row0 = s_rowoff[lo + 1] - BM;
    return c;
}

// Tile i of 256-row unit tiles.  s_units[g] = number of 256-row units before
// group g (a group of 128*m padded rows has ceil(m/2) units); row0 is the first
// row of the unit, whose upper half may lie past the group's end.
__device__ __forceinline__ TileCoord decode_unit_tile(int i, const int *s_rowoff, const int *s_units, int G,
                                                      int n_tiles, int dense_units) {
    TileCoord c;
    if (s_rowoff == nullptr) {
        c.g = 0;
        c.nt = i / dense_units;
        c.row0 = (i - c.nt * dense_units) * 2 * BM;
        return c;
    }
    int lo = 0, hi = G - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_units[mid] * n_tiles <= i) lo = mid;
        else hi = mid - 1;
    }
    const int u0 = s_units[lo];
    const int un = s_units[lo + 1] - u0;
    const int local = i - u0 * n_tiles;
    c.g = lo;
    c.nt = local / un;
    c.row0 = s_rowoff[lo] + (local - c.nt * un) * 2 * BM;
    return c;
}

// GELU(v) = v Phi(v), exact-erf form, on a pair of values.  With
// Phi(-|v|) = erfc(|v| / sqrt 2) / 2 from Abramowitz & Stegun, Handbook of
// Mathematical Functions, formula 7.1.26 (absolute error of erf at most
// 1.5e-7):
//   erfc(z) ~ (a1 t + a2 t^2 + a3 t^3 + a4 t^4 + a5 t^5) exp(-z^2),  t = 1 / (1 + p z),
// and v Phi(v) = relu(v) - |v| Phi(-|v|) for either sign of v (no
// cancellation for v < 0).  The factor -1/2 is folded into the coefficients,
// p into p / sqrt 2; exp(-v^2 / 2) = 2^(-v^2 log2(e) / 2).  Per pair: eleven
// f32x2 instructions, two reciprocals and two exponentials on the
// special-function unit.  Returns the two results rounded to bf16.
__device__ __forceinline__ uint32_t gelu_erf_bf16x2(float v0, float v1) {
    constexpr float kP = 0.2316418882663604f;          // p / sqrt 2, p = 0.3275911
    constexpr float kB1 = -0.127414796f, kB2 = 0.142248368f, kB3 = -0.7107068705f,
                    kB4 = 0.7265760135f, kB5 = -0.5307027145f;   // -a_i / 2
    constexpr float kL = 0.7213475204444817f;          // log2(e) / 2
    const float a0 = fabsf(v0), a1 = fabsf(v1);
    const uint64_t v = f2_pack(v0, v1), a = f2_pack(a0, a1);
    float d0, d1;
    f2_unpack(f2_fma(a, f2_splat(kP), f2_splat(1.0f)), d0, d1);
    const uint64_t t = f2_pack(rcp_approx(d0), rcp_approx(d1));
    uint64_t q = f2_fma(t, f2_splat(kB5), f2_splat(kB4));
    q = f2_fma(t, q, f2_splat(kB3));
    q = f2_fma(t, q, f2_splat(kB2));
    q = f2_fma(t, q, f2_splat(kB1));
    q = f2_mul(q, t);                                   // -erfc-series / 2 without the Gaussian
    float g0, g1;
    f2_unpack(f2_mul(f2_mul(v, f2_splat(-kL)), v), g0, g1);
    const uint64_t nphi = f2_mul(q, f2_pack(ex2_approx(g0), ex2_approx(g1)));   // -Phi(-|v|)
    const uint64_t out = f2_fma(f2_add(v, a), f2_splat(0.5f), f2_mul(a, nphi));
    float o0, o1;
    f2_unpack(out, o0, o1);
    return pack_bf16x2(o0, o1);
}

// SwiGLU on a pair: silu(g) u = g u / (1 + 2^(-g log2 e)), rounded to bf16.
__device__ __forceinline__ uint32_t swiglu_bf16x2(float g0, float g1, float u0, float u1) {
    constexpr float kLog2e = 1.4426950408889634f;
    const uint64_t g = f2_pack(g0, g1);
    float e0, e1;
    f2_unpack(f2_mul(g, f2_splat(-kLog2e)), e0, e1);
    float d0, d1;
    f2_unpack(f2_add(f2_pack(ex2_approx(e0), ex2_approx(e1)), f2_splat(1.0f)), d0, d1);
    float o0, o1;
    f2_unpack(f2_mul(f2_mul(g, f2_pack(u0, u1)), f2_pack(rcp_approx(d0), rcp_approx(d1))), o0, o1);
    return pack_bf16x2(o0, o1);
}

__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

// tcgen05.wait::ld that also names the registers of the load it completes, so
// that their uses cannot be scheduled above it.
__device__ __forceinline__ void tmem_ld_wait_regs(uint32_t (&r)[16]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
                 :
                 : "memory");
}

__device__ __forceinline__ void store_bf16x16(__nv_bfloat16 *dst, const uint32_t (&pk)[8], int n0, int n_valid) {
    if (n0 + 16 <= n_valid) {
        reinterpret_cast<uint4 *>(dst)[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        reinterpret_cast<uint4 *>(dst)[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
    } else {
#pragma unroll
        for (int k = 0; k < 16; ++k)
            if (n0 + k < n_valid)
                dst[k] = __ushort_as_bfloat16(static_cast<unsigned short>((pk[k >> 1] >> ((k & 1) * 16)) & 0xffffu));
    }
}

// Epilogue of one accumulator tile for the calling warp.  The warp reads TMEM
// lanes 32*(warp%4).. (this thread: output row `row`) from `tbase`; column
// group `grp` (of kEpiGroups) of the tile is its share, in 16-column chunks.
// Rows at or beyond row_limit are not stored.  Every lane executes the TMEM
// loads (they are warp-wide).
// Stores one warp's 32 rows x 16 bf16 columns (pk: this lane's row) at
// (column n0, row row0): through the warp's shared staging tile and one bulk
// tensor store when all 32 rows are valid (rows of a 128-row aligned segment),
// else row by row.
__device__ __forceinline__ void store_h_chunk(const CUtensorMap *tmO, uint8_t *stage, __nv_bfloat16 *out,
                                              int64_t ldo, int row, bool row_ok, const uint32_t (&pk)[8], int n0,
                                              int n_valid) {
    const int lane = threadIdx.x & 31;
    if (__all_sync(0xffffffffu, row_ok)) {
        if (lane == 0) bulk_wait_read_all();   // the previous store has read the staging tile
        __syncwarp();
        uint4 *dst = reinterpret_cast<uint4 *>(stage + lane * 32);
        dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            tma_store_2d(tmO, stage, n0, row - lane);
            bulk_commit();
        }
    } else if (row_ok) {
        store_bf16x16(out + (int64_t)row * ldo + n0, pk, n0, n_valid);
    }
}

// EPI_SCATTER: the row's slot and gate weight, loaded by the caller before it
// waits for the accumulator (two dependent global loads off the critical path).
struct RowGate {
    int slot = -1;
    float gw = 0.f;
};
template <int EPI>
__device__ __forceinline__ RowGate load_row_gate(const Params &p, int row, int row_limit) {
    RowGate r;
    if (EPI == EPI_SCATTER && row < row_limit) {
        if (p.perm_slot) {
            r.slot = p.perm_slot[row];
            if (r.slot >= 0 && !MOE_BOUNDS(p.slot_limit <= 0 || r.slot < p.slot_limit)) r.slot = -1;
            if (r.slot >= 0) r.gw = p.gate_w[r.slot];
        } else {   // dense rows (shared expert): row r is token r, weight 1
            r.slot = row;
            r.gw = 1.f;
        }
    }
    return r;
}

// Stores one warp's 32 rows x 16 fp32 columns (v: this lane's row) at (column
// n0, row row0) as two 32 x 8 bulk tensor stores through the warp's shared
// staging tile when all 32 rows are valid, else row by row.
__device__ __forceinline__ void store_z_chunk(const CUtensorMap *tmO, uint8_t *stage, float *out, int64_t ldo, int row,
                                              bool row_ok, const float (&v)[16], int n0, int n_valid) {
    const int lane = threadIdx.x & 31;
    if (__all_sync(0xffffffffu, row_ok)) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            if (lane == 0) bulk_wait_read_all();   // the previous store has read the staging tile
            __syncwarp();
            float4 *dst = reinterpret_cast<float4 *>(stage + lane * 32);
            dst[0] = make_float4(v[8 * h], v[8 * h + 1], v[8 * h + 2], v[8 * h + 3]);
            dst[1] = make_float4(v[8 * h + 4], v[8 * h + 5], v[8 * h + 6], v[8 * h + 7]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                tma_store_2d(tmO, stage, n0 + 8 * h, row - lane);
                bulk_commit();
            }
        }
    } else if (row_ok) {
        float *dst = out + (int64_t)row * ldo + n0;
#pragma unroll
        for (int k = 0; k < 16; ++k)
            if (n0 + k < n_valid) dst[k] = v[k];
    }
}

template <int BN, int EPI>
__device__ __forceinline__ void epilogue_tile(const Params &p, const TileCoord &c, int row, int row_limit,
                                              uint32_t tbase, int grp, const CUtensorMap *tmO, uint8_t *stage,
                                              const RowGate rg) {
    const bool row_ok = row < row_limit;
    if (EPI == EPI_SWIGLU) {
        constexpr int kOutCols = BN / 2;                  // h columns per tile
        constexpr int kPerGroup = kOutCols / kEpiGroups;  // per epilogue warp
        __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(p.out);
#pragma unroll 1
        for (int cc = 0; cc < kPerGroup; cc += 16) {
            const int col = grp * kPerGroup + cc;
            uint32_t rg[16], ru[16];
            tmem_ld_32x32b_x16(tbase + col, rg);
            tmem_ld_32x32b_x16(tbase + kOutCols + col, ru);
            tmem_ld_wait();
            const int n0 = c.nt * kOutCols + col;
            if (!__any_sync(0xffffffffu, row_ok) || n0 >= p.n_valid) continue;   // warp-uniform
            uint32_t pk[8];
#pragma unroll
            for (int k = 0; k < 8; ++k)
                pk[k] = swiglu_bf16x2(__uint_as_float(rg[2 * k]), __uint_as_float(rg[2 * k + 1]),
                                      __uint_as_float(ru[2 * k]), __uint_as_float(ru[2 * k + 1]));
            store_h_chunk(tmO, stage, out, p.ldo, row, row_ok, pk, n0, p.n_valid);
        }
        return;
    }
    constexpr int kPerGroup = BN / kEpiGroups;
    constexpr int kChunks = kPerGroup / 16;
    const int slot = rg.slot;
    const float gw = rg.gw;
    const float *bias_row = p.bias ? p.bias + (int64_t)c.g * p.n_valid : nullptr;
    // Chunks of 16 columns, software-pipelined: tcgen05.wait::ld waits for all
    // of a thread's outstanding loads, so chunk i+1's TMEM load is issued right
    // after chunk i's wait and runs while chunk i is computed; chunk i's bias
    // loads go out before its wait.
    uint32_t r[2][16];
    tmem_ld_32x32b_x16(tbase + grp * kPerGroup, r[0]);
#pragma unroll
    for (int ci = 0; ci < kChunks; ++ci) {
        const int col = grp * kPerGroup + ci * 16;
        const int n0 = c.nt * BN + col;
        // bulk-stored outputs (GELU, row-ordered z): the store is warp-collective,
        // so lanes of invalid rows come along
        const bool warp_store = EPI == EPI_GELU || (EPI == EPI_SCATTER && p.scatter_rows);
        const bool active = (warp_store ? __any_sync(0xffffffffu, row_ok) : row_ok) && n0 < p.n_valid &&
                            !(EPI == EPI_SCATTER && !p.scatter_rows && slot < 0);
        const bool full_chunk = n0 + 16 <= p.n_valid;
        float bv[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) bv[k] = 0.f;
        if (bias_row && active) {
            const float *bias = bias_row + n0;
            if (full_chunk) {
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float4 b4 = __ldg(reinterpret_cast<const float4 *>(bias) + u);
                    bv[4 * u] = b4.x; bv[4 * u + 1] = b4.y; bv[4 * u + 2] = b4.z; bv[4 * u + 3] = b4.w;
                }
            } else {
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    if (n0 + k < p.n_valid) bv[k] = __ldg(bias + k);
            }
        }
        tmem_ld_wait_regs(r[ci & 1]);
        if (ci + 1 < kChunks) tmem_ld_32x32b_x16(tbase + col + 16, r[(ci + 1) & 1]);
        if (active) {
            float v[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) v[k] = __uint_as_float(r[ci & 1][k]) + bv[k];
            if (EPI == EPI_GELU) {
                uint32_t pk[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) pk[k] = gelu_erf_bf16x2(v[2 * k], v[2 * k + 1]);
                store_h_chunk(tmO, stage, static_cast<__nv_bfloat16 *>(p.out), p.ldo, row, row_ok, pk, n0, p.n_valid);
            } else if (EPI == EPI_SCATTER) {
                if (p.scatter_rows) {
                    float sv[16];
#pragma unroll
                    for (int k = 0; k < 16; ++k) sv[k] = gw * v[k];
                    store_z_chunk(tmO, stage, static_cast<float *>(p.out), p.ldo, row, row_ok, sv, n0, p.n_valid);
                } else if (p.accum_k > 0) {
                    float *dst = static_cast<float *>(p.out) + (int64_t)(slot / p.accum_k) * p.ldo + n0;
                    if (full_chunk) {
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            red_add_v4(dst + 4 * u, gw * v[4 * u], gw * v[4 * u + 1], gw * v[4 * u + 2],
                                       gw * v[4 * u + 3]);
                    } else {
#pragma unroll
                        for (int k = 0; k < 16; ++k)
                            if (n0 + k < p.n_valid) atomicAdd(dst + k, gw * v[k]);
                    }
                } else {
                    float *dst = static_cast<float *>(p.out) + (int64_t)slot * p.ldo + n0;
                    if (full_chunk) {
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            reinterpret_cast<float4 *>(dst)[u] =
                                make_float4(gw * v[4 * u], gw * v[4 * u + 1], gw * v[4 * u + 2], gw * v[4 * u + 3]);
                    } else {
#pragma unroll
                        for (int k = 0; k < 16; ++k)
                            if (n0 + k < p.n_valid) dst[k] = gw * v[k];
                    }
                }
            } else {  // EPI_LOGITS
                float *dst = static_cast<float *>(p.out) + (int64_t)row * p.ldo + n0;
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    if (n0 + k < p.n_valid) dst[k] = v[k];
            }
        }
    }
}
template <int BN, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                           const __grid_constant__ CUtensorMap tmO, const Params p) {
    if (p.tail_mode == 2) pdl_launch_dependents();   // reads only what the pair kernel's wait covered
    else pdl_enter();
    using S = Shape<BN>;
    constexpr int kStages = S::kStages;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = smem + kStages * S::kABytes;
    uint8_t *sOut = sB + kStages * S::kBBytes;
    uint64_t *full = reinterpret_cast<uint64_t *>(sOut + kOutStageBytes);
    uint64_t *empty = full + kStages;
    uint64_t *tfull = empty + kStages;
    uint64_t *tempty = tfull + 2;
    uint64_t *drain = tempty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    int *s_rowoff = reinterpret_cast<int *>(tmem_slot + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = p.num_groups;
    int *s_tcum = s_rowoff + (G + 1);
    if (p.row_offsets) {
        for (int i = threadIdx.x; i <= G; i += blockDim.x) s_rowoff[i] = p.row_offsets[i];
        if (p.tail_mode == 2) {
            __syncthreads();
            if (warp == 0) {   // groups before each one whose segment has an odd number of blocks
                int carry = 0;
                for (int g0 = 0; g0 <= G; g0 += 32) {
                    const int g = g0 + lane;
                    const int u = g < G ? ((s_rowoff[g + 1] - s_rowoff[g]) / BM) & 1 : 0;
                    int incl = u;
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const int n = __shfl_up_sync(0xffffffffu, incl, o);
                        if (lane >= o) incl += n;
                    }
                    if (g <= G) s_tcum[g] = carry + incl - u;
                    carry += __shfl_sync(0xffffffffu, incl, 31);
                }
            }
        }
    }
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
    const bool tails = rowoff && p.tail_mode == 2;
    // a table that fails the bounds-check build's test: no tiles at all
    const bool tbl_ok = !rowoff || MOE_BOUNDS(group_table_ok(s_rowoff, G));
    const int total = !tbl_ok ? 0 : tails ? s_tcum[G] * p.n_tiles : m_tiles * p.n_tiles;
    auto tile_of = [&](int i) {
        return tails ? decode_tail_tile(i, s_rowoff, s_tcum, G, p.n_tiles)
                     : decode_tile(i, rowoff, G, p.n_tiles, dense_mtiles);
    };

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            IssuedSlots iss;
            for (int i = blockIdx.x; i < total && ok; i += gridDim.x) {
                const TileCoord c = tile_of(i);
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
        const int grp = ew >> 2;
        const int r_in_tile = q * 32 + lane;
        int local = 0;
        for (int i = blockIdx.x; i < total; i += gridDim.x, ++local) {
            const int a = local & 1;
            const uint32_t aph = (local >> 1) & 1;
            const TileCoord c = tile_of(i);
            const int row_limit = rowoff ? s_rowoff[c.g + 1] : p.dense_rows;
            const RowGate rg = load_row_gate<EPI>(p, c.row0 + r_in_tile, row_limit);
            // warp-uniform decision: the TMEM loads below are warp-collective
            if (!__all_sync(0xffffffffu, mbar_wait(&tfull[a], aph, p.timeout_ns))) break;
            tc_fence_after();
            epilogue_tile<BN, EPI>(p, c, c.row0 + r_in_tile, row_limit,
                                   tmem_base + (static_cast<uint32_t>(q * 32) << 16) + a * BN, grp, &tmO,
                                   sOut + ew * kOutStageWarpBytes, rg);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[a]);
        }
        if (lane == 0) bulk_wait_all();   // this warp's bulk stores are complete before the CTA exits
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, S::kTmemCols);
    }
    if (p.tail_mode == 2) pdl_wait();   // complete only after the pair kernel beside it
}

// =====================================================================================
// Two CTAs (one cluster) per 256-row x 256-column tile.
// =====================================================================================
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t nclusters_x() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// shared::cluster address of the variable at shared::cta address `local` in CTA `rank`
__device__ __forceinline__ uint32_t mapa_shared(uint32_t local, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
    return r;
}
// Allocation shared by the CTA pair: one warp of each CTA executes it.
__device__ __forceinline__ void tmem_alloc2(uint32_t *slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc2(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_mma2_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive once on the barrier at the offset of `bar` in every CTA of cta_mask
// when all tcgen05 operations issued so far by this thread have completed.
__device__ __forceinline__ void tc_commit2_mc(uint64_t *bar, uint16_t cta_mask) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_u32(bar)),
        "h"(cta_mask)
        : "memory");
}
__device__ __forceinline__ void tc_commit2(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
// TMA load into this CTA's shared memory; completion is counted on the barrier
// at shared::cluster address `mbar_cluster` (the leader CTA's barrier).
__device__ __forceinline__ void tma_load_2d_pair(const CUtensorMap *map, uint32_t mbar_cluster, void *smem_dst,
                                                 int32_t c0, int32_t c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
        "%4}], [%2];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(mbar_cluster), "r"(c0), "r"(c1)
        : "memory");
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t bar_cluster) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait with cluster-scope acquire (arrivals come from the peer CTA).
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t *bar, uint32_t parity, uint64_t timeout_ns) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait_cluster(bar, parity)) return true;
        if (globaltimer_ns() - t0 > timeout_ns) {
            set_status(kStatusTimeout);
            return false;
        }
    }
}

template <int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    grouped_gemm_tc2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                            const __grid_constant__ CUtensorMap tmO, const Params p) {
    if (p.tail_mode == 1) {
        pdl_wait();                 // the dependent (the tail kernel, run beside this one) launches
        pdl_launch_dependents();    // only once everything before this kernel is complete
    } else {
        pdl_enter();
    }
    using S = Shape2;
    constexpr int BN = 256;
    constexpr int kStages = S::kStages;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = smem + kStages * S::kABytes;
    uint8_t *sOut = sB + kStages * S::kBBytes;
    uint64_t *full = reinterpret_cast<uint64_t *>(sOut + kOutStageBytes);
    uint64_t *empty = full + kStages;
    uint64_t *tfull = empty + kStages;
    uint64_t *tempty = tfull + 2;
    uint64_t *drain = tempty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    int *s_rowoff = reinterpret_cast<int *>(tmem_slot + 4);
    const int G = p.num_groups;
    int *s_units = s_rowoff + (G + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int cid = (int)cluster_id_x(), ncl = (int)nclusters_x();
    if (p.row_offsets) {
        for (int i = threadIdx.x; i <= G; i += blockDim.x) s_rowoff[i] = p.row_offsets[i];
        __syncthreads();
        if (warp == 0) {   // 256-row units before each group
            int carry = 0;
            for (int g0 = 0; g0 <= G; g0 += 32) {
                const int g = g0 + lane;
                const int blocks = g < G ? (s_rowoff[g + 1] - s_rowoff[g]) / BM : 0;
                const int u = p.tail_mode == 1 ? blocks / 2 : (blocks + 1) / 2;   // tail_mode 1: odd tails left out
                int incl = u;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int n = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += n;
                }
                if (g <= G) s_units[g] = carry + incl - u;
                carry += __shfl_sync(0xffffffffu, incl, 31);
            }
        }
    }
    if (warp == 0 && lane == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 2 * kEpiWarps);
        }
        mbar_init(drain, 1);
        fence_mbar_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) tmem_alloc2(tmem_slot, S::kTmemCols);
    tc_fence_before();
    __syncthreads();
    cluster_sync();   // both CTAs' barriers initialised and TMEM allocated before any cross-CTA traffic
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int *rowoff = p.row_offsets ? s_rowoff : nullptr;
    const int dense_units = (p.dense_rows + 2 * BM - 1) / (2 * BM);
    const int units = rowoff ? s_units[G] : dense_units;
    const bool tbl_ok = !rowoff || MOE_BOUNDS(group_table_ok(s_rowoff, G));
    const int total = tbl_ok ? units * p.n_tiles : 0;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            IssuedSlots iss;
            for (int i = cid; i < total && ok; i += ncl) {
                const TileCoord c = decode_unit_tile(i, rowoff, s_units, G, p.n_tiles, dense_units);
                const int arow = c.row0 + (int)rank * BM;
                int brow;
                if (EPI == EPI_SWIGLU)   // CTA 0: 128 gate rows, CTA 1: the matching 128 up rows
                    brow = c.g * p.b_group_rows + c.nt * (BN / 2) + (rank ? p.b_up_offset : 0);
                else
                    brow = c.g * p.b_group_rows + c.nt * BN + (int)rank * (BN / 2);
                for (int kb = 0; kb < p.num_k_blocks; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * (S::kABytes + S::kBBytes));
                    const uint32_t leader_full = mapa_shared(smem_u32(&full[stage]), 0);
                    tma_load_2d_pair(&tmA, leader_full, sA + stage * S::kABytes, kb * BK, arow);
                    tma_load_2d_pair(&tmB, leader_full, sB + stage * S::kBBytes, kb * BK, brow);
                    iss.note(stage, phase);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            // both CTAs' copies complete on the leader's barriers: the leader waits
            // (bounded) for every slot's last copies; the cluster barrier at the end
            // keeps the other CTA resident until then
            if (!ok && rank == 0) iss.drain(full, p.timeout_ns);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (leader CTA only)
        if (lane == 0 && rank == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(2 * BM, BN);
            int stage = 0;
            uint32_t phase = 0;
            int local = 0;
            bool ok = true;
            for (int i = cid; i < total && ok; i += ncl, ++local) {
                const int a = local & 1;
                const uint32_t aph = (local >> 1) & 1;
                if (!mbar_wait_cluster(&tempty[a], aph ^ 1, p.timeout_ns)) {
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
                        tc_mma2_bf16(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
                    tc_commit2_mc(&empty[stage], 0x3);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (ok) tc_commit2_mc(&tfull[a], 0x3);
            }
            if (!ok) {
                tc_commit2(drain);
                mbar_wait(drain, 0, p.timeout_ns);
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int ew = warp - 2;
        const int q = warp & 3;
        const int grp = ew >> 2;
        const int r_in_tile = q * 32 + lane;
        int local = 0;
        for (int i = cid; i < total; i += ncl, ++local) {
            const int a = local & 1;
            const uint32_t aph = (local >> 1) & 1;
            const TileCoord c = decode_unit_tile(i, rowoff, s_units, G, p.n_tiles, dense_units);
            const int row_limit = rowoff ? s_rowoff[c.g + 1] : p.dense_rows;
            const RowGate rg = load_row_gate<EPI>(p, c.row0 + (int)rank * BM + r_in_tile, row_limit);
            // warp-uniform decision: the TMEM loads below are warp-collective
            if (!__all_sync(0xffffffffu, mbar_wait(&tfull[a], aph, p.timeout_ns))) break;
            tc_fence_after();
            epilogue_tile<BN, EPI>(p, c, c.row0 + (int)rank * BM + r_in_tile, row_limit,
                                   tmem_base + (static_cast<uint32_t>(q * 32) << 16) + a * BN, grp, &tmO,
                                   sOut + ew * kOutStageWarpBytes, rg);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(mapa_shared(smem_u32(&tempty[a]), 0));
        }
        if (lane == 0) bulk_wait_all();   // this warp's bulk stores are complete before the CTA exits
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();   // the leader's last MMAs read this CTA's shared memory and TMEM
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc2(tmem_base, S::kTmemCols);
    }
}

}  // namespace tc
}  // namespace moe
