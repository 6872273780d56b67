// moe_decode_stream.cuh -- the whole layer for one or two tokens as one
// uninterrupted stream of whole weight rows.
//
// At T = 1 the layer reads K experts' weights (three D x H matrices each for
// SwiGLU) and does one multiply-add per weight element: the time is the time
// the live experts' weights take to come in from HBM (the Transformers-v5 MoE
// article's gpt-oss decode estimate).  Tensor cores bring nothing here, and
// 128-row weight tiles (the decode GEMM's MMA operand) read every weight row in
// 128-byte pieces; a plain read of a few hundred MB also needs ~10 us before it
// reaches full rate.  So this kernel keeps the memory system busy with one
// stream per SM that never drains between the two projections:
//   routing  as the fused decode kernel (R1 slab scores, grid barrier, R2 in
//            every CTA, R3 tables; moe_decode_fused.cuh)
//   U        unit u = (live expert l, hidden unit j), the units of all live
//            experts cut into equal contiguous ranges, one per CTA; a unit is one
//            weight row of W1 (GELU) or the gate row and the up row of W_gu
//            (SwiGLU), each row one bulk copy of D*2 contiguous bytes into a
//            shared-memory ring; h[slot, j] = act(row . x_t) for every kept slot
//            of the expert, rounded to bf16 as the tensor-core path does
//   --- grid barrier (h complete); the producer keeps loading through it
//   D        row r = (output d, live expert l), d-major, cut the same way; each
//            row of W_down is one bulk copy of H*2 bytes; z[slot, d] =
//            w_slot (row . h_slot + b2[d])
//   --- grid barrier (z complete)
//   C        y[t] = the kept slots' z rows in slot order
// A single thread of warp 0 issues the copies; warps 1-16 take the units and rows
// round-robin.  The producer's only dependency is the routing: the rows of the
// down projection are loaded while the up projection finishes and the barrier
// is waited on.  Every wait is bounded (status MOE_STATUS_TIMEOUT on expiry).
#pragma once

#include "moe_common.cuh"
#include "moe_decode_fused.cuh"
#include "moe_gemm_tc.cuh"

namespace moe {
namespace dst {

using dfu::Params;
using dfu::Tables;
constexpr int kConsumers = 16;            // consumer warps (warp 0 issues the copies)
constexpr int kThreads = 32 * (kConsumers + 1);
constexpr int kMaxT = 4;                  // tokens whose x rows are held in shared memory
constexpr int kMaxSlots = 8;              // T * K: h rows held in shared memory (bf16)
constexpr int kMaxStages = 32;            // IssuedSlots tracks at most 32 ring slots
constexpr uint32_t kTableBytes = 2 * dfu::kMaxSlots * 2 + 8 * 40 * 4;

__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// Count of ring stages the producer has issued, published to the consumer
// warps through shared memory.
__device__ __forceinline__ void publish_issued(uint32_t *ctr, uint32_t n) {
    asm volatile("st.release.cta.shared::cta.u32 [%0], %1;" ::"r"(smem_u32(ctr)), "r"(n) : "memory");
}
__device__ __forceinline__ uint32_t read_issued(const uint32_t *ctr) {
    uint32_t n;
    asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(n) : "r"(smem_u32(ctr)) : "memory");
    return n;
}

// Barrier among the consumer warps only (named barrier 1).
__device__ __forceinline__ void consumers_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumers * 32) : "memory");
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// A 32-bit word of two bf16 (low element first) as a pair of fp32.
__device__ __forceinline__ uint64_t bf16x2_as_f2(uint32_t w) {
    return f2_pack(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// NR weight rows (n8 16-byte words of bf16 each, in shared memory) against KC
// bf16 vectors in shared memory (rows of `vec`, ld elements apart, selected by
// idx[m]); with NR = 2 (the gate and up rows of one SwiGLU unit) each vector
// word is loaded and widened once for both rows.  Each lane keeps two
// fp32-pair accumulators per row and vector (sm_100 f32x2 FMA); the four
// partial sums and then the lanes are added in a fixed order.  out[r][m] for
// m >= KC is 0.
template <int KC, int NR>
__device__ __forceinline__ void row_dot(const uint4 *w0, const uint4 *w1, int n8, const __nv_bfloat16 *vec, int ld,
                                        const int (&idx)[kMaxT], float (&out)[2][kMaxT]) {
    const int lane = threadIdx.x & 31;
    uint64_t acc[NR][KC][2];
#pragma unroll
    for (int r = 0; r < NR; ++r)
#pragma unroll
        for (int m = 0; m < KC; ++m) acc[r][m][0] = acc[r][m][1] = 0ull;   // pairs of +0.0f
#pragma unroll 2
    for (int v = lane; v < n8; v += 32) {
        uint4 q[NR];
        q[0] = w0[v];
        if (NR == 2) q[NR - 1] = w1[v];
#pragma unroll
        for (int m = 0; m < KC; ++m) {
            const uint4 hq = reinterpret_cast<const uint4 *>(vec + (size_t)idx[m] * ld)[v];
            const uint64_t x0 = bf16x2_as_f2(hq.x), x1 = bf16x2_as_f2(hq.y), x2 = bf16x2_as_f2(hq.z),
                           x3 = bf16x2_as_f2(hq.w);
#pragma unroll
            for (int r = 0; r < NR; ++r) {
                acc[r][m][0] = f2_fma(bf16x2_as_f2(q[r].x), x0, acc[r][m][0]);
                acc[r][m][1] = f2_fma(bf16x2_as_f2(q[r].y), x1, acc[r][m][1]);
                acc[r][m][0] = f2_fma(bf16x2_as_f2(q[r].z), x2, acc[r][m][0]);
                acc[r][m][1] = f2_fma(bf16x2_as_f2(q[r].w), x3, acc[r][m][1]);
            }
        }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int m = 0; m < kMaxT; ++m) out[r][m] = 0.f;
#pragma unroll
    for (int r = 0; r < NR; ++r)
#pragma unroll
        for (int m = 0; m < KC; ++m) {
            float a0, a1, b0, b1;
            f2_unpack(acc[r][m][0], a0, a1);
            f2_unpack(acc[r][m][1], b0, b1);
            out[r][m] = warp_sum((a0 + a1) + (b0 + b1));
        }
}

// row_dot for the expert's kc kept slots (1 <= kc <= kMaxT, warp-uniform).
template <int NR>
__device__ __forceinline__ void row_dot_kc(int kc, const uint4 *w0, const uint4 *w1, int n8,
                                           const __nv_bfloat16 *vec, int ld, const int (&idx)[kMaxT],
                                           float (&out)[2][kMaxT]) {
    switch (kc) {
        case 1: row_dot<1, NR>(w0, w1, n8, vec, ld, idx, out); break;
        case 2: row_dot<2, NR>(w0, w1, n8, vec, ld, idx, out); break;
        case 3: row_dot<3, NR>(w0, w1, n8, vec, ld, idx, out); break;
        default: row_dot<4, NR>(w0, w1, n8, vec, ld, idx, out); break;
    }
}

// Shared-memory plan of the kernel for a layer: ring stages of stage_bytes,
// then the x / h area, the routing tables and the barriers.
struct Smem {
    uint32_t stage_bytes, stages, xh_bytes;
    __host__ __device__ uint32_t ring_bytes() const { return stages * stage_bytes; }
    __host__ __device__ size_t total() const {
        return 1024 + (size_t)ring_bytes() + xh_bytes + kTableBytes + (2 * kMaxStages + 8) * 8 + 64;
    }
};

template <int EPI_UP>
__global__ void __launch_bounds__(kThreads, 1) decode_stream_kernel(const Params p, const Smem sm) {
    pdl_enter();
    constexpr bool kSwiglu = EPI_UP == dec::EPI_SWIGLU;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = align_smem_1024(smem_raw);
    uint8_t *ring = smem;
    uint8_t *sXH = smem + sm.ring_bytes();
    uint8_t *sT = sXH + sm.xh_bytes;
    Tables tb;
    tb.row = reinterpret_cast<int16_t *>(sT);
    tb.ent = tb.row + dfu::kMaxSlots;
    tb.cnt = reinterpret_cast<int *>(tb.ent + dfu::kMaxSlots);
    tb.kept = tb.cnt + 40;
    tb.rowoff = tb.kept + 40;
    tb.koff = tb.rowoff + 40;
    tb.live = tb.koff + 40;
    tb.nlive = tb.live + 40;
    int *s_flag = tb.nlive + 40;   // [4], then the gate weights of the T*K slots
    uint64_t *full = reinterpret_cast<uint64_t *>(sT + kTableBytes);
    uint64_t *empty = full + kMaxStages;
    uint32_t *issued = reinterpret_cast<uint32_t *>(empty + kMaxStages);   // stages issued so far

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = (int)sm.stages;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        fence_mbar_init();
        *issued = 0;
    }
    __syncthreads();

    // ---------------------------------------------------------------- routing
    bool ok = true;
    if ((int)blockIdx.x < p.n_slabs) dfu::route_r1<16, EPI_UP>(p, smem);
    ok = dfu::grid_sync_all(p, 1, s_flag);
    if (ok) dfu::route_r2_all(p, smem);
    if (ok) dfu::route_r3(p, tb, smem, true);
    if (threadIdx.x == 0) s_flag[1] = 0;   // set by a consumer warp whose wait ran out
    __syncthreads();   // the routing scratch in the ring is free from here on

    const int D = p.D, H = p.H, K = p.K;
    const int nlive = ok ? *tb.nlive : 0;
    const int G = (int)gridDim.x, c = (int)blockIdx.x;
    const int64_t U = (int64_t)nlive * H, R = (int64_t)nlive * D;
    const int64_t u0 = U * c / G, u1 = U * (c + 1) / G;
    const int64_t r0 = R * c / G, r1 = R * (c + 1) / G;
    constexpr int kSpu = kSwiglu ? 2 : 1;   // ring stages per unit
    const int64_t n_up = u1 - u0, n_dn = r1 - r0;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0 && ok) {
            const __nv_bfloat16 *W1 = static_cast<const __nv_bfloat16 *>(p.W1);
            const __nv_bfloat16 *W2 = static_cast<const __nv_bfloat16 *>(p.W2);
            // stage g of this CTA: the U rows (a unit's gate row, then its up row),
            // then the D rows
            const int64_t n_stages = n_up * kSpu + n_dn;
            auto row_of = [&](int64_t g) -> const __nv_bfloat16 * {
                if (g < n_up * kSpu) {
                    const int64_t u = u0 + g / kSpu;
                    const int l = (int)(u / H), j = (int)(u - (int64_t)l * H);
                    const int e = tb.live[l];
                    const int64_t row = kSwiglu ? (int64_t)e * 2 * H + (g % kSpu) * H + j : (int64_t)e * H + j;
                    return W1 + row * D;
                }
                const int64_t r = r0 + (g - n_up * kSpu);
                const int d = (int)(r / nlive), l = (int)(r - (int64_t)d * nlive);
                return W2 + ((int64_t)tb.live[l] * D + d) * H;
            };
            int st = 0;
            uint32_t ph = 0;
            IssuedSlots iss;
            for (int64_t g = 0; g < n_stages && ok; ++g) {
                if (!mbar_wait(&empty[st], ph ^ 1, p.timeout_ns)) {
                    ok = false;
                    break;
                }
                const uint32_t bytes = (uint32_t)(g < n_up * kSpu ? D : H) * 2;
                mbar_arrive_expect_tx(&full[st], bytes);
                bulk_load(ring + (size_t)st * sm.stage_bytes, row_of(g), bytes, &full[st]);
                publish_issued(issued, (uint32_t)(g + 1));
                iss.note(st, ph);
                if (++st == S) {
                    st = 0;
                    ph ^= 1;
                }
            }
            if (!ok) iss.drain(full, p.timeout_ns);   // copies in flight land before the CTA leaves
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    const int cw = warp - 1, ct = threadIdx.x - 32;
    // bf16 rows in shared memory: one conflict-free 16-byte load per lane and step
    __nv_bfloat16 *xs = reinterpret_cast<__nv_bfloat16 *>(sXH);  // [T][D] (U phase)
    __nv_bfloat16 *hs = reinterpret_cast<__nv_bfloat16 *>(sXH);  // [T*K][H] (D phase)
    float *s_w = reinterpret_cast<float *>(s_flag + 4);          // [T*K] gate weights (D phase)
    if (ok) {
        for (int i = ct; i < p.T * D / 8; i += kConsumers * 32)
            reinterpret_cast<uint4 *>(xs)[i] = __ldg(reinterpret_cast<const uint4 *>(p.x) + i);
    }
    consumers_sync();
    bool cok = ok;
    // Warps take stages round-robin, so a warp can reach a slot before the
    // slot's previous stage has even been issued; a parity wait there would
    // match the phase before.  So a consumer first waits (bounded) until the
    // producer has issued its stage, which also means that the slot's previous
    // phase is complete, and then waits on that stage's phase.
    auto stage_wait = [&](int64_t si) -> const uint4 * {
        bool w = true;
        if (lane == 0 && read_issued(issued) <= (uint32_t)si) {
            const uint64_t t0 = globaltimer_ns();
            while (read_issued(issued) <= (uint32_t)si) {
                if (globaltimer_ns() - t0 > p.timeout_ns) {
                    set_status(kStatusTimeout);
                    w = false;
                    break;
                }
            }
        }
        if (!__shfl_sync(0xffffffffu, w, 0)) return nullptr;
        const int s = (int)(si % S);
        if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (uint32_t)((si / S) & 1), p.timeout_ns))) return nullptr;
        return reinterpret_cast<const uint4 *>(ring + (size_t)s * sm.stage_bytes);
    };
    auto stage_free = [&](int64_t si) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[(int)(si % S)]);
    };
    // U: units of this CTA, round-robin over the consumer warps
    for (int64_t i = cw; i < n_up && cok; i += kConsumers) {
        const int64_t u = u0 + i;
        const int l = (int)(u / H), j = (int)(u - (int64_t)l * H);
        const int e = tb.live[l];
        const int kc = tb.kept[e], kb = tb.koff[e];
        int slot[kMaxT], tok[kMaxT];
#pragma unroll
        for (int m = 0; m < kMaxT; ++m) {
            slot[m] = m < kc ? tb.ent[kb + m] : 0;
            tok[m] = slot[m] / K;
        }
        const float b = (!kSwiglu && p.b1) ? __ldg(p.b1 + (int64_t)e * H + j) : 0.f;   // in flight meanwhile
        const int64_t si = i * kSpu;
        const uint4 *wg = stage_wait(si);
        const uint4 *wu = (kSwiglu && wg) ? stage_wait(si + 1) : wg;
        if (!wg || !wu) {
            cok = false;
            break;
        }
        float acc[2][kMaxT];
        row_dot_kc<kSwiglu ? 2 : 1>(kc, wg, wu, D / 8, xs, D, tok, acc);
        stage_free(si);
        if (kSwiglu) stage_free(si + 1);
        // h[slot, j], rounded to bf16 as the tensor-core epilogues do
        if (lane < kc) {
            float gl = acc[0][0], ul = acc[1][0];
            int sl = slot[0];
#pragma unroll
            for (int m = 1; m < kMaxT; ++m)
                if (lane == m) {
                    gl = acc[0][m];
                    ul = acc[1][m];
                    sl = slot[m];
                }
            const uint32_t hv = kSwiglu ? tc::swiglu_bf16x2(gl, gl, ul, ul) : tc::gelu_erf_bf16x2(gl + b, gl + b);
            p.h[(int64_t)tb.row[sl] * H + j] = __ushort_as_bfloat16(static_cast<unsigned short>(hv & 0xffffu));
        }
    }
    // h of this CTA written: release it to the grid; the producer goes on loading
    if (!cok && lane == 0) s_flag[1] = 1;
    consumers_sync();
    cok = cok && s_flag[1] == 0;
    if (ct == 0) {
        int f = 0;
        if (cok) {
            __threadfence();
            dfu::grid_arrive(p.bar4);
            f = dfu::grid_wait(p.bar4, gridDim.x, p.timeout_ns) ? 1 : 0;
        }
        s_flag[2] = f;
    }
    consumers_sync();
    cok = cok && s_flag[2] != 0;
    const int TK = p.T * K;
    if (cok) {
        // every kept slot's h row and the gate weights into shared memory (the x
        // rows are no longer needed)
        const int hv8 = H / 8;
        for (int i = ct; i < TK * hv8; i += kConsumers * 32) {
            const int s = i / hv8, v = i - s * hv8;
            const int r = tb.row[s];
            if (r >= 0)
                reinterpret_cast<uint4 *>(hs)[(size_t)s * hv8 + v] =
                    __ldcg(reinterpret_cast<const uint4 *>(p.h + (int64_t)r * H) + v);
        }
        for (int i = ct; i < TK; i += kConsumers * 32) s_w[i] = __ldcg(p.topk_w + i);
    }
    consumers_sync();
    // D: rows of the down projection, round-robin over the consumer warps
    for (int64_t i = cw; i < n_dn && cok; i += kConsumers) {
        const int64_t r = r0 + i;
        const int d = (int)(r / nlive), l = (int)(r - (int64_t)d * nlive);
        const int e = tb.live[l];
        const int kc = tb.kept[e], kb = tb.koff[e];
        int slot[kMaxT];
#pragma unroll
        for (int m = 0; m < kMaxT; ++m) slot[m] = m < kc ? tb.ent[kb + m] : 0;
        const float b = p.b2 ? __ldg(p.b2 + (int64_t)e * D + d) : 0.f;   // in flight meanwhile
        const int64_t si = n_up * kSpu + i;
        const uint4 *wd = stage_wait(si);
        if (!wd) {
            cok = false;
            break;
        }
        float acc[2][kMaxT];
        row_dot_kc<1>(kc, wd, wd, H / 8, hs, H, slot, acc);
        stage_free(si);
        if (lane < kc) {
            float a = acc[0][0];
            int sl = slot[0];
#pragma unroll
            for (int m = 1; m < kMaxT; ++m)
                if (lane == m) {
                    a = acc[0][m];
                    sl = slot[m];
                }
            __stcg(p.z + (int64_t)sl * D + d, s_w[sl] * (a + b));
        }
    }
    // C: once every CTA's z values are written, y[t, d] = the kept slots' z in slot order
    if (!cok && lane == 0) s_flag[1] = 1;
    consumers_sync();
    cok = cok && s_flag[1] == 0;
    if (ct == 0) {
        int f = 0;
        if (cok) {
            __threadfence();
            dfu::grid_arrive(p.bar5);
            f = dfu::grid_wait(p.bar5, gridDim.x, p.timeout_ns) ? 1 : 0;
        }
        s_flag[3] = f;
    }
    consumers_sync();
    if (!cok || !s_flag[3]) return;
    const int O = p.T * D;
    for (int o = c * kConsumers * 32 + ct; o < O; o += G * kConsumers * 32) {
        const int t = o / D, d = o - t * D;
        float acc = 0.f;
        bool any = false;
        for (int k = 0; k < K; ++k) {
            if (tb.row[t * K + k] < 0) continue;   // dropped by the capacity
            const float v = __ldcg(p.z + ((int64_t)t * K + k) * D + d);
            acc = any ? acc + v : v;
            any = true;
        }
        if (p.y_bf16) static_cast<__nv_bfloat16 *>(p.y)[o] = __float2bfloat16_rn(acc);
        else static_cast<float *>(p.y)[o] = acc;
    }
}

}  // namespace dst
}  // namespace moe
