// moe_backward.cuh -- the layer's backward pass ("Extending Raschka's GPT-2 ...",
// section on making the router trainable: the router learns through the gate
// weights it produces and through the auxiliary loss, the experts through the
// outputs they are weighted into).
//
// Given the upstream gradient dy of y (and the weights of the two trainable
// auxiliary losses), with the routing and the dispatch of the forward (the
// same router, tables and permuted rows; recomputed here, nothing is kept
// from a forward call):
//   per routed row r (token t, slot j, expert e, weight w):
//     pre  = W1[e] x + b1          (recomputed: GELU pre-activation, or gate | up)
//     h    = act(pre)
//     dh   = w W2[e]^T dy[t]       dw = <W2[e]^T dy[t], h> + <dy[t], b2[e]>
//     da   = dh * act'(pre)        dx_r = W1[e]^T da
//     dW2[e] += w dy[t] h^T,  db2[e] += w dy[t],  dW1[e] += da x^T,  db1[e] += da
//   per token: the softmax over the kept scores backwards,
//     ds_kept_j = w_j (dw_j - sum_m w_m dw_m)   (+ the auxiliary losses' terms)
//     dW_g += x ds^T, db_g += ds, dx[t] = sum_j dx_r(t, j) + W_g ds
// The contractions run on the CUDA cores in fp32 (strided grouped GEMM below:
// row-grouped for the per-row products, K-grouped for the per-expert weight
// gradients, whose contraction runs over each expert's routed rows); inputs in
// bf16 are widened exactly.  Every sum has a fixed order: results are bitwise
// reproducible.
#pragma once

#include "moe_common.cuh"
#include "moe_route.cuh"

namespace moe {
namespace bwd {

constexpr int TM = 64, TN = 64, TK = 16;

// C[m, n] = sum_k A(m, k) B(n, k),  A(m, k) = A[a_off + m a_sm + k a_sk],
// B(n, k) = B[b_off + n b_sn + k b_sk], C[c_off + m c_sm + n c_sn], per group g:
//   ROWS mode (row_offsets, counts): the M rows of group g are the permuted
//     rows [row_offsets[g], row_offsets[g] + counts[g]); b_off = g * b_group
//   KGRP mode (row_offsets, counts): the contraction of group g runs over
//     k in [row_offsets[g], row_offsets[g] + counts[g]); M, N fixed; c_off = g * c_group
//   dense: one group, M rows, K columns
enum { DENSE = 0, ROWS = 1, KGRP = 2 };

template <typename TA, typename TB>
struct GemmParams {
    const TA *A;
    int64_t a_sm, a_sk;
    const TB *B;
    int64_t b_sn, b_sk, b_group;
    float *C;
    int64_t c_sm, c_sn, c_group;
    int M, N, K;                 // dense / KGRP: output M x N; dense and ROWS: contraction length K
    const int *row_offsets;      // ROWS / KGRP: [G+1] segment starts (multiples of 128)
    const int *counts;           // ROWS / KGRP: rows of each group
    int groups;
    int mode;
};

template <typename T>
__device__ __forceinline__ float ld_f(const T *p) { return to_f32(*p); }

template <typename TA, typename TB>
__global__ void __launch_bounds__(256) gemm_strided_kernel(const GemmParams<TA, TB> p) {
    __shared__ float As[TK][TM + 4];
    __shared__ float Bs[TK][TN + 4];
    const int tid = threadIdx.x;
    int g = 0, m_lo, m_hi, k_lo, k_hi;
    int64_t b_off = 0, c_off = 0;
    if (p.mode == ROWS) {
        const int row0 = blockIdx.x * TM;
        const int G = p.groups;
        if (row0 >= p.row_offsets[G]) return;
        int lo = 0, hi = G - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (p.row_offsets[mid] <= row0) lo = mid;
            else hi = mid - 1;
        }
        g = lo;
        m_lo = row0;
        m_hi = min(row0 + TM, p.row_offsets[g] + p.counts[g]);
        if (m_lo >= m_hi) return;   // padding rows of the segment: nothing to compute
        k_lo = 0;
        k_hi = p.K;
        b_off = (int64_t)g * p.b_group;
    } else if (p.mode == KGRP) {
        g = blockIdx.z;
        m_lo = blockIdx.x * TM;
        m_hi = min(m_lo + TM, p.M);
        k_lo = p.row_offsets[g];
        k_hi = k_lo + p.counts[g];
        c_off = (int64_t)g * p.c_group;
    } else {
        m_lo = blockIdx.x * TM;
        m_hi = min(m_lo + TM, p.M);
        k_lo = 0;
        k_hi = p.K;
    }
    const int n_lo = blockIdx.y * TN;
    const int n_hi = min(n_lo + TN, p.N);
    if (m_lo >= m_hi || n_lo >= n_hi) return;
    const int tx = tid & 15, ty = tid >> 4;
    float acc[4][4] = {};
    const bool a_m_fast = p.a_sm == 1, b_n_fast = p.b_sn == 1;
    for (int k0 = k_lo; k0 < k_hi; k0 += TK) {
        for (int i = tid; i < TM * TK; i += 256) {
            // coalesced along whichever index is contiguous in memory
            const int m = a_m_fast ? i % TM : i / TK, k = a_m_fast ? i / TM : i % TK;
            const int r = m_lo + m, kk = k0 + k;
            As[k][m] = (r < m_hi && kk < k_hi) ? ld_f(p.A + r * p.a_sm + kk * p.a_sk) : 0.f;
            const int n = b_n_fast ? i % TN : i / TK, k2 = b_n_fast ? i / TN : i % TK;
            const int c = n_lo + n, kk2 = k0 + k2;
            Bs[k2][n] = (c < n_hi && kk2 < k_hi) ? ld_f(p.B + b_off + c * p.b_sn + kk2 * p.b_sk) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < TK; ++k) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = As[k][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = Bs[k][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = m_lo + ty * 4 + i;
        if (r >= m_hi) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c = n_lo + tx * 4 + j;
            if (c < n_hi) p.C[c_off + r * p.c_sm + c * p.c_sn] = acc[i][j];
        }
    }
}

// The upstream gradient per permuted row: g[r] = dy[token of r] (fp32), 0 on
// padding rows and on the rows past the last segment (*row_end = the end of
// the last expert's segment; perm_slot holds nothing there).  Grid-stride over
// rows_cap * D / 4 float4s.
__global__ void __launch_bounds__(256) gather_rows_kernel(const float *__restrict__ dy, int64_t rows_cap, int D, int K,
                                                          const int *__restrict__ perm_slot,
                                                          const int *__restrict__ row_end, float *__restrict__ g) {
    const int64_t nq = rows_cap * (D / 4);
    const int64_t rend = *row_end;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < nq; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / (D / 4);
        const int d = (int)(i - r * (D / 4)) * 4;
        const int slot = r < rend ? perm_slot[r] : -1;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (slot >= 0) v = *reinterpret_cast<const float4 *>(dy + (int64_t)(slot / K) * D + d);
        *reinterpret_cast<float4 *>(g + r * D + d) = v;
    }
}

__device__ __forceinline__ float gelu_f(float v) { return 0.5f * v * (1.0f + erff(v * 0.70710678118654752f)); }
__device__ __forceinline__ float gelu_grad_f(float v) {
    return 0.5f * (1.0f + erff(v * 0.70710678118654752f)) + v * expf(-0.5f * v * v) * 0.39894228040143268f;
}
__device__ __forceinline__ float sigmoid_f(float v) { return 1.0f / (1.0f + expf(-v)); }

// Per permuted row (one warp per row): the activation and its backward.
//   pre [rows, rows1] (W1 x, without b1), dhr [rows, H] (W2^T dy), g [rows, D] (dy rows)
//   -> h [rows, H] fp32, dA [rows, rows1], gw [rows, D] = w g, dw [rows] = <dhr, h> + <g, b2>
// Padding rows (and the rows past the last segment, *row_end on) get zeros everywhere.
__global__ void __launch_bounds__(256) act_backward_kernel(const float *__restrict__ pre, const float *__restrict__ dhr,
                                                           const float *__restrict__ g, int64_t rows_cap, int D, int H,
                                                           int swiglu, const int *__restrict__ perm_slot,
                                                           const int *__restrict__ row_end,
                                                           const int *__restrict__ topk_idx,
                                                           const float *__restrict__ topk_w,
                                                           const float *__restrict__ b1, const float *__restrict__ b2,
                                                           float *__restrict__ h, float *__restrict__ dA,
                                                           float *__restrict__ gw, float *__restrict__ dw) {
    const int lane = threadIdx.x & 31;
    const int64_t r = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    if (r >= rows_cap) return;
    const int rows1 = swiglu ? 2 * H : H;
    const int slot = r < (int64_t)*row_end ? perm_slot[r] : -1;
    const float *pr = pre + r * rows1;
    const float *dr = dhr + r * H;
    float *hr = h + r * H, *ar = dA + r * rows1, *gwr = gw + r * D;
    if (slot < 0) {
        for (int n = lane; n < H; n += 32) hr[n] = 0.f;
        for (int n = lane; n < rows1; n += 32) ar[n] = 0.f;
        for (int c = lane; c < D; c += 32) gwr[c] = 0.f;
        if (lane == 0) dw[r] = 0.f;
        return;
    }
    const int e = topk_idx[slot];
    const float w = topk_w[slot];
    float dot = 0.f;   // <W2^T dy, h> + <dy, b2>: lanes stride the columns, then a fixed xor tree
    for (int n = lane; n < H; n += 32) {
        float hv, da_g, da_u = 0.f;
        const float dh = w * dr[n];
        if (swiglu) {
            const float gt = pr[n], up = pr[H + n];
            const float sg = sigmoid_f(gt);
            hv = gt * sg * up;
            da_g = dh * up * sg * (1.0f + gt * (1.0f - sg));
            da_u = dh * gt * sg;
            ar[H + n] = da_u;
        } else {
            const float a = pr[n] + (b1 ? b1[(int64_t)e * H + n] : 0.f);
            hv = gelu_f(a);
            da_g = dh * gelu_grad_f(a);
        }
        ar[n] = da_g;
        hr[n] = hv;
        dot = fmaf(dr[n], hv, dot);
    }
    const float *gr = g + r * D;
    for (int c = lane; c < D; c += 32) {
        gwr[c] = w * gr[c];
        if (b2) dot = fmaf(gr[c], b2[(int64_t)e * D + c], dot);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    if (lane == 0) dw[r] = dot;
}

// Per-expert statistics the auxiliary losses' gradients need, from the exact
// integer partials (moe_aux_partials layout): f_e = counts / (T K) and
// dCV^2/dimportance_e = 2 (imp_e - m) / (N m^2) - 2 var / (N m^3).
__global__ void aux_grad_prep_kernel(int N, int K, const long long *__restrict__ part, float *__restrict__ f,
                                     float *__restrict__ dimp) {
    if (blockIdx.x != 0 || threadIdx.x != 0) return;
    const long long T = part[3 * N];
    double m = 0.0, var = 0.0;
    for (int e = 0; e < N; ++e) m += (double)part[N + e] / kFixScale;
    m /= N;
    for (int e = 0; e < N; ++e) {
        const double d = (double)part[N + e] / kFixScale - m;
        var += d * d;
    }
    var /= N;
    for (int e = 0; e < N; ++e) {
        f[e] = T > 0 ? (float)((double)part[e] / ((double)T * K)) : 0.f;
        const double im = (double)part[N + e] / kFixScale;
        dimp[e] = m != 0.0 ? (float)(2.0 * (im - m) / (N * m * m) - 2.0 * var / (N * m * m * m)) : 0.f;
    }
}

// Per token (one warp): the router scores' gradient ds [T, N].
//   dw_j = dw[row of slot j] + a_imp dimp[e_j]; ds_kept = w (dw - sum_m w_m dw_m)
//   Switch-style loss: ds_e += a_sw (N / T) p_e (f_e - sum_e' f_e' p_e'), p the full softmax
__global__ void __launch_bounds__(256) router_backward_kernel(const float *__restrict__ logits,
                                                              const int *__restrict__ topk_idx,
                                                              const float *__restrict__ topk_w,
                                                              const int *__restrict__ slot_row,
                                                              const float *__restrict__ dw, const float *__restrict__ f,
                                                              const float *__restrict__ dimp, int T, int N, int K,
                                                              float a_sw, float a_imp, float *__restrict__ ds) {
    const int lane = threadIdx.x & 31;
    const int t = (int)((blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5);
    if (t >= T) return;
    const float *s = logits + (size_t)t * N;
    float *dst = ds + (size_t)t * N;
    float mx = -INFINITY;
    for (int e = lane; e < N; e += 32) mx = fmaxf(mx, s[e] != s[e] ? -INFINITY : s[e]);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float z = 0.f, fp = 0.f;
    for (int e = lane; e < N; e += 32) {
        const float ex = (s[e] != s[e] || mx == -INFINITY) ? 0.f : expf(s[e] - mx);
        z += ex;
        fp += f[e] * ex;
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        z += __shfl_xor_sync(0xffffffffu, z, o);
        fp += __shfl_xor_sync(0xffffffffu, fp, o);
    }
    fp = z > 0.f ? fp / z : 0.f;
    const float cs = a_sw * (float)N / (float)T;
    for (int e = lane; e < N; e += 32) {
        const float pe = (s[e] != s[e] || mx == -INFINITY || z == 0.f) ? 0.f : expf(s[e] - mx) / z;
        dst[e] = a_sw != 0.f ? cs * pe * (f[e] - fp) : 0.f;
    }
    __syncwarp();
    // the kept slots (K <= 32: one per lane)
    float wj = 0.f, dwj = 0.f;
    int ej = -1;
    if (lane < K) {
        ej = topk_idx[(size_t)t * K + lane];
        wj = topk_w[(size_t)t * K + lane];
        const int r = slot_row[(size_t)t * K + lane];
        dwj = (r >= 0 ? dw[r] : 0.f) + a_imp * dimp[ej];
    }
    float wdw = 0.f;
    for (int j = 0; j < K; ++j) wdw += __shfl_sync(0xffffffffu, wj * dwj, j);   // slot order
    if (lane < K) dst[ej] += wj * (dwj - wdw);
}

// Column sums over each group's rows, in row order: out[g, c] = sum_{r in group g} in[r, c].
// Grid (ceil(C / 256), groups); a group's rows: [row_offsets[g], + counts[g]) or, without
// row_offsets, all rows (one group).
__global__ void __launch_bounds__(256) column_sums_kernel(const float *__restrict__ in, int64_t ld, int C,
                                                          const int *__restrict__ row_offsets,
                                                          const int *__restrict__ counts, int64_t dense_rows,
                                                          float *__restrict__ out) {
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    const int g = blockIdx.y;
    if (c >= C) return;
    const int64_t r0 = row_offsets ? row_offsets[g] : 0;
    const int64_t r1 = row_offsets ? r0 + counts[g] : dense_rows;
    float acc = 0.f;
    for (int64_t r = r0; r < r1; ++r) acc += in[r * ld + c];
    out[(int64_t)g * C + c] = acc;
}

}  // namespace bwd
}  // namespace moe
