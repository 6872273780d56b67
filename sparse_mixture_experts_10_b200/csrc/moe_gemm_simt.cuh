// moe_gemm_simt.cuh -- fp32 grouped GEMM on the CUDA cores.
//
// The tensor cores have no full-fp32 operand kind (only tf32, which cannot meet
// an fp32 1e-4 tolerance), so fp32 layers use this plain tiled kernel: 64 x 64
// output tiles, 16-deep K slices staged in shared memory, 4 x 4 outputs per
// thread.  Same operand conventions, tile-to-expert mapping and epilogues as
// the tensor-core kernel (moe_gemm_tc.cuh); fp32 hidden activations.
#pragma once

#include "moe_common.cuh"

namespace moe {
namespace simt {

constexpr int TM = 64, TN = 64, TK = 16;
enum { EPI_GELU = 0, EPI_SWIGLU = 1, EPI_SCATTER = 2, EPI_LOGITS = 3 };

struct Params {
    const float *A;
    int64_t lda;
    const float *B;
    int64_t ldb;
    int K;
    int num_groups;
    const int *row_offsets;   // [G+1] or nullptr (dense)
    int dense_rows;
    int b_group_rows;
    int b_up_offset;
    int n_valid;
    float *out;
    int64_t ldo;
    const float *bias;
    const int *perm_slot;
    const float *gate_w;
};

__device__ __forceinline__ float gelu_erf(float v) { return 0.5f * v * (1.0f + erff(v * 0.70710678118654752f)); }

template <int EPI>
__global__ void __launch_bounds__(256) grouped_gemm_simt_kernel(const Params p) {
    __shared__ float As[TK][TM + 4];
    __shared__ float Bs[TK][TN + 4];
    __shared__ float Cs[TM][TN + 1];
    const int tid = threadIdx.x;
    const int row0 = blockIdx.x * TM;
    int g = 0, rows_end;
    if (p.row_offsets) {
        const int G = p.num_groups;
        if (row0 >= p.row_offsets[G]) return;
        int lo = 0, hi = G - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (p.row_offsets[mid] <= row0) lo = mid;
            else hi = mid - 1;
        }
        g = lo;
        rows_end = p.row_offsets[g + 1];
    } else {
        if (row0 >= p.dense_rows) return;
        rows_end = p.dense_rows;
    }
    const int nt = blockIdx.y;
    // B row of local column n (0..63) and whether that output feature exists
    auto b_row = [&](int n, bool &valid) -> int64_t {
        if (EPI == EPI_SWIGLU) {
            const int f = nt * (TN / 2) + (n & 31);
            valid = f < p.n_valid;
            return (int64_t)g * p.b_group_rows + (n < 32 ? 0 : p.b_up_offset) + f;
        }
        const int f = nt * TN + n;
        valid = f < p.n_valid;
        return (int64_t)g * p.b_group_rows + f;
    };
    const int tx = tid & 15, ty = tid >> 4;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < p.K; k0 += TK) {
        for (int i = tid; i < TM * TK; i += 256) {
            const int m = i / TK, k = i % TK;
            const int r = row0 + m;
            As[k][m] = (r < rows_end && k0 + k < p.K) ? p.A[(int64_t)r * p.lda + k0 + k] : 0.f;
            bool valid;
            const int64_t br = b_row(m, valid);
            Bs[k][m] = (valid && k0 + k < p.K) ? p.B[br * p.ldb + k0 + k] : 0.f;
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
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) Cs[ty * 4 + i][tx * 4 + j] = acc[i][j];
    __syncthreads();
    if (EPI == EPI_SWIGLU) {
        for (int i = tid; i < TM * 32; i += 256) {
            const int m = i / 32, n = i % 32;
            const int r = row0 + m, f = nt * 32 + n;
            if (r >= rows_end || f >= p.n_valid) continue;
            const float gt = Cs[m][n], up = Cs[m][n + 32];
            p.out[(int64_t)r * p.ldo + f] = gt / (1.0f + expf(-gt)) * up;
        }
        return;
    }
    for (int i = tid; i < TM * TN; i += 256) {
        const int m = i / TN, n = i % TN;
        const int r = row0 + m, f = nt * TN + n;
        if (r >= rows_end || f >= p.n_valid) continue;
        float v = Cs[m][n] + (p.bias ? p.bias[(int64_t)g * p.n_valid + f] : 0.f);
        if (EPI == EPI_GELU) {
            p.out[(int64_t)r * p.ldo + f] = gelu_erf(v);
        } else if (EPI == EPI_SCATTER) {   // no perm_slot (dense rows, shared expert): row r is token r, weight 1
            const int slot = p.perm_slot ? p.perm_slot[r] : r;
            if (slot >= 0) p.out[(int64_t)slot * p.ldo + f] = (p.perm_slot ? p.gate_w[slot] : 1.f) * v;
        } else {
            p.out[(int64_t)r * p.ldo + f] = v;
        }
    }
}

}  // namespace simt
}  // namespace moe
