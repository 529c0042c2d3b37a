// Column gather and scatter of bf16 matrices, for weights quantized in a
// permuted input-channel order (act-order, the GPTQ-style variant the
// TensorRT-LLM page "Modify small-batched weight only quantization" sets beside
// the channel-wise and group-wise AWQ/GPTQ kernels): with the packed columns
// j = 0 .. K-1 holding input channel perm[j],
//     forward     Y  = X[:, perm] . w_hat^T          (gather X's columns first)
//     transposed  dX[:, perm] = dY . w_hat           (scatter the result's columns)
// Rows that fit in shared memory are staged there (whole rows move with
// coalesced accesses); longer rows take plain copies, one thread per element.  An index outside the source (gather) or destination
// (scatter) is skipped (a gathered element reads as 0) and records
// kErrBadIndex in the device error word.
#pragma once

#include "common.cuh"

namespace w4 {

__global__ void __launch_bounds__(256) gather_columns_kernel(const uint16_t* __restrict__ A, int M, int src_cols,
                                                             const int32_t* __restrict__ idx, int L,
                                                             uint16_t* __restrict__ out) {
    const long long total = static_cast<long long>(M) * L;
    bool bad = false;
    for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
         e += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int m = static_cast<int>(e / L), j = static_cast<int>(e - static_cast<long long>(m) * L);
        const int c = __ldg(idx + j);
        uint16_t v = 0;
        if (c >= 0 && c < src_cols) v = A[static_cast<size_t>(m) * src_cols + c];
        else bad = true;
        out[e] = v;
    }
    if (bad) record_error(kErrBadIndex);
}

__global__ void __launch_bounds__(256) scatter_columns_kernel(const uint16_t* __restrict__ A, int M, int L,
                                                              const int32_t* __restrict__ idx, int dst_cols,
                                                              uint16_t* __restrict__ out) {
    const long long total = static_cast<long long>(M) * L;
    bool bad = false;
    for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
         e += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int m = static_cast<int>(e / L), j = static_cast<int>(e - static_cast<long long>(m) * L);
        const int c = __ldg(idx + j);
        if (c >= 0 && c < dst_cols) out[static_cast<size_t>(m) * dst_cols + c] = A[e];
        else bad = true;
    }
    if (bad) record_error(kErrBadIndex);
}

// The same copies with each row staged in shared memory, for rows that fit
// (both sides then move whole rows with coalesced accesses): one block per
// row (grid-stride), `row` holds src_cols (gather) or dst_cols (scatter)
// bf16.  Launched as programmatic dependents: they wait for the work before
// them, then let the matmul that follows start its prologue.
// (plain loads: the scatter reads the rows it later writes)
__device__ __forceinline__ void copy_row_in(uint16_t* row, const uint16_t* src, int n) {
    if ((reinterpret_cast<uintptr_t>(src) & 15) == 0 && (n & 7) == 0) {
        for (int i = threadIdx.x; i < n / 8; i += blockDim.x)
            reinterpret_cast<uint4*>(row)[i] = reinterpret_cast<const uint4*>(src)[i];
    } else {
        for (int i = threadIdx.x; i < n; i += blockDim.x) row[i] = src[i];
    }
}

__device__ __forceinline__ void copy_row_out(uint16_t* __restrict__ dst, const uint16_t* row, int n) {
    if ((reinterpret_cast<uintptr_t>(dst) & 15) == 0 && (n & 7) == 0) {
        for (int i = threadIdx.x; i < n / 8; i += blockDim.x)
            reinterpret_cast<uint4*>(dst)[i] = reinterpret_cast<const uint4*>(row)[i];
    } else {
        for (int i = threadIdx.x; i < n; i += blockDim.x) dst[i] = row[i];
    }
}

constexpr int kGatherChunk = 2048;   // output columns per block of gather_rows_kernel (4 per thread)

__global__ void __launch_bounds__(512) gather_rows_kernel(const uint16_t* __restrict__ A, int M, int src_cols,
                                                          const int32_t* __restrict__ idx, int L,
                                                          uint16_t* __restrict__ out) {
    // block (x, y): output columns x * kGatherChunk .. + kGatherChunk of rows y, y + gridDim.y, ...
    extern __shared__ __align__(16) uint16_t row[];
    pdl_wait();
    pdl_launch_dependents();
    bool bad = false;
    const int j0 = blockIdx.x * kGatherChunk + threadIdx.x;
    int c[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int j = j0 + 512 * u;
        c[u] = j < L ? __ldg(idx + j) : 0;     // independent loads, in flight together
    }
    for (int m = blockIdx.y; m < M; m += gridDim.y) {
        copy_row_in(row, A + static_cast<size_t>(m) * src_cols, src_cols);
        __syncthreads();
        uint16_t* o = out + static_cast<size_t>(m) * L;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int j = j0 + 512 * u;
            if (j < L) {
                const bool ok = c[u] >= 0 && c[u] < src_cols;
                bad = bad || !ok;
                o[j] = ok ? row[c[u]] : static_cast<uint16_t>(0);
            }
        }
        __syncthreads();
    }
    if (bad) record_error(kErrBadIndex);
}

// inv[perm[j]] = j for j < n (perm a permutation of [0, n); an entry out of
// range is skipped and recorded), so that a scatter by perm is a gather by inv.
__global__ void __launch_bounds__(256) invert_permutation_kernel(const int32_t* __restrict__ perm, int n,
                                                                 int32_t* __restrict__ inv) {
    pdl_wait();
    pdl_launch_dependents();
    bool bad = false;
    for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < n; j += gridDim.x * blockDim.x) {
        const int c = __ldg(perm + j);
        if (c >= 0 && c < n) inv[c] = j;
        else bad = true;
    }
    if (bad) record_error(kErrBadIndex);
}

__global__ void __launch_bounds__(512) scatter_rows_kernel(const uint16_t* __restrict__ A, int M, int L,
                                                           const int32_t* __restrict__ idx, int dst_cols,
                                                           uint16_t* __restrict__ out) {
    extern __shared__ __align__(16) uint16_t row[];
    pdl_wait();
    pdl_launch_dependents();
    bool bad = false;
    for (int m = blockIdx.x; m < M; m += gridDim.x) {
        uint16_t* o = out + static_cast<size_t>(m) * dst_cols;
        copy_row_in(row, o, dst_cols);            // columns no index names keep their values
        __syncthreads();
        const uint16_t* a = A + static_cast<size_t>(m) * L;
        for (int j = threadIdx.x; j < L; j += blockDim.x) {
            const int c = __ldg(idx + j);
            if (c >= 0 && c < dst_cols) row[c] = a[j];
            else bad = true;
        }
        __syncthreads();
        copy_row_out(o, row, dst_cols);
        __syncthreads();
    }
    if (bad) record_error(kErrBadIndex);
}

}  // namespace w4
