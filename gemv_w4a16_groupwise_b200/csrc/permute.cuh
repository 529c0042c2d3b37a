// Column gather and scatter of bf16 matrices, for weights quantized in a
// permuted input-channel order (act-order, the GPTQ-style variant the
// TensorRT-LLM page "Modify small-batched weight only quantization" sets beside
// the channel-wise and group-wise AWQ/GPTQ kernels): with the packed columns
// j = 0 .. K-1 holding input channel perm[j],
//     forward     Y  = X[:, perm] . w_hat^T          (gather X's columns first)
//     transposed  dX[:, perm] = dY . w_hat           (scatter the result's columns)
// Plain copies: one thread per element, rows of the output written
// contiguously.  An index outside the source (gather) or destination
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

}  // namespace w4
