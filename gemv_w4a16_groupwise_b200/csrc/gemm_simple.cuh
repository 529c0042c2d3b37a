// Plain CUDA-core W4A16 matmul for M > 4 on the shapes the tensor-core GEMM
// cannot stream: packed rows not 16-byte strided (K % 32 != 0), or, in
// transposed mode, dY rows not 16-byte strided (N % 8 != 0).  A CTA computes
// a 64 x 64 tile of the output from 32-long slices of the reduction staged in
// shared memory: the activations as fp32 and the weights dequantized to
// (q - z) s in fp32 (exact for an integer z: a 5-bit integer times an 11-bit
// significand; a fractional z rounds it once);
// each thread keeps 4 x 4 outputs and adds x w_hat with fp32 fma (every
// product exact), in ascending reduction order, then adds the bias and
// rounds once to bf16.
//   forward:    Y[m, n]  = sum_k X[m, k] w_hat[n, k]    (reduction over k)
//   transposed: dX[m, k] = sum_n dY[m, n] w_hat[n, k]   (reduction over n)
#pragma once

#include "gemv.cuh"

namespace w4 {

struct GemmSimpleArgs {
    const uint16_t* A;        // X [M, K] or dY [M, N], bf16
    const uint32_t* packed;   // [N, K / 8]
    const __half* S;
    const __half* Z;
    const uint16_t* bias;     // [output columns] bf16 or nullptr
    uint16_t* Y;              // [M, output columns] bf16
    int M, N, K, g, G, sz_row;
    int fmt;                  // format flags: kFmtZeroFloat, kFmtMetaBf16
};

constexpr int kGsTile = 64;   // output tile (rows of A x output columns)
constexpr int kGsRed = 32;    // reduction slice

template <bool TR>
__global__ void __launch_bounds__(256) gemm_simple_kernel(const GemmSimpleArgs a) {
    __shared__ float xs[kGsRed][kGsTile + 1];   // [reduction][row of A]
    __shared__ float ws[kGsRed][kGsTile + 1];   // [reduction][output column]
    const int L = TR ? a.K : a.N;               // output columns
    const int R = TR ? a.N : a.K;               // reduction length
    const int row0 = blockIdx.y * kGsTile, col0 = blockIdx.x * kGsTile;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    const int W8 = a.K / 8;
    for (int r0 = 0; r0 < R; r0 += kGsRed) {
        for (int e = threadIdx.x; e < kGsRed * kGsTile; e += 256) {
            const int rr = e % kGsRed, i = e / kGsRed;
            const int m = row0 + i, r = r0 + rr;
            xs[rr][i] = (m < a.M && r < R) ? bf16_bits_to_float(a.A[static_cast<size_t>(m) * R + r]) : 0.f;
            // weight (n, k) for output column col0 + i and reduction index r
            const int n = TR ? r : col0 + i, k = TR ? col0 + i : r;
            float w = 0.f;
            if (n < a.N && k < a.K) {
                const uint32_t word = __ldg(a.packed + static_cast<size_t>(n) * W8 + k / 8);
                const int grp = a.G == 1 ? 0 : k / a.g;
                const bool mbf = (a.fmt & kFmtMetaBf16) != 0;
                const float s = meta_to_float(a.S[static_cast<size_t>(n) * a.sz_row + grp], mbf);
                const float z = meta_to_float(a.Z[static_cast<size_t>(n) * a.sz_row + grp], mbf);
                w = (static_cast<float>((word >> (4 * (k & 7))) & 0xFu) - z) * s;
            }
            ws[rr][i] = w;
        }
        __syncthreads();
#pragma unroll 8
        for (int rr = 0; rr < kGsRed; ++rr) {
            float xv[4], wv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) xv[i] = xs[rr][ty + 16 * i];
#pragma unroll
            for (int j = 0; j < 4; ++j) wv[j] = ws[rr][tx + 16 * j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(xv[i], wv[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int m = row0 + ty + 16 * i, c = col0 + tx + 16 * j;
            if (m < a.M && c < L) {
                float v = acc[i][j];
                if (a.bias) v += bf16_bits_to_float(a.bias[c]);
                a.Y[static_cast<size_t>(m) * L + c] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
            }
        }
}

}  // namespace w4
