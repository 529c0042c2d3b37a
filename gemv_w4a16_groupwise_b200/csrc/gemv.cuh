// CUDA-core pieces of the small-batch (M <= 4) W4A16 products: the kernels
// that cover what the tensor-pipe GEMV kernels do not take, and the split
// finalize they share:
//
//  * gemv_fwd_simple_kernel: the forward product for shapes the streaming
//    kernels do not take (K or the group length not a multiple of 32): one
//    warp per output row, lanes along K, plain fp32 arithmetic;
//  * splits_finalize_kernel, splits_finalize_vec4_kernel: add the fp32
//    partials of a split reduction (and the bias) in a fixed order;
//  * gemv_t_kernel: the transposed product dX = dY . dequant(W) for M <= 4
//    on shapes the tensor-pipe kernel does not take.
//
// The forward GEMV proper is in gemv_q8.cuh and gemv_mma.cuh (tensor pipe);
// the transposed one in gemv_t_mma.cuh.
#pragma once

#include "tma.cuh"

namespace w4 {

// Arguments of gemv_fwd_simple_kernel.
struct GemvFwdArgs {
    const uint16_t* X;       // [M, K] bf16
    const __half* S;         // scales
    const __half* Z;         // zeros
    const uint16_t* bias;    // [N] bf16 or nullptr
    uint16_t* Y;             // [M, N] bf16
    int N, K, g, G, sz_row;  // group of (n, k): n * sz_row + min(k / g, G - 1)
    int fmt;                 // format flags: kFmtZeroFloat, kFmtMetaBf16
};

// A scale or zero (fp16 or bf16 bits) through the read-only cache.
__device__ __forceinline__ float meta_ldg(const __half* p, bool bf16) {
    return meta_to_float(__ldg(reinterpret_cast<const unsigned short*>(p)), bf16);
}


// Finalize a split reduction: out[m, l] = bf16(sum_s partial[s, m, l] + bias[l]).
// A block takes 64 consecutive outputs; thread (q, o) adds slices q, q + 4,
// q + 8, ... of output o in ascending order (independent loads, so many are
// in flight), and the four partial sums are then added in the order
// q = 0, 1, 2, 3: a fixed order, so the result does not depend on timing.
constexpr int kFinOut = 64;
__global__ void __launch_bounds__(256) splits_finalize_kernel(const float* __restrict__ partial,
                                                              int splits, int M, int L,
                                                              const uint16_t* __restrict__ bias,
                                                              uint16_t* __restrict__ out) {
    pdl_wait();   // when launched as a programmatic dependent of the split kernel
    __shared__ float red[4][kFinOut];
    const long long total = static_cast<long long>(M) * L;
    const int o = threadIdx.x % kFinOut, q = threadIdx.x / kFinOut;
    for (long long b0 = static_cast<long long>(blockIdx.x) * kFinOut; b0 < total;
         b0 += static_cast<long long>(gridDim.x) * kFinOut) {
        const long long idx = b0 + o;
        float s = 0.0f;
        if (idx < total) {
#pragma unroll 4
            for (int sp = q; sp < splits; sp += 4) s += __ldg(partial + static_cast<long long>(sp) * total + idx);
        }
        red[q][o] = s;
        __syncthreads();
        if (q == 0 && idx < total) {
            float v = ((red[0][o] + red[1][o]) + red[2][o]) + red[3][o];
            const int l = static_cast<int>(idx % L);
            if (bias) v += bf16_bits_to_float(bias[l]);
            out[idx] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
        }
        __syncthreads();
    }
}

// The same sum for L a multiple of 4, four outputs per thread: a block
// takes 64 consecutive outputs (16 float4 columns); thread (q, c) adds
// slices q, q + 16, q + 32, ... of column c in ascending order.  Its loads
// go out together, eight at a time (indices past the last slice are clamped
// to it, so every load is unconditional, and those values are dropped); the
// sixteen partial sums are then added in the order q = 0 .. 15.
constexpr int kFin4Cols = 16;
constexpr int kFin4Q = 16;
__global__ void __launch_bounds__(256) splits_finalize_vec4_kernel(const float* __restrict__ partial,
                                                                   int splits, int M, int L,
                                                                   const uint16_t* __restrict__ bias,
                                                                   uint16_t* __restrict__ out) {
    pdl_wait();   // when launched as a programmatic dependent of the split kernel
    __shared__ float4 red[kFin4Q][kFin4Cols];
    const long long total4 = static_cast<long long>(M) * L / 4;
    const int c = threadIdx.x % kFin4Cols, q = threadIdx.x / kFin4Cols;
    const float4* p4 = reinterpret_cast<const float4*>(partial);
    for (long long b0 = static_cast<long long>(blockIdx.x) * kFin4Cols; b0 < total4;
         b0 += static_cast<long long>(gridDim.x) * kFin4Cols) {
        const long long idx = min(b0 + c, total4 - 1);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int sp0 = q; sp0 < splits; sp0 += kFin4Q * 8) {
            float4 v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j)
                v[j] = __ldg(p4 + static_cast<long long>(min(sp0 + kFin4Q * j, splits - 1)) * total4 + idx);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (sp0 + kFin4Q * j < splits) {
                    acc.x += v[j].x;
                    acc.y += v[j].y;
                    acc.z += v[j].z;
                    acc.w += v[j].w;
                }
        }
        red[q][c] = acc;
        __syncthreads();
        if (q == 0 && b0 + c < total4) {
            float r[4] = {red[0][c].x, red[0][c].y, red[0][c].z, red[0][c].w};
#pragma unroll
            for (int i = 1; i < kFin4Q; ++i) {
                r[0] += red[i][c].x;
                r[1] += red[i][c].y;
                r[2] += red[i][c].z;
                r[3] += red[i][c].w;
            }
            const int l = static_cast<int>((idx * 4) % L);
            if (bias) {
#pragma unroll
                for (int e = 0; e < 4; ++e) r[e] += bf16_bits_to_float(bias[l + e]);
            }
            uint2 o;
            o.x = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(r[0]))) |
                  (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(r[1]))) << 16);
            o.y = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(r[2]))) |
                  (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(r[3]))) << 16);
            *reinterpret_cast<uint2*>(out + idx * 4) = o;
        }
        __syncthreads();
    }
}

// Plain forward GEMV for shapes the TMA path does not take (K % 32 != 0):
// one warp per row, lanes stride over packed words, per-element dequant.
template <int M>
__global__ void __launch_bounds__(256) gemv_fwd_simple_kernel(const GemvFwdArgs a,
                                                              const uint32_t* __restrict__ packed) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= a.N) return;
    const int n = warp;
    const int W8 = a.K / 8;
    float acc[M];
#pragma unroll
    for (int m = 0; m < M; ++m) acc[m] = 0.0f;
    for (int j = lane; j < W8; j += 32) {
        const uint32_t w = __ldg(packed + static_cast<size_t>(n) * W8 + j);
        const int grp = min((8 * j) / a.g, a.G - 1);
        const bool mbf = (a.fmt & kFmtMetaBf16) != 0;
        const float s = meta_ldg(a.S + n * a.sz_row + grp, mbf);
        const float z = meta_ldg(a.Z + n * a.sz_row + grp, mbf);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float wv = (static_cast<float>((w >> (4 * e)) & 0xF) - z) * s;
#pragma unroll
            for (int m = 0; m < M; ++m)
                acc[m] = fmaf(bf16_bits_to_float(a.X[static_cast<size_t>(m) * a.K + 8 * j + e]), wv, acc[m]);
        }
    }
#pragma unroll
    for (int m = 0; m < M; ++m) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc[m] += __shfl_xor_sync(0xFFFFFFFFu, acc[m], off);
    }
    if (lane == 0) {
#pragma unroll
        for (int m = 0; m < M; ++m) {
            float s = acc[m];
            if (a.bias) s += bf16_bits_to_float(a.bias[n]);
            a.Y[static_cast<size_t>(m) * a.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(s));
        }
    }
}

// ---------------------------------------------------------------------------
// Transposed GEMV: dX[m, k] = sum_n dY[m, n] * w_hat[n, k]  (M <= 4)
// ("Re-write HQQ Fused Gemm Transpose": same packed W, scales and zeros), for
// the shapes the tensor-pipe kernel does not take.  Lanes own two
// consecutive packed words (16 k) of a row, so a warp reads 256 contiguous
// bytes of each row it visits; the 4 warps of a CTA take interleaved rows of
// the CTA's row range and meet in shared memory.  Per code the lane forms
// (q - z) exactly ((2^23 + q) - (2^23 + z) in fp32) and multiplies it by
// c = dY[m, n] s (exact: 8 x 11 significant bits) in an fp32 fma, so every
// product is exact and the sums are fp32.  A fractional zero point takes
// (128 + q) - (128 + z) instead, q - z rounded at most once.  Row ranges are
// split over CTAs; fp32 partials go to the workspace.
// ---------------------------------------------------------------------------
struct GemvTArgs {
    const uint16_t* dY;      // [M, N] bf16
    const uint32_t* packed;  // [N, K/8]
    const __half* S;
    const __half* Z;
    const uint16_t* bias;    // [K] or nullptr
    uint16_t* dX;            // [M, K] bf16
    float* partial;          // [splits, M, K] when splits > 1
    int N, K, g, G, sz_row;
    int rows_per_split, splits;
    int fmt;                 // format flags: kFmtZeroFloat, kFmtMetaBf16
};

constexpr int kGemvTThreads = 128;
constexpr int kGemvTWordsPerCta = 64;  // 32 lanes x 2 words = 512 k

template <int M>
__global__ void __launch_bounds__(kGemvTThreads)
    gemv_t_kernel(const GemvTArgs a) {
    __shared__ float red[kGemvTThreads / 32][M][16][32 + 1];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int W8 = a.K / 8;
    const int j0 = blockIdx.x * kGemvTWordsPerCta + 2 * lane;  // first word of this lane
    const int split = blockIdx.y;
    const int r0 = split * a.rows_per_split;
    const int r1 = min(a.N, r0 + a.rows_per_split);
    const bool has0 = j0 < W8, has1 = (j0 + 1) < W8;
    const int grp0 = has0 ? min((8 * j0) / a.g, a.G - 1) : 0;
    const int grp1 = has1 ? min((8 * (j0 + 1)) / a.g, a.G - 1) : 0;

    float acc[M][16];
#pragma unroll
    for (int m = 0; m < M; ++m)
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[m][e] = 0.0f;

    for (int n = r0 + warp; n < r1; n += kGemvTThreads / 32) {
        const uint32_t* rowp = a.packed + static_cast<size_t>(n) * W8;
        const uint32_t w[2] = {has0 ? ldg_stream_u32(rowp + j0) : 0u, has1 ? ldg_stream_u32(rowp + j0 + 1) : 0u};
        const bool mbf = (a.fmt & kFmtMetaBf16) != 0;
        const float s[2] = {meta_ldg(a.S + n * a.sz_row + grp0, mbf), meta_ldg(a.S + n * a.sz_row + grp1, mbf)};
        // off + z, so that (off + q) - (off + z) = q - z: off = 2^23 for an
        // integer z (exact), 128 for a fractional one (exact unless z has
        // bits below 2^-16)
        const float off = (a.fmt & kFmtZeroFloat) ? 128.0f : 8388608.0f;
        const uint32_t ob = (a.fmt & kFmtZeroFloat) ? 0x43000000u : 0x4B000000u;
        const int qsh = (a.fmt & kFmtZeroFloat) ? 16 : 0;     // code position in (off + q)
        const float zo[2] = {off + meta_ldg(a.Z + n * a.sz_row + grp0, mbf),
                             off + meta_ldg(a.Z + n * a.sz_row + grp1, mbf)};
        float qz[16];
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int e = 0; e < 8; ++e)
                qz[8 * h + e] = __uint_as_float(ob | (((w[h] >> (4 * e)) & 0xFu) << qsh)) - zo[h];
#pragma unroll
        for (int m = 0; m < M; ++m) {
            const float d = bf16_bits_to_float(__ldg(a.dY + static_cast<size_t>(m) * a.N + n));
            const float c[2] = {d * s[0], d * s[1]};
#pragma unroll
            for (int e = 0; e < 16; ++e) acc[m][e] = fmaf(c[e >> 3], qz[e], acc[m][e]);
        }
    }

#pragma unroll
    for (int m = 0; m < M; ++m)
#pragma unroll
        for (int e = 0; e < 16; ++e) red[warp][m][e][lane] = acc[m][e];
    __syncthreads();
    // the warps' sums in warp order; lanes cover the 16 k of one lane-slot
    for (int o = threadIdx.x; o < M * 16 * 32; o += kGemvTThreads) {
        const int m = o / (16 * 32);
        const int rem = o - m * 16 * 32;
        const int ln = rem / 16, kk = rem % 16;
        float s = 0.0f;
#pragma unroll
        for (int w = 0; w < kGemvTThreads / 32; ++w) s += red[w][m][kk][ln];
        const int j = blockIdx.x * kGemvTWordsPerCta + 2 * ln + kk / 8;
        if (j < W8) {
            const int k = 8 * j + (kk & 7);
            if (a.splits == 1) {
                if (a.bias) s += bf16_bits_to_float(a.bias[k]);
                a.dX[static_cast<size_t>(m) * a.K + k] = __bfloat16_as_ushort(__float2bfloat16_rn(s));
            } else {
                a.partial[(static_cast<size_t>(split) * M + m) * a.K + k] = s;
            }
        }
    }
}

}  // namespace w4
