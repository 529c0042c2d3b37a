// Small-batch (M <= 4) W4A16 GEMV on CUDA cores.
//
// The decode-time product Y[m, n] = sum_k X[m, k] * w_hat[n, k] is bound by
// streaming the packed weights from HBM (TensorRT-LLM "Modify
// small-batched weight only quantization": small-batch weight-only GEMV
// suffers global-memory load stalls; scale/zero loads are deduplicated and
// copies are double buffered).  The B200 design here:
//
//  * One lane owns whole weight rows (4 rows, stride 32), so each lane
//    finishes its dot products alone and the activations it multiplies are
//    the same for all 32 lanes: they are read from shared memory as
//    warp-uniform broadcasts, which costs one wavefront per load.
//  * Packed weights arrive by TMA in boxes of 128 rows x 64 bytes (128 k),
//    64-byte swizzled so that 32 lanes reading 32 different rows hit
//    different banks; a 16-stage mbarrier ring keeps up to 128 KB per SM in
//    flight.
//  * The 8 consumer warps of a CTA split the K slice box by box: box i (in
//    the CTA's global box order) goes to warp i % 8 and stage i % 16, so
//    every stage has exactly one consumer that takes its uses in order (a
//    parity wait can then never mistake an old phase for the awaited one).
//    Their partial sums meet in shared memory once per 128-row tile.
//  * Dequantization in registers: each code lands in the mantissa of an
//    fp32 "magic" value (2048 + q or 128 + q) with one lop3, and packed
//    f32x2 FMAs multiply two codes at a time.  The scale and zero point are
//    applied once per fold granule F (a run of k inside one group):
//        sum_k (q_k - z) s x_k = s * (sum_k (off_k + q_k) x_k - O - z X)
//    where O = sum off_k x_k and X = sum x_k are computed once per CTA
//    when the activations are staged.
//  * Persistent CTAs (one per SM) walk a contiguous range of (K slice,
//    row tile) units; the activation slice is staged once per K slice.
//    When K is split, fp32 partials go to the caller's workspace and a
//    finalize kernel adds the slices (and the bias) in a fixed order.
#pragma once

#include "tma.cuh"

namespace w4 {

constexpr int kGemvConsumerWarps = 8;
constexpr int kGemvThreads = (kGemvConsumerWarps + 1) * 32;
constexpr int kGemvTileRows = 128;
constexpr int kGemvBoxK = 128;
constexpr int kGemvBoxWords = kGemvBoxK / 8;
constexpr int kGemvBoxBytes = kGemvTileRows * (kGemvBoxK / 2);
constexpr int kGemvStages = 2 * kGemvConsumerWarps;

// Position of element e (k % 8) of a word inside its 8-float activation
// record: pairs (x3,x4) (x5,x6) (x1,x2) (x0,x7) match the magic-value pairs.
__host__ __device__ constexpr int gemv_pair_pos(int e) { return (0x73210546 >> (4 * e)) & 7; }

struct GemvFwdArgs {
    const uint16_t* X;       // [M, K] bf16
    const __half* S;         // scales
    const __half* Z;         // zeros
    const uint16_t* bias;    // [N] bf16 or nullptr
    uint16_t* Y;             // [M, N] bf16
    float* partial;          // [splits, M, N] fp32 when splits > 1
    int N, K, g, G, sz_row;  // group of (n, k): n * sz_row + min(k / g, G - 1)
    int TK, splits, row_tiles, units;
};

__host__ __device__ inline size_t gemv_fwd_smem_bytes(int M, int TK, int F) {
    size_t b = 1024;                                        // alignment slack
    b += static_cast<size_t>(kGemvStages) * kGemvBoxBytes;  // weight ring
    b += static_cast<size_t>(M) * TK * 4;                   // activations (fp32)
    b += 2ull * M * (TK / F) * 4;                           // O and X per granule
    b += static_cast<size_t>(kGemvConsumerWarps) * M * kGemvTileRows * 4;  // reduction
    b += 2ull * kGemvStages * 8 + 16;                       // barriers + flag
    return b;
}

__device__ __forceinline__ float half_to_float_ldg(const __half* p) {
    return __half2float(__ldg(p));
}

template <int M, int F>
__global__ void __launch_bounds__(kGemvThreads, 1)
    gemv_fwd_tma_kernel(const __grid_constant__ CUtensorMap wmap, const GemvFwdArgs a) {
    static_assert(M >= 1 && M <= 4, "M");
    static_assert(F >= 32 && F <= kGemvBoxK && (kGemvBoxK % F) == 0, "F");
    constexpr int FW = F / 8;                // words per granule
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* ring = base;
    float* xs = reinterpret_cast<float*>(ring + kGemvStages * kGemvBoxBytes);
    const int ngran = a.TK / F;
    float* osum = xs + M * a.TK;
    float* xsum = osum + M * ngran;
    float* red = xsum + M * ngran;
    uint64_t* full = reinterpret_cast<uint64_t*>(red + kGemvConsumerWarps * M * kGemvTileRows);
    uint64_t* empty = full + kGemvStages;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kGemvStages);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kGemvStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);  // each box is consumed by exactly one warp
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();

    const long long C = gridDim.x;
    const int u_begin = static_cast<int>(blockIdx.x * static_cast<long long>(a.units) / C);
    const int u_end = static_cast<int>((blockIdx.x + 1) * static_cast<long long>(a.units) / C);
    auto boxes_of = [&](int slice) {
        const int len = min(a.TK, a.K - slice * a.TK);
        return (len + kGemvBoxK - 1) / kGemvBoxK;
    };

    if (warp == kGemvConsumerWarps) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            tma_prefetch_desc(&wmap);
            int it = 0;
            for (int u = u_begin; u < u_end && !*abort_flag; ++u) {
                const int slice = u / a.row_tiles, tile = u - slice * a.row_tiles;
                const int nb = boxes_of(slice);
                for (int b = 0; b < nb; ++b, ++it) {
                    const int st = it % kGemvStages;
                    const uint32_t use = static_cast<uint32_t>(it / kGemvStages);
                    if (use > 0 &&
                        !mbar_wait_bounded(&empty[st], (use - 1) & 1u, abort_flag, kErrTimeoutEmpty))
                        break;
                    mbar_arrive_expect_tx(&full[st], kGemvBoxBytes);
                    tma_load_2d(ring + st * kGemvBoxBytes, &wmap,
                                (slice * a.TK + b * kGemvBoxK) / 8, tile * kGemvTileRows, &full[st]);
                }
            }
            if (*abort_flag) {
                // let copies already issued land before the CTA can exit
                const unsigned long long t0 = global_timer_ns();
                while (global_timer_ns() - t0 < 1000000ull) {
                }
            }
        }
        return;
    }

    // ---------------- consumers ----------------
    const int tid = threadIdx.x;  // 0 .. 255
    int it = 0;
    int cur_slice = -1;
    for (int u = u_begin; u < u_end; ++u) {
        const int slice = u / a.row_tiles, tile = u - slice * a.row_tiles;
        const int nb = boxes_of(slice);
        const int k_slice = slice * a.TK;
        if (slice != cur_slice) {
            // stage the activation slice in pair order, zero past K
            const int len = min(a.TK, a.K - k_slice);
            for (int idx = tid; idx < M * a.TK; idx += 256) {
                const int m = idx / a.TK, kk = idx - m * a.TK;
                float v = 0.0f;
                if (kk < len) v = bf16_bits_to_float(a.X[static_cast<size_t>(m) * a.K + k_slice + kk]);
                xs[m * a.TK + (kk & ~7) + gemv_pair_pos(kk & 7)] = v;
            }
            named_barrier_sync(1, 256);
            // per-granule sums O = sum off_k x_k and X = sum x_k from the staged
            // copy: one warp per granule, lanes stride over its F values, fixed
            // shuffle tree (deterministic)
            for (int gidx = warp; gidx < M * ngran; gidx += kGemvConsumerWarps) {
                const int m = gidx / ngran, gi = gidx - m * ngran;
                float o = 0.0f, xsm = 0.0f;
                for (int e = lane; e < F; e += 32) {
                    const int kk = gi * F + e;
                    const float v = xs[m * a.TK + (kk & ~7) + gemv_pair_pos(kk & 7)];
                    o = fmaf((kk & 1) ? 2048.0f : 128.0f, v, o);
                    xsm += v;
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    o += __shfl_xor_sync(0xFFFFFFFFu, o, off);
                    xsm += __shfl_xor_sync(0xFFFFFFFFu, xsm, off);
                }
                if (lane == 0) {
                    osum[gidx] = o;
                    xsum[gidx] = xsm;
                }
            }
            named_barrier_sync(1, 256);
            cur_slice = slice;
        }

        float y[4][M];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int m = 0; m < M; ++m) y[i][m] = 0.0f;

        // s / z index base per row (clamped to a valid row)
        int szbase[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int n = min(tile * kGemvTileRows + lane + 32 * i, a.N - 1);
            szbase[i] = n * a.sz_row;
        }

        const int b_first = ((warp - it) % kGemvConsumerWarps + kGemvConsumerWarps) % kGemvConsumerWarps;
        for (int b = b_first; b < nb; b += kGemvConsumerWarps) {
            const int bit = it + b;  // global box index: bit % 8 == warp
            const int st = bit % kGemvStages;
            const uint32_t par = static_cast<uint32_t>(bit / kGemvStages) & 1u;
            const int kbox = k_slice + b * kGemvBoxK;  // global k of the box

            const bool ok = __all_sync(0xFFFFFFFFu,
                                       mbar_wait_bounded(&full[st], par, abort_flag, kErrTimeoutTmaFull));
            if (!ok) continue;
            const uint8_t* sb = ring + st * kGemvBoxBytes;
            const float* xbox = xs + b * kGemvBoxK;
            const int gbox = (b * kGemvBoxK) / F;  // granule index of the box start

            float2 acc[4][M];
            float sv[4], zv[4];
#pragma unroll
            for (int c = 0; c < kGemvBoxWords / 4; ++c) {
                uint4 wv[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    // 64-byte TMA swizzle: 16-byte chunk c of row r sits at c ^ ((r >> 1) & 3)
                    const int row = lane + 32 * i;
                    wv[i] = *reinterpret_cast<const uint4*>(sb + row * (kGemvBoxK / 2) +
                                                            ((c ^ ((lane >> 1) & 3)) << 4));
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int wb = c * 4 + j;  // word within box
                    const int gi = wb / FW;
                    if (wb % FW == 0) {
                        // scale / zero of this granule for the 4 rows; used at its end
                        const int grp = min((kbox + gi * F) / a.g, a.G - 1);
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            sv[i] = half_to_float_ldg(a.S + szbase[i] + grp);
                            zv[i] = half_to_float_ldg(a.Z + szbase[i] + grp);
                        }
#pragma unroll
                        for (int m = 0; m < M; ++m) {
                            const float o = osum[m * ngran + gbox + gi];
#pragma unroll
                            for (int i = 0; i < 4; ++i) acc[i][m] = make_float2(-o, 0.0f);
                        }
                    }
                    float2 xp[M][4];
#pragma unroll
                    for (int m = 0; m < M; ++m) {
                        const float4 xa = *reinterpret_cast<const float4*>(xbox + m * a.TK + wb * 8);
                        const float4 xb =
                            *reinterpret_cast<const float4*>(xbox + m * a.TK + wb * 8 + 4);
                        xp[m][0] = make_float2(xa.x, xa.y);
                        xp[m][1] = make_float2(xa.z, xa.w);
                        xp[m][2] = make_float2(xb.x, xb.y);
                        xp[m][3] = make_float2(xb.z, xb.w);
                    }
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const uint32_t w = (j == 0) ? wv[i].x : (j == 1) ? wv[i].y : (j == 2) ? wv[i].z : wv[i].w;
                        const uint32_t r8 = w >> 8, l8 = w << 8;
                        const float2 p0 = make_float2(__uint_as_float(lop3_and_or(w, 0xF000u, 0x45000000u)),
                                                      __uint_as_float(lop3_and_or(w, 0xF0000u, 0x43000000u)));
                        const float2 p1 = make_float2(__uint_as_float(lop3_and_or(r8, 0xF000u, 0x45000000u)),
                                                      __uint_as_float(lop3_and_or(r8, 0xF0000u, 0x43000000u)));
                        const float2 p2 = make_float2(__uint_as_float(lop3_and_or(l8, 0xF000u, 0x45000000u)),
                                                      __uint_as_float(lop3_and_or(l8, 0xF0000u, 0x43000000u)));
                        const float2 p3 =
                            make_float2(__uint_as_float(lop3_and_or(w << 16, 0xF0000u, 0x43000000u)),
                                        __uint_as_float(lop3_and_or(w >> 16, 0xF000u, 0x45000000u)));
#pragma unroll
                        for (int m = 0; m < M; ++m) {
                            acc[i][m] = ffma2(p0, xp[m][0], acc[i][m]);
                            acc[i][m] = ffma2(p1, xp[m][1], acc[i][m]);
                            acc[i][m] = ffma2(p2, xp[m][2], acc[i][m]);
                            acc[i][m] = ffma2(p3, xp[m][3], acc[i][m]);
                        }
                    }
                    if ((wb + 1) % FW == 0) {
#pragma unroll
                        for (int m = 0; m < M; ++m) {
                            const float xg = xsum[m * ngran + gbox + gi];
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const float part = acc[i][m].x + acc[i][m].y;
                                const float t = fmaf(-zv[i], xg, part);
                                y[i][m] = fmaf(sv[i], t, y[i][m]);
                            }
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
        }
        it += nb;

        // combine the 8 warps' partial sums for this tile
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int m = 0; m < M; ++m) red[(warp * M + m) * kGemvTileRows + lane + 32 * i] = y[i][m];
        named_barrier_sync(1, 256);
        for (int o = tid; o < M * kGemvTileRows; o += 256) {
            const int m = o / kGemvTileRows, r = o - m * kGemvTileRows;
            float s = 0.0f;
#pragma unroll
            for (int w = 0; w < kGemvConsumerWarps; ++w) s += red[(w * M + m) * kGemvTileRows + r];
            const int n = tile * kGemvTileRows + r;
            if (n < a.N) {
                if (a.splits == 1) {
                    if (a.bias) s += bf16_bits_to_float(a.bias[n]);
                    a.Y[static_cast<size_t>(m) * a.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(s));
                } else {
                    a.partial[(static_cast<size_t>(slice) * M + m) * a.N + n] = s;
                }
            }
        }
        named_barrier_sync(1, 256);
    }
}

// Finalize a split reduction: out[m, l] = bf16(sum_s partial[s, m, l] + bias[l]),
// slices added in ascending order.
__global__ void __launch_bounds__(256) splits_finalize_kernel(const float* __restrict__ partial,
                                                              int splits, int M, int L,
                                                              const uint16_t* __restrict__ bias,
                                                              uint16_t* __restrict__ out) {
    const long long total = static_cast<long long>(M) * L;
    for (long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
         idx += static_cast<long long>(gridDim.x) * blockDim.x) {
        float s = 0.0f;
        for (int sp = 0; sp < splits; ++sp) s += partial[static_cast<long long>(sp) * total + idx];
        const int l = static_cast<int>(idx % L);
        if (bias) s += bf16_bits_to_float(bias[l]);
        out[idx] = __bfloat16_as_ushort(__float2bfloat16_rn(s));
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
        const float s = half_to_float_ldg(a.S + n * a.sz_row + grp);
        const float z = half_to_float_ldg(a.Z + n * a.sz_row + grp);
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
// ("Re-write HQQ Fused Gemm Transpose": same packed W, scales and zeros).
// Lanes own two consecutive packed words (16 k) of a row, so a warp reads
// 256 contiguous bytes of each row it visits; the 8 warps of a CTA take
// interleaved rows of the CTA's row range and meet in shared memory.  With
// c = dY[m, n] * s:   sum_n c (q - z) = sum_n c (off + q) - sum_n c (off + z)
// so per word only sum_n c and sum_n c z are kept besides the 16 products.
// Row ranges are split over CTAs; fp32 partials go to the workspace.
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
    float csum[M][2], czsum[M][2];
#pragma unroll
    for (int m = 0; m < M; ++m) {
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[m][e] = 0.0f;
        csum[m][0] = csum[m][1] = czsum[m][0] = czsum[m][1] = 0.0f;
    }

    for (int n = r0 + warp; n < r1; n += kGemvTThreads / 32) {
        const uint32_t* rowp = a.packed + static_cast<size_t>(n) * W8;
        const uint32_t w0 = has0 ? ldg_stream_u32(rowp + j0) : 0u;
        const uint32_t w1 = has1 ? ldg_stream_u32(rowp + j0 + 1) : 0u;
        const float s0 = half_to_float_ldg(a.S + n * a.sz_row + grp0);
        const float z0 = half_to_float_ldg(a.Z + n * a.sz_row + grp0);
        const float s1 = half_to_float_ldg(a.S + n * a.sz_row + grp1);
        const float z1 = half_to_float_ldg(a.Z + n * a.sz_row + grp1);
#pragma unroll
        for (int m = 0; m < M; ++m) {
            const float d = bf16_bits_to_float(__ldg(a.dY + static_cast<size_t>(m) * a.N + n));
            const float c0 = d * s0, c1 = d * s1;
            csum[m][0] += c0;
            csum[m][1] += c1;
            czsum[m][0] = fmaf(c0, z0, czsum[m][0]);
            czsum[m][1] = fmaf(c1, z1, czsum[m][1]);
            const float2 cc0 = make_float2(c0, c0), cc1 = make_float2(c1, c1);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t w = h ? w1 : w0;
                const float2 cc = h ? cc1 : cc0;
                const uint32_t r8 = w >> 8, l8 = w << 8;
                // (q3,q4) (q5,q6) (q1,q2) (q0,q7) as (off + q) magic pairs
                const float2 p0 = make_float2(__uint_as_float(lop3_and_or(w, 0xF000u, 0x45000000u)),
                                              __uint_as_float(lop3_and_or(w, 0xF0000u, 0x43000000u)));
                const float2 p1 = make_float2(__uint_as_float(lop3_and_or(r8, 0xF000u, 0x45000000u)),
                                              __uint_as_float(lop3_and_or(r8, 0xF0000u, 0x43000000u)));
                const float2 p2 = make_float2(__uint_as_float(lop3_and_or(l8, 0xF000u, 0x45000000u)),
                                              __uint_as_float(lop3_and_or(l8, 0xF0000u, 0x43000000u)));
                const float2 p3 =
                    make_float2(__uint_as_float(lop3_and_or(w << 16, 0xF0000u, 0x43000000u)),
                                __uint_as_float(lop3_and_or(w >> 16, 0xF000u, 0x45000000u)));
                float2* A = reinterpret_cast<float2*>(&acc[m][8 * h]);
                A[0] = ffma2(p0, cc, A[0]);  // k3, k4
                A[1] = ffma2(p1, cc, A[1]);  // k5, k6
                A[2] = ffma2(p2, cc, A[2]);  // k1, k2
                A[3] = ffma2(p3, cc, A[3]);  // k0, k7
            }
        }
    }

    // slot order inside acc[m][8h + slot]: k3,k4,k5,k6,k1,k2,k0,k7 ; offsets
    // 2048 for odd k, 128 for even k
#pragma unroll
    for (int m = 0; m < M; ++m)
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int slot = 0; slot < 8; ++slot) {
                const int e = (0x70216543 >> (4 * slot)) & 7;  // k offset of the slot
                const float off = (e & 1) ? 2048.0f : 128.0f;
                const float v = acc[m][8 * h + slot] - fmaf(off, csum[m][h], czsum[m][h]);
                red[warp][m][8 * h + e][lane] = v;
            }
    __syncthreads();
    // warps 0..M-1 each finish one m; lanes cover the 16 k of one lane-slot
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
