// Transposed GEMV for M <= 4 (the fine-tuning backward from the same packed
// tensors, "Re-write HQQ Fused Gemm Transpose": dX = dY . dequant(W), no
// repack, no reshaped scales or zeros):
//     dX[m, k] = sum_n dY[m, n] * s[n, g(k)] * (q[n, k] - z[n, g(k)]).
//
// The reduction runs over the weight rows, which the packed layout keeps
// apart (rows are contiguous along K), so each CTA owns a strip of 2048 k
// (one box width) and walks a range of rows:
//   * a producer warp streams 4-row x 1 KB boxes of the strip (and the
//     rows' scale / zero boxes) through a CTA-wide
//     ring; a stage is refilled once all 8 consumer warps released it;
//   * consumer warp w owns k = 256 w .. 256 w + 255 of the strip, lane l
//     one packed word (8 k, inside one group) of it;
//   * per row n the lane forms c = dY[m, n] * s[n, g] and adds
//     c * (off + q) for its 8 codes with the magic-number unpack (one lop3
//     turns a code into the fp32 value off + q, off = 128 or 2048) and
//     paired FMAs, while it also keeps sum_n c and sum_n c * z; at the end
//         dX = sum c (off + q) - off * sum c - sum c z
//     gives sum c (q - z) for every k of the lane.
// Row ranges are split over CTAs so the grid covers the SMs; the fp32
// partials of the splits are added (with the bias) by
// splits_finalize_kernel in a fixed order.
#pragma once

#include "gemv_mma.cuh"

namespace w4 {

constexpr int kTSW = 8;          // consumer warps per CTA
constexpr int kTSThreads = (kTSW + 1) * 32;
constexpr int kTSStrip = kSBK;   // k per CTA strip (one box width)

struct GemvTStreamArgs {
    const uint16_t* dY;      // [M, N] bf16
    const __half* S;
    const __half* Z;
    const uint16_t* bias;    // [K] bf16 or nullptr
    uint16_t* dX;            // [M, K] bf16
    float* partial;          // [splits, M, K] when splits > 1
    int N, K, g, G, sz_row;
    int strips;              // ceil(K / 2048)
    int splits;              // row ranges
    int rows_per_split;      // a multiple of 4
    int stages;
};

// A stage: one 4-row x 1 KB box of packed words, then the S and Z boxes
// (4 rows x 16 groups each, or the 8 rows' values around the box with one
// group per row), each starting on a 128-byte boundary.
__host__ __device__ inline int gemv_t_stage_bytes(int sz) {
    return (kSBBytes + (sz == kSzTma2d ? 2 * 128 : sz == kSzTma1d ? 128 + 16 : 0) + 127) / 128 * 128;
}

// Ring, barriers, and dY of the CTA's rows as one float4 per row.
__host__ __device__ inline size_t gemv_t_stream_smem_bytes(int stages, int sz, int rows_per_split) {
    return 1024 + static_cast<size_t>(stages) * gemv_t_stage_bytes(sz) + static_cast<size_t>(stages) * 16 + 16 +
           static_cast<size_t>(rows_per_split) * 16;
}

template <int M, int GK, int SZ>
__global__ void __launch_bounds__(kTSThreads, 1)
    gemv_t_stream_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap smap,
                         const __grid_constant__ CUtensorMap zmap, const GemvTStreamArgs a) {
    static_assert(M >= 1 && M <= 4, "M");
    static_assert(SZ == kSzConst || SZ == kSzTma2d || SZ == kSzTma1d, "scale / zero path");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int NS = a.stages;
    const int SB = gemv_t_stage_bytes(SZ);
    constexpr int kSzTx = SZ == kSzTma2d ? 2 * kSR * 16 * 2 : SZ == kSzTma1d ? 2 * 8 * 2 : 0;
    uint8_t* ring = base;                                                    // [stage][SB]
    uint64_t* full = reinterpret_cast<uint64_t*>(ring + NS * SB);
    uint64_t* empty = full + NS;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + NS);
    float4* dys = reinterpret_cast<float4*>(reinterpret_cast<uint8_t*>(empty + NS) + 16);   // [row of the split] (dY[0..3][n])
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const int strip = blockIdx.x % a.strips, split = blockIdx.x / a.strips;
    const int k0 = strip * kTSStrip;
    const int r0 = split * a.rows_per_split;
    const int r1 = min(a.N, r0 + a.rows_per_split);
    const int nboxes = r1 > r0 ? (r1 - r0 + kSR - 1) / kSR : 0;
    int gshift = 0;
    if (GK == kGroupsPow2) gshift = __ffs(a.g) - 1;
    auto group_of = [&](int k) {
        if (GK == kGroupsOne) return 0;
        if (GK == kGroupsPow2) return k >> gshift;
        return k / a.g;
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kTSW);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (threadIdx.x == kTSW * 32) {
        tma_prefetch_desc(&wmap);
        if (SZ != kSzConst) {
            tma_prefetch_desc(&smap);
            tma_prefetch_desc(&zmap);
        }
    }
    // dY of this split's rows, transposed to one float4 per row (rows past
    // r1 and absent m read as 0, so rows a box carries past r1 add nothing)
    for (int r = threadIdx.x; r < nboxes * kSR; r += kTSThreads) {
        const int n = r0 + r;
        float v[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int m = 0; m < M; ++m)
            if (n < r1) v[m] = bf16_bits_to_float(__ldg(a.dY + static_cast<size_t>(m) * a.N + n));
        dys[r] = make_float4(v[0], v[1], v[2], v[3]);
    }
    __syncthreads();

    if (warp == kTSW) {
        // ------------------------------------------------ producer
        const int x_sz = group_of(k0) & ~7;
        for (int b = 0; b < nboxes; ++b) {
            const int s = b % NS;
            if (b >= NS) {
                const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&empty[s], ((b / NS) - 1) & 1u,
                                                                          abort_flag, kErrTimeoutEmpty));
                if (!ok) break;
            }
            uint8_t* sd = ring + s * SB;
            const int row0 = r0 + b * kSR;
            if (SZ == kSzTma2d)
                tma_issue_elected<3>(&full[s], kSBBytes + kSzTx, sd, &wmap, k0 / 8, row0, sd + kSBBytes, &smap, x_sz,
                                     row0, sd + kSBBytes + 128, &zmap, x_sz, row0);
            else if (SZ == kSzTma1d)
                tma_issue_elected<3>(&full[s], kSBBytes + kSzTx, sd, &wmap, k0 / 8, row0, sd + kSBBytes, &smap,
                                     row0 & ~7, 0, sd + kSBBytes + 128, &zmap, row0 & ~7, 0);
            else
                tma_issue_elected<1>(&full[s], kSBBytes, sd, &wmap, k0 / 8, row0);
        }
    } else {
        // ------------------------------------------------ consumers
        const int wi = warp * 32 + lane;                 // word of the strip
        const int k_lane = k0 + 8 * wi;
        const bool valid = k_lane < a.K;
        const int grp = min(group_of(k_lane), a.G - 1);
        const int x_sz = group_of(k0) & ~7;
        const int sz_off = grp - x_sz;                   // 2-D boxes: the lane's group in the S / Z box
        float s_const = 0.f, z_const = 0.f;
        if (SZ == kSzConst) {
            s_const = __half2float(a.S[0]);
            z_const = __half2float(a.Z[0]);
        }
        float acc[M][8];
#pragma unroll
        for (int m = 0; m < M; ++m)
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[m][e] = 0.0f;
        // sum_n c and sum_n c z for m pairs (0,1) and (2,3), as packed f32x2
        float2 csum2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        float2 czsum2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        const float2 zero2 = make_float2(0.f, 0.f), one2 = make_float2(1.f, 1.f);
        for (int b = 0; b < nboxes; ++b) {
            const int s = b % NS;
            const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&full[s], (b / NS) & 1u, abort_flag,
                                                                      kErrTimeoutTmaFull));
            if (!ok) break;
            const uint8_t* sb = ring + s * SB;
            const __half* sh = reinterpret_cast<const __half*>(sb + kSBBytes);
            const int row0 = r0 + b * kSR;
#pragma unroll
            for (int i = 0; i < kSR; ++i) {
                const uint32_t w = valid ? *reinterpret_cast<const uint32_t*>(sb + i * 1024 + wi * 4) : 0u;
                const float4 d4 = dys[b * kSR + i];
                float sv, zv;
                if (SZ == kSzConst) {
                    sv = s_const;
                    zv = z_const;
                } else if (SZ == kSzTma2d) {
                    sv = __half2float(sh[i * 16 + sz_off]);
                    zv = __half2float(sh[64 + i * 16 + sz_off]);
                } else {
                    sv = __half2float(sh[(row0 & 7) + i]);
                    zv = __half2float(sh[64 + (row0 & 7) + i]);
                }
                const float2 ss = make_float2(sv, sv), zz = make_float2(zv, zv);
                float2 c2[2];
                c2[0] = ffma2(make_float2(d4.x, d4.y), ss, zero2);
                csum2[0] = ffma2(c2[0], one2, csum2[0]);
                czsum2[0] = ffma2(c2[0], zz, czsum2[0]);
                if (M > 2) {
                    c2[1] = ffma2(make_float2(d4.z, d4.w), ss, zero2);
                    csum2[1] = ffma2(c2[1], one2, csum2[1]);
                    czsum2[1] = ffma2(c2[1], zz, czsum2[1]);
                } else {
                    c2[1] = zero2;
                }
                const uint32_t r8 = w >> 8, l8 = w << 8;
                // (q3,q4) (q5,q6) (q1,q2) (q0,q7) as (off + q) magic pairs
                const float2 p0 = make_float2(__uint_as_float(lop3_and_or(w, 0xF000u, 0x45000000u)),
                                              __uint_as_float(lop3_and_or(w, 0xF0000u, 0x43000000u)));
                const float2 p1 = make_float2(__uint_as_float(lop3_and_or(r8, 0xF000u, 0x45000000u)),
                                              __uint_as_float(lop3_and_or(r8, 0xF0000u, 0x43000000u)));
                const float2 p2 = make_float2(__uint_as_float(lop3_and_or(l8, 0xF000u, 0x45000000u)),
                                              __uint_as_float(lop3_and_or(l8, 0xF0000u, 0x43000000u)));
                const float2 p3 = make_float2(__uint_as_float(lop3_and_or(w << 16, 0xF0000u, 0x43000000u)),
                                              __uint_as_float(lop3_and_or(w >> 16, 0xF000u, 0x45000000u)));
#pragma unroll
                for (int m = 0; m < M; ++m) {
                    const float c = (m & 1) ? c2[m >> 1].y : c2[m >> 1].x;
                    const float2 cc = make_float2(c, c);
                    float2* A = reinterpret_cast<float2*>(&acc[m][0]);
                    A[0] = ffma2(p0, cc, A[0]);  // k3, k4
                    A[1] = ffma2(p1, cc, A[1]);  // k5, k6
                    A[2] = ffma2(p2, cc, A[2]);  // k1, k2
                    A[3] = ffma2(p3, cc, A[3]);  // k0, k7
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
        float csum[4], czsum[4];
        csum[0] = csum2[0].x;
        csum[1] = csum2[0].y;
        csum[2] = csum2[1].x;
        csum[3] = csum2[1].y;
        czsum[0] = czsum2[0].x;
        czsum[1] = czsum2[0].y;
        czsum[2] = czsum2[1].x;
        czsum[3] = czsum2[1].y;
        // slot order inside acc[m][slot]: k3,k4,k5,k6,k1,k2,k0,k7; the
        // offset is 2048 for odd k and 128 for even k
        if (valid) {
#pragma unroll
            for (int m = 0; m < M; ++m) {
                float v[8];
#pragma unroll
                for (int slot = 0; slot < 8; ++slot) {
                    const int e = (0x70216543 >> (4 * slot)) & 7;   // k offset of the slot
                    const float off = (e & 1) ? 2048.0f : 128.0f;
                    v[e] = acc[m][slot] - fmaf(off, csum[m], czsum[m]);
                }
                if (a.splits == 1) {
                    uint32_t outw[4];
#pragma unroll
                    for (int e = 0; e < 8; e += 2) {
                        float x0 = v[e], x1 = v[e + 1];
                        if (a.bias) {
                            x0 += bf16_bits_to_float(a.bias[k_lane + e]);
                            x1 += bf16_bits_to_float(a.bias[k_lane + e + 1]);
                        }
                        outw[e / 2] = bf162_bits(__floats2bfloat162_rn(x0, x1));
                    }
                    *reinterpret_cast<uint4*>(a.dX + static_cast<size_t>(m) * a.K + k_lane) =
                        make_uint4(outw[0], outw[1], outw[2], outw[3]);
                } else {
                    float4* pp = reinterpret_cast<float4*>(a.partial + (static_cast<size_t>(split) * M + m) * a.K + k_lane);
                    pp[0] = make_float4(v[0], v[1], v[2], v[3]);
                    pp[1] = make_float4(v[4], v[5], v[6], v[7]);
                }
            }
        }
    }
    if (*abort_flag) {
        const unsigned long long t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 1000000ull) {
        }
    }
}

}  // namespace w4
