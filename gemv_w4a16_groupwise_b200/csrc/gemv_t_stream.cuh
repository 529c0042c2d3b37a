// Transposed GEMV for M <= 4 (the fine-tuning backward from the same packed
// tensors, "Re-write HQQ Fused Gemm Transpose": dX = dY . dequant(W), no
// repack, no reshaped scales or zeros):
//     dX[m, k] = sum_n dY[m, n] * s[n, g(k)] * (q[n, k] - z[n, g(k)]).
//
// The reduction runs over the weight rows, which the packed layout keeps
// apart (rows are contiguous along K), so each CTA owns a strip of 2048 k
// (one box width) and walks a range of rows:
//   * a producer warp streams 4-row x 1 KB boxes of the strip (and the
//     rows' scale / zero boxes) through a CTA-wide ring; a stage is
//     refilled once all 16 consumer warps released it;
//   * a table warp turns each landed box into c[m] = dY[m, n] * s[n, g]
//     for its 4 rows and the strip's groups, stored as duplicated pairs for
//     the paired FMAs, and keeps sum_n c and sum_n c z per group;
//   * consumer warp w owns k = 256 (w % 8) .. + 255 of the strip and rows
//     2 (w / 8), 2 (w / 8) + 1 of every box, lane l one packed word (8 k,
//     inside one group); per row it adds c * (off + q) for its 8 codes with
//     the magic-number unpack (one lop3 turns a code into the fp32 value
//     off + q, off = 128 or 2048) and paired FMAs.
// At the end the two row halves are added and
//     dX = sum c (off + q) - off * sum c - sum c z = sum c (q - z).
// Row ranges are split over CTAs so the grid covers the SMs; the fp32
// partials of the splits are added (with the bias) by
// splits_finalize_kernel in a fixed order.
#pragma once

#include "gemv_mma.cuh"

namespace w4 {

constexpr int kTSW = 16;         // consumer warps per CTA
constexpr int kTSThreads = (kTSW + 2) * 32;   // + the producer warp and the table warp
constexpr int kTSStrip = kSBK;   // k per CTA strip (one box width)
constexpr int kTSTab = kSBBytes + 256;        // offset of a stage's c table
constexpr int kTSTabBytes = kSR * 16 * 32;    // [4 rows][16 groups] x 2 float4

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
// group per row; each starting on a 128-byte boundary), then the box's c
// table.
__host__ __device__ inline int gemv_t_stage_bytes(int) { return kTSTab + kTSTabBytes; }

// Ring, barriers, the groups' correction sums, and dY of the CTA's rows as
// one float4 per row.
__host__ __device__ inline size_t gemv_t_stream_smem_bytes(int stages, int sz, int rows_per_split) {
    return 1024 + static_cast<size_t>(stages) * gemv_t_stage_bytes(sz) + static_cast<size_t>(stages) * 24 + 16 + 15 +
           16 * 2 * 16 + static_cast<size_t>(rows_per_split) * 16;
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
    uint64_t* ready = empty + NS;                                            // the stage's c table is built
    volatile int* abort_flag = reinterpret_cast<volatile int*>(ready + NS);
    float4* corr = reinterpret_cast<float4*>(ring + ((NS * SB + NS * 24 + 16 + 15) & ~15));   // [16 groups][2]
    float4* dys = corr + 2 * 16;                                             // [row of the split] (dY[0..3][n])
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
    const int fgs = group_of(k0);                                  // the strip's first group
    const int ngl = group_of(min(k0 + kTSStrip, a.K) - 1) - fgs + 1;   // groups the strip touches (<= 16)
    const int x_sz = fgs & ~7;                                     // 2-D boxes: their first group

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kTSW);
            mbar_init(&ready[s], 1);
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
        int s = 0;
        uint32_t round = 0;
        for (int b = 0; b < nboxes; ++b) {
            if (round > 0) {
                const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&empty[s], (round - 1) & 1u, abort_flag,
                                                                          kErrTimeoutEmpty));
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
            if (++s == NS) {
                s = 0;
                ++round;
            }
        }
    } else if (warp == kTSW + 1) {
        // ------------------------------------------------ c tables
        // lane (group lg, row pair rp): c[m] = dY[m, n] s[n, g] for rows
        // 2 rp, 2 rp + 1 of each box, stored as {c0, c0, c1, c1},
        // {c2, c2, c3, c3}; sums of c and c z per group stay in registers
        const int lg = lane & 15, rp = lane >> 4;
        const bool act = lg < ngl;
        float cs[4] = {0.f, 0.f, 0.f, 0.f}, czs[4] = {0.f, 0.f, 0.f, 0.f};
        float s_const = 0.f, z_const = 0.f;
        if (SZ == kSzConst) {
            s_const = __half2float(a.S[0]);
            z_const = __half2float(a.Z[0]);
        }
        int s = 0;
        uint32_t phase = 0;
        for (int b = 0; b < nboxes; ++b) {
            if (!mbar_wait_bounded(&full[s], phase, abort_flag, kErrTimeoutTmaFull)) break;
            uint8_t* sb = ring + s * SB;
            const __half* sh = reinterpret_cast<const __half*>(sb + kSBBytes);
            float4* tab = reinterpret_cast<float4*>(sb + kTSTab);
            const int row0 = r0 + b * kSR;
            if (act) {
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int i = 2 * rp + j;
                    float sv, zv;
                    if (SZ == kSzConst) {
                        sv = s_const;
                        zv = z_const;
                    } else if (SZ == kSzTma2d) {
                        sv = __half2float(sh[i * 16 + fgs - x_sz + lg]);
                        zv = __half2float(sh[64 + i * 16 + fgs - x_sz + lg]);
                    } else {
                        sv = __half2float(sh[(row0 & 7) + i]);
                        zv = __half2float(sh[64 + (row0 & 7) + i]);
                    }
                    const float4 d4 = dys[b * kSR + i];
                    const float c[4] = {d4.x * sv, d4.y * sv, d4.z * sv, d4.w * sv};
#pragma unroll
                    for (int m = 0; m < M; ++m) {
                        cs[m] += c[m];
                        czs[m] = fmaf(c[m], zv, czs[m]);
                    }
                    tab[(i * 16 + lg) * 2] = make_float4(c[0], c[0], c[1], c[1]);
                    if (M > 2) tab[(i * 16 + lg) * 2 + 1] = make_float4(c[2], c[2], c[3], c[3]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&ready[s]);
            if (++s == NS) {
                s = 0;
                phase ^= 1u;
            }
        }
        // per group: the two row pairs' sums, first pair first
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const float o = __shfl_xor_sync(0xFFFFFFFFu, cs[m], 16);
            const float oz = __shfl_xor_sync(0xFFFFFFFFu, czs[m], 16);
            cs[m] = rp ? o + cs[m] : cs[m] + o;
            czs[m] = rp ? oz + czs[m] : czs[m] + oz;
        }
        if (rp == 0) {
            corr[lg * 2] = make_float4(cs[0], cs[1], cs[2], cs[3]);
            corr[lg * 2 + 1] = make_float4(czs[0], czs[1], czs[2], czs[3]);
        }
        named_barrier_sync(1, (kTSW + 1) * 32);
    } else {
        // ------------------------------------------------ consumers
        const int wi = (warp & 7) * 32 + lane;           // word of the strip
        const int rp = warp >> 3;                        // rows 2 rp, 2 rp + 1 of each box
        const int k_lane = k0 + 8 * wi;
        const bool valid = k_lane < a.K;
        const int lg = valid ? group_of(k_lane) - fgs : 0;
        float acc[M][8];
#pragma unroll
        for (int m = 0; m < M; ++m)
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[m][e] = 0.0f;
        int s = 0;
        uint32_t phase = 0;
        for (int b = 0; b < nboxes; ++b) {
            // the table warp has seen the box land and built its c table
            __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&ready[s], phase, abort_flag, kErrTimeoutTmaFull));
            __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&full[s], phase, abort_flag, kErrTimeoutTmaFull));
            const uint8_t* sb = ring + s * SB;
            const float4* tab = reinterpret_cast<const float4*>(sb + kTSTab);
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int i = 2 * rp + j;
                const uint32_t w = valid ? *reinterpret_cast<const uint32_t*>(sb + i * 1024 + wi * 4) : 0u;
                const float4 c01 = tab[(i * 16 + lg) * 2];
                float4 c23 = make_float4(0.f, 0.f, 0.f, 0.f);
                if (M > 2) c23 = tab[(i * 16 + lg) * 2 + 1];
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
                    const float2 cc = m == 0 ? make_float2(c01.x, c01.y)
                                    : m == 1 ? make_float2(c01.z, c01.w)
                                    : m == 2 ? make_float2(c23.x, c23.y)
                                             : make_float2(c23.z, c23.w);
                    float2* A = reinterpret_cast<float2*>(&acc[m][0]);
                    A[0] = ffma2(p0, cc, A[0]);  // k3, k4
                    A[1] = ffma2(p1, cc, A[1]);  // k5, k6
                    A[2] = ffma2(p2, cc, A[2]);  // k1, k2
                    A[3] = ffma2(p3, cc, A[3]);  // k0, k7
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            if (++s == NS) {
                s = 0;
                phase ^= 1u;
            }
        }
        // every box is consumed (and the ring idle): the second row pair's
        // sums go through the ring's memory to the first
        named_barrier_sync(1, (kTSW + 1) * 32);
        float* xacc = reinterpret_cast<float*>(ring) + ((warp & 7) * 32 + lane) * (8 * M);
        if (rp == 1) {
#pragma unroll
            for (int m = 0; m < M; ++m)
#pragma unroll
                for (int e = 0; e < 8; ++e) xacc[m * 8 + e] = acc[m][e];
        }
        named_barrier_sync(2, kTSW * 32);
        // slot order inside acc[m][slot]: k3,k4,k5,k6,k1,k2,k0,k7; the
        // offset is 2048 for odd k and 128 for even k
        if (rp == 0 && valid) {
            const float4 cs4 = corr[lg * 2], czs4 = corr[lg * 2 + 1];
            const float csum[4] = {cs4.x, cs4.y, cs4.z, cs4.w}, czsum[4] = {czs4.x, czs4.y, czs4.z, czs4.w};
#pragma unroll
            for (int m = 0; m < M; ++m) {
                float v[8];
#pragma unroll
                for (int slot = 0; slot < 8; ++slot) {
                    const int e = (0x70216543 >> (4 * slot)) & 7;   // k offset of the slot
                    const float off = (e & 1) ? 2048.0f : 128.0f;
                    v[e] = (acc[m][slot] + xacc[m * 8 + slot]) - fmaf(off, csum[m], czsum[m]);
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
