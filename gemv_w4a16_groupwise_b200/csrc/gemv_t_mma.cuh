// Transposed GEMV for M <= 4 with its integer dot products on the tensor
// pipe (the fine-tuning backward from the same packed tensors, "Re-write
// HQQ Fused Gemm Transpose": dX = dY . dequant(W), no repack, no reshaped
// scales or zeros):
//     dX[m, k] = sum_n c[m, n, g(k)] (q[n, k] - z[n, g(k)]),
//     c[m, n, g] = dY[m, n] s[n, g].
//
// The reduction runs over weight rows, while a packed word holds 8
// consecutive k of one row, so the codes are transposed in registers:
//
// Stream.  Each CTA owns a strip of 2048 k (1 KB of every row) and a range
// of rows.  A producer warp brings the range 32 rows at a time into a
// CTA-wide ring: one TMA box of 32 rows x 1040 bytes (the packed words seen
// as 8-byte elements, 130 per row: the strip's 1 KB and the next 16 bytes,
// which no warp reads), so that rows sit 1040 bytes apart and the words
// that one load instruction of a warp reads fall into 32 different banks;
// plus TMA boxes of the 32 rows' scales and zeros.
//
// Arithmetic.  Consumer warp w owns k = 128 w .. 128 w + 127 of the strip
// (16 packed words of every row, inside one group) and, per stage, issues
// 8 mma.sync m16n8k32 (u8 x s8 -> s32):
//   A (16 x 32, u8)  rows are k, columns are the stage's 32 rows.  Lane
//                    (gid, tig) reads word columns 16 w + 2 gid + S (S < 2,
//                    one 8-byte load) of rows 8 i + 2 tig + h (i < 4,
//                    h < 2), transposes the 4 x 4
//                    bytes of each h with byte permutes, and takes byte p of
//                    the rows: the low nibbles (code 2p, A row gid) and the
//                    whole bytes q_2p + 16 q_2p+1 (A row gid + 8).
//                    A column 4 tig + i + 16 h is stage row 8 i + 2 tig + h.
//   B (32 x 8, s8)   c of the stage's rows for the warp's group in 16-bit
//                    fixed point, c' = rint(c 2^(140 - e)) with e the
//                    largest fp32 exponent of c seen so far in the CTA's
//                    rows (a running value per m; so |c'| <= 2^14; when it
//                    rises the integer sums so far move into fp32 sums),
//                    split into digits hi = (c' + 128) >> 8
//                    and lo = c' - 256 hi; column 2 m + d is digit d of m.
//                    Lane r of the warp converts stage row r and leaves its
//                    digits in a per-warp table laid out as the fragments.
//   D (16 x 8, s32)  accumulates over stages: lane (gid, tig) holds, for
//                    m = tig, the two digit sums of k = 8 col + 2p (row gid)
//                    and of the whole bytes (row gid + 8), whose difference
//                    is 16 x the sums of k + 1.
// At the end, with xs = 2^(e - 140) and V = 256 D_hi + D_lo per row,
//     dX[k] = xs V_gid - xs sum_n c' z,
//     dX[k + 1] = xs (V_gid+8 - V_gid) / 16 - xs sum_n c' z,
// the last sum kept by the converting lanes.  Row ranges are split over
// CTAs so that the grid covers the SMs; the fp32 partials of the splits are
// added (with the bias) by splits_finalize_vec4_kernel in a fixed order.
#pragma once

#include "gemv_mma.cuh"

namespace w4 {

constexpr int kTMW = 16;                          // consumer warps
constexpr int kTMThreads = (kTMW + 1) * 32;       // + the producer warp
constexpr int kTMRows = 32;                       // weight rows per stage
constexpr int kTMStrip = 2048;                    // k per CTA strip
constexpr int kTMPitch = 1040;                    // bytes per row slot: 1 KB of words + 16
constexpr int kTMBoxX = kTMPitch / 8;             // box width in 8-byte elements
constexpr int kTMSzOff = kTMRows * kTMPitch;      // scale box, then the zero box 1 KB later
constexpr int kTMStageBytes = kTMSzOff + 2 * 1024;
constexpr int kTMTabBytes = 256;                  // per consumer warp: [digit][m][h][tig][i] bytes

struct GemvTMmaArgs {
    const uint16_t* dY;      // [M, N] bf16
    const uint32_t* packed;  // [N, K / 8]
    const __half* S;
    const __half* Z;
    const uint16_t* bias;    // [K] bf16 or nullptr
    uint16_t* dX;            // [M, K] bf16
    float* partial;          // [splits, M, K] when splits > 1
    int N, K, g, G, sz_row;
    int strips;              // ceil(K / 2048)
    int splits;              // row ranges
    int rows_per_split;      // a multiple of 32
    int stages;
};

// Ring, the warps' digit tables, dY of the split's rows (one float4 per
// row), barriers and the abort flag.
__host__ __device__ inline size_t gemv_t_mma_smem_bytes(int stages, int rows_per_split) {
    return 1024 + static_cast<size_t>(stages) * kTMStageBytes + kTMW * kTMTabBytes +
           static_cast<size_t>(rows_per_split) * 16 + static_cast<size_t>(stages) * 16 + 16;
}

// Bytes i of the four words, for i = 0..3: x[i] = {w0.i, w1.i, w2.i, w3.i}.
__device__ __forceinline__ void transpose_bytes4(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3,
                                                 uint32_t (&x)[4]) {
    const uint32_t t0 = prmt(w0, w1, 0x5140u), t1 = prmt(w0, w1, 0x7362u);
    const uint32_t t2 = prmt(w2, w3, 0x5140u), t3 = prmt(w2, w3, 0x7362u);
    x[0] = prmt(t0, t2, 0x5410u);
    x[1] = prmt(t0, t2, 0x7632u);
    x[2] = prmt(t1, t3, 0x5410u);
    x[3] = prmt(t1, t3, 0x7632u);
}

template <int M, int SZ>
__global__ void __launch_bounds__(kTMThreads, 1)
    gemv_t_mma_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap smap,
                      const __grid_constant__ CUtensorMap zmap, const GemvTMmaArgs a) {
    static_assert(M >= 1 && M <= 4, "M");
    static_assert(SZ == kSzConst || SZ == kSzTma2d || SZ == kSzTma1d, "scale / zero path");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int NS = a.stages;
    constexpr uint32_t kSzTx = SZ == kSzTma2d ? 2 * kTMRows * 16 * 2 : SZ == kSzTma1d ? 2 * kTMRows * 2 : 0;
    uint8_t* ring = base;                                                        // [stage][kTMStageBytes]
    uint8_t* tabs = ring + NS * kTMStageBytes;                                   // [warp][256]
    float4* dys = reinterpret_cast<float4*>(tabs + kTMW * kTMTabBytes);          // [row of the split]
    uint64_t* full = reinterpret_cast<uint64_t*>(dys + a.rows_per_split);
    uint64_t* empty = full + NS;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + NS);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const int strip = blockIdx.x % a.strips, split = blockIdx.x / a.strips;
    const int k0 = strip * kTMStrip;
    const int r0 = split * a.rows_per_split;
    const int r1 = min(a.N, r0 + a.rows_per_split);
    const int nst = r1 > r0 ? (r1 - r0 + kTMRows - 1) / kTMRows : 0;
    auto group_of = [&](int k) { return a.G == 1 ? 0 : k / a.g; };
    const int x_sz = group_of(k0) & ~7;        // first group of the 2-D scale / zero boxes

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kTMW);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (threadIdx.x == kTMW * 32) {
        tma_prefetch_desc(&wmap);
        if (SZ != kSzConst) {
            tma_prefetch_desc(&smap);
            tma_prefetch_desc(&zmap);
        }
    }
    __syncthreads();
    // launched as a programmatic dependent: let the finalize launch, then
    // wait for the work before this kernel before reading any input
    pdl_launch_dependents();
    pdl_wait();

    if (warp == kTMW) {
        // ------------------------------------------------ producer
        // rows past N and columns past K read as 0; rows of the next split
        // that a last stage carries meet c = 0
        int s = 0;
        uint32_t round = 0;
        for (int b = 0; b < nst; ++b) {
            if (round > 0) {
                const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&empty[s], (round - 1) & 1u, abort_flag,
                                                                          kErrTimeoutEmpty));
                if (!ok) break;
            }
            uint8_t* sd = ring + s * kTMStageBytes;
            const int row0 = r0 + b * kTMRows;
            if (SZ == kSzTma2d)
                tma_issue_elected<3>(&full[s], kTMRows * kTMPitch + kSzTx, sd, &wmap, k0 / 16, row0,
                                     sd + kTMSzOff, &smap, x_sz, row0, sd + kTMSzOff + 1024, &zmap, x_sz, row0);
            else if (SZ == kSzTma1d)
                tma_issue_elected<3>(&full[s], kTMRows * kTMPitch + kSzTx, sd, &wmap, k0 / 16, row0,
                                     sd + kTMSzOff, &smap, row0, 0, sd + kTMSzOff + 1024, &zmap, row0, 0);
            else
                tma_issue_elected<1>(&full[s], kTMRows * kTMPitch, sd, &wmap, k0 / 16, row0);
            if (++s == NS) {
                s = 0;
                ++round;
            }
        }
    } else {
        // ------------------------------------------------ consumers
        const int gid = lane >> 2, tig = lane & 3;
        const int kw = k0 + 128 * warp;                  // the warp's first k
        const int grp = group_of(min(kw, a.K - 1));
        float s_const = 0.f, z_const = 0.f;
        if (SZ == kSzConst) {
            s_const = __half2float(a.S[0]);
            z_const = __half2float(a.Z[0]);
        }
        // dY of the CTA's rows into shared memory, one float4 per row (absent
        // m and rows past r1 read as 0, so rows a stage carries past r1 add
        // nothing); one coalesced pass while the first stages are in flight
        for (int r = threadIdx.x; r < nst * kTMRows; r += kTMW * 32) {
            const int n = r0 + r;
            float v[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int m = 0; m < M; ++m)
                if (n < r1) v[m] = bf16_bits_to_float(__ldg(a.dY + static_cast<size_t>(m) * a.N + n));
            dys[r] = make_float4(v[0], v[1], v[2], v[3]);
        }
        named_barrier_sync(1, kTMW * 32);
        // Running exponents: E[m] is the largest fp32 exponent of c seen so
        // far (at least 14), c' = rint(c 2^(140 - E)), and the integer sums
        // in acc are in units of xs = 2^(E - 140).  When a stage raises E[m],
        // the lanes of m first move acc into the fp32 sums fac (in units of
        // the old xs) and clear it, and every lane rescales its sum of c' z.
        // The precision of c' is never below that of one exponent for all
        // of the CTA's rows.
        // thr[m] = 2^(E[m] - 126): |c| >= thr[m] means an exponent above E[m];
        // from its bits, 2^(140 - E) = bits 0x86000000 - thr and
        // 2^(E - 140) = bits thr - 0x07000000
        float thr[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) thr[m] = __int_as_float((14 + 1) << 23);
        auto xs_of = [](float th) { return __int_as_float(__float_as_int(th) - 0x07000000); };
        // this lane's stage row r = 8 i + 2 t + h and its table bytes
        const int ti = lane >> 3, tt = (lane >> 1) & 3, th = lane & 1;
        uint8_t* tab = tabs + warp * kTMTabBytes;
        const int tbyte = th * 16 + tt * 4 + ti;         // + (d * 4 + m) * 32
        const uint32_t* tabw = reinterpret_cast<const uint32_t*>(tab);
        const int bsel = ((gid & 1) * 4 + (gid >> 1)) * 8 + tig;   // word of b0; b1 is 4 words on
        float zt[4] = {0.f, 0.f, 0.f, 0.f};
        int acc[2][4][4];
        float fac[2][4][2];
#pragma unroll
        for (int S = 0; S < 2; ++S)
#pragma unroll
            for (int p = 0; p < 4; ++p) {
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[S][p][j] = 0;
                fac[S][p][0] = fac[S][p][1] = 0.f;
            }
        // acc (units xs) -> fac, for the lane's m = tig: rows gid carry the
        // even codes q_e, rows gid + 8 whole bytes q_e + 16 q_o
        auto fold = [&](float x) {
            const float x16 = x * 0.0625f;
#pragma unroll
            for (int S = 0; S < 2; ++S)
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const float ve = fmaf(256.0f, static_cast<float>(acc[S][p][0]), static_cast<float>(acc[S][p][1]));
                    const float vb = fmaf(256.0f, static_cast<float>(acc[S][p][2]), static_cast<float>(acc[S][p][3]));
                    fac[S][p][0] = fmaf(ve, x, fac[S][p][0]);
                    fac[S][p][1] = fmaf(vb - ve, x16, fac[S][p][1]);
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[S][p][j] = 0;
                }
        };
        auto pick = [&](const auto (&v)[4]) { return tig == 0 ? v[0] : tig == 1 ? v[1] : tig == 2 ? v[2] : v[3]; };
        // word pair (columns 16 w + 2 gid, + 1) of rows 8 i + 2 tig + h
        const uint32_t col0 = static_cast<uint32_t>((16 * warp + 2 * gid) * 4 + (2 * tig) * kTMPitch);

        int s = 0;
        uint32_t phase = 0;
        for (int b = 0; b < nst; ++b) {
            const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&full[s], phase, abort_flag,
                                                                      kErrTimeoutTmaFull));
            if (!ok) break;
            const uint8_t* sb = ring + s * kTMStageBytes;
            // ---- this lane's code words first, so that their latency overlaps
            // the digits: words 2 gid (S = 0) and 2 gid + 1 (S = 1) of the
            // warp's 16, rows 8 i + 2 tig + h
            uint2 w[2][4];
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    w[h][i] = *reinterpret_cast<const uint2*>(sb + col0 + (8 * i + h) * kTMPitch);
            // ---- digits of c for stage row `lane` and the warp's group
            {
                float sv, zv;
                if (SZ == kSzConst) {
                    sv = s_const;
                    zv = z_const;
                } else if (SZ == kSzTma2d) {
                    const __half* sh = reinterpret_cast<const __half*>(sb + kTMSzOff);
                    sv = __half2float(sh[lane * 16 + grp - x_sz]);
                    zv = __half2float(sh[512 + lane * 16 + grp - x_sz]);
                } else {
                    const __half* sh = reinterpret_cast<const __half*>(sb + kTMSzOff);
                    sv = __half2float(sh[lane]);
                    zv = __half2float(sh[512 + lane]);
                }
                const float4 d4 = dys[b * kTMRows + lane];
                const float c[4] = {d4.x * sv, d4.y * sv, d4.z * sv, d4.w * sv};
                const bool up = fabsf(c[0]) >= thr[0] || fabsf(c[1]) >= thr[1] || fabsf(c[2]) >= thr[2] ||
                                fabsf(c[3]) >= thr[3];
                if (__any_sync(0xFFFFFFFFu, up)) {              // rare: an exponent rises
                    float tn[4];
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const int e = min(static_cast<int>(__reduce_max_sync(0xFFFFFFFFu, __float_as_uint(c[m]) & 0x7FFFFFFFu) >> 23),
                                          254);
                        tn[m] = fmaxf(thr[m], __int_as_float((e + 1) << 23));
                    }
                    if (pick(tn) > pick(thr)) fold(xs_of(pick(thr)));
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        // 2^(E_old - E_new) from the exponent fields (thr may
                        // be +inf, the bits of E = 254), or 0 below 2^-126
                        const int f = 127 + ((__float_as_int(thr[m]) - __float_as_int(tn[m])) >> 23);
                        zt[m] *= f > 0 ? __int_as_float(f << 23) : 0.0f;
                        thr[m] = tn[m];
                    }
                }
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    // t = 1.5 * 2^23 + c' with c' = rint(c 2^(140 - E)), |c'| <= 2^14,
                    // in one rounding; the bit pattern of t is 0x4B400000 + c', so
                    // its low byte is the low digit lo = c' - 256 hi (as a signed
                    // byte) and byte 1 of bits + 128 is hi = (c' + 128) >> 8
                    const float t = fmaf(c[m], __int_as_float(0x86000000 - __float_as_int(thr[m])), 12582912.0f);
                    const uint32_t tb = __float_as_uint(t);
                    tab[m * 32 + tbyte] = static_cast<uint8_t>((tb + 128u) >> 8);
                    tab[(4 + m) * 32 + tbyte] = static_cast<uint8_t>(tb);
                    zt[m] = fmaf(t - 12582912.0f, zv, zt[m]);
                }
            }
            __syncwarp();
            const uint32_t b0 = tabw[bsel], b1 = tabw[bsel + 4];
            // ---- codes: four nibble pairs of each word
#pragma unroll
            for (int S = 0; S < 2; ++S) {
                uint32_t x0[4], x1[4];
                if (S == 0) {
                    transpose_bytes4(w[0][0].x, w[0][1].x, w[0][2].x, w[0][3].x, x0);
                    transpose_bytes4(w[1][0].x, w[1][1].x, w[1][2].x, w[1][3].x, x1);
                } else {
                    transpose_bytes4(w[0][0].y, w[0][1].y, w[0][2].y, w[0][3].y, x0);
                    transpose_bytes4(w[1][0].y, w[1][1].y, w[1][2].y, w[1][3].y, x1);
                }
#pragma unroll
                for (int p = 0; p < 4; ++p)
                    mma_u8s8_16832(acc[S][p], x0[p] & 0x0F0F0F0Fu, x0[p], x1[p] & 0x0F0F0F0Fu, x1[p], b0, b1);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            if (++s == NS) {
                s = 0;
                phase ^= 1u;
            }
        }
        // ---- outputs: sum_n c' z over the warp, the last fold, 16 k per lane
#pragma unroll
        for (int m = 0; m < 4; ++m)
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) zt[m] += __shfl_xor_sync(0xFFFFFFFFu, zt[m], o);
        const float xsm = xs_of(pick(thr));
        fold(xsm);
        const float zterm = pick(zt) * xsm;
        const int k = kw + 16 * gid;                     // words 2 gid, 2 gid + 1
        if (!*abort_flag && tig < M && k < a.K) {
            float v[16];
#pragma unroll
            for (int S = 0; S < 2; ++S)
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    v[8 * S + 2 * p] = fac[S][p][0] - zterm;
                    v[8 * S + 2 * p + 1] = fac[S][p][1] - zterm;
                }
            if (a.splits == 1) {
                uint32_t outw[8];
#pragma unroll
                for (int e = 0; e < 16; e += 2) {
                    float y0 = v[e], y1 = v[e + 1];
                    if (a.bias) {
                        y0 += bf16_bits_to_float(a.bias[k + e]);
                        y1 += bf16_bits_to_float(a.bias[k + e + 1]);
                    }
                    outw[e / 2] = bf162_bits(__floats2bfloat162_rn(y0, y1));
                }
                uint4* o = reinterpret_cast<uint4*>(a.dX + static_cast<size_t>(tig) * a.K + k);
                o[0] = make_uint4(outw[0], outw[1], outw[2], outw[3]);
                o[1] = make_uint4(outw[4], outw[5], outw[6], outw[7]);
            } else {
                float4* pp = reinterpret_cast<float4*>(a.partial + (static_cast<size_t>(split) * M + tig) * a.K + k);
#pragma unroll
                for (int q = 0; q < 4; ++q) pp[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
            }
        }
    }
    if (*abort_flag) {
        // let copies still in flight land before the CTA's memory is released
        const unsigned long long t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 1000000ull) {
        }
    }
}

}  // namespace w4
