// Transposed GEMV for M <= 4 on the tensor pipe (the fine-tuning backward
// from the same packed tensors, "Re-write HQQ Fused Gemm Transpose":
// dX = dY . dequant(W), no repack, no reshaped scales or zeros):
//     dX[m, k] = sum_n c[m, n] (q[n, k] - z[n, g(k)]),   c[m, n] = dY[m, n] s[n, g(k)].
//
// Exact operands.  c is the fp32 product of a bf16 and an fp16 (at most 19
// significant bits), so it is exactly the sum of three bf16 parts
// c = c0 + c1 + c2 (c0 = bf16(c), c1 = bf16(c - c0), c2 = c - c0 - c1); the
// codes enter as exact bf16 (q - z), unpacked from the packed words with one
// AND-OR (the bf16 pair (128 + q, 128 + q')) and one bf16x2 subtraction of
// (128 + z, 128 + z').  The mma (m16n8k16, bf16 x bf16 -> fp32) then forms
// every product exactly and accumulates in fp32; the three parts are
// separate columns, added once at the end.
//
// The reduction runs over weight rows, while a packed word holds 8
// consecutive k of one row, so the codes are transposed on the way in.
//
// Stream.  Each CTA owns a strip of 16 KW k and a range of rows.  A
// producer warp brings the range 32 rows at a time into a CTA-wide ring: one
// TMA box of 32 rows x (8 KW + 16) bytes (the packed words seen as 8-byte
// elements: the strip's bytes and the next 16, which no warp reads), plus
// TMA boxes of the 32 rows' scales and zeros.
//
// Arithmetic.  Consumer warp w owns k = KW w .. KW w + KW - 1 of the strip
// (inside one group: KW divides the group length).  Per stage and n-tile t
// (stage rows 16 t .. 16 t + 15) the mma's 16 reduction columns are the rows
// 16 t + 4 tig + {0, 1} (register pair 0) and + {2, 3} (pair 1) of lane
// (gid, tig); its 16 k-rows are, for tile j, k-row gid = nibble j % 4 of the
// lane's word j / 4 (words 2 gid, 2 gid + 1 of the warp's KW k when KW =
// 128; word gid when KW = 64) and k-row gid + 8 = nibble j % 4 + 4 of the
// same word.  So a lane reads one (or two) words of four rows, pairs the rows
// with one byte permute each, and every (shift, AND-OR, subtract) yields one
// A register: no codes move between lanes.  B is (c0, c1, c2) of each
// activation row: columns 3 m' + p of set m / 2 (m' = m % 2), written by the
// lane that converts stage row r into a per-warp table laid out as the B
// fragments.  Accumulators stay in registers across all the CTA's stages.
//
// At the end a lane adds the three parts of each of its columns with one
// shuffle, and the lanes holding whole rows write 16 (or 8) consecutive dX,
// or fp32 partials when the rows are split over CTAs (added, with the bias,
// by splits_finalize_vec4_kernel in a fixed order).
#pragma once

#include "gemv_q8.cuh"

namespace w4 {

constexpr int kTMW = 16;                          // consumer warps
constexpr int kTMThreads = (kTMW + 1) * 32;       // + the producer warp
constexpr int kTMRows = 32;                       // weight rows per stage

// Geometry for a warp k-width KW (128 or 64): strip 16 KW k; a stage row is
// the strip's 8 KW bytes plus 16.
__host__ __device__ constexpr int tm_strip(int KW) { return kTMW * KW; }
__host__ __device__ constexpr int tm_pitch(int KW) { return kTMW * KW / 2 + 16; }
__host__ __device__ constexpr int tm_sz_off(int KW) { return kTMRows * tm_pitch(KW); }
__host__ __device__ constexpr int tm_stage_bytes(int KW) { return tm_sz_off(KW) + 2 * 1024; }
// per warp: B table [set][n-tile][register][lane] u32, then (128 + z) of the
// stage's rows as bf16
__host__ __device__ constexpr int tm_tab_bytes(int nset) { return nset * 2 * 2 * 32 * 4 + kTMRows * 2; }

struct GemvTMmaArgs {
    const uint16_t* dY;      // [M, N] bf16
    const uint32_t* packed;  // [N, K / 8]
    const __half* S;
    const __half* Z;
    const uint16_t* bias;    // [K] bf16 or nullptr
    uint16_t* dX;            // [M, K] bf16
    float* partial;          // [splits, M, K] when splits > 1
    int N, K, g, G, sz_row;
    int strips;              // ceil(K / strip)
    int splits;              // row ranges
    int rows_per_split;      // a multiple of 32
    int stages;
    int fmt;                 // format flags: kFmtZeroFloat, kFmtMetaBf16
};

// Ring, the warps' tables, dY of the split's rows (one float4 per row),
// barriers and the abort flag.
__host__ __device__ inline size_t gemv_t_mma_smem_bytes(int KW, int nset, int stages, int rows_per_split) {
    return 1024 + static_cast<size_t>(stages) * tm_stage_bytes(KW) + kTMW * tm_tab_bytes(nset) +
           static_cast<size_t>(rows_per_split) * 16 + static_cast<size_t>(stages) * 16 + 16;
}

template <int M, int KW, int SZ, bool FZ>
__global__ void __launch_bounds__(kTMThreads, 1)
    gemv_t_mma_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap smap,
                      const __grid_constant__ CUtensorMap zmap, const GemvTMmaArgs a) {
    static_assert(M >= 1 && M <= 4, "M");
    static_assert(KW == 128 || KW == 64, "KW");
    static_assert(SZ == kSzConst || SZ == kSzTma2d || SZ == kSzTma1d, "scale / zero path");
    // the test hook that withholds a stage (-1 unless a test injects a lost
    // stage) is set by the host before the launch: read it first thing, so
    // that its global-memory latency overlaps the set-up instead of delaying
    // the producer's first copy
    const int withhold = threadIdx.x >= kTMW * 32 ? *reinterpret_cast<volatile int*>(&g_withhold_stage) : -1;
    constexpr int NSET = (M + 1) / 2;
    constexpr int NT = KW / 16;                   // k-tiles per warp
    constexpr int NWD = KW / 64;                  // packed words per row and lane
    constexpr int kStrip = tm_strip(KW), kPitch = tm_pitch(KW), kSzOff = tm_sz_off(KW);
    constexpr int kStage = tm_stage_bytes(KW), kTab = tm_tab_bytes(NSET);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int NS = a.stages;
    constexpr uint32_t kSzTx = SZ == kSzTma2d ? 2 * kTMRows * 16 * 2 : SZ == kSzTma1d ? 2 * kTMRows * 2 : 0;
    uint8_t* ring = base;                                                        // [stage][kStage]
    uint8_t* tabs = ring + NS * kStage;                                          // [warp][kTab]
    float4* dys = reinterpret_cast<float4*>(tabs + kTMW * kTab);                 // [row of the split]
    uint64_t* full = reinterpret_cast<uint64_t*>(dys + a.rows_per_split);
    uint64_t* empty = full + NS;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + NS);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const int strip = blockIdx.x % a.strips, split = blockIdx.x / a.strips;
    const int k0 = strip * kStrip;
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
    // the B tables start at zero: columns no activation row uses stay zero
    for (int i = threadIdx.x; i < kTMW * kTab / 4; i += blockDim.x) reinterpret_cast<uint32_t*>(tabs)[i] = 0u;
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
            uint8_t* sd = ring + s * kStage;
            const int row0 = r0 + b * kTMRows;
            if (b == withhold) {
                // injected loss: the copy is never issued (nothing in flight)
                if (++s == NS) {
                    s = 0;
                    ++round;
                }
                continue;
            }
            if (SZ == kSzTma2d)
                tma_issue_elected<3>(&full[s], kTMRows * kPitch + kSzTx, sd, &wmap, k0 / 16, row0, sd + kSzOff,
                                     &smap, x_sz, row0, sd + kSzOff + 1024, &zmap, x_sz, row0);
            else if (SZ == kSzTma1d)
                tma_issue_elected<3>(&full[s], kTMRows * kPitch + kSzTx, sd, &wmap, k0 / 16, row0, sd + kSzOff,
                                     &smap, row0, 0, sd + kSzOff + 1024, &zmap, row0, 0);
            else
                tma_issue_elected<1>(&full[s], kTMRows * kPitch, sd, &wmap, k0 / 16, row0);
            if (++s == NS) {
                s = 0;
                ++round;
            }
        }
    } else {
        // ------------------------------------------------ consumers
        const int gid = lane >> 2, tig = lane & 3;
        const int kw = k0 + KW * warp;                   // the warp's first k
        const int grp = group_of(min(kw, a.K - 1));
        const bool mbf = (a.fmt & kFmtMetaBf16) != 0;
        // a fractional zero point z is taken as zi + (z - zi), zi = clamp(rint(z), 0, 15):
        // the codes enter the mma as the exact bf16 q - zi, and since the
        // warp's k columns share one group, the rest is one fp32 sum per
        // activation row, sum_n c[n] (z - zi)[n], taken off every output
        constexpr bool fz = FZ;     // a.fmt & kFmtZeroFloat, as a template argument
        float corr[4] = {0.f, 0.f, 0.f, 0.f};
        float s_const = 0.f, z_const = 0.f;
        if (SZ == kSzConst) {
            s_const = meta_to_float(a.S[0], mbf);
            z_const = meta_to_float(a.Z[0], mbf);
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
        uint8_t* tab = tabs + warp * kTab;
        uint16_t* tab16 = reinterpret_cast<uint16_t*>(tab);
        const uint32_t* tabw = reinterpret_cast<const uint32_t*>(tab);
        uint16_t* zzt = reinterpret_cast<uint16_t*>(tab + NSET * 2 * 2 * 32 * 4);
        // the converting lane's stage row r = lane: its place in the B fragments
        const int ct = lane >> 4, rr = lane & 15;
        const int bt = rr >> 2, breg = (rr & 3) >> 1, bhalf = rr & 1;
        float acc[NSET][NT][4];
#pragma unroll
        for (int st = 0; st < NSET; ++st)
#pragma unroll
            for (int j = 0; j < NT; ++j) acc[st][j][0] = acc[st][j][1] = acc[st][j][2] = acc[st][j][3] = 0.f;
        // this lane's words: (2 gid, 2 gid + 1) or gid of the warp's KW k
        const int wbyte = KW * warp / 2 + (NWD == 2 ? 8 * gid : 4 * gid);

        int s = 0;
        uint32_t phase = 0;
        for (int b = 0; b < nst; ++b) {
            const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&full[s], phase, abort_flag,
                                                                      kErrTimeoutTmaFull));
            if (!ok) break;
            const uint8_t* sb = ring + s * kStage;
            // ---- this lane's code words first, so that their latency overlaps
            // the conversion: rows 16 t + 4 tig + i
            uint32_t wv[2][4][NWD];
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint8_t* p = sb + (16 * t + 4 * tig + i) * kPitch + wbyte;
                    if (NWD == 2) {
                        const uint2 w2 = *reinterpret_cast<const uint2*>(p);
                        wv[t][i][0] = w2.x;
                        wv[t][i][NWD - 1] = w2.y;
                    } else {
                        wv[t][i][0] = *reinterpret_cast<const uint32_t*>(p);
                    }
                }
            // ---- stage row `lane`: (c0, c1, c2) of each activation row into
            // the B table, (128 + z) into the zero table
            {
                float sv, zv;
                if (SZ == kSzConst) {
                    sv = s_const;
                    zv = z_const;
                } else if (SZ == kSzTma2d) {
                    const __half* sh = reinterpret_cast<const __half*>(sb + kSzOff);
                    sv = meta_to_float(sh[lane * 16 + grp - x_sz], mbf);
                    zv = meta_to_float(sh[512 + lane * 16 + grp - x_sz], mbf);
                } else {
                    const __half* sh = reinterpret_cast<const __half*>(sb + kSzOff);
                    sv = meta_to_float(sh[lane], mbf);
                    zv = meta_to_float(sh[512 + lane], mbf);
                }
                const float4 d4 = dys[b * kTMRows + lane];
                const float dv[4] = {d4.x, d4.y, d4.z, d4.w};
                float zfr = 0.f;
                if (fz) {
                    const float zi = fminf(fmaxf(rintf(zv), 0.f), 15.f);
                    zfr = zv - zi;                         // exact
                    zv = zi;
                }
                __syncwarp();                              // the last stage's table reads are done
#pragma unroll
                for (int m = 0; m < M; ++m) {
                    const float c = dv[m] * sv;            // exact: 8 x 11 significant bits
                    if (fz) corr[m] = fmaf(c, zfr, corr[m]);
                    const __nv_bfloat16 p0 = __float2bfloat16_rn(c);
                    const float q1 = c - __bfloat162float(p0);
                    const __nv_bfloat16 p1 = __float2bfloat16_rn(q1);
                    const __nv_bfloat16 p2 = __float2bfloat16_rn(q1 - __bfloat162float(p1));
                    const __nv_bfloat16 pv[3] = {p0, p1, p2};
#pragma unroll
                    for (int p = 0; p < 3; ++p) {
                        const int col = 3 * (m & 1) + p;
                        const int idx = ((((m >> 1) * 2 + ct) * 2 + breg) * 32 + col * 4 + bt) * 2 + bhalf;
                        tab16[idx] = __bfloat16_as_ushort(pv[p]);
                    }
                }
                zzt[lane] = __bfloat16_as_ushort(__float2bfloat16_rn(128.0f + zv));
                __syncwarp();
            }
            // ---- the mma: per n-tile, pairs (rows 4 tig, 4 tig + 1) and (+2, +3)
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                uint32_t bq[NSET][2];
#pragma unroll
                for (int st = 0; st < NSET; ++st) {
                    bq[st][0] = tabw[((st * 2 + t) * 2 + 0) * 32 + lane];
                    bq[st][1] = tabw[((st * 2 + t) * 2 + 1) * 32 + lane];
                }
                const uint32_t zab = *reinterpret_cast<const uint32_t*>(zzt + 16 * t + 4 * tig);
                const uint32_t zcd = *reinterpret_cast<const uint32_t*>(zzt + 16 * t + 4 * tig + 2);
#pragma unroll
                for (int wd = 0; wd < NWD; ++wd) {
                    // nibbles 0..3 of rows (A, B) as bf16 pairs in u, 4..7 in v
                    const uint32_t uab = prmt(wv[t][0][wd], wv[t][1][wd], 0x5410u);
                    const uint32_t vab = prmt(wv[t][0][wd], wv[t][1][wd], 0x7632u);
                    const uint32_t ucd = prmt(wv[t][2][wd], wv[t][3][wd], 0x5410u);
                    const uint32_t vcd = prmt(wv[t][2][wd], wv[t][3][wd], 0x7632u);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint32_t a0 = bf16x2_sub(lop3_and_or(uab >> (4 * q), 0x000F000Fu, 0x43004300u), zab);
                        const uint32_t a1 = bf16x2_sub(lop3_and_or(vab >> (4 * q), 0x000F000Fu, 0x43004300u), zab);
                        const uint32_t a2 = bf16x2_sub(lop3_and_or(ucd >> (4 * q), 0x000F000Fu, 0x43004300u), zcd);
                        const uint32_t a3 = bf16x2_sub(lop3_and_or(vcd >> (4 * q), 0x000F000Fu, 0x43004300u), zcd);
#pragma unroll
                        for (int st = 0; st < NSET; ++st)
                            mma_bf16_16816(acc[st][4 * wd + q], a0, a1, a2, a3, bq[st][0], bq[st][1]);
                    }
                }
            }
            __syncwarp();
            mbar_arrive_elected(&empty[s]);
            if (++s == NS) {
                s = 0;
                phase ^= 1u;
            }
        }
        if (fz) {
#pragma unroll
            for (int m = 0; m < M; ++m)
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) corr[m] += __shfl_xor_sync(0xFFFFFFFFu, corr[m], o);
        }
        // ---- outputs: the three parts of each activation row meet in lane
        // tig = 0 (row 2 st) and tig = 1 (row 2 st + 1) of each gid: columns
        // (0, 1 | 2) and (3 | 4, 5) of the set
#pragma unroll
        for (int st = 0; st < NSET; ++st) {
            float v[NT * 2];
#pragma unroll
            for (int j = 0; j < NT; ++j)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float first = acc[st][j][2 * h], second = acc[st][j][2 * h + 1];
                    const float whole = first + second;
                    const float recv = __shfl_down_sync(0xFFFFFFFFu, tig == 1 ? first : whole, 1);
                    v[2 * j + h] = tig == 0 ? whole + recv : second + recv;
                }
            const int m = 2 * st + tig;
            // k of value (j, h): word j / 4, nibble j % 4 + 4 h of the lane's words
            const int kl = kw + (NWD == 2 ? 16 * gid : 8 * gid);
            if (!*abort_flag && tig < 2 && m < M && kl < a.K) {
                float o[8 * NWD];
#pragma unroll
                for (int j = 0; j < NT; ++j)
#pragma unroll
                    for (int h = 0; h < 2; ++h) o[8 * (j >> 2) + (j & 3) + 4 * h] = v[2 * j + h];
                if (fz) {
                    const float cm = m == 0 ? corr[0] : m == 1 ? corr[1] : m == 2 ? corr[2] : corr[3];
#pragma unroll
                    for (int e = 0; e < 8 * NWD; ++e) o[e] -= cm;
                }
                if (a.splits == 1) {
                    uint32_t outw[4 * NWD];
#pragma unroll
                    for (int e = 0; e < 8 * NWD; e += 2) {
                        float y0 = o[e], y1 = o[e + 1];
                        if (a.bias) {
                            y0 += bf16_bits_to_float(a.bias[kl + e]);
                            y1 += bf16_bits_to_float(a.bias[kl + e + 1]);
                        }
                        outw[e / 2] = bf162_bits(__floats2bfloat162_rn(y0, y1));
                    }
                    uint4* op = reinterpret_cast<uint4*>(a.dX + static_cast<size_t>(m) * a.K + kl);
#pragma unroll
                    for (int q = 0; q < NWD; ++q)
                        op[q] = make_uint4(outw[4 * q], outw[4 * q + 1], outw[4 * q + 2], outw[4 * q + 3]);
                } else {
                    float4* pp = reinterpret_cast<float4*>(a.partial + (static_cast<size_t>(split) * M + m) * a.K + kl);
#pragma unroll
                    for (int q = 0; q < 2 * NWD; ++q) pp[q] = make_float4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
                }
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
