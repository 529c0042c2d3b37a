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
//    warp-uniform broadcasts.
//  * Packed weights arrive by TMA in boxes of 128 rows x 64 bytes (128 k),
//    64-byte swizzled so that 32 lanes reading 32 different rows hit
//    different banks.  Each warp owns two stages of the 16-stage ring and
//    refills a stage itself as soon as it has consumed it (box i of the
//    CTA's order goes to warp i % 8), so every stage has one consumer that
//    takes its phases in order and no cross-warp release is needed.
//  * Integer arithmetic on CUDA cores: a packed word splits into its even
//    and odd nibbles as two words of four bytes with two ANDs and a shift,
//    and dp4a multiplies four codes by four activation bytes at a time.
//    The activations of each fold granule (a run of F k inside one group)
//    are staged as 24-bit fixed point with one shared exponent, in three
//    byte planes (signed high, unsigned middle and low byte), so that
//        sum_k q_k x_k = 2^e (65536 sum q hi + 256 sum q mid + sum q lo)
//    is accumulated exactly in int32.  A bf16 value within 2^15 of the
//    granule's largest magnitude is represented exactly; smaller ones are
//    rounded to 2^-23 of that maximum.  Per granule the fold adds
//        s * 2^e * (sum_k q_k x_k - z * sum_k x_k)
//    in fp32, with the integer sum of the granule's activations staged too.
//  * Persistent CTAs (one per SM) walk a contiguous range of (K slice,
//    row tile) units; the 8 warps split each unit box by box and meet in
//    shared memory once per 128-row tile.  When K is split, fp32 partials
//    go to the caller's workspace and a finalize kernel adds the slices
//    (and the bias) in a fixed order.
#pragma once

#include "tma.cuh"

namespace w4 {

constexpr int kGemvConsumerWarps = 8;
constexpr int kGemvThreads = kGemvConsumerWarps * 32;
constexpr int kGemvTileRows = 128;
constexpr int kGemvBoxK = 128;
constexpr int kGemvBoxWords = kGemvBoxK / 8;
constexpr int kGemvBoxBytes = kGemvTileRows * (kGemvBoxK / 2);
constexpr int kGemvStages = 2 * kGemvConsumerWarps;

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
    b += static_cast<size_t>(M) * (TK / 8) * 32;            // activation planes, 32 B per word
    b += 4ull * M * (TK / F) * 4;                           // per granule: exponent, int sum, scale, sum
    b += static_cast<size_t>(kGemvConsumerWarps) * M * kGemvTileRows * 4;  // reduction
    b += 1ull * kGemvStages * 8 + 16;                       // barriers + flag
    return b;
}

// dp4a with unsigned codes and signed / unsigned activation bytes
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
    int d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ uint32_t dp4a_uu(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("dp4a.u32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// Biased exponent of a bf16 (1 for zero and subnormals) and its significand
// with the implicit bit: value = mant * 2^(e - 134).
__device__ __forceinline__ int bf16_exp1(uint32_t b) {
    const int e = (b >> 7) & 0xFF;
    return e ? e : 1;
}
__device__ __forceinline__ int bf16_fixed(uint32_t b, int emax) {
    // b * 2^(149 - emax): exact when the exponent is within 15 of emax
    const int e = (b >> 7) & 0xFF;
    const int mant = e ? (0x80 | (b & 0x7F)) : (b & 0x7F);
    const int sh = (e ? e : 1) - emax + 15;
    int v;
    if (sh >= 0) v = mant << sh;
    else if (sh > -9) v = (mant + (1 << (-sh - 1))) >> (-sh);
    else v = 0;
    return (b & 0x8000u) ? -v : v;
}

__device__ __forceinline__ float half_to_float_ldg(const __half* p) {
    return __half2float(__ldg(p));
}

// Position of a warp in its own box sequence: unit u (whose boxes start at
// global index it_u in the CTA's order) and box b of that unit.  Box i of
// the CTA's order belongs to warp i % 8.
struct GemvBoxCursor {
    int u, it_u, b;
};

template <int M, int F>
__global__ void __launch_bounds__(kGemvThreads, 1)
    gemv_fwd_tma_kernel(const __grid_constant__ CUtensorMap wmap, const GemvFwdArgs a) {
    static_assert(M >= 1 && M <= 4, "M");
    static_assert(F >= 32 && F <= kGemvBoxK && (kGemvBoxK % F) == 0, "F");
    constexpr int FW = F / 8;                // words per granule
    constexpr int GPB = kGemvBoxK / F;       // fold granules per box
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* ring = base;
    // activation record of (m, word j): 8 uint32 = hi(even k), hi(odd k),
    // mid(even), mid(odd), lo(even), lo(odd), 2 unused; byte i of an "even"
    // word is k = 8j + 2i, of an "odd" word k = 8j + 2i + 1
    uint4* xrec = reinterpret_cast<uint4*>(ring + kGemvStages * kGemvBoxBytes);
    const int wps = a.TK / 8;                // words per slice
    const int ngran = a.TK / F;
    int* gexp = reinterpret_cast<int*>(xrec + 2 * M * wps);
    int* gsum = gexp + M * ngran;
    float* gscale = reinterpret_cast<float*>(gsum + M * ngran);
    float* gxsum = gscale + M * ngran;
    float* red = gxsum + M * ngran;
    uint64_t* full = reinterpret_cast<uint64_t*>(red + kGemvConsumerWarps * M * kGemvTileRows);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(full + kGemvStages);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int tid = threadIdx.x;
    if (tid == 0) {
        for (int s = 0; s < kGemvStages; ++s) mbar_init(&full[s], 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (tid == 32) tma_prefetch_desc(&wmap);
    __syncthreads();

    const long long C = gridDim.x;
    const int u_begin = static_cast<int>(blockIdx.x * static_cast<long long>(a.units) / C);
    const int u_end = static_cast<int>((blockIdx.x + 1) * static_cast<long long>(a.units) / C);
    auto boxes_of = [&](int u) {
        const int slice = u / a.row_tiles;
        const int len = min(a.TK, a.K - slice * a.TK);
        return (len + kGemvBoxK - 1) / kGemvBoxK;
    };
    auto settle = [&](GemvBoxCursor& c) {  // skip units in which this warp has no box
        while (c.u < u_end && c.b >= boxes_of(c.u)) {
            c.it_u += boxes_of(c.u);
            ++c.u;
            c.b = ((warp - c.it_u) % kGemvConsumerWarps + kGemvConsumerWarps) % kGemvConsumerWarps;
        }
    };
    auto advance = [&](GemvBoxCursor& c) {
        c.b += kGemvConsumerWarps;
        settle(c);
    };
    // The warp's k-th box lives in its private stage warp + 8 * (k & 1):
    // every stage has one consumer, which is also the warp that refills it.
    auto issue = [&](const GemvBoxCursor& c, int k) {
        if (c.u >= u_end || *abort_flag) return;
        if (lane == 0) {
            const int slice = c.u / a.row_tiles, tile = c.u - slice * a.row_tiles;
            const int st = warp + kGemvConsumerWarps * (k & 1);
            fence_proxy_async_smem();  // this warp's reads of the stage precede the refill
            mbar_arrive_expect_tx(&full[st], kGemvBoxBytes);
            tma_load_2d(ring + st * kGemvBoxBytes, &wmap, (slice * a.TK + c.b * kGemvBoxK) / 8,
                        tile * kGemvTileRows, &full[st]);
        }
    };
    // fp16 scale / zero of every fold granule of a box, for the lane's 4 rows
    auto load_sz = [&](const GemvBoxCursor& c, float (&s_)[GPB][4], float (&z_)[GPB][4]) {
        const int cu = min(c.u, u_end - 1);
        const int slice = cu / a.row_tiles, tile = cu - slice * a.row_tiles;
#pragma unroll
        for (int gi = 0; gi < GPB; ++gi) {
            const int grp = min((slice * a.TK + c.b * kGemvBoxK + gi * F) / a.g, a.G - 1);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int n = min(tile * kGemvTileRows + lane + 32 * i, a.N - 1);
                s_[gi][i] = half_to_float_ldg(a.S + n * a.sz_row + grp);
                z_[gi][i] = half_to_float_ldg(a.Z + n * a.sz_row + grp);
            }
        }
    };

    const int swz = (lane >> 1) & 3;  // 64-byte TMA swizzle of this lane's rows
    GemvBoxCursor cc{u_begin, 0, warp};  // next box to consume
    settle(cc);
    GemvBoxCursor ic = cc;               // next box to issue (two ahead of cc)
    issue(ic, 0);
    advance(ic);
    issue(ic, 1);
    advance(ic);
    int k = 0;  // boxes consumed by this warp
    float sc[GPB][4], zc[GPB][4];
    load_sz(cc, sc, zc);

    int cur_slice = -1;
    for (int u = u_begin; u < u_end; ++u) {
        const int slice = u / a.row_tiles, tile = u - slice * a.row_tiles;
        const int k_slice = slice * a.TK;
        if (slice != cur_slice) {
            // ---- stage the activation slice as per-granule fixed point ----
            const int len = min(a.TK, a.K - k_slice);
            for (int i = tid; i < M * ngran; i += 256) {
                gexp[i] = 1;
                gsum[i] = 0;
            }
            named_barrier_sync(1, 256);
            auto load8 = [&](int v) -> uint4 {  // 8 bf16 of (m, word) v, zero past K
                const int m = v / wps, kk = (v - m * wps) * 8;
                if (kk >= len) return make_uint4(0u, 0u, 0u, 0u);
                return __ldg(reinterpret_cast<const uint4*>(a.X + static_cast<size_t>(m) * a.K +
                                                            k_slice + kk));
            };
            // pass 1: largest exponent of each granule (integer max, order-free)
#pragma unroll 1
            for (int v0 = tid; v0 < M * wps; v0 += 256 * 4) {
                uint4 raw[4];
#pragma unroll
                for (int t = 0; t < 4; ++t)
                    raw[t] = (v0 + t * 256 < M * wps) ? load8(v0 + t * 256) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const int v = v0 + t * 256;
                    if (v < M * wps) {
                        const uint32_t r[4] = {raw[t].x, raw[t].y, raw[t].z, raw[t].w};
                        int e = 1;
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            e = max(e, max(bf16_exp1(r[q] & 0xFFFFu), bf16_exp1(r[q] >> 16)));
                        const int m = v / wps, j = v - m * wps;
                        atomicMax(&gexp[m * ngran + j / FW], e);
                    }
                }
            }
            named_barrier_sync(1, 256);
            // pass 2: fixed-point byte planes and the exact granule sums
#pragma unroll 1
            for (int v0 = tid; v0 < M * wps; v0 += 256 * 4) {
                uint4 raw[4];
#pragma unroll
                for (int t = 0; t < 4; ++t)
                    raw[t] = (v0 + t * 256 < M * wps) ? load8(v0 + t * 256) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const int v = v0 + t * 256;
                    if (v < M * wps) {
                        const int m = v / wps, j = v - m * wps;
                        const int emax = gexp[m * ngran + j / FW];
                        const uint32_t r[4] = {raw[t].x, raw[t].y, raw[t].z, raw[t].w};
                        uint32_t hi[2] = {0u, 0u}, mid[2] = {0u, 0u}, lo[2] = {0u, 0u};
                        int sum = 0;
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const uint32_t bits = (e & 1) ? (r[e >> 1] >> 16) : (r[e >> 1] & 0xFFFFu);
                            const int xf = bf16_fixed(bits, emax);
                            sum += xf;
                            const int par = e & 1, pos = e >> 1;  // even/odd word, byte slot
                            hi[par] |= (static_cast<uint32_t>(xf >> 16) & 0xFFu) << (8 * pos);
                            mid[par] |= (static_cast<uint32_t>(xf >> 8) & 0xFFu) << (8 * pos);
                            lo[par] |= (static_cast<uint32_t>(xf) & 0xFFu) << (8 * pos);
                        }
                        xrec[2 * v] = make_uint4(hi[0], hi[1], mid[0], mid[1]);
                        xrec[2 * v + 1] = make_uint4(lo[0], lo[1], 0u, 0u);
                        atomicAdd(&gsum[m * ngran + j / FW], sum);
                    }
                }
            }
            named_barrier_sync(1, 256);
            for (int i = tid; i < M * ngran; i += 256) {
                gscale[i] = ldexpf(1.0f, gexp[i] - 149);   // 2^e of the granule's fixed point
                gxsum[i] = static_cast<float>(gsum[i]);
            }
            named_barrier_sync(1, 256);
            cur_slice = slice;
        }

        float y[4][M];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int m = 0; m < M; ++m) y[i][m] = 0.0f;

        for (; cc.u == u; ++k) {
            const int b = cc.b;
            const int st = warp + kGemvConsumerWarps * (k & 1);
            const uint32_t par = static_cast<uint32_t>(k >> 1) & 1u;
            GemvBoxCursor nc = cc;
            advance(nc);
            float sn[GPB][4], zn[GPB][4];
            load_sz(nc, sn, zn);  // next box's scale / zero, in flight during this box

            const bool ok = __all_sync(0xFFFFFFFFu,
                                       mbar_wait_bounded(&full[st], par, abort_flag, kErrTimeoutTmaFull));
            if (ok) {
                const uint8_t* sb = ring + st * kGemvBoxBytes;
                const uint4* xbox = xrec + 2 * (b * kGemvBoxWords);
                const int gbox = (b * kGemvBoxK) / F;  // granule index of the box start
                int acc_h[4][M];
                uint32_t acc_m[4][M], acc_l[4][M];
                uint4 wc[4];
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    wc[i] = *reinterpret_cast<const uint4*>(sb + (lane + 32 * i) * (kGemvBoxK / 2) + (swz << 4));
#pragma unroll
                for (int c = 0; c < kGemvBoxWords / 4; ++c) {
                    uint4 wn[4];
                    if (c + 1 < kGemvBoxWords / 4) {
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            wn[i] = *reinterpret_cast<const uint4*>(
                                sb + (lane + 32 * i) * (kGemvBoxK / 2) + (((c + 1) ^ swz) << 4));
                    }
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int wb = c * 4 + j;  // word within box
                        const int gi = wb / FW;
                        if (wb % FW == 0) {
#pragma unroll
                            for (int i = 0; i < 4; ++i)
#pragma unroll
                                for (int m = 0; m < M; ++m) {
                                    acc_h[i][m] = 0;
                                    acc_m[i][m] = 0u;
                                    acc_l[i][m] = 0u;
                                }
                        }
                        uint32_t ev[4], od[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const uint32_t w =
                                (j == 0) ? wc[i].x : (j == 1) ? wc[i].y : (j == 2) ? wc[i].z : wc[i].w;
                            ev[i] = w & 0x0F0F0F0Fu;           // codes of k = 8j + 0, 2, 4, 6
                            od[i] = (w >> 4) & 0x0F0F0F0Fu;    // codes of k = 8j + 1, 3, 5, 7
                        }
#pragma unroll
                        for (int m = 0; m < M; ++m) {
                            const uint4 r0 = xbox[2 * (m * wps + wb)];
                            const uint4 r1 = xbox[2 * (m * wps + wb) + 1];
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                acc_h[i][m] = dp4a_us(ev[i], r0.x, acc_h[i][m]);
                                acc_h[i][m] = dp4a_us(od[i], r0.y, acc_h[i][m]);
                                acc_m[i][m] = dp4a_uu(ev[i], r0.z, acc_m[i][m]);
                                acc_m[i][m] = dp4a_uu(od[i], r0.w, acc_m[i][m]);
                                acc_l[i][m] = dp4a_uu(ev[i], r1.x, acc_l[i][m]);
                                acc_l[i][m] = dp4a_uu(od[i], r1.y, acc_l[i][m]);
                            }
                        }
                        if ((wb + 1) % FW == 0) {
#pragma unroll
                            for (int m = 0; m < M; ++m) {
                                const int gidx = m * ngran + gbox + gi;
                                const float xg = gxsum[gidx];
                                const float sx = gscale[gidx];
#pragma unroll
                                for (int i = 0; i < 4; ++i) {
                                    // sum q x in units of the granule's fixed point; mid and low
                                    // planes combine exactly in int32 (< 2^31)
                                    const int ml = static_cast<int>(acc_m[i][m] * 256u + acc_l[i][m]);
                                    const float qx = fmaf(static_cast<float>(acc_h[i][m]), 65536.0f,
                                                          static_cast<float>(ml));
                                    const float t = fmaf(-zc[gi][i], xg, qx);
                                    y[i][m] = fmaf(sc[gi][i] * sx, t, y[i][m]);
                                }
                            }
                        }
                    }
                    if (c + 1 < kGemvBoxWords / 4) {
#pragma unroll
                        for (int i = 0; i < 4; ++i) wc[i] = wn[i];
                    }
                }
            }
            __syncwarp();
            issue(ic, k + 2);  // refill this stage with the box two ahead
            advance(ic);
            cc = nc;
#pragma unroll
            for (int gi = 0; gi < GPB; ++gi)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    sc[gi][i] = sn[gi][i];
                    zc[gi][i] = zn[gi][i];
                }
        }

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
    if (*abort_flag) {
        // a wait gave up: let copies already issued land before the CTA exits
        const unsigned long long t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 1000000ull) {
        }
    }
}

// ---------------------------------------------------------------------------
// M <= 2 forward GEMV with lanes along K.  A warp item is 16 weight rows x
// 1024 k: lane l owns the 32 k [32l, 32l + 32) of the k-block, loads 16
// bytes of each row directly (a warp reads 512 contiguous bytes per row,
// 8 rows in flight per lane) and holds its activation chunk in registers as
// 24-bit fixed point in three byte planes (exponent shared by the 32 k).
// Per row: two ANDs and a shift split each word into even / odd nibble
// bytes, dp4a accumulates exactly in int32, and one fold applies
// s * 2^e * (sum q x - z sum x) (the chunk lies inside one group).  A
// butterfly reduce-scatter over the lanes yields one row total per lane
// pair; the CTA adds the k-blocks of each row in a fixed order and writes Y
// (+ bias): no workspace, no finalize launch.
// ---------------------------------------------------------------------------
struct GemvRowsArgs {
    const uint16_t* X;
    const uint32_t* packed;
    const __half* S;
    const __half* Z;
    const uint16_t* bias;
    uint16_t* Y;
    int N, K, g, G, sz_row;
    int KB;          // k-blocks of 1024 k
    int RBP;         // 16-row blocks per round
    int rounds;      // total rounds (ceil(row blocks / RBP))
};

constexpr int kRowsRB = 16;   // rows per warp item

__host__ __device__ inline size_t gemv_rows_smem_bytes(int M, int KB, int RBP) {
    size_t b = 0;
    b += static_cast<size_t>(M) * KB * 32 * 6 * 16;  // planes: 6 x uint4 per (m, lane chunk)
    b += static_cast<size_t>(M) * KB * 32 * 8;      // scale, integer sum per chunk
    b += static_cast<size_t>(RBP) * KB * kRowsRB * M * 4;  // per-item row totals
    return b;
}

template <int M>
__global__ void __launch_bounds__(512) gemv_rows_kernel(const GemvRowsArgs a) {
    static_assert(M >= 1 && M <= 2, "M");
    extern __shared__ uint4 smem_rows[];
    const int NW = blockDim.x >> 5;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nchunk = a.KB * 32;              // lane chunks per m
    uint4* planes = smem_rows;                 // [m][6][nchunk]
    float* cscale = reinterpret_cast<float*>(planes + M * 6 * nchunk);   // [m][nchunk]
    float* csum = cscale + M * nchunk;                                   // [m][nchunk]
    float* part = csum + M * nchunk;                                     // [RBP][KB][16][M]

    // ---- stage every activation chunk once: exponent, planes, exact sum
    for (int idx = threadIdx.x; idx < M * nchunk; idx += blockDim.x) {
        const int m = idx / nchunk, c = idx - m * nchunk;
        const int k0 = c * 32;
        uint32_t r[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (k0 + 8 * q < a.K)
                v = __ldg(reinterpret_cast<const uint4*>(a.X + static_cast<size_t>(m) * a.K + k0 + 8 * q));
            r[4 * q] = v.x;
            r[4 * q + 1] = v.y;
            r[4 * q + 2] = v.z;
            r[4 * q + 3] = v.w;
        }
        int emax = 1;
#pragma unroll
        for (int q = 0; q < 16; ++q) emax = max(emax, max(bf16_exp1(r[q] & 0xFFFFu), bf16_exp1(r[q] >> 16)));
        int sum = 0;
#pragma unroll
        for (int w = 0; w < 4; ++w) {  // word w of the chunk: k0 + 8w .. k0 + 8w + 7
            uint32_t hi[2] = {0u, 0u}, mid[2] = {0u, 0u}, lo[2] = {0u, 0u};
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const uint32_t bits = (e & 1) ? (r[4 * w + (e >> 1)] >> 16) : (r[4 * w + (e >> 1)] & 0xFFFFu);
                const int xf = bf16_fixed(bits, emax);
                sum += xf;
                const int par = e & 1, pos = e >> 1;
                hi[par] |= (static_cast<uint32_t>(xf >> 16) & 0xFFu) << (8 * pos);
                mid[par] |= (static_cast<uint32_t>(xf >> 8) & 0xFFu) << (8 * pos);
                lo[par] |= (static_cast<uint32_t>(xf) & 0xFFu) << (8 * pos);
            }
            // six uint4 per chunk: (hiE,hiO,midE,midO) of words w = 0..3 and lo
            // plane word q = 6w + t of chunk c lives in component q % 4 of
            // uint4 (m * 6 + q / 4) * nchunk + c: lanes read consecutive uint4
            uint32_t* pl = reinterpret_cast<uint32_t*>(planes);
            const size_t base_u4 = static_cast<size_t>(m) * 6 * nchunk;
            const int q0 = 6 * w;
            const uint32_t vals[6] = {hi[0], hi[1], mid[0], mid[1], lo[0], lo[1]};
#pragma unroll
            for (int t = 0; t < 6; ++t) {
                const int qq = q0 + t;  // 0 .. 23
                pl[(base_u4 + static_cast<size_t>(qq >> 2) * nchunk + c) * 4 + (qq & 3)] = vals[t];
            }
        }
        cscale[idx] = ldexpf(1.0f, emax - 149);
        csum[idx] = static_cast<float>(sum);
    }
    __syncthreads();

    const int items = a.RBP * a.KB;
    const int r_begin = static_cast<int>(static_cast<long long>(blockIdx.x) * a.rounds / gridDim.x);
    const int r_end = static_cast<int>(static_cast<long long>(blockIdx.x + 1) * a.rounds / gridDim.x);
    const int W8 = a.K / 8;
    int cached_kb = -1;
    uint32_t xp[M][24];
    float xscale[M], xsum[M];

    for (int rd = r_begin; rd < r_end; ++rd) {
        for (int t = warp; t < items; t += NW) {
            const int rbl = t / a.KB, kb = t - rbl * a.KB;
            const int rb = rd * a.RBP + rbl;
            const int c = kb * 32 + lane;            // this lane's chunk
            const bool kvalid = c * 32 < a.K;
            if (kb != cached_kb) {
#pragma unroll
                for (int m = 0; m < M; ++m) {
#pragma unroll
                    for (int q4 = 0; q4 < 6; ++q4) {
                        const uint4 v = planes[(static_cast<size_t>(m) * 6 + q4) * nchunk + c];
                        xp[m][4 * q4] = v.x;
                        xp[m][4 * q4 + 1] = v.y;
                        xp[m][4 * q4 + 2] = v.z;
                        xp[m][4 * q4 + 3] = v.w;
                    }
                    xscale[m] = cscale[m * nchunk + c];
                    xsum[m] = csum[m * nchunk + c];
                }
                cached_kb = kb;
            }
            const int grp = min((c * 32) / a.g, a.G - 1);
            float y[kRowsRB][M];
#pragma unroll
            for (int h = 0; h < 2; ++h) {  // two batches of 8 rows, loads first
                uint4 wv[8];
                float sv[8], zv[8];
#pragma unroll
                for (int r = 0; r < 8; ++r) {
                    const int n = rb * kRowsRB + 8 * h + r;
                    const bool ok = kvalid && n < a.N;
                    const int nc = min(n, a.N - 1);
                    wv[r] = ok ? ldg_stream_v4(a.packed + static_cast<size_t>(nc) * W8 + 4 * c)
                               : make_uint4(0u, 0u, 0u, 0u);
                    sv[r] = half_to_float_ldg(a.S + nc * a.sz_row + grp);
                    zv[r] = half_to_float_ldg(a.Z + nc * a.sz_row + grp);
                }
#pragma unroll
                for (int r = 0; r < 8; ++r) {
                    int ah[M];
                    uint32_t am[M], al[M];
#pragma unroll
                    for (int m = 0; m < M; ++m) {
                        ah[m] = 0;
                        am[m] = 0u;
                        al[m] = 0u;
                    }
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        const uint32_t word = (w == 0) ? wv[r].x : (w == 1) ? wv[r].y : (w == 2) ? wv[r].z : wv[r].w;
                        const uint32_t ev = word & 0x0F0F0F0Fu, od = (word >> 4) & 0x0F0F0F0Fu;
#pragma unroll
                        for (int m = 0; m < M; ++m) {
                            ah[m] = dp4a_us(ev, xp[m][6 * w + 0], ah[m]);
                            ah[m] = dp4a_us(od, xp[m][6 * w + 1], ah[m]);
                            am[m] = dp4a_uu(ev, xp[m][6 * w + 2], am[m]);
                            am[m] = dp4a_uu(od, xp[m][6 * w + 3], am[m]);
                            al[m] = dp4a_uu(ev, xp[m][6 * w + 4], al[m]);
                            al[m] = dp4a_uu(od, xp[m][6 * w + 5], al[m]);
                        }
                    }
#pragma unroll
                    for (int m = 0; m < M; ++m) {
                        const int ml = static_cast<int>(am[m] * 256u + al[m]);
                        const float qx = fmaf(static_cast<float>(ah[m]), 65536.0f, static_cast<float>(ml));
                        y[8 * h + r][m] = (sv[r] * xscale[m]) * fmaf(-zv[r], xsum[m], qx);
                    }
                }
            }
            // butterfly reduce-scatter of the 16 row partials over the 32 lanes:
            // afterwards lanes 2r and 2r+1 hold the total of row r
#pragma unroll
            for (int m = 0; m < M; ++m) {
                float v16[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) v16[i] = y[i][m];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const bool up = lane & 16;
                    const float send = up ? v16[i] : v16[i + 8];
                    const float keep = up ? v16[i + 8] : v16[i];
                    v16[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, 16);
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const bool up = lane & 8;
                    const float send = up ? v16[i] : v16[i + 4];
                    const float keep = up ? v16[i + 4] : v16[i];
                    v16[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, 8);
                }
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const bool up = lane & 4;
                    const float send = up ? v16[i] : v16[i + 2];
                    const float keep = up ? v16[i + 2] : v16[i];
                    v16[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, 4);
                }
                {
                    const bool up = lane & 2;
                    const float send = up ? v16[0] : v16[1];
                    const float keep = up ? v16[1] : v16[0];
                    v16[0] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, 2);
                }
                v16[0] += __shfl_xor_sync(0xFFFFFFFFu, v16[0], 1);
                if ((lane & 1) == 0) part[((rbl * a.KB + kb) * kRowsRB + (lane >> 1)) * M + m] = v16[0];
            }
        }
        __syncthreads();
        // add the k-blocks of every row in ascending order and write Y
        for (int o = threadIdx.x; o < a.RBP * kRowsRB * M; o += blockDim.x) {
            const int rbl = o / (kRowsRB * M);
            const int rem = o - rbl * kRowsRB * M;
            const int r = rem / M, m = rem - r * M;
            const int n = (rd * a.RBP + rbl) * kRowsRB + r;
            if (n < a.N) {
                float s = 0.0f;
                for (int kb = 0; kb < a.KB; ++kb) s += part[((rbl * a.KB + kb) * kRowsRB + r) * M + m];
                if (a.bias) s += bf16_bits_to_float(a.bias[n]);
                a.Y[static_cast<size_t>(m) * a.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(s));
            }
        }
        __syncthreads();
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
