// Forward GEMV for M <= 4 whose integer dot products run on the tensor
// pipe (mma.sync m16n8k32, s8 x u8 -> s32), for group lengths that are a
// multiple of 128 (or one group per row).
//
// Streaming is the same as in gemv_stream_kernel: each warp walks 4
// consecutive weight rows along K in 4 rows x 1 KB TMA boxes, with the
// box's scales and zeros copied into the same stage by cp.async.  What
// changes is the arithmetic, which on CUDA cores costs 4 dp4a per packed
// word and activation row; here one mma covers 4 weight rows x 64 k for
// every M <= 4:
//
//   B (32 x 8, u8)  column n = (weight row i = n / 2, half h = n % 2): the
//                   4-bit codes themselves, one byte each, the even and odd
//                   nibbles of one packed word per lane;
//   A (16 x 32, s8) row r = (half h = r / 8, activation row m, digit p):
//                   X in 16-bit fixed point per 128-k granule, split into a
//                   high and a low signed byte (balanced digits, so both
//                   fit s8);
//   D (16 x 8, s32) entries with equal halves in A and B are exact integer
//                   dot products; the two other entries are not used.
//
// A quad-window is 256 k of the box: lane (g, tig) loads one 16-byte chunk
// of weight row g / 2, chunk (g % 2) * 4 + tig, and its 4 words feed the 4
// mma of the window, word t to mma t.  So mma t pairs slot 4 tig + e with
// k = 128 h + 32 tig + 8 t + 2 e (even nibbles) and slot 16 + 4 tig + e
// with the odd k after it, and half h = 0 / 1 is the first / second 128 k
// of the window.  A small kernel (gemv_xfrag_kernel) writes the A
// fragments in exactly this order, once per call, with the granule scales.
//
// Each lane then holds, per window, the exact sums sum_k q x' of weight row
// tig against (m, p) = (g / 2, g % 2) for both halves, and folds them:
//   y += s * (f1 * D - z * f2),  f1 = xs * 256^(1 - p),  f2 = [p == 1] xs * sum_k x'
// with xs = 2^(e - 140), e the granule's largest bf16 exponent.  The two
// digits meet in one shuffle when a row block is done; the work split and
// the output are described at the kernel.
#pragma once

#include "gemv_stream.cuh"

namespace w4 {

constexpr int kMFrac = 6;          // fixed-point bits below the granule's leading binade
constexpr int kMMaxWarps = 16;

// One slice's activation block: A fragments [window][mma t][8 M lanes]
// (16 bytes each), then the fold constants [window][g = 2 m + p] as float4
// {f1_h0, f2_h0, f1_h1, f2_h1} with f1 = xs * 256^(1 - p) and
// f2 = [p == 1] xs * sum x'.
__host__ __device__ inline size_t gemv_mma_xblock_bytes(int M, int TKC) {
    const size_t nqw = static_cast<size_t>(TKC) / 256;
    return nqw * M * (4 * 8 * 16 + 2 * 16);
}

// Programmatic dependent launch: the prep kernel lets the GEMV start early,
// and the GEMV waits for the prep kernel's results only where it needs them.
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// One warp per (slice, window, m); lane = 16 h + 4 t + tig converts the 8
// activations k = 128 h + 32 tig + 8 t .. + 7 of the window (zero past K).
// The grid also clears the GEMV's row-block counters.
__global__ void __launch_bounds__(256) gemv_xfrag_kernel(const uint16_t* __restrict__ X, int M, int K,
                                                         int TKC, int splits, uint8_t* __restrict__ out,
                                                         int* __restrict__ counters, int ncounters) {
    pdl_launch_dependents();
    // the GEMV's per-row-block box counters start from zero on every call
    for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < ncounters;
         i += static_cast<long long>(gridDim.x) * blockDim.x)
        counters[i] = 0;
    const int nqw = TKC / 256;
    const long long unit = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    if (unit >= static_cast<long long>(splits) * nqw * M) return;   // whole warps
    const int lane = threadIdx.x & 31;
    const int m = static_cast<int>(unit % M);
    const long long sq = unit / M;
    const int slice = static_cast<int>(sq / nqw), qw = static_cast<int>(sq - static_cast<long long>(slice) * nqw);
    const int h = lane >> 4, t = (lane >> 2) & 3, tig = lane & 3;
    const long long k = static_cast<long long>(slice) * TKC + qw * 256 + h * 128 + 32 * tig + 8 * t;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (k < K) v = __ldg(reinterpret_cast<const uint4*>(X + static_cast<size_t>(m) * K + k));
    const uint32_t r[4] = {v.x, v.y, v.z, v.w};
    int emax = 1;
#pragma unroll
    for (int q = 0; q < 4; ++q) emax = max(emax, max(bf16_exp1(r[q] & 0xFFFFu), bf16_exp1(r[q] >> 16)));
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) emax = max(emax, __shfl_xor_sync(0xFFFFFFFFu, emax, o));
    uint32_t hi[2] = {0u, 0u}, lo[2] = {0u, 0u};   // [even / odd k] digit bytes
    int sum = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const uint32_t bits = (j & 1) ? (r[j >> 1] >> 16) : (r[j >> 1] & 0xFFFFu);
        const int xf = bf16_fixed_bits(bits, emax, kMFrac);   // |xf| <= 255 * 2^6
        sum += xf;
        const int dl = ((xf + 128) & 255) - 128;             // balanced low digit in [-128, 127]
        const int dh = (xf - dl) >> 8;                        // high digit in [-64, 64]
        hi[j & 1] |= (static_cast<uint32_t>(dh) & 0xFFu) << (8 * (j >> 1));
        lo[j & 1] |= (static_cast<uint32_t>(dl) & 0xFFu) << (8 * (j >> 1));
    }
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
    const size_t nqw8 = static_cast<size_t>(nqw);
    uint8_t* block = out + static_cast<size_t>(slice) * gemv_mma_xblock_bytes(M, TKC);
    uint32_t* frag = reinterpret_cast<uint32_t*>(block);
    // lane (g = 2 m + p, tig) of mma t: {even h0, even h1, odd h0, odd h1}
#pragma unroll
    for (int p = 0; p < 2; ++p) {
        const size_t rec = (static_cast<size_t>(qw) * 4 + t) * (8 * M) + (2 * m + p) * 4 + tig;
        frag[rec * 4 + h] = p ? lo[0] : hi[0];
        frag[rec * 4 + 2 + h] = p ? lo[1] : hi[1];
    }
    if ((lane & 15) == 0) {
        float* fs = reinterpret_cast<float*>(block + nqw8 * M * 512);
        const float xs = ldexpf(1.0f, emax - 134 - kMFrac);
        const size_t f0 = (static_cast<size_t>(qw) * 2 * M + 2 * m) * 4 + 2 * h;   // p = 0
        fs[f0] = 256.0f * xs;
        fs[f0 + 1] = 0.0f;
        fs[f0 + 4] = xs;                                                           // p = 1
        fs[f0 + 5] = xs * static_cast<float>(sum);
    }
}

// D = A B + C and D = A B (C = 0); the fragments are plain values, so the
// compiler may schedule these freely.
__device__ __forceinline__ void mma_s8u8_16832(int (&d)[4], const uint4& a, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_s8u8_16832_z(int (&d)[4], const uint4& a, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%10,%10,%10};"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
        : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b0), "r"(b1), "r"(0));
}

// How the scales and zeros reach a stage:
//   kSzConst  one scale and zero for the whole matrix (global mode): read
//             once per thread, no per-box data;
//   kSzTma2d  groupwise with G % 8 == 0: a TMA box of 4 rows x 16 groups of
//             S and of Z, starting at the 8-aligned group at or below the
//             box's first group;
//   kSzTma1d  one group per row: a TMA box of the 8 rows' values around the
//             box's 4 rows (S and Z seen as one-row 2-D tensors);
//   kSzCopy   anything else: 4-byte cp.async copies (gemv_stream_kernel's
//             scheme), tracked by the same barrier.
enum SzKind { kSzConst = 0, kSzTma2d = 1, kSzTma1d = 2, kSzCopy = 3 };

// Shared-memory footprint of a stage's scales and zeros.  Tiled TMA writes
// must start on a 128-byte boundary, so the Z box sits 128 bytes after the
// S box in both TMA layouts.
__host__ __device__ inline int gemv_mma_sz_bytes(int sz, int szw) {
    return sz == kSzTma2d ? 2 * 128 : sz == kSzTma1d ? 128 + 16 : sz == kSzCopy ? 2 * kSR * szw * 4 : 0;
}
__host__ __device__ inline int gemv_mma_stage_bytes(int sz, int szw) {
    return (kSBBytes + gemv_mma_sz_bytes(sz, szw) + 127) / 128 * 128;
}
__host__ __device__ inline size_t gemv_mma_smem_bytes(int M, int TKC, int warps, int stages, int sz, int szw) {
    size_t b = 1024;
    b += static_cast<size_t>(warps) * stages * gemv_mma_stage_bytes(sz, szw);
    b += static_cast<size_t>(warps) * kSR * 8 * 16;                 // per-box fp32 scale / zero table
    b += gemv_mma_xblock_bytes(M, TKC);
    b += static_cast<size_t>(warps) * stages * 8 + 8 + 16;
    return b;
}

// Arguments of gemv_mma_kernel.
struct GemvMmaArgs {
    const uint8_t* xblocks;   // [splits] activation blocks from gemv_xfrag_kernel
    const __half* S;
    const __half* Z;
    const uint16_t* bias;
    uint16_t* Y;
    float* partial;           // [splits, M, N] when splits > 1
    float* slots;             // [splits, warps of a slice, 2, 4 rows, M] shared row blocks
    int* counters;            // [splits, row blocks] boxes finished (zeroed by the prep kernel)
    int N, K, g, G, sz_row;
    int TKC;                  // k per slice (a whole number of boxes)
    int splits;               // slices; CTA c works on slice c / cps
    int nbs;                  // boxes per slice and row block
    int nrb;                  // row blocks (4 rows each)
    int cps;                  // CTAs per slice
    int stages;               // TMA stages per warp
    int szw;                  // copy path: scale / zero words per row and stage
    long long sz_total;       // halves in each of S and Z (N * sz_row, or 1)
};

// Work split: the boxes of a slice, row block major (box b = row block
// b / nbs, k box b % nbs), are cut into one contiguous range per warp of
// the slice's CTAs, so every warp streams the same number of boxes to
// within one and no warp waits for another.  A row block that one warp
// covers completely is written at once; a row block shared by neighbouring
// warps (at most the first and the last of each range) goes through
// per-warp partial slots, and the warp that completes its box count sums
// the slots in warp order, so the result does not depend on timing.
template <int M, int GK, int SZ>
__global__ void __launch_bounds__(kMMaxWarps * 32, 1)
    gemv_mma_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap smap,
                    const __grid_constant__ CUtensorMap zmap, const GemvMmaArgs a) {
    static_assert(M >= 1 && M <= 4, "M");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int NW = blockDim.x >> 5;
    const int NS = a.stages;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
    const int g = lane >> 2, tig = lane & 3;
    const int nqw = a.TKC / 256;
    const uint32_t xbytes = static_cast<uint32_t>(gemv_mma_xblock_bytes(M, a.TKC));
    const int SB = gemv_mma_stage_bytes(SZ, a.szw);
    // bytes the scale / zero boxes add to a stage's transaction count
    constexpr int kSzTx = SZ == kSzTma2d ? 2 * kSR * 16 * 2 : SZ == kSzTma1d ? 2 * 8 * 2 : 0;
    uint8_t* ring = base;                                                    // [warp][stage][SB]
    float4* table = reinterpret_cast<float4*>(ring + NW * NS * SB);          // [warp][8 windows][4 rows]
    uint8_t* xblk = reinterpret_cast<uint8_t*>(table + NW * kSR * 8);
    const uint4* frag = reinterpret_cast<const uint4*>(xblk);                // [qw][t][8M]
    const float4* fsc = reinterpret_cast<const float4*>(xblk + static_cast<size_t>(nqw) * M * 512);  // [qw][2M]
    uint64_t* full = reinterpret_cast<uint64_t*>(xblk + xbytes);
    uint64_t* xbar = full + NW * NS;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(xbar + 1);

    if (tid == 0) {
        // a stage completes on the elected lane's expect-tx arrival and its
        // bytes; the copy path adds one cp.async arrival per lane
        for (int i = 0; i < NW * NS; ++i) mbar_init(&full[i], SZ == kSzCopy ? 33 : 1);
        mbar_init(xbar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (tid == 32) {
        tma_prefetch_desc(&wmap);
        if (SZ == kSzTma2d || SZ == kSzTma1d) {
            tma_prefetch_desc(&smap);
            tma_prefetch_desc(&zmap);
        }
    }
    __syncthreads();

    const int slice = blockIdx.x / a.cps;
    const int W = a.cps * NW;                                   // warps of this slice
    const int w = (blockIdx.x - slice * a.cps) * NW + warp;
    const long long T = static_cast<long long>(a.nrb) * a.nbs;  // boxes of the slice
    auto wstart = [&](int ww) { return static_cast<int>(static_cast<long long>(ww) * T / W); };
    // the warp whose range holds box b
    auto warp_of = [&](int b) {
        return static_cast<int>((static_cast<long long>(b + 1) * W - 1) / T);
    };
    const int b_begin = wstart(w), b_end = wstart(w + 1);
    int gshift = 0;
    if (GK == kGroupsPow2) gshift = __ffs(a.g) - 1;

    struct Cur {
        int b, rb, kb;
    };
    auto advance = [&](Cur& c) {
        ++c.b;
        if (++c.kb == a.nbs) {
            c.kb = 0;
            ++c.rb;
        }
    };
    const Cur start{b_begin, b_begin / a.nbs, b_begin - (b_begin / a.nbs) * a.nbs};
    auto box_k0 = [&](const Cur& c) { return slice * a.TKC + c.kb * kSBK; };
    auto box_row0 = [&](const Cur& c) { return c.rb * kSR; };
    auto first_group = [&](int k0) {
        if (GK == kGroupsOne) return 0;
        if (GK == kGroupsPow2) return k0 >> gshift;
        return k0 / a.g;
    };

    const int sz_arr = (lane >> 2) & 1, sz_row_i = lane & 3;   // copy path: lane's array and row
    int islot = 0;
    Cur ic = start;
    auto issue = [&]() {
        if (ic.b < b_end) {
            const int k0 = box_k0(ic), row0 = box_row0(ic);
            const int st = warp * NS + islot;
            uint8_t* sd = ring + st * SB;
            if (SZ == kSzCopy) {
                const long long h0 =
                    (static_cast<long long>(row0 + sz_row_i) * a.sz_row + first_group(k0)) & ~1ll;
                uint32_t* szd = reinterpret_cast<uint32_t*>(sd + kSBBytes) + (sz_arr * kSR + sz_row_i) * a.szw;
                const __half* src = sz_arr ? a.Z : a.S;
                for (int q = lane >> 3; q < a.szw; q += 4) {
                    const long long hh = h0 + 2 * q;
                    const long long avail = a.sz_total - hh;
                    const uint32_t bytes = avail >= 2 ? 4u : (avail == 1 ? 2u : 0u);
                    cp_async_4(szd + q, src + (bytes ? hh : 0), bytes);
                }
                cp_async_arrive_noinc(&full[st]);
            }
            // (after a timed-out wait the loads keep coming; the kernel lets
            // them land before it exits)
            if (SZ == kSzTma2d) {
                const int x = first_group(k0) & ~7;
                tma_issue_elected<3>(&full[st], kSBBytes + kSzTx, sd, &wmap, k0 / 8, row0, sd + kSBBytes, &smap, x,
                                     row0, sd + kSBBytes + 128, &zmap, x, row0);
            } else if (SZ == kSzTma1d) {
                tma_issue_elected<3>(&full[st], kSBBytes + kSzTx, sd, &wmap, k0 / 8, row0, sd + kSBBytes, &smap,
                                     row0 & ~7, 0, sd + kSBBytes + 128, &zmap, row0 & ~7, 0);
            } else {
                tma_issue_elected<1>(&full[st], kSBBytes, sd, &wmap, k0 / 8, row0);
            }
            if (++islot == NS) islot = 0;
            advance(ic);
        }
    };
    // one stage of weights first; then, once the prep kernel is done, the
    // activation block (so that it does not queue behind the whole ring);
    // then the rest of the ring
    issue();
    pdl_wait();
    if (tid == 0 && b_begin < wstart(NW * (blockIdx.x - slice * a.cps + 1))) {
        mbar_arrive_expect_tx(xbar, xbytes);
        bulk_load_1d(xblk, a.xblocks + static_cast<size_t>(slice) * xbytes, xbytes, xbar);
    }
    for (int b = 1; b < NS; ++b) issue();

    const int wrow = g >> 1, wchunk = (g & 1) * 4 + tig;   // the B chunk this lane loads
    const bool f_lane = g < 2 * M;
    // lanes without activation rows (g >= 2M) never load: their fragments
    // and fold constants stay zero for the whole kernel
    uint4 af[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) af[t] = make_uint4(0u, 0u, 0u, 0u);
    float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
    float s_const = 0.f, z_const = 0.f;
    if (SZ == kSzConst) {
        s_const = __half2float(a.S[0]);
        z_const = __half2float(a.Z[0]);
    }
    float4* wtable = table + warp * kSR * 8;
    const int tq = lane & 7, ti = lane >> 3;               // table entry this lane builds
    if (b_begin < b_end) mbar_wait_bounded(xbar, 0, abort_flag, kErrTimeoutTmaFull);

    // the outputs of row block rb: lanes with even g < 2M hold (m = g / 2,
    // row tig) after the digit shuffle
    auto store = [&](int m, int n, float v) {
        if (a.splits == 1) {
            if (a.bias) v += bf16_bits_to_float(a.bias[n]);
            a.Y[static_cast<size_t>(m) * a.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
        } else {
            a.partial[(static_cast<size_t>(slice) * M + m) * a.N + n] = v;
        }
    };
    const int first_rb = start.rb;
    auto finish = [&](int rb, int nb, float y) {
        const float v = y + __shfl_xor_sync(0xFFFFFFFFu, y, 4);
        const bool out_lane = !(g & 1) && f_lane;
        if (nb == a.nbs) {
            const int n = rb * kSR + tig;
            if (out_lane && n < a.N) store(g >> 1, n, v);
            return;
        }
        float* sl = a.slots + ((static_cast<size_t>(slice) * W + w) * 2 + (rb == first_rb ? 0 : 1)) * (kSR * M);
        if (out_lane) sl[tig * M + (g >> 1)] = v;
        __threadfence();
        __syncwarp();
        int last = 0;
        if (lane == 0) last = (atomicAdd(&a.counters[slice * a.nrb + rb], nb) + nb == a.nbs);
        last = __shfl_sync(0xFFFFFFFFu, last, 0);
        if (!last) return;
        __threadfence();
        const int w0 = warp_of(rb * a.nbs), w1 = warp_of(rb * a.nbs + a.nbs - 1);
        if (lane < kSR * M) {
            const int r = lane / M, m = lane - (lane / M) * M;
            float s = 0.0f;
            for (int ww = w0; ww <= w1; ++ww) {
                const int ws = wstart(ww);
                if (ws == wstart(ww + 1)) continue;
                const int sslot = (ws / a.nbs == rb) ? 0 : 1;
                s += __ldcg(a.slots + ((static_cast<size_t>(slice) * W + ww) * 2 + sslot) * (kSR * M) + r * M + m);
            }
            const int n = rb * kSR + r;
            if (n < a.N) store(m, n, s);
        }
    };

    int cslot = 0;
    uint32_t cpar = 0;
    Cur cc = start;
    float y = 0.0f;
    int nb_rb = 0;
    for (int b = b_begin; b < b_end; ++b) {
        const int k0 = box_k0(cc), row0 = box_row0(cc);
        const int st = warp * NS + cslot;
        __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&full[st], cpar, abort_flag, kErrTimeoutTmaFull));
        if (++cslot == NS) {
            cslot = 0;
            cpar ^= 1u;
        }
        const uint8_t* sb = ring + st * SB;
        if (SZ != kSzConst) {
            // fp32 table of (s, z) for window tq, row ti, both halves (the 4
            // rows of a window are adjacent: the readers hit 4 distinct banks)
            const int grp_lo = first_group(k0);
            int o0, o1;
            if (GK == kGroupsOne) {
                o0 = 0;
                o1 = 0;
            } else if (GK == kGroupsPow2) {
                o0 = (tq * 256) >> gshift;
                o1 = (tq * 256 + 128) >> gshift;
            } else {
                const int r0 = k0 - grp_lo * a.g;
                o0 = (r0 + tq * 256) / a.g;
                o1 = (r0 + tq * 256 + 128) / a.g;
            }
            const __half* sh = reinterpret_cast<const __half*>(sb + kSBBytes);
            const __half *ps, *pz;
            if (SZ == kSzTma2d) {
                ps = sh + ti * 16 + (grp_lo & 7);
                pz = ps + 64;                    // Z box 128 bytes after the S box
            } else if (SZ == kSzTma1d) {
                ps = sh + (row0 & 7) + ti;
                pz = ps + 64;
            } else {
                ps = sh + ti * 2 * a.szw + ((((row0 + ti) & a.sz_row) ^ grp_lo) & 1);
                pz = ps + kSR * 2 * a.szw;
            }
            wtable[tq * kSR + ti] = make_float4(__half2float(ps[o0]), __half2float(pz[o0]), __half2float(ps[o1]),
                                                __half2float(pz[o1]));
            __syncwarp();
        }
        // per-box bases: every window below is an immediate offset from them
        const uint8_t* wsrc = sb + wrow * 1024 + wchunk * 16;
        const int qw0 = cc.kb * (kSBK / 256);
        const uint4* fb = frag + qw0 * (32 * M) + lane;
        const float4* cb = fsc + qw0 * (2 * M) + g;
#pragma unroll
        for (int qwl = 0; qwl < kSBK / 256; ++qwl) {
            const uint4 wv = *reinterpret_cast<const uint4*>(wsrc + qwl * 128);
            if (lane < 8 * M) {
#pragma unroll
                for (int t = 0; t < 4; ++t) af[t] = fb[(qwl * 4 + t) * (8 * M)];
            }
            if (f_lane) f = cb[qwl * 2 * M];
            int acc[2][4];
            mma_s8u8_16832_z(acc[0], af[0], wv.x & 0x0F0F0F0Fu, (wv.x >> 4) & 0x0F0F0F0Fu);
            mma_s8u8_16832_z(acc[1], af[1], wv.y & 0x0F0F0F0Fu, (wv.y >> 4) & 0x0F0F0F0Fu);
            mma_s8u8_16832(acc[0], af[2], wv.z & 0x0F0F0F0Fu, (wv.z >> 4) & 0x0F0F0F0Fu);
            mma_s8u8_16832(acc[1], af[3], wv.w & 0x0F0F0F0Fu, (wv.w >> 4) & 0x0F0F0F0Fu);
            const int d0 = acc[0][0] + acc[1][0];   // half 0: A row g, B column (tig, 0)
            const int d1 = acc[0][3] + acc[1][3];   // half 1: A row g + 8, B column (tig, 1)
            float4 sz;
            if (SZ == kSzConst) sz = make_float4(s_const, z_const, s_const, z_const);
            else sz = wtable[qwl * kSR + tig];
            y = fmaf(sz.x, fmaf(f.x, static_cast<float>(d0), -sz.y * f.y), y);
            y = fmaf(sz.z, fmaf(f.z, static_cast<float>(d1), -sz.w * f.w), y);
        }
        __syncwarp();
        issue();
        ++nb_rb;
        const int rb = cc.rb;
        const bool rb_done = (cc.kb == a.nbs - 1) || (b == b_end - 1);
        advance(cc);
        if (rb_done) {
            finish(rb, nb_rb, y);
            y = 0.0f;
            nb_rb = 0;
        }
    }
    if (*abort_flag) {
        const unsigned long long t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 1000000ull) {
        }
    }
}

}  // namespace w4
