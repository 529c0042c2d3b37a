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

// One warp converts activation row m of window qw (256 k starting at
// k_first) into `block`, a slice's activation block: lane = 16 h + 4 t + tig
// converts the 8 activations k_first + 128 h + 32 tig + 8 t .. + 7 (zero past
// K).  `block` may be global (the prep kernel) or shared memory (the GEMV
// converting its own slice).
// The 8 activations of the lane (zero past K).
__device__ __forceinline__ uint4 xfrag_load(const uint16_t* __restrict__ X, int K, long long k_first, int m,
                                            int lane) {
    const int h = lane >> 4, t = (lane >> 2) & 3, tig = lane & 3;
    const long long k = k_first + h * 128 + 32 * tig + 8 * t;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (k < K) v = __ldg(reinterpret_cast<const uint4*>(X + static_cast<size_t>(m) * K + k));
    return v;
}

// Fixed point, digits and fold constants from the lane's 8 activations v.
// x' = round(x * 2^(140 - e)) with e the largest bf16 exponent of the lane's
// half (128 k); the power of two is exact in fp32 unless e < 14 (values
// below 2^-113), where the integer path below is used instead.  The digits
// are dh = floor((x' + 128) / 256) and dl = x' - 256 dh, so dl is in
// [-128, 127] and |dh| <= 64.
__device__ __forceinline__ void xfrag_store(uint4 v, int M, int nqw, int qw, int m, int lane, uint8_t* block) {
    const int h = lane >> 4, t = (lane >> 2) & 3, tig = lane & 3;
    const uint32_t r[4] = {v.x, v.y, v.z, v.w};
    // largest magnitude: bf16 bit patterns order like their magnitudes
    uint32_t mx = __vmaxu2(__vmaxu2(r[0] & 0x7FFF7FFFu, r[1] & 0x7FFF7FFFu), __vmaxu2(r[2] & 0x7FFF7FFFu, r[3] & 0x7FFF7FFFu));
    mx = max(mx & 0xFFFFu, mx >> 16);
    int emax = max(static_cast<int>(mx >> 7), 1);
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) emax = max(emax, __shfl_xor_sync(0xFFFFFFFFu, emax, o));
    int xf[8];
    if (emax >= 14) {
        const float scale = __int_as_float((267 - emax) << 23);   // 2^(140 - emax), exact
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t bits = (j & 1) ? (r[j >> 1] & 0xFFFF0000u) : (r[j >> 1] << 16);
            xf[j] = __float2int_rn(__uint_as_float(bits) * scale);
        }
    } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t bits = (j & 1) ? (r[j >> 1] >> 16) : (r[j >> 1] & 0xFFFFu);
            xf[j] = bf16_fixed_bits(bits, emax, kMFrac);
        }
    }
    int sum = 0;
    uint32_t dh[8], dl[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        sum += xf[j];
        const int hi = (xf[j] + 128) >> 8;
        dh[j] = static_cast<uint32_t>(hi);
        dl[j] = static_cast<uint32_t>(xf[j] - (hi << 8));
    }
    // bytes of elements 0,2,4,6 (even k) and 1,3,5,7 (odd k), low byte first
    auto pack4 = [](uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3) {
        return __byte_perm(__byte_perm(a0, a1, 0x0040), __byte_perm(a2, a3, 0x0040), 0x5410);
    };
    const uint32_t hi_e = pack4(dh[0], dh[2], dh[4], dh[6]), hi_o = pack4(dh[1], dh[3], dh[5], dh[7]);
    const uint32_t lo_e = pack4(dl[0], dl[2], dl[4], dl[6]), lo_o = pack4(dl[1], dl[3], dl[5], dl[7]);
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
    uint32_t* frag = reinterpret_cast<uint32_t*>(block);
    // lane (g = 2 m + p, tig) of mma t: {even h0, even h1, odd h0, odd h1}
    const size_t rec = (static_cast<size_t>(qw) * 4 + t) * (8 * M) + (2 * m) * 4 + tig;
    frag[rec * 4 + h] = hi_e;
    frag[rec * 4 + 2 + h] = hi_o;
    frag[(rec + 4) * 4 + h] = lo_e;
    frag[(rec + 4) * 4 + 2 + h] = lo_o;
    if ((lane & 15) == 0) {
        float* fs = reinterpret_cast<float*>(block + static_cast<size_t>(nqw) * M * 512);
        // 2^(emax - 140): a normal float unless emax < 14
        const float xs_exact = emax >= 14 ? __int_as_float((emax - 13) << 23) : ldexpf(1.0f, emax - 134 - kMFrac);
        const size_t f0 = (static_cast<size_t>(qw) * 2 * M + 2 * m) * 4 + 2 * h;   // p = 0
        fs[f0] = 256.0f * xs_exact;
        fs[f0 + 1] = 0.0f;
        fs[f0 + 4] = xs_exact;                                                     // p = 1
        fs[f0 + 5] = xs_exact * static_cast<float>(sum);
    }
}

__device__ __forceinline__ void xfrag_convert(const uint16_t* __restrict__ X, int M, int K, long long k_first,
                                              int nqw, int qw, int m, int lane, uint8_t* block) {
    xfrag_store(xfrag_load(X, K, k_first, m, lane), M, nqw, qw, m, lane, block);
}

// Prep kernel for shapes whose conversion is too much to repeat in every
// CTA: one warp per (slice, window, m).
__global__ void __launch_bounds__(256) gemv_xfrag_kernel(const uint16_t* __restrict__ X, int M, int K,
                                                         int TKC, int splits, uint8_t* __restrict__ out) {
    pdl_launch_dependents();
    const int nqw = TKC / 256;
    const long long unit = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    if (unit >= static_cast<long long>(splits) * nqw * M) return;   // whole warps
    const int m = static_cast<int>(unit % M);
    const long long sq = unit / M;
    const int slice = static_cast<int>(sq / nqw), qw = static_cast<int>(sq - static_cast<long long>(slice) * nqw);
    xfrag_convert(X, M, K, static_cast<long long>(slice) * TKC + qw * 256, nqw, qw, m, threadIdx.x & 31,
                  out + static_cast<size_t>(slice) * gemv_mma_xblock_bytes(M, TKC));
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
    b += static_cast<size_t>(warps) * 2 * kSR * M * 4;             // shared-row-block slots
    b += gemv_mma_xblock_bytes(M, TKC);
    b += static_cast<size_t>(warps) * stages * 8 + 8 + 16;
    return b;
}

// Arguments of gemv_mma_kernel.
struct GemvMmaArgs {
    const uint16_t* X;        // [M, K] bf16 (converted in the kernel when xblocks is null)
    const uint8_t* xblocks;   // [splits] activation blocks from gemv_xfrag_kernel, or null
    const __half* S;
    const __half* Z;
    const uint16_t* bias;
    uint16_t* Y;
    float* partial;           // [splits, M, N] when splits > 1
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

// Work split: each CTA of a slice takes a contiguous range of whole row
// blocks (balanced to within one row block), and its warps cut the CTA's
// boxes, row block major (box b = row block b / nbs, k box b % nbs), into
// one contiguous range each, equal to within one box; no warp waits for
// another until the end.  A row block one warp covers completely is written
// at once.  A row block shared by neighbouring warps goes through per-warp
// slots in shared memory: after the CTA's single barrier, the warp holding
// the row block's last box sums the slots in warp order, so the result does
// not depend on timing.
//
// Activations: with `xblocks` null every CTA converts its K slice of X into
// the fragment layout itself while its first weight boxes are in flight (the
// planner picks this when the conversion is a few units per warp); else the
// kernel is a programmatic dependent of gemv_xfrag_kernel and fetches the
// prepared block with one bulk copy.
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
    float* slots = reinterpret_cast<float*>(table + NW * kSR * 8);           // [warp][2][4 rows][M]
    uint8_t* xblk = reinterpret_cast<uint8_t*>(slots + NW * 2 * kSR * M);
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

    const int slice = blockIdx.x / a.cps, cta = blockIdx.x - (blockIdx.x / a.cps) * a.cps;
    const int rb_lo = static_cast<int>(static_cast<long long>(cta) * a.nrb / a.cps);
    const int rb_hi = static_cast<int>(static_cast<long long>(cta + 1) * a.nrb / a.cps);
    const int T = (rb_hi - rb_lo) * a.nbs;                       // boxes of this CTA
    auto wstart = [&](int ww) { return static_cast<int>(static_cast<long long>(ww) * T / NW); };
    auto warp_of = [&](int b) { return static_cast<int>((static_cast<long long>(b + 1) * NW - 1) / T); };
    const int b_begin = wstart(warp), b_end = wstart(warp + 1);
    int gshift = 0;
    if (GK == kGroupsPow2) gshift = __ffs(a.g) - 1;

    struct Cur {
        int b, rb, kb;   // CTA-local box, its row block (absolute) and k box
    };
    auto advance = [&](Cur& c) {
        ++c.b;
        if (++c.kb == a.nbs) {
            c.kb = 0;
            ++c.rb;
        }
    };
    const Cur start{b_begin, rb_lo + b_begin / a.nbs, b_begin - (b_begin / a.nbs) * a.nbs};
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
    if (a.xblocks == nullptr) {
        // this warp's activation units (at most 4: the planner's limit) are
        // loaded first, the ring is filled while they are in flight, and
        // the conversion runs while the first boxes are in flight
        constexpr int kMaxUnits = 4;
        const long long k_slice = static_cast<long long>(slice) * a.TKC;
        uint4 raw[kMaxUnits];
#pragma unroll
        for (int i = 0; i < kMaxUnits; ++i) {
            const int u = warp + i * NW;
            raw[i] = make_uint4(0u, 0u, 0u, 0u);
            if (u < nqw * M) raw[i] = xfrag_load(a.X, a.K, k_slice + (u / M) * 256, u - (u / M) * M, lane);
        }
        for (int b = 0; b < NS; ++b) issue();
#pragma unroll
        for (int i = 0; i < kMaxUnits; ++i) {
            const int u = warp + i * NW;
            if (u < nqw * M) xfrag_store(raw[i], M, nqw, u / M, u - (u / M) * M, lane, xblk);
        }
        __syncthreads();
    } else {
        // one stage of weights first; then, once the prep kernel is done,
        // the activation block (so that it does not queue behind the whole
        // ring); then the rest of the ring
        issue();
        pdl_wait();
        if (tid == 0 && T > 0) {
            mbar_arrive_expect_tx(xbar, xbytes);
            bulk_load_1d(xblk, a.xblocks + static_cast<size_t>(slice) * xbytes, xbytes, xbar);
        }
        for (int b = 1; b < NS; ++b) issue();
        if (T > 0) mbar_wait_bounded(xbar, 0, abort_flag, kErrTimeoutTmaFull);
    }

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

    // outputs: after the digit shuffle, lanes with even g < 2M hold
    // (m = g / 2, row tig) of the row block
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
        if (!(g & 1) && f_lane) {
            if (nb == a.nbs) {
                const int n = rb * kSR + tig;
                if (n < a.N) store(g >> 1, n, v);
            } else {
                slots[((warp * 2) + (rb == first_rb ? 0 : 1)) * (kSR * M) + tig * M + (g >> 1)] = v;
            }
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

    // row blocks shared by neighbouring warps: the warp with a shared row
    // block's last box adds the slots of all its contributors in warp order
    __syncthreads();
    if (b_begin < b_end) {
        const int last_rb = rb_lo + (b_end - 1) / a.nbs;
        for (int side = 0; side < 2; ++side) {
            const int rb = side ? last_rb : first_rb;
            if (side && rb == first_rb) break;
            const int lb0 = (rb - rb_lo) * a.nbs, lb1 = lb0 + a.nbs - 1;   // CTA-local boxes of rb
            const bool partial = b_begin > lb0 || b_end - 1 < lb1;
            if (!partial || warp_of(lb1) != warp) continue;
            if (lane < kSR * M) {
                const int r = lane / M, m = lane - (lane / M) * M;
                float s = 0.0f;
                for (int ww = warp_of(lb0); ww <= warp; ++ww) {
                    const int ws = wstart(ww);
                    if (ws == wstart(ww + 1)) continue;
                    const int sslot = (rb_lo + ws / a.nbs == rb) ? 0 : 1;
                    s += slots[(ww * 2 + sslot) * (kSR * M) + r * M + m];
                }
                const int n = rb * kSR + r;
                if (n < a.N) store(m, n, s);
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
