// Forward GEMV for M <= 4 whose integer dot products run on the tensor
// pipe (mma.sync m16n8k32, u8 x s8 -> s32), for group lengths that are a
// multiple of 128 (or one group per row).
//
// Stream.  A producer warp walks the CTA's 16-row blocks along K and brings
// each 16 rows x 2048 k piece (16 rows x 1 KB of packed words, one TMA box)
// and its scales and zeros into a CTA-wide ring of stages.  Sixteen consumer
// warps share every stage: warp w takes granule w (k = 128 w .. 128 w + 127
// of the stage) of all 16 rows.  Row segments of 1 KB keep DRAM pages busy,
// and the per-stage bookkeeping is paid once per 16 KB, not once per warp.
//
// Arithmetic.  One mma multiplies 16 weight rows by 32 k:
//   A (16 x 32, u8)  the 4-bit codes, one per byte: A row r is weight row r
//                    of the stage.  Lane (g, tig) holds four consecutive
//                    packed words of rows g and g + 8 (words 4 tig .. 4 tig + 3
//                    of the granule).  The even codes of a word are
//                    w & 0x0F0F0F0F, the odd ones w & 0xF0F0F0F0 (16 q, still
//                    a byte), so four mma cover the granule: the even and the
//                    odd codes of words {0, 1} and of words {2, 3}.
//   B (32 x 8, s8)   the activations in 16-bit fixed point per 128-k granule
//                    (scaled by the granule's largest bf16 exponent), split
//                    into a high and a low signed digit: column 2 m + p is
//                    digit p of activation row m, so one mma serves any M <= 4.
//   D (16 x 8, s32)  exact sums over the granule: lane (g, tig) holds rows g
//                    and g + 8 for m = tig, digits 0 and 1, separately for the
//                    even codes (D_e) and the odd ones (D_o, 16 times larger).
// Per granule each lane folds
//   16 V = 16 (256 D_e,0 + D_e,1) + 256 D_o,0 + D_o,1   (= 16 sum_k x' q)
//   y   += s * ((xs / 16) * 16 V - z * xs * sum_k x')
// with xs = 2^(e - 140), e the granule's largest bf16 exponent, so y
// accumulates s * sum_k x (q - z) for its two rows.
//
// Output.  At the end of a row block each consumer warp leaves its sums in
// shared memory and moves on; a reducer warp adds the sixteen in a fixed
// order (so results do not depend on timing), then biases and rounds once,
// or writes fp32 partials when K is split into slices.
#pragma once

#include "gemv_stream.cuh"

namespace w4 {

constexpr int kMFrac = 6;          // fixed-point bits below the granule's leading binade
constexpr int kMR = 16;            // weight rows per stage (the mma's A rows)
constexpr int kMK = 2048;          // k per stage
constexpr int kMW = 16;            // consumer warps: one 128-k granule of each stage apiece
constexpr int kMThreads = (kMW + 2) * 32;  // + the producer warp and the reducer warp
constexpr int kMWBytes = kMR * kMK / 2;    // 16 KB of packed weights per stage
constexpr int kMRedStride = 68;            // floats per warp in the row-block reduction (64 + pad)

// One slice's activation block: the B fragments [granule][2 halves][8 M
// lanes][16 bytes] (lane 4 (2 m + p) + tig; half 0 holds words 0..3 of the
// lane's 8-word record, half 1 words 4..7), then the fold constants
// [granule][M] float2 {xs / 16, xs * sum x'}.
__host__ __device__ inline size_t gemv_mma_xfrag_bytes(int M, int TKC) {
    return static_cast<size_t>(TKC) / 128 * M * 256;
}
__host__ __device__ inline size_t gemv_mma_xblock_bytes(int M, int TKC) {
    return static_cast<size_t>(TKC) / 128 * M * (256 + 8);
}

// A conversion unit is 256 k of one activation row: lane = 16 h + 4 t + tig
// converts the 8 activations k_first + 128 h + 32 tig + 8 t .. + 7 (zero past
// K), i.e. chunk t of B lane tig's 32 k in granule h of the unit.
__device__ __forceinline__ uint4 xfrag_load(const uint16_t* __restrict__ X, int K, long long k_first, int m,
                                            int lane) {
    const int h = lane >> 4, t = (lane >> 2) & 3, tig = lane & 3;
    const long long k = k_first + h * 128 + 32 * tig + 8 * t;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (k < K) v = __ldg(reinterpret_cast<const uint4*>(X + static_cast<size_t>(m) * K + k));
    return v;
}

// Fixed point, digits and fold constants from the lane's 8 activations v,
// stored into `block` (global for the prep kernel, shared when the GEMV
// converts its own slice) for unit qw of activation row m; ngran is the
// slice's number of granules.
// x' = round(x * 2^(140 - e)) with e the largest bf16 exponent of the
// granule; the power of two is exact in fp32 unless e < 14 (values below
// 2^-113), where the integer path is used instead.  The digits are
// dh = floor((x' + 128) / 256) and dl = x' - 256 dh: dl is in [-128, 127]
// and |dh| <= 64.
__device__ __forceinline__ void xfrag_store(uint4 v, int M, int ngran, int qw, int m, int lane, uint8_t* block) {
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
    // the 8-word record of B lane (2 m + p, tig) is {e0.b0, e0.b1, o0.b0,
    // o0.b1, e1.b0, e1.b1, o1.b0, o1.b1}: chunk t fills word
    // 4 (t >> 1) + (t & 1) (even k) and 4 (t >> 1) + 2 + (t & 1) (odd k)
    const size_t gran = static_cast<size_t>(qw) * 2 + h;
    uint32_t* half = reinterpret_cast<uint32_t*>(block + (gran * 2 + (t >> 1)) * (8 * M * 16));
    const int l_hi = (2 * m) * 4 + tig, l_lo = l_hi + 4;
    half[l_hi * 4 + (t & 1)] = hi_e;
    half[l_hi * 4 + 2 + (t & 1)] = hi_o;
    half[l_lo * 4 + (t & 1)] = lo_e;
    half[l_lo * 4 + 2 + (t & 1)] = lo_o;
    if ((lane & 15) == 0) {
        float2* fc = reinterpret_cast<float2*>(block + static_cast<size_t>(ngran) * M * 256);
        // 2^(emax - 140): a normal float unless emax < 14
        const float xs_exact = emax >= 14 ? __int_as_float((emax - 13) << 23) : ldexpf(1.0f, emax - 134 - kMFrac);
        fc[gran * M + m] = make_float2(xs_exact * 0.0625f, xs_exact * static_cast<float>(sum));
    }
}

// Prep kernel for shapes whose conversion is too much to repeat in every
// CTA: one warp per (slice, unit of 256 k, m).
__global__ void __launch_bounds__(256) gemv_xfrag_kernel(const uint16_t* __restrict__ X, int M, int K,
                                                         int TKC, int splits, uint8_t* __restrict__ out) {
    pdl_launch_dependents();
    const int nqw = TKC / 256;
    const long long unit = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    if (unit >= static_cast<long long>(splits) * nqw * M) return;   // whole warps
    const int m = static_cast<int>(unit % M);
    const long long sq = unit / M;
    const int slice = static_cast<int>(sq / nqw), qw = static_cast<int>(sq - static_cast<long long>(slice) * nqw);
    const int lane = threadIdx.x & 31;
    xfrag_store(xfrag_load(X, K, static_cast<long long>(slice) * TKC + qw * 256, m, lane), M, TKC / 128, qw, m,
                lane, out + static_cast<size_t>(slice) * gemv_mma_xblock_bytes(M, TKC));
}

// D = A B + C with A the u8 weight codes and B the s8 activation digits.
__device__ __forceinline__ void mma_u8s8_16832(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// How the scales and zeros reach a stage:
//   kSzConst  one scale and zero for the whole matrix (global mode): read
//             once per thread, no per-stage data;
//   kSzTma2d  groupwise with G % 8 == 0: a TMA box of the stage's rows x 16
//             groups of S and of Z, starting at the 8-aligned group at or
//             below the stage's first group;
//   kSzTma1d  one group per row: a TMA box of the rows' values (S and Z seen
//             as one-row 2-D tensors);
//   kSzCopy   anything else: 4-byte cp.async copies by the producer warp,
//             tracked by the same barrier.
enum SzKind { kSzConst = 0, kSzTma2d = 1, kSzTma1d = 2, kSzCopy = 3 };

// Shared-memory footprint of a stage: 16 KB of weights, then S and Z
// (tiled TMA writes start on 128-byte boundaries).
__host__ __device__ inline int gemv_mma_sz_bytes(int sz, int szw) {
    return sz == kSzTma2d ? 2 * kMR * 16 * 2 : sz == kSzTma1d ? 2 * 128 : sz == kSzCopy ? 2 * kMR * szw * 4 : 0;
}
__host__ __device__ inline int gemv_mma_stage_bytes(int sz, int szw) {
    return (kMWBytes + gemv_mma_sz_bytes(sz, szw) + 127) / 128 * 128;
}
__host__ __device__ inline size_t gemv_mma_smem_bytes(int M, int TKC, int stages, int sz, int szw) {
    size_t b = 1024;                                                   // alignment slack
    b += static_cast<size_t>(stages) * gemv_mma_stage_bytes(sz, szw);
    b += (gemv_mma_xblock_bytes(M, TKC) + 15) / 16 * 16;
    b += static_cast<size_t>(2) * kMW * kMRedStride * 4;               // row-block reduction, 2 buffers
    b += static_cast<size_t>(stages) * 16 + 32 + 8 + 16;               // barriers, abort flag
    return b;
}
// Scale / zero words per row and stage on the copy path: the groups a
// stage touches, plus one half for the 4-byte alignment, rounded up.
__host__ __device__ inline int gemv_mma_sz_words(int g) { return ((kMK + g - 1) / g + 3) / 2; }

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
    int TKC;                  // k per slice (a whole number of stages)
    int splits;               // slices; CTA c works on slice c / cps
    int nks;                  // stages per row block and slice
    int nrb;                  // row blocks (16 rows each)
    int cps;                  // CTAs per slice
    int stages;               // ring depth
    int szw;                  // copy path: scale / zero words per row and stage
    long long sz_total;       // halves in each of S and Z (N * sz_row, or 1)
};

// Work split: each CTA of a slice takes a contiguous range of whole row
// blocks (balanced to within one row block) and walks them row block by row
// block, stage by stage along its K slice.
//
// Activations: with `xblocks` null every CTA converts its K slice of X into
// the fragment layout itself while the producer fills the ring (the planner
// picks this when the conversion is at most a few units per warp); else the
// kernel is a programmatic dependent of gemv_xfrag_kernel and fetches the
// prepared block with one bulk copy.
template <int M, int GK, int SZ>
__global__ void __launch_bounds__(kMThreads, 1)
    gemv_mma_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap smap,
                    const __grid_constant__ CUtensorMap zmap, const GemvMmaArgs a) {
    static_assert(M >= 1 && M <= 4, "M");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int NS = a.stages;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
    const int g = lane >> 2, tig = lane & 3;
    const int ngran = a.TKC / 128;
    const uint32_t xbytes = static_cast<uint32_t>(gemv_mma_xblock_bytes(M, a.TKC));
    const int SB = gemv_mma_stage_bytes(SZ, a.szw);
    constexpr int kSzTx = SZ == kSzTma2d ? 2 * kMR * 16 * 2 : SZ == kSzTma1d ? 2 * kMR * 2 : 0;
    uint8_t* ring = base;                                                   // [stage][SB]
    uint8_t* xblk = ring + NS * SB;                                         // fragments, then constants
    float* red = reinterpret_cast<float*>(xblk + ((xbytes + 15) & ~15u));   // [2][warp][kMRedStride]
    uint64_t* full = reinterpret_cast<uint64_t*>(red + 2 * kMW * kMRedStride);
    uint64_t* empty = full + NS;
    uint64_t* rfull = empty + NS;              // [2] a row block's 16 warp sums are in
    uint64_t* rempty = rfull + 2;              // [2] the reducer is done with a buffer
    uint64_t* xbar = rempty + 2;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(xbar + 1);

    if (tid == 0) {
        for (int i = 0; i < NS; ++i) {
            // a stage completes on the elected lane's expect-tx arrival and its
            // bytes; the copy path adds one cp.async arrival per producer lane
            mbar_init(&full[i], SZ == kSzCopy ? 33 : 1);
            mbar_init(&empty[i], kMW);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&rfull[i], kMW);
            mbar_init(&rempty[i], 1);
        }
        mbar_init(xbar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (tid == kMW * 32) {
        tma_prefetch_desc(&wmap);
        if (SZ == kSzTma2d || SZ == kSzTma1d) {
            tma_prefetch_desc(&smap);
            tma_prefetch_desc(&zmap);
        }
    }
    __syncthreads();
    // Programmatic dependent launch: the next kernel in the stream may start
    // its own prologue as SMs free up.  This kernel itself was launched as a
    // dependent of the work before it, so it touches no global memory until
    // that work is complete -- except, after a prep kernel (which started
    // only once everything before it was done), the weights, which no kernel
    // in between writes.
    pdl_launch_dependents();
    if (a.xblocks == nullptr) pdl_wait();

    const int slice = blockIdx.x / a.cps, cta = blockIdx.x - (blockIdx.x / a.cps) * a.cps;
    const int rb_lo = static_cast<int>(static_cast<long long>(cta) * a.nrb / a.cps);
    const int rb_hi = static_cast<int>(static_cast<long long>(cta + 1) * a.nrb / a.cps);
    const int items = (rb_hi - rb_lo) * a.nks;
    const int k_slice = slice * a.TKC;
    int gshift = 0;
    if (GK == kGroupsPow2) gshift = __ffs(a.g) - 1;
    auto group_of = [&](int k) {
        if (GK == kGroupsOne) return 0;
        if (GK == kGroupsPow2) return k >> gshift;
        return k / a.g;
    };

    if (warp == kMW) {
        // ------------------------------------------------------ producer
        int rb = rb_lo, ks = 0;
        int s = 0;
        uint32_t round = 0;                      // completed passes over the ring
        for (int it = 0; it < items; ++it) {
            if (round > 0) {
                const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&empty[s], (round - 1) & 1u, abort_flag,
                                                                          kErrTimeoutEmpty));
                if (!ok) break;
            }
            uint8_t* sd = ring + s * SB;
            const int k0 = k_slice + ks * kMK, row0 = rb * kMR;
            if (SZ == kSzCopy) {
                // lane -> (array, row): the row's szw words around the stage's
                // groups, zero-filled past the end of S / Z
                const int arr = lane >> 4, r = lane & 15;
                const long long h0 = (static_cast<long long>(row0 + r) * a.sz_row + group_of(k0)) & ~1ll;
                uint32_t* dst = reinterpret_cast<uint32_t*>(sd + kMWBytes) + (arr * kMR + r) * a.szw;
                const __half* src = arr ? a.Z : a.S;
                for (int q = 0; q < a.szw; ++q) {
                    const long long hh = h0 + 2 * q;
                    const long long avail = a.sz_total - hh;
                    const uint32_t bytes = avail >= 2 ? 4u : (avail == 1 ? 2u : 0u);
                    cp_async_4(dst + q, src + (bytes ? hh : 0), bytes);
                }
                cp_async_arrive_noinc(&full[s]);
            }
            if (SZ == kSzTma2d) {
                const int x = group_of(k0) & ~7;
                tma_issue_elected<3>(&full[s], kMWBytes + kSzTx, sd, &wmap, k0 / 8, row0, sd + kMWBytes, &smap, x,
                                     row0, sd + kMWBytes + kMR * 32, &zmap, x, row0);
            } else if (SZ == kSzTma1d) {
                tma_issue_elected<3>(&full[s], kMWBytes + kSzTx, sd, &wmap, k0 / 8, row0, sd + kMWBytes, &smap, row0,
                                     0, sd + kMWBytes + 128, &zmap, row0, 0);
            } else {
                tma_issue_elected<1>(&full[s], kMWBytes, sd, &wmap, k0 / 8, row0);
            }
            if (it == 0 && a.xblocks != nullptr) {
                // the prepared activation block right after the first stage,
                // so that it does not queue behind the whole ring
                pdl_wait();
                if (lane == 0) {
                    // every CTA of the slice copies the same block: in 8
                    // pieces, each CTA starting at a different one
                    mbar_arrive_expect_tx(xbar, xbytes);
                    const uint8_t* src = a.xblocks + static_cast<size_t>(slice) * xbytes;
                    const uint32_t piece = (xbytes / 8 + 15) & ~15u;
                    for (int q = 0; q < 8; ++q) {
                        const uint32_t o = ((q + blockIdx.x) & 7) * piece;
                        if (o < xbytes) bulk_load_1d(xblk + o, src + o, min(piece, xbytes - o), xbar);
                    }
                }
                __syncwarp();
            }
            if (++ks == a.nks) {
                ks = 0;
                ++rb;
            }
            if (++s == NS) {
                s = 0;
                ++round;
            }
        }
    } else if (warp == kMW + 1) {
        // ------------------------------------------------------ reducer
        // adds the 16 consumer warps' sums of each row block in warp order
        // (so results do not depend on timing), then biases and rounds once,
        // or writes fp32 partials when K is split into slices
        const int nrows = rb_hi - rb_lo;
        for (int i = 0; i < nrows; ++i) {
            const int b = i & 1;
            if (!mbar_wait_bounded(&rfull[b], (i >> 1) & 1u, abort_flag, kErrTimeoutTmaFull)) break;
            const float* rbuf = red + b * (kMW * kMRedStride);
            const int rb = rb_lo + i;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int v = lane + 32 * h;            // output (row r, m)
                const int r = v >> 2, m = v & 3;
                const int src = ((r & 7) * 4 + m) * 2 + (r >> 3);
                float sum = 0.f;
#pragma unroll
                for (int w = 0; w < kMW; ++w) sum += rbuf[w * kMRedStride + src];
                const int n = rb * kMR + r;
                if (m < M && n < a.N) {
                    if (a.splits == 1) {
                        float o = sum;
                        if (a.bias) o += bf16_bits_to_float(a.bias[n]);
                        a.Y[static_cast<size_t>(m) * a.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(o));
                    } else {
                        a.partial[(static_cast<size_t>(slice) * M + m) * a.N + n] = sum;
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&rempty[b]);
        }
    } else {
        // ------------------------------------------------------ consumers
        if (a.xblocks == nullptr) {
            // this warp's activation units (at most 4: the planner's limit)
            // are loaded, converted and stored while the ring fills.  Every
            // CTA reads all of X; each starts at a different unit, so that
            // the CTAs do not all queue on the same L2 lines at once.
            constexpr int kMaxUnits = 4;
            const int nunits = (a.TKC / 256) * M;
            const int rot = static_cast<int>((static_cast<unsigned>(blockIdx.x) * 7u) % static_cast<unsigned>(nunits));
            uint4 raw[kMaxUnits];
#pragma unroll
            for (int i = 0; i < kMaxUnits; ++i) {
                int u = warp + i * kMW;
                raw[i] = make_uint4(0u, 0u, 0u, 0u);
                if (u < nunits) {
                    u = u + rot < nunits ? u + rot : u + rot - nunits;
                    raw[i] = xfrag_load(a.X, a.K, k_slice + (u / M) * 256, u - (u / M) * M, lane);
                }
            }
#pragma unroll
            for (int i = 0; i < kMaxUnits; ++i) {
                int u = warp + i * kMW;
                if (u < nunits) {
                    u = u + rot < nunits ? u + rot : u + rot - nunits;
                    xfrag_store(raw[i], M, ngran, u / M, u - (u / M) * M, lane, xblk);
                }
            }
            named_barrier_sync(1, kMW * 32);
        } else if (items > 0) {
            // the producer fetches the prepared block once the prep kernel is done
            mbar_wait_bounded(xbar, 0, abort_flag, kErrTimeoutTmaFull);
        }

        const bool b_lane = lane < 8 * M;        // lanes whose B columns hold activations
        const int mf = min(tig, M - 1);          // fold constants of activation row m = tig
        float s_const = 0.f, z_const = 0.f;
        if (SZ == kSzConst) {
            s_const = __half2float(a.S[0]);
            z_const = __half2float(a.Z[0]);
        }
        const uint4* xb4 = reinterpret_cast<const uint4*>(xblk);
        const float2* fcs = reinterpret_cast<const float2*>(xblk + static_cast<size_t>(ngran) * M * 256);
        float y0 = 0.f, y1 = 0.f;                // rows g and g + 8 of the row block, m = tig
        int rb = rb_lo, ks = 0, rbi = 0;
        int s = 0;
        uint32_t phase = 0;
        for (int it = 0; it < items; ++it) {
            __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&full[s], phase, abort_flag, kErrTimeoutTmaFull));
            const uint8_t* sb = ring + s * SB;
            const int gl = ks * (kMK / 128) + warp;               // granule within the slice
            const int kg = k_slice + gl * 128;                    // its first k
            if (kg < a.K) {
                const uint8_t* wrow = sb + g * 1024 + warp * 64 + tig * 16;
                const uint4 wa = *reinterpret_cast<const uint4*>(wrow);
                const uint4 wb = *reinterpret_cast<const uint4*>(wrow + 8 * 1024);
                uint4 b0 = make_uint4(0u, 0u, 0u, 0u), b1 = b0;
                if (b_lane) {
                    const uint4* xg = xb4 + static_cast<size_t>(gl) * (16 * M);
                    b0 = xg[lane];
                    b1 = xg[8 * M + lane];
                }
                const float2 fc = fcs[gl * M + mf];
                int de[4] = {0, 0, 0, 0}, dd[4] = {0, 0, 0, 0};
                constexpr uint32_t kLo = 0x0F0F0F0Fu, kHi = 0xF0F0F0F0u;
                mma_u8s8_16832(de, wa.x & kLo, wb.x & kLo, wa.y & kLo, wb.y & kLo, b0.x, b0.y);
                mma_u8s8_16832(dd, wa.x & kHi, wb.x & kHi, wa.y & kHi, wb.y & kHi, b0.z, b0.w);
                mma_u8s8_16832(de, wa.z & kLo, wb.z & kLo, wa.w & kLo, wb.w & kLo, b1.x, b1.y);
                mma_u8s8_16832(dd, wa.z & kHi, wb.z & kHi, wa.w & kHi, wb.w & kHi, b1.z, b1.w);
                // scales and zeros of rows g and g + 8 for this granule's group
                float s0, z0, s1, z1;
                if (SZ == kSzConst) {
                    s0 = s1 = s_const;
                    z0 = z1 = z_const;
                } else {
                    const __half* sh = reinterpret_cast<const __half*>(sb + kMWBytes);
                    const int grp = group_of(kg);
                    if (SZ == kSzTma2d) {
                        const int gi = grp - (group_of(k_slice + ks * kMK) & ~7);
                        s0 = __half2float(sh[g * 16 + gi]);
                        s1 = __half2float(sh[(g + 8) * 16 + gi]);
                        z0 = __half2float(sh[kMR * 16 + g * 16 + gi]);
                        z1 = __half2float(sh[kMR * 16 + (g + 8) * 16 + gi]);
                    } else if (SZ == kSzTma1d) {
                        s0 = __half2float(sh[g]);
                        s1 = __half2float(sh[g + 8]);
                        z0 = __half2float(sh[64 + g]);
                        z1 = __half2float(sh[64 + g + 8]);
                    } else {
                        // row r's words start at half (row r, first group)
                        // rounded down to even
                        const int fg = group_of(k_slice + ks * kMK);
                        const int row0 = rb * kMR;
                        const int o0 = grp - fg + ((((row0 + g) & a.sz_row) ^ fg) & 1);
                        const int o1 = grp - fg + ((((row0 + g + 8) & a.sz_row) ^ fg) & 1);
                        const int w2 = 2 * a.szw;
                        s0 = __half2float(sh[g * w2 + o0]);
                        s1 = __half2float(sh[(g + 8) * w2 + o1]);
                        z0 = __half2float(sh[(kMR + g) * w2 + o0]);
                        z1 = __half2float(sh[(kMR + g + 8) * w2 + o1]);
                    }
                }
                const int v0 = (de[0] * 256 + de[1]) * 16 + dd[0] * 256 + dd[1];
                const int v1 = (de[2] * 256 + de[3]) * 16 + dd[2] * 256 + dd[3];
                y0 = fmaf(s0, fmaf(fc.x, static_cast<float>(v0), -z0 * fc.y), y0);
                y1 = fmaf(s1, fmaf(fc.x, static_cast<float>(v1), -z1 * fc.y), y1);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            if (++s == NS) {
                s = 0;
                phase ^= 1u;
            }
            if (++ks == a.nks) {
                // row block done: hand this warp's sums to the reducer (its
                // buffer is free once the reducer finished the row block two
                // before)
                const int b = rbi & 1;
                if (rbi >= 2)
                    __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&rempty[b], ((rbi >> 1) - 1) & 1u, abort_flag,
                                                              kErrTimeoutTmaFull));
                float* rbuf = red + b * (kMW * kMRedStride);
                reinterpret_cast<float2*>(rbuf + warp * kMRedStride)[lane] = make_float2(y0, y1);
                __syncwarp();
                if (lane == 0) mbar_arrive(&rfull[b]);
                y0 = 0.f;
                y1 = 0.f;
                ks = 0;
                ++rb;
                ++rbi;
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
