// Forward GEMV for M <= 4 with its dot products on the tensor pipe
// (mma.sync m16n8k16, bf16 operands, fp32 accumulation), for K and the group
// length multiples of 32 (or one group per row).
//
// Stream.  A producer warp walks the CTA's 16-row blocks along K and brings
// each 16 rows x 2048 k piece (16 rows x 1 KB of packed words, one TMA box)
// and its scales and zeros into a CTA-wide ring of stages.  Sixteen consumer
// warps share every stage: warp w takes granule w (k = 128 w .. 128 w + 127
// of the stage) of all 16 rows.  Row segments of 1 KB keep DRAM pages busy,
// and the per-stage bookkeeping is paid once per 16 KB, not once per warp.
//
// Arithmetic.  One mma multiplies 16 weight rows by 16 k:
//   A (16 x 16, bf16)  the exact differences q - z.  For a packed word w,
//                      ((w >> 4 s) & 0x000F000F) | 0x43004300 is the bf16 pair
//                      (128 + q_s, 128 + q_s+4) exactly, and one bf16x2
//                      subtraction of (128 + z, 128 + z) leaves
//                      (q_s - z, q_s+4 - z): every value is an integer below
//                      2^8, so nothing rounds.
//   B (16 x 8, bf16)   the activations themselves: column m is activation
//                      row m (columns M..7 are zero).  The k order inside an
//                      mma is free, so each lane's A registers come straight
//                      from its packed words and B is X permuted to match.
//   D (16 x 8, fp32)   sum over k of (q - z) x: each product is exact in fp32
//                      (a 5-bit integer times an 8-bit significand) and the
//                      tensor pipe adds them in fp32.
// Lane (gid, tig) holds rows gid and gid + 8; per group it folds
// y += s * D for its two rows and activation rows m = 2 tig, 2 tig + 1.
//
// Which packed words a lane holds.  The four tig lanes of a row hold four
// words each (32 of the granule's 128 k).  Every mma step takes word i of
// all four lanes, so the four words of one step must lie in one group:
//   kCls128  (g a multiple of 128, or one group per row) words 4 tig .. +3,
//            one 16-byte load per row;
//   kCls64   (g a multiple of 64) words 2 tig, 2 tig + 1 of each 64-k half;
//   kCls32   (g a multiple of 32) word tig of each 32-k quarter.
// Word i gives two steps: nibbles (0, 4 | 1, 5) and (2, 6 | 3, 7), and B
// lane (m, tig) holds x at the same k: (x0, x4 | x1, x5), (x2, x6 | x3, x7)
// of the 8 activations under the word.
//
// Activations.  Warp w only ever reads the granules w, w + 16, ... of its K
// slice, so each warp converts its own granules (16-byte loads of X and
// byte permutes) into shared memory before its first stage, while the
// producer fills the ring; no other warp reads them and no CTA barrier is
// needed.
//
// Output.  At the end of a row block each consumer warp leaves its sums in
// shared memory and moves on; a reducer warp adds the sixteen in a fixed
// order (so results do not depend on timing), then biases and rounds once,
// or writes fp32 partials when K is split into slices.
#pragma once

#include "gemv.cuh"

namespace w4 {

constexpr int kMR = 16;                    // weight rows per stage (the mma's A rows)
constexpr int kMK = 2048;                  // k per stage
constexpr int kMW = 16;                    // consumer warps: one 128-k granule of each stage apiece
constexpr int kMThreads = (kMW + 2) * 32;  // + the producer warp and the reducer warp
constexpr int kMWBytes = kMR * kMK / 2;    // 16 KB of packed weights per stage
constexpr int kMRedStride = 68;            // floats per warp in the row-block reduction (64 + pad)

// Word layouts of a lane's four packed words in a 16-word granule row.
enum WordClass { kCls128 = 0, kCls64 = 1, kCls32 = 2 };

template <int CLS>
__host__ __device__ __forceinline__ int cls_word(int i, int tig) {
    return CLS == kCls128 ? 4 * tig + i : CLS == kCls64 ? 8 * (i >> 1) + 2 * tig + (i & 1) : 4 * i + tig;
}
// k blocks of a granule that each lie in one group (word i is in block
// i / (4 / blocks)).
template <int CLS>
__host__ __device__ constexpr int cls_blocks() {
    return CLS == kCls128 ? 1 : CLS == kCls64 ? 2 : 4;
}

// One slice's activation fragments: [warp][j < nks][i < 4][lb < 4 M] uint4,
// the B registers of lane lb = 4 m + tig for the two steps of word i of the
// warp's granule 16 j + w.  Exactly the bytes of X's slice.
__host__ __device__ inline size_t gemv_mma_xblock_bytes(int M, int TKC) {
    return static_cast<size_t>(TKC) * 2 * M;
}

// Converts this warp's granules j < nks (granule 16 j + warp of the slice):
// unit u = (4 j + i) * 4 M + lb is one 16-byte load of x[m][k .. k + 7],
// k the first k of word cls_word(i, tig) (zeros past K), and one 16-byte
// store of (x0 x4 | x1 x5 | x2 x6 | x3 x7).  Loads go out eight at a time.
template <int M, int CLS>
__device__ __forceinline__ void convert_x_block(const uint16_t* __restrict__ X, int K, int k_slice, int nks,
                                                int warp, int lane, uint4* dst) {
    constexpr int kLB = 4 * M;
    const int units = nks * 4 * kLB;
    for (int u0 = 0; u0 < units; u0 += 32 * 8) {
        uint4 v[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            const int u = u0 + 32 * t + lane;
            v[t] = make_uint4(0u, 0u, 0u, 0u);
            if (u < units) {
                const int lb = u % kLB, ji = u / kLB;
                const int i = ji & 3, j = ji >> 2;
                const int m = lb >> 2, tig = lb & 3;
                const int k = k_slice + (16 * j + warp) * 128 + 8 * cls_word<CLS>(i, tig);
                if (k < K) v[t] = __ldg(reinterpret_cast<const uint4*>(X + static_cast<size_t>(m) * K + k));
            }
        }
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            const int u = u0 + 32 * t + lane;
            if (u < units)
                dst[u] = make_uint4(prmt(v[t].x, v[t].z, 0x5410u), prmt(v[t].x, v[t].z, 0x7632u),
                                    prmt(v[t].y, v[t].w, 0x5410u), prmt(v[t].y, v[t].w, 0x7632u));
        }
    }
}

// D = A B + C, bf16 operands, fp32 accumulators.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// (v, v) as a bf16 pair (v an integer below 2^8 here, so exact).
__device__ __forceinline__ uint32_t bf16x2_splat(float v) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %1;" : "=r"(r) : "f"(v));
    return r;
}

// The four A registers of one packed word: p[s] = (q_s - z, q_s+4 - z) as
// bf16, zz = (128 + z, 128 + z).
__device__ __forceinline__ void unpack_word_bf16(uint32_t w, uint32_t zz, uint32_t (&p)[4]) {
    p[0] = bf16x2_sub(lop3_and_or(w, 0x000F000Fu, 0x43004300u), zz);
    p[1] = bf16x2_sub(lop3_and_or(w >> 4, 0x000F000Fu, 0x43004300u), zz);
    p[2] = bf16x2_sub(lop3_and_or(w >> 8, 0x000F000Fu, 0x43004300u), zz);
    p[3] = bf16x2_sub(lop3_and_or(w >> 12, 0x000F000Fu, 0x43004300u), zz);
}

// The same registers for a fractional zero point, where q - z is not a
// bf16 value: (128 + q) - (128 + z) in fp32 (zo = 128 + z), rounded once to
// bf16.
__device__ __forceinline__ void unpack_word_bf16_rounded(uint32_t w, float zo, uint32_t (&p)[4]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float lo = __uint_as_float(lop3_and_or(w << (16 - 4 * i), 0x000F0000u, 0x43000000u));
        const float hi = __uint_as_float(lop3_and_or(w >> (4 * i), 0x000F0000u, 0x43000000u));
        p[i] = bf162_bits(__floats2bfloat162_rn(lo - zo, hi - zo));
    }
}

// How the scales and zeros reach a stage:
//   kSzConst  one scale and zero for the whole matrix (global mode): read
//             once per thread, no per-stage data;
//   kSzTma2d  groupwise with G % 8 == 0: a TMA box of the stage's rows x
//             `szw` groups of S and of Z, starting at the 8-aligned group at
//             or below the stage's first group;
//   kSzTma1d  one group per row: a TMA box of the rows' values (S and Z seen
//             as one-row 2-D tensors);
//   kSzCopy   anything else: 4-byte cp.async copies by the producer warp,
//             `szw` words per row, tracked by the same barrier.
enum SzKind { kSzConst = 0, kSzTma2d = 1, kSzTma1d = 2, kSzCopy = 3 };

// Shared-memory footprint of a stage: 16 KB of weights, then S and Z
// (tiled TMA writes start on 128-byte boundaries).
__host__ __device__ inline int gemv_mma_sz_bytes(int sz, int szw) {
    return sz == kSzTma2d ? 2 * kMR * szw * 2 : sz == kSzTma1d ? 2 * 128 : sz == kSzCopy ? 2 * kMR * szw * 4 : 0;
}
__host__ __device__ inline int gemv_mma_stage_bytes(int sz, int szw) {
    return (kMWBytes + gemv_mma_sz_bytes(sz, szw) + 127) / 128 * 128;
}
__host__ __device__ inline size_t gemv_mma_smem_bytes(int M, int TKC, int stages, int sz, int szw) {
    size_t b = 1024;                                                   // alignment slack
    b += static_cast<size_t>(stages) * gemv_mma_stage_bytes(sz, szw);
    b += gemv_mma_xblock_bytes(M, TKC);
    b += static_cast<size_t>(2) * kMW * kMRedStride * 4;               // row-block reduction, 2 buffers
    b += static_cast<size_t>(stages) * 16 + 32 + 16;                   // barriers, abort flag
    return b;
}
// Scale / zero words per row and stage on the copy path: the groups a
// stage touches, plus one half for the 4-byte alignment, rounded up.
__host__ __device__ inline int gemv_mma_sz_words(int g) { return ((kMK + g - 1) / g + 3) / 2; }
// Groups per row of the 2-D scale / zero box: a stage's groups from the
// 8-aligned one at or below its first.
__host__ __device__ inline int gemv_mma_sz_box(int g) {
    if (kMK % g == 0 && (kMK / g) % 8 == 0) return kMK / g;
    return ((kMK + g - 1) / g + 1 + 7 + 7) / 8 * 8;
}

// Arguments of gemv_mma_kernel.
struct GemvMmaArgs {
    const uint16_t* X;        // [M, K] bf16
    const __half* S;
    const __half* Z;
    const uint16_t* bias;
    uint16_t* Y;
    float* partial;           // [splits, M, N] when splits > 1
    int N, K, g, G, sz_row;
    unsigned long long gmul;  // group of k = (k * gmul) >> gshift, exact for 0 <= k < 2^31
    int gshift;
    int TKC;                  // k per slice (a whole number of stages)
    int splits;               // slices; CTA c works on slice c / cps
    int nks;                  // stages per row block and slice
    int nrb;                  // row blocks (16 rows each)
    int cps;                  // CTAs per slice
    int stages;               // ring depth
    int szw;                  // 2-D box: groups per row; copy path: words per row and stage
    long long sz_total;       // halves in each of S and Z (N * sz_row, or 1)
    int fmt;                  // format flags: kFmtZeroFloat, kFmtMetaBf16
};

// Work split: each CTA of a slice takes a contiguous range of whole row
// blocks (balanced to within one row block) and walks them row block by row
// block, stage by stage along its K slice.
template <int M, int CLS, int SZ, bool FZ>
__global__ void __launch_bounds__(kMThreads, 1)
    gemv_mma_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap smap,
                    const __grid_constant__ CUtensorMap zmap, const GemvMmaArgs a) {
    static_assert(M >= 1 && M <= 4, "M");
    constexpr int NB = cls_blocks<CLS>();
    constexpr int kLB = 4 * M;                 // lanes whose B columns hold activations
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int NS = a.stages;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
    const int gid = lane >> 2, tig = lane & 3;
    const int SB = gemv_mma_stage_bytes(SZ, a.szw);
    const int kSzTx = SZ == kSzTma2d ? 2 * kMR * a.szw * 2 : SZ == kSzTma1d ? 2 * kMR * 2 : 0;
    uint8_t* ring = base;                                                   // [stage][SB]
    uint4* xblk = reinterpret_cast<uint4*>(ring + NS * SB);                 // activation fragments
    float* red = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(xblk) + gemv_mma_xblock_bytes(M, a.TKC));
    uint64_t* full = reinterpret_cast<uint64_t*>(red + 2 * kMW * kMRedStride);
    uint64_t* empty = full + NS;
    uint64_t* rfull = empty + NS;              // [2] a row block's 16 warp sums are in
    uint64_t* rempty = rfull + 2;              // [2] the reducer is done with a buffer
    volatile int* abort_flag = reinterpret_cast<volatile int*>(rempty + 2);

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
    // dependent of the work before it, so it reads no global memory until
    // that work is complete.
    pdl_launch_dependents();
    pdl_wait();

    const int slice = blockIdx.x / a.cps, cta = blockIdx.x - (blockIdx.x / a.cps) * a.cps;
    const int rb_lo = static_cast<int>(static_cast<long long>(cta) * a.nrb / a.cps);
    const int rb_hi = static_cast<int>(static_cast<long long>(cta + 1) * a.nrb / a.cps);
    const int items = (rb_hi - rb_lo) * a.nks;
    const int k_slice = slice * a.TKC;
    auto group_of = [&](int k) {
        return a.G == 1 ? 0 : static_cast<int>((static_cast<unsigned long long>(k) * a.gmul) >> a.gshift);
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
                                     row0, sd + kMWBytes + kMR * a.szw * 2, &zmap, x, row0);
            } else if (SZ == kSzTma1d) {
                tma_issue_elected<3>(&full[s], kMWBytes + kSzTx, sd, &wmap, k0 / 8, row0, sd + kMWBytes, &smap, row0,
                                     0, sd + kMWBytes + 128, &zmap, row0, 0);
            } else {
                tma_issue_elected<1>(&full[s], kMWBytes, sd, &wmap, k0 / 8, row0);
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
                float sum = 0.f;
#pragma unroll
                for (int w = 0; w < kMW; ++w) sum += rbuf[w * kMRedStride + v];
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
        uint4* xw = xblk + static_cast<size_t>(warp) * a.nks * 4 * kLB;   // this warp's fragments
        if (items > 0) convert_x_block<M, CLS>(a.X, a.K, k_slice, a.nks, warp, lane, xw);
        __syncwarp();

        const bool mbf = (a.fmt & kFmtMetaBf16) != 0;
        constexpr bool fz = FZ;     // a.fmt & kFmtZeroFloat, as a template argument
        float s_const = 0.f, zo_const = 0.f;
        uint32_t zz_const = 0u;
        if (SZ == kSzConst) {
            s_const = meta_to_float(a.S[0], mbf);
            zo_const = 128.0f + meta_to_float(a.Z[0], mbf);
            zz_const = bf16x2_splat(zo_const);
        }
        float y0a = 0.f, y0b = 0.f, y1a = 0.f, y1b = 0.f;   // rows gid / gid + 8, m = 2 tig / 2 tig + 1
        int rb = rb_lo, ks = 0, rbi = 0;
        int s = 0;
        uint32_t phase = 0;
        for (int it = 0; it < items; ++it) {
            const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&full[s], phase, abort_flag,
                                                                      kErrTimeoutTmaFull));
            if (!ok) break;
            const uint8_t* sb = ring + s * SB;
            const int k0 = k_slice + ks * kMK;                    // the stage's first k
            const int kg = k0 + warp * 128;                       // the warp's granule
            if (kg < a.K) {
                // ---- packed words of rows gid and gid + 8
                uint32_t wa[4], wb[4];
                const uint8_t* ra = sb + gid * 1024 + warp * 64;
                if (CLS == kCls128) {
                    const uint4 t0 = *reinterpret_cast<const uint4*>(ra + tig * 16);
                    const uint4 t1 = *reinterpret_cast<const uint4*>(ra + 8 * 1024 + tig * 16);
                    wa[0] = t0.x; wa[1] = t0.y; wa[2] = t0.z; wa[3] = t0.w;
                    wb[0] = t1.x; wb[1] = t1.y; wb[2] = t1.z; wb[3] = t1.w;
                } else if (CLS == kCls64) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint2 t0 = *reinterpret_cast<const uint2*>(ra + 32 * h + tig * 8);
                        const uint2 t1 = *reinterpret_cast<const uint2*>(ra + 8 * 1024 + 32 * h + tig * 8);
                        wa[2 * h] = t0.x; wa[2 * h + 1] = t0.y;
                        wb[2 * h] = t1.x; wb[2 * h + 1] = t1.y;
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        wa[i] = *reinterpret_cast<const uint32_t*>(ra + 16 * i + tig * 4);
                        wb[i] = *reinterpret_cast<const uint32_t*>(ra + 8 * 1024 + 16 * i + tig * 4);
                    }
                }
                // ---- activation fragments of the granule
                uint4 bq[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) bq[i] = make_uint4(0u, 0u, 0u, 0u);
                if (lane < kLB) {
                    const uint4* xq = xw + static_cast<size_t>(ks) * 4 * kLB + lane;
#pragma unroll
                    for (int i = 0; i < 4; ++i) bq[i] = xq[i * kLB];
                }
                // ---- scales and zeros of rows gid and gid + 8, per k block
                float sv[NB][2], zo[NB][2];
                uint32_t zz[NB][2];
#pragma unroll
                for (int b = 0; b < NB; ++b) {
                    float zv0, zv1;
                    if (SZ == kSzConst) {
                        sv[b][0] = sv[b][1] = s_const;
                        zz[b][0] = zz[b][1] = zz_const;
                        zo[b][0] = zo[b][1] = zo_const;
                        continue;
                    }
                    const __half* sh = reinterpret_cast<const __half*>(sb + kMWBytes);
                    if (SZ == kSzTma1d) {
                        sv[b][0] = meta_to_float(sh[gid], mbf);
                        sv[b][1] = meta_to_float(sh[gid + 8], mbf);
                        zv0 = meta_to_float(sh[64 + gid], mbf);
                        zv1 = meta_to_float(sh[64 + gid + 8], mbf);
                    } else {
                        const int grp = group_of(kg + b * (128 / NB));
                        const int fg = group_of(k0);
                        if (SZ == kSzTma2d) {
                            const int gi = grp - (fg & ~7);
                            const int w2 = a.szw;
                            sv[b][0] = meta_to_float(sh[gid * w2 + gi], mbf);
                            sv[b][1] = meta_to_float(sh[(gid + 8) * w2 + gi], mbf);
                            zv0 = meta_to_float(sh[kMR * w2 + gid * w2 + gi], mbf);
                            zv1 = meta_to_float(sh[kMR * w2 + (gid + 8) * w2 + gi], mbf);
                        } else {
                            // row r's words start at half (row r, first group)
                            // rounded down to even
                            const int row0 = rb * kMR;
                            const int o0 = grp - fg + ((((row0 + gid) & a.sz_row) ^ fg) & 1);
                            const int o1 = grp - fg + ((((row0 + gid + 8) & a.sz_row) ^ fg) & 1);
                            const int w2 = 2 * a.szw;
                            sv[b][0] = meta_to_float(sh[gid * w2 + o0], mbf);
                            sv[b][1] = meta_to_float(sh[(gid + 8) * w2 + o1], mbf);
                            zv0 = meta_to_float(sh[(kMR + gid) * w2 + o0], mbf);
                            zv1 = meta_to_float(sh[(kMR + gid + 8) * w2 + o1], mbf);
                        }
                    }
                    zo[b][0] = 128.0f + zv0;
                    zo[b][1] = 128.0f + zv1;
                    zz[b][0] = bf16x2_splat(zo[b][0]);
                    zz[b][1] = bf16x2_splat(zo[b][1]);
                }
                // ---- eight mma steps, one accumulator per k block
                float d[NB][4];
#pragma unroll
                for (int b = 0; b < NB; ++b) d[b][0] = d[b][1] = d[b][2] = d[b][3] = 0.f;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    constexpr int kPer = 4 / NB;
                    const int b = i / kPer;
                    uint32_t pa[4], pb[4];
                    if (!fz) {
                        unpack_word_bf16(wa[i], zz[b][0], pa);
                        unpack_word_bf16(wb[i], zz[b][1], pb);
                    } else {
                        unpack_word_bf16_rounded(wa[i], zo[b][0], pa);
                        unpack_word_bf16_rounded(wb[i], zo[b][1], pb);
                    }
                    mma_bf16_16816(d[b], pa[0], pb[0], pa[1], pb[1], bq[i].x, bq[i].y);
                    mma_bf16_16816(d[b], pa[2], pb[2], pa[3], pb[3], bq[i].z, bq[i].w);
                }
#pragma unroll
                for (int b = 0; b < NB; ++b) {
                    y0a = fmaf(sv[b][0], d[b][0], y0a);
                    y0b = fmaf(sv[b][0], d[b][1], y0b);
                    y1a = fmaf(sv[b][1], d[b][2], y1a);
                    y1b = fmaf(sv[b][1], d[b][3], y1b);
                }
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
                if (rbi >= 2) {
                    const bool ok2 = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&rempty[b], ((rbi >> 1) - 1) & 1u,
                                                                               abort_flag, kErrTimeoutTmaFull));
                    if (!ok2) break;
                }
                float* rbuf = red + b * (kMW * kMRedStride) + warp * kMRedStride;
                if (tig < 2) {
                    reinterpret_cast<float2*>(rbuf + gid * 4 + 2 * tig)[0] = make_float2(y0a, y0b);
                    reinterpret_cast<float2*>(rbuf + (gid + 8) * 4 + 2 * tig)[0] = make_float2(y1a, y1b);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&rfull[b]);
                y0a = y0b = y1a = y1b = 0.f;
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
