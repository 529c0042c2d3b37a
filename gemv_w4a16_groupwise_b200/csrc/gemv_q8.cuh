// Forward GEMV for M <= 4 on the int8 tensor pipe with exact activations,
// for group lengths that are a multiple of 128 (or one group per row).
//
// Why int8.  On B200 a legacy mma.sync keeps the tensor pipe of its SM
// sub-partition busy about 32 cycles, bf16 m16n8k16 and int8 m16n8k32 alike,
// so the number of mma per weight sets a ceiling: a bf16 GEMV (256 codes per
// mma) tops out near 32 weights per clock and SM, while the HBM roofline
// needs about 44.  The int8 form takes 512 codes per mma, and its weight
// operand costs one AND per four codes; the activations then need an integer
// form that is exact.
//
// Activations as three digits.  Per 128-k granule and activation row, let E
// be the largest bf16 exponent; every x becomes c' = x 2^(148 - E), so the
// largest |c'| lies in [2^21, 2^22) and every x within 2^15 of the largest
// (15 binades) is an exact integer.  c' is split into balanced signed digits
//     c' = 65536 c2 + 256 d1 + d0,   d0, d1 in [-128, 127], c2 in [-64, 64],
// read straight from the bits of t = c' + 1.5 * 2^23 (one FMA): d0 is byte 0
// of t, d1 byte 1 of t + 128, c2 byte 2 of t + 32896 - 2^22.  One mma set
// (u8 codes x s8 digits) holds two activation rows: columns 4 j .. 4 j + 2
// are c2, d1, d0 of row 2 s + j of set s (column 4 j + 3 is zero); M <= 2
// takes one set per mma step, M = 3 or 4 two.  With the even codes as bytes q
// and the odd ones as 16 q (one AND each per word, as in the codes' own byte
// layout), each lane gets exact integers V_d = 16 sum q d for its columns,
// and with the granule's digit sums T_d,
//     t_d = V_d - 16 z T_d = 16 sum (q - z) d   (exact, |t| < 2^30),
// so that 16 sum (q - z) c' = 65536 t_c2 + 256 t_d1 + t_d0, folded into y in
// fp32 with the scale s 2^(E - 152).  Every product and sum up to that fold
// is exact; the fold rounds like an fp32 accumulation (balanced digits keep
// each level's term within twice the value's own size, so nothing cancels
// catastrophically).  With one set, the lane holding (c2, d1) of a row folds
// 256 (256 t_c2 + t_d1) and its neighbour, holding d0, folds t_d0: two
// partial sums that the end-of-chunk reduction adds.  With two sets, each
// lane folds one whole row after one exchange with its neighbour.
//
// Granules outside that window.  A bf16 x is m 2^(e - 134) with an 8-bit m
// and exponent field e, so x 2^(148 - E) is an integer whenever e >= E - 14;
// the conversion checks that every non-zero activation of the granule meets
// it (the smallest non-zero magnitude, found with one add, one AND and one
// 16-bit min per pair of bf16 values).  A granule that does not (a spread
// above 15 binades, activations below 2^-100 or above 2^28, or subnormal
// ones) takes the bf16 path instead: the codes unpacked to exact bf16
// (q - z), the activations themselves as bf16, mma.sync m16n8k16 with fp32
// accumulation.  Both paths are exact up to fp32 accumulation; the choice is
// per granule and warp-uniform, and the bf16 path is a separate function
// that reloads its activations from L2, so that the common path keeps its
// registers.
//
// Schedule.  A producer warp streams 16-row x 2048-k boxes (16 rows x 1 KB
// of packed words) with their scales and zeros through a ring of stages;
// warp w takes granule w (k = 128 w .. 128 w + 127) of every stage.  The
// CTA's row blocks are taken in chunks of up to 8: for each 2048-k step of
// the K slice, the chunk's row blocks follow one another, so a warp converts
// its granule once per chunk and keeps the digits in registers for all of
// the chunk's row blocks (the activations never sit in shared memory); each
// lane's running sums of the chunk's row blocks live in the warp's slice of
// shared memory.  At the end of a chunk the sixteen warps' sums are added in
// a fixed order (results do not depend on timing), biased and rounded once,
// or written as fp32 partials when K is split into slices.
#pragma once

#include "gemv_mma.cuh"

namespace w4 {

constexpr int kQW = 16;                          // consumer warps
constexpr int kQThreads = (kQW + 1) * 32;        // + the producer warp
constexpr int kQChunk = 8;                       // row blocks per chunk
constexpr int kQYWords = kQChunk * 32 * 2;       // per warp: running sums [row block][lane][2 rows]
constexpr int kQTabWords = 2 * 32 * 8;           // per warp: digit exchange [set][lane][8 registers]

__host__ __device__ inline size_t gemv_q8_smem_bytes(int stages, int sz, int szw) {
    size_t b = 1024;
    b += static_cast<size_t>(stages) * gemv_mma_stage_bytes(sz, szw);
    b += static_cast<size_t>(kQW) * (kQYWords + kQTabWords) * 4;
    b += static_cast<size_t>(stages) * 16 + 16;
    return b;
}

__device__ __forceinline__ void mma_u8s8_16832(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Arrive once per warp on `bar` (one elected lane, no divergent branch).
__device__ __forceinline__ void mbar_arrive_elected(uint64_t* bar) {
    asm volatile(
        "{\n .reg .pred P;\n elect.sync _|P, 0xffffffff;\n"
        " @P mbarrier.arrive.shared::cta.b64 _, [%0];\n}\n" ::"r"(smem_u32(bar))
        : "memory");
}

// One warp's activation granule (k = kg .. kg + 127, all M rows): the lane's
// B registers of each mma set and the constants of its fold.
template <int NSET>
struct Q8Granule {
    uint32_t b[NSET][8];    // per set: [pair][parity][half] B registers of this lane
    int thi, tlo;           // digit sums that go with this lane's fold (see q8_convert)
    int khi;                // one set: 256 for a (c2, d1) lane, 1 for a d0 lane
    float xs;               // scale of the lane's fold: 2^(E - 152), times 256 on (c2, d1) lanes of one set
    bool bf16;              // warp-uniform: the granule takes the bf16 path
};

// The activation row whose sums a lane accumulates: with one set, row tig / 2
// (even lanes its (c2, d1) part, odd lanes its d0 part); with two, row tig / 2
// of set 0 on even lanes and row 2 + tig / 2 of set 1 on odd lanes.
template <int NSET>
__device__ __forceinline__ int q8_fold_row(int tig) {
    return NSET == 1 ? (tig >> 1) : ((tig & 1) ? 2 + (tig >> 1) : (tig >> 1));
}

// Digit bytes of four scaled values: byte `sel` of each, in k order.
__device__ __forceinline__ uint32_t gather4(uint32_t a, uint32_t b, uint32_t c, uint32_t d, uint32_t sel2) {
    return prmt(prmt(a, b, sel2), prmt(c, d, sel2), 0x5410u);
}

// Converts the warp's granule at kg.  Unit u = 16 m + j (word j of the
// granule, 8 activations of row m) belongs to lane u % 32 (two units per
// lane when M > 2); the sixteen lanes of a row reduce its largest and
// smallest non-zero magnitude with shuffles, and each unit's digit registers
// go through the warp's table `tab` to the lanes that hold them as B
// fragments.  Those lanes then sum their column's digits (dp4a over their 32
// k, then over the row of four lanes), and each lane fetches the sums its
// fold needs.
template <int M>
__device__ __forceinline__ void q8_convert(const uint16_t* __restrict__ X, int K, int kg, int lane, uint32_t* tab,
                                           Q8Granule<(M + 1) / 2>& g) {
    constexpr int NSET = (M + 1) / 2;
    constexpr int kRounds = NSET;                   // units 16 m + j over 32 lanes
    constexpr float kMagic = 12582912.0f;          // 1.5 * 2^23
    const int gid = lane >> 2, tig = lane & 3;
    bool inexact = false;
    float XS[kRounds];
    __syncwarp();                                  // the table's last readers are done
#pragma unroll
    for (int rr = 0; rr < kRounds; ++rr) {
        const int u = lane + 32 * rr;
        const int m = u >> 4, j = u & 15;
        const bool real = m < M;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (real && kg + 8 * j < K) v = __ldg(reinterpret_cast<const uint4*>(X + static_cast<size_t>(m) * K + kg + 8 * j));
        // magnitudes as bf16 bit patterns (they order like the values); for
        // the smallest non-zero one each half becomes a - 1, or 0x7FFF for a
        // zero, with no carry between the halves
        const uint32_t a0 = v.x & 0x7FFF7FFFu, a1 = v.y & 0x7FFF7FFFu, a2 = v.z & 0x7FFF7FFFu, a3 = v.w & 0x7FFF7FFFu;
        uint32_t mx = __vmaxu2(__vmaxu2(a0, a1), __vmaxu2(a2, a3));
        uint32_t mn = __vminu2(__vminu2((a0 + 0x7FFF7FFFu) & 0x7FFF7FFFu, (a1 + 0x7FFF7FFFu) & 0x7FFF7FFFu),
                               __vminu2((a2 + 0x7FFF7FFFu) & 0x7FFF7FFFu, (a3 + 0x7FFF7FFFu) & 0x7FFF7FFFu));
        mx = max(mx & 0xFFFFu, mx >> 16);
        mn = min(mn & 0xFFFFu, mn >> 16);
#pragma unroll
        for (int o = 8; o >= 1; o >>= 1) {
            mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
            mn = min(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, o));
        }
        int e = static_cast<int>(mx >> 7);         // exponent field of the largest
        const bool big = e > 155;
        e = min(max(e, 26), 155);
        // exact when every non-zero magnitude has an exponent field >= E - 14
        inexact = inexact || big || (static_cast<int>(mn) + 1 < ((e - 14) << 7));
        const float scale = __int_as_float((275 - e) << 23);       // 2^(148 - E)
        XS[rr] = real ? __int_as_float((e - 25) << 23) : 0.f;      // 2^(E - 152)
        uint32_t tb[8], e1[8], e2[8];
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float xf = __uint_as_float((i & 1) ? (w4[i >> 1] & 0xFFFF0000u) : (w4[i >> 1] << 16));
            tb[i] = __float_as_uint(fmaf(xf, scale, kMagic));       // 0x4B400000 + c'
            e1[i] = tb[i] + 128u;                   // byte 1: d1
            e2[i] = tb[i] + (32896u - 0x400000u);   // byte 2: c2 (two's complement)
        }
        if (real) {
            // owners: word j sits in lane tig_o = j / 4 of a row, as half j % 2
            // of pair (j % 4) / 2, register [pair][parity][half]; row m's digits
            // are columns 4 (m % 2) + {0, 1, 2} of set m / 2
            const int tig_o = j >> 2, ri = ((j & 3) >> 1) * 4 + (j & 1);
            uint32_t* ts = tab + (m >> 1) * (32 * 8);
            const int l2 = 4 * (4 * (m & 1)) + tig_o;
            ts[l2 * 8 + ri] = gather4(e2[0], e2[2], e2[4], e2[6], 0x62u);
            ts[l2 * 8 + ri + 2] = gather4(e2[1], e2[3], e2[5], e2[7], 0x62u);
            ts[(l2 + 4) * 8 + ri] = gather4(e1[0], e1[2], e1[4], e1[6], 0x51u);
            ts[(l2 + 4) * 8 + ri + 2] = gather4(e1[1], e1[3], e1[5], e1[7], 0x51u);
            ts[(l2 + 8) * 8 + ri] = gather4(tb[0], tb[2], tb[4], tb[6], 0x40u);
            ts[(l2 + 8) * 8 + ri + 2] = gather4(tb[1], tb[3], tb[5], tb[7], 0x40u);
        }
    }
    __syncwarp();
    int colsum[NSET];
#pragma unroll
    for (int st = 0; st < NSET; ++st) {
        // column gid of set st: row 2 st + gid / 4, digit gid % 4 (3: zero)
        const bool own = (gid & 3) != 3 && 2 * st + (gid >> 2) < M;
        uint4 b0 = make_uint4(0u, 0u, 0u, 0u), b1 = b0;
        if (own) {
            const uint4* tv = reinterpret_cast<const uint4*>(tab + st * (32 * 8) + lane * 8);
            b0 = tv[0];
            b1 = tv[1];
        }
        g.b[st][0] = b0.x; g.b[st][1] = b0.y; g.b[st][2] = b0.z; g.b[st][3] = b0.w;
        g.b[st][4] = b1.x; g.b[st][5] = b1.y; g.b[st][6] = b1.z; g.b[st][7] = b1.w;
        int cs = 0;
#pragma unroll
        for (int q = 0; q < 8; ++q) cs = __dp4a(static_cast<int>(g.b[st][q]), 0x01010101, cs);
        cs += __shfl_xor_sync(0xFFFFFFFFu, cs, 1);
        cs += __shfl_xor_sync(0xFFFFFFFFu, cs, 2);
        colsum[st] = cs;                           // the digit sum of column gid over the granule
    }
    // the lane's fold row f: set f / 2, columns 4 (f % 2) + {0, 1, 2}, whose
    // sums live in lanes 4 column ..; its scale in lanes 16 (f % 2) .. of
    // round f / 2
    {
        const int f = q8_fold_row<NSET>(tig);
        const int sf = f >> 1, c0 = 4 * (f & 1);
        int tc[3];
#pragma unroll
        for (int d = 0; d < 3; ++d) {
            tc[d] = __shfl_sync(0xFFFFFFFFu, colsum[0], 4 * (c0 + d));
            if (NSET == 2) {
                const int t1 = __shfl_sync(0xFFFFFFFFu, colsum[NSET - 1], 4 * (c0 + d));
                if (sf) tc[d] = t1;
            }
        }
        float xs = __shfl_sync(0xFFFFFFFFu, XS[0], 16 * (f & 1));
        if (kRounds == 2) {
            const float us = __shfl_sync(0xFFFFFFFFu, XS[kRounds - 1], 16 * (f & 1));
            if (sf) xs = us;
        }
        const bool live = f < M;
        if (NSET == 1) {
            // (c2, d1) lanes fold 256 (256 t_c2 + t_d1), d0 lanes fold t_d0
            const bool hi = (tig & 1) == 0;
            g.khi = hi ? 256 : 1;
            g.thi = live ? (hi ? 256 * tc[0] + tc[1] : tc[2]) : 0;
            g.tlo = 0;
            g.xs = live ? (hi ? 256.0f * xs : xs) : 0.f;
        } else {
            g.khi = 256;
            g.thi = live ? 256 * tc[0] + tc[1] : 0;
            g.tlo = live ? tc[2] : 0;
            g.xs = live ? xs : 0.f;
        }
    }
    g.bf16 = __any_sync(0xFFFFFFFFu, inexact);
}

// bf16 B registers of lane (m, tig) = 4 m + tig for the four words of lane
// tig: x[m][kg + 32 tig + 8 i ..], (x0 x4 | x1 x5 | x2 x6 | x3 x7) each.
template <int M>
__device__ __forceinline__ void q8_bf16_fragments(const uint16_t* __restrict__ X, int K, int kg, int lane,
                                                  uint32_t (&h)[16]) {
    const int tig = lane & 3;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint4 u = make_uint4(0u, 0u, 0u, 0u);
        const int k = kg + 32 * tig + 8 * i;
        if (lane < 4 * M && k < K)
            u = __ldg(reinterpret_cast<const uint4*>(X + static_cast<size_t>(lane >> 2) * K + k));
        h[4 * i] = prmt(u.x, u.z, 0x5410u);
        h[4 * i + 1] = prmt(u.x, u.z, 0x7632u);
        h[4 * i + 2] = prmt(u.y, u.w, 0x5410u);
        h[4 * i + 3] = prmt(u.y, u.w, 0x7632u);
    }
}

// One stage of a granule on the bf16 path: returns the lane's share of the
// two rows' sums (rows gid and gid + 8 of the lane's fold row), before the
// scale.  Kept out of line so that the int8 path keeps its registers.
template <int M, int NSET>
__device__ __noinline__ float2 q8_bf16_stage(const uint16_t* __restrict__ X, int K, int kg, int lane, uint4 wa,
                                             uint4 wb, uint32_t zz0, uint32_t zz1, bool fz, float zo0, float zo1) {
    uint32_t hx[16];
    q8_bf16_fragments<M>(X, K, kg, lane, hx);
    float dh[4] = {0.f, 0.f, 0.f, 0.f};
    const uint32_t wa4[4] = {wa.x, wa.y, wa.z, wa.w}, wb4[4] = {wb.x, wb.y, wb.z, wb.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t pa[4], pb[4];
        if (!fz) {
            unpack_word_bf16(wa4[i], zz0, pa);
            unpack_word_bf16(wb4[i], zz1, pb);
        } else {
            unpack_word_bf16_rounded(wa4[i], zo0, pa);
            unpack_word_bf16_rounded(wb4[i], zo1, pb);
        }
        mma_bf16_16816(dh, pa[0], pb[0], pa[1], pb[1], hx[4 * i], hx[4 * i + 1]);
        mma_bf16_16816(dh, pa[2], pb[2], pa[3], pb[3], hx[4 * i + 2], hx[4 * i + 3]);
    }
    // lane (gid, tig) holds m = 2 tig, 2 tig + 1: move the lane's fold row f
    // here (from lane gid * 4 + f / 2); with one set the d0 lanes take no part
    const int gid = lane >> 2, tig = lane & 3;
    const int fr = q8_fold_row<NSET>(tig);
    const int src = gid * 4 + (fr >> 1);
    const float v00 = __shfl_sync(0xFFFFFFFFu, dh[0], src);
    const float v01 = __shfl_sync(0xFFFFFFFFu, dh[1], src);
    const float v10 = __shfl_sync(0xFFFFFFFFu, dh[2], src);
    const float v11 = __shfl_sync(0xFFFFFFFFu, dh[3], src);
    const bool take = NSET == 2 || (tig & 1) == 0;
    return take ? make_float2((fr & 1) ? v01 : v00, (fr & 1) ? v11 : v10) : make_float2(0.f, 0.f);
}

// Arguments of gemv_q8_kernel.
struct GemvQ8Args {
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

template <int M, int SZ, bool FZ>
__global__ void __launch_bounds__(kQThreads, 1)
    gemv_q8_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap smap,
                   const __grid_constant__ CUtensorMap zmap, const GemvQ8Args a) {
    static_assert(M >= 1 && M <= 4, "M");
    constexpr int NSET = (M + 1) / 2;
    // the test hook that withholds a stage (-1 unless a test injects a lost
    // stage) is set by the host before the launch: read it first thing, so
    // that its global-memory latency overlaps the set-up instead of delaying
    // the producer's first copy
    const int withhold = threadIdx.x >= kQW * 32 ? *reinterpret_cast<volatile int*>(&g_withhold_stage) : -1;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int NS = a.stages;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
    const int gid = lane >> 2, tig = lane & 3;
    const int SB = gemv_mma_stage_bytes(SZ, a.szw);
    const int kSzTx = SZ == kSzTma2d ? 2 * kMR * a.szw * 2 : SZ == kSzTma1d ? 2 * kMR * 2 : 0;
    uint8_t* ring = base;
    float* ysum = reinterpret_cast<float*>(ring + NS * SB);                 // [warp][kQYWords]
    uint32_t* tabs = reinterpret_cast<uint32_t*>(ysum + kQW * kQYWords);   // [warp][kQTabWords]
    uint64_t* full = reinterpret_cast<uint64_t*>(tabs + kQW * kQTabWords);
    uint64_t* empty = full + NS;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + NS);

    if (tid == 0) {
        for (int i = 0; i < NS; ++i) {
            mbar_init(&full[i], SZ == kSzCopy ? 33 : 1);
            mbar_init(&empty[i], kQW);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (tid == kQW * 32) {
        tma_prefetch_desc(&wmap);
        if (SZ == kSzTma2d || SZ == kSzTma1d) {
            tma_prefetch_desc(&smap);
            tma_prefetch_desc(&zmap);
        }
    }
    __syncthreads();
    // launched as a programmatic dependent of the work before it: no global
    // memory is read until that work is complete
    pdl_launch_dependents();
    pdl_wait();

    const int slice = blockIdx.x / a.cps, cta = blockIdx.x - (blockIdx.x / a.cps) * a.cps;
    const int rb_lo = static_cast<int>(static_cast<long long>(cta) * a.nrb / a.cps);
    const int rb_hi = static_cast<int>(static_cast<long long>(cta + 1) * a.nrb / a.cps);
    const int nrows = rb_hi - rb_lo;
    const int nch = (nrows + kQChunk - 1) / kQChunk;
    const int k_slice = slice * a.TKC;
    auto chunk_lo = [&](int c) { return rb_lo + static_cast<int>(static_cast<long long>(c) * nrows / nch); };
    auto group_of = [&](int k) {
        return a.G == 1 ? 0 : static_cast<int>((static_cast<unsigned long long>(k) * a.gmul) >> a.gshift);
    };

    if (warp == kQW) {
        // ------------------------------------------------------ producer
        int s = 0, it = 0;
        uint32_t round = 0;
        bool alive = true;
        for (int c = 0; c < nch && alive; ++c) {
            const int r0 = chunk_lo(c), rc = chunk_lo(c + 1) - r0;
            for (int ks = 0; ks < a.nks && alive; ++ks) {
                const int k0 = k_slice + ks * kMK;
                const int x2 = SZ == kSzTma2d ? group_of(k0) & ~7 : 0;
                for (int r = 0; r < rc; ++r, ++it) {
                    if (round > 0) {
                        alive = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&empty[s], (round - 1) & 1u, abort_flag,
                                                                          kErrTimeoutEmpty));
                        if (!alive) break;
                    }
                    uint8_t* sd = ring + s * SB;
                    const int row0 = (r0 + r) * kMR;
                    if (it == withhold) {
                        // injected loss: this stage's copy is never issued, so its
                        // consumers' bounded waits run out; nothing is left in flight
                        if (++s == NS) {
                            s = 0;
                            ++round;
                        }
                        continue;
                    }
                    if (SZ == kSzCopy) {
                        const int arr = lane >> 4, rr = lane & 15;
                        const long long h0 = (static_cast<long long>(row0 + rr) * a.sz_row + group_of(k0)) & ~1ll;
                        uint32_t* dst = reinterpret_cast<uint32_t*>(sd + kMWBytes) + (arr * kMR + rr) * a.szw;
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
                        tma_issue_elected<3>(&full[s], kMWBytes + kSzTx, sd, &wmap, k0 / 8, row0, sd + kMWBytes, &smap,
                                             x2, row0, sd + kMWBytes + kMR * a.szw * 2, &zmap, x2, row0);
                    } else if (SZ == kSzTma1d) {
                        tma_issue_elected<3>(&full[s], kMWBytes + kSzTx, sd, &wmap, k0 / 8, row0, sd + kMWBytes, &smap,
                                             row0, 0, sd + kMWBytes + 128, &zmap, row0, 0);
                    } else {
                        tma_issue_elected<1>(&full[s], kMWBytes, sd, &wmap, k0 / 8, row0);
                    }
                    if (++s == NS) {
                        s = 0;
                        ++round;
                    }
                }
            }
        }
    } else {
        // ------------------------------------------------------ consumers
        uint32_t* tab = tabs + warp * kQTabWords;
        float2* yw = reinterpret_cast<float2*>(ysum + warp * kQYWords) + lane;   // [row block] stride 32
        const bool mbf = (a.fmt & kFmtMetaBf16) != 0;
        // a fractional zero point z is taken as zi + (z - zi), zi = clamp(rint(z), 0, 15):
        // the integer part goes through the exact integer sums, the rest is an fp32
        // correction of the fold
        constexpr bool fz = FZ;     // a.fmt & kFmtZeroFloat, as a template argument
        float s_const = 0.f, z_const = 0.f;
        int z16_const = 0;
        uint32_t zz_const = 0u;
        if (SZ == kSzConst) {
            z_const = meta_to_float(a.Z[0], mbf);
            s_const = meta_to_float(a.S[0], mbf);
            z16_const = __float_as_int(fmaf(z_const, 16.0f, 12582912.0f)) - 0x4B400000;
            zz_const = bf16x2_splat(128.0f + z_const);
        }
        const uint8_t* ra_base = ring + gid * 1024 + warp * 64 + tig * 16;
#pragma unroll
        for (int r = 0; r < kQChunk; ++r) yw[r * 32] = make_float2(0.f, 0.f);
        int s = 0;
        uint32_t phase = 0;
        bool alive = true;
        for (int c = 0; c < nch; ++c) {
            const int r0 = chunk_lo(c), rc = chunk_lo(c + 1) - r0;
            for (int ks = 0; ks < a.nks; ++ks) {
                const int k0 = k_slice + ks * kMK;
                const int kg = k0 + warp * 128;
                const bool active = kg < a.K && alive;
                Q8Granule<NSET> xg;
                if (active) q8_convert<M>(a.X, a.K, kg, lane, tab, xg);
                // where rows gid, gid + 8 find their scale and zero in a stage
                int so0 = 0, so1 = 0, zo = 0;
                int grp = 0, fg = 0;
                if (SZ == kSzTma2d) {
                    grp = group_of(kg);
                    const int gi = grp - (group_of(k0) & ~7);
                    so0 = gid * a.szw + gi;
                    so1 = (gid + 8) * a.szw + gi;
                    zo = kMR * a.szw;
                } else if (SZ == kSzTma1d) {
                    so0 = gid;
                    so1 = gid + 8;
                    zo = 64;
                } else if (SZ == kSzCopy) {
                    grp = group_of(kg);
                    fg = group_of(k0);
                    zo = kMR * 2 * a.szw;
                }
                for (int r = 0; r < rc; ++r) {
                    if (alive)
                        alive = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&full[s], phase, abort_flag,
                                                                          kErrTimeoutTmaFull));
                    float2 yv = yw[r * 32];
                    if (alive && active) {
                        const uint8_t* sb = ring + s * SB;
                        const uint4 wa = *reinterpret_cast<const uint4*>(ra_base + s * SB);
                        const uint4 wb = *reinterpret_cast<const uint4*>(ra_base + s * SB + 8 * 1024);
                        // scale and zero of rows gid and gid + 8 for the granule's group
                        float s0, s1, z0, z1;
                        if (SZ == kSzConst) {
                            s0 = s1 = s_const;
                            z0 = z1 = z_const;
                        } else {
                            const __half* sh = reinterpret_cast<const __half*>(sb + kMWBytes);
                            int o0 = so0, o1 = so1;
                            if (SZ == kSzCopy) {
                                // row r's words start at half (row r, first group)
                                // rounded down to even
                                const int row0 = (r0 + r) * kMR;
                                const int w2 = 2 * a.szw;
                                o0 = gid * w2 + grp - fg + ((((row0 + gid) & a.sz_row) ^ fg) & 1);
                                o1 = (gid + 8) * w2 + grp - fg + ((((row0 + gid + 8) & a.sz_row) ^ fg) & 1);
                            }
                            s0 = meta_to_float(sh[o0], mbf);
                            s1 = meta_to_float(sh[o1], mbf);
                            z0 = meta_to_float(sh[zo + o0], mbf);
                            z1 = meta_to_float(sh[zo + o1], mbf);
                        }
                        if (!xg.bf16) {
                            // ---- int8 path: four mma per set, exact integer sums
                            int de[NSET][4], dd[NSET][4];
#pragma unroll
                            for (int st = 0; st < NSET; ++st)
#pragma unroll
                                for (int q = 0; q < 4; ++q) de[st][q] = dd[st][q] = 0;
                            constexpr uint32_t kLo = 0x0F0F0F0Fu, kHi = 0xF0F0F0F0u;
                            const uint32_t wa4[4] = {wa.x, wa.y, wa.z, wa.w}, wb4[4] = {wb.x, wb.y, wb.z, wb.w};
#pragma unroll
                            for (int pr = 0; pr < 2; ++pr) {
                                const uint32_t a0 = wa4[2 * pr] & kLo, a1 = wb4[2 * pr] & kLo;
                                const uint32_t a2 = wa4[2 * pr + 1] & kLo, a3 = wb4[2 * pr + 1] & kLo;
                                const uint32_t o0 = wa4[2 * pr] & kHi, o1 = wb4[2 * pr] & kHi;
                                const uint32_t o2 = wa4[2 * pr + 1] & kHi, o3 = wb4[2 * pr + 1] & kHi;
#pragma unroll
                                for (int st = 0; st < NSET; ++st) {
                                    mma_u8s8_16832(de[st], a0, a1, a2, a3, xg.b[st][4 * pr], xg.b[st][4 * pr + 1]);
                                    mma_u8s8_16832(dd[st], o0, o1, o2, o3, xg.b[st][4 * pr + 2], xg.b[st][4 * pr + 3]);
                                }
                            }
                            int zq0, zq1;          // 16 z (16 zi for a fractional zero), an integer
                            float zr0 = 0.f, zr1 = 0.f;   // 16 (z - zi)
                            if (!fz) {
                                zq0 = SZ == kSzConst ? z16_const
                                                     : __float_as_int(fmaf(z0, 16.0f, 12582912.0f)) - 0x4B400000;
                                zq1 = SZ == kSzConst ? z16_const
                                                     : __float_as_int(fmaf(z1, 16.0f, 12582912.0f)) - 0x4B400000;
                            } else {
                                const float zi0 = fminf(fmaxf(rintf(z0), 0.f), 15.f);
                                const float zi1 = fminf(fmaxf(rintf(z1), 0.f), 15.f);
                                zq0 = __float_as_int(fmaf(zi0, 16.0f, 12582912.0f)) - 0x4B400000;
                                zq1 = __float_as_int(fmaf(zi1, 16.0f, 12582912.0f)) - 0x4B400000;
                                zr0 = 16.0f * (z0 - zi0);
                                zr1 = 16.0f * (z1 - zi1);
                            }
                            float f[2];
#pragma unroll
                            for (int h = 0; h < 2; ++h) {
                                const int z16 = h ? zq1 : zq0;
                                const float zr = h ? zr1 : zr0;
                                // V = 16 sum q d of the lane's two columns of set 0
                                const int va = 16 * de[0][2 * h] + dd[0][2 * h];
                                const int vb = 16 * de[0][2 * h + 1] + dd[0][2 * h + 1];
                                if (NSET == 1) {
                                    // (c2, d1) lanes: 256 V_c2 + V_d1; d0 lanes: V_d0 (vb = 0)
                                    f[h] = static_cast<float>(xg.khi * va + vb - z16 * xg.thi);
                                    if (fz) f[h] = fmaf(-zr, static_cast<float>(xg.thi), f[h]);
                                } else {
                                    const int wa_ = 16 * de[NSET - 1][2 * h] + dd[NSET - 1][2 * h];
                                    const int wb_ = 16 * de[NSET - 1][2 * h + 1] + dd[NSET - 1][2 * h + 1];
                                    // even lanes: set 0 (c2, d1) here, d0 from the odd neighbour;
                                    // odd lanes: set 1 d0 here, (c2, d1) from the even neighbour
                                    const bool odd = tig & 1;
                                    const int mine = odd ? wa_ : 256 * va + vb;
                                    const int other = __shfl_xor_sync(0xFFFFFFFFu, odd ? va : 256 * wa_ + wb_, 1);
                                    const int hi = odd ? other : mine, lo = odd ? mine : other;
                                    float fh = static_cast<float>(hi - z16 * xg.thi);
                                    float fl = static_cast<float>(lo - z16 * xg.tlo);
                                    if (fz) {
                                        fh = fmaf(-zr, static_cast<float>(xg.thi), fh);
                                        fl = fmaf(-zr, static_cast<float>(xg.tlo), fl);
                                    }
                                    f[h] = fmaf(fh, 256.0f, fl);
                                }
                            }
                            yv.x = fmaf(s0 * xg.xs, f[0], yv.x);
                            yv.y = fmaf(s1 * xg.xs, f[1], yv.y);
                        } else {
                            // ---- bf16 path (rare): exact (q - z) x bf16 activations, fp32 sums
                            const uint32_t zz0 = SZ == kSzConst ? zz_const : bf16x2_splat(128.0f + z0);
                            const uint32_t zz1 = SZ == kSzConst ? zz_const : bf16x2_splat(128.0f + z1);
                            const float2 d = q8_bf16_stage<M, NSET>(a.X, a.K, kg, lane, wa, wb, zz0, zz1, fz,
                                                                    128.0f + z0, 128.0f + z1);
                            yv.x = fmaf(s0, d.x, yv.x);
                            yv.y = fmaf(s1, d.y, yv.y);
                        }
                    }
                    yw[r * 32] = yv;
                    __syncwarp();
                    mbar_arrive_elected(&empty[s]);
                    if (++s == NS) {
                        s = 0;
                        phase ^= 1u;
                    }
                }
            }
            // ---- chunk done: add the sixteen warps' sums in warp order
            named_barrier_sync(1, kQW * 32);
            for (int o = tid; o < rc * 64; o += kQW * 32) {
                const int r = o >> 6, row = (o >> 2) & 15, m = o & 3;
                const int n = (r0 + r) * kMR + row;
                if (m >= M || n >= a.N) continue;
                // lane holding (row, m): gid = row % 8, h = row / 8, tig from the fold layout
                const int h = row >> 3, g8 = row & 7;
                const int tg = NSET == 1 ? 2 * m : (m < 2 ? 2 * m : 2 * (m - 2) + 1);
                const int idx = (r * 32 + g8 * 4 + tg) * 2 + h;
                float sum = 0.f;
#pragma unroll
                for (int w = 0; w < kQW; ++w) {
                    float v = ysum[w * kQYWords + idx];
                    if (NSET == 1) v += ysum[w * kQYWords + idx + 2];     // the d0 lane's part
                    sum += v;
                }
                if (!*abort_flag) {
                    if (a.splits == 1) {
                        if (a.bias) sum += bf16_bits_to_float(a.bias[n]);
                        a.Y[static_cast<size_t>(m) * a.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(sum));
                    } else {
                        a.partial[(static_cast<size_t>(slice) * M + m) * a.N + n] = sum;
                    }
                }
            }
            named_barrier_sync(1, kQW * 32);            // every sum is read: clear this lane's
#pragma unroll
            for (int r = 0; r < kQChunk; ++r) yw[r * 32] = make_float2(0.f, 0.f);
        }
    }
    if (*abort_flag) {
        const unsigned long long t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 1000000ull) {
        }
    }
}

}  // namespace w4
