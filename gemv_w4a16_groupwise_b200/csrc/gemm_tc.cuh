// Tensor-core W4A16 GEMM for M > 4 on sm_100a: TMA -> in-register int4
// dequantization -> tcgen05.mma (bf16 x bf16 -> fp32 in TMEM) -> epilogue.
//
// Forward  (llm-quantization, "Objectives" 2, Y = X_bf16 @ W_int4^T):
//     D[n, m] = sum_k w_hat[n, k] X[m, k]          A = w_hat tile, K-major
// Transposed ("Re-write HQQ Fused Gemm Transpose", same packed W, s, z):
//     D[k, m] = sum_n w_hat[n, k] dY[m, n]         A = w_hat^T tile, MN-major
// Both run "swap-AB": the 128-row MMA side carries weight rows (n, or k when
// transposed) and the MMA N side carries tokens, so one kernel serves M = 5
// to thousands with a token tile BN in {16, 32, 64, 128, 256}.  The bias is
// added to the fp32 accumulator before the single bf16 rounding (vLLM
// "Adding bias epilogue support for cutlass_scaled_mm").
//
// Persistent: one CTA per SM walks work units blockIdx.x, + gridDim.x, ...;
// the stage ring runs on across unit boundaries and the fp32 accumulator is
// double-buffered in TMEM, so one unit's epilogue overlaps the next unit's
// main loop.  A unit is a whole tile, or, for the tiles of a last partial
// wave (from tile F on), one of S slices of the tile's k-blocks: those
// units write fp32 partial tiles, which gemm_tail_finalize_kernel adds in
// slice order (with the bias) and rounds, so the last wave takes about
// 1 / S of a tile's time instead of a whole one.  Warp roles (704 threads):
//   warp 0       TMA producer: packed weight tile + activation tile per stage,
//                and, for groupwise scales whose row stride is a multiple of
//                16 bytes, a box of 8 groups x the tile's rows of S and of Z,
//                so that the scales arrive with the weights a ring ahead.  The
//                weights (with their scales) complete one barrier and the
//                activation tile another, so the dequantization of a stage does
//                not wait for the activation bytes, which only the MMA reads
//   warp 1       TMEM allocator; lane 0 issues tcgen05.mma and commits
//   warps 2..17  dequantize packed codes into the bf16 A tile of a stage
//                (128-byte swizzled UMMA layout).  Two groups of 8 warps take
//                alternate stages, four packed words per thread, so two
//                stages are being dequantized at any time: a warp's share of
//                a stage is a chain of dependent steps (wait, scale and code
//                loads, arithmetic, stores, proxy fence, arrival) whose
//                latency hardly depends on how many words it converts, so
//                one group of 16 warps on every stage (kTcDeqGroups = 1, two
//                words per thread) measured 25 % slower.
//   warps 18..21 epilogue: TMEM -> registers, fp32 bias, one bf16 rounding,
//                store (warp w reads the TMEM lanes 32 (w % 4) .. + 31).
// Every mbarrier wait is bounded; a wait that runs out records the reason in
// the device error word and the CTA unwinds without hanging.
//
// Dequantization of one packed word (8 codes) is exact up to the single
// bf16 rounding: each code becomes the fp32 value off + q (off = 128 or
// 2048) with one lop3, and one packed FMA per pair gives
//     (off + q) * s - (off + z) * s = (q - z) * s
// exactly in fp32 (both products need at most 23 significand bits), which
// cvt.rn.bf16x2 rounds once.  A fractional zero point (more significand
// bits) takes (off + q) - (off + z) and then the product with s instead,
// the product rounded in fp32 before the bf16 rounding.
#pragma once

#include "tma.cuh"

namespace w4 {

constexpr int kTcDeqWarps = 16;                      // dequantizing warps
constexpr int kTcDeqGroups = 2;                      // groups of them that take alternate stages
constexpr int kTcEpiWarps = 4;
constexpr int kTcThreads = 64 + kTcDeqWarps * 32 + kTcEpiWarps * 32;
constexpr int kTcBM = 128;     // MMA M (weight rows per tile)
constexpr int kTcBK = 64;      // reduction depth per pipeline stage
constexpr int kTcDeqGroupThreads = kTcDeqWarps * 32 / kTcDeqGroups;
constexpr int kTcWpt = kTcBM * kTcBK / 8 / kTcDeqGroupThreads;   // packed words per thread and stage
static_assert(kTcWpt == 2 || kTcWpt == 4, "dequantization mapping");
constexpr int kTcABytes = kTcBM * kTcBK * 2;   // 16 KB dequantized tile
constexpr int kTcPBytes = kTcBM * kTcBK / 2;   // 4 KB packed tile

struct TcArgs {
    const __half* S;
    const __half* Z;
    int fmt;              // format flags: kFmtZeroFloat, kFmtMetaBf16
    const uint16_t* bias;
    uint16_t* Y;
    float* part;          // [(tiles - F) * nslice][BN][128] fp32 partial tiles of the split tail
    int M, N, K;
    int g, G, sz_row;
    int stages;
    int stage_bytes;      // tc_stage_bytes(BN), plus the scale / zero boxes when sz_tma
    int sz_tma;           // scales and zeros come with each stage (TMA boxes)
    int F;                // tiles 0 .. F - 1 are whole work units
    int nslice;           // k slices of each tile from F on (1: no split)
};

struct TcProblem {
    const void* A;
    int M, N, K;
    const uint32_t* packed;
    const void* S;
    const void* Z;
    int g, G, sz_row;
    int fmt;
    const void* bias;
    int transposed;
    void* Y;
    int sms;
};

__host__ __device__ constexpr int tc_stage_bytes(int BN) { return kTcABytes + BN * 128 + kTcPBytes; }

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor (sm_100 "version 1"), 128-byte swizzle.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t smem_addr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
    d |= 1ull << 46;                 // descriptor version for tcgen05
    d |= 2ull << 61;                 // SWIZZLE_128B
    return d;
}

// Instruction descriptor: bf16 x bf16 -> fp32, M = 128, N = BN.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int BN, bool a_mn_major) {
    return (1u << 4)                              // D format f32
           | (1u << 7)                            // A format bf16
           | (1u << 10)                           // B format bf16
           | ((a_mn_major ? 1u : 0u) << 15)       // A major
           | (static_cast<uint32_t>(BN >> 3) << 17)
           | (static_cast<uint32_t>(kTcBM >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tmem_ld_x8(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Eight codes of one packed word -> eight bf16 (q - z) * s in k order.
__device__ __forceinline__ uint4 dequant_word_bf16(uint32_t w, float s, float c_lo, float c_hi, bool fz) {
    const uint32_t l16 = w << 16, l8 = w << 8, r8 = w >> 8, r16 = w >> 16;
    const float2 ss = make_float2(s, s);
    const float2 cc = make_float2(c_lo, c_hi);
    // (128 + q_even, 2048 + q_odd) for the pairs (0,1) (2,3) (4,5) (6,7)
    const float2 v01 = make_float2(__uint_as_float(lop3_and_or(l16, 0xF0000u, 0x43000000u)),
                                   __uint_as_float(lop3_and_or(l8, 0xF000u, 0x45000000u)));
    const float2 v23 = make_float2(__uint_as_float(lop3_and_or(l8, 0xF0000u, 0x43000000u)),
                                   __uint_as_float(lop3_and_or(w, 0xF000u, 0x45000000u)));
    const float2 v45 = make_float2(__uint_as_float(lop3_and_or(w, 0xF0000u, 0x43000000u)),
                                   __uint_as_float(lop3_and_or(r8, 0xF000u, 0x45000000u)));
    const float2 v67 = make_float2(__uint_as_float(lop3_and_or(r8, 0xF0000u, 0x43000000u)),
                                   __uint_as_float(lop3_and_or(r16, 0xF000u, 0x45000000u)));
    float2 f01, f23, f45, f67;
    if (!fz) {
        f01 = ffma2(v01, ss, cc);
        f23 = ffma2(v23, ss, cc);
        f45 = ffma2(v45, ss, cc);
        f67 = ffma2(v67, ss, cc);
    } else {
        // cc = -(off + z) here
        f01 = fmul2(fadd2(v01, cc), ss);
        f23 = fmul2(fadd2(v23, cc), ss);
        f45 = fmul2(fadd2(v45, cc), ss);
        f67 = fmul2(fadd2(v67, cc), ss);
    }
    uint4 out;
    out.x = bf162_bits(__floats2bfloat162_rn(f01.x, f01.y));
    out.y = bf162_bits(__floats2bfloat162_rn(f23.x, f23.y));
    out.z = bf162_bits(__floats2bfloat162_rn(f45.x, f45.y));
    out.w = bf162_bits(__floats2bfloat162_rn(f67.x, f67.y));
    return out;
}

template <bool TR, int BN, bool PWG, bool FZ>
__global__ void __launch_bounds__(kTcThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap pmap, const __grid_constant__ CUtensorMap bmap,
                   const __grid_constant__ CUtensorMap smap, const __grid_constant__ CUtensorMap zmap,
                   const TcArgs a) {
    static_assert(BN == 16 || BN == 32 || BN == 64 || BN == 128 || BN == 256, "BN");
    const int kStageBytes = a.stage_bytes;
    constexpr int kSzOff = tc_stage_bytes(BN);                  // the stage's scale / zero boxes
    constexpr int kSzRows = TR ? kTcBK : kTcBM;                 // weight rows of a stage
    constexpr uint32_t kAccCols = BN < 32 ? 32 : BN;          // one accumulator buffer
    constexpr uint32_t kTmemCols = 2 * kAccCols;              // two, a power of two >= 64
    constexpr uint32_t kBTxBytes = BN * 128;
    constexpr uint32_t kIdesc = umma_idesc_bf16(BN, TR);

    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int NS = a.stages;
    // tma_full: the stage's packed weights (and scale / zero boxes), which the
    // dequantizing warps wait for; b_full: its activation tile, which only
    // the MMA needs.  Separate barriers let the dequantization start as soon
    // as its 8 KB land, while the larger activation tile is still arriving.
    uint64_t* tma_full = reinterpret_cast<uint64_t*>(base + NS * kStageBytes);
    uint64_t* b_full = tma_full + NS;
    uint64_t* deq_full = b_full + NS;
    uint64_t* empty = deq_full + NS;
    uint64_t* acc_full = empty + NS;          // [2] an accumulator buffer holds a finished tile
    uint64_t* acc_empty = acc_full + 2;       // [2] the epilogue has drained a buffer
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int L_out = TR ? a.K : a.N;        // output row length
    const int red_len = TR ? a.N : a.K;      // reduction length
    const int num_kb = (red_len + kTcBK - 1) / kTcBK;
    const int tiles_m = (a.M + BN - 1) / BN;
    const int tiles = tiles_m * ((L_out + kTcBM - 1) / kTcBM);
    const int units = a.F + (tiles - a.F) * a.nslice;
    // this CTA's units: blockIdx.x, + gridDim.x, ...; tile t covers tokens
    // (t % tiles_m) * BN .. and output rows (t / tiles_m) * 128 ..
    const int my_units = blockIdx.x < units ? (units - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    struct Unit {
        int t, kb0, kb1;
        int part;        // index of the partial tile, or -1 for a whole tile
    };
    auto unit_of = [&](int i) {
        const int u = blockIdx.x + i * gridDim.x;
        Unit w;
        if (u < a.F) {
            w.t = u;
            w.kb0 = 0;
            w.kb1 = num_kb;
            w.part = -1;
        } else {
            const int v = u - a.F, sl = v % a.nslice;
            w.t = a.F + v / a.nslice;
            w.kb0 = sl * num_kb / a.nslice;
            w.kb1 = (sl + 1) * num_kb / a.nslice;
            w.part = v;
        }
        return w;
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&tma_full[s], 1);
            mbar_init(&b_full[s], 1);
            mbar_init(&deq_full[s], kTcDeqWarps / kTcDeqGroups);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], kTcEpiWarps);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_d = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&pmap);
            tma_prefetch_desc(&bmap);
            if (a.sz_tma) {
                tma_prefetch_desc(&smap);
                tma_prefetch_desc(&zmap);
            }
            int s = 0;
            uint32_t round = 0;
            bool ok = true;
            for (int i = 0; i < my_units && ok; ++i) {
                const Unit w = unit_of(i);
                const int m0 = (w.t % tiles_m) * BN, r0 = (w.t / tiles_m) * kTcBM;
                for (int kb = w.kb0; kb < w.kb1; ++kb) {
                    if (round > 0 && !mbar_wait_bounded(&empty[s], (round - 1) & 1u, abort_flag, kErrTimeoutEmpty)) {
                        ok = false;
                        break;
                    }
                    uint8_t* st = base + s * kStageBytes;
                    mbar_arrive_expect_tx(&tma_full[s], kTcPBytes + (a.sz_tma ? 2 * kSzRows * 16 : 0));
                    if (TR)
                        tma_load_2d(st + kTcABytes + BN * 128, &pmap, r0 / 8, kb * kTcBK, &tma_full[s]);
                    else
                        tma_load_2d(st + kTcABytes + BN * 128, &pmap, kb * (kTcBK / 8), r0, &tma_full[s]);
                    if (a.sz_tma) {
                        // groups from the stage's first one, rounded down to a
                        // multiple of 8 (16 bytes), for the stage's weight rows
                        const int x0 = (min((TR ? r0 : kb * kTcBK) / a.g, a.G - 1)) & ~7;
                        const int y0 = TR ? kb * kTcBK : r0;
                        tma_load_2d(st + kSzOff, &smap, x0, y0, &tma_full[s]);
                        tma_load_2d(st + kSzOff + kSzRows * 16, &zmap, x0, y0, &tma_full[s]);
                    }
                    mbar_arrive_expect_tx(&b_full[s], kBTxBytes);
                    tma_load_2d(st + kTcABytes, &bmap, kb * kTcBK, m0, &b_full[s]);
                    if (++s == NS) {
                        s = 0;
                        ++round;
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            bool ok = true;
            int s = 0;
            uint32_t phase = 0;
            for (int i = 0; i < my_units && ok; ++i) {
                const Unit w = unit_of(i);
                const int buf = i & 1;
                // the epilogue has drained this buffer (tile i - 2)
                if (i >= 2) ok = mbar_wait_bounded(&acc_empty[buf], ((i >> 1) - 1) & 1u, abort_flag, kErrTimeoutAccum);
                if (!ok) break;
                tc_fence_after();
                const uint32_t acc = tmem_d + static_cast<uint32_t>(buf) * kAccCols;
                for (int kb = w.kb0; kb < w.kb1; ++kb) {
                    // deq_full implies tma_full: every dequantizing warp waited for it
                    ok = mbar_wait_bounded(&deq_full[s], phase, abort_flag, kErrTimeoutDequant) &&
                         mbar_wait_bounded(&b_full[s], phase, abort_flag, kErrTimeoutTmaFull);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(base + s * kStageBytes);
                    const uint32_t b_addr = a_addr + kTcABytes;
#pragma unroll
                    for (int j = 0; j < kTcBK / 16; ++j) {
                        const uint64_t adesc = TR ? umma_desc_sw128(a_addr + j * 2048, 8192, 1024)
                                                  : umma_desc_sw128(a_addr + j * 32, 16, 1024);
                        const uint64_t bdesc = umma_desc_sw128(b_addr + j * 32, 16, 1024);
                        umma_bf16(acc, adesc, bdesc, kIdesc, (kb != w.kb0 || j != 0) ? 1u : 0u);
                    }
                    umma_commit(&empty[s]);
                    if (++s == NS) {
                        s = 0;
                        phase ^= 1u;
                    }
                }
                umma_commit(&acc_full[buf]);   // also tracks any MMA issued before an abort
            }
        }
    } else if (warp < 2 + kTcDeqWarps) {
        // ------------------------------------------------ dequantize
        // Stages are numbered across the CTA's units, in order; group grp_id
        // takes stages grp_id, grp_id + kTcDeqGroups, ...  Each thread of a
        // group dequantizes kTcWpt packed words (8 codes each) of one weight row.
        const int grp_id = (threadIdx.x - 64) / kTcDeqGroupThreads;
        const int t = (threadIdx.x - 64) % kTcDeqGroupThreads;
        int prow, pw;          // the thread's row in the stage and its first word in that row
        if (kTcWpt == 4) {
            // forward: row t / 2, words 4 (t % 2) .. + 3 of the 8 in a k-block (a phase of
            //   8 lanes reads 4 rows' 32 bytes: 128 contiguous bytes, no bank conflict; its
            //   swizzled 16-byte stores still land in 8 distinct banks)
            // transposed: words 4q .. 4q+3 of the 16 of a k-tile, with (row, q) spread so
            //   that a phase of 8 lanes takes 4 rows x 2 quads of one 64-k atom: its 16-byte
            //   loads meet at most 2 to a bank and its MN-major stores fall into 8 distinct banks
            prow = TR ? (((t >> 4) << 2) | ((t >> 1) & 3)) : (t >> 1);
            pw = 4 * (TR ? ((((t >> 3) & 1) << 1) | (t & 1)) : (t & 1));
        } else {
            // forward: row t / 4, words 2 (t % 4), + 1 (a half warp reads 4 rows' 32 bytes,
            //   128 contiguous bytes; 8 lanes store 2 rows x 4 chunks of one parity, which
            //   the swizzle puts in 8 distinct banks)
            // transposed: lane = (row bit 1, atom, row bit 0, pair 0..3), 4 rows per warp: a
            //   half warp reads 2 rows' 64 bytes (128 contiguous bytes); 8 lanes store 2 rows
            //   x 4 chunks of one atom, again 8 distinct banks
            const int l = t & 31;
            prow = TR ? ((t >> 5) * 4 + ((l >> 4) & 1) * 2 + ((l >> 2) & 1)) : (t >> 2);
            pw = TR ? (((l >> 3) & 1) * 8 + (l & 3) * 2) : 2 * (t & 3);
        }
        const int W8 = a.K / 8;
        // swizzled 16-byte destinations of this thread's words in the A tile
        uint32_t off[kTcWpt];
#pragma unroll
        for (int j = 0; j < kTcWpt; ++j) {
            if (TR) {
                const int kk = 8 * (pw + j);               // k within the 128-wide tile
                const int atom = kk >> 6, c = (kk & 63) >> 3;
                off[j] = atom * 8192 + (prow >> 3) * 1024 + (prow & 7) * 128 + ((c ^ (prow & 7)) << 4);
            } else {
                const int c = pw + j;                      // 16-byte chunk within the row
                off[j] = prow * 128 + ((c ^ (prow & 7)) << 4);
            }
        }
        int gshift = -1;                                  // log2(g) when g is a power of two
        if ((a.g & (a.g - 1)) == 0) gshift = __ffs(a.g) - 1;
        auto group_of = [&](int k) { return min(gshift >= 0 ? (k >> gshift) : k / a.g, a.G - 1); };
        const bool mbf = (a.fmt & kFmtMetaBf16) != 0;
        constexpr bool fz = FZ;     // a.fmt & kFmtZeroFloat, as a template argument
        // Scale / zero of one stage (tile i, block kb); with g a multiple of
        // 32 the thread's words share one group.
        constexpr int NG = PWG ? kTcWpt : 1;
        auto tile_r0 = [&](int i) { return (unit_of(i).t / tiles_m) * kTcBM; };
        auto load_sz = [&](int r0, int kb, float (&sv)[NG], float (&zv)[NG]) {
            const int n = TR ? kb * kTcBK + prow : r0 + prow;
            const int nc = min(n, a.N - 1);
            const __half* sp = a.S + static_cast<size_t>(nc) * a.sz_row;
            const __half* zp = a.Z + static_cast<size_t>(nc) * a.sz_row;
            const int kw0 = TR ? r0 / 8 + pw : kb * (kTcBK / 8) + pw;
#pragma unroll
            for (int j = 0; j < NG; ++j) {
                const int grp = group_of(8 * (kw0 + j));
                sv[j] = meta_to_float(__ldg(reinterpret_cast<const unsigned short*>(sp + grp)), mbf);
                zv[j] = meta_to_float(__ldg(reinterpret_cast<const unsigned short*>(zp + grp)), mbf);
            }
        };
        // (ci, ckb): unit and k-block of this group's current stage; cb1 is
        // the end of the unit's k-blocks.  Advancing by `step` stages walks
        // into the following units.
        auto advance = [&](int& i, int& kb, int& kb1, int step) {
            kb += step;
            while (i < my_units && kb >= kb1) {
                const int over = kb - kb1;
                if (++i >= my_units) break;
                const Unit w = unit_of(i);
                kb = w.kb0 + over;
                kb1 = w.kb1;
            }
        };
        int ci = 0, ckb = 0, cb1 = 0;
        if (my_units > 0) {
            const Unit w0 = unit_of(0);
            ckb = w0.kb0;
            cb1 = w0.kb1;
            advance(ci, ckb, cb1, grp_id);
        }
        int s = grp_id % NS;
        uint32_t phase = static_cast<uint32_t>(grp_id / NS) & 1u;
        float sv[NG], zv[NG], svn[NG], zvn[NG];
        int cr0 = ci < my_units ? tile_r0(ci) : 0;           // output row offset of the current tile
        if (ci < my_units && !a.sz_tma) load_sz(cr0, ckb, sv, zv);
        while (ci < my_units) {
            // the next stage of this group, whose scales are fetched now
            int ni = ci, nkb = ckb, nb1 = cb1;
            advance(ni, nkb, nb1, kTcDeqGroups);
            const bool more = ni < my_units;
            const int nr0 = (more && ni != ci) ? tile_r0(ni) : cr0;
            if (more && !a.sz_tma) load_sz(nr0, nkb, svn, zvn);
            const int r0 = cr0;
            const int n = TR ? ckb * kTcBK + prow : r0 + prow;
            const int kw0 = TR ? r0 / 8 + pw : ckb * (kTcBK / 8) + pw;
            const bool row_ok = n < a.N;
            const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&tma_full[s], phase, abort_flag,
                                                                      kErrTimeoutTmaFull));
            if (ok) {
                uint8_t* st = base + s * kStageBytes;
                if (a.sz_tma) {
                    // this stage's boxes: [S rows][8 groups] then [Z rows][8 groups]
                    const uint16_t* hs = reinterpret_cast<const uint16_t*>(st + kSzOff) + prow * 8;
                    const uint16_t* hz = hs + kSzRows * 8;
                    const int x0 = group_of(TR ? r0 : ckb * kTcBK) & ~7;
#pragma unroll
                    for (int j = 0; j < NG; ++j) {
                        const int idx = group_of(8 * (kw0 + j)) - x0;
                        sv[j] = meta_to_float(hs[idx], mbf);
                        zv[j] = meta_to_float(hz[idx], mbf);
                    }
                }
                const uint8_t* pk = st + kTcABytes + BN * 128 + prow * (TR ? 64 : 32) + pw * 4;
                uint32_t wv[kTcWpt];
                if constexpr (kTcWpt == 4) {
                    const uint4 v = *reinterpret_cast<const uint4*>(pk);
                    wv[0] = v.x;
                    wv[1] = v.y;
                    wv[2] = v.z;
                    wv[3] = v.w;
                } else {
                    const uint2 v = *reinterpret_cast<const uint2*>(pk);
                    wv[0] = v.x;
                    wv[1] = v.y;
                }
#pragma unroll
                for (int j = 0; j < kTcWpt; ++j) {
                    const uint32_t w = wv[j];
                    const float sj = sv[PWG ? j : 0], zj = zv[PWG ? j : 0];
                    uint4 out = make_uint4(0u, 0u, 0u, 0u);
                    if (row_ok && (kw0 + j) < W8)
                        out = fz ? dequant_word_bf16(w, sj, -(128.0f + zj), -(2048.0f + zj), true)
                                 : dequant_word_bf16(w, sj, -(128.0f + zj) * sj, -(2048.0f + zj) * sj, false);
                    *reinterpret_cast<uint4*>(st + off[j]) = out;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&deq_full[s]);
            }
            if (!a.sz_tma) {
#pragma unroll
                for (int j = 0; j < NG; ++j) {
                    sv[j] = svn[j];
                    zv[j] = zvn[j];
                }
            }
            ci = ni;
            ckb = nkb;
            cb1 = nb1;
            cr0 = nr0;
            s += kTcDeqGroups;
            while (s >= NS) {
                s -= NS;
                phase ^= 1u;
            }
        }
    } else {
        // ------------------------------------------------ epilogue
        const int q = warp & 3;                 // TMEM lanes 32 q .. 32 q + 31
        for (int i = 0; i < my_units; ++i) {
            const int buf = i & 1;
            const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&acc_full[buf], (i >> 1) & 1u, abort_flag,
                                                                      kErrTimeoutAccum));
            if (!ok || *abort_flag) break;
            tc_fence_after();
            const Unit w = unit_of(i);
            const int t = w.t;
            const int m0 = (t % tiles_m) * BN, r0 = (t / tiles_m) * kTcBM;
            const int row = r0 + 32 * q + lane;
            const bool rv = row < L_out;
            const float bias_f = (a.bias && rv) ? bf16_bits_to_float(a.bias[row]) : 0.0f;
            const uint32_t acc = tmem_d + static_cast<uint32_t>(buf) * kAccCols + (static_cast<uint32_t>(32 * q) << 16);
            // lanes pair up: for token column c0 + e the even lane of a pair
            // stores rows (row, row + 1) when e is even and the odd lane when
            // e is odd, as one 4-byte bf16x2; with L_out odd such a pair
            // would be misaligned, so every lane stores its own row instead
            const bool odd = (lane & 1) != 0;
            const int prow = row - (odd ? 1 : 0);            // first row of the pair
            const bool pv = prow < L_out;
            if (w.part >= 0) {
                // a k slice of a tail tile: fp32 partial [token][row] of the tile
                float* pt = a.part + static_cast<size_t>(w.part) * (BN * kTcBM) + 32 * q + lane;
#pragma unroll 1
                for (int c0 = 0; c0 < BN; c0 += 8) {
                    uint32_t r[8];
                    tmem_ld_x8(acc + static_cast<uint32_t>(c0), r);
#pragma unroll
                    for (int e = 0; e < 8; ++e) pt[(c0 + e) * kTcBM] = __uint_as_float(r[e]);
                }
            } else if (L_out & 1) {
#pragma unroll 1
                for (int c0 = 0; c0 < BN; c0 += 8) {
                    uint32_t r[8];
                    tmem_ld_x8(acc + static_cast<uint32_t>(c0), r);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int m = m0 + c0 + e;
                        if (rv && m < a.M)
                            a.Y[static_cast<size_t>(m) * L_out + row] =
                                __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(r[e]) + bias_f));
                    }
                }
            } else {
#pragma unroll 1
            for (int c0 = 0; c0 < BN; c0 += 8) {
                uint32_t r[8];
                tmem_ld_x8(acc + static_cast<uint32_t>(c0), r);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float v = __uint_as_float(r[e]) + bias_f;
                    const float o = __shfl_xor_sync(0xFFFFFFFFu, v, 1);
                    const int m = m0 + c0 + e;
                    if (((e & 1) != 0) == odd && pv && m < a.M) {
                        const float lo = odd ? o : v, hi = odd ? v : o;
                        *reinterpret_cast<uint32_t*>(a.Y + static_cast<size_t>(m) * L_out + prow) =
                            bf162_bits(__floats2bfloat162_rn(lo, hi));
                    }
                }
            }
            }
            // this warp's reads of the buffer are complete
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[buf]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        // a role gave up: let copies and mma already issued land (bounded)
        // before the tensor memory and the CTA's shared memory are released
        const unsigned long long t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 1000000ull) {
        }
    }
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_d),
                     "r"(kTmemCols)
                     : "memory");
    }
}

// The tail tiles of a split GEMM: out[m, row] = bf16(sum over the S slices
// of the tile's fp32 partials, in slice order, + bias[row]).  One thread per
// four consecutive rows of one token of a tile: its slice loads (float4,
// up to 8 at a time, indices past the last slice clamped to it and the
// values dropped) go out together; rows fastest, so reads and stores are
// coalesced.
__global__ void __launch_bounds__(256) gemm_tail_finalize_kernel(const float* __restrict__ part, int F, int S,
                                                                 int ntail, int tiles_m, int BN, int M, int L_out,
                                                                 const uint16_t* __restrict__ bias,
                                                                 uint16_t* __restrict__ Y) {
    pdl_wait();   // launched as a programmatic dependent of the GEMM
    const long long per_tile4 = static_cast<long long>(BN) * (kTcBM / 4);
    const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= per_tile4 * ntail) return;
    const int tt = static_cast<int>(idx / per_tile4);           // tail tile
    const int e4 = static_cast<int>(idx - tt * per_tile4);
    const int ml = e4 / (kTcBM / 4), rl = (e4 % (kTcBM / 4)) * 4;
    const int t = F + tt;
    const int m = (t % tiles_m) * BN + ml, row = (t / tiles_m) * kTcBM + rl;
    if (m >= M || row >= L_out) return;
    const float4* p = reinterpret_cast<const float4*>(part) + static_cast<size_t>(tt) * S * per_tile4 + e4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = 0; s0 < S; s0 += 8) {
        float4 v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = __ldg(p + static_cast<size_t>(min(s0 + j, S - 1)) * per_tile4);
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (s0 + j < S) {
                acc.x += v[j].x;
                acc.y += v[j].y;
                acc.z += v[j].z;
                acc.w += v[j].w;
            }
    }
    float r[4] = {acc.x, acc.y, acc.z, acc.w};
    uint16_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        if (bias && row + q < L_out) r[q] += bf16_bits_to_float(bias[row + q]);
        o[q] = __bfloat16_as_ushort(__float2bfloat16_rn(r[q]));
    }
    uint16_t* y = Y + static_cast<size_t>(m) * L_out + row;
    if ((L_out & 3) == 0) {              // row + 3 < L_out, and y is 8-byte aligned
        *reinterpret_cast<uint2*>(y) = make_uint2(o[0] | (static_cast<uint32_t>(o[1]) << 16),
                                                  o[2] | (static_cast<uint32_t>(o[3]) << 16));
    } else {
#pragma unroll
        for (int q = 0; q < 4; ++q)
            if (row + q < L_out) y[q] = o[q];
    }
}

}  // namespace w4
