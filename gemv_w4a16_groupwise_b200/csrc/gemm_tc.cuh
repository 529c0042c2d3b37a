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
// Warp roles (576 threads, one CTA per SM):
//   warp 0       TMA producer: packed weight tile + activation tile per stage
//   warp 1       TMEM allocator; lane 0 issues tcgen05.mma and commits
//   warps 2..17  dequantize packed codes into the bf16 A tile of a stage
//                (128-byte swizzled UMMA layout), then run the epilogue.
//                Two groups of 8 warps take alternate stages, so two stages
//                are being dequantized at any time and the tensor pipe is not
//                left waiting on one stage's dequantization latency.
// Every mbarrier wait is bounded; a wait that runs out records the reason in
// the device error word and the CTA unwinds without hanging.
//
// Dequantization of one packed word (8 codes) is exact up to the single
// bf16 rounding: each code becomes the fp32 value off + q (off = 128 or
// 2048) with one lop3, and one packed FMA per pair gives
//     (off + q) * s - (off + z) * s = (q - z) * s
// exactly in fp32 (both products need at most 23 significand bits), which
// cvt.rn.bf16x2 rounds once.
#pragma once

#include "tma.cuh"

namespace w4 {

constexpr int kTcDeqGroups = 2;                      // dequantizing warp groups (8 warps each)
constexpr int kTcThreads = 64 + kTcDeqGroups * 256;
constexpr int kTcBM = 128;     // MMA M (weight rows per tile)
constexpr int kTcBK = 64;      // reduction depth per pipeline stage
constexpr int kTcABytes = kTcBM * kTcBK * 2;   // 16 KB dequantized tile
constexpr int kTcPBytes = kTcBM * kTcBK / 2;   // 4 KB packed tile

struct TcArgs {
    const __half* S;
    const __half* Z;
    const uint16_t* bias;
    uint16_t* Y;
    int M, N, K;
    int g, G, sz_row;
    int stages;
};

struct TcProblem {
    const void* A;
    int M, N, K;
    const uint32_t* packed;
    const void* S;
    const void* Z;
    int g, G, sz_row;
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

__device__ __forceinline__ uint32_t bf162_bits(__nv_bfloat162 v) {
    return *reinterpret_cast<uint32_t*>(&v);
}

// Eight codes of one packed word -> eight bf16 (q - z) * s in k order.
__device__ __forceinline__ uint4 dequant_word_bf16(uint32_t w, float s, float c_lo, float c_hi) {
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
    const float2 f01 = ffma2(v01, ss, cc);
    const float2 f23 = ffma2(v23, ss, cc);
    const float2 f45 = ffma2(v45, ss, cc);
    const float2 f67 = ffma2(v67, ss, cc);
    uint4 out;
    out.x = bf162_bits(__floats2bfloat162_rn(f01.x, f01.y));
    out.y = bf162_bits(__floats2bfloat162_rn(f23.x, f23.y));
    out.z = bf162_bits(__floats2bfloat162_rn(f45.x, f45.y));
    out.w = bf162_bits(__floats2bfloat162_rn(f67.x, f67.y));
    return out;
}

template <bool TR, int BN, bool PWG>
__global__ void __launch_bounds__(kTcThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap pmap, const __grid_constant__ CUtensorMap bmap,
                   const TcArgs a) {
    static_assert(BN == 16 || BN == 32 || BN == 64 || BN == 128 || BN == 256, "BN");
    constexpr int kStageBytes = tc_stage_bytes(BN);
    constexpr uint32_t kTmemCols = BN < 32 ? 32 : BN;
    constexpr uint32_t kTxBytes = kTcPBytes + BN * 128;
    constexpr uint32_t kIdesc = umma_idesc_bf16(BN, TR);

    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int NS = a.stages;
    uint64_t* tma_full = reinterpret_cast<uint64_t*>(base + NS * kStageBytes);
    uint64_t* deq_full = tma_full + NS;
    uint64_t* empty = deq_full + NS;
    uint64_t* acc_full = empty + NS;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.x * BN;          // first token of the tile
    const int r0 = blockIdx.y * kTcBM;       // first output row (n, or k when transposed)
    const int L_out = TR ? a.K : a.N;        // output row length
    const int red_len = TR ? a.N : a.K;      // reduction length
    const int num_kb = (red_len + kTcBK - 1) / kTcBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&tma_full[s], 1);
            mbar_init(&deq_full[s], 8);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
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
            for (int kb = 0; kb < num_kb; ++kb) {
                const int s = kb % NS;
                const uint32_t use = static_cast<uint32_t>(kb / NS);
                if (use > 0 && !mbar_wait_bounded(&empty[s], (use - 1) & 1u, abort_flag, kErrTimeoutEmpty))
                    break;
                uint8_t* st = base + s * kStageBytes;
                mbar_arrive_expect_tx(&tma_full[s], kTxBytes);
                if (TR)
                    tma_load_2d(st + kTcABytes + BN * 128, &pmap, r0 / 8, kb * kTcBK, &tma_full[s]);
                else
                    tma_load_2d(st + kTcABytes + BN * 128, &pmap, kb * (kTcBK / 8), r0, &tma_full[s]);
                tma_load_2d(st + kTcABytes, &bmap, kb * kTcBK, m0, &tma_full[s]);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            bool ok = true;
            for (int kb = 0; kb < num_kb && ok; ++kb) {
                const int s = kb % NS;
                const uint32_t par = static_cast<uint32_t>(kb / NS) & 1u;
                ok = mbar_wait_bounded(&tma_full[s], par, abort_flag, kErrTimeoutTmaFull) &&
                     mbar_wait_bounded(&deq_full[s], par, abort_flag, kErrTimeoutDequant);
                if (!ok) break;
                tc_fence_after();
                const uint32_t a_addr = smem_u32(base + s * kStageBytes);
                const uint32_t b_addr = a_addr + kTcABytes;
#pragma unroll
                for (int i = 0; i < kTcBK / 16; ++i) {
                    const uint64_t adesc = TR ? umma_desc_sw128(a_addr + i * 2048, 8192, 1024)
                                              : umma_desc_sw128(a_addr + i * 32, 16, 1024);
                    const uint64_t bdesc = umma_desc_sw128(b_addr + i * 32, 16, 1024);
                    umma_bf16(tmem_d, adesc, bdesc, kIdesc, (kb | i) != 0 ? 1u : 0u);
                }
                umma_commit(&empty[s]);
            }
            umma_commit(acc_full);  // also tracks any MMA issued before an abort
        }
    } else {
        // ------------------------------------------------ dequantize
        const int grp_id = (threadIdx.x - 64) >> 8;           // this warp's group: stages kb = grp_id mod 2
        const int t = (threadIdx.x - 64) & 255;               // 0 .. 255 within the group
        // forward: row n = r0 + t % 128, words 4h .. 4h+3 of the 8 in a k-block
        // transposed: row n = kb * 64 + t % 64, words 4q .. 4q+3 of the 16 of a k-tile
        const int prow = TR ? (t & 63) : (t & 127);
        const int pquad = TR ? (t >> 6) : (t >> 7);
        const int W8 = a.K / 8;
        // swizzled 16-byte destinations of this thread's 4 words in the A tile
        uint32_t off[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (TR) {
                const int kk = 32 * pquad + 8 * j;        // k within the 128-wide tile
                const int atom = kk >> 6, c = (kk & 63) >> 3;
                off[j] = atom * 8192 + (prow >> 3) * 1024 + (prow & 7) * 128 + ((c ^ (prow & 7)) << 4);
            } else {
                const int c = 4 * pquad + j;               // 16-byte chunk within the row
                off[j] = prow * 128 + ((c ^ (prow & 7)) << 4);
            }
        }
        // Scale / zero of block kb, fetched one block ahead.  With g a
        // multiple of 32 the thread's 4 words share one group: forward, the
        // group moves by at most 64 / g per block and is tracked by
        // subtraction; transposed, it is fixed and only the row moves.
        constexpr int NG = PWG ? 4 : 1;
        const int kw_t = TR ? r0 / 8 + 4 * pquad : 4 * pquad;   // forward: + kb * 8
        int grp_f = 0, rem_f = 0;                               // forward: (8 kw0) = grp_f * g + rem_f
        if (!PWG && !TR) {
            grp_f = (8 * kw_t) / a.g;
            rem_f = 8 * kw_t - grp_f * a.g;
        }
        const int grp_t = (!PWG && TR) ? min((8 * kw_t) / a.g, a.G - 1) : 0;
        auto load_sz = [&](int kb, float (&sv)[NG], float (&zv)[NG]) {
            const int n = TR ? kb * kTcBK + prow : r0 + prow;
            const int nc = min(n, a.N - 1);
            const __half* sp = a.S + static_cast<size_t>(nc) * a.sz_row;
            const __half* zp = a.Z + static_cast<size_t>(nc) * a.sz_row;
            if (PWG) {
                const int kw0 = TR ? kw_t : kb * (kTcBK / 8) + kw_t;
#pragma unroll
                for (int j = 0; j < NG; ++j) {
                    const int grp = min((8 * (kw0 + j)) / a.g, a.G - 1);
                    sv[j] = __half2float(__ldg(sp + grp));
                    zv[j] = __half2float(__ldg(zp + grp));
                }
            } else {
                const int grp = TR ? grp_t : min(grp_f, a.G - 1);
                sv[0] = __half2float(__ldg(sp + grp));
                zv[0] = __half2float(__ldg(zp + grp));
            }
        };
        auto next_group = [&]() {   // forward, g a multiple of 32: advance this group's stride of k-blocks
            if (!PWG && !TR) {
                rem_f += kTcBK * kTcDeqGroups;
                while (rem_f >= a.g) {
                    rem_f -= a.g;
                    ++grp_f;
                }
            }
        };
        if (!PWG && !TR) {   // start at this group's first block
            rem_f += kTcBK * grp_id;
            while (rem_f >= a.g) {
                rem_f -= a.g;
                ++grp_f;
            }
        }
        float sv[NG], zv[NG], svn[NG], zvn[NG];
        if (grp_id < num_kb) load_sz(grp_id, sv, zv);
        next_group();
        for (int kb = grp_id; kb < num_kb; kb += kTcDeqGroups) {
            const int s = kb % NS;
            const uint32_t par = static_cast<uint32_t>(kb / NS) & 1u;
            if (kb + kTcDeqGroups < num_kb) load_sz(kb + kTcDeqGroups, svn, zvn);
            next_group();
            const int n = TR ? kb * kTcBK + prow : r0 + prow;
            const int kw0 = TR ? kw_t : kb * (kTcBK / 8) + kw_t;
            const bool row_ok = n < a.N;
            const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&tma_full[s], par, abort_flag,
                                                                      kErrTimeoutTmaFull));
            if (ok) {
                uint8_t* st = base + s * kStageBytes;
                const uint8_t* pk = st + kTcABytes + BN * 128;
                const uint4 wv = TR ? *reinterpret_cast<const uint4*>(pk + prow * 64 + pquad * 16)
                                    : *reinterpret_cast<const uint4*>(pk + prow * 32 + pquad * 16);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t w = (j == 0) ? wv.x : (j == 1) ? wv.y : (j == 2) ? wv.z : wv.w;
                    const float sj = sv[PWG ? j : 0], zj = zv[PWG ? j : 0];
                    uint4 out = make_uint4(0u, 0u, 0u, 0u);
                    if (row_ok && (kw0 + j) < W8)
                        out = dequant_word_bf16(w, sj, -(128.0f + zj) * sj, -(2048.0f + zj) * sj);
                    *reinterpret_cast<uint4*>(st + off[j]) = out;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&deq_full[s]);
            }
#pragma unroll
            for (int j = 0; j < NG; ++j) {
                sv[j] = svn[j];
                zv[j] = zvn[j];
            }
        }

        // ------------------------------------------------ epilogue
        const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(acc_full, 0u, abort_flag,
                                                                  kErrTimeoutAccum));
        if (ok && !*abort_flag) {
            tc_fence_after();
            // warp w reads TMEM lanes 32 (w % 4) .. + 31; the 16 epilogue
            // warps split the BN columns into up to 4 parts of >= 8
            const int q = warp & 3;
            constexpr int kParts = BN / 8 < 4 ? BN / 8 : 4;
            const int part = (warp - 2) >> 2;
            const int row = r0 + 32 * q + lane;
            const bool rv = row < L_out;
            const float bias_f = (a.bias && rv) ? bf16_bits_to_float(a.bias[row]) : 0.0f;
#pragma unroll 1
            for (int c0 = part * (BN / kParts); part < kParts && c0 < (part + 1) * (BN / kParts); c0 += 8) {
                uint32_t r[8];
                tmem_ld_x8(tmem_d + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(c0), r);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int m = m0 + c0 + e;
                    if (rv && m < a.M)
                        a.Y[static_cast<size_t>(m) * L_out + row] =
                            __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(r[e]) + bias_f));
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_d),
                     "r"(kTmemCols)
                     : "memory");
    }
}

}  // namespace w4

