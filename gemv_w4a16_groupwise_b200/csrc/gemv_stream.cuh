// Forward GEMV for M <= 4 that streams contiguous weight rows.
//
// On B200, HBM reaches its measured copy bandwidth only when each request
// stream covers long contiguous runs: boxes of 4 rows x 1 KB read at
// ~6.3 TB/s with two 4 KB stages per warp, while 128-row x 64-byte boxes (a
// lane per row) stay near 3 TB/s.  So each warp here owns 4 consecutive
// weight rows and walks them along K in boxes of 4 rows x 1024 bytes
// (2048 k), delivered by TMA into the warp's private stages and refilled by
// the warp itself as soon as it has read them (one consumer per stage, its
// phases in order).
//
// Activations.  A small kernel (gemv_xprep_kernel) first turns X into the
// form the inner loop consumes, once per call: per 32-k chunk, the largest
// bf16 exponent e of the chunk and every value as a 16-bit fixed-point
// integer x' = round(x * 2^(141 - e)) (exact for values within 2^7 of the
// chunk maximum, rounded to 2^-15 of it below), split into a signed high
// byte and an unsigned low byte, with the bytes of even and odd k in
// separate words so that they line up with the even / odd nibbles of a
// packed word; plus the chunk's scale 2^(e - 141) and the exact sum of x'.
// The block of a K slice is laid out exactly as the stream kernel keeps it
// in shared memory, and each CTA fetches it with one bulk copy.
//
// Inner loop.  Lanes work along K: in a box, lane l owns the 32-k chunks l
// and l + 32 of every row.  A packed word splits into its even and odd
// nibbles (4 codes each, one per byte), and dp4a multiplies four codes by
// four activation bytes, so a word costs 4 dp4a per activation row; sums
// are exact in int32.  Per (row, chunk), with the chunk inside one group,
//     y += s * 2^(e - 141) * (sum_k q_k x'_k - z * sum_k x'_k)
// in fp32.
//
// Work: a warp item is 4 rows x one k-part of the CTA's K slice; a round
// gives each of the 8 warps one item (RBP row blocks x KP k-parts).  At the
// end of an item a butterfly over the lanes reduces the 4 rows; at the end
// of a round the CTA adds the k-parts of every row in a fixed order and
// writes Y (+ bias), or fp32 partials when K is split across slices (only
// when the M x K activation block does not fit in shared memory).
// Persistent CTAs walk a contiguous range of (slice, round) units.
#pragma once

#include "gemv.cuh"

namespace w4 {

constexpr int kSW = 8;                 // warps per CTA
constexpr int kSR = 4;                 // rows per box / item
constexpr int kSBK = 2048;             // k per box (1024 bytes of packed row)
constexpr int kSBBytes = kSR * 1024;   // 4 KB per box
constexpr int kSRecs = 4;              // 16-byte records per 32-k chunk and activation row
constexpr int kSFrac = 7;              // fixed-point bits below the chunk's leading binade

// One slice's activation block: [m][record][chunk] uint4, then the chunk
// scales [m][chunk] and the chunk sums [m][chunk] (fp32).
__host__ __device__ inline size_t gemv_stream_xblock_bytes(int M, int TKC) {
    const size_t nchunk = static_cast<size_t>(TKC) / 32;
    return static_cast<size_t>(M) * nchunk * (kSRecs * 16 + 8);
}

// 32-bit words of scale (or zero) that one row of a box needs: the fp16
// values of the groups that 2048 k touch, starting at the aligned word that
// holds the first one.
__host__ __device__ inline int gemv_stream_sz_words(int g) {
    return ((kSBK + g - 1) / g + 3 + 1) / 2;
}

// One stage: the 4 x 1 KB weight box, then [s|z][4 rows][szw] words.
__host__ __device__ inline int gemv_stream_stage_bytes(int szw) {
    return (kSBBytes + 2 * kSR * szw * 4 + 127) / 128 * 128;
}

__host__ __device__ inline size_t gemv_stream_smem_bytes(int M, int TKC, int stages, int szw) {
    size_t b = 1024;                                                      // alignment slack
    b += static_cast<size_t>(kSW) * stages * gemv_stream_stage_bytes(szw); // TMA ring
    b += gemv_stream_xblock_bytes(M, TKC);                                // activation block
    b += static_cast<size_t>(kSW) * kSR * M * 4;                          // item row totals
    b += static_cast<size_t>(kSW) * stages * 8 + 8 + 16;                  // barriers + flag
    return b;
}

// b * 2^(134 - emax + frac) rounded to an integer (half away from zero):
// a bf16 is mant * 2^(e - 134), mant holding the implicit bit.
__device__ __forceinline__ int bf16_fixed_bits(uint32_t b, int emax, int frac) {
    const int e = (b >> 7) & 0xFF;
    const int mant = e ? (0x80 | (b & 0x7F)) : (b & 0x7F);
    const int sh = (e ? e : 1) - emax + frac;
    int v;
    if (sh >= 0) v = mant << sh;
    else if (sh > -9) v = (mant + (1 << (-sh - 1))) >> (-sh);
    else v = 0;
    return (b & 0x8000u) ? -v : v;
}

// One thread per (slice, m, chunk): writes that chunk's 4 records, scale
// and sum into the slice's block.  Chunks past K read as zero.
__global__ void __launch_bounds__(256) gemv_xprep_kernel(const uint16_t* __restrict__ X, int M, int K,
                                                         int TKC, int splits, uint8_t* __restrict__ out) {
    const int nchunk = TKC / 32;
    const long long total = static_cast<long long>(splits) * M * nchunk;
    const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= total) return;
    const int slice = static_cast<int>(idx / (static_cast<long long>(M) * nchunk));
    const int rem = static_cast<int>(idx - static_cast<long long>(slice) * M * nchunk);
    const int m = rem / nchunk, c = rem - (rem / nchunk) * nchunk;
    const long long k0 = static_cast<long long>(slice) * TKC + static_cast<long long>(c) * 32;
    uint32_t r[16];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (k0 + 8 * q < K)
            v = __ldg(reinterpret_cast<const uint4*>(X + static_cast<size_t>(m) * K + k0 + 8 * q));
        r[4 * q] = v.x;
        r[4 * q + 1] = v.y;
        r[4 * q + 2] = v.z;
        r[4 * q + 3] = v.w;
    }
    int emax = 1;
#pragma unroll
    for (int q = 0; q < 16; ++q) emax = max(emax, max(bf16_exp1(r[q] & 0xFFFFu), bf16_exp1(r[q] >> 16)));
    uint8_t* block = out + static_cast<size_t>(slice) * gemv_stream_xblock_bytes(M, TKC);
    uint4* planes = reinterpret_cast<uint4*>(block);
    float* cscale = reinterpret_cast<float*>(planes + static_cast<size_t>(M) * kSRecs * nchunk);
    float* csum = cscale + static_cast<size_t>(M) * nchunk;
    int sum = 0;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        uint32_t hi[2] = {0u, 0u}, lo[2] = {0u, 0u};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            // element 8w + e of the chunk; even e pair with the low nibbles
            const uint32_t word = r[4 * w + (e >> 1)];
            const uint32_t bits = (e & 1) ? (word >> 16) : (word & 0xFFFFu);
            const int xf = bf16_fixed_bits(bits, emax, kSFrac);
            sum += xf;
            hi[e & 1] |= (static_cast<uint32_t>(xf >> 8) & 0xFFu) << (8 * (e >> 1));
            lo[e & 1] |= (static_cast<uint32_t>(xf) & 0xFFu) << (8 * (e >> 1));
        }
        planes[(static_cast<size_t>(m) * kSRecs + w) * nchunk + c] = make_uint4(hi[0], hi[1], lo[0], lo[1]);
    }
    cscale[m * nchunk + c] = ldexpf(1.0f, emax - 134 - kSFrac);
    csum[m * nchunk + c] = static_cast<float>(sum);
}

struct GemvStreamArgs {
    const uint8_t* xblocks;   // [splits] activation blocks from gemv_xprep_kernel
    const __half* S;
    const __half* Z;
    const uint16_t* bias;
    uint16_t* Y;
    float* partial;           // [splits, M, N] when splits > 1
    int N, K, g, G, sz_row;
    int TKC;                  // k per slice (a whole number of boxes)
    int splits;               // slices
    int nbs;                  // boxes per slice
    int KP;                   // k-parts per slice
    int RBP;                  // 4-row blocks per round (RBP * KP == kSW)
    int rounds;               // rounds per slice
    int units;                // splits * rounds
    int stages;               // TMA stages per warp
    int szw;                  // scale / zero words per row and stage
    long long sz_total;       // halves in each of S and Z (N * sz_row, or 1)
    int M;                    // activation rows (the tensor-pipe kernel takes it at run time)
};

// 1-D bulk copy global -> shared, completing on `bar` (16-byte aligned
// addresses, size a multiple of 16).
__device__ __forceinline__ void bulk_load_1d(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(gsrc)), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// 4-byte cp.async that reads `src_bytes` (0, 2 or 4) and zero-fills the rest.
__device__ __forceinline__ void cp_async_4(void* smem_dst, const void* gsrc, uint32_t src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(smem_dst)),
                 "l"(reinterpret_cast<uint64_t>(gsrc)), "r"(src_bytes)
                 : "memory");
}

// Arrive on `bar` once this thread's earlier cp.async copies have landed
// (the arrival is counted in the barrier's initial count).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Where the groups of a box's chunks lie, fixed per launch:
//   kGroupsOne   one group per row (rowwise / global): group 0 everywhere;
//   kGroupsPow2  g divides 2048 (a power of two): chunk d of a box is in
//                group k0 / g + (32 d) >> log2(g);
//   kGroupsAny   any other multiple of 32: divisions per box.
enum GroupKind { kGroupsOne = 0, kGroupsPow2 = 1, kGroupsAny = 2 };

template <int M, int GK>
__global__ void __launch_bounds__(kSW * 32, 1)
    gemv_stream_kernel(const __grid_constant__ CUtensorMap wmap, const GemvStreamArgs a) {
    static_assert(M >= 1 && M <= 4, "M");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int NS = a.stages;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
    const int nchunk = a.TKC / 32;
    const uint32_t xbytes = static_cast<uint32_t>(gemv_stream_xblock_bytes(M, a.TKC));
    const int SB = gemv_stream_stage_bytes(a.szw);
    uint8_t* ring = base;                                                       // [warp][stage][SB]
    uint8_t* xblk = ring + kSW * NS * SB;
    const uint4* planes = reinterpret_cast<const uint4*>(xblk);                 // [m][rec][chunk]
    const float* cscale = reinterpret_cast<const float*>(planes + M * kSRecs * nchunk);
    const float* csum = cscale + M * nchunk;
    float* part = reinterpret_cast<float*>(xblk + xbytes);                      // [warp][4 rows][M]
    uint64_t* full = reinterpret_cast<uint64_t*>(part + kSW * kSR * M);
    uint64_t* xbar = full + kSW * NS;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(xbar + 1);

    if (tid == 0) {
        // a stage completes on lane 0's expect-tx arrival plus the TMA bytes
        // and one cp.async arrival from each of the 32 lanes
        for (int i = 0; i < kSW * NS; ++i) mbar_init(&full[i], 33);
        mbar_init(xbar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (tid == 32) tma_prefetch_desc(&wmap);
    __syncthreads();

    const int u_begin = static_cast<int>(static_cast<long long>(blockIdx.x) * a.units / gridDim.x);
    const int u_end = static_cast<int>(static_cast<long long>(blockIdx.x + 1) * a.units / gridDim.x);
    // this warp's item in every round: row block rbl, k-part kp = boxes
    // [b_lo, b_lo + BPI) of the slice
    const int rbl = warp / a.KP, kp = warp - rbl * a.KP;
    const int b_lo = kp * a.nbs / a.KP;
    const int BPI = (kp + 1) * a.nbs / a.KP - b_lo;
    int gshift = 0;
    if (GK == kGroupsPow2) gshift = __ffs(a.g) - 1;

    // position in the warp's box sequence: unit u = (slice, round rd), box bi
    struct Cur {
        int u, slice, rd, bi;
    };
    auto advance = [&](Cur& c) {
        if (++c.bi >= BPI) {
            c.bi = 0;
            ++c.u;
            if (++c.rd == a.rounds) {
                c.rd = 0;
                ++c.slice;
            }
        }
    };
    const int slice0 = u_begin / a.rounds;
    const Cur start{u_begin, slice0, u_begin - slice0 * a.rounds, 0};
    auto box_k0 = [&](const Cur& c) { return c.slice * a.TKC + (b_lo + c.bi) * kSBK; };
    auto box_row0 = [&](const Cur& c) { return (c.rd * a.RBP + rbl) * kSR; };
    auto first_group = [&](int k0) {
        if (GK == kGroupsOne) return 0;
        if (GK == kGroupsPow2) return k0 >> gshift;
        return k0 / a.g;
    };

    // Filling a stage: the weight box by TMA, and the scale / zero words of
    // the box's groups for its 4 rows by cp.async (lane l copies words
    // l >> 3, + 4, ... of array (l >> 2) & 1, row l & 3), so that they arrive
    // as far ahead as the weights.  Words past the end of S / Z read as 0.
    const int sz_arr = (lane >> 2) & 1, sz_row_i = lane & 3;
    const __half* sz_src = sz_arr ? a.Z : a.S;
    int islot = 0;
    Cur ic = start;
    auto issue = [&]() {
        if (BPI > 0 && ic.u < u_end) {
            const int k0 = box_k0(ic), row0 = box_row0(ic);
            const int st = warp * NS + islot;
            uint8_t* sd = ring + st * SB;
            const long long h0 =
                (static_cast<long long>(row0 + sz_row_i) * a.sz_row + first_group(k0)) & ~1ll;
            uint32_t* szd = reinterpret_cast<uint32_t*>(sd + kSBBytes) + (sz_arr * kSR + sz_row_i) * a.szw;
            for (int w = lane >> 3; w < a.szw; w += 4) {
                const long long h = h0 + 2 * w;
                const long long avail = a.sz_total - h;
                const uint32_t bytes = avail >= 2 ? 4u : (avail == 1 ? 2u : 0u);
                cp_async_4(szd + w, sz_src + (bytes ? h : 0), bytes);
            }
            cp_async_arrive_noinc(&full[st]);
            if (lane == 0 && !*abort_flag) {
                fence_proxy_async_smem();
                mbar_arrive_expect_tx(&full[st], kSBBytes);
                tma_load_2d(sd, &wmap, k0 / 8, row0, &full[st]);
            }
            if (++islot == NS) islot = 0;
            advance(ic);
        }
    };
    for (int b = 0; b < NS; ++b) issue();

    // group offset of this lane's chunk j (k offset 32 lane + 1024 j in the
    // box) from the box's first group
    int dj[2] = {0, 0};
    if (GK == kGroupsPow2) {
        dj[0] = (32 * lane) >> gshift;
        dj[1] = (32 * lane + 1024) >> gshift;
    }

    int cslot = 0;
    uint32_t cpar = 0, xpar = 0;
    Cur cc = start;
    int cur_slice = -1;
    float y[kSR][M];

    for (int u = u_begin; u < u_end; ++u) {
        const int slice = cc.slice, rd = cc.rd;
        if (slice != cur_slice) {
            // every warp is past the previous round's final barrier, so the
            // old block is no longer read: fetch this slice's block
            if (tid == 0 && !*abort_flag) {
                fence_proxy_async_smem();
                mbar_arrive_expect_tx(xbar, xbytes);
                bulk_load_1d(xblk, a.xblocks + static_cast<size_t>(slice) * xbytes, xbytes, xbar);
            }
            mbar_wait_bounded(xbar, xpar, abort_flag, kErrTimeoutTmaFull);
            xpar ^= 1u;
            cur_slice = slice;
        }
#pragma unroll
        for (int i = 0; i < kSR; ++i)
#pragma unroll
            for (int m = 0; m < M; ++m) y[i][m] = 0.0f;

        for (int bi = 0; bi < BPI; ++bi) {
            const int k0 = box_k0(cc), row0 = box_row0(cc);
            const int st = warp * NS + cslot;
            __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&full[st], cpar, abort_flag, kErrTimeoutTmaFull));
            if (++cslot == NS) {
                cslot = 0;
                cpar ^= 1u;
            }
            const uint8_t* sb = ring + st * SB;
            const __half* szh = reinterpret_cast<const __half*>(sb + kSBBytes);
            const int grp_lo = first_group(k0);
            if (GK == kGroupsAny) {
                const int r0 = k0 - grp_lo * a.g;
                dj[0] = (r0 + 32 * lane) / a.g;
                dj[1] = (r0 + 32 * lane + 1024) / a.g;
            }
            // half offset of row i's first group in its copied words
            int roff[kSR];
#pragma unroll
            for (int i = 0; i < kSR; ++i)
                roff[i] = i * 2 * a.szw + ((((row0 + i) & a.sz_row) ^ grp_lo) & 1);
            const int cbase = (b_lo + bi) * (kSBK / 32);   // first chunk of the box in the slice
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int c = cbase + lane + 32 * j;           // this lane's chunk
                float sc[kSR], zc[kSR];
#pragma unroll
                for (int i = 0; i < kSR; ++i) {
                    sc[i] = __half2float(szh[roff[i] + dj[j]]);
                    zc[i] = __half2float(szh[roff[i] + kSR * 2 * a.szw + dj[j]]);
                }
                uint4 wv[kSR];
#pragma unroll
                for (int i = 0; i < kSR; ++i)
                    wv[i] = *reinterpret_cast<const uint4*>(sb + i * 1024 + (lane + 32 * j) * 16);
                int ah[kSR][M];
                uint32_t al[kSR][M];
#pragma unroll
                for (int i = 0; i < kSR; ++i)
#pragma unroll
                    for (int m = 0; m < M; ++m) {
                        ah[i][m] = 0;
                        al[i][m] = 0u;
                    }
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    uint32_t ev[kSR], od[kSR];
#pragma unroll
                    for (int i = 0; i < kSR; ++i) {
                        const uint32_t word = (w == 0) ? wv[i].x : (w == 1) ? wv[i].y : (w == 2) ? wv[i].z : wv[i].w;
                        ev[i] = word & 0x0F0F0F0Fu;          // codes of k = 8w + 0, 2, 4, 6
                        od[i] = (word >> 4) & 0x0F0F0F0Fu;   // codes of k = 8w + 1, 3, 5, 7
                    }
#pragma unroll
                    for (int m = 0; m < M; ++m) {
                        const uint4 xr = planes[(m * kSRecs + w) * nchunk + c];
#pragma unroll
                        for (int i = 0; i < kSR; ++i) {
                            ah[i][m] = dp4a_us(ev[i], xr.x, ah[i][m]);
                            ah[i][m] = dp4a_us(od[i], xr.y, ah[i][m]);
                            al[i][m] = dp4a_uu(ev[i], xr.z, al[i][m]);
                            al[i][m] = dp4a_uu(od[i], xr.w, al[i][m]);
                        }
                    }
                }
                // fold the chunk: s * 2^(e - 141) * (sum q x' - z sum x')
#pragma unroll
                for (int m = 0; m < M; ++m) {
                    const float xs = cscale[m * nchunk + c];
                    const float xsum = csum[m * nchunk + c];
#pragma unroll
                    for (int i = 0; i < kSR; ++i) {
                        const float qx = static_cast<float>(ah[i][m] * 256 + static_cast<int>(al[i][m]));
                        y[i][m] = fmaf(sc[i] * xs, fmaf(-zc[i], xsum, qx), y[i][m]);
                    }
                }
            }
            __syncwarp();
            issue();                                   // refill the stage just read
            advance(cc);
        }

        // end of this warp's item: butterfly over the lanes; afterwards the
        // lanes with (lane & 7) == 0 hold row 2 * (lane >> 4) + ((lane >> 3) & 1)
#pragma unroll
        for (int m = 0; m < M; ++m) {
            float v0, v1;
            {
                const bool up = lane & 16;
                const float s0 = up ? y[0][m] : y[2][m], s1 = up ? y[1][m] : y[3][m];
                const float k0 = up ? y[2][m] : y[0][m], k1 = up ? y[3][m] : y[1][m];
                v0 = k0 + __shfl_xor_sync(0xFFFFFFFFu, s0, 16);
                v1 = k1 + __shfl_xor_sync(0xFFFFFFFFu, s1, 16);
            }
            {
                const bool up = lane & 8;
                const float s = up ? v0 : v1, k = up ? v1 : v0;
                v0 = k + __shfl_xor_sync(0xFFFFFFFFu, s, 8);
            }
            v0 += __shfl_xor_sync(0xFFFFFFFFu, v0, 4);
            v0 += __shfl_xor_sync(0xFFFFFFFFu, v0, 2);
            v0 += __shfl_xor_sync(0xFFFFFFFFu, v0, 1);
            if ((lane & 7) == 0) {
                const int row = 2 * (lane >> 4) + ((lane >> 3) & 1);
                part[(warp * kSR + row) * M + m] = v0;
            }
        }
        // end of the round: add the k-parts of each row in ascending order,
        // then write Y (+ bias) or the slice's partials
        __syncthreads();
        for (int o = tid; o < a.RBP * kSR * M; o += kSW * 32) {
            const int rb2 = o / (kSR * M);
            const int rem = o - rb2 * kSR * M;
            const int r = rem / M, m = rem - (rem / M) * M;
            const int n = (rd * a.RBP + rb2) * kSR + r;
            if (n < a.N) {
                float sacc = 0.0f;
                for (int p = 0; p < a.KP; ++p) sacc += part[((rb2 * a.KP + p) * kSR + r) * M + m];
                if (a.splits == 1) {
                    if (a.bias) sacc += bf16_bits_to_float(a.bias[n]);
                    a.Y[static_cast<size_t>(m) * a.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(sacc));
                } else {
                    a.partial[(static_cast<size_t>(slice) * M + m) * a.N + n] = sacc;
                }
            }
        }
        __syncthreads();
    }
    if (*abort_flag) {
        // a wait gave up: let copies already issued land before the CTA exits
        const unsigned long long t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 1000000ull) {
        }
    }
}

}  // namespace w4
