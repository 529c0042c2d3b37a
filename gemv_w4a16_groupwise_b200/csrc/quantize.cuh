// Quantize bf16 W [N, K] to uint4 codes and pack eight codes per uint32
// along K (llm-quantization, "Objectives" 1; modes GLOBAL / ROWWISE /
// GROUPWISE from its mode table).  Memory bound: W is read once (twice for
// groups that do not fit a warp segment, the second read hitting L2), the
// packed words and the fp16 scale / zero are written once.
//
// Per group, in IEEE fp32 with round-half-even and no contraction:
//     s = fp16((max - min) / 15); if s == 0: s = fp16(max(|min|, 2^-14))
//     z = clamp(rint(-min / s), 0, 15)
//     q = clamp(rint(w / s) + z, 0, 15)
// Clamps use fmaxf/fminf (a NaN lands on 0) and then convert to int, so a
// negative zero never reaches the stored fp16 zero point.
// Format flags (or-ed into the mode) give the HQQ-style variant of
// "Re-write HQQ Fused Gemm Transpose" and bf16 metadata:
//     fractional zero:  z = meta(-min / s) (kept finite in its type, not
//                       rounded or clamped), q = clamp(rint(w / s + z), 0, 15)
//     bf16 metadata:    every fp16 rounding above is a bf16 rounding.
#pragma once

#include "common.cuh"

namespace w4 {

struct GroupParams {
    uint16_t sb, zb;   // stored bits of s and z (fp16, or bf16)
    float sf;          // value of s
    float rs;          // 1 / sf, correctly rounded
    float zf;          // value of z (an integer unless the zero is fractional)
    bool fz;           // fractional zero point
};

// Nearest value of the metadata type (fp16 or bf16), as stored bits.
__device__ __forceinline__ uint16_t meta_bits_rn(float v, bool bf16) {
    return bf16 ? __bfloat16_as_ushort(__float2bfloat16_rn(v)) : __half_as_ushort(__float2half_rn(v));
}

__device__ __forceinline__ GroupParams group_params_from_range(float mn, float mx, int flags) {
    GroupParams p;
    const bool bf = (flags & kFmtMetaBf16) != 0;
    p.fz = (flags & kFmtZeroFloat) != 0;
    const float range = __fsub_rn(mx, mn);
    uint16_t sb = meta_bits_rn(__fdiv_rn(range, 15.0f), bf);
    if (meta_to_float(sb, bf) == 0.0f) sb = meta_bits_rn(fmaxf(fabsf(mn), 0x1p-14f), bf);
    p.sb = sb;
    p.sf = meta_to_float(sb, bf);
    p.rs = __frcp_rn(p.sf);
    if (p.fz) {
        const float zmax = bf ? 0x1.FEp127f : 65504.0f;      // largest finite value of the type
        p.zb = meta_bits_rn(fminf(fmaxf(__fdiv_rn(-mn, p.sf), -zmax), zmax), bf);
        p.zf = meta_to_float(p.zb, bf);
    } else {
        p.zf = fminf(fmaxf(rintf(__fdiv_rn(-mn, p.sf)), 0.0f), 15.0f);
        p.zb = meta_bits_rn(static_cast<float>(static_cast<int>(p.zf)), bf);   // no negative zero
    }
    return p;
}

// rint(w / s) as IEEE fp32 division followed by rint gives it, without the
// division for all but near-tie quotients.  t = w * (1/s) is within about
// 2^-23 relative of w / s, and so is the correctly rounded quotient.  The
// exact integer only matters while the code is not clamped, i.e. for
// |t| <= 15 + 15 (z <= 15); there both lie within 2^-18 of w / s, so when t
// is farther than 2^-11 from every half-integer they round to the same
// integer.  For larger |t| the clamp gives 0 or 15 either way.  Otherwise
// (and for NaN or infinity) the division is done exactly.
__device__ __forceinline__ float rint_quotient(float w, const GroupParams& p) {
    const float t = w * p.rs;
    const float k = rintf(t);
    if (fabsf(t - k) < 0.5f - 0x1p-11f) return k;
    return rintf(__fdiv_rn(w, p.sf));
}

// rint(fp32(fp32(w / s) + z)) for a fractional z, through the same
// reciprocal: t = w * (1/s) is within 2^-22 |t| of fp32(w / s), so u = t + z
// is within 2^-22 |t| + one ulp of u of the exact sum's fp32 value; when u
// is farther than that from every half-integer both round alike, else the
// division and the sum are done exactly.
__device__ __forceinline__ float rint_shifted_quotient(float w, const GroupParams& p) {
    const float t = w * p.rs;
    const float u = __fadd_rn(t, p.zf);
    const float k = rintf(u);
    const float margin = (fabsf(t) + 4.0f * fabsf(u)) * 0x1p-22f;
    if (fabsf(u - k) < 0.5f - margin) return k;
    return rintf(__fadd_rn(__fdiv_rn(w, p.sf), p.zf));
}

__device__ __forceinline__ uint32_t quantize_code(float w, const GroupParams& p) {
    float t = p.fz ? rint_shifted_quotient(w, p) : __fadd_rn(rint_quotient(w, p), p.zf);
    t = fminf(fmaxf(t, 0.0f), 15.0f);
    // t is an integer in [0, 15]: adding 2^23 leaves it in the low mantissa bits
    return __float_as_uint(__fadd_rn(t, 8388608.0f)) & 0xFu;
}

__device__ __forceinline__ void unpack8_bf16(const uint4 raw, float (&v)[8]) {
    const uint32_t r[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(r[i] << 16);
        v[2 * i + 1] = __uint_as_float(r[i] & 0xFFFF0000u);
    }
}

__device__ __forceinline__ uint32_t pack8(const float (&v)[8], const GroupParams& p) {
    uint32_t word = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) word |= quantize_code(v[i], p) << (4 * i);
    return word;
}

// Groups of g = 8 * WPT * LPG elements, LPG a power of two <= 32: each
// thread owns WPT consecutive 16-byte chunks (8 values, one packed word
// each) of one group; the LPG lanes of a group reduce min / max with
// shuffles inside their aligned lane segment.  The format flags are a
// template argument: the choice between the integer and the fractional
// zero point's rounding is then made at compile time instead of once per
// code (a runtime flag cost this kernel 8 %).
template <int LPG, int WPT, int FLAGS>
__global__ void __launch_bounds__(256) quantize_segmented_kernel(
    const uint16_t* __restrict__ W, long long total_words, uint32_t* __restrict__ packed,
    uint16_t* __restrict__ scales, uint16_t* __restrict__ zeros) {
    constexpr int flags = FLAGS;
    const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    const long long w0 = t * WPT;                      // first word of the thread
    const bool active = w0 < total_words;
    const long long tw = active ? w0 : (total_words - WPT);
    float v[WPT][8];
#pragma unroll
    for (int j = 0; j < WPT; ++j) unpack8_bf16(__ldg(reinterpret_cast<const uint4*>(W) + tw + j), v[j]);
    float mn = v[0][0], mx = v[0][0];
#pragma unroll
    for (int j = 0; j < WPT; ++j)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            mn = fminf(mn, v[j][i]);
            mx = fmaxf(mx, v[j][i]);
        }
#pragma unroll
    for (int off = 1; off < LPG; off <<= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, off));
        mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
    }
    const GroupParams p = group_params_from_range(mn, mx, flags);
    if (!active) return;
    if (WPT == 2) {
        *reinterpret_cast<uint2*>(packed + w0) = make_uint2(pack8(v[0], p), pack8(v[1], p));
    } else {
#pragma unroll
        for (int j = 0; j < WPT; ++j) packed[w0 + j] = pack8(v[j], p);
    }
    if ((threadIdx.x & (LPG - 1)) == 0) {
        const long long grp = t / LPG;
        scales[grp] = p.sb;
        zeros[grp] = p.zb;
    }
}

// Any group length g (multiple of 8): one warp per group, lanes stride over
// the group's 16-byte chunks; min / max first, then a second pass quantizes
// (the re-read is an L2 hit for all but the longest rows).
__global__ void __launch_bounds__(256) quantize_warp_group_kernel(
    const uint16_t* __restrict__ W, long long num_groups, int words_per_group,
    uint32_t* __restrict__ packed, uint16_t* __restrict__ scales, uint16_t* __restrict__ zeros, int flags) {
    const int lane = threadIdx.x & 31;
    const long long grp =
        static_cast<long long>(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5);
    if (grp >= num_groups) return;
    const long long base = grp * words_per_group;
    const uint4* src = reinterpret_cast<const uint4*>(W) + base;
    float mn = __int_as_float(0x7f800000), mx = -__int_as_float(0x7f800000);
    for (int c = lane; c < words_per_group; c += 32) {
        float v[8];
        unpack8_bf16(__ldg(src + c), v);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            mn = fminf(mn, v[i]);
            mx = fmaxf(mx, v[i]);
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, off));
        mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
    }
    const GroupParams p = group_params_from_range(mn, mx, flags);
    for (int c = lane; c < words_per_group; c += 32) {
        float v[8];
        unpack8_bf16(__ldg(src + c), v);
        packed[base + c] = pack8(v, p);
    }
    if (lane == 0) {
        scales[grp] = p.sb;
        zeros[grp] = p.zb;
    }
}

// GLOBAL mode, pass 1: grid-stride min / max, one partial pair per block.
__global__ void __launch_bounds__(256) global_minmax_kernel(const uint16_t* __restrict__ W,
                                                            long long total_words,
                                                            float2* __restrict__ partial) {
    __shared__ float smn[8], smx[8];
    float mn = __int_as_float(0x7f800000), mx = -__int_as_float(0x7f800000);
    for (long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
         t < total_words; t += static_cast<long long>(gridDim.x) * blockDim.x) {
        float v[8];
        unpack8_bf16(__ldg(reinterpret_cast<const uint4*>(W) + t), v);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            mn = fminf(mn, v[i]);
            mx = fmaxf(mx, v[i]);
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, off));
        mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) {
        smn[warp] = mn;
        smx[warp] = mx;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < static_cast<int>(blockDim.x >> 5); ++w) {
            mn = fminf(mn, smn[w]);
            mx = fmaxf(mx, smx[w]);
        }
        partial[blockIdx.x] = make_float2(mn, mx);
    }
}

// GLOBAL mode, pass 2: every block folds the partials (min / max are exact
// and order-free, so all blocks agree), derives (s, z), quantizes a
// grid-stride share of W; block 0 stores s and z.
__global__ void __launch_bounds__(256) global_quantize_kernel(
    const uint16_t* __restrict__ W, long long total_words, const float2* __restrict__ partial,
    int num_partial, uint32_t* __restrict__ packed, uint16_t* __restrict__ scales,
    uint16_t* __restrict__ zeros, int flags) {
    __shared__ GroupParams sp;
    if (threadIdx.x < 32) {
        float mn = __int_as_float(0x7f800000), mx = -__int_as_float(0x7f800000);
        for (int i = threadIdx.x; i < num_partial; i += 32) {
            const float2 pm = partial[i];
            mn = fminf(mn, pm.x);
            mx = fmaxf(mx, pm.y);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            mn = fminf(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, off));
            mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
        }
        if (threadIdx.x == 0) sp = group_params_from_range(mn, mx, flags);
    }
    __syncthreads();
    const GroupParams p = sp;
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        scales[0] = p.sb;
        zeros[0] = p.zb;
    }
    for (long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
         t < total_words; t += static_cast<long long>(gridDim.x) * blockDim.x) {
        float v[8];
        unpack8_bf16(__ldg(reinterpret_cast<const uint4*>(W) + t), v);
        packed[t] = pack8(v, p);
    }
}

// Debug-mode input check: sets g_nonfinite when any of the n bf16 values is
// a NaN or an infinity (exponent field all ones).  n is a multiple of 8.
__global__ void __launch_bounds__(256) nonfinite_check_kernel(const uint16_t* __restrict__ W, long long n) {
    const long long n8 = n / 8;
    bool bad = false;
    for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(W) + i);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
            bad = bad || ((w[j] & 0x7F80u) == 0x7F80u) || ((w[j] & 0x7F800000u) == 0x7F800000u);
    }
    if (__any_sync(0xFFFFFFFFu, bad) && (threadIdx.x & 31) == 0) atomicOr(&g_nonfinite, 1u);
}

}  // namespace w4
