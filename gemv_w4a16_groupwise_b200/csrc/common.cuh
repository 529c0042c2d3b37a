// Shared device helpers of the W4A16 library (sm_100a only).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "this library targets sm_100a (B200) only"
#endif

namespace w4 {

// Device-side error word: kernels whose waits are bounded record why they
// gave up here instead of hanging (read and cleared by w4_device_error).
__device__ unsigned int g_error_word;

enum DeviceError : unsigned int {
    kErrNone = 0,
    kErrTimeoutTmaFull = 1,     // a consumer waited too long for a TMA stage
    kErrTimeoutDequant = 2,     // the MMA issuer waited too long for dequantized tiles
    kErrTimeoutEmpty = 3,       // the producer waited too long for a free stage
    kErrTimeoutAccum = 4,       // the epilogue waited too long for the accumulator
    kErrBadIndex = 5,           // a column index of a gather / scatter was out of range
};

// Debug controls, set from the host (w4_debug_set_wait_limit,
// w4_debug_withhold_stage): how long a bounded wait may last, and a stage
// index whose copy the GEMV producers leave unissued (-1: none), so that a
// test can make a wait run out without any fault.
__device__ unsigned long long g_wait_limit_ns = 2000000000ull;
__device__ int g_withhold_stage = -1;
// Set by the debug-mode input check when it meets a NaN or an infinity.
__device__ unsigned int g_nonfinite;

__device__ __forceinline__ void record_error(unsigned int code) {
    atomicCAS(&g_error_word, 0u, code);
}

// Programmatic dependent launch: a kernel lets its dependents start early;
// a dependent waits for the kernels before it where it needs their results.
// Both are no-ops in a kernel launched without the programmatic attribute.
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// Format flags of the scale / zero metadata, or-ed into the mode (the same
// values as W4_ZERO_FLOAT and W4_META_BF16 of the public header).
constexpr int kFmtZeroFloat = 0x10;   // fractional zero point
constexpr int kFmtMetaBf16 = 0x20;    // scales and zeros stored as bf16

// Value of a scale or zero stored as fp16 bits, or bf16 bits.
__device__ __forceinline__ float meta_to_float(uint16_t b, bool bf16) {
    return bf16 ? bf16_bits_to_float(b) : __half2float(__ushort_as_half(b));
}
__device__ __forceinline__ float meta_to_float(__half h, bool bf16) {
    return meta_to_float(__half_as_ushort(h), bf16);
}

__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a, uint32_t mask, uint32_t orv) {
    // (a & mask) | orv in one instruction
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(a), "r"(mask), "r"(orv));
    return r;
}

// Byte permute: result byte i = byte sel_i of {b:a} (PTX prmt default mode).
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

__device__ __forceinline__ uint32_t ldg_stream_u32(const void* p) {
    uint32_t v;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t bf162_bits(__nv_bfloat162 v) {
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    return __ffma2_rn(a, b, c);
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) { return __fmul2_rn(a, b); }

}  // namespace w4
