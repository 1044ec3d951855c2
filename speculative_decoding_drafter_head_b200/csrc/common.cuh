// common.cuh -- status codes, the per-device error word and small helpers.
#pragma once
#include <cstdint>

#include "../../include/dspark.h"

namespace dspark {

// First problem seen on the device since the last dspark_get_error; 0 = none.
__device__ unsigned int g_error_word;

__device__ __forceinline__ void record_error(unsigned int code)
{
    atomicCAS(&g_error_word, 0u, code);
}

// Optional timeline trace of the draft kernel (build with -DDSPARK_TRACE): per CTA and
// per position k, 32 slots of %globaltimer stamps or accumulated wait times in ns.
#ifdef DSPARK_TRACE
__device__ unsigned long long g_trace[256 * 64 * 32];
#define DSPARK_TRACE_AT(k, slot)                                                              \
    do {                                                                                      \
        if ((k) <= 64 && blockIdx.x < 256) {                                                  \
            uint64_t t_;                                                                      \
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                            \
            g_trace[(blockIdx.x * 64 + ((k) - 1)) * 32 + (slot)] = t_;                        \
        }                                                                                     \
    } while (0)
#define DSPARK_TRACE_ADD(k, slot, v)                                                          \
    do {                                                                                      \
        if ((k) <= 64 && blockIdx.x < 256) g_trace[(blockIdx.x * 64 + ((k) - 1)) * 32 + (slot)] += (v); \
    } while (0)
#else
#define DSPARK_TRACE_AT(k, slot) \
    do {                         \
    } while (0)
#define DSPARK_TRACE_ADD(k, slot, v) \
    do {                             \
    } while (0)
#endif

__device__ __forceinline__ float bf16lo_to_f32(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi_to_f32(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Two fp32 additions in one packed instruction (add.rn.f32x2): d0 = a0 + b0, d1 = a1 + b1,
// each rounded to nearest as a plain fp32 addition would be.
__device__ __forceinline__ void add_f32x2(float &d0, float &d1, float a0, float a1, float b0,
                                          float b1)
{
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\t"
        "mov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\t"
        "mov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d0), "=f"(d1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
}

// Monotone map of fp32 onto uint32 (larger float -> larger integer).
__device__ __forceinline__ uint32_t float_order_bits(float f)
{
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// 64-bit argmax key: larger value wins, then the smaller index.
__device__ __forceinline__ unsigned long long argmax_key(float value, uint32_t index)
{
    return (static_cast<unsigned long long>(float_order_bits(value + 0.0f)) << 32) |
           static_cast<unsigned long long>(0xFFFFFFFFu - index);
}

__device__ __forceinline__ uint32_t argmax_key_index(unsigned long long key)
{
    return 0xFFFFFFFFu - static_cast<uint32_t>(key);
}

}  // namespace dspark
