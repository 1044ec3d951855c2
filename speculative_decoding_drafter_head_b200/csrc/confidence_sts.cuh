// confidence_sts.cuh -- confidence head, Sequential Temperature Scaling, prefix survival.
//
// gdymind.com, "DSpark: DeepSeek's new speculative decoding work", section 5: the
// confidence head is a linear projection followed by a sigmoid over the backbone
// hidden state at position k and the Markov embedding of the previous draft token;
// temperatures are calibrated per position ("Sequential Temperature Scaling") and
// the scheduler consumes the cumulative product of the calibrated scores.
//
// One CTA per request.  Warp w computes the logits of positions k = w, w + 8, ...
// with 16-byte loads of h (the dominant byte stream) and of the W1 row, against the
// projection vector staged once in shared memory; one thread then forms the fp32
// product along the request in position order.
#pragma once
#include "common.cuh"

namespace dspark {
namespace conf {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxGamma = 64;

__device__ __forceinline__ float dot8_bf16(const int4 a, const int4 b, float acc)
{
    const uint32_t aw[4] = {static_cast<uint32_t>(a.x), static_cast<uint32_t>(a.y),
                            static_cast<uint32_t>(a.z), static_cast<uint32_t>(a.w)};
    const uint32_t bw[4] = {static_cast<uint32_t>(b.x), static_cast<uint32_t>(b.y),
                            static_cast<uint32_t>(b.z), static_cast<uint32_t>(b.w)};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        acc = fmaf(bf16lo_to_f32(aw[q]), bf16lo_to_f32(bw[q]), acc);
        acc = fmaf(bf16hi_to_f32(aw[q]), bf16hi_to_f32(bw[q]), acc);
    }
    return acc;
}

__global__ void __launch_bounds__(kThreads)
    confidence_sts_kernel(const uint16_t *__restrict__ h, const int32_t *__restrict__ anchor,
                          const int32_t *__restrict__ x, const uint16_t *__restrict__ W1,
                          const uint16_t *__restrict__ w, float b_conf,
                          const float *__restrict__ T, int B, int gamma, int d, int r, int V,
                          float *__restrict__ c_out, float *__restrict__ P_out)
{
    extern __shared__ int4 s_w[];   // projection vector w, (d + r) bf16
    __shared__ float s_c[kMaxGamma];
    const int b = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nvec = (d + r) / 8;
    for (int i = threadIdx.x; i < nvec; i += kThreads)
        s_w[i] = __ldg(reinterpret_cast<const int4 *>(w) + i);
    __syncthreads();

    const int dv = d / 8, rv = r / 8;
    for (int k = warp; k < gamma; k += kWarps) {
        int prev = (k == 0) ? anchor[b] : x[static_cast<size_t>(b) * gamma + (k - 1)];
        if (prev < 0 || prev >= V) {
            if (lane == 0) record_error(DSPARK_INVALID_TOKEN);
            prev = 0;
        }
        const int4 *hk = reinterpret_cast<const int4 *>(h + (static_cast<size_t>(b) * gamma + k) * d);
        const int4 *ek = reinterpret_cast<const int4 *>(W1 + static_cast<size_t>(prev) * r);
        float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
        int i = lane;
        for (; i + 96 < dv; i += 128) {
            const int4 h0 = __ldcs(hk + i), h1 = __ldcs(hk + i + 32);
            const int4 h2 = __ldcs(hk + i + 64), h3 = __ldcs(hk + i + 96);
            acc0 = dot8_bf16(h0, s_w[i], acc0);
            acc1 = dot8_bf16(h1, s_w[i + 32], acc1);
            acc2 = dot8_bf16(h2, s_w[i + 64], acc2);
            acc3 = dot8_bf16(h3, s_w[i + 96], acc3);
        }
        for (; i < dv; i += 32) acc0 = dot8_bf16(__ldcs(hk + i), s_w[i], acc0);
        for (int j = lane; j < rv; j += 32) acc1 = dot8_bf16(__ldg(ek + j), s_w[dv + j], acc1);
        const float z = warp_sum((acc0 + acc1) + (acc2 + acc3)) + b_conf;
        if (lane == 0) s_c[k] = 1.0f / (1.0f + expf(-z / T[k]));
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        float P = 1.0f;
        for (int k = 0; k < gamma; ++k) {
            const float c = s_c[k];
            P = __fmul_rn(P, c);
            c_out[static_cast<size_t>(b) * gamma + k] = c;
            P_out[static_cast<size_t>(b) * gamma + k] = P;
        }
    }
}

}  // namespace conf
}  // namespace dspark
