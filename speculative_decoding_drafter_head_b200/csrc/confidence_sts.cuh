// confidence_sts.cuh -- confidence head, Sequential Temperature Scaling, prefix survival.
//
// gdymind.com, "DSpark: DeepSeek's new speculative decoding work", section 5: the
// confidence head is a linear projection followed by a sigmoid over the backbone
// hidden state at position k and the Markov embedding of the previous draft token;
// temperatures are calibrated per position ("Sequential Temperature Scaling") and
// the scheduler consumes the cumulative product of the calibrated scores.
//
// A cluster of up to 8 CTAs per request: CTA q of the cluster computes the logits of
// positions q*ppc .. q*ppc + ppc - 1 (ppc = ceil(gamma / 8)), splitting each position's
// dot product over 8 / ppc warps with 16-byte loads of h (the dominant byte stream), of
// the W1 row and of the projection vector; the calibrated scores are stored into the
// shared memory of the cluster's first CTA, and after a cluster barrier one thread of it
// forms the fp32 product along the request in position order.  With B = 64 and
// gamma = 16 that is 512 CTAs instead of 64, so the h stream is read by the whole GPU.
#pragma once
#include <cooperative_groups.h>

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

// Positions per CTA and CTAs per cluster (one cluster per request).
__host__ __device__ constexpr int pos_per_cta(int gamma) { return (gamma + kWarps - 1) / kWarps; }
__host__ __device__ constexpr int cluster_ctas(int gamma)
{
    return (gamma + pos_per_cta(gamma) - 1) / pos_per_cta(gamma);
}

__global__ void __launch_bounds__(kThreads)
    confidence_sts_kernel(const uint16_t *__restrict__ h, const int32_t *__restrict__ anchor,
                          const int32_t *__restrict__ x, const uint16_t *__restrict__ W1,
                          const uint16_t *__restrict__ w, float b_conf,
                          const float *__restrict__ T, int B, int gamma, int d, int r, int V,
                          float *__restrict__ c_out, float *__restrict__ P_out)
{
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    __shared__ float s_c[kMaxGamma];               // used in the cluster's first CTA
    __shared__ float s_part[kWarps];
    const int b = blockIdx.y;
    const int q = static_cast<int>(cluster.block_rank());
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ppc = pos_per_cta(gamma);
    const int wpp = kWarps / ppc;                   // warps per position (>= 1)
    const int j = warp / wpp, part = warp % wpp;    // this warp's position slot and share
    const int k = q * ppc + j;
    const bool active = j < ppc && k < gamma;

    const int dv = d / 8, nvec = (d + r) / 8;
    const int per = (nvec + wpp - 1) / wpp;
    const int i0 = part * per, i1 = min(nvec, i0 + per);
    float acc0 = 0.f, acc1 = 0.f;
    if (active) {
        int prev = (k == 0) ? anchor[b] : x[static_cast<size_t>(b) * gamma + (k - 1)];
        if (prev < 0 || prev >= V) {
            if (lane == 0) record_error(DSPARK_INVALID_TOKEN);
            prev = 0;
        }
        const int4 *hk = reinterpret_cast<const int4 *>(h + (static_cast<size_t>(b) * gamma + k) * d);
        const int4 *ek = reinterpret_cast<const int4 *>(W1 + static_cast<size_t>(prev) * r);
        const int4 *wv = reinterpret_cast<const int4 *>(w);
        int i = i0 + lane;
        for (; i + 32 < i1 && i + 32 < dv; i += 64) {     // two h vectors in flight per lane
            const int4 h0 = __ldcs(hk + i), h1 = __ldcs(hk + i + 32);
            acc0 = dot8_bf16(h0, __ldg(wv + i), acc0);
            acc1 = dot8_bf16(h1, __ldg(wv + i + 32), acc1);
        }
        for (; i < i1; i += 32)
            acc0 = dot8_bf16(i < dv ? __ldcs(hk + i) : __ldg(ek + (i - dv)), __ldg(wv + i), acc0);
    }
    const float zpart = warp_sum(acc0 + acc1);
    if (lane == 0) s_part[warp] = zpart;
    __syncthreads();
    if (active && part == 0 && lane == 0) {
        float z = b_conf;
        for (int pw = 0; pw < wpp; ++pw) z += s_part[warp + pw];
        const float c = 1.0f / (1.0f + expf(-z / T[k]));
        float *dst = cluster.map_shared_rank(s_c, 0);
        dst[k] = c;
    }
    cluster.sync();                                 // every score of the request is in CTA 0
    if (q == 0 && threadIdx.x == 0) {
        float P = 1.0f;
        for (int kk = 0; kk < gamma; ++kk) {
            const float c = s_c[kk];
            P = __fmul_rn(P, c);
            c_out[static_cast<size_t>(b) * gamma + kk] = c;
            P_out[static_cast<size_t>(b) * gamma + kk] = P;
        }
    }
}

}  // namespace conf
}  // namespace dspark
