// verify_prefix.cuh -- strict prefix-match verification.
//
// seventnews.com, "DeepSeek's DSpark just fixed the two things that held back faster
// AI inference": the target verifies the whole proposal in one pass, accepted tokens
// stick, and the first rejected token and everything after it are dropped.  The
// target's token at the first rejected position (or after the last accepted draft)
// is emitted as the bonus token.
//
// One thread per request; the compare loop reads at most gamma + 1 ids per request.
#pragma once
#include "common.cuh"

namespace dspark {
namespace verify {

constexpr int kThreads = 128;

// Request b with verify length len: the first position among its first len drafts where
// the draft and the target differ (len if none) and the target's token there.  Drafts are
// read through L2: in the draft kernel's tail they were written earlier in the launch.
__device__ __forceinline__ void verify_request_len(const int32_t *x, int len,
                                                   const int32_t *__restrict__ target, int b,
                                                   int gamma, int32_t *accepted_out,
                                                   int32_t *bonus_out)
{
    if (len < 0 || len > gamma) {
        record_error(DSPARK_INVALID_TOKEN);
        len = min(max(len, 0), gamma);
    }
    const int32_t *xb = x + static_cast<size_t>(b) * gamma;
    const int32_t *tb = target + static_cast<size_t>(b) * (gamma + 1);
    // sixteen positions per round, all their loads in flight together
    int a = len;
    for (int k0 = 0; k0 < len && a == len; k0 += 16) {
        int xs[16], ts[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const bool in = k0 + j < len;
            xs[j] = in ? __ldcg(xb + k0 + j) : 0;
            ts[j] = in ? tb[k0 + j] : 0;
        }
#pragma unroll
        for (int j = 15; j >= 0; --j)
            if (k0 + j < len && xs[j] != ts[j]) a = k0 + j;
    }
    accepted_out[b] = a;
    bonus_out[b] = tb[a];
}

// The same with the length read from L[b].
__device__ __forceinline__ void verify_request(const int32_t *x, const int32_t *L,
                                               const int32_t *__restrict__ target, int b,
                                               int gamma, int32_t *accepted_out,
                                               int32_t *bonus_out)
{
    verify_request_len(x, __ldcg(L + b), target, b, gamma, accepted_out, bonus_out);
}

__global__ void __launch_bounds__(kThreads)
    verify_prefix_kernel(const int32_t *__restrict__ x, const int32_t *__restrict__ L,
                         const int32_t *__restrict__ target, int B, int gamma,
                         int32_t *__restrict__ accepted_out, int32_t *__restrict__ bonus_out)
{
    const int b = blockIdx.x * kThreads + threadIdx.x;
    if (b >= B) return;
    verify_request(x, L, target, b, gamma, accepted_out, bonus_out);
}

}  // namespace verify
}  // namespace dspark
