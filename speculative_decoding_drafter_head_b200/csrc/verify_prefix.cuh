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

__global__ void __launch_bounds__(kThreads)
    verify_prefix_kernel(const int32_t *__restrict__ x, const int32_t *__restrict__ L,
                         const int32_t *__restrict__ target, int B, int gamma,
                         int32_t *__restrict__ accepted_out, int32_t *__restrict__ bonus_out)
{
    const int b = blockIdx.x * kThreads + threadIdx.x;
    if (b >= B) return;
    int len = L[b];
    if (len < 0 || len > gamma) {
        record_error(DSPARK_INVALID_TOKEN);
        len = min(max(len, 0), gamma);
    }
    const int32_t *xb = x + static_cast<size_t>(b) * gamma;
    const int32_t *tb = target + static_cast<size_t>(b) * (gamma + 1);
    int a = len;
    for (int k = 0; k < len; ++k) {
        if (xb[k] != tb[k]) {
            a = k;
            break;
        }
    }
    accepted_out[b] = a;
    bonus_out[b] = tb[a];
}

}  // namespace verify
}  // namespace dspark
