// schedule_prefix.cuh -- the hardware-aware prefix scheduler.
//
// wispaper.ai, "DSpark: Overcoming the Efficiency Wall in LLM Speculative Decoding",
// "The Hardware-Aware Prefix Scheduler", and gdymind.com "DSpark", section 6: verify
// lengths are chosen by a global throughput maximisation against the current
// steps-per-second curve.  Prefix survival falls along every request, so the best
// choice for any total N keeps the N largest scores (a global top-N); a scan over N
// then picks the best total.
//
// One launch.  Phase 1 (all CTAs): the rank of every score in the order
// (P desc, b asc, k asc) -- each request's row is already in that order, so the rank
// of (b, k) is the sum over rows b' of a binary search in row b'.  Phase 2 (the last
// CTA to finish, found with a completion counter, no spinning): scatter the
// fixed-point scores q = floor(P 2^46) into rank order, prefix-sum them in int64,
// evaluate F(N) = double(B 2^46 + S_N) / Tstep[B + N] for every N, take the first
// maximum, and count each request's entries below it.  With B <= 32768 and
// B gamma <= 65536 the numerator stays below (B + B gamma) 2^46 < 2^63.
#pragma once
#include "common.cuh"

namespace dspark {
namespace sched {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;

struct Params {
    const float *P;
    int B, gamma, n;
    const double *Tstep;
    int32_t *L_out;
    int32_t *N_out;
    double *objective_out;
    int32_t *rank;          // [n]
    long long *q_sorted;    // [n]
    unsigned int *done;     // completion counter, zeroed before launch
};

// Bits of a score for ordering.  Valid scores lie in [0, 1], where the fp32 bit
// patterns of non-negative values sort like the values, once -0.0 (sign bit set, equal
// to +0.0 as a number) is mapped onto +0.0 by adding +0.0.
__device__ __forceinline__ uint32_t score_bits(float p) { return __float_as_uint(p + 0.0f); }

// Number of entries of row `row` ordered before the score (bits pb, flat index ib).
__device__ __forceinline__ int count_before(const float *__restrict__ P, int gamma, int row,
                                            uint32_t pb, int ib)
{
    const float *pr = P + static_cast<size_t>(row) * gamma;
    int lo = 0, hi = gamma;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        const uint32_t m = score_bits(__ldg(pr + mid));
        const bool before = (m > pb) || (m == pb && row * gamma + mid < ib);
        if (before)
            lo = mid + 1;
        else
            hi = mid;
    }
    return lo;
}

__device__ __forceinline__ long long block_exclusive_scan(long long v, long long *s_warp,
                                                          long long &total)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    long long incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const long long t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        long long w = (lane < kWarps) ? s_warp[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long t = __shfl_up_sync(0xFFFFFFFFu, w, o);
            if (lane >= o) w += t;
        }
        if (lane < kWarps) s_warp[lane] = w;   // inclusive warp prefix
    }
    __syncthreads();
    total = s_warp[kWarps - 1];
    const long long before_warp = (warp == 0) ? 0 : s_warp[warp - 1];
    return before_warp + incl - v;
}

__global__ void __launch_bounds__(kThreads) schedule_prefix_kernel(const Params p)
{
    __shared__ long long s_warp[kWarps];
    __shared__ double s_bestF[kWarps];
    __shared__ int s_bestN[kWarps];
    __shared__ int s_last;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // ---------------- phase 1: ranks
    for (int i = blockIdx.x * kWarps + warp; i < p.n; i += gridDim.x * kWarps) {
        const float pi = __ldg(p.P + i);
        const uint32_t pb = score_bits(pi);
        int cnt = 0;
        for (int row = lane; row < p.B; row += 32) cnt += count_before(p.P, p.gamma, row, pb, i);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xFFFFFFFFu, cnt, o);
        if (lane == 0) {
            const int k = i % p.gamma;
            const bool bad = !(pi >= 0.0f && pi <= 1.0f) || (k > 0 && pi > __ldg(p.P + i - 1));
            if (bad) record_error(DSPARK_NOT_MONOTONE);
            p.rank[i] = min(max(cnt, 0), p.n - 1);
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        s_last = (atomicAdd(p.done, 1u) == gridDim.x - 1);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    // ---------------- phase 2 (last CTA): scatter, scan, objective, lengths
    for (int i = threadIdx.x; i < p.n; i += kThreads) {
        const int pos = __ldcg(p.rank + i);
        const float pi = __ldg(p.P + i);
        p.q_sorted[pos] = __float2ll_rz(pi * 0x1p46f);
    }
    __syncthreads();

    const int per = (p.n + kThreads - 1) / kThreads;
    const int lo = min(p.n, static_cast<int>(threadIdx.x) * per);
    const int hi = min(p.n, lo + per);
    long long part = 0;
    for (int i = lo; i < hi; ++i) part += __ldcg(p.q_sorted + i);
    long long total;
    long long S = block_exclusive_scan(part, s_warp, total);

    const long long base = static_cast<long long>(p.B) << 46;
    double best = -1.0;
    int bestN = 0;
    if (threadIdx.x == 0) {
        const double t = __ldg(p.Tstep + p.B);
        if (!(t > 0.0)) record_error(DSPARK_INVALID_ARG);
        best = __ll2double_rn(base) / t;
        bestN = 0;
    }
    for (int i = lo; i < hi; ++i) {
        S += __ldcg(p.q_sorted + i);
        const int N = i + 1;
        const double t = __ldg(p.Tstep + p.B + N);
        if (!(t > 0.0)) record_error(DSPARK_INVALID_ARG);
        const double F = __ll2double_rn(base + S) / t;
        if (F > best) {
            best = F;
            bestN = N;
        }
    }
    // first maximum: larger F, then smaller N
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const double oF = __shfl_xor_sync(0xFFFFFFFFu, best, o);
        const int oN = __shfl_xor_sync(0xFFFFFFFFu, bestN, o);
        if (oF > best || (oF == best && oN < bestN)) {
            best = oF;
            bestN = oN;
        }
    }
    if (lane == 0) {
        s_bestF[warp] = best;
        s_bestN[warp] = bestN;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < kWarps; ++w) {
            if (s_bestF[w] > s_bestF[0] || (s_bestF[w] == s_bestF[0] && s_bestN[w] < s_bestN[0])) {
                s_bestF[0] = s_bestF[w];
                s_bestN[0] = s_bestN[w];
            }
        }
        *p.N_out = s_bestN[0];
        *p.objective_out = s_bestF[0] * 0x1p-46;
        *p.done = 0u;
    }
    __syncthreads();
    const int Nstar = s_bestN[0];
    for (int b = threadIdx.x; b < p.B; b += kThreads) {
        int L = 0;
        for (int k = 0; k < p.gamma; ++k)
            L += (__ldcg(p.rank + b * p.gamma + k) < Nstar) ? 1 : 0;
        p.L_out[b] = L;
    }
}

}  // namespace sched
}  // namespace dspark
