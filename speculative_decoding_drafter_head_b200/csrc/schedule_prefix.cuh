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

// How phase 1 reads the scores: through the read-only path when they are an input of
// the launch, or with plain loads (a copy in shared memory, say).
struct LoadReadOnly {
    __device__ __forceinline__ float operator()(const float *p) const { return __ldg(p); }
};
struct LoadPlain {
    __device__ __forceinline__ float operator()(const float *p) const { return *p; }
};

// Number of entries of row `row` ordered before the score (bits pb, flat index ib).
template <typename Load>
__device__ __forceinline__ int count_before(const float *__restrict__ P, int gamma, int row,
                                            uint32_t pb, int ib, Load ld)
{
    const float *pr = P + static_cast<size_t>(row) * gamma;
    int lo = 0, hi = gamma;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        const uint32_t m = score_bits(ld(pr + mid));
        const bool before = (m > pb) || (m == pb && row * gamma + mid < ib);
        if (before)
            lo = mid + 1;
        else
            hi = mid;
    }
    return lo;
}

// Phase 1 for score i, by one warp: its rank (the sum over rows of a binary search),
// written to rank[i]; a score outside [0, 1] or above its predecessor records
// DSPARK_NOT_MONOTONE.
template <typename Load>
__device__ __forceinline__ void rank_score(const float *__restrict__ P, int B, int gamma, int n,
                                           int i, int32_t *rank, Load ld)
{
    const int lane = threadIdx.x & 31;
    const float pi = ld(P + i);
    const uint32_t pb = score_bits(pi);
    int cnt = 0;
    for (int row = lane; row < B; row += 32) cnt += count_before(P, gamma, row, pb, i, ld);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xFFFFFFFFu, cnt, o);
    if (lane == 0) {
        const int k = i % gamma;
        const bool bad = !(pi >= 0.0f && pi <= 1.0f) || (k > 0 && pi > ld(P + i - 1));
        if (bad) record_error(DSPARK_NOT_MONOTONE);
        rank[i] = min(max(cnt, 0), n - 1);
    }
}

// Shared scratch of phase 2 for a group of kW warps.
template <int kW>
struct ScanSmem {
    long long warp_sum[kW];
    double best_F[kW];
    int best_N[kW];
};

// Exclusive scan of one int64 per thread over the group's kW warps (threads t = 0 ..
// 32 kW - 1 of the group, which `sync` synchronises); `total` gets the sum.
template <int kW, typename Sync>
__device__ __forceinline__ long long group_exclusive_scan(long long v, ScanSmem<kW> &sm, int t,
                                                          Sync sync, long long &total)
{
    const int warp = t >> 5, lane = t & 31;
    long long incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const long long u = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += u;
    }
    if (lane == 31) sm.warp_sum[warp] = incl;
    sync();
    if (warp == 0) {
        long long w = (lane < kW) ? sm.warp_sum[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long u = __shfl_up_sync(0xFFFFFFFFu, w, o);
            if (lane >= o) w += u;
        }
        if (lane < kW) sm.warp_sum[lane] = w;   // inclusive warp prefix
    }
    sync();
    total = sm.warp_sum[kW - 1];
    const long long before_warp = (warp == 0) ? 0 : sm.warp_sum[warp - 1];
    sync();                                     // warp_sum is free again when this returns
    return before_warp + incl - v;
}

// Phase 2, by one group of kW warps (thread t of 32 kW) once every rank is written (ranks
// and scores are read through L2: other CTAs wrote them): scatter the fixed-point scores
// q = floor(P 2^46) into rank order, prefix-sum them in int64, evaluate
// F(N) = double(B 2^46 + S_N) / Tstep[B + N] for every N, take the first maximum (largest
// F, then smallest N), and count each request's entries ranked below it.  q_sorted is
// this group's own scratch (global or shared memory); s_rank, when not null, is shared
// memory for a copy of the ranks, so that the counts read shared memory, and s_L, when
// not null, receives the lengths as well.
template <int kW, typename Sync>
__device__ void scan_and_lengths(const float *__restrict__ P, int B, int gamma, int n,
                                 const double *__restrict__ Tstep, const int32_t *rank,
                                 long long *q_sorted, int32_t *L_out, int32_t *N_out,
                                 double *objective_out, ScanSmem<kW> &sm, int t, Sync sync,
                                 int32_t *s_rank = nullptr, int32_t *s_L = nullptr)
{
    constexpr int kT = 32 * kW;
    const int warp = t >> 5, lane = t & 31;
    // the loops below are unrolled so that their independent loads are in flight together
#pragma unroll 8
    for (int i = t; i < n; i += kT) {
        const int pos = __ldcg(rank + i);
        const float pi = __ldcg(P + i);
        q_sorted[pos] = __float2ll_rz(pi * 0x1p46f);
        if (s_rank) s_rank[i] = pos;
    }
    sync();

    const int per = (n + kT - 1) / kT;
    const int lo = min(n, t * per);
    const int hi = min(n, lo + per);
    long long part = 0;
#pragma unroll 8
    for (int i = lo; i < hi; ++i) part += q_sorted[i];
    long long total;
    long long S = group_exclusive_scan<kW>(part, sm, t, sync, total);

    const long long base = static_cast<long long>(B) << 46;
    double best = -1.0;
    int bestN = 0;
    if (t == 0) {
        const double tb = __ldg(Tstep + B);
        if (!(tb > 0.0)) record_error(DSPARK_INVALID_ARG);
        best = __ll2double_rn(base) / tb;
        bestN = 0;
    }
#pragma unroll 8
    for (int i = lo; i < hi; ++i) {
        S += q_sorted[i];
        const int N = i + 1;
        const double tN = __ldg(Tstep + B + N);
        if (!(tN > 0.0)) record_error(DSPARK_INVALID_ARG);
        const double F = __ll2double_rn(base + S) / tN;
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
        sm.best_F[warp] = best;
        sm.best_N[warp] = bestN;
    }
    sync();
    if (t == 0) {
        for (int w = 1; w < kW; ++w) {
            if (sm.best_F[w] > sm.best_F[0] || (sm.best_F[w] == sm.best_F[0] && sm.best_N[w] < sm.best_N[0])) {
                sm.best_F[0] = sm.best_F[w];
                sm.best_N[0] = sm.best_N[w];
            }
        }
        *N_out = sm.best_N[0];
        *objective_out = sm.best_F[0] * 0x1p-46;
    }
    sync();
    const int Nstar = sm.best_N[0];
    // L_b: one warp per request, a ballot over its gamma <= 64 ranks
    for (int b = warp; b < B; b += kW) {
        const int32_t *rb = s_rank ? s_rank + b * gamma : rank + b * gamma;
        int L = 0;
        for (int k0 = 0; k0 < gamma; k0 += 32) {
            const int k = k0 + lane;
            const bool below = k < gamma && (s_rank ? rb[k] : __ldcg(rb + k)) < Nstar;
            L += __popc(__ballot_sync(0xFFFFFFFFu, below));
        }
        if (lane == 0) {
            L_out[b] = L;
            if (s_L) s_L[b] = L;
        }
    }
}

__global__ void __launch_bounds__(kThreads) schedule_prefix_kernel(const Params p)
{
    __shared__ ScanSmem<kWarps> sm;
    __shared__ int s_last;
    const int warp = threadIdx.x >> 5;

    // ---------------- phase 1: ranks
    for (int i = blockIdx.x * kWarps + warp; i < p.n; i += gridDim.x * kWarps)
        rank_score(p.P, p.B, p.gamma, p.n, i, p.rank, LoadReadOnly{});
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        s_last = (atomicAdd(p.done, 1u) == gridDim.x - 1);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    // ---------------- phase 2 (last CTA): scatter, scan, objective, lengths
    scan_and_lengths<kWarps>(p.P, p.B, p.gamma, p.n, p.Tstep, p.rank, p.q_sorted, p.L_out,
                             p.N_out, p.objective_out, sm, static_cast<int>(threadIdx.x),
                             [] { __syncthreads(); });
    if (threadIdx.x == 0) *p.done = 0u;
}

}  // namespace sched
}  // namespace dspark
