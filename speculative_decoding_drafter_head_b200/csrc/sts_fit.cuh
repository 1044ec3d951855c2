// sts_fit.cuh -- Sequential Temperature Scaling, fitting the per-position temperatures.
//
// gdymind.com, "DSpark: DeepSeek's new speculative decoding work", section 5,
// "Sequential Temperature Scaling": the survival product is calibrated from left to
// right; at each position k a one-dimensional grid search picks the temperature whose
// cumulative product has the smallest expected calibration error (ECE), with the
// temperatures of positions 1..k-1 already fixed.
//
// On a held-out set of N draft blocks with raw confidence logits z [N, gamma] and
// accepted lengths a [N], the label at position k is y = (a >= k), and for candidate
// T_i = t_min + i * t_step
//     p_i[n] = P_{k-1}[n] / (1 + exp(-z[n, k-1] / T_i)),   P_0 = 1
//     ECE_i  = sum over equal-width bins m of |sum_{n in m} y - sum_{n in m} p_i| / N,
// bin(p) = min(floor(p * n_bins), n_bins - 1).  The smallest i with the smallest
// ECE_i wins, and P_k = P_{k-1} / (1 + exp(-z[., k-1] / T_k)).
//
// Work per position is N * n_t sigmoids in fp64 (exp is the cost); it is ALU-bound,
// the data (z, a, P: 17 bytes per block) is read once per position.
//
// Layout of the work: one thread per candidate temperature (up to 512 per CTA), each
// with a private histogram column in shared memory (count and fp64 sum of p per bin),
// so the inner loop needs no atomics; blocks of 256 samples are staged in shared memory
// and read by every thread as broadcasts.  At the end each CTA rounds its column sums
// to 2^-40 fixed point and adds them into global per-(position, candidate, bin) totals
// with integer atomics: integer addition is associative, so the totals, the ECE
// numerators and the chosen index do not depend on the order in which CTAs finish.
//
// Per candidate the thread computes e = exp(-z / T) as exp(-z * (1/T)) with 1/T
// formed once, and 1 / (1 + e) by two Newton-Raphson steps r <- r (2 - d r) from the
// hardware's approximate fp64 reciprocal: each differs from the correctly rounded
// quotient by a few ulp, far below the resolution at which two ECEs are compared.
#pragma once
#include "common.cuh"

namespace dspark {
namespace stsfit {

constexpr int kStage = 256;                    // samples staged per round
constexpr int kMaxThreads = 512;               // candidates per CTA
constexpr int kMaxBins = 256;
constexpr int kMaxN = (1 << 23) - 1;           // keeps N * 2^40 below 2^63
constexpr double kFix = 1099511627776.0;       // 2^40
constexpr int kPickThreads = 1024;

struct Params {
    const float *z;             // [N, gamma]
    const int32_t *acc;         // [N]
    int N, gamma, k;            // k: 1-based position being fitted
    double t_min, t_step;
    int n_t, n_bins;
    double *P;                  // [2][N]: P_{j} lives in buffer (j & 1)
    int32_t *idx;               // [gamma] chosen grid indices (output, read by later positions)
    float *T_out;               // [gamma]
    double *ece_out;            // [gamma]
    unsigned int *cnt;          // [gamma][n_t][n_bins] label counts
    unsigned long long *sq;     // [gamma][n_t][n_bins] fixed-point sums of p
};

inline size_t hist_smem_bytes(int tpb, int n_bins)
{
    return static_cast<size_t>(n_bins) * tpb * 12 + kStage * (8 + 8 + 4);
}

// 1 / d for d >= 1: approximate reciprocal, refined by two Newton-Raphson steps.
__device__ __forceinline__ double recip_ge1(double d)
{
    double r;
    asm("rcp.approx.ftz.f64 %0, %1;" : "=d"(r) : "d"(d));
    if (!(d < 1.0e300)) return 0.0;          // exp overflowed: the sigmoid is 0 to fp64
    double t = fma(-d, r, 1.0);
    r = fma(r, t, r);
    t = fma(-d, r, 1.0);
    return fma(r, t, r);
}

__global__ void __launch_bounds__(kMaxThreads) sts_hist_kernel(Params p)
{
    extern __shared__ __align__(16) unsigned char smem[];
    const int tpb = blockDim.x;
    const int tid = threadIdx.x;
    const int nb = p.n_bins;
    double *hsp = reinterpret_cast<double *>(smem);                            // [nb][tpb]
    unsigned int *hcnt = reinterpret_cast<unsigned int *>(hsp + nb * tpb);     // [nb][tpb]
    double *sP = reinterpret_cast<double *>(hcnt + nb * tpb);                  // [kStage]
    double *snz = sP + kStage;                                                 // [kStage] -z
    unsigned int *sy = reinterpret_cast<unsigned int *>(snz + kStage);         // [kStage]

    for (int m = 0; m < nb; ++m) {
        hsp[m * tpb + tid] = 0.0;
        hcnt[m * tpb + tid] = 0u;
    }
    const int k = p.k;
    const int i = blockIdx.y * tpb + tid;
    const bool active = i < p.n_t;
    const double invT = 1.0 / (p.t_min + i * p.t_step);
    const double Tprev = k >= 2 ? p.t_min + p.idx[k - 2] * p.t_step : 1.0;
    const double nbd = static_cast<double>(nb);

    // an even share of the samples per CTA (every CTA slot on the GPU gets one share)
    const int n_begin = static_cast<int>(static_cast<long long>(p.N) * blockIdx.x / gridDim.x);
    const int n_end = static_cast<int>(static_cast<long long>(p.N) * (blockIdx.x + 1) / gridDim.x);
    for (int base = n_begin; base < n_end; base += kStage) {
        const int cnt = min(kStage, n_end - base);
        __syncthreads();
        for (int j = tid; j < cnt; j += tpb) {
            const int n = base + j;
            const float *zn = p.z + static_cast<size_t>(n) * p.gamma;
            double Pp = 1.0;
            if (k >= 2) {
                // P_{k-1} from P_{k-2} and the frozen temperature of position k-1
                const double Pb = k >= 3 ? p.P[static_cast<size_t>(k & 1) * p.N + n] : 1.0;
                Pp = Pb / (1.0 + exp(-static_cast<double>(zn[k - 2]) / Tprev));
                if (blockIdx.y == 0) p.P[static_cast<size_t>((k - 1) & 1) * p.N + n] = Pp;
            }
            sP[j] = Pp;
            snz[j] = -static_cast<double>(zn[k - 1]);
            sy[j] = p.acc[n] >= k ? 1u : 0u;
        }
        __syncthreads();
        if (active) {
            for (int j = 0; j < cnt; ++j) {
                const double pj = sP[j] * recip_ge1(1.0 + exp(snz[j] * invT));
                int m = static_cast<int>(pj * nbd);
                m = max(0, min(m, nb - 1));       // also keeps a NaN logit in range
                hsp[m * tpb + tid] += pj;
                hcnt[m * tpb + tid] += sy[j];
            }
        }
    }
    if (!active) return;
    const size_t row = (static_cast<size_t>(k - 1) * p.n_t + i) * nb;
    for (int m = 0; m < nb; ++m) {
        const unsigned long long s =
            static_cast<unsigned long long>(__double2ll_rn(hsp[m * tpb + tid] * kFix));
        const unsigned int c = hcnt[m * tpb + tid];
        if (s) atomicAdd(p.sq + row + m, s);
        if (c) atomicAdd(p.cnt + row + m, c);
    }
}

// One CTA: the ECE numerator of every candidate as an exact integer
// (sum_m |count_m 2^40 - fixed-point sum_m|), then the smallest index of the minimum.
__global__ void __launch_bounds__(kPickThreads) sts_pick_kernel(Params p)
{
    __shared__ unsigned long long s_num[kPickThreads / 32];
    __shared__ int s_idx[kPickThreads / 32];
    const int k = p.k;
    unsigned long long best = ~0ull;
    int best_i = 0x7FFFFFFF;
    for (int i = threadIdx.x; i < p.n_t; i += kPickThreads) {
        const size_t row = (static_cast<size_t>(k - 1) * p.n_t + i) * p.n_bins;
        unsigned long long num = 0;
        for (int m = 0; m < p.n_bins; ++m) {
            const unsigned long long y = static_cast<unsigned long long>(p.cnt[row + m]) << 40;
            const unsigned long long s = p.sq[row + m];
            num += y > s ? y - s : s - y;
        }
        if (num < best) {     // i increases within a thread: strict < keeps the smallest
            best = num;
            best_i = i;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const unsigned long long on = __shfl_xor_sync(0xFFFFFFFFu, best, o);
        const int oi = __shfl_xor_sync(0xFFFFFFFFu, best_i, o);
        if (on < best || (on == best && oi < best_i)) {
            best = on;
            best_i = oi;
        }
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) {
        s_num[warp] = best;
        s_idx[warp] = best_i;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < kPickThreads / 32; ++w)
            if (s_num[w] < best || (s_num[w] == best && s_idx[w] < best_i)) {
                best = s_num[w];
                best_i = s_idx[w];
            }
        p.idx[k - 1] = best_i;
        p.T_out[k - 1] = static_cast<float>(p.t_min + best_i * p.t_step);
        p.ece_out[k - 1] = static_cast<double>(best) / kFix / static_cast<double>(p.N);
    }
}

}  // namespace stsfit
}  // namespace dspark
