// markov_draft.cuh -- the sequential Markov head of DSpark on tcgen05 tensor cores.
//
// gdymind.com, "DSpark: DeepSeek's new speculative decoding work", section 4
// ("Sequential stage", "Markov head"): position k adds a first-order transition
// bias B(x_{k-1}, .) = W1[x_{k-1}] W2 (rank r = 256) to the backbone's base logits
// U_k and picks x_k from them.
//
// One persistent cooperative kernel runs all gamma positions.  Each CTA owns a
// contiguous slice of the vocabulary, cut into tiles of 32 columns, and for every
// position k and every block of 128 requests it computes
//     D[b, v] = sum_j A[b, j] W2[j, v],   A[b, :] = W1[x_{k-1, b}, :]
// as M=128, N=32, K=256 tcgen05.mma (bf16 in, fp32 accumulate in TMEM).  The
// epilogue adds U_k, applies greedy or Gumbel-max selection and keeps a running
// (max, index) per request row, so the [B, V] logits never reach memory.  Rows are
// combined across CTAs by a 64-bit atomicMax on (ordered value, inverted index);
// a bounded grid barrier ends each position, after which every CTA reads x_k for
// the next gather and the CTA that owns the winning column writes the outputs.
//
// Warp roles (192 threads): warps 0-3 epilogue (TMEM lanes 0-127) and A gather,
// warp 4 TMA producer (W2 tile + U tile per stage), warp 5 MMA issuer + TMEM owner.
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "ptx.cuh"

namespace dspark {
namespace draft {

constexpr int kTileN = 32;                       // vocabulary columns per tile
constexpr int kRank = 256;                       // r, the contraction length
constexpr int kMTile = 128;                      // requests per M tile
constexpr int kStages = 6;                       // W2/U smem ring depth
constexpr int kAcc = 4;                          // TMEM accumulator buffers
constexpr int kABytes = kMTile * kRank * 2;      // 64 KB gathered W1 rows
constexpr int kAChunk = kMTile * 128;            // one 64-column (128 B) K chunk
constexpr int kW2Bytes = kTileN * kRank * 2;     // 16 KB per W2 tile
constexpr int kUBytes = kMTile * kTileN * 2;     // 8 KB per U tile (max rows)
constexpr int kStageBytes = kW2Bytes + kUBytes;  // 24 KB
constexpr int kDynSmem = kABytes + kStages * kStageBytes + 1024;  // + alignment slack
constexpr int kThreads = 192;
constexpr int kEpiThreads = 128;
constexpr uint32_t kTmemCols = kAcc * kTileN;    // 128 columns
constexpr int kMaxB = 1024;
constexpr float kGumbelMax = 17.0f;              // above any noise value the epilogue makes

struct Params {
    const int32_t *anchor;
    const uint16_t *W1;
    int B, gamma, V, mode;
    float inv_tau;
    uint32_t seed_lo, seed_hi;
    int b_offset;
    int32_t *x_out;
    float *logit_out;
    unsigned long long *slots;   // [gamma][B] argmax keys, zeroed before launch
    unsigned int *barrier;       // grid barrier arrival counter, zeroed before launch
    unsigned int *abort_flag;    // set by any CTA that gives up, zeroed before launch
    int ntiles_total;            // ceil(V / 32)
    int ub;                      // rows of the U TMA box: min(B, 128)
    unsigned long long timeout_ns;
    int barrier_extra;
};

struct Ctl {
    unsigned long long full[kStages];
    unsigned long long empty[kStages];
    unsigned long long tfull[kAcc];
    unsigned long long tempty[kAcc];
    unsigned long long afull, aempty, drain;
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ void give_up(Ctl &ctl, const Params &p, unsigned code)
{
    record_error(code);
    *reinterpret_cast<volatile int *>(&ctl.abort) = 1;
    atomicExch(p.abort_flag, 1u);
}

// Wait for an mbarrier phase; false once the CTA gives up or the wait runs out.
__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity, Ctl &ctl,
                                           const Params &p)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t n = 1;; ++n) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((n & 63u) == 0) {
            if (*reinterpret_cast<volatile int *>(&ctl.abort)) return false;
            if (globaltimer_ns() - t0 > p.timeout_ns) {
                give_up(ctl, p, DSPARK_TIMEOUT);
                return false;
            }
        }
    }
}

// Bounded wait used while draining: ignores the abort flag, only the time limit.
__device__ __forceinline__ void wait_drain(uint32_t bar, uint32_t parity, const Params &p)
{
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > p.timeout_ns) {
            record_error(DSPARK_TIMEOUT);
            return;
        }
    }
}

__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ unsigned int ld_acquire_u32(const unsigned int *ptr)
{
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ptr) : "memory");
    return v;
}

// Philox4x32-10 (Salmon et al., SC'11): 10 rounds of the 4-word S-box with round
// multipliers 0xD2511F53, 0xCD9E8D57 and key increments 0x9E3779B9, 0xBB67AE85.
__device__ __forceinline__ uint4 philox(uint4 c, uint32_t k0, uint32_t k1)
{
#pragma unroll
    for (int round = 0; round < 10; ++round) {
        const uint32_t hi0 = __umulhi(0xD2511F53u, c.x), lo0 = 0xD2511F53u * c.x;
        const uint32_t hi1 = __umulhi(0xCD9E8D57u, c.z), lo1 = 0xCD9E8D57u * c.z;
        c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
    return c;
}

// g = -ln(-ln u), u = ((w >> 9) + 0.5) 2^-23.  E = -ln u is taken from the hardware
// log2 when u <= 1 - 2^-6 and, closer to 1, from the Mercator series
// -ln(1 - t) = t + t^2/2 + t^3/3 + ... in t = 1 - u (exact), where the hardware
// log loses relative accuracy.  Truncating after t^5/5 leaves < 1e-10 relative error.
__device__ __forceinline__ float gumbel_from_word(uint32_t w)
{
    const uint32_t m = w >> 9;
    const float u = (static_cast<float>(m) + 0.5f) * 0x1p-23f;
    const float t = (static_cast<float>(0x7FFFFFu - m) + 0.5f) * 0x1p-23f;
    const float e_series = t * (1.0f + t * (0.5f + t * (1.0f / 3.0f + t * (0.25f + t * 0.2f))));
    const float e_log = -__logf(u);
    const float e = (t < 0.015625f) ? e_series : e_log;
    return -__logf(e);
}

__device__ __forceinline__ void lds128(uint32_t addr, uint32_t &a, uint32_t &b, uint32_t &c,
                                       uint32_t &d)
{
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(a), "=r"(b), "=r"(c), "=r"(d)
                 : "r"(addr));
}

__device__ __forceinline__ void sts128(uint32_t addr, int4 v)
{
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

// Token x_{k-1} of request b (k is 1-based): the anchor at k = 1, else the winner of
// position k-1 read from the combined argmax keys.  Out-of-range ids are recorded and
// replaced by 0 so that no gather leaves W1.
__device__ __forceinline__ int prev_token(const Params &p, int b, int k)
{
    int tok;
    if (k == 1) {
        tok = p.anchor[b];
    } else {
        const unsigned long long key = __ldcg(&p.slots[static_cast<size_t>(k - 2) * p.B + b]);
        tok = static_cast<int>(argmax_key_index(key));
    }
    if (tok < 0 || tok >= p.V) {
        record_error(DSPARK_INVALID_TOKEN);
        tok = 0;
    }
    return tok;
}

__global__ void __launch_bounds__(kThreads, 1)
    markov_draft_kernel(const __grid_constant__ CUtensorMap tm_w2,
                        const __grid_constant__ CUtensorMap tm_u, const Params p)
{
    extern __shared__ uint8_t dyn_smem[];
    __shared__ Ctl ctl;
    __shared__ unsigned long long row_key[kMaxB];
    __shared__ float row_logit[kMaxB];

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t base = (smem_u32(dyn_smem) + 1023u) & ~1023u;
    const uint32_t sA = base;
    const uint32_t sStage = base + kABytes;

    const int G = gridDim.x;
    const int t_begin = static_cast<int>(static_cast<long long>(blockIdx.x) * p.ntiles_total / G);
    const int t_end =
        static_cast<int>(static_cast<long long>(blockIdx.x + 1) * p.ntiles_total / G);
    const int ntiles = t_end - t_begin;
    const int num_mt = (p.B + kMTile - 1) / kMTile;

    const uint32_t bar_full = smem_u32(&ctl.full[0]);
    const uint32_t bar_empty = smem_u32(&ctl.empty[0]);
    const uint32_t bar_tfull = smem_u32(&ctl.tfull[0]);
    const uint32_t bar_tempty = smem_u32(&ctl.tempty[0]);
    const uint32_t bar_afull = smem_u32(&ctl.afull);
    const uint32_t bar_aempty = smem_u32(&ctl.aempty);
    const uint32_t bar_drain = smem_u32(&ctl.drain);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 1 + 4);
        }
        for (int a = 0; a < kAcc; ++a) {
            mbar_init(bar_tfull + 8 * a, 1);
            mbar_init(bar_tempty + 8 * a, 4);
        }
        mbar_init(bar_afull, 4);
        mbar_init(bar_aempty, 1);
        mbar_init(bar_drain, 1);
        ctl.abort = 0;
        mbar_fence_init();
    }
    if (warp == 5) {
        tmem_alloc(smem_u32(&ctl.tmem_base), kTmemCols);
        tmem_relinquish();
    }
    if (warp == 4 && lane == 0) {
        tma_prefetch_desc(&tm_w2);
        tma_prefetch_desc(&tm_u);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl.tmem_base;

    if (warp == 4) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint64_t pol_w2 = l2_policy_evict_last();
            const uint64_t pol_u = l2_policy_evict_first();
            const uint32_t tx = kW2Bytes + static_cast<uint32_t>(p.ub) * kTileN * 2;
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            bool ok = true;
            for (int k = 1; k <= p.gamma && ok; ++k) {
                for (int mt = 0; mt < num_mt && ok; ++mt) {
                    for (int j = 0; j < ntiles; ++j) {
                        if (!wait_phase(bar_empty + 8 * stage, phase ^ 1u, ctl, p)) {
                            ok = false;
                            break;
                        }
                        const int v0 = (t_begin + j) * kTileN;
                        const uint32_t sW = sStage + stage * kStageBytes;
                        const uint32_t sU = sW + kW2Bytes;
                        mbar_arrive_expect_tx(bar_full + 8 * stage, tx);
                        tma_load_2d(sW, &tm_w2, bar_full + 8 * stage, v0, 0, pol_w2);
                        tma_load_3d(sU, &tm_u, bar_full + 8 * stage, v0, k - 1, mt * kMTile, pol_u);
                        ++issued;
                        if (++stage == kStages) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                }
            }
            // every issued copy must land before the CTA may exit
            for (int s = 0; s < kStages; ++s) {
                const long long uses = issued / kStages + (s < issued % kStages ? 1 : 0);
                if (uses > 0) wait_drain(bar_full + 8 * s, static_cast<uint32_t>((uses - 1) & 1), p);
            }
        }
    } else if (warp == 5) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(kMTile, kTileN, 1);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t aphase = 0;
            uint32_t mt_count = 0;
            bool issued_any = false;
            bool ok = true;
            for (int k = 1; k <= p.gamma && ok; ++k) {
                for (int mt = 0; mt < num_mt && ok; ++mt) {
                    if (!wait_phase(bar_afull, mt_count & 1u, ctl, p)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    for (int j = 0; j < ntiles; ++j) {
                        if (!wait_phase(bar_full + 8 * stage, phase, ctl, p) ||
                            !wait_phase(bar_tempty + 8 * acc, aphase ^ 1u, ctl, p)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t d_tmem = tmem + static_cast<uint32_t>(acc * kTileN);
                        const uint32_t sW = sStage + stage * kStageBytes;
#pragma unroll
                        for (int kk = 0; kk < kRank / 16; ++kk) {
                            const uint64_t a_desc = smem_desc(
                                sA + (kk >> 2) * kAChunk + (kk & 3) * 32, 1024, 1024, kSwizzle128B);
                            const uint64_t b_desc = smem_desc(sW + kk * 1024, 512, 512, kSwizzle64B);
                            umma_bf16(d_tmem, a_desc, b_desc, idesc, kk > 0 ? 1u : 0u);
                        }
                        issued_any = true;
                        umma_commit(bar_tfull + 8 * acc);
                        umma_commit(bar_empty + 8 * stage);
                        if (++stage == kStages) {
                            stage = 0;
                            phase ^= 1u;
                        }
                        if (++acc == kAcc) {
                            acc = 0;
                            aphase ^= 1u;
                        }
                    }
                    if (!ok) break;
                    umma_commit(bar_aempty);
                    ++mt_count;
                }
            }
            if (issued_any) {
                umma_commit(bar_drain);
                wait_drain(bar_drain, 0, p);
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue (warps 0-3)
        const int row = warp * 32 + lane;
        const uint32_t t_lane = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        int stage = 0;
        uint32_t phase = 0;
        int acc = 0;
        uint32_t aphase = 0;
        uint32_t mt_count = 0;
        bool ok = true;

        for (int k = 1; k <= p.gamma && ok; ++k) {
            for (int mt = 0; mt < num_mt && ok; ++mt) {
                const int m0 = mt * kMTile;
                // ---- gather A = W1[x_{k-1}] for this block of requests (K-major, 128B swizzle)
                if (!__all_sync(0xFFFFFFFFu, wait_phase(bar_aempty, (mt_count & 1u) ^ 1u, ctl, p))) {
                    ok = false;
                    break;
                }
                const int my_b = m0 + row;
                const int my_tok = (my_b < p.B) ? prev_token(p, my_b, k) : -1;
                const int chunk = lane >> 3, unit = lane & 7;
#pragma unroll 1
                for (int i0 = 0; i0 < 32; i0 += 8) {
                    int4 v[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const int tok = __shfl_sync(0xFFFFFFFFu, my_tok, i0 + q);
                        if (tok >= 0) {
                            v[q] = __ldg(reinterpret_cast<const int4 *>(
                                p.W1 + static_cast<size_t>(tok) * kRank + lane * 8));
                        } else {
                            v[q] = make_int4(0, 0, 0, 0);
                        }
                    }
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const int r = warp * 32 + i0 + q;
                        sts128(sA + chunk * kAChunk + r * 128 + ((unit ^ (r & 7)) << 4), v[q]);
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_afull);
                ++mt_count;

                // ---- vocabulary tiles of this CTA
                const bool active = (m0 + warp * 32) < p.B;
                const int b_glob = my_b + p.b_offset;
                float best_s = -INFINITY, best_l = 0.0f;
                uint32_t best_v = 0xFFFFFFFFu;
                for (int j = 0; j < ntiles; ++j) {
                    // warp-uniform outcome: tcgen05.ld below needs every lane of the warp
                    if (!__all_sync(0xFFFFFFFFu, wait_phase(bar_tfull + 8 * acc, aphase, ctl, p))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (active) {
                        uint32_t a[32];
                        tmem_ld_32x32b_x32(t_lane + static_cast<uint32_t>(acc * kTileN), a);
                        tmem_wait_ld();
                        const uint32_t sU = sStage + stage * kStageBytes + kW2Bytes;
                        const int v0 = (t_begin + j) * kTileN;
                        float l[32];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            uint32_t w0, w1, w2, w3;
                            lds128(sU + row * 64 + ((u ^ ((row >> 1) & 3)) << 4), w0, w1, w2, w3);
                            l[8 * u + 0] = __uint_as_float(a[8 * u + 0]) + bf16lo_to_f32(w0);
                            l[8 * u + 1] = __uint_as_float(a[8 * u + 1]) + bf16hi_to_f32(w0);
                            l[8 * u + 2] = __uint_as_float(a[8 * u + 2]) + bf16lo_to_f32(w1);
                            l[8 * u + 3] = __uint_as_float(a[8 * u + 3]) + bf16hi_to_f32(w1);
                            l[8 * u + 4] = __uint_as_float(a[8 * u + 4]) + bf16lo_to_f32(w2);
                            l[8 * u + 5] = __uint_as_float(a[8 * u + 5]) + bf16hi_to_f32(w2);
                            l[8 * u + 6] = __uint_as_float(a[8 * u + 6]) + bf16lo_to_f32(w3);
                            l[8 * u + 7] = __uint_as_float(a[8 * u + 7]) + bf16hi_to_f32(w3);
                        }
                        if (v0 + kTileN > p.V) {
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                if (v0 + i >= p.V) l[i] = -INFINITY;
                        }
                        float s[32];
                        if (p.mode == 0) {
#pragma unroll
                            for (int i = 0; i < 32; ++i) s[i] = l[i];
                        } else {
#pragma unroll
                            for (int q = 0; q < 8; ++q) {
                                const float lmax = fmaxf(fmaxf(l[4 * q], l[4 * q + 1]),
                                                         fmaxf(l[4 * q + 2], l[4 * q + 3]));
                                // noise cannot lift this group above the running best
                                const bool skip =
                                    !(fmaf(lmax, p.inv_tau, kGumbelMax) >= best_s);
                                if (__all_sync(0xFFFFFFFFu, skip)) {
                                    s[4 * q] = s[4 * q + 1] = s[4 * q + 2] = s[4 * q + 3] = -INFINITY;
                                } else {
                                    const uint4 w = philox(
                                        make_uint4(static_cast<uint32_t>(v0 / 4 + q),
                                                   static_cast<uint32_t>(k - 1),
                                                   static_cast<uint32_t>(b_glob), 0u),
                                        p.seed_lo, p.seed_hi);
                                    s[4 * q + 0] = fmaf(l[4 * q + 0], p.inv_tau, gumbel_from_word(w.x));
                                    s[4 * q + 1] = fmaf(l[4 * q + 1], p.inv_tau, gumbel_from_word(w.y));
                                    s[4 * q + 2] = fmaf(l[4 * q + 2], p.inv_tau, gumbel_from_word(w.z));
                                    s[4 * q + 3] = fmaf(l[4 * q + 3], p.inv_tau, gumbel_from_word(w.w));
                                    if (skip) s[4 * q] = s[4 * q + 1] = s[4 * q + 2] = s[4 * q + 3] = -INFINITY;
                                }
                            }
                        }
                        float mx = s[0];
#pragma unroll
                        for (int i = 1; i < 32; ++i) mx = fmaxf(mx, s[i]);
                        if (mx > best_s) {
                            int idx = 31;
#pragma unroll
                            for (int i = 31; i >= 0; --i)
                                if (s[i] == mx) idx = i;
                            best_s = mx;
                            best_v = static_cast<uint32_t>(v0 + idx);
                            float li = l[0];
#pragma unroll
                            for (int i = 1; i < 32; ++i)
                                if (i == idx) li = l[i];
                            best_l = li;
                        }
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive(bar_tempty + 8 * acc);
                        mbar_arrive(bar_empty + 8 * stage);
                    }
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                    if (++acc == kAcc) {
                        acc = 0;
                        aphase ^= 1u;
                    }
                }
                if (!ok) break;
                if (my_b < p.B) {
                    const unsigned long long key = argmax_key(best_s, best_v);
                    atomicMax(&p.slots[static_cast<size_t>(k - 1) * p.B + my_b], key);
                    row_key[my_b] = key;
                    row_logit[my_b] = best_l;
                }
            }

            // ---- grid barrier: every CTA has combined its rows of position k
            epi_sync();
            if (threadIdx.x == 0 && ok && !*reinterpret_cast<volatile int *>(&ctl.abort)) {
                __threadfence();
                atomicAdd(p.barrier, 1u);
                const uint32_t target =
                    static_cast<uint32_t>(k) * static_cast<uint32_t>(G) + static_cast<uint32_t>(p.barrier_extra);
                const uint64_t t0 = globaltimer_ns();
                while (ld_acquire_u32(p.barrier) < target) {
                    if (*reinterpret_cast<volatile unsigned int *>(p.abort_flag)) {
                        *reinterpret_cast<volatile int *>(&ctl.abort) = 1;
                        break;
                    }
                    if (globaltimer_ns() - t0 > p.timeout_ns) {
                        give_up(ctl, p, DSPARK_TIMEOUT);
                        break;
                    }
                    __nanosleep(64);
                }
                __threadfence();
            }
            epi_sync();
            if (!ok || *reinterpret_cast<volatile int *>(&ctl.abort)) {
                ok = false;
                break;
            }
            // ---- outputs of position k: written by the CTA that owns the winning column
            for (int b = threadIdx.x; b < p.B; b += kEpiThreads) {
                const unsigned long long key =
                    __ldcg(&p.slots[static_cast<size_t>(k - 1) * p.B + b]);
                if (key == row_key[b]) {
                    p.x_out[static_cast<size_t>(b) * p.gamma + (k - 1)] =
                        static_cast<int32_t>(argmax_key_index(key));
                    p.logit_out[static_cast<size_t>(b) * p.gamma + (k - 1)] = row_logit[b];
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace draft
}  // namespace dspark
