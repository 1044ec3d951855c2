// markov_pair.cuh -- the Markov head for large batches (B > 128) on CTA pairs.
//
// gdymind.com, "DSpark: DeepSeek's new speculative decoding work", section 4 ("Sequential
// stage", "Markov head"): position k adds the transition bias W1[x_{k-1}] W2 (rank
// r = 256) to the backbone's base logits U_k and picks x_k from them.  The arithmetic is
// that of markov_draft_kernel; this kernel arranges it for many requests.
//
// With more than 128 requests the bias GEMM has several 128-row M tiles, and a single
// CTA streams its whole W2 slice once per M tile.  Here the CTAs run as pairs (clusters
// of two on one TPC) and every MMA is a pair MMA (tcgen05.mma.cta_group::2, M = 256): the
// even CTA issues it, each CTA holds the A rows of its own 128 requests and half of the
// W2 tile's columns, and each CTA's TMEM receives its 128 rows of the accumulator.  Every
// W2 byte a CTA loads therefore serves 256 requests instead of 128.  The A rows sit in
// tensor memory, in two buffers (written there by the epilogue warps with tcgen05.st), so
// that the next block's rows are in place before its first MMA and the tensor core reads
// only W2 from shared memory, whose bandwidth the TMA copies and the epilogue's U reads
// share.  Each pair owns a contiguous vocabulary slice cut into 128-column tiles; for
// every position k it walks the tiles once per super-pass, alternating direction from
// one walk to the next, so that the tiles read last are read again first and are still
// in L2.  In greedy drafting a super-pass is two blocks of 256 requests: every W2 tile
// then feeds 16 MMAs per block (one accumulator each) before its stages are released.
// Gumbel-max, bound by its selection arithmetic, walks once per block.
//
// Per CTA: 16 epilogue warps (four per TMEM lane quadrant, one 32-column chunk of every
// tile each), warp 16 the W2 producer (TMA, 64 columns x 128 K rows per stage), warp 17
// the U producer (TMA, 128 rows x 64 columns per box), warp 18 the MMA issuer in the even
// CTA, and in the kConf instances warp 19 the confidence head (as in
// markov_draft_kernel).  Signals that cross the pair: the odd CTA's W2 copies complete
// on the even CTA's stage barrier (.cta_group::2 copies; the even CTA arms it for both
// halves), and its A gathers and accumulator releases arrive on the even CTA's barriers;
// the even CTA's MMA completions arrive on both CTAs' barriers through one pair commit.
//
// Selection as in markov_draft_kernel: greedy argmax with the smallest index on ties, or
// Gumbel-max with Philox noise keyed (seed, request, position, vocabulary index).  Here the
// Gumbel scores are taken in the log2 domain, l log2(e)/tau - log2(-log2 u), which is
// log2(e) times the natural-log score minus a constant, so the chosen index is the same.
// Rows are combined within the CTA through shared memory and across CTAs by a 64-bit
// atomicMax; a bounded grid barrier ends each position.
#pragma once
#include "markov_draft.cuh"

namespace dspark {
namespace draft {
namespace pairk {

constexpr int kEpiWarps = 16;
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kWarpW2 = kEpiWarps, kWarpU = kEpiWarps + 1, kWarpMma = kEpiWarps + 2;
constexpr int kThreads = (kEpiWarps + 3) * 32;        // 608
constexpr int kWarpConfPair = kEpiWarps + 3;          // confidence head (kConf instances)
constexpr int kThreadsConfPair = kThreads + 32;       // 640
constexpr int kRows = 128;                            // requests per CTA per block
constexpr int kPairRows = 2 * kRows;                  // the pair MMA's M
constexpr int kW2Stages = 7;
constexpr int kW2StageBytes = 64 * kKSlice * 2;       // 64 columns x 128 K rows: 16 KB
constexpr int kUSlots = 6;
constexpr int kUSlotBytes = kRows * kUBoxCols * 2;    // 128 rows x 64 columns: 16 KB
constexpr int kDynSmem = kW2Stages * kW2StageBytes + kUSlots * kUSlotBytes + 1024;
// TMEM (512 columns): two 128-column accumulators, then two buffers of A = W1[x_{k-1}]
// for the CTA's 128 rows (row m in lane m, K = 256 bf16 packed two per column: 128
// columns each): one per block of a super-pass
constexpr int kPairAcc = 2;
constexpr int kABufs = 2;
constexpr uint32_t kACol = kPairAcc * kAccCols;       // 256: A buffer b at 256 + 128 b
constexpr int kMaxPasses = kMaxB / kPairRows;         // 256-request blocks: 4
constexpr int kChunks = 4;                            // 32-column chunks of a tile
constexpr int kBoxWarps = 2 * 4;                      // warps reading one U box: 2 chunks x 4 quadrants
constexpr float kLog2e = 1.4426950408889634f;
// above any log2-domain noise value: -log2(-log2 u) <= -log2(2^-24 log2 e) < 23.5
constexpr float kGumbel2Max = 24.0f;

struct Ctl {
    unsigned long long w2_full[kW2Stages];   // even CTA: both CTAs' W2 halves have landed
    unsigned long long w2_empty[kW2Stages];  // both: the pair MMAs have read the stage
    unsigned long long u_full[kUSlots];
    unsigned long long u_empty[kUSlots];
    unsigned long long tfull[kPairAcc];      // both: the accumulator holds a tile
    unsigned long long tempty[kPairAcc];     // even CTA: all 32 epilogue warps have read it
    unsigned long long afull[kABufs];        // even CTA: all 32 epilogue warps gathered A
    unsigned long long aempty[kABufs];       // both: the pair MMAs no longer read A
    unsigned long long drain;
    uint32_t tmem_base;
    int abort;
};

struct Shared {
    Ctl ctl;
    unsigned long long part_key[kChunks][kRows];   // per chunk warp, before the CTA combine
    float part_logit[kChunks][kRows];
    unsigned long long cta_key[kMaxPasses][kRows];  // this CTA's best per row and block
    float cta_logit[kMaxPasses][kRows];
    int tok[kMaxPasses][kRows];                     // x_{k-1} of this CTA's rows (-1: none)
    int go;                                         // verdict of the last grid barrier
};

// Optional per-tile timeline (build with -DDSPARK_TRACE): for position 2, block 0, tile j
// and event e, a %globaltimer stamp in g_trace[(blockIdx.x * 64 + j) * 32 + e].
#ifdef DSPARK_TRACE
#define PAIR_TRACE(k, ps, j, e)                                                               \
    do {                                                                                      \
        if ((k) == 2 && (ps) == 0 && (j) < 64 && blockIdx.x < 256)                            \
            g_trace[(blockIdx.x * 64 + (j)) * 32 + (e)] = globaltimer_ns();                   \
    } while (0)
#else
#define PAIR_TRACE(k, ps, j, e) \
    do {                        \
    } while (0)
#endif

// Named barrier of the 16 epilogue warps.
__device__ __forceinline__ void epi_sync512() { asm volatile("bar.sync 1, 512;" ::: "memory"); }

__device__ __forceinline__ void give_up(Ctl &ctl, const Params &p, unsigned code)
{
    record_error(code);
    *reinterpret_cast<volatile int *>(&ctl.abort) = 1;
    atomicExch(p.abort_flag, 1u);
}

// Bounded wait on an mbarrier phase.  CTA-scope acquire also for the barriers that the
// other CTA of the pair arrives on: what those arrivals order is tensor-core work (A
// stores, accumulator reads, TMA landings), which the tcgen05 fences around the arrive and
// the wait order (the pairing CUTLASS's two-SM pipelines use too).  False once this CTA or
// any other gave up, or the wait ran out.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, Ctl &ctl, const Params &p)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        if (mbar_try_wait_sleep(bar, parity, kWaitHintNs)) return true;
        if (*reinterpret_cast<volatile int *>(&ctl.abort) ||
            *reinterpret_cast<volatile unsigned int *>(p.abort_flag)) {
            *reinterpret_cast<volatile int *>(&ctl.abort) = 1;
            return false;
        }
        if (globaltimer_ns() - t0 > p.timeout_ns) {
            give_up(ctl, p, DSPARK_TIMEOUT);
            return false;
        }
    }
}

// Wait for the last use of every slot of a ring after `issued` uses in total.  If the
// kernel is aborting, a stage may never be used or completed: then the copies this CTA may
// still have in flight get a fixed time to land, and the result is false.
constexpr uint64_t kSettleNs = 200000;
__device__ __forceinline__ bool drain_or_settle(uint32_t bar0, int n, long long issued, Ctl &ctl,
                                                const Params &p)
{
    for (int s = 0; s < n; ++s) {
        const long long uses = issued / n + (s < issued % n ? 1 : 0);
        if (uses > 0 && !wait_bar(bar0 + 8 * s, static_cast<uint32_t>((uses - 1) & 1), ctl, p)) {
            const uint64_t t0 = globaltimer_ns();
            while (globaltimer_ns() - t0 < kSettleNs) __nanosleep(1000);
            return false;
        }
    }
    return true;
}

// The j-th tile of super-pass S: forward on even super-passes, backward on odd ones.
__device__ __forceinline__ int snake(int S, int j, int ntiles)
{
    return (S & 1) ? ntiles - 1 - j : j;
}

// Request block ps always reads A buffer ps mod 2.  Uses of that buffer before block ps
// of position k: every earlier position's blocks of the same parity, and this position's
// blocks ps - 2, ps - 4, ...
__device__ __forceinline__ uint32_t abuf_uses(int k, int ps, int npass)
{
    const int per_position = (ps & 1) ? npass / 2 : (npass + 1) / 2;
    return static_cast<uint32_t>((k - 1) * per_position + (ps >> 1));
}

// ------------------------------------------------------------------ Philox, one request row
// Philox4x32-10 (Salmon et al., SC'11) on the counter (x, y, z, 0), where y = k - 1 and
// z = the request are fixed for a row: the parts of the first two rounds that depend only
// on them are computed once per row and position.
constexpr uint32_t kPhM0 = 0xD2511F53u, kPhM1 = 0xCD9E8D57u;
constexpr uint32_t kPhW0 = 0x9E3779B9u, kPhW1 = 0xBB67AE85u;

struct RowNoise {
    uint32_t r0, l1, h0p, l0p;
};

__device__ __forceinline__ RowNoise row_noise(uint32_t y, uint32_t z, uint32_t k0, uint32_t k1)
{
    RowNoise n;
    n.r0 = __umulhi(kPhM1, z) ^ y ^ k0;     // word 0 after round 1
    n.l1 = kPhM1 * z;                       // word 1 after round 1
    n.h0p = __umulhi(kPhM0, n.r0);          // round 2 products of word 0
    n.l0p = kPhM0 * n.r0;
    (void)k1;
    return n;
}

// hi and lo halves of a 32 x 32-bit product from one wide multiply
__device__ __forceinline__ void mul_wide(uint32_t a, uint32_t b, uint32_t &hi, uint32_t &lo)
{
    uint64_t r;
    asm("mul.wide.u32 %0, %1, %2;" : "=l"(r) : "r"(a), "r"(b));
    hi = static_cast<uint32_t>(r >> 32);
    lo = static_cast<uint32_t>(r);
}

// Philox4x32-10 of the counter (x, y, z, 0) for the row `n` describes.  The round keys
// come precomputed from the launch parameters (constant memory), so that no round spends
// instructions on the key schedule, and each round's two products are wide multiplies.
__device__ __forceinline__ uint4 philox_row(uint32_t x, const RowNoise &n, const Params &p)
{
    uint32_t hi0, lo0, hi1, lo1;
    mul_wide(kPhM0, x, hi0, lo0);                                 // round 1
    const uint32_t cz = hi0 ^ p.rk1[0];
    mul_wide(kPhM1, cz, hi1, lo1);                                // round 2
    uint4 c = make_uint4(hi1 ^ n.l1 ^ p.rk0[1], lo1, n.h0p ^ lo0 ^ p.rk1[1], n.l0p);
#pragma unroll
    for (int round = 2; round < 10; ++round) {
        uint32_t a0, b0, a1, b1;
        mul_wide(kPhM0, c.x, a0, b0);
        mul_wide(kPhM1, c.z, a1, b1);
        c = make_uint4(a1 ^ c.y ^ p.rk0[round], b1, a0 ^ c.w ^ p.rk1[round], b0);
    }
    return c;
}

// Log2-domain noise of one Philox word: u = ((w >> 9) + 0.5) 2^-23 (exact), and the result
// is -log2(e2) with e2 = -log2 u, which equals log2(e) (-ln(-ln u)) - log2(log2 e).  e2 is
// the hardware log2 except within 2^-6 of u = 1, where the hardware log2 loses relative
// accuracy and e2 = log2(e) (t + t^2/2) with t = 1 - u (exact) is used instead: the
// series -ln(1 - t) = t + t^2/2 + t^3/3 + ... cut after two terms, relative error < t^2/3.
__device__ __forceinline__ float gumbel2_from_word(uint32_t w)
{
    const float u = fmaf(static_cast<float>(w >> 9), 0x1p-23f, 0x1p-24f);
    const float t = 1.0f - u;
    const float e_series = t * fmaf(t, 0.5f * kLog2e, kLog2e);
    const float e_log = -__log2f(u);
    const float e = (t < 0.015625f) ? e_series : e_log;
    return -__log2f(e);
}

// One 32-column chunk of one request row: l = acc + U; greedy keeps the largest logit,
// Gumbel-max the largest l c2 + noise (c2 = log2(e)/tau); strict improvement keeps the
// smallest column on ties.  Greedy and Gumbel are separate kernel instances (kGumbel), so
// that the greedy one carries none of the noise code.
template <bool kGumbel>
__device__ __forceinline__ void chunk_update(RowBest &best, const uint32_t (&a)[32], uint32_t sU,
                                             int row, int h, int v0, const Params &p,
                                             const RowNoise &rn, float c2)
{
    float l[32];
    add_u32(l, a, sU, row, h);
    if (v0 + kUnit > p.V) {
#pragma unroll
        for (int i = 0; i < 32; ++i)
            if (v0 + i >= p.V) l[i] = -INFINITY;
    }
    if constexpr (!kGumbel) {
        const float mx = max32(l);
        if (mx > best.s) {
            best.v = static_cast<uint32_t>(v0 + first_index(l, mx));
            best.s = mx;
            best.l = mx;
        }
        return;
    }
    // exact pruning, one vote per warp: skip the noise when no row of the warp can beat its
    // running best with the largest noise value
    if (__all_sync(0xFFFFFFFFu, !(fmaf(max32(l), c2, kGumbel2Max) >= best.s))) return;
    float s[32];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const uint4 w = philox_row(static_cast<uint32_t>((v0 >> 2) + q), rn, p);
        s[4 * q + 0] = fmaf(l[4 * q + 0], c2, gumbel2_from_word(w.x));
        s[4 * q + 1] = fmaf(l[4 * q + 1], c2, gumbel2_from_word(w.y));
        s[4 * q + 2] = fmaf(l[4 * q + 2], c2, gumbel2_from_word(w.z));
        s[4 * q + 3] = fmaf(l[4 * q + 3], c2, gumbel2_from_word(w.w));
    }
    const float mx = max32(s);
    if (mx > best.s) {
        const int idx = first_index(s, mx);
        best.v = static_cast<uint32_t>(v0 + idx);
        best.s = mx;
        best.l = pick(l, idx);
    }
}

template <bool kGumbel, bool kConf>
__global__ void __launch_bounds__(kConf ? kThreadsConfPair : kThreads, 1)
    markov_pair_kernel(const __grid_constant__ CUtensorMap tm_w2,
                       const __grid_constant__ CUtensorMap tm_u, const Params p)
{
    extern __shared__ uint8_t dyn_smem[];
    __shared__ Shared sh;
    Ctl &ctl = sh.ctl;

    // everything below assumes clusters of exactly two CTAs and whole pairs: a launch in
    // any other shape (a tool re-issuing it without the cluster, say) stops here, before
    // any pair instruction or cross-CTA access
    if (cluster_nctarank() != 2u || (gridDim.x & 1u) ||
        blockDim.x != static_cast<unsigned>(kConf ? kThreadsConfPair : kThreads)) {
        if (threadIdx.x == 0) record_error(DSPARK_BAD_LAUNCH);
        return;
    }
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();          // 0: even CTA (issues the MMAs)
    const bool lead = rank == 0;
    const uint32_t base = (smem_u32(dyn_smem) + 1023u) & ~1023u;
    const uint32_t sW2 = base;
    const uint32_t sU = sW2 + kW2Stages * kW2StageBytes;

    const int npairs = gridDim.x >> 1;
    const int pair = blockIdx.x >> 1;
    const int u_begin = static_cast<int>(static_cast<long long>(pair) * p.units_total / npairs);
    const int u_end = static_cast<int>(static_cast<long long>(pair + 1) * p.units_total / npairs);
    const int n_units = u_end - u_begin;
    const int ntiles = (n_units + kMaxUnits - 1) / kMaxUnits;
    const int npass = (p.B + kPairRows - 1) / kPairRows;   // 256-request blocks per position
    // super-pass: the request blocks that take their MMAs from the same W2 stages, tile by
    // tile (two for greedy drafting; one for Gumbel-max, whose selection arithmetic, not
    // the W2 stream, bounds it)
    constexpr int kSpMax = kGumbel ? 1 : 2;
    const int nsp = (npass + kSpMax - 1) / kSpMax;          // super-passes per position
    auto sp_blocks = [&](int sp) { return min(kSpMax, npass - kSpMax * sp); };
    // A buffer of block ps at position k, and its uses before that: the block's parity with
    // two blocks per super-pass; with one, the launch-wide pass number's parity (so that
    // consecutive passes, also across positions, alternate)
    auto a_buf = [&](int k, int ps) -> int {
        return kSpMax == 2 ? (ps & 1) : (((k - 1) * npass + ps) & 1);
    };
    auto a_uses = [&](int k, int ps) -> uint32_t {
        return kSpMax == 2 ? abuf_uses(k, ps, npass) : static_cast<uint32_t>(((k - 1) * npass + ps) >> 1);
    };

    const uint32_t bar_w2_full = smem_u32(&ctl.w2_full[0]);
    const uint32_t bar_w2_empty = smem_u32(&ctl.w2_empty[0]);
    const uint32_t bar_u_full = smem_u32(&ctl.u_full[0]);
    const uint32_t bar_u_empty = smem_u32(&ctl.u_empty[0]);
    const uint32_t bar_tfull = smem_u32(&ctl.tfull[0]);
    const uint32_t bar_tempty = smem_u32(&ctl.tempty[0]);
    const uint32_t bar_afull = smem_u32(&ctl.afull[0]);
    const uint32_t bar_aempty = smem_u32(&ctl.aempty[0]);
    const uint32_t bar_drain = smem_u32(&ctl.drain);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kW2Stages; ++s) {
            mbar_init(bar_w2_full + 8 * s, 1);
            mbar_init(bar_w2_empty + 8 * s, 1);
        }
        for (int s = 0; s < kUSlots; ++s) {
            mbar_init(bar_u_full + 8 * s, 1);
            mbar_init(bar_u_empty + 8 * s, kBoxWarps);
        }
        for (int a = 0; a < kPairAcc; ++a) {
            mbar_init(bar_tfull + 8 * a, 1);
            mbar_init(bar_tempty + 8 * a, 2 * kEpiWarps);
        }
        for (int b = 0; b < kABufs; ++b) {
            mbar_init(bar_afull + 8 * b, 2 * kEpiWarps);
            mbar_init(bar_aempty + 8 * b, 1);
        }
        mbar_init(bar_drain, 1);
        ctl.abort = 0;
        mbar_fence_init();
    }
    if (warp == kWarpMma) {
        tmem_alloc_pair(smem_u32(&ctl.tmem_base), kTmemCols);
        tmem_relinquish_pair();
    }
    if (warp == kWarpW2 && lane == 0) {
        tma_prefetch_desc(&tm_w2);
        tma_prefetch_desc(&tm_u);
    }
    tc_fence_before();
    cluster_sync();                  // both CTAs' barriers exist before any cross-CTA signal
    tc_fence_after();
    const uint32_t tmem = ctl.tmem_base;

    if (warp == kWarpW2) {
        // ------------------------------------------------------------ W2 producer (both CTAs)
        if (lane == 0) {
            const uint64_t pol_w2 = l2_policy_evict_last();
            const uint32_t w2_full_lead = mapa_shared(bar_w2_full, 0);
            Ring w2;
            long long issued = 0;
            bool ok = true;
            for (int k = 1; k <= p.gamma && ok; ++k)
                for (int sp = 0; sp < nsp && ok; ++sp) {
                    const int S = (k - 1) * nsp + sp;
                    [[maybe_unused]] const int ps = kSpMax * sp;
                    for (int j = 0; j < ntiles && ok; ++j) {
                        int first, count;
                        tile_span(snake(S, j, ntiles), n_units, ntiles, first, count);
                        // this CTA's half of the tile: columns rank * N/2 .. + N/2 (a 64-column box)
                        const int x = (u_begin + first) * kUnit + static_cast<int>(rank) * count * (kUnit / 2);
                        for (int ks = 0; ks < kKSlices; ++ks) {
                            if (!wait_bar(bar_w2_empty + 8 * w2.slot, w2.phase ^ 1u, ctl, p)) {
                                ok = false;
                                break;
                            }
                            PAIR_TRACE(k, ps, j, 8 + ks);
                            // both halves count on the even CTA's barrier, armed there for both
                            const uint32_t bar = bar_w2_full + 8 * w2.slot;
                            if (lead) {
                                mbar_arrive_expect_tx(bar, 2 * kW2StageBytes);
                                tma_load_2d(sW2 + w2.slot * kW2StageBytes, &tm_w2, bar, x,
                                            ks * kKSlice, pol_w2);
                            } else {
                                tma_load_2d_pair(sW2 + w2.slot * kW2StageBytes, &tm_w2, w2_full_lead + 8 * w2.slot,
                                                 x, ks * kKSlice, pol_w2);
                            }
                            ++issued;
                            w2.next(kW2Stages);
                        }
                    }
                }
            // the copies land before exit: the even CTA sees both halves on w2_full, and every
            // stage the MMAs released (w2_empty, in both CTAs) had landed
            if (!lead || drain_or_settle(bar_w2_full, kW2Stages, issued, ctl, p))
                drain_or_settle(bar_w2_empty, kW2Stages, issued, ctl, p);
        }
    } else if (warp == kWarpU) {
        // ------------------------------------------------------------ U producer (both CTAs)
        if (lane == 0) {
            const uint64_t pol_u = l2_policy_evict_first();
            Ring ur;
            long long issued = 0;
            bool ok = true;
            for (int k = 1; k <= p.gamma && ok; ++k)
                for (int sp = 0; sp < nsp && ok; ++sp) {
                    const int S = (k - 1) * nsp + sp;
                    const int nb = sp_blocks(sp);
                    for (int j = 0; j < ntiles && ok; ++j) {
                        int first, count;
                        tile_span(snake(S, j, ntiles), n_units, ntiles, first, count);
                        const int v0 = (u_begin + first) * kUnit;
                        for (int bi = 0; bi < nb && ok; ++bi) {
                            const int ps = kSpMax * sp + bi;
                            const int row0 = ps * kPairRows + static_cast<int>(rank) * kRows;
                            for (int u = 0; u < count; u += 2) {
                                if (!wait_bar(bar_u_empty + 8 * ur.slot, ur.phase ^ 1u, ctl, p)) {
                                    ok = false;
                                    break;
                                }
                                PAIR_TRACE(k, ps, j, 10 + u / 2);
                                const uint32_t bar = bar_u_full + 8 * ur.slot;
                                mbar_arrive_expect_tx(bar, kUSlotBytes);
                                tma_load_3d(sU + ur.slot * kUSlotBytes, &tm_u, bar, v0 + u * kUnit, k - 1,
                                            row0, pol_u);
                                ++issued;
                                ur.next(kUSlots);
                            }
                        }
                    }
                }
            drain_ring(bar_u_full, kUSlots, issued, p);
        }
    } else if (kConf && warp == kWarpConfPair) {
        // ------------------------------------------------------------ confidence head
        confidence_warp(p, static_cast<int>(gridDim.x));
    } else if (warp == kWarpMma) {
#ifdef DSPARK_TRACE
        if (lane == 0 && !lead) {
            // trace only: when each accumulator of positions 1-2 completes, by polling
            Ring acc;
            bool live = true;
            for (int k = 1; k <= 2 && k <= p.gamma && live; ++k)
                for (int ps = 0; ps < npass && live; ++ps)
                    for (int j = 0; j < ntiles && live; ++j) {
                        const uint64_t t0 = globaltimer_ns();
                        while (!mbar_test_wait(bar_tfull + 8 * acc.slot, acc.phase))
                            if (globaltimer_ns() - t0 > p.timeout_ns) {
                                live = false;
                                break;
                            }
                        PAIR_TRACE(k, ps, j, 5);
                        acc.next(kPairAcc);
                    }
        }
#endif
        if (lane == 0 && lead) {
            // -------------------------------------------------------- pair MMA issuer (even CTA)
            Ring w2, acc;
            const uint64_t b_desc0 = smem_desc(sW2, kW2StageBytes, 1024, kSwizzle128B);
            const uint16_t both = 0x3;
            bool issued_any = false;
            bool ok = true;
            for (int k = 1; k <= p.gamma && ok; ++k)
                for (int sp = 0; sp < nsp && ok; ++sp) {
                    const int S = (k - 1) * nsp + sp;
                    const int nb = sp_blocks(sp);
                    // block ps = kSpMax sp + bi reads A buffer ps mod 2; its rows are waited
                    // for right before its first MMAs (the first tile's), so that block 0's
                    // MMAs start while block 1's rows are still being gathered
                    for (int j = 0; j < ntiles && ok; ++j) {
                        [[maybe_unused]] const int ps = kSpMax * sp;
                        int first, count;
                        tile_span(snake(S, j, ntiles), n_units, ntiles, first, count);
                        const uint32_t idesc = idesc_bf16_f32(static_cast<uint32_t>(kPairRows),
                                                              static_cast<uint32_t>(count * kUnit), 1);
                        static_assert(kKSlices == 2, "a tile's K is two W2 stages");
                        // both K halves are waited for up front, so that the tile's MMAs issue
                        // back to back: the tensor core's queue is short, and a wait between
                        // them leaves it idle.  Every block of the super-pass then takes its 16
                        // MMAs from the same two stages, into its own accumulator.
                        Ring w2b = w2;
                        w2b.next(kW2Stages);
#pragma unroll
                        for (int bi = 0; bi < kSpMax; ++bi) {
                            if (bi >= nb) break;
                            PAIR_TRACE(k, ps + bi, j, 0);
                            if (!wait_bar(bar_tempty + 8 * acc.slot, acc.phase ^ 1u, ctl, p)) {
                                ok = false;
                                break;
                            }
                            PAIR_TRACE(k, ps + bi, j, 1);
                            if (bi == 0 && (!wait_bar(bar_w2_full + 8 * w2.slot, w2.phase, ctl, p) ||
                                            !wait_bar(bar_w2_full + 8 * w2b.slot, w2b.phase, ctl, p))) {
                                ok = false;
                                break;
                            }
                            PAIR_TRACE(k, ps + bi, j, 2);
                            if (j == 0 && !wait_bar(bar_afull + 8 * a_buf(k, ps + bi),
                                                    a_uses(k, ps + bi) & 1u, ctl, p)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
                            const uint32_t d_tmem = tmem + static_cast<uint32_t>(acc.slot * kAccCols);
                            const uint32_t a_col = kACol + static_cast<uint32_t>(a_buf(k, ps + bi) * kAccCols);
#pragma unroll
                            for (int ks = 0; ks < kKSlices; ++ks) {
                                const uint32_t slot = ks ? w2b.slot : w2.slot;
                                const uint64_t b_k = b_desc0 + static_cast<uint64_t>((slot * kW2StageBytes) >> 4);
#pragma unroll
                                for (int kk = 0; kk < kKSlice / 16; ++kk) {
                                    // K elements ks*128 + 16 kk .. + 15: 8 TMEM columns of A
                                    const uint32_t a_tmem =
                                        tmem + a_col + static_cast<uint32_t>((ks * kKSlice + 16 * kk) >> 1);
                                    const uint64_t b_desc = b_k + static_cast<uint64_t>((kk * 2048) >> 4);
                                    umma_bf16_pair_ts(d_tmem, a_tmem, b_desc, idesc, (ks | kk) ? 1u : 0u);
                                }
                            }
                            issued_any = true;
                            umma_commit_pair_mask(bar_tfull + 8 * acc.slot, both);
                            PAIR_TRACE(k, ps + bi, j, 4);
                            acc.next(kPairAcc);
                        }
                        if (!ok) break;
                        umma_commit_pair_mask(bar_w2_empty + 8 * w2.slot, both);
                        umma_commit_pair_mask(bar_w2_empty + 8 * w2b.slot, both);
                        w2b.next(kW2Stages);
                        w2 = w2b;
                    }
                    if (!ok) break;
                    for (int bi = 0; bi < nb; ++bi)
                        umma_commit_pair_mask(bar_aempty + 8 * a_buf(k, kSpMax * sp + bi), both);
                }
            if (issued_any) {
                umma_commit_pair(bar_drain);
                wait_drain(bar_drain, 0, p);
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue (warps 0-15)
        // Every epilogue warp runs the same sequence of named barriers whatever happens:
        // after a failed wait a warp only skips work (waits, loads, copies), so that no
        // bar.sync is ever left short of arrivals.
        const int et = threadIdx.x;                       // 0 .. 511
        const int q = warp & 3;                           // TMEM lane quadrant
        const int c = warp >> 2;                          // chunk of every tile: columns 32c ..
        const int row = q * 32 + lane;                    // row of this CTA's 128
        const uint32_t t_lane = tmem + (static_cast<uint32_t>(q * 32) << 16);
        const uint32_t afull_lead = mapa_shared(bar_afull, 0);
        const uint32_t tempty_lead = mapa_shared(bar_tempty, 0);
        const float c2 = p.inv_tau * kLog2e;
        Ring acc, ur;
        bool ok = true;                                   // uniform within a warp

        for (int i = et; i < kMaxPasses * kRows; i += kEpiThreads) {
            const int ps = i / kRows, r = i % kRows;
            const int b = ps * kPairRows + static_cast<int>(rank) * kRows + r;
            sh.tok[ps][r] = (ps < npass && b < p.B) ? checked_token(p.anchor[b], p.V) : -1;
        }
        epi_sync512();

        // this warp's share of A for block ps of position k: K elements 64c .. 64c + 63 of
        // the W1 rows of its quadrant's 32 requests (zeros for rows without a request),
        // loaded into registers (a whole 128-byte line per lane) and stored into the block's
        // A buffer in TMEM, once the MMAs of that buffer's previous use have released it
        // (bounded wait).  The result says whether the rows were stored.
        auto gather = [&](int k, int ps) -> bool {
            const int abuf = a_buf(k, ps);
            const uint32_t free_parity = (a_uses(k, ps) & 1u) ^ 1u;
            if (!__all_sync(0xFFFFFFFFu, wait_bar(bar_aempty + 8 * abuf, free_parity, ctl, p))) {
                ok = false;
                return false;
            }
            const int tok = sh.tok[ps][row];
            uint32_t v[32];
            if (tok >= 0) {
                const uint4 *src = reinterpret_cast<const uint4 *>(
                    p.W1 + static_cast<size_t>(tok) * kRank + c * 64);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint4 t = __ldg(src + i);
                    v[4 * i] = t.x;
                    v[4 * i + 1] = t.y;
                    v[4 * i + 2] = t.z;
                    v[4 * i + 3] = t.w;
                }
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = 0u;
            }
            tmem_st_32x32b_x32(t_lane + kACol + static_cast<uint32_t>(abuf * kAccCols + c * 32), v);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (lead) mbar_arrive(bar_afull + 8 * abuf);
                else mbar_arrive_remote(afull_lead + 8 * abuf);
            }
            return true;
        };

        // bounded grid barrier number nth; the verdict is taken by one thread and shared, so
        // that all epilogue threads agree on it
        auto grid_sync = [&](uint32_t nth) -> bool {
            if (!ok) *reinterpret_cast<volatile int *>(&ctl.abort) = 1;   // this warp failed: stop
            epi_sync512();
            if (et == 0) {
                bool good = !*reinterpret_cast<volatile int *>(&ctl.abort);
                if (good) {
                    red_release_add_u32(p.barrier, 1u);
                    const uint32_t target = nth * static_cast<uint32_t>(gridDim.x) +
                                            static_cast<uint32_t>(p.barrier_extra);
                    const uint64_t t0 = globaltimer_ns();
                    while (ld_acquire_u32(p.barrier) < target) {
                        if (*reinterpret_cast<volatile unsigned int *>(p.abort_flag)) {
                            good = false;
                            break;
                        }
                        if (globaltimer_ns() - t0 > p.timeout_ns) {
                            give_up(ctl, p, DSPARK_TIMEOUT);
                            good = false;
                            break;
                        }
                    }
                }
                if (!good) *reinterpret_cast<volatile int *>(&ctl.abort) = 1;
                sh.go = good ? 1 : 0;
            }
            epi_sync512();
            return sh.go != 0;
        };

        for (int k = 1; k <= p.gamma; ++k) {
            if (ok) {
                // L2 prefetch of the W1 lines the later blocks of this position will gather
                for (int ps = 1; ps < npass; ++ps) {
                    const int tok = sh.tok[ps][row];
                    if (tok >= 0) prefetch_l2(p.W1 + static_cast<size_t>(tok) * kRank + c * 64);
                }
                // the rows of the first super-pass's blocks, each into its own A buffer
                if (gather(k, 0) && npass > 1) gather(k, 1);
            }
            for (int sp = 0; sp < nsp; ++sp) {
                const int S = (k - 1) * nsp + sp;
                const int nb = sp_blocks(sp);
                RowBest best[kSpMax];
                // Gumbel-max runs one block per super-pass: its row's noise key, once
                static_assert(!kGumbel || kSpMax == 1, "one block per super-pass with noise");
                const RowNoise rn = kGumbel ? row_noise(static_cast<uint32_t>(k - 1),
                                                        static_cast<uint32_t>(sp * kPairRows + static_cast<int>(rank) * kRows +
                                                                              row + p.b_offset),
                                                        p.seed_lo, p.seed_hi)
                                            : RowNoise{0u, 0u, 0u, 0u};
                for (int j = 0; j < ntiles; ++j) {
                    int first, count;
                    tile_span(snake(S, j, ntiles), n_units, ntiles, first, count);
                    const int nbox = (count + 1) >> 1;
                    const int box = c >> 1;
#pragma unroll
                    for (int bi = 0; bi < kSpMax; ++bi) {
                        if (bi >= nb) break;
                        const int ps = kSpMax * sp + bi;
                        const bool active = ps * kPairRows + static_cast<int>(rank) * kRows + q * 32 < p.B;
                        // the U box first (it is usually there already), then the accumulator:
                        // the chunk goes to registers and the slot is released at once, so that
                        // the next MMAs into it overlap the arithmetic below
                        Ring my = ur;
                        for (int i = 0; i < box; ++i) my.next(kUSlots);
                        const bool has_box = box < nbox;
                        if (ok && has_box &&
                            !__all_sync(0xFFFFFFFFu, wait_bar(bar_u_full + 8 * my.slot, my.phase, ctl, p)))
                            ok = false;
                        if (lane == 0 && (warp == 0 || warp == 12)) PAIR_TRACE(k, ps, j, 12 + (warp == 12));
                        // warp-uniform: tcgen05.ld below needs every lane of the warp
                        if (ok && !__all_sync(0xFFFFFFFFu,
                                              wait_bar(bar_tfull + 8 * acc.slot, acc.phase, ctl, p)))
                            ok = false;
                        if (lane == 0 && (warp == 0 || warp == 12)) PAIR_TRACE(k, ps, j, 16 + (warp == 12) * 4);
                        if (ok) {
                            auto release = [&]() {
                                tc_fence_before();
                                __syncwarp();
                                if (lane == 0) {
                                    if (lead) mbar_arrive(bar_tempty + 8 * acc.slot);
                                    else mbar_arrive_remote(tempty_lead + 8 * acc.slot);
                                }
                            };
                            tc_fence_after();
                            if (active && c < count) {
                                uint32_t a[32];
                                tmem_ld_32x32b_x32(
                                    t_lane + static_cast<uint32_t>(acc.slot * kAccCols + c * kUnit), a);
                                tmem_wait_ld();
                                release();
                                if (lane == 0 && (warp == 0 || warp == 12)) PAIR_TRACE(k, ps, j, 17 + (warp == 12) * 4);
                                chunk_update<kGumbel>(best[bi], a, sU + my.slot * kUSlotBytes, row, c & 1,
                                                      (u_begin + first + c) * kUnit, p, rn, c2);
                            } else {
                                release();
                            }
                            __syncwarp();
                            if (lane == 0 && has_box) mbar_arrive(bar_u_empty + 8 * my.slot);
                        }
                        if (lane == 0 && (warp == 0 || warp == 12)) PAIR_TRACE(k, ps, j, 18 + (warp == 12) * 4);
                        for (int i = 0; i < nbox; ++i) ur.next(kUSlots);
                        acc.next(kPairAcc);
                    }
                }
                // combine the four chunk warps of each row, one atomic per row and CTA, block
                // by block
#pragma unroll
                for (int bi = 0; bi < kSpMax; ++bi) {
                    if (bi >= nb) break;
                    const int ps = kSpMax * sp + bi;
                    const int b_row = ps * kPairRows + static_cast<int>(rank) * kRows + row;
                    sh.part_key[c][row] = argmax_key(best[bi].s, best[bi].v);
                    sh.part_logit[c][row] = best[bi].l;
                    epi_sync512();
                    if (c == 0) {
                        unsigned long long kb = sh.part_key[0][row];
                        float lb = sh.part_logit[0][row];
#pragma unroll
                        for (int i = 1; i < kChunks; ++i) {
                            const unsigned long long ki = sh.part_key[i][row];
                            if (ki > kb) {
                                kb = ki;
                                lb = sh.part_logit[i][row];
                            }
                        }
                        sh.cta_key[ps][row] = kb;
                        sh.cta_logit[ps][row] = lb;
                        if (ok && b_row < p.B)
                            atomicMax(&p.slots[static_cast<size_t>(k - 1) * p.B + b_row], kb);
                    }
                    epi_sync512();
                }
                // the blocks that reuse this super-pass's A buffers (blocks 0 and 1 went in at
                // the position's start), once its MMAs have released them
                for (int ps = kSpMax * sp + 2; ps < kSpMax * sp + kSpMax + 2 && ps < npass; ++ps)
                    if (ok) gather(k, ps);
            }

            // ---- grid barrier: every CTA has combined its rows of position k
            if (!grid_sync(static_cast<uint32_t>(k))) ok = false;
            // ---- x_k of this CTA's rows: the next gather's tokens; the owner writes the outputs
            if (ok) {
                for (int i = et; i < npass * kRows; i += kEpiThreads) {
                    const int ps = i / kRows, r = i % kRows;
                    const int b = ps * kPairRows + static_cast<int>(rank) * kRows + r;
                    if (b >= p.B) continue;
                    const size_t o = static_cast<size_t>(k - 1) * p.B + b;
                    const unsigned long long key = __ldcg(&p.slots[o]);
                    const int tok = static_cast<int>(argmax_key_index(key));
                    sh.tok[ps][r] = checked_token(tok, p.V);
                    if (key == sh.cta_key[ps][r]) {
                        p.x_out[static_cast<size_t>(b) * p.gamma + (k - 1)] = tok;
                        p.logit_out[static_cast<size_t>(b) * p.gamma + (k - 1)] = sh.cta_logit[ps][r];
                    }
                }
            }
            epi_sync512();
        }
        // the last pair commit on aempty may still be arriving on this CTA's barrier
        if (ok) {
            for (int b = 0; b < kABufs; ++b) {
                // uses over the launch: the count before block b of a position past the last
                const uint32_t uses = kSpMax == 2 ? (b < npass ? abuf_uses(p.gamma + 1, b, npass) : 0u)
                                                  : static_cast<uint32_t>((p.gamma * npass + 1 - b) / 2);
                if (uses > 0) wait_drain(bar_aempty + 8 * b, (uses - 1) & 1u, p);
            }
        }
    }

    __syncwarp();
    tc_fence_before();
    cluster_sync();                  // no cross-CTA signal is in flight past this point
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, kTmemCols);
    }
}

}  // namespace pairk
}  // namespace draft
}  // namespace dspark
