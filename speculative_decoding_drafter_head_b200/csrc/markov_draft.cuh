// markov_draft.cuh -- the sequential head of DSpark (Markov or RNN) on tcgen05 tensor cores.
//
// gdymind.com, "DSpark: DeepSeek's new speculative decoding work", section 4
// ("Sequential stage", "Markov head"): position k adds a first-order transition
// bias B(x_{k-1}, .) = W1[x_{k-1}] W2 (rank r = 256) to the backbone's base logits
// U_k and picks x_k from them.  The same section names an RNN head, a recurrent state
// over the block's prefix; with kRnn the bias is bf16(s_k) W2 instead, where
// s_k = tanh(W1[x_{k-1}] + s_{k-1} Whh) (our reading; the pages give no equations).
//
// One persistent cooperative kernel runs all gamma positions.  Each CTA owns a
// contiguous slice of the vocabulary (a whole number of 32-column units, balanced
// over the grid) cut into tiles of 128 columns, and for every position k and every
// block of M requests it computes
//     D[b, v] = sum_j A[b, j] W2[j, v],   A[b, :] = W1[x_{k-1, b}, :]  (or bf16(s_k[b, :]))
// as tcgen05.mma M=64/128, N<=128, K=16 (bf16 in, fp32 accumulate in TMEM), with W2
// streamed by TMA in two K-halves of 128 rows (MN-major, 128-byte swizzle).  A single
// MMA instruction costs the same for any N up to 128 and for M = 64 or 128, so tiles
// are 128 columns wide and a CTA's remainder becomes one narrower tile.  The epilogue
// adds U_k (staged by TMA), applies greedy or Gumbel-max selection and keeps a running
// (max, index) per request row, so the [B, V] logits never reach memory.  Rows are
// combined across CTAs by a 64-bit atomicMax on (ordered value, inverted index); a
// bounded grid barrier ends each position, after which every CTA reads x_k for the
// next gather and the CTA that owns the winning column writes the outputs.  The RNN
// instance adds, before each gather, the state update of the CTA's rows and a second
// grid barrier that publishes them.
//
// W2 is read with an L2 evict-last policy and U with evict-first: within one launch
// W2 (at most 134 MB) is re-read every position and mostly stays in L2.
//
// Warp roles (352 threads): warps 0-7 epilogue and A gather (warps q and q + 4 read
// TMEM lane quadrant q and take alternate 64-column boxes of each tile), warp 8 W2
// producer, warp 9 U producer, warp 10 MMA issuer and TMEM owner; with the confidence
// head fused in (kConf, 384 threads) warp 11 computes c and P beside the drafting, and
// with kTail the epilogue warps run the prefix scheduler and the verification after the
// last position (the scheduler and verify kernels' device code).  With B <= 64 the MMA
// uses M = 64 (rows 16q..16q+15 sit in TMEM lanes 32q..32q+15, read with 16x256b loads),
// else M = 128 (32x32b loads).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "ptx.cuh"
#include "schedule_prefix.cuh"
#include "verify_prefix.cuh"

namespace dspark {
namespace draft {

constexpr int kUnit = 32;                         // columns per epilogue chunk
constexpr int kUBoxCols = 64;                     // columns per U TMA box (two chunks)
constexpr int kMaxUnits = 4;                      // 128 columns per MMA tile
constexpr int kRank = 256;                        // r, the contraction length
constexpr int kKSlice = 128;                      // W2 rows per ring stage
constexpr int kKSlices = kRank / kKSlice;         // 2
constexpr int kMaxW2Stages = 5;
constexpr int kW2BoxBytes = 64 * kKSlice * 2;     // one TMA box: 64 columns x 128 rows (16 KB)
constexpr int kW2StageBytes = 2 * kW2BoxBytes;    // 32 KB: 128 columns x 128 rows
constexpr int kUMaxSlots = 16;
constexpr int kAcc = 4;                           // TMEM accumulators of 128 columns
constexpr int kAccCols = 128;
constexpr uint32_t kTmemCols = 512;
// A (M x 256 bf16) + W2 ring + U ring in 224 KB (+ alignment slack)
constexpr int kRingSmem = 224 * 1024;
constexpr int kDynSmem = kRingSmem + 1024;
constexpr int kEpiWarps = 8;                      // two per TMEM lane quadrant
constexpr int kThreads = (kEpiWarps + 3) * 32;    // + W2 producer, U producer, MMA issuer
constexpr int kWarpW2 = kEpiWarps, kWarpU = kEpiWarps + 1, kWarpMma = kEpiWarps + 2;
constexpr int kWarpConf = kEpiWarps + 3;          // confidence head (fused instances only)
constexpr int kThreadsConf = kThreads + 32;
constexpr int kMaxB = 1024;
constexpr int kMaxMTiles = kMaxB / 64;
constexpr float kGumbelMax = 17.0f;               // above any noise value the epilogue makes
constexpr uint32_t kWaitHintNs = 20000;           // longest hardware suspension per try_wait

struct Params {
    const int32_t *anchor;
    const uint16_t *W1;
    int B, gamma, V, mode;
    float inv_tau;
    uint32_t seed_lo, seed_hi;
    uint32_t rk0[10], rk1[10];   // Philox round keys: (seed_lo + r W0, seed_hi + r W1), r = 0..9
    int b_offset;
    int32_t *x_out;
    float *logit_out;
    unsigned long long *slots;   // [gamma][B] argmax keys, zeroed before launch
    unsigned int *barrier;       // grid barrier arrival counter, zeroed before launch
    unsigned int *abort_flag;    // set by any CTA that gives up, zeroed before launch
    int units_total;             // ceil(V / 32)
    int M;                       // requests per MMA tile: 64 (B <= 64) or 128
    int w2_stages;               // W2 ring depth
    int w2_stage_bytes;          // one K half of a tile: tile_units / 2 boxes of 16 KB
    int tile_units;              // 32-column units per MMA tile (N = 32 tile_units)
    int acc_cols;                // TMEM columns of one accumulator (32 tile_units)
    int acc_slots;               // accumulators in TMEM (512 / acc_cols, at most kAcc)
    int ub;                      // rows of the U TMA box: min(B, M)
    int u_slots;                 // U ring depth (boxes of 64 columns)
    int u_slot_bytes;
    unsigned long long timeout_ns;
    int barrier_extra;
    // RNN head (Whh != nullptr): s_k = tanh(W1[x_{k-1}] + s_{k-1} Whh), A_k = bf16(s_k)
    const uint16_t *Whh;         // [r][r] bf16
    float *state;                // [B][r] fp32, s_{k-1} then s_k (workspace)
    uint16_t *a_rows;            // [B][r] bf16 copy of s_k, the rows the gather reads
    // confidence head fused in (kConf): z = w . [h_k ; W1[x_{k-1}]] + b_conf,
    // c = sigmoid(z / T_k), P_k = P_{k-1} c
    const uint16_t *h;           // [B][gamma][d] bf16
    const uint16_t *wconf;       // [d + r] bf16
    float b_conf;
    const float *T;              // [gamma]
    int d;
    float *c_out, *P_out;        // [B][gamma]
    float *zh;                   // [B][gamma] workspace: the hidden-state part of z
    unsigned int *zh_done;       // workspace counter: CTAs whose zh share is written
    unsigned int *conf_done;     // workspace counter: CTAs whose confidence warp is done
    // scheduler and verification in the same launch (kTail): the global top-N over all
    // B gamma survival scores and the scan over N, then strict prefix-match verification
    const double *Tstep;         // [B (gamma + 1) + 1] step time for n verified tokens
    const int32_t *target;       // [B][gamma + 1]
    int32_t *L_out, *N_out;      // [B], [1]
    double *objective_out;       // [1]
    int32_t *accepted_out, *bonus_out;   // [B]
    int32_t *rank;               // [B gamma] workspace
    unsigned int *tail_done;     // workspace counter: CTAs whose ranks are written
};

struct Ctl {
    unsigned long long w2_full[kMaxW2Stages];
    unsigned long long w2_empty[kMaxW2Stages];
    unsigned long long u_full[kUMaxSlots];
    unsigned long long u_empty[kUMaxSlots];
    unsigned long long tfull[kAcc];
    unsigned long long tempty[kAcc];
    unsigned long long afull, aempty, drain;
    uint32_t tmem_base;
    int abort;
    int go;          // verdict of the last grid barrier, shared by all epilogue threads
};

// A ring position: slot index and the parity of its current use.
struct Ring {
    int slot = 0;
    uint32_t phase = 0;
    __device__ __forceinline__ void next(int n)
    {
        if (++slot == n) {
            slot = 0;
            phase ^= 1u;
        }
    }
};

// The t-th tile of a CTA that owns n_units units, in tiles of `units` units: full tiles,
// then the remainder.
__device__ __forceinline__ void tile_span_n(int t, int n_units, int units, int &first, int &count)
{
    first = t * units;
    count = min(units, n_units - first);
}

// The t-th tile of a CTA that owns n_units units: full tiles of kMaxUnits units, then
// the remainder (an MMA costs the same for any N <= 128, so this minimises the count).
__device__ __forceinline__ void tile_span(int t, int n_units, int ntiles, int &first, int &count)
{
    (void)ntiles;
    first = t * kMaxUnits;
    count = min(kMaxUnits, n_units - first);
}

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
    for (;;) {
        if (mbar_try_wait_sleep(bar, parity, kWaitHintNs)) return true;
        if (*reinterpret_cast<volatile int *>(&ctl.abort)) return false;
        if (globaltimer_ns() - t0 > p.timeout_ns) {
            give_up(ctl, p, DSPARK_TIMEOUT);
            return false;
        }
    }
}

// Bounded wait used while draining: ignores the abort flag, only the time limit.
__device__ __forceinline__ void wait_drain(uint32_t bar, uint32_t parity, const Params &p)
{
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait_sleep(bar, parity, kWaitHintNs)) {
        if (globaltimer_ns() - t0 > p.timeout_ns) {
            record_error(DSPARK_TIMEOUT);
            return;
        }
    }
}

// Wait for the last use of every slot of a ring of n slots after `issued` uses in total.
__device__ __forceinline__ void drain_ring(uint32_t bar0, int n, long long issued, const Params &p)
{
    for (int s = 0; s < n; ++s) {
        const long long uses = issued / n + (s < issued % n ? 1 : 0);
        if (uses > 0) wait_drain(bar0 + 8 * s, static_cast<uint32_t>((uses - 1) & 1), p);
    }
}

__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

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

__device__ __forceinline__ void sts128_zero(uint32_t addr)
{
    asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(addr), "r"(0) : "memory");
}

__device__ __forceinline__ int checked_token(int tok, int V)
{
    if (tok < 0 || tok >= V) {
        record_error(DSPARK_INVALID_TOKEN);
        return 0;
    }
    return tok;
}

// Running best of one request row over one 32-column chunk: l = acc + U, greedy or
// Gumbel-max score s, strict improvement keeps the smallest column on ties.
struct RowBest {
    float s = -INFINITY;
    float l = 0.0f;
    uint32_t v = 0xFFFFFFFFu;
};

__device__ __forceinline__ float fmax3(float a, float b, float c)
{
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Largest of 32 values with three-input max (17 instructions instead of 31).
__device__ __forceinline__ float max32(const float (&s)[32])
{
    float m[11];
#pragma unroll
    for (int i = 0; i < 10; ++i) m[i] = fmax3(s[3 * i], s[3 * i + 1], s[3 * i + 2]);
    m[10] = fmaxf(s[30], s[31]);
    const float a = fmax3(m[0], m[1], m[2]), b = fmax3(m[3], m[4], m[5]);
    const float c = fmax3(m[6], m[7], m[8]), d = fmaxf(m[9], m[10]);
    return fmaxf(fmax3(a, b, c), d);
}

__device__ __forceinline__ void lds128(uint32_t addr, uint32_t &a, uint32_t &b, uint32_t &c,
                                       uint32_t &d)
{
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(a), "=r"(b), "=r"(c), "=r"(d)
                 : "r"(addr));
}

// l = acc + U for 32 columns: the U row sits in a 64-column box in shared memory
// (128-byte rows, 128-byte swizzle) and these are its columns 32 h .. 32 h + 31.
__device__ __forceinline__ void add_u32(float (&l)[32], const uint32_t (&a)[32], uint32_t sU,
                                        int row, int h)
{
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        uint32_t w0, w1, w2, w3;
        lds128(sU + row * 128 + (((4 * h + u) ^ (row & 7)) << 4), w0, w1, w2, w3);
        add_f32x2(l[8 * u + 0], l[8 * u + 1], __uint_as_float(a[8 * u + 0]),
                  __uint_as_float(a[8 * u + 1]), bf16lo_to_f32(w0), bf16hi_to_f32(w0));
        add_f32x2(l[8 * u + 2], l[8 * u + 3], __uint_as_float(a[8 * u + 2]),
                  __uint_as_float(a[8 * u + 3]), bf16lo_to_f32(w1), bf16hi_to_f32(w1));
        add_f32x2(l[8 * u + 4], l[8 * u + 5], __uint_as_float(a[8 * u + 4]),
                  __uint_as_float(a[8 * u + 5]), bf16lo_to_f32(w2), bf16hi_to_f32(w2));
        add_f32x2(l[8 * u + 6], l[8 * u + 7], __uint_as_float(a[8 * u + 6]),
                  __uint_as_float(a[8 * u + 7]), bf16lo_to_f32(w3), bf16hi_to_f32(w3));
    }
}

// Scores of 32 logits starting at column v0: the logits themselves (greedy) or
// l / tau + Gumbel noise; columns at or beyond V get -inf.
__device__ __forceinline__ void scores32(float (&s)[32], float (&l)[32], int v0, const Params &p,
                                         int k, int b_glob, float best_s)
{
    if (v0 + kUnit > p.V) {
#pragma unroll
        for (int i = 0; i < 32; ++i)
            if (v0 + i >= p.V) l[i] = -INFINITY;
    }
    if (p.mode == 0) {
#pragma unroll
        for (int i = 0; i < 32; ++i) s[i] = l[i];
        return;
    }
    // exact pruning, one warp vote per chunk: skip the noise only when no lane's chunk can
    // beat its running best even with the largest noise value; otherwise the eight Philox
    // blocks run without branches so that their round chains interleave
    const bool skip = !(fmaf(max32(l), p.inv_tau, kGumbelMax) >= best_s);
    if (__all_sync(0xFFFFFFFFu, skip)) {
#pragma unroll
        for (int i = 0; i < 32; ++i) s[i] = -INFINITY;
        return;
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const uint4 w = philox(make_uint4(static_cast<uint32_t>(v0 / 4 + q),
                                          static_cast<uint32_t>(k - 1),
                                          static_cast<uint32_t>(b_glob), 0u),
                               p.seed_lo, p.seed_hi);
        s[4 * q + 0] = fmaf(l[4 * q + 0], p.inv_tau, gumbel_from_word(w.x));
        s[4 * q + 1] = fmaf(l[4 * q + 1], p.inv_tau, gumbel_from_word(w.y));
        s[4 * q + 2] = fmaf(l[4 * q + 2], p.inv_tau, gumbel_from_word(w.z));
        s[4 * q + 3] = fmaf(l[4 * q + 3], p.inv_tau, gumbel_from_word(w.w));
    }
}

// First index of the largest of 32 scores (the caller knows the largest is mx).
__device__ __forceinline__ int first_index(const float (&s)[32], float mx)
{
    int idx = 31;
#pragma unroll
    for (int i = 31; i >= 0; --i)
        if (s[i] == mx) idx = i;
    return idx;
}

__device__ __forceinline__ float pick(const float (&l)[32], int idx)
{
    float li = l[0];
#pragma unroll
    for (int i = 1; i < 32; ++i)
        if (i == idx) li = l[i];
    return li;
}

// Running best of one request row over one 64-column U box: chunk 0 holds columns
// v0 .. v0 + 31 and, when `two`, chunk 1 holds v0 + 32 .. v0 + 63.  The two 32-column
// chains are independent until one compare against the running best, which keeps the
// smallest column on ties.
__device__ __forceinline__ void box_update(RowBest &best, const uint32_t (&a0)[32],
                                           const uint32_t (&a1)[32], bool two, uint32_t sU,
                                           int row, int v0, const Params &p, int k, int b_glob)
{
    float l0[32], l1[32], s0[32], s1[32];
    add_u32(l0, a0, sU, row, 0);
    add_u32(l1, a1, sU, row, 1);
    scores32(s0, l0, v0, p, k, b_glob, best.s);
    scores32(s1, l1, v0 + kUnit, p, k, b_glob, best.s);
    const float m0 = max32(s0);
    const float m1 = two ? max32(s1) : -INFINITY;
    const float mx = fmaxf(m0, m1);
    if (mx > best.s) {
        if (m0 == mx) {
            const int idx = first_index(s0, mx);
            best.v = static_cast<uint32_t>(v0 + idx);
            best.l = p.mode == 0 ? mx : pick(l0, idx);     // greedy: the score is the logit
        } else {
            const int idx = first_index(s1, mx);
            best.v = static_cast<uint32_t>(v0 + kUnit + idx);
            best.l = p.mode == 0 ? mx : pick(l1, idx);
        }
        best.s = mx;
    }
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr)
{
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

// M = 64 (rows 16q..16q+15 of the tile in TMEM lanes 32q..32q+15): one 64-column box
// read with 16x256b loads, so all 32 lanes work.  Thread t holds rows ra = t/4 and
// rb = t/4 + 8 of the quadrant and, of the box, columns 8i + 2(t%4) + e (i = 0..7,
// e = 0, 1): a[4i + e] is row ra, a[4i + 2 + e] row rb.  Each thread keeps a running
// best per row over its own columns; the four threads of a row are combined by the
// caller.  `two` is false when the box's second 32 columns lie outside the tile.
__device__ __forceinline__ void box_update_m64(RowBest (&best)[2], const uint32_t (&a)[32],
                                               bool two, uint32_t sU, int ua, int ub, int v0,
                                               const Params &p, int k, int bg_a, int bg_b)
{
    const int w = threadIdx.x & 3;
    float l[32], s[32];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint32_t wa = lds32(sU + ua * 128 + ((i ^ (ua & 7)) << 4) + w * 4);
        const uint32_t wb = lds32(sU + ub * 128 + ((i ^ (ub & 7)) << 4) + w * 4);
        add_f32x2(l[4 * i + 0], l[4 * i + 1], __uint_as_float(a[4 * i + 0]),
                  __uint_as_float(a[4 * i + 1]), bf16lo_to_f32(wa), bf16hi_to_f32(wa));
        add_f32x2(l[4 * i + 2], l[4 * i + 3], __uint_as_float(a[4 * i + 2]),
                  __uint_as_float(a[4 * i + 3]), bf16lo_to_f32(wb), bf16hi_to_f32(wb));
    }
    const int vw = v0 + 2 * w;                    // column of a[0]
    if (!two || v0 + 2 * kUnit > p.V) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int e = 0; e < 2; ++e)
                if ((!two && i >= 4) || vw + 8 * i + e >= p.V) {
                    l[4 * i + e] = -INFINITY;
                    l[4 * i + 2 + e] = -INFINITY;
                }
    }
    if (p.mode == 0) {
#pragma unroll
        for (int j = 0; j < 32; ++j) s[j] = l[j];
    } else {
        // one vote per box: skip the noise only when no thread's columns can beat its row's
        // running best even with the largest noise value
        float lm0 = -INFINITY, lm1 = -INFINITY;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            lm0 = fmax3(lm0, l[4 * i + 0], l[4 * i + 1]);
            lm1 = fmax3(lm1, l[4 * i + 2], l[4 * i + 3]);
        }
        const bool skip = !(fmaf(lm0, p.inv_tau, kGumbelMax) >= best[0].s) &&
                          !(fmaf(lm1, p.inv_tau, kGumbelMax) >= best[1].s);
        if (__all_sync(0xFFFFFFFFu, skip)) {
#pragma unroll
            for (int j = 0; j < 32; ++j) s[j] = -INFINITY;
        } else {
            // columns 8i + 2w + {0,1} are words 2(w&1) + {0,1} of Philox block 2i + (w>>1);
            // threads w and w^1 need the same block for both rows, so each computes it for
            // one row (w&1 ? rb : ra) and passes the other thread its two words
            const int own_b = (w & 1) ? bg_b : bg_a;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint4 g = philox(make_uint4(static_cast<uint32_t>((v0 >> 2) + 2 * i + (w >> 1)),
                                                  static_cast<uint32_t>(k - 1),
                                                  static_cast<uint32_t>(own_b), 0u),
                                       p.seed_lo, p.seed_hi);
                const uint32_t send0 = (w & 1) ? g.x : g.z, send1 = (w & 1) ? g.y : g.w;
                const uint32_t recv0 = __shfl_xor_sync(0xFFFFFFFFu, send0, 1);
                const uint32_t recv1 = __shfl_xor_sync(0xFFFFFFFFu, send1, 1);
                // row ra: own words when w is even, else the neighbour's; row rb the reverse
                const uint32_t a0 = (w & 1) ? recv0 : g.x, a1 = (w & 1) ? recv1 : g.y;
                const uint32_t b0 = (w & 1) ? g.z : recv0, b1 = (w & 1) ? g.w : recv1;
                s[4 * i + 0] = fmaf(l[4 * i + 0], p.inv_tau, gumbel_from_word(a0));
                s[4 * i + 1] = fmaf(l[4 * i + 1], p.inv_tau, gumbel_from_word(a1));
                s[4 * i + 2] = fmaf(l[4 * i + 2], p.inv_tau, gumbel_from_word(b0));
                s[4 * i + 3] = fmaf(l[4 * i + 3], p.inv_tau, gumbel_from_word(b1));
            }
        }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        float m4[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            m4[i] = fmaxf(fmax3(s[8 * i + 2 * h], s[8 * i + 2 * h + 1], s[8 * i + 4 + 2 * h]),
                          s[8 * i + 4 + 2 * h + 1]);
        const float mx = fmaxf(fmax3(m4[0], m4[1], m4[2]), m4[3]);
        if (mx > best[h].s) {
            int idx = 31;
#pragma unroll
            for (int i = 7; i >= 0; --i)
#pragma unroll
                for (int e = 1; e >= 0; --e)
                    if (s[4 * i + 2 * h + e] == mx) idx = 4 * i + 2 * h + e;
            float li = mx;                      // greedy: the score is the logit
            if (p.mode != 0) {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (j == idx) li = l[j];
            }
            best[h].v = static_cast<uint32_t>(vw + 8 * (idx >> 2) + (idx & 1));
            best[h].l = li;
            best[h].s = mx;
        }
    }
}

// 8 bf16 products of two 16-byte vectors added to acc (low half, then high half, of each
// 32-bit word).
__device__ __forceinline__ float dot8(const uint4 a, const uint4 b, float acc)
{
    acc = fmaf(bf16lo_to_f32(a.x), bf16lo_to_f32(b.x), acc);
    acc = fmaf(bf16hi_to_f32(a.x), bf16hi_to_f32(b.x), acc);
    acc = fmaf(bf16lo_to_f32(a.y), bf16lo_to_f32(b.y), acc);
    acc = fmaf(bf16hi_to_f32(a.y), bf16hi_to_f32(b.y), acc);
    acc = fmaf(bf16lo_to_f32(a.z), bf16lo_to_f32(b.z), acc);
    acc = fmaf(bf16hi_to_f32(a.z), bf16hi_to_f32(b.z), acc);
    acc = fmaf(bf16lo_to_f32(a.w), bf16lo_to_f32(b.w), acc);
    acc = fmaf(bf16hi_to_f32(a.w), bf16hi_to_f32(b.w), acc);
    return acc;
}

// Bounded wait of one thread until *ctr >= target (acquire); false on abort or time-out.
__device__ __forceinline__ bool wait_counter(const unsigned int *ctr, uint32_t target,
                                             const Params &p)
{
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire_u32(ctr) < target) {
        if (*reinterpret_cast<volatile unsigned int *>(p.abort_flag)) return false;
        if (globaltimer_ns() - t0 > p.timeout_ns) {
            record_error(DSPARK_TIMEOUT);
            atomicExch(p.abort_flag, 1u);
            return false;
        }
        __nanosleep(200);
    }
    return true;
}

// The confidence head, fused (gdymind.com "DSpark", section 5: a linear projection of the
// backbone hidden state at position k and of the Markov embedding of the previous draft
// token, a sigmoid, sequential temperature scaling, and the cumulative product of the
// calibrated scores).  One warp of every CTA:
//   1. z_h[b, k] = sum_i w[i] h[b, k-1, i] for the pairs n = b gamma + k - 1 with
//      n = blockIdx.x (mod G), published with a release-add on a workspace counter;
//   2. for k = 1..gamma, once the grid barrier of position k - 1 has passed (x_{k-1} is
//      final): for the requests b = blockIdx.x (mod G), z = z_h + w[d..] . W1[x_{k-1}]
//      + b_conf, c_k = 1 / (1 + exp(-z / T_k)), P_k = P_{k-1} c_k in fp32, k order.
// It waits only on the grid barrier's counter, so it runs beside the drafting, off its
// critical path.
__device__ __forceinline__ void confidence_warp(const Params &p, int G)
{
    const int lane = threadIdx.x & 31;
    const int n_pairs = p.B * p.gamma;
    const int dv = p.d >> 3;                                    // 16-byte vectors of h
    const uint4 *wv = reinterpret_cast<const uint4 *>(p.wconf);
    for (int n = blockIdx.x; n < n_pairs; n += G) {
        const uint4 *hk = reinterpret_cast<const uint4 *>(p.h + static_cast<size_t>(n) * p.d);
        float a0 = 0.f, a1 = 0.f;
        int i = lane;
        for (; i + 32 < dv; i += 64) {                          // two vectors in flight per lane
            const uint4 h0 = __ldcs(hk + i), h1 = __ldcs(hk + i + 32);
            a0 = dot8(h0, __ldg(wv + i), a0);
            a1 = dot8(h1, __ldg(wv + i + 32), a1);
        }
        if (i < dv) a0 = dot8(__ldcs(hk + i), __ldg(wv + i), a0);
        const float z = warp_sum(a0 + a1);
        if (lane == 0) p.zh[n] = z;
    }
    __syncwarp();
    if (lane == 0) red_release_add_u32(p.zh_done, 1u);
    bool ok = true;
    if (lane == 0) ok = wait_counter(p.zh_done, static_cast<uint32_t>(G), p);
    ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
    const uint4 *wr = wv + dv;                                  // the W1-row part of w
    const int rv = kRank >> 3;                                  // 32 vectors: one per lane
    for (int k = 1; k <= p.gamma && ok; ++k) {
        if (k >= 2 && lane == 0)                                // x_{k-1} final after barrier k-1
            ok = wait_counter(p.barrier, static_cast<uint32_t>(k - 1) * static_cast<uint32_t>(G), p);
        ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
        if (!ok) break;
        const float Tk = __ldg(p.T + (k - 1));
        for (int b = blockIdx.x; b < p.B; b += G) {
            int tok = k == 1 ? __ldg(p.anchor + b)
                             : static_cast<int>(argmax_key_index(
                                   __ldcg(&p.slots[static_cast<size_t>(k - 2) * p.B + b])));
            if (tok < 0 || tok >= p.V) {
                if (lane == 0) record_error(DSPARK_INVALID_TOKEN);
                tok = 0;
            }
            const uint4 *e = reinterpret_cast<const uint4 *>(p.W1 + static_cast<size_t>(tok) * kRank);
            float zr = lane < rv ? dot8(__ldg(e + lane), __ldg(wr + lane), 0.f) : 0.f;
            zr = warp_sum(zr);
            if (lane == 0) {
                const size_t o = static_cast<size_t>(b) * p.gamma + (k - 1);
                const float z = __ldcg(p.zh + o) + zr + p.b_conf;
                const float c = 1.0f / (1.0f + expf(-z / Tk));
                const float P = k == 1 ? c : __fmul_rn(p.P_out[o - 1], c);
                p.c_out[o] = c;
                p.P_out[o] = P;
            }
        }
    }
    // with the scheduler in the launch, it starts once every CTA's scores are written
    // (also after a failure: the waiter then sees the abort flag)
    __syncwarp();
    if (p.conf_done && lane == 0) red_release_add_u32(p.conf_done, 1u);
}

// kM is the MMA's M (64 when B <= 64, else 128); p.M equals it.  kRnn selects the RNN
// head (p.Whh set); the Markov instances carry none of its code.  kConf adds the
// confidence warp (Markov head only), kTail (with kConf) the scheduler and the
// verification after the last position.
template <int kM, bool kRnn, bool kConf = false, bool kTail = false>
__global__ void __launch_bounds__(kConf ? kThreadsConf : kThreads, 1)
    markov_draft_kernel(const __grid_constant__ CUtensorMap tm_w2,
                        const __grid_constant__ CUtensorMap tm_u, const Params p)
{
    extern __shared__ uint8_t dyn_smem[];
    __shared__ Ctl ctl;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    constexpr int M = kM;
    const int a_chunk = M * 128;                  // one 64-column K chunk of A
    const uint32_t base = (smem_u32(dyn_smem) + 1023u) & ~1023u;
    const uint32_t sA = base;
    const uint32_t sW2 = base + static_cast<uint32_t>(M * kRank * 2);
    const uint32_t sU = sW2 + static_cast<uint32_t>(p.w2_stages * p.w2_stage_bytes);

    const int G = gridDim.x;
    const int u_begin = static_cast<int>(static_cast<long long>(blockIdx.x) * p.units_total / G);
    const int u_end =
        static_cast<int>(static_cast<long long>(blockIdx.x + 1) * p.units_total / G);
    const int n_units = u_end - u_begin;
    const int ntiles = (n_units + p.tile_units - 1) / p.tile_units;
    const int num_mt = (p.B + M - 1) / M;

    const uint32_t bar_w2_full = smem_u32(&ctl.w2_full[0]);
    const uint32_t bar_w2_empty = smem_u32(&ctl.w2_empty[0]);
    const uint32_t bar_u_full = smem_u32(&ctl.u_full[0]);
    const uint32_t bar_u_empty = smem_u32(&ctl.u_empty[0]);
    const uint32_t bar_tfull = smem_u32(&ctl.tfull[0]);
    const uint32_t bar_tempty = smem_u32(&ctl.tempty[0]);
    const uint32_t bar_afull = smem_u32(&ctl.afull);
    const uint32_t bar_aempty = smem_u32(&ctl.aempty);
    const uint32_t bar_drain = smem_u32(&ctl.drain);

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.w2_stages; ++s) {
            mbar_init(bar_w2_full + 8 * s, 1);
            mbar_init(bar_w2_empty + 8 * s, 1);
        }
        for (int s = 0; s < p.u_slots; ++s) {
            mbar_init(bar_u_full + 8 * s, 1);
            mbar_init(bar_u_empty + 8 * s, kEpiWarps / 2);
        }
        for (int a = 0; a < kAcc; ++a) {
            mbar_init(bar_tfull + 8 * a, 1);
            mbar_init(bar_tempty + 8 * a, kEpiWarps);
        }
        mbar_init(bar_afull, kEpiWarps);
        mbar_init(bar_aempty, 1);
        mbar_init(bar_drain, 1);
        ctl.abort = 0;
        mbar_fence_init();
    }
    if (warp == kWarpMma) {
        tmem_alloc(smem_u32(&ctl.tmem_base), kTmemCols);
        tmem_relinquish();
    }
    if (warp == kWarpW2 && lane == 0) {
        tma_prefetch_desc(&tm_w2);
        tma_prefetch_desc(&tm_u);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl.tmem_base;

    if (warp == kWarpW2) {
        // ------------------------------------------------------------ W2 producer
        if (lane == 0) {
            const uint64_t pol_w2 = l2_policy_evict_last();
            Ring w2;
            long long issued = 0;
            bool ok = true;
            for (int k = 1; k <= p.gamma && ok; ++k) {
                for (int mt = 0; mt < num_mt && ok; ++mt) {
                    for (int t = 0; t < ntiles && ok; ++t) {
                        int first, count;
                        tile_span_n(t, n_units, p.tile_units, first, count);
                        const int v0 = (u_begin + first) * kUnit;
                        const int nbox = (count + 1) >> 1;          // 64-column boxes
                        if (mt == 0 && t == 0) DSPARK_TRACE_AT(k, 7);
                        if (mt == num_mt - 1 && t == ntiles - 1) DSPARK_TRACE_AT(k, 8);
                        for (int ks = 0; ks < kKSlices; ++ks) {
                            if (!wait_phase(bar_w2_empty + 8 * w2.slot, w2.phase ^ 1u, ctl, p)) {
                                ok = false;
                                break;
                            }
                            const uint32_t bar = bar_w2_full + 8 * w2.slot;
                            const uint32_t dst = sW2 + w2.slot * p.w2_stage_bytes;
                            mbar_arrive_expect_tx(bar, nbox * kW2BoxBytes);
                            for (int i = 0; i < nbox; ++i)
                                tma_load_2d(dst + i * kW2BoxBytes, &tm_w2, bar, v0 + 64 * i,
                                            ks * kKSlice, pol_w2);
                            ++issued;
                            w2.next(p.w2_stages);
                        }
                    }
                }
            }
            drain_ring(bar_w2_full, p.w2_stages, issued, p);   // copies must land before exit
        }
    } else if (warp == kWarpU) {
        // ------------------------------------------------------------ U producer
        if (lane == 0) {
            const uint64_t pol_u = l2_policy_evict_first();
            const uint32_t u_tx = static_cast<uint32_t>(p.ub) * kUBoxCols * 2;
            Ring ur;
            long long issued = 0;
            bool ok = true;
            for (int k = 1; k <= p.gamma && ok; ++k) {
                for (int mt = 0; mt < num_mt && ok; ++mt) {
                    for (int t = 0; t < ntiles && ok; ++t) {
                        int first, count;
                        tile_span_n(t, n_units, p.tile_units, first, count);
                        const int v0 = (u_begin + first) * kUnit;
                        for (int u = 0; u < count; u += 2) {
                            if (!wait_phase(bar_u_empty + 8 * ur.slot, ur.phase ^ 1u, ctl, p)) {
                                ok = false;
                                break;
                            }
                            const uint32_t bar = bar_u_full + 8 * ur.slot;
                            if (mt == 0 && t == 0 && u == 0) DSPARK_TRACE_AT(k, 11);
                            if (mt == num_mt - 1 && t == ntiles - 1 && u + 2 >= count) DSPARK_TRACE_AT(k, 12);
                            mbar_arrive_expect_tx(bar, u_tx);
                            tma_load_3d(sU + ur.slot * p.u_slot_bytes, &tm_u, bar, v0 + u * kUnit,
                                        k - 1, mt * M, pol_u);

                            ++issued;
                            ur.next(p.u_slots);
                        }
                    }
                }
            }
            drain_ring(bar_u_full, p.u_slots, issued, p);
        }
    } else if (warp == kWarpMma) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            Ring w2, acc;
            const uint64_t a_desc0 = smem_desc(sA, 1024, 1024, kSwizzle128B);
            const uint64_t b_desc0 = smem_desc(sW2, kW2BoxBytes, 1024, kSwizzle128B);
            uint32_t mt_count = 0;
            bool issued_any = false;
            bool ok = true;
            for (int k = 1; k <= p.gamma && ok; ++k) {
                for (int mt = 0; mt < num_mt && ok; ++mt) {
                    if (!wait_phase(bar_afull, mt_count & 1u, ctl, p)) {
                        ok = false;
                        break;
                    }
                    if (mt == 0) DSPARK_TRACE_AT(k, 16);
                    tc_fence_after();
                    for (int t = 0; t < ntiles && ok; ++t) {
                        int first, count;
                        tile_span_n(t, n_units, p.tile_units, first, count);
                        const uint32_t idesc = idesc_bf16_f32(static_cast<uint32_t>(M),
                                                              static_cast<uint32_t>(count * kUnit), 1);
#ifdef DSPARK_TRACE
                        const uint64_t tw0 = globaltimer_ns();
#endif
                        if (!wait_phase(bar_tempty + 8 * acc.slot, acc.phase ^ 1u, ctl, p)) {
                            ok = false;
                            break;
                        }
                        DSPARK_TRACE_ADD(k, 14, globaltimer_ns() - tw0);
                        tc_fence_after();
                        const uint32_t d_tmem = tmem + static_cast<uint32_t>(acc.slot * p.acc_cols);
                        for (int ks = 0; ks < kKSlices; ++ks) {
#ifdef DSPARK_TRACE
                            const uint64_t tw1 = globaltimer_ns();
#endif
                            if (!wait_phase(bar_w2_full + 8 * w2.slot, w2.phase, ctl, p)) {
                                ok = false;
                                break;
                            }
                            DSPARK_TRACE_ADD(k, 13, globaltimer_ns() - tw1);
                            if (mt == 0 && t == 0 && ks == 0) DSPARK_TRACE_AT(k, 17);
                            tc_fence_after();
                            // descriptors differ only in the start-address field (bits 0..13,
                            // 16-byte units): advance them with plain adds
                            const uint64_t a_k = a_desc0 + static_cast<uint64_t>((2 * ks * a_chunk) >> 4);
                            const uint64_t b_k = b_desc0 + static_cast<uint64_t>((w2.slot * p.w2_stage_bytes) >> 4);
#pragma unroll
                            for (int kk = 0; kk < kKSlice / 16; ++kk) {
                                const uint64_t a_desc =
                                    a_k + static_cast<uint64_t>(((kk >> 2) * a_chunk + (kk & 3) * 32) >> 4);
                                const uint64_t b_desc = b_k + static_cast<uint64_t>((kk * 2048) >> 4);
                                umma_bf16(d_tmem, a_desc, b_desc, idesc, (ks | kk) ? 1u : 0u);
                            }
                            issued_any = true;
                            umma_commit(bar_w2_empty + 8 * w2.slot);
                            w2.next(p.w2_stages);
                        }
                        if (!ok) break;
                        if (!ok) break;
                        if (mt == 0 && t == 0) DSPARK_TRACE_AT(k, 9);
                        if (mt == num_mt - 1 && t == ntiles - 1) DSPARK_TRACE_AT(k, 10);
                        umma_commit(bar_tfull + 8 * acc.slot);
                        acc.next(p.acc_slots);
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
    } else if (kConf && warp == kWarpConf) {
        // ------------------------------------------------------------ confidence head
        if constexpr (kConf) confidence_warp(p, G);
    } else {
        // ------------------------------------------------------------ epilogue (warps 0-7)
        const int q = warp & 3;                   // TMEM lane quadrant
        const int half = warp >> 2;               // which 32-column chunks of a tile
        const int rq = M / 4;                     // rows per quadrant: 16 or 32
        const bool lane_row = lane < rq;
        const int row = q * rq + lane;            // row of the M tile held by this lane
        const int urow = lane_row ? min(row, p.ub - 1) : 0;   // U tile row (stays in the slot)
        const uint32_t t_lane = tmem + (static_cast<uint32_t>(q * 32) << 16);
        const int chunk = lane >> 3, unit = lane & 7;
        const int gather_rows = rq / 2;           // rows of the quadrant this warp gathers
        Ring acc, ur;                             // accumulator and U box sequence
        uint32_t mt_count = 0;
        bool ok = true;
        int next_tok[kMaxMTiles];
        unsigned long long my_key[kMaxMTiles];
        float my_logit[kMaxMTiles];
        // M = 64 (one M tile): this thread's rows ra = lane/4 and rb = lane/4 + 8 of the quadrant
        const int r64 = q * 16 + (lane >> 2);
        const int ua64 = min(r64, p.ub - 1), ub64 = min(r64 + 8, p.ub - 1);
        unsigned long long key64[2] = {0ull, 0ull};
        float logit64[2] = {0.0f, 0.0f};
        for (int mt = 0; mt < num_mt; ++mt) {
            const int b = mt * M + row;
            next_tok[mt] = (lane_row && b < p.B) ? checked_token(p.anchor[b], p.V) : -1;
        }

        // gather A = W1[x_{k-1}] of M tile gmt (K-major, 128-byte swizzle), all rows in
        // flight; the MMA must have released A (aempty) before this is called
        auto gather = [&](int gmt) {
            const int my_tok = next_tok[gmt];
            for (int i = 0; i < gather_rows; ++i) {
                const int src_lane = half * gather_rows + i;
                const int tok = __shfl_sync(0xFFFFFFFFu, my_tok, src_lane);
                const int r = q * rq + src_lane;
                const uint32_t dst = sA + chunk * a_chunk + r * 128 + ((unit ^ (r & 7)) << 4);
                if (tok >= 0) {
                    const uint16_t *src = kRnn
                        ? p.a_rows + static_cast<size_t>(gmt * M + r) * kRank    // row b of s_k
                        : p.W1 + static_cast<size_t>(tok) * kRank;              // W1[x_{k-1}]
                    cp_async_16(dst, src + lane * 8);
                } else {
                    sts128_zero(dst);
                }
            }
            cp_async_wait_all();
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_afull);
            ++mt_count;
        };

        // bounded grid barrier number nth (counted from 1 over the whole launch); false
        // once this CTA or any other gave up.  trace_k > 0 stamps the trace of position k.
        // The verdict is taken by one thread and shared, so that every epilogue thread
        // agrees on it; a warp that failed earlier marks the CTA as stopping first.
        auto grid_sync = [&](uint32_t nth, int trace_k) -> bool {
            if (!ok) *reinterpret_cast<volatile int *>(&ctl.abort) = 1;
            epi_sync();
            if (threadIdx.x == 0) {
                bool good = !*reinterpret_cast<volatile int *>(&ctl.abort);
                if (good) {
                    red_release_add_u32(p.barrier, 1u);
                    if (trace_k > 0) DSPARK_TRACE_AT(trace_k, 4);
                    const uint32_t target =
                        nth * static_cast<uint32_t>(G) + static_cast<uint32_t>(p.barrier_extra);
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
                    if (trace_k > 0) DSPARK_TRACE_AT(trace_k, 5);
                }
                if (!good) *reinterpret_cast<volatile int *>(&ctl.abort) = 1;
                ctl.go = good ? 1 : 0;
            }
            epi_sync();
            return *reinterpret_cast<volatile int *>(&ctl.go) != 0;
        };
        constexpr uint32_t bars_per_pos = kRnn ? 2u : 1u;

        // RNN head: this CTA's rows b = blockIdx.x + j G get s_k = tanh(W1[x_{k-1}] +
        // s_{k-1} Whh).  Warp w multiplies Whh rows 32w .. 32w + 31 (16-byte loads, lane l
        // holds columns 8l .. 8l + 7), the eight partial rows are summed through shared
        // memory, and thread t finishes element t.  The A tile's shared memory, free until
        // the gather that follows, holds s_{k-1} and the partial sums.
        // After a failure it skips the work but keeps its named barriers.
        auto rnn_update = [&](int k) {
            float *scr = reinterpret_cast<float *>(dyn_smem + (sA - smem_u32(dyn_smem)));
            float *s_prev = scr;                          // [256]
            float *part = scr + kRank;                    // [8][256]
            const int t = threadIdx.x, w = t >> 5, ln = t & 31;
            for (int b = blockIdx.x; b < p.B; b += G) {
                if (!ok) {
                    epi_sync();
                    epi_sync();
                    epi_sync();
                    continue;
                }
                int tok = k == 1 ? p.anchor[b]
                                 : static_cast<int>(argmax_key_index(
                                       __ldcg(&p.slots[static_cast<size_t>(k - 2) * p.B + b])));
                tok = checked_token(tok, p.V);
                float *st = p.state + static_cast<size_t>(b) * kRank;
                s_prev[t] = k == 1 ? 0.0f : __ldcg(st + t);
                epi_sync();
                float acc8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
                for (int ii = 0; ii < 32; ++ii) {
                    const int i = 32 * w + ii;
                    const float si = s_prev[i];
                    const uint4 wv = __ldg(reinterpret_cast<const uint4 *>(
                        p.Whh + static_cast<size_t>(i) * kRank + 8 * ln));
                    acc8[0] = fmaf(si, bf16lo_to_f32(wv.x), acc8[0]);
                    acc8[1] = fmaf(si, bf16hi_to_f32(wv.x), acc8[1]);
                    acc8[2] = fmaf(si, bf16lo_to_f32(wv.y), acc8[2]);
                    acc8[3] = fmaf(si, bf16hi_to_f32(wv.y), acc8[3]);
                    acc8[4] = fmaf(si, bf16lo_to_f32(wv.z), acc8[4]);
                    acc8[5] = fmaf(si, bf16hi_to_f32(wv.z), acc8[5]);
                    acc8[6] = fmaf(si, bf16lo_to_f32(wv.w), acc8[6]);
                    acc8[7] = fmaf(si, bf16hi_to_f32(wv.w), acc8[7]);
                }
                float4 *pw = reinterpret_cast<float4 *>(part + w * kRank + 8 * ln);
                pw[0] = make_float4(acc8[0], acc8[1], acc8[2], acc8[3]);
                pw[1] = make_float4(acc8[4], acc8[5], acc8[6], acc8[7]);
                epi_sync();
                float acc = __uint_as_float(
                    static_cast<uint32_t>(p.W1[static_cast<size_t>(tok) * kRank + t]) << 16);
#pragma unroll
                for (int q8 = 0; q8 < kEpiWarps; ++q8) acc += part[q8 * kRank + t];
                const float sn = tanhf(acc);
                st[t] = sn;
                p.a_rows[static_cast<size_t>(b) * kRank + t] =
                    __bfloat16_as_ushort(__float2bfloat16_rn(sn));
                epi_sync();                   // the scratch is rewritten for the next row
            }
            __threadfence();                  // the rows are read by every CTA after the barrier
        };

        // Every epilogue warp runs the same sequence of named barriers whatever happens:
        // after a failed wait a warp only skips work, so that no bar.sync is left short.
        for (int k = 1; k <= p.gamma; ++k) {
            if (ok && !__all_sync(0xFFFFFFFFu, wait_phase(bar_aempty, (mt_count & 1u) ^ 1u, ctl, p)))
                ok = false;
            if constexpr (kRnn) {
                rnn_update(k);
                if (!grid_sync(static_cast<uint32_t>(2 * k - 1), 0)) ok = false;
            }
            if (threadIdx.x == 0) DSPARK_TRACE_AT(k, 0);
            if (ok) gather(0);
            if (threadIdx.x == 0) DSPARK_TRACE_AT(k, 1);
            for (int mt = 0; mt < num_mt; ++mt) {
                const int m0 = mt * M;
                const int my_b = m0 + row;
                // the next M tile's rows are gathered as soon as the MMA has released A, so
                // the tensor core does not wait for this tile's epilogue to finish
                bool next_gathered = mt + 1 >= num_mt;

                // ---- vocabulary tiles of this CTA: this warp takes chunks u with u % 2 == half
                const bool active = (m0 + q * rq) < p.B;
                const int b_glob = my_b + p.b_offset;
                RowBest best;
                RowBest best64[2];
                for (int t = 0; t < ntiles; ++t) {
                    int first, count;
                    tile_span_n(t, n_units, p.tile_units, first, count);
                    const int nbox = (count + 1) >> 1;
#ifdef DSPARK_TRACE
                    const uint64_t tfw0 = globaltimer_ns();
#endif
                    // warp-uniform outcome: tcgen05.ld below needs every lane of the warp
                    if (ok && !__all_sync(0xFFFFFFFFu,
                                          wait_phase(bar_tfull + 8 * acc.slot, acc.phase, ctl, p)))
                        ok = false;
                    if (ok) {
                        tc_fence_after();
                        if (threadIdx.x == 0 && mt == 0 && t == 0) DSPARK_TRACE_AT(k, 2);
                        if (threadIdx.x == 0 && mt == num_mt - 1 && t == ntiles - 1) DSPARK_TRACE_AT(k, 21);
                        if (threadIdx.x == 0 && t > 0) DSPARK_TRACE_ADD(k, 20, globaltimer_ns() - tfw0);
#ifdef DSPARK_TRACE
                        const uint64_t tbusy0 = globaltimer_ns();
#endif
                        // box i of the tile holds chunks 2i and 2i + 1; this warp takes boxes
                        // i = s, s + 2, ... and reduces both chunks of a box together, where
                        // s = half, swapped on odd tiles when a tile has an odd number of
                        // boxes so that the two warps of a quadrant share them evenly
                        const uint32_t t_acc = t_lane + static_cast<uint32_t>(acc.slot * p.acc_cols);
                        const int s0 = ((nbox & 1) && (t & 1)) ? (half ^ 1) : half;
                        Ring my = ur;
                        if (s0) my.next(p.u_slots);
                        for (int i = s0; i < nbox; i += 2) {
#ifdef DSPARK_TRACE
                            const uint64_t tw2 = globaltimer_ns();
#endif
                            if (!__all_sync(0xFFFFFFFFu,
                                            wait_phase(bar_u_full + 8 * my.slot, my.phase, ctl, p))) {
                                ok = false;
                                break;
                            }
                            if (threadIdx.x == 0) DSPARK_TRACE_ADD(k, 15, globaltimer_ns() - tw2);
                            const uint32_t u_box = sU + my.slot * p.u_slot_bytes;
                            if (active && M == 64) {
                                uint32_t a[32];
                                tmem_ld_16x256b_x8(t_acc + 2 * i * kUnit, a);
                                tmem_wait_ld();
                                box_update_m64(best64, a, 2 * i + 1 < count, u_box, ua64, ub64,
                                               (u_begin + first + 2 * i) * kUnit, p, k,
                                               r64 + p.b_offset, r64 + 8 + p.b_offset);
                            } else if (active) {
                                const bool two = 2 * i + 1 < count;
                                uint32_t a0[32], a1[32];
                                tmem_ld_32x32b_x32(t_acc + 2 * i * kUnit, a0);
                                tmem_ld_32x32b_x32(t_acc + (two ? 2 * i + 1 : 2 * i) * kUnit, a1);
                                tmem_wait_ld();
                                box_update(best, a0, a1, two, u_box, urow,
                                           (u_begin + first + 2 * i) * kUnit, p, k, b_glob);
                            }
                            __syncwarp();
                            if (lane == 0) mbar_arrive(bar_u_empty + 8 * my.slot);
                            my.next(p.u_slots);
                            my.next(p.u_slots);
                        }
                        if (threadIdx.x == 0) DSPARK_TRACE_ADD(k, 19, globaltimer_ns() - tbusy0);
                    }
                    for (int i = 0; i < nbox; ++i) ur.next(p.u_slots);
                    if (ok) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar_tempty + 8 * acc.slot);
                    }
                    acc.next(p.acc_slots);
                    if (ok && !next_gathered &&
                        __all_sync(0xFFFFFFFFu, mbar_test_wait(bar_aempty, (mt_count & 1u) ^ 1u))) {
                        gather(mt + 1);
                        next_gathered = true;
                    }
                }
                if (ok && !next_gathered) {
                    if (__all_sync(0xFFFFFFFFu, wait_phase(bar_aempty, (mt_count & 1u) ^ 1u, ctl, p)))
                        gather(mt + 1);
                    else
                        ok = false;
                }
                if (!ok) continue;
                if (M == 64) {
                    // the four threads of a row hold disjoint columns: combine, one atomic per row
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const unsigned long long key = argmax_key(best64[h].s, best64[h].v);
                        key64[h] = key;
                        logit64[h] = best64[h].l;
                        unsigned long long kr = key;
                        kr = max(kr, __shfl_xor_sync(0xFFFFFFFFu, kr, 1));
                        kr = max(kr, __shfl_xor_sync(0xFFFFFFFFu, kr, 2));
                        const int b = r64 + 8 * h;
                        if ((lane & 3) == 0 && b < p.B)
                            atomicMax(&p.slots[static_cast<size_t>(k - 1) * p.B + b], kr);
                    }
                } else if (lane_row && my_b < p.B) {
                    const unsigned long long key = argmax_key(best.s, best.v);
                    atomicMax(&p.slots[static_cast<size_t>(k - 1) * p.B + my_b], key);
                    my_key[mt] = key;
                    my_logit[mt] = best.l;
                }
            }

            // ---- grid barrier: every CTA has combined its rows of position k
            if (threadIdx.x == 0) DSPARK_TRACE_AT(k, 3);
            if (!grid_sync(static_cast<uint32_t>(k) * bars_per_pos, k)) ok = false;
            if (!ok) continue;
            // ---- x_k of my rows: next gather's tokens; the owning CTA/half writes the outputs
            for (int mt = 0; mt < num_mt; ++mt) {
                const int b = mt * M + row;
                if (!lane_row || b >= p.B) continue;
                const size_t o = static_cast<size_t>(k - 1) * p.B + b;
                const unsigned long long key = __ldcg(&p.slots[o]);
                const int tok = static_cast<int>(argmax_key_index(key));
                next_tok[mt] = checked_token(tok, p.V);
                if (M != 64 && key == my_key[mt]) {
                    p.x_out[static_cast<size_t>(b) * p.gamma + (k - 1)] = tok;
                    p.logit_out[static_cast<size_t>(b) * p.gamma + (k - 1)] = my_logit[mt];
                }
            }
            if (M == 64) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int b = r64 + 8 * h;
                    if (b >= p.B) continue;
                    const size_t o = static_cast<size_t>(k - 1) * p.B + b;
                    const unsigned long long key = __ldcg(&p.slots[o]);
                    if (key == key64[h]) {
                        p.x_out[static_cast<size_t>(b) * p.gamma + (k - 1)] =
                            static_cast<int>(argmax_key_index(key));
                        p.logit_out[static_cast<size_t>(b) * p.gamma + (k - 1)] = logit64[h];
                    }
                }
            }
            if (threadIdx.x == 0) DSPARK_TRACE_AT(k, 6);
        }

        if constexpr (kTail) {
            // ---- the scheduler and the verification, once every score of the launch is
            // written: ranks by all CTAs (one warp per score), then the last CTA to finish
            // its ranks scans, picks N*, writes the lengths and verifies every request, with
            // the same device code as the scheduler and verify kernels
            __shared__ sched::ScanSmem<kEpiWarps> tail_sm;
            __shared__ int tail_last;
            const int n = p.B * p.gamma;
            if (threadIdx.x == 0) {
                ctl.go = (ok && wait_counter(p.conf_done, static_cast<uint32_t>(G), p)) ? 1 : 0;
                DSPARK_TRACE_AT(p.gamma, 22);
            }
            epi_sync();
            const bool go = *reinterpret_cast<volatile int *>(&ctl.go) != 0;
            // the scores into this CTA's shared memory (the rings are idle once the last
            // position is drafted: every copy has landed and every MMA has completed), so
            // that the binary searches read shared memory
            float *sP = reinterpret_cast<float *>(dyn_smem + (base - smem_u32(dyn_smem)));
            if (go) {
#pragma unroll 8
                for (int i = threadIdx.x; i < n; i += kEpiWarps * 32) sP[i] = __ldcg(p.P_out + i);
            }
            epi_sync();
            if (go)
                for (int i = blockIdx.x * kEpiWarps + warp; i < n; i += G * kEpiWarps)
                    sched::rank_score(sP, p.B, p.gamma, n, i, p.rank, sched::LoadPlain{});
            epi_sync();
            if (threadIdx.x == 0) DSPARK_TRACE_AT(p.gamma, 23);
            if (threadIdx.x == 0) {
                __threadfence();
                const bool last = atomicAdd(p.tail_done, 1u) == static_cast<unsigned int>(G) - 1u;
                tail_last = (last && go && !*reinterpret_cast<volatile unsigned int *>(p.abort_flag)) ? 1 : 0;
                DSPARK_TRACE_AT(p.gamma, 24);
            }
            epi_sync();
            if (tail_last) {
                __threadfence();
                // the sorted scores and a copy of the ranks in shared memory, after sP
                long long *sQ = reinterpret_cast<long long *>(sP + ((n + 1) & ~1));
                int32_t *sRank = reinterpret_cast<int32_t *>(sQ + n);
                int32_t *sL = sRank + n;
                sched::scan_and_lengths<kEpiWarps>(p.P_out, p.B, p.gamma, n, p.Tstep, p.rank, sQ,
                                                   p.L_out, p.N_out, p.objective_out, tail_sm,
                                                   static_cast<int>(threadIdx.x),
                                                   [] { epi_sync(); }, sRank, sL);
                epi_sync();
                if (threadIdx.x == 0) DSPARK_TRACE_AT(p.gamma, 25);
                for (int b = threadIdx.x; b < p.B; b += kEpiWarps * 32)
                    verify::verify_request_len(p.x_out, sL[b], p.target, b, p.gamma,
                                               p.accepted_out, p.bonus_out);
                epi_sync();
                if (threadIdx.x == 0) DSPARK_TRACE_AT(p.gamma, 26);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace draft
}  // namespace dspark
