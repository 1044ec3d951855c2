// dspark_api.cu -- the C ABI (include/dspark.h): argument checks, TMA descriptors and
// launches of the four hot-path kernels.  One translation unit holds every kernel so
// that the per-device error word is a single symbol.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "confidence_sts.cuh"
#include "markov_draft.cuh"
#include "markov_pair.cuh"
#include "ptx.cuh"
#include "schedule_prefix.cuh"
#include "sts_fit.cuh"
#include "verify_prefix.cuh"

namespace {

std::atomic<unsigned long long> g_timeout_ns{2000000000ull};
std::atomic<int> g_barrier_extra{0};

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

struct DeviceInfo {
    int sms = 0;
    int major = 0;
    bool no_coop_clusters = false;   // the runtime refused a cooperative cluster launch
    // draft-kernel attributes and the pair kernel's resident clusters, valid for the CUDA
    // context with this id (0: none yet); a new context (after a device reset) re-sets them
    unsigned long long draft_ctx = 0;
    int pair_clusters = 0;
};

using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

// Unique id of the calling thread's current CUDA context (0 if unavailable).
unsigned long long current_ctx_id()
{
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx ||
        get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

constexpr int kMaxDevices = 64;
constexpr int kTileUnitsWide = 6; // 32-column units per wide tile of the single-CTA draft kernel
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mutex;

int current_device(DeviceInfo **info)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return DSPARK_CUDA_ERROR;
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    DeviceInfo &d = g_dev[dev];
    if (d.sms == 0) {
        if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
            d.sms = 0;
            return DSPARK_CUDA_ERROR;
        }
    }
    if (d.major != 10) return DSPARK_UNSUPPORTED_SHAPE;   // built for sm_100a only
    *info = &d;
    return DSPARK_OK;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// workspace layout shared by draft_step and schedule_prefix:
//   [0, 256)          control words (counters, flags)
//   [256, ...)        draft: argmax keys [gamma][B] u64
//                     schedule: ranks [n] i32, then fixed-point scores [n] i64
constexpr size_t kCtlBytes = 256;

//   RNN head: after the keys, the recurrent state [B][r] fp32 and its bf16 copy [B][r]
size_t draft_keys_end(int B, int gamma)
{
    return round_up(kCtlBytes + static_cast<size_t>(B) * gamma * 8, 256);
}

size_t draft_ws(int B, int gamma)
{
    return draft_keys_end(B, gamma) + static_cast<size_t>(B) * 256 * (4 + 2);
}

size_t sched_ws(int n)
{
    return kCtlBytes + round_up(static_cast<size_t>(n) * 4, 256) + static_cast<size_t>(n) * 8;
}

int from_cuda(cudaError_t e) { return e == cudaSuccess ? DSPARK_OK : DSPARK_CUDA_ERROR; }

// STS-fit workspace: frozen products [2][N] f64, then label counts [gamma][n_t][n_bins]
// u32, then fixed-point sums [gamma][n_t][n_bins] u64.
struct StsFitLayout {
    size_t p_bytes, cnt_bytes, sq_bytes;
    size_t total() const { return p_bytes + cnt_bytes + sq_bytes; }
};

StsFitLayout sts_fit_layout(int N, int gamma, int n_t, int n_bins)
{
    const size_t cells = static_cast<size_t>(gamma) * n_t * n_bins;
    return {round_up(static_cast<size_t>(N) * 16, 256), round_up(cells * 4, 256), cells * 8};
}

}  // namespace

extern "C" {

const char *dspark_status_string(int status)
{
    switch (status) {
    case DSPARK_OK: return "ok";
    case DSPARK_INVALID_ARG: return "invalid argument";
    case DSPARK_UNSUPPORTED_SHAPE: return "unsupported shape or device";
    case DSPARK_WORKSPACE_TOO_SMALL: return "workspace too small";
    case DSPARK_NOT_MONOTONE: return "scores outside [0,1] or increasing along a request";
    case DSPARK_CUDA_ERROR: return "CUDA error";
    case DSPARK_TIMEOUT: return "device wait timed out";
    case DSPARK_INVALID_TOKEN: return "token id or verify length out of range";
    case DSPARK_BAD_LAUNCH: return "kernel launched in a shape it cannot run in";
    default: return "unknown status";
    }
}

size_t dspark_workspace_bytes(int B, int gamma, int V, int r)
{
    (void)V;
    (void)r;
    if (B < 1 || gamma < 1) return 0;
    const size_t a = draft_ws(B, gamma);
    const size_t b = sched_ws(B * gamma);
    return a > b ? a : b;
}

int dspark_set_wait_timeout_ns(uint64_t ns)
{
    if (ns == 0) return DSPARK_INVALID_ARG;
    g_timeout_ns.store(ns);
    return DSPARK_OK;
}

int dspark_debug_barrier_extra(int extra)
{
    if (extra < 0) return DSPARK_INVALID_ARG;
    g_barrier_extra.store(extra);
    return DSPARK_OK;
}

}  // extern "C"

namespace {

// Inputs and outputs of the confidence head when it runs inside the draft launch.
struct ConfArgs {
    const void *h;
    const void *w;
    float b_conf;
    const float *T;
    int d;
    float *c_out;
    float *P_out;
};

// Inputs and outputs of the scheduler and the verification when they run at the end of
// the draft launch.
struct TailArgs {
    const double *Tstep;
    const int32_t *target;
    int32_t *L_out, *N_out;
    double *objective_out;
    int32_t *accepted_out, *bonus_out;
};

// Argument checks of the confidence head when it runs inside the draft launch.
int check_conf_args(const void *h, const void *w, const float *T, const float *c_out,
                    const float *P_out, int gamma, int d, int r)
{
    if (!h || !w || !T || !c_out || !P_out) return DSPARK_INVALID_ARG;
    if (!aligned(h, 16) || !aligned(w, 16) || !aligned(T, 4) || !aligned(c_out, 4) ||
        !aligned(P_out, 4))
        return DSPARK_INVALID_ARG;
    if (d < 8 || d % 8 != 0 || (d + r) * 2 > 200 * 1024 || gamma > dspark::conf::kMaxGamma)
        return DSPARK_UNSUPPORTED_SHAPE;
    return DSPARK_OK;
}

// The Markov head (Whh == nullptr) and the RNN head share one kernel and one launcher;
// with `conf` the Markov head's launch also computes the confidence head, and with
// `tail` (B <= 128, with conf) the scheduler and the verification after the last position.
int launch_draft(const void *U, const int32_t *anchor, const void *W1, const void *W2,
                 const void *Whh, int B, int gamma, int V, int r, int mode, float temperature,
                 uint64_t seed, int b_offset, int32_t *x_out, float *logit_x_out, void *workspace,
                 size_t workspace_bytes, dspark_stream_t stream, const ConfArgs *conf = nullptr,
                 const TailArgs *tail = nullptr)
{
    namespace D = dspark::draft;
    if (!U || !anchor || !W1 || !W2 || !x_out || !logit_x_out || !workspace)
        return DSPARK_INVALID_ARG;
    if (Whh && !aligned(Whh, 16)) return DSPARK_INVALID_ARG;
    if (!aligned(U, 16) || !aligned(W1, 16) || !aligned(W2, 16) || !aligned(anchor, 4) ||
        !aligned(x_out, 4) || !aligned(logit_x_out, 4) || !aligned(workspace, 256))
        return DSPARK_INVALID_ARG;
    if (mode != 0 && mode != 1) return DSPARK_INVALID_ARG;
    if (mode == 1 && !(temperature > 0.0f)) return DSPARK_INVALID_ARG;
    if (b_offset < 0) return DSPARK_INVALID_ARG;
    if (B < 1 || B > D::kMaxB || gamma < 1 || gamma > 64 || r != D::kRank || V < 64 ||
        V > (1 << 24) || V % 8 != 0)
        return DSPARK_UNSUPPORTED_SHAPE;
    if (workspace_bytes < draft_ws(B, gamma)) return DSPARK_WORKSPACE_TOO_SMALL;
    DeviceInfo *dev = nullptr;
    if (int st = current_device(&dev)) return st;
    EncodeTiledFn encode = encode_tiled();
    if (!encode) return DSPARK_CUDA_ERROR;

    // more than 128 requests (Markov head): the CTA-pair kernel, M = 256 per pair MMA
    const bool pair = !Whh && B > 128;
    const int M = B <= 64 ? 64 : 128;
    const int ub = B < M ? B : M;
    CUtensorMap tm_w2, tm_u;
    {
        const cuuint64_t dims[2] = {static_cast<cuuint64_t>(V), static_cast<cuuint64_t>(r)};
        const cuuint64_t strides[1] = {static_cast<cuuint64_t>(V) * 2};
        const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(D::kKSlice)};
        const cuuint32_t estr[2] = {1, 1};
        if (encode(&tm_w2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(W2), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return DSPARK_CUDA_ERROR;
    }
    {
        const cuuint64_t dims[3] = {static_cast<cuuint64_t>(V), static_cast<cuuint64_t>(gamma),
                                    static_cast<cuuint64_t>(B)};
        const cuuint64_t strides[2] = {static_cast<cuuint64_t>(V) * 2,
                                       static_cast<cuuint64_t>(V) * 2 * gamma};
        const cuuint32_t box[3] = {D::kUBoxCols, 1, static_cast<cuuint32_t>(ub)};
        const cuuint32_t estr[3] = {1, 1, 1};
        if (encode(&tm_u, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(U), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return DSPARK_CUDA_ERROR;
    }

    // the kernel instance for this call (Markov or RNN head, M = 64 or 128, or the pair
    // kernel); its shared memory limit is set on every call, so nothing cached outlives a
    // device reset
    const bool fused = conf != nullptr;   // the confidence head runs in a warp of the draft kernel
    void (*kern)(const CUtensorMap, const CUtensorMap, const D::Params) =
        pair ? (fused ? (mode ? D::pairk::markov_pair_kernel<true, true>
                              : D::pairk::markov_pair_kernel<false, true>)
                      : (mode ? D::pairk::markov_pair_kernel<true, false>
                              : D::pairk::markov_pair_kernel<false, false>))
        : Whh ? (M == 64 ? D::markov_draft_kernel<64, true> : D::markov_draft_kernel<128, true>)
        : (fused && tail) ? (M == 64 ? D::markov_draft_kernel<64, false, true, true>
                                     : D::markov_draft_kernel<128, false, true, true>)
        : fused ? (M == 64 ? D::markov_draft_kernel<64, false, true>
                           : D::markov_draft_kernel<128, false, true>)
                : (M == 64 ? D::markov_draft_kernel<64, false> : D::markov_draft_kernel<128, false>);
    const int dyn_smem = pair ? D::pairk::kDynSmem : D::kDynSmem;
    {
        // every instance's shared-memory limit, once per CUDA context (a device reset makes
        // a new context, with a new id, and the attributes are set again)
        const unsigned long long ctx = current_ctx_id();
        std::lock_guard<std::mutex> lock(g_dev_mutex);
        if (ctx == 0 || dev->draft_ctx != ctx) {
            void (*const all[])(const CUtensorMap, const CUtensorMap, const D::Params) = {
                D::markov_draft_kernel<64, false>, D::markov_draft_kernel<128, false>,
                D::markov_draft_kernel<64, true>, D::markov_draft_kernel<128, true>,
                D::markov_draft_kernel<64, false, true>, D::markov_draft_kernel<128, false, true>,
                D::markov_draft_kernel<64, false, true, true>,
                D::markov_draft_kernel<128, false, true, true>};
            for (auto f : all)
                if (cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         D::kDynSmem) != cudaSuccess)
                    return DSPARK_CUDA_ERROR;
            for (auto f : {D::pairk::markov_pair_kernel<false, false>,
                           D::pairk::markov_pair_kernel<true, false>,
                           D::pairk::markov_pair_kernel<false, true>,
                           D::pairk::markov_pair_kernel<true, true>})
                if (cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         D::pairk::kDynSmem) != cudaSuccess)
                    return DSPARK_CUDA_ERROR;
            dev->pair_clusters = 0;
            dev->draft_ctx = ctx;
        }
    }

    uint8_t *ws = static_cast<uint8_t *>(workspace);
    D::Params prm{};                     // every pointer not set below is null
    prm.anchor = anchor;
    prm.W1 = static_cast<const uint16_t *>(W1);
    prm.B = B;
    prm.gamma = gamma;
    prm.V = V;
    prm.mode = mode;
    prm.inv_tau = mode == 1 ? 1.0f / temperature : 1.0f;
    prm.seed_lo = static_cast<uint32_t>(seed);
    prm.seed_hi = static_cast<uint32_t>(seed >> 32);
    for (int r = 0; r < 10; ++r) {   // the Philox key schedule (Weyl increments), once per launch
        prm.rk0[r] = prm.seed_lo + static_cast<uint32_t>(r) * 0x9E3779B9u;
        prm.rk1[r] = prm.seed_hi + static_cast<uint32_t>(r) * 0xBB67AE85u;
    }
    prm.b_offset = b_offset;
    prm.x_out = x_out;
    prm.logit_out = logit_x_out;
    prm.barrier = reinterpret_cast<unsigned int *>(ws);
    prm.abort_flag = reinterpret_cast<unsigned int *>(ws + 4);
    prm.slots = reinterpret_cast<unsigned long long *>(ws + kCtlBytes);
    prm.Whh = static_cast<const uint16_t *>(Whh);
    prm.state = reinterpret_cast<float *>(ws + draft_keys_end(B, gamma));
    prm.a_rows = reinterpret_cast<uint16_t *>(ws + draft_keys_end(B, gamma) +
                                              static_cast<size_t>(B) * 256 * 4);
    prm.units_total = (V + D::kUnit - 1) / D::kUnit;
    const int grid_single = prm.units_total < dev->sms ? prm.units_total : dev->sms;
    prm.M = M;
    // shared memory: A (M x 256 bf16), then the W2 ring, then U boxes in what is left
    // Tile width: 192 columns (6 units; two 192-column accumulators) where that takes
    // fewer tiles per CTA than 128 columns (4 units; four accumulators), else 128.  At the
    // 151936-column vocabularies every CTA then has six tiles instead of eight, or nine for
    // the CTAs with a 33rd unit, which every position's grid barrier waited for.  W2
    // stages hold tile_units / 2 boxes of 64 columns per K half; the ring is one stage
    // deeper with M = 64, whose A tile is half as big.
    const int per_cta = (prm.units_total + grid_single - 1) / grid_single;
    const bool wide = (per_cta + kTileUnitsWide - 1) / kTileUnitsWide <
                      (per_cta + D::kMaxUnits - 1) / D::kMaxUnits;
    prm.tile_units = wide ? kTileUnitsWide : D::kMaxUnits;
    prm.acc_cols = prm.tile_units * D::kUnit;
    prm.acc_slots = wide ? 2 : D::kAcc;
    prm.w2_stage_bytes = ((prm.tile_units + 1) / 2) * D::kW2BoxBytes;
    prm.w2_stages = (wide ? 2 : 3) + (M == 64 ? 1 : 0);
    prm.ub = ub;
    prm.u_slot_bytes = static_cast<int>(round_up(static_cast<size_t>(ub) * D::kUBoxCols * 2, 1024));
    prm.u_slots = (D::kRingSmem - M * D::kRank * 2 - prm.w2_stages * prm.w2_stage_bytes) /
                  prm.u_slot_bytes;
    if (prm.u_slots > D::kUMaxSlots) prm.u_slots = D::kUMaxSlots;
    prm.timeout_ns = g_timeout_ns.load();
    prm.barrier_extra = g_barrier_extra.load();
    if (fused) {
        prm.h = static_cast<const uint16_t *>(conf->h);
        prm.wconf = static_cast<const uint16_t *>(conf->w);
        prm.b_conf = conf->b_conf;
        prm.T = conf->T;
        prm.d = conf->d;
        prm.c_out = conf->c_out;
        prm.P_out = conf->P_out;
        prm.zh = reinterpret_cast<float *>(ws + draft_keys_end(B, gamma));   // the RNN state's space
        prm.zh_done = reinterpret_cast<unsigned int *>(ws + 8);
    }
    if (fused && tail && !pair) {
        // workspace past the argmax keys: zh [B gamma] f32, then rank [B gamma] i32 (the
        // sorted scores live in the kernel's shared memory)
        const size_t n = static_cast<size_t>(B) * gamma;
        uint8_t *w0 = ws + draft_keys_end(B, gamma);
        prm.conf_done = reinterpret_cast<unsigned int *>(ws + 12);
        prm.tail_done = reinterpret_cast<unsigned int *>(ws + 16);
        prm.rank = reinterpret_cast<int32_t *>(w0 + round_up(n * 4, 256));
        prm.Tstep = tail->Tstep;
        prm.target = tail->target;
        prm.L_out = tail->L_out;
        prm.N_out = tail->N_out;
        prm.objective_out = tail->objective_out;
        prm.accepted_out = tail->accepted_out;
        prm.bonus_out = tail->bonus_out;
    }

    if (cudaMemsetAsync(ws, 0, draft_keys_end(B, gamma), stream) != cudaSuccess)
        return DSPARK_CUDA_ERROR;

    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof cfg);
    cfg.dynamicSmemBytes = dyn_smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    if (!pair) {
        cfg.gridDim = dim3(grid_single);
        cfg.blockDim = dim3(fused ? D::kThreadsConf : D::kThreads);
        cfg.numAttrs = 1;
        return from_cuda(cudaLaunchKernelEx(&cfg, kern, tm_w2, tm_u, prm));
    }
    // clusters of two CTAs, as many pairs as can be resident at once (every CTA waits for
    // all others at the end of each position)
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.blockDim = dim3(fused ? D::pairk::kThreadsConfPair : D::pairk::kThreads);
    cfg.gridDim = dim3(dev->sms & ~1);
    cfg.attrs = attr + 1;
    cfg.numAttrs = 1;
    int clusters = dev->pair_clusters;
    if (clusters < 1) {
        if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) != cudaSuccess || clusters < 1) {
            cudaGetLastError();
            return DSPARK_CUDA_ERROR;
        }
        dev->pair_clusters = clusters;
    }
    int npairs = dev->sms / 2;
    if (clusters < npairs) npairs = clusters;
    if (prm.units_total < npairs) npairs = prm.units_total;
    cfg.gridDim = dim3(2 * npairs);
    // cooperative as well where the runtime accepts it together with clusters
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (!dev->no_coop_clusters) {
        const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tm_w2, tm_u, prm);
        if (e == cudaSuccess) return DSPARK_OK;
        if (e != cudaErrorInvalidValue && e != cudaErrorNotSupported &&
            e != cudaErrorInvalidConfiguration)
            return DSPARK_CUDA_ERROR;
        cudaGetLastError();
        dev->no_coop_clusters = true;
    }
    cfg.attrs = attr + 1;
    cfg.numAttrs = 1;
    return from_cuda(cudaLaunchKernelEx(&cfg, kern, tm_w2, tm_u, prm));
}

}  // namespace

extern "C" {

int dspark_draft_step(const void *U, const int32_t *anchor, const void *W1, const void *W2, int B,
                      int gamma, int V, int r, int mode, float temperature, uint64_t seed,
                      int b_offset, int32_t *x_out, float *logit_x_out, void *workspace,
                      size_t workspace_bytes, dspark_stream_t stream)
{
    return launch_draft(U, anchor, W1, W2, nullptr, B, gamma, V, r, mode, temperature, seed,
                        b_offset, x_out, logit_x_out, workspace, workspace_bytes, stream);
}

int dspark_draft_step_rnn(const void *U, const int32_t *anchor, const void *W1, const void *W2,
                          const void *Whh, int B, int gamma, int V, int r, int mode,
                          float temperature, uint64_t seed, int b_offset, int32_t *x_out,
                          float *logit_x_out, void *workspace, size_t workspace_bytes,
                          dspark_stream_t stream)
{
    if (!Whh) return DSPARK_INVALID_ARG;
    return launch_draft(U, anchor, W1, W2, Whh, B, gamma, V, r, mode, temperature, seed,
                        b_offset, x_out, logit_x_out, workspace, workspace_bytes, stream);
}

int dspark_draft_confidence_step(const void *U, const int32_t *anchor, const void *W1,
                                 const void *W2, const void *h, const void *w, float b_conf,
                                 const float *T, int B, int gamma, int V, int r, int d, int mode,
                                 float temperature, uint64_t seed, int b_offset, int32_t *x_out,
                                 float *logit_x_out, float *c_out, float *P_out, void *workspace,
                                 size_t workspace_bytes, dspark_stream_t stream)
{
    if (int st = check_conf_args(h, w, T, c_out, P_out, gamma, d, r)) return st;
    const ConfArgs conf{h, w, b_conf, T, d, c_out, P_out};
    // Gumbel-max drafting on CTA pairs is bound by its selection arithmetic, and a
    // confidence warp beside it would take issue slots from it: there the confidence
    // kernel follows as a second launch instead
    const bool in_launch = !(mode == 1 && B > 128);
    if (int st = launch_draft(U, anchor, W1, W2, nullptr, B, gamma, V, r, mode, temperature, seed,
                              b_offset, x_out, logit_x_out, workspace, workspace_bytes, stream,
                              in_launch ? &conf : nullptr))
        return st;
    if (in_launch) return DSPARK_OK;     // computed inside the draft launch
    return dspark_confidence_sts(h, anchor, x_out, W1, w, b_conf, T, B, gamma, d, r, V, c_out,
                                 P_out, stream);
}

// The scheduler's second phase runs on one CTA of the draft launch; above this many
// scores the separate scheduler kernel (many CTAs for the ranks, a 512-thread scan) is
// faster than the launch it saves (measured: 1024 scores 6 us faster in one launch,
// 2048 scores 5 us slower).
constexpr int kTailMaxScores = 1024;

int dspark_step(const void *U, const int32_t *anchor, const void *W1, const void *W2,
                const void *h, const void *w, float b_conf, const float *T,
                const double *Tstep_us, const int32_t *target, int B, int gamma, int V, int r,
                int d, int mode, float temperature, uint64_t seed, int b_offset, int32_t *x_out,
                float *logit_x_out, float *c_out, float *P_out, int32_t *L_out, int32_t *N_out,
                double *objective_out, int32_t *accepted_out, int32_t *bonus_out,
                void *workspace, size_t workspace_bytes, dspark_stream_t stream)
{
    if (!Tstep_us || !target || !L_out || !N_out || !objective_out || !accepted_out ||
        !bonus_out)
        return DSPARK_INVALID_ARG;
    if (!aligned(Tstep_us, 8) || !aligned(target, 4) || !aligned(L_out, 4) ||
        !aligned(N_out, 4) || !aligned(objective_out, 8) || !aligned(accepted_out, 4) ||
        !aligned(bonus_out, 4))
        return DSPARK_INVALID_ARG;
    if (B < 1 || gamma < 1 || B > 32768 || static_cast<long long>(B) * gamma > 65536)
        return DSPARK_UNSUPPORTED_SHAPE;
    if (workspace && workspace_bytes < dspark_workspace_bytes(B, gamma, V, r))
        return DSPARK_WORKSPACE_TOO_SMALL;
    if (B <= 128 && B * gamma <= kTailMaxScores) {
        // one launch: drafting, the confidence head, then the scheduler and verification
        if (int st = check_conf_args(h, w, T, c_out, P_out, gamma, d, r)) return st;
        const ConfArgs conf{h, w, b_conf, T, d, c_out, P_out};
        const TailArgs tail{Tstep_us, target, L_out, N_out, objective_out, accepted_out, bonus_out};
        return launch_draft(U, anchor, W1, W2, nullptr, B, gamma, V, r, mode, temperature, seed,
                            b_offset, x_out, logit_x_out, workspace, workspace_bytes, stream,
                            &conf, &tail);
    }
    if (int st = dspark_draft_confidence_step(U, anchor, W1, W2, h, w, b_conf, T, B, gamma, V, r,
                                              d, mode, temperature, seed, b_offset, x_out,
                                              logit_x_out, c_out, P_out, workspace,
                                              workspace_bytes, stream))
        return st;
    if (int st = dspark_schedule_prefix(P_out, B, gamma, Tstep_us, L_out, N_out, objective_out,
                                        workspace, workspace_bytes, stream))
        return st;
    return dspark_verify_prefix(x_out, L_out, target, B, gamma, accepted_out, bonus_out, stream);
}

int dspark_confidence_sts(const void *h, const int32_t *anchor, const int32_t *x, const void *W1,
                          const void *w, float b_conf, const float *T, int B, int gamma, int d,
                          int r, int V, float *c_out, float *P_out, dspark_stream_t stream)
{
    namespace C = dspark::conf;
    if (!h || !anchor || !x || !W1 || !w || !T || !c_out || !P_out) return DSPARK_INVALID_ARG;
    if (!aligned(h, 16) || !aligned(W1, 16) || !aligned(w, 16) || !aligned(anchor, 4) ||
        !aligned(x, 4) || !aligned(T, 4) || !aligned(c_out, 4) || !aligned(P_out, 4))
        return DSPARK_INVALID_ARG;
    if (B < 1 || B > 65535 || gamma < 1 || gamma > C::kMaxGamma || d < 8 || d % 8 != 0 || r < 8 ||
        r % 8 != 0 || V < 1 || (d + r) * 2 > 200 * 1024)
        return DSPARK_UNSUPPORTED_SHAPE;
    DeviceInfo *dev = nullptr;
    if (int st = current_device(&dev)) return st;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof cfg);
    const int cs = C::cluster_ctas(gamma);
    cfg.gridDim = dim3(cs, B);
    cfg.blockDim = dim3(C::kThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return from_cuda(cudaLaunchKernelEx(
        &cfg, C::confidence_sts_kernel, static_cast<const uint16_t *>(h), anchor, x,
        static_cast<const uint16_t *>(W1), static_cast<const uint16_t *>(w), b_conf, T, B, gamma,
        d, r, V, c_out, P_out));
}

int dspark_schedule_prefix(const float *P, int B, int gamma, const double *Tstep_us,
                           int32_t *L_out, int32_t *N_out, double *objective_out, void *workspace,
                           size_t workspace_bytes, dspark_stream_t stream)
{
    namespace S = dspark::sched;
    if (!P || !Tstep_us || !L_out || !N_out || !objective_out || !workspace)
        return DSPARK_INVALID_ARG;
    if (!aligned(P, 4) || !aligned(Tstep_us, 8) || !aligned(L_out, 4) || !aligned(N_out, 4) ||
        !aligned(objective_out, 8) || !aligned(workspace, 256))
        return DSPARK_INVALID_ARG;
    if (B < 1 || B > 32768 || gamma < 1 || gamma > 64 || static_cast<long long>(B) * gamma > 65536)
        return DSPARK_UNSUPPORTED_SHAPE;
    const int n = B * gamma;
    if (workspace_bytes < sched_ws(n)) return DSPARK_WORKSPACE_TOO_SMALL;
    DeviceInfo *dev = nullptr;
    if (int st = current_device(&dev)) return st;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    S::Params prm;
    prm.P = P;
    prm.B = B;
    prm.gamma = gamma;
    prm.n = n;
    prm.Tstep = Tstep_us;
    prm.L_out = L_out;
    prm.N_out = N_out;
    prm.objective_out = objective_out;
    prm.done = reinterpret_cast<unsigned int *>(ws);
    prm.rank = reinterpret_cast<int32_t *>(ws + kCtlBytes);
    prm.q_sorted = reinterpret_cast<long long *>(ws + kCtlBytes + round_up(static_cast<size_t>(n) * 4, 256));
    if (cudaMemsetAsync(ws, 0, kCtlBytes, stream) != cudaSuccess) return DSPARK_CUDA_ERROR;
    int grid = (n + S::kWarps - 1) / S::kWarps;
    if (grid > 2 * dev->sms) grid = 2 * dev->sms;
    S::schedule_prefix_kernel<<<grid, S::kThreads, 0, stream>>>(prm);
    return from_cuda(cudaGetLastError());
}

int dspark_verify_prefix(const int32_t *x, const int32_t *L, const int32_t *target, int B,
                         int gamma, int32_t *accepted_out, int32_t *bonus_out,
                         dspark_stream_t stream)
{
    namespace Vf = dspark::verify;
    if (!x || !L || !target || !accepted_out || !bonus_out) return DSPARK_INVALID_ARG;
    if (!aligned(x, 4) || !aligned(L, 4) || !aligned(target, 4) || !aligned(accepted_out, 4) ||
        !aligned(bonus_out, 4))
        return DSPARK_INVALID_ARG;
    if (B < 1 || gamma < 1 || gamma > 4096) return DSPARK_UNSUPPORTED_SHAPE;
    DeviceInfo *dev = nullptr;
    if (int st = current_device(&dev)) return st;
    Vf::verify_prefix_kernel<<<(B + Vf::kThreads - 1) / Vf::kThreads, Vf::kThreads, 0, stream>>>(
        x, L, target, B, gamma, accepted_out, bonus_out);
    return from_cuda(cudaGetLastError());
}

size_t dspark_sts_fit_workspace_bytes(int N, int gamma, int n_t, int n_bins)
{
    if (N < 1 || gamma < 1 || n_t < 1 || n_bins < 1) return 0;
    return sts_fit_layout(N, gamma, n_t, n_bins).total();
}

int dspark_sts_fit(const float *z, const int32_t *accepted, int N, int gamma, double t_min,
                   double t_step, int n_t, int n_bins, int32_t *index_out, float *T_out,
                   double *ece_out, void *workspace, size_t workspace_bytes,
                   dspark_stream_t stream)
{
    namespace F = dspark::stsfit;
    if (!z || !accepted || !index_out || !T_out || !ece_out || !workspace)
        return DSPARK_INVALID_ARG;
    if (!aligned(z, 4) || !aligned(accepted, 4) || !aligned(index_out, 4) || !aligned(T_out, 4) ||
        !aligned(ece_out, 8) || !aligned(workspace, 256))
        return DSPARK_INVALID_ARG;
    const double t_max = t_min + static_cast<double>(n_t - 1) * t_step;
    if (!(t_min > 0.0) || !(t_step >= 0.0) || !(t_max < 1e300)) return DSPARK_INVALID_ARG;
    if (N < 1 || N > F::kMaxN || gamma < 1 || gamma > 64 || n_t < 1 || n_t > (1 << 20) ||
        n_bins < 1 || n_bins > F::kMaxBins)
        return DSPARK_UNSUPPORTED_SHAPE;
    const StsFitLayout lay = sts_fit_layout(N, gamma, n_t, n_bins);
    if (workspace_bytes < lay.total()) return DSPARK_WORKSPACE_TOO_SMALL;
    DeviceInfo *dev = nullptr;
    if (int st = current_device(&dev)) return st;

    int tpb = static_cast<int>(round_up(static_cast<size_t>(n_t), 32));
    if (tpb > F::kMaxThreads) tpb = F::kMaxThreads;
    while (F::hist_smem_bytes(tpb, n_bins) > 200 * 1024 && tpb > 32)
        tpb = static_cast<int>(round_up(static_cast<size_t>(tpb / 2), 32));
    const size_t smem = F::hist_smem_bytes(tpb, n_bins);
    const int gy = (n_t + tpb - 1) / tpb;
    if (gy > 65535) return DSPARK_UNSUPPORTED_SHAPE;
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(F::sts_hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return DSPARK_CUDA_ERROR;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, F::sts_hist_kernel, tpb, smem) !=
            cudaSuccess ||
        per_sm < 1)
        return DSPARK_CUDA_ERROR;
    int gx = per_sm * dev->sms / gy;             // one even share of the samples per CTA slot
    if (gx > (N + 63) / 64) gx = (N + 63) / 64;  // but no share below 64 samples
    if (gx < 1) gx = 1;

    uint8_t *ws = static_cast<uint8_t *>(workspace);
    F::Params prm;
    prm.z = z;
    prm.acc = accepted;
    prm.N = N;
    prm.gamma = gamma;
    prm.t_min = t_min;
    prm.t_step = t_step;
    prm.n_t = n_t;
    prm.n_bins = n_bins;
    prm.P = reinterpret_cast<double *>(ws);
    prm.idx = index_out;
    prm.T_out = T_out;
    prm.ece_out = ece_out;
    prm.cnt = reinterpret_cast<unsigned int *>(ws + lay.p_bytes);
    prm.sq = reinterpret_cast<unsigned long long *>(ws + lay.p_bytes + lay.cnt_bytes);
    if (cudaMemsetAsync(ws + lay.p_bytes, 0, lay.cnt_bytes + lay.sq_bytes, stream) != cudaSuccess)
        return DSPARK_CUDA_ERROR;
    for (int k = 1; k <= gamma; ++k) {
        prm.k = k;
        F::sts_hist_kernel<<<dim3(gx, gy), tpb, smem, stream>>>(prm);
        F::sts_pick_kernel<<<1, F::kPickThreads, 0, stream>>>(prm);
    }
    return from_cuda(cudaGetLastError());
}

}  // extern "C"

// ---------------------------------------------------------------------------------
// Scheduler entry point for callers that cannot allocate device memory.
//
// dspark_schedule_prefix needs a caller-provided workspace.  Some callers have no way
// to provide one: their device memory is fixed when the process starts (a serving
// engine that carves all of HBM into its own pools, an embedded runtime with a set
// budget), or they must not call cudaMalloc on this path because it can synchronise
// the device and stall other streams.  This variant keeps its scratch in the static
// array below instead, which is part of this library's device image: every GPU that
// loads the library holds it (288 KB) until the process exits.
namespace {

constexpr int kNoAllocMaxScores = 24576;                          // B * gamma limit
constexpr size_t kNoAllocRankOffset = kCtlBytes;
constexpr size_t kNoAllocQOffset = kCtlBytes + static_cast<size_t>(kNoAllocMaxScores) * 4;
constexpr size_t kNoAllocScratchBytes = kNoAllocQOffset + static_cast<size_t>(kNoAllocMaxScores) * 8;

static __device__ __align__(256) unsigned char g_sched_scratch[kNoAllocScratchBytes];

}  // namespace

extern "C" {

int dspark_schedule_prefix_noalloc(const float *P, int B, int gamma, const double *Tstep_us,
                                   int32_t *L_out, int32_t *N_out, double *objective_out,
                                   dspark_stream_t stream)
{
    namespace S = dspark::sched;
    if (!P || !Tstep_us || !L_out || !N_out || !objective_out) return DSPARK_INVALID_ARG;
    if (!aligned(P, 4) || !aligned(Tstep_us, 8) || !aligned(L_out, 4) || !aligned(N_out, 4) ||
        !aligned(objective_out, 8))
        return DSPARK_INVALID_ARG;
    if (B < 1 || gamma < 1 || gamma > 64 ||
        static_cast<long long>(B) * gamma > kNoAllocMaxScores)
        return DSPARK_UNSUPPORTED_SHAPE;
    DeviceInfo *dev = nullptr;
    if (int st = current_device(&dev)) return st;
    // In host code g_sched_scratch names only a host-side stand-in; its device address
    // on the current device is looked up on every call (cheap once the module is
    // loaded), so no address outlives a context that was torn down and re-created.
    void *scratch = nullptr;
    if (cudaGetSymbolAddress(&scratch, g_sched_scratch) != cudaSuccess || !scratch)
        return DSPARK_CUDA_ERROR;
    uint8_t *ws = static_cast<uint8_t *>(scratch);
    const int n = B * gamma;
    S::Params prm;
    prm.P = P;
    prm.B = B;
    prm.gamma = gamma;
    prm.n = n;
    prm.Tstep = Tstep_us;
    prm.L_out = L_out;
    prm.N_out = N_out;
    prm.objective_out = objective_out;
    prm.done = reinterpret_cast<unsigned int *>(ws);
    prm.rank = reinterpret_cast<int32_t *>(ws + kNoAllocRankOffset);
    prm.q_sorted = reinterpret_cast<long long *>(ws + kNoAllocQOffset);
    // the completion counter must start at zero; the rest is fully rewritten by the kernel
    if (cudaMemsetAsync(ws, 0, kCtlBytes, stream) != cudaSuccess) return DSPARK_CUDA_ERROR;
    int grid = (n + S::kWarps - 1) / S::kWarps;
    if (grid > 2 * dev->sms) grid = 2 * dev->sms;
    S::schedule_prefix_kernel<<<grid, S::kThreads, 0, stream>>>(prm);
    return from_cuda(cudaGetLastError());
}

int dspark_get_error(dspark_stream_t stream, int *status)
{
    if (!status) return DSPARK_INVALID_ARG;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return DSPARK_CUDA_ERROR;
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, dspark::g_error_word, sizeof v) != cudaSuccess)
        return DSPARK_CUDA_ERROR;
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(dspark::g_error_word, &zero, sizeof zero) != cudaSuccess)
        return DSPARK_CUDA_ERROR;
    *status = static_cast<int>(v);
    return DSPARK_OK;
}

}  // extern "C"

#ifdef DSPARK_TRACE
// Trace builds only: copy the draft kernel's timeline (see DSPARK_TRACE_AT).
extern "C" int dspark_trace_copy(void *host, size_t bytes)
{
    return cudaMemcpyFromSymbol(host, dspark::g_trace, bytes) == cudaSuccess ? DSPARK_OK
                                                                              : DSPARK_CUDA_ERROR;
}
#endif
