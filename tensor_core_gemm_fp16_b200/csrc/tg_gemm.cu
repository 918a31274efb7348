// tg_gemm.cu -- host side of the C ABI declared in include/tg_gemm.h:
// argument validation, per-shape configuration choice, TMA tensor-map
// encoding, operand repacking for unaligned pitches, and kernel launch.
//
// The operation is the tutorial's tiled fp16 tensor-core GEMM with an fp32
// accumulator ("Designing High-Performance GPU Kernels with TileLang",
// thecryptopost.io, make_matmul and the 2048^3 section) with the fused
// bias + GELU epilogue of its fused-epilogue section (ainovat.com).  Its
// schedule knobs (tile sizes, stages, L2 swizzle; the schedule-sweep
// section) become the compiled configuration table below.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>

#include "tg_gemm.h"
#include "tg_internal.h"
#include "tg_aux.cuh"

// Per-device error word: bounded-wait expiries are OR-ed in here.
__device__ unsigned g_tg_error_word;

namespace {

constexpr int kMaxDevices = 64;
constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;   // 2 s

// ------------------------------------------------------------------ configs
using LaunchFn = cudaError_t (*)(const CUtensorMap &, const CUtensorMap &, const CUtensorMap &,
                                 const tg::GemmParams &, int, cudaStream_t);
using ClusterQueryFn = int (*)(int num_sms);

// One bit per device: the kernel's dynamic shared-memory limit has been raised.
template <class Kernel>
cudaError_t ensure_smem_attr(Kernel kern, int smem, std::atomic<uint64_t> &attr_set)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = dev < 64 ? (1ull << dev) : 0;
    if (!bit || !(attr_set.load() & bit)) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        attr_set.fetch_or(bit);
    }
    return cudaSuccess;
}

template <int BN, int BK, int ST_REQ, int EPI, bool PAIR, int EW, int STORE, int LOAD,
          bool SHARE = false>
cudaError_t launch_gemm(const CUtensorMap &ta, const CUtensorMap &tb, const CUtensorMap &tc,
                        const tg::GemmParams &p, int grid, cudaStream_t stream)
{
    constexpr int ST = tg::FittedStages<BN, BK, ST_REQ, PAIR, EW, STORE, LOAD>::value;
    using S = tg::KernelShape<BN, BK, ST, PAIR, EW, STORE, LOAD>;
    auto kern = tg::gemm_persistent_kernel<BN, BK, ST, EPI, PAIR, EW, STORE, LOAD, SHARE>;
    static std::atomic<uint64_t> attr_set{0};
    cudaError_t e = ensure_smem_attr(kern, S::kDynamicBytes, attr_set);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.blockDim = dim3(S::kThreads, 1, 1);
    cfg.dynamicSmemBytes = S::kDynamicBytes;
    cfg.stream = stream;
    // Programmatic stream serialisation: the kernel's prologue may overlap the
    // previous kernel in the stream; it waits (griddepcontrol.wait) before
    // touching global memory.
    cudaLaunchAttribute attr[2];
    unsigned n_attr = 0;
    attr[n_attr].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n_attr].val.programmaticStreamSerializationAllowed = 1;
    ++n_attr;
    if (PAIR) {
        attr[n_attr].id = cudaLaunchAttributeClusterDimension;
        attr[n_attr].val.clusterDim.x = 2;
        attr[n_attr].val.clusterDim.y = 1;
        attr[n_attr].val.clusterDim.z = 1;
        ++n_attr;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n_attr;
    e = cudaLaunchKernelEx(&cfg, kern, ta, tb, tc, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// The row-softmax epilogue needs each epilogue thread to own a whole row,
// i.e. 4 epilogue warps; other shapes have no softmax kernel.
template <int BN, int BK, int ST, bool PAIR, int EW, int STORE, int LOAD>
constexpr LaunchFn softmax_fn()
{
    if constexpr (EW == 4)
        return launch_gemm<BN, BK, ST, TG_EPILOGUE_BIAS_SOFTMAX, PAIR, EW, STORE, LOAD>;
    else
        return nullptr;
}

constexpr int kNumEpilogues = 5;

template <int BN, int BK, int ST, int EPI, bool PAIR, int EW, int STORE, int LOAD>
constexpr LaunchFn share_fn()
{
    if constexpr (LOAD == tg::kLoadTma)
        return launch_gemm<BN, BK, ST, EPI, PAIR, EW, STORE, LOAD, true>;
    else
        return nullptr;
}

struct KernelConfig {
    tg_config_t info;
    int store_pref;                  // store mode when C rows are 16-byte aligned
    LaunchFn fn[kNumEpilogues][2];   // [epilogue][0: element stores, 1: store_pref]
    // Variants for an even stream-K split with a shared fold (store_pref, no
    // row softmax; nullptr for the plain loader).
    LaunchFn fn_share[kNumEpilogues - 1];
};

#define TG_FNS(BN, BK, ST, PAIR, EW, SP, LD)                                                \
    {                                                                                       \
        {launch_gemm<BN, BK, ST, 0, PAIR, EW, tg::kStoreScalar, LD>,                        \
         launch_gemm<BN, BK, ST, 0, PAIR, EW, SP, LD>},                                     \
            {launch_gemm<BN, BK, ST, 1, PAIR, EW, tg::kStoreScalar, LD>,                    \
             launch_gemm<BN, BK, ST, 1, PAIR, EW, SP, LD>},                                 \
            {launch_gemm<BN, BK, ST, 2, PAIR, EW, tg::kStoreScalar, LD>,                    \
             launch_gemm<BN, BK, ST, 2, PAIR, EW, SP, LD>},                                 \
            {launch_gemm<BN, BK, ST, 3, PAIR, EW, tg::kStoreScalar, LD>,                    \
             launch_gemm<BN, BK, ST, 3, PAIR, EW, SP, LD>},                                 \
            {softmax_fn<BN, BK, ST, PAIR, EW, tg::kStoreScalar, LD>(),                      \
             softmax_fn<BN, BK, ST, PAIR, EW, SP, LD>()},                                   \
    }

#define TG_FNS_SHARE(BN, BK, ST, PAIR, EW, SP, LD)                                          \
    {share_fn<BN, BK, ST, 0, PAIR, EW, SP, LD>(), share_fn<BN, BK, ST, 1, PAIR, EW, SP, LD>(),  \
     share_fn<BN, BK, ST, 2, PAIR, EW, SP, LD>(), share_fn<BN, BK, ST, 3, PAIR, EW, SP, LD>()}

#define TG_CONFIG(ID, BN, BK, ST, PAIR, EW, SP, GROUP, LD)                                  \
    {{ID, 128 * ((PAIR) ? 2 : 1), BN, BK, ST, (PAIR) ? 1 : 0, GROUP, EW, 0, LD}, SP,        \
     TG_FNS(BN, BK, ST, PAIR, EW, SP, LD), TG_FNS_SHARE(BN, BK, ST, PAIR, EW, SP, LD)}

// {id, BN, BK, stages, CTA pair, epilogue warps, store mode for aligned C, group_m, loader}
// Configurations 9 and 10 load operands with plain loads (any row pitch, no
// repacking); the others use TMA and repack operands whose rows are not
// 16-byte aligned.
const KernelConfig kConfigs[] = {
    TG_CONFIG(0, 256, 128, 3, true, 8, tg::kStoreTma, 8, tg::kLoadTma),
    TG_CONFIG(1, 256, 64, 6, true, 8, tg::kStoreTma, 8, tg::kLoadTma),
    TG_CONFIG(2, 128, 64, 8, true, 8, tg::kStoreTma, 8, tg::kLoadTma),
    TG_CONFIG(3, 256, 64, 4, false, 8, tg::kStoreTma, 8, tg::kLoadTma),
    TG_CONFIG(4, 128, 64, 6, false, 8, tg::kStoreTma, 8, tg::kLoadTma),
    TG_CONFIG(5, 64, 64, 8, false, 4, tg::kStoreTma, 8, tg::kLoadTma),
    TG_CONFIG(6, 256, 128, 3, true, 4, tg::kStoreTma, 8, tg::kLoadTma),
    TG_CONFIG(7, 256, 64, 6, true, 4, tg::kStoreTma, 8, tg::kLoadTma),
    TG_CONFIG(8, 256, 64, 4, false, 4, tg::kStoreVec, 8, tg::kLoadTma),
    TG_CONFIG(9, 256, 64, 4, false, 4, tg::kStoreTma, 8, tg::kLoadPlain),
    TG_CONFIG(10, 128, 64, 6, false, 4, tg::kStoreTma, 8, tg::kLoadPlain),
};
constexpr int kNumConfigs = sizeof(kConfigs) / sizeof(kConfigs[0]);

struct TableRow {
    int64_t M, N, K;
    int epilogue;
    int config;
    int split;   // TG_SPLIT_TILES or TG_SPLIT_STREAM_K, as the sweep timed it
};
#include "tg_configs.inc"

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Cost model for choosing a configuration and a work division, in
// microseconds at the power-capped clock of a busy B200 (about 1.4 GHz).
//   One k-block of one SM takes max(MMA, operand load): the MMA does
//   128 x BN x BK multiply-adds at 8192 flops per clock; the loads bring
//   (128 + BN / CG) x BK fp16 values at about 64 bytes per clock from L2.
//   Whole tiles: the busiest SM runs ceil(tiles / units) tiles of all k-blocks.
//   Stream-K: every unit runs ceil(tiles x k-blocks / units) k-blocks, plus a
//   fixed 6 us for writing, flagging and waiting, plus the head's fold of its
//   contributors' partials (128 x BN fp32 per CTA each) at about 75 GB/s.
// The constants were fitted to whole-tile and stream-K timings of the
// compiled configurations on deep-K and square shapes.
constexpr double kClockGhz = 1.4;
constexpr double kStreamKFixedUs = 6.0;
constexpr double kFoldGBs = 75.0;

struct Choice {
    int config;
    int split;   // TG_SPLIT_TILES or TG_SPLIT_STREAM_K
};

// Stream-K units (CTAs, or CTA pairs): at most one per iteration, so that no
// unit's range is empty.  When every tile can go to two or more units, each
// tile's k-blocks are split evenly over S of them (S as large as fits and
// divides the k-blocks): every tile then has one head and S - 1 contributors
// that start and finish together, instead of ranges that straddle tiles.
int64_t streamk_units(int64_t tiles, int64_t kb, int64_t units, int *share = nullptr)
{
    if (share) *share = 0;
    if (tiles > 0 && tiles <= units / 2) {
        int64_t S = units / tiles;
        while (S > 1 && kb % S != 0) --S;
        if (S >= 2) {
            if (share) *share = static_cast<int>(S);
            return tiles * S;
        }
    }
    return std::min<int64_t>(tiles * kb, units);
}

void split_costs(int id, int64_t M, int64_t N, int64_t K, int sms, double *dp, double *sk)
{
    const tg_config_t &ci = kConfigs[id].info;
    const int cg = ci.cta_pair ? 2 : 1;
    const int64_t tiles = ceil_div(M, ci.block_m) * ceil_div(N, ci.block_n);
    const int64_t kb = ceil_div(K, ci.block_k);
    const int64_t units = ci.cta_pair ? sms / 2 : sms;
    const double mma_clk = static_cast<double>(ci.block_n) * ci.block_k / 32.0;
    const double load_clk = (128.0 + static_cast<double>(ci.block_n) / cg) * ci.block_k * 2.0 / 64.0;
    const double iter_us = (mma_clk > load_clk ? mma_clk : load_clk) / (kClockGhz * 1e3);
    *dp = static_cast<double>(ceil_div(tiles, units) * kb) * iter_us;
    const int64_t sk_units = streamk_units(tiles, kb, units);
    const double contributors =
        sk_units > tiles ? static_cast<double>(sk_units) / static_cast<double>(tiles) : 1.0;
    const double partial_bytes = 128.0 * ci.block_n * 4.0;
    *sk = static_cast<double>(ceil_div(tiles * kb, sk_units)) * iter_us + kStreamKFixedUs +
          contributors * partial_bytes / (kFoldGBs * 1e3);
}

int rule_split(int id, int64_t M, int64_t N, int64_t K, int epilogue, int sms)
{
    if (epilogue == TG_EPILOGUE_BIAS_SOFTMAX) return TG_SPLIT_TILES;
    double dp, sk;
    split_costs(id, M, N, K, sms, &dp, &sk);
    return sk < 0.8 * dp ? TG_SPLIT_STREAM_K : TG_SPLIT_TILES;
}

// Shapes missing from the table: the cheapest (configuration, split) among
// the general-purpose TMA tiles.  Operands whose rows are not 16-byte aligned
// are repacked for them: on B200 the repacking pass plus TMA is 8 to 20 times
// faster than the plain loader (whose loads are latency-bound), so the plain
// loader runs only when chosen explicitly or by a table row.
Choice rule_choice(int64_t M, int64_t N, int64_t K, int epilogue, int sms)
{
    static const int cands[] = {0, 2, 4, 5};
    const int n_cands = 4;
    Choice best{cands[0], TG_SPLIT_TILES};
    double best_cost = 0;
    bool first = true;
    for (int c = 0; c < n_cands; ++c) {
        const int id = cands[c];
        const int split = rule_split(id, M, N, K, epilogue, sms);
        double dp, sk;
        split_costs(id, M, N, K, sms, &dp, &sk);
        const double cost = split == TG_SPLIT_STREAM_K ? sk : dp;
        if (first || cost < best_cost - 1e-9) {
            best = {id, split};
            best_cost = cost;
            first = false;
        }
    }
    return best;
}

// Softmax rows must fit one tile with whole rows per thread: 4 epilogue
// warps and block_n >= N (N <= 256).
bool softmax_capable(const tg_config_t &c, int64_t N) { return c.epi_warps == 4 && c.block_n >= N; }

// `allow_plain`: a table row may select a plain-loader configuration (not for
// the allocation-free entry point, which keeps its repacking scratch).
Choice choose_config(int64_t M, int64_t N, int64_t K, int epilogue, int num_sms,
                     bool allow_plain = true)
{
    const int sms = num_sms > 1 ? num_sms : 148;
    for (const TableRow &r : kShapeTable)
        if (r.M >= 0 && r.M == M && r.N == N && r.K == K &&
            (r.epilogue < 0 || r.epilogue == epilogue) && r.config >= 0 &&
            r.config < kNumConfigs &&
            (allow_plain || kConfigs[r.config].info.loader == tg::kLoadTma) &&
            (epilogue != TG_EPILOGUE_BIAS_SOFTMAX || softmax_capable(kConfigs[r.config].info, N)))
            return {r.config, (r.split == TG_SPLIT_TILES || r.split == TG_SPLIT_STREAM_K)
                                  ? r.split
                                  : rule_split(r.config, M, N, K, epilogue, sms)};
    if (epilogue == TG_EPILOGUE_BIAS_SOFTMAX) {
        // narrow rows: the 64-column single-CTA tile; otherwise the 256-column
        // CTA pair when it fills the SM pairs, else the 256-column single CTA
        const int id = N <= 64 ? 5 : (ceil_div(M, 256) >= sms / 2 ? 6 : 8);
        return {id, TG_SPLIT_TILES};
    }
    return rule_choice(M, N, K, epilogue, sms);
}

// ------------------------------------------------------------------ devices
struct DeviceState {
    bool init = false;
    tg_status_t status = TG_OK;
    int num_sms = 0;
    unsigned *error_word = nullptr;
    cudaMemPool_t pool = nullptr;
};
DeviceState g_devices[kMaxDevices];
std::mutex g_mutex;

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// Stream-K workspace of one (device, stream): an fp32 128 x 256 partial tile
// per CTA and one completion flag per (CTA, epilogue warp).  Flags hold the
// epoch of the launch that wrote them, so they never need clearing again.
struct StreamKWorkspace {
    float *partials = nullptr;
    unsigned *flags = nullptr;
    unsigned epoch = 0;
};
constexpr int kMaxEpiWarps = 8;
std::map<std::pair<int, cudaStream_t>, StreamKWorkspace> g_streamk;   // under g_mutex

// The workspace for (current device, stream) and a fresh epoch; created on
// first use (cudaMalloc, flags zeroed on `stream`).
tg_status_t streamk_workspace(int num_sms, cudaStream_t stream, float **partials,
                              unsigned **flags, unsigned *epoch)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return TG_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    StreamKWorkspace &w = g_streamk[std::make_pair(dev, stream)];
    if (!w.partials) {
        const size_t part_bytes = static_cast<size_t>(num_sms) * tg::kBlockM * 256 * sizeof(float);
        const size_t flag_bytes = static_cast<size_t>(num_sms) * kMaxEpiWarps * sizeof(unsigned);
        void *mem = nullptr;
        if (cudaMalloc(&mem, part_bytes + flag_bytes) != cudaSuccess) {
            cudaGetLastError();
            g_streamk.erase(std::make_pair(dev, stream));
            return TG_ERR_OOM;
        }
        w.partials = static_cast<float *>(mem);
        w.flags = reinterpret_cast<unsigned *>(static_cast<char *>(mem) + part_bytes);
        if (cudaMemsetAsync(w.flags, 0, flag_bytes, stream) != cudaSuccess) {
            cudaGetLastError();
            return TG_ERR_CUDA;
        }
    }
    if (++w.epoch == 0) w.epoch = 1;
    *partials = w.partials;
    *flags = w.flags;
    *epoch = w.epoch;
    return TG_OK;
}

tg_status_t device_state(DeviceState **out, int *dev_out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return TG_ERR_UNSUPPORTED_DEVICE;
    }
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceState &d = g_devices[dev];
    if (!d.init) {
        d.init = true;
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            major != 10 || minor != 0) {
            d.status = TG_ERR_UNSUPPORTED_DEVICE;
        } else if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) !=
                       cudaSuccess ||
                   cudaGetSymbolAddress(reinterpret_cast<void **>(&d.error_word),
                                        g_tg_error_word) != cudaSuccess) {
            d.status = TG_ERR_CUDA;
        } else {
            // A private stream-ordered pool for repacking temporaries; it
            // keeps freed memory for reuse instead of returning it at every
            // synchronisation.
            cudaMemPoolProps props;
            std::memset(&props, 0, sizeof(props));
            props.allocType = cudaMemAllocationTypePinned;
            props.location.type = cudaMemLocationTypeDevice;
            props.location.id = dev;
            if (cudaMemPoolCreate(&d.pool, &props) != cudaSuccess) {
                d.pool = nullptr;
                d.status = TG_ERR_CUDA;
            } else {
                uint64_t keep = 1ull << 30;
                cudaMemPoolSetAttribute(d.pool, cudaMemPoolAttrReleaseThreshold, &keep);
            }
        }
        if (d.status == TG_OK && !g_encode) {
            cudaDriverEntryPointQueryResult q;
            void *fn = nullptr;
            if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000,
                                                 cudaEnableDefault, &q) != cudaSuccess ||
                q != cudaDriverEntryPointSuccess || !fn)
                d.status = TG_ERR_CUDA;
            else
                g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
        }
        cudaGetLastError();
    }
    *out = &d;
    if (dev_out) *dev_out = dev;
    return d.status;
}

bool encode_2d(CUtensorMap *tm, const void *base, uint64_t inner, uint64_t outer,
               uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_outer,
               CUtensorMapSwizzle swizzle)
{
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {pitch_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool overlaps(const void *a, int64_t a_bytes, const void *b, int64_t b_bytes)
{
    if (!a || !b || a_bytes <= 0 || b_bytes <= 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + static_cast<uintptr_t>(b_bytes) && b0 < a0 + static_cast<uintptr_t>(a_bytes);
}

bool aligned(const void *p, uintptr_t n) { return (reinterpret_cast<uintptr_t>(p) % n) == 0; }

constexpr int64_t kDimLimit = (1ll << 31) - 1;
constexpr int64_t kSoftmaxMaxN = 256;

// Checks that need no device.
tg_status_t validate(const void *A, const void *B, const void *bias, const void *C, int64_t M,
                     int64_t N, int64_t K, int epilogue)
{
    if (epilogue < TG_EPILOGUE_NONE || epilogue > TG_EPILOGUE_BIAS_SOFTMAX) return TG_ERR_INVALID_ARG;
    if (M < 0 || N < 0 || K < 0 || M > kDimLimit || N > kDimLimit || K > kDimLimit)
        return TG_ERR_INVALID_ARG;
    if (epilogue == TG_EPILOGUE_BIAS_SOFTMAX && N > kSoftmaxMaxN) return TG_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return TG_OK;
    if (!C || (K > 0 && (!A || !B))) return TG_ERR_INVALID_ARG;
    if (!aligned(C, 2) || (A && !aligned(A, 2)) || (B && !aligned(B, 2)) ||
        (bias && !aligned(bias, 2)))
        return TG_ERR_MISALIGNED;
    if (ceil_div(M, tg::kBlockM) * ceil_div(N, 64) > kDimLimit) return TG_ERR_INVALID_ARG;
    const int64_t c_bytes = 2 * M * N;
    if (overlaps(C, c_bytes, A, 2 * M * K) || overlaps(C, c_bytes, B, 2 * K * N) ||
        (epilogue != TG_EPILOGUE_NONE && overlaps(C, c_bytes, bias, 2 * N)))
        return TG_ERR_INVALID_ARG;
    return TG_OK;
}

tg_status_t launch_k0(const void *bias, void *C, int64_t M, int64_t N, int epilogue,
                      cudaStream_t stream, int num_sms)
{
    const int64_t total = M * N;
    const int grid = static_cast<int>(std::min<int64_t>(ceil_div(total, 256), 8ll * num_sms));
    const __half *b = static_cast<const __half *>(bias);
    __half *c = static_cast<__half *>(C);
    if (epilogue == TG_EPILOGUE_NONE)
        tg::k0_epilogue_kernel<0><<<grid, 256, 0, stream>>>(b, c, M, N);
    else if (epilogue == TG_EPILOGUE_BIAS)
        tg::k0_epilogue_kernel<1><<<grid, 256, 0, stream>>>(b, c, M, N);
    else if (epilogue == TG_EPILOGUE_BIAS_GELU)
        tg::k0_epilogue_kernel<2><<<grid, 256, 0, stream>>>(b, c, M, N);
    else if (epilogue == TG_EPILOGUE_BIAS_GELU_TANH)
        tg::k0_epilogue_kernel<3><<<grid, 256, 0, stream>>>(b, c, M, N);
    else
        tg::k0_epilogue_kernel<4><<<grid, 256, 0, stream>>>(b, c, M, N);
    return cudaGetLastError() == cudaSuccess ? TG_OK : TG_ERR_LAUNCH;
}

// Thin N remainder: when N = q * BN + r with 0 < r <= kTailMaxCols and the
// last, nearly empty column of tiles would cost the persistent GEMM a whole
// extra wave, the GEMM covers the first q * BN columns and tail_cols_kernel
// the last r on the CUDA cores, alongside the GEMM.  Whole-tile TMA
// configurations only (the tail kernel reads A with 16-byte loads), not the
// row softmax (it needs whole rows).  Measured on 3000 x (1536 + r) x 2048
// (bias + GELU, cold L2): the tail path takes 42.0, 42.1, 48.3, 56.7 and
// 80.9 us for r = 1, 2, 4, 8, 16; the extra wave of whole tiles 50.3 us for
// r = 4 (B repacked, C stored element by element) and 36.9-37.7 us for the
// aligned r = 8, 16.  So r <= 4 goes to the tail (N is then not a multiple
// of 8).
constexpr int kTailMaxCols = 4;

int tail_round(int r) { return r <= 1 ? 1 : r <= 2 ? 2 : 4; }

int tail_cols(const tg_config_t &ci, int64_t M, int64_t N, int64_t K, int epilogue, int split,
              int num_sms)
{
    (void)K;
    if (split == TG_SPLIT_STREAM_K || epilogue == TG_EPILOGUE_BIAS_SOFTMAX ||
        ci.loader != tg::kLoadTma)
        return 0;
    const int64_t r = N % ci.block_n;
    if (r == 0 || r > kTailMaxCols || N < ci.block_n) return 0;
    const int64_t units = ci.cta_pair ? num_sms / 2 : num_sms;
    const int64_t m_tiles = ceil_div(M, ci.block_m);
    const int64_t waves_all = ceil_div(m_tiles * ceil_div(N, ci.block_n), units);
    const int64_t waves_main = ceil_div(m_tiles * (N / ci.block_n), units);
    return waves_main < waves_all ? static_cast<int>(r) : 0;
}

// The tail kernel's launch: programmatic stream serialisation, so that it may
// start while the GEMM before it runs (the GEMM allows it once its CTAs are
// resident; the tail waits for the GEMM's completion at its end).
struct TailArgs {
    const __half *A, *slab;
    int64_t ld;
    const __half *bias;
    __half *C;
    int64_t ldc, M, n0;
    int r;
    unsigned long long *next_row;
};

template <int EPI, int RT>
cudaError_t launch_tail_kernel(const TailArgs &t, int grid, cudaStream_t stream)
{
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.blockDim = dim3(tg::kTailThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, tg::tail_cols_kernel<EPI, RT>, t.A, t.slab, t.ld, t.bias, t.C,
                              t.ldc, t.M, t.n0, t.r, t.next_row);
}

template <int EPI>
cudaError_t launch_tail_epi(const TailArgs &t, int grid, cudaStream_t stream)
{
    switch (tail_round(t.r)) {
    case 1: return launch_tail_kernel<EPI, 1>(t, grid, stream);
    case 2: return launch_tail_kernel<EPI, 2>(t, grid, stream);
    default: return launch_tail_kernel<EPI, 4>(t, grid, stream);
    }
}

// The tail kernel's blocks share SMs with the GEMM's CTAs, which take nearly
// all of the shared memory: an SM runs blocks of one shared-memory
// configuration at a time, so the tail kernels ask for the largest carveout
// too (once per device), else they would run only on SMs without a GEMM CTA.
template <int EPI>
cudaError_t tail_carveout_epi()
{
    cudaError_t e = cudaSuccess;
    auto set = [&](auto kern) {
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                     static_cast<int>(cudaSharedmemCarveoutMaxShared));
    };
    set(tg::tail_cols_kernel<EPI, 1>);
    set(tg::tail_cols_kernel<EPI, 2>);
    set(tg::tail_cols_kernel<EPI, 4>);
    return e;
}

tg_status_t tail_carveout()
{
    static std::atomic<uint64_t> attr_set{0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return TG_ERR_CUDA;
    }
    const uint64_t bit = dev < 64 ? (1ull << dev) : 0;
    if (bit && (attr_set.load() & bit)) return TG_OK;
    if (tail_carveout_epi<0>() != cudaSuccess || tail_carveout_epi<1>() != cudaSuccess ||
        tail_carveout_epi<2>() != cudaSuccess || tail_carveout_epi<3>() != cudaSuccess) {
        cudaGetLastError();
        return TG_ERR_CUDA;
    }
    attr_set.fetch_or(bit);
    return TG_OK;
}

tg_status_t launch_tail(const TailArgs &t, int epilogue, int num_sms, cudaStream_t stream)
{
    const tg_status_t st = tail_carveout();
    if (st != TG_OK) return st;
    // one warp per row, up to eight two-warp blocks per SM in the grid
    const int grid = static_cast<int>(std::min<int64_t>(ceil_div(t.M, 2), 8ll * num_sms));
    cudaError_t e;
    if (epilogue == TG_EPILOGUE_NONE)
        e = launch_tail_epi<0>(t, grid, stream);
    else if (epilogue == TG_EPILOGUE_BIAS)
        e = launch_tail_epi<1>(t, grid, stream);
    else if (epilogue == TG_EPILOGUE_BIAS_GELU)
        e = launch_tail_epi<2>(t, grid, stream);
    else
        e = launch_tail_epi<3>(t, grid, stream);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return TG_ERR_LAUNCH;
    }
    return TG_OK;
}

// A repacking job for an operand of rows x cols at src into dst with pitch
// ld_dst, or an empty job when src is null.
tg::PackJob pack_job(const void *src, int64_t rows, int64_t cols, void *dst, int64_t ld_dst)
{
    tg::PackJob j;
    j.src = static_cast<const __half *>(src);
    j.dst = static_cast<__half *>(dst);
    j.cols = cols;
    j.ld_dst = ld_dst;
    j.groups_per_row = static_cast<uint32_t>(ld_dst / 8);
    j.groups = src ? static_cast<uint64_t>(rows) * static_cast<uint64_t>(ld_dst / 8) : 0;
    return j;
}

// Where a GEMM's operands come from: the operands as the GEMM reads them and
// the tail's columns and slab.
struct Staging {
    const void *A = nullptr, *B = nullptr;
    int64_t lda = 0, ldb = 0;
    int tail = 0;                      // thin remainder columns (0: none)
    __half *slab = nullptr;            // tail: B's last columns, r rows of lda
    unsigned long long *next_row = nullptr;   // tail: its row counter
};

// Bytes of scratch a call needs: A and B repacked (when not 16-byte
// addressable) and the tail's slab and row counter, each part 256-byte
// aligned.
struct ScratchPlan {
    size_t a_off = 0, b_off = 0, slab_off = 0, counter_off = 0, bytes = 0;
};

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

ScratchPlan scratch_plan(bool a_direct, bool b_direct, int64_t M, int64_t N, int64_t K, int tail)
{
    ScratchPlan s;
    const int64_t lda = a_direct ? K : (K + 7) / 8 * 8;
    const int64_t ldb = b_direct ? N : (N + 7) / 8 * 8;
    s.a_off = 0;
    s.b_off = s.a_off + round256(a_direct ? 0 : static_cast<size_t>(2 * M * lda));
    s.slab_off = s.b_off + round256(b_direct ? 0 : static_cast<size_t>(2 * K * ldb));
    s.counter_off = s.slab_off + round256(static_cast<size_t>(2 * tail * lda));
    s.bytes = s.counter_off + (tail > 0 ? 256 : 0);
    return s;
}

// The repacking pre-pass: one launch makes every copy a call needs (the
// repacked operands and the tail's slab) before the GEMM: up to eight
// 256-thread blocks per SM, each thread kPackGroups 16-byte groups per step.
tg_status_t launch_pack(const tg::PackJob &a, const tg::PackJob &b, const tg::SlabJob &sl,
                        int num_sms, cudaStream_t stream)
{
    const uint64_t total = a.groups + b.groups + sl.groups;
    if (total == 0) return TG_OK;
    const uint64_t per_block = 256ull * tg::kPackGroups;
    const int grid = static_cast<int>(std::min<uint64_t>((total + per_block - 1) / per_block,
                                                         8ull * static_cast<uint64_t>(num_sms)));
    tg::pack_pad2_kernel<<<grid, 256, 0, stream>>>(a, b, sl);
    return cudaGetLastError() == cudaSuccess ? TG_OK : TG_ERR_LAUNCH;
}

// Repacking scratch of one (device, stream), kept from call to call: the
// calls on one stream are ordered by it, so each may reuse the same bytes,
// and a call saves the stream-ordered allocation and release of its own
// (about 2 µs on a 3000 x 1537 x 2050 call).  It grows, stream-ordered, when a
// call needs more.  Calls that need more than kCachedScratchMax, and calls
// while the stream is capturing a graph, take a pool allocation of their own.
constexpr size_t kCachedScratchMax = 64ull << 20;
struct CachedScratch {
    void *ptr = nullptr;
    size_t bytes = 0;
};
std::map<std::pair<int, cudaStream_t>, CachedScratch> g_scratch;   // under g_mutex

tg_status_t cached_scratch(cudaMemPool_t pool, cudaStream_t stream, size_t bytes, void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return TG_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(g_mutex);
    CachedScratch &c = g_scratch[std::make_pair(dev, stream)];
    if (c.bytes < bytes) {
        if (c.ptr) cudaFreeAsync(c.ptr, stream);
        c.ptr = nullptr;
        c.bytes = 0;
        void *p = nullptr;
        if (cudaMallocFromPoolAsync(&p, bytes, pool, stream) != cudaSuccess) {
            cudaGetLastError();
            return TG_ERR_OOM;
        }
        c.ptr = p;
        c.bytes = bytes;
    }
    *out = c.ptr;
    return TG_OK;
}

// Fills in where the GEMM reads its operands and launches the repacking
// pre-pass a call needs (repacked operands and the tail's slab, in `scratch`
// as `plan` lays them out), if any.
tg_status_t stage_operands(const void *A, const void *B, int64_t M, int64_t N, int64_t K,
                           bool a_direct, bool b_direct, const ScratchPlan &plan,
                           unsigned char *scratch, int num_sms, cudaStream_t stream, Staging *sg)
{
    sg->lda = a_direct ? K : (K + 7) / 8 * 8;
    sg->ldb = b_direct ? N : (N + 7) / 8 * 8;
    sg->A = a_direct ? A : scratch + plan.a_off;
    sg->B = b_direct ? B : scratch + plan.b_off;
    sg->slab = sg->tail > 0 ? reinterpret_cast<__half *>(scratch + plan.slab_off) : nullptr;
    sg->next_row = sg->tail > 0 ? reinterpret_cast<unsigned long long *>(scratch + plan.counter_off)
                                : nullptr;
    if (plan.bytes == 0) return TG_OK;
    const tg::PackJob ja = pack_job(a_direct ? nullptr : A, M, K, scratch + plan.a_off, sg->lda);
    const tg::PackJob jb = pack_job(b_direct ? nullptr : B, K, N, scratch + plan.b_off, sg->ldb);
    tg::SlabJob js;
    js.src = static_cast<const __half *>(B);
    js.dst = sg->slab;
    js.ldb = N;
    js.n0 = N - sg->tail;
    js.K = K;
    js.ld_slab = sg->lda;
    js.groups = static_cast<uint64_t>(sg->tail) * static_cast<uint64_t>(sg->lda / 8);
    js.next_row = sg->next_row;
    return launch_pack(ja, jb, js, num_sms, stream);
}

// Tensor maps, kernel parameters, work division and launch of the GEMM on
// operands already in a form the configuration can read (TMA: 16-byte
// aligned bases and pitches lda, ldb; the plain loader: any 2-byte aligned
// pitch).  Shared by tg_gemm and tg_gemm_noalloc, which differ only in where
// repacked operands live.  `split` is TG_SPLIT_TILES or TG_SPLIT_STREAM_K;
// stream-K takes the (device, stream) workspace.
tg_status_t launch_staged(const KernelConfig &cfg, const Staging &sg, const void *bias, void *C,
                          int64_t M, int64_t N, int64_t K, int epilogue, int split,
                          const tg_options_t *opts, int num_sms, unsigned *error_word,
                          cudaStream_t stream)
{
    const void *Aeff = sg.A, *Beff = sg.B;
    const int64_t lda = sg.lda, ldb = sg.ldb;
    const bool plain = cfg.info.loader == tg::kLoadPlain;
    const bool c_rows16 = aligned(C, 16) && (N % 8 == 0);
    const int store = c_rows16 ? cfg.store_pref : tg::kStoreScalar;
    // The GEMM covers columns [0, n_main); a thin remainder goes to the tail kernel.
    const int tail = sg.tail;
    const int64_t n_main = N - tail;
    CUtensorMap ta, tb, tc;
    std::memset(&ta, 0, sizeof(ta));
    std::memset(&tb, 0, sizeof(tb));
    std::memset(&tc, 0, sizeof(tc));
    if ((!plain && (!encode_2d(&ta, Aeff, K, M, 2 * lda, tg::kAtomK, tg::kBlockM,
                               CU_TENSOR_MAP_SWIZZLE_128B) ||
                    !encode_2d(&tb, Beff, n_main, K, 2 * ldb, tg::kBChunkN, cfg.info.block_k,
                               CU_TENSOR_MAP_SWIZZLE_128B))) ||
        (store == tg::kStoreTma &&
         !encode_2d(&tc, C, n_main, M, 2 * N, tg::kStoreCols, 32, CU_TENSOR_MAP_SWIZZLE_64B)))
        return TG_ERR_CUDA;

    tg::GemmParams p;
    p.A = static_cast<const __half *>(Aeff);
    p.B = static_cast<const __half *>(Beff);
    p.lda = lda;
    p.ldb = ldb;
    p.bias = static_cast<const __half *>(bias);
    p.C = static_cast<__half *>(C);
    p.M = M;
    p.N = n_main;
    p.K = K;
    p.ldc = N;
    p.num_m_tiles = static_cast<int>(ceil_div(M, cfg.info.block_m));
    p.num_n_tiles = static_cast<int>(ceil_div(n_main, cfg.info.block_n));
    p.num_k_blocks = static_cast<int>(ceil_div(K, cfg.info.block_k));
    p.num_tiles = p.num_m_tiles * p.num_n_tiles;
    p.group_m = (opts && opts->group_m > 0) ? opts->group_m : cfg.info.group_m;
    p.inject = opts ? opts->inject : 0;
    p.bias_vec = (bias && aligned(bias, 16)) ? 1 : 0;
    p.wait_limit_ns = (opts && opts->wait_limit_ns) ? opts->wait_limit_ns : kDefaultWaitLimitNs;
    p.error_word = error_word;
    p.early_trigger = tail > 0 ? 1 : 0;
    // Persistent grid: one CTA (or CTA pair) per SM (pair of SMs).  Whole
    // tiles: never more units than tiles; stream-K: streamk_units.
    const int units = cfg.info.cta_pair ? num_sms / 2 : num_sms;
    const bool stream_k = split == TG_SPLIT_STREAM_K;
    p.stream_k = stream_k ? 1 : 0;
    p.sk_partials = nullptr;
    p.sk_flags = nullptr;
    p.sk_epoch = 0;
    if (stream_k) {
        const tg_status_t st =
            streamk_workspace(num_sms, stream, &p.sk_partials, &p.sk_flags, &p.sk_epoch);
        if (st != TG_OK) return st;
    }
    // An even stream-K split shares each tile's fold among its units (not for
    // the row softmax, whose epilogue needs whole rows).
    int share = 0;
    const int grid =
        static_cast<int>(stream_k ? streamk_units(p.num_tiles, p.num_k_blocks, units, &share)
                                  : std::min<int64_t>(p.num_tiles, units)) *
        (cfg.info.cta_pair ? 2 : 1);
    p.sk_share = (stream_k && epilogue != TG_EPILOGUE_BIAS_SOFTMAX) ? share : 0;

    LaunchFn fn = cfg.fn[epilogue][store == tg::kStoreScalar ? 0 : 1];
    if (p.sk_share > 0) {
        // The shared-fold variant exists for the preferred store mode only;
        // otherwise the tile's first unit folds alone.
        LaunchFn shared = store == tg::kStoreScalar ? nullptr : cfg.fn_share[epilogue];
        if (shared)
            fn = shared;
        else
            p.sk_share = 0;
    }
    const cudaError_t e = fn(ta, tb, tc, p, grid, stream);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return TG_ERR_LAUNCH;
    }
    if (tail > 0) {
        TailArgs t;
        t.A = static_cast<const __half *>(Aeff);
        t.slab = sg.slab;
        t.ld = lda;
        t.bias = static_cast<const __half *>(bias);
        t.C = static_cast<__half *>(C);
        t.ldc = N;
        t.M = M;
        t.n0 = n_main;
        t.r = tail;
        t.next_row = sg.next_row;
        return launch_tail(t, epilogue, num_sms, stream);
    }
    return TG_OK;
}

tg_status_t gemm_impl(const void *A, const void *B, const void *bias, void *C, int64_t M,
                      int64_t N, int64_t K, int epilogue, const tg_options_t *opts,
                      cudaStream_t stream)
{
    tg_status_t st = validate(A, B, bias, C, M, N, K, epilogue);
    if (st != TG_OK || M == 0 || N == 0) return st;
    if (opts && (opts->config_id < -1 || opts->config_id >= kNumConfigs)) return TG_ERR_INVALID_ARG;
    if (opts && (opts->inject != 0 && opts->inject != TG_INJECT_SKIP_FIRST_LOAD &&
                 opts->inject != TG_INJECT_SKIP_STREAMK_FLAGS))
        return TG_ERR_INVALID_ARG;
    if (opts && (opts->split < TG_SPLIT_AUTO || opts->split > TG_SPLIT_STREAM_K))
        return TG_ERR_INVALID_ARG;
    if (opts && (opts->group_m < 0 || opts->group_m > 64)) return TG_ERR_INVALID_ARG;
    DeviceState *dev = nullptr;
    st = device_state(&dev, nullptr);
    if (st != TG_OK) return st;
    if (epilogue == TG_EPILOGUE_NONE) bias = nullptr;
    if (K == 0) return launch_k0(bias, C, M, N, epilogue, stream, dev->num_sms);

    // TMA needs 16-byte aligned bases and pitches; otherwise repack, or load
    // with the plain loader.
    const bool a_aligned = aligned(A, 16) && (K % 8 == 0);
    const bool b_aligned = aligned(B, 16) && (N % 8 == 0);
    Choice choice{0, TG_SPLIT_TILES};
    if (opts && opts->config_id >= 0)
        choice = {opts->config_id, rule_split(opts->config_id, M, N, K, epilogue, dev->num_sms)};
    else
        choice = choose_config(M, N, K, epilogue, dev->num_sms);
    if (opts && opts->split != TG_SPLIT_AUTO) choice.split = opts->split;
    // Stream-K flags hold a per-call epoch, which a replayed graph would
    // repeat: whole tiles while the stream is capturing.
    const bool capturing = tg_internal_capturing(stream);
    if (capturing) {
        if (opts && opts->split == TG_SPLIT_STREAM_K) return TG_ERR_INVALID_ARG;
        choice.split = TG_SPLIT_TILES;
    }
    const int cfg_id = choice.config;
    const KernelConfig &cfg = kConfigs[cfg_id];
    if (epilogue == TG_EPILOGUE_BIAS_SOFTMAX && !softmax_capable(cfg.info, N))
        return TG_ERR_INVALID_ARG;
    const bool plain = cfg.info.loader == tg::kLoadPlain;
    const bool a_direct = plain || a_aligned;
    const bool b_direct = plain || b_aligned;
    Staging sg;
    sg.tail = tail_cols(cfg.info, M, N, K, epilogue, choice.split, dev->num_sms);
    const ScratchPlan plan = scratch_plan(a_direct, b_direct, M, N, K, sg.tail);
    void *tmp = nullptr;      // a pool allocation of this call's own, freed after it
    void *scratch = nullptr;
    if (plan.bytes > 0) {
        if (!capturing && plan.bytes <= kCachedScratchMax) {
            st = cached_scratch(dev->pool, stream, plan.bytes, &scratch);
            if (st != TG_OK) return st;
        } else {
            if (cudaMallocFromPoolAsync(&tmp, plan.bytes, dev->pool, stream) != cudaSuccess) {
                cudaGetLastError();
                return TG_ERR_OOM;
            }
            scratch = tmp;
        }
        st = stage_operands(A, B, M, N, K, a_direct, b_direct, plan,
                            static_cast<unsigned char *>(scratch), dev->num_sms, stream, &sg);
    } else {
        st = stage_operands(A, B, M, N, K, true, true, plan, nullptr, dev->num_sms, stream, &sg);
    }
    if (st == TG_OK)
        st = launch_staged(cfg, sg, bias, C, M, N, K, epilogue, choice.split, opts, dev->num_sms,
                           dev->error_word, stream);
    if (tmp) cudaFreeAsync(tmp, stream);
    return st;
}

// The end-to-end entry point overlaps its copies with the GEMM: B (and the
// bias) go up first, then A in row panels on an internal copy-in stream;
// panel i's GEMM runs on the caller's stream as soon as its rows have
// arrived, and its rows of C go down on an internal copy-out stream while the
// next panels are uploaded and computed.  Streams and events are created once
// per (device, caller stream) and reused; everything joins back into the
// caller's stream before the call returns.
// Panels of about kHostPanelRows rows (at most kMaxPanelsEqual), the last one
// halved: what is left after the final upload (that panel's GEMM and its
// download) is then a short tail.
constexpr int kMaxPanelsEqual = 16;
constexpr int kMaxHostPanels = kMaxPanelsEqual + 1;
constexpr int64_t kHostPanelRows = 1024;

// Row boundaries of the panels: edge[0] = 0 < edge[1] < ... < edge[n] = M.
int host_panels(int64_t M, int64_t (&edge)[kMaxHostPanels + 1])
{
    const int64_t n = std::min<int64_t>(kMaxPanelsEqual, std::max<int64_t>(1, ceil_div(M, kHostPanelRows)));
    const int64_t rows = ceil_div(M, n);
    int k = 0;
    edge[0] = 0;
    for (int64_t r = 0; r < M; r += rows) edge[++k] = std::min<int64_t>(M, r + rows);
    const int64_t last = edge[k] - edge[k - 1];
    if (k >= 2 && last >= 256) {
        edge[k + 1] = edge[k];
        edge[k] = edge[k - 1] + last / 2;
        ++k;
    }
    return k;
}

struct HostPipe {
    cudaStream_t in = nullptr, out = nullptr;
    cudaEvent_t entry = nullptr, b_ready = nullptr, out_done = nullptr;
    cudaEvent_t a_ready[kMaxHostPanels] = {}, c_ready[kMaxHostPanels] = {};
};
std::map<std::pair<int, cudaStream_t>, HostPipe> g_host_pipes;

tg_status_t host_pipe(cudaStream_t caller, HostPipe **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return TG_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(g_mutex);
    auto it = g_host_pipes.find(std::make_pair(dev, caller));
    if (it != g_host_pipes.end()) {
        *out = &it->second;
        return TG_OK;
    }
    HostPipe hp;
    bool ok = cudaStreamCreateWithFlags(&hp.in, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&hp.out, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&hp.entry, cudaEventDisableTiming) == cudaSuccess &&
              cudaEventCreateWithFlags(&hp.b_ready, cudaEventDisableTiming) == cudaSuccess &&
              cudaEventCreateWithFlags(&hp.out_done, cudaEventDisableTiming) == cudaSuccess;
    for (int i = 0; ok && i < kMaxHostPanels; ++i)
        ok = cudaEventCreateWithFlags(&hp.a_ready[i], cudaEventDisableTiming) == cudaSuccess &&
             cudaEventCreateWithFlags(&hp.c_ready[i], cudaEventDisableTiming) == cudaSuccess;
    if (!ok) {
        cudaGetLastError();
        return TG_ERR_CUDA;
    }
    *out = &(g_host_pipes[std::make_pair(dev, caller)] = hp);
    return TG_OK;
}

}  // namespace

tg_status_t tg_internal_device(int *num_sms, unsigned **error_word,
                               PFN_cuTensorMapEncodeTiled_v12000 *encode)
{
    DeviceState *dev = nullptr;
    const tg_status_t st = device_state(&dev, nullptr);
    if (st != TG_OK) return st;
    *num_sms = dev->num_sms;
    *error_word = dev->error_word;
    *encode = g_encode;
    return g_encode ? TG_OK : TG_ERR_CUDA;
}

extern "C" {

tg_status_t tg_gemm(const void *A, const void *B, const void *bias, void *C, int64_t M, int64_t N,
                    int64_t K, int epilogue, void *stream)
{
    return gemm_impl(A, B, bias, C, M, N, K, epilogue, nullptr,
                     static_cast<cudaStream_t>(stream));
}

tg_status_t tg_gemm_ex(const void *A, const void *B, const void *bias, void *C, int64_t M,
                       int64_t N, int64_t K, int epilogue, const tg_options_t *opts, void *stream)
{
    return gemm_impl(A, B, bias, C, M, N, K, epilogue, opts, static_cast<cudaStream_t>(stream));
}

int tg_num_configs(void) { return kNumConfigs; }

tg_status_t tg_config_info(int id, tg_config_t *out)
{
    if (!out || id < 0 || id >= kNumConfigs) return TG_ERR_INVALID_ARG;
    *out = kConfigs[id].info;
    return TG_OK;
}

tg_status_t tg_gemm_select_config(int64_t M, int64_t N, int64_t K, int epilogue, int num_sms,
                                  tg_config_t *out)
{
    if (!out || M < 0 || N < 0 || K < 0 || epilogue < TG_EPILOGUE_NONE ||
        epilogue > TG_EPILOGUE_BIAS_SOFTMAX || num_sms <= 0 ||
        (epilogue == TG_EPILOGUE_BIAS_SOFTMAX && N > kSoftmaxMaxN))
        return TG_ERR_INVALID_ARG;
    const Choice c = choose_config(M, N, K, epilogue, num_sms);
    *out = kConfigs[c.config].info;
    out->split = c.split;
    return TG_OK;
}

size_t tg_gemm_host_workspace_size(int64_t M, int64_t N, int64_t K, int has_bias)
{
    if (M < 0 || N < 0 || K < 0) return 0;
    return round256(2 * static_cast<size_t>(M * K)) + round256(2 * static_cast<size_t>(K * N)) +
           round256(has_bias ? 2 * static_cast<size_t>(N) : 0) +
           round256(2 * static_cast<size_t>(M * N));
}

tg_status_t tg_gemm_host(const void *A_host, const void *B_host, const void *bias_host,
                         void *C_host, int64_t M, int64_t N, int64_t K, int epilogue,
                         void *workspace, size_t workspace_bytes, void *stream)
{
    tg_status_t st = validate(A_host, B_host, bias_host, C_host, M, N, K, epilogue);
    if (st != TG_OK || M == 0 || N == 0) return st;
    const bool has_bias = bias_host != nullptr && epilogue != TG_EPILOGUE_NONE;
    if (!workspace || !aligned(workspace, 256) ||
        workspace_bytes < tg_gemm_host_workspace_size(M, N, K, has_bias ? 1 : 0))
        return TG_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    char *w = static_cast<char *>(workspace);
    const size_t a_bytes = 2 * static_cast<size_t>(M * K), b_bytes = 2 * static_cast<size_t>(K * N);
    const size_t bias_bytes = has_bias ? 2 * static_cast<size_t>(N) : 0;
    char *dA = w;
    char *dB = dA + round256(a_bytes);
    char *dbias = dB + round256(b_bytes);
    char *dC = dbias + round256(bias_bytes);
    HostPipe *hp = nullptr;
    st = host_pipe(s, &hp);
    if (st != TG_OK) return st;
    int64_t edge[kMaxHostPanels + 1];
    const int panels = host_panels(M, edge);
    const char *Ah = static_cast<const char *>(A_host);
    char *Ch = static_cast<char *>(C_host);
    bool ok = cudaEventRecord(hp->entry, s) == cudaSuccess &&
              cudaStreamWaitEvent(hp->in, hp->entry, 0) == cudaSuccess &&
              cudaStreamWaitEvent(hp->out, hp->entry, 0) == cudaSuccess;
    // Up: bias and B, then the panels of A.
    ok = ok &&
         (!bias_bytes || cudaMemcpyAsync(dbias, bias_host, bias_bytes, cudaMemcpyHostToDevice,
                                         hp->in) == cudaSuccess) &&
         (!b_bytes ||
          cudaMemcpyAsync(dB, B_host, b_bytes, cudaMemcpyHostToDevice, hp->in) == cudaSuccess) &&
         cudaEventRecord(hp->b_ready, hp->in) == cudaSuccess;
    for (int i = 0; ok && i < panels; ++i) {
        const int64_t r0 = edge[i], r1 = edge[i + 1];
        const size_t off = 2 * static_cast<size_t>(r0 * K), len = 2 * static_cast<size_t>((r1 - r0) * K);
        ok = (!len || cudaMemcpyAsync(dA + off, Ah + off, len, cudaMemcpyHostToDevice, hp->in) ==
                          cudaSuccess) &&
             cudaEventRecord(hp->a_ready[i], hp->in) == cudaSuccess;
    }
    // Compute: each panel once its rows are up.
    ok = ok && cudaStreamWaitEvent(s, hp->b_ready, 0) == cudaSuccess;
    for (int i = 0; ok && i < panels; ++i) {
        const int64_t r0 = edge[i], r1 = edge[i + 1];
        ok = cudaStreamWaitEvent(s, hp->a_ready[i], 0) == cudaSuccess;
        if (!ok) break;
        if (r1 > r0) {
            st = gemm_impl(dA + 2 * static_cast<size_t>(r0 * K), dB, has_bias ? dbias : nullptr,
                           dC + 2 * static_cast<size_t>(r0 * N), r1 - r0, N, K, epilogue, nullptr,
                           s);
            if (st != TG_OK) break;
        }
        ok = cudaEventRecord(hp->c_ready[i], s) == cudaSuccess;
    }
    // Down: each panel of C once computed.
    for (int i = 0; ok && st == TG_OK && i < panels; ++i) {
        const int64_t r0 = edge[i], r1 = edge[i + 1];
        const size_t off = 2 * static_cast<size_t>(r0 * N), len = 2 * static_cast<size_t>((r1 - r0) * N);
        ok = cudaStreamWaitEvent(hp->out, hp->c_ready[i], 0) == cudaSuccess &&
             (!len || cudaMemcpyAsync(Ch + off, dC + off, len, cudaMemcpyDeviceToHost, hp->out) ==
                          cudaSuccess);
    }
    // Join both internal streams back into the caller's stream, whatever happened.
    const bool joined = cudaEventRecord(hp->out_done, hp->out) == cudaSuccess &&
                        cudaStreamWaitEvent(s, hp->out_done, 0) == cudaSuccess &&
                        cudaEventRecord(hp->b_ready, hp->in) == cudaSuccess &&
                        cudaStreamWaitEvent(s, hp->b_ready, 0) == cudaSuccess;
    if (st != TG_OK) return st;
    if (!ok || !joined) {
        cudaGetLastError();
        return TG_ERR_CUDA;
    }
    return TG_OK;
}

int tg_gemm_launch_count(const void *A, const void *B, const void *bias, const void *C,
                         int64_t M, int64_t N, int64_t K, int epilogue)
{
    if (validate(A, B, bias, C, M, N, K, epilogue) != TG_OK) return -1;
    if (M == 0 || N == 0) return 0;
    if (K == 0) return 1;
    const Choice c = choose_config(M, N, K, epilogue, 148);
    const tg_config_t &ci = kConfigs[c.config].info;
    if (ci.loader == tg::kLoadPlain) return 1;
    const bool a_direct = aligned(A, 16) && (K % 8 == 0);
    const bool b_direct = aligned(B, 16) && (N % 8 == 0);
    const int tail = tail_cols(ci, M, N, K, epilogue, c.split, 148);
    // the GEMM, one repacking pass (operands or the tail's slab), the tail
    return 1 + ((a_direct && b_direct && tail == 0) ? 0 : 1) + (tail > 0 ? 1 : 0);
}

tg_status_t tg_gemm_check_error(void *stream)
{
    DeviceState *dev = nullptr;
    tg_status_t st = device_state(&dev, nullptr);
    if (st != TG_OK) return st;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) {
        cudaGetLastError();
        return TG_ERR_CUDA;
    }
    unsigned word = 0;
    if (cudaMemcpy(&word, dev->error_word, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) {
        cudaGetLastError();
        return TG_ERR_CUDA;
    }
    if (word) {
        const unsigned zero = 0;
        cudaMemcpy(dev->error_word, &zero, sizeof(zero), cudaMemcpyHostToDevice);
        return TG_ERR_TIMEOUT;
    }
    return TG_OK;
}

const char *tg_status_string(int status)
{
    switch (status) {
    case TG_OK: return "TG_OK";
    case TG_ERR_INVALID_ARG: return "TG_ERR_INVALID_ARG: invalid argument";
    case TG_ERR_MISALIGNED: return "TG_ERR_MISALIGNED: pointer not 2-byte aligned";
    case TG_ERR_UNSUPPORTED_DEVICE: return "TG_ERR_UNSUPPORTED_DEVICE: needs an sm_100 GPU";
    case TG_ERR_LAUNCH: return "TG_ERR_LAUNCH: kernel launch failed";
    case TG_ERR_TIMEOUT: return "TG_ERR_TIMEOUT: a device-side wait expired";
    case TG_ERR_OOM: return "TG_ERR_OOM: temporary allocation failed";
    case TG_ERR_CUDA: return "TG_ERR_CUDA: CUDA runtime error";
    case TG_ERR_SCRATCH_LIMIT:
        return "TG_ERR_SCRATCH_LIMIT: tg_gemm_noalloc needs more repacking scratch than "
               "TG_NOALLOC_SCRATCH_BYTES";
    default: return "unknown tg_status_t";
    }
}

int tg_version(void) { return 100; }

}  // extern "C"

// ---------------------------------------------------------------------------
// tg_gemm_noalloc: the same GEMM with the repacking scratch taken from a fixed
// file-scope device array instead of a memory pool.  Nothing here allocates.

static __device__ __align__(256) unsigned char g_tg_noalloc_scratch[TG_NOALLOC_SCRATCH_BYTES];

namespace {

struct NoallocDevice {
    bool init = false;
    tg_status_t status = TG_OK;
    int num_sms = 0;
    unsigned *error_word = nullptr;
    unsigned char *scratch = nullptr;   // device address of g_tg_noalloc_scratch
};
NoallocDevice g_noalloc_devices[kMaxDevices];

// One-time set-up per device, with that device current: the device checks
// of device_state() (without its memory pool) plus the device addresses of
// the error word and of the scratch array.  In host code the array's name is
// only a host-side stand-in; cudaGetSymbolAddress gives the address to pass.
tg_status_t noalloc_device(NoallocDevice **out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return TG_ERR_UNSUPPORTED_DEVICE;
    }
    std::lock_guard<std::mutex> lock(g_mutex);
    NoallocDevice &d = g_noalloc_devices[dev];
    if (!d.init) {
        d.init = true;
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            major != 10 || minor != 0) {
            d.status = TG_ERR_UNSUPPORTED_DEVICE;
        } else if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) !=
                       cudaSuccess ||
                   cudaGetSymbolAddress(reinterpret_cast<void **>(&d.error_word),
                                        g_tg_error_word) != cudaSuccess ||
                   cudaGetSymbolAddress(reinterpret_cast<void **>(&d.scratch),
                                        g_tg_noalloc_scratch) != cudaSuccess ||
                   !d.scratch) {
            d.status = TG_ERR_CUDA;
        }
        if (d.status == TG_OK && !g_encode) {
            cudaDriverEntryPointQueryResult q;
            void *fn = nullptr;
            if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000,
                                                 cudaEnableDefault, &q) != cudaSuccess ||
                q != cudaDriverEntryPointSuccess || !fn)
                d.status = TG_ERR_CUDA;
            else
                g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
        }
        cudaGetLastError();
    }
    *out = &d;
    return d.status;
}

tg_status_t gemm_noalloc_impl(const void *A, const void *B, const void *bias, void *C, int64_t M,
                              int64_t N, int64_t K, int epilogue, cudaStream_t stream)
{
    tg_status_t st = validate(A, B, bias, C, M, N, K, epilogue);
    if (st != TG_OK || M == 0 || N == 0) return st;
    // Scratch needed by the repacking step, checked before any device call.
    const bool a_direct = aligned(A, 16) && (K % 8 == 0);
    const bool b_direct = aligned(B, 16) && (N % 8 == 0);
    const Choice choice = K == 0 ? Choice{0, TG_SPLIT_TILES} : choose_config(M, N, K, epilogue, 148, false);
    const int tail = K == 0 ? 0 : tail_cols(kConfigs[choice.config].info, M, N, K, epilogue,
                                            TG_SPLIT_TILES, 148);
    if (K > 0 && scratch_plan(a_direct, b_direct, M, N, K, tail).bytes >
                     static_cast<size_t>(TG_NOALLOC_SCRATCH_BYTES))
        return TG_ERR_SCRATCH_LIMIT;

    NoallocDevice *dev = nullptr;
    st = noalloc_device(&dev);
    if (st != TG_OK) return st;
    if (epilogue == TG_EPILOGUE_NONE) bias = nullptr;
    if (K == 0) return launch_k0(bias, C, M, N, epilogue, stream, dev->num_sms);

    const int cfg_id =
        choose_config(M, N, K, epilogue, dev->num_sms, false).config;
    const KernelConfig &cfg = kConfigs[cfg_id];
    // stream-K needs a workspace; this entry point allocates nothing
    Staging sg;
    sg.tail = tail_cols(cfg.info, M, N, K, epilogue, TG_SPLIT_TILES, dev->num_sms);
    const ScratchPlan plan = scratch_plan(a_direct, b_direct, M, N, K, sg.tail);
    if (plan.bytes > static_cast<size_t>(TG_NOALLOC_SCRATCH_BYTES)) return TG_ERR_SCRATCH_LIMIT;
    st = stage_operands(A, B, M, N, K, a_direct, b_direct, plan, dev->scratch, dev->num_sms,
                        stream, &sg);
    if (st != TG_OK) return st;
    return launch_staged(cfg, sg, bias, C, M, N, K, epilogue, TG_SPLIT_TILES, nullptr,
                         dev->num_sms, dev->error_word, stream);
}

}  // namespace

extern "C" tg_status_t tg_gemm_noalloc(const void *A, const void *B, const void *bias, void *C,
                                       int64_t M, int64_t N, int64_t K, int epilogue,
                                       void *stream)
{
    return gemm_noalloc_impl(A, B, bias, C, M, N, K, epilogue, static_cast<cudaStream_t>(stream));
}
