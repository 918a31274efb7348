// tg_kernels.cuh -- sm_100a kernels of the fused fp16 GEMM.
//
//   gemm_persistent_kernel  C = g(A.B + beta) with tcgen05 MMA into TMEM,
//                           TMA-fed swizzled shared-memory ring, one CTA per
//                           SM walking an L2-grouped tile order.
// (The kernels around it -- operand repacking, the thin N remainder, K == 0 --
// are in tg_aux.cuh.)
//
// Operation: "Designing High-Performance GPU Kernels with TileLang"
// (thecryptopost.io), make_matmul -- per output tile, clear an fp32
// accumulator, loop over K in block_K steps copying an A tile and a B tile
// to shared memory and accumulating their product, then write the tile.
// Fused epilogue (bias add + GELU on the accumulator before the one store):
// the same tutorial (ainovat.com), fused-epilogue section.
//
// B200 design (not the tutorial's): the copies are TMA bulk tensor loads
// into a STAGES-deep mbarrier ring in the 128-byte-swizzled layouts that
// tcgen05.mma reads directly; one thread issues the MMAs; the accumulator
// lives in tensor memory, double-buffered so the epilogue of one tile
// overlaps the main loop of the next; the grid is persistent.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "tg_ptx.cuh"

namespace tg {

constexpr int kBlockM = 128;   // rows of A (and of C) per CTA: one TMEM lane per row
constexpr int kAtomK = 64;     // K of one A box: 64 fp16 = one 128-byte swizzle row
constexpr int kBChunkN = 64;   // B is loaded in 64-column boxes (128 bytes wide)
constexpr int kUmmaK = 16;     // K of one kind::f16 MMA instruction
constexpr int kAAtomBytes = kBlockM * kAtomK * 2;     // one 128 x 64 A box: 16 KiB
constexpr int kStoreCols = 32;                        // C columns per TMEM load / TMA store box
constexpr int kStoreBoxBytes = 32 * kStoreCols * 2;   // 32 rows x 32 fp16 = 2 KiB
constexpr int kFoldSlotBytes = 32 * kStoreCols * 4;   // 32 rows x 32 fp32 columns

// Error word bits (OR-ed into the per-device error word on a wait expiry).
constexpr unsigned kErrProducerWait = 1u;
constexpr unsigned kErrMmaWait = 2u;
constexpr unsigned kErrEpilogueWait = 4u;
constexpr unsigned kErrDrain = 8u;
constexpr unsigned kErrStreamKWait = 16u;
constexpr unsigned kErrFoldWait = 32u;

enum : int { kEpiNone = 0, kEpiBias = 1, kEpiBiasGelu = 2, kEpiBiasGeluTanh = 3, kEpiBiasSoftmax = 4 };
// How the epilogue writes C: element stores (any pitch), 16-byte stores
// (16-byte aligned rows), or TMA stores from a swizzled staging tile.
enum : int { kStoreScalar = 0, kStoreVec = 1, kStoreTma = 2 };
// How operand tiles reach shared memory: TMA (16-byte aligned bases and row
// pitches), or plain loads by four loader warps (any pitch; 2-byte alignment).
enum : int { kLoadTma = 0, kLoadPlain = 1 };

struct GemmParams {
    const __half *A;        // [M, lda], read by the plain loader only
    const __half *B;        // [K, ldb], read by the plain loader only
    int64_t lda, ldb;
    const __half *bias;     // [N] or nullptr
    __half *C;              // [M, ldc]
    int64_t M, N, K;
    int64_t ldc;
    int num_m_tiles;        // ceil(M / tile_m), tile_m = 128 (single CTA) or 256 (CTA pair)
    int num_n_tiles;        // ceil(N / BN)
    int num_k_blocks;       // ceil(K / 64)
    int num_tiles;
    int group_m;
    int inject;             // 1: the first CTA skips its first operand load;
                            // 2: stream-K partials are never flagged (timeout tests)
    int bias_vec;           // bias is 16-byte aligned: load it 8 values at a time
    uint64_t wait_limit_ns;
    unsigned *error_word;   // device address of the per-device error word
    // Stream-K: the tiles' k-block iterations are split evenly over the units
    // (CTAs, or CTA pairs) instead of whole tiles.
    int stream_k;
    float *sk_partials;     // per CTA: 128 x BN fp32 partial accumulator, laid out
                            // so that each warp store is one contiguous 512-B run
    unsigned *sk_flags;     // per CTA and epilogue warp: epoch at which that warp's
                            // rows / columns of the CTA's partial are complete
    unsigned sk_epoch;      // this launch's epoch (never 0)
    // Stream-K with every tile split evenly over sk_share consecutive units
    // (0: not so): the units of a tile share its fold.  Each writes its
    // partial of the 32-column chunks it does not own, then adds the others'
    // partials to the chunks it owns (chunk c: unit c mod sk_share of the
    // tile) and runs their epilogue.  Not for the row softmax.
    int sk_share;
    // A tail kernel follows: let it start as soon as every CTA is resident.
    int early_trigger;
};

// The work of one unit, as segments (tile, k-blocks [k0, k1)).
//   data-parallel: whole tiles unit, unit + num_units, ...
//   stream-K:      the iterations [unit * I / U, (unit + 1) * I / U) of the
//                  I = tiles * k-blocks iteration space, cut at tile borders.
// Roles: kSegFull (whole tile), kSegHead (holds k-block 0 but not the last:
// adds the later units' partials, then runs the epilogue), kSegPartial (starts
// after k-block 0: writes its partial for the head).  A unit's partial
// segment, if any, is its first and its head segment its last, so a head
// only ever waits on work that the other units do before any waiting.
enum : int { kSegFull = 0, kSegHead = 1, kSegPartial = 2 };

struct WorkIter {
    long long cur, end;
    int kb, step;
    bool sk;

    __device__ __forceinline__ static long long sk_begin(const GemmParams &p, int unit, int units)
    {
        return static_cast<long long>(p.num_tiles) * p.num_k_blocks * unit / units;
    }

    // The last unit whose range starts before iteration `tile_end` (a head
    // at `unit` adds the partials of units unit + 1 .. that one).  The range
    // starts floor(I u / U) are stepped by adding I / U and carrying the
    // remainder, so the search costs two divisions however long it is.  The
    // host launches at most I units, so every unit's range is non-empty.
    __device__ __forceinline__ static int last_contributor(const GemmParams &p, int unit, int units,
                                                           long long tile_end)
    {
        const long long iters = static_cast<long long>(p.num_tiles) * p.num_k_blocks;
        const long long q_step = iters / units;
        const long long r_step = iters - q_step * units;
        const long long num = iters * (unit + 1);
        long long q = num / units;   // start of unit + 1
        long long r = num - q * units;
        int last = unit;
        while (last + 1 < units && q < tile_end) {
            ++last;
            q += q_step;
            r += r_step;
            if (r >= units) {
                r -= units;
                ++q;
            }
        }
        return last;
    }

    __device__ __forceinline__ WorkIter(const GemmParams &p, int unit, int units)
    {
        kb = p.num_k_blocks;
        sk = p.stream_k != 0;
        step = units;
        if (sk) {
            cur = sk_begin(p, unit, units);
            end = sk_begin(p, unit + 1, units);
        } else {
            cur = unit;
            end = p.num_tiles;
        }
    }

    __device__ __forceinline__ bool next(int &tile, int &k0, int &k1, int &role)
    {
        if (cur >= end) return false;
        if (!sk) {
            tile = static_cast<int>(cur);
            k0 = 0;
            k1 = kb;
            role = kSegFull;
            cur += step;
            return true;
        }
        tile = static_cast<int>(cur / kb);
        const long long base = static_cast<long long>(tile) * kb;
        const long long seg_end = end < base + kb ? end : base + kb;
        k0 = static_cast<int>(cur - base);
        k1 = static_cast<int>(seg_end - base);
        role = (k0 == 0 && k1 == kb) ? kSegFull : (k0 == 0 ? kSegHead : kSegPartial);
        cur = seg_end;
        return true;
    }
};

// Compile-time shape of one kernel variant.
//   BN        output columns per tile (the MMA's N)
//   BK        K per pipeline stage (64 or 128): A arrives as BK/64 boxes of
//             128 x 64, each B chunk as one 64-column x BK box
//   STAGES    depth of the shared-memory operand ring
//   PAIR      two CTAs of a cluster run one cta_group::2 MMA on a 256-row tile;
//             each loads 128 rows of A and BN/2 columns of B
//   EPI_WARPS 4 or 8 warps drain TMEM (8: two per lane quarter, halving columns)
//   LOAD      kLoadTma (one producer lane) or kLoadPlain (four loader warps;
//             single CTA with 4 epilogue warps only)
template <int BN, int BK, int STAGES, bool PAIR, int EPI_WARPS, int STORE, int LOAD = kLoadTma>
struct KernelShape {
    static_assert(BN == 64 || BN == 128 || BN == 256, "BN must be 64, 128 or 256");
    static_assert(BK == 64 || BK == 128, "BK must be 64 or 128");
    static_assert(!PAIR || BN >= 128, "a CTA pair needs BN >= 128");
    static_assert(EPI_WARPS == 4 || EPI_WARPS == 8, "4 or 8 epilogue warps");
    static_assert(LOAD == kLoadTma || (!PAIR && EPI_WARPS == 4),
                  "the plain loader runs single CTAs with 4 epilogue warps");
    static constexpr int kCG = PAIR ? 2 : 1;
    static constexpr int kTileM = kBlockM * kCG;
    static constexpr int kCtaN = BN / kCG;                       // B columns loaded per CTA
    static constexpr int kBChunks = kCtaN / kBChunkN;
    static constexpr int kAAtoms = BK / kAtomK;
    static constexpr int kABytes = kAAtoms * kAAtomBytes;       // A part of a stage
    static constexpr int kBChunkBytes = kBChunkN * BK * 2;      // one B box
    static constexpr int kStageBytes = kABytes + kBChunks * kBChunkBytes;
    static constexpr uint32_t kTxBytes = kCG * kStageBytes;      // both CTAs land on the leader
    static constexpr int kRingBytes = STAGES * kStageBytes;
    static constexpr int kStagingBytes = STORE != kStoreVec ? EPI_WARPS * 2 * kStoreBoxBytes : 0;
    // Stream-K fold: once a head segment's MMAs are done the operand ring is
    // idle, and each epilogue warp streams the contributors' partials into its
    // own kFoldSlots slots of kFoldSlotBytes (one warp's 32 rows x 32 columns
    // of fp32) there with bulk copies.
    static constexpr int kFoldSlots =
        kRingBytes / (EPI_WARPS * kFoldSlotBytes) < 8 ? kRingBytes / (EPI_WARPS * kFoldSlotBytes)
                                                      : 8;
    static_assert(kFoldSlots >= 2, "the operand ring must hold two fold slots per epilogue warp");
    static_assert(kRingBytes >= EPI_WARPS * (BN / kStoreCols / (EPI_WARPS / 4)) * kStoreBoxBytes,
                  "the operand ring must hold a staging box per chunk of the last tile");
    // barriers: full[STAGES], empty[STAGES], tmem_full[2], tmem_empty[2], drain,
    // fold[EPI_WARPS][kFoldSlots]
    static constexpr int kFoldBar = 2 * STAGES + 5;
    static constexpr int kNumBars = kFoldBar + EPI_WARPS * kFoldSlots;
    static constexpr int kStagingOffset = kRingBytes;
    static constexpr int kBarOffset = kRingBytes + kStagingBytes;
    static constexpr int kTmemSlotOffset = kBarOffset + kNumBars * 8;
    static constexpr int kAbortOffset = kTmemSlotOffset + 4;
    static constexpr int kUsedBytes = kAbortOffset + 4;
    static constexpr int kDynamicBytes = kUsedBytes + 1024;     // slack for 1024-B alignment
    static constexpr uint32_t kTmemCols = 2 * BN;               // double-buffered accumulator
    static constexpr int kLoaderWarps = LOAD == kLoadPlain ? 4 : 1;
    static constexpr int kProducerWarp = EPI_WARPS;             // the first loader warp
    static constexpr int kMmaWarp = EPI_WARPS + kLoaderWarps;
    static constexpr int kThreads = 32 * (EPI_WARPS + kLoaderWarps + 1);
    static constexpr int kChunksPerWarp = (BN / kStoreCols) / (EPI_WARPS / 4);
    static constexpr uint32_t kTmemEmptyArrivals = kCG * EPI_WARPS;
};

constexpr int kMaxDynamicSmem = 232448;   // 227 KiB: the sm_100 per-block opt-in limit

// STAGES, reduced by one when this store mode's staging buffers would push
// the block past the shared-memory limit (the element-store fallback of a
// configuration tuned for direct vector stores).
template <int BN, int BK, int STAGES, bool PAIR, int EPI_WARPS, int STORE, int LOAD = kLoadTma>
struct FittedStages {
    static constexpr int value =
        KernelShape<BN, BK, STAGES, PAIR, EPI_WARPS, STORE, LOAD>::kDynamicBytes <= kMaxDynamicSmem
            ? STAGES
            : STAGES - 1;
    static_assert(KernelShape<BN, BK, value, PAIR, EPI_WARPS, STORE, LOAD>::kDynamicBytes <=
                      kMaxDynamicSmem,
                  "shared-memory budget exceeded");
};

// Eight consecutive fp16 values src[0 .. 8) of a row with `valid` of them in
// bounds (the rest read as zero), by the widest loads their alignment allows:
// one 16-byte load, four 4-byte loads, or element loads.  Nothing outside the
// valid range is read.
__device__ __forceinline__ uint4 load8_any(const __half *src, int64_t valid)
{
    if (valid <= 0) return make_uint4(0u, 0u, 0u, 0u);
    const uintptr_t addr = reinterpret_cast<uintptr_t>(src);
    if (valid >= 8) {
        if ((addr & 15u) == 0) return __ldg(reinterpret_cast<const uint4 *>(src));
        if ((addr & 3u) == 0) {
            const unsigned *w = reinterpret_cast<const unsigned *>(src);
            return make_uint4(__ldg(w), __ldg(w + 1), __ldg(w + 2), __ldg(w + 3));
        }
    }
    const unsigned short *h = reinterpret_cast<const unsigned short *>(src);
    unsigned short e[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) e[i] = i < valid ? __ldg(h + i) : static_cast<unsigned short>(0);
    return make_uint4(e[0] | (static_cast<unsigned>(e[1]) << 16),
                      e[2] | (static_cast<unsigned>(e[3]) << 16),
                      e[4] | (static_cast<unsigned>(e[5]) << 16),
                      e[6] | (static_cast<unsigned>(e[7]) << 16));
}

// Tile index -> (m tile, n tile), walking group_m M-tiles per panel so that
// CTAs running at the same time share A rows and B columns in L2.
__device__ __forceinline__ void tile_coords(int tile, int num_m, int num_n, int group_m, int &mt,
                                            int &nt)
{
    const int per_group = group_m * num_n;
    const int g = tile / per_group;
    const int first_m = g * group_m;
    const int rows = min(num_m - first_m, group_m);
    const int r = tile - g * per_group;
    mt = first_m + r % rows;
    nt = r / rows;
}

__device__ __forceinline__ float rcp_approx(float x)
{
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ float exp2_approx(float x)
{
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// Two fp32 values in one 64-bit register, for the packed f32x2 arithmetic of
// sm_100 (two lanes' worth of FMA per instruction).
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ void f2_unpack(uint64_t r, float &lo, float &hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(r));
}

__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// GELU(v) = v * Phi(v), Phi the standard normal CDF.  With a = |v| and the
// lower tail T = Phi(-a), GELU(v) = max(v, 0) - a * T for either sign of v.
// log2 T(a) is the Gaussian exponent -a^2 log2(e) / 2 plus a smooth
// remainder (the logarithm of the Mills ratio, falling like -log2(a) for
// large a); on a in [0, 6] the whole of it is fitted by a degree-7
// polynomial Q in x = a / 3 - 1 to 5e-6 in log2 units (csrc/fit_gelu.py; our
// coefficients), so
//   T = 2^Q(x)   (a <= 6),   T = 0   (a > 6).
// Past a = 6, a * T is below half the smallest fp16 subnormal for every fp16
// input, so the cut changes no fp16 result but the sign of a zero.  One
// exponential, no division, 9 multiply-adds; in fp32 the result is within
// one fp16 ulp of the correctly rounded GELU for every fp16 input (0.4% of
// them off by one).
constexpr float kGeluQ0 = -9.532936096e+00f, kGeluQ1 = -1.420956707e+01f,
                kGeluQ2 = -6.033975601e+00f, kGeluQ3 = -2.038841099e-01f,
                kGeluQ4 = 9.168275446e-02f, kGeluQ5 = -4.095217586e-02f,
                kGeluQ6 = 1.681641303e-02f, kGeluQ7 = -4.013689235e-03f;
constexpr float kGeluAMax = 6.0f;

__device__ __forceinline__ float gelu_erf(float v)
{
    const float a = fabsf(v);
    const float x = fmaf(fminf(a, kGeluAMax), 2.0f / kGeluAMax, -1.0f);
    float p = fmaf(kGeluQ7, x, kGeluQ6);
    p = fmaf(p, x, kGeluQ5);
    p = fmaf(p, x, kGeluQ4);
    p = fmaf(p, x, kGeluQ3);
    p = fmaf(p, x, kGeluQ2);
    p = fmaf(p, x, kGeluQ1);
    p = fmaf(p, x, kGeluQ0);
    const float t = a > kGeluAMax ? 0.0f : exp2_approx(p);
    return fmaf(-a, t, fmaxf(v, 0.0f));
}

// gelu_erf of two values at once: the polynomial runs as packed f32x2
// operations (the same roundings as the scalar form).
__device__ __forceinline__ void gelu_erf2(float &v0, float &v1)
{
    const float a0 = fabsf(v0), a1 = fabsf(v1);
    const uint64_t x = f2_fma(f2_pack(fminf(a0, kGeluAMax), fminf(a1, kGeluAMax)),
                              f2_pack(2.0f / kGeluAMax, 2.0f / kGeluAMax), f2_pack(-1.0f, -1.0f));
    uint64_t p = f2_fma(f2_pack(kGeluQ7, kGeluQ7), x, f2_pack(kGeluQ6, kGeluQ6));
    p = f2_fma(p, x, f2_pack(kGeluQ5, kGeluQ5));
    p = f2_fma(p, x, f2_pack(kGeluQ4, kGeluQ4));
    p = f2_fma(p, x, f2_pack(kGeluQ3, kGeluQ3));
    p = f2_fma(p, x, f2_pack(kGeluQ2, kGeluQ2));
    p = f2_fma(p, x, f2_pack(kGeluQ1, kGeluQ1));
    p = f2_fma(p, x, f2_pack(kGeluQ0, kGeluQ0));
    float e0, e1;
    f2_unpack(p, e0, e1);
    const float t0 = a0 > kGeluAMax ? 0.0f : exp2_approx(e0);
    const float t1 = a1 > kGeluAMax ? 0.0f : exp2_approx(e1);
    v0 = fmaf(-a0, t0, fmaxf(v0, 0.0f));
    v1 = fmaf(-a1, t1, fmaxf(v1, 0.0f));
}

// tanh approximation of GELU (Hendrycks & Gimpel, "Gaussian Error Linear
// Units", section 2): v/2 (1 + tanh(u)), u = sqrt(2/pi) (v + 0.044715 v^3),
// evaluated as v / (1 + exp(-2u)) = v / (1 + 2^(-2 log2(e) u)).
__device__ __forceinline__ float gelu_tanh(float v)
{
    constexpr float k = 2.302208198115997f;   // 2 log2(e) sqrt(2/pi)
    const float x = v * fmaf(v * v, -k * 0.044715f, -k);
    return v * rcp_approx(1.0f + exp2_approx(x));
}

template <int EPI>
__device__ __forceinline__ float apply_epilogue(float acc, float beta)
{
    if (EPI == kEpiNone) return acc;
    float v = acc + beta;
    if (EPI == kEpiBiasGelu) v = gelu_erf(v);
    if (EPI == kEpiBiasGeluTanh) v = gelu_tanh(v);
    return v;
}

constexpr float kLog2e = 1.4426950408889634f;

// The 32 bias values of columns [col0, col0 + 32) as packed fp16 (zeros past N
// or without bias).  Issued ahead of their use so that the load latency
// overlaps other work: the first chunk's before the accumulator wait, each
// next chunk's while the current one is processed.
template <int EPI>
__device__ __forceinline__ void fetch_bias32(const __half *bias, int64_t col0, int64_t N, bool vec,
                                             uint4 (&out)[4])
{
    if (EPI == kEpiNone || bias == nullptr || col0 >= N) {
#pragma unroll
        for (int q = 0; q < 4; ++q) out[q] = make_uint4(0u, 0u, 0u, 0u);
        return;
    }
    if (vec && col0 + 32 <= N) {
        const uint4 *src = reinterpret_cast<const uint4 *>(bias + col0);
#pragma unroll
        for (int q = 0; q < 4; ++q) out[q] = __ldg(src + q);
    } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            __half h[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int64_t col = col0 + q * 8 + e;
                h[e] = col < N ? bias[col] : __ushort_as_half(static_cast<unsigned short>(0));
            }
            out[q] = *reinterpret_cast<const uint4 *>(h);
        }
    }
}

// Eight packed fp16 bias values -> floats.
__device__ __forceinline__ void unpack_bias8(const uint4 &u, float (&b)[8])
{
    const __half2 *h = reinterpret_cast<const __half2 *>(&u);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(h[e]);
        b[2 * e] = f.x;
        b[2 * e + 1] = f.y;
    }
}

// Eight fp32 accumulators + bias -> epilogue -> eight fp16 packed in a uint4.
// For the row softmax, r holds exp(v - m_c) already (written back by the
// statistics pass, m_c the running maximum when that chunk was read) and
// sm_scale is the chunk's exp(m_c - max) / sum(exp(v - max)); sm_max is unused.
template <int EPI>
__device__ __forceinline__ uint4 epilogue8(const uint32_t *r, const float (&b)[8],
                                           float sm_max = 0.f, float sm_scale = 0.f)
{
    uint4 u;
    __half2 *h = reinterpret_cast<__half2 *>(&u);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        float lo, hi;
        if constexpr (EPI == kEpiBiasGelu) {
            const uint64_t v = f2_add(f2_pack(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1])),
                                      f2_pack(b[2 * e], b[2 * e + 1]));
            f2_unpack(v, lo, hi);
            gelu_erf2(lo, hi);
        } else if constexpr (EPI == kEpiBiasSoftmax) {
            lo = __uint_as_float(r[2 * e]) * sm_scale;
            hi = __uint_as_float(r[2 * e + 1]) * sm_scale;
        } else {
            lo = apply_epilogue<EPI>(__uint_as_float(r[2 * e]), b[2 * e]);
            hi = apply_epilogue<EPI>(__uint_as_float(r[2 * e + 1]), b[2 * e + 1]);
        }
        h[e] = __floats2half2_rn(lo, hi);
    }
    return u;
}

// The low (hi == 0) or high half of a packed pair of fp16 values.
__device__ __forceinline__ __half half_of(uint32_t w, int hi)
{
    return __ushort_as_half(static_cast<unsigned short>(hi ? w >> 16 : w & 0xFFFFu));
}

// ---------------------------------------------------------------------------
// Persistent warp-specialised GEMM.
//   warps [0, EPI_WARPS)  epilogue: TMEM -> registers -> bias/GELU -> fp16 -> C
//   warp EPI_WARPS        TMA producer (one lane)
//   warp EPI_WARPS + 1    TMEM allocator; MMA issuer (one lane; the leader CTA
//                         of a pair issues for both)
// SHARE: the kernel variant launched for an even stream-K split, whose
// tile's units share the fold (GemmParams::sk_share); the other variants
// carry none of that code.
template <int BN, int BK, int STAGES, int EPI, bool PAIR, int EPI_WARPS, int STORE, int LOAD,
          bool SHARE = false>
__global__ void __launch_bounds__(KernelShape<BN, BK, STAGES, PAIR, EPI_WARPS, STORE, LOAD>::kThreads,
                                  1)
    gemm_persistent_kernel(const __grid_constant__ CUtensorMap tmA,
                           const __grid_constant__ CUtensorMap tmB,
                           const __grid_constant__ CUtensorMap tmC, const GemmParams p)
{
    using S = KernelShape<BN, BK, STAGES, PAIR, EPI_WARPS, STORE, LOAD>;
    constexpr int CG = S::kCG;
    constexpr uint32_t kIdesc = idesc_f16_f32(S::kTileM, BN);

    extern __shared__ uint8_t smem_raw[];
    // Round the dynamic shared-memory base up to 1024 B (128-byte swizzle atom);
    // the offset is the same in both CTAs of a pair.
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + S::kBarOffset);
    uint64_t *full_bar = bars;
    uint64_t *empty_bar = bars + STAGES;
    uint64_t *tmem_full_bar = bars + 2 * STAGES;
    uint64_t *tmem_empty_bar = bars + 2 * STAGES + 2;
    uint64_t *drain_bar = bars + 2 * STAGES + 4;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + S::kTmemSlotOffset);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + S::kAbortOffset);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t cta_rank = PAIR ? cluster_cta_rank() : 0u;
    const bool leader = cta_rank == 0;
    const int unit = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
    const int num_units = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], LOAD == kLoadPlain ? 32 * S::kLoaderWarps : 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tmem_full_bar[b], 1);
            mbar_init(&tmem_empty_bar[b], S::kTmemEmptyArrivals);
        }
        mbar_init(drain_bar, 1);
        for (int f = 0; f < EPI_WARPS * S::kFoldSlots; ++f) mbar_init(&bars[S::kFoldBar + f], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == S::kProducerWarp && lane == 0) {
        if (LOAD == kLoadTma) {
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmB);
        }
        if (STORE == kStoreTma) tma_prefetch_desc(&tmC);
    }
    if (warp == S::kMmaWarp) {
        tmem_alloc<CG>(tmem_slot, S::kTmemCols);
        tmem_relinquish<CG>();
    }
    tc_fence_before_sync();
    __syncthreads();
    if (PAIR) cluster_sync();   // peer barriers initialised before any remote use
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;
    // Everything above touches only this CTA's own resources, so it may overlap
    // the previous kernel in the stream; A, B, bias and C are touched only after
    // that kernel has completed.  A tail kernel that follows may start once
    // every CTA is here.
    grid_dependency_wait();
    if (p.early_trigger) grid_launch_dependents();

    const uint32_t smem_base = smem_u32(smem);
    const uint64_t limit = p.wait_limit_ns;

    if (LOAD == kLoadPlain && warp >= S::kProducerWarp && warp < S::kMmaWarp) {
        // Plain loader: 128 threads copy each stage's A and B tiles with global
        // loads into the same 128-byte-swizzled layout TMA would produce (16-byte
        // chunk c of row r at chunk c ^ (r % 8)), zero-filling past M, N and K,
        // then publish them to the tensor core (each thread: proxy fence, then
        // its arrival on the stage's full barrier).  Consecutive threads take
        // consecutive chunks of one 128-byte row: coalesced reads.
        const int lt = (warp - S::kProducerWarp) * 32 + lane;
        int stage = 0;
        uint32_t phase = 0;
        bool skip_next = (p.inject == 1 && blockIdx.x == 0 && warp == S::kProducerWarp);
        WorkIter work(p, unit, num_units);
        int tile, k0, k1, role;
        bool ok = true;
        while (ok && work.next(tile, k0, k1, role)) {
            int mt, nt;
            tile_coords(tile, p.num_m_tiles, p.num_n_tiles, p.group_m, mt, nt);
            const int64_t a_row0 = static_cast<int64_t>(mt) * kBlockM;
            const int64_t b_col0 = static_cast<int64_t>(nt) * BN;
            for (int kb = k0; kb < k1; ++kb) {
                int okw = 1;
                if (lane == 0)
                    okw = mbar_wait_bounded(&empty_bar[stage], phase ^ 1u, abort_flag, limit,
                                            p.error_word, kErrProducerWait)
                              ? 1
                              : 0;
                okw = __shfl_sync(0xffffffffu, okw, 0);
                if (!okw) {
                    ok = false;
                    break;
                }
                const uint32_t a_dst = smem_base + stage * S::kStageBytes;
                const uint32_t b_dst = a_dst + S::kABytes;
                const int64_t kbase = static_cast<int64_t>(kb) * BK;
#pragma unroll 2
                for (int i = lt; i < S::kAAtoms * kBlockM * 8; i += 128) {
                    const int q = i >> 10, r = (i >> 3) & 127, c = i & 7;
                    const int64_t gm = a_row0 + r;
                    const int64_t gk = kbase + q * kAtomK + c * 8;
                    const uint4 v = gm < p.M ? load8_any(p.A + gm * p.lda + gk, p.K - gk)
                                             : make_uint4(0u, 0u, 0u, 0u);
                    const uint32_t addr = a_dst + q * kAAtomBytes + r * 128 +
                                          ((static_cast<uint32_t>(c) ^ (r & 7)) * 16u);
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                                 "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                                 : "memory");
                }
#pragma unroll 2
                for (int i = lt; i < S::kBChunks * BK * 8; i += 128) {
                    const int j = i / (BK * 8), rem = i % (BK * 8), r = rem >> 3, c = rem & 7;
                    const int64_t gk = kbase + r;
                    const int64_t gn = b_col0 + j * kBChunkN + c * 8;
                    const uint4 v = gk < p.K ? load8_any(p.B + gk * p.ldb + gn, p.N - gn)
                                             : make_uint4(0u, 0u, 0u, 0u);
                    const uint32_t addr = b_dst + j * S::kBChunkBytes + r * 128 +
                                          ((static_cast<uint32_t>(c) ^ (r & 7)) * 16u);
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                                 "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                                 : "memory");
                }
                fence_proxy_async_smem();
                if (skip_next)
                    skip_next = false;   // injected fault: this stage never fills
                else
                    mbar_arrive(&full_bar[stage]);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        __syncwarp();
    } else if (LOAD == kLoadTma && warp == S::kProducerWarp) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            // Per stage: 1 + parity of the last load whose bytes this CTA's
            // full barrier expects, or 0 for none (drained before exit).
            uint32_t pending[STAGES];
#pragma unroll
            for (int s = 0; s < STAGES; ++s) pending[s] = 0;
            bool skip_next = (p.inject == 1 && blockIdx.x == 0);
            WorkIter work(p, unit, num_units);
            int tile, k0, k1, role;
            while (work.next(tile, k0, k1, role)) {
                int mt, nt;
                tile_coords(tile, p.num_m_tiles, p.num_n_tiles, p.group_m, mt, nt);
                const int a_row = mt * S::kTileM + static_cast<int>(cta_rank) * kBlockM;
                const int b_col = nt * BN + static_cast<int>(cta_rank) * S::kCtaN;
                bool ok = true;
                for (int kb = k0; kb < k1; ++kb) {
                    if (!mbar_wait_bounded(&empty_bar[stage], phase ^ 1u, abort_flag, limit,
                                           p.error_word, kErrProducerWait)) {
                        ok = false;
                        break;
                    }
                    if (skip_next) {
                        skip_next = false;   // injected fault: this stage never fills
                    } else {
                        const uint32_t a_dst = smem_base + stage * S::kStageBytes;
                        const uint32_t b_dst = a_dst + S::kABytes;
                        if (leader) {
                            mbar_arrive_expect_tx(&full_bar[stage], S::kTxBytes);
                            pending[stage] = 1u + phase;
                        }
                        if constexpr (PAIR) {
                            const uint32_t bar = map_to_cta(smem_u32(&full_bar[stage]), 0);
#pragma unroll
                            for (int q = 0; q < S::kAAtoms; ++q)
                                tma_load_2d_pair(a_dst + q * kAAtomBytes, &tmA, bar,
                                                 kb * BK + q * kAtomK, a_row);
#pragma unroll
                            for (int j = 0; j < S::kBChunks; ++j)
                                tma_load_2d_pair(b_dst + j * S::kBChunkBytes, &tmB, bar,
                                                 b_col + j * kBChunkN, kb * BK);
                        } else {
#pragma unroll
                            for (int q = 0; q < S::kAAtoms; ++q)
                                tma_load_2d(a_dst + q * kAAtomBytes, &tmA, &full_bar[stage],
                                            kb * BK + q * kAtomK, a_row);
#pragma unroll
                            for (int j = 0; j < S::kBChunks; ++j)
                                tma_load_2d(b_dst + j * S::kBChunkBytes, &tmB, &full_bar[stage],
                                            b_col + j * kBChunkN, kb * BK);
                        }
                    }
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
            }
            // Let the loads this CTA's full barriers track land before exit.
            // (A pair's peer CTA is covered by the leader's drain plus the
            // cluster barrier at teardown.)
#pragma unroll
            for (int s = 0; s < STAGES; ++s)
                if (pending[s] != 0 && !mbar_wait_drain(&full_bar[s], pending[s] - 1u, limit))
                    atomicOr(p.error_word, kErrDrain);
        }
        __syncwarp();
    } else if (warp == S::kMmaWarp) {
        if (lane == 0 && leader) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool issued_any = false;
            // Result of a non-blocking probe of full_bar[stage] made while the
            // previous stage's MMAs were being issued: when it already saw the
            // data, the blocking wait (and its latency) is skipped.
            bool ready = false;
            // Shared-memory descriptors of stage 0; stage s adds s * kStageBytes
            // to the 14-bit start-address field (units of 16 B, no carry out for
            // addresses below 256 KiB).
            // A: K-major, 128-B swizzle; 8-row groups 1024 B apart.
            const uint64_t a_desc0 = smem_desc_sw128(smem_base, 16, 1024);
            // B: MN-major, 128-B swizzle; 64-column chunks kBChunkBytes apart
            // (leading), 8-k-row groups 1024 B apart (stride).
            const uint64_t b_desc0 =
                smem_desc_sw128(smem_base + S::kABytes, S::kBChunkBytes, 1024);
            WorkIter work(p, unit, num_units);
            int tile, k0, k1, role;
            while (work.next(tile, k0, k1, role)) {
                if (!mbar_wait_bounded(&tmem_empty_bar[acc], acc_phase ^ 1u, abort_flag, limit,
                                       p.error_word, kErrMmaWait))
                    break;
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
                bool ok = true;
                for (int kb = k0; kb < k1; ++kb) {
                    if (!ready && !mbar_wait_bounded(&full_bar[stage], phase, abort_flag, limit,
                                                     p.error_word, kErrMmaWait)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const int next_stage = stage + 1 == STAGES ? 0 : stage + 1;
                    const uint32_t next_phase = next_stage == 0 ? phase ^ 1u : phase;
                    ready = mbar_test_wait(&full_bar[next_stage], next_phase);
                    const uint64_t stage_off =
                        static_cast<uint64_t>((stage * S::kStageBytes) >> 4);
#pragma unroll
                    for (int kk = 0; kk < BK / kUmmaK; ++kk) {
                        // K step: for A, the next 32 B inside a 128-B swizzle row,
                        // moving to the next 128 x 64 box every 4 steps; for B,
                        // the next 16 k-rows (2 KiB).
                        constexpr int kStepsPerAtom = kAtomK / kUmmaK;
                        const uint64_t a_k =
                            a_desc0 + stage_off +
                            static_cast<uint64_t>(((kk / kStepsPerAtom) * kAAtomBytes +
                                                   (kk % kStepsPerAtom) * kUmmaK * 2) >>
                                                  4);
                        const uint64_t b_k =
                            b_desc0 + stage_off + static_cast<uint64_t>((kk * kUmmaK * 128) >> 4);
                        mma_f16_ss<CG>(d_tmem, a_k, b_k, kIdesc, (kb != k0 || kk != 0) ? 1u : 0u);
                    }
                    issued_any = true;
                    // the stage is free (in both CTAs) once these MMAs finish
                    if constexpr (PAIR)
                        mma_commit_pair_multicast(&empty_bar[stage], 0x3);
                    else
                        mma_commit<1>(&empty_bar[stage]);
                    stage = next_stage;
                    phase = next_phase;
                }
                if (!ok) break;
                // accumulator ready for the epilogue (of both CTAs)
                if constexpr (PAIR)
                    mma_commit_pair_multicast(&tmem_full_bar[acc], 0x3);
                else
                    mma_commit<1>(&tmem_full_bar[acc]);
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
            // Wait for every MMA this thread issued before TMEM is released.
            if (issued_any) {
                mma_commit<CG>(drain_bar);
                if (!mbar_wait_drain(drain_bar, 0, limit)) atomicOr(p.error_word, kErrDrain);
            }
        }
        __syncwarp();
    } else {
        // Epilogue warp w: TMEM lanes [32 (w % 4), +32) = 32 tile rows; with 8
        // warps, w / 4 selects the half of the columns.
        const int quarter = warp & 3;
        const int chunk0 = (warp >> 2) * S::kChunksPerWarp;
        const uint32_t empty_bar_leader =
            PAIR ? map_to_cta(smem_u32(&tmem_empty_bar[0]), 0) : 0u;
        const uint32_t staging = smem_base + S::kStagingOffset + warp * 2 * kStoreBoxBytes;
        const bool bias_vec = p.bias_vec != 0;
        int acc = 0;
        uint32_t acc_phase = 0;
        uint32_t store_count = 0;
        WorkIter work(p, unit, num_units);
        int tile, k0, k1, role;
        while (work.next(tile, k0, k1, role)) {
            int mt, nt;
            tile_coords(tile, p.num_m_tiles, p.num_n_tiles, p.group_m, mt, nt);
            uint4 bias_next[4];
            fetch_bias32<EPI>(p.bias, static_cast<int64_t>(nt) * BN + chunk0 * kStoreCols, p.N,
                              bias_vec, bias_next);
            int ok = 0;
            if (lane == 0)
                ok = mbar_wait_bounded(&tmem_full_bar[acc], acc_phase, abort_flag, limit,
                                       p.error_word, kErrEpilogueWait)
                         ? 1
                         : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after_sync();

            const int64_t row0 = static_cast<int64_t>(mt) * S::kTileM +
                                 static_cast<int64_t>(cta_rank) * kBlockM + quarter * 32;
            const int64_t row = row0 + lane;
            const bool row_ok = row < p.M;
            __half *crow = p.C + row * p.ldc;
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                   static_cast<uint32_t>(acc * BN);
            // Stream-K partials of a CTA (slot = unit * CG + rank) hold 128 x BN
            // fp32 values as uint4 groups indexed ((warp * chunks + chunk) * 8 + q)
            // * 32 + lane: lane l of warp w keeps columns 4q .. 4q + 3 of its row
            // of chunk c there, so a warp writes 512 contiguous bytes per store and
            // each (warp, chunk) block is 4 KiB of contiguous memory.
            auto partial_group = [&](int slot, int c, int q) {
                return reinterpret_cast<uint4 *>(p.sk_partials +
                                                 static_cast<size_t>(slot) * kBlockM * BN) +
                       ((warp * S::kChunksPerWarp + (c - chunk0)) * 8 + q) * 32 + lane;
            };
            // Shared fold (an even split, sk_share units per tile): this unit is
            // member `me` of the tile's units and owns its chunks c with
            // c mod sk_share == me.
            const bool shared =
                SHARE && EPI != kEpiBiasSoftmax && p.sk_share > 0 && role != kSegFull;
            const int share = shared ? p.sk_share : 1;
            const int me = shared ? unit % share : 0;
            auto owned = [&](int c) { return !shared || c % share == me; };
            int first_contrib = 0, last_contrib = -1;   // units whose partials this unit adds,
            int skip_v = -1;                            // except this one
            if (shared) {
                // First the chunks this unit does not own, for their owners.
#pragma unroll 1
                for (int c = chunk0; c < chunk0 + S::kChunksPerWarp; ++c) {
                    if (owned(c)) continue;
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(c * kStoreCols), r);
                    tmem_wait_ld();
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        __stcg(partial_group(unit * CG + cta_rank, c, q),
                               make_uint4(r[4 * q], r[4 * q + 1], r[4 * q + 2], r[4 * q + 3]));
                }
                __threadfence();
                __syncwarp();
                if (lane == 0 && p.inject != 2)
                    st_release_gpu(p.sk_flags + (unit * CG + cta_rank) * EPI_WARPS + warp,
                                   p.sk_epoch);
                first_contrib = unit - me;
                last_contrib = unit - me + share - 1;
                skip_v = unit;
            } else if (role == kSegHead) {
                const long long tile_end = static_cast<long long>(tile + 1) * p.num_k_blocks;
                first_contrib = unit + 1;
                last_contrib = WorkIter::last_contributor(p, unit, num_units, tile_end);
            }
            // The contributing units in the order their partials are added.
            const int v_begin = first_contrib == skip_v ? first_contrib + 1 : first_contrib;
            auto next_v = [&](int v) { return v + 1 == skip_v ? v + 2 : v + 1; };
            {
                // Warp w reads exactly the rows and columns that warp w of each
                // contributing CTA wrote, so it waits for those flags only.
                for (int v = v_begin; v <= last_contrib; v = next_v(v)) {
                    const unsigned *flag = p.sk_flags + (v * CG + cta_rank) * EPI_WARPS + warp;
                    if (ld_acquire_gpu(flag) == p.sk_epoch) continue;
                    const uint64_t t0 = global_timer_ns();
                    while (ld_acquire_gpu(flag) != p.sk_epoch) {
                        if (*abort_flag) break;
                        if (global_timer_ns() - t0 > limit) {
                            *abort_flag = 1;
                            atomicOr(p.error_word, kErrStreamKWait);
                            break;
                        }
                    }
                }
            }
            __syncwarp();   // reconverge before the warp-collective TMEM loads
            // The chunks this warp's epilogue visits: up to the first one past N
            // (none when all 32 rows are past M).
            int chunk_end = chunk0;
            if (row0 < p.M)
                while (chunk_end < chunk0 + S::kChunksPerWarp &&
                       static_cast<int64_t>(nt) * BN + chunk_end * kStoreCols < p.N)
                    ++chunk_end;
            // Fold (heads only).  A head segment is the last of its unit, so its
            // tmem_full means every MMA of this CTA is done and the operand ring
            // is idle.  Items (chunk c, contributor v) are visited c-major, v
            // ascending -- the order the sums are taken in -- and item i is
            // copied into slot i % kFoldSlots of this warp's part of the ring,
            // kFoldSlots items ahead of its use.
            // The first chunk this warp finishes (shared fold: the first it owns).
            int first_owned = chunk0;
            while (first_owned < chunk_end && !owned(first_owned)) ++first_owned;
            const int chunk_step = shared ? share : 1;
            bool folding =
                v_begin <= last_contrib && first_owned < chunk_end && *abort_flag == 0;
            bool fold_ok = true;
            uint64_t *fold_bar = bars + S::kFoldBar + warp * S::kFoldSlots;
            const uint32_t fold_smem =
                smem_base + static_cast<uint32_t>(warp * S::kFoldSlots * kFoldSlotBytes);
            int issue_c = first_owned, issue_v = v_begin;
            uint32_t issued = 0, waited = 0;
            auto fold_issue = [&]() {
                if (!folding || !fold_ok || issue_c >= chunk_end) return;
                const uint32_t slot = issued % S::kFoldSlots;
                if (lane == 0) {
                    // 4 KiB: this warp's 32 rows x 32 columns of chunk issue_c
                    // in contributor issue_v's partial (the layout below).
                    const float *src =
                        p.sk_partials +
                        static_cast<size_t>(issue_v * CG + cta_rank) * kBlockM * BN +
                        static_cast<size_t>(warp * S::kChunksPerWarp + (issue_c - chunk0)) *
                            (kFoldSlotBytes / 4);
                    mbar_arrive_expect_tx(&fold_bar[slot], kFoldSlotBytes);
                    bulk_load_g2s(fold_smem + slot * kFoldSlotBytes, src, kFoldSlotBytes,
                                  &fold_bar[slot]);
                }
                ++issued;
                issue_v = next_v(issue_v);
                if (issue_v > last_contrib) {
                    issue_v = v_begin;
                    issue_c += chunk_step;
                }
            };
            if (folding) {
                // The flags were acquired through the generic proxy; the bulk
                // copies read the partials through the async proxy.
                if (lane == 0) fence_proxy_async_all();
                __syncwarp();
                for (int i = 0; i < S::kFoldSlots; ++i) fold_issue();
            }
            // One 32-column chunk of the accumulator: TMEM, plus (for a head)
            // the partials of the later units, added in unit order.
            auto load_acc_chunk = [&](int c, uint32_t (&r)[32]) {
                tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(c * kStoreCols), r);
                tmem_wait_ld();
                if (!folding) return;
                for (int v = v_begin; v <= last_contrib; v = next_v(v)) {
                    const uint32_t slot = waited % S::kFoldSlots;
                    if (fold_ok) {
                        const int ok = mbar_wait_bounded(&fold_bar[slot],
                                                         (waited / S::kFoldSlots) & 1u, abort_flag,
                                                         limit, p.error_word, kErrFoldWait)
                                           ? 1
                                           : 0;
                        fold_ok = __all_sync(0xffffffffu, ok) != 0;
                    }
                    if (!fold_ok) return;
                    const uint32_t src = fold_smem + slot * kFoldSlotBytes + lane * 16u;
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        uint32_t u0, u1, u2, u3;
                        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                     : "=r"(u0), "=r"(u1), "=r"(u2), "=r"(u3)
                                     : "r"(src + static_cast<uint32_t>(q) * 512u)
                                     : "memory");
                        r[4 * q + 0] = __float_as_uint(__uint_as_float(r[4 * q + 0]) + __uint_as_float(u0));
                        r[4 * q + 1] = __float_as_uint(__uint_as_float(r[4 * q + 1]) + __uint_as_float(u1));
                        r[4 * q + 2] = __float_as_uint(__uint_as_float(r[4 * q + 2]) + __uint_as_float(u2));
                        r[4 * q + 3] = __float_as_uint(__uint_as_float(r[4 * q + 3]) + __uint_as_float(u3));
                    }
                    ++waited;
                    __syncwarp();   // every lane has read the slot before it is refilled
                    fold_issue();
                }
            };
            // Copies still in flight after a failed wait land before the ring's
            // shared memory is released.
            auto fold_drain = [&]() {
                if (lane == 0)
                    for (uint32_t i = waited; i < issued; ++i)
                        if (!mbar_wait_drain(&fold_bar[i % S::kFoldSlots],
                                             (i / S::kFoldSlots) & 1u, limit))
                            atomicOr(p.error_word, kErrDrain);
                __syncwarp();
            };
            if (role == kSegPartial && !shared) {
                // Write this warp's rows / columns of the unit's partial
                // accumulator; once every lane's stores are fenced, flag them.
#pragma unroll 1
                for (int c = chunk0; c < chunk0 + S::kChunksPerWarp; ++c) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(c * kStoreCols), r);
                    tmem_wait_ld();
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        __stcg(partial_group(unit * CG + cta_rank, c, q),
                               make_uint4(r[4 * q], r[4 * q + 1], r[4 * q + 2], r[4 * q + 3]));
                }
                __threadfence();
                __syncwarp();
                if (lane == 0 && p.inject != 2)
                    st_release_gpu(p.sk_flags + (unit * CG + cta_rank) * EPI_WARPS + warp,
                                   p.sk_epoch);
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) {
                    if (PAIR)
                        mbar_arrive_cluster(empty_bar_leader + static_cast<uint32_t>(acc * 8));
                    else
                        mbar_arrive(&tmem_empty_bar[acc]);
                }
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
                continue;
            }
            // Row softmax (4 epilogue warps: each thread owns its whole row).  One
            // pass over the accumulator in TMEM gives the row maximum and the sum
            // of exp(v - max) over the valid columns, kept as a running pair: a
            // chunk raising the maximum from m to m' rescales the sum by
            // exp(m - m').  Two chunks are read per TMEM wait, and each chunk's
            // maximum and sum are taken over eight independent partials.  The
            // chunk's exponentials go back into TMEM in place of its accumulator,
            // with the maximum they were taken against (chunk_shift, in log2
            // units), so that the output pass multiplies instead of exponentiating
            // again.
            float sm_max = 0.f, sm_scale = 0.f;
            float chunk_shift[S::kChunksPerWarp];
            if constexpr (EPI == kEpiBiasSoftmax) {
                static_assert(EPI_WARPS == 4, "the softmax epilogue needs whole rows per thread");
                // The statistics pass and the output pass both read the
                // accumulator; fold the contributors into it in TMEM once, first.
                if (folding) {
#pragma unroll 1
                    for (int c = chunk0; c < chunk_end; ++c) {
                        uint32_t r[32];
                        load_acc_chunk(c, r);
                        tmem_st_32x32b_x32(t_row + static_cast<uint32_t>(c * kStoreCols), r);
                    }
                    tmem_wait_st();
                    folding = false;
                }
                float run_max = -INFINITY, run_sum = 0.f;
                auto stats_chunk = [&](const uint32_t (&r)[32], const uint4 (&bq)[4], int64_t col0,
                                       int ci, uint32_t taddr) {
                    float v[32];
                    const bool full = col0 + kStoreCols <= p.N;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        float b[8];
                        unpack_bias8(bq[q], b);
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const float x = __uint_as_float(r[q * 8 + e]) + b[e];
                            v[q * 8 + e] = (full || col0 + q * 8 + e < p.N) ? x : -INFINITY;
                        }
                    }
                    float m[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        m[j] = fmaxf(fmaxf(v[j], v[j + 8]), fmaxf(v[j + 16], v[j + 24]));
#pragma unroll
                    for (int j = 0; j < 4; ++j) m[j] = fmaxf(m[j], m[j + 4]);
                    const float cmax = fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]));
                    const float new_max = fmaxf(run_max, cmax);   // finite: a chunk has a valid column
                    const float shift = new_max * kLog2e;
                    float sp[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) sp[j] = 0.f;
                    uint32_t ex[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const float x = exp2_approx(fmaf(v[e], kLog2e, -shift));
                        ex[e] = __float_as_uint(x);
                        sp[e & 7] += x;
                    }
                    tmem_st_32x32b_x32(taddr, ex);
                    chunk_shift[ci] = shift;
#pragma unroll
                    for (int j = 0; j < 4; ++j) sp[j] += sp[j + 4];
                    const float csum = (sp[0] + sp[1]) + (sp[2] + sp[3]);
                    run_sum = fmaf(run_sum, exp2_approx(fmaf(run_max, kLog2e, -shift)), csum);
                    run_max = new_max;
                };
#pragma unroll 1
                for (int c = chunk0; c < chunk_end; c += 2) {
                    const bool two = c + 1 < chunk_end;
                    const int64_t col0 = static_cast<int64_t>(nt) * BN + c * kStoreCols;
                    uint32_t ra[32], rb[32];
                    tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(c * kStoreCols), ra);
                    if (two)
                        tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>((c + 1) * kStoreCols), rb);
                    uint4 ba[4], bb[4];
                    fetch_bias32<EPI>(p.bias, col0, p.N, bias_vec, ba);
                    if (two) fetch_bias32<EPI>(p.bias, col0 + kStoreCols, p.N, bias_vec, bb);
                    tmem_wait_ld_dep(ra);
                    if (two) tmem_wait_ld_dep(rb);
                    stats_chunk(ra, ba, col0, c - chunk0,
                                t_row + static_cast<uint32_t>(c * kStoreCols));
                    if (two)
                        stats_chunk(rb, bb, col0 + kStoreCols, c + 1 - chunk0,
                                    t_row + static_cast<uint32_t>((c + 1) * kStoreCols));
                }
                tmem_wait_st();
                sm_max = run_max;
                sm_scale = rcp_approx(run_sum);
            }
            // The CTA's last tile (no segment follows): every MMA of the CTA (of
            // both CTAs of a pair) is complete once its accumulator is, so the
            // operand ring is idle -- unless a stream-K fold copies into it.
            const bool ring_staging = work.cur >= work.end && !folding;
            // One chunk: epilogue on its 32 accumulator columns r, then its store.
            // The bias of chunk c is in bias_next on entry; the next chunk's is
            // fetched here.
            auto emit = [&](int c, const uint32_t (&r)[32]) {
                const int64_t col0 = static_cast<int64_t>(nt) * BN + c * kStoreCols;
                // row softmax: this chunk's factor exp(m_c - max) / sum
                float chunk_scale = 0.f;
                if constexpr (EPI == kEpiBiasSoftmax)
                    chunk_scale =
                        exp2_approx(fmaf(sm_max, -kLog2e, chunk_shift[c - chunk0])) * sm_scale;
                uint4 bias_cur[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) bias_cur[q] = bias_next[q];
                if (c + 1 < chunk_end)
                    fetch_bias32<EPI>(p.bias, col0 + kStoreCols, p.N, bias_vec, bias_next);
                if constexpr (STORE == kStoreVec) {
                    if (row_ok) {
                        const bool full = col0 + kStoreCols <= p.N;
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            float b[8];
                            unpack_bias8(bias_cur[q], b);
                            const uint4 u = epilogue8<EPI>(r + q * 8, b, sm_max, chunk_scale);
                            if (full) {
                                *reinterpret_cast<uint4 *>(crow + col0 + q * 8) = u;
                            } else {
                                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                                for (int e = 0; e < 8; ++e)
                                    if (col0 + q * 8 + e < p.N)
                                        crow[col0 + q * 8 + e] = half_of(w[e >> 1], e & 1);
                            }
                        }
                    }
                    return;
                }
                // TMA stores and element stores both stage a 32 x 32 fp16 box
                // (64-B rows, 64-B swizzle) first; two boxes alternate.  On the
                // CTA's last tile the TMA path gives every chunk a box of its own
                // in the idle operand ring, so no store waits for an earlier one
                // to be read out.
                const uint32_t slot = store_count & 1u;
                const bool own_box = STORE == kStoreTma && ring_staging;
                const uint32_t buf =
                    own_box ? smem_base + static_cast<uint32_t>(
                                              (warp * S::kChunksPerWarp + (c - chunk0)) *
                                              kStoreBoxBytes)
                            : staging + slot * kStoreBoxBytes;
                if (STORE == kStoreTma && !own_box && store_count >= 2) {
                    if (lane == 0) bulk_wait_group_read<1>();
                    __syncwarp();
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float b[8];
                    unpack_bias8(bias_cur[q], b);
                    const uint4 u = epilogue8<EPI>(r + q * 8, b, sm_max, chunk_scale);
                    const uint32_t phys = static_cast<uint32_t>(q) ^ ((lane >> 1) & 3u);
                    const uint32_t addr = buf + lane * 64u + phys * 16u;
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                                 "r"(u.x), "r"(u.y), "r"(u.z), "r"(u.w)
                                 : "memory");
                }
                if constexpr (STORE == kStoreTma) {
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&tmC, buf, static_cast<int32_t>(col0),
                                     static_cast<int32_t>(row0));
                        bulk_commit_group();
                    }
                } else {
                    // Any pitch: the box goes back out one row per instruction,
                    // lane l storing column l (64 contiguous bytes of a row per
                    // store: on rows that are not 16-byte aligned this beats
                    // per-row vector stores, which touch 32 rows per store).
                    __syncwarp();
                    const bool col_ok = col0 + lane < p.N;
                    const unsigned short *box = reinterpret_cast<const unsigned short *>(
                        smem + S::kStagingOffset + (warp * 2 + slot) * kStoreBoxBytes);
                    const uint32_t q = static_cast<uint32_t>(lane) >> 3;
                    const uint32_t within = static_cast<uint32_t>(lane) & 7u;
                    __half *dst = p.C + row0 * p.ldc + col0 + lane;
                    const int rows = p.M - row0 < 32 ? static_cast<int>(p.M - row0) : 32;
#pragma unroll 8
                    for (int rr = 0; rr < 32; ++rr) {
                        const uint32_t phys = q ^ ((static_cast<uint32_t>(rr) >> 1) & 3u);
                        const unsigned short h = box[rr * 32 + phys * 8 + within];
                        if (col_ok && rr < rows) dst[rr * p.ldc] = __ushort_as_half(h);
                    }
                    __syncwarp();
                }
                ++store_count;
            };
            // Each chunk's TMEM load is issued one chunk ahead, so that it is in
            // flight while the previous chunk is converted and stored.  (Heads
            // of a stream-K split load through the fold, one chunk at a time.)
            uint32_t ra[32], rb[32];
            if (shared) {
                // The chunks this unit owns, each with every unit's partial.
#pragma unroll 1
                for (int c = first_owned; c < chunk_end; c += share) {
                    fetch_bias32<EPI>(p.bias, static_cast<int64_t>(nt) * BN + c * kStoreCols, p.N,
                                      bias_vec, bias_next);
                    if (folding) {
                        load_acc_chunk(c, ra);
                    } else {
                        tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(c * kStoreCols), ra);
                        tmem_wait_ld_dep(ra);
                    }
                    emit(c, ra);
                }
            }
            if (!shared && !folding && chunk_end > chunk0)
                tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(chunk0 * kStoreCols), ra);
#pragma unroll 1
            for (int c = chunk0; !shared && c < chunk_end; c += 2) {
                if (folding)
                    load_acc_chunk(c, ra);
                else
                    tmem_wait_ld_dep(ra);
                if (!folding && c + 1 < chunk_end)
                    tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>((c + 1) * kStoreCols), rb);
                emit(c, ra);
                if (c + 1 >= chunk_end) break;
                if (folding)
                    load_acc_chunk(c + 1, rb);
                else
                    tmem_wait_ld_dep(rb);
                if (!folding && c + 2 < chunk_end)
                    tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>((c + 2) * kStoreCols), ra);
                emit(c + 1, rb);
            }
            fold_drain();
            // All TMEM reads of this accumulator are complete (wait::ld above).
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) {
                if (PAIR)
                    mbar_arrive_cluster(empty_bar_leader + static_cast<uint32_t>(acc * 8));
                else
                    mbar_arrive(&tmem_empty_bar[acc]);
            }
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
        if (STORE == kStoreTma && lane == 0) bulk_wait_group_read<0>();
        __syncwarp();
    }

    // Teardown: every role has returned (all waits are bounded), so no thread
    // still reads TMEM and no MMA or copy tracked by this CTA is in flight.
    // The next kernel in the stream may start its prologue now.
    if (!p.early_trigger) grid_launch_dependents();
    tc_fence_before_sync();
    __syncthreads();
    if (PAIR) cluster_sync();   // the leader's MMAs into this CTA's TMEM are done
    if (warp == S::kMmaWarp) {
        tc_fence_after_sync();
        tmem_dealloc<CG>(tmem_base, S::kTmemCols);
    }
}

// ---------------------------------------------------------------------------
}  // namespace tg
