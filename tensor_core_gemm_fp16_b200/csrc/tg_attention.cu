// tg_attention.cu -- fused attention forward for sm_100a (tcgen05 + TMEM + TMA)
// and the host side of include/tg_attention.h.
//
// The operation is the FlashAttention forward of "Designing High-Performance
// GPU Kernels with TileLang" (ainovat.com, FlashAttention section): per
// (batch, head) and tile of queries, the key/value tiles are visited in
// order; the scores S = Q K^T of one tile never leave the SM; an online
// softmax keeps each row's running maximum m and sum l, rescaling the output
// accumulator when m grows; O += P V; at the end O / l is written once.
//
// B200 design: one CTA per (batch x head, pair of 128-query tiles t = 0, 1),
// ten warps.
//   warps 4t .. 4t+3  softmax of tile t: thread r owns query row r of the tile
//              (TMEM lane r).  Reads S_t from TMEM, masks, exponentiates, and
//              writes P_t (fp16), where the tensor core reads it as the A
//              operand of P_t V; rescales O_t in TMEM when needed; stores
//              O_t / l at the end.
//   warp 8     TMA producer (one lane): Q for both tiles, then the K and V
//              tiles into their rings, polling both rings' empty barriers
//              without blocking so neither ring waits on the other.
//   warp 9     TMEM allocator and MMA issuer (one lane).
// TMEM: tile t owns columns [256 t, 256 t + 256).  Head width 64: S_t in the
// first 128, P_t (two fp16 per 32-bit column) in the next 64, O_t in the last
// 64.  Head width 128: S_t in the first 128 and O_t in the next 128, which
// fills TMEM, so P_t goes to shared memory instead: a 128 x 128 fp16 tile per
// query tile in the 128-byte-swizzled layout of the tensor core's A operand
// (room for it comes from a single V stage).  Either way P never overwrites
// S, so S_t,j+1 can be issued as soon as the softmax group has read S_t,j,
// while it still exponentiates; the group's next step then finds its scores
// ready.  The two tiles' softmax phases run side by side on the SM, sharing
// the SFU, while the tensor core's products proceed; a quarter of the
// exponentials (head width 128) are computed on the FMA pipe instead of the
// SFU, so that both units work.
//
// Order of the MMA issuer per key tile j (each wait bounded): S_0,j+1 and
// S_1,j+1 as soon as the groups have read S_t,j (s_free), then P_0,j V_j and
// P_1,j V_j as the groups publish P (p_full).  A group waits for
// P_t,j-1 V_j-1 itself before it rescales O_t or writes P_t.
//
// Lazy rescaling: a row keeps its maximum m until a tile raises it by more
// than 8 (in log2 units), so exponentials stay below 2^8 and O is rescaled
// in TMEM only on those tiles; O / l uses the same m, so the result is the
// same softmax.
//
// Key-half split (non-causal): when the last wave of units would fill at
// most half of the SMs, each of its units runs as two CTAs over the first and
// the second half of the key tiles.  Each half publishes its unnormalised O,
// m and l; the warp that finds its partner's publication (an epoch swapped
// into a flag word) merges the two with the same rescaling, half 0's terms
// first.  Nothing waits on the other half.
//
// Every mbarrier wait is bounded by a global-timer limit; on expiry a CTA
// abort flag is set, a site bit is OR-ed into the library error word, and
// the CTA tears down after letting its own copies and MMAs land.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>

#include "tg_attention.h"
#include "tg_internal.h"
#include "tg_ptx.cuh"

namespace tga {

using namespace tg;

constexpr int kTileQ = 128;        // queries per tile (TMEM lanes)
constexpr int kTilesPerCta = 2;
constexpr int kTileK = 128;        // keys per tile (score columns)
constexpr int kAtom = 64;          // head-dim elements per 128-byte swizzle atom
constexpr int kAtomBytes = 128 * 128;   // one 128-row x 64-element fp16 box
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kThreads = 32 * 10;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTileCols = 256;     // per tile, see the layout above

// Error word bits (shared word with the GEMM kernels; these sites are the
// attention kernel's).
constexpr unsigned kErrAttnProducer = 64u;
constexpr unsigned kErrAttnMma = 128u;
constexpr unsigned kErrAttnSoftmax = 256u;
constexpr unsigned kErrAttnDrain = 512u;

struct AttnParams {
    __half *O;
    int64_t Sq, Sk;
    int num_bh;          // batch x heads
    int num_qp;          // pairs of query tiles per (batch, head)
    int causal;
    float scale_log2;    // scale * log2(e)
    int inject;
    uint64_t wait_limit_ns;
    unsigned *error_word;
    // Work division.  A unit is one (batch x head, pair of query tiles); units
    // [0, num_full) take one CTA each, the next split_units take two CTAs,
    // one per half of the key tiles, and are combined by whichever half
    // finishes second (non-causal only).
    int num_full;
    int split_units;
    float *part;         // [split unit][key half][tile][D + 2][128]: O (unnormalised), m, l
    unsigned *flags;     // [split unit][tile][lane quarter]: epoch of the first half to finish
    unsigned epoch;
};

template <int D>
struct AttnShape {
    static_assert(D == 64 || D == 128, "head_dim 64 or 128");
    static constexpr int kAtoms = D / kAtom;
    static constexpr int kKStages = D == 64 ? 4 : 2;    // K ring depth
    static constexpr int kVStages = D == 64 ? 4 : 1;    // V ring depth
    // P in its own TMEM columns (head width 64) or in shared memory (128)
    static constexpr bool kPSmem = D == 128;
    static constexpr uint32_t kPCol = 128u;             // head width 64
    static constexpr uint32_t kOCol = kPSmem ? 128u : 192u;
    // One pair of scores in kEmuShare takes the FMA-pipe exponential (0: none)
    static constexpr int kEmuShare = D == 128 ? 4 : 0;
    static constexpr int kTileBytes = kAtoms * kAtomBytes;   // one 128-row Q, K or V tile
    static constexpr int kQOff = 0;                          // Q of both query tiles
    static constexpr int kKOff = kQOff + kTilesPerCta * kTileBytes;
    static constexpr int kVOff = kKOff + kKStages * kTileBytes;
    // P of each query tile, 128 rows x 128 keys as two 64-key atoms (head width 128)
    static constexpr int kPTileBytes = kTileQ * kTileK * 2;
    static constexpr int kPOff = kVOff + kVStages * kTileBytes;
    static constexpr int kPBytes = kPSmem ? kTilesPerCta * kPTileBytes : 0;
    // barriers: q_full, k_full[SK], k_empty[SK], v_full[SV], v_empty[SV],
    // s_full[2], p_full[2], pv_done[2], s_free[2], drain
    static constexpr int kNumBars = 1 + 2 * kKStages + 2 * kVStages + 8 + 1;
    static constexpr int kBarOff = kPOff + kPBytes;
    static constexpr int kTmemSlotOff = kBarOff + kNumBars * 8;
    static constexpr int kAbortOff = kTmemSlotOff + 4;
    static constexpr int kDynamicBytes = kAbortOff + 4 + 1024;
    static_assert(kDynamicBytes <= 232448, "shared-memory budget");
};

// Instruction descriptor for kind::f16 with fp32 D and both operands K-major
// (S = Q K^T: rows of Q and of K are contiguous along the head dimension).
__host__ __device__ constexpr uint32_t idesc_f16_f32_kk(int m, int n)
{
    return (1u << 4) | (static_cast<uint32_t>(n >> 3) << 17) |
           (static_cast<uint32_t>(m >> 4) << 24);
}

// D (TMEM) += A (TMEM: 128 lanes x 16 fp16, two per 32-bit column) x B (shared
// memory descriptor).
__device__ __forceinline__ void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst_smem, const CUtensorMap *tm,
                                            uint64_t *bar, int32_t x, int32_t y, int32_t z)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst_smem),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
        : "memory");
}

__device__ __forceinline__ float ex2(float x)
{
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ float rcp(float x)
{
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// Two fp32 values in one 64-bit register, and the packed f32x2 arithmetic of
// sm_100 (one instruction for both halves).
__device__ __forceinline__ uint64_t f2(float lo, float hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ void f2split(uint64_t v, float &lo, float &hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// 2^x for two values on the FMA pipe, so that part of the softmax's
// exponentials leave the SFU (fit_exp2.py fits R and checks this sequence):
// x = n + r with n = round(x), r in [-1/2, 1/2]; R(r) = 1 + c1 r + c2 r^2 +
// c3 r^3 ~ 2^r by Horner in packed f32x2 arithmetic; n is added to R's
// exponent field, taken from the low bits of x + 1.5 * 2^23.  x is first
// raised to -125 (a masked score, -inf, gives about 2^-125, which rounds to
// 0 in fp16 P).  Integer x gives 2^x exactly; elsewhere the relative error
// stays below 1.1e-4, under the fp16 rounding P gets next.  A NaN score does
// not propagate here; the row maximum carries it instead.
constexpr float kExp2C1 = 6.932827830e-01f;
constexpr float kExp2C2 = 2.422083467e-01f;
constexpr float kExp2C3 = 5.500787124e-02f;
constexpr float kExp2Round = 12582912.0f;   // 1.5 * 2^23

__device__ __forceinline__ float max_nan(float a, float b)
{
    float r;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}

__device__ __forceinline__ float min_nan(float a, float b)
{
    float r;
    asm("min.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}

__device__ __forceinline__ uint64_t exp2_fma2(float x0, float x1)
{
    const uint64_t x2 = f2(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
    const uint64_t t2 = fadd2(x2, f2(kExp2Round, kExp2Round));
    const uint64_t n2 = fadd2(t2, f2(-kExp2Round, -kExp2Round));
    const uint64_t r2 = ffma2(n2, f2(-1.f, -1.f), x2);
    uint64_t p2 = ffma2(f2(kExp2C3, kExp2C3), r2, f2(kExp2C2, kExp2C2));
    p2 = ffma2(p2, r2, f2(kExp2C1, kExp2C1));
    p2 = ffma2(p2, r2, f2(1.f, 1.f));
    float t0, t1, q0, q1;
    f2split(t2, t0, t1);
    f2split(p2, q0, q1);
    return f2(__uint_as_float(__float_as_uint(q0) + (__float_as_uint(t0) << 23)),
              __uint_as_float(__float_as_uint(q1) + (__float_as_uint(t1) << 23)));
}

// 16 consecutive 32-bit TMEM columns of this thread's lane from r (the
// 16-column form of tmem_st_32x32b_x32).
__device__ __forceinline__ void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
        : "memory");
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d)
{
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi)
{
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

// Keys visible to query tile (pair qp, tile t): all key tiles, or with the
// causal mask those up to the one holding the tile's last query; 0 for a tile
// that lies entirely past seq_q.
__device__ __forceinline__ int tile_key_tiles(const AttnParams &p, int64_t q0)
{
    if (q0 >= p.Sq) return 0;
    const int64_t kv_tiles = (p.Sk + kTileK - 1) / kTileK;
    const int64_t kv_causal = (q0 + kTileQ - 1) / kTileK + 1;
    return static_cast<int>(p.causal && kv_causal < kv_tiles ? kv_causal : kv_tiles);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ,
                    const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const AttnParams p)
{
    using S = AttnShape<D>;
    constexpr int SK = S::kKStages;
    constexpr int SV = S::kVStages;

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(smem);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + S::kBarOff);
    uint64_t *q_full = bars;
    uint64_t *k_full = bars + 1;
    uint64_t *k_empty = k_full + SK;
    uint64_t *v_full = k_empty + SK;
    uint64_t *v_empty = v_full + SV;
    uint64_t *s_full = v_empty + SV;     // [2]: S_t of the current key tile is in TMEM
    uint64_t *p_full = s_full + 2;       // [2]: P_t written to TMEM (4 arrivals)
    uint64_t *pv_done = p_full + 2;      // [2]: P_t V complete
    uint64_t *s_free = pv_done + 2;      // [2]: S_t read out of TMEM (4 arrivals)
    uint64_t *drain_bar = s_free + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + S::kTmemSlotOff);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + S::kAbortOff);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // Unit of this CTA, and its key half (-1: all key tiles).
    int unit = static_cast<int>(blockIdx.x), half = -1;
    if (unit >= p.num_full) {
        const int i = unit - p.num_full;
        unit = p.num_full + (i >> 1);
        half = i & 1;
    }
    // Heavier query pairs first (causal: later queries see more keys).
    const int qp = p.num_qp - 1 - unit / p.num_bh;
    const int bh = unit % p.num_bh;
    const int64_t qbase = static_cast<int64_t>(qp) * kTilesPerCta * kTileQ;
    const int n0_all = tile_key_tiles(p, qbase);
    const int n1_all = tile_key_tiles(p, qbase + kTileQ);
    const int n_units = n0_all > n1_all ? n0_all : n1_all;
    // Key tiles [kv_lo, kv_lo + n_t) for tile t; j below counts from kv_lo.
    // A split unit is non-causal, so each tile has all key tiles or none.
    const int kv_lo = half == 1 ? n_units / 2 : 0;
    const int kv_n = half < 0 ? n_units : (half == 0 ? n_units / 2 : n_units - n_units / 2);
    const int n0 = half < 0 ? n0_all : (n0_all > 0 ? kv_n : 0);
    const int n1 = half < 0 ? n1_all : (n1_all > 0 ? kv_n : 0);
    const int n_all = n0 > n1 ? n0 : n1;
    const uint64_t limit = p.wait_limit_ns;

    if (threadIdx.x == 0) {
        for (int b = 0; b < S::kNumBars; ++b) {
            uint64_t *bar = &bars[b];
            mbar_init(bar, (bar == &p_full[0] || bar == &p_full[1] || bar == &s_free[0] ||
                            bar == &s_free[1])
                               ? 4u
                               : 1u);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kProducerWarp && lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
    }
    if (warp == kMmaWarp) {
        tmem_alloc<1>(tmem_slot, kTmemCols);
        tmem_relinquish<1>();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == kProducerWarp) {
        if (lane == 0 && n_all > 0) {
            // Q of both tiles (rows past seq_q read as zero), then both rings.
            mbar_arrive_expect_tx(q_full, kTilesPerCta * S::kTileBytes);
            for (int t = 0; t < kTilesPerCta; ++t)
                for (int a = 0; a < S::kAtoms; ++a)
                    tma_load_3d(sbase + S::kQOff + t * S::kTileBytes + a * kAtomBytes, &tmQ,
                                q_full, a * kAtom, static_cast<int32_t>(qbase + t * kTileQ), bh);
            int jk = 0, jv = 0;
            int k_filled[SK], v_filled[SV];
            for (int st = 0; st < SK; ++st) k_filled[st] = 0;
            for (int st = 0; st < SV; ++st) v_filled[st] = 0;
            uint64_t t_idle = 0;
            bool ok = true;
            while (ok && (jk < n_all || jv < n_all)) {
                bool progress = false;
                if (jk < n_all &&
                    (jk < SK || mbar_test_wait(&k_empty[jk % SK], ((jk / SK) - 1) & 1))) {
                    const int st = jk % SK;
                    const uint32_t kdst = sbase + S::kKOff + st * S::kTileBytes;
                    mbar_arrive_expect_tx(&k_full[st], S::kTileBytes);
                    if (!(p.inject == 1 && blockIdx.x == 0 && jk == 0))
                        for (int a = 0; a < S::kAtoms; ++a)
                            tma_load_3d(kdst + a * kAtomBytes, &tmK, &k_full[st], a * kAtom,
                                        (kv_lo + jk) * kTileK, bh);
                    k_filled[st] = jk / SK + 1;
                    ++jk;
                    progress = true;
                }
                if (jv < n_all &&
                    (jv < SV || mbar_test_wait(&v_empty[jv % SV], ((jv / SV) - 1) & 1))) {
                    const int st = jv % SV;
                    const uint32_t vdst = sbase + S::kVOff + st * S::kTileBytes;
                    mbar_arrive_expect_tx(&v_full[st], S::kTileBytes);
                    for (int a = 0; a < S::kAtoms; ++a)
                        tma_load_3d(vdst + a * kAtomBytes, &tmV, &v_full[st], a * kAtom,
                                    (kv_lo + jv) * kTileK, bh);
                    v_filled[st] = jv / SV + 1;
                    ++jv;
                    progress = true;
                }
                if (progress) {
                    t_idle = 0;
                } else {
                    // Bounded: give up after the wait limit without progress.
                    if (*abort_flag) break;
                    const uint64_t now = global_timer_ns();
                    if (t_idle == 0) {
                        t_idle = now;
                    } else if (now - t_idle > limit) {
                        *abort_flag = 1;
                        atomicOr(p.error_word, kErrAttnProducer);
                        ok = false;
                    }
                }
            }
            // Let every copy this thread issued land before shared memory goes away
            // (the injected test skips one load, whose barrier never completes).
            if (!mbar_wait_drain(q_full, 0, limit)) atomicOr(p.error_word, kErrAttnDrain);
            for (int st = 0; st < SK; ++st)
                if (k_filled[st] > 0 && !(p.inject == 1 && blockIdx.x == 0 && st == 0 &&
                                          k_filled[st] == 1) &&
                    !mbar_wait_drain(&k_full[st], (k_filled[st] - 1) & 1, limit))
                    atomicOr(p.error_word, kErrAttnDrain);
            for (int st = 0; st < SV; ++st)
                if (v_filled[st] > 0 &&
                    !mbar_wait_drain(&v_full[st], (v_filled[st] - 1) & 1, limit))
                    atomicOr(p.error_word, kErrAttnDrain);
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        if (lane == 0 && n_all > 0) {
            constexpr uint32_t kIdescS = idesc_f16_f32_kk(kTileQ, kTileK);
            constexpr uint32_t kIdescO = idesc_f16_f32(kTileQ, D);
            const int nt[2] = {n0, n1};
            bool ok = mbar_wait_bounded(q_full, 0, abort_flag, limit, p.error_word, kErrAttnMma);
            bool issued = false;
            auto wait = [&](uint64_t *bar, uint32_t parity) {
                if (ok)
                    ok = mbar_wait_bounded(bar, parity, abort_flag, limit, p.error_word,
                                           kErrAttnMma);
                return ok;
            };
            // S_t,j = Q_t K_j^T into tile t's score columns.
            auto issue_s = [&](int t, int j) {
                const uint32_t qa = sbase + S::kQOff + t * S::kTileBytes;
                const uint32_t ka = sbase + S::kKOff + (j % SK) * S::kTileBytes;
                tc_fence_after_sync();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kAtomBytes + (kk & 3) * 32;
                    mma_f16_ss<1>(tmem_base + t * kTileCols, smem_desc_sw128(qa + off, 16, 1024),
                                  smem_desc_sw128(ka + off, 16, 1024), kIdescS, kk > 0);
                }
                mma_commit<1>(&s_full[t]);
                issued = true;
            };
            // O_t += P_t,j V_j: P from shared memory (head width 128, the
            // same 64-key atoms as Q) or from TMEM (8 columns per 16 keys).
            auto issue_pv = [&](int t, int j) {
                const uint32_t va = sbase + S::kVOff + (j % SV) * S::kTileBytes;
                tc_fence_after_sync();
#pragma unroll
                for (int kk = 0; kk < kTileK / 16; ++kk) {
                    const uint64_t vdesc = smem_desc_sw128(va + kk * 2048, kAtomBytes, 1024);
                    const uint32_t acc = (j > 0 || kk > 0) ? 1u : 0u;
                    if constexpr (S::kPSmem) {
                        const uint32_t off = (kk >> 2) * kAtomBytes + (kk & 3) * 32;
                        mma_f16_ss<1>(tmem_base + t * kTileCols + S::kOCol,
                                      smem_desc_sw128(sbase + S::kPOff + t * S::kPTileBytes + off,
                                                      16, 1024),
                                      vdesc, kIdescO, acc);
                    } else {
                        mma_f16_ts(tmem_base + t * kTileCols + S::kOCol,
                                   tmem_base + t * kTileCols + S::kPCol +
                                       static_cast<uint32_t>(kk * 8),
                                   vdesc, kIdescO, acc);
                    }
                }
                mma_commit<1>(&pv_done[t]);
                issued = true;
            };
            if (wait(&k_full[0], 0)) {
                for (int t = 0; t < 2; ++t)
                    if (nt[t] > 0) issue_s(t, 0);
                mma_commit<1>(&k_empty[0]);
            }
            for (int j = 0; ok && j < n_all; ++j) {
                // S_t,j+1 as soon as group t has read S_t,j.
                bool k_next = false;   // K_j+1 waited for
                for (int t = 0; t < 2 && ok; ++t) {
                    if (j + 1 < nt[t]) {
                        if (!k_next && !wait(&k_full[(j + 1) % SK], ((j + 1) / SK) & 1)) break;
                        k_next = true;
                        if (!wait(&s_free[t], j & 1)) break;
                        issue_s(t, j + 1);
                    }
                }
                if (!ok || !wait(&v_full[j % SV], (j / SV) & 1)) break;
                for (int t = 0; t < 2 && ok; ++t)
                    if (j < nt[t]) {
                        if (!wait(&p_full[t], j & 1)) break;
                        issue_pv(t, j);
                    }
                if (!ok) break;
                mma_commit<1>(&v_empty[j % SV]);
                if (j + 1 < n_all) mma_commit<1>(&k_empty[(j + 1) % SK]);
            }
            if (issued) {
                mma_commit<1>(drain_bar);
                if (!mbar_wait_drain(drain_bar, 0, limit)) atomicOr(p.error_word, kErrAttnDrain);
            }
        }
        __syncwarp();
    } else {
        // Softmax group t = warp / 4: row r = 32 (warp % 4) + lane of query tile t.
        const int t = warp >> 2;
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const int64_t q0 = qbase + static_cast<int64_t>(t) * kTileQ;
        const int64_t qi = q0 + row;
        const int n_kv = t == 0 ? n0 : n1;
        const uint32_t t_lane =
            tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + t * kTileCols;
        const float sl2 = p.scale_log2;
        const bool pos = sl2 > 0.f;
        float m = -INFINITY;   // running maximum of the scaled scores, log2 units
        float l = 0.f;         // running sum of 2^(score - m)
        bool ok = true;
        for (int j = 0; j < n_kv; ++j) {
            int okw = 1;
            if (lane == 0)
                okw = mbar_wait_bounded(&s_full[t], j & 1, abort_flag, limit, p.error_word,
                                        kErrAttnSoftmax)
                          ? 1
                          : 0;
            okw = __shfl_sync(0xffffffffu, okw, 0);
            if (!okw) {
                ok = false;
                break;
            }
            tc_fence_after_sync();
            // Mask keys past seq_k and, causal, past qi, on the raw scores: the
            // masked value turns into -inf once scaled (the scale's sign decides
            // which infinity).  The row maximum of the scaled scores is the scale
            // times the raw maximum (or minimum, for a negative scale), and each
            // exponent is one fused multiply-add: 2^(s * scale * log2 e - m).
            const int64_t key0 = static_cast<int64_t>(kv_lo + j) * kTileK;
            const bool need_mask =
                key0 + kTileK > p.Sk || (p.causal && key0 + kTileK - 1 > q0);
            int64_t lim = kTileK;   // valid columns: keys [key0, Sk) and, causal, <= qi
            if (need_mask) {
                lim = p.Sk - key0;
                if (p.causal && qi + 1 - key0 < lim) lim = qi + 1 - key0;
            }
            const float masked = pos ? -INFINITY : INFINITY;
            // The whole 128-score row comes out of TMEM in one round trip (four
            // loads behind one wait) and stays in registers for both the
            // maximum and the exponentials.
            uint32_t s0[32], s1[32], s2[32], s3[32];
            tmem_ld_32x32b_x32(t_lane + 0u, s0);
            tmem_ld_32x32b_x32(t_lane + 32u, s1);
            tmem_ld_32x32b_x32(t_lane + 64u, s2);
            tmem_ld_32x32b_x32(t_lane + 96u, s3);
            tmem_wait_ld_dep(s0);
            tmem_wait_ld_dep(s1);
            tmem_wait_ld_dep(s2);
            tmem_wait_ld_dep(s3);
            // All of S_t,j is in registers: S_t,j+1 may land.
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_free[t]);
            auto mask32 = [&](uint32_t (&x)[32], int c0) {
                if (need_mask) {
#pragma unroll
                    for (int c = 0; c < 32; ++c)
                        if (c0 + c >= lim) x[c] = __float_as_uint(masked);
                }
            };
            mask32(s0, 0);
            mask32(s1, 32);
            mask32(s2, 64);
            mask32(s3, 96);
            float mx[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) mx[u] = masked;
            // The extreme keeps NaN (a NaN score makes the row NaN, as the
            // exact softmax would).
            auto ext32 = [&](const uint32_t (&x)[32]) {
                if (pos) {
#pragma unroll
                    for (int c = 0; c < 32; ++c) mx[c & 7] = max_nan(mx[c & 7], __uint_as_float(x[c]));
                } else {
#pragma unroll
                    for (int c = 0; c < 32; ++c) mx[c & 7] = min_nan(mx[c & 7], __uint_as_float(x[c]));
                }
            };
            ext32(s0);
            ext32(s1);
            ext32(s2);
            ext32(s3);
            const float rext =
                pos ? max_nan(max_nan(max_nan(mx[0], mx[1]), max_nan(mx[2], mx[3])),
                              max_nan(max_nan(mx[4], mx[5]), max_nan(mx[6], mx[7])))
                    : min_nan(min_nan(min_nan(mx[0], mx[1]), min_nan(mx[2], mx[3])),
                              min_nan(min_nan(mx[4], mx[5]), min_nan(mx[6], mx[7])));
            const float tmax = rext * sl2;
            // Lazy rescale: move m only when the tile raises it by more than 8
            // (or brings a NaN, which then reaches every exponential).
            float alpha = 1.f;
            const bool raise = !(tmax <= m + 8.f);
            if (raise) {
                alpha = (m == -INFINITY) ? 0.f : ex2(m - tmax);
                m = tmax;
            }
            const float mu = (m == -INFINITY) ? 0.f : m;
            // Before O_t is rescaled or P_t written, P_t,j-1 V_j-1 must be
            // complete.
            auto wait_prev = [&]() -> bool {
                int okv = 1;
                if (lane == 0 && j > 0)
                    okv = mbar_wait_bounded(&pv_done[t], (j - 1) & 1, abort_flag, limit,
                                            p.error_word, kErrAttnSoftmax)
                              ? 1
                              : 0;
                okv = __shfl_sync(0xffffffffu, okv, 0);
                tc_fence_after_sync();
                return okv != 0;
            };
            auto rescale_o = [&]() {
                if (j > 0 && __any_sync(0xffffffffu, raise)) {
#pragma unroll 1
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t o[32];
                        const uint32_t t_o = t_lane + S::kOCol + static_cast<uint32_t>(c * 32);
                        tmem_ld_32x32b_x32(t_o, o);
                        tmem_wait_ld_dep(o);
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        tmem_st_32x32b_x32(t_o, o);
                    }
                }
            };
            // P row: head width 64 into TMEM columns [128, 192), keys 2i, 2i + 1
            // packed into column i; head width 128 into the shared P tile, row
            // r of each 64-key atom at 128 r with its 16-byte chunks swizzled
            // by r mod 8.  Arguments and partial sums use the packed f32x2 FMA
            // and add.
            const uint64_t sl2x2 = f2(sl2, sl2);
            const uint64_t nmu2 = f2(-mu, -mu);
            uint64_t ps2[4] = {0, 0, 0, 0};
            // 32 scores -> 16 packed P values.
            auto exp32 = [&](const uint32_t (&x)[32], uint32_t *hp) {
#pragma unroll
                for (int c = 0; c < 32; c += 2) {
                    const int pr = c >> 1;
                    const uint64_t a2 =
                        ffma2(f2(__uint_as_float(x[c]), __uint_as_float(x[c + 1])), sl2x2, nmu2);
                    float a0, a1, e0, e1;
                    f2split(a2, a0, a1);
                    if (S::kEmuShare > 0 && pr % S::kEmuShare == S::kEmuShare - 1) {
                        f2split(exp2_fma2(a0, a1), e0, e1);
                    } else {
                        e0 = ex2(a0);
                        e1 = ex2(a1);
                    }
                    ps2[pr & 3] = fadd2(ps2[pr & 3], f2(e0, e1));
                    hp[pr] = pack_half2(e0, e1);
                }
            };
            if constexpr (S::kPSmem) {
                // The whole P row in registers first, then (P_t,j-1 V_j-1 done)
                // into the tile's P tile.
                uint32_t hp[64];
                exp32(s0, hp);
                exp32(s1, hp + 16);
                exp32(s2, hp + 32);
                exp32(s3, hp + 48);
                if (!wait_prev()) {
                    ok = false;
                    break;
                }
                rescale_o();
                const uint32_t prow = sbase + S::kPOff + t * S::kPTileBytes + row * 128;
#pragma unroll
                for (int c = 0; c < 16; ++c)   // 16-byte chunk c: keys 8c .. 8c + 7
                    st_shared_v4(prow + (c >> 3) * kAtomBytes + (((c & 7) ^ (row & 7)) << 4),
                                 hp[4 * c], hp[4 * c + 1], hp[4 * c + 2], hp[4 * c + 3]);
            } else {
                if (!wait_prev()) {
                    ok = false;
                    break;
                }
                rescale_o();
                // 32 scores -> 16 packed P columns at a time (keeps the live
                // registers within the launch's budget).
                auto exp_store = [&](const uint32_t (&x)[32], int q) {
                    uint32_t hp[16];
                    exp32(x, hp);
                    tmem_st_32x32b_x16(t_lane + S::kPCol + static_cast<uint32_t>(q * 16), hp);
                };
                exp_store(s0, 0);
                exp_store(s1, 1);
                exp_store(s2, 2);
                exp_store(s3, 3);
            }
            float q0, q1, q2, q3;
            f2split(fadd2(ps2[0], ps2[1]), q0, q1);
            f2split(fadd2(ps2[2], ps2[3]), q2, q3);
            l = fmaf(l, alpha, (q0 + q1) + (q2 + q3));
            tmem_wait_st();
            if constexpr (S::kPSmem) fence_proxy_async_smem();   // P visible to the tensor core
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[t]);
        }
        if (ok && n_kv > 0) {
            int okw = 1;
            if (lane == 0)
                okw = mbar_wait_bounded(&pv_done[t], (n_kv - 1) & 1, abort_flag, limit,
                                        p.error_word, kErrAttnSoftmax)
                          ? 1
                          : 0;
            okw = __shfl_sync(0xffffffffu, okw, 0);
            if (okw) {
                tc_fence_after_sync();
                // Whole unit: O / l.  Split unit: publish this half's O, m and l
                // (column-major over the tile's rows, so a warp's accesses are
                // coalesced); the half that finishes second merges both:
                //   O = (O_a 2^(m_a - m) + O_b 2^(m_b - m)) / (l_a 2^(m_a - m) + l_b 2^(m_b - m)),
                //   m = max(m_a, m_b).
                float wa = 1.f, wb = 0.f;   // weights of this half's O and of the other's
                const float *other = nullptr;
                bool store = true;
                if (half >= 0) {
                    const int us = unit - p.num_full;
                    float *mine =
                        p.part + static_cast<size_t>((us * 2 + half) * 2 + t) * (D + 2) * kTileQ;
                    other = p.part +
                            static_cast<size_t>((us * 2 + (1 - half)) * 2 + t) * (D + 2) * kTileQ;
#pragma unroll 1
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t o[32];
                        tmem_ld_32x32b_x32(t_lane + S::kOCol + static_cast<uint32_t>(c * 32), o);
                        tmem_wait_ld_dep(o);
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            __stcg(mine + (c * 32 + e) * kTileQ + row, __uint_as_float(o[e]));
                    }
                    __stcg(mine + D * kTileQ + row, m);
                    __stcg(mine + (D + 1) * kTileQ + row, l);
                    __threadfence();
                    __syncwarp();
                    unsigned prev = 0;
                    if (lane == 0) prev = atomicExch(&p.flags[(us * 2 + t) * 4 + quarter], p.epoch);
                    prev = __shfl_sync(0xffffffffu, prev, 0);
                    store = prev == p.epoch;
                    if (store) {
                        __threadfence();
                        const float mo = __ldcg(other + D * kTileQ + row);
                        const float lo = __ldcg(other + (D + 1) * kTileQ + row);
                        const float mm = fmaxf(m, mo);
                        wa = m == -INFINITY ? 0.f : ex2(m - mm);
                        wb = mo == -INFINITY ? 0.f : ex2(mo - mm);
                        // Half 0's terms first, whichever half merges: the
                        // result does not depend on which finished second.
                        l = half == 0 ? fmaf(lo, wb, l * wa) : fmaf(l, wa, lo * wb);
                    }
                }
                if (store) {
                    const float inv_l = l > 0.f ? rcp(l) : 0.f;
                    const float sa = wa * inv_l, sb = wb * inv_l;
                    __half *orow = p.O + (static_cast<int64_t>(bh) * p.Sq + qi) * D;
#pragma unroll 1
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t o[32];
                        tmem_ld_32x32b_x32(t_lane + S::kOCol + static_cast<uint32_t>(c * 32), o);
                        tmem_wait_ld_dep(o);
                        if (qi < p.Sq) {
                            float v[32];
#pragma unroll
                            for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(o[e]) * sa;
                            if (other) {
#pragma unroll
                                for (int e = 0; e < 32; ++e) {
                                    const float x = __ldcg(other + (c * 32 + e) * kTileQ + row);
                                    v[e] = half == 0 ? fmaf(x, sb, v[e])
                                                     : fmaf(__uint_as_float(o[e]), sa, x * sb);
                                }
                            }
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                uint4 u;
                                u.x = pack_half2(v[q * 8 + 0], v[q * 8 + 1]);
                                u.y = pack_half2(v[q * 8 + 2], v[q * 8 + 3]);
                                u.z = pack_half2(v[q * 8 + 4], v[q * 8 + 5]);
                                u.w = pack_half2(v[q * 8 + 6], v[q * 8 + 7]);
                                *reinterpret_cast<uint4 *>(orow + c * 32 + q * 8) = u;
                            }
                        }
                    }
                }
            }
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after_sync();
        tmem_dealloc<1>(tmem_base, kTmemCols);
    }
}

}  // namespace tga

namespace {

constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;

bool encode_3d(PFN_cuTensorMapEncodeTiled_v12000 encode, CUtensorMap *tm, const void *base,
               uint64_t d, uint64_t s, uint64_t bh)
{
    const cuuint64_t dims[3] = {d, s, bh};
    const cuuint64_t strides[2] = {d * 2, s * d * 2};
    const cuuint32_t box[3] = {tga::kAtom, tga::kTileQ, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return encode(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void *>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Workspace of the key-half split, per (device, stream): the halves' partial
// results and one flag word per (split unit, tile, lane quarter).  It grows
// in stream order (cudaFreeAsync / cudaMallocAsync on the caller's stream);
// each launch takes a fresh epoch, so flags need no reset between launches.
struct SplitWorkspace {
    void *mem = nullptr;
    int units = 0;
    unsigned epoch = 0;
};
std::mutex g_ws_mutex;
std::map<std::pair<int, cudaStream_t>, SplitWorkspace> g_split_ws;

// Floats of partial results per split unit: 2 key halves x 2 tiles x (O of
// up to 128 columns, m, l) x 128 rows.
constexpr size_t split_part_floats(int units)
{
    return static_cast<size_t>(units) * 2 * 2 * (128 + 2) * tga::kTileQ;
}

tg_status_t split_workspace(int units, cudaStream_t stream, float **part, unsigned **flags,
                            unsigned *epoch)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return TG_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(g_ws_mutex);
    SplitWorkspace &w = g_split_ws[std::make_pair(dev, stream)];
    if (units > w.units) {
        const size_t part_bytes = split_part_floats(units) * sizeof(float);
        const size_t flag_bytes = static_cast<size_t>(units) * 2 * 4 * sizeof(unsigned);
        if (w.mem && cudaFreeAsync(w.mem, stream) != cudaSuccess) {
            cudaGetLastError();
            return TG_ERR_CUDA;
        }
        w.mem = nullptr;
        w.units = 0;
        if (cudaMallocAsync(&w.mem, part_bytes + flag_bytes, stream) != cudaSuccess) {
            cudaGetLastError();
            w.mem = nullptr;
            return TG_ERR_OOM;
        }
        if (cudaMemsetAsync(static_cast<char *>(w.mem) + part_bytes, 0, flag_bytes, stream) !=
            cudaSuccess) {
            cudaGetLastError();
            return TG_ERR_CUDA;
        }
        w.units = units;
    }
    if (++w.epoch == 0) w.epoch = 1;
    *part = static_cast<float *>(w.mem);
    *flags = reinterpret_cast<unsigned *>(static_cast<char *>(w.mem) +
                                          split_part_floats(w.units) * sizeof(float));
    *epoch = w.epoch;
    return TG_OK;
}

// Units split into key halves.  Auto: when the last wave of units would fill
// at most half of the SMs, its units are split, so that it takes half as
// long; never for causal attention or a single key tile.
int split_units(int64_t units, int num_sms, int64_t key_tiles, int causal, int mode)
{
    if (causal || key_tiles < 2 || mode == TG_ATTN_SPLIT_NEVER) return 0;
    if (mode == TG_ATTN_SPLIT_ALL) return static_cast<int>(units);
    const int64_t rem = units % num_sms;
    return rem > 0 && 2 * rem <= num_sms ? static_cast<int>(rem) : 0;
}

bool overlaps(const void *a, size_t na, const void *b, size_t nb)
{
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return na && nb && x < y + nb && y < x + na;
}

template <int D>
tg_status_t launch_attn(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                        const tga::AttnParams &p, int grid, cudaStream_t stream)
{
    constexpr int smem = tga::AttnShape<D>::kDynamicBytes;
    // One bit per device: the kernel's dynamic shared-memory limit is raised.
    static std::atomic<uint64_t> attr_set{0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return TG_ERR_UNSUPPORTED_DEVICE;
    }
    const uint64_t bit = uint64_t(1) << dev;
    if (!(attr_set.load() & bit)) {
        if (cudaFuncSetAttribute(tga::attn_fwd_kernel<D>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 smem) != cudaSuccess) {
            cudaGetLastError();
            return TG_ERR_LAUNCH;
        }
        attr_set.fetch_or(bit);
    }
    tga::attn_fwd_kernel<D><<<grid, tga::kThreads, smem, stream>>>(tq, tk, tv, p);
    if (cudaGetLastError() != cudaSuccess) return TG_ERR_LAUNCH;
    return TG_OK;
}

tg_status_t attention_impl(const void *Q, const void *K, const void *V, void *O, int64_t B,
                           int64_t H, int64_t Sq, int64_t Sk, int64_t D, int causal, float scale,
                           const tg_attention_options_t *opts, cudaStream_t stream)
{
    if (B < 0 || H < 0 || Sq < 0 || Sk < 0 || (D != 64 && D != 128) ||
        (causal != 0 && causal != 1) ||
        !std::isfinite(scale) || (scale != 0.f && std::fabs(scale) < 1e-30f))
        return TG_ERR_INVALID_ARG;
    if (opts && opts->inject != 0 && opts->inject != TG_INJECT_SKIP_FIRST_LOAD)
        return TG_ERR_INVALID_ARG;
    if (opts && (opts->kv_split < TG_ATTN_SPLIT_AUTO || opts->kv_split > TG_ATTN_SPLIT_ALL))
        return TG_ERR_INVALID_ARG;
    const int64_t bh = B * H;
    if (B > 0 && H > (int64_t(1) << 31) / B) return TG_ERR_INVALID_ARG;
    if (bh == 0 || Sq == 0) return TG_OK;
    if (Sq > (int64_t(1) << 31) - tga::kTileQ || Sk > (int64_t(1) << 31) - tga::kTileK)
        return TG_ERR_INVALID_ARG;
    if (!Q || !O || (Sk > 0 && (!K || !V))) return TG_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(O) || (Sk > 0 && (!aligned16(K) || !aligned16(V))))
        return TG_ERR_MISALIGNED;
    const size_t qbytes = static_cast<size_t>(bh * Sq * D) * 2;
    const size_t kvbytes = static_cast<size_t>(bh * Sk * D) * 2;
    if (overlaps(O, qbytes, Q, qbytes) || overlaps(O, qbytes, K, kvbytes) ||
        overlaps(O, qbytes, V, kvbytes))
        return TG_ERR_INVALID_ARG;
    const int64_t pair_rows = static_cast<int64_t>(tga::kTilesPerCta) * tga::kTileQ;
    const int64_t num_qp = (Sq + pair_rows - 1) / pair_rows;
    if (bh * num_qp > 0x7fffffff) return TG_ERR_INVALID_ARG;

    int num_sms = 0;
    unsigned *error_word = nullptr;
    PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    tg_status_t st = tg_internal_device(&num_sms, &error_word, &encode);
    if (st != TG_OK) return st;
    if (Sk == 0) return cudaMemsetAsync(O, 0, qbytes, stream) == cudaSuccess ? TG_OK : TG_ERR_CUDA;

    CUtensorMap tq, tk, tv;
    if (!encode_3d(encode, &tq, Q, D, Sq, bh) || !encode_3d(encode, &tk, K, D, Sk, bh) ||
        !encode_3d(encode, &tv, V, D, Sk, bh))
        return TG_ERR_CUDA;
    tga::AttnParams p;
    p.O = static_cast<__half *>(O);
    p.Sq = Sq;
    p.Sk = Sk;
    p.num_bh = static_cast<int>(bh);
    p.num_qp = static_cast<int>(num_qp);
    p.causal = causal;
    const float sc = scale != 0.f ? scale : 1.0f / std::sqrt(static_cast<float>(D));
    p.scale_log2 = sc * 1.4426950408889634f;
    p.inject = opts ? opts->inject : 0;
    p.wait_limit_ns = (opts && opts->wait_limit_ns) ? opts->wait_limit_ns : kDefaultWaitLimitNs;
    p.error_word = error_word;
    const int64_t units = bh * num_qp;
    const int64_t key_tiles = (Sk + tga::kTileK - 1) / tga::kTileK;
    // The merge flags hold a per-call epoch, which a replayed graph would
    // repeat: no split while the stream is capturing.
    const int mode = opts ? opts->kv_split : TG_ATTN_SPLIT_AUTO;
    const bool capturing = tg_internal_capturing(stream);
    if (capturing && mode == TG_ATTN_SPLIT_ALL) return TG_ERR_INVALID_ARG;
    const int split = capturing ? 0 : split_units(units, num_sms, key_tiles, causal, mode);
    if (units + split > 0x7fffffff) return TG_ERR_INVALID_ARG;
    p.num_full = static_cast<int>(units - split);
    p.split_units = split;
    p.part = nullptr;
    p.flags = nullptr;
    p.epoch = 0;
    if (split > 0) {
        st = split_workspace(split, stream, &p.part, &p.flags, &p.epoch);
        if (st != TG_OK) return st;
    }
    const int grid = static_cast<int>(units + split);
    return D == 64 ? launch_attn<64>(tq, tk, tv, p, grid, stream)
                   : launch_attn<128>(tq, tk, tv, p, grid, stream);
}

}  // namespace

extern "C" {

tg_status_t tg_attention_fwd(const void *Q, const void *K, const void *V, void *O, int64_t batch,
                             int64_t heads, int64_t seq_q, int64_t seq_k, int64_t head_dim,
                             int causal, float scale, void *stream)
{
    return attention_impl(Q, K, V, O, batch, heads, seq_q, seq_k, head_dim, causal, scale, nullptr,
                          static_cast<cudaStream_t>(stream));
}

tg_status_t tg_attention_plan(int64_t batch, int64_t heads, int64_t seq_q, int64_t seq_k,
                              int64_t head_dim, int causal, int kv_split, int num_sms,
                              int64_t *units, int64_t *split, int64_t *grid)
{
    if (!units || !split || !grid || num_sms <= 0 || batch < 0 || heads < 0 || seq_q < 0 ||
        seq_k < 0 || (head_dim != 64 && head_dim != 128) || (causal != 0 && causal != 1) ||
        kv_split < TG_ATTN_SPLIT_AUTO || kv_split > TG_ATTN_SPLIT_ALL)
        return TG_ERR_INVALID_ARG;
    if (batch > 0 && heads > (int64_t(1) << 31) / batch) return TG_ERR_INVALID_ARG;
    if (seq_q > (int64_t(1) << 31) - tga::kTileQ || seq_k > (int64_t(1) << 31) - tga::kTileK)
        return TG_ERR_INVALID_ARG;
    *units = *split = *grid = 0;
    const int64_t bh = batch * heads;
    if (bh == 0 || seq_q == 0 || seq_k == 0) return TG_OK;   // nothing launched
    const int64_t pair_rows = static_cast<int64_t>(tga::kTilesPerCta) * tga::kTileQ;
    const int64_t n_units = bh * ((seq_q + pair_rows - 1) / pair_rows);
    if (n_units > 0x7fffffff) return TG_ERR_INVALID_ARG;
    const int64_t key_tiles = (seq_k + tga::kTileK - 1) / tga::kTileK;
    const int s = split_units(n_units, num_sms, key_tiles, causal, kv_split);
    if (n_units + s > 0x7fffffff) return TG_ERR_INVALID_ARG;
    *units = n_units;
    *split = s;
    *grid = n_units + s;
    return TG_OK;
}

tg_status_t tg_attention_fwd_ex(const void *Q, const void *K, const void *V, void *O,
                                int64_t batch, int64_t heads, int64_t seq_q, int64_t seq_k,
                                int64_t head_dim, int causal, float scale,
                                const tg_attention_options_t *opts, void *stream)
{
    return attention_impl(Q, K, V, O, batch, heads, seq_q, seq_k, head_dim, causal, scale, opts,
                          static_cast<cudaStream_t>(stream));
}

}  // extern "C"
