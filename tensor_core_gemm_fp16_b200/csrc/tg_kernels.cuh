// tg_kernels.cuh -- sm_100a kernels of the fused fp16 GEMM.
//
//   gemm_persistent_kernel  C = g(A.B + beta) with tcgen05 MMA into TMEM,
//                           TMA-fed swizzled shared-memory ring, one CTA per
//                           SM walking an L2-grouped tile order.
//   pack_pad_kernel         copies a row-major fp16 matrix into a copy whose
//                           row pitch is a multiple of 8 elements (16 bytes),
//                           zero-padded, so TMA can address it.
//   k0_epilogue_kernel      the K == 0 case: C = g(beta).
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

constexpr int kBlockM = 128;   // rows of the MMA tile (one TMEM lane per row)
constexpr int kBlockK = 64;    // K per stage: 64 fp16 = one 128-byte swizzle row
constexpr int kBChunkN = 64;   // B is loaded in 64-column boxes (128 bytes wide)
constexpr int kUmmaK = 16;     // K of one kind::f16 MMA instruction
constexpr int kABytesStage = kBlockM * kBlockK * 2;   // 16 KiB
constexpr int kBChunkBytes = kBChunkN * kBlockK * 2;  // 8 KiB

constexpr int kEpiWarps = 4;                       // warps 0..3 drain TMEM
constexpr int kProducerWarp = 4;                   // TMA producer
constexpr int kMmaWarp = 5;                        // MMA issuer + TMEM owner
constexpr int kThreads = 32 * 6;

// Error word bits (OR-ed into the per-device error word on a wait expiry).
constexpr unsigned kErrProducerWait = 1u;
constexpr unsigned kErrMmaWait = 2u;
constexpr unsigned kErrEpilogueWait = 4u;
constexpr unsigned kErrDrain = 8u;

enum : int { kEpiNone = 0, kEpiBias = 1, kEpiBiasGelu = 2 };

struct GemmParams {
    const __half *bias;     // [N] or nullptr
    __half *C;              // [M, ldc]
    int64_t M, N, K;
    int64_t ldc;
    int num_m_tiles;
    int num_n_tiles;
    int num_k_blocks;
    int num_tiles;
    int group_m;
    int inject;             // 1: CTA 0 skips its first operand load (timeout test)
    uint64_t wait_limit_ns;
    unsigned *error_word;   // device address of the per-device error word
};

template <int BN, int STAGES>
struct SmemLayout {
    static constexpr int kBBytesStage = BN / kBChunkN * kBChunkBytes;
    static constexpr int kStageBytes = kABytesStage + kBBytesStage;
    static constexpr int kRingBytes = STAGES * kStageBytes;
    // barriers: full[STAGES], empty[STAGES], tmem_full[2], tmem_empty[2], drain
    static constexpr int kNumBars = 2 * STAGES + 5;
    static constexpr int kBarOffset = kRingBytes;
    static constexpr int kTmemSlotOffset = kBarOffset + kNumBars * 8;
    static constexpr int kAbortOffset = kTmemSlotOffset + 4;
    static constexpr int kUsedBytes = kAbortOffset + 4;
    static constexpr int kDynamicBytes = kUsedBytes + 1024;   // slack for 1024-B alignment
    static constexpr uint32_t kTmemCols = 2 * BN;             // double-buffered accumulator
};

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

__device__ __forceinline__ float gelu_erf(float v)
{
    // v * Phi(v) with Phi(v) = erfc(-v / sqrt 2) / 2; erfc keeps relative
    // accuracy in the far negative tail where 1 + erf(.) would cancel.
    return 0.5f * v * erfcf(-v * 0.70710678118654752f);
}

template <int EPI>
__device__ __forceinline__ float apply_epilogue(float acc, float beta)
{
    if (EPI == kEpiNone) return acc;
    float v = acc + beta;
    if (EPI == kEpiBiasGelu) v = gelu_erf(v);
    return v;
}

// ---------------------------------------------------------------------------
// Persistent warp-specialised GEMM.
//   warps 0-3  epilogue: TMEM -> registers -> bias/GELU -> fp16 -> global
//   warp 4     TMA producer (one lane)
//   warp 5     TMEM allocator + MMA issuer (one lane)
// VEC: C rows and bias are 16-byte addressable (N % 8 == 0, aligned bases).
template <int BN, int STAGES, int EPI, bool VEC>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_persistent_kernel(const __grid_constant__ CUtensorMap tmA,
                           const __grid_constant__ CUtensorMap tmB, const GemmParams p)
{
    using L = SmemLayout<BN, STAGES>;
    static_assert(BN == 64 || BN == 128 || BN == 256, "BN must be 64, 128 or 256");
    constexpr uint32_t kIdesc = idesc_f16_f32(kBlockM, BN);
    constexpr uint32_t kTxBytes = L::kStageBytes;

    extern __shared__ uint8_t smem_raw[];
    // Round the dynamic shared-memory base up to 1024 B (128-byte swizzle atom).
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kBarOffset);
    uint64_t *full_bar = bars;
    uint64_t *empty_bar = bars + STAGES;
    uint64_t *tmem_full_bar = bars + 2 * STAGES;
    uint64_t *tmem_empty_bar = bars + 2 * STAGES + 2;
    uint64_t *drain_bar = bars + 2 * STAGES + 4;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kTmemSlotOffset);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kAbortOffset);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tmem_full_bar[b], 1);
            mbar_init(&tmem_empty_bar[b], kEpiWarps);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kProducerWarp && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, L::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;

    const uint32_t smem_base = smem_u32(smem);
    const uint64_t limit = p.wait_limit_ns;

    if (warp == kProducerWarp) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            // Per stage: parity of the last load issued into it, or -1.
            int pending_parity[STAGES];
#pragma unroll
            for (int s = 0; s < STAGES; ++s) pending_parity[s] = -1;
            bool skip_next = (p.inject == 1 && blockIdx.x == 0);
            for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
                int mt, nt;
                tile_coords(tile, p.num_m_tiles, p.num_n_tiles, p.group_m, mt, nt);
                bool ok = true;
                for (int kb = 0; kb < p.num_k_blocks; ++kb) {
                    if (!mbar_wait_bounded(&empty_bar[stage], phase ^ 1u, abort_flag, limit,
                                           p.error_word, kErrProducerWait)) {
                        ok = false;
                        break;
                    }
                    if (skip_next) {
                        skip_next = false;   // injected fault: this stage never fills
                    } else {
                        const uint32_t a_dst = smem_base + stage * L::kStageBytes;
                        const uint32_t b_dst = a_dst + kABytesStage;
                        mbar_arrive_expect_tx(&full_bar[stage], kTxBytes);
                        tma_load_2d(a_dst, &tmA, &full_bar[stage], kb * kBlockK, mt * kBlockM);
#pragma unroll
                        for (int j = 0; j < BN / kBChunkN; ++j)
                            tma_load_2d(b_dst + j * kBChunkBytes, &tmB, &full_bar[stage],
                                        nt * BN + j * kBChunkN, kb * kBlockK);
                        pending_parity[stage] = static_cast<int>(phase);
                    }
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
            }
            // Let every load this thread issued land before the CTA can exit.
#pragma unroll
            for (int s = 0; s < STAGES; ++s)
                if (pending_parity[s] >= 0 &&
                    !mbar_wait_drain(&full_bar[s], static_cast<uint32_t>(pending_parity[s]), limit))
                    atomicOr(p.error_word, kErrDrain);
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool issued_any = false;
            for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
                if (!mbar_wait_bounded(&tmem_empty_bar[acc], acc_phase ^ 1u, abort_flag, limit,
                                       p.error_word, kErrMmaWait))
                    break;
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
                bool ok = true;
                for (int kb = 0; kb < p.num_k_blocks; ++kb) {
                    if (!mbar_wait_bounded(&full_bar[stage], phase, abort_flag, limit,
                                           p.error_word, kErrMmaWait)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t a_addr = smem_base + stage * L::kStageBytes;
                    const uint32_t b_addr = a_addr + kABytesStage;
                    // A: K-major, 128-B swizzle; 8-row groups 1024 B apart.
                    const uint64_t a_desc = smem_desc_sw128(a_addr, 16, 1024);
                    // B: MN-major, 128-B swizzle; 64-column chunks kBChunkBytes
                    // apart (leading), 8-k-row groups 1024 B apart (stride).
                    const uint64_t b_desc = smem_desc_sw128(b_addr, kBChunkBytes, 1024);
#pragma unroll
                    for (int kk = 0; kk < kBlockK / kUmmaK; ++kk) {
                        // K step inside the swizzle row: +32 B for A; +16 rows
                        // (2 KiB) for B.  Both are added to the start-address
                        // field (units of 16 B).
                        const uint64_t a_k = a_desc + static_cast<uint64_t>((kk * kUmmaK * 2) >> 4);
                        const uint64_t b_k =
                            b_desc + static_cast<uint64_t>((kk * kUmmaK * 128) >> 4);
                        mma_f16_ss(d_tmem, a_k, b_k, kIdesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    issued_any = true;
                    mma_commit(&empty_bar[stage]);   // stage free once these MMAs finish
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                mma_commit(&tmem_full_bar[acc]);     // accumulator ready for the epilogue
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
            // Wait for every MMA this thread issued before TMEM is released.
            if (issued_any) {
                mma_commit(drain_bar);
                if (!mbar_wait_drain(drain_bar, 0, limit)) atomicOr(p.error_word, kErrDrain);
            }
        }
        __syncwarp();
    } else {
        // Epilogue warps 0..3: warp w owns TMEM lanes [32w, 32w + 32) = tile rows.
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
            int mt, nt;
            tile_coords(tile, p.num_m_tiles, p.num_n_tiles, p.group_m, mt, nt);
            int ok = 0;
            if (lane == 0)
                ok = mbar_wait_bounded(&tmem_full_bar[acc], acc_phase, abort_flag, limit,
                                       p.error_word, kErrEpilogueWait)
                         ? 1
                         : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after_sync();

            const int64_t row = static_cast<int64_t>(mt) * kBlockM + warp * 32 + lane;
            const bool row_ok = row < p.M;
            __half *crow = p.C + row * p.ldc;
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(warp * 32) << 16) +
                                   static_cast<uint32_t>(acc * BN);
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                const int64_t col0 = static_cast<int64_t>(nt) * BN + c * 32;
                if (col0 >= p.N) break;          // warp-uniform: whole chunk past N
                uint32_t r[32];
                tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(c * 32), r);
                tmem_wait_ld();
                const bool full_chunk = col0 + 32 <= p.N;
                float beta[32];
                if (EPI != kEpiNone && p.bias != nullptr) {
                    if (VEC && full_chunk) {
                        const uint4 *bp = reinterpret_cast<const uint4 *>(p.bias + col0);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            uint4 u = __ldg(bp + q);
                            const __half2 *h = reinterpret_cast<const __half2 *>(&u);
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                float2 f = __half22float2(h[e]);
                                beta[q * 8 + 2 * e] = f.x;
                                beta[q * 8 + 2 * e + 1] = f.y;
                            }
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            beta[j] = (col0 + j < p.N) ? __half2float(p.bias[col0 + j]) : 0.f;
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) beta[j] = 0.f;
                }
                if (row_ok) {
                    if (VEC && full_chunk) {
                        uint4 *dst = reinterpret_cast<uint4 *>(crow + col0);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            uint4 u;
                            __half2 *h = reinterpret_cast<__half2 *>(&u);
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int j = q * 8 + 2 * e;
                                const float lo = apply_epilogue<EPI>(__uint_as_float(r[j]), beta[j]);
                                const float hi =
                                    apply_epilogue<EPI>(__uint_as_float(r[j + 1]), beta[j + 1]);
                                h[e] = __floats2half2_rn(lo, hi);
                            }
                            dst[q] = u;
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (col0 + j < p.N)
                                crow[col0 + j] = __float2half_rn(
                                    apply_epilogue<EPI>(__uint_as_float(r[j]), beta[j]));
                    }
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tmem_empty_bar[acc]);
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
    }

    // Teardown: every role has returned (all waits are bounded), so no thread
    // still reads TMEM and no MMA or copy is in flight.
    tc_fence_before_sync();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, L::kTmemCols);
    }
}

// ---------------------------------------------------------------------------
// dst[r, c] = src[r, c] for c < cols, 0 for cols <= c < ld_dst.  Each thread
// writes one 16-byte group of 8 destination elements; ld_dst % 8 == 0.
__global__ void pack_pad_kernel(const __half *__restrict__ src, int64_t rows, int64_t cols,
                                __half *__restrict__ dst, int64_t ld_dst)
{
    const int64_t groups_per_row = ld_dst / 8;
    const int64_t total = rows * groups_per_row;
    for (int64_t g = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; g < total;
         g += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t r = g / groups_per_row;
        const int64_t c0 = (g - r * groups_per_row) * 8;
        const __half *s = src + r * cols;
        uint4 u;
        __half *h = reinterpret_cast<__half *>(&u);
#pragma unroll
        for (int e = 0; e < 8; ++e)
            h[e] = (c0 + e < cols) ? s[c0 + e] : __ushort_as_half(static_cast<unsigned short>(0));
        *reinterpret_cast<uint4 *>(dst + r * ld_dst + c0) = u;
    }
}

// K == 0: the accumulator is zero, so C[i, j] = g(beta[j]).
template <int EPI>
__global__ void k0_epilogue_kernel(const __half *__restrict__ bias, __half *__restrict__ C,
                                   int64_t M, int64_t N)
{
    const int64_t total = M * N;
    for (int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; t < total;
         t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t j = t % N;
        const float beta = (EPI != kEpiNone && bias != nullptr) ? __half2float(bias[j]) : 0.f;
        C[t] = __float2half_rn(apply_epilogue<EPI>(0.f, beta));
    }
}

}  // namespace tg
