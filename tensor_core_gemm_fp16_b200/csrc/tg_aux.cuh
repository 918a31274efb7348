// tg_aux.cuh -- sm_100a kernels around the fused fp16 GEMM of tg_kernels.cuh.
//
//   pack_pad2_kernel        copies up to two row-major fp16 matrices into
//                           copies whose row pitch is a multiple of 8
//                           elements (16 bytes), zero-padded, so TMA can
//                           address them, and gathers a thin remainder's
//                           columns of B for tail_cols_kernel.
//   tail_cols_kernel        a thin remainder of C's columns on the CUDA cores,
//                           alongside the GEMM.
//   k0_epilogue_kernel      the K == 0 case: C = g(beta).
//
// They compute the same operation as the GEMM ("Designing High-Performance
// GPU Kernels with TileLang", thecryptopost.io, make_matmul; the fused
// epilogue of the same tutorial, ainovat.com) for the parts of a call the
// tensor-core kernel does not take.
#pragma once

#include "tg_kernels.cuh"

namespace tg {

// ---------------------------------------------------------------------------
// Repacking of operands whose base or row pitch is not a multiple of 16 bytes:
// dst[r, c] = src[r, c] for c < cols, 0 for cols <= c < ld_dst (ld_dst % 8 == 0,
// dst 16-byte aligned).
struct PackJob {
    const __half *src;
    __half *dst;
    int64_t cols, ld_dst;
    uint32_t groups_per_row;   // ld_dst / 8: 16-byte groups of one dst row
    uint64_t groups;           // rows * groups_per_row (0: nothing to do)
};

// The thin remainder's B operand for tail_cols_kernel: columns [n0, n0 + r) of
// B (K x N, pitch ldb), r <= 16, transposed into r rows of ld_slab fp16
// (ld_slab a multiple of 8, at least K), zero past K.
struct SlabJob {
    const __half *src;   // B
    __half *dst;
    int64_t ldb, n0, K, ld_slab;
    uint64_t groups;     // r * ld_slab / 8 (0: no slab)
    unsigned long long *next_row;   // the tail kernel's row counter, zeroed here
};

// The eight fp16 values src[0 .. 8), of which the first `valid` (1..8) are
// in bounds and the rest read as zero, from any 2-byte aligned address: the
// aligned 16-byte vector holding src[0], the next one only when valid
// elements reach into it, and a byte permutation that shifts the 16 bytes
// into place.  A 16-byte aligned vector that holds a valid element never
// crosses a page, so reading its other bytes is always safe; they are
// discarded.
__device__ __forceinline__ uint4 load8_any16(const __half *src, int valid)
{
    const uintptr_t addr = reinterpret_cast<uintptr_t>(src);
    const uint32_t b = static_cast<uint32_t>(addr & 15u);   // even
    const uint4 *v = reinterpret_cast<const uint4 *>(addr - b);
    const uint4 lo = __ldg(v);
    const uint4 hi = (b != 0 && b + 2u * static_cast<uint32_t>(valid) > 16u)
                         ? __ldg(v + 1)
                         : make_uint4(0u, 0u, 0u, 0u);
    const uint32_t W[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
    // output word j = bytes [b + 4j, b + 4j + 4) of lo:hi
    const uint32_t sel = (b & 2u) ? 0x5432u : 0x3210u;
    uint32_t w[4];
    switch (b >> 2) {
    case 0:
#pragma unroll
        for (int j = 0; j < 4; ++j) w[j] = __byte_perm(W[j], W[j + 1], sel);
        break;
    case 1:
#pragma unroll
        for (int j = 0; j < 4; ++j) w[j] = __byte_perm(W[j + 1], W[j + 2], sel);
        break;
    case 2:
#pragma unroll
        for (int j = 0; j < 4; ++j) w[j] = __byte_perm(W[j + 2], W[j + 3], sel);
        break;
    default:
#pragma unroll
        for (int j = 0; j < 4; ++j) w[j] = __byte_perm(W[j + 3], W[j + 4], sel);
        break;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (2 * i >= valid)
            w[i] = 0u;
        else if (2 * i + 1 >= valid)
            w[i] &= 0xFFFFu;
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// Destination group g of a job: its source elements (nullptr when the group
// lies wholly in the zero padding), how many of its 8 are valid, and where
// it goes.
__device__ __forceinline__ void pack_group(const PackJob &j, uint64_t g, const __half *&src,
                                           int &valid, uint4 *&dst)
{
    uint64_t r;
    uint32_t cg;
    if (g < (1ull << 32)) {
        const uint32_t g32 = static_cast<uint32_t>(g);
        r = g32 / j.groups_per_row;
        cg = g32 - static_cast<uint32_t>(r) * j.groups_per_row;
    } else {
        r = g / j.groups_per_row;
        cg = static_cast<uint32_t>(g - r * j.groups_per_row);
    }
    const int64_t c0 = static_cast<int64_t>(cg) * 8;
    const int64_t left = j.cols - c0;
    valid = left <= 0 ? 0 : (left < 8 ? static_cast<int>(left) : 8);
    src = valid > 0 ? j.src + static_cast<int64_t>(r) * j.cols + c0 : nullptr;
    dst = reinterpret_cast<uint4 *>(j.dst + static_cast<int64_t>(r) * j.ld_dst + c0);
}

// Grid-stride over the 16-byte destination groups of job a, then of job b,
// kPackGroups groups per thread and step with all their loads in flight
// together (the copy is bound by DRAM latency otherwise), then over the
// slab's groups (each gathers 8 rows of one column of B).  Consecutive
// threads take consecutive groups of a row: coalesced reads and writes.  The
// launch lets the dependent GEMM start its prologue as soon as SMs free up
// (it still waits for this grid's completion before reading the copies).
// The copy needs the whole GPU's occupancy to keep enough loads in flight,
// which is why it runs before the GEMM rather than beside it: next to a GEMM
// CTA (nearly all of an SM's shared memory, most of its registers) an SM has
// room for a few warps only.
constexpr int kPackGroups = 4;

__global__ void __launch_bounds__(256) pack_pad2_kernel(const PackJob a, const PackJob b,
                                                        const SlabJob sl)
{
    grid_launch_dependents();
    const uint64_t total = a.groups + b.groups;
    const uint64_t stride = static_cast<uint64_t>(gridDim.x) * blockDim.x;
    const uint64_t t0 = blockIdx.x * static_cast<uint64_t>(blockDim.x) + threadIdx.x;
    for (uint64_t g0 = t0; g0 < total; g0 += kPackGroups * stride) {
        const __half *src[kPackGroups];
        int valid[kPackGroups];
        uint4 *dst[kPackGroups];
#pragma unroll
        for (int i = 0; i < kPackGroups; ++i) {
            const uint64_t g = g0 + i * stride;
            src[i] = nullptr;
            dst[i] = nullptr;
            valid[i] = 0;
            if (g < total)
                pack_group(g < a.groups ? a : b, g < a.groups ? g : g - a.groups, src[i], valid[i],
                           dst[i]);
        }
        uint4 u[kPackGroups];
#pragma unroll
        for (int i = 0; i < kPackGroups; ++i)
            u[i] = src[i] ? load8_any16(src[i], valid[i]) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int i = 0; i < kPackGroups; ++i)
            if (dst[i]) *dst[i] = u[i];
    }
    if (sl.groups > 0 && t0 == 0) *sl.next_row = 0ull;
    const uint64_t per_row = static_cast<uint64_t>(sl.ld_slab / 8);
    for (uint64_t g = t0; g < sl.groups; g += stride) {
        const uint64_t j = g / per_row;
        const int64_t k0 = static_cast<int64_t>(g - j * per_row) * 8;
        const unsigned short *col =
            reinterpret_cast<const unsigned short *>(sl.src) + k0 * sl.ldb + sl.n0 + j;
        uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int e = 0; e < 8; ++e)
            if (k0 + e < sl.K)
                w[e >> 1] |= static_cast<uint32_t>(__ldg(col + e * sl.ldb)) << (16 * (e & 1));
        *reinterpret_cast<uint4 *>(sl.dst + j * sl.ld_slab + k0) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// ---------------------------------------------------------------------------
// The last r columns of C, when a thin remainder past a multiple of the tile
// width would cost the tensor-core kernel a whole extra wave of tiles:
//   C[i][n0 + j] = g( sum_k A[i][k] B[k][n0 + j] + beta[n0 + j] ),  j < r <= RT,
// on the CUDA cores.  A is the operand as the GEMM reads it (row pitch ld, a
// multiple of 8, rows 16-byte aligned and zero past K); B's r columns come as
// the slab (r rows of pitch ld, zero past K).  One warp per row of A: each
// lane takes 8 consecutive k per 16-byte load of A and of each slab row,
// products summed in fp32, then a warp reduction per column.  Warps claim
// rows one at a time from a counter (next_row, zeroed by the repacking
// pre-pass), so that the warps that start first, on the SMs the GEMM leaves
// free, keep working until no row is left.
// It is launched right after the GEMM, which lets it start once every GEMM
// CTA is resident: it runs on the SMs' spare resources while the GEMM runs
// (the repacking pre-pass that made the slab, and A's copy if any, completed
// before the GEMM passed its own wait, and so before the GEMM let this kernel
// start).  A streams through L2 only (ld.global.cg); the slab, which every
// row reads, stays in L1.  It completes only after the GEMM has
// (griddepcontrol.wait at its end).
constexpr int kTailThreads = 64;

template <int EPI, int RT>
__global__ void __launch_bounds__(kTailThreads) tail_cols_kernel(
    const __half *A, const __half *slab, int64_t ld, const __half *bias, __half *C, int64_t ldc,
    int64_t M, int64_t n0, int r, unsigned long long *next_row)
{
    constexpr int kLoads = RT >= 8 ? 1 : 8 / RT;   // groups of A in flight per lane and step
    grid_launch_dependents();
    {
        const int lane = threadIdx.x & 31;
        const int64_t k8 = ld / 8;
        for (;;) {
            unsigned long long claimed = 0ull;
            if (lane == 0) claimed = atomicAdd(next_row, 1ull);
            const int64_t m = static_cast<int64_t>(__shfl_sync(0xffffffffu, claimed, 0));
            if (m >= M) break;
            float acc[RT];
#pragma unroll
            for (int j = 0; j < RT; ++j) acc[j] = 0.f;
            const uint4 *arow = reinterpret_cast<const uint4 *>(A + m * ld);
            for (int64_t g0 = lane; g0 < k8; g0 += 32 * kLoads) {
                uint4 ua[kLoads], us[kLoads][RT];
#pragma unroll
                for (int t = 0; t < kLoads; ++t) {
                    const int64_t g = g0 + 32 * t;
                    ua[t] = g < k8 ? __ldcg(arow + g) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                    for (int j = 0; j < RT; ++j)
                        us[t][j] = (g < k8 && j < r)
                                       ? reinterpret_cast<const uint4 *>(slab + j * ld)[g]
                                       : make_uint4(0u, 0u, 0u, 0u);
                }
#pragma unroll
                for (int t = 0; t < kLoads; ++t) {
                    const uint32_t wa[4] = {ua[t].x, ua[t].y, ua[t].z, ua[t].w};
#pragma unroll
                    for (int j = 0; j < RT; ++j) {
                        const uint32_t ws[4] = {us[t][j].x, us[t][j].y, us[t][j].z, us[t][j].w};
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            acc[j] = fmaf(__half2float(half_of(wa[e >> 1], e & 1)),
                                          __half2float(half_of(ws[e >> 1], e & 1)), acc[j]);
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < RT; ++j)
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], o);
#pragma unroll
            for (int j = 0; j < RT; ++j)
                if (lane == j && j < r) {
                    const float beta =
                        (EPI != kEpiNone && bias != nullptr) ? __half2float(bias[n0 + j]) : 0.f;
                    C[m * ldc + n0 + j] = __float2half_rn(apply_epilogue<EPI>(acc[j], beta));
                }
        }
    }
    grid_dependency_wait();
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
        if constexpr (EPI == kEpiBiasSoftmax) {
            // every row is softmax(bias); N is small (at most 256)
            float m = -INFINITY, sum = 0.f;
            for (int64_t q = 0; q < N; ++q) m = fmaxf(m, bias ? __half2float(bias[q]) : 0.f);
            for (int64_t q = 0; q < N; ++q)
                sum += exp2_approx(((bias ? __half2float(bias[q]) : 0.f) - m) * kLog2e);
            C[t] = __float2half_rn(exp2_approx((beta - m) * kLog2e) * rcp_approx(sum));
        } else {
            C[t] = __float2half_rn(apply_epilogue<EPI>(0.f, beta));
        }
    }
}

}  // namespace tg
