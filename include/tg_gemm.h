/*
 * tg_gemm.h -- C ABI of the B200 (sm_100a) fused fp16 tensor-core GEMM.
 *
 * Operation (all entry points):
 *
 *     C[i][j] = g( sum_k A[i][k] * B[k][j]  +  beta[j] )      (fp32 accumulate)
 *
 *   A is M x K, B is K x N, C is M x N, all fp16 (IEEE binary16), dense and
 *   row-major (leading dimensions K, N and N elements).  Products are formed
 *   from the fp16 inputs and summed in fp32; the epilogue runs on the fp32
 *   accumulator and the result is rounded once to fp16 (nearest, ties to
 *   even) and stored.
 *   Definition: "Designing High-Performance GPU Kernels with TileLang"
 *   (thecryptopost.io), the make_matmul kernel and its 2048^3 benchmark
 *   section: float16 A (M,K), B (K,N), C (M,N) with a "float" accumulator
 *   fragment.
 *
 *   beta[j] = bias[j] (converted to fp32) for every epilogue except
 *   TG_EPILOGUE_NONE (beta = 0).  bias == NULL means a zero bias.  g is the
 *   identity for NONE and BIAS, and for
 *     TG_EPILOGUE_BIAS_GELU       g(v) = v * Phi(v) = 0.5 v (1 + erf(v / sqrt 2)),
 *                                 the erf form of GELU.  Definition: the same
 *                                 tutorial (ainovat.com), fused-epilogue
 *                                 section: bias add and GELU applied to the
 *                                 register-resident accumulator before the
 *                                 single write of the output;
 *     TG_EPILOGUE_BIAS_GELU_TANH  g(v) = 0.5 v (1 + tanh(sqrt(2/pi)(v + 0.044715 v^3))),
 *                                 the tanh approximation (Hendrycks & Gimpel,
 *                                 "Gaussian Error Linear Units", section 2);
 *     TG_EPILOGUE_BIAS_SOFTMAX    not elementwise: each row of z = A.B + beta is
 *                                 replaced by softmax(z_i) = exp(z_i - max z_i) /
 *                                 sum exp(z_i - max z_i) over its N columns.
 *                                 Definition: the same tutorial (ainovat.com),
 *                                 row-wise softmax section (per-row max and sum
 *                                 reductions in registers), here fused as a GEMM
 *                                 epilogue.  Requires N <= 256 (one tile per
 *                                 row), else TG_ERR_INVALID_ARG.
 *
 * Conventions shared by every entry point:
 *   - Pointers are DEVICE pointers on the current CUDA device (except where
 *     an entry point says "host"); the caller owns every buffer.  The library
 *     keeps no pointer after the call returns.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls are asynchronous with respect to the host and never
 *     synchronise the device, except tg_gemm_check_error.
 *   - Arguments are validated on the host before anything is launched; a
 *     non-TG_OK status means nothing was launched (except TG_ERR_LAUNCH /
 *     TG_ERR_CUDA, which report a CUDA runtime failure).  Nothing throws
 *     across this ABI.
 *   - M == 0 or N == 0: nothing to do, TG_OK.  K == 0: C = g(beta).
 *   - Each of M, N, K must be below 2^31 and the number of 128 x 64 output
 *     tiles below 2^31, else TG_ERR_INVALID_ARG.
 *   - A, B, C, bias must be 2-byte aligned (TG_ERR_MISALIGNED otherwise).
 *     Any 2-byte-aligned address and any K, N are accepted: when a row pitch
 *     or base address is not a multiple of 16 bytes the operands are first
 *     repacked into a padded temporary, a stream-ordered allocation on
 *     `stream` from a memory pool private to the library; TG_ERR_OOM if that
 *     allocation fails.  Up to 64 MiB of it is kept for the next call on the
 *     same stream (and grown, stream-ordered, when a call needs more); a
 *     larger temporary, or one made while `stream` is capturing a graph, is
 *     freed on `stream` after the GEMM.  One repacking kernel makes the
 *     copies before the GEMM kernel.
 *   - C must not overlap A, B or bias (TG_ERR_INVALID_ARG).
 *   - The device must be compute capability 10.0 (B200 class, sm_100a);
 *     otherwise TG_ERR_UNSUPPORTED_DEVICE.  There is no CPU fallback.
 *   - Device-side waits are bounded.  If one expires (it should not in a
 *     correct run) the kernel records the fact in a per-device error word,
 *     leaves C partly written and exits cleanly; tg_gemm_check_error reports
 *     it as TG_ERR_TIMEOUT.
 */
#ifndef TG_GEMM_H
#define TG_GEMM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    TG_EPILOGUE_NONE = 0,           /* C = A.B                          */
    TG_EPILOGUE_BIAS = 1,           /* C = A.B + bias                   */
    TG_EPILOGUE_BIAS_GELU = 2,      /* C = GELU_erf(A.B + bias)         */
    TG_EPILOGUE_BIAS_GELU_TANH = 3, /* C = GELU_tanh(A.B + bias)        */
    TG_EPILOGUE_BIAS_SOFTMAX = 4    /* C = row_softmax(A.B + bias), N <= 256 */
} tg_epilogue_t;

typedef enum {
    TG_OK = 0,
    TG_ERR_INVALID_ARG = 1,        /* null pointer, bad size/epilogue, overlap  */
    TG_ERR_MISALIGNED = 2,         /* a pointer is not 2-byte aligned           */
    TG_ERR_UNSUPPORTED_DEVICE = 3, /* current device is not sm_100              */
    TG_ERR_LAUNCH = 4,             /* a kernel launch failed                    */
    TG_ERR_TIMEOUT = 5,            /* a device-side bounded wait expired        */
    TG_ERR_OOM = 6,                /* a temporary could not be allocated        */
    TG_ERR_CUDA = 7,               /* another CUDA runtime error                */
    TG_ERR_SCRATCH_LIMIT = 8       /* tg_gemm_noalloc: the repacking scratch the
                                      problem needs exceeds TG_NOALLOC_SCRATCH_BYTES */
} tg_status_t;

/*
 * tg_gemm -- C = g(A.B + beta) as defined above, on `stream`.
 *
 *   A     device, fp16 [M, K] row-major (leading dimension K), read only
 *   B     device, fp16 [K, N] row-major (leading dimension N), read only
 *   bias  device, fp16 [N], or NULL; read only; ignored for TG_EPILOGUE_NONE
 *   C     device, fp16 [M, N] row-major (leading dimension N), written
 *   epilogue  one of tg_epilogue_t
 *   stream    cudaStream_t or NULL
 *
 * The tile configuration (tile width, pipeline depth, CTA pairing,
 * rasterisation) comes from a per-shape table built by an offline sweep;
 * see tg_gemm_select_config.  Results are deterministic: the same inputs and
 * configuration give bit-identical C.
 *
 * Work split: a problem with at least two waves of output tiles is computed
 * tile by tile.  A smaller one is computed "stream-K": the tiles' K loops are
 * divided evenly over all SMs (or SM pairs); a unit that covers the later
 * part of a tile's K loop writes an fp32 partial tile, and the unit that
 * covers its start adds those partials (always in the same order) before the
 * epilogue.  The partials live in a workspace owned by the library, created
 * once per (device, stream) on first use (a cudaMalloc of about
 * 148 x 128 KiB plus flags), so stream-K calls on one stream are ordered by
 * that stream; a first call inside a stream capture cannot create it.  While
 * `stream` is capturing a CUDA graph, stream-K is never used: its flags carry
 * a per-call epoch, which every replay of the graph would repeat.  Such calls
 * run whole tiles (an explicit TG_SPLIT_STREAM_K returns TG_ERR_INVALID_ARG).
 *
 * Thin N remainder: when N = q * BN + r with 0 < r <= 4 (BN the tile width
 * of the chosen configuration) and the last, nearly empty column of tiles
 * would add a whole wave to a whole-tile launch, the tensor-core kernel
 * covers the first q * BN columns and a second kernel computes the last r
 * columns on the CUDA cores (fp32 sums of the same fp16 products, the same
 * epilogue), launched after it on `stream` and running alongside it; the
 * repacking gathers those r columns of B for it (into the same temporary).
 * Not for the row softmax.
 */
tg_status_t tg_gemm(const void *A, const void *B, const void *bias, void *C,
                    int64_t M, int64_t N, int64_t K, int epilogue, void *stream);

/*
 * Tile configuration descriptor (read-only view of one table entry).
 *   id         index in [0, tg_num_configs())
 *   block_m    output rows per MMA tile (128 per CTA; 256 with a CTA pair)
 *   block_n    output columns per MMA tile (64, 128 or 256)
 *   block_k    K elements per pipeline stage (64 or 128)
 *   stages     depth of the shared-memory operand ring
 *   cta_pair   1 if two CTAs of a cluster share one 2-SM MMA (cta_group::2)
 *   group_m    M-tiles per rasterisation panel (L2 reuse)
 *   epi_warps  warps that drain the accumulator
 *   split      from tg_gemm_select_config: how tg_gemm divides that problem
 *              among the SMs, TG_SPLIT_TILES or TG_SPLIT_STREAM_K; 0 from
 *              tg_config_info
 *   loader     how operand tiles reach shared memory: 0 TMA (operands whose
 *              rows are not 16-byte aligned are first repacked into padded
 *              scratch), 1 plain loads by four loader warps (any row pitch,
 *              no repacking; latency-bound, so chosen only by config_id or a
 *              table row -- the default for unaligned rows is the repack)
 */
typedef struct {
    int id;
    int block_m;
    int block_n;
    int block_k;
    int stages;
    int cta_pair;
    int group_m;
    int epi_warps;
    int split;
    int loader;
} tg_config_t;

/* Number of compiled tile configurations. */
int tg_num_configs(void);

/* Describe configuration `id`.  Host only, no device call.
 * TG_ERR_INVALID_ARG for a bad id or a NULL `out`. */
tg_status_t tg_config_info(int id, tg_config_t *out);

/*
 * The configuration tg_gemm would use for this problem (host only, no device
 * call; `num_sms` is the device's SM count, 148 on B200).  The choice comes
 * from the compiled per-shape table (an offline sweep's winners, with the
 * split each was timed with) and falls back to a cost rule for shapes the
 * table does not list: per configuration, the k-blocks the busiest SM runs
 * when whole tiles are dealt out in waves, against the k-blocks of an even
 * stream-K share plus a fixed cost for the partial-sum exchange; the
 * cheapest (configuration, split) wins.  The softmax epilogue always runs
 * whole tiles under this rule.
 */
tg_status_t tg_gemm_select_config(int64_t M, int64_t N, int64_t K, int epilogue,
                                  int num_sms, tg_config_t *out);

/*
 * tg_gemm_ex -- tg_gemm with explicit options.  `opts` may be NULL (same as
 * tg_gemm).  Used by the offline sweep and the tests.
 *
 *   config_id      -1: table choice; otherwise a configuration id (for
 *                  TG_EPILOGUE_BIAS_SOFTMAX it must have 4 epilogue warps and
 *                  block_n >= N, else TG_ERR_INVALID_ARG)
 *   wait_limit_ns  0: default (2 s); else the limit of every device-side wait
 *   inject         0 normally.  TG_INJECT_SKIP_FIRST_LOAD makes the first CTA
 *                  skip one operand load, so that the consumer's bounded
 *                  wait expires; for testing the timeout path only.  The
 *                  kernel then exits cleanly and tg_gemm_check_error returns
 *                  TG_ERR_TIMEOUT.
 *                  TG_INJECT_SKIP_STREAMK_FLAGS makes stream-K partial
 *                  results never be flagged, so the units that wait for them
 *                  time out the same way.
 *   group_m        0: the configuration's rasterisation panel height; else
 *                  the number of M-tiles per panel (1 .. 64)
 *   split          TG_SPLIT_AUTO: the table's split for a listed shape, else
 *                  the cost rule of tg_gemm_select_config (for a forced
 *                  config_id too); TG_SPLIT_TILES: always whole tiles;
 *                  TG_SPLIT_STREAM_K: always stream-K (see tg_gemm; not
 *                  while the stream is capturing a graph).
 */
#define TG_INJECT_SKIP_FIRST_LOAD 1
#define TG_INJECT_SKIP_STREAMK_FLAGS 2
#define TG_SPLIT_AUTO 0
#define TG_SPLIT_TILES 1
#define TG_SPLIT_STREAM_K 2
typedef struct {
    int config_id;
    uint64_t wait_limit_ns;
    int inject;
    int group_m;
    int split;
} tg_options_t;

tg_status_t tg_gemm_ex(const void *A, const void *B, const void *bias, void *C,
                       int64_t M, int64_t N, int64_t K, int epilogue,
                       const tg_options_t *opts, void *stream);

/*
 * tg_gemm_host -- the same GEMM on HOST buffers (end-to-end path).
 *
 *   A_host, B_host, bias_host (or NULL)  host fp16 inputs, row-major as above
 *                                        (pinned memory gives async copies)
 *   C_host                               host fp16 output [M, N]
 *   workspace                            device buffer of at least
 *                                        tg_gemm_host_workspace_size(M, N, K, has_bias)
 *                                        bytes, 256-byte aligned; owned by the caller
 *
 * Enqueues host-to-device copies of the inputs into the workspace, tg_gemm,
 * and the device-to-host copy of C, overlapped: B and the bias go up first,
 * then A in panels of about 1024 rows (at most 16, the last one split in
 * two halves so that little is left to do after the last upload); each
 * panel's GEMM runs on `stream` as soon as its rows are up, and its rows of C
 * go down while later panels are uploaded and computed.  The copies run on two
 * library streams (created once per device and caller stream) that are
 * joined back into `stream` before the call returns, so the call is ordered
 * on `stream` like any other work.  Returns after enqueueing; synchronise
 * `stream` before reading C_host.  Allocates no memory (the first call on a
 * stream creates the two streams and their events).
 */
size_t tg_gemm_host_workspace_size(int64_t M, int64_t N, int64_t K, int has_bias);

tg_status_t tg_gemm_host(const void *A_host, const void *B_host, const void *bias_host,
                         void *C_host, int64_t M, int64_t N, int64_t K, int epilogue,
                         void *workspace, size_t workspace_bytes, void *stream);

/*
 * tg_gemm_launch_count -- number of kernels tg_gemm would launch for these
 * arguments (host only, no device call; the configuration choice assumes
 * 148 SMs): 0 for an empty problem, 1 for the GEMM kernel (or the K == 0
 * kernel), plus one repacking kernel (it repacks both operands and gathers
 * the thin remainder's columns of B) when the base address or row pitch of A
 * or B is not a multiple of 16 bytes and the chosen configuration loads with
 * TMA (a table row choosing a plain-loader configuration repacks nothing) or
 * when there is a thin remainder, plus one kernel for the last N mod 256 (at
 * most 4) columns when that thin remainder would otherwise cost the
 * tensor-core kernel a whole extra wave of tiles (see tg_gemm).  Returns -1
 * if the arguments would be rejected.
 */
int tg_gemm_launch_count(const void *A, const void *B, const void *bias, const void *C,
                         int64_t M, int64_t N, int64_t K, int epilogue);

/*
 * tg_gemm_check_error -- synchronise `stream`, then read and clear the
 * current device's error word.  TG_ERR_TIMEOUT if a bounded wait expired in
 * any kernel since the last check, TG_ERR_CUDA if the stream reports a CUDA
 * error, else TG_OK.
 */
tg_status_t tg_gemm_check_error(void *stream);

/*
 * tg_gemm_noalloc -- tg_gemm for callers that must not allocate device memory.
 *
 * The paper has no counterpart to this entry point; it exists for users of
 * this library.  tg_gemm repacks operands whose base address or row pitch is
 * not a multiple of 16 bytes into a temporary taken from a stream-ordered
 * memory pool.  Some callers cannot have the library allocate at all: a
 * serving engine that has handed nearly all of HBM to its own allocator (a
 * KV cache, a caching allocator) and must not see a foreign allocation fail
 * or fragment its arena, or a latency-critical loop that must not enter the
 * driver's allocator.  This entry point performs the same computation with
 * the same arguments, results and conventions as tg_gemm, but takes any
 * repacking scratch from a fixed array compiled into the library
 * (file-scope __device__ memory of TG_NOALLOC_SCRATCH_BYTES bytes, which
 * every GPU that loads the library holds until the process exits).  It
 * calls no cudaMalloc, cudaFree, memory-pool or other allocating routine.
 *
 *   - The scratch a call needs is 2*M*K8 bytes (rounded up to 256) when A
 *     must be repacked, plus 2*K*N8 bytes (rounded up to 256) when B must be
 *     repacked, plus 2*r*KA bytes (rounded up to 256) and 256 more for a
 *     thin remainder of r columns (K8, N8 = K, N rounded up to a multiple of
 *     8; KA = K8 when A is repacked, else K); aligned operands without a
 *     remainder need none.  A call needing more than
 *     TG_NOALLOC_SCRATCH_BYTES returns TG_ERR_SCRATCH_LIMIT and launches
 *     nothing.
 *   - The first call on each device performs a one-time set-up on that
 *     device (it looks up the device address of the scratch array, which may
 *     load the library's GPU module); make that first call before any stream
 *     capture begins on the device.
 *   - Every call on a device shares the one scratch array and it keeps the
 *     last call's contents (the repacking kernels rewrite every byte a call
 *     reads, padding included).  Calls whose kernels can overlap on the GPU,
 *     e.g. on two streams without ordering between them, race on it: order
 *     them on one stream or with events.
 */
#define TG_NOALLOC_SCRATCH_BYTES (32u << 20)

tg_status_t tg_gemm_noalloc(const void *A, const void *B, const void *bias, void *C,
                            int64_t M, int64_t N, int64_t K, int epilogue, void *stream);

/* Static, human-readable name of a status code (never NULL). */
const char *tg_status_string(int status);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int tg_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TG_GEMM_H */
