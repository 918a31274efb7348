/*
 * tg_attention.h -- C ABI of the fused attention forward kernel (sm_100a).
 *
 * The operation is the FlashAttention forward of "Designing High-Performance
 * GPU Kernels with TileLang: Tensor-Core GEMM, Fused Softmax, FlashAttention,
 * and Autotuning" (ainovat.com copy, FlashAttention section): query, key and
 * value tiles are processed without writing the score matrix to global
 * memory, with an online softmax (running row maxima, normalisation sums,
 * rescaling) and tensor-core products, causal or not, as PyTorch's scaled
 * dot-product attention defines it:
 *
 *   O[b,h,i,:] = sum_j softmax_j( scale * Q[b,h,i,:] . K[b,h,j,:] ) V[b,h,j,:]
 *
 * over the keys j < seq_k, and with `causal` only j <= i (the lower-triangular
 * mask, aligned at the top-left corner when seq_q != seq_k).  Scores and the
 * softmax are fp32; the probabilities enter the second product as fp16, both
 * products accumulate in fp32, and O is rounded to fp16 (nearest even).
 *
 * Status codes and tg_gemm_check_error / tg_status_string are shared with
 * tg_gemm.h.
 */
#ifndef TG_ATTENTION_H
#define TG_ATTENTION_H

#include <stdint.h>

#include "tg_gemm.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * tg_attention_fwd -- O = attention(Q, K, V) on the current CUDA device.
 *
 *   Q        fp16 [batch, heads, seq_q, head_dim], row-major (contiguous)
 *   K, V     fp16 [batch, heads, seq_k, head_dim], row-major (contiguous)
 *   O        fp16 [batch, heads, seq_q, head_dim], row-major; written
 *   head_dim 64 or 128
 *   causal   0: every key; 1: key j only for query i >= j
 *   scale    factor on the scores (|scale| >= 1e-30); 0 selects 1/sqrt(head_dim)
 *   stream   cudaStream_t (NULL: the legacy default stream)
 *
 * All four are device pointers owned by the caller, 16-byte aligned (else
 * TG_ERR_MISALIGNED); O must not overlap Q, K or V (TG_ERR_INVALID_ARG).
 * The call is asynchronous and keeps no pointer after it returns.
 * batch * heads * seq_q == 0 is a no-op; seq_k == 0 writes O = 0.
 *
 * Work division: one CTA per (batch x head, 256 queries).  Non-causal calls
 * whose last wave of CTAs would occupy at most half of the SMs split each
 * of that wave's units into two CTAs, one per half of the keys; the half
 * that finishes second merges the two partial results (the FlashAttention
 * rescaling by the row maxima).  Such a call uses a library workspace per
 * (device, stream) of about 266 KB per split unit, allocated in stream
 * order on first need (cudaMallocAsync; TG_ERR_OOM if that fails) and kept
 * for the process; calls that share a stream are ordered by it, calls on
 * different streams use different workspaces.  While `stream` is capturing a
 * CUDA graph nothing is split (the merge flags carry a per-call epoch, which
 * every replay would repeat).  Bad sizes, head_dim, causal
 * or a non-finite scale return TG_ERR_INVALID_ARG before anything is
 * launched; a device other than compute capability 10.0 returns
 * TG_ERR_UNSUPPORTED_DEVICE (there is no CPU path).  Every device-side wait
 * is bounded (2 s by default); an expiry is reported by tg_gemm_check_error
 * as TG_ERR_TIMEOUT.
 */
tg_status_t tg_attention_fwd(const void *Q, const void *K, const void *V, void *O, int64_t batch,
                             int64_t heads, int64_t seq_q, int64_t seq_k, int64_t head_dim,
                             int causal, float scale, void *stream);

/* Key-half split of tg_attention_options_t.kv_split. */
enum {
    TG_ATTN_SPLIT_AUTO = 0,   /* split the units of a sparse last wave (non-causal) */
    TG_ATTN_SPLIT_NEVER = 1,  /* one CTA per unit */
    TG_ATTN_SPLIT_ALL = 2     /* split every unit (non-causal, at least 2 key tiles) */
};

/*
 * Options of tg_attention_fwd_ex (NULL: the defaults of tg_attention_fwd).
 *   wait_limit_ns  0: default (2 s); else the limit of every device-side wait
 *   inject         0 normally.  TG_INJECT_SKIP_FIRST_LOAD makes the first CTA
 *                  skip its first key-tile load, so that the MMA issuer's
 *                  bounded wait expires (testing the timeout path only); the
 *                  kernel exits cleanly and tg_gemm_check_error returns
 *                  TG_ERR_TIMEOUT.
 *   kv_split       TG_ATTN_SPLIT_*; other values: TG_ERR_INVALID_ARG.  Causal
 *                  calls and calls with seq_k <= 128 never split, nor calls
 *                  on a capturing stream (TG_ATTN_SPLIT_ALL there returns
 *                  TG_ERR_INVALID_ARG).
 */
typedef struct {
    uint64_t wait_limit_ns;
    int inject;
    int kv_split;
} tg_attention_options_t;

tg_status_t tg_attention_fwd_ex(const void *Q, const void *K, const void *V, void *O,
                                int64_t batch, int64_t heads, int64_t seq_q, int64_t seq_k,
                                int64_t head_dim, int causal, float scale,
                                const tg_attention_options_t *opts, void *stream);

/*
 * tg_attention_plan -- host only: the launch tg_attention_fwd_ex would make
 * for these arguments on a device with num_sms SMs (148 on B200), without
 * touching a device.
 *   units  out: work units, (batch x heads) x ceil(seq_q / 256)
 *   split  out: units split into two key halves (kv_split, causal and
 *          seq_k decide, as for tg_attention_fwd_ex)
 *   grid   out: CTAs launched, units + split
 * All three are 0 when nothing would be launched (an empty call, seq_k == 0).
 * The plan is that of a stream that is not capturing a graph.
 * Returns TG_ERR_INVALID_ARG for a null output, num_sms <= 0, or the sizes,
 * head_dim, causal or kv_split that tg_attention_fwd_ex rejects as such.
 */
tg_status_t tg_attention_plan(int64_t batch, int64_t heads, int64_t seq_q, int64_t seq_k,
                              int64_t head_dim, int causal, int kv_split, int num_sms,
                              int64_t *units, int64_t *split, int64_t *grid);

#ifdef __cplusplus
}
#endif

#endif /* TG_ATTENTION_H */
