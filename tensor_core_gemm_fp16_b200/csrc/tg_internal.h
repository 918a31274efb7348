// tg_internal.h -- library-internal hooks shared by the GEMM and attention
// translation units (not part of the C ABI, not exported).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "tg_gemm.h"

// The calling thread's current device, checked to be compute capability 10.0
// and initialised once: its SM count, the device address of the library's
// error word (bounded-wait expiries are OR-ed into it; tg_gemm_check_error
// reads and clears it) and the driver's tensor-map encoder.
__attribute__((visibility("hidden"))) tg_status_t tg_internal_device(
    int *num_sms, unsigned **error_word, PFN_cuTensorMapEncodeTiled_v12000 *encode);

// True while `stream` is capturing a CUDA graph.  A graph replays a kernel
// with the parameters it was captured with, so the launches whose cross-CTA
// flags carry a per-call epoch (stream-K GEMM, key-half split attention)
// would meet their own epoch on every replay; callers avoid them then.
static inline bool tg_internal_capturing(cudaStream_t stream)
{
    cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &st) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return st != cudaStreamCaptureStatusNone;
}
