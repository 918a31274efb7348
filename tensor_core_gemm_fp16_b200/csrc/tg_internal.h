// tg_internal.h -- library-internal hooks shared by the GEMM and attention
// translation units (not part of the C ABI, not exported).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include "tg_gemm.h"

// The calling thread's current device, checked to be compute capability 10.0
// and initialised once: its SM count, the device address of the library's
// error word (bounded-wait expiries are OR-ed into it; tg_gemm_check_error
// reads and clears it) and the driver's tensor-map encoder.
__attribute__((visibility("hidden"))) tg_status_t tg_internal_device(
    int *num_sms, unsigned **error_word, PFN_cuTensorMapEncodeTiled_v12000 *encode);
