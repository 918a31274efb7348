"""B200-native (sm_100a) fused fp16 tensor-core GEMM: C = g(A.B + bias).

The computation lives in libtg_gemm.so (C ABI, include/tg_gemm.h), built
from csrc/ by ``tensor_core_gemm_fp16_b200.build``.  ``binding`` is its thin
ctypes layer; ``workloads`` holds the seeded synthetic inputs.
"""
from .binding import (  # noqa: F401
    TG_EPILOGUE_BIAS, TG_EPILOGUE_BIAS_GELU, TG_EPILOGUE_NONE, TG_OK, TgError, gemm, gemm_host,
    load, tg_config_info, tg_gemm, tg_gemm_check_error, tg_gemm_ex, tg_gemm_host,
    tg_gemm_host_workspace_size, tg_gemm_select_config, tg_num_configs, tg_status_string,
    tg_version,
)

__version__ = "0.1.0"
