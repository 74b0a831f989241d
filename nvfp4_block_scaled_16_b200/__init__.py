"""NVFP4 linear-layer inference on NVIDIA B200 (sm_100a).

The work happens in ``libnvfp4.so`` (CUDA kernels behind the C ABI of
``include/nvfp4.h``).  This package is a thin ctypes binding with the same names as the
C entry points: it checks tensor placement, allocates outputs the caller did not pass,
and forwards raw device pointers and the current CUDA stream.  PyTorch supplies device
memory and streams only; there is no fallback path.  Importing works without a GPU, but
calling any kernel entry point requires the built library and a compute-capability-10.0
device, and raises otherwise.
"""
from .binding import (  # noqa: F401
    NVFP4Error,
    library_path,
    load_library,
    EXPORTED_SYMBOLS,
    nvfp4_scale_bytes,
    nvfp4_status_string,
    nvfp4_global_scale,
    nvfp4_global_scale_batched,
    nvfp4_global_scale_batched_noalloc,
    nvfp4_quantize,
    nvfp4_global_scale_quantize,
    nvfp4_quantize_masked_batched,
    nvfp4_silu_mul_quantize_batched,
    nvfp4_gemm,
    nvfp4_gemm_bf16a,
    nvfp4_gemm_bf16a_static,
    nvfp4_grouped_gemm_masked,
    nvfp4_gemm_lowrank_bias,
    nvfp4_gemm_silu_mul_quantize,
    nvfp4_grouped_gemm_silu_mul_quantize_masked,
    nvfp4_silu_and_mul,
    nvfp4_quantize_smooth,
    nvfp4_lora_down,
    nvfp4_quantize_smooth_lora_down,
    nvfp4_set_pdl,
    nvfp4_get_pdl,
    nvfp4_selftest_bounded_wait,
    nvfp4_selftest_gemm_stall,
    nvfp4_selftest_grid_barrier,
    nvfp4_selftest_index_check,
    nvfp4_debug_index_checks,
    nvfp4_device_status,
)
