"""B200-native fused GEMM + ReLU: C = relu(A . op(B)) on sm_100a tensor cores.

The compute path is libgemmrelu.so (hand-written CUDA + inline PTX: TMA,
mbarrier pipeline, tcgen05 MMA into TMEM, fused ReLU/cast epilogue); this
package only marshals arguments to its C ABI (include/gemm_relu.h).
"""
from ._abi import (  # noqa: F401
    EXPORTS,
    GEMM_BF16,
    GEMM_CTA_AUTO,
    GEMM_CTA_PAIR,
    GEMM_CTA_SINGLE,
    GEMM_ERR_CUDA,
    GEMM_ERR_INVALID_ARG,
    GEMM_ERR_MISALIGNED,
    GEMM_ERR_NO_DEVICE,
    GEMM_ERR_TIMEOUT,
    GEMM_ERR_UNSUPPORTED_DTYPE,
    GEMM_F16,
    GEMM_F32,
    GEMM_OK,
    LIB_PATH,
    NOALLOC_SCRATCH_BYTES,
    GemmError,
    GemmOptions,
    gemm_relu,
    gemm_relu_ex,
    gemm_relu_last_cuda_error,
    gemm_relu_last_device_error,
    gemm_relu_plan,
    gemm_relu_plan_unit,
    gemm_relu_release_workspace,
    gemm_relu_selftest_timeout,
    gemm_relu_splitk_noalloc,
    gemm_relu_status_string,
    gemm_relu_version,
    load,
    matmul_relu,
)
