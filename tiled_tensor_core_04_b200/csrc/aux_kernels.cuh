// aux_kernels.cuh -- the small memory-bound kernels around the GEMM:
//   * split-K reduction: C = relu(sum over splits of the fp32 partials),
//     slices added in increasing split order (deterministic);
//   * re-pitch: copy a row-major 16-bit matrix whose row pitch or base is not
//     16-byte aligned into a buffer with a 16-byte-multiple pitch, so the
//     Tensor Memory Accelerator can read it;
//   * the bounded-wait self-test (failure detection without a fault).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

#include "gemm_kernel.cuh"

namespace gr {

// ws: `splits` slices of M x N fp32 partial sums, slice s at ws + s*split_stride,
// row pitch N.  C: M x N, row pitch N.  n_total = M*N.
template <typename OutT>
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const float *__restrict__ ws,
                                                            OutT *__restrict__ C, int64_t n_total,
                                                            int splits, int64_t split_stride,
                                                            int relu, int vec4)
{
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (vec4) {
        const int64_t n4 = n_total / 4;
        for (int64_t i = tid; i < n4; i += stride) {
            float4 acc = reinterpret_cast<const float4 *>(ws)[i];
            for (int s = 1; s < splits; ++s) {
                const float4 v = reinterpret_cast<const float4 *>(ws + s * split_stride)[i];
                acc.x += v.x;
                acc.y += v.y;
                acc.z += v.z;
                acc.w += v.w;
            }
            float r[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                if (relu) r[e] = fmaxf(r[e], 0.0f);
                C[4 * i + e] = convert_out<OutT>(r[e]);
            }
        }
    } else {
        for (int64_t i = tid; i < n_total; i += stride) {
            float acc = ws[i];
            for (int s = 1; s < splits; ++s) acc += ws[s * split_stride + i];
            if (relu) acc = fmaxf(acc, 0.0f);
            C[i] = convert_out<OutT>(acc);
        }
    }
}

// dst[r * dst_pitch + c] = src[r * cols + c] for r < rows, c < cols (16-bit).
__global__ void __launch_bounds__(256) repitch_kernel(const uint16_t *__restrict__ src,
                                                      int64_t rows, int64_t cols,
                                                      uint16_t *__restrict__ dst,
                                                      int64_t dst_pitch)
{
    for (int64_t r = blockIdx.y; r < rows; r += gridDim.y) {
        const uint16_t *s = src + r * cols;
        uint16_t *d = dst + r * dst_pitch;
        for (int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; c < cols;
             c += static_cast<int64_t>(gridDim.x) * blockDim.x)
            d[c] = s[c];
    }
}

// One warp waits, bounded by timeout_ns, on an mbarrier that nothing arrives
// on.  out[0] = 1 if the wait completed (never expected), 0 if it ran out.
__global__ void selftest_timeout_kernel(uint64_t timeout_ns, int *out)
{
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_addr(&bar), 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    const WaitCtx wc{&abort_flag, timeout_ns, 1000};
    const bool ok = wait_phase<false>(smem_addr(&bar), 0, wc, kErrSelfTest);
    if (threadIdx.x == 0) out[0] = ok ? 1 : 0;
}

}  // namespace gr
