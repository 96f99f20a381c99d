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

// Stream-K fix-up for the skinny kernel: for every column tile split between
// CTAs, C[m, n] = relu(sum of its pieces' partials, in slot order), cast.
// Tiles owned whole by one CTA were written by the GEMM kernel and are skipped.
template <typename OutT>
__global__ void __launch_bounds__(256) streamk_reduce_kernel(const float *__restrict__ ws,
                                                             OutT *__restrict__ C, int M, int N,
                                                             int64_t ldc, int tiles, int kblocks,
                                                             int64_t T, int G, int max_seg, int relu)
{
    constexpr int kTileN = 128;
    const int64_t per_tile = static_cast<int64_t>(M) * kTileN;
    const int64_t total = per_tile * tiles;
    for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int tile = static_cast<int>(idx / per_tile);
        const int64_t r = idx - static_cast<int64_t>(tile) * per_tile;
        const int m = static_cast<int>(r / kTileN);
        const int nl = static_cast<int>(r - static_cast<int64_t>(m) * kTileN);
        const int n = tile * kTileN + nl;
        if (n >= N) continue;
        const int first = sk_owner(static_cast<int64_t>(tile) * kblocks, T, G);
        const int last = sk_owner(static_cast<int64_t>(tile + 1) * kblocks - 1, T, G);
        if (last == first) continue;  // written whole by its owner
        const float *src = ws + static_cast<int64_t>(tile) * max_seg * per_tile + r;
        float acc = src[0];
        for (int s = 1; s <= last - first; ++s) acc += src[static_cast<int64_t>(s) * per_tile];
        if (relu) acc = fmaxf(acc, 0.0f);
        C[static_cast<int64_t>(m) * ldc + n] = convert_out<OutT>(acc);
    }
}

// dst[r * dst_pitch + c] = src[r * cols + c] for r < rows, c < cols (16-bit).
// dst is 16-byte aligned with a pitch of a multiple of 8 elements; src rows
// may start on any 2-byte boundary.  One warp copies a row at a time, lane l
// taking 8-element chunks l, l + 32, ...: 16-byte stores, and 4-byte loads
// where the source row is 4-byte aligned (2-byte loads otherwise).
__global__ void __launch_bounds__(256) repitch_kernel(const uint16_t *__restrict__ src,
                                                      int64_t rows, int64_t cols,
                                                      uint16_t *__restrict__ dst,
                                                      int64_t dst_pitch)
{
    const int lane = static_cast<int>(threadIdx.x & 31);
    const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const int64_t chunks = cols / 8;
    for (int64_t r = warp0; r < rows; r += nwarps) {
        const uint16_t *srow = src + r * cols;
        uint16_t *drow = dst + r * dst_pitch;
        if ((reinterpret_cast<uintptr_t>(srow) & 3u) == 0) {
            for (int64_t c = lane; c < chunks; c += 32) {
                const uint32_t *s4 = reinterpret_cast<const uint32_t *>(srow + c * 8);
                *reinterpret_cast<uint4 *>(drow + c * 8) = make_uint4(s4[0], s4[1], s4[2], s4[3]);
            }
        } else {
            for (int64_t c = lane; c < chunks; c += 32) {
                const uint16_t *s2 = srow + c * 8;
                uint32_t w[4];
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    w[i] = static_cast<uint32_t>(s2[2 * i]) | (static_cast<uint32_t>(s2[2 * i + 1]) << 16);
                *reinterpret_cast<uint4 *>(drow + c * 8) = make_uint4(w[0], w[1], w[2], w[3]);
            }
        }
        for (int64_t e = chunks * 8 + lane; e < cols; e += 32) drow[e] = srow[e];
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
