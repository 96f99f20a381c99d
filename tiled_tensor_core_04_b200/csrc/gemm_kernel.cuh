// gemm_kernel.cuh -- the fused GEMM + ReLU kernel for sm_100a.
//
//   C = relu(A . op(B)),  fp16/bf16 operands, fp32 accumulation in TMEM.
//
// This is the hot path of the matmul_relu method (TileLang technical notes,
// section 3.2: stage A and B tiles global -> shared over a multi-stage
// pipelined K loop, multiply on the tensor cores into a fp32 accumulator
// cleared by the first step, apply max(acc, 0), cast and store; section 3.3:
// the same with B stored (N, K) and transposed, a fixed set of persistent
// blocks walking the output tiles).  The B200 design:
//
//  * persistent grid: one CTA per SM (or one 2-CTA cluster per SM pair),
//    each walking work units u = cluster_id, cluster_id + num_clusters, ...
//    A unit is (output tile, K split).  Units are numbered so that tiles come
//    in panels of `panel` tile rows (a threadblock swizzle for L2 reuse:
//    consecutive units share A rows and B columns).
//  * warp 0: TMA producer.  For every 64-wide K block it waits until a ring
//    slot is free, then issues the bulk tensor copies of the A tile
//    (128 rows x 64) and the B tile (256 or 128 columns x 64) into the slot;
//    the copy engine counts the bytes on the slot's "full" mbarrier.
//  * warp 1: MMA issuer (one thread).  Waits on "full", issues four
//    tcgen05.mma (K = 16 each) into the TMEM accumulator, then
//    tcgen05.commit frees the slot ("empty").  After the unit's last K
//    block it commits to the accumulator's "tmem_full" barrier.
//  * warps 2-5: epilogue.  Each warp owns 32 TMEM lanes (= 32 output rows);
//    it reads 32 fp32 columns at a time (tcgen05.ld), applies ReLU, rounds
//    to the output type and stores to global memory, then releases the
//    accumulator ("tmem_empty").  Two accumulators (2 x 256 TMEM columns)
//    let the epilogue of one unit overlap the main loop of the next.
//  * CTA pair (cta_group::2): the two CTAs of a cluster compute one
//    256 x 256 tile; each holds 128 rows of A and half (128 columns) of B,
//    the leader CTA issues the 256-row MMA, and each CTA's TMEM receives its
//    own 128 rows of the accumulator.
//  * split-K: a unit covers K blocks [kb0, kb1); with more than one split
//    the epilogue writes fp32 partial sums (no ReLU) to a workspace slice and
//    a separate pass adds the slices in fixed order, then applies ReLU.
//  * tails: TMA zero-fills rows/columns/K outside the matrices (zeros add
//    nothing), and the epilogue writes only the in-range part of a tile.
//
// Every mbarrier wait is bounded (timeout_ns).  A wait that runs out sets the
// CTA's abort flag and a bit in g_gemm_device_error and every role leaves its
// loop; the kernel then drains what it can (bounded), frees TMEM and returns.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>
#include <type_traits>

#include "ptx.cuh"

namespace gr {

// Sticky device error word (bit per kind of wait that gave up).
__device__ uint32_t g_gemm_device_error = 0;

enum : uint32_t {
    kErrProducer = 1u,
    kErrMmaOperands = 2u,
    kErrMmaAccum = 4u,
    kErrEpilogue = 8u,
    kErrDrain = 16u,
    kErrSelfTest = 32u,
};

struct GemmParams {
    void *C;               // output (or the split-K workspace)
    int64_t ldc;           // elements between rows of C
    int64_t split_stride;  // elements between split-K slices (0 without split)
    int M, N, K;
    int tiles_m, tiles_n, splits, kblocks, panel, num_units;
    int relu;
    int vec_ok;            // 16-byte vector stores are aligned
    uint32_t idesc;        // tcgen05 instruction descriptor
    uint64_t timeout_ns;
    int l2_a, l2_b;        // L2 eviction priority of the A / B loads (0 normal, 1 first, 2 last)
    int c_stream;          // 1: store C with evict-first (streaming) stores
    uint32_t sleep_ns;     // suspend-time hint for the epilogue's accumulator waits
    int c_tma;             // wide kernel: 1 = write C through shared memory + TMA stores
    // stream-K (skinny kernel): sk_iters > 0 spreads tiles_n * kblocks K blocks
    // evenly over the CTAs; tiles split between CTAs leave fp32 partials in
    // sk_ws, slot (tile * sk_max_seg + segment), each M x 128, row pitch 128
    int64_t sk_iters;
    int sk_max_seg;
    float *sk_ws;
};

// ------------------------------------------------------------------ stream-K
// CTA c of G owns K-block iterations [sk_begin(c), sk_begin(c + 1)) of the
// T = tiles * kblocks iterations, tile-major.
__host__ __device__ __forceinline__ int64_t sk_begin(int64_t c, int64_t T, int64_t G)
{
    return c * T / G;
}

// The CTA whose range contains iteration x.
__host__ __device__ __forceinline__ int sk_owner(int64_t x, int64_t T, int64_t G)
{
    int64_t c = (x * G) / T;
    while (c + 1 < G && sk_begin(c + 1, T, G) <= x) ++c;
    while (c > 0 && sk_begin(c, T, G) > x) --c;
    return static_cast<int>(c);
}

constexpr int kThreads = 192;  // 6 warps
constexpr int kBM = 128;       // rows of A per CTA
constexpr int kBN = 256;       // MMA N (tile columns)
constexpr int kBK = 64;        // K per pipeline stage (128 bytes of 16-bit data)
constexpr uint32_t kTmemCols = 512;

// PAIR: 2-CTA (cta_group::2) tile of 256 x 256, else 1-CTA tile of 128 x 256.
// KK: 64-wide K sub-blocks per pipeline stage (stage K = 64 * KK).  Each
// sub-block of A is one 128-row x 128-byte TMA box (16 KB, 128-byte swizzle);
// B sub-blocks hold the CTA's kBNCta columns for the same 64 K.
template <bool PAIR, int KK>
struct TileCfg {
    static constexpr int kBNCta = PAIR ? kBN / 2 : kBN;           // B columns held per CTA
    static constexpr int kStageK = kBK * KK;
    static constexpr int kASub = kBM * kBK * 2;                    // 16 KB
    static constexpr int kBSub = kBNCta * kBK * 2;                 // 16 or 32 KB
    static constexpr int kABytes = KK * kASub;
    static constexpr int kBBytes = KK * kBSub;
    static constexpr int kStageBytes = kABytes + kBBytes;
    // as many stages as fit in 227 KB next to 1 KB of static shared memory
    // and 1 KB of alignment slack (at most 8)
    static constexpr int kStagesFit = (232448 - 2048) / kStageBytes;
    static constexpr int kStages = kStagesFit > 8 ? 8 : kStagesFit;
    static constexpr uint32_t kTxBytes = kStageBytes * (PAIR ? 2 : 1);
    static constexpr int kTileM = PAIR ? 2 * kBM : kBM;
    static constexpr int kSmemBytes = kStages * kStageBytes + 1024;  // + alignment slack
};

struct WorkUnit {
    int m_tile, n_tile, kb0, kb1, split;
};

// Unit -> (tile, split).  Splits of one tile are adjacent; tiles are walked
// panel by panel (`panel` tile rows per panel, all tile columns), column-major
// inside a panel, and every other panel walks its columns backwards so the
// first tiles of a panel reuse the B columns the previous panel read last.
__host__ __device__ __forceinline__ WorkUnit decode_unit(int u, int tiles_m, int tiles_n,
                                                         int splits, int kblocks, int panel)
{
    WorkUnit w;
    w.split = u % splits;
    const int t = u / splits;
    const int per_panel = panel * tiles_n;
    const int pi = t / per_panel;
    const int r = t - pi * per_panel;
    const int left = tiles_m - pi * panel;
    const int rows_here = panel < left ? panel : left;
    w.m_tile = pi * panel + r % rows_here;
    w.n_tile = r / rows_here;
    if (pi & 1) w.n_tile = tiles_n - 1 - w.n_tile;
    w.kb0 = static_cast<int>(static_cast<int64_t>(w.split) * kblocks / splits);
    w.kb1 = static_cast<int>(static_cast<int64_t>(w.split + 1) * kblocks / splits);
    return w;
}

// The i-th K block a CTA processes for its `local`-th unit.  Consecutive
// units of a CTA alternate the direction of the K loop: at a wave boundary
// the next tiles start on the K range whose A rows (same panel) were read
// most recently and are still in L2.  The sum order changes, nothing else.
__device__ __forceinline__ int k_block_at(const WorkUnit &w, int i, int local)
{
    return (local & 1) ? w.kb1 - 1 - i : w.kb0 + i;
}

struct WaitCtx {
    int *abort_flag;  // shared, per CTA
    uint64_t timeout_ns;
    uint32_t sleep_ns;  // suspend-time hint of the warp-wide (epilogue) waits
};

// Bounded wait on an mbarrier phase, executed by all 32 lanes of a warp.
// Returns true (warp-uniformly) once the phase with `parity` completed;
// false if the wait ran out (this warp sets the abort flag and the error
// bit) or another warp of the CTA already aborted.
template <bool CLUSTER_SCOPE>
__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity, const WaitCtx &wc,
                                           uint32_t code)
{
    auto probe = [&]() {
        if (CLUSTER_SCOPE) return mbar_try_wait_cluster(bar, parity);
        return wc.sleep_ns ? mbar_try_wait_sleep(bar, parity, wc.sleep_ns)
                           : mbar_try_wait(bar, parity);
    };
    bool ok = probe();
    if (!ok) {
        const uint64_t t0 = global_timer_ns();
        for (uint32_t n = 1;; ++n) {
            if (probe()) {
                ok = true;
                break;
            }
            if ((n & 15u) == 0u) {
                if (*reinterpret_cast<volatile int *>(wc.abort_flag)) break;
                if (global_timer_ns() - t0 > wc.timeout_ns) {
                    *reinterpret_cast<volatile int *>(wc.abort_flag) = 1;
                    atomicOr(&g_gemm_device_error, code);
                    break;
                }
            }
        }
    }
    return __all_sync(0xffffffffu, ok);
}

// Bounded wait executed by ONE thread (the TMA producer and MMA issuer run on
// a single elected lane, so their waits carry no warp-wide vote).  Same
// return convention as wait_phase.
template <bool CLUSTER_SCOPE>
__device__ __forceinline__ bool wait_phase_thread(uint32_t bar, uint32_t parity,
                                                  const WaitCtx &wc, uint32_t code)
{
    auto probe = [&]() {
        return CLUSTER_SCOPE ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity);
    };
    if (probe()) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t n = 1;; ++n) {
        if (probe()) return true;
        if ((n & 15u) == 0u) {
            if (*reinterpret_cast<volatile int *>(wc.abort_flag)) return false;
            if (global_timer_ns() - t0 > wc.timeout_ns) {
                *reinterpret_cast<volatile int *>(wc.abort_flag) = 1;
                atomicOr(&g_gemm_device_error, code);
                return false;
            }
        }
    }
}

// Single-thread bounded wait used only while tearing down after an abort.
__device__ __forceinline__ bool wait_phase_one(uint32_t bar, uint32_t parity, uint64_t limit_ns)
{
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > limit_ns) return false;
    }
    return true;
}

// ------------------------------------------------------------------ epilogue
template <typename OutT>
__device__ __forceinline__ uint32_t pack_pair(float a, float b)
{
    if constexpr (std::is_same_v<OutT, __half>) {
        __half2 h = __floats2half2_rn(a, b);  // a -> low half (lower address)
        return *reinterpret_cast<uint32_t *>(&h);
    } else {
        __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
        return *reinterpret_cast<uint32_t *>(&h);
    }
}

template <typename OutT>
__device__ __forceinline__ OutT convert_out(float x)
{
    if constexpr (std::is_same_v<OutT, float>)
        return x;
    else if constexpr (std::is_same_v<OutT, __half>)
        return __float2half_rn(x);
    else
        return __float2bfloat16_rn(x);
}

// Store 32 consecutive outputs of one row (ReLU + round), `valid` of them in
// range.  `vec`: the destination is 16-byte aligned.
template <typename OutT>
__device__ __forceinline__ void store_row32(OutT *dst, const uint32_t (&v)[32], int valid,
                                            bool vec, int relu, bool stream)
{
    float f[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const float x = __uint_as_float(v[i]);
        f[i] = relu ? fmaxf(x, 0.0f) : x;
    }
    if (vec && valid >= 32) {
        if constexpr (std::is_same_v<OutT, float>) {
            float4 *d4 = reinterpret_cast<float4 *>(dst);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float4 q = make_float4(f[4 * i], f[4 * i + 1], f[4 * i + 2], f[4 * i + 3]);
                if (stream)
                    __stcs(d4 + i, q);
                else
                    d4[i] = q;
            }
        } else {
            uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint4 q = make_uint4(pack_pair<OutT>(f[8 * i + 0], f[8 * i + 1]),
                                           pack_pair<OutT>(f[8 * i + 2], f[8 * i + 3]),
                                           pack_pair<OutT>(f[8 * i + 4], f[8 * i + 5]),
                                           pack_pair<OutT>(f[8 * i + 6], f[8 * i + 7]));
                if (stream)
                    __stcs(d4 + i, q);
                else
                    d4[i] = q;
            }
        }
    } else {
#pragma unroll
        for (int i = 0; i < 32; ++i)
            if (i < valid) dst[i] = convert_out<OutT>(f[i]);
    }
}

// ------------------------------------------------------------------ kernel
template <bool PAIR, int KK, bool B_MN, typename OutT>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_relu_tc_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB, const GemmParams p)
{
    using Cfg = TileCfg<PAIR, KK>;
    constexpr int CG = PAIR ? 2 : 1;
    constexpr int kStages = Cfg::kStages;

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full_bar[kStages];
    __shared__ __align__(8) uint64_t empty_bar[kStages];
    __shared__ __align__(8) uint64_t tfull_bar[2];
    __shared__ __align__(8) uint64_t tempty_bar[2];
    __shared__ __align__(8) uint64_t drain_bar;
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag;

    const int warp = static_cast<int>(threadIdx.x >> 5);
    const int lane = static_cast<int>(threadIdx.x & 31);
    const uint32_t rank = PAIR ? cluster_cta_rank() : 0u;
    const uint32_t tiles_base = (smem_addr(smem_raw) + 1023u) & ~1023u;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_addr(&full_bar[s]), 1);
            mbar_init(smem_addr(&empty_bar[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_addr(&tfull_bar[b]), 1);
            mbar_init(smem_addr(&tempty_bar[b]), PAIR ? 8 : 4);
        }
        mbar_init(smem_addr(&drain_bar), 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensor_map(&tmA);
        prefetch_tensor_map(&tmB);
    }
    if (warp == 1) {
        tmem_alloc<CG>(smem_addr(&tmem_slot), kTmemCols);
        tmem_relinquish<CG>();
    }
    tc_fence_before_sync();
    if constexpr (PAIR)
        cluster_sync_all();
    else
        __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = tmem_slot;

    const WaitCtx wc{&abort_flag, p.timeout_ns, p.sleep_ns};
    const int cluster_id = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
    const int num_clusters = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
    bool aborted = false;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer (one lane)
        if (lane == 0) {
            const uint64_t pol_a = make_l2_policy(p.l2_a);
            const uint64_t pol_b = make_l2_policy(p.l2_b);
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued_mask = 0;  // stages that received at least one load
            uint32_t last_parity = 0;  // parity of the last phase issued per stage (bit s)
            int local = 0;
            for (int u = cluster_id; u < p.num_units && !aborted; u += num_clusters, ++local) {
                const WorkUnit w = decode_unit(u, p.tiles_m, p.tiles_n, p.splits, p.kblocks, p.panel);
                const int m_row = w.m_tile * Cfg::kTileM + static_cast<int>(rank) * kBM;
                const int n_col = w.n_tile * kBN + static_cast<int>(rank) * Cfg::kBNCta;
                // K direction alternates per unit (see k_block_at)
                for (int i = 0; i < w.kb1 - w.kb0; ++i) {
                    const int kb = k_block_at(w, i, local);
                    // the slot is released by the MMA's tcgen05.commit (local in both CTAs)
                    if (!wait_phase_thread<false>(smem_addr(&empty_bar[stage]), phase ^ 1u, wc,
                                                  kErrProducer)) {
                        aborted = true;
                        break;
                    }
                    const uint32_t fb = smem_addr(&full_bar[stage]);
                    const uint32_t a_dst = tiles_base + static_cast<uint32_t>(stage * Cfg::kStageBytes);
                    const uint32_t b_dst = a_dst + Cfg::kABytes;
                    const int k0 = kb * Cfg::kStageK;
                    if constexpr (PAIR) {
                        const uint32_t fb_leader = map_shared_to_rank(fb, 0);
                        if (rank == 0) mbar_arrive_expect_tx(fb, Cfg::kTxBytes);
#pragma unroll
                        for (int kk = 0; kk < KK; ++kk) {
                            const int kx = k0 + kk * kBK;
                            tma_load_2d_pair_hint(a_dst + kk * Cfg::kASub, &tmA, fb_leader, kx, m_row,
                                                  pol_a);
                            if constexpr (B_MN) {
#pragma unroll
                                for (int c = 0; c < Cfg::kBNCta / 64; ++c)
                                    tma_load_2d_pair_hint(b_dst + kk * Cfg::kBSub + c * 8192, &tmB,
                                                          fb_leader, n_col + c * 64, kx, pol_b);
                            } else {
                                tma_load_2d_pair_hint(b_dst + kk * Cfg::kBSub, &tmB, fb_leader, kx,
                                                      n_col, pol_b);
                            }
                        }
                    } else {
                        mbar_arrive_expect_tx(fb, Cfg::kTxBytes);
#pragma unroll
                        for (int kk = 0; kk < KK; ++kk) {
                            const int kx = k0 + kk * kBK;
                            tma_load_2d_hint(a_dst + kk * Cfg::kASub, &tmA, fb, kx, m_row, pol_a);
                            if constexpr (B_MN) {
#pragma unroll
                                for (int c = 0; c < Cfg::kBNCta / 64; ++c)
                                    tma_load_2d_hint(b_dst + kk * Cfg::kBSub + c * 8192, &tmB, fb,
                                                     n_col + c * 64, kx, pol_b);
                            } else {
                                tma_load_2d_hint(b_dst + kk * Cfg::kBSub, &tmB, fb, kx, n_col, pol_b);
                            }
                        }
                    }
                    issued_mask |= 1u << stage;
                    last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (aborted && (!PAIR || rank == 0)) {
                // let copies still in flight land before the CTA goes away
                for (int s = 0; s < kStages; ++s)
                    if (issued_mask & (1u << s))
                        if (!wait_phase_one(smem_addr(&full_bar[s]), (last_parity >> s) & 1u, 20000000ull))
                            atomicOr(&g_gemm_device_error, kErrDrain);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (one lane of the leader)
        if (rank == 0 && lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int local = 0;
            bool issued_any = false;
            // Descriptors of stage 0, k = 0; a stage / K step only moves the
            // start address (bits 0-13, in 16-byte units).
            const uint64_t a_desc0 = smem_desc_sw128(tiles_base, 16, 1024);
            const uint64_t b_desc0 = B_MN ? smem_desc_sw128(tiles_base + Cfg::kABytes, 8192, 1024)
                                          : smem_desc_sw128(tiles_base + Cfg::kABytes, 16, 1024);
            constexpr uint64_t kAStep = 32 >> 4;                  // 16 K elements of a K-major row
            constexpr uint64_t kBStep = B_MN ? (2048 >> 4) : (32 >> 4);  // 16 K rows / elements
            constexpr uint64_t kStageStep = Cfg::kStageBytes >> 4;
            constexpr uint64_t kASubStep = Cfg::kASub >> 4;
            constexpr uint64_t kBSubStep = Cfg::kBSub >> 4;
            // whether the next slot's operands were seen to have landed (peeked
            // before the current slot's MMAs are issued, so the barrier check
            // does not sit between two MMA groups)
            bool next_ready = mbar_test_wait(smem_addr(&full_bar[0]), 0);
            for (int u = cluster_id; u < p.num_units && !aborted; u += num_clusters, ++local) {
                const WorkUnit w = decode_unit(u, p.tiles_m, p.tiles_n, p.splits, p.kblocks, p.panel);
                const int buf = local & 1;
                const uint32_t tphase = static_cast<uint32_t>(local >> 1) & 1u;
                // the accumulator is released by the epilogue warps of both CTAs
                if (!wait_phase_thread<PAIR>(smem_addr(&tempty_bar[buf]), tphase ^ 1u, wc,
                                             kErrMmaAccum)) {
                    aborted = true;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * kBN);
                for (int i = 0; i < w.kb1 - w.kb0; ++i) {
                    if (!next_ready &&
                        !wait_phase_thread<false>(smem_addr(&full_bar[stage]), phase, wc,
                                                  kErrMmaOperands)) {
                        aborted = true;
                        break;
                    }
                    const int next_stage = stage + 1 == kStages ? 0 : stage + 1;
                    const uint32_t next_phase = next_stage == 0 ? phase ^ 1u : phase;
                    next_ready = mbar_test_wait(smem_addr(&full_bar[next_stage]), next_phase);
                    const uint64_t so = static_cast<uint64_t>(stage) * kStageStep;
#pragma unroll
                    for (int k = 0; k < KK * (kBK / 16); ++k) {
                        const uint64_t sub = static_cast<uint64_t>(k / (kBK / 16));
                        const uint64_t kin = static_cast<uint64_t>(k % (kBK / 16));
                        umma_f16<CG>(d_tmem, a_desc0 + so + sub * kASubStep + kin * kAStep,
                                     b_desc0 + so + sub * kBSubStep + kin * kBStep, p.idesc,
                                     (i > 0 || k > 0) ? 1u : 0u);
                    }
                    if constexpr (PAIR)
                        umma_commit_pair(smem_addr(&empty_bar[stage]), 0x3);
                    else
                        umma_commit(smem_addr(&empty_bar[stage]));
                    issued_any = true;
                    stage = next_stage;
                    phase = next_phase;
                }
                if (aborted) break;
                if constexpr (PAIR)
                    umma_commit_pair(smem_addr(&tfull_bar[buf]), 0x3);
                else
                    umma_commit(smem_addr(&tfull_bar[buf]));
            }
            if (aborted && issued_any) {
                // wait for the MMAs already issued before TMEM is released
                if constexpr (PAIR)
                    umma_commit_pair(smem_addr(&drain_bar), 0x1);
                else
                    umma_commit(smem_addr(&drain_bar));
                if (!wait_phase_one(smem_addr(&drain_bar), 0, 20000000ull))
                    atomicOr(&g_gemm_device_error, kErrDrain);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue (warps 2..5)
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        int local = 0;
        for (int u = cluster_id; u < p.num_units && !aborted; u += num_clusters, ++local) {
            const WorkUnit w = decode_unit(u, p.tiles_m, p.tiles_n, p.splits, p.kblocks, p.panel);
            const int buf = local & 1;
            const uint32_t tphase = static_cast<uint32_t>(local >> 1) & 1u;
            if (!wait_phase<false>(smem_addr(&tfull_bar[buf]), tphase, wc, kErrEpilogue)) {
                aborted = true;
                break;
            }
            tc_fence_after_sync();
            const int row = w.m_tile * Cfg::kTileM + static_cast<int>(rank) * kBM + q * 32 + lane;
            const int col0 = w.n_tile * kBN;
            OutT *out = reinterpret_cast<OutT *>(p.C) + static_cast<int64_t>(w.split) * p.split_stride;
            OutT *rowp = out + static_cast<int64_t>(row) * p.ldc + col0;
            const bool row_ok = row < p.M;
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                   static_cast<uint32_t>(buf * kBN);
#pragma unroll 1
            for (int c = 0; c < kBN; c += 32) {
                if (col0 + c >= p.N) break;  // warp-uniform
                uint32_t v[32];
                tmem_load_32cols(taddr + static_cast<uint32_t>(c), v);
                tmem_load_wait();
                const int valid = min(32, p.N - (col0 + c));
                if (row_ok) store_row32<OutT>(rowp + c, v, valid, p.vec_ok != 0, p.relu, p.c_stream != 0);
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) {
                if constexpr (PAIR)
                    mbar_arrive_cluster(map_shared_to_rank(smem_addr(&tempty_bar[buf]), 0));
                else
                    mbar_arrive_local(smem_addr(&tempty_bar[buf]));
            }
        }
    }

    __syncwarp();
    tc_fence_before_sync();
    if constexpr (PAIR)
        cluster_sync_all();
    else
        __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc<CG>(tmem_base, kTmemCols);
    }
}

}  // namespace gr
