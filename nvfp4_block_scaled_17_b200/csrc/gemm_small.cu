// gemm_small.cu -- the block-scaled FP4 GEMM for few activation rows (the kernel takes
// M <= 128; nvfp4_gemm routes M <= 32 here, where it measured faster than the general
// kernel's split-K build).
//
// Pages: "minimax_h3_nvfp4_decoder" -- nvfp4_linear_inference (mm_fp4 with alpha =
// 1/(global_sf_x * global_sf_w), bf16 output, then the bias); the operation is the one
// gemm.cu computes: y[m, n] = bf16(fp32(alpha * acc) + bias[n]).
//
// With M of 16 or 128 rows (a decode step, or the Qwen3-VL projections at small batch)
// the output has too few 128-row tiles to fill the tensor cores: an M = 128 MMA would
// spend 7/8 of its work on padding rows, and the weight stream (N x K / 2 bytes, read
// once) is what bounds the call.  So the operands swap: the tensor cores compute
// y^T = W x^T, 128 weight rows filling the MMA's M and the activation rows the MMA's N
// (M rounded up to a multiple of 16).
//
// Design (320 threads, one CTA per SM):
//   * a tile is 256 weight rows (output columns), two M = 128 MMAs per K step sharing
//     the activation operand; K is split over the S CTAs of a thread-block cluster,
//     S chosen so that every tile's cluster is resident at once;
//   * warp 0 loads, per 256-value K stage, the 256 x 128-byte weight box and the
//     M x 128-byte activation box (128-byte swizzle, rows past M zero-filled), the
//     activation's 128x4 scale chunks and the weight's: the 128x4 chunks of both row
//     tiles, or, from prepared weight scales, the stage's 4 KiB block (the same chunks
//     in the same shared-memory order, one bulk copy);
//   * warp 1 copies each K step's three scale chunks into a five-slot tensor-memory
//     ring and issues the two MMAs (kind::mxf4nvf4, block16, M = 128, N = M padded),
//     the whole warp running the loop converged and one elected lane issuing;
//   * warps 2..9 move the two fp32 partial accumulators into shared memory (the idle
//     stage buffers), then, after a cluster barrier, each CTA sums its share of the
//     tile over the S partials in rank order (distributed shared memory) and applies
//     alpha and the bias: deterministic, and the unrounded-output build (F32) stores
//     the same fp32 value the bf16 build rounds.
// With weights_ready (the linear paths) the weight copies of the first stages go out
// before the wait for the previous kernel, so the weight stream overlaps the activation
// quantizer; the activation's copies follow the wait.
// Every wait is bounded; on expiry the kernel records NVFP4_ERR_TIMEOUT, drains its
// copies and MMAs, frees tensor memory and returns.  No load uses cluster multicast.
#include <atomic>

#include "common.cuh"
#include "kernels.h"

namespace nvfp4 {

namespace {

constexpr int XW_ROWS = 256;                 // weight rows per tile (two MMAs)
constexpr int XBKB = 128;                    // packed K bytes per stage (256 values)
constexpr int XSTAGES = 4;
constexpr int XMAX = 128;                    // activation rows at most (the MMA's N)
constexpr int XTHREADS = 320;
constexpr int XS_W = XW_ROWS * XBKB;         // 32 KiB
constexpr int XS_X = XMAX * XBKB;            // 16 KiB
constexpr int XS_SFW = 4096;                 // two row tiles x four steps x 512 B
constexpr int XS_SFX = 2048;                 // four steps x 512 B
constexpr int XS_STAGE = XS_W + XS_X + XS_SFW + XS_SFX;
constexpr int XSMEM = 1024 + XSTAGES * XS_STAGE + 256;
static_assert(XSMEM <= 232448, "dynamic shared memory above the 227 KiB a CTA can have");
static_assert(XMAX * XW_ROWS * 4 <= XSTAGES * XS_STAGE, "partial tile must fit the stages");
constexpr int XTMEM_COLS = 512;
constexpr uint32_t XTMEM_ACC1 = 128;         // second accumulator (weight rows 128..255)
constexpr uint32_t XTMEM_SF = 256;           // scale ring: 5 slots x 12 columns
constexpr int XSF_SLOTS = 5;

struct SmallParams {
    const uint8_t* sfw;        // weight scales: 128x4, or prepared (RSB)
    const uint8_t* sfx;        // activation 128x4 scales
    const float* alpha;
    const uint16_t* bias;      // bf16 [N] or null
    uint16_t* y;               // bf16 [M, N]
    float* y32;                // fp32 [M, N] (the unrounded-output build)
    int M, N;
    int mpad;                  // the MMA's N: M rounded up to 16
    uint32_t idesc;
    int k_tiles;               // ceil(K / 256)
    int kchunks;               // K / 64
    int w_row_tiles;           // ceil(N / 128)
    int splits;
    // 1: the weights (W and its scales) were complete before the previous kernel on the
    // stream started, so the producer loads them before waiting for it
    int w_early;
    int* status;
    uint64_t budget_ns;
};

// One K step, warp-issued under a single election: the weight scales of row tile 0 (and,
// with TWO, of row tile 1, 2048 bytes further) and the activation's into the slot's
// columns 0, 4 and 8, then the M = 128 MMA of each row tile (row tile 1's W rows 16 KiB,
// 1024 descriptor units, after tile 0's).
template <bool TWO>
__device__ __forceinline__ void small_step_w(uint32_t acc0, uint32_t acc1, uint64_t wd,
                                             uint64_t xd, uint32_t idesc, uint32_t sf_t,
                                             uint64_t sfw_d, uint64_t sfx_d,
                                             uint32_t accumulate) {
    if constexpr (TWO) {
        asm volatile(
            "{\n\t"
            ".reg .pred p, e;\n\t"
            ".reg .b32 t4, t8;\n\t"
            ".reg .b64 s2, w1;\n\t"
            "elect.sync _|e, 0xffffffff;\n\t"
            "setp.ne.b32 p, %8, 0;\n\t"
            "add.u32 t4, %5, 4;\n\t"
            "add.u32 t8, %5, 8;\n\t"
            "add.u64 s2, %6, 128;\n\t"
            "add.u64 w1, %2, 1024;\n\t"
            "@e tcgen05.cp.cta_group::1.32x128b.warpx4 [%5], %6;\n\t"
            "@e tcgen05.cp.cta_group::1.32x128b.warpx4 [t4], s2;\n\t"
            "@e tcgen05.cp.cta_group::1.32x128b.warpx4 [t8], %7;\n\t"
            "@e tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %2, %3, %4, "
            "[%5], [t8], p;\n\t"
            "@e tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%1], w1, %3, %4, "
            "[t4], [t8], p;\n\t"
            "}" ::"r"(acc0),
            "r"(acc1), "l"(wd), "l"(xd), "r"(idesc), "r"(sf_t), "l"(sfw_d), "l"(sfx_d),
            "r"(accumulate)
            : "memory");
    } else {
        asm volatile(
            "{\n\t"
            ".reg .pred p, e;\n\t"
            ".reg .b32 t8;\n\t"
            "elect.sync _|e, 0xffffffff;\n\t"
            "setp.ne.b32 p, %8, 0;\n\t"
            "add.u32 t8, %5, 8;\n\t"
            "@e tcgen05.cp.cta_group::1.32x128b.warpx4 [%5], %6;\n\t"
            "@e tcgen05.cp.cta_group::1.32x128b.warpx4 [t8], %7;\n\t"
            "@e tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %2, %3, %4, "
            "[%5], [t8], p;\n\t"
            "}" ::"r"(acc0),
            "r"(acc1), "l"(wd), "l"(xd), "r"(idesc), "r"(sf_t), "l"(sfw_d), "l"(sfx_d),
            "r"(accumulate)
            : "memory");
    }
}

template <bool RSB, bool F32>
__global__ void __launch_bounds__(XTHREADS, 1)
gemm_small_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                  const SmallParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + XSTAGES * XS_STAGE);
    uint64_t* empty = full + XSTAGES;
    uint64_t* acc_full = empty + XSTAGES;
    uint64_t* drain = acc_full + 1;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < XSTAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc(tmem_holder, XTMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    const int splits = p.splits;
    const int rank = (int)cluster_rank();
    const int tile = (int)blockIdx.x / splits;
    const int kt_begin = rank * p.k_tiles / splits;
    const int kt_end = (rank + 1) * p.k_tiles / splits;
    const bool two = 2 * tile + 1 < p.w_row_tiles;   // the second 128-row MMA has rows

    // One stage's weight copies (the W box and its scales), completing on full[stage].
    auto load_w = [&](int stage, int kt, int steps) {
        uint8_t* sW = smem + stage * XS_STAGE;
        uint8_t* sSFW = sW + XS_W + XS_X;
        tma_load_2d_w(sW, &tmW, &full[stage], kt * XBKB, tile * XW_ROWS);
        if constexpr (RSB) {
            bulk_load_w(sSFW, p.sfw + ((size_t)tile * p.k_tiles + kt) * 4096, 4096u, &full[stage]);
        } else {
            for (int t = 0; t < (two ? 2 : 1); ++t)
                bulk_load_w(sSFW + t * 2048,
                            p.sfw + ((size_t)(2 * tile + t) * p.kchunks + 4 * kt) * 512,
                            (uint32_t)steps * 512u, &full[stage]);
        }
    };
    auto stage_bytes = [&](int steps) -> uint32_t {
        const uint32_t sfx_bytes = (uint32_t)steps * 512u;
        const uint32_t sfw_bytes = RSB ? 4096u : sfx_bytes * (two ? 2u : 1u);
        return XS_W + (uint32_t)p.mpad * XBKB + sfw_bytes + sfx_bytes;
    };
    // With w_early the weight copies of the first stages go out before the wait for the
    // previous kernel (which wrote the activation, not the weights); the activation's
    // copies follow the wait.
    // Warp 0 issues its copies converged, one elected lane per copy (the _w forms).
    int n_early = 0;
    if (warp == 0) {
        if (lane == 0) {
            prefetch_tensormap(&tmW);
            prefetch_tensormap(&tmX);
        }
        if (p.w_early) {
            n_early = min(XSTAGES, kt_end - kt_begin);
            for (int i = 0; i < n_early; ++i) {
                const int kt = kt_begin + i;
                const int steps = min(4, p.kchunks - 4 * kt);
                mbar_arrive_expect_tx_w(&full[i], stage_bytes(steps));
                load_w(i, kt, steps);
            }
        }
    }
    griddep_wait();
    griddep_launch_dependents();

    if (warp == 0) {
        {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued = 0, issued_phase = 0;
            for (int kt = kt_begin; kt < kt_end; ++kt) {
                const int steps = min(4, p.kchunks - 4 * kt);
                if (kt - kt_begin >= n_early) {
                    if (!mbar_wait_bounded_warp(&empty[stage], phase ^ 1, abort_flag, p.status,
                                                p.budget_ns))
                        break;
                    mbar_arrive_expect_tx_w(&full[stage], stage_bytes(steps));
                    load_w(stage, kt, steps);
                }
                uint8_t* sX = smem + stage * XS_STAGE + XS_W;
                uint8_t* sSFX = sX + XS_X + XS_SFW;
                const uint32_t sfx_bytes = (uint32_t)steps * 512u;
                tma_load_2d_w(sX, &tmX, &full[stage], kt * XBKB, 0);
                bulk_load_w(sSFX, p.sfx + (size_t)(4 * kt) * 512, sfx_bytes, &full[stage]);
                issued |= 1u << stage;
                issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
                if (++stage == XSTAGES) {
                    stage = 0;
                    phase ^= 1;
                }
            }
            // every fill this warp started must land before the block can exit
            for (int s = 0; s < XSTAGES; ++s)
                if (issued & (1u << s)) {
                    volatile int no_abort = 0;
                    mbar_wait_bounded(&full[s], (issued_phase >> s) & 1, &no_abort, p.status,
                                      p.budget_ns);
                }
        }
    } else if (warp == 1) {
        {   // the whole warp runs the issue loop; one elected lane issues (the _w forms)
            int stage = 0;
            uint32_t phase = 0;
            int slot = 0;
            bool ok = true;
            for (int kt = kt_begin; kt < kt_end; ++kt) {
                if (!mbar_wait_bounded_warp(&full[stage], phase, abort_flag, p.status, p.budget_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int steps = min(4, p.kchunks - 4 * kt);
                // the stage's descriptors; step kk adds 32 bytes to W and x (2 units) and
                // 512 to the scale chunks (32 units).  Both weight scale layouts leave the
                // stage's chunks in the same shared-memory order.
                const uint32_t w0 = smem_u32(smem + stage * XS_STAGE);
                const uint64_t wd = sdesc_kmajor_sw128(w0);
                const uint64_t xd = sdesc_kmajor_sw128(w0 + XS_W);
                const uint64_t sfw_d = sdesc_sf(w0 + XS_W + XS_X);
                const uint64_t sfx_d = sdesc_sf(w0 + XS_W + XS_X + XS_SFW);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    if (kk < steps) {
                        const uint32_t sf_t = tmem + XTMEM_SF + 12u * (uint32_t)slot;
                        const uint32_t acc = (kt > kt_begin || kk > 0) ? 1u : 0u;
                        if (two)
                            small_step_w<true>(tmem, tmem + XTMEM_ACC1, wd + 2 * kk, xd + 2 * kk,
                                               p.idesc, sf_t, sfw_d + 32 * kk, sfx_d + 32 * kk, acc);
                        else
                            small_step_w<false>(tmem, tmem + XTMEM_ACC1, wd + 2 * kk, xd + 2 * kk,
                                                p.idesc, sf_t, sfw_d + 32 * kk, sfx_d + 32 * kk, acc);
                        slot = slot == XSF_SLOTS - 1 ? 0 : slot + 1;
                    }
                }
                tc_commit_w(&empty[stage]);
                if (++stage == XSTAGES) {
                    stage = 0;
                    phase ^= 1;
                }
            }
            if (ok) tc_commit_w(acc_full);
            tc_commit_w(drain);
            volatile int no_abort = 0;
            mbar_wait_bounded(drain, 0, &no_abort, p.status, p.budget_ns);
        }
        __syncwarp();
    } else {
        // the fp32 partial of this CTA's K range into shared memory, [m][256] floats:
        // warp (t, q) holds weight rows t * 128 + 32 q + lane of the tile
        const int t = (warp - 2) >> 2;
        const int quad = warp & 3;
        if ((t == 0 || two) &&
            mbar_wait_bounded(acc_full, 0, abort_flag, p.status, p.budget_ns)) {
            tc_fence_after();
            float* part = reinterpret_cast<float*>(smem);
            const int nl = t * 128 + quad * 32 + lane;
            const uint32_t base = tmem + ((uint32_t)(quad * 32) << 16) + (t ? XTMEM_ACC1 : 0u);
            for (int c = 0; c * 32 < p.M; ++c) {
                uint32_t r[32];
                tmem_ld32(base + (uint32_t)c * 32, r);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int m = c * 32 + j;
                    if (m < p.M) part[m * XW_ROWS + nl] = __uint_as_float(r[j]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    // Every thread of the cluster gets here after bounded work, so the barriers below
    // cannot hang.  Rank r then reduces granules [r G / S, (r + 1) G / S) of the M x 256
    // partials (4 floats each) in rank order and stores them; the second barrier keeps
    // every partial alive until all ranks have read it.
    cluster_sync_all();
    if (warp >= 2 && !*abort_flag) {
        const int G = p.M * (XW_ROWS / 4);
        const int lo = rank * G / splits, hi = (rank + 1) * G / splits;
        const uint32_t part = smem_u32(smem);
        const float alpha = *p.alpha;
        for (int idx = lo + (int)threadIdx.x - 64; idx < hi; idx += XTHREADS - 64) {
            const int m = idx >> 6, g = idx & 63;
            const int n = tile * XW_ROWS + 4 * g;
            if (n >= p.N) continue;
            const uint32_t off = part + (uint32_t)((m * XW_ROWS + 4 * g) * 4);
            float4 acc = ld_dsmem_f4(dsmem_addr(off, 0));
            for (int r = 1; r < splits; ++r) {
                const float4 v = ld_dsmem_f4(dsmem_addr(off, (uint32_t)r));
                acc.x = __fadd_rn(acc.x, v.x);
                acc.y = __fadd_rn(acc.y, v.y);
                acc.z = __fadd_rn(acc.z, v.z);
                acc.w = __fadd_rn(acc.w, v.w);
            }
            float v[4] = {__fmul_rn(alpha, acc.x), __fmul_rn(alpha, acc.y),
                          __fmul_rn(alpha, acc.z), __fmul_rn(alpha, acc.w)};
            if (p.bias) {
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    v[j] = __fadd_rn(v[j], __uint_as_float((uint32_t)p.bias[min(n + j, p.N - 1)] << 16));
            }
            if constexpr (F32) {
                float* yp = p.y32 + (size_t)m * p.N + n;
                for (int j = 0; j < 4 && n + j < p.N; ++j) yp[j] = v[j];
            } else {
                const uint32_t lo2 = bf16x2_rn(v[0], v[1]), hi2 = bf16x2_rn(v[2], v[3]);
                uint16_t* yp = p.y + (size_t)m * p.N + n;
                if ((p.N & 3) == 0) {
                    *reinterpret_cast<uint2*>(yp) = make_uint2(lo2, hi2);
                } else {
                    const uint16_t hv[4] = {(uint16_t)lo2, (uint16_t)(lo2 >> 16), (uint16_t)hi2,
                                            (uint16_t)(hi2 >> 16)};
                    for (int j = 0; j < 4 && n + j < p.N; ++j) yp[j] = hv[j];
                }
            }
        }
    }
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, XTMEM_COLS);
    }
}

cudaLaunchConfig_t small_config(int grid, int splits, cudaStream_t stream,
                                cudaLaunchAttribute* attr) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid, 1, 1);
    cfg.blockDim = dim3(XTHREADS, 1, 1);
    cfg.dynamicSmemBytes = XSMEM;
    cfg.stream = stream;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)splits;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cfg;
}

template <bool RSB, bool F32>
bool small_attr(int device) {
    static std::atomic<int> done[64];
    if (done[device & 63].load(std::memory_order_acquire)) return true;
    if (cudaFuncSetAttribute(gemm_small_kernel<RSB, F32>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, XSMEM) != cudaSuccess)
        return false;
    done[device & 63].store(1, std::memory_order_release);
    return true;
}

// K splits: the largest S <= 8 (a portable cluster) with S <= the K stages and
// tiles * S <= SMs whose clusters are all resident at once (cached per device and S).
template <bool RSB, bool F32>
int small_splits(int tiles, int k_tiles, const DeviceInfo& dev) {
    static std::atomic<int> cap[64][9];   // max active clusters + 1 (0 = not queried yet)
    int smax = min(8, k_tiles);
    if (tiles * smax > dev.sms) smax = max(1, dev.sms / tiles);
    for (int sp = smax; sp >= 2; --sp) {
        int c = cap[dev.device & 63][sp].load(std::memory_order_relaxed) - 1;
        if (c < 0) {
            cudaLaunchAttribute attr[2];
            const cudaLaunchConfig_t cfg = small_config(sp * tiles, sp, nullptr, attr);
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, gemm_small_kernel<RSB, F32>, &cfg) != cudaSuccess) {
                (void)cudaGetLastError();
                n = 0;
            }
            c = n;
            cap[dev.device & 63][sp].store(c + 1, std::memory_order_relaxed);
        }
        if (c >= tiles) return sp;
    }
    return 1;
}

template <bool RSB, bool F32>
nvfp4_status launch_small_impl(const uint8_t* a, const uint8_t* sfa, const uint8_t* b,
                               const uint8_t* sfb, const float* alpha, const void* bias, void* y,
                               int64_t M, int64_t N, int64_t K, cudaStream_t stream,
                               bool weights_ready) {
    DeviceInfo dev;
    nvfp4_status st = device_info(&dev);
    if (st != NVFP4_OK) return st;
    int* status = nullptr;
    if ((st = status_word(&status)) != NVFP4_OK) return st;
    if (!small_attr<RSB, F32>(dev.device)) return NVFP4_ERR_CUDA;

    SmallParams p{};
    p.mpad = (int)((M + 15) / 16 * 16);
    CUtensorMap mapW, mapX;
    if (!make_operand_map(&mapW, b, N, K / 2, XW_ROWS) || !make_operand_map(&mapX, a, M, K / 2, p.mpad))
        return NVFP4_ERR_CUDA;
    p.sfw = sfb;
    p.sfx = sfa;
    p.alpha = alpha;
    p.bias = static_cast<const uint16_t*>(bias);
    p.y = F32 ? nullptr : static_cast<uint16_t*>(y);
    p.y32 = F32 ? static_cast<float*>(y) : nullptr;
    p.M = (int)M;
    p.N = (int)N;
    // E2M1 x E2M1, UE4M3 block scales, both K-major; N = padded M, M = 128
    p.idesc = (1u << 7) | (1u << 10) | ((uint32_t)(p.mpad >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
    p.k_tiles = (int)((K / 2 + XBKB - 1) / XBKB);
    p.kchunks = (int)(K / 64);
    p.w_row_tiles = (int)((N + 127) / 128);
    p.w_early = weights_ready ? 1 : 0;
    p.status = status;
    p.budget_ns = 4000000000ull;   // 4 s
    const int tiles = (int)((N + XW_ROWS - 1) / XW_ROWS);
    p.splits = small_splits<RSB, F32>(tiles, p.k_tiles, dev);
    cudaLaunchAttribute attr[2];
    const cudaLaunchConfig_t cfg = small_config(tiles * p.splits, p.splits, stream, attr);
    if (cudaLaunchKernelEx(&cfg, gemm_small_kernel<RSB, F32>, mapW, mapX, p) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    return NVFP4_OK;
}

}  // namespace

nvfp4_status launch_gemm_small(const uint8_t* a, const uint8_t* sfa, const uint8_t* b,
                               const uint8_t* sfb, bool sfb_prepared, bool f32_out,
                               const float* alpha, const void* bias, void* y, int64_t M,
                               int64_t N, int64_t K, cudaStream_t stream, bool weights_ready) {
    if (M < 1 || M > XMAX) return NVFP4_ERR_INVALID_ARG;
    const bool w = weights_ready;
    if (sfb_prepared)
        return f32_out ? launch_small_impl<true, true>(a, sfa, b, sfb, alpha, bias, y, M, N, K, stream, w)
                       : launch_small_impl<true, false>(a, sfa, b, sfb, alpha, bias, y, M, N, K, stream, w);
    return f32_out ? launch_small_impl<false, true>(a, sfa, b, sfb, alpha, bias, y, M, N, K, stream, w)
                   : launch_small_impl<false, false>(a, sfa, b, sfb, alpha, bias, y, M, N, K, stream, w);
}

}  // namespace nvfp4
