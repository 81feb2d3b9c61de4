// gemm.cu -- block-scaled FP4 x FP4 GEMM on the sm_100a tensor cores.
//
// Pages: "minimax_h3_nvfp4_decoder" -- nvfp4_linear_inference: mm_fp4 over the
// packed activation and weight with their E4M3 block scales (block_size 16, 128x4
// layout), alpha = 1/(global_sf_x * global_sf_w) applied to the product, bf16
// output, then the bias added.  Here alpha and the bias are fused into the
// epilogue: y = bf16(fp32(alpha * acc) + bias).
//
// Design (one CTA per SM, persistent over 128 x 256 output tiles):
//   warp 0      TMA producer: per 256-wide K step, a 128 x 128-byte A box and a
//               256 x 128-byte B box (128-byte swizzle), plus the matching 512-byte
//               chunks of the 128x4 scale layout with plain bulk copies (the layout
//               already is the tensor-memory copy order, so no reshuffle is needed);
//               or, for prepared weight scales (RSB), the B scales of the stage as one
//               4 KiB bulk copy of its prepared block.
//   warp 1      MMA issuer (the whole warp runs the loop converged; one elected lane
//               issues each K step's operations, under a single election): per K=64
//               step, tcgen05.cp of the step's three scale chunks (A and the two B
//               halves, 32x128b.warpx4 each) into a ring of five tensor-memory slots,
//               then tcgen05.mma kind::mxf4nvf4 block16 (M=128, N=256, K=64),
//               accumulating in tensor memory; tcgen05.commit releases the stage and,
//               at the end of a tile, hands the accumulator to the epilogue.  The copy
//               for step g overwrites the slot of step g-5, long finished, so the
//               in-order tensor pipe never waits for an MMA to stop reading the scales
//               it is about to replace.  The issue loop is kept short -- descriptors
//               advanced by adds, one election per step -- because the single issuing
//               warp's instruction stream sets the pace at which MMAs reach the pipe.
//   warps 2..9  epilogue, two warps per 32-lane tensor-memory quadrant (one per
//               128-column half): tcgen05.ld, alpha, bias, bf16, a 64-byte-swizzled
//               shared staging tile (two per warp), TMA store (bounds clipped by the
//               tensor map).
//
// Accumulator double buffering within 512 tensor-memory columns: tile buffers
// occupy columns [0, 256) and [192, 448), the scale-factor ring [448, 508).  The two
// buffers share columns [192, 256); the epilogue drains that shared part of a tile
// first and releases it, so the MMAs of the next tile start while the rest of the
// previous accumulator is still being stored.
//
// Small grids (at most half as many tiles as SMs, e.g. M <= 128 at N = 5120) take the
// split-K build instead: a cluster of S CTAs per tile, CTA r of the cluster running the
// same pipeline over its share of the K tiles; the raw fp32 partial tile goes to that
// CTA's own (now idle) stage buffers, and after a cluster barrier rank r sums its share
// of the rows over all S partials (distributed shared memory, rank order) and applies
// alpha and the bias.  One full wave plus a short second one of long tiles runs the
// full wave persistent and splits the leftover tiles that way right behind it.
//
// Launches use programmatic stream serialization: set-up overlaps the previous
// kernel's tail, and griddepcontrol.wait precedes every global access -- except, when the
// caller says the weights were complete before the previous kernel began (the linear
// paths, whose previous kernel is their own activation quantizer), the first stages' B
// copies, which go out before the wait and overlap the quantizer.
//
// Every wait is bounded (globaltimer); on expiry the kernel records
// NVFP4_ERR_TIMEOUT, drains its own copies and MMAs, frees tensor memory and exits.
// No load uses cluster multicast.
#include "common.cuh"
#include "kernels.h"

#include <atomic>

#include <cudaTypedefs.h>

namespace nvfp4 {

namespace {

constexpr int BM = 128;                 // rows of A per tile (= tensor-memory lanes)
constexpr int BN = 256;                 // rows of B per tile (= accumulator columns)
constexpr int BKB = 128;                // bytes of packed K per stage (256 values)
constexpr int STAGES = 3;
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 64 + 32 * EPI_WARPS;
constexpr int SMEM_A = BM * BKB;        // 16 KiB
constexpr int SMEM_B = BN * BKB;        // 32 KiB
constexpr int SMEM_SFA = 4 * 512;       // four K=64 scale chunks for 128 rows
constexpr int STG_BYTES = 32 * 64;      // one 32 x 32 bf16 staging tile
constexpr int SMEM_BIAS = EPI_WARPS * 256;   // each epilogue warp's 128 bias values of a tile
// Shared memory of one build.  B scales per stage: four 512-byte chunks per 128-row half,
// copied from the 128x4 layout (two bulk copies) or, with RSB (prepared weight scales),
// as the stage's one 4 KiB block, already in this order.
template <bool RSB>
struct GemmSmem {
    static constexpr int SFB = 4 * 1024;
    static constexpr int STG_BUFS = 2;
    static constexpr int STG = EPI_WARPS * STG_BUFS * STG_BYTES;
    static constexpr int BYTES =
        1024 + STAGES * (SMEM_A + SMEM_B + SMEM_SFA + SFB) + STG + SMEM_BIAS + 256;
};
static_assert(GemmSmem<false>::BYTES <= 232448 && GemmSmem<true>::BYTES <= 232448,
              "dynamic shared memory above the 227 KiB a CTA can have");
constexpr int TMEM_COLS = 512;
constexpr uint32_t TMEM_BUF1 = 192;     // second accumulator buffer (overlaps [192, 256))
constexpr uint32_t TMEM_SF = 448;       // ring of scale-factor slots
constexpr int SF_SLOTS = 5;             // 12 columns each: 4 for A, 8 for B (256 rows)

// Instruction descriptor: E2M1 x E2M1 (format 1), both K-major, UE4M3 scales,
// N = 256, M = 128, dense K = 64.
constexpr uint32_t IDESC = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                           ((uint32_t)(BM >> 4) << 24);
// kind::i8: int32 accumulator (D format 2), signed int8 A and B (format 1), K-major.
constexpr uint32_t IDESC_I8 = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                              ((uint32_t)(BM >> 4) << 24);

struct GemmParams {
    const uint8_t* sfa;
    const uint8_t* sfb;
    const float* alpha;
    const uint16_t* bias;      // bf16 [N] or null
    uint16_t* y;               // bf16 [M, N]
    float* y32;                // fp32 [M, N] (the unrounded-output build)
    int M, N;
    int m_blocks, n_blocks;
    int k_tiles;               // ceil(K / 256)
    int kchunks;               // K / 64: scale chunks per 128-row tile
    int sf_row_tiles_b;        // ceil(N / 128)
    int tma_store;             // 1: y through the tensor map (N % 8 == 0)
    int n_fast;                // tile order: 1 = consecutive tiles walk N (B re-read from L2)
    int splits;                // split-K build: CTAs (one cluster) sharing the K range of a tile
    int tile_base, tile_count; // the tiles of this launch: [tile_base, tile_base + tile_count)
    // quantized output (the NVFP4 input of the next linear), when the kernel is built for it
    uint8_t* q_packed;         // [M, N/2]
    uint8_t* q_sf;             // 128x4 scales of an [M, N] operand
    const float* q_gsf;        // static global scale of the next linear's input
    int q_cgroups;             // N / 64
    // int8 operands (the W8A8 linear): fp32 row scales of A and of B
    const float* sx;
    const float* sw;
    // 1: the weight operand (B and its scales) was complete before the previous kernel on
    // the stream started, so the producer loads the first stages' B before waiting for it
    int w_early;
    int* status;
    uint64_t budget_ns;
};

__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) { return bf16x2_rn(lo, hi); }

// NVFP4 encoding of one 16-value block given as 8 bf16 pairs, exactly as the activation
// quantizer encodes it under a static global scale: bmax, E4M3 scale of rn(gsf*bmax)/6,
// codes E2M1(rn(x * rn(gsf / scale))), all codes 0 under a zero scale.  Returns the
// scale byte; c0 / c1 receive the codes of values 0..7 / 8..15.
template <int OFF>
__device__ __forceinline__ uint32_t quantize_block(const uint32_t (&words)[16], float gsf,
                                                   uint32_t& c0, uint32_t& c1) {
    const uint32_t* w = words + OFF;   // compile-time offset: the array stays in registers
    const uint32_t tm = absmax2_bf16(absmax2_bf16(absmax2_bf16(w[0], w[1]), absmax2_bf16(w[2], w[3])),
                                     absmax2_bf16(absmax2_bf16(w[4], w[5]), absmax2_bf16(w[6], w[7])));
    const uint32_t s8 = e4m3_scale_of_scaled_max(__fmul_rn(gsf, absmax_of_pair(tm)));
    const float inv = (s8 == 0u || s8 == 127u) ? 0.0f : __fdiv_rn(gsf, f32_from_e4m3(s8));
    float q[2][8];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t x = w[4 * h + j];
            q[h][2 * j] = __fmul_rn(__uint_as_float(x << 16), inv);
            q[h][2 * j + 1] = __fmul_rn(__uint_as_float(x & 0xffff0000u), inv);
        }
    c0 = s8 ? e2m1x8_from_f32(q[0]) : 0u;
    c1 = s8 ? e2m1x8_from_f32(q[1]) : 0u;
    return s8;
}

// Tile order.  The CTAs of one wave work on consecutive tiles; walking N first keeps
// the few A row blocks of a wave hot while the (smaller) B panel is re-read from L2,
// walking M first does the opposite.
__device__ __forceinline__ void tile_coords(const GemmParams& p, int tile, int& m_blk, int& n_blk) {
    if (p.n_fast) {
        n_blk = tile % p.n_blocks;
        m_blk = tile / p.n_blocks;
    } else {
        m_blk = tile % p.m_blocks;
        n_blk = tile / p.m_blocks;
    }
}

template <bool QOUT, bool I8, bool SPLITK, bool RSB, bool F32 = false>
__global__ void __launch_bounds__(THREADS, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
            const __grid_constant__ CUtensorMap tmY, const GemmParams p) {
    using SM = GemmSmem<RSB>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = sA + STAGES * SMEM_A;
    uint8_t* sStg = sB + STAGES * SMEM_B;
    uint8_t* sSFA = sStg + SM::STG;
    uint8_t* sSFB = sSFA + STAGES * SMEM_SFA;
    uint8_t* sBias = sSFB + STAGES * SM::SFB;
    uint64_t* full = reinterpret_cast<uint64_t*>(sBias + SMEM_BIAS);
    uint64_t* empty = full + STAGES;
    uint64_t* acc_full = empty + STAGES;     // [2]
    uint64_t* acc_free = acc_full + 2;       // [2]
    uint64_t* ovl_free = acc_free + 2;
    uint64_t* drain = ovl_free + 1;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_free[b], EPI_WARPS);
        }
        mbar_init(ovl_free, EPI_WARPS / 2);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc(tmem_holder, TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    const int num_tiles = p.tile_count;
    // This CTA's work: whole tiles, persistent over the grid; or (split-K) the K range
    // [kt_begin, kt_end) of the one tile that its cluster shares.
    const int splits = SPLITK ? p.splits : 1;
    const int rank = SPLITK ? (int)cluster_rank() : 0;
    const int tile_first = SPLITK ? (int)blockIdx.x / splits : (int)blockIdx.x;
    const int tile_step = SPLITK ? num_tiles : (int)gridDim.x;
    const int kt_begin = SPLITK ? rank * p.k_tiles / splits : 0;
    const int kt_end = SPLITK ? (rank + 1) * p.k_tiles / splits : p.k_tiles;

    // One stage's B copies: the B box and its scales (per 128-row half, or with RSB the
    // stage's prepared 4 KiB block), completing on full[stage].
    auto load_b = [&](int stage, int kt, int n_blk, int steps, int sfb_tiles) {
        tma_load_2d(sB + stage * SMEM_B, &tmB, &full[stage], kt * BKB, n_blk * BN);
        if constexpr (!I8) {
            if constexpr (RSB) {
                bulk_load(sSFB + stage * SM::SFB, p.sfb + ((size_t)n_blk * p.k_tiles + kt) * 4096,
                          4096u, &full[stage]);
            } else {
                for (int t = 0; t < sfb_tiles; ++t)
                    bulk_load(sSFB + stage * SM::SFB + t * 2048,
                              p.sfb + ((size_t)(2 * n_blk + t) * p.kchunks + 4 * kt) * 512,
                              (uint32_t)steps * 512u, &full[stage]);
            }
        }
    };
    auto stage_bytes = [&](int steps, int sfb_tiles) -> uint32_t {
        const uint32_t sf_bytes = I8 ? 0u : (uint32_t)steps * 512u;
        const uint32_t sfb_bytes = I8 ? 0u : (RSB ? 4096u : sf_bytes * sfb_tiles);
        return SMEM_A + SMEM_B + sf_bytes + sfb_bytes;
    };
    // With w_early the producer issues the first tile's first stages of B before waiting
    // for the previous kernel (which wrote A, not B); their A copies follow the wait.
    int n_early = 0;
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
        if (p.w_early && tile_first < num_tiles) {
            int m_blk, n_blk;
            tile_coords(p, p.tile_base + tile_first, m_blk, n_blk);
            const int sfb_tiles = (2 * n_blk + 1 < p.sf_row_tiles_b) ? 2 : 1;
            n_early = min(STAGES, kt_end - kt_begin);
            for (int i = 0; i < n_early; ++i) {
                const int kt = kt_begin + i;
                const int steps = min(4, p.kchunks - 4 * kt);
                mbar_arrive_expect_tx(&full[i], stage_bytes(steps, sfb_tiles));
                load_b(i, kt, n_blk, steps, sfb_tiles);
            }
        }
    }
    griddep_wait();
    griddep_launch_dependents();

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued = 0, issued_phase = 0;   // per-stage bit masks
            bool ok = true;
            int fills = 0;   // stages filled so far; the first n_early already hold B
            for (int tile = tile_first; ok && tile < num_tiles; tile += tile_step) {
                int m_blk, n_blk;
                tile_coords(p, p.tile_base + tile, m_blk, n_blk);
                const int sfb_tiles = (2 * n_blk + 1 < p.sf_row_tiles_b) ? 2 : 1;
                for (int kt = kt_begin; kt < kt_end; ++kt, ++fills) {
                    const int steps = min(4, p.kchunks - 4 * kt);
                    const uint32_t sf_bytes = I8 ? 0u : (uint32_t)steps * 512u;
                    if (fills >= n_early) {
                        if (!mbar_wait_bounded(&empty[stage], phase ^ 1, abort_flag, p.status,
                                               p.budget_ns)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&full[stage], stage_bytes(steps, sfb_tiles));
                        load_b(stage, kt, n_blk, steps, sfb_tiles);
                    }
                    tma_load_2d(sA + stage * SMEM_A, &tmA, &full[stage], kt * BKB, m_blk * BM);
                    if constexpr (!I8)
                        bulk_load(sSFA + stage * SMEM_SFA,
                                  p.sfa + ((size_t)m_blk * p.kchunks + 4 * kt) * 512, sf_bytes,
                                  &full[stage]);
                    issued |= 1u << stage;
                    issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            // Every fill this thread started must land before the block can exit.
            for (int s = 0; s < STAGES; ++s)
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
            bool ok = true;
            int it = 0;
            int sf_slot = 0;
            for (int tile = tile_first; ok && tile < num_tiles; tile += tile_step, ++it) {
                const int b = it & 1;
                const uint32_t use = (uint32_t)(it >> 1);
                // buffer b fully drained (tile it-2) and the shared columns drained (tile it-1)
                if (!mbar_wait_bounded_warp(&acc_free[b], (use & 1) ^ 1, abort_flag, p.status,
                                            p.budget_ns) ||
                    !mbar_wait_bounded_warp(ovl_free, (uint32_t)(it & 1) ^ 1, abort_flag, p.status,
                                            p.budget_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t acc = tmem + (b ? TMEM_BUF1 : 0u);
                for (int kt = kt_begin; kt < kt_end; ++kt) {
                    if (!mbar_wait_bounded_warp(&full[stage], phase, abort_flag, p.status,
                                                p.budget_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int steps = min(4, p.kchunks - 4 * kt);
                    // Descriptors of the stage's first K step; step kk adds 32 bytes to the
                    // A and B start addresses and 512 to the scale chunks' (2 and 32 in the
                    // descriptors' address fields).  B's second 128-row half is 2048 bytes
                    // (128 units) after the first.
                    const uint64_t ad = sdesc_kmajor_sw128(smem_u32(sA + stage * SMEM_A));
                    const uint64_t bd = sdesc_kmajor_sw128(smem_u32(sB + stage * SMEM_B));
                    const uint64_t sad = sdesc_sf(smem_u32(sSFA + stage * SMEM_SFA));
                    const uint64_t sbd = sdesc_sf(smem_u32(sSFB + stage * SM::SFB));
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        if (kk < steps) {
                            const uint32_t accumulate = (kt > kt_begin || kk > 0) ? 1u : 0u;
                            if constexpr (I8) {
                                mma_i8_w(acc, ad + 2 * kk, bd + 2 * kk, IDESC_I8, accumulate);
                            } else {
                                mma_step_nvf4_w<128>(acc, ad + 2 * kk, bd + 2 * kk, IDESC,
                                                     tmem + TMEM_SF + 12u * (uint32_t)sf_slot,
                                                     sad + 32 * kk, sbd + 32 * kk, accumulate);
                                sf_slot = sf_slot == SF_SLOTS - 1 ? 0 : sf_slot + 1;
                            }
                        }
                    }
                    tc_commit_w(&empty[stage]);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (!ok) break;
                tc_commit_w(&acc_full[b]);
            }
            // Wait until every tensor-core operation the warp issued has finished.
            tc_commit_w(drain);
            volatile int no_abort = 0;
            mbar_wait_bounded(drain, 0, &no_abort, p.status, p.budget_ns);
        }
        __syncwarp();
    } else {
        // epilogue: quadrant q = warp % 4 (tensor-memory lanes 32q..32q+31), column half h
        const int quad = warp & 3;
        const int half = (warp - 2) >> 2;
        const float alpha = I8 ? 0.0f : *p.alpha;
        const float qgsf = QOUT ? *p.q_gsf : 0.0f;
        uint8_t* stg = sStg + (warp - 2) * SM::STG_BUFS * STG_BYTES;
        uint32_t* sbias = reinterpret_cast<uint32_t*>(sBias + (warp - 2) * 256);
        int stg_sel = 0;
        int it = 0;
        bool ok = true;
        for (int tile = tile_first; ok && tile < num_tiles; tile += tile_step, ++it) {
            int m_blk, n_blk;
            tile_coords(p, p.tile_base + tile, m_blk, n_blk);
            const int b = it & 1;
            const uint32_t use = (uint32_t)(it >> 1);
            // The bias of this warp's 128 columns goes to shared memory before the
            // accumulator wait, so its global-load latency stays off the drain path
            // (columns past N repeat the last bias; they are never stored).
            const int n_half = n_blk * BN + half * 128;
            if (p.bias) {
                const int n = n_half + 4 * lane;
                uint2 v;
                if (n + 4 <= p.N) {
                    v = *reinterpret_cast<const uint2*>(p.bias + n);
                } else {
                    v.x = (uint32_t)p.bias[min(n, p.N - 1)] | ((uint32_t)p.bias[min(n + 1, p.N - 1)] << 16);
                    v.y = (uint32_t)p.bias[min(n + 2, p.N - 1)] | ((uint32_t)p.bias[min(n + 3, p.N - 1)] << 16);
                }
                __syncwarp();   // every lane is done with the previous tile's bias
                reinterpret_cast<uint2*>(sbias)[lane] = v;
                __syncwarp();
            }
            if (!mbar_wait_bounded(&acc_full[b], use & 1, abort_flag, p.status, p.budget_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
            // The shared columns [192, 256) are chunks 6, 7 of buffer 0 (half 1) and chunks
            // 0, 1 of buffer 1 (half 0): the owning half drains them first.
            const bool owns_overlap = (b == 0) ? (half == 1) : (half == 0);
            const uint32_t buf_col = b ? TMEM_BUF1 : 0u;
            const int row0 = m_blk * BM + quad * 32;
            const float sx_row = (I8 && row0 + lane < p.M) ? p.sx[row0 + lane] : 0.0f;
            // bf16(alpha * acc + bias) of one 32-column chunk, as 16 bf16 pairs
            auto make_words = [&](const uint32_t (&r)[32], int n0, uint32_t (&packed)[16]) {
                // the bias as 16 bf16 pairs (shared-memory broadcast), widened pair by pair below
                uint32_t bw[16];
                if (p.bias) {
                    const uint4* bp = reinterpret_cast<const uint4*>(sbias + (n0 - n_half) / 2);
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const uint4 w = bp[q4];
                        bw[4 * q4] = w.x; bw[4 * q4 + 1] = w.y;
                        bw[4 * q4 + 2] = w.z; bw[4 * q4 + 3] = w.w;
                    }
                }
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                    float v0, v1;
                    if constexpr (I8) {
                        // (fp32(acc) * s_x[row]) * s_w[col], s_w read per column pair
                        const float2 sw2 = (n0 + j + 1 < p.N)
                                               ? *reinterpret_cast<const float2*>(p.sw + n0 + j)
                                               : make_float2(p.sw[min(n0 + j, p.N - 1)],
                                                             p.sw[min(n0 + j + 1, p.N - 1)]);
                        v0 = __fmul_rn(__fmul_rn(__int2float_rn((int)r[j]), sx_row), sw2.x);
                        v1 = __fmul_rn(__fmul_rn(__int2float_rn((int)r[j + 1]), sx_row), sw2.y);
                    } else {
                        v0 = __fmul_rn(alpha, __uint_as_float(r[j]));
                        v1 = __fmul_rn(alpha, __uint_as_float(r[j + 1]));
                    }
                    if (p.bias) {
                        v0 = __fadd_rn(v0, bf16lo(bw[j / 2]));
                        v1 = __fadd_rn(v1, bf16hi(bw[j / 2]));
                    }
                    packed[j / 2] = bf16x2_bits(v0, v1);
                }
            };
            // the bf16 chunk, staged and stored
            auto store_words = [&](const uint32_t (&packed)[16], int n0) {
                if (p.tma_store) {
                    uint8_t* sb = stg + (SM::STG_BUFS == 2 ? stg_sel * STG_BYTES : 0);
                    if (lane == 0) {   // this buffer's previous store has read it
                        if constexpr (SM::STG_BUFS == 2) bulk_wait_read<1>();
                        else bulk_wait_read<0>();
                    }
                    __syncwarp();
                    // 64-byte swizzle: 16-byte chunk c of row r sits at c ^ ((r >> 1) & 3)
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        *reinterpret_cast<uint4*>(sb + lane * 64 + ((c ^ ((lane >> 1) & 3)) << 4)) =
                            make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2],
                                       packed[4 * c + 3]);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&tmY, sb, n0, row0);
                        bulk_commit();
                    }
                    stg_sel ^= 1;
                } else {
                    const int row = row0 + lane;
                    if (row < p.M) {
                        uint16_t* yrow = p.y + (size_t)row * p.N;
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (n0 + j < p.N) yrow[n0 + j] = (uint16_t)(packed[j / 2] >> (16 * (j & 1)));
                    }
                }
            };
            // the unrounded-output build: fp32(alpha * acc) + bias in fp32, stored as is
            auto store_f32 = [&](const uint32_t (&r)[32], int n0) {
                const int row = row0 + lane;
                if (n0 >= p.N || row >= p.M) return;
                float* yrow = p.y32 + (size_t)row * p.N;
                const uint32_t* bw = sbias + (n0 - n_half) / 2;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    float v = __fmul_rn(alpha, __uint_as_float(r[j]));
                    if (p.bias) v = __fadd_rn(v, (j & 1) ? bf16hi(bw[j / 2]) : bf16lo(bw[j / 2]));
                    if (n0 + j < p.N) yrow[n0 + j] = v;
                }
            };
            // Two chunks at a time: both tensor-memory loads are in flight together, and
            // the columns are released as soon as they are in registers -- the shared
            // columns first, so the next tile's MMAs start before this tile is stored.
            const uint32_t lane_col = tmem + ((uint32_t)(quad * 32) << 16) + buf_col;
            for (int i = 0; i < 4; i += 2) {
                const int c0 = (b == 0 && half == 1) ? ((i + 2) & 3) + 4 : half * 4 + i;
                const int c1 = (b == 0 && half == 1) ? ((i + 3) & 3) + 4 : half * 4 + i + 1;
                uint32_t r0[32], r1[32];
                tmem_ld32(lane_col + (uint32_t)c0 * 32, r0);
                tmem_ld32(lane_col + (uint32_t)c1 * 32, r1);
                tmem_ld_wait();
                if (i == 0 && owns_overlap) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(ovl_free);
                }
                if (i == 2) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&acc_free[b]);
                }
                if constexpr (SPLITK) {
                    // the raw fp32 partial into this CTA's partial tile (the stage buffers,
                    // idle now): row-major 1 KiB rows, 16-byte granule g of row r at
                    // g ^ (r & 7), so eight lanes of a store phase hit eight bank groups
                    const int row = quad * 32 + lane;
                    uint8_t* prow = smem + row * 1024;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        *reinterpret_cast<uint4*>(prow + (((c0 * 8 + j) ^ (row & 7)) << 4)) =
                            make_uint4(r0[4 * j], r0[4 * j + 1], r0[4 * j + 2], r0[4 * j + 3]);
                        *reinterpret_cast<uint4*>(prow + (((c1 * 8 + j) ^ (row & 7)) << 4)) =
                            make_uint4(r1[4 * j], r1[4 * j + 1], r1[4 * j + 2], r1[4 * j + 3]);
                    }
                    continue;
                }
                const int n00 = n_blk * BN + c0 * 32, n01 = n_blk * BN + c1 * 32;
                if constexpr (F32) {
                    store_f32(r0, n00);
                    store_f32(r1, n01);
                    continue;
                }
                uint32_t w0[16], w1[16];
                if (n00 < p.N) make_words(r0, n00, w0);   // warp-uniform
                if (n01 < p.N) make_words(r1, n01, w1);
                if constexpr (!QOUT) {
                    if (n00 < p.N) store_words(w0, n00);
                    if (n01 < p.N) store_words(w1, n01);
                }
                if constexpr (QOUT) {
                    // chunks c0, c1 are the 64 columns of one 4-block scale word (N % 64 == 0)
                    if (n00 < p.N) {
                        const int row = row0 + lane;
                        uint32_t codes[8];
                        const uint32_t s0 = quantize_block<0>(w0, qgsf, codes[0], codes[1]);
                        const uint32_t s1 = quantize_block<8>(w0, qgsf, codes[2], codes[3]);
                        const uint32_t s2 = quantize_block<0>(w1, qgsf, codes[4], codes[5]);
                        const uint32_t s3 = quantize_block<8>(w1, qgsf, codes[6], codes[7]);
                        const bool live = row < p.M;       // padding rows get zero scales
                        const uint32_t word = live ? (s0 | (s1 << 8) | (s2 << 16) | (s3 << 24)) : 0u;
                        const size_t off = ((size_t)(row >> 7) * p.q_cgroups + (size_t)(n00 >> 6)) * 512 +
                                           (size_t)((row & 31) << 4) + (size_t)(((row >> 5) & 3) << 2);
                        *reinterpret_cast<uint32_t*>(p.q_sf + off) = word;
                        if (live) {
                            uint4* dst = reinterpret_cast<uint4*>(p.q_packed + (size_t)row * (p.N / 2) + n00 / 2);
                            dst[0] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
                            dst[1] = make_uint4(codes[4], codes[5], codes[6], codes[7]);
                        }
                    }
                }
            }
        }
        if (lane == 0) bulk_wait_all();
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if constexpr (SPLITK) {
        // Every thread of the cluster gets here after bounded work (all waits above are
        // bounded), so the two cluster barriers cannot hang.  Rank r then sums rows
        // [r R / S, (r + 1) R / S) of the S partial tiles in rank order over distributed
        // shared memory and stores them; the second barrier keeps every partial alive
        // until all ranks have read it.
        cluster_sync_all();
        if (warp >= 2) {
            int m_blk, n_blk;
            tile_coords(p, p.tile_base + tile_first, m_blk, n_blk);
            const int rows = min(BM, p.M - m_blk * BM);
            const int r_lo = rank * rows / splits, r_hi = (rank + 1) * rows / splits;
            const uint32_t part = smem_u32(smem);
            const float alpha = *p.alpha;
            for (int idx = threadIdx.x - 64; idx < (r_hi - r_lo) * 64; idx += 32 * EPI_WARPS) {
                const int row = r_lo + (idx >> 6), g = idx & 63;
                const int col = n_blk * BN + 4 * g;
                if (col >= p.N) continue;
                const uint32_t off = part + (uint32_t)(row * 1024 + ((g ^ (row & 7)) << 4));
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
                        v[j] = __fadd_rn(v[j], __uint_as_float((uint32_t)p.bias[min(col + j, p.N - 1)] << 16));
                }
                if constexpr (F32) {
                    float* yp32 = p.y32 + (size_t)(m_blk * BM + row) * p.N + col;
                    for (int j = 0; j < 4 && col + j < p.N; ++j) yp32[j] = v[j];
                    continue;
                }
                const uint32_t lo = bf16x2_bits(v[0], v[1]), hi = bf16x2_bits(v[2], v[3]);
                uint16_t* yp = p.y + (size_t)(m_blk * BM + row) * p.N + col;
                if ((p.N & 3) == 0 && col + 4 <= p.N) {
                    *reinterpret_cast<uint2*>(yp) = make_uint2(lo, hi);
                } else {
                    const uint16_t hv[4] = {(uint16_t)lo, (uint16_t)(lo >> 16), (uint16_t)hi,
                                            (uint16_t)(hi >> 16)};
                    for (int j = 0; j < 4 && col + j < p.N; ++j) yp[j] = hv[j];
                }
            }
        }
        cluster_sync_all();
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// bf16 [M, N] output with a 32 x 32 box and 64-byte swizzle (N % 8 == 0).
bool make_output_map(CUtensorMap* map, void* base, int64_t M, int64_t N) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)M};
    cuuint64_t strides[1] = {(cuuint64_t)N * 2};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                     CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace

// 2-D uint8 view [rows, row_bytes] with a [box_rows, 128-byte] box, 128-byte swizzle.
bool make_operand_map(CUtensorMap* map, const void* base, int64_t rows, int64_t row_bytes,
                      int box_rows) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    cuuint32_t box[2] = {(cuuint32_t)BKB, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

namespace {

// Quantized-output request of the fused epilogue (the next linear's NVFP4 input; the
// bf16 product itself is not written).
struct QuantOut {
    uint8_t* packed;
    uint8_t* sf;
    const float* gsf;
};

// Split-K build: clusters of `splits` CTAs, one tile per cluster.
template <bool RSB>
cudaLaunchConfig_t split_k_config(int grid, int splits, cudaStream_t stream,
                                  cudaLaunchAttribute* attr, bool pdl = false) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid, 1, 1);
    cfg.blockDim = dim3(THREADS, 1, 1);
    cfg.dynamicSmemBytes = GemmSmem<RSB>::BYTES;
    cfg.stream = stream;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)splits;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    return cfg;
}

template <bool RSB, bool F32>
bool split_k_attr(int device) {
    static std::atomic<int> done[64];
    if (done[device & 63].load(std::memory_order_acquire)) return true;
    if (cudaFuncSetAttribute(gemm_kernel<false, false, true, RSB, F32>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             GemmSmem<RSB>::BYTES) != cudaSuccess)
        return false;
    done[device & 63].store(1, std::memory_order_release);
    return true;
}

// K splits for a grid with too few tiles to fill the SMs: the largest S <= 8 (a portable
// cluster) with S <= ceil(K / 256) and tiles * S <= SMs whose clusters are all resident
// at once (cudaOccupancyMaxActiveClusters, cached per device and S); 1 = no split.
template <bool RSB, bool F32>
int choose_splits(int tiles, int k_tiles, const DeviceInfo& dev) {
    if (tiles * 2 > dev.sms || k_tiles < 2) return 1;
    if (!split_k_attr<RSB, F32>(dev.device)) return 1;
    static std::atomic<int> cap[64][9];   // max active clusters + 1 (0 = not queried yet)
    const int smax = min(8, min(k_tiles, dev.sms / tiles));
    for (int sp = smax; sp >= 2; --sp) {
        int c = cap[dev.device & 63][sp].load(std::memory_order_relaxed) - 1;
        if (c < 0) {
            cudaLaunchAttribute attr[2];
            const cudaLaunchConfig_t cfg = split_k_config<RSB>(sp * tiles, sp, nullptr, attr);
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, gemm_kernel<false, false, true, RSB, F32>, &cfg) !=
                cudaSuccess) {
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
nvfp4_status launch_split_k(const CUtensorMap& mapA, const CUtensorMap& mapB,
                            const CUtensorMap& mapY, const GemmParams& p, int grid, int splits,
                            cudaStream_t stream) {
    cudaLaunchAttribute attr[2];
    const cudaLaunchConfig_t cfg = split_k_config<RSB>(grid, splits, stream, attr, true);
    if (cudaLaunchKernelEx(&cfg, gemm_kernel<false, false, true, RSB, F32>, mapA, mapB, mapY, p) !=
        cudaSuccess)
        return NVFP4_ERR_CUDA;
    return NVFP4_OK;
}

// One launcher for the builds of the kernel: NVFP4 (sfa = 128x4 scales; sfb = 128x4
// scales, or with RSB the prepared weight scales; alpha), NVFP4 with the quantized
// output, int8 (sfa/sfb unused; sx/sw = fp32 row scales of A and B), and (F32) the
// NVFP4 GEMM with an unrounded fp32 output y.
template <bool QOUT, bool I8, bool RSB = false, bool F32 = false>
nvfp4_status launch_gemm_impl(const uint8_t* a, const uint8_t* sfa, const uint8_t* b,
                              const uint8_t* sfb, const float* alpha, const void* bias, void* y,
                              int64_t M, int64_t N, int64_t K, const QuantOut* q,
                              const float* sx, const float* sw, cudaStream_t stream,
                              bool weights_ready = false) {
    DeviceInfo dev;
    nvfp4_status st = device_info(&dev);
    if (st != NVFP4_OK) return st;
    int* status = nullptr;
    if ((st = status_word(&status)) != NVFP4_OK) return st;

    // few activation rows: the swapped-operand kernel (gemm_small.cu)
    if constexpr (!QOUT && !I8) {
        if (M <= kSmallMaxRows)
            return launch_gemm_small(a, sfa, b, sfb, RSB, F32, alpha, bias, y, M, N, K, stream,
                                     weights_ready);
    }
    const int64_t kbytes = I8 ? K : K / 2;   // bytes of one operand row
    CUtensorMap mapA, mapB, mapY;
    if (!make_operand_map(&mapA, a, M, kbytes, BM) || !make_operand_map(&mapB, b, N, kbytes, BN))
        return NVFP4_ERR_CUDA;
    const bool tma_store = !QOUT && !F32 && (N % 8) == 0;
    if (tma_store) {
        if (!make_output_map(&mapY, y, M, N)) return NVFP4_ERR_CUDA;
    } else {
        mapY = mapA;   // unused
    }

    static std::atomic<int> attr_set[64];
    if (!attr_set[dev.device & 63].load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(gemm_kernel<QOUT, I8, false, RSB, F32>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 GemmSmem<RSB>::BYTES) != cudaSuccess)
            return NVFP4_ERR_CUDA;
        attr_set[dev.device & 63].store(1, std::memory_order_release);
    }

    GemmParams p{};
    p.sfa = sfa;
    p.sfb = sfb;
    p.alpha = alpha;
    p.bias = static_cast<const uint16_t*>(bias);
    p.y = F32 ? nullptr : static_cast<uint16_t*>(y);
    p.y32 = F32 ? static_cast<float*>(y) : nullptr;
    p.M = (int)M;
    p.N = (int)N;
    p.m_blocks = (int)((M + BM - 1) / BM);
    p.n_blocks = (int)((N + BN - 1) / BN);
    p.k_tiles = (int)((kbytes + BKB - 1) / BKB);
    p.kchunks = (int)(kbytes / 32);          // 32-byte MMA K steps
    p.sx = sx;
    p.sw = sw;
    p.sf_row_tiles_b = (int)((N + 127) / 128);
    p.tma_store = tma_store ? 1 : 0;
    p.n_fast = (N <= M) ? 1 : 0;
    p.splits = 1;
    p.tile_base = 0;
    p.tile_count = p.m_blocks * p.n_blocks;
    if (QOUT) {
        p.q_packed = q->packed;
        p.q_sf = q->sf;
        p.q_gsf = q->gsf;
        p.q_cgroups = (int)(N / 64);
    }
    p.w_early = weights_ready ? 1 : 0;
    p.status = status;
    p.budget_ns = 4000000000ull;   // 4 s

    const int tiles = p.m_blocks * p.n_blocks;
    if constexpr (!QOUT && !I8) {

        const int splits = choose_splits<RSB, F32>(tiles, p.k_tiles, dev);
        if (splits > 1) {
            p.splits = splits;
            return launch_split_k<RSB, F32>(mapA, mapB, mapY, p, tiles * splits, splits, stream);
        }
        // One full wave plus a short second one (at most SMs / 2 tiles) of long tiles
        // (K >= 4096): the full wave runs persistent, the leftover tiles split K over
        // clusters right behind it (1024 x 5120 x 5120: 148 + 12 tiles, 37.1 -> 34.1 us
        // on B200).  A split-K launch costs about 15 us of fixed time, so it loses where
        // it replaces only the last of many waves or a short-K wave.
        const int tail = tiles % dev.sms;
        if (tiles > dev.sms && tiles < 2 * dev.sms && tail > 0 && p.k_tiles >= 16) {
            const int ts = choose_splits<RSB, F32>(tail, p.k_tiles, dev);
            if (ts > 1) {
                GemmParams full = p;
                full.tile_count = tiles - tail;
                if (launch_pdl(gemm_kernel<false, false, false, RSB, F32>, (unsigned)dev.sms, THREADS,
                               GemmSmem<RSB>::BYTES, stream, mapA, mapB, mapY, full) != cudaSuccess)
                    return NVFP4_ERR_CUDA;
                GemmParams rest = p;
                rest.tile_base = tiles - tail;
                rest.tile_count = tail;
                rest.splits = ts;
                return launch_split_k<RSB, F32>(mapA, mapB, mapY, rest, tail * ts, ts, stream);
            }
        }
    }
    const int grid = tiles < dev.sms ? tiles : dev.sms;
    if (launch_pdl(gemm_kernel<QOUT, I8, false, RSB, F32>, (unsigned)grid, THREADS,
                   GemmSmem<RSB>::BYTES, stream, mapA, mapB, mapY, p) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    return NVFP4_OK;
}

// Prepared weight scales: the 4 KiB block of (256-row block nb, K stage s of 256 values)
// holds at h * 2048 + j * 512 the 512-byte 128x4 chunk of row tile 2 nb + h and K step
// 4 s + j -- the order in which a stage's B scales sit in shared memory -- with zeros for
// row tiles past the last one and steps past K / 64.  One thread per 16 bytes.
__global__ void __launch_bounds__(256) prepare_scales_kernel(const uint8_t* __restrict__ sf,
                                                             uint8_t* __restrict__ out,
                                                             int64_t pieces, int kchunks,
                                                             int kstages, int row_tiles) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < pieces;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t blk = i >> 8;
        const int q = (int)(i & 255);
        const int h = q >> 7, j = (q >> 5) & 3, part = q & 31;
        const int64_t nb = blk / kstages, st = blk - nb * kstages;
        const int64_t tile = 2 * nb + h, k = 4 * st + j;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (tile < row_tiles && k < kchunks)
            v = *reinterpret_cast<const uint4*>(sf + (tile * kchunks + k) * 512 + part * 16);
        *reinterpret_cast<uint4*>(out + blk * 4096 + h * 2048 + j * 512 + part * 16) = v;
    }
}

}  // namespace

size_t prepared_scale_bytes(int64_t N, int64_t K) {
    return (size_t)((N + 255) / 256) * (size_t)((K / 64 + 3) / 4) * 4096u;
}

nvfp4_status launch_prepare_scales(const uint8_t* sf, int64_t N, int64_t K, uint8_t* out,
                                   cudaStream_t stream) {
    DeviceInfo dev;
    nvfp4_status st = device_info(&dev);
    if (st != NVFP4_OK) return st;
    const int kchunks = (int)(K / 64);
    const int kstages = (kchunks + 3) / 4;
    const int64_t pieces = (int64_t)((N + 255) / 256) * kstages * 256;
    const int64_t need = (pieces + 255) / 256;
    const int64_t cap = (int64_t)dev.sms * 8;
    const int grid = (int)(need < cap ? (need > 0 ? need : 1) : cap);
    prepare_scales_kernel<<<grid, 256, 0, stream>>>(sf, out, pieces, kchunks, kstages,
                                                    (int)((N + 127) / 128));
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

nvfp4_status launch_gemm(const uint8_t* a, const uint8_t* sfa, const uint8_t* b,
                         const uint8_t* sfb, const float* alpha, const void* bias, void* y,
                         int64_t M, int64_t N, int64_t K, cudaStream_t stream,
                         bool weights_ready) {
    return launch_gemm_impl<false, false>(a, sfa, b, sfb, alpha, bias, y, M, N, K, nullptr,
                                          nullptr, nullptr, stream, weights_ready);
}

nvfp4_status launch_gemm_prepared(const uint8_t* a, const uint8_t* sfa, const uint8_t* b,
                                  const uint8_t* sfb_prepared, const float* alpha,
                                  const void* bias, void* y, int64_t M, int64_t N, int64_t K,
                                  cudaStream_t stream, bool weights_ready) {
    return launch_gemm_impl<false, false, true>(a, sfa, b, sfb_prepared, alpha, bias, y, M, N, K,
                                                nullptr, nullptr, nullptr, stream, weights_ready);
}

nvfp4_status launch_gemm_f32(const uint8_t* a, const uint8_t* sfa, const uint8_t* b,
                             const uint8_t* sfb, bool sfb_prepared, const float* alpha,
                             const void* bias, float* y, int64_t M, int64_t N, int64_t K,
                             cudaStream_t stream) {
    if (sfb_prepared)
        return launch_gemm_impl<false, false, true, true>(a, sfa, b, sfb, alpha, bias, y, M, N,
                                                          K, nullptr, nullptr, nullptr, stream);
    return launch_gemm_impl<false, false, false, true>(a, sfa, b, sfb, alpha, bias, y, M, N, K,
                                                       nullptr, nullptr, nullptr, stream);
}

nvfp4_status launch_gemm_quant_out(const uint8_t* a, const uint8_t* sfa, const uint8_t* b,
                                   const uint8_t* sfb, const float* alpha, const void* bias,
                                   const float* gsf_out, uint8_t* out_packed, uint8_t* out_sf,
                                   int64_t M, int64_t N, int64_t K, cudaStream_t stream) {
    QuantOut q{out_packed, out_sf, gsf_out};
    return launch_gemm_impl<true, false>(a, sfa, b, sfb, alpha, bias, nullptr, M, N, K, &q,
                                         nullptr, nullptr, stream);
}

nvfp4_status launch_int8_gemm(const int8_t* a, const float* sa, const int8_t* b, const float* sb,
                              const void* bias, void* y, int64_t M, int64_t N, int64_t K,
                              cudaStream_t stream) {
    return launch_gemm_impl<false, true>(reinterpret_cast<const uint8_t*>(a), nullptr,
                                         reinterpret_cast<const uint8_t*>(b), nullptr, nullptr,
                                         bias, y, M, N, K, nullptr, sa, sb, stream);
}

}  // namespace nvfp4
