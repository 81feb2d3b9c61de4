// dequant.cu -- NVFP4 -> bf16 expansion of a packed tensor.
//
// Pages: "decode dynamic-scale NVFP4 H3 VAE tiles one at a time" --
// FASTVIDEO_H3_ENCODER_FUSED_DEQUANT (one fused pass that expands the serialized NVFP4
// text encoder to bf16 on GPUs without an FP4 GEMM).  The value of element (r, k) is
// E2M1(code) * E4M3(block scale) -- exact in fp32 -- divided by the global scale in fp32
// and rounded to nearest even to bf16.
//
// The result depends only on the (scale byte, code) pair of an element, so every CTA
// first fills a 256 x 16 table of bf16 results in shared memory (one correctly rounded
// division per entry) and then expands by table lookup.  A warp handles a 256-value
// segment of one row: lane t reads the 4 packed bytes of values 8t..8t+7 (one 128-byte
// line per warp) and writes their 16 bf16 bytes (one 512-byte run per warp).  A warp's
// work unit is four consecutive segments of a row, loaded before they are expanded.
// CTAs of 1024 threads, two per SM: the table is built 296 times per launch instead of
// 1184 with 256-thread CTAs, at the same 64 warps per SM.
#include <atomic>

#include "common.cuh"
#include "kernels.h"

namespace nvfp4 {

namespace {

constexpr int kDeqThreads = 1024;

constexpr int kDeqSegs = 4;           // 256-value segments per warp work unit (1024 values)

struct DeqParams {
    const uint8_t* packed;
    const uint8_t* sf;
    const float* gsf;
    uint16_t* y;
    int64_t rows, K;
    uint32_t upr;           // 1024-value units per row
    uint32_t total;         // rows * upr (< 2^31)
    FastDiv upr_div;
    int64_t cgroups;        // K / 64 rounded up: 4-block column groups of the scale layout
};

__global__ void __launch_bounds__(kDeqThreads) dequant_kernel(const DeqParams p) {
    __shared__ uint16_t tab[256 * 16];
    const float gsf = *p.gsf;
    for (int i = threadIdx.x; i < 256 * 16; i += kDeqThreads) {
        const uint32_t s8 = (uint32_t)i >> 4, code = (uint32_t)i & 15u;
        const float s = f32_from_e4m3(s8 & 0x7fu);
        const float c = e2m1_value(code);
        const float v = __fmul_rn(c, (s8 & 0x80u) ? -s : s);   // exact
        const float q = __fdiv_rn(v, gsf);
        tab[i] = (uint16_t)(bf16x2_rn(q, 0.0f) & 0xffffu);
    }
    __syncthreads();

    const int lane = threadIdx.x & 31;
    const uint32_t warp = (blockIdx.x * kDeqThreads + threadIdx.x) >> 5;
    const uint32_t n_warps = (gridDim.x * kDeqThreads) >> 5;
    for (uint32_t u = warp; u < p.total; u += n_warps) {
        const uint32_t row = fast_div(u, p.upr_div);
        const int64_t k = (int64_t)(u - row * p.upr) * 1024 + 8 * lane;   // segment 0
        // lane's block in segment j: k/16 + 16 j, i.e. 4-block column group k/64 + 4 j
        const uint8_t* pk = p.packed + (int64_t)row * (p.K / 2) + k / 2;
        const uint8_t* ps = p.sf + ((((int64_t)row >> 7) * p.cgroups + (k >> 6)) << 9) +
                            ((row & 31) << 4) + (((row >> 5) & 3) << 2) + ((k >> 4) & 3);
        uint16_t* py = p.y + (int64_t)row * p.K + k;
        uint32_t codes[kDeqSegs], base[kDeqSegs];
#pragma unroll
        for (int j = 0; j < kDeqSegs; ++j) {
            codes[j] = 0;
            base[j] = 0;
            if (k + 256 * j < p.K) {
                codes[j] = __ldg(reinterpret_cast<const uint32_t*>(pk + 128 * j));
                base[j] = (uint32_t)__ldg(ps + 2048 * j) << 4;
            }
        }
#pragma unroll
        for (int j = 0; j < kDeqSegs; ++j) {
            if (k + 256 * j >= p.K) continue;
            uint32_t w[4];
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const uint32_t lo = tab[base[j] | ((codes[j] >> (8 * b)) & 15u)];
                const uint32_t hi = tab[base[j] | ((codes[j] >> (8 * b + 4)) & 15u)];
                w[b] = lo | (hi << 16);
            }
            *reinterpret_cast<uint4*>(py + 256 * j) = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
}

}  // namespace

nvfp4_status launch_dequantize(const uint8_t* packed, const uint8_t* sf, const float* gsf,
                               int64_t rows, int64_t K, void* y, cudaStream_t stream) {
    if (rows * ((K + 1023) / 1024) >= (int64_t(1) << 31)) return NVFP4_ERR_SHAPE;
    DeviceInfo dev;
    nvfp4_status st = device_info(&dev);
    if (st != NVFP4_OK) return st;
    DeqParams p{};
    p.packed = packed;
    p.sf = sf;
    p.gsf = gsf;
    p.y = static_cast<uint16_t*>(y);
    p.rows = rows;
    p.K = K;
    p.upr = (uint32_t)((K + 1023) / 1024);
    p.total = (uint32_t)(rows * (int64_t)p.upr);
    p.upr_div = make_fastdiv(p.upr);
    p.cgroups = (K + 63) / 64;
    // one resident wave: every CTA builds the table once
    static std::atomic<int> per_sm[64];
    int resident = per_sm[dev.device & 63].load(std::memory_order_relaxed);
    if (!resident) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&resident, dequant_kernel, kDeqThreads,
                                                          0) != cudaSuccess ||
            resident <= 0)
            resident = 2;
        per_sm[dev.device & 63].store(resident, std::memory_order_relaxed);
    }
    const int64_t need = ((int64_t)p.total + kDeqThreads / 32 - 1) / (kDeqThreads / 32);
    const int64_t cap = (int64_t)dev.sms * resident;
    const int grid = (int)(need < cap ? (need > 0 ? need : 1) : cap);
    dequant_kernel<<<grid, kDeqThreads, 0, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

}  // namespace nvfp4
