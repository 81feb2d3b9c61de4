// int8.cu -- per-row int8 quantizer of the W8A8 linear.
//
// Page: "FastH3-4-step-Preview-v1-r16-int8" -- "What is inside": every quantized linear
// stores round(W / scale) clamped to -127..127 with scale = amax(|W[row]|) / 127 per
// output row, and activations are quantized per row at call time before the int8 GEMM.
// The division and the scale are fp32 (round to nearest even), round() is half to even,
// and an all-zero row has scale 0 and codes 0.
//
// One warp per row, grid-stride over rows: a pass over the row for its amax (packed bf16
// maxima, 16-byte loads), then a pass that divides (one reciprocal per row and an FMA
// correction per value), rounds and packs 8 codes per lane (the second read comes back
// from L1/L2).
#include "common.cuh"
#include "kernels.h"

namespace nvfp4 {

namespace {

constexpr int kI8Threads = 256;

__global__ void __launch_bounds__(kI8Threads) int8_rows_kernel(const uint16_t* __restrict__ x,
                                                               int64_t R, int64_t K,
                                                               int8_t* __restrict__ q,
                                                               float* __restrict__ scale) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * kI8Threads + threadIdx.x) >> 5;
    const int64_t n_warps = ((int64_t)gridDim.x * kI8Threads) >> 5;
    for (int64_t row = warp; row < R; row += n_warps) {
        const uint16_t* xr = x + row * K;
        uint32_t m = 0u;
        for (int64_t k = 8 * lane; k < K; k += 256)
            m = absmax2_bf16(m, absmax_word4(*reinterpret_cast<const uint4*>(xr + k)));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = absmax2_bf16(m, __shfl_xor_sync(0xffffffffu, m, o));
        const float s = __fdiv_rn(absmax_of_pair(m), 127.0f);
        if (lane == 0) scale[row] = s;
        // rn(x / s) for every x of the row: with r = rn(1/s) (within half an ulp of 1/s) the
        // first quotient x*r is faithful, the remainder x - s*q0 is exact in one FMA, and
        // q0 + rem*r rounded once is the correctly rounded quotient (Markstein's theorem);
        // |x| <= 127 s keeps every step finite.  A subnormal s (whose reciprocal would
        // overflow) takes the plain division instead.
        const bool fast = s >= 1.17549435e-38f;
        const float r = fast ? __frcp_rn(s) : 0.0f;
        int8_t* qr = q + row * K;
        // one loop per case, so the inner loop carries no per-value branch
        auto encode = [=](auto quotient) {
            for (int64_t k = 8 * lane; k < K; k += 256) {
                const uint4 v = *reinterpret_cast<const uint4*>(xr + k);
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
                int c[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint32_t word = w[j >> 1];
                    c[j] = __float2int_rn(quotient(
                        __uint_as_float((j & 1) ? (word & 0xffff0000u) : (word << 16))));
                }
                uint32_t out[2];
#pragma unroll
                for (int hh = 0; hh < 2; ++hh)
                    out[hh] = __byte_perm(__byte_perm(c[4 * hh], c[4 * hh + 1], 0x0040),
                                          __byte_perm(c[4 * hh + 2], c[4 * hh + 3], 0x0040), 0x5410);
                *reinterpret_cast<uint2*>(qr + k) = make_uint2(out[0], out[1]);
            }
        };
        // |x| <= amax keeps |x / s| <= 127 (1 + 2^-23): the rounded code is within -127..127
        // without a clamp.
        if (fast) {
            encode([r, s](float xv) {
                const float q0 = __fmul_rn(xv, r);
                return __fmaf_rn(__fmaf_rn(-q0, s, xv), r, q0);
            });
        } else if (s != 0.0f) {
            encode([s](float xv) { return __fdiv_rn(xv, s); });
        } else {
            encode([](float) { return 0.0f; });
        }
    }
}

}  // namespace

nvfp4_status launch_int8_quantize_rows(const void* x, int64_t rows, int64_t K, int8_t* q,
                                       float* scale, cudaStream_t stream) {
    DeviceInfo dev;
    nvfp4_status st = device_info(&dev);
    if (st != NVFP4_OK) return st;
    const int64_t need = (rows + kI8Threads / 32 - 1) / (kI8Threads / 32);
    const int64_t cap = (int64_t)dev.sms * 8;
    const int grid = (int)(need < cap ? (need > 0 ? need : 1) : cap);
    int8_rows_kernel<<<grid, kI8Threads, 0, stream>>>(static_cast<const uint16_t*>(x), rows, K, q,
                                                     scale);
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

}  // namespace nvfp4
