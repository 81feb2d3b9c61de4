// debug.cu -- two diagnostics the test suite drives through the C ABI:
//   * a sweep that runs the quantizer's own fp32 -> E2M1 and fp32 -> E4M3 device
//     conversions over a range of fp32 bit patterns, so they can be compared with
//     the CPU oracle pattern by pattern;
//   * a kernel whose barrier wait is bound to run out, to exercise the timeout
//     reporting path without hanging or faulting the GPU.
#include "common.cuh"
#include "kernels.h"

namespace nvfp4 {

namespace {

__global__ void cvt_sweep_kernel(uint32_t first, int64_t n, uint8_t* e2m1, uint8_t* e4m3,
                                 uint8_t* scale) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const float v = __uint_as_float(first + (uint32_t)i);
        e2m1[i] = (uint8_t)(e2m1x2_from_f32(v, 0.0f) & 0xfu);
        e4m3[i] = (uint8_t)e4m3_from_f32(fabsf(v));
        scale[i] = (uint8_t)e4m3_scale_of_scaled_max(fabsf(v));
    }
}

__global__ void wait_timeout_kernel(uint64_t budget_ns, int* status) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // nothing arrives on `bar`: the wait must give up after budget_ns
        mbar_wait_bounded(&bar, 0, &abort_flag, status, budget_ns);
    }
    __syncthreads();
}

}  // namespace

nvfp4_status launch_cvt_sweep(uint32_t first, int64_t n, uint8_t* e2m1, uint8_t* e4m3,
                              uint8_t* scale, cudaStream_t stream) {
    DeviceInfo dev;
    nvfp4_status st = device_info(&dev);
    if (st != NVFP4_OK) return st;
    int64_t blocks = (n + 255) / 256;
    const int grid = (int)(blocks < dev.sms * 16 ? blocks : dev.sms * 16);
    cvt_sweep_kernel<<<grid, 256, 0, stream>>>(first, n, e2m1, e4m3, scale);
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

nvfp4_status launch_wait_timeout(int64_t budget_us, cudaStream_t stream) {
    int* status = nullptr;
    nvfp4_status st = status_word(&status);
    if (st != NVFP4_OK) return st;
    wait_timeout_kernel<<<1, 32, 0, stream>>>((uint64_t)budget_us * 1000ull, status);
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

}  // namespace nvfp4
