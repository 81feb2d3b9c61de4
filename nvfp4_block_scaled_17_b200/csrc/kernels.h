// kernels.h -- host-side launchers shared between the translation units.
#pragma once

#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include "nvfp4.h"

namespace nvfp4 {

// Cached per-device facts (multiprocessor count, compute capability).
// Launch with programmatic stream serialization (the kernel overlaps its set-up with the
// tail of the previous kernel on the stream and runs griddep_wait() before any global
// memory access).  Used for the persistent kernels, whose grid is resident at once.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), unsigned grid, unsigned block,
                              size_t smem, cudaStream_t stream, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(block, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

struct DeviceInfo {
    int device = -1;
    int sms = 0;
    int major = 0, minor = 0;
};
nvfp4_status device_info(DeviceInfo* out);

// Rotation scale rn(1/sqrt(g)) for g in {16, 32, 64, 128}.
float hadamard_scale(int g);

// Quantizer: [rotate] -> [amax pass] -> encode pass.  `partials` (kMaxPartials
// floats) is required when gsf_in == nullptr.  When gsf_w and alpha_out are
// given the encode pass also writes alpha = rn(1 / rn(gsf * gsf_w)).
nvfp4_status launch_quantize(const void* x, int64_t rows, int64_t K, int group,
                             const float* gsf_in, float* gsf_out, uint8_t* packed, uint8_t* sf,
                             float* partials, const float* gsf_w, float* alpha_out,
                             cudaStream_t stream);

nvfp4_status launch_rotate(const void* x, void* y, int64_t rows, int64_t K, int group,
                           cudaStream_t stream);

// weights_ready (here and below): b and sfb were complete before the previous kernel on
// the stream started -- the linear paths, whose previous kernel is their own activation
// quantizer, which itself waited for all earlier work -- so the kernel may start loading
// them before it waits for that kernel.  False for a bare GEMM call, whose predecessor may
// be the kernel that writes the weights.
nvfp4_status launch_gemm(const uint8_t* a, const uint8_t* sfa, const uint8_t* b,
                         const uint8_t* sfb, const float* alpha, const void* bias, void* y,
                         int64_t M, int64_t N, int64_t K, cudaStream_t stream,
                         bool weights_ready = false);

// The same GEMM with the weight's scales in the prepared order (launch_prepare_scales):
// one 4 KiB block per 256-row block and 256-value K stage, in shared-memory order.
nvfp4_status launch_gemm_prepared(const uint8_t* a, const uint8_t* sfa, const uint8_t* b,
                                  const uint8_t* sfb_prepared, const float* alpha,
                                  const void* bias, void* y, int64_t M, int64_t N, int64_t K,
                                  cudaStream_t stream, bool weights_ready = false);
size_t prepared_scale_bytes(int64_t N, int64_t K);
nvfp4_status launch_prepare_scales(const uint8_t* sf, int64_t N, int64_t K, uint8_t* out,
                                   cudaStream_t stream);

// The same GEMM (128x4 or prepared weight scales) with an unrounded fp32 output:
// y[m, n] = fp32(alpha * acc) + bias[n], the value the bf16 builds round once.
nvfp4_status launch_gemm_f32(const uint8_t* a, const uint8_t* sfa, const uint8_t* b,
                             const uint8_t* sfb, bool sfb_prepared, const float* alpha,
                             const void* bias, float* y, int64_t M, int64_t N, int64_t K,
                             cudaStream_t stream);

// The GEMM for M <= kSmallMaxRows activation rows with the operands swapped
// (y^T = W x^T: weight rows on the MMA's M, activation rows on its N), K split over a
// thread-block cluster; same arguments and result as launch_gemm / launch_gemm_prepared
// (sfb_prepared) / launch_gemm_f32 (f32_out, y is then float*).  The kernel takes up to
// 128 rows; the dispatch uses it up to 32, where it measured faster than the general
// kernel's split-K build (its reduction grows with M).
constexpr int64_t kSmallMaxRows = 32;
nvfp4_status launch_gemm_small(const uint8_t* a, const uint8_t* sfa, const uint8_t* b,
                               const uint8_t* sfb, bool sfb_prepared, bool f32_out,
                               const float* alpha, const void* bias, void* y, int64_t M,
                               int64_t N, int64_t K, cudaStream_t stream,
                               bool weights_ready = false);

// 2-D uint8 tensor map [rows, row_bytes] with a [box_rows, 128-byte] box and the
// 128-byte swizzle (the GEMM operand loads).
bool make_operand_map(CUtensorMap* map, const void* base, int64_t rows, int64_t row_bytes,
                      int box_rows);

// The GEMM whose epilogue emits the NVFP4 encoding of its bf16 output instead of the
// output itself (static global scale gsf_out, 128x4 scales, N % 64 == 0).
nvfp4_status launch_gemm_quant_out(const uint8_t* a, const uint8_t* sfa, const uint8_t* b,
                                   const uint8_t* sfb, const float* alpha, const void* bias,
                                   const float* gsf_out, uint8_t* out_packed, uint8_t* out_sf,
                                   int64_t M, int64_t N, int64_t K, cudaStream_t stream);

// int8 per-row W8A8: row quantizer and GEMM with y = bf16((acc * sa[m]) * sb[n] + bias).
nvfp4_status launch_int8_quantize_rows(const void* x, int64_t rows, int64_t K, int8_t* q,
                                       float* scale, cudaStream_t stream);
nvfp4_status launch_int8_gemm(const int8_t* a, const float* sa, const int8_t* b, const float* sb,
                              const void* bias, void* y, int64_t M, int64_t N, int64_t K,
                              cudaStream_t stream);

// NVFP4 -> bf16 expansion: y = bf16(fp32(E2M1 * E4M3) / gsf).
nvfp4_status launch_dequantize(const uint8_t* packed, const uint8_t* sf, const float* gsf,
                               int64_t rows, int64_t K, void* y, cudaStream_t stream);

nvfp4_status launch_cvt_sweep(uint32_t first, int64_t n, uint8_t* e2m1, uint8_t* e4m3,
                              uint8_t* scale, cudaStream_t stream);
nvfp4_status launch_wait_timeout(int64_t budget_us, cudaStream_t stream);

// The driver's cuTensorMapEncodeTiled (looked up once through the runtime), or
// nullptr when the driver does not provide it.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

// The per-device asynchronous status word (device address for the current device).
nvfp4_status status_word(int** dev_ptr);

}  // namespace nvfp4
