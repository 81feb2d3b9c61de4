// api.cu -- the C ABI: argument checks, workspace carving, launches.
//
// Every entry point checks its arguments on the host first and launches nothing
// when a check fails.  The checks mirror the pages' own: "minimax_h3_nvfp4_decoder"
// -- NVFP4DecoderLinear.__init__ (in_features % 16, in_features % rotation_group)
// and from_packed (packed weight shape); "convert_minimax_h3_text_encoder_nvfp4.py"
// -- quantize_language_linear (exact packed and scale shapes).
#include <cmath>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace nvfp4 {

// Per-device asynchronous status word (see nvfp4_last_device_status).
__device__ int g_status_word;

namespace {

constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
int* g_status_ptr[kMaxDevices];
std::mutex g_mu;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

bool valid_group(int g) { return g == 0 || g == 16 || g == 32 || g == 64 || g == 128; }

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// Workspace carving for nvfp4_linear: packed x | scales | {gsf_x, alpha} | partials.
struct LinearWs {
    size_t packed, sf, scalars, partials, total;
};

LinearWs linear_ws(int64_t M, int64_t K) {
    LinearWs w;
    w.packed = 0;
    w.sf = align256((size_t)M * (size_t)K / 2);
    w.scalars = w.sf + align256(nvfp4_scale_bytes(M, K));
    w.partials = w.scalars + 256;
    w.total = w.partials + align256(kQuantWorkspace);
    return w;
}

}  // namespace

nvfp4_status device_info(DeviceInfo* out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return NVFP4_ERR_DEVICE;
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_dev[dev].device != dev) {
        cudaDeviceProp prop;
        if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return NVFP4_ERR_CUDA;
        g_dev[dev].sms = prop.multiProcessorCount;
        g_dev[dev].major = prop.major;
        g_dev[dev].minor = prop.minor;
        g_dev[dev].device = dev;
    }
    *out = g_dev[dev];
    if (out->major != 10 || out->minor != 0) return NVFP4_ERR_DEVICE;
    return NVFP4_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000,
                                             cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

nvfp4_status status_word(int** dev_ptr) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return NVFP4_ERR_DEVICE;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_status_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return NVFP4_ERR_CUDA;
        g_status_ptr[dev] = static_cast<int*>(p);
    }
    *dev_ptr = g_status_ptr[dev];
    return NVFP4_OK;
}

// Fixed scratch of nvfp4_linear_fixed_scratch: one per device, placed when the
// module loads.  Holds the same carve as a caller workspace of nvfp4_linear.
static __device__ __align__(256) uint8_t g_fixed_scratch[NVFP4_FIXED_SCRATCH_BYTES];

namespace {

uint8_t* g_fixed_scratch_ptr[kMaxDevices];

// Address of this device's fixed scratch; looked up once per device, with the
// device current.
nvfp4_status fixed_scratch(uint8_t** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return NVFP4_ERR_DEVICE;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_fixed_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_fixed_scratch) != cudaSuccess) return NVFP4_ERR_CUDA;
        g_fixed_scratch_ptr[dev] = static_cast<uint8_t*>(p);
    }
    *out = g_fixed_scratch_ptr[dev];
    return NVFP4_OK;
}
}  // namespace

}  // namespace nvfp4

using namespace nvfp4;

extern "C" {

const char* nvfp4_status_string(int s) {
    switch (s) {
        case NVFP4_OK: return "NVFP4_OK";
        case NVFP4_ERR_INVALID_ARG: return "NVFP4_ERR_INVALID_ARG";
        case NVFP4_ERR_SHAPE: return "NVFP4_ERR_SHAPE";
        case NVFP4_ERR_ALIGN: return "NVFP4_ERR_ALIGN";
        case NVFP4_ERR_WORKSPACE: return "NVFP4_ERR_WORKSPACE";
        case NVFP4_ERR_DEVICE: return "NVFP4_ERR_DEVICE";
        case NVFP4_ERR_CUDA: return "NVFP4_ERR_CUDA";
        case NVFP4_ERR_TIMEOUT: return "NVFP4_ERR_TIMEOUT";
        default: return "NVFP4_ERR_UNKNOWN";
    }
}

int nvfp4_abi_version(void) { return 1; }

size_t nvfp4_scale_bytes(int64_t rows, int64_t K) {
    if (rows <= 0 || K <= 0) return 0;
    return (size_t)((rows + 127) / 128 * 128) * (size_t)((K / 16 + 3) / 4 * 4);
}

size_t nvfp4_packed_bytes(int64_t rows, int64_t K) {
    if (rows <= 0 || K <= 0) return 0;
    return (size_t)rows * (size_t)(K / 2);
}

nvfp4_status hadamard_rotate(const void* x, void* y, int64_t rows, int64_t K, int group,
                             void* stream) {
    if (!x || !y || rows < 0 || group == 0 || !valid_group(group)) return NVFP4_ERR_INVALID_ARG;
    if (K <= 0 || K % group) return NVFP4_ERR_SHAPE;
    if (!aligned(x, 16) || !aligned(y, 16)) return NVFP4_ERR_ALIGN;
    DeviceInfo dev;
    nvfp4_status st = device_info(&dev);
    if (st != NVFP4_OK) return st;
    if (rows == 0) return NVFP4_OK;
    return launch_rotate(x, y, rows, K, group, static_cast<cudaStream_t>(stream));
}

size_t nvfp4_quantize_workspace_bytes(void) { return kQuantWorkspace; }

nvfp4_status nvfp4_quantize(const void* x, int64_t rows, int64_t K, int group,
                            const float* gsf_in, float* gsf_out, uint8_t* packed, uint8_t* sf,
                            const float* gsf_w, float* alpha_out, void* workspace,
                            size_t ws_bytes, void* stream) {
    if (!x || !packed || !sf || rows < 0 || !valid_group(group)) return NVFP4_ERR_INVALID_ARG;
    if (!gsf_in && !gsf_out) return NVFP4_ERR_INVALID_ARG;
    if ((gsf_w == nullptr) != (alpha_out == nullptr)) return NVFP4_ERR_INVALID_ARG;
    if ((gsf_w && !aligned(gsf_w, 4)) || (alpha_out && !aligned(alpha_out, 4)))
        return NVFP4_ERR_ALIGN;
    if (K <= 0 || K % 16 || (group && K % group)) return NVFP4_ERR_SHAPE;
    if (!aligned(x, 16) || !aligned(packed, 16) || !aligned(sf, 16)) return NVFP4_ERR_ALIGN;
    if ((gsf_in && !aligned(gsf_in, 4)) || (gsf_out && !aligned(gsf_out, 4)))
        return NVFP4_ERR_ALIGN;
    if (!gsf_in) {
        if (!workspace || ws_bytes < kQuantWorkspace) return NVFP4_ERR_WORKSPACE;
        if (!aligned(workspace, 16)) return NVFP4_ERR_ALIGN;
    }
    DeviceInfo dev;
    nvfp4_status st = device_info(&dev);
    if (st != NVFP4_OK) return st;
    if (rows == 0) return NVFP4_OK;
    return launch_quantize(x, rows, K, group, gsf_in, gsf_out, packed, sf,
                           static_cast<float*>(workspace), gsf_w, alpha_out,
                           static_cast<cudaStream_t>(stream));
}

nvfp4_status nvfp4_gemm(const uint8_t* a, const uint8_t* sfa, const uint8_t* b,
                        const uint8_t* sfb, const float* alpha, const void* bias, void* y,
                        int64_t M, int64_t N, int64_t K, void* stream) {
    if (!a || !sfa || !b || !sfb || !alpha || !y || M < 0 || N < 0) return NVFP4_ERR_INVALID_ARG;
    if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31)) return NVFP4_ERR_INVALID_ARG;
    if (K <= 0 || K % 64 || K >= (int64_t(1) << 31)) return NVFP4_ERR_SHAPE;
    if (!aligned(a, 16) || !aligned(sfa, 16) || !aligned(b, 16) || !aligned(sfb, 16) ||
        !aligned(y, 16) || !aligned(alpha, 4) || (bias && !aligned(bias, 16)))
        return NVFP4_ERR_ALIGN;
    DeviceInfo dev;
    nvfp4_status st = device_info(&dev);
    if (st != NVFP4_OK) return st;
    if (M == 0 || N == 0) return NVFP4_OK;
    return launch_gemm(a, sfa, b, sfb, alpha, bias, y, M, N, K, static_cast<cudaStream_t>(stream));
}

nvfp4_status nvfp4_gemm_prepared(const uint8_t* a, const uint8_t* sfa, const uint8_t* b,
                                 const uint8_t* sfb_prepared, const float* alpha, const void* bias,
                                 void* y, int64_t M, int64_t N, int64_t K, void* stream) {
    if (!a || !sfa || !b || !sfb_prepared || !alpha || !y || M < 0 || N < 0)
        return NVFP4_ERR_INVALID_ARG;
    if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31)) return NVFP4_ERR_INVALID_ARG;
    if (K <= 0 || K % 64 || K >= (int64_t(1) << 31)) return NVFP4_ERR_SHAPE;
    if (!aligned(a, 16) || !aligned(sfa, 16) || !aligned(b, 16) || !aligned(sfb_prepared, 16) ||
        !aligned(y, 16) || !aligned(alpha, 4) || (bias && !aligned(bias, 16)))
        return NVFP4_ERR_ALIGN;
    DeviceInfo dev;
    nvfp4_status st = device_info(&dev);
    if (st != NVFP4_OK) return st;
    if (M == 0 || N == 0) return NVFP4_OK;
    return launch_gemm_prepared(a, sfa, b, sfb_prepared, alpha, bias, y, M, N, K,
                                static_cast<cudaStream_t>(stream));
}

size_t nvfp4_prepared_scale_bytes(int64_t N, int64_t K) {
    if (N < 0 || K <= 0 || K % 64 || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31)) return 0;
    return prepared_scale_bytes(N, K);
}

nvfp4_status nvfp4_prepare_weight_scales(const uint8_t* sf, int64_t N, int64_t K, uint8_t* out,
                                         void* stream) {
    if (!sf || !out || N < 0 || N >= (int64_t(1) << 31)) return NVFP4_ERR_INVALID_ARG;
    if (K <= 0 || K % 64 || K >= (int64_t(1) << 31)) return NVFP4_ERR_SHAPE;
    if (!aligned(sf, 16) || !aligned(out, 16)) return NVFP4_ERR_ALIGN;
    DeviceInfo dev;
    nvfp4_status st = device_info(&dev);
    if (st != NVFP4_OK) return st;
    if (N == 0) return NVFP4_OK;
    return launch_prepare_scales(sf, N, K, out, static_cast<cudaStream_t>(stream));
}

nvfp4_status nvfp4_dequantize(const uint8_t* packed, const uint8_t* sf, const float* gsf,
                              int64_t rows, int64_t K, void* y, void* stream) {
    if (!packed || !sf || !gsf || !y || rows < 0) return NVFP4_ERR_INVALID_ARG;
    if (K <= 0 || K % 16) return NVFP4_ERR_SHAPE;
    if (!aligned(packed, 16) || !aligned(sf, 16) || !aligned(y, 16) || !aligned(gsf, 4))
        return NVFP4_ERR_ALIGN;
    DeviceInfo dev;
    nvfp4_status st = device_info(&dev);
    if (st != NVFP4_OK) return st;
    if (rows == 0) return NVFP4_OK;
    return launch_dequantize(packed, sf, gsf, rows, K, y, static_cast<cudaStream_t>(stream));
}

nvfp4_status nvfp4_gemm_quantize_out(const uint8_t* a, const uint8_t* sfa, const uint8_t* b,
                                     const uint8_t* sfb, const float* alpha, const void* bias,
                                     const float* gsf_out, uint8_t* out_packed, uint8_t* out_sf,
                                     int64_t M, int64_t N, int64_t K, void* stream) {
    if (!a || !sfa || !b || !sfb || !alpha || !gsf_out || !out_packed || !out_sf || M < 0 ||
        N < 0)
        return NVFP4_ERR_INVALID_ARG;
    if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31)) return NVFP4_ERR_INVALID_ARG;
    if (K <= 0 || K % 64 || K >= (int64_t(1) << 31) || N % 64) return NVFP4_ERR_SHAPE;
    if (!aligned(a, 16) || !aligned(sfa, 16) || !aligned(b, 16) || !aligned(sfb, 16) ||
        !aligned(out_packed, 16) || !aligned(out_sf, 16) || !aligned(alpha, 4) ||
        !aligned(gsf_out, 4) || (bias && !aligned(bias, 16)))
        return NVFP4_ERR_ALIGN;
    DeviceInfo dev;
    nvfp4_status st = device_info(&dev);
    if (st != NVFP4_OK) return st;
    if (M == 0 || N == 0) return NVFP4_OK;
    return launch_gemm_quant_out(a, sfa, b, sfb, alpha, bias, gsf_out, out_packed, out_sf, M, N,
                                 K, static_cast<cudaStream_t>(stream));
}

nvfp4_status int8_quantize_rows(const void* x, int64_t rows, int64_t K, int8_t* q, float* scale,
                                void* stream) {
    if (!x || !q || !scale || rows < 0) return NVFP4_ERR_INVALID_ARG;
    if (K <= 0 || K % 16) return NVFP4_ERR_SHAPE;
    if (!aligned(x, 16) || !aligned(q, 16) || !aligned(scale, 4)) return NVFP4_ERR_ALIGN;
    DeviceInfo dev;
    nvfp4_status st = device_info(&dev);
    if (st != NVFP4_OK) return st;
    if (rows == 0) return NVFP4_OK;
    return launch_int8_quantize_rows(x, rows, K, q, scale, static_cast<cudaStream_t>(stream));
}

nvfp4_status int8_gemm(const int8_t* a, const float* sa, const int8_t* b, const float* sb,
                       const void* bias, void* y, int64_t M, int64_t N, int64_t K, void* stream) {
    if (!a || !sa || !b || !sb || !y || M < 0 || N < 0) return NVFP4_ERR_INVALID_ARG;
    if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31)) return NVFP4_ERR_INVALID_ARG;
    if (K <= 0 || K % 32 || K >= (int64_t(1) << 31)) return NVFP4_ERR_SHAPE;
    if (!aligned(a, 16) || !aligned(b, 16) || !aligned(y, 16) || !aligned(sa, 16) ||
        !aligned(sb, 16) || (bias && !aligned(bias, 16)))
        return NVFP4_ERR_ALIGN;
    DeviceInfo dev;
    nvfp4_status st = device_info(&dev);
    if (st != NVFP4_OK) return st;
    if (M == 0 || N == 0) return NVFP4_OK;
    return launch_int8_gemm(a, sa, b, sb, bias, y, M, N, K, static_cast<cudaStream_t>(stream));
}

size_t int8_linear_workspace_bytes(int64_t M, int64_t K) {
    if (M < 0 || K <= 0) return 0;
    return align256((size_t)M * (size_t)K) + align256((size_t)M * 4);
}

nvfp4_status int8_linear(const void* x, int64_t M, int64_t K, const int8_t* wq, const float* sw,
                         int64_t N, const void* bias, void* workspace, size_t ws_bytes, void* y,
                         void* stream) {
    if (!x || !wq || !sw || !y || M < 0 || N < 0) return NVFP4_ERR_INVALID_ARG;
    if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31)) return NVFP4_ERR_INVALID_ARG;
    if (K <= 0 || K % 32 || K >= (int64_t(1) << 31)) return NVFP4_ERR_SHAPE;
    if (!aligned(x, 16) || !aligned(wq, 16) || !aligned(sw, 16) || !aligned(y, 16) ||
        (bias && !aligned(bias, 16)))
        return NVFP4_ERR_ALIGN;
    const size_t need = int8_linear_workspace_bytes(M, K);
    if (!workspace || ws_bytes < need) return NVFP4_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return NVFP4_ERR_ALIGN;
    DeviceInfo dev;
    nvfp4_status st = device_info(&dev);
    if (st != NVFP4_OK) return st;
    if (M == 0 || N == 0) return NVFP4_OK;
    int8_t* xq = static_cast<int8_t*>(workspace);
    float* sx = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                         align256((size_t)M * (size_t)K));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    st = launch_int8_quantize_rows(x, M, K, xq, sx, s);
    if (st != NVFP4_OK) return st;
    return launch_int8_gemm(xq, sx, wq, sw, bias, y, M, N, K, s);
}

size_t nvfp4_linear_workspace_bytes(int64_t M, int64_t K) {
    if (M < 0 || K <= 0) return 0;
    return linear_ws(M, K).total;
}

// nvfp4_linear and nvfp4_linear_prepared: the same checks and launches; `prepared` says
// which order w_sf is in (128x4, or nvfp4_prepare_weight_scales).
static nvfp4_status linear_impl(const void* x, int64_t M, int64_t K, const uint8_t* w_packed,
                         const uint8_t* w_sf, const float* gsf_w, int64_t N, const void* bias,
                         const float* gsf_x, int group, void* workspace, size_t ws_bytes,
                         void* y, void* stream, bool prepared) {
    if (!x || !w_packed || !w_sf || !gsf_w || !y || M < 0 || N < 0 || !valid_group(group))
        return NVFP4_ERR_INVALID_ARG;
    if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31)) return NVFP4_ERR_INVALID_ARG;
    if (K <= 0 || K % 64 || (group && K % group) || K >= (int64_t(1) << 31))
        return NVFP4_ERR_SHAPE;
    if (!aligned(x, 16) || !aligned(w_packed, 16) || !aligned(w_sf, 16) || !aligned(y, 16) ||
        !aligned(gsf_w, 4) || (gsf_x && !aligned(gsf_x, 4)) || (bias && !aligned(bias, 16)))
        return NVFP4_ERR_ALIGN;
    const LinearWs ws = linear_ws(M, K);
    if (!workspace || ws_bytes < ws.total) return NVFP4_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return NVFP4_ERR_ALIGN;
    DeviceInfo dev;
    nvfp4_status st = device_info(&dev);
    if (st != NVFP4_OK) return st;
    if (M == 0 || N == 0) return NVFP4_OK;

    uint8_t* base = static_cast<uint8_t*>(workspace);
    uint8_t* xp = base + ws.packed;
    uint8_t* xsf = base + ws.sf;
    float* scalars = reinterpret_cast<float*>(base + ws.scalars);
    float* partials = reinterpret_cast<float*>(base + ws.partials);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    st = launch_quantize(x, M, K, group, gsf_x, &scalars[0], xp, xsf, partials, gsf_w, &scalars[1],
                         s);
    if (st != NVFP4_OK) return st;
    // the weights were complete before the quantizer began: the GEMM may load them early
    if (prepared)
        return launch_gemm_prepared(xp, xsf, w_packed, w_sf, &scalars[1], bias, y, M, N, K, s,
                                    true);
    return launch_gemm(xp, xsf, w_packed, w_sf, &scalars[1], bias, y, M, N, K, s, true);
}

nvfp4_status nvfp4_linear(const void* x, int64_t M, int64_t K, const uint8_t* w_packed,
                          const uint8_t* w_sf, const float* gsf_w, int64_t N, const void* bias,
                          const float* gsf_x, int group, void* workspace, size_t ws_bytes,
                          void* y, void* stream) {
    return linear_impl(x, M, K, w_packed, w_sf, gsf_w, N, bias, gsf_x, group, workspace,
                       ws_bytes, y, stream, false);
}

nvfp4_status nvfp4_linear_prepared(const void* x, int64_t M, int64_t K, const uint8_t* w_packed,
                                   const uint8_t* w_sf_prepared, const float* gsf_w, int64_t N,
                                   const void* bias, const float* gsf_x, int group,
                                   void* workspace, size_t ws_bytes, void* y, void* stream) {
    return linear_impl(x, M, K, w_packed, w_sf_prepared, gsf_w, N, bias, gsf_x, group, workspace,
                       ws_bytes, y, stream, true);
}

nvfp4_status nvfp4_linear_fixed_scratch(const void* x, int64_t M, int64_t K,
                                        const uint8_t* w_packed, const uint8_t* w_sf,
                                        const float* gsf_w, int64_t N, const void* bias,
                                        const float* gsf_x, int group, void* y, void* stream) {
    if (!x || !w_packed || !w_sf || !gsf_w || !y || M < 0 || N < 0 || !valid_group(group))
        return NVFP4_ERR_INVALID_ARG;
    if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31)) return NVFP4_ERR_INVALID_ARG;
    if (K <= 0 || K % 64 || (group && K % group) || K >= (int64_t(1) << 31))
        return NVFP4_ERR_SHAPE;
    if (!aligned(x, 16) || !aligned(w_packed, 16) || !aligned(w_sf, 16) || !aligned(y, 16) ||
        !aligned(gsf_w, 4) || (gsf_x && !aligned(gsf_x, 4)) || (bias && !aligned(bias, 16)))
        return NVFP4_ERR_ALIGN;
    const LinearWs ws = linear_ws(M, K);
    if (ws.total > NVFP4_FIXED_SCRATCH_BYTES) return NVFP4_ERR_WORKSPACE;
    DeviceInfo dev;
    nvfp4_status st = device_info(&dev);
    if (st != NVFP4_OK) return st;
    uint8_t* base = nullptr;
    st = fixed_scratch(&base);
    if (st != NVFP4_OK) return st;
    if (M == 0 || N == 0) return NVFP4_OK;

    uint8_t* xp = base + ws.packed;
    uint8_t* xsf = base + ws.sf;
    float* scalars = reinterpret_cast<float*>(base + ws.scalars);
    float* partials = reinterpret_cast<float*>(base + ws.partials);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    st = launch_quantize(x, M, K, group, gsf_x, &scalars[0], xp, xsf, partials, gsf_w, &scalars[1],
                         s);
    if (st != NVFP4_OK) return st;
    return launch_gemm(xp, xsf, w_packed, w_sf, &scalars[1], bias, y, M, N, K, s, true);
}

nvfp4_status nvfp4_debug_gemm_f32(const uint8_t* a, const uint8_t* sfa, const uint8_t* b,
                                  const uint8_t* sfb, int sfb_prepared, const float* alpha,
                                  const void* bias, float* y_f32, int64_t M, int64_t N, int64_t K,
                                  void* stream) {
    if (!a || !sfa || !b || !sfb || !alpha || !y_f32 || M < 0 || N < 0 ||
        (sfb_prepared != 0 && sfb_prepared != 1))
        return NVFP4_ERR_INVALID_ARG;
    if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31)) return NVFP4_ERR_INVALID_ARG;
    if (K <= 0 || K % 64 || K >= (int64_t(1) << 31)) return NVFP4_ERR_SHAPE;
    if (!aligned(a, 16) || !aligned(sfa, 16) || !aligned(b, 16) || !aligned(sfb, 16) ||
        !aligned(y_f32, 16) || !aligned(alpha, 4) || (bias && !aligned(bias, 16)))
        return NVFP4_ERR_ALIGN;
    DeviceInfo dev;
    nvfp4_status st = device_info(&dev);
    if (st != NVFP4_OK) return st;
    if (M == 0 || N == 0) return NVFP4_OK;
    return launch_gemm_f32(a, sfa, b, sfb, sfb_prepared != 0, alpha, bias, y_f32, M, N, K,
                           static_cast<cudaStream_t>(stream));
}

nvfp4_status nvfp4_last_device_status(void* stream, int* status) {
    if (!status) return NVFP4_ERR_INVALID_ARG;
    int* dev_ptr = nullptr;
    nvfp4_status st = status_word(&dev_ptr);
    if (st != NVFP4_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int host = 0;
    if (cudaStreamSynchronize(s) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (cudaMemcpyAsync(&host, dev_ptr, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    if (cudaMemsetAsync(dev_ptr, 0, sizeof(int), s) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return NVFP4_ERR_CUDA;
    *status = host;
    return NVFP4_OK;
}

nvfp4_status nvfp4_debug_cvt_sweep(uint32_t first, int64_t n, uint8_t* e2m1, uint8_t* e4m3,
                                   uint8_t* scale, void* stream) {
    if (!e2m1 || !e4m3 || !scale || n < 0 || n > (int64_t(1) << 32)) return NVFP4_ERR_INVALID_ARG;
    DeviceInfo dev;
    nvfp4_status st = device_info(&dev);
    if (st != NVFP4_OK) return st;
    if (n == 0) return NVFP4_OK;
    return launch_cvt_sweep(first, n, e2m1, e4m3, scale, static_cast<cudaStream_t>(stream));
}

nvfp4_status nvfp4_debug_wait_timeout(int64_t budget_us, void* stream) {
    if (budget_us < 1 || budget_us > 2000000) return NVFP4_ERR_INVALID_ARG;
    DeviceInfo dev;
    nvfp4_status st = device_info(&dev);
    if (st != NVFP4_OK) return st;
    return launch_wait_timeout(budget_us, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
