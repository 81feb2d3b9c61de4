// quantize.cu -- the NVFP4 activation/weight quantizer, the dynamic-scale amax
// pass and the block Hadamard rotation, as one family of streaming kernels.
//
// Pages: "minimax_h3_nvfp4_decoder" -- nvfp4_linear_inference (dynamic global scale
// when global_sf_x is None, then the fenced quantizer with the 128x4 scale layout),
// _activation_global_sf (FP4_E4M3_RANGE / amax), rotate_activation and the module
// docstring (block Hadamard applied to the activation before FP4 rounding);
// "convert_minimax_h3_text_encoder_nvfp4.py" -- quantize_language_linear (weights go
// through the same quantizer with their own global scale).
//
// Work decomposition.  A "unit" is E consecutive values of one row (E = 64, or 128
// for a 128-wide rotation), handled by a pair of adjacent lanes: lane h of the pair
// owns the 8-value chunks 2i+h of the unit, so every load instruction of a warp
// reads 16 whole 32-byte sectors and each 16-value block lies half in each lane.
// With that split the only cross-lane step of the butterfly is the h = 8 stage
// (one shuffle per value); stages 1, 2, 4 stay inside a chunk and 16, 32, 64 inside
// a lane.  Block maxima need one shuffle per block; the scale bytes of four blocks
// form one aligned 32-bit word of the 128x4 layout.
#include <cmath>

#include "common.cuh"
#include "kernels.h"

namespace nvfp4 {

namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kThreads = 256;
constexpr int kUnitsPerCta = kThreads / 2;

struct UnitParams {
    const uint16_t* x;      // bf16 [rows, K]
    int64_t rows;           // rows holding data
    int64_t K;
    int64_t upr;            // units per row
    int64_t total_units;    // units to visit (padded rows included for the encode pass)
    float hscale;           // rn(1/sqrt(g))
    // encode pass
    uint8_t* packed;
    uint8_t* sf;
    int64_t cgroups;        // ceil(K/64): 4-block groups per row
    const float* gsf_in;
    const float* partials;
    int n_partials;
    float* gsf_out;
    const float* gsf_w;
    float* alpha_out;
    // amax pass
    float* partials_out;
    // rotate-only pass
    uint16_t* y;
};

template <int G>
struct UnitShape {
    static constexpr int E = (G == 128) ? 128 : 64;   // values per unit
    static constexpr int NCT = E / 16;                // 8-value chunks per lane
};

__device__ __forceinline__ uint4 ld_stream(const uint16_t* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint4 ld_plain(const uint16_t* p) {
    return *reinterpret_cast<const uint4*>(p);
}

__device__ __forceinline__ void unpack8(const uint4& w, float (&f)[8]) {
    f[0] = bf16lo(w.x); f[1] = bf16hi(w.x);
    f[2] = bf16lo(w.y); f[3] = bf16hi(w.y);
    f[4] = bf16lo(w.z); f[5] = bf16hi(w.z);
    f[6] = bf16lo(w.w); f[7] = bf16hi(w.w);
}

// One butterfly stage on a pair: (a, b) -> (a + b, a - b), each correctly rounded.
__device__ __forceinline__ void bfly(float& a, float& b) {
    float s = __fadd_rn(a, b);
    float d = __fsub_rn(a, b);
    a = s;
    b = d;
}

// Rotates every g-group of the unit in place (the values stay bf16 words).
template <int G>
__device__ __forceinline__ void rotate_unit(uint4 (&w)[UnitShape<G>::NCT], int h, float hscale) {
    constexpr int NCT = UnitShape<G>::NCT;
    float f[NCT][8];
#pragma unroll
    for (int i = 0; i < NCT; ++i) unpack8(w[i], f[i]);
    // stages h = 1, 2, 4 inside each chunk
#pragma unroll
    for (int i = 0; i < NCT; ++i) {
#pragma unroll
        for (int s = 1; s < 8; s *= 2)
#pragma unroll
            for (int e = 0; e < 8; ++e)
                if ((e & s) == 0) bfly(f[i][e], f[i][e + s]);
    }
    // stage h = 8: chunk 2i (lane h = 0) with chunk 2i + 1 (lane h = 1)
#pragma unroll
    for (int i = 0; i < NCT; ++i)
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            float o = __shfl_xor_sync(kFull, f[i][e], 1);
            f[i][e] = h ? __fsub_rn(o, f[i][e]) : __fadd_rn(f[i][e], o);
        }
    // stages h = 16, 32, 64: chunk pairs two, four, eight apart = local pairs 1, 2, 4 apart
#pragma unroll
    for (int s = 1; s < G / 16; s *= 2)
#pragma unroll
        for (int i = 0; i < NCT; ++i)
            if ((i & s) == 0)
#pragma unroll
                for (int e = 0; e < 8; ++e) bfly(f[i][e], f[i + s][e]);
#pragma unroll
    for (int i = 0; i < NCT; ++i) {
        float g[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) g[e] = __fmul_rn(f[i][e], hscale);
        w[i] = make_uint4(bf16x2_rn(g[0], g[1]), bf16x2_rn(g[2], g[3]), bf16x2_rn(g[4], g[5]),
                          bf16x2_rn(g[6], g[7]));
    }
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
    return v;
}

__device__ __forceinline__ float block_max(float v, float* red) {
    v = warp_max(v);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    v = (threadIdx.x < (blockDim.x >> 5)) ? red[threadIdx.x] : 0.0f;
    if (warp == 0) v = warp_max(v);
    return v;   // valid in warp 0
}

// MODE 0: amax partials.  MODE 1: quantize.  MODE 2: rotate only (G > 0).
template <int G, int MODE>
__global__ void __launch_bounds__(kThreads) unit_kernel(const UnitParams p) {
    constexpr int E = UnitShape<G>::E;
    constexpr int NCT = UnitShape<G>::NCT;
    __shared__ float red[32];
    __shared__ float s_gsf;

    const int lane = threadIdx.x & 31;
    const int h = lane & 1;
    const int64_t warp_id = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
    const int64_t n_warps = (int64_t)gridDim.x * (kThreads / 32);

    float gsf = 0.0f;
    if constexpr (MODE == 1) {
        if (p.gsf_in != nullptr) {
            gsf = *p.gsf_in;
        } else {
            float m = 0.0f;
            for (int i = threadIdx.x; i < p.n_partials; i += kThreads) m = fmaxf(m, p.partials[i]);
            m = block_max(m, red);
            if (threadIdx.x == 0) s_gsf = __fdiv_rn(kFp4E4m3Range, fmaxf(m, kAmaxFloor));
            __syncthreads();
            gsf = s_gsf;
        }
        if (blockIdx.x == 0 && threadIdx.x == 0) {
            if (p.gsf_out) *p.gsf_out = gsf;
            if (p.alpha_out) *p.alpha_out = __fdiv_rn(1.0f, __fmul_rn(gsf, *p.gsf_w));
        }
    }
    float tmax = 0.0f;

    for (int64_t base = warp_id * 16; base < p.total_units; base += n_warps * 16) {
        const int64_t unit = base + (lane >> 1);
        const bool active = unit < p.total_units;
        int64_t row = 0, u = 0;
        if (active) {
            row = unit / p.upr;
            u = unit - row * p.upr;
        }
        const int64_t e0 = u * E;
        const int valid = active ? (int)min((int64_t)E, p.K - e0) : 0;
        const bool data_row = active && row < p.rows;

        uint4 w[NCT];
        const uint16_t* src = p.x + row * p.K + e0;
#pragma unroll
        for (int i = 0; i < NCT; ++i) {
            const int c = 2 * i + h;
            // the rotate-only pass may run in place, so it does not use the read-only path
            w[i] = (data_row && c * 8 < valid)
                       ? (MODE == 2 ? ld_plain(src + c * 8) : ld_stream(src + c * 8))
                       : make_uint4(0, 0, 0, 0);
        }
        if constexpr (G > 0) rotate_unit<G>(w, h, p.hscale);

        if constexpr (MODE == 2) {
            uint16_t* dst = p.y + row * p.K + e0;
#pragma unroll
            for (int i = 0; i < NCT; ++i) {
                const int c = 2 * i + h;
                if (data_row && c * 8 < valid) *reinterpret_cast<uint4*>(dst + c * 8) = w[i];
            }
        } else if constexpr (MODE == 0) {
#pragma unroll
            for (int i = 0; i < NCT; ++i) tmax = fmaxf(tmax, absmax_words4(w[i]));
        } else {
            // block i of the unit = chunks 2i (lane h = 0) and 2i + 1 (lane h = 1)
            uint32_t codes[NCT];
            uint32_t s8[NCT];
#pragma unroll
            for (int i = 0; i < NCT; ++i) {
                const float tm = absmax_words4(w[i]);
                const float bmax = fmaxf(tm, __shfl_xor_sync(kFull, tm, 1));
                const float s_raw = __fdiv_rn(__fmul_rn(gsf, bmax), 6.0f);
                s8[i] = e4m3_from_f32(s_raw);
                const float s = f32_from_e4m3(s8[i]);
                codes[i] = 0u;
                if (s != 0.0f) {
                    const float inv = __fdiv_rn(gsf, s);
                    float v[8];
                    unpack8(w[i], v);
#pragma unroll
                    for (int e = 0; e < 8; ++e) v[e] = __fmul_rn(v[e], inv);
                    codes[i] = e2m1x8_from_f32(v);
                }
            }
            // scale words: blocks 4q..4q+3 -> one aligned 32-bit word, lane h = q & 1
#pragma unroll
            for (int q = 0; q < NCT / 4; ++q) {
                if (active && (q & 1) == h) {
                    const uint32_t word = s8[4 * q] | (s8[4 * q + 1] << 8) | (s8[4 * q + 2] << 16) |
                                          (s8[4 * q + 3] << 24);
                    const int64_t cg = e0 / 64 + q;
                    const int64_t off = (((row >> 7) * p.cgroups + cg) << 9) + ((row & 31) << 4) +
                                        (((row >> 5) & 3) << 2);
                    *reinterpret_cast<uint32_t*>(p.sf + off) = word;
                }
            }
            // packed bytes: each lane of the pair writes 16 contiguous bytes per 8-word half
            const int valid_words = valid / 8;
            uint8_t* dst = p.packed + row * (p.K / 2) + e0 / 2;
            const bool al16 = ((row * (p.K / 2)) & 15) == 0;
#pragma unroll
            for (int hh = 0; hh < NCT / 4; ++hh) {
                const uint32_t c0 = codes[4 * hh], c1 = codes[4 * hh + 1];
                const uint32_t c2 = codes[4 * hh + 2], c3 = codes[4 * hh + 3];
                const uint32_t r0 = __shfl_xor_sync(kFull, h ? c0 : c2, 1);
                const uint32_t r1 = __shfl_xor_sync(kFull, h ? c1 : c3, 1);
                const uint4 out = h ? make_uint4(r0, c2, r1, c3) : make_uint4(c0, r0, c1, r1);
                const int wb = 8 * hh + 4 * h;
                uint32_t* d = reinterpret_cast<uint32_t*>(dst + wb * 4);
                if (data_row) {
                    if (wb + 4 <= valid_words) {
                        if (al16) {
                            *reinterpret_cast<uint4*>(d) = out;
                        } else {
                            reinterpret_cast<uint2*>(d)[0] = make_uint2(out.x, out.y);
                            reinterpret_cast<uint2*>(d)[1] = make_uint2(out.z, out.w);
                        }
                    } else {
                        const uint32_t o[4] = {out.x, out.y, out.z, out.w};
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            if (wb + j < valid_words) d[j] = o[j];
                    }
                }
            }
        }
    }
    if constexpr (MODE == 0) {
        const float m = block_max(tmax, red);
        if (threadIdx.x == 0) p.partials_out[blockIdx.x] = m;
    }
}

template <int G, int MODE>
nvfp4_status launch_unit(const UnitParams& p, int grid, cudaStream_t stream) {
    unit_kernel<G, MODE><<<grid, kThreads, 0, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

template <int MODE>
nvfp4_status dispatch(int g, const UnitParams& p, int grid, cudaStream_t stream) {
    switch (g) {
        case 0: if constexpr (MODE != 2) return launch_unit<0, MODE>(p, grid, stream); break;
        case 16: return launch_unit<16, MODE>(p, grid, stream);
        case 32: return launch_unit<32, MODE>(p, grid, stream);
        case 64: return launch_unit<64, MODE>(p, grid, stream);
        case 128: return launch_unit<128, MODE>(p, grid, stream);
        default: break;
    }
    return NVFP4_ERR_INVALID_ARG;
}

int64_t unit_elems(int g) { return g == 128 ? 128 : 64; }

int grid_for(int64_t units, int sms) {
    const int64_t need = (units + kUnitsPerCta - 1) / kUnitsPerCta;
    const int64_t cap = (int64_t)sms * 8;   // 8 resident CTAs of 256 threads per SM
    return (int)(need < cap ? (need > 0 ? need : 1) : cap);
}

}  // namespace

float hadamard_scale(int g) { return (float)(1.0 / sqrt((double)g)); }

nvfp4_status launch_quantize(const void* x, int64_t rows, int64_t K, int group,
                             const float* gsf_in, float* gsf_out, uint8_t* packed, uint8_t* sf,
                             float* partials, const float* gsf_w, float* alpha_out,
                             cudaStream_t stream) {
    DeviceInfo dev;
    nvfp4_status st = device_info(&dev);
    if (st != NVFP4_OK) return st;

    UnitParams p{};
    p.x = static_cast<const uint16_t*>(x);
    p.rows = rows;
    p.K = K;
    p.upr = (K + unit_elems(group) - 1) / unit_elems(group);
    p.hscale = group ? hadamard_scale(group) : 1.0f;
    p.packed = packed;
    p.sf = sf;
    p.cgroups = (K + 63) / 64;
    p.gsf_in = gsf_in;
    p.gsf_out = gsf_out;
    p.gsf_w = gsf_w;
    p.alpha_out = alpha_out;

    if (gsf_in == nullptr) {
        UnitParams a = p;
        a.total_units = rows * p.upr;
        int n = grid_for(a.total_units, dev.sms);
        n = n < dev.sms * 4 ? n : dev.sms * 4;
        n = n < kMaxPartials ? n : kMaxPartials;
        a.partials_out = partials;
        st = dispatch<0>(group, a, n, stream);
        if (st != NVFP4_OK) return st;
        p.partials = partials;
        p.n_partials = n;
    }
    const int64_t rows_padded = (rows + 127) / 128 * 128;
    p.total_units = rows_padded * p.upr;
    return dispatch<1>(group, p, grid_for(p.total_units, dev.sms), stream);
}

nvfp4_status launch_rotate(const void* x, void* y, int64_t rows, int64_t K, int group,
                           cudaStream_t stream) {
    DeviceInfo dev;
    nvfp4_status st = device_info(&dev);
    if (st != NVFP4_OK) return st;
    UnitParams p{};
    p.x = static_cast<const uint16_t*>(x);
    p.y = static_cast<uint16_t*>(y);
    p.rows = rows;
    p.K = K;
    p.upr = (K + unit_elems(group) - 1) / unit_elems(group);
    p.total_units = rows * p.upr;
    p.hscale = hadamard_scale(group);
    return dispatch<2>(group, p, grid_for(p.total_units, dev.sms), stream);
}

}  // namespace nvfp4
