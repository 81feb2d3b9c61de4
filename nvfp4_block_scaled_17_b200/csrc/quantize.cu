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
#include <atomic>
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


// Packed fp32 pairs (sm_100 FADD2/FMUL2): each lane of the pair is an IEEE binary32
// operation rounded to nearest even, exactly like its scalar form.
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
// a - b as one fused op: b * (-1) is exact, so the single rounding equals rn(a - b)
// (signed zeros included).
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
    return __ffma2_rn(b, make_float2(-1.0f, -1.0f), a);
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 word_to_f2(uint32_t w) { return make_float2(bf16lo(w), bf16hi(w)); }

// One butterfly on two packed pairs: (a, b) -> (a + b, a - b) lane-wise.
__device__ __forceinline__ void bfly2(float2& a, float2& b) {
    const float2 s = add2(a, b);
    const float2 d = sub2(a, b);
    a = s;
    b = d;
}

// rn(lo + hi) and rn(lo - hi) of one bf16 pair, with hi widened to fp32 and lo used
// as a bf16 operand of the mixed-precision add and subtract (exact widening, one
// rounding each, so both equal the plain fp32 results, signed zeros included).
__device__ __forceinline__ float2 pair_sum_diff(uint32_t w) {
    const float hi = bf16hi(w);
    const uint16_t lo = (uint16_t)(w & 0xffffu);
    float s, d;
    asm("add.rn.f32.bf16 %0, %1, %2;" : "=f"(s) : "h"(lo), "f"(hi));
    asm("sub.rn.f32.bf16 %0, %1, %2;" : "=f"(d) : "h"(lo), "f"(hi));
    return make_float2(s, d);
}

// The butterfly stages of a unit's g-groups in fp32, up to but not including the
// in-lane stage that is LOCAL_END local chunks apart (G / 16: every stage).  Values are
// held as pairs (2k, 2k+1) of a chunk, so the h = 1 stage works inside a pair and all
// later stages on whole pairs.
template <int G, int LOCAL_END>
__device__ __forceinline__ void butterfly(const uint4 (&w)[UnitShape<G>::NCT], int h,
                                          float2 (&v)[UnitShape<G>::NCT][4]) {
    constexpr int NCT = UnitShape<G>::NCT;
#pragma unroll
    for (int i = 0; i < NCT; ++i) {
        // h = 1: inside each pair, straight from the bf16 words
        v[i][0] = pair_sum_diff(w[i].x);
        v[i][1] = pair_sum_diff(w[i].y);
        v[i][2] = pair_sum_diff(w[i].z);
        v[i][3] = pair_sum_diff(w[i].w);
        // h = 2, 4: pairs one and two apart
        bfly2(v[i][0], v[i][1]);
        bfly2(v[i][2], v[i][3]);
        bfly2(v[i][0], v[i][2]);
        bfly2(v[i][1], v[i][3]);
    }
    // h = 8: chunk 2i (lane h = 0) with chunk 2i + 1 (lane h = 1); the lower lane keeps
    // v + o, the upper lane o - v, both as o + v * (+-1) with one rounding
    const float sg = h ? -1.0f : 1.0f;
    const float2 sgn = make_float2(sg, sg);
#pragma unroll
    for (int i = 0; i < NCT; ++i)
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 o = make_float2(__shfl_xor_sync(kFull, v[i][k].x, 1),
                                         __shfl_xor_sync(kFull, v[i][k].y, 1));
            v[i][k] = __ffma2_rn(v[i][k], sgn, o);
        }
    // h = 16, 32, 64: chunks two, four, eight apart = local chunks 1, 2, 4 apart
#pragma unroll
    for (int s = 1; s < LOCAL_END; s *= 2)
#pragma unroll
        for (int i = 0; i < NCT; ++i)
            if ((i & s) == 0)
#pragma unroll
                for (int k = 0; k < 4; ++k) bfly2(v[i][k], v[i + s][k]);
}

// Rotates every g-group of the unit in place (the values stay bf16 words): the whole
// butterfly, the 1/sqrt(g) scale and the rounding to bf16.
template <int G>
__device__ __forceinline__ void rotate_unit(uint4 (&w)[UnitShape<G>::NCT], int h, float hscale) {
    constexpr int NCT = UnitShape<G>::NCT;
    float2 v[NCT][4];
    butterfly<G, G / 16>(w, h, v);
    const float2 hs = make_float2(hscale, hscale);
#pragma unroll
    for (int i = 0; i < NCT; ++i) {
        float2 g[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) g[k] = mul2(v[i][k], hs);
        w[i] = make_uint4(bf16x2_rn(g[0].x, g[0].y), bf16x2_rn(g[1].x, g[1].y),
                          bf16x2_rn(g[2].x, g[2].y), bf16x2_rn(g[3].x, g[3].y));
    }
}

__device__ __forceinline__ float max3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Running maximum of |v| over the unit's rotated values before the 1/sqrt(g) scale and
// the bf16 rounding (G >= 32, where the last stage is in-lane).  The last stage maps
// (a, b) to rn(a + b) and rn(a - b); one of |a + b|, |a - b| is |a| + |b| exactly and
// rounding is monotone and odd, so the larger magnitude of the two outputs is
// rn(|a| + |b|).  The rotated bf16 value is bf16(rn(v * hscale)), also monotone in |v|,
// so the bf16 amax of the unit is bf16(rn(m * hscale)) of this maximum m.
template <int G>
__device__ __forceinline__ float rotate_amax(const uint4 (&w)[UnitShape<G>::NCT], int h, float m) {
    static_assert(G >= 32, "the last stage must be in-lane");
    constexpr int NCT = UnitShape<G>::NCT;
    constexpr int S = G / 32;
    float2 v[NCT][4];
    butterfly<G, S>(w, h, v);
#pragma unroll
    for (int i = 0; i < NCT; ++i)
        if ((i & S) == 0)
#pragma unroll
            for (int k = 0; k < 4; ++k)
                m = max3(m, __fadd_rn(fabsf(v[i][k].x), fabsf(v[i + S][k].x)),
                         __fadd_rn(fabsf(v[i][k].y), fabsf(v[i + S][k].y)));
    return m;
}

// bf16(rn(m * hscale)) as fp32: the amax of the rotated bf16 values (see rotate_amax).
__device__ __forceinline__ float rotated_amax_bf16(float m, float hscale) {
    return bf16lo(bf16x2_rn(__fmul_rn(m, hscale), 0.0f));
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

// Encode-pass prologue of every CTA: the global scale (given, or reduced from the
// amax partials: FP4_E4M3_RANGE / max(amax, floor)), alpha and gsf written once by
// block 0, and the table rn(gsf / dec(s)) for every non-negative E4M3 scale byte
// (0 and NaN map to 0).  Ends with a block barrier.
template <int THREADS>
__device__ __forceinline__ float encode_prologue(const UnitParams& p, float* red, float* s_gsf,
                                                 float* inv_tab) {
    float gsf;
    if (p.gsf_in != nullptr) {
        gsf = *p.gsf_in;
    } else {
        float m = 0.0f;
        for (int i = threadIdx.x; i < p.n_partials; i += THREADS) m = fmaxf(m, p.partials[i]);
        m = block_max(m, red);
        if (threadIdx.x == 0) *s_gsf = __fdiv_rn(kFp4E4m3Range, fmaxf(m, kAmaxFloor));
        __syncthreads();
        gsf = *s_gsf;
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        if (p.gsf_out) *p.gsf_out = gsf;
        if (p.alpha_out) *p.alpha_out = __fdiv_rn(1.0f, __fmul_rn(gsf, *p.gsf_w));
    }
    if (threadIdx.x < 128) {
        const float sv = f32_from_e4m3(threadIdx.x);
        inv_tab[threadIdx.x] = (threadIdx.x == 0 || threadIdx.x == 127) ? 0.0f : __fdiv_rn(gsf, sv);
    }
    __syncthreads();
    return gsf;
}

// Encode pass of one unit: block maxima, E4M3 scales, E2M1 codes; writes the
// packed bytes (rows < p.rows only) and the scale words of the 128x4 layout.
template <int G>
__device__ __forceinline__ void encode_unit(const uint4 (&w)[UnitShape<G>::NCT], int h, float gsf,
                                            const float* inv_tab, const UnitParams& p,
                                            int64_t row, int64_t e0, int valid, bool data_row,
                                            bool active) {
    constexpr int NCT = UnitShape<G>::NCT;
    // block i of the unit = chunks 2i (lane h = 0) and 2i + 1 (lane h = 1).  Each
    // lane derives the scale of the blocks i with (i & 1) == h; the pair swaps them.
    float bm[NCT];
#pragma unroll
    for (int i = 0; i < NCT; ++i) {
        const uint32_t tm = absmax_word4(w[i]);
        bm[i] = absmax_of_pair(absmax2_bf16(tm, __shfl_xor_sync(kFull, tm, 1)));
    }
    uint32_t s8[NCT];
#pragma unroll
    for (int j = 0; j < NCT / 2; ++j) {
        const float mine_bm = h ? bm[2 * j + 1] : bm[2 * j];
        const uint32_t mine = e4m3_scale_of_scaled_max(__fmul_rn(gsf, mine_bm));
        const uint32_t other = __shfl_xor_sync(kFull, mine, 1);
        s8[2 * j] = h ? other : mine;
        s8[2 * j + 1] = h ? mine : other;
    }
    uint32_t codes[NCT];
#pragma unroll
    for (int i = 0; i < NCT; ++i) {
        // inv_tab[s8] = rn(gsf / dec(s8)); a zero scale zeroes the whole block
        const float inv = inv_tab[s8[i]];
        const float2 iv = make_float2(inv, inv);
        const float2 a = mul2(word_to_f2(w[i].x), iv), b = mul2(word_to_f2(w[i].y), iv);
        const float2 c = mul2(word_to_f2(w[i].z), iv), d = mul2(word_to_f2(w[i].w), iv);
        const float q[8] = {a.x, a.y, b.x, b.y, c.x, c.y, d.x, d.y};
        codes[i] = s8[i] ? e2m1x8_from_f32(q) : 0u;
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

// MODE 0: amax partials.  MODE 1: quantize.  MODE 2: rotate only (G > 0).
template <int G, int MODE>
__global__ void __launch_bounds__(kThreads) unit_kernel(const UnitParams p) {
    constexpr int E = UnitShape<G>::E;
    constexpr int NCT = UnitShape<G>::NCT;
    __shared__ float red[32];
    __shared__ float s_gsf;
    __shared__ float inv_tab[128];

    const int lane = threadIdx.x & 31;
    const int h = lane & 1;
    const int64_t warp_id = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
    const int64_t n_warps = (int64_t)gridDim.x * (kThreads / 32);

    float gsf = 0.0f;
    if constexpr (MODE == 1) gsf = encode_prologue<kThreads>(p, red, &s_gsf, inv_tab);
    uint32_t tmax = 0u;       // packed bf16 maxima (G < 32)
    float fmax_rot = 0.0f;    // pre-scale rotated maximum (G >= 32)

    // (row, u) of this lane's unit, advanced by the grid stride without dividing again
    const int64_t stride = n_warps * 16;
    int64_t unit = warp_id * 16 + (lane >> 1);
    int64_t row = unit / p.upr, u = unit - (unit / p.upr) * p.upr;
    const int64_t srow = stride / p.upr, su = stride - srow * p.upr;
    for (int64_t base = warp_id * 16; base < p.total_units; base += stride,
                 unit += stride, row += srow, u += su) {
        if (u >= p.upr) {
            u -= p.upr;
            ++row;
        }
        const bool active = unit < p.total_units;
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
        if constexpr (MODE == 0 && G >= 32) {
            fmax_rot = rotate_amax<G>(w, h, fmax_rot);
            continue;
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
            for (int i = 0; i < NCT; ++i) tmax = absmax2_bf16(tmax, absmax_word4(w[i]));
        } else {
            encode_unit<G>(w, h, gsf, inv_tab, p, row, e0, valid, data_row, active);
        }
    }
    if constexpr (MODE == 0) {
        const float mine = G >= 32 ? rotated_amax_bf16(fmax_rot, p.hscale) : absmax_of_pair(tmax);
        const float m = block_max(mine, red);
        if (threadIdx.x == 0) p.partials_out[blockIdx.x] = m;
    }
}

// ---------------------------------------------------------------------------
// TMA-fed form (K % 64 == 0): the same per-unit arithmetic, with x staged in
// shared memory by the tensor-memory accelerator.
//
// x is viewed as a flat 2-D array of 64-value rows (128 bytes each); an item is
// the 16 units one warp handles (16 or 32 flat rows), loaded as one box with the
// 128-byte swizzle, so the lane-pair reads below hit 8 distinct 16-byte bank
// groups per quarter-warp.  Every warp keeps its own ring of kSlots items and
// issues the load of item k + kSlots as soon as it has read item k into
// registers, so HBM latency overlaps the arithmetic of the items in between.
// One CTA of 16 warps per SM, persistent over the items.
// ---------------------------------------------------------------------------

constexpr int kTmaWarps = 16;
constexpr int kTmaThreads = kTmaWarps * 32;
constexpr int kSlots = 3;
constexpr int kItemRows = 32;                       // flat 64-value rows per item (4 KiB)
constexpr uint64_t kTmaWaitBudgetNs = 2000000000ull;

template <int G>
struct TmaShape {
    static constexpr int E = UnitShape<G>::E;
    static constexpr int SUBS = 128 / E;                // units per lane pair per item
    static constexpr int UPI = 16 * SUBS;               // units per item
    static constexpr int ITEM_BYTES = kItemRows * 128;
    static constexpr int RING_BYTES = kTmaWarps * kSlots * ITEM_BYTES;
    static constexpr int SMEM = 1024 + RING_BYTES + kTmaWarps * kSlots * 8;
};

struct TmaParams {
    uint32_t total_units;   // rows * K / E  (< 2^31)
    uint32_t n_items;
    uint32_t upr;           // units per row
    FastDiv upr_div;
};

// Unit of the item read by lane pair `pair` in sub-step `sub`.  With 128-value units a
// pair reads two flat rows; with 64-value units the order 0,2,4,6 | 1,3,5,7 | 8,10,..
// keeps the four pairs of a quarter-warp on distinct swizzle phases.
template <int E>
__device__ __forceinline__ int item_unit(int pair, int sub) {
    if constexpr (E == 128) return pair;
    return sub * 16 + ((pair & 8) | ((pair & 3) << 1) | ((pair >> 2) & 1));
}

template <int G, int MODE>
__global__ void __launch_bounds__(kTmaThreads, 1)
    tma_unit_kernel(const __grid_constant__ CUtensorMap tmX, const UnitParams p,
                    const TmaParams t, int* status) {
    using S = TmaShape<G>;
    constexpr int E = S::E;
    constexpr int NCT = UnitShape<G>::NCT;
    constexpr int SUBS = S::SUBS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::RING_BYTES);
    __shared__ float red[32];
    __shared__ float s_gsf;
    __shared__ float inv_tab[128];
    __shared__ int s_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = lane & 1;
    if (threadIdx.x == 0) s_abort = 0;
    if (lane == 0)
        for (int s = 0; s < kSlots; ++s) mbar_init(&full[warp * kSlots + s], 1);
    fence_barrier_init();
    __syncthreads();
    griddep_wait();
    griddep_launch_dependents();

    float gsf = 0.0f;
    if constexpr (MODE == 1) {
        gsf = encode_prologue<kTmaThreads>(p, red, &s_gsf, inv_tab);
        // scale bytes of the padding rows (up to the next multiple of 128) are zero
        const int64_t pad_rows = (p.rows + 127) / 128 * 128 - p.rows;
        for (int64_t i = (int64_t)blockIdx.x * kTmaThreads + threadIdx.x; i < pad_rows * p.cgroups;
             i += (int64_t)gridDim.x * kTmaThreads) {
            const int64_t row = p.rows + i / p.cgroups, cg = i % p.cgroups;
            const int64_t off = (((row >> 7) * p.cgroups + cg) << 9) + ((row & 31) << 4) +
                                (((row >> 5) & 3) << 2);
            *reinterpret_cast<uint32_t*>(p.sf + off) = 0u;
        }
    }

    const uint64_t policy = MODE == 0 ? l2_policy_evict_last() : l2_policy_evict_first();
    const uint32_t stride = gridDim.x * kTmaWarps;
    uint8_t* ring = smem + warp * kSlots * S::ITEM_BYTES;
    uint64_t* bars = full + warp * kSlots;
    const uint32_t first = blockIdx.x * kTmaWarps + warp;
    if (lane == 0) {
        for (int s = 0; s < kSlots; ++s) {
            const uint32_t it = first + s * stride;
            if (it < t.n_items) {
                mbar_arrive_expect_tx(&bars[s], S::ITEM_BYTES);
                tma_load_2d_hint(ring + s * S::ITEM_BYTES, &tmX, &bars[s], 0,
                                 (int32_t)(it * kItemRows), policy);
            }
        }
    }

    const int pair = lane >> 1;
    uint32_t tmax = 0u;       // packed bf16 maxima (G < 32)
    float fmax_rot = 0.0f;    // pre-scale rotated maximum (G >= 32)
    uint32_t k = 0;
    for (uint32_t item = first; item < t.n_items; item += stride, ++k) {
        const int s = (int)(k % kSlots);
        if (!mbar_wait_bounded(&bars[s], (k / kSlots) & 1u, &s_abort, status, kTmaWaitBudgetNs))
            break;
        const uint8_t* slot = ring + s * S::ITEM_BYTES;
        uint4 w[SUBS][NCT];
#pragma unroll
        for (int sub = 0; sub < SUBS; ++sub) {
            const int m = item_unit<E>(pair, sub);
#pragma unroll
            for (int i = 0; i < NCT; ++i) {
                const int j = 2 * i + h;                            // chunk of the unit
                const int fr = (E == 128) ? 2 * m + (j >> 3) : m;   // flat row of the item
                const int pos = (j & 7) ^ (fr & 7);
                w[sub][i] = *reinterpret_cast<const uint4*>(slot + fr * 128 + pos * 16);
            }
        }
        __syncwarp();
        if (lane == 0) {
            const uint32_t nxt = item + kSlots * stride;
            if (nxt < t.n_items) {
                fence_proxy_async_smem();
                mbar_arrive_expect_tx(&bars[s], S::ITEM_BYTES);
                tma_load_2d_hint(ring + s * S::ITEM_BYTES, &tmX, &bars[s], 0,
                                 (int32_t)(nxt * kItemRows), policy);
            }
        }
#pragma unroll
        for (int sub = 0; sub < SUBS; ++sub) {
            const uint32_t unit = item * S::UPI + item_unit<E>(pair, sub);
            const bool active = unit < t.total_units;
            const uint32_t row = fast_div(unit, t.upr_div);
            const int64_t e0 = (int64_t)(unit - row * t.upr) * E;
            if constexpr (MODE == 0 && G >= 32) {
                fmax_rot = rotate_amax<G>(w[sub], h, fmax_rot);
            } else if constexpr (MODE == 0) {
                if constexpr (G > 0) rotate_unit<G>(w[sub], h, p.hscale);
#pragma unroll
                for (int i = 0; i < NCT; ++i) tmax = absmax2_bf16(tmax, absmax_word4(w[sub][i]));
            } else {
                if constexpr (G > 0) rotate_unit<G>(w[sub], h, p.hscale);
                encode_unit<G>(w[sub], h, gsf, inv_tab, p, (int64_t)row, e0, E, active, active);
            }
        }
    }
    if constexpr (MODE == 0) {
        const float mine = G >= 32 ? rotated_amax_bf16(fmax_rot, p.hscale) : absmax_of_pair(tmax);
        const float mx = block_max(mine, red);
        if (threadIdx.x == 0) p.partials_out[blockIdx.x] = mx;
    }
    // after a timeout, let this warp's loads still in flight land before the CTA exits
    if (s_abort && lane == 0) {
        volatile int no_abort = 0;
        for (uint32_t s = 0; s < (uint32_t)kSlots; ++s) {
            const uint32_t kk = k + s;
            const uint64_t it = first + (uint64_t)kk * stride;
            if (it < t.n_items)
                mbar_wait_bounded(&bars[kk % kSlots], (kk / kSlots) & 1u, &no_abort, nullptr,
                                  100000000ull);
        }
    }
}

// ---------------------------------------------------------------------------
// Single pass for a dynamic scale when the whole call fits in shared memory at once
// (every warp's items fit its three ring slots; 14.5 M values on 148 SMs -- a 4096 x
// 1024 tile is 4.2 M).  Each warp loads its items once, rotates them in place in shared
// memory while taking the amax, the CTAs meet at a grid barrier (cooperative launch, so
// all of them are resident; the wait is bounded), and every warp then encodes its items
// from shared memory with the global scale: one HBM read and one rotation instead of two.
// The arithmetic is the two-pass kernels' own, so the results are identical.
// ---------------------------------------------------------------------------

template <int G>
__global__ void __launch_bounds__(kTmaThreads, 1)
    single_pass_kernel(const __grid_constant__ CUtensorMap tmX, const UnitParams p,
                       const TmaParams t, float* partials, unsigned int* arrive, int* status) {
    using S = TmaShape<G>;
    constexpr int E = S::E;
    constexpr int NCT = UnitShape<G>::NCT;
    constexpr int SUBS = S::SUBS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::RING_BYTES);
    __shared__ float red[32];
    __shared__ float s_gsf;
    __shared__ float inv_tab[128];
    __shared__ int s_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = lane & 1;
    const int pair = lane >> 1;
    if (threadIdx.x == 0) s_abort = 0;
    if (lane == 0)
        for (int s = 0; s < kSlots; ++s) mbar_init(&full[warp * kSlots + s], 1);
    fence_barrier_init();
    __syncthreads();

    const uint32_t stride = gridDim.x * kTmaWarps;
    const uint32_t first = blockIdx.x * kTmaWarps + warp;
    uint8_t* ring = smem + warp * kSlots * S::ITEM_BYTES;
    uint64_t* bars = full + warp * kSlots;
    if (lane == 0)
        for (int k = 0; k < kSlots; ++k) {
            const uint32_t it = first + k * stride;
            if (it < t.n_items) {
                mbar_arrive_expect_tx(&bars[k], S::ITEM_BYTES);
                tma_load_2d(ring + k * S::ITEM_BYTES, &tmX, &bars[k], 0, (int32_t)(it * kItemRows));
            }
        }

    // the swizzled position of chunk i of sub-unit `sub` of this lane in an item
    auto chunk_ptr = [&](uint8_t* slot, int sub, int i) -> uint4* {
        const int m = item_unit<E>(pair, sub);
        const int j = 2 * i + h;
        const int fr = (E == 128) ? 2 * m + (j >> 3) : m;
        return reinterpret_cast<uint4*>(slot + fr * 128 + (((j & 7) ^ (fr & 7)) << 4));
    };

    // pass over the own items: rotate in place, amax of the rotated values
    uint32_t tmax = 0u;
    bool ok = true;
    for (int k = 0; k < kSlots; ++k) {
        const uint32_t item = first + k * stride;
        if (item >= t.n_items) break;
        if (!mbar_wait_bounded(&bars[k], 0u, &s_abort, status, kTmaWaitBudgetNs)) {
            ok = false;
            break;
        }
        uint8_t* slot = ring + k * S::ITEM_BYTES;
#pragma unroll
        for (int sub = 0; sub < SUBS; ++sub) {
            uint4 w[NCT];
#pragma unroll
            for (int i = 0; i < NCT; ++i) w[i] = *chunk_ptr(slot, sub, i);
            if constexpr (G > 0) {
                rotate_unit<G>(w, h, p.hscale);
#pragma unroll
                for (int i = 0; i < NCT; ++i) *chunk_ptr(slot, sub, i) = w[i];
            }
            // units past the end hold the zeros the copy filled in: they add nothing
#pragma unroll
            for (int i = 0; i < NCT; ++i) tmax = absmax2_bf16(tmax, absmax_word4(w[i]));
        }
    }
    if (!ok) {
        // let this warp's other loads land before the CTA can leave
        if (lane == 0) {
            volatile int no_abort = 0;
            for (int k = 0; k < kSlots; ++k)
                if (first + k * stride < t.n_items)
                    mbar_wait_bounded(&bars[k], 0u, &no_abort, nullptr, 100000000ull);
        }
    }

    // grid-wide amax: per-CTA partials, then a bounded barrier on the arrival count
    const float m = block_max(absmax_of_pair(tmax), red);
    if (threadIdx.x == 0) {
        partials[blockIdx.x] = m;
        __threadfence();
        atomicAdd(arrive, 1u);
        const uint64_t t0 = globaltimer_ns();
        while (atomicAdd(arrive, 0u) < gridDim.x) {
            if (s_abort || globaltimer_ns() - t0 > kTmaWaitBudgetNs) {
                record_status(status, NVFP4_ERR_TIMEOUT);
                s_abort = 1;
                break;
            }
        }
        __threadfence();
    }
    __syncthreads();
    if (s_abort) return;

    // the global scale from every CTA's partial (read past L1), then the encode table
    float mm = 0.0f;
    for (int i = threadIdx.x; i < (int)gridDim.x; i += kTmaThreads) mm = fmaxf(mm, __ldcg(partials + i));
    mm = block_max(mm, red);
    if (threadIdx.x == 0) s_gsf = __fdiv_rn(kFp4E4m3Range, fmaxf(mm, kAmaxFloor));
    __syncthreads();
    const float gsf = s_gsf;
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        if (p.gsf_out) *p.gsf_out = gsf;
        if (p.alpha_out) *p.alpha_out = __fdiv_rn(1.0f, __fmul_rn(gsf, *p.gsf_w));
    }
    if (threadIdx.x < 128) {
        const float sv = f32_from_e4m3(threadIdx.x);
        inv_tab[threadIdx.x] = (threadIdx.x == 0 || threadIdx.x == 127) ? 0.0f : __fdiv_rn(gsf, sv);
    }
    // scale bytes of the padding rows (up to the next multiple of 128) are zero
    const int64_t pad_rows = (p.rows + 127) / 128 * 128 - p.rows;
    for (int64_t i = (int64_t)blockIdx.x * kTmaThreads + threadIdx.x; i < pad_rows * p.cgroups;
         i += (int64_t)gridDim.x * kTmaThreads) {
        const int64_t row = p.rows + i / p.cgroups, cg = i % p.cgroups;
        const int64_t off = (((row >> 7) * p.cgroups + cg) << 9) + ((row & 31) << 4) +
                            (((row >> 5) & 3) << 2);
        *reinterpret_cast<uint32_t*>(p.sf + off) = 0u;
    }
    __syncthreads();

    // encode the own items from shared memory
    for (int k = 0; k < kSlots; ++k) {
        const uint32_t item = first + k * stride;
        if (item >= t.n_items) break;
        uint8_t* slot = ring + k * S::ITEM_BYTES;
#pragma unroll
        for (int sub = 0; sub < SUBS; ++sub) {
            uint4 w[NCT];
#pragma unroll
            for (int i = 0; i < NCT; ++i) w[i] = *chunk_ptr(slot, sub, i);
            const uint32_t unit = item * S::UPI + item_unit<E>(pair, sub);
            const bool active = unit < t.total_units;
            const uint32_t row = fast_div(unit, t.upr_div);
            const int64_t e0 = (int64_t)(unit - row * t.upr) * E;
            encode_unit<G>(w, h, gsf, inv_tab, p, (int64_t)row, e0, E, active, active);
        }
    }
}

template <int G>
nvfp4_status launch_single_pass(const CUtensorMap& map, const UnitParams& p, const TmaParams& t,
                                int grid, float* partials, int device, int* status,
                                cudaStream_t stream) {
    constexpr int smem = TmaShape<G>::SMEM;
    static std::atomic<int> attr_set[64];
    if (device < 0 || device >= 64) return NVFP4_ERR_DEVICE;
    if (!attr_set[device].load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(single_pass_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 smem) != cudaSuccess)
            return NVFP4_ERR_CUDA;
        attr_set[device].store(1, std::memory_order_release);
    }
    // the arrival counter lives in the last word of the caller's 4 KiB workspace
    unsigned int* arrive = reinterpret_cast<unsigned int*>(partials) + (kMaxPartials - 1);
    if (cudaMemsetAsync(arrive, 0, sizeof(unsigned int), stream) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    const CUtensorMap* mp = &map;
    void* args[] = {const_cast<CUtensorMap*>(mp), const_cast<UnitParams*>(&p),
                    const_cast<TmaParams*>(&t), &partials, &arrive, &status};
    if (cudaLaunchCooperativeKernel(reinterpret_cast<void*>(single_pass_kernel<G>), dim3(grid),
                                    dim3(kTmaThreads), args, smem, stream) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    return NVFP4_OK;
}

nvfp4_status dispatch_single_pass(int g, const CUtensorMap& map, const UnitParams& p,
                                  const TmaParams& t, int grid, float* partials, int device,
                                  int* status, cudaStream_t stream) {
    switch (g) {
        case 0: return launch_single_pass<0>(map, p, t, grid, partials, device, status, stream);
        case 16: return launch_single_pass<16>(map, p, t, grid, partials, device, status, stream);
        case 32: return launch_single_pass<32>(map, p, t, grid, partials, device, status, stream);
        case 64: return launch_single_pass<64>(map, p, t, grid, partials, device, status, stream);
        case 128: return launch_single_pass<128>(map, p, t, grid, partials, device, status, stream);
        default: break;
    }
    return NVFP4_ERR_INVALID_ARG;
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

template <int G, int MODE>
nvfp4_status launch_tma_unit(const CUtensorMap& map, const UnitParams& p, const TmaParams& t,
                             int grid, int device, int* status, cudaStream_t stream) {
    constexpr int smem = TmaShape<G>::SMEM;
    static std::atomic<int> attr_set[64];
    if (device < 0 || device >= 64) return NVFP4_ERR_DEVICE;
    if (!attr_set[device].load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(tma_unit_kernel<G, MODE>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return NVFP4_ERR_CUDA;
        attr_set[device].store(1, std::memory_order_release);
    }
    if (launch_pdl(tma_unit_kernel<G, MODE>, (unsigned)grid, kTmaThreads, smem, stream, map, p, t,
                   status) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    return NVFP4_OK;
}

template <int MODE>
nvfp4_status dispatch_tma(int g, const CUtensorMap& map, const UnitParams& p, const TmaParams& t,
                          int grid, int device, int* status, cudaStream_t stream) {
    switch (g) {
        case 0: return launch_tma_unit<0, MODE>(map, p, t, grid, device, status, stream);
        case 16: return launch_tma_unit<16, MODE>(map, p, t, grid, device, status, stream);
        case 32: return launch_tma_unit<32, MODE>(map, p, t, grid, device, status, stream);
        case 64: return launch_tma_unit<64, MODE>(map, p, t, grid, device, status, stream);
        case 128: return launch_tma_unit<128, MODE>(map, p, t, grid, device, status, stream);
        default: break;
    }
    return NVFP4_ERR_INVALID_ARG;
}

// x as [rows*K/64, 64] bf16 with a [BR, 64] box and the 128-byte swizzle.
bool make_flat_map(CUtensorMap* map, const void* x, int64_t flat_rows, int box_rows) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {64, (cuuint64_t)flat_rows};
    cuuint64_t strides[1] = {128};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void*>(x), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
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

    const int64_t flat_rows = rows * K / 64;
    if (K % 64 == 0 && flat_rows < (int64_t(1) << 31) - 256) {
        int* status = nullptr;
        if ((st = status_word(&status)) != NVFP4_OK) return st;
        CUtensorMap map;
        if (!make_flat_map(&map, x, flat_rows, kItemRows)) return NVFP4_ERR_CUDA;
        const int upi = group == 128 ? 16 : 32;
        p.total_units = rows * p.upr;
        TmaParams t;
        t.total_units = (uint32_t)p.total_units;
        t.n_items = (uint32_t)((p.total_units + upi - 1) / upi);
        t.upr = (uint32_t)p.upr;
        t.upr_div = make_fastdiv(t.upr);
        // dynamic scale that fits on chip: one pass, every warp holding at most kSlots items
        const int64_t per_cta = (int64_t)kTmaWarps * kSlots;
        if (gsf_in == nullptr && (int64_t)t.n_items <= (int64_t)dev.sms * per_cta) {
            // as many CTAs as give every warp one item, up to one per SM
            const int64_t g1 = ((int64_t)t.n_items + kTmaWarps - 1) / kTmaWarps;
            return dispatch_single_pass(group, map, p, t, (int)(g1 < dev.sms ? (g1 > 0 ? g1 : 1) : dev.sms),
                                        partials, dev.device, status, stream);
        }
        const int64_t need = (t.n_items + kTmaWarps - 1) / kTmaWarps;
        const int grid = (int)(need < dev.sms ? (need > 0 ? need : 1) : dev.sms);
        if (gsf_in == nullptr) {
            UnitParams a = p;
            a.partials_out = partials;
            st = dispatch_tma<0>(group, map, a, t, grid, dev.device, status, stream);
            if (st != NVFP4_OK) return st;
            p.partials = partials;
            p.n_partials = grid;
        }
        return dispatch_tma<1>(group, map, p, t, grid, dev.device, status, stream);
    }

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
