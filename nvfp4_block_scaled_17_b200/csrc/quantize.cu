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
// Two work decompositions.
//   * Rows made of whole 128-value units (K % 128 == 0, every workload here): one
//     thread owns a unit, loaded through the tensor-memory accelerator, and keeps the
//     whole butterfly, the block maxima and the encoding in its registers (row_kernel,
//     row_single_kernel below).
//   * Any other K % 16 == 0 (unit_kernel): a unit is E consecutive values of one row (E
//     = 64, or 128 for a 128-wide rotation), handled by a pair of adjacent lanes: lane h
//     of the pair owns the 8-value chunks 2i+h of the unit, so every load instruction of
//     a warp reads 16 whole 32-byte sectors and each 16-value block lies half in each
//     lane.  With that split the only cross-lane step of the butterfly is the h = 8 stage
//     (one shuffle per value); stages 1, 2, 4 stay inside a chunk and 16, 32, 64 inside a
//     lane.  Block maxima need one shuffle per block; the scale bytes of four blocks form
//     one aligned 32-bit word of the 128x4 layout.
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
        for (int i = threadIdx.x; i < p.n_partials; i += THREADS) m = fmaxf(m, __ldcg(p.partials + i));
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

// Plain-load form for any K % 16 == 0 (the calls whose rows are not whole 128-value
// units).  MODE 0: amax partials.  MODE 1: quantize.  MODE 2: rotate only (G > 0).
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
// Row-unit form (K % 128 == 0): one thread owns a unit of 128 consecutive values of a
// row, so the whole 128-wide butterfly, the block maxima and the encoding stay in its
// registers: no shuffles and no lane-pair exchanges.
//
// x is read as units (256 bytes each) through two tensor maps over the same memory with
// a 256-byte row stride: one for the first 64 values of every unit, one (based 128 bytes
// further) for the second 64.  An item is 32 consecutive units, one per lane: one 4 KiB
// box from each map, 128-byte swizzle, so lane t reads row t of each box and the eight
// lanes of a quarter-warp hit eight distinct 16-byte bank groups.  Every warp keeps its
// own ring of kRSlots items and issues the load of its piece r + kRSlots as soon as its
// lanes have read piece r into registers.  One CTA of kRWarps warps per SM, persistent.
// These kernels run the single pass of small dynamic calls for every g and the two
// streaming passes for g = 128; the streaming passes of g <= 64 use the half-unit form.
// ---------------------------------------------------------------------------

constexpr int kRWarps = 12;
constexpr int kRThreads = kRWarps * 32;
constexpr int kRSlots = 2;
constexpr int kRHalfBytes = 32 * 128;              // one 64-value half of 32 units
constexpr int kRItemBytes = 2 * kRHalfBytes;       // 8 KiB: 32 units
constexpr int kRRingBytes = kRWarps * kRSlots * kRItemBytes;
constexpr int kRSmem = 1024 + kRRingBytes + kRWarps * kRSlots * 8;
constexpr uint64_t kTmaWaitBudgetNs = 2000000000ull;
static_assert(kRSmem <= 232448, "dynamic shared memory above the 227 KiB a CTA can have");

struct RowParams {
    uint32_t total_units;   // rows * K / 128  (< 2^31)
    uint32_t n_items;       // items of the pass (32 units each; 16 in the half-unit form)
    uint32_t upr;           // units per row, K / 128
    FastDiv upr_div;
    uint32_t reverse;       // 1: visit the items last to first
};

// The streaming passes hand item j to warp slot j % W (W warps in the grid), and slot q is
// warp q / gridDim.x of CTA q % gridDim.x: the items of a last, partial round spread over
// all CTAs first, so every SM gets the same number of items to within one.
__device__ __forceinline__ uint32_t warp_slot(int warp) {
    return (uint32_t)warp * gridDim.x + blockIdx.x;
}

// fp32 bit pattern of bf16(a) (round to nearest even): a goes to the upper half of the
// packed pair, +0 to the lower half.
__device__ __forceinline__ float bf16_round(float a) {
    uint32_t d;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(a), "f"(0.0f));
    return __uint_as_float(d);
}

// Two fp32 values that are bf16-exact back into one bf16 pair (lo in bits 0..15).
__device__ __forceinline__ uint32_t pack_bf16_pair(float lo, float hi) {
    return __byte_perm(__float_as_uint(lo), __float_as_uint(hi), 0x7632);
}

// Byte address of chunk c (8 values) of lane `lane`'s unit in an item slot.
__device__ __forceinline__ uint32_t unit_chunk_off(int lane, int c) {
    return (uint32_t)((c >> 3) * kRHalfBytes + lane * 128 + (((c & 7) ^ (lane & 7)) << 4));
}

__device__ __forceinline__ void load_unit(const uint8_t* slot, int lane, uint4 (&w)[16]) {
#pragma unroll
    for (int c = 0; c < 16; ++c) w[c] = *reinterpret_cast<const uint4*>(slot + unit_chunk_off(lane, c));
}

// The butterfly stages h = 1, 2, 4, ... < STOP of every G-group of the unit in fp32.  The
// values are held as pairs (2i, 2i + 1): stage 1 works inside each bf16 pair, straight
// from the words; stage h >= 2 on pairs h / 2 apart (the pair index bit h / 2 clear keeps
// both partners in one aligned group of 2h <= G values).
template <int STOP>
__device__ __forceinline__ void unit_butterfly(const uint4 (&w)[16], float2 (&v)[64]) {
#pragma unroll
    for (int c = 0; c < 16; ++c) {
        v[4 * c] = pair_sum_diff(w[c].x);
        v[4 * c + 1] = pair_sum_diff(w[c].y);
        v[4 * c + 2] = pair_sum_diff(w[c].z);
        v[4 * c + 3] = pair_sum_diff(w[c].w);
    }
#pragma unroll
    for (int h = 2; h < STOP; h *= 2)
#pragma unroll
        for (int i = 0; i < 64; ++i)
            if ((i & (h / 2)) == 0) bfly2(v[i], v[i + h / 2]);
}

// The unit's values as fp32: rotated (every G-group times H / sqrt(G), rounded to bf16)
// or, for G = 0, the bf16 input itself.
template <int G>
__device__ __forceinline__ void unit_values(const uint4 (&w)[16], float hscale, float (&r)[128]) {
    if constexpr (G == 0) {
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            const uint32_t q[4] = {w[c].x, w[c].y, w[c].z, w[c].w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                r[8 * c + 2 * k] = bf16lo(q[k]);
                r[8 * c + 2 * k + 1] = bf16hi(q[k]);
            }
        }
    } else {
        float2 v[64];
        unit_butterfly<G>(w, v);
        const float2 hs = make_float2(hscale, hscale);
#pragma unroll
        for (int i = 0; i < 64; ++i) {
            const float2 g = mul2(v[i], hs);
            r[2 * i] = bf16_round(g.x);
            r[2 * i + 1] = bf16_round(g.y);
        }
    }
}

// Running maximum for the amax pass.  G = 0: the bf16 maxima of the words (packed).
// G > 0: the butterfly up to its last stage, then max(|a| + |b|) over the last stage's
// pairs -- one of rn(a + b), rn(a - b) has magnitude rn(|a| + |b|) and rounding is
// monotone, so this is the largest pre-scale magnitude of the rotated values; the
// rotated bf16 amax is bf16(rn(m * hscale)) of it (rotated_amax_bf16).
template <int G>
__device__ __forceinline__ void unit_amax(const uint4 (&w)[16], uint32_t& tmax, float& fmax_) {
    if constexpr (G == 0) {
#pragma unroll
        for (int c = 0; c < 16; ++c) tmax = absmax2_bf16(tmax, absmax_word4(w[c]));
    } else {
        float2 v[64];
        unit_butterfly<G / 2>(w, v);
        constexpr int S = G / 4;   // pair distance of the last stage
#pragma unroll
        for (int i = 0; i < 64; ++i)
            if ((i & S) == 0)
                fmax_ = max3(fmax_, __fadd_rn(fabsf(v[i].x), fabsf(v[i + S].x)),
                             __fadd_rn(fabsf(v[i].y), fabsf(v[i + S].y)));
    }
}

// E4M3 block-scale bytes of two blocks from their scaled maxima y0, y1 >= 0 (or NaN):
// e4m3_scale_of_scaled_max on each, converted in one instruction; y0's byte is the low one.
__device__ __forceinline__ uint32_t e4m3_scales2(float y0, float y1) {
    const float r = __uint_as_float(0x3e2aaaabu);   // rn(1/6)
    y0 = (y0 > 6000.0f) ? 6000.0f : y0;
    y1 = (y1 > 6000.0f) ? 6000.0f : y1;
    const float q0 = __fmul_rn(y0, r), q1 = __fmul_rn(y1, r);
    const float a0 = __fmaf_rn(__fmaf_rn(-q0, 6.0f, y0), r, q0);
    const float a1 = __fmaf_rn(__fmaf_rn(-q1, 6.0f, y1), r, q1);
    uint16_t d;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(a1), "f"(a0));
    return d;
}

// max |r[k]| over one 16-value block
__device__ __forceinline__ float block_absmax16(const float* r) {
    float m = max3(fabsf(r[0]), fabsf(r[1]), fabsf(r[2]));
#pragma unroll
    for (int k = 3; k < 15; k += 2) m = max3(m, fabsf(r[k]), fabsf(r[k + 1]));
    return fmaxf(m, fabsf(r[15]));
}

// Encode one unit (values r, bf16-exact): per 16-value block bmax, the E4M3 scale of
// rn(gsf * bmax) / 6, codes E2M1(rn(x * rn(gsf / scale))), all codes 0 under a zero
// scale; 64 bytes of packed codes and two scale words of the 128x4 layout.
__device__ __forceinline__ void encode_unit128(const float (&r)[128], float gsf,
                                               const float* inv_tab, const UnitParams& p,
                                               int64_t row, int64_t e0) {
    uint32_t s8[8];
#pragma unroll
    for (int b = 0; b < 8; b += 2) {
        const uint32_t s = e4m3_scales2(__fmul_rn(gsf, block_absmax16(r + 16 * b)),
                                        __fmul_rn(gsf, block_absmax16(r + 16 * b + 16)));
        s8[b] = s & 0xffu;
        s8[b + 1] = s >> 8;
    }
    uint32_t codes[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) {
        const float inv = inv_tab[s8[c >> 1]];   // rn(gsf / dec(s8)); 0 for a zero scale
        const float2 iv = make_float2(inv, inv);
        const float* x = r + 8 * c;
        const float2 a = mul2(make_float2(x[0], x[1]), iv), b = mul2(make_float2(x[2], x[3]), iv);
        const float2 cc = mul2(make_float2(x[4], x[5]), iv), d = mul2(make_float2(x[6], x[7]), iv);
        const float q[8] = {a.x, a.y, b.x, b.y, cc.x, cc.y, d.x, d.y};
        codes[c] = s8[c >> 1] ? e2m1x8_from_f32(q) : 0u;
    }
    uint4* dst = reinterpret_cast<uint4*>(p.packed + row * (p.K / 2) + e0 / 2);
#pragma unroll
    for (int k = 0; k < 4; ++k)
        dst[k] = make_uint4(codes[4 * k], codes[4 * k + 1], codes[4 * k + 2], codes[4 * k + 3]);
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        const int64_t cg = e0 / 64 + q;
        const int64_t off = (((row >> 7) * p.cgroups + cg) << 9) + ((row & 31) << 4) +
                            (((row >> 5) & 3) << 2);
        *reinterpret_cast<uint32_t*>(p.sf + off) = s8[4 * q] | (s8[4 * q + 1] << 8) |
                                                   (s8[4 * q + 2] << 16) | (s8[4 * q + 3] << 24);
    }
}

// Scale bytes of the padding rows (rows .. up to the next multiple of 128) are zero.
template <int THREADS>
__device__ __forceinline__ void zero_padding_scales(const UnitParams& p) {
    const int64_t pad_rows = (p.rows + 127) / 128 * 128 - p.rows;
    for (int64_t i = (int64_t)blockIdx.x * THREADS + threadIdx.x; i < pad_rows * p.cgroups;
         i += (int64_t)gridDim.x * THREADS) {
        const int64_t row = p.rows + i / p.cgroups, cg = i % p.cgroups;
        const int64_t off = (((row >> 7) * p.cgroups + cg) << 9) + ((row & 31) << 4) +
                            (((row >> 5) & 3) << 2);
        *reinterpret_cast<uint32_t*>(p.sf + off) = 0u;
    }
}

// The 32 units from `base` (rows past the end of x arrive as zeros).
__device__ __forceinline__ void load_units(uint8_t* slot, const CUtensorMap* tmE,
                                           const CUtensorMap* tmO, uint64_t* bar, uint32_t base,
                                           uint64_t policy) {
    mbar_arrive_expect_tx(bar, kRItemBytes);
    tma_load_2d_hint(slot, tmE, bar, 0, (int32_t)base, policy);
    tma_load_2d_hint(slot + kRHalfBytes, tmO, bar, 0, (int32_t)base, policy);
}

__device__ __forceinline__ void load_item(uint8_t* slot, const CUtensorMap* tmE,
                                          const CUtensorMap* tmO, uint64_t* bar, uint32_t item,
                                          uint64_t policy) {
    load_units(slot, tmE, tmO, bar, item * 32, policy);
}

// MODE 0: amax partials (one per CTA).  MODE 1: quantize; after an amax pass it walks the
// pieces last to first, so that it starts on those still in L2.
template <int G, int MODE>
__global__ void __launch_bounds__(kRThreads, 1)
    row_kernel(const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmO,
               const UnitParams p, const RowParams t, int* status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kRRingBytes);
    __shared__ float red[32];
    __shared__ float s_gsf;
    __shared__ float inv_tab[128];
    __shared__ int s_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) s_abort = 0;
    if (lane == 0)
        for (int s = 0; s < kRSlots; ++s) mbar_init(&full[warp * kRSlots + s], 1);
    if (threadIdx.x == 0) {   // the descriptors do not depend on the previous kernel
        prefetch_tensormap(&tmE);
        prefetch_tensormap(&tmO);
    }
    fence_barrier_init();
    __syncthreads();
    griddep_wait();
    griddep_launch_dependents();

    const uint32_t stride = gridDim.x * kRWarps;
    const uint32_t first = warp_slot(warp);
    uint8_t* ring = smem + warp * kRSlots * kRItemBytes;
    uint64_t* bars = full + warp * kRSlots;
    uint32_t k = 0;   // uses of this warp's ring so far; slot k % kRSlots, parity (k / kRSlots) & 1

    // A streaming pass over this warp's items (last to first when `reverse`): prime issues
    // the first kRSlots loads, run waits for each item, reads it into registers, refills
    // the slot and calls body(item, words).
    auto at = [&](bool reverse, uint32_t j) { return reverse ? t.n_items - 1 - j : j; };
    auto prime = [&](bool reverse, uint64_t policy) {
        if (lane == 0)
            for (uint32_t s = 0; s < (uint32_t)kRSlots; ++s) {
                const uint32_t jj = first + s * stride;
                const int slot = (int)((k + s) % kRSlots);
                if (jj < t.n_items)
                    load_item(ring + slot * kRItemBytes, &tmE, &tmO, &bars[slot], at(reverse, jj),
                              policy);
            }
    };
    auto run = [&](bool reverse, uint64_t policy, auto&& body) -> bool {
        for (uint32_t j = first; j < t.n_items; j += stride, ++k) {
            const int s = (int)(k % kRSlots);
            if (!mbar_wait_bounded(&bars[s], (k / kRSlots) & 1u, &s_abort, status, kTmaWaitBudgetNs))
                return false;
            uint8_t* slot = ring + s * kRItemBytes;
            uint4 w[16];
            load_unit(slot, lane, w);
            __syncwarp();
            if (lane == 0) {
                const uint32_t nxt = j + kRSlots * stride;
                if (nxt < t.n_items) {
                    fence_proxy_async_smem();
                    load_item(slot, &tmE, &tmO, &bars[s], at(reverse, nxt), policy);
                }
            }
            body(at(reverse, j), w);
        }
        return true;
    };
    // units past the end were zero-filled by the copy: they add nothing to the amax
    auto amax_body = [&](uint32_t, const uint4 (&w)[16], uint32_t& tmax, float& fmax_rot) {
        unit_amax<G>(w, tmax, fmax_rot);
    };
    auto encode_body = [&](uint32_t item, const uint4 (&w)[16], float gsf) {
        const uint32_t unit = item * 32 + lane;
        if (unit < t.total_units) {
            const uint32_t row = fast_div(unit, t.upr_div);
            float r[128];
            unit_values<G>(w, p.hscale, r);
            encode_unit128(r, gsf, inv_tab, p, (int64_t)row, (int64_t)(unit - row * t.upr) * 128);
        }
    };

    bool ok = true;
    static_assert(MODE == 0 || MODE == 1, "amax or encode");
    if constexpr (MODE == 0) {
        uint32_t tmax = 0u;       // packed bf16 maxima (G = 0)
        float fmax_rot = 0.0f;    // pre-scale rotated maximum (G > 0)
        prime(false, l2_policy_evict_last());
        ok = run(false, l2_policy_evict_last(),
                 [&](uint32_t item, const uint4 (&w)[16]) { amax_body(item, w, tmax, fmax_rot); });
        const float mine = G > 0 ? rotated_amax_bf16(fmax_rot, p.hscale) : absmax_of_pair(tmax);
        const float mx = block_max(mine, red);
        if (threadIdx.x == 0) p.partials_out[blockIdx.x] = mx;
    }
    if constexpr (MODE == 1) {
        // the prologue's loads go out before the pass's first copies, which would delay them
        const float gsf = encode_prologue<kRThreads>(p, red, &s_gsf, inv_tab);
        zero_padding_scales<kRThreads>(p);
        prime(t.reverse, l2_policy_evict_first());
        ok = run(t.reverse, l2_policy_evict_first(),
                 [&](uint32_t item, const uint4 (&w)[16]) { encode_body(item, w, gsf); });
    }
    // after a timeout, let this warp's loads still in flight land before the CTA exits
    if (!ok && lane == 0) {
        volatile int no_abort = 0;
        for (uint32_t s = 0; s < (uint32_t)kRSlots; ++s) {
            const uint32_t kk = k + s;
            mbar_wait_bounded(&bars[kk % kRSlots], (kk / kRSlots) & 1u, &no_abort, nullptr,
                              100000000ull);
        }
    }
}

// ---------------------------------------------------------------------------
// Half-unit form (K % 128 == 0, multi-pass calls, g <= 64): two threads share a 128-value
// unit, each owning 64 consecutive values (one 128-byte half).  Every g-group of g <= 64
// lies inside a half, so the whole butterfly stays in-thread; a thread holds 64 fp32
// values instead of 128 and a CTA runs kHWarps warps instead of kRWarps.  (For g = 128
// the h = 64 stage would pair the two halves: swapping 64 fp32 values per thread through
// shared memory cost more than the extra warps gained, so g = 128 keeps a whole unit per
// thread.)
//
// An item is 16 consecutive units: a [16, 64] box from each half map (128-byte swizzle),
// 4 KiB.  Lane l owns half l >> 4 of unit l & 15, so the eight lanes of a quarter-warp
// read eight rows of one box: eight distinct 16-byte bank groups.
// ---------------------------------------------------------------------------

constexpr int kHWarps = 16;
constexpr int kHThreads = kHWarps * 32;
constexpr int kHSlots = 2;
constexpr int kHBoxBytes = 16 * 128;               // one 64-value half of 16 units
constexpr int kHItemBytes = 2 * kHBoxBytes;        // 4 KiB: 16 units
constexpr int kHRingBytes = kHWarps * kHSlots * kHItemBytes;
constexpr int kHSmem = 1024 + kHRingBytes + kHWarps * kHSlots * 8;
static_assert(kHSmem <= 232448, "dynamic shared memory above the 227 KiB a CTA can have");

// The 16 units from `base` (rows past the end of x arrive as zeros).
__device__ __forceinline__ void load_half_units(uint8_t* slot, const CUtensorMap* tmE,
                                                const CUtensorMap* tmO, uint64_t* bar,
                                                uint32_t base, uint64_t policy) {
    mbar_arrive_expect_tx(bar, kHItemBytes);
    tma_load_2d_hint(slot, tmE, bar, 0, (int32_t)base, policy);
    tma_load_2d_hint(slot + kHBoxBytes, tmO, bar, 0, (int32_t)base, policy);
}

// The eight 8-value chunks of this lane's half-unit.
__device__ __forceinline__ void load_half(const uint8_t* slot, int lane, uint4 (&w)[8]) {
    const int u = lane & 15;
    const uint8_t* base = slot + (lane >> 4) * kHBoxBytes + u * 128;
#pragma unroll
    for (int c = 0; c < 8; ++c)
        w[c] = *reinterpret_cast<const uint4*>(base + ((c ^ (u & 7)) << 4));
}

// Stages h = 1, 2, ... < STOP of the half's butterfly on pairs (2i, 2i + 1).
template <int STOP>
__device__ __forceinline__ void half_butterfly(const uint4 (&w)[8], float2 (&v)[32]) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        v[4 * c] = pair_sum_diff(w[c].x);
        v[4 * c + 1] = pair_sum_diff(w[c].y);
        v[4 * c + 2] = pair_sum_diff(w[c].z);
        v[4 * c + 3] = pair_sum_diff(w[c].w);
    }
#pragma unroll
    for (int h = 2; h < STOP; h *= 2)
#pragma unroll
        for (int i = 0; i < 32; ++i)
            if ((i & (h / 2)) == 0) bfly2(v[i], v[i + h / 2]);
}

// Amax of a half-unit.  G = 0: bf16 maxima of the words.  G > 0: the in-thread butterfly
// up to its last stage, then max(|a| + |b|) over that stage's pairs (see rotate_amax).
template <int G>
__device__ __forceinline__ void half_amax(const uint4 (&w)[8], uint32_t& tmax, float& fmax_) {
    static_assert(G <= 64, "g = 128 groups span both halves of a unit");
    if constexpr (G == 0) {
#pragma unroll
        for (int c = 0; c < 8; ++c) tmax = absmax2_bf16(tmax, absmax_word4(w[c]));
    } else {
        float2 v[32];
        half_butterfly<G / 2>(w, v);
        constexpr int S = G / 4;
#pragma unroll
        for (int i = 0; i < 32; ++i)
            if ((i & S) == 0)
                fmax_ = max3(fmax_, __fadd_rn(fabsf(v[i].x), fabsf(v[i + S].x)),
                             __fadd_rn(fabsf(v[i].y), fabsf(v[i + S].y)));
    }
}

// The half-unit's 64 values as fp32: rotated (every G-group times H / sqrt(G), rounded to
// bf16) or, for G = 0, the bf16 input itself.
template <int G>
__device__ __forceinline__ void half_values(const uint4 (&w)[8], float hscale, float (&r)[64]) {
    static_assert(G <= 64, "g = 128 groups span both halves of a unit");
    if constexpr (G == 0) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const uint32_t q[4] = {w[c].x, w[c].y, w[c].z, w[c].w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                r[8 * c + 2 * k] = bf16lo(q[k]);
                r[8 * c + 2 * k + 1] = bf16hi(q[k]);
            }
        }
    } else {
        float2 v[32];
        half_butterfly<G>(w, v);
        const float2 hs = make_float2(hscale, hscale);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const float2 g = mul2(v[i], hs);
            r[2 * i] = bf16_round(g.x);
            r[2 * i + 1] = bf16_round(g.y);
        }
    }
}

// Encode 64 values (bf16-exact) of one half-unit: four 16-value blocks, 32 bytes of codes
// and the scale word of its 64-value group in the 128x4 layout.
__device__ __forceinline__ void encode_half64(const float (&r)[64], float gsf,
                                              const float* inv_tab, const UnitParams& p,
                                              int64_t row, int64_t e0) {
    uint32_t s8[4];
#pragma unroll
    for (int b = 0; b < 4; b += 2) {
        const uint32_t s = e4m3_scales2(__fmul_rn(gsf, block_absmax16(r + 16 * b)),
                                        __fmul_rn(gsf, block_absmax16(r + 16 * b + 16)));
        s8[b] = s & 0xffu;
        s8[b + 1] = s >> 8;
    }
    uint32_t codes[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const float inv = inv_tab[s8[c >> 1]];   // rn(gsf / dec(s8)); 0 for a zero scale
        const float2 iv = make_float2(inv, inv);
        const float* x = r + 8 * c;
        const float2 a = mul2(make_float2(x[0], x[1]), iv), b = mul2(make_float2(x[2], x[3]), iv);
        const float2 cc = mul2(make_float2(x[4], x[5]), iv), d = mul2(make_float2(x[6], x[7]), iv);
        const float q[8] = {a.x, a.y, b.x, b.y, cc.x, cc.y, d.x, d.y};
        codes[c] = s8[c >> 1] ? e2m1x8_from_f32(q) : 0u;
    }
    uint4* dst = reinterpret_cast<uint4*>(p.packed + row * (p.K / 2) + e0 / 2);
    dst[0] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
    dst[1] = make_uint4(codes[4], codes[5], codes[6], codes[7]);
    const int64_t cg = e0 / 64;
    const int64_t off = (((row >> 7) * p.cgroups + cg) << 9) + ((row & 31) << 4) +
                        (((row >> 5) & 3) << 2);
    *reinterpret_cast<uint32_t*>(p.sf + off) = s8[0] | (s8[1] << 8) | (s8[2] << 16) | (s8[3] << 24);
}

// MODE 0: amax partials (one per CTA).  MODE 1: quantize.  MODE 4: amax phase, bounded grid
// barrier on `arrive` (zeroed before the launch; cooperative launch), encode phase.  The
// RowParams count items of 16 units here.
template <int G, int MODE>
__global__ void __launch_bounds__(kHThreads, 1)
    half_kernel(const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmO,
                const UnitParams p, const RowParams t, unsigned int* arrive, int* status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kHRingBytes);
    __shared__ float red[32];
    __shared__ float s_gsf;
    __shared__ float inv_tab[128];
    __shared__ int s_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) s_abort = 0;
    if (lane == 0)
        for (int s = 0; s < kHSlots; ++s) mbar_init(&full[warp * kHSlots + s], 1);
    if (threadIdx.x == 0) {   // the descriptors do not depend on the previous kernel
        prefetch_tensormap(&tmE);
        prefetch_tensormap(&tmO);
    }
    fence_barrier_init();
    __syncthreads();
    griddep_wait();
    griddep_launch_dependents();

    const uint32_t stride = gridDim.x * kHWarps;
    const uint32_t first = warp_slot(warp);
    uint8_t* ring = smem + warp * kHSlots * kHItemBytes;
    uint64_t* bars = full + warp * kHSlots;
    uint32_t k = 0;   // uses of this warp's ring so far; slot k % kHSlots, parity (k / kHSlots) & 1

    // A streaming pass over this warp's items of 16 units (last to first when `reverse`):
    // prime issues the first kHSlots loads, run waits for each item, reads the lane's
    // half-unit, refills the slot and calls body(item, words).
    auto at = [&](bool reverse, uint32_t j) { return reverse ? t.n_items - 1 - j : j; };
    auto prime = [&](bool reverse, uint64_t policy) {
        if (lane == 0)
            for (uint32_t s = 0; s < (uint32_t)kHSlots; ++s) {
                const uint32_t jj = first + s * stride;
                const int slot = (int)((k + s) % kHSlots);
                if (jj < t.n_items)
                    load_half_units(ring + slot * kHItemBytes, &tmE, &tmO, &bars[slot],
                                    at(reverse, jj) * 16, policy);
            }
    };
    auto run = [&](bool reverse, uint64_t policy, auto&& body) -> bool {
        for (uint32_t j = first; j < t.n_items; j += stride, ++k) {
            const int s = (int)(k % kHSlots);
            if (!mbar_wait_bounded(&bars[s], (k / kHSlots) & 1u, &s_abort, status, kTmaWaitBudgetNs))
                return false;
            uint8_t* slot = ring + s * kHItemBytes;
            uint4 w[8];
            load_half(slot, lane, w);
            __syncwarp();
            if (lane == 0) {
                const uint32_t nxt = j + kHSlots * stride;
                if (nxt < t.n_items) {
                    fence_proxy_async_smem();
                    load_half_units(slot, &tmE, &tmO, &bars[s], at(reverse, nxt) * 16, policy);
                }
            }
            body(at(reverse, j), w);
        }
        return true;
    };
    bool ok = true;
    if constexpr (MODE == 0 || MODE == 4) {
        uint32_t tmax = 0u;       // packed bf16 maxima (G = 0)
        float fmax_rot = 0.0f;    // pre-scale rotated maximum (G > 0)
        // half-units past the end were zero-filled by the copy: they add nothing
        prime(false, l2_policy_evict_last());
        ok = run(false, l2_policy_evict_last(),
                 [&](uint32_t, const uint4 (&w)[8]) { half_amax<G>(w, tmax, fmax_rot); });
        const float mine = G > 0 ? rotated_amax_bf16(fmax_rot, p.hscale) : absmax_of_pair(tmax);
        const float mx = block_max(mine, red);
        if (threadIdx.x == 0) p.partials_out[blockIdx.x] = mx;
    }
    if constexpr (MODE == 4) {
        // the encode phase's first loads go out before the barrier wait
        if (ok) prime(true, l2_policy_evict_first());
        if (threadIdx.x == 0) {
            __threadfence();
            atomicAdd(arrive, 1u);
            const uint64_t t0 = globaltimer_ns();
            while (atomicAdd(arrive, 0u) < gridDim.x) {
                if (globaltimer_ns() - t0 > kTmaWaitBudgetNs) {
                    record_status(status, NVFP4_ERR_TIMEOUT);
                    s_abort = 1;
                    break;
                }
            }
            __threadfence();
        }
        __syncthreads();
        if (s_abort) ok = false;
    }
    if constexpr (MODE == 1 || MODE == 4) {
        const bool rev = MODE == 4 || t.reverse;
        if (ok) {
            // the prologue's loads go out before the pass's first copies, which would delay
            // them (MODE 4 issued its first copies before the barrier wait)
            const float gsf = encode_prologue<kHThreads>(p, red, &s_gsf, inv_tab);
            zero_padding_scales<kHThreads>(p);
            if constexpr (MODE == 1) prime(rev, l2_policy_evict_first());
            ok = run(rev, l2_policy_evict_first(), [&](uint32_t item, const uint4 (&w)[8]) {
                const uint32_t unit = item * 16 + (lane & 15);
                if (unit < t.total_units) {
                    float r[64];
                    half_values<G>(w, p.hscale, r);
                    const uint32_t row = fast_div(unit, t.upr_div);
                    encode_half64(r, gsf, inv_tab, p, (int64_t)row,
                                  (int64_t)(unit - row * t.upr) * 128 + 64 * (lane >> 4));
                }
            });
        }
    }
    if (!ok && lane == 0) {
        volatile int no_abort = 0;
        for (uint32_t s = 0; s < (uint32_t)kHSlots; ++s) {
            const uint32_t kk = k + s;
            mbar_wait_bounded(&bars[kk % kHSlots], (kk / kHSlots) & 1u, &no_abort, nullptr,
                              100000000ull);
        }
    }
}

// ---------------------------------------------------------------------------
// Single pass for a small dynamic-scale call: one CTA whose warps hold every item of
// the call at once (at most kRWarps * kRSlots items of 4096 values; calls of up to kRWarps
// items are routed here, one item per warp).  Each warp loads its items once, rotates them
// in place in shared memory while taking the amax, the block reduces the maximum, and
// every warp encodes its items from shared memory with the global scale: one read, one
// rotation and one launch, with no grid barrier.  The arithmetic is the streaming passes'
// own, so the results are identical.  (A multi-CTA form with a grid barrier under a
// cooperative launch measured slower than the two streaming passes at every size it
// covered, so larger calls take those.)
// ---------------------------------------------------------------------------

template <int G>
__global__ void __launch_bounds__(kRThreads, 1)
    row_single_kernel(const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmO,
                      const UnitParams p, const RowParams t, int* status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kRRingBytes);
    __shared__ float red[32];
    __shared__ float s_gsf;
    __shared__ float inv_tab[128];
    __shared__ int s_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) s_abort = 0;
    if (lane == 0)
        for (int s = 0; s < kRSlots; ++s) mbar_init(&full[warp * kRSlots + s], 1);
    if (threadIdx.x == 0) {   // the descriptors do not depend on the previous kernel
        prefetch_tensormap(&tmE);
        prefetch_tensormap(&tmO);
    }
    fence_barrier_init();
    __syncthreads();
    griddep_wait();
    griddep_launch_dependents();

    uint8_t* ring = smem + warp * kRSlots * kRItemBytes;
    uint64_t* bars = full + warp * kRSlots;
    if (lane == 0)
        for (int s = 0; s < kRSlots; ++s) {
            const uint32_t it = warp + s * kRWarps;
            if (it < t.n_items)
                load_item(ring + s * kRItemBytes, &tmE, &tmO, &bars[s], it, l2_policy_evict_first());
        }

    // pass over the own items: rotate in place, amax of the rotated values
    uint32_t tmax = 0u;
    bool ok = true;
    for (int s = 0; s < kRSlots; ++s) {
        const uint32_t item = warp + s * kRWarps;
        if (item >= t.n_items) break;
        if (!mbar_wait_bounded(&bars[s], 0u, &s_abort, status, kTmaWaitBudgetNs)) {
            ok = false;
            break;
        }
        uint8_t* slot = ring + s * kRItemBytes;
        uint4 w[16];
        load_unit(slot, lane, w);
        if constexpr (G > 0) {
            float r[128];
            unit_values<G>(w, p.hscale, r);
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                w[c] = make_uint4(pack_bf16_pair(r[8 * c], r[8 * c + 1]),
                                  pack_bf16_pair(r[8 * c + 2], r[8 * c + 3]),
                                  pack_bf16_pair(r[8 * c + 4], r[8 * c + 5]),
                                  pack_bf16_pair(r[8 * c + 6], r[8 * c + 7]));
                *reinterpret_cast<uint4*>(slot + unit_chunk_off(lane, c)) = w[c];
            }
        }
        // units past the end hold the zeros the copy filled in: they add nothing
#pragma unroll
        for (int c = 0; c < 16; ++c) tmax = absmax2_bf16(tmax, absmax_word4(w[c]));
    }
    if (!ok && lane == 0) {
        // let this warp's other loads land before the CTA can leave
        volatile int no_abort = 0;
        for (int s = 0; s < kRSlots; ++s)
            if (warp + s * kRWarps < t.n_items)
                mbar_wait_bounded(&bars[s], 0u, &no_abort, nullptr, 100000000ull);
    }

    // the call's amax (warp 0 holds it), the global scale, then the encode table
    const float m = block_max(absmax_of_pair(tmax), red);
    if (threadIdx.x == 0) s_gsf = __fdiv_rn(kFp4E4m3Range, fmaxf(m, kAmaxFloor));
    __syncthreads();
    if (s_abort) return;
    const float gsf = s_gsf;
    if (threadIdx.x == 0) {
        if (p.gsf_out) *p.gsf_out = gsf;
        if (p.alpha_out) *p.alpha_out = __fdiv_rn(1.0f, __fmul_rn(gsf, *p.gsf_w));
    }
    if (threadIdx.x < 128) {
        const float sv = f32_from_e4m3(threadIdx.x);
        inv_tab[threadIdx.x] = (threadIdx.x == 0 || threadIdx.x == 127) ? 0.0f : __fdiv_rn(gsf, sv);
    }
    zero_padding_scales<kRThreads>(p);
    __syncthreads();

    // encode the own items from shared memory
    for (int s = 0; s < kRSlots; ++s) {
        const uint32_t item = warp + s * kRWarps;
        if (item >= t.n_items) break;
        const uint32_t unit = item * 32 + lane;
        if (unit >= t.total_units) continue;
        uint4 w[16];
        load_unit(ring + s * kRItemBytes, lane, w);
        float r[128];
        unit_values<0>(w, 1.0f, r);
        const uint32_t row = fast_div(unit, t.upr_div);
        encode_unit128(r, gsf, inv_tab, p, (int64_t)row, (int64_t)(unit - row * t.upr) * 128);
    }
}

template <typename Kernel>
bool set_smem_once(Kernel* k, std::atomic<int> (&flags)[64], int device, int bytes) {
    if (flags[device].load(std::memory_order_acquire)) return true;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
        return false;
    flags[device].store(1, std::memory_order_release);
    return true;
}

template <int G>
nvfp4_status launch_row_single(const CUtensorMap& mE, const CUtensorMap& mO, const UnitParams& p,
                               const RowParams& t, int device, int* status, cudaStream_t stream) {
    static std::atomic<int> attr_set[64];
    if (device < 0 || device >= 64) return NVFP4_ERR_DEVICE;
    if (!set_smem_once(row_single_kernel<G>, attr_set, device, kRSmem)) return NVFP4_ERR_CUDA;
    if (launch_pdl(row_single_kernel<G>, 1u, kRThreads, kRSmem, stream, mE, mO, p, t, status) !=
        cudaSuccess)
        return NVFP4_ERR_CUDA;
    return NVFP4_OK;
}

nvfp4_status dispatch_row_single(int g, const CUtensorMap& mE, const CUtensorMap& mO,
                                 const UnitParams& p, const RowParams& t, int device, int* status,
                                 cudaStream_t stream) {
    switch (g) {
        case 0: return launch_row_single<0>(mE, mO, p, t, device, status, stream);
        case 16: return launch_row_single<16>(mE, mO, p, t, device, status, stream);
        case 32: return launch_row_single<32>(mE, mO, p, t, device, status, stream);
        case 64: return launch_row_single<64>(mE, mO, p, t, device, status, stream);
        case 128: return launch_row_single<128>(mE, mO, p, t, device, status, stream);
        default: break;
    }
    return NVFP4_ERR_INVALID_ARG;
}

template <int G, int MODE>
nvfp4_status launch_row(const CUtensorMap& mE, const CUtensorMap& mO, const UnitParams& p,
                        const RowParams& t, int grid, int device, int* status, cudaStream_t stream) {
    static std::atomic<int> attr_set[64];
    if (device < 0 || device >= 64) return NVFP4_ERR_DEVICE;
    if (!set_smem_once(row_kernel<G, MODE>, attr_set, device, kRSmem)) return NVFP4_ERR_CUDA;
    if (launch_pdl(row_kernel<G, MODE>, (unsigned)grid, kRThreads, kRSmem, stream, mE, mO, p, t,
                   status) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    return NVFP4_OK;
}

// The whole-unit streaming passes serve g = 128 (a group spans a whole unit).
template <int MODE>
nvfp4_status dispatch_row(int g, const CUtensorMap& mE, const CUtensorMap& mO, const UnitParams& p,
                          const RowParams& t, int grid, int device, int* status,
                          cudaStream_t stream) {
    if (g == 128) return launch_row<128, MODE>(mE, mO, p, t, grid, device, status, stream);
    return NVFP4_ERR_INVALID_ARG;
}

// MODE 4 is a cooperative launch (its CTAs meet at a grid barrier, so all must be resident)
// after a 4-byte memset of the arrival counter; the others use programmatic dependent
// launch.
template <int G, int MODE>
nvfp4_status launch_half(const CUtensorMap& mE, const CUtensorMap& mO, const UnitParams& p,
                         const RowParams& t, int grid, int device, unsigned int* arrive, int* status,
                         cudaStream_t stream) {
    static std::atomic<int> attr_set[64];
    if (device < 0 || device >= 64) return NVFP4_ERR_DEVICE;
    if (!set_smem_once(half_kernel<G, MODE>, attr_set, device, kHSmem)) return NVFP4_ERR_CUDA;
    if constexpr (MODE == 4) {
        if (cudaMemsetAsync(arrive, 0, sizeof(unsigned int), stream) != cudaSuccess)
            return NVFP4_ERR_CUDA;
        void* args[] = {const_cast<CUtensorMap*>(&mE), const_cast<CUtensorMap*>(&mO),
                        const_cast<UnitParams*>(&p), const_cast<RowParams*>(&t), &arrive, &status};
        if (cudaLaunchCooperativeKernel(reinterpret_cast<void*>(half_kernel<G, MODE>), dim3(grid),
                                        dim3(kHThreads), args, kHSmem, stream) != cudaSuccess)
            return NVFP4_ERR_CUDA;
        return NVFP4_OK;
    }
    if (launch_pdl(half_kernel<G, MODE>, (unsigned)grid, kHThreads, kHSmem, stream, mE, mO, p, t,
                   arrive, status) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    return NVFP4_OK;
}

template <int MODE>
nvfp4_status dispatch_half(int g, const CUtensorMap& mE, const CUtensorMap& mO, const UnitParams& p,
                           const RowParams& t, int grid, int device, unsigned int* arrive,
                           int* status, cudaStream_t stream) {
    switch (g) {
        case 0: return launch_half<0, MODE>(mE, mO, p, t, grid, device, arrive, status, stream);
        case 16: return launch_half<16, MODE>(mE, mO, p, t, grid, device, arrive, status, stream);
        case 32: return launch_half<32, MODE>(mE, mO, p, t, grid, device, arrive, status, stream);
        case 64: return launch_half<64, MODE>(mE, mO, p, t, grid, device, arrive, status, stream);
        default: break;
    }
    return NVFP4_ERR_INVALID_ARG;
}

// One half of every 128-value unit of x: [n_units, 64] bf16 rows 256 bytes apart, based at
// x (first halves) or x + 128 bytes (second halves), with a [box_rows, 64] box and the
// 128-byte swizzle.
bool make_half_map(CUtensorMap* map, const void* base, int64_t n_units, uint32_t box_rows) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {64, (cuuint64_t)n_units};
    cuuint64_t strides[1] = {256};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void*>(base), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
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

    const int64_t n_units = rows * (K / 128);
    if (K % 128 == 0 && n_units < (int64_t(1) << 31) - 64) {
        int* status = nullptr;
        if ((st = status_word(&status)) != NVFP4_OK) return st;
        CUtensorMap mE, mO;
        if (!make_half_map(&mE, x, n_units, 32) ||
            !make_half_map(&mO, static_cast<const uint8_t*>(x) + 128, n_units, 32))
            return NVFP4_ERR_CUDA;
        p.total_units = n_units;
        RowParams t{};
        t.total_units = (uint32_t)n_units;
        t.n_items = (uint32_t)((n_units + 31) / 32);
        t.upr = (uint32_t)(K / 128);
        t.upr_div = make_fastdiv(t.upr);
        t.reverse = 0;
        // a small dynamic call: one CTA holds it all, one item per warp (one launch)
        if (gsf_in == nullptr && t.n_items <= (uint32_t)kRWarps)
            return dispatch_row_single(group, mE, mO, p, t, dev.device, status, stream);
        // multi-pass calls.  g = 128 keeps a whole unit per thread (row_kernel, pieces of 32
        // units); g <= 64 has every group inside a 64-value half and runs the half-unit
        // kernels (half_kernel, pieces of 16 units, 16 warps per SM).
        const bool whole = group == 128;
        const uint32_t iu = whole ? 32u : 16u;
        const int warps = whole ? kRWarps : kHWarps;
        if (!whole && (!make_half_map(&mE, x, n_units, 16) ||
                       !make_half_map(&mO, static_cast<const uint8_t*>(x) + 128, n_units, 16)))
            return NVFP4_ERR_CUDA;
        t.n_items = (uint32_t)((n_units + iu - 1) / iu);
        const int64_t need = ((int64_t)t.n_items + warps - 1) / warps;
        const int grid = (int)(need < dev.sms ? (need > 0 ? need : 1) : dev.sms);
        // the grid-barrier arrival counter lives in the last word of the caller's 4 KiB
        // workspace (a static call has none and needs none)
        unsigned int* arrive =
            partials ? reinterpret_cast<unsigned int*>(partials) + (kMaxPartials - 1) : nullptr;
        if (gsf_in == nullptr && group == 0) {
            // amax phase, grid barrier, encode phase in one cooperative kernel: for the
            // bandwidth-bound unrotated calls (weight packing) this saves a launch, a ramp-up
            // and a tail
            p.partials_out = partials;
            p.partials = partials;
            p.n_partials = grid;
            return launch_half<0, 4>(mE, mO, p, t, grid, dev.device, arrive, status, stream);
        }
        if (gsf_in == nullptr) {
            // rotated: two launches, the amax pass then the encode pass, both with
            // programmatic dependent launch (a cooperative launch cannot overlap the previous
            // kernel's tail)
            UnitParams a = p;
            a.partials_out = partials;
            st = whole ? dispatch_row<0>(group, mE, mO, a, t, grid, dev.device, status, stream)
                       : dispatch_half<0>(group, mE, mO, a, t, grid, dev.device, arrive, status, stream);
            if (st != NVFP4_OK) return st;
            p.partials = partials;
            p.n_partials = grid;
            t.reverse = 1;   // the encode pass starts where the amax pass ended (in L2)
        }
        return whole ? dispatch_row<1>(group, mE, mO, p, t, grid, dev.device, status, stream)
                     : dispatch_half<1>(group, mE, mO, p, t, grid, dev.device, arrive, status, stream);
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
