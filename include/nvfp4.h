/*
 * nvfp4.h -- C ABI of the B200 (sm_100a) NVFP4 W4A4 linear library
 *
 *     y = dequant(Q(x.H)) . dequant(Q(W.H))^T + b
 *
 * Format (the pages: "minimax_h3_nvfp4_decoder" -- nvfp4_linear_inference and
 * NVFP4DecoderLinear; "convert_minimax_h3_text_encoder_nvfp4.py" -- module
 * docstring and quantize_language_linear; "FastH3-QAD-v2 and NVFP4 VAE Decoders" --
 * "The whole stack in NVFP4"):
 *   - E2M1 4-bit values, 16 consecutive values along K share one FP8-E4M3 scale,
 *     one FP32 global scale per tensor: value = e2m1 * e4m3 / global_scale.
 *   - packed data: uint8 [rows, K/2], row-major; element 2i in bits 0..3 of byte i,
 *     element 2i+1 in bits 4..7.
 *   - scales: uint8, nvfp4_scale_bytes(rows, K) bytes in the 128x4 tile layout:
 *     rows padded to Rp = ceil(rows/128)*128, scale columns (K/16) padded to
 *     Cp = ceil(K/64)*4, byte (r, c) at ((r/128)*(Cp/4) + c/4)*512 + (r%32)*16
 *     + ((r%128)/32)*4 + c%4; padding bytes are 0 (the quantizer writes them).
 *   - global scale: gsf = 2688 / max(amax, 1e-12) (2688 = 448 * 6); dynamic =
 *     amax over the whole call, static = a device scalar the caller computed.
 *   - GEMM epilogue: y = bf16(alpha * acc + bias), alpha = 1 / (gsf_x * gsf_w).
 *
 * Conventions for every entry point:
 *   - Every pointer except those marked "host" is a device pointer on the current
 *     device, owned by the caller.  The library never allocates, frees or
 *     synchronises (except nvfp4_last_device_status, which says so); each call only
 *     enqueues kernels on `stream` (a cudaStream_t; NULL = legacy default stream),
 *     so calls are stream-ordered and may be captured in a CUDA graph
 *     (nvfp4_linear_fixed_scratch states its own set-up condition).  The quantizer
 *     and GEMM kernels are launched with programmatic stream serialization: their
 *     set-up (barriers, tensor memory) may overlap the end of the previous kernel on
 *     the stream, but they wait for it to complete before touching any global
 *     memory, so the stream order holds for every input and output.
 *   - bf16 tensors are row-major with no padding; tensor pointers must be 16-byte
 *     aligned, scalar pointers 4-byte aligned.
 *   - Argument checks run on the host before anything is enqueued; on any error
 *     nothing is launched and the status says why.  A zero-size call (rows, M or N
 *     equal to 0) returns NVFP4_OK and launches nothing.
 *   - Device-side waits are bounded; a kernel that gives up records
 *     NVFP4_ERR_TIMEOUT in a per-device status word (see nvfp4_last_device_status)
 *     and returns instead of hanging.
 *   - NaN or Inf inputs are outside the contract (results unspecified, no fault).
 */
#ifndef NVFP4_B200_H
#define NVFP4_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NVFP4_API __attribute__((visibility("default")))
#else
#define NVFP4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    NVFP4_OK = 0,
    NVFP4_ERR_INVALID_ARG = 1,  /* null pointer, negative size, unsupported group */
    NVFP4_ERR_SHAPE = 2,        /* K not a multiple of 16 (64 for the GEMM), K % group != 0 */
    NVFP4_ERR_ALIGN = 3,        /* tensor pointer not 16-byte aligned */
    NVFP4_ERR_WORKSPACE = 4,    /* workspace missing or smaller than required */
    NVFP4_ERR_DEVICE = 5,       /* current device is not compute capability 10.0 (B200) */
    NVFP4_ERR_CUDA = 6,         /* a CUDA runtime/driver call failed (launch, tensor map) */
    NVFP4_ERR_TIMEOUT = 7       /* a device-side wait ran out (reported asynchronously) */
} nvfp4_status;

/* Human-readable name of a status code (static string). */
NVFP4_API const char* nvfp4_status_string(int status);

/* Version of this ABI (bumped on any signature change). */
NVFP4_API int nvfp4_abi_version(void);

/* Bytes of the 128x4 scale tensor for a [rows, K] operand: ceil(rows/128)*128 *
 * ceil(K/64)*4 ("convert_minimax_h3_text_encoder_nvfp4.py" -- nvfp4_scale_shape).
 * Returns 0 for rows <= 0 or K <= 0. */
NVFP4_API size_t nvfp4_scale_bytes(int64_t rows, int64_t K);

/* Bytes of the packed data for a [rows, K] operand: rows * K / 2
 * ("minimax_h3_nvfp4_decoder" -- from_packed: [out_features, in_features // 2]). */
NVFP4_API size_t nvfp4_packed_bytes(int64_t rows, int64_t K);

/*
 * hadamard_rotate -- block Hadamard rotation along the last dimension
 * ("minimax_h3_nvfp4_decoder" -- rotate_activation, module docstring, from_linear:
 * an orthonormal symmetric block Hadamard applied per group of `group` values).
 *   x_bf16 : in,  bf16 [rows, K]
 *   y_bf16 : out, bf16 [rows, K]; may equal x_bf16 (in place)
 *   group  : 16, 32, 64 or 128; K % group == 0
 * Each group y = H_g x / sqrt(g) with the Sylvester H_g, computed as an fp32
 * butterfly (stages h = 1, 2, ..., g/2), one fp32 multiply by rn(1/sqrt(g)) and
 * round-to-nearest-even to bf16.  Used offline on W (the weight fold) and, fused
 * into nvfp4_quantize, on activations.
 * Errors: INVALID_ARG (null, rows < 0, bad group), SHAPE (K <= 0, K % group),
 * ALIGN, DEVICE, CUDA.
 */
NVFP4_API nvfp4_status hadamard_rotate(const void* x_bf16, void* y_bf16, int64_t rows, int64_t K,
                             int group, void* stream);

/* Workspace bytes nvfp4_quantize needs when gsf_in == NULL (dynamic scale); a
 * constant, independent of the shape.  A static call needs none. */
NVFP4_API size_t nvfp4_quantize_workspace_bytes(void);

/*
 * nvfp4_quantize -- NVFP4 quantizer for activations (per call) and weights
 * (offline), with the optional rotation fused in
 * ("minimax_h3_nvfp4_decoder" -- nvfp4_linear_inference: nvfp4_quantize_fenced with
 * layout_128x4; _activation_global_sf; "convert_minimax_h3_text_encoder_nvfp4.py" --
 * quantize_language_linear: nvfp4_weight_global_scale then _nvfp4_quantize).
 *   x_bf16       : in,  bf16 [rows, K]; K % 16 == 0
 *   rotate_group : 0 (none) or 16/32/64/128 (K % group == 0): x is rotated exactly
 *                  as hadamard_rotate does, then quantized (one HBM pass per pass)
 *   gsf_in       : in,  device fp32 scalar = static global scale, or NULL = dynamic:
 *                  gsf = 2688 / max(amax, 1e-12) with amax = max |x (rotated)| over
 *                  all rows*K values (two passes over x)
 *   gsf_out      : out, device fp32 scalar, always written with the scale used
 *                  (may be NULL when gsf_in is given)
 *   packed       : out, uint8 [rows, K/2]
 *   sf           : out, uint8 [nvfp4_scale_bytes(rows, K)], padding written as 0
 *   gsf_w        : in,  optional device fp32 scalar (the weight's global scale of the
 *                  GEMM this activation feeds); with alpha_out, the kernel also writes
 *   alpha_out    : out, optional device fp32 scalar alpha = rn(1 / rn(gsf * gsf_w)),
 *                  ready for nvfp4_gemm; both NULL or both given
 *   workspace    : scratch of nvfp4_quantize_workspace_bytes() bytes (dynamic only;
 *                  may be NULL for a static call), 16-byte aligned, caller-owned,
 *                  contents need no initialisation
 * Per block of 16: bmax = max|x|; s8 = E4M3(rn(rn(gsf*bmax)/6)) (RNE, saturating);
 * if dec(s8) == 0 all codes are 0, else code = E2M1(rn(x * rn(gsf/dec(s8)))) (RNE,
 * saturating, sign kept).
 * Errors: INVALID_ARG, SHAPE (K <= 0, K % 16, K % group), ALIGN, WORKSPACE, DEVICE, CUDA.
 */
NVFP4_API nvfp4_status nvfp4_quantize(const void* x_bf16, int64_t rows, int64_t K, int rotate_group,
                                      const float* gsf_in, float* gsf_out, uint8_t* packed,
                                      uint8_t* sf, const float* gsf_w, float* alpha_out,
                                      void* workspace, size_t ws_bytes, void* stream);

/*
 * nvfp4_gemm -- block-scaled FP4 GEMM on the tcgen05 tensor cores with the
 * rescale and bias fused into the epilogue
 * ("minimax_h3_nvfp4_decoder" -- nvfp4_linear_inference: mm_fp4(x_fp4, packed.T,
 * x_sf, w_sf.T, 1/(gsf_x*gsf_w), bf16, out, block_size=16) then out.add_(bias)).
 *   a, sfa  : in,  packed [M, K/2] + 128x4 scales of the activation (K-major)
 *   b, sfb  : in,  packed [N, K/2] + 128x4 scales of the weight (K-major, "TN")
 *   alpha   : in,  device fp32 scalar, 1 / (gsf_x * gsf_w)
 *   bias    : in,  bf16 [N] or NULL
 *   y_bf16  : out, bf16 [M, N] row-major
 *   K % 64 == 0 (32-byte packed rows keep the tensor-map rows aligned and match the
 *   128x4 scale tiling); M, N >= 0, each below 2^31.
 * y[m,n] = bf16(fp32(alpha * acc) + bias[n]), acc = the fp32 tensor-core sum of
 * (e2m1_a * e4m3_a) * (e2m1_b * e4m3_b) over k.  When the 128 x 256 output tiles
 * fill at most half of the SMs (small M), K is split over a thread-block cluster and
 * the partial sums are added in a fixed order, so results are deterministic either way.
 * Errors: INVALID_ARG, SHAPE, ALIGN, DEVICE, CUDA.
 */
NVFP4_API nvfp4_status nvfp4_gemm(const uint8_t* a, const uint8_t* sfa, const uint8_t* b,
                        const uint8_t* sfb, const float* alpha, const void* bias_bf16,
                        void* y_bf16, int64_t M, int64_t N, int64_t K, void* stream);

/*
 * nvfp4_prepare_weight_scales -- a weight's 128x4 block scales rearranged once, offline,
 * for nvfp4_gemm_prepared / nvfp4_linear_prepared (same page and operation as
 * nvfp4_gemm; only the order of the B scale bytes differs).  For each 256-row block nb of
 * W and each K stage s of 256 values there is one 4 KiB block, at (nb * ceil(K/256) + s)
 * * 4096; inside it, the 512 bytes at h*2048 + j*512 (h = 0, 1; j = 0..3) are the 128x4
 * chunk of row tile 2*nb + h and K step 4*s + j (zero where that row tile is past N or
 * that step past K/64).  That is the order in which the GEMM holds a stage's B scales in
 * shared memory, so a stage takes one 4 KiB bulk copy instead of two.
 *   sf  : in,  the weight's 128x4 scales (nvfp4_scale_bytes(N, K) bytes)
 *   out : out, nvfp4_prepared_scale_bytes(N, K) bytes, caller-owned
 *   K % 64 == 0.  Errors: INVALID_ARG, SHAPE, ALIGN (16-byte), DEVICE, CUDA.
 */
NVFP4_API size_t nvfp4_prepared_scale_bytes(int64_t N, int64_t K);
NVFP4_API nvfp4_status nvfp4_prepare_weight_scales(const uint8_t* sf, int64_t N, int64_t K,
                                                   uint8_t* out, void* stream);

/*
 * nvfp4_gemm_prepared -- nvfp4_gemm with the weight scales from
 * nvfp4_prepare_weight_scales (sfb_prepared); arguments, result (bit for bit) and errors
 * otherwise as nvfp4_gemm.  Two tensor-memory scale copies per K step instead of three.
 */
NVFP4_API nvfp4_status nvfp4_gemm_prepared(const uint8_t* a, const uint8_t* sfa, const uint8_t* b,
                                           const uint8_t* sfb_prepared, const float* alpha,
                                           const void* bias_bf16, void* y_bf16, int64_t M,
                                           int64_t N, int64_t K, void* stream);

/*
 * nvfp4_gemm_quantize_out -- nvfp4_gemm whose epilogue hands the next linear its NVFP4
 * input directly: the bf16 product y = bf16(alpha * acc + bias) is encoded in
 * registers under a static global scale and only the codes and scales are written
 * ("minimax_h3_nvfp4_decoder" -- NVFP4FusedState and NVFP4DecoderLinear.fused_state:
 * the fused kernels quantize with a precomputed global scale and alpha, so dynamic
 * scales and the activation rotation stay on the unfused path; "FastH3-QAD-v2 and NVFP4
 * VAE Decoders" -- "Fused FP4 kernels": quantize, scale and GEMM without round trips
 * through memory, bit-exact with the unfused path).
 *   a, sfa, b, sfb, alpha, bias_bf16, M, N, K : as nvfp4_gemm
 *   gsf_out    : in,  device fp32 scalar, the static global scale of the next linear's input
 *   out_packed : out, uint8 [M, N/2]
 *   out_sf     : out, uint8 [nvfp4_scale_bytes(M, N)], 128x4 layout, padding rows 0
 * The encoding is exactly nvfp4_quantize(y, rotate_group 0, gsf_in = gsf_out) applied to
 * the bf16 y nvfp4_gemm would have written; y itself is not written.  N % 64 == 0.
 * Errors: as nvfp4_gemm; SHAPE also for N % 64; ALIGN for out_packed, out_sf (16 bytes)
 * and gsf_out (4 bytes).
 */
NVFP4_API nvfp4_status nvfp4_gemm_quantize_out(const uint8_t* a, const uint8_t* sfa, const uint8_t* b,
                                               const uint8_t* sfb, const float* alpha,
                                               const void* bias_bf16, const float* gsf_out,
                                               uint8_t* out_packed, uint8_t* out_sf, int64_t M,
                                               int64_t N, int64_t K, void* stream);

/* Workspace bytes nvfp4_linear needs for an [M, K] activation: the packed
 * activation, its scales, the two scalars and the dynamic-scale scratch, each
 * 256-byte aligned. */
NVFP4_API size_t nvfp4_linear_workspace_bytes(int64_t M, int64_t K);

/*
 * nvfp4_linear -- the whole W4A4 linear on one stream: [rotate] -> [amax] ->
 * quantize -> GEMM ("minimax_h3_nvfp4_decoder" -- NVFP4DecoderLinear.forward and
 * nvfp4_linear_inference).
 *   x_bf16       : in,  bf16 [M, K]
 *   w_packed     : in,  packed weight [N, K/2]; w_sf its 128x4 scales
 *   gsf_w        : in,  device fp32 scalar, the weight's global scale
 *   bias_bf16    : in,  bf16 [N] or NULL
 *   gsf_x        : in,  device fp32 scalar (static / unit scale) or NULL (dynamic)
 *   rotate_group : 0 or 16/32/64/128; the weight must already be rotated with the
 *                  same group (hadamard_rotate on W before nvfp4_quantize)
 *   workspace    : nvfp4_linear_workspace_bytes(M, K) bytes, 256-byte aligned
 *   y_bf16       : out, bf16 [M, N]
 *   K % 64 == 0.  alpha = rn(1 / rn(gsf_x * gsf_w)) is computed on the device.
 * Errors: as nvfp4_quantize and nvfp4_gemm.
 */
NVFP4_API nvfp4_status nvfp4_linear(const void* x_bf16, int64_t M, int64_t K, const uint8_t* w_packed,
                          const uint8_t* w_sf, const float* gsf_w, int64_t N,
                          const void* bias_bf16, const float* gsf_x, int rotate_group,
                          void* workspace, size_t ws_bytes, void* y_bf16, void* stream);

/*
 * nvfp4_linear_prepared -- nvfp4_linear with the weight scales from
 * nvfp4_prepare_weight_scales (w_sf_prepared); arguments, workspace, result (bit for bit)
 * and errors otherwise as nvfp4_linear.
 */
NVFP4_API nvfp4_status nvfp4_linear_prepared(const void* x_bf16, int64_t M, int64_t K,
                                             const uint8_t* w_packed,
                                             const uint8_t* w_sf_prepared, const float* gsf_w,
                                             int64_t N, const void* bias_bf16,
                                             const float* gsf_x, int rotate_group,
                                             void* workspace, size_t ws_bytes, void* y_bf16,
                                             void* stream);

/*
 * nvfp4_dequantize -- NVFP4 -> bf16 expansion of a packed tensor, the W4A16 path for
 * GPUs without an FP4 GEMM ("decode dynamic-scale NVFP4 H3 VAE tiles one at a time" --
 * FASTVIDEO_H3_ENCODER_FUSED_DEQUANT: one fused pass that expands the serialized NVFP4
 * text encoder to bf16).
 *   packed : in,  uint8 [rows, K/2] (element 2i in the low nibble of byte i)
 *   sf     : in,  uint8 [nvfp4_scale_bytes(rows, K)], 128x4 layout
 *   gsf    : in,  device fp32 scalar, the tensor's global scale
 *   y_bf16 : out, bf16 [rows, K]
 * y = RNE_bf16(fp32(E2M1(code) * E4M3(scale)) / gsf), the division in IEEE fp32.  Scale
 * bytes are expected in 0..0x7E (what nvfp4_quantize writes); other bytes give the
 * negative or NaN values their E4M3 decoding implies.  K % 16 == 0.
 * Errors: INVALID_ARG, SHAPE (K <= 0 or K % 16), ALIGN (packed, sf, y not 16-byte
 * aligned; gsf not 4-byte aligned), DEVICE, CUDA.
 */
NVFP4_API nvfp4_status nvfp4_dequantize(const uint8_t* packed, const uint8_t* sf, const float* gsf,
                                        int64_t rows, int64_t K, void* y_bf16, void* stream);

/* ---- int8 per-row W8A8 linear ------------------------------------------------ */
/*
 * The pages' second quantized linear ("FastH3-4-step-Preview-v1-r16-int8" -- "What is
 * inside"): int8 codes round(x / s) clamped to -127..127 with one fp32 scale
 * s = amax(|row|) / 127 per row, weights per output row offline and activations per row
 * at call time; the product runs on the int8 tensor cores with an exact int32
 * accumulator.  Division and scale in fp32 (round to nearest even), round() half to
 * even, an all-zero row gives s = 0 and codes 0.
 */

/*
 * int8_quantize_rows -- per-row int8 quantizer.
 *   x_bf16 : in,  bf16 [rows, K], K % 16 == 0
 *   q      : out, int8 [rows, K]
 *   scale  : out, fp32 [rows]
 * Errors: INVALID_ARG, SHAPE (K <= 0 or K % 16), ALIGN (x, q 16-byte; scale 4-byte),
 * DEVICE, CUDA.
 */
NVFP4_API nvfp4_status int8_quantize_rows(const void* x_bf16, int64_t rows, int64_t K, int8_t* q,
                                          float* scale, void* stream);

/*
 * int8_gemm -- y = bf16((fp32(acc) * sa[m]) * sb[n] + bias[n]), acc = sum_k a[m,k] b[n,k]
 * in int32 (tcgen05.mma kind::i8).
 *   a, sa : in, int8 [M, K] and fp32 [M];  b, sb : in, int8 [N, K] and fp32 [N]
 *   bias_bf16 : in, bf16 [N] or NULL;  y_bf16 : out, bf16 [M, N]
 * K % 32 == 0.  Errors: as nvfp4_gemm (ALIGN: a, b, y, bias 16-byte; sa, sb 16-byte).
 */
NVFP4_API nvfp4_status int8_gemm(const int8_t* a, const float* sa, const int8_t* b, const float* sb,
                                 const void* bias_bf16, void* y_bf16, int64_t M, int64_t N,
                                 int64_t K, void* stream);

/* Workspace bytes int8_linear needs for an [M, K] activation: the codes and the row
 * scales, 256-byte aligned. */
NVFP4_API size_t int8_linear_workspace_bytes(int64_t M, int64_t K);

/*
 * int8_linear -- int8_quantize_rows(x) then int8_gemm with the stored weight, one stream.
 *   x_bf16 : in, bf16 [M, K];  wq, sw : in, int8 [N, K] and fp32 [N] (offline codes)
 *   bias_bf16 : in, bf16 [N] or NULL;  workspace : int8_linear_workspace_bytes(M, K) bytes,
 *   256-byte aligned;  y_bf16 : out, bf16 [M, N].  K % 32 == 0.
 * Errors: as int8_quantize_rows and int8_gemm; WORKSPACE.
 */
NVFP4_API nvfp4_status int8_linear(const void* x_bf16, int64_t M, int64_t K, const int8_t* wq,
                                   const float* sw, int64_t N, const void* bias_bf16,
                                   void* workspace, size_t ws_bytes, void* y_bf16, void* stream);

/* Size of the library's own fixed device scratch used by
 * nvfp4_linear_fixed_scratch: 8 MiB. */
#define NVFP4_FIXED_SCRATCH_BYTES ((size_t)8 << 20)

/*
 * nvfp4_linear_fixed_scratch -- nvfp4_linear without a caller workspace.  The
 * pages have no counterpart: this is a convenience of the library, not a step
 * of the method.  It computes exactly what nvfp4_linear computes (same kernels,
 * same arguments minus the workspace).
 *
 * Who it is for: callers that cannot allocate device memory at call time or
 * have none to lend -- a C host program without a device allocator of its own,
 * a serving process that reserved all device memory up front, or a path where
 * a cudaMalloc would synchronise the device and stall the other streams.  The
 * call itself allocates nothing: the packed activation, its scales, the two
 * device scalars and the amax partials live in one fixed array of
 * NVFP4_FIXED_SCRATCH_BYTES bytes inside the library, placed in device memory
 * when the library's module is loaded.
 *
 * Limit: nvfp4_linear_workspace_bytes(M, K) <= NVFP4_FIXED_SCRATCH_BYTES
 * (for example M*K up to about 14.8 M values: 4096 x 3584, or one
 * 4096 x 1024 tile); a larger call returns NVFP4_ERR_WORKSPACE and launches
 * nothing.
 *
 * Set-up: the first call on each device (with that device current) looks up the
 * scratch address once; make that first call before any stream capture.
 * Nothing in the scratch has to start at zero: each call writes every scratch
 * byte it reads before reading it.
 *
 * Races: the scratch is one per device, so two calls on the same device that
 * can overlap (different streams, or different host threads without ordering)
 * race on it and corrupt each other.  Calls on one stream are ordered and safe.
 *
 * Arguments, layouts, alignment and the other errors: as nvfp4_linear.
 */
NVFP4_API nvfp4_status nvfp4_linear_fixed_scratch(const void* x_bf16, int64_t M, int64_t K,
                                                  const uint8_t* w_packed, const uint8_t* w_sf,
                                                  const float* gsf_w, int64_t N,
                                                  const void* bias_bf16, const float* gsf_x,
                                                  int rotate_group, void* y_bf16, void* stream);

/*
 * nvfp4_last_device_status -- synchronises `stream`, then returns (in *status,
 * host pointer) and clears the current device's asynchronous status word:
 * NVFP4_OK, or NVFP4_ERR_TIMEOUT when a kernel's bounded wait ran out since the
 * last call.  Returns NVFP4_ERR_CUDA if the synchronisation itself failed.
 */
NVFP4_API nvfp4_status nvfp4_last_device_status(void* stream, int* status);

/* ---- diagnostics used by the test suite ---------------------------------- */

/*
 * nvfp4_debug_cvt_sweep -- runs the quantizer's own device conversions over the
 * fp32 bit patterns first, first+1, ..., first+n-1 (wrapping mod 2^32):
 *   e2m1[i]  = E2M1 code of the pattern (RNE, saturating, sign kept)
 *   e4m3[i]  = E4M3 byte of |pattern| (RNE, saturating)
 *   scale[i] = the block-scale byte the quantizer derives from a scaled block
 *              maximum y = |pattern|: E4M3(rn(y / 6))
 * All outputs: device uint8 [n].  Errors: INVALID_ARG, DEVICE, CUDA.
 */
NVFP4_API nvfp4_status nvfp4_debug_cvt_sweep(uint32_t first, int64_t n, uint8_t* e2m1, uint8_t* e4m3,
                                             uint8_t* scale, void* stream);

/*
 * nvfp4_debug_wait_timeout -- launches one block that waits on a barrier nothing
 * will ever arrive at, with a wait budget of `budget_us` microseconds (1..2000000),
 * so that the bounded-wait path runs: the kernel records NVFP4_ERR_TIMEOUT in the
 * device status word and returns.  Used to test failure reporting without hanging
 * or faulting the GPU.  Errors: INVALID_ARG, DEVICE, CUDA.
 */
NVFP4_API nvfp4_status nvfp4_debug_wait_timeout(int64_t budget_us, void* stream);

/*
 * nvfp4_debug_gemm_f32 -- nvfp4_gemm (sfb_prepared = 0) or nvfp4_gemm_prepared
 * (sfb_prepared = 1) built with an unrounded output: the same tile schedule, mainloop
 * and accumulation order, and the epilogue stores y[m,n] = fp32(alpha * acc) + bias[n]
 * (fp32 add) instead of rounding it to bf16.  The operation is the one the decoder page
 * defines ("minimax_h3_nvfp4_decoder" -- nvfp4_linear_inference: mm_fp4 then the bias);
 * the page's mm_fp4 writes bf16, and the bf16 result of nvfp4_gemm equals this output
 * rounded to nearest even.  It exists so that the GEMM's accumulation error can be
 * checked against an fp64 reference without the bf16 output rounding on top.
 *   a, sfa, b, sfb, alpha, bias_bf16, M, N, K : as nvfp4_gemm / nvfp4_gemm_prepared
 *   y_f32 : out, fp32 [M, N] row-major, 16-byte aligned, caller-owned
 * Errors: as nvfp4_gemm; INVALID_ARG also for sfb_prepared other than 0 or 1.
 */
NVFP4_API nvfp4_status nvfp4_debug_gemm_f32(const uint8_t* a, const uint8_t* sfa, const uint8_t* b,
                                            const uint8_t* sfb, int sfb_prepared,
                                            const float* alpha, const void* bias_bf16,
                                            float* y_f32, int64_t M, int64_t N, int64_t K,
                                            void* stream);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_B200_H */
