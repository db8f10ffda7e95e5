/*
 * fp4.h -- C ABI of the B200 (sm_100a) W4A4 block-scaled FP4 library.
 *
 * Formats (sources are web pages, cited by title and section):
 *  NVFP4  E2M1 codes {0, +-0.5, +-1, +-1.5, +-2, +-3, +-4, +-6}; every 16
 *         consecutive values along K share an E4M3 scale chosen so the block
 *         maximum lands on 6; a per-tensor FP32 global scale g keeps the
 *         block scales inside E4M3's range (saturating, never NaN).
 *         "Hardware FP4 inference for speech on Blackwell", section "NVFP4,
 *         and the two ways it fails".
 *  MXFP4  the OCP MX variant: 32 values per block share an E8M0 power-of-two
 *         scale; no global scale.  "FP4 n'existe pas : il existe des FP4, et
 *         chaque runtime choisit son dialecte", section "Deux dialectes, deux
 *         strategies de scaling" and its format table.
 *
 * Operation (the W4A4 GEMM of the first page, "fp4-cuda-kernel" forum post:
 * weights quantized once at load, activations quantized on the fly per call):
 *     C[m, n] = alpha * sum_k  s_a[m, k/B] * q_a[m, k] * s_w[n, k/B] * q_w[n, k]
 * with alpha = g_a * g_w (NVFP4) or 1 (MXFP4), accumulation in FP32.
 *
 * Conventions shared by every entry point
 *  - Every pointer argument is a DEVICE pointer unless stated otherwise.
 *    The caller allocates and owns all memory; the library never allocates,
 *    frees or synchronizes (fp4_device_status is the one exception and says
 *    so).  Work is enqueued on `stream` (a cudaStream_t; NULL = legacy
 *    default stream) and is asynchronous; global scales stay on the device.
 *  - Argument checks happen before any launch and return a status; nothing
 *    is enqueued when a check fails.  A failed launch returns FP4_ERR_CUDA.
 *  - Shapes: rows (M or N) >= 0, K > 0 and K % 32 == 0 (a packed row of K/2
 *    bytes must be a multiple of 16 bytes for the tensor-memory-accelerator
 *    loads).  rows == 0 (or M == 0 / N == 0) is a no-op that returns FP4_OK
 *    after the shape and enum checks, without looking at the pointers.
 *    N % 8 == 0 for the GEMMs.
 *  - Alignment: bf16 inputs, code and scale buffers and C are 16-byte
 *    aligned; ldc * sizeof(element) is a multiple of 16; g pointers 4-byte.
 *  - Packed codes: row-major [rows, K/2] bytes; element 2j of a row is the
 *    low nibble of byte j, element 2j+1 the high nibble; a code is
 *    sign<<3 | exponent<<1 | mantissa.
 *  - Scales, FP4_SCALES_ROWMAJOR: [rows, K/B] bytes (B = 16 or 32).
 *    FP4_SCALES_MMA: the order the tensor cores read.  Scales are grouped in
 *    atoms of 128 rows x 4 scale columns (512 bytes); in an atom, row r and
 *    column c sit at byte (r%32)*16 + (r/32)*4 + c; atom (rb, cb) starts at
 *    byte (rb * ceil(nsf/4) + cb) * 512 with nsf = K/B.  Rows are padded to
 *    a multiple of 128 and columns to a multiple of 4; the library writes
 *    the padding as 0.
 */
#ifndef FP4_B200_H
#define FP4_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FP4_OK = 0,
    FP4_ERR_INVALID_ARG = 1,        /* null pointer, bad enum, ldc < N, ... */
    FP4_ERR_UNSUPPORTED_SHAPE = 2,  /* K % 32 != 0, N % 8 != 0, negative size */
    FP4_ERR_MISALIGNED = 3,         /* a pointer or leading dimension misaligned */
    FP4_ERR_WORKSPACE_TOO_SMALL = 4,
    FP4_ERR_CUDA = 5,               /* a CUDA runtime call or launch failed */
    FP4_ERR_DEVICE_TIMEOUT = 6,     /* a kernel's bounded wait ran out */
    FP4_ERR_NO_DEVICE = 7,          /* no sm_100 device is current */
    FP4_ERR_NONFINITE = 8           /* a DYNAMIC amax met an Inf or NaN input
                                       (reported by fp4_device_status) */
} fp4_status_t;

typedef enum { FP4_NVFP4 = 0, FP4_MXFP4 = 1 } fp4_format_t;
typedef enum { FP4_SCALES_MMA = 0, FP4_SCALES_ROWMAJOR = 1 } fp4_scale_layout_t;
/* NVFP4 only: DYNAMIC computes g = amax(tensor) / 2688 on the device (g = 1
 * for an all-zero tensor) and writes it to *g; STATIC reads a caller-chosen
 * g from *g.  2688 = 6 * 448 ("Hardware FP4 inference for speech on
 * Blackwell", section "NVFP4, and the two ways it fails"). */
typedef enum { FP4_GLOBAL_DYNAMIC = 0, FP4_GLOBAL_STATIC = 1 } fp4_global_mode_t;
typedef enum { FP4_OUT_BF16 = 0, FP4_OUT_F32 = 1 } fp4_out_t;

/* Bytes of packed codes for a [rows, K] tensor: rows * K / 2. */
size_t fp4_packed_bytes(int rows, int K);

/* Bytes of scales for a [rows, K] tensor in the given layout (MMA layout
 * includes its padding).  Returns 0 for an unsupported K. */
size_t fp4_scale_bytes(int rows, int K, fp4_format_t fmt, fp4_scale_layout_t layout);

/* Device workspace (bytes) that fp4_quantize_act / fp4_quantize_weights /
 * fp4_gemm / fp4_gemm_fused need for a problem of this size.  The workspace
 * holds per-block partial maxima of the DYNAMIC global-scale reduction and,
 * for the small-M path, split-K partial sums; it needs no initialisation. */
size_t fp4_workspace_bytes(int M, int N, int K, fp4_format_t fmt);

/* Activation quantization, run per call: one pass of amax (DYNAMIC only) and
 * one fused pass block-amax -> scale -> round-to-nearest-even to E2M1 ->
 * nibble pack.  "Hardware FP4 inference for speech on Blackwell", section
 * "NVFP4, and the two ways it fails" (s = E4M3(max|x|/6), x_hat = s*q, 448,
 * 2688); MXFP4 per the format table of "FP4 n'existe pas".
 *   x       bf16 [rows, K] row-major, contiguous
 *   g       NVFP4: DYNAMIC writes g, STATIC reads g; MXFP4: ignored (may be NULL)
 *   codes   [rows, K/2] bytes out; scales out in `layout`
 *   ws      workspace of at least fp4_workspace_bytes(rows, 0, K, fmt) bytes
 * Floating-point steps (one IEEE binary32 rounding each): g = amax/2688;
 * sb = amax_b / (6 g); s = E4M3 round-to-nearest-even, saturating at 448;
 * r = 1 / (s g); q = E2M1 round-to-nearest-even of x r, saturating at 6,
 * sign kept (a negative value that rounds to zero is code 0x8); a block
 * whose scale rounds to 0 gets all-zero codes.  MXFP4: e = floor(log2
 * amax_b) - 2 clamped to [-127, 127], scale byte e + 127, q = E2M1(x 2^-e). */
fp4_status_t fp4_quantize_act(const void* x, int rows, int K, fp4_format_t fmt,
                              fp4_scale_layout_t layout, fp4_global_mode_t gmode,
                              float* g, uint8_t* codes, uint8_t* scales,
                              void* ws, size_t ws_bytes, void* stream);

/* Options of the extended quantizer entry points below.  Passing NULL, or a
 * zeroed struct, gives exactly the plain entry points' results.
 *  hadamard  0: none.  16 or 32: an online rotation of every n consecutive
 *            values of a row (blocks from k = 0) by the Walsh-Hadamard
 *            matrix of order n, Sylvester order H[i][j] = (-1)^popcount(i&j),
 *            ahead of the quantizer (the DYNAMIC amax is that of the rotated
 *            tensor).  Computed in binary32 by the fast transform (for
 *            h = 1, 2, 4, ... < n every pair (i, i + h) with bit h of i clear
 *            becomes (RN(a + b), RN(a - b))), then multiplied by 2^-shift
 *            (exact): shift = ceil(log2(n) / 2) for activations
 *            (fp4_quantize_act_ex, fp4_gemm_fused_ex) and floor(log2(n) / 2)
 *            for weights (fp4_quantize_weights_ex), so that a rotated
 *            activation times a weight rotated with the same n gives the
 *            plain product: H H^T = n I.  Needs K % n == 0 (always true for
 *            K % 32 == 0).  "FP4 on a consumer RTX 5090: the Blackwell
 *            headline loses to plain int4", section "Finding 3 -- the
 *            real-FP4 path (QuTLASS MXFP4)" (the online Hadamard rotation +
 *            activation quantization every layer pays).
 *  mx_rule   MXFP4 shared-exponent rule.  FP4_MX_RULE_OCP: e = floor(log2
 *            amax_b) - 2 (values in (6, 8) * 2^e clip to 6).
 *            FP4_MX_RULE_OAS (overflow-aware): the smallest e with
 *            amax_b <= 6 * 2^e, so no value of the block saturates ("FP4
 *            n'existe pas", section "L'ecart de qualite -- et comment il se
 *            reduit").  Both clamp e to [-127, 127].  Must be
 *            FP4_MX_RULE_OCP for NVFP4 (FP4_ERR_INVALID_ARG otherwise). */
typedef enum { FP4_MX_RULE_OCP = 0, FP4_MX_RULE_OAS = 1 } fp4_mx_rule_t;
typedef struct {
    int hadamard;
    fp4_mx_rule_t mx_rule;
    /* MXFP4 macro-block scaling (MBS; "FP4 n'existe pas", section "L'ecart
     * de qualite -- et comment il se reduit": a second-level scale over a
     * macro-block of several 32-blocks, the base format unchanged).  Here a
     * macro-block is one row (all K / 32 blocks of a token or an output
     * channel), so that fp4_gemm_mbs applies the second level in its
     * epilogue.  NULL: off.  Otherwise a DEVICE array of `rows` floats that
     * the call writes: per row, with A its largest magnitude, sigma = the
     * significand of RN(A / 6) (in [1, 2); 1 for an all-zero row); the row
     * is multiplied by RN(1 / sigma) (one rounding per value) before the
     * MXFP4 quantizer (mx_rule applies), so that x_hat = sigma * 2^e * q.
     * MXFP4 only, without rotation (FP4_ERR_INVALID_ARG otherwise); not
     * accepted by fp4_gemm_fused_ex or fp4_gemm_quant.  A non-finite row
     * maximum is reported as FP4_ERR_NONFINITE by fp4_device_status. */
    float* mbs_scale;
} fp4_quant_opts_t;

/* fp4_quantize_act with options (above).  opts == NULL is fp4_quantize_act.
 * FP4_ERR_INVALID_ARG for a hadamard other than 0, 16, 32 or an unknown
 * rule. */
fp4_status_t fp4_quantize_act_ex(const void* x, int rows, int K, fp4_format_t fmt,
                                 fp4_scale_layout_t layout, fp4_global_mode_t gmode,
                                 const fp4_quant_opts_t* opts, float* g, uint8_t* codes,
                                 uint8_t* scales, void* ws, size_t ws_bytes, void* stream);

/* One-time weight quantization at load time ("fp4-cuda-kernel" forum post:
 * quantize weights once at model load).  Same arithmetic as
 * fp4_quantize_act with DYNAMIC global scale and scales written in the MMA
 * layout.  w: bf16 [N, K]; g: NVFP4 out (may be NULL for MXFP4). */
fp4_status_t fp4_quantize_weights(const void* w, int N, int K, fp4_format_t fmt,
                                  uint8_t* codes, uint8_t* scales, float* g,
                                  void* ws, size_t ws_bytes, void* stream);

/* fp4_quantize_weights with options (the weight shift of the rotation). */
fp4_status_t fp4_quantize_weights_ex(const void* w, int N, int K, fp4_format_t fmt,
                                     const fp4_quant_opts_t* opts, uint8_t* codes,
                                     uint8_t* scales, float* g, void* ws, size_t ws_bytes,
                                     void* stream);

/* Block-scaled FP4 GEMM on the tcgen05 tensor cores:
 *     C[M, N] = alpha * A_hat[M, K] . W_hat[N, K]^T
 * A and W are both K-major packed codes with MMA-layout scales (as written
 * by the two quantizers above).  alpha = RN(g_a * g_w) for NVFP4 (g_a, g_w
 * are device pointers) and 1 for MXFP4 (g_a, g_w may be NULL).  The sum is
 * accumulated in FP32 in tensor memory; C = RN(alpha * acc) is written as
 * bf16 (round to nearest even) or fp32, row-major with leading dimension
 * ldc (elements).  Any M >= 0 (no padding asked of the caller), N % 8 == 0.
 * The launch shape follows the problem (fp4_gemm_plan): when output tiles
 * are few, K may be split over a thread-block cluster whose partial sums are
 * added in a fixed order, so repeated calls give identical bits.
 * max_sms: the SMs the launch shape is chosen for (0 = the whole device).
 * A caller that runs several GEMMs at once on different streams gives each
 * its share, so that their CTAs run side by side; it changes the tile width
 * and K split (hence the FP32 summation order), never the arithmetic.
 * The pages' W4A4 GEMM: "fp4-cuda-kernel" forum post; cuBLAS's refusal of
 * M < 128 that this entry point does not share: "Hardware FP4 inference for
 * speech on Blackwell", section "Do the FP4 tensor cores even engage?". */
fp4_status_t fp4_gemm(const uint8_t* a_codes, const uint8_t* a_scales, const float* g_a,
                      const uint8_t* w_codes, const uint8_t* w_scales, const float* g_w,
                      int M, int N, int K, fp4_format_t fmt,
                      void* C, int ldc, fp4_out_t out,
                      void* ws, size_t ws_bytes, int max_sms, void* stream);

/* Small-M path (decode): quantize the bf16 activation a [M, K] on the fly
 * and multiply it with pre-quantized weights.  Small activations (M*K up to
 * 32768 values) take ONE kernel: every CTA streams its weight tile from its
 * first instruction, then takes the activation's global amax, quantizes its
 * own K slice into shared memory and runs its MMAs.  Larger ones are a
 * chain of programmatic dependent launches on `stream`: amax (DYNAMIC only)
 * -> quantize (into the workspace) -> a swap-AB, split-K tcgen05 GEMM for
 * M <= 32 that starts streaming the weights before the quantized activation
 * is ready.  Either way the kernels may begin reading w_codes / w_scales
 * before the kernel preceding them on `stream` has finished, so the
 * weights must not be written by that kernel (quantize them earlier, as at
 * load time, or synchronize the stream first).
 * "FP4 n'existe pas", runtime survey (quantization, scaling, matmul and
 * de-scaling chained in one go); the small-M regime: "Hardware FP4
 * inference for speech on Blackwell", section "Do the FP4 tensor cores even
 * engage?".  g_a: DYNAMIC writes it, STATIC reads it (NVFP4; MXFP4 ignores
 * it).  Results equal fp4_quantize_act followed by fp4_gemm up to FP32
 * summation order; the split-K reduction runs in a fixed order, so repeated
 * calls give identical bits.  Requires 1 <= M <= 32 (M == 0 is a no-op;
 * FP4_ERR_UNSUPPORTED_SHAPE above 32).  The workspace (fp4_workspace_bytes)
 * holds the partial maxima and the quantized activation.  max_sms as for
 * fp4_gemm: the SMs the K split is chosen for (0 = all). */
fp4_status_t fp4_gemm_fused(const void* a, const uint8_t* w_codes, const uint8_t* w_scales,
                            const float* g_w, int M, int N, int K, fp4_format_t fmt,
                            fp4_global_mode_t gmode, float* g_a,
                            void* C, int ldc, fp4_out_t out,
                            void* ws, size_t ws_bytes, int max_sms, void* stream);

/* fp4_gemm_fused with quantizer options for the activation (the activation
 * shift of the rotation; the weights must have been quantized by
 * fp4_quantize_weights_ex with the same hadamard order).  opts == NULL is
 * fp4_gemm_fused. */
fp4_status_t fp4_gemm_fused_ex(const void* a, const uint8_t* w_codes, const uint8_t* w_scales,
                               const float* g_w, int M, int N, int K, fp4_format_t fmt,
                               fp4_global_mode_t gmode, const fp4_quant_opts_t* opts,
                               float* g_a, void* C, int ldc, fp4_out_t out,
                               void* ws, size_t ws_bytes, int max_sms, void* stream);

/* Block-scaled FP4 GEMM whose epilogue emits the next layer's FP4
 * activation: C = alpha * A_hat . W_hat^T as fp4_gemm computes it, rounded
 * to bf16 exactly as fp4_gemm writes it, then quantized in the same launch
 * (no HBM round trip of C) with the activation quantizer's arithmetic:
 * NVFP4 with the STATIC global scale *g_out (a DYNAMIC scale would need the
 * whole C before any block could be coded), or MXFP4 (g_out ignored, may be
 * NULL), with out_opts' rotation (activation shift) and MXFP4 rule.  The
 * results equal fp4_quantize_act_ex(STATIC g_out) applied to that bf16 C,
 * bit for bit.
 *   out_codes   [M, N/2] packed codes; out_scales in out_layout for a
 *               [M, N] tensor (the MMA order pads rows to 128 and scale
 *               columns to 4, written as 0), i.e. what the next fp4_gemm
 *               takes as its activation with K = N.
 *   C, ldc      optional: when C is not NULL the bf16 C is stored as well
 *               (row-major, leading dimension ldc).
 * N % 32 == 0 (N is the next layer's K).  The launch shape is fp4_gemm's
 * without a K split (every output row of a tile is quantized by the thread
 * that holds it), so for shapes where fp4_gemm_plan reports a split the
 * FP32 summation order can differ from fp4_gemm's.  ws unused (may be
 * NULL).  "FP4 n'existe pas : il existe des FP4, et chaque runtime choisit
 * son dialecte", section "TensorRT-LLM 1.3 : NVFP4 natif, verrouille
 * NVIDIA" (quantization, scaling, matmul and de-scaling in one launch, no
 * HBM round trip between the steps). */
fp4_status_t fp4_gemm_quant(const uint8_t* a_codes, const uint8_t* a_scales, const float* g_a,
                            const uint8_t* w_codes, const uint8_t* w_scales, const float* g_w,
                            int M, int N, int K, fp4_format_t fmt, fp4_format_t out_fmt,
                            fp4_scale_layout_t out_layout, const fp4_quant_opts_t* out_opts,
                            const float* g_out, uint8_t* out_codes, uint8_t* out_scales,
                            void* C, int ldc, void* ws, size_t ws_bytes, int max_sms,
                            void* stream);

/* MXFP4 GEMM with macro-block scaling: A and W quantized with
 * fp4_quant_opts_t.mbs_scale (fp4_quantize_act_ex, fp4_quantize_weights_ex)
 * and their per-row macro scales sigma_a [M], sigma_w [N] (device arrays):
 *     C[m, n] = RN(RN(sigma_a[m] * sigma_w[n]) * acc[m, n]),
 * acc the FP32 block-scaled accumulation of the MXFP4 codes and E8M0
 * scales (as fp4_gemm), bf16 or fp32 out.  The launch shape is fp4_gemm's
 * without a K split.  Shapes, alignment and errors as fp4_gemm (sigma
 * pointers 4-byte aligned, never NULL).  "FP4 n'existe pas", section
 * "L'ecart de qualite -- et comment il se reduit" (the GEMM pays a small
 * overhead for the second level). */
fp4_status_t fp4_gemm_mbs(const uint8_t* a_codes, const uint8_t* a_scales, const float* sigma_a,
                          const uint8_t* w_codes, const uint8_t* w_scales, const float* sigma_w,
                          int M, int N, int K, void* C, int ldc, fp4_out_t out,
                          void* ws, size_t ws_bytes, int max_sms, void* stream);

/* Grouped block-scaled FP4 GEMM (mixture of experts: many per-expert GEMMs
 * in one launch).  Group e (0 <= e < E) is rows [offsets[e], offsets[e+1])
 * of A and C and expert weight e:
 *     C[r, :] = alpha_e * A_hat[r, :] . W_hat_e^T   for r in group e,
 * alpha_e = RN(g_a * g_w[e]) (NVFP4; 1 for MXFP4), FP32 accumulation in
 * tensor memory, bf16 (round to nearest even) or fp32 out.
 *   a_codes, a_scales, g_a   the routed activation [M, K] as written by
 *               fp4_quantize_act (MMA scale order, one global scale for all
 *               rows); groups may start on any row.
 *   w_codes     E experts' packed codes back to back, [E, N, K/2];
 *   w_scales    E per-expert MMA-order scale blocks back to back, each
 *               fp4_scale_bytes(N, K, fmt, FP4_SCALES_MMA) bytes (what
 *               fp4_quantize_weights writes for one expert);
 *   g_w         E global scales (NVFP4; may be NULL for MXFP4);
 *   offsets     DEVICE array of E + 1 ints, offsets[0] = 0, non-decreasing,
 *               offsets[E] = M (routing results stay on the device; no host
 *               synchronization).  Out-of-range or decreasing entries are
 *               clamped into [0, M] and made non-decreasing, so no row
 *               outside A and C is read or written.
 * 1 <= E <= 256, N % 8 == 0, K % 32 == 0.  Empty groups are allowed.  Every
 * tile has all of K (no split): 256 x 256 tiles on CTA pairs when the
 * groups average at least 512 rows (M >= 512 E), N > 128 and the pair
 * tiles keep at least half the SMs busy, else 128 x 256 tiles (N > 128) or
 * 128 x 128.  ws unused (may be NULL).
 * "FP4 n'existe pas : il existe des FP4, et chaque runtime choisit son
 * dialecte", section "Les runtimes et leurs dialectes : qui parle quoi"
 * (fused NVFP4 MoE kernels, W4A4 MegaMoE). */
fp4_status_t fp4_gemm_grouped(const uint8_t* a_codes, const uint8_t* a_scales, const float* g_a,
                              const uint8_t* w_codes, const uint8_t* w_scales, const float* g_w,
                              const int* offsets, int E, int M, int N, int K, fp4_format_t fmt,
                              void* C, int ldc, fp4_out_t out, void* ws, size_t ws_bytes,
                              int max_sms, void* stream);

/* The launch shape fp4_gemm takes for an M x N x K problem on the current
 * device, for tests and profiling (nothing is launched; the pages have no
 * counterpart).  *tile_m x *tile_n output tiles (256 x 256: the CTA-pair
 * kernel; 128 x {256, 128, 64}: one CTA per tile) and *splits CTAs per tile
 * along K: a thread-block cluster whose CTAs each accumulate one slice of K
 * and then add their FP32 partial sums in a fixed order (split 0 first), so
 * repeated calls give identical bits.  Narrow tiles and splits are taken
 * when 256-wide tiles would leave most of the max_sms SMs (0 = all of the
 * device's) idle.  Errors as fp4_gemm's shape checks, FP4_ERR_INVALID_ARG
 * for a NULL output pointer or a negative max_sms. */
fp4_status_t fp4_gemm_plan(int M, int N, int K, fp4_format_t fmt, int max_sms,
                           int* tile_m, int* tile_n, int* splits);

/* Activation quantization without a workspace argument, for callers that
 * cannot allocate device memory: engines that reserve all device memory at
 * start-up for weights and caches and allow no later allocation, plug-ins
 * that run inside a host framework which owns the allocator and hands them
 * no scratch, and latency-critical paths that cannot pay for cudaMalloc's
 * implicit device synchronization.  The pages have no counterpart of this
 * entry point.
 * Same arguments (minus ws / ws_bytes), arithmetic and results as
 * fp4_quantize_act.  The DYNAMIC global-scale reduction keeps its partial
 * maxima in a fixed 4 KiB device array inside the library instead of a
 * caller workspace; the array exists on every GPU that loads the library
 * until the process exits.  Limit: the call is rejected with
 * FP4_ERR_WORKSPACE_TOO_SMALL if the scratch that fp4_quantize_act needs for
 * this size (the same rule) exceeds those 4 KiB; today that need is 4 KiB
 * for every accepted size.  The first DYNAMIC call on a device looks up the
 * array's device address (cudaGetSymbolAddress, once per device); make that
 * first call before any stream capture.  All calls share the array: calls
 * that overlap on the GPU (other streams, other host threads on the same
 * device) race and must not be issued.  The array keeps the last call's
 * contents; no clearing is needed since every call writes each slot before
 * reading it.  No cudaMalloc / cudaFree or other allocating call is made. */
fp4_status_t fp4_quantize_act_noalloc(const void* x, int rows, int K, fp4_format_t fmt,
                                      fp4_scale_layout_t layout, fp4_global_mode_t gmode,
                                      float* g, uint8_t* codes, uint8_t* scales,
                                      void* stream);

/* Reads and clears, in one atomic exchange on the device, the library's
 * status word: kernels OR a bit into it when one of their bounded waits runs
 * out (bits 0-6) and when a DYNAMIC global-scale reduction meets a
 * non-finite input (bit 7, FP4_STATUS_NONFINITE_BIT).  A bit set by a kernel
 * on another stream is never lost: it is either returned by this call or
 * left for the next, also when several host threads call this at once
 * (their calls are serialized).  Synchronizes `stream` (the exchange runs on
 * it after the work queued before).  *code receives the raw word (0 = nothing
 * happened).  Returns FP4_ERR_DEVICE_TIMEOUT if a wait ran out, else
 * FP4_ERR_NONFINITE if only the non-finite bit was set, else FP4_OK.
 * Non-finite inputs are outside the format's contract ("Hardware FP4
 * inference for speech on Blackwell", section "NVFP4, and the two ways it
 * fails": the scale saturates, never NaN): the reduction still derives a
 * finite g from the largest finite bf16 (so no NaN reaches g or alpha), and
 * the status word reports the input. */
#define FP4_STATUS_NONFINITE_BIT 0x80u
fp4_status_t fp4_device_status(unsigned* code, void* stream);

/* Self-test of the failure detection (the pages have no counterpart): one
 * kernel waits on a device barrier that nothing signals, with a bounded wait
 * of limit_ns (0 < limit_ns <= 1 s), then sets the watchdog word and
 * returns, as every kernel of this library does when one of its waits runs
 * out.  A following fp4_device_status returns FP4_ERR_DEVICE_TIMEOUT and the
 * CUDA context stays usable.  Nothing is faulted, trapped or hung. */
fp4_status_t fp4_watchdog_selftest(unsigned long long limit_ns, void* stream);

/* A static string naming the status (never NULL). */
const char* fp4_status_string(fp4_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* FP4_B200_H */
