/*
 * lora_gemm.h -- C ABI of the B200 (sm_100a) merged-LoRA refiner hot path.
 *
 * The operations come from the Open-H3-Regenerate-2K pages:
 *
 *   lg_lora_merge   "Open-H3-Regenerate-2K：MiniMax H3 的开源 4K 精修方案"
 *                   (comfyui-wiki.com news), section "三个步如何完成工作":
 *                   adapters merged by concatenating factors along the rank
 *                   axis (384 + 128 + 64 = 576), stored in FP32.
 *   lg_lora_linear  the frozen transformer's linear layer carrying that merged
 *                   LoRA ("Open-H3-Regenerate-2K: High-Resolution Video
 *                   Refinement with Few-Step Diffusion", section "The
 *                   four-stage refinement pipeline"):
 *                   y = x W^T + (x A_cat^T) B_cat^T.
 *   lg_renoise      same page, section "Three steps instead of dozens":
 *                   z = (1 - sigma0) z_up + sigma0 eps, eps ~ N(0, I).
 *   lg_euler_step   same section: z_{k+1} = z_k + (sigma_{k+1} - sigma_k) v on
 *                   the schedule 0.909 -> 0.857 -> 0.667 -> 0.
 *
 * and, from the same article's section "Where the 3.9x speedup comes from":
 *
 *   lg_mx_quantize, lg_lora_linear_mxfp8   the linear layer with its base term
 *                   as MXFP8 GEMMs, activations re-quantized per call;
 *   lg_lora_linear_swiglu_mxfp8   the MLP input projection with SwiGLU and
 *                   the activation quantizer fused;
 *   lg_lora_linear_euler   the step's last projection with the Euler update
 *                   (and the bf16 copy of the new latent) fused;
 *   lg_shift_ladder the sampler routes of "Open-H3-Regenerate-2K-IC"
 *                   (wujieai.com) on HyperFlow's shift-12 table (host only);
 *   lg_lora_linear_noalloc   lg_lora_linear without a caller workspace.
 *
 * The pages name no random number generator.  This library draws eps from a
 * Philox4x32-10 stream (Salmon et al., "Parallel Random Numbers: As Easy as
 * 1, 2, 3", SC'11) with key = (seed mod 2^32, seed >> 32) and counter
 * (j mod 2^32, j >> 32, 0, 0) for 4-element block j, turned into normals by
 * the Box-Muller transform (see lg_philox_normal).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers on the current CUDA device,
 *     owned by the caller.  The library allocates no device memory; the
 *     scratch that lg_lora_linear needs is the caller's workspace.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls are asynchronous on that stream.  The return value
 *     reports argument validation and launch errors only; a device-side
 *     timeout is reported later by lg_get_last_device_error().
 *   - Arguments are validated before anything is launched; on any error
 *     nothing is launched and nothing is written.
 *   - Kernels are compiled for sm_100a only; on another device every compute
 *     entry point returns LG_ERR_NOT_SM100.
 *   - Element counts of zero are valid and launch nothing.
 */
#ifndef LORA_GEMM_H
#define LORA_GEMM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum lg_status {
  LG_OK = 0,
  LG_ERR_INVALID_ARG = 1,       /* null pointer, negative size, bad sigma, ... */
  LG_ERR_UNSUPPORTED_SHAPE = 2, /* a dimension outside the supported set */
  LG_ERR_MISALIGNED = 3,        /* a pointer not aligned as documented */
  LG_ERR_WORKSPACE = 4,         /* workspace missing or too small */
  LG_ERR_CUDA = 5,              /* a CUDA runtime/driver call failed */
  LG_ERR_DEVICE_TIMEOUT = 6,    /* a bounded wait inside a kernel ran out */
  LG_ERR_NOT_SM100 = 7          /* current device is not compute capability 10.0 */
} lg_status;

/* Short English description of a status code (static storage). */
const char* lg_status_string(int status);

/* Library version as 10000*major + 100*minor + patch. */
int lg_version(void);

/* Number of kernels this library has launched in this process (all devices).
 * A monotone counter; callers take differences around a region of interest. */
uint64_t lg_launch_count(void);

/* Synchronizes `stream`, then reads and clears the current device's error
 * word.  Returns LG_OK if no kernel recorded an error since the last call,
 * LG_ERR_DEVICE_TIMEOUT if a bounded wait in a kernel gave up (the kernel
 * then abandoned its work, drained its own copies, freed its tensor memory
 * and returned; its outputs are undefined), or LG_ERR_CUDA if the
 * synchronization itself failed. */
lg_status lg_get_last_device_error(void* stream);

/* Upper bound, in nanoseconds, on any single wait inside lg_lora_linear's
 * pipeline (default 4e9).  Process-wide; applies to launches made after the
 * call.  0 restores the default.  Meant for fault-injection tests: a tiny
 * limit makes the waits run out so the timeout path can be exercised. */
void lg_set_wait_limit_ns(uint64_t limit_ns);

/* Thread-block cluster size of lg_lora_linear: the CTAs (one per SM) that
 * share one panel of x -- 1, 2, 4 or 8 -- or 0 (the default) to choose
 * per shape.  Sharing a panel lets the cluster's CTAs split the N tiles while
 * the panel is read from DRAM once; each computes its slice of the rank-R
 * intermediate and they exchange the slices through distributed shared
 * memory.  For the SM-pair variant the size counts both CTAs of each pair
 * (2, 4 or 8).  Process-wide; for tuning and tests.  Returns
 * LG_ERR_INVALID_ARG for other values. */
lg_status lg_set_cluster_size(int g);

/* MMA variant of lg_lora_linear: 1 = single-SM tcgen05.mma (128 x 224
 * tiles), 2 = SM-pair tcgen05.mma.cta_group::2 (256 x 256 tiles, each SM
 * loads half of every B tile), 0 (the default) = chosen per shape (single-SM
 * for K <= 2048, pairs beyond).  Process-wide; for
 * tuning and tests.  Returns LG_ERR_INVALID_ARG for other values. */
lg_status lg_set_kernel_variant(int v);

/* ------------------------------------------------------------------------
 * lg_lora_merge -- concatenate n_adapters LoRA adapters along the rank axis.
 *
 *   A_cat[off_i + r][k] = scales[i] * A[i][r][k]      (FP32, one rounding)
 *   B_cat[o][off_i + r] = B[i][o][r]                  (FP32, exact copy)
 *
 * with off_i = ranks[0] + ... + ranks[i-1] and R = sum of ranks, so that
 * B_cat A_cat = sum_i scales[i] B_i A_i.  The scale sits on A (the pages do
 * not say which factor carries it).
 *
 *   A, B        HOST arrays of n_adapters DEVICE pointers.  A[i] is row-major
 *               [ranks[i], d_in] FP32; B[i] is row-major [d_out, ranks[i]].
 *   ranks       HOST array, each >= 1 and a multiple of 4.
 *   scales      HOST array of n_adapters FP32 scales.
 *   A_cat       DEVICE [R, d_in] FP32 row-major (output).
 *   B_cat       DEVICE [d_out, R] FP32 row-major (output).
 *   1 <= n_adapters <= 8; d_in, d_out >= 1 and multiples of 4; all device
 *   pointers 16-byte aligned (else LG_ERR_MISALIGNED).  Outputs must not
 *   overlap inputs.
 * ---------------------------------------------------------------------- */
lg_status lg_lora_merge(int n_adapters, const float* const* A, const float* const* B,
                        const int* ranks, const float* scales, int d_in, int d_out,
                        float* A_cat, float* B_cat, void* stream);

/* Bytes of workspace lg_lora_linear needs for this shape (bf16 copies of the
 * merged factors, each padded to 256 bytes).  Returns 0 when no workspace is
 * needed (R = 0) or the shape is unsupported (lg_lora_linear then says
 * which argument is wrong). */
size_t lg_lora_linear_workspace_size(int64_t M, int K, int N, int R);

/* ------------------------------------------------------------------------
 * lg_lora_linear -- merged-LoRA linear layer over latent tokens:
 *
 *   y = x W^T + (x A_cat^T) B_cat^T
 *
 *   x      DEVICE [M, K] bf16 row-major (token activations).
 *   W      DEVICE [N, K] bf16 row-major (frozen weight, y = x W^T).
 *   A_cat  DEVICE [R, K] FP32 row-major (merged down-projection factor).
 *   B_cat  DEVICE [N, R] FP32 row-major (merged up-projection factor).
 *   y      DEVICE [M, N] bf16 row-major (output, round-to-nearest-even).
 *   workspace, ws_bytes  DEVICE scratch of at least
 *          lg_lora_linear_workspace_size(M, K, N, R) bytes; contents on
 *          entry are ignored and clobbered.
 *
 * Arithmetic: the FP32 factors are rounded to bf16 (RNE) for the tensor
 * cores; all products accumulate in FP32; the rank-R intermediate
 * h = x A_cat^T is rounded to bf16 and kept on chip (tensor memory), never
 * written to global memory.
 *
 * Shapes: M >= 0 (0 launches nothing; M < 2^31); K a multiple of 64 and
 * >= 64; N a multiple of 32 and >= 32; R a multiple of 64 with
 * 0 <= R <= 576 (R = 0: plain GEMM, A_cat and B_cat may be NULL).  All
 * pointers 16-byte aligned.  y must not overlap x, W, A_cat, B_cat or the
 * workspace.
 * ---------------------------------------------------------------------- */
lg_status lg_lora_linear(const void* x, const void* W, const float* A_cat, const float* B_cat,
                         void* y, int64_t M, int K, int N, int R,
                         void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * lg_lora_linear_mxfp8 -- the merged-LoRA linear layer with the base term as
 * MXFP8 GEMMs ("Open-H3-Regenerate-2K: High-Resolution Video Refinement with
 * Few-Step Diffusion", section "Where the 3.9x speedup comes from"):
 *
 *   y = deq(x_codes, x_scales) deq(W_codes, W_scales)^T + (x A_cat^T) B_cat^T
 *
 * with deq the exact values of lg_mx_quantize's output (code value times the
 * block's 2^e); the LoRA term is that of lg_lora_linear, from the bf16 x.
 *
 *   x                  DEVICE [M, K] bf16 (the activations x_codes came from).
 *   x_codes, x_scales  DEVICE lg_mx_quantize(x) output ([M, K] codes,
 *                      lg_mx_scale_bytes(M, K) scale bytes).
 *   W_codes, W_scales  DEVICE lg_mx_quantize(W) output for W [N, K].
 *   A_cat, B_cat, y, workspace, ws_bytes  as for lg_lora_linear.
 *
 * Arithmetic: tcgen05.mma kind::mxf8f6f4 with E8M0 block scales for the
 * base term, FP32 accumulation; the LoRA term as in lg_lora_linear.
 * Shapes: as lg_lora_linear, and K a multiple of 128.  All pointers 16-byte
 * aligned; y must not overlap any input or the workspace.
 * ---------------------------------------------------------------------- */
lg_status lg_lora_linear_mxfp8(const void* x, const void* x_codes, const void* x_scales, const void* W_codes,
                               const void* W_scales, const float* A_cat, const float* B_cat, void* y,
                               int64_t M, int K, int N, int R, void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * lg_lora_linear_swiglu_mxfp8 -- the MLP's input projection with SwiGLU and
 * the activation quantizer fused into its epilogue ("Open-H3-Regenerate-2K:
 * High-Resolution Video Refinement with Few-Step Diffusion", section "Where
 * the 3.9x speedup comes from": fused SwiGLU with MXFP8, one-pass activation
 * quantization):
 *
 *   z = deq(x_codes) deq(W_codes)^T + (x A_cat^T) B_cat^T     [M, 2F]
 *   s = silu(z[:, :F]) * z[:, F:]                             [M, F]
 *   (out_codes, out_scales) = MXFP8 of s (the lg_mx_quantize rule and layout)
 *
 * W has 2F rows: the F gate rows, then the F up rows (this library's layout;
 * converters must order the halves so); B_cat is [2F, R] in the same order.
 * The products are formed, quantized and written from the FP32 accumulator:
 * z is never stored.  silu(g) = g / (1 + e^-g) in FP32.
 *
 *   out_codes   DEVICE [M, F] uint8.
 *   out_scales  DEVICE lg_mx_scale_bytes(M, F) bytes.
 *   workspace   lg_lora_linear_workspace_size(M, K, 2F, R) bytes.
 *   other arguments as for lg_lora_linear_mxfp8 with N = 2F.
 *
 * Shapes: F a multiple of 128; K a multiple of 128; R as for lg_lora_linear.
 * ---------------------------------------------------------------------- */
lg_status lg_lora_linear_swiglu_mxfp8(const void* x, const void* x_codes, const void* x_scales, const void* W_codes,
                                      const void* W_scales, const float* A_cat, const float* B_cat, void* out_codes,
                                      void* out_scales, int64_t M, int K, int F, int R, void* workspace,
                                      size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * lg_lora_linear_euler -- the step's last projection (token activations to
 * the latent's velocity channels) with the Euler update of "Open-H3-
 * Regenerate-2K: High-Resolution Video Refinement with Few-Step Diffusion",
 * section "Three steps instead of dozens", folded into its epilogue:
 *
 *   v = x W^T + (x A_cat^T) B_cat^T                    [M, N], FP32, not stored
 *   z[f][c][p] = fmaf(sigma_next - sigma, v[f T + p][c], z[f][c][p])
 *   z_bf16[f][c][p] = bf16(z[f][c][p])  (round to nearest even; next input)
 *
 * Token m is cell p = m mod T of frame f = m / T (T = frame_tokens, the H W
 * cells of one latent frame), and the latent keeps its [frames, channels,
 * cells] layout (the [F, C, H, W] latent with N = C channels).  The step
 * sigma_next - sigma is rounded to FP32 first, as in lg_euler_step; v is the
 * FP32 accumulator itself (lg_lora_linear would round it to bf16).
 *
 *   x, W, A_cat, B_cat  as for lg_lora_linear (W [N, K], B_cat [N, R]).
 *   z       DEVICE [M / T, N, T] FP32, updated in place.
 *   z_bf16  DEVICE [M / T, N, T] bf16, written; or NULL to skip the copy.
 *   frame_tokens  T >= 1, M a multiple of T.
 *   workspace, ws_bytes  at least lg_lora_linear_euler_workspace_size(M, K,
 *          N, R) bytes (R = 0: none).
 *
 * Shapes: K and R as for lg_lora_linear; any N >= 1 (one tile covers
 * N <= 224, and its MMAs then run with N rounded up to 16).  Variant as for
 * lg_lora_linear (lg_set_kernel_variant applies: single-SM for K <= 2048,
 * SM pairs beyond), always with one CTA or pair per panel
 * (lg_set_cluster_size does not apply).  z and z_bf16 must not overlap each
 * other, an input or the workspace.
 * ---------------------------------------------------------------------- */
size_t lg_lora_linear_euler_workspace_size(int64_t M, int K, int N, int R);
lg_status lg_lora_linear_euler(const void* x, const void* W, const float* A_cat, const float* B_cat, float* z,
                               void* z_bf16, int64_t M, int K, int N, int R, int64_t frame_tokens, float sigma,
                               float sigma_next, void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * lg_lora_linear_noalloc -- lg_lora_linear for callers that cannot allocate
 * device memory.  The pages have no counterpart; this is an interface
 * addition of this library.
 *
 * Some callers have no device allocator at the point of the call: a plugin
 * inside an inference engine whose device memory is planned before the run
 * and which may not allocate when it is enqueued, or a serving loop that must
 * never call cudaMalloc (it synchronizes the device and stalls every other
 * stream).  They cannot provide lg_lora_linear's workspace.  This entry point
 * takes the same arguments minus the workspace and keeps the bf16 copies of
 * the merged factors in an array of LG_NOALLOC_SCRATCH_BYTES that is part of
 * the library's device image: every GPU on which the library's kernels are
 * loaded holds that memory until the process exits.  The call itself
 * allocates nothing (no cudaMalloc, cudaFree or allocating library routine).
 *
 *   - Result, validation, arithmetic and kernels are those of lg_lora_linear;
 *     its argument checks run first, so a bad argument gives the status
 *     lg_lora_linear would give, before any CUDA call.
 *   - Limit: lg_lora_linear_workspace_size(M, K, N, R) must not exceed
 *     LG_NOALLOC_SCRATCH_BYTES (about 2 (K + N) R bytes; with R = 576 this is
 *     K + N <= 43,690, e.g. the 7168 -> 7168, 7168 -> 21504 and
 *     28672 -> 7168 layers); a larger shape returns LG_ERR_WORKSPACE and
 *     launches nothing.
 *   - The first call on a device looks up the array's device address on that
 *     device (cudaGetSymbolAddress, with that device current); make that
 *     first call before any stream capture.  The address belongs to the
 *     current CUDA context: it is cached per device and context, so the first
 *     call after a context was destroyed and recreated (cudaDeviceReset), or
 *     under another context, looks it up again (and is then also a first
 *     call in the sense above).
 *   - Every call uses the same array.  Calls that can overlap on the GPU
 *     (different streams without ordering between them) race on it; keep
 *     such calls on one stream or order them with events.
 * ---------------------------------------------------------------------- */
#define LG_NOALLOC_SCRATCH_BYTES ((size_t)48 << 20)
lg_status lg_lora_linear_noalloc(const void* x, const void* W, const float* A_cat, const float* B_cat,
                                 void* y, int64_t M, int K, int N, int R, void* stream);

/* ------------------------------------------------------------------------
 * lg_mx_quantize -- MXFP8 quantization of bf16 rows along K.  "Open-H3-
 * Regenerate-2K: High-Resolution Video Refinement with Few-Step Diffusion",
 * section "Where the 3.9x speedup comes from", runs the linear layers as MXFP8
 * GEMMs with the activations re-quantized at every stage; the pages name the
 * format only, so the block rule is the OCP Microscaling (MX) one:
 *
 *   blocks of 32 consecutive values along K share the scale 2^e with
 *   e = floor(log2 max|v|) - 8 clamped to [-127, 127] (-127 for an all-zero
 *   block), stored as the E8M0 byte e + 127; each value becomes the E4M3
 *   (OCP E4M3FN) code of v 2^-e, round to nearest even, saturated at +-448.
 *
 *   in      DEVICE [rows, K] bf16 row-major.
 *   codes   DEVICE [rows, K] uint8 row-major (E4M3 codes).
 *   scales  DEVICE lg_mx_scale_bytes(rows, K) bytes of E8M0 scales, blocked:
 *           rows in groups of 128, K in groups of 128 (four blocks); group
 *           (g, kg) is 512 contiguous bytes at ((g * K / 128) + kg) * 512, the
 *           byte of row r (0..127 in the group) and block b (0..3 in the K
 *           group) at 16 (r mod 32) + 4 (r / 32) + b.  Rows past `rows`, up to
 *           the next multiple of 128, get byte 0.
 *
 * Shapes: 0 <= rows < 2^31; K a multiple of 128.  in and codes 16-byte
 * aligned; no buffer may overlap another.
 * ---------------------------------------------------------------------- */
size_t lg_mx_scale_bytes(int64_t rows, int K);
lg_status lg_mx_quantize(const void* in, int64_t rows, int K, void* codes, void* scales, void* stream);

/* ------------------------------------------------------------------------
 * lg_renoise -- partial re-noise of an upscaled latent:
 *
 *   x[i] = (1 - sigma) * up[i] + sigma * eps[offset + i],  i in [0, n)
 *
 * eps[e] is element e of the Philox/Box-Muller stream for `seed` (see
 * lg_philox_normal).  The blend is evaluated from the unrounded eps and
 * rounded once to FP32.
 *
 *   up, x   DEVICE FP32 arrays of n elements (flat [F, C, H, W] latent);
 *           x == up (in place) is allowed, partial overlap is not.
 *   sigma   0 <= sigma <= 1.
 *   offset  flat index of up[0] in the global latent; a multiple of 4.
 *   Pointers 16-byte aligned.
 * ---------------------------------------------------------------------- */
lg_status lg_renoise(const float* up, float* x, int64_t n, float sigma, uint64_t seed,
                     uint64_t offset, void* stream);

/* ------------------------------------------------------------------------
 * lg_euler_step -- one flow-matching Euler step, in place:
 *
 *   x[i] = x[i] + (sigma_next - sigma) * v[i]
 *
 * computed as fmaf(sigma_next - sigma, v[i], x[i]) with the difference taken
 * in FP32 (exact for the schedule 0.909 -> 0.857 -> 0.667 -> 0 by
 * Sterbenz's lemma).
 *
 *   x, v    DEVICE FP32 arrays of n elements; must not overlap.
 *   Pointers 16-byte aligned; sigma, sigma_next finite.
 * ---------------------------------------------------------------------- */
lg_status lg_euler_step(float* x, const float* v, int64_t n, float sigma, float sigma_next,
                        void* stream);

/* ------------------------------------------------------------------------
 * lg_shift_ladder -- the sigmas a sampling route visits on a time-shifted
 * flow-matching table.  Host computation only (no device work, no stream):
 *
 *   table_k = shift t_k / (1 + (shift - 1) t_k),  t_k = 1 - k / n_steps,
 *             k = 0..n_steps (1 down to 0), evaluated in double and rounded
 *             to FP32;
 *   ladder  = sigma0, then every table value strictly below sigma0.
 *
 * Page "Open-H3-Regenerate-2K-IC", section "三步接着放大的草稿画，八步从噪声重画":
 * the up3, up4 and hf8 routes share HyperFlow's eight-step table with video
 * shift 12; they start at 0.835, 0.923 and 1 and take 3, 4 and 8 steps.  The
 * page prints no formula; the time shift above is this library's reading of
 * "video shift 12" (it puts the table point at t = 1/2 at 12/13 = 0.923...).
 * The route is then: lg_renoise at ladder[0], lg_euler_step from ladder[k] to
 * ladder[k + 1] for each k.
 *
 *   sigma0   0 < sigma0 <= 1.
 *   n_steps  1 .. 4096.   shift  finite, > 0.
 *   out      HOST FP32 array with room for `cap` values; the ladder has at
 *            most n_steps + 1 values.  *len receives the count.
 *   Returns LG_ERR_INVALID_ARG (writing nothing) for an argument out of range,
 *   null pointers, or cap smaller than the ladder.
 * ---------------------------------------------------------------------- */
lg_status lg_shift_ladder(float sigma0, int n_steps, double shift, float* out, int cap, int* len);

/* ------------------------------------------------------------------------
 * Generator hooks (same generator as lg_renoise), for testing.
 *
 * lg_philox_u32: out[4b + t] = word t of Philox4x32-10(counter of block
 *   block_offset + b, key of seed), b in [0, n_blocks).  out: DEVICE uint32,
 *   4 * n_blocks words, 16-byte aligned.
 *
 * lg_philox_normal: eps[i] = FP32 rounding of element offset + i of the
 *   normal stream.  Element e uses block j = e / 4, slot t = e % 4; words
 *   (a, b) = (r0, r1) for slots 0-1 and (r2, r3) for slots 2-3;
 *   u1 = ((a >> 8) + 1) 2^-24, u2 = (b >> 8) 2^-24; slot 0/2 is
 *   sqrt(-2 ln u1) cos(2 pi u2), slot 1/3 is sqrt(-2 ln u1) sin(2 pi u2).
 *   eps: DEVICE FP32, n elements, 16-byte aligned; offset a multiple of 4.
 * ---------------------------------------------------------------------- */
lg_status lg_philox_u32(uint32_t* out, int64_t n_blocks, uint64_t seed, uint64_t block_offset,
                        void* stream);
lg_status lg_philox_normal(float* eps, int64_t n, uint64_t seed, uint64_t offset, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LORA_GEMM_H */
