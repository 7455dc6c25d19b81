/*
 * fluxdit.h -- C ABI of the B200 (sm_100a) FLUX.2-klein denoising transformer
 * (and of its FLUX.3 Image Klein variant, flux3_dit_*, further below).
 *
 * The library evaluates the velocity field of the FLUX.2-klein image generator
 * once per Euler flow-matching step: 5 double-stream blocks (separate text and
 * image weights, joint attention over the concatenated sequence) and 20
 * single-stream blocks, width 3072, 24 heads of 128 ("Flux 2 Klein: Reine
 * C-basierte Inferenz", section "Modellarchitektur und Leistung"; hakusoku.com
 * story 4662, section "技術詳細"), on image tokens that are 2x2 patches of a
 * 32-channel, 8x-downsampled latent packed to 128 channels ("FLUX.3 Image Klein
 * in Diffusers: Architektur, ...", section "Zweistufiger Transformer und
 * Tokenisierung").
 *
 * Conventions for every entry point:
 *   - Tensor pointers are DEVICE pointers owned by the caller, unless stated.
 *     Layouts are row-major and dense.  "bf16" arrays are uint16_t bit patterns.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream).  Nothing synchronises the host except
 *     flux_dit_create (blob upload) and flux_device_error.
 *   - Return 0 on success or a negative errno-style code: FLUX_EINVAL for a bad
 *     argument (null pointer, shape out of range), FLUX_ENOMEM when a device
 *     allocation fails, FLUX_EIO for a CUDA launch or runtime error.  Pointer
 *     returning calls return NULL on failure.  flux_get_error() then holds a
 *     message for the calling thread.
 *   - Kernels never trap: a pipeline wait that exceeds one second makes the
 *     kernel stop, record a code in a device error word and return;
 *     flux_device_error() reads and clears it.
 *   - Kernels are launched with programmatic dependent launch: a kernel's set-up
 *     may overlap the end of the previous kernel on the stream, and it waits for
 *     that kernel's completion before touching memory, so results do not change.
 *     FLUX_PDL=0 in the environment (read at every launch) turns this off.
 */
#ifndef FLUXDIT_H
#define FLUXDIT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define FLUX_API __attribute__((visibility("default")))
#else
#define FLUX_API
#endif

#define FLUX_OK 0
#define FLUX_EIO (-5)
#define FLUX_ENOMEM (-12)
#define FLUX_EINVAL (-22)

typedef struct flux_dit flux_dit;

/* Model hyper-parameters.  Defaults (FLUX.2-klein): 5, 20, 3072, 24, 128, 9216,
 * 128, 3072, 256, 1e4, 1e-6, 1e-6.  hidden == heads * head_dim, head_dim == 128. */
typedef struct {
  int n_double, n_single, hidden, heads, head_dim, mlp_hidden, in_ch, txt_dim, t_freq_dim;
  float rope_theta, eps_ln, eps_rms;
} flux_dit_config;

/* Last error message of the calling thread ("" if none).  Valid until the next call. */
FLUX_API const char *flux_get_error(void);

/* Code (FLUX_EINVAL, FLUX_ENOMEM, FLUX_EIO) of the calling thread's last failure, 0 if none has
 * happened: lets a caller of a pointer-returning call (flux_dit_create, flux3_dit_create) tell a
 * device out of memory from a bad argument. */
FLUX_API int flux_get_error_code(void);

/* Bytes of a weight blob for `cfg` (header + tensors), or 0 if cfg is invalid.
 *
 * Blob format (little endian): a 256-byte header
 *   char magic[8] = "FLUXDIT\0"; uint32 version = 1; uint32 n_tensors;
 *   int32 n_double, n_single, hidden, heads, head_dim, mlp_hidden, in_ch, txt_dim, t_freq_dim;
 *   float32 rope_theta, eps_ln, eps_rms; uint64 data_offset (= 256); uint64 data_bytes;
 * then every tensor as bf16, row-major, each starting on a 256-byte boundary, in this order:
 *   time_in.{w1 [D,256], b1 [D], w2 [D,D], b2 [D]}, img_in.{w [D,128], b [D]},
 *   txt_in.{w [D,txt_dim], b [D]},
 *   for each double block i, for stream s in (img, txt):
 *     mod.{w [6D,D], b [6D]}        rows: shift1, scale1, gate1, shift2, scale2, gate2
 *     qkv.{w [3D,D], b [3D]}        rows: q, k, v (head h = rows h*128 .. h*128+127)
 *     q_gain [128], k_gain [128]    QK-RMSNorm gains
 *     proj.{w [D,D], b [D]}
 *     mlp_in.{w [2F,D], b [2F]}     rows: a, b of SwiGLU, silu(a) * b
 *     mlp_out.{w [D,F], b [D]}
 *   for each single block i:
 *     mod.{w [3D,D], b [3D]}        rows: shift, scale, gate
 *     lin1.{w [3D+2F,D], b}         rows: q, k, v, a, b
 *     q_gain [128], k_gain [128]
 *     lin2.{w [D,D+F], b [D]}       input: [attention output ; silu(a) * b]
 *   final.mod.{w [2D,D], b [2D]}    rows: shift, scale
 *   final.out.{w [128,D], b [128]}
 * (D = hidden, F = mlp_hidden.) */
FLUX_API size_t flux_blob_expected_bytes(const flux_dit_config *cfg);

/* Create a model from a weight blob in HOST memory (format above).  The blob is
 * copied to the device (and SwiGLU rows re-interleaved for the GEMM epilogue);
 * the caller keeps ownership of `blob`.  `cfg` may be NULL (take the header's),
 * otherwise it must equal the header's.  Synchronises `stream`.  NULL on error. */
FLUX_API flux_dit *flux_dit_create(const void *blob, size_t blob_bytes, const flux_dit_config *cfg, void *stream);

/* Release the model's device memory.  NULL is allowed. */
FLUX_API void flux_dit_destroy(flux_dit *m);

/* One transformer forward: the velocity of the image tokens at time t.
 *   img_tok  fp32 [grid_h*grid_w, 128]    packed noisy latent tokens (flux_pack_latents)
 *   txt      fp32 [n_txt, txt_dim]         text features
 *   ref_tok  fp32 [ref_h*ref_w, 128] or NULL   packed reference-image tokens
 *   v_out    fp32 [grid_h*grid_w, 128]    velocity (written)
 * The joint sequence is text | image | reference; reference tokens use the image
 * stream's weights, the same timestep, and RoPE coordinates (0, row, col, -1)
 * (FLUX.3 Image Klein in Diffusers write-up, section "Modulation pro Token-Typ,
 * Flow-Map-Destillation und 4D-RoPE"); only image tokens reach the output layer
 * (section "Entkoppelte Vorverarbeitung und gemeinsame Attention-Blöcke").
 * Shapes: 4 <= grid_h, grid_w <= 64 (64..1024 px in steps of 16 px, "Flux 2
 * Klein: Reine C-basierte Inferenz", "Build und Ausführung"); ref_h = ref_w = 0
 * or in 4..64; 0 <= n_txt <= 4096.  The first call with a larger sequence grows
 * the model's workspace (cudaMalloc), so it must not be inside a stream capture. */
FLUX_API int flux_dit_forward(flux_dit *m, const float *img_tok, int grid_h, int grid_w, const float *txt, int n_txt,
                     const float *ref_tok, int ref_h, int ref_w, float t, float *v_out, void *stream);

/* One forward with several reference images (at most 10): their packed tokens are
 * concatenated in order in ref_tok (fp32 [sum_k h_k*w_k, 128]); ref_grids is a HOST
 * array of n_refs (h, w) pairs, each in 4..64.  Reference k sits at RoPE coordinate
 * l = -(k+1) ("FLUX.3 Image Klein in Diffusers: ...", section "Modulation pro Token-Typ,
 * Flow-Map-Destillation und 4D-RoPE"; up to ten reference images: we0.ai FLUX.3 Image
 * Klein article).  n_refs = 0 is a text-to-image forward.  Otherwise as flux_dit_forward. */
FLUX_API int flux_dit_forward_refs(flux_dit *m, const float *img_tok, int grid_h, int grid_w, const float *txt,
                                   int n_txt, const float *ref_tok, int n_refs, const int *ref_grids, float t,
                                   float *v_out, void *stream);

/* Classifier-free guidance forward: the velocities of the prompt and of the unconditional
 * text for the same image, references and t, as ONE batch of two sequences (every GEMM
 * and attention launch covers both).  txt_cond and txt_uncond are fp32 [n_txt, 3072]
 * device buffers with the same token count (prompts are padded to one length and the
 * padding is attended: "FLUX.3 Image Klein in Diffusers: ...", section "Verarbeitung
 * einzelner Prompts und Batching-Architektur"); v_cond and v_uncond are distinct fp32
 * [grid_h*grid_w, 128] outputs.  The guidance scale is a sampler parameter (hakusoku.com
 * story 4662, "CライブラリAPI": guidance_scale; base checkpoint: 50 steps at guidance 3.5,
 * we0.ai FLUX 3 Image Klein article, checkpoint table); combine the two velocities with
 * flux_cfg_euler_step.  The workspace holds both sequences (twice the rows of a
 * single-text forward).  Otherwise as flux_dit_forward_refs; each velocity equals, bit for
 * bit, what flux_dit_forward_refs returns for that text alone. */
FLUX_API int flux_dit_forward_cfg(flux_dit *m, const float *img_tok, int grid_h, int grid_w, const float *txt_cond,
                                  const float *txt_uncond, int n_txt, const float *ref_tok, int n_refs,
                                  const int *ref_grids, float t, float *v_cond, float *v_uncond, void *stream);

/* Precision of the block linears (qkv, projection, MLP in / out; linear1 / linear2) of later
 * forwards.  FLUX_PRECISION_BF16 (the default): bf16 operands.  FLUX_PRECISION_FP8: row-wise FP8,
 * the "fp8r" format of the FLUX.3 Image Klein in Diffusers write-up, section "Hardwareanforderungen,
 * Quantisierung und Inferenzlatenz": every weight row and every activation row is quantised to
 * e4m3 with its own fp32 scale (amax / 448; codes e4m3(x * 448 / amax), round to nearest even,
 * saturating), the products are accumulated in fp32 and scaled by both rows' scales.  The first
 * switch to FP8 quantises the block weights once (a device allocation of one byte per weight, and
 * a host synchronisation); the input / output projections, the modulation, attention and the
 * residual stream keep their precision.  Needs hidden in {1024, 2048, 3072, 4096} and
 * hidden + mlp_hidden <= 16384.
 * FLUX_PRECISION_NVFP4: the "nvfp4" format of the same section, which needs a Blackwell GPU: the
 * same operands as 4-bit e2m1 codes with one e4m3 scale per 16 elements and one fp32 scale per
 * row (flux_quantize_rows_nvfp4), multiplied by tcgen05 block-scaled MMAs; the first switch
 * quantises the block weights once (half a byte per weight plus the scales).  Needs hidden in
 * {1024, 2048, 3072, 4096}, mlp_hidden a multiple of 256 and hidden + mlp_hidden <= 16384. */
#define FLUX_PRECISION_BF16 0
#define FLUX_PRECISION_FP8 1
#define FLUX_PRECISION_NVFP4 2
FLUX_API int flux_dit_set_precision(flux_dit *m, int precision);

/* Diagnostic: run only the first n_double double blocks and n_single single
 * blocks in later forwards (-1 = all).  Used to bisect parity; not a model change. */
FLUX_API int flux_dit_set_active_blocks(flux_dit *m, int n_double, int n_single);

/* The modulation vector for time t: SiLU(vec(t)) through every block's
 * modulation linear, fp32 [flux_dit_modulation_size(m)], in blob order of the
 * mod tensors (double i img, double i txt, ..., single i, ..., final). */
FLUX_API size_t flux_dit_modulation_size(const flux_dit *m);
FLUX_API int flux_dit_modulation(flux_dit *m, float t, float *mods_out, void *stream);

/* Compute the modulation vectors of n timesteps (a sampler's schedule, n <= 64, HOST array) in
 * passes of up to four that read the time-MLP and modulation weights once per pass, and keep them:
 * a later forward (or flux_dit_modulation) whose t equals one of them exactly uses the kept vector
 * instead of computing it (the modulation linears read 2.3 GB of weights per forward at the
 * default size; "Modulation pro Token-Typ, Flow-Map-Destillation und 4D-RoPE": shift, scale and
 * gate depend on the timestep only).  A new call replaces the kept set; n = 0 clears it.  Uses a
 * stream-ordered temporary allocation; the first call allocates the cache (64 vectors). */
FLUX_API int flux_dit_prepare_timesteps(flux_dit *m, const float *ts, int n, void *stream);

/* Euler flow-matching update x += dt * v over n fp32 values, in place
 * ("Flux 2 Klein: Reine C-basierte Inferenz", "Modellarchitektur und Leistung":
 * 4 sampling steps; t_i = linspace(1, 0, S+1), dt = t_{i+1} - t_i). */
FLUX_API int flux_euler_step(float *x, const float *v, size_t n, float dt, void *stream);

/* Guided Euler update in one pass: x += dt * (v_uncond + guidance * (v_cond - v_uncond)) over
 * n fp32 values, in place.  The combination is the usual classifier-free guidance
 * extrapolation; the pages name the scale but not the formula (see flux_dit_forward_cfg).
 * x, v_cond, v_uncond 16-byte aligned device buffers; guidance and dt finite. */
FLUX_API int flux_cfg_euler_step(float *x, const float *v_cond, const float *v_uncond, size_t n, float guidance,
                                 float dt, void *stream);

/* flux_cfg_euler_step that also writes the guided velocity v_uncond + guidance * (v_cond - v_uncond)
 * to v_guided (fp32, n values, a distinct 16-byte aligned device buffer, caller-owned), the same
 * values the update adds to x, for a sampler that reports each step's velocity.  Errors as
 * flux_cfg_euler_step; a NULL v_guided is FLUX_EINVAL. */
FLUX_API int flux_cfg_euler_step_out(float *x, const float *v_cond, const float *v_uncond, float *v_guided,
                                     size_t n, float guidance, float dt, void *stream);

/* img2img start state: out = (1 - t) x + t noise over n fp32 values (x the latent of the
 * image to edit, noise N(0,1)): the flow-matching state at time t.  With strength s the
 * sampler starts at the first of the last floor(S*s) schedule times; s = 0 keeps the image
 * and s = 1 regenerates it ("Flux 2 Klein: Reine C-basierte Inferenz", "Nutzungsbeispiele";
 * hakusoku.com story 4662, "コマンドラインオプション": -t/--strength, default 0.75). */
FLUX_API int flux_blend_latents(const float *x, const float *noise, float t, float *out, size_t n, void *stream);

/* 2x2 latent packing ("Zweistufiger Transformer und Tokenisierung"):
 *   lat fp32 [32, h8, w8]  <->  tok fp32 [(h8/2)*(w8/2), 128],
 *   tok[i*(w8/2)+j][c*4 + py*2 + px] = lat[c][2i+py][2j+px].  h8, w8 even, >= 2.
 * Device pointers, 16-byte aligned, owned by the caller; the call is asynchronous on `stream`.
 * FLUX_EINVAL (nothing launched) for a NULL or misaligned pointer or an odd / too small size. */
FLUX_API int flux_pack_latents(const float *lat, float *tok, int h8, int w8, void *stream);
FLUX_API int flux_unpack_latents(const float *tok, float *lat, int h8, int w8, void *stream);

/* Joint attention O = softmax(Q K^T * scale) V per head, no mask, non-causal
 * (FLUX.3 Image Klein in Diffusers write-up, "Entkoppelte Vorverarbeitung und
 * gemeinsame Attention-Blöcke").  q, k, v, o bf16 [n, heads, head_dim],
 * head_dim == 128, n >= 1.  fp32 softmax statistics, bf16 P, fp32 accumulation. */
FLUX_API int flux_joint_attention(const uint16_t *q, const uint16_t *k, const uint16_t *v, uint16_t *o, int n, int heads,
                         int head_dim, float scale, void *stream);

/* The same over a batch of independent sequences of n tokens each, stored one after
 * another: q, k, v, o bf16 [batch * n, heads, 128]; sequence b attends only to its own
 * rows [b n, (b + 1) n).  1 <= batch <= 65535. */
FLUX_API int flux_joint_attention_batch(const uint16_t *q, const uint16_t *k, const uint16_t *v, uint16_t *o, int batch,
                                        int n, int heads, int head_dim, float scale, void *stream);

/* Kernel-level entry points of the forward's steps (for parity tests and reuse). */

/* Linear layer on the tensor cores: acc = A W^T, A bf16 [m, k] (row stride lda
 * elements), W bf16 [n, k] (nn.Linear layout), bias bf16 [n].  k % 64 == 0,
 * n % 32 == 0, lda % 8 == 0.  mode:
 *   0  out bf16 [m, ldo]: acc + bias
 *   1  out fp32 [m, ldo]: acc + bias
 *   2  out bf16 [m, ldo]: silu(a + bias_a) * (b + bias_b) for n/2 output columns;
 *      W and bias rows in GEMM order: for output columns [128g, 128g+128) the
 *      128 a-rows then the 128 matching b-rows; n % 256 == 0
 *   3  out fp32 [m, ldo] residual: out += gate * (acc + bias), gate fp32 [n] */
FLUX_API int flux_linear(const uint16_t *a, int m, int k, int lda, const uint16_t *w, int n, const uint16_t *bias, int mode,
                void *out, int ldo, const float *gate, void *stream);

/* Fused qkv projection on the tensor cores: qkv = A W^T + bias, bf16 [m, 3*heads*128] in
 * q | k | v order (W bf16 [3*heads*128, k], bias bf16), then each 128-value head of q and k
 * is RMS-normalised (eps), scaled by q_gain / k_gain (bf16 [128]) and rotated by rows
 * table_row0 .. table_row0+m-1 of a flux_rope_table table ("Entkoppelte Vorverarbeitung und
 * gemeinsame Attention-Blöcke": QK-RMSNorm before attention; "Modulation pro Token-Typ,
 * Flow-Map-Destillation und 4D-RoPE": 4-axis RoPE).  k % 64 == 0, heads even. */
FLUX_API int flux_qkv_projection(const uint16_t *a, int m, int k, int lda, const uint16_t *w, const uint16_t *bias,
                                 int heads, const uint16_t *q_gain, const uint16_t *k_gain, const float *table,
                                 int table_row0, float eps, uint16_t *qkv, void *stream);

/* y = LayerNorm(x) * (1 + scale) + shift per row (no learned affine; eps):
 * x fp32 [rows, dim], shift/scale fp32 [dim], y bf16 [rows, dim]
 * ("Modulation pro Token-Typ, Flow-Map-Destillation und 4D-RoPE"). */
FLUX_API int flux_layernorm_modulate(const float *x, uint16_t *y, int rows, int dim, const float *shift, const float *scale,
                            float eps, void *stream);

/* RoPE (cos, sin) table for the joint sequence [n_txt text; gh x gw image;
 * rh x rw reference], head_dim 128, axes (t, h, w, l) of 32 dims, frequency
 * theta^(-2m/32): table fp32 [n, 64, 2] with n = n_txt + gh*gw + rh*rw. */
FLUX_API int flux_rope_table(float *table, int n_txt, int gh, int gw, int rh, int rw, float theta, void *stream);

/* In place on a bf16 [rows, ld] buffer: q = columns [0, heads*128), k = columns
 * [k_col, k_col + heads*128).  Each head's 128 values are RMS-normalised and
 * scaled by the gain (bf16 [128]), then rotated by the table (flux_rope_table). */
FLUX_API int flux_qk_rmsnorm_rope(uint16_t *qkv, int rows, int ld, int k_col, int heads, const uint16_t *q_gain,
                         const uint16_t *k_gain, const float *table, float eps, void *stream);

/* Row-wise e4m3 quantisation (see flux_dit_set_precision): for each of `rows` rows of x (bf16,
 * row stride ldx elements) q[r, j] = e4m3(x[r, j] * inv_r) (uint8 codes, row stride ldq bytes) and
 * scale[r] = amax_r / 448 with amax_r = max_j |x[r, j]| and inv_r = 448 / amax_r (0 for a zero row),
 * the division and the product rounded to float32.  cols % 8 == 0, cols <= 16384; x 16-byte, q
 * 8-byte aligned. */
FLUX_API int flux_quantize_rows_e4m3(const uint16_t *x, int rows, int cols, int ldx, uint8_t *q, int ldq,
                                     float *scale, void *stream);

/* NVFP4 quantisation of rows (see flux_dit_set_precision with FLUX_PRECISION_NVFP4): x bf16 [rows, k]
 * (row stride ldx elements) to 4-bit e2m1 codes q ([rows, k/2] bytes, row stride ldq bytes,
 * element 2i in the low nibble of byte i), e4m3 block scales sf (one per 16 elements, in the
 * tensor-core layout: byte ((r/128)*(k/64) + j/64)*512 + 16*(r%32) + 4*((r%128)/32) + (j/16)%4
 * for element j of row r; flux_nvfp4_scale_bytes(rows, k) bytes, padding rows untouched) and fp32
 * row scales S: amax = max |x|, S = amax / 2688, s_b = e4m3(amax_b * (448 / amax)),
 * code = e2m1(x * (1 / (s_b * S))), each step rounded to float32, round to nearest even and
 * saturating; a zero row or a block whose scale rounds to 0 gets codes 0 (the nvfp4 checkpoint
 * format, "FLUX.3 Image Klein in Diffusers: ...", section "Hardwareanforderungen, Quantisierung
 * und Inferenzlatenz"; block size and block-scale type as in NVIDIA's NVFP4).
 * k % 64 == 0, k <= 16384, ldx % 8 == 0, ldq % 16 == 0; pointers 16-byte aligned. */
FLUX_API size_t flux_nvfp4_scale_bytes(int rows, int k);
FLUX_API int flux_quantize_rows_nvfp4(const uint16_t *x, int rows, int k, int ldx, uint8_t *q, int ldq, uint8_t *sf,
                                      float *row_scale, void *stream);

/* flux_layernorm_modulate with its output quantised to NVFP4 in the same pass (codes [rows, dim/2],
 * block scales and row scales as flux_quantize_rows_nvfp4; the modulated values are quantised from
 * float32).  dim in {1024, 2048, 3072, 4096}. */
FLUX_API int flux_layernorm_modulate_nvfp4(const float *x, uint8_t *q, uint8_t *sf, float *row_scale, int rows,
                                           int dim, const float *shift, const float *scale, float eps,
                                           void *stream);

/* NVFP4 linear layer on the tensor cores (tcgen05 kind::mxf4nvf4 with block scales, CTA pairs):
 * acc = sum over 16-element blocks of (codes_A . codes_W) * s_A * s_W for A [m, k] (codes with row
 * stride lda bytes, scales a_sf) and W [n, k] (codes row stride k/2), both as written by
 * flux_quantize_rows_nvfp4; then acc[i][j] * a_scale[i] * w_scale[j] goes through the epilogue
 * `mode` of flux_linear.  k % 256 == 0, n % 32 == 0, lda % 16 == 0; pointers 16-byte aligned. */
FLUX_API int flux_linear_nvfp4(const uint8_t *a, const uint8_t *a_sf, const float *a_scale, int m, int k, int lda,
                               const uint8_t *w, const uint8_t *w_sf, const float *w_scale, int n,
                               const uint16_t *bias, int mode, void *out, int ldo, const float *gate, void *stream);

/* flux_layernorm_modulate with its output quantised row-wise to e4m3 in the same pass: q uint8
 * [rows, dim] codes and q_scale fp32 [rows] as in flux_quantize_rows_e4m3 (the modulated values
 * are quantised from float32).  dim in {1024, 2048, 3072, 4096}. */
FLUX_API int flux_layernorm_modulate_fp8(const float *x, uint8_t *q, float *q_scale, int rows, int dim,
                                         const float *shift, const float *scale, float eps, void *stream);

/* FP8 linear layer on the tensor cores (tcgen05 kind::f8f6f4, CTA pairs): acc = (A W^T) with A e4m3
 * codes [m, k] (row stride lda bytes) and W e4m3 codes [n, k], then acc[i][j] * a_scale[i] *
 * w_scale[j] goes through the epilogue `mode` of flux_linear (0 bf16 + bias, 1 fp32 + bias,
 * 2 SwiGLU, 3 gated residual).  k % 128 == 0, n % 32 == 0, lda % 16 == 0; pointers 16-byte aligned. */
FLUX_API int flux_linear_fp8(const uint8_t *a, const float *a_scale, int m, int k, int lda, const uint8_t *w,
                             const float *w_scale, int n, const uint16_t *bias, int mode, void *out, int ldo,
                             const float *gate, void *stream);

/* Measurement hooks (used by the benchmark).
 * flux_dit_profile(m, 1) starts bracketing every kernel launch of later
 * forwards with CUDA events on the launch's stream (0 stops); both reset the
 * totals.  flux_dit_profile_read synchronises the device and returns, for one
 * kernel kind (0 GEMM, 1 attention, 2 LayerNorm+modulation, 3 QK-RMSNorm+RoPE,
 * 4 GEMV, 5 other), the summed device time in ms, the algorithmic FLOPs and
 * HBM bytes of those launches, and their number.  Any pointer may be NULL. */
FLUX_API int flux_dit_profile(flux_dit *m, int enable);
FLUX_API int flux_dit_profile_read(flux_dit *m, int kind, double *ms, double *flops, double *bytes, long long *launches);

/* Number of kernel launches the library has enqueued since it was loaded. */
FLUX_API unsigned long long flux_kernel_launches(void);

/* Timestep conditioning that allocates no device memory (the pages have no
 * counterpart; this is a deployment convenience).  For callers that may not
 * call cudaMalloc once running -- runtimes that hand all device memory to a
 * pre-sized pool at start-up, or latency-critical loops that cannot take the
 * stall of cudaMalloc/cudaFree (cudaFree can synchronise the whole device).
 * Computes what flux_dit_modulation computes, from caller-owned weights:
 *   temb = [cos(t*1000*f_j), sin(t*1000*f_j)], vec = w2 silu(w1 temb + b1) + b2,
 *   mods_out = wmod silu(vec) + bmod
 * w1 bf16 [hidden, t_freq_dim], w2 bf16 [hidden, hidden], wmod bf16 [mod_rows,
 * hidden] (every modulation linear stacked in blob order), biases bf16,
 * mods_out fp32 [mod_rows]; weight and output pointers 16-byte aligned.
 * Limits: hidden <= 8192 and t_freq_dim <= 1024, both multiples of 8; larger
 * sizes return FLUX_EINVAL.  The intermediates live in one 68 KiB device array
 * inside the library, which every GPU that loads the library holds until the
 * process exits.  The first call in a CUDA context (normally a device's primary
 * context) looks up that array's address (cudaGetSymbolAddress) with the device
 * current and keeps it for that context; make that first call before any stream
 * capture.  All calls on a device share the array: calls whose
 * kernels overlap on the GPU (different streams without ordering) race.  Each
 * call writes every scratch element before reading it, so nothing is cleared. */
FLUX_API int flux_timestep_modulation_noalloc(const uint16_t *w1, const uint16_t *b1, const uint16_t *w2,
                                              const uint16_t *b2, const uint16_t *wmod, const uint16_t *bmod,
                                              int hidden, int t_freq_dim, int mod_rows, float t, float *mods_out,
                                              void *stream);

/* ======================================================================
 * FLUX.3 Image Klein ("FLUX.3 Image Klein in Diffusers: Architektur, Layout-Steuerung und
 * Systemanforderungen im Überblick", mindverse).  The same kernels in the FLUX.3 block
 * structure:
 *   - "Zweistufiger Transformer und Tokenisierung": text features are the hidden states of 8
 *     encoder layers (8 x 2560 = 20480 values per token) projected to the width by one linear;
 *   - "Entkoppelte Vorverarbeitung und gemeinsame Attention-Blöcke": n_mode (5) per-mode blocks
 *     in which the text, image and reference streams have their own weights and attend only to
 *     themselves, then n_joint (28) joint blocks with one weight set over text | image |
 *     reference; in every block attention and the SwiGLU MLP run in parallel on one
 *     normalised input (the FLUX.2 single-stream block);
 *   - "Modulation pro Token-Typ, Flow-Map-Destillation und 4D-RoPE": image tokens are modulated
 *     with the current t, text and reference tokens with t = 0; the time-distilled checkpoint
 *     (flow_map = 1) embeds the step's target time with its own MLP and adds it to the time
 *     vector of every token.
 * Readings where the page is silent: the modulation linears are shared by the blocks of a phase
 * (one per stream for the per-mode phase, one for the joint phase: 5.49 B parameters against the
 * page's 5.6 B; per-block linears would give 6.7 B); the target embedding has the time MLP's
 * shape and is added before SiLU; the reference stream of the per-mode phase is every reference
 * image together; block arithmetic as in the FLUX.2 single-stream block. */
typedef struct flux3_dit flux3_dit;

/* Defaults (FLUX.3 Image Klein): 5, 28, 3072, 24, 128, 9216, 128, 20480, 256, 1, 1e4, 1e-6, 1e-6.
 * hidden == heads * head_dim, head_dim == 128, heads even, hidden and t_freq_dim <= 6144. */
typedef struct {
  int n_mode, n_joint, hidden, heads, head_dim, mlp_hidden, in_ch, txt_dim, t_freq_dim, flow_map;
  float rope_theta, eps_ln, eps_rms;
} flux3_dit_config;

/* Bytes of a FLUX.3 weight blob for `cfg`, or 0 if cfg is invalid.
 * Blob format (little endian, fields packed without padding): a 256-byte header
 *   char magic[8] = "FLUX3DT\0"; uint32 version = 1; uint32 n_tensors;
 *   int32 n_mode, n_joint, hidden, heads, head_dim, mlp_hidden, in_ch, txt_dim, t_freq_dim, flow_map;
 *   float32 rope_theta, eps_ln, eps_rms; uint64 data_offset (= 256, at byte 68); uint64 data_bytes;
 * then every tensor as bf16, row-major, each starting on a 256-byte boundary, in this order:
 *   time_in.{w1 [D,256], b1, w2 [D,D], b2}, (flow_map only) target_in.{w1, b1, w2, b2},
 *   img_in.{w [D,128], b}, txt_in.{w [D,txt_dim], b},
 *   mode_mod.{txt, img, ref}.{w [3D,D], b [3D]}      rows: shift, scale, gate
 *   for each per-mode block i, for stream s in (txt, img, ref):
 *     lin1.{w [3D+2F,D], b}  q_gain [128]  k_gain [128]  lin2.{w [D,D+F], b [D]}
 *   joint_mod.{w [3D,D], b [3D]}
 *   for each joint block i: lin1, q_gain, k_gain, lin2 as above
 *   final.mod.{w [2D,D], b [2D]} (shift, scale), final.out.{w [128,D], b [128]}. */
FLUX_API size_t flux3_blob_expected_bytes(const flux3_dit_config *cfg);

/* Create a FLUX.3 model from a weight blob in HOST memory (format above); as flux_dit_create. */
FLUX_API flux3_dit *flux3_dit_create(const void *blob, size_t blob_bytes, const flux3_dit_config *cfg, void *stream);
FLUX_API void flux3_dit_destroy(flux3_dit *m);

/* One FLUX.3 forward: the velocity of the image tokens at time t.
 *   img_tok fp32 [grid_h*grid_w, 128], txt fp32 [n_txt, txt_dim], ref_tok fp32 [sum_k h_k*w_k, 128]
 *   (n_refs <= 10 references, ref_grids a HOST array of (h, w) pairs, RoPE l = -(k+1)),
 *   v_out fp32 [grid_h*grid_w, 128].
 * t_target: the step's target time (the sampler's next schedule point), read only by the
 * flow-map model.  Shapes and workspace growth as flux_dit_forward_refs. */
FLUX_API int flux3_dit_forward(flux3_dit *m, const float *img_tok, int grid_h, int grid_w, const float *txt,
                               int n_txt, const float *ref_tok, int n_refs, const int *ref_grids, float t,
                               float t_target, float *v_out, void *stream);

/* Classifier-free guidance forward of a FLUX.3 model: the velocities of the prompt and of the
 * unconditional text for the same image, references, t and t_target as ONE batch of two
 * sequences.  The base checkpoint samples 50 steps at guidance 3.5 (we0.ai FLUX 3 Image Klein
 * article, checkpoint table); combine the two velocities with flux_cfg_euler_step.  In the
 * per-mode blocks the image and reference streams attend only to themselves ("FLUX.3 Image Klein
 * in Diffusers: ...", section "Entkoppelte Vorverarbeitung und gemeinsame Attention-Blöcke"), so
 * they do not depend on the text: they are computed once for both sequences; the text streams
 * and every joint block run per sequence.  txt_cond and txt_uncond are fp32 [n_txt, txt_dim]
 * device buffers with the same token count; v_cond and v_uncond are distinct fp32
 * [grid_h*grid_w, 128] outputs.  The workspace holds both sequences.  Otherwise as
 * flux3_dit_forward; each velocity equals, bit for bit, what flux3_dit_forward returns for that
 * text alone. */
FLUX_API int flux3_dit_forward_cfg(flux3_dit *m, const float *img_tok, int grid_h, int grid_w, const float *txt_cond,
                                   const float *txt_uncond, int n_txt, const float *ref_tok, int n_refs,
                                   const int *ref_grids, float t, float t_target, float *v_cond, float *v_uncond,
                                   void *stream);

/* Precision of the block linears of later FLUX.3 forwards (linear1 / linear2 of the per-mode and
 * joint blocks): FLUX_PRECISION_BF16, FLUX_PRECISION_FP8 or FLUX_PRECISION_NVFP4, as
 * flux_dit_set_precision. */
FLUX_API int flux3_dit_set_precision(flux3_dit *m, int precision);

/* Diagnostic: run only the first n_mode per-mode and n_joint joint blocks (-1 = all). */
FLUX_API int flux3_dit_set_active_blocks(flux3_dit *m, int n_mode, int n_joint);

/* Every modulation vector of a forward at (t, t_target), fp32 [17 * hidden]:
 * per-mode text (shift, scale, gate; from the t = 0 time vector) | per-mode image (from t) |
 * per-mode reference (t = 0) | joint image (t) | joint text and reference (t = 0) |
 * output layer (shift, scale; from t). */
FLUX_API size_t flux3_dit_modulation_size(const flux3_dit *m);
FLUX_API int flux3_dit_modulation(flux3_dit *m, float t, float t_target, float *mods_out, void *stream);

/* Per-kernel timing of later forwards; as flux_dit_profile / flux_dit_profile_read. */
FLUX_API int flux3_dit_profile(flux3_dit *m, int enable);
FLUX_API int flux3_dit_profile_read(flux3_dit *m, int kind, double *ms, double *flops, double *bytes,
                                    long long *launches);

/* Attention over n_seg (1..4) independent segments stored one after another: segment z is
 * the seg_len[z] rows that follow segment z-1 and attends only to itself (the per-mode blocks'
 * stream-local attention).  q, k, v, o bf16 [sum seg_len, heads, 128]; seg_len a HOST array,
 * entries >= 0 (0 = empty segment).  Otherwise as flux_joint_attention. */
FLUX_API int flux_joint_attention_segments(const uint16_t *q, const uint16_t *k, const uint16_t *v, uint16_t *o,
                                           int n_seg, const int *seg_len, int heads, int head_dim, float scale,
                                           void *stream);

/* Synchronise `stream`, then read and clear the kernels' device error words:
 * 0 when no kernel gave up waiting, else the first nonzero code (FLUX_DEVERR_*). */
FLUX_API int flux_device_error(void *stream);

/* Device error codes: which role of a kernel gave up waiting. */
#define FLUX_DEVERR_TIMEOUT_PRODUCER 1 /* a TMA producer waited for a free stage */
#define FLUX_DEVERR_TIMEOUT_MMA 2      /* the MMA issuer waited for operands or an empty accumulator */
#define FLUX_DEVERR_TIMEOUT_EPILOGUE 3 /* the epilogue waited for a finished accumulator */
#define FLUX_DEVERR_TIMEOUT_SOFTMAX 4  /* an attention softmax warpgroup waited for scores */
#define FLUX_DEVERR_BAD_LAUNCH 5       /* a kernel found its launch shape inconsistent */
#define FLUX_DEVERR_TIMEOUT_SELFTEST 6 /* flux_selftest_bounded_wait gave up, as asked */

/* Check of the error path above, with no kernel stalled for real (hakusoku.com story 4662,
 * "エラーハンドリング": failures surface as a status code and a message).  Launches one CTA
 * that waits on a shared-memory mbarrier through the bounded wait every pipeline uses.  With
 * arrive = 1 the CTA first arrives on the barrier, so the wait succeeds at once and nothing is
 * recorded.  With arrive = 0 nothing ever arrives: the wait gives up after limit_ns nanoseconds
 * (0 < limit_ns <= 1e9, else FLUX_EINVAL), the kernel records FLUX_DEVERR_TIMEOUT_SELFTEST in its
 * device error word and returns normally, leaving the context usable; flux_device_error() then
 * reports and clears it.  Asynchronous on `stream`; no memory arguments. */
FLUX_API int flux_selftest_bounded_wait(unsigned long long limit_ns, int arrive, void *stream);

/* Test hook for the out-of-memory path (same convention: hakusoku.com story 4662,
 * "エラーハンドリング").  After this call the library's next n device allocations succeed and
 * the one after them fails as if the device were out of memory (n = 0: the very next one); the
 * hook then disarms itself.  n < 0 disarms it at once.  Every entry point that allocates (model
 * creation, the first forward at a larger token count or a new precision, timestep preparation)
 * then returns FLUX_ENOMEM with a message in flux_get_error(), frees what it had allocated in that
 * call and leaves the model as it was, so that a later call succeeds.  Process-wide; no device
 * work. */
FLUX_API void flux_test_fail_alloc_after(long long n);

#ifdef __cplusplus
}
#endif

#endif /* FLUXDIT_H */
