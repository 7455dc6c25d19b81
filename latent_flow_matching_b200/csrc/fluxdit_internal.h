// Internal interfaces between the kernel files and the C-ABI layer (not exported).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>

namespace fdit {

// Kernel attributes (the dynamic shared-memory size) are a per-device setting: cudaFuncSetAttribute
// applies to the current device.  `set` runs once per device ordinal (below 64; beyond that, on
// every call), and again after a failure.
template <class SetAttributes>
cudaError_t once_per_device(std::atomic<unsigned long long>& done, SetAttributes set) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = dev < 64 ? 1ull << dev : 0ull;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = set();
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

// ------------------------------------------------------------------ GEMM
enum EpiMode : int { kEpiBf16Bias = 0, kEpiF32Bias = 1, kEpiSwiGLU = 2, kEpiResidGate = 3, kEpiQKNormRope = 4 };
constexpr int kMaxProblems = 8;

struct GemmProblem {
  int M, N, K;                    // out rows, W rows, reduction (K % 64 == 0, N % 32 == 0)
  int mode;                       // EpiMode
  int ldo;                        // leading dimension of out, elements
  int tiles_m, tiles_n, tile_begin;   // filled by gemm_launch
  void* out;                      // bf16 or f32 (see mode); kEpiResidGate: the f32 residual
  const __nv_bfloat16* bias;      // [N]
  const float* gate;              // [N], kEpiResidGate only
  // kEpiQKNormRope (bf16 out, N = 3 * heads * 128 in q | k | v order, BN = 256): each 128-column
  // head of q and k is RMS-normalised (eps), scaled by its gain and rotated by the RoPE table row
  // rope_row0 + m; v columns get the plain bias epilogue.
  const __nv_bfloat16* gain_q;    // [128]
  const __nv_bfloat16* gain_k;    // [128]
  const float2* rope;             // (cos, sin) [tokens, 64]
  int rope_row0;
  float eps;
  // 8-bit operands (gemm2 launched with fp8): the accumulator is scaled by scale_a[m] (per row of
  // A, [M]) and scale_b[n] (per row of W, [N]) before the epilogue above
  const float* scale_a;
  const float* scale_b;
};

struct GemmParams {
  CUtensorMap mapA[kMaxProblems];     // activations [M, K], box {64, 128}
  CUtensorMap mapB[kMaxProblems];     // weights [N, K], box {64, BN}
  GemmProblem prob[kMaxProblems];
  int num_problems;
  int total_tiles;
};

int gemm_bn_for(int n);
cudaError_t gemm_launch(GemmParams& P, int bn, int num_sms, cudaStream_t stream);
int gemm_read_device_error(cudaStream_t stream);
// CTA-pair variant (cta_group::2, 256 x 256 tiles, W maps with a 128-row box): same problems and epilogues.
// fp8: A and W are e4m3 codes (u8 maps with a 128-byte box, K % 128 == 0) with per-row scales.
cudaError_t gemm2_launch(GemmParams& P, int num_sms, cudaStream_t stream, bool fp8 = false);
int gemm2_read_device_error(cudaStream_t stream);

// ------------------------------------------------------------------ attention
constexpr int kMaxSegs = 4;       // independent segments of one attention launch
struct AttnParams {
  CUtensorMap mapQ, mapK, mapV;   // 2D bf16 [rows = n, cols], box {64, 128}, 128B swizzle
  __nv_bfloat16* out;             // O row i, head h at out + i*ldo + h*128
  int ldo;
  int n, heads;                   // tokens per sequence, heads
  int batch;                      // sequences of n rows each, one after another (grid.z)
  int q_col0, k_col0, v_col0;     // column of head 0's first element in each map
  float scale_log2;               // softmax scale * log2(e)
  // nseg > 0 replaces the batch: grid.z = segment, segment z is rows [seg_row0[z], +seg_n[z]) and
  // attends only to itself (n and batch are then ignored)
  int nseg = 0;
  int seg_row0[kMaxSegs], seg_n[kMaxSegs];
};
cudaError_t attention_launch(const AttnParams& P, cudaStream_t stream);
int attention_read_device_error(cudaStream_t stream);

// ------------------------------------------------------------------ HBM-bound kernels
cudaError_t pack_latents_launch(const float* lat, float* tok, int c, int h8, int w8, cudaStream_t s);
cudaError_t unpack_latents_launch(const float* tok, float* lat, int c, int h8, int w8, cudaStream_t s);
cudaError_t euler_launch(float* x, const float* v, size_t n, float dt, cudaStream_t s);
// v = vu + g * (vc - vu) and x += dt * v, element-wise; v is also written to vg unless vg is null
cudaError_t cfg_euler_launch(float* x, const float* vc, const float* vu, float* vg, size_t n, float g, float dt,
                             cudaStream_t s);
cudaError_t cast_bf16_launch(const float* x, __nv_bfloat16* y, size_t n, cudaStream_t s);

// Modulation sets of a LayerNorm + modulation launch: row r uses set 0 when r % period < split, set 1
// when it is < split2, else set 2.  (Scalar members: a runtime index into a kernel-parameter array
// would copy it to the stack.)
struct LnModSets {
  int split, split2, period;
  const float *sh0, *sh1, *sh2;
  const float *sc0, *sc1, *sc2;
  __device__ __forceinline__ const float* shift(int row) const {
    const int r = row % period;
    return r < split ? sh0 : (r < split2 ? sh1 : sh2);
  }
  __device__ __forceinline__ const float* scale(int row) const {
    const int r = row % period;
    return r < split ? sc0 : (r < split2 ? sc1 : sc2);
  }
};

// y[r, :] = LN(x[r, :]) * (1 + scale) + shift; rows with r % period < split use (shift0, scale0), the
// others (shift1, scale1) (period: rows per sequence of a batch, the row count for one sequence)
cudaError_t ln_modulate_launch(const float* x, __nv_bfloat16* y, int rows, int dim, int split, int period,
                               const float* shift0, const float* scale0, const float* shift1,
                               const float* scale1, float eps, cudaStream_t s);
// Three row regions: r % period in [0, split) set 0, [split, split2) set 1, [split2, period) set 2
// (FLUX.3 per-token-type modulation: text | image | reference).
cudaError_t ln_modulate3_launch(const float* x, __nv_bfloat16* y, int rows, int dim, int split, int split2,
                                int period, const float* shift0, const float* scale0, const float* shift1,
                                const float* scale1, const float* shift2, const float* scale2, float eps,
                                cudaStream_t s);

// In place on q (columns [0, heads*hd)) and k (columns [kcol, kcol + heads*hd)) of a [rows, ld] bf16 buffer:
// RMSNorm over each head's hd values with gain (rows < split: gq0/gk0, else gq1/gk1), then RoPE from
// the [rows, hd/2] float2 (cos, sin) table.
cudaError_t qk_norm_rope_launch(__nv_bfloat16* qkv, int rows, int ld, int kcol, int heads, int split,
                                const __nv_bfloat16* gq0, const __nv_bfloat16* gk0,
                                const __nv_bfloat16* gq1, const __nv_bfloat16* gk1,
                                const float2* rope, float eps, cudaStream_t s);

// Token grids of the reference images, in sequence order.
constexpr int kMaxRefs = 10;
struct RefGrids {
  int count;
  int h[kMaxRefs], w[kMaxRefs];
};

// (cos, sin) table for the joint sequence [text; image grid; reference grids], head_dim 128, 4 axes.
cudaError_t rope_table_launch(float2* table, int n_txt, int gh, int gw, const RefGrids& refs, float theta,
                              cudaStream_t s);

// out = (1 - t) x + t noise over n floats
cudaError_t blend_launch(const float* x, const float* noise, float t, float* out, size_t n, cudaStream_t s);

// temb[j] = cos(t*1000*f_j), temb[128+j] = sin(...), f_j = 1e4^(-j/128)
cudaError_t timestep_embed_launch(float* temb, float t, int dim, cudaStream_t s);

// y[r] = act_out(sum_k W[r,k] * act_in(x[k]) + b[r]); W bf16 [rows, k], b bf16 [rows]
cudaError_t gemv_launch(const __nv_bfloat16* W, const __nv_bfloat16* b, const float* x, float* y, int rows,
                        int k, int silu_in, int silu_out, cudaStream_t s);
// nvec (1 to 4) input vectors of k floats, one after another, against one read of W: output v is
// y[v * rows .. v * rows + rows); add (NULL or [rows]) is added before act_out.  nvec * k <= 12288.
cudaError_t gemv_multi_launch(const __nv_bfloat16* W, const __nv_bfloat16* b, const float* x, int nvec, float* y,
                              const float* add, int rows, int k, int silu_in, int silu_out, cudaStream_t s);

// ------------------------------------------------------------------ row-wise e4m3 (fp8.cu)
// codes[r, 0..cols) = e4m3(x[r, j] * 448 / amax_r), scale[r] = amax_r / 448; x bf16 rows of stride
// ldx, codes of stride ldq (bytes); cols % 8 == 0, cols <= 16384.
cudaError_t quantize_rows_launch(const __nv_bfloat16* x, int ldx, int rows, int cols, uint8_t* q, int ldq,
                                 float* scale, cudaStream_t s);
// ln_modulate3_launch whose modulated rows are quantised to e4m3 codes [rows, dim] + scales [rows];
// dim in {1024, 2048, 3072, 4096}.
cudaError_t ln_modulate_fp8_launch(const float* x, uint8_t* q, float* qscale, int rows, int dim, int split,
                                   int split2, int period, const float* shift0, const float* scale0,
                                   const float* shift1, const float* scale1, const float* shift2,
                                   const float* scale2, float eps, cudaStream_t s);

// ------------------------------------------------------------------ NVFP4 (nvfp4.cu, gemm_fp4.cu)
// Rows of x (bf16, stride ldx elements) to e2m1 codes (q, [rows, k/2] bytes, stride ldq), e4m3
// block scales (sf, nvfp4_scale_bytes(rows, k) bytes, 512-byte blocks of 128 rows x 64 elements)
// and fp32 row scales; k % 64 == 0, k <= 16384.
inline size_t nvfp4_scale_bytes(size_t rows, size_t k) { return (rows + 127) / 128 * 128 * (k / 16); }
// Row segments of one quantisation: segment z is rows [row0, row0 + rows) and its block scales
// start at 128-row block blk0 of the scale buffer (q4_segments packs them one after another).
constexpr int kMaxQ4Segs = 8;
struct Q4Segs {
  int n;
  int row0[kMaxQ4Segs], rows[kMaxQ4Segs], blk0[kMaxQ4Segs];
};
Q4Segs q4_segments(const int* row0, const int* rows, int n);
cudaError_t quantize_nvfp4_launch(const __nv_bfloat16* x, int ldx, int k, uint8_t* q, int ldq, uint8_t* sf,
                                  float* row_scale, const Q4Segs& segs, cudaStream_t s);
// LayerNorm + modulation (fp32 rows of x, dim values each) rounded to bf16 and quantised to NVFP4 as
// quantize_nvfp4_launch (codes row stride dim / 2), over the rows of `segs`; dim in {1024, 2048, 3072, 4096}.
cudaError_t ln_modulate_nvfp4_launch(const float* x, int dim, uint8_t* q, uint8_t* sf, float* row_scale,
                                     const Q4Segs& segs, const LnModSets& ms, float eps, cudaStream_t s);
// Problems of the NVFP4 pair GEMM: mapA / mapB over the codes (u8 maps, 128-byte box), K in elements
// (K % 256 == 0), scale_a / scale_b the fp32 row scales, and the block scales' maps (make_tmap_sf).
struct GemmParams4 {
  GemmParams g;
  CUtensorMap mapSFA[kMaxProblems];
  CUtensorMap mapSFB[kMaxProblems];
  CUtensorMap mapOut[kMaxProblems];     // filled by gemm_fp4_launch: the epilogue writes by TMA
};
cudaError_t gemm_fp4_launch(GemmParams4& P, int num_sms, cudaStream_t stream);
int gemm_fp4_read_device_error(cudaStream_t stream);

// ------------------------------------------------------------------ kernel launches
// Programmatic dependent launches are on unless the environment sets FLUX_PDL=0 (read at every
// launch, so a process can compare both; a CUDA graph keeps what was set when it was captured).
bool pdl_enabled();

// Every device allocation of the library goes through dev_alloc / dev_alloc_async: a failed
// cudaMalloc leaves *p null and its error is cleared from the runtime's last-error state (so that a
// later launch check does not report it again), and flux_test_fail_alloc_after can make the n-th
// following allocation fail the same way without asking the driver.
cudaError_t dev_alloc(void** p, size_t bytes);
cudaError_t dev_alloc_async(void** p, size_t bytes, cudaStream_t s);
template <typename T>
cudaError_t dev_alloc(T** p, size_t bytes) {
  return dev_alloc(reinterpret_cast<void**>(p), bytes);
}
template <typename T>
cudaError_t dev_alloc_async(T** p, size_t bytes, cudaStream_t s) {
  return dev_alloc_async(reinterpret_cast<void**>(p), bytes, s);
}
// Launch `kernel` on `s` with programmatic stream serialisation (when enabled): the kernel may be
// scheduled before the previous kernel on the stream has finished, and waits for it with
// pdl_wait() (common.cuh) before touching global memory.  Only kernels that call pdl_wait()
// before their first global access may be launched this way.
template <typename... KernelArgs, typename... Args>
cudaError_t launch_kernel(void (*kernel)(KernelArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                          Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

// ------------------------------------------------------------------ host helpers
// Record `msg` as the calling thread's flux_get_error() message and return `code`.
int record_error(int code, const char* msg);
// Counts kernel launches enqueued by the library (reported by flux_kernel_launches).
void count_launch();
// the bounded-wait self-test kernel's device error word (read and cleared)
int selftest_read_device_error(cudaStream_t stream);
// 2D bf16 tensor map: rows x cols, row stride in bytes, box {64 cols, box_rows}, 128B swizzle.
bool make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t row_stride_bytes,
                    uint32_t box_rows);
// 2D u8 tensor map (e4m3 codes): rows x cols bytes, box {128 bytes, box_rows}, 128B swizzle.
bool make_tmap_u8(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t row_stride_bytes,
                  uint32_t box_rows);
// Block scales of an NVFP4 matrix as 256-byte rows, box 8 rows (2 KB: one stage of 128 rows), no swizzle.
bool make_tmap_sf(CUtensorMap* map, const void* base, uint64_t bytes);
// GEMM output written by TMA: 64-byte box rows (16 fp32 or 32 bf16 columns) x 32 rows, 64-byte swizzle.
bool make_tmap_out(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t row_stride_bytes,
                   bool f32);
// The output map of problem pr for a TMA-store epilogue (fp32 for kEpiF32Bias / kEpiResidGate, N / 2
// columns for SwiGLU), encoded once per (buffer, shape) and kept.
bool gemm_out_map(CUtensorMap* map, const GemmProblem& pr);
int num_sms_current();

}  // namespace fdit
