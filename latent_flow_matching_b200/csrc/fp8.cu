// Row-wise e4m3 quantisation for the FP8 block linears ("FLUX.3 Image Klein in Diffusers: ...",
// section "Hardwareanforderungen, Quantisierung und Inferenzlatenz": the fp8r format, row-wise FP8).
//
// Every row gets one fp32 scale from its absolute maximum:
//   scale = amax / 448, inv = 448 / amax (0 for an all-zero row), code_j = e4m3_rn_satfinite(x_j * inv)
// with IEEE-rounded float32 division and product, so the codes are a function of the row's
// values alone.  The GEMM multiplies its accumulator by scale_a[m] * scale_b[n].
//
//   quantize_rows_kernel  bf16 rows (weights at model set-up; attention output and SwiGLU hidden
//                         inside the forward) -> codes + scales, one CTA per row, the row held in
//                         registers between the max and the conversion
//   ln_mod_fp8_kernel     LayerNorm + adaLN modulation (as ln_mod_kernel) whose modulated row is
//                         quantised in the same pass instead of being written as bf16
#include <cuda_fp8.h>

#include "common.cuh"
#include "fluxdit_internal.h"

namespace fdit {
namespace {

constexpr float kE4M3Max = 448.0f;
constexpr int kQThreads = 256;
constexpr int kQMaxChunks = 8;                 // 8 bf16 per chunk: rows of up to 16384 values

__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
  return static_cast<uint16_t>(__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3));
}

// Maximum over the CTA (256 threads); `red` holds 8 floats.
__device__ __forceinline__ float block_max(float v, float* red) {
  v = redux_max(v, 0xffffffffu);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int w = 1; w < kQThreads / 32; ++w) r = fmaxf(r, red[w]);
  return r;
}

__device__ __forceinline__ void row_scale(float amax, float* scale, float* inv) {
  *scale = amax / kE4M3Max;
  *inv = amax > 0.f ? kE4M3Max / amax : 0.f;
}

__global__ void __launch_bounds__(kQThreads) quantize_rows_kernel(const __nv_bfloat16* __restrict__ x, int ldx,
                                                                  int cols, uint8_t* __restrict__ q, int ldq,
                                                                  float* __restrict__ scale) {
  pdl_trigger();
  pdl_wait();
  __shared__ float red[kQThreads / 32];
  const int row = blockIdx.x;
  const int nch = cols / 8;
  const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<size_t>(row) * ldx);
  uint4 v[kQMaxChunks];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < kQMaxChunks; ++i) {
    const int c = i * kQThreads + threadIdx.x;
    v[i] = c < nch ? __ldcs(src + c) : make_uint4(0u, 0u, 0u, 0u);
    const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) amax = fmaxf(amax, fmaxf(fabsf(bf16lo(w[e])), fabsf(bf16hi(w[e]))));
  }
  amax = block_max(amax, red);
  float sc, inv;
  row_scale(amax, &sc, &inv);
  if (threadIdx.x == 0) scale[row] = sc;
  uint2* dst = reinterpret_cast<uint2*>(q + static_cast<size_t>(row) * ldq);
#pragma unroll
  for (int i = 0; i < kQMaxChunks; ++i) {
    const int c = i * kQThreads + threadIdx.x;
    if (c >= nch) continue;
    const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
    uint32_t o[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const uint32_t lo = e4m3x2(__fmul_rn(bf16lo(w[2 * e]), inv), __fmul_rn(bf16hi(w[2 * e]), inv));
      const uint32_t hi = e4m3x2(__fmul_rn(bf16lo(w[2 * e + 1]), inv), __fmul_rn(bf16hi(w[2 * e + 1]), inv));
      o[e] = lo | (hi << 16);
    }
    dst[c] = make_uint2(o[0], o[1]);
  }
}

// LayerNorm + modulation of one row per CTA (dim = 1024 VPT), the modulated values quantised to
// e4m3 with the row's scale.  Rows with r % period < split use set 0, < split2 set 1, else set 2.
template <int VPT>
__global__ void __launch_bounds__(kQThreads) ln_mod_fp8_kernel(const float* __restrict__ x, uint8_t* __restrict__ q,
                                                               float* __restrict__ qscale, int split, int split2,
                                                               int period, const float* __restrict__ sh0,
                                                               const float* __restrict__ sc0,
                                                               const float* __restrict__ sh1,
                                                               const float* __restrict__ sc1,
                                                               const float* __restrict__ sh2,
                                                               const float* __restrict__ sc2, float eps) {
  pdl_trigger();
  pdl_wait();
  constexpr int dim = 1024 * VPT;
  __shared__ float red[3][kQThreads / 32];
  const int row = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float4* xr = reinterpret_cast<const float4*>(x + static_cast<size_t>(row) * dim);
  float4 v[VPT];
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    v[i] = __ldcs(xr + i * kQThreads + tid);
    s += (v[i].x + v[i].y) + (v[i].z + v[i].w);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) red[0][warp] = s;
  __syncthreads();
  s = 0.f;
#pragma unroll
  for (int w = 0; w < kQThreads / 32; ++w) s += red[0][w];
  const float mean = s * (1.0f / dim);
  float qs = 0.f;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const float a = v[i].x - mean, b = v[i].y - mean, c = v[i].z - mean, d = v[i].w - mean;
    qs += (a * a + b * b) + (c * c + d * d);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) qs += __shfl_xor_sync(0xffffffffu, qs, o);
  if (lane == 0) red[1][warp] = qs;
  __syncthreads();
  qs = 0.f;
#pragma unroll
  for (int w = 0; w < kQThreads / 32; ++w) qs += red[1][w];
  const float rstd = rsqrtf(qs * (1.0f / dim) + eps);
  const int r = row % period;
  const float* shp = r < split ? sh0 : (r < split2 ? sh1 : sh2);
  const float* scp = r < split ? sc0 : (r < split2 ? sc1 : sc2);
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const float4 sh = __ldg(reinterpret_cast<const float4*>(shp) + i * kQThreads + tid);
    const float4 sc = __ldg(reinterpret_cast<const float4*>(scp) + i * kQThreads + tid);
    v[i].x = (v[i].x - mean) * rstd * (1.f + sc.x) + sh.x;
    v[i].y = (v[i].y - mean) * rstd * (1.f + sc.y) + sh.y;
    v[i].z = (v[i].z - mean) * rstd * (1.f + sc.z) + sh.z;
    v[i].w = (v[i].w - mean) * rstd * (1.f + sc.w) + sh.w;
    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v[i].x), fabsf(v[i].y)), fmaxf(fabsf(v[i].z), fabsf(v[i].w))));
  }
  amax = redux_max(amax, 0xffffffffu);
  if (lane == 0) red[2][warp] = amax;
  __syncthreads();
  amax = red[2][0];
#pragma unroll
  for (int w = 1; w < kQThreads / 32; ++w) amax = fmaxf(amax, red[2][w]);
  float scl, inv;
  row_scale(amax, &scl, &inv);
  if (tid == 0) qscale[row] = scl;
  uint32_t* dst = reinterpret_cast<uint32_t*>(q + static_cast<size_t>(row) * dim);
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const uint32_t lo = e4m3x2(__fmul_rn(v[i].x, inv), __fmul_rn(v[i].y, inv));
    const uint32_t hi = e4m3x2(__fmul_rn(v[i].z, inv), __fmul_rn(v[i].w, inv));
    dst[i * kQThreads + tid] = lo | (hi << 16);
  }
}

}  // namespace

cudaError_t quantize_rows_launch(const __nv_bfloat16* x, int ldx, int rows, int cols, uint8_t* q, int ldq,
                                 float* scale, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  if (cols <= 0 || cols % 8 || cols > kQThreads * kQMaxChunks * 8 || ldx % 8 || ldq % 8)
    return cudaErrorInvalidValue;
  count_launch();
  launch_kernel(quantize_rows_kernel, rows, kQThreads, 0, s, x, ldx, cols, q, ldq, scale);
  return cudaGetLastError();
}

cudaError_t ln_modulate_fp8_launch(const float* x, uint8_t* q, float* qscale, int rows, int dim, int split,
                                   int split2, int period, const float* shift0, const float* scale0,
                                   const float* shift1, const float* scale1, const float* shift2,
                                   const float* scale2, float eps, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  if (period <= 0) return cudaErrorInvalidValue;
  count_launch();
  switch (dim) {
    case 1024:
      launch_kernel(ln_mod_fp8_kernel<1>, rows, kQThreads, 0, s, x, q, qscale, split, split2, period, shift0, scale0, shift1,
                                                       scale1, shift2, scale2, eps);
      break;
    case 2048:
      launch_kernel(ln_mod_fp8_kernel<2>, rows, kQThreads, 0, s, x, q, qscale, split, split2, period, shift0, scale0, shift1,
                                                       scale1, shift2, scale2, eps);
      break;
    case 3072:
      launch_kernel(ln_mod_fp8_kernel<3>, rows, kQThreads, 0, s, x, q, qscale, split, split2, period, shift0, scale0, shift1,
                                                       scale1, shift2, scale2, eps);
      break;
    case 4096:
      launch_kernel(ln_mod_fp8_kernel<4>, rows, kQThreads, 0, s, x, q, qscale, split, split2, period, shift0, scale0, shift1,
                                                       scale1, shift2, scale2, eps);
      break;
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace fdit
