// NVFP4 quantisation of token / weight rows: 4-bit e2m1 codes, one e4m3 scale per 16 elements and
// one fp32 scale per row (the second-level scale).  The transformer's nvfp4 checkpoint format
// ("FLUX.3 Image Klein in Diffusers: ...", section "Hardwareanforderungen, Quantisierung und
// Inferenzlatenz") with NVIDIA's block size of 16 and e4m3 block scales; one row:
//   amax = max |x|, S = amax / 2688, inv = 448 / amax,
//   s_b  = e4m3(amax_b * inv)            (round to nearest even, saturating),
//   code = e2m1(x * (1 / (s_b * S)))     (round to nearest even, saturating at +-6),
// every intermediate rounded to fp32; an all-zero row or a block whose scale rounds to 0 gets
// codes 0.  value = code * s_b * S.
//
// Output layouts (the ones the tcgen05 block-scaled MMA reads):
//   codes  [rows, k/2] bytes, element 2i in the low nibble of byte i;
//   scales e4m3 bytes in 512-byte blocks of 128 rows x 64 elements (4 scales per row):
//          byte ((r/128)*(k/64) + j/64)*512 + 16*(r%32) + 4*((r%128)/32) + (j/16)%4 for element j,
//          so that 32 rows of 16 bytes, copied to tensor memory and broadcast to the four lane
//          quarters, put row r's four scales in lane r, column r/32 of the block's four columns;
//   row scales fp32 [rows].
#include <cuda_fp4.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "fluxdit_internal.h"

namespace fdit {
namespace {

constexpr int kQ4Threads = 128;
constexpr int kQ4MaxUnits = 2;          // 64-element units per thread: k <= 128 * 64 * 2

__device__ __forceinline__ float bf16_abs_max8(const uint4& w, float m) {
  const uint32_t x[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) m = fmaxf(m, fmaxf(fabsf(bf16lo(x[e])), fabsf(bf16hi(x[e]))));
  return m;
}

// One CTA per row.  Rows come in segments (Q4Segs): segment z is rows [row0, row0 + rows) of x, q
// and row_scale, and its scales start at 128-row block blk0 of sf, so that a GEMM problem over
// that segment finds its first row at the start of a scale block.
__global__ void __launch_bounds__(kQ4Threads) quantize_nvfp4_kernel(const __nv_bfloat16* __restrict__ x, int ldx,
                                                                    int k, uint8_t* __restrict__ q, int ldq,
                                                                    uint8_t* __restrict__ sf, float* __restrict__ row_scale,
                                                                    const Q4Segs segs) {
  __shared__ float red[kQ4Threads / 32];
  int z = 0, l = blockIdx.x;
  while (z + 1 < segs.n && l >= segs.rows[z]) l -= segs.rows[z++];
  const int r = segs.row0[z] + l;                  // row of x, q and row_scale
  const int sfr = segs.blk0[z] * 128 + l;          // row of the scale layout
  const int units = k / 64;
  const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<size_t>(r) * ldx);
  uint4 v[kQ4MaxUnits][8];
  float bmax[kQ4MaxUnits][4];
  float amax = 0.f;
#pragma unroll
  for (int u = 0; u < kQ4MaxUnits; ++u) {
    const int unit = threadIdx.x + u * kQ4Threads;
#pragma unroll
    for (int b = 0; b < 4; ++b) bmax[u][b] = 0.f;
    if (unit < units) {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[u][i] = __ldg(xr + unit * 8 + i);
#pragma unroll
      for (int b = 0; b < 4; ++b) bmax[u][b] = bf16_abs_max8(v[u][2 * b + 1], bf16_abs_max8(v[u][2 * b], 0.f));
      amax = fmaxf(amax, fmaxf(fmaxf(bmax[u][0], bmax[u][1]), fmaxf(bmax[u][2], bmax[u][3])));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  const float inv = amax > 0.f ? __fdiv_rn(448.0f, amax) : 0.f;
  const float S = __fdiv_rn(amax, 2688.0f);
  if (threadIdx.x == 0) row_scale[r] = S;
  uint8_t* qr = q + static_cast<size_t>(r) * ldq;
  const size_t sf_row = 16 * (sfr & 31) + 4 * ((sfr & 127) >> 5);
#pragma unroll
  for (int u = 0; u < kQ4MaxUnits; ++u) {
    const int unit = threadIdx.x + u * kQ4Threads;
    if (unit >= units) continue;
    uint32_t sfw = 0;
    uint32_t codes[8];                               // 64 codes, 8 per word
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const __nv_fp8_storage_t s8 = __nv_cvt_float_to_fp8(__fmul_rn(bmax[u][b], inv), __NV_SATFINITE, __NV_E4M3);
      const float sb = __half2float(__half(__nv_cvt_fp8_to_halfraw(s8, __NV_E4M3)));
      const float d = __fmul_rn(sb, S);
      const float rcp = d > 0.f ? __frcp_rn(d) : 0.f;
      sfw |= static_cast<uint32_t>(s8) << (8 * b);
#pragma unroll
      for (int h = 0; h < 2; ++h) {                  // 8 elements per uint4
        const uint4 w = v[u][2 * b + h];
        const uint32_t xw[4] = {w.x, w.y, w.z, w.w};
        uint32_t word = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = make_float2(__fmul_rn(bf16lo(xw[e]), rcp), __fmul_rn(bf16hi(xw[e]), rcp));
          word |= static_cast<uint32_t>(__nv_cvt_float2_to_fp4x2(f, __NV_E2M1, cudaRoundNearest)) << (8 * e);
        }
        codes[2 * b + h] = word;
      }
    }
    uint4* dq = reinterpret_cast<uint4*>(qr + unit * 32);
    dq[0] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
    dq[1] = make_uint4(codes[4], codes[5], codes[6], codes[7]);
    const size_t blk = static_cast<size_t>(sfr >> 7) * units + unit;
    *reinterpret_cast<uint32_t*>(sf + blk * 512 + sf_row) = sfw;
  }
}

}  // namespace

cudaError_t quantize_nvfp4_launch(const __nv_bfloat16* x, int ldx, int k, uint8_t* q, int ldq, uint8_t* sf,
                                  float* row_scale, const Q4Segs& segs, cudaStream_t s) {
  if (k <= 0 || k % 64 != 0 || k > kQ4Threads * 64 * kQ4MaxUnits || ldx < k || ldx % 8 != 0 || ldq < k / 2 ||
      ldq % 16 != 0 || segs.n < 1 || segs.n > kMaxQ4Segs)
    return cudaErrorInvalidValue;
  long total = 0;
  for (int z = 0; z < segs.n; ++z) {
    if (segs.rows[z] < 0 || segs.row0[z] < 0 || segs.blk0[z] < 0) return cudaErrorInvalidValue;
    total += segs.rows[z];
  }
  if (total == 0) return cudaSuccess;
  count_launch();
  quantize_nvfp4_kernel<<<static_cast<unsigned>(total), kQ4Threads, 0, s>>>(x, ldx, k, q, ldq, sf, row_scale, segs);
  return cudaGetLastError();
}

Q4Segs q4_segments(const int* row0, const int* rows, int n) {
  Q4Segs g{};
  g.n = n;
  int blk = 0;
  for (int z = 0; z < n; ++z) {
    g.row0[z] = row0[z];
    g.rows[z] = rows[z];
    g.blk0[z] = blk;
    blk += (rows[z] + 127) / 128;
  }
  return g;
}

}  // namespace fdit
