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
#include <cuda_fp8.h>

#include "common.cuh"
#include "fluxdit_internal.h"

namespace fdit {
namespace {

// One 256-thread CTA per row.  A row is read with coalesced 16-byte loads (element group j, of 8
// bf16 values or 4 fp32 values, goes to thread j % 256), kept in registers, and every 16-element
// block is held by neighbouring threads of one warp (2 threads for bf16 groups, 4 for fp32), so
// a block's maximum takes one or two shuffles and the row's maximum one CTA reduction.
constexpr int kQ4Threads = 256;

__device__ __forceinline__ float bf16_abs_max8(const uint4& w, float m) {
  const uint32_t x[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) m = fmaxf(m, fmaxf(fabsf(bf16lo(x[e])), fabsf(bf16hi(x[e]))));
  return m;
}

// Sum (or maximum) over the CTA; every thread gets the result.  red: one float per warp.
template <bool kMax>
__device__ __forceinline__ float cta_reduce(float v, float* red) {
  if constexpr (kMax) {
    v = redux_max(v, 0xffffffffu);
  } else {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  }
  __syncthreads();                                   // red may still be read by the previous reduction
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  v = red[0];
#pragma unroll
  for (int w = 1; w < kQ4Threads / 32; ++w) v = kMax ? fmaxf(v, red[w]) : v + red[w];
  return v;
}

// The row and the scale-layout row of CTA blockIdx.x in a segment list.
struct Q4Row {
  int r, sfr;
};
__device__ __forceinline__ Q4Row q4_row(const Q4Segs& segs) {
  int z = 0, l = blockIdx.x;
  while (z + 1 < segs.n && l >= segs.rows[z]) l -= segs.rows[z++];
  return {segs.row0[z] + l, segs.blk0[z] * 128 + l};
}

// Row quantities from the row's absolute maximum: inv = 448 / amax (0 for a zero row), S = amax / 2688.
__device__ __forceinline__ void q4_row_scales(float amax, float* inv, float* S) {
  *inv = amax > 0.f ? __fdiv_rn(448.0f, amax) : 0.f;
  *S = __fdiv_rn(amax, 2688.0f);
}

// The e4m3 scale of a block with maximum bmax, and the reciprocal of its dequantisation factor.
__device__ __forceinline__ __nv_fp8_storage_t q4_block_scale(float bmax, float inv, float S, float* rcp) {
  const __nv_fp8_storage_t s8 = __nv_cvt_float_to_fp8(__fmul_rn(bmax, inv), __NV_SATFINITE, __NV_E4M3);
  const float sb = __half2float(__half(__nv_cvt_fp8_to_halfraw(s8, __NV_E4M3)));
  const float d = __fmul_rn(sb, S);
  *rcp = d > 0.f ? __frcp_rn(d) : 0.f;
  return s8;
}

// Two e2m1 codes, a * rcp in the low nibble and b * rcp in the high one, by the sm_100a conversion
// instruction (nearest even, saturating at +-6; it places its first source in the high nibble).
// The toolkit's conversion helper emulates this in integer arithmetic unless the family-specific
// target macro is defined, which an sm_100a build does not define.
__device__ __forceinline__ uint32_t e2m1x2(float a, float b, float rcp) {
  uint32_t r;
  asm("{\n\t.reg .b8 c;\n\tcvt.rn.satfinite.e2m1x2.f32 c, %2, %1;\n\tcvt.u32.u8 %0, c;\n}"
      : "=r"(r)
      : "f"(__fmul_rn(a, rcp)), "f"(__fmul_rn(b, rcp)));
  return r;
}

// Byte offset of the scale of 16-element block g of scale-layout row sfr (k elements per row).
__device__ __forceinline__ size_t q4_sf_offset(int sfr, int g, int k) {
  return (static_cast<size_t>(sfr >> 7) * (k / 64) + (g >> 2)) * 512 + 16 * (sfr & 31) + 4 * ((sfr & 127) >> 5) +
         (g & 3);
}

// Rows come in segments (Q4Segs): segment z is rows [row0, row0 + rows) of x, q and row_scale, and
// its scales start at 128-row block blk0 of sf, so that a GEMM problem over that segment finds its
// first row at the start of a scale block.  U: groups of 8 values per thread (k <= 2048 U).
template <int U>
__global__ void __launch_bounds__(kQ4Threads) quantize_nvfp4_kernel(const __nv_bfloat16* __restrict__ x, int ldx,
                                                                    int k, uint8_t* __restrict__ q, int ldq,
                                                                    uint8_t* __restrict__ sf,
                                                                    float* __restrict__ row_scale, const Q4Segs segs) {
  pdl_trigger();
  pdl_wait();
  __shared__ float red[kQ4Threads / 32];
  const int tid = threadIdx.x;
  const Q4Row rr = q4_row(segs);
  const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<size_t>(rr.r) * ldx);
  const int n8 = k / 8;
  uint4 v[U];
  float amax = 0.f;
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int j = tid + u * kQ4Threads;
    v[u] = j < n8 ? __ldg(xr + j) : make_uint4(0u, 0u, 0u, 0u);
    amax = bf16_abs_max8(v[u], amax);
  }
  float inv, S;
  q4_row_scales(cta_reduce<true>(amax, red), &inv, &S);
  if (tid == 0) row_scale[rr.r] = S;
  uint32_t* qr = reinterpret_cast<uint32_t*>(q + static_cast<size_t>(rr.r) * ldq);
  // Group pairs (u0, u1) = (2w, 2w + 1): the two threads of a block each compute one of the pair's
  // two block scales (thread parity p takes u_p) and exchange the reciprocals.
  const int p = tid & 1;
#pragma unroll
  for (int w = 0; w < (U + 1) / 2; ++w) {
    float m[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float a = 2 * w + h < U ? bf16_abs_max8(v[2 * w + h], 0.f) : 0.f;
      m[h] = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
    }
    float my_rcp;
    const __nv_fp8_storage_t s8 = q4_block_scale(p ? m[1] : m[0], inv, S, &my_rcp);
    const float other = __shfl_xor_sync(0xffffffffu, my_rcp, 1);
    const int jp = tid + (2 * w + p) * kQ4Threads;  // n8 % 8 == 0: both threads of a block agree on j < n8
    if (2 * w + p < U && jp < n8) sf[q4_sf_offset(rr.sfr, jp >> 1, k)] = s8;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int u = 2 * w + h;
      if (u < U) {
        const int j = tid + u * kQ4Threads;
        const float rcp = h == p ? my_rcp : other;
        const uint32_t e4[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
        uint32_t c = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) c |= e2m1x2(bf16lo(e4[e]), bf16hi(e4[e]), rcp) << (8 * e);
        if (j < n8) qr[j] = c;
      }
    }
  }
}

// LayerNorm + modulation of one row per CTA (dim = 1024 VPT: VPT float4 per thread), the modulated
// float32 row quantised to NVFP4 as above; row r uses the modulation set that `ms` gives it.
template <int VPT>
__global__ void __launch_bounds__(kQ4Threads) ln_mod_nvfp4_kernel(const float* __restrict__ x,
                                                                  uint8_t* __restrict__ q, uint8_t* __restrict__ sf,
                                                                  float* __restrict__ row_scale, const Q4Segs segs,
                                                                  LnModSets ms, float eps) {
  pdl_trigger();
  pdl_wait();
  static_assert(VPT >= 1 && VPT <= 4, "one block scale per quad lane");
  constexpr int dim = 1024 * VPT;
  __shared__ float red[kQ4Threads / 32];
  const int tid = threadIdx.x;
  const Q4Row rr = q4_row(segs);
  const float4* xr = reinterpret_cast<const float4*>(x + static_cast<size_t>(rr.r) * dim) + tid;
  float4 v[VPT];
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    v[i] = __ldcs(xr + i * kQ4Threads);
    s += (v[i].x + v[i].y) + (v[i].z + v[i].w);
  }
  const float mean = cta_reduce<false>(s, red) * (1.0f / dim);
  float qs = 0.f;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const float a = v[i].x - mean, b = v[i].y - mean, c = v[i].z - mean, d = v[i].w - mean;
    qs += (a * a + b * b) + (c * c + d * d);
  }
  const float rstd = rsqrtf(cta_reduce<false>(qs, red) * (1.0f / dim) + eps);
  const float4* sh = reinterpret_cast<const float4*>(ms.shift(rr.r)) + tid;
  const float4* sc = reinterpret_cast<const float4*>(ms.scale(rr.r)) + tid;
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const float4 a = __ldg(sh + i * kQ4Threads), c = __ldg(sc + i * kQ4Threads);
    v[i].x = (v[i].x - mean) * rstd * (1.f + c.x) + a.x;
    v[i].y = (v[i].y - mean) * rstd * (1.f + c.y) + a.y;
    v[i].z = (v[i].z - mean) * rstd * (1.f + c.z) + a.z;
    v[i].w = (v[i].w - mean) * rstd * (1.f + c.w) + a.w;
    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v[i].x), fabsf(v[i].y)), fmaxf(fabsf(v[i].z), fabsf(v[i].w))));
  }
  float inv, S;
  q4_row_scales(cta_reduce<true>(amax, red), &inv, &S);
  if (tid == 0) row_scale[rr.r] = S;
  // Float4 group g = tid + 256 i belongs to block g / 4: the quad of threads 4b..4b+3 shares block
  // b + 64 i for every i.  Thread 4b + i computes the scale of the quad's i-th block once and the
  // quad exchanges the reciprocals (lanes with 4b + i, i >= VPT, compute a spare copy of block 0).
  const int quad_lane = tid & 3;
  float mine = 0.f;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    float m = fmaxf(fmaxf(fabsf(v[i].x), fabsf(v[i].y)), fmaxf(fabsf(v[i].z), fabsf(v[i].w)));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
    mine = (i == 0 || quad_lane == i) ? m : mine;
  }
  float my_rcp;
  const __nv_fp8_storage_t s8 = q4_block_scale(mine, inv, S, &my_rcp);
  if (quad_lane < VPT) sf[q4_sf_offset(rr.sfr, (tid >> 2) + 64 * quad_lane, dim)] = s8;
  uint16_t* qr = reinterpret_cast<uint16_t*>(q + static_cast<size_t>(rr.r) * (dim / 2)) + tid;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const float rcp = __shfl_sync(0xffffffffu, my_rcp, (tid & 28) | i);
    qr[i * kQ4Threads] = static_cast<uint16_t>(e2m1x2(v[i].x, v[i].y, rcp) | (e2m1x2(v[i].z, v[i].w, rcp) << 8));
  }
}

}  // namespace

static bool q4_segs_ok(const Q4Segs& segs, long* total) {
  if (segs.n < 1 || segs.n > kMaxQ4Segs) return false;
  *total = 0;
  for (int z = 0; z < segs.n; ++z) {
    if (segs.rows[z] < 0 || segs.row0[z] < 0 || segs.blk0[z] < 0) return false;
    *total += segs.rows[z];
  }
  return *total < (1l << 31);
}

cudaError_t quantize_nvfp4_launch(const __nv_bfloat16* x, int ldx, int k, uint8_t* q, int ldq, uint8_t* sf,
                                  float* row_scale, const Q4Segs& segs, cudaStream_t s) {
  long total = 0;
  if (k <= 0 || k % 64 != 0 || k > 16384 || ldx < k || ldx % 8 != 0 || ldq < k / 2 || ldq % 16 != 0 ||
      !q4_segs_ok(segs, &total))
    return cudaErrorInvalidValue;
  if (total == 0) return cudaSuccess;
  const unsigned grid = static_cast<unsigned>(total);
  count_launch();
  switch ((k / 8 + kQ4Threads - 1) / kQ4Threads) {
    case 1: launch_kernel(quantize_nvfp4_kernel<1>, grid, kQ4Threads, 0, s, x, ldx, k, q, ldq, sf, row_scale, segs); break;
    case 2: launch_kernel(quantize_nvfp4_kernel<2>, grid, kQ4Threads, 0, s, x, ldx, k, q, ldq, sf, row_scale, segs); break;
    case 3: launch_kernel(quantize_nvfp4_kernel<3>, grid, kQ4Threads, 0, s, x, ldx, k, q, ldq, sf, row_scale, segs); break;
    case 4: launch_kernel(quantize_nvfp4_kernel<4>, grid, kQ4Threads, 0, s, x, ldx, k, q, ldq, sf, row_scale, segs); break;
    case 5: launch_kernel(quantize_nvfp4_kernel<5>, grid, kQ4Threads, 0, s, x, ldx, k, q, ldq, sf, row_scale, segs); break;
    case 6: launch_kernel(quantize_nvfp4_kernel<6>, grid, kQ4Threads, 0, s, x, ldx, k, q, ldq, sf, row_scale, segs); break;
    case 7: launch_kernel(quantize_nvfp4_kernel<7>, grid, kQ4Threads, 0, s, x, ldx, k, q, ldq, sf, row_scale, segs); break;
    default: launch_kernel(quantize_nvfp4_kernel<8>, grid, kQ4Threads, 0, s, x, ldx, k, q, ldq, sf, row_scale, segs); break;
  }
  return cudaGetLastError();
}

cudaError_t ln_modulate_nvfp4_launch(const float* x, int dim, uint8_t* q, uint8_t* sf, float* row_scale,
                                     const Q4Segs& segs, const LnModSets& ms, float eps, cudaStream_t s) {
  long total = 0;
  if (!q4_segs_ok(segs, &total)) return cudaErrorInvalidValue;
  if (total == 0) return cudaSuccess;
  const unsigned grid = static_cast<unsigned>(total);
  switch (dim) {
    case 1024: count_launch(); launch_kernel(ln_mod_nvfp4_kernel<1>, grid, kQ4Threads, 0, s, x, q, sf, row_scale, segs, ms, eps); break;
    case 2048: count_launch(); launch_kernel(ln_mod_nvfp4_kernel<2>, grid, kQ4Threads, 0, s, x, q, sf, row_scale, segs, ms, eps); break;
    case 3072: count_launch(); launch_kernel(ln_mod_nvfp4_kernel<3>, grid, kQ4Threads, 0, s, x, q, sf, row_scale, segs, ms, eps); break;
    case 4096: count_launch(); launch_kernel(ln_mod_nvfp4_kernel<4>, grid, kQ4Threads, 0, s, x, q, sf, row_scale, segs, ms, eps); break;
    default: return cudaErrorInvalidValue;
  }
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
