// HBM-bound kernels of the transformer forward and the sampler:
//   2x2 latent pack / unpack, Euler update, fp32 -> bf16 casts, LayerNorm + adaLN
//   modulation, QK-RMSNorm + RoPE, the RoPE (cos, sin) table, the sinusoidal
//   timestep embedding and the GEMV used for the time MLP and the modulation vectors.
//
// Sources: FLUX.3 Image Klein in Diffusers write-up (mindverse): "Zweistufiger
// Transformer und Tokenisierung" (2x2 packing to 128 channels), "Entkoppelte
// Vorverarbeitung und gemeinsame Attention-Blöcke" (QK-RMSNorm, SwiGLU),
// "Modulation pro Token-Typ, Flow-Map-Destillation und 4D-RoPE" (LayerNorm
// without affine, shift/scale/gate from the timestep embedding, 4-axis RoPE).
// The Euler step x += dt * v follows the 4-step sampler of the FLUX.2-klein
// pages ("Modellarchitektur und Leistung").
#include <math.h>

#include "common.cuh"
#include "fluxdit_internal.h"

namespace fdit {
namespace {

inline int blocks_for(size_t n, int per_block) {
  size_t b = (n + per_block - 1) / per_block;
  return static_cast<int>(b < 1 ? 1 : (b > 1048576 ? 1048576 : b));
}

// ------------------------------------------------------------------ pack / unpack
// token (i, j) channel c*4 + py*2 + px  <->  lat[c, 2i+py, 2j+px]
//
// The packing transposes channels and tokens: a latent row is contiguous along j, a token is
// contiguous along its 128 channels.  One CTA takes a tile of kPackT consecutive tokens of one
// token row i (all 32 channels, 2 latent rows each) and stages it in shared memory, so that both
// the latent side (8 bytes per thread, a warp spans 256 contiguous bytes of one latent row) and the
// token side (16 bytes per thread, the tile is kPackT * 512 contiguous bytes) are coalesced.
constexpr int kPackC = 32;            // latent channels; 4 * kPackC = 128 token channels
constexpr int kPackT = 32;            // tokens per tile
constexpr int kPackLd = 4 * kPackC + 4;   // shared row stride in floats: 16-byte rows, 4-bank skew
constexpr int kPackThreads = 256;

struct PackTile {
  int i, j0, gw;
};
__device__ __forceinline__ PackTile pack_tile(int w8) {
  const int gw = w8 / 2, tiles_w = (gw + kPackT - 1) / kPackT;
  return {static_cast<int>(blockIdx.x / tiles_w), static_cast<int>(blockIdx.x % tiles_w) * kPackT, gw};
}

__global__ void __launch_bounds__(kPackThreads) pack_kernel(const float* __restrict__ lat, float* __restrict__ tok,
                                                            int h8, int w8) {
  pdl_trigger();
  pdl_wait();
  __shared__ __align__(16) float st[kPackT * kPackLd];
  const PackTile tl = pack_tile(w8);
  // latent side: item (c, py, jj), jj fastest
#pragma unroll
  for (int s = 0; s < kPackC * 2 * kPackT / kPackThreads; ++s) {
    const int item = threadIdx.x + s * kPackThreads;
    const int jj = item % kPackT, cp = item / kPackT, c = cp >> 1, py = cp & 1;
    if (tl.j0 + jj < tl.gw) {
      const float2 v = __ldcs(reinterpret_cast<const float2*>(
          lat + (static_cast<size_t>(c) * h8 + 2 * tl.i + py) * w8 + 2 * (tl.j0 + jj)));
      *reinterpret_cast<float2*>(st + jj * kPackLd + c * 4 + py * 2) = v;
    }
  }
  __syncthreads();
  // token side: item (jj, quad), quad fastest
  float4* dst = reinterpret_cast<float4*>(tok + (static_cast<size_t>(tl.i) * tl.gw + tl.j0) * (4 * kPackC));
#pragma unroll
  for (int s = 0; s < kPackT * kPackC / kPackThreads; ++s) {
    const int item = threadIdx.x + s * kPackThreads;
    const int jj = item / kPackC, qd = item % kPackC;
    if (tl.j0 + jj < tl.gw) dst[item] = *reinterpret_cast<const float4*>(st + jj * kPackLd + qd * 4);
  }
}

__global__ void __launch_bounds__(kPackThreads) unpack_kernel(const float* __restrict__ tok, float* __restrict__ lat,
                                                              int h8, int w8) {
  pdl_trigger();
  pdl_wait();
  __shared__ __align__(16) float st[kPackT * kPackLd];
  const PackTile tl = pack_tile(w8);
  const float4* src =
      reinterpret_cast<const float4*>(tok + (static_cast<size_t>(tl.i) * tl.gw + tl.j0) * (4 * kPackC));
#pragma unroll
  for (int s = 0; s < kPackT * kPackC / kPackThreads; ++s) {
    const int item = threadIdx.x + s * kPackThreads;
    const int jj = item / kPackC, qd = item % kPackC;
    if (tl.j0 + jj < tl.gw) *reinterpret_cast<float4*>(st + jj * kPackLd + qd * 4) = __ldcs(src + item);
  }
  __syncthreads();
#pragma unroll
  for (int s = 0; s < kPackC * 2 * kPackT / kPackThreads; ++s) {
    const int item = threadIdx.x + s * kPackThreads;
    const int jj = item % kPackT, cp = item / kPackT, c = cp >> 1, py = cp & 1;
    if (tl.j0 + jj < tl.gw)
      *reinterpret_cast<float2*>(lat + (static_cast<size_t>(c) * h8 + 2 * tl.i + py) * w8 + 2 * (tl.j0 + jj)) =
          *reinterpret_cast<const float2*>(st + jj * kPackLd + c * 4 + py * 2);
  }
}

// ------------------------------------------------------------------ Euler, casts
__global__ void euler_kernel(float* __restrict__ x, const float* __restrict__ v, size_t n, float dt) {
  pdl_trigger();
  pdl_wait();
  const size_t n4 = n / 4;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n4; i += stride) {
    float4 a = reinterpret_cast<float4*>(x)[i];
    const float4 b = reinterpret_cast<const float4*>(v)[i];
    a.x = fmaf(dt, b.x, a.x);
    a.y = fmaf(dt, b.y, a.y);
    a.z = fmaf(dt, b.z, a.z);
    a.w = fmaf(dt, b.w, a.w);
    reinterpret_cast<float4*>(x)[i] = a;
  }
  for (size_t i = n4 * 4 + blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n; i += stride)
    x[i] = fmaf(dt, v[i], x[i]);
}

__global__ void cast_bf16_kernel(const float* __restrict__ x, __nv_bfloat16* __restrict__ y, size_t n) {
  pdl_trigger();
  pdl_wait();
  const size_t n4 = n / 4;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n4; i += stride) {
    const float4 a = reinterpret_cast<const float4*>(x)[i];
    reinterpret_cast<uint2*>(y)[i] = make_uint2(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w));
  }
  for (size_t i = n4 * 4 + blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n; i += stride)
    y[i] = __float2bfloat16_rn(x[i]);
}

// ------------------------------------------------------------------ LayerNorm + adaLN modulation
// One 256-thread CTA per row: each thread keeps VPT float4 of the row in registers (dim = 1024 VPT),
// mean and variance come from two block reductions, so many CTAs stay resident per SM.
// Row r uses modulation set 0 when r % period < split, set 1 when it is < split2, else set 2
// (LnModSets, fluxdit_internal.h).

template <int VPT>
__global__ void __launch_bounds__(256) ln_mod_kernel(const float* __restrict__ x, __nv_bfloat16* __restrict__ y,
                                                     int rows, const LnModSets m, float eps) {
  pdl_trigger();
  pdl_wait();
  constexpr int dim = 1024 * VPT;
  __shared__ float red[2][8];
  const int row = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float4* xr = reinterpret_cast<const float4*>(x + static_cast<size_t>(row) * dim);
  float4 v[VPT];
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    v[i] = __ldcs(xr + i * 256 + tid);
    s += (v[i].x + v[i].y) + (v[i].z + v[i].w);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) red[0][warp] = s;
  __syncthreads();
  s = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) s += red[0][w];
  const float mean = s * (1.0f / dim);
  float q = 0.f;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const float a = v[i].x - mean, b = v[i].y - mean, c = v[i].z - mean, d = v[i].w - mean;
    q += (a * a + b * b) + (c * c + d * d);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
  if (lane == 0) red[1][warp] = q;
  __syncthreads();
  q = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) q += red[1][w];
  const float rstd = rsqrtf(q * (1.0f / dim) + eps);
  const float4* shp = reinterpret_cast<const float4*>(m.shift(row));
  const float4* scp = reinterpret_cast<const float4*>(m.scale(row));
  uint2* yr = reinterpret_cast<uint2*>(y + static_cast<size_t>(row) * dim);
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const float4 sh = __ldg(shp + i * 256 + tid), sc = __ldg(scp + i * 256 + tid);
    const float a = (v[i].x - mean) * rstd * (1.f + sc.x) + sh.x;
    const float b = (v[i].y - mean) * rstd * (1.f + sc.y) + sh.y;
    const float c = (v[i].z - mean) * rstd * (1.f + sc.z) + sh.z;
    const float d = (v[i].w - mean) * rstd * (1.f + sc.w) + sh.w;
    yr[i * 256 + tid] = make_uint2(pack_bf16x2(a, b), pack_bf16x2(c, d));
  }
}

// Any dim that is a multiple of 4: three passes over the row in global memory.
__global__ void ln_mod_generic_kernel(const float* __restrict__ x, __nv_bfloat16* __restrict__ y, int rows, int dim,
                                      const LnModSets m, float eps) {
  pdl_trigger();
  pdl_wait();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= rows) return;
  const float* xr = x + static_cast<size_t>(warp) * dim;
  float s = 0.f;
  for (int i = lane; i < dim; i += 32) s += xr[i];
  for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float mean = s / dim;
  float q = 0.f;
  for (int i = lane; i < dim; i += 32) q += (xr[i] - mean) * (xr[i] - mean);
  for (int o = 16; o; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
  const float rstd = rsqrtf(q / dim + eps);
  const float* sh = m.shift(warp);
  const float* sc = m.scale(warp);
  for (int i = lane; i < dim; i += 32)
    y[static_cast<size_t>(warp) * dim + i] = __float2bfloat16_rn((xr[i] - mean) * rstd * (1.f + sc[i]) + sh[i]);
}

// ------------------------------------------------------------------ QK-RMSNorm + RoPE (head_dim 128)
// One warp per (row, q or k); a half-warp per head, 8 dims (4 rotation pairs) per lane.
__global__ void __launch_bounds__(256) qk_norm_rope_kernel(__nv_bfloat16* __restrict__ qkv, int rows, int ld, int kcol,
                                                           int heads, int split, const __nv_bfloat16* __restrict__ gq0,
                                                           const __nv_bfloat16* __restrict__ gk0,
                                                           const __nv_bfloat16* __restrict__ gq1,
                                                           const __nv_bfloat16* __restrict__ gk1,
                                                           const float2* __restrict__ rope, float eps) {
  pdl_trigger();
  pdl_wait();
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int row = gw >> 1;
  const int which = gw & 1;                       // 0: q, 1: k
  if (row >= rows) return;
  const int hl = lane & 15;                       // dims [8 hl, 8 hl + 8)
  const int hsub = lane >> 4;                     // which head of the pair
  const __nv_bfloat16* gain = which == 0 ? (row < split ? gq0 : gq1) : (row < split ? gk0 : gk1);
  const uint4 g4 = __ldg(reinterpret_cast<const uint4*>(gain) + hl);
  const float g[8] = {bf16lo(g4.x), bf16hi(g4.x), bf16lo(g4.y), bf16hi(g4.y),
                      bf16lo(g4.z), bf16hi(g4.z), bf16lo(g4.w), bf16hi(g4.w)};
  const float4* rp = reinterpret_cast<const float4*>(rope + static_cast<size_t>(row) * 64 + 4 * hl);
  const float4 r01 = __ldg(rp), r23 = __ldg(rp + 1);
  const float cs[4] = {r01.x, r01.z, r23.x, r23.z};
  const float sn[4] = {r01.y, r01.w, r23.y, r23.w};
  __nv_bfloat16* base = qkv + static_cast<size_t>(row) * ld + (which ? kcol : 0);
  // every lane takes every shuffle: with an odd head count the second half-warp idles on the last pair
  for (int h0 = 0; h0 < heads; h0 += 2) {
    const int h = h0 + hsub;
    const bool act = h < heads;
    uint4* p = reinterpret_cast<uint4*>(base + (act ? h : 0) * 128) + hl;
    const uint4 w = act ? *p : make_uint4(0u, 0u, 0u, 0u);
    float x[8] = {bf16lo(w.x), bf16hi(w.x), bf16lo(w.y), bf16hi(w.y),
                  bf16lo(w.z), bf16hi(w.z), bf16lo(w.w), bf16hi(w.w)};
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) ss += x[e] * x[e];
#pragma unroll
    for (int o = 8; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float r = rsqrtf(ss * (1.0f / 128.0f) + eps);
    uint32_t out[4];
#pragma unroll
    for (int pr = 0; pr < 4; ++pr) {
      const float a = x[2 * pr] * r * g[2 * pr];
      const float b = x[2 * pr + 1] * r * g[2 * pr + 1];
      out[pr] = pack_bf16x2(a * cs[pr] - b * sn[pr], a * sn[pr] + b * cs[pr]);
    }
    if (act) *p = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

// (cos, sin) of pos_axis * theta^(-2m/32) for the 64 pairs of a 128-dim head, axes (t, h, w, l).
// text i: (0,0,0,i); image (r,c): (0,r,c,0); reference k (r,c): (0,r,c,-(k+1)).
__global__ void rope_table_kernel(float2* __restrict__ table, int n_txt, int gh, int gw, RefGrids refs,
                                  float theta) {
  pdl_trigger();
  pdl_wait();
  int n = n_txt + gh * gw;
  for (int k = 0; k < refs.count; ++k) n += refs.h[k] * refs.w[k];
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= n * 64) return;
  const int row = idx >> 6, pr = idx & 63;
  const int axis = pr >> 4, m = pr & 15;
  double pos[4] = {0.0, 0.0, 0.0, 0.0};
  if (row < n_txt) {
    pos[3] = row;
  } else if (row < n_txt + gh * gw) {
    const int t = row - n_txt;
    pos[1] = t / gw;
    pos[2] = t % gw;
  } else {
    int t = row - n_txt - gh * gw;
    int k = 0;
    while (k + 1 < refs.count && t >= refs.h[k] * refs.w[k]) {
      t -= refs.h[k] * refs.w[k];
      ++k;
    }
    pos[1] = t / refs.w[k];
    pos[2] = t % refs.w[k];
    pos[3] = -(k + 1.0);
  }
  const double ang = pos[axis] * pow(static_cast<double>(theta), -2.0 * m / 32.0);
  double s, c;
  sincos(ang, &s, &c);
  table[idx] = make_float2(static_cast<float>(c), static_cast<float>(s));
}

// (1 - t) x + t noise: the flow-matching state at time t between data (t = 0) and noise (t = 1)
// x += dt * (v_u + g (v_c - v_u)): the guided velocity and the Euler step in one pass.
__global__ void cfg_euler_kernel(float* __restrict__ x, const float* __restrict__ vc, const float* __restrict__ vu,
                                 float* __restrict__ vg, size_t n, float g, float dt) {
  pdl_trigger();
  pdl_wait();
  const size_t n4 = n / 4;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n4; i += stride) {
    float4 a = reinterpret_cast<float4*>(x)[i];
    const float4 c = reinterpret_cast<const float4*>(vc)[i];
    const float4 u = reinterpret_cast<const float4*>(vu)[i];
    const float4 v = make_float4(fmaf(g, c.x - u.x, u.x), fmaf(g, c.y - u.y, u.y), fmaf(g, c.z - u.z, u.z),
                                 fmaf(g, c.w - u.w, u.w));
    a.x = fmaf(dt, v.x, a.x);
    a.y = fmaf(dt, v.y, a.y);
    a.z = fmaf(dt, v.z, a.z);
    a.w = fmaf(dt, v.w, a.w);
    reinterpret_cast<float4*>(x)[i] = a;
    if (vg) reinterpret_cast<float4*>(vg)[i] = v;
  }
  for (size_t i = n4 * 4 + blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n; i += stride) {
    const float v = fmaf(g, vc[i] - vu[i], vu[i]);
    x[i] = fmaf(dt, v, x[i]);
    if (vg) vg[i] = v;
  }
}

__global__ void blend_kernel(const float* __restrict__ x, const float* __restrict__ noise, float t,
                             float* __restrict__ out, size_t n) {
  pdl_trigger();
  pdl_wait();
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n; i += stride)
    out[i] = (1.0f - t) * x[i] + t * noise[i];
}

// ------------------------------------------------------------------ timestep embedding, GEMV
__global__ void timestep_embed_kernel(float* __restrict__ out, float t, int dim) {
  pdl_trigger();
  pdl_wait();
  const int half = dim / 2;
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= half) return;
  const double f = exp(-log(10000.0) * j / half);
  const double a = static_cast<double>(t) * 1000.0 * f;
  double s, c;
  sincos(a, &s, &c);
  out[j] = static_cast<float>(c);
  out[half + j] = static_cast<float>(s);
}

constexpr int kGemvRowsPerWarp = 4;
constexpr int kGemvWarps = 8;

// NV input vectors x[v] (k floats each, one after another) against one read of W:
// y[v * rows + r] = act_out(W[r] . act_in(x[v]) + b[r] + add[r]) (add may be NULL).
template <int NV>
__global__ void __launch_bounds__(256) gemv_kernel(const __nv_bfloat16* __restrict__ W,
                                                   const __nv_bfloat16* __restrict__ b, const float* __restrict__ x,
                                                   float* __restrict__ y, const float* __restrict__ add, int rows,
                                                   int k, int silu_in, int silu_out) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ float xs[];
  for (int i = threadIdx.x; i < NV * k; i += blockDim.x) {
    const float v = x[i];
    xs[i] = silu_in ? silu_f(v) : v;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunks = k / 8;
  for (int r0 = (blockIdx.x * kGemvWarps + warp) * kGemvRowsPerWarp; r0 < rows;
       r0 += gridDim.x * kGemvWarps * kGemvRowsPerWarp) {
    float acc[NV][kGemvRowsPerWarp] = {};
#pragma unroll 4
    for (int c = lane; c < chunks; c += 32) {
      uint4 w[kGemvRowsPerWarp];
#pragma unroll
      for (int rr = 0; rr < kGemvRowsPerWarp; ++rr)
        w[rr] = r0 + rr < rows ? __ldcs(reinterpret_cast<const uint4*>(W + static_cast<size_t>(r0 + rr) * k) + c)
                               : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        const float4 x0 = reinterpret_cast<const float4*>(xs + v * k)[2 * c];
        const float4 x1 = reinterpret_cast<const float4*>(xs + v * k)[2 * c + 1];
#pragma unroll
        for (int rr = 0; rr < kGemvRowsPerWarp; ++rr)
          acc[v][rr] += bf16lo(w[rr].x) * x0.x + bf16hi(w[rr].x) * x0.y + bf16lo(w[rr].y) * x0.z +
                        bf16hi(w[rr].y) * x0.w + bf16lo(w[rr].z) * x1.x + bf16hi(w[rr].z) * x1.y +
                        bf16lo(w[rr].w) * x1.z + bf16hi(w[rr].w) * x1.w;
      }
    }
#pragma unroll
    for (int v = 0; v < NV; ++v)
#pragma unroll
      for (int rr = 0; rr < kGemvRowsPerWarp; ++rr) {
        float a = acc[v][rr];
#pragma unroll
        for (int o = 16; o; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
        if (lane == 0 && r0 + rr < rows) {
          a += __bfloat162float(b[r0 + rr]);
          if (add) a += add[r0 + rr];
          y[static_cast<size_t>(v) * rows + r0 + rr] = silu_out ? silu_f(a) : a;
        }
      }
  }
}

}  // namespace

// One CTA per tile of kPackT tokens of one token row.
static cudaError_t pack_grid(int c, int h8, int w8, unsigned* tiles) {
  if (c != kPackC || h8 < 2 || w8 < 2 || (h8 | w8) & 1) return cudaErrorInvalidValue;
  const long t = static_cast<long>(h8 / 2) * ((w8 / 2 + kPackT - 1) / kPackT);
  if (t >= (1l << 31)) return cudaErrorInvalidValue;
  *tiles = static_cast<unsigned>(t);
  return cudaSuccess;
}

cudaError_t pack_latents_launch(const float* lat, float* tok, int c, int h8, int w8, cudaStream_t s) {
  unsigned tiles;
  if (const cudaError_t e = pack_grid(c, h8, w8, &tiles)) return e;
  count_launch();
  launch_kernel(pack_kernel, tiles, kPackThreads, 0, s, lat, tok, h8, w8);
  return cudaGetLastError();
}

cudaError_t unpack_latents_launch(const float* tok, float* lat, int c, int h8, int w8, cudaStream_t s) {
  unsigned tiles;
  if (const cudaError_t e = pack_grid(c, h8, w8, &tiles)) return e;
  count_launch();
  launch_kernel(unpack_kernel, tiles, kPackThreads, 0, s, tok, lat, h8, w8);
  return cudaGetLastError();
}

cudaError_t euler_launch(float* x, const float* v, size_t n, float dt, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  count_launch();
  launch_kernel(euler_kernel, blocks_for((n + 3) / 4, 256), 256, 0, s, x, v, n, dt);
  return cudaGetLastError();
}

cudaError_t cfg_euler_launch(float* x, const float* vc, const float* vu, float* vg, size_t n, float g, float dt,
                             cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  count_launch();
  launch_kernel(cfg_euler_kernel, blocks_for((n + 3) / 4, 256), 256, 0, s, x, vc, vu, vg, n, g, dt);
  return cudaGetLastError();
}

cudaError_t cast_bf16_launch(const float* x, __nv_bfloat16* y, size_t n, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  count_launch();
  launch_kernel(cast_bf16_kernel, blocks_for((n + 3) / 4, 256), 256, 0, s, x, y, n);
  return cudaGetLastError();
}

cudaError_t ln_modulate3_launch(const float* x, __nv_bfloat16* y, int rows, int dim, int split, int split2,
                                int period, const float* shift0, const float* scale0, const float* shift1,
                                const float* scale1, const float* shift2, const float* scale2, float eps,
                                cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  if (period <= 0) return cudaErrorInvalidValue;
  const LnModSets m = {split, split2, period, shift0, shift1, shift2, scale0, scale1, scale2};
  count_launch();
  if (dim == 3072)
    launch_kernel(ln_mod_kernel<3>, rows, 256, 0, s, x, y, rows, m, eps);
  else
    launch_kernel(ln_mod_generic_kernel, (rows + 7) / 8, 256, 0, s, x, y, rows, dim, m, eps);
  return cudaGetLastError();
}

cudaError_t ln_modulate_launch(const float* x, __nv_bfloat16* y, int rows, int dim, int split, int period,
                               const float* shift0, const float* scale0, const float* shift1, const float* scale1,
                               float eps, cudaStream_t s) {
  return ln_modulate3_launch(x, y, rows, dim, split, period, period, shift0, scale0, shift1, scale1, shift1, scale1,
                             eps, s);
}

cudaError_t qk_norm_rope_launch(__nv_bfloat16* qkv, int rows, int ld, int kcol, int heads, int split,
                                const __nv_bfloat16* gq0, const __nv_bfloat16* gk0, const __nv_bfloat16* gq1,
                                const __nv_bfloat16* gk1, const float2* rope, float eps, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  const int warps = rows * 2;
  count_launch();
  launch_kernel(qk_norm_rope_kernel, (warps + 7) / 8, 256, 0, s, qkv, rows, ld, kcol, heads, split, gq0, gk0, gq1, gk1, rope,
                                                      eps);
  return cudaGetLastError();
}

cudaError_t rope_table_launch(float2* table, int n_txt, int gh, int gw, const RefGrids& refs, float theta,
                              cudaStream_t s) {
  int n = n_txt + gh * gw;
  for (int k = 0; k < refs.count; ++k) n += refs.h[k] * refs.w[k];
  if (n <= 0) return cudaSuccess;
  count_launch();
  launch_kernel(rope_table_kernel, (n * 64 + 255) / 256, 256, 0, s, table, n_txt, gh, gw, refs, theta);
  return cudaGetLastError();
}

cudaError_t blend_launch(const float* x, const float* noise, float t, float* out, size_t n, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  count_launch();
  launch_kernel(blend_kernel, blocks_for(n, 256), 256, 0, s, x, noise, t, out, n);
  return cudaGetLastError();
}

cudaError_t timestep_embed_launch(float* temb, float t, int dim, cudaStream_t s) {
  count_launch();
  launch_kernel(timestep_embed_kernel, (dim / 2 + 127) / 128, 128, 0, s, temb, t, dim);
  return cudaGetLastError();
}

cudaError_t gemv_multi_launch(const __nv_bfloat16* W, const __nv_bfloat16* b, const float* x, int nvec, float* y,
                              const float* add, int rows, int k, int silu_in, int silu_out, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  if (nvec < 1 || nvec > 4 || k % 8) return cudaErrorInvalidValue;
  const int per_block = kGemvWarps * kGemvRowsPerWarp;
  int grid = (rows + per_block - 1) / per_block;
  const int cap = num_sms_current() * 8;
  if (grid > cap) grid = cap;
  const size_t smem = static_cast<size_t>(nvec) * k * sizeof(float);
  if (smem > 48 * 1024) return cudaErrorInvalidValue;
  count_launch();
  if (nvec == 1)
    launch_kernel(gemv_kernel<1>, grid, 256, smem, s, W, b, x, y, add, rows, k, silu_in, silu_out);
  else if (nvec == 2)
    launch_kernel(gemv_kernel<2>, grid, 256, smem, s, W, b, x, y, add, rows, k, silu_in, silu_out);
  else if (nvec == 3)
    launch_kernel(gemv_kernel<3>, grid, 256, smem, s, W, b, x, y, add, rows, k, silu_in, silu_out);
  else
    launch_kernel(gemv_kernel<4>, grid, 256, smem, s, W, b, x, y, add, rows, k, silu_in, silu_out);
  return cudaGetLastError();
}

cudaError_t gemv_launch(const __nv_bfloat16* W, const __nv_bfloat16* b, const float* x, float* y, int rows, int k,
                        int silu_in, int silu_out, cudaStream_t s) {
  return gemv_multi_launch(W, b, x, 1, y, nullptr, rows, k, silu_in, silu_out, s);
}

}  // namespace fdit
