// Fused epilogue shared by the one-CTA (gemm_tc.cu) and CTA-pair (gemm_tc2.cu) tcgen05 GEMMs.
//
// Called by one epilogue warp for one accumulator tile; thread i of the warp owns accumulator
// row m (global row of this problem) whose BN fp32 columns start at TMEM address `tbase`.  With
// kParts > 1 the tile's columns are shared by kParts warps of the same lane quarter and this call
// handles part `part`: a contiguous 1/kParts of the columns (of the a/b pairs for SwiGLU, of the
// 128-wide heads for the fused QK-RMSNorm).
// Every tcgen05.ld is warp-collective, so rows outside the problem still load and only skip
// their global stores.
#pragma once

#include "common.cuh"
#include "fluxdit_internal.h"

namespace fdit {

// kScale (8-bit operands): acc[m][n] *= scale_a[m] * scale_b[n] as each 32-column chunk is read.
template <bool kScale>
__device__ __forceinline__ void scale_chunk(uint32_t (&r)[32], float sa, const float* sb) {
  if constexpr (kScale) {
    const float4* s4 = reinterpret_cast<const float4*>(sb);
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      const float4 w = __ldg(s4 + v);
      r[4 * v + 0] = __float_as_uint(__uint_as_float(r[4 * v + 0]) * sa * w.x);
      r[4 * v + 1] = __float_as_uint(__uint_as_float(r[4 * v + 1]) * sa * w.y);
      r[4 * v + 2] = __float_as_uint(__uint_as_float(r[4 * v + 2]) * sa * w.z);
      r[4 * v + 3] = __float_as_uint(__uint_as_float(r[4 * v + 3]) * sa * w.w);
    }
  }
}

// 32 bf16 values (16 packed words) of one row: two 32-byte stores when aligned, else four 16-byte ones.
__device__ __forceinline__ void store_bf16x32(__nv_bfloat16* dst, const uint32_t (&w)[16], bool v8) {
  if (v8) {
    st_global_v8(reinterpret_cast<uint32_t*>(dst), w);
    st_global_v8(reinterpret_cast<uint32_t*>(dst) + 8, w + 8);
  } else {
    uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int v = 0; v < 4; ++v) d[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
  }
}

// Overlapping accumulators (kOvl, the NVFP4 kernel): the tile's TMEM columns share 32 columns with
// the other accumulator buffer, the last 32 (ovl_side 0) or the first 32 (ovl_side 1).  The part
// that owns them drains that chunk first and then arrives on the barrier at `ovl_bar` (a
// shared::cluster address), so the next tile's MMAs may start while the rest of this tile drains.
// Under the fused QK-RMSNorm a head is read twice, so the owning part arrives when its head is done.
__device__ __forceinline__ void ovl_release(uint32_t ovl_bar) {
  tc_fence_before();
  __syncwarp();
  if ((threadIdx.x & 31) == 0)
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(ovl_bar) : "memory");
}

template <int BN, bool kScale = false, int kParts = 1, bool kOvl = false>
__device__ __forceinline__ void gemm_epilogue_tile(const GemmProblem& pr, uint32_t tbase, int m, int n0,
                                                   int part = 0, int ovl_side = -1, uint32_t ovl_bar = 0) {
  static_assert(BN % (128 * kParts) == 0, "each part must hold whole 128-wide heads");
  // this part owns the shared columns: the last part for side 0, the first for side 1
  const bool ovl_mine = kOvl && ((ovl_side == 0 && part == kParts - 1) || (ovl_side == 1 && part == 0));
  const bool row_ok = m < pr.M;
  // fp32 outputs whose rows start on 32-byte boundaries take 256-bit loads / stores
  const bool v8_ok = ((reinterpret_cast<uintptr_t>(pr.out) | (static_cast<uintptr_t>(pr.ldo) * 4)) & 31) == 0;
  const bool v8b_ok = ((reinterpret_cast<uintptr_t>(pr.out) | (static_cast<uintptr_t>(pr.ldo) * 2)) & 31) == 0;
  float sa = 0.f;                          // row scale (kScale only; rows outside the problem read none)
  if constexpr (kScale) sa = row_ok ? __ldg(pr.scale_a + m) : 0.f;
  if (pr.mode == kEpiSwiGLU) {
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(pr.out);
    const int on0 = n0 / 2;                // output column of this tile's first pair
    constexpr int kSw = BN / 2 / kParts;             // pairs per part
#pragma unroll 1
    for (int c0 = part * kSw; c0 < (part + 1) * kSw; c0 += 32) {
      // side 0 shares the last b chunk: the owning part walks its pairs from the end
      const int c = (kOvl && ovl_mine && ovl_side == 0) ? (part + 1) * kSw - 32 - (c0 - part * kSw) : c0;
      uint32_t ra[32], rb[32];
      tmem_ld32(tbase + c, ra);
      tmem_ld32(tbase + BN / 2 + c, rb);
      tmem_ld_wait();
      if constexpr (kOvl) {
        if (ovl_mine && c0 == part * kSw) ovl_release(ovl_bar);
      }
      if (row_ok && n0 + c < pr.N) {
        const uint4* ba = reinterpret_cast<const uint4*>(pr.bias + n0 + c);
        const uint4* bb = reinterpret_cast<const uint4*>(pr.bias + n0 + BN / 2 + c);
        __nv_bfloat16* dstp = out + static_cast<size_t>(m) * pr.ldo + on0 + c;
        uint32_t ob[16];                             // this chunk's 32 outputs, packed
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const uint4 wa = __ldg(ba + v), wb = __ldg(bb + v);
          const uint32_t xa[4] = {wa.x, wa.y, wa.z, wa.w}, xb[4] = {wb.x, wb.y, wb.z, wb.w};
          float fa[8], fb[8];                        // accumulators of these 8 columns, scaled (kScale)
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            fa[e] = __uint_as_float(ra[v * 8 + e]);
            fb[e] = __uint_as_float(rb[v * 8 + e]);
          }
          if constexpr (kScale) {
            const float4* sa4 = reinterpret_cast<const float4*>(pr.scale_b + n0 + c + v * 8);
            const float4* sb4 = reinterpret_cast<const float4*>(pr.scale_b + n0 + BN / 2 + c + v * 8);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const float4 ka = __ldg(sa4 + h), kb = __ldg(sb4 + h);
              fa[4 * h] *= sa * ka.x; fa[4 * h + 1] *= sa * ka.y; fa[4 * h + 2] *= sa * ka.z; fa[4 * h + 3] *= sa * ka.w;
              fb[4 * h] *= sa * kb.x; fb[4 * h + 1] *= sa * kb.y; fb[4 * h + 2] *= sa * kb.z; fb[4 * h + 3] *= sa * kb.w;
            }
          }
          uint32_t o[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float a0 = fa[2 * e] + bf16lo(xa[e]);
            const float a1 = fa[2 * e + 1] + bf16hi(xa[e]);
            const float b0 = fb[2 * e] + bf16lo(xb[e]);
            const float b1 = fb[2 * e + 1] + bf16hi(xb[e]);
            o[e] = pack_bf16x2(silu_f(a0) * b0, silu_f(a1) * b1);
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) ob[4 * v + e] = o[e];
        }
        store_bf16x32(dstp, ob, v8b_ok);
      }
    }
  } else if (pr.mode == kEpiQKNormRope && n0 < 2 * (pr.N / 3)) {
    const bool is_k = n0 >= pr.N / 3;
    const __nv_bfloat16* gain = is_k ? pr.gain_k : pr.gain_q;
    const float4* rrow = reinterpret_cast<const float4*>(pr.rope + static_cast<size_t>(pr.rope_row0 + (row_ok ? m : 0)) * 64);
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(pr.out);
#pragma unroll 1
    for (int hh = part * (BN / 128 / kParts); hh < (part + 1) * (BN / 128 / kParts); ++hh) {
      const uint32_t hb = tbase + hh * 128;
      const __nv_bfloat16* bh = pr.bias + n0 + hh * 128;
      float ss = 0.f;
#pragma unroll 1
      for (int c = 0; c < 128; c += 32) {           // pass 1: sum of squares of the head
        uint32_t r[32];
        tmem_ld32(hb + c, r);
        tmem_ld_wait();
        if (row_ok) scale_chunk<kScale>(r, sa, pr.scale_b + n0 + hh * 128 + c);
        const uint4* bsrc = reinterpret_cast<const uint4*>(bh + c);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const uint4 w = __ldg(bsrc + v);
          const uint32_t x[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float a0 = __uint_as_float(r[v * 8 + e * 2]) + bf16lo(x[e]);
            const float a1 = __uint_as_float(r[v * 8 + e * 2 + 1]) + bf16hi(x[e]);
            ss = fmaf(a0, a0, fmaf(a1, a1, ss));
          }
        }
      }
      const float rstd = rsqrtf(ss * (1.0f / 128.0f) + pr.eps);
#pragma unroll 1
      for (int c = 0; c < 128; c += 32) {           // pass 2: normalise, gain, rotate, store
        uint32_t r[32];
        tmem_ld32(hb + c, r);
        tmem_ld_wait();
        if (!row_ok) continue;
        scale_chunk<kScale>(r, sa, pr.scale_b + n0 + hh * 128 + c);
        const uint4* bsrc = reinterpret_cast<const uint4*>(bh + c);
        const uint4* gsrc = reinterpret_cast<const uint4*>(gain + c);
        __nv_bfloat16* dstp = out + static_cast<size_t>(m) * pr.ldo + n0 + hh * 128 + c;
        uint32_t ob[16];
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const uint4 w = __ldg(bsrc + v), g = __ldg(gsrc + v);
          const uint32_t x[4] = {w.x, w.y, w.z, w.w}, gg[4] = {g.x, g.y, g.z, g.w};
          const float4 cs01 = __ldg(rrow + (c + v * 8) / 4);       // (cos, sin) of pairs p, p+1
          const float4 cs23 = __ldg(rrow + (c + v * 8) / 4 + 1);   // pairs p+2, p+3
          const float cs[4] = {cs01.x, cs01.z, cs23.x, cs23.z};
          const float sn[4] = {cs01.y, cs01.w, cs23.y, cs23.w};
          uint32_t o[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float a0 = (__uint_as_float(r[v * 8 + e * 2]) + bf16lo(x[e])) * rstd * bf16lo(gg[e]);
            const float a1 = (__uint_as_float(r[v * 8 + e * 2 + 1]) + bf16hi(x[e])) * rstd * bf16hi(gg[e]);
            o[e] = pack_bf16x2(a0 * cs[e] - a1 * sn[e], a0 * sn[e] + a1 * cs[e]);
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) ob[4 * v + e] = o[e];
        }
        store_bf16x32(dstp, ob, v8b_ok);
      }
    }
    if constexpr (kOvl) {
      if (ovl_mine) ovl_release(ovl_bar);
    }
  } else {
    constexpr int kCols = BN / kParts;              // columns per part
#pragma unroll 1
    for (int c0 = part * kCols; c0 < (part + 1) * kCols; c0 += 32) {
      // side 0 shares the tile's last chunk: the owning part walks its columns from the end
      const int c = (kOvl && ovl_mine && ovl_side == 0) ? (part + 1) * kCols - 32 - (c0 - part * kCols) : c0;
      uint32_t r[32];
      tmem_ld32(tbase + c, r);
      tmem_ld_wait();
      if constexpr (kOvl) {
        if (ovl_mine && c0 == part * kCols) ovl_release(ovl_bar);
      }
      const int n = n0 + c;
      if (!row_ok || n >= pr.N) continue;
      scale_chunk<kScale>(r, sa, pr.scale_b + n);
      const uint4* bsrc = reinterpret_cast<const uint4*>(pr.bias + n);
      float f[32];
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const uint4 w = __ldg(bsrc + v);
        const uint32_t x[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          f[v * 8 + e * 2] = __uint_as_float(r[v * 8 + e * 2]) + bf16lo(x[e]);
          f[v * 8 + e * 2 + 1] = __uint_as_float(r[v * 8 + e * 2 + 1]) + bf16hi(x[e]);
        }
      }
      if (pr.mode == kEpiBf16Bias || pr.mode == kEpiQKNormRope) {
        uint32_t ob[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) ob[e] = pack_bf16x2(f[2 * e], f[2 * e + 1]);
        store_bf16x32(static_cast<__nv_bfloat16*>(pr.out) + static_cast<size_t>(m) * pr.ldo + n, ob, v8b_ok);
      } else if (pr.mode == kEpiF32Bias) {
        float* dstp = static_cast<float*>(pr.out) + static_cast<size_t>(m) * pr.ldo + n;
        if (v8_ok) {                        // one 32-byte access per 8 values: half the L1 wavefronts
#pragma unroll
          for (int v = 0; v < 4; ++v) st_global_v8(dstp + 8 * v, f + 8 * v);
        } else {
          float4* dst = reinterpret_cast<float4*>(dstp);
#pragma unroll
          for (int v = 0; v < 8; ++v) dst[v] = make_float4(f[v * 4], f[v * 4 + 1], f[v * 4 + 2], f[v * 4 + 3]);
        }
      } else if (v8_ok) {                   // kEpiResidGate, 32-byte accesses
        float* xp = static_cast<float*>(pr.out) + static_cast<size_t>(m) * pr.ldo + n;
        const float4* g = reinterpret_cast<const float4*>(pr.gate + n);
        float xv[4][8];
#pragma unroll
        for (int v = 0; v < 4; ++v) ld_global_v8(xp + 8 * v, xv[v]);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const float4 g0 = __ldg(g + 2 * v), g1 = __ldg(g + 2 * v + 1);
          xv[v][0] = fmaf(g0.x, f[8 * v + 0], xv[v][0]);
          xv[v][1] = fmaf(g0.y, f[8 * v + 1], xv[v][1]);
          xv[v][2] = fmaf(g0.z, f[8 * v + 2], xv[v][2]);
          xv[v][3] = fmaf(g0.w, f[8 * v + 3], xv[v][3]);
          xv[v][4] = fmaf(g1.x, f[8 * v + 4], xv[v][4]);
          xv[v][5] = fmaf(g1.y, f[8 * v + 5], xv[v][5]);
          xv[v][6] = fmaf(g1.z, f[8 * v + 6], xv[v][6]);
          xv[v][7] = fmaf(g1.w, f[8 * v + 7], xv[v][7]);
          st_global_v8(xp + 8 * v, xv[v]);
        }
      } else {                              // kEpiResidGate
        float4* x = reinterpret_cast<float4*>(static_cast<float*>(pr.out) + static_cast<size_t>(m) * pr.ldo + n);
        const float4* g = reinterpret_cast<const float4*>(pr.gate + n);
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          float4 xv = x[v];
          const float4 gv = __ldg(g + v);
          xv.x += gv.x * f[v * 4];
          xv.y += gv.y * f[v * 4 + 1];
          xv.z += gv.z * f[v * 4 + 2];
          xv.w += gv.w * f[v * 4 + 3];
          x[v] = xv;
        }
      }
    }
  }
}

}  // namespace fdit
