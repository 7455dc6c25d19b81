// Fused GEMM epilogue with TMA stores (the NVFP4 pair kernel, gemm_fp4.cu).
//
// Same modes and arithmetic as gemm_epilogue.cuh, but a warp does not write its 32 accumulator rows
// with per-thread global stores (one row per thread: 32 separate 32-byte segments per store
// instruction).  Results are staged 64 bytes per row (32 bf16 or 16 fp32 columns) in one of this
// warp's two 2 KB shared memory buffers, in the 64-byte swizzled layout of a 32-row TMA box, and
// written by one bulk tensor store per box; the gated residual (X += gate * y) becomes a bulk
// tensor reduce-add of gate * y into X, so X is never read.  Rows and columns outside the output
// are clipped by the tensor map.  A buffer is refilled once the store issued from it two boxes
// earlier has read it.
#pragma once

#include "common.cuh"
#include "fluxdit_internal.h"
#include "gemm_epilogue.cuh"

namespace fdit {

struct EpiTma {
  const CUtensorMap* map;   // output of this problem (make_tmap_out)
  uint32_t buf0;            // shared address of this warp's two 2 KB staging buffers (1024-byte aligned)
  int y0;                   // output row of lane 0
  int rows;                 // output rows: a box starting at or past them is not issued
  uint32_t* which;          // the buffer the next chunk fills (0 or 1), kept across tiles
  __device__ __forceinline__ uint32_t buf() const { return buf0 + (*which << 11); }
};

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// The store issued from the buffer about to be filled (two chunks ago) has read it.
__device__ __forceinline__ void epi_tma_reuse() {
  if ((threadIdx.x & 31) == 0) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
  __syncwarp();
}

// Row `lane` of half h of a fp32 chunk (16 of its 32 values) into the 64-byte swizzled box layout.
__device__ __forceinline__ void epi_stage_f32(const EpiTma& e, const float (&f)[32], int h) {
  const uint32_t t = threadIdx.x & 31;
#pragma unroll
  for (uint32_t u = 0; u < 4; ++u)
    st_shared_v4(e.buf() + t * 64 + ((u ^ ((t >> 1) & 3)) << 4), __float_as_uint(f[16 * h + 4 * u]),
                 __float_as_uint(f[16 * h + 4 * u + 1]), __float_as_uint(f[16 * h + 4 * u + 2]),
                 __float_as_uint(f[16 * h + 4 * u + 3]));
}
// Row `lane` of a bf16 chunk (32 values, 16 packed words) into the 64-byte swizzled box layout.
__device__ __forceinline__ void epi_stage_bf16(const EpiTma& e, const uint32_t (&w)[16]) {
  const uint32_t t = threadIdx.x & 31;
#pragma unroll
  for (uint32_t u = 0; u < 4; ++u)
    st_shared_v4(e.buf() + t * 64 + ((u ^ ((t >> 1) & 3)) << 4), w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
}

// Store (or, with add, reduce-add) the staged 32-row box at output column x; the next box
// takes the other buffer.  Lane 0 (which issues and waits for every store of the warp) commits a
// group, possibly empty, per chunk, so that "all but the latest group" is always the buffer being
// refilled.
__device__ __forceinline__ void epi_tma_issue(const EpiTma& e, int x, bool add) {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // staged values visible to the bulk copy
  __syncwarp();
  const uint32_t buf = e.buf();
  *e.which ^= 1u;
  if ((threadIdx.x & 31) == 0) {
    if (e.y0 < e.rows) {
      if (add)
        asm volatile(
            "cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                reinterpret_cast<uint64_t>(e.map)),
            "r"(buf), "r"(x), "r"(e.y0)
            : "memory");
      else
        asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                         reinterpret_cast<uint64_t>(e.map)),
                     "r"(buf), "r"(x), "r"(e.y0)
                     : "memory");
    }
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
  }
}

// Every bulk store of this warp has completed (before the kernel exits).
__device__ __forceinline__ void epi_tma_drain() {
  if ((threadIdx.x & 31) == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  __syncwarp();
}

// One accumulator tile, as gemm_epilogue_tile<BN, kScale, kParts, kOvl>, with TMA stores.
template <int BN, bool kScale, int kParts, bool kOvl>
__device__ __forceinline__ void gemm_epilogue_tile_tma(const GemmProblem& pr, uint32_t tbase, int m, int n0, int part,
                                                       int ovl_side, uint32_t ovl_bar, const EpiTma& e) {
  static_assert(BN % (128 * kParts) == 0, "each part must hold whole 128-wide heads");
  const bool row_ok = m < pr.M;
  const bool ovl_mine = kOvl && ((ovl_side == 0 && part == kParts - 1) || (ovl_side == 1 && part == 0));
  float sa = 0.f;
  if constexpr (kScale) sa = row_ok ? __ldg(pr.scale_a + m) : 0.f;
  if (pr.mode == kEpiSwiGLU) {
    const int on0 = n0 / 2;
    constexpr int kSw = BN / 2 / kParts;
#pragma unroll 1
    for (int c0 = part * kSw; c0 < (part + 1) * kSw; c0 += 32) {
      const int c = (kOvl && ovl_mine && ovl_side == 0) ? (part + 1) * kSw - 32 - (c0 - part * kSw) : c0;
      uint32_t ra[32], rb[32];
      tmem_ld32(tbase + c, ra);
      tmem_ld32(tbase + BN / 2 + c, rb);
      tmem_ld_wait();
      if constexpr (kOvl) {
        if (ovl_mine && c0 == part * kSw) ovl_release(ovl_bar);
      }
      if (n0 + c >= pr.N) continue;
      const uint4* ba = reinterpret_cast<const uint4*>(pr.bias + n0 + c);
      const uint4* bb = reinterpret_cast<const uint4*>(pr.bias + n0 + BN / 2 + c);
      uint32_t ob[16];
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const uint4 wa = __ldg(ba + v), wb = __ldg(bb + v);
        const uint32_t xa[4] = {wa.x, wa.y, wa.z, wa.w}, xb[4] = {wb.x, wb.y, wb.z, wb.w};
        float fa[8], fb[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          fa[q] = __uint_as_float(ra[v * 8 + q]);
          fb[q] = __uint_as_float(rb[v * 8 + q]);
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
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float a0 = fa[2 * q] + bf16lo(xa[q]);
          const float a1 = fa[2 * q + 1] + bf16hi(xa[q]);
          const float b0 = fb[2 * q] + bf16lo(xb[q]);
          const float b1 = fb[2 * q + 1] + bf16hi(xb[q]);
          ob[4 * v + q] = pack_bf16x2(silu_f(a0) * b0, silu_f(a1) * b1);
        }
      }
      epi_tma_reuse();
      epi_stage_bf16(e, ob);
      epi_tma_issue(e, on0 + c, false);
    }
  } else if (pr.mode == kEpiQKNormRope && n0 < 2 * (pr.N / 3)) {
    const bool is_k = n0 >= pr.N / 3;
    const __nv_bfloat16* gain = is_k ? pr.gain_k : pr.gain_q;
    const float4* rrow =
        reinterpret_cast<const float4*>(pr.rope + static_cast<size_t>(pr.rope_row0 + (row_ok ? m : 0)) * 64);
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
          for (int q = 0; q < 4; ++q) {
            const float a0 = __uint_as_float(r[v * 8 + q * 2]) + bf16lo(x[q]);
            const float a1 = __uint_as_float(r[v * 8 + q * 2 + 1]) + bf16hi(x[q]);
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
        scale_chunk<kScale>(r, sa, pr.scale_b + n0 + hh * 128 + c);
        const uint4* bsrc = reinterpret_cast<const uint4*>(bh + c);
        const uint4* gsrc = reinterpret_cast<const uint4*>(gain + c);
        uint32_t ob[16];
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const uint4 w = __ldg(bsrc + v), g = __ldg(gsrc + v);
          const uint32_t x[4] = {w.x, w.y, w.z, w.w}, gg[4] = {g.x, g.y, g.z, g.w};
          const float4 cs01 = __ldg(rrow + (c + v * 8) / 4);
          const float4 cs23 = __ldg(rrow + (c + v * 8) / 4 + 1);
          const float cs[4] = {cs01.x, cs01.z, cs23.x, cs23.z};
          const float sn[4] = {cs01.y, cs01.w, cs23.y, cs23.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float a0 = (__uint_as_float(r[v * 8 + q * 2]) + bf16lo(x[q])) * rstd * bf16lo(gg[q]);
            const float a1 = (__uint_as_float(r[v * 8 + q * 2 + 1]) + bf16hi(x[q])) * rstd * bf16hi(gg[q]);
            ob[4 * v + q] = pack_bf16x2(a0 * cs[q] - a1 * sn[q], a0 * sn[q] + a1 * cs[q]);
          }
        }
        epi_tma_reuse();
        epi_stage_bf16(e, ob);
        epi_tma_issue(e, n0 + hh * 128 + c, false);
      }
    }
    if constexpr (kOvl) {
      if (ovl_mine) ovl_release(ovl_bar);
    }
  } else {
    constexpr int kCols = BN / kParts;
#pragma unroll 1
    for (int c0 = part * kCols; c0 < (part + 1) * kCols; c0 += 32) {
      const int c = (kOvl && ovl_mine && ovl_side == 0) ? (part + 1) * kCols - 32 - (c0 - part * kCols) : c0;
      uint32_t r[32];
      tmem_ld32(tbase + c, r);
      tmem_ld_wait();
      if constexpr (kOvl) {
        if (ovl_mine && c0 == part * kCols) ovl_release(ovl_bar);
      }
      const int n = n0 + c;
      if (n >= pr.N) continue;
      scale_chunk<kScale>(r, sa, pr.scale_b + n);
      const uint4* bsrc = reinterpret_cast<const uint4*>(pr.bias + n);
      float f[32];
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const uint4 w = __ldg(bsrc + v);
        const uint32_t x[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          f[v * 8 + q * 2] = __uint_as_float(r[v * 8 + q * 2]) + bf16lo(x[q]);
          f[v * 8 + q * 2 + 1] = __uint_as_float(r[v * 8 + q * 2 + 1]) + bf16hi(x[q]);
        }
      }
      epi_tma_reuse();
      if (pr.mode == kEpiBf16Bias || pr.mode == kEpiQKNormRope) {
        uint32_t ob[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) ob[q] = pack_bf16x2(f[2 * q], f[2 * q + 1]);
        epi_stage_bf16(e, ob);
        epi_tma_issue(e, n, false);
      } else {
        if (pr.mode == kEpiResidGate) {            // the residual takes gate * y by reduce-add
          const float4* g = reinterpret_cast<const float4*>(pr.gate + n);
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            const float4 gv = __ldg(g + v);
            f[4 * v] *= gv.x; f[4 * v + 1] *= gv.y; f[4 * v + 2] *= gv.z; f[4 * v + 3] *= gv.w;
          }
        }
        epi_stage_f32(e, f, 0);
        epi_tma_issue(e, n, pr.mode == kEpiResidGate);
        epi_tma_reuse();
        epi_stage_f32(e, f, 1);
        epi_tma_issue(e, n + 16, pr.mode == kEpiResidGate);
      }
    }
  }
}

}  // namespace fdit
