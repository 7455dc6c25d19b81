// Persistent tcgen05 GEMM for the transformer's linear layers, C = A W^T (+ fused epilogue).
//
//   A [M, K] bf16 row-major (activations), W [N, K] bf16 row-major (nn.Linear
//   [out, in] layout), fp32 accumulation in tensor memory.
//
// One launch runs up to kMaxProblems independent problems (the text and image
// streams of a double block, or the qkv and SwiGLU halves of a single block's
// fused first linear), so both fill one persistent grid.
//
// CTA = 6 warps: warp 0 issues TMA loads into a STAGES-deep shared-memory ring,
// one thread of warp 1 issues tcgen05.mma into one of two TMEM accumulators
// (BN columns each), warps 2..5 drain the other accumulator through the fused
// epilogue, so tile i's epilogue overlaps tile i+1's MMAs.
//
// Epilogues (the transformer operations they implement, FLUX.3 Image Klein in
// Diffusers write-up, "Entkoppelte Vorverarbeitung und gemeinsame
// Attention-Blöcke" and "Modulation pro Token-Typ ..."):
//   kEpiBf16Bias    out_bf16 = acc + bias                  (qkv projections)
//   kEpiF32Bias     out_f32  = acc + bias                  (input / output projections)
//   kEpiSwiGLU      out_bf16 = silu(a + ba) * (b + bb)     (SwiGLU MLP; W rows pre-interleaved
//                                                          so a tile holds BN/2 a-rows then
//                                                          the matching BN/2 b-rows)
//   kEpiResidGate   X_f32   += gate * (acc + bias)         (gated residual add)
#include <cstdio>

#include "common.cuh"
#include "fluxdit_internal.h"

namespace fdit {

__device__ int g_gemm_error;

namespace {

constexpr int BM = 128;
constexpr int BK = 64;

template <int BN>
struct GemmCfg {
  static constexpr int STAGES = BN == 256 ? 4 : 6;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TMEM_COLS = 2 * BN;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
};

__device__ __forceinline__ int find_problem(const GemmParams& P, int tile) {
  int p = 0;
#pragma unroll 1
  for (int i = 1; i < P.num_problems; ++i)
    if (tile >= P.prob[i].tile_begin) p = i;
  return p;
}

template <int BN>
__global__ void __launch_bounds__(192, 1) gemm_bf16_tc_kernel(const __grid_constant__ GemmParams P) {
  using C = GemmCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::STAGES * C::A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* acc_full = empty + C::STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < P.num_problems; ++i) {
      tma_prefetch_map(&P.mapA[i]);
      tma_prefetch_map(&P.mapB[i]);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0;             // bit s: stage s was armed at least once
      uint32_t armed_phase = 0;       // bit s: phase parity of the last arming of stage s
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < P.total_tiles; tile += gridDim.x) {
        const int p = find_problem(P, tile);
        const GemmProblem& pr = P.prob[p];
        const int lt = tile - pr.tile_begin;
        const int m0 = (lt % pr.tiles_m) * BM;
        const int n0 = (lt / pr.tiles_m) * BN;
        const int nk = pr.K / BK;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
          tma_load_2d(sA + stage * C::A_BYTES, &P.mapA[p], &full[stage], kb * BK, m0);
          tma_load_2d(sB + stage * C::B_BYTES, &P.mapB[p], &full[stage], kb * BK, n0);
          armed |= 1u << stage;
          armed_phase = (armed_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        atomicExch(&g_gemm_error, kErrTimeoutProducer);
        for (int s = 0; s < C::STAGES; ++s)      // let issued copies land before the CTA exits
          if (armed & (1u << s)) mbar_drain(&full[s], (armed_phase >> s) & 1u);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < P.total_tiles; tile += gridDim.x) {
        const int p = find_problem(P, tile);
        const GemmProblem& pr = P.prob[p];
        const int nk = pr.K / BK;
        const uint32_t idesc = idesc_bf16_f32(BM, BN, 0, 0);
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * C::A_BYTES);
          const uint32_t b_addr = smem_u32(sB + stage * C::B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t ad = sw128_desc(a_addr + k * 32, 16, 1024);
            const uint64_t bd = sw128_desc(b_addr + k * 32, 16, 1024);
            mma_ss(d_tmem, ad, bd, idesc, (kb | k) != 0 ? 1u : 0u);
          }
          mma_commit(&empty[stage]);           // frees the smem stage once these MMAs retire
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(&acc_full[acc]);            // accumulator ready for the epilogue
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (!ok) atomicExch(&g_gemm_error, kErrTimeoutMma);
      mma_commit(drain);                       // every MMA issued by this thread has retired ...
      mbar_drain(drain, 0);                    // ... before TMEM is released
    }
  } else {
    // -------------------------------------------------------------- epilogue warps 2..5
    const int quarter = warp & 3;              // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;       // accumulator row of this thread
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < P.total_tiles; tile += gridDim.x) {
      const int p = find_problem(P, tile);
      const GemmProblem& pr = P.prob[p];
      const int lt = tile - pr.tile_begin;
      const int m = (lt % pr.tiles_m) * BM + row;
      const int n0 = (lt / pr.tiles_m) * BN;
      if (!mbar_wait(&acc_full[acc], acc_phase, abort_flag)) {
        atomicExch(&g_gemm_error, kErrTimeoutEpilogue);
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem_base + lane_addr + static_cast<uint32_t>(acc * BN);
      const bool row_ok = m < pr.M;
      if (pr.mode == kEpiSwiGLU) {
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(pr.out);
        const int on0 = n0 / 2;                // output column of this tile's first pair
#pragma unroll 1
        for (int c = 0; c < BN / 2; c += 32) {
          uint32_t ra[32], rb[32];
          tmem_ld32(tbase + c, ra);
          tmem_ld32(tbase + BN / 2 + c, rb);
          tmem_ld_wait();
          if (row_ok && n0 + c < pr.N) {
            const uint4* ba = reinterpret_cast<const uint4*>(pr.bias + n0 + c);
            const uint4* bb = reinterpret_cast<const uint4*>(pr.bias + n0 + BN / 2 + c);
            uint4* dst = reinterpret_cast<uint4*>(out + static_cast<size_t>(m) * pr.ldo + on0 + c);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const uint4 wa = __ldg(ba + v), wb = __ldg(bb + v);
              const uint32_t xa[4] = {wa.x, wa.y, wa.z, wa.w}, xb[4] = {wb.x, wb.y, wb.z, wb.w};
              uint32_t o[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int j = v * 8 + e * 2;
                const float a0 = __uint_as_float(ra[j]) + bf16lo(xa[e]);
                const float a1 = __uint_as_float(ra[j + 1]) + bf16hi(xa[e]);
                const float b0 = __uint_as_float(rb[j]) + bf16lo(xb[e]);
                const float b1 = __uint_as_float(rb[j + 1]) + bf16hi(xb[e]);
                o[e] = pack_bf16x2(silu_f(a0) * b0, silu_f(a1) * b1);
              }
              dst[v] = make_uint4(o[0], o[1], o[2], o[3]);
            }
          }
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t r[32];
          tmem_ld32(tbase + c, r);
          tmem_ld_wait();
          const int n = n0 + c;
          if (!row_ok || n >= pr.N) continue;
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
          if (pr.mode == kEpiBf16Bias) {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(pr.out) +
                                                  static_cast<size_t>(m) * pr.ldo + n);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              dst[v] = make_uint4(pack_bf16x2(f[v * 8 + 0], f[v * 8 + 1]), pack_bf16x2(f[v * 8 + 2], f[v * 8 + 3]),
                                  pack_bf16x2(f[v * 8 + 4], f[v * 8 + 5]), pack_bf16x2(f[v * 8 + 6], f[v * 8 + 7]));
          } else if (pr.mode == kEpiF32Bias) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(pr.out) + static_cast<size_t>(m) * pr.ldo + n);
#pragma unroll
            for (int v = 0; v < 8; ++v) dst[v] = make_float4(f[v * 4], f[v * 4 + 1], f[v * 4 + 2], f[v * 4 + 3]);
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
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

template <int BN>
cudaError_t launch_bn(GemmParams& P, int num_sms, cudaStream_t stream) {
  using C = GemmCfg<BN>;
  static bool attr_set = false;          // per process; the attribute is per function
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(gemm_bf16_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int grid = P.total_tiles < num_sms ? P.total_tiles : num_sms;
  count_launch();
  gemm_bf16_tc_kernel<BN><<<grid, 192, C::SMEM_BYTES, stream>>>(P);
  return cudaGetLastError();
}

}  // namespace

int gemm_bn_for(int n) { return n <= 128 ? 128 : 256; }

// Fill tile bookkeeping and launch.  Problems with no rows are dropped.
cudaError_t gemm_launch(GemmParams& P, int bn, int num_sms, cudaStream_t stream) {
  int w = 0, total = 0;
  for (int i = 0; i < P.num_problems; ++i) {
    GemmProblem pr = P.prob[i];
    if (pr.M <= 0 || pr.N <= 0) continue;
    pr.tiles_m = (pr.M + BM - 1) / BM;
    pr.tiles_n = (pr.N + bn - 1) / bn;
    pr.tile_begin = total;
    total += pr.tiles_m * pr.tiles_n;
    if (w != i) {
      P.mapA[w] = P.mapA[i];
      P.mapB[w] = P.mapB[i];
    }
    P.prob[w++] = pr;
  }
  P.num_problems = w;
  P.total_tiles = total;
  if (total == 0) return cudaSuccess;
  return bn == 128 ? launch_bn<128>(P, num_sms, stream) : launch_bn<256>(P, num_sms, stream);
}

int gemm_read_device_error(cudaStream_t stream) {
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbolAsync(&v, g_gemm_error, sizeof(int), 0, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return -1;
  cudaMemcpyToSymbolAsync(g_gemm_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, stream);
  cudaStreamSynchronize(stream);
  return v;
}

}  // namespace fdit
