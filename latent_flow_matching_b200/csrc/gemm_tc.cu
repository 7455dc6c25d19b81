// Persistent one-CTA tcgen05 GEMM, C = A W^T (+ fused epilogue), 128 x 128 tiles: used for the
// 128-wide output projection and small standalone calls.  The wide linear layers of the forward
// run on the CTA-pair kernel (gemm_tc2.cu), which shares this file's epilogue (gemm_epilogue.cuh).
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
//   kEpiQKNormRope  out_bf16 = rope(rms(acc + bias) * gain) on the q and k heads, acc + bias on v
//                                                          (fused qkv projection + QK-RMSNorm + RoPE;
//                                                          a 256-column tile is two whole heads)
#include <cstdio>

#include "common.cuh"
#include "fluxdit_internal.h"
#include "gemm_epilogue.cuh"

namespace fdit {

__device__ int g_gemm_error;

namespace {

constexpr int BM = 128;
constexpr int BK = 64;

template <int BN>
struct GemmCfg {
  static constexpr int STAGES = 6;
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
  pdl_trigger();                                    // after this CTA's tensor-memory allocation
  pdl_wait();                                       // the previous kernel's writes are visible

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
    {
      // ------------------------------------------------------------ MMA issuer (whole warp, one elected lane issues)
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      const uint64_t a_desc0 = sw128_desc(smem_u32(sA), 16, 1024);
      const uint64_t b_desc0 = sw128_desc(smem_u32(sB), 16, 1024);
      for (int tile = blockIdx.x; ok && tile < P.total_tiles; tile += gridDim.x) {
        const int p = find_problem(P, tile);
        const GemmProblem& pr = P.prob[p];
        const int nk = pr.K / BK;
        const uint32_t idesc = idesc_bf16_f32(BM, BN, 0, 0);
        if (!mbar_wait_warp(&acc_empty[acc], acc_phase ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait_warp(&full[stage], phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = desc_advance(a_desc0, stage * C::A_BYTES);
          const uint64_t bd = desc_advance(b_desc0, stage * C::B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            mma_ss_warp(d_tmem, desc_advance(ad, k * 32), desc_advance(bd, k * 32), idesc, (kb | k) != 0 ? 1u : 0u);
          mma_commit_warp(&empty[stage]);           // frees the smem stage once these MMAs retire
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit_warp(&acc_full[acc]);            // accumulator ready for the epilogue
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (!ok && lane == 0) atomicExch(&g_gemm_error, kErrTimeoutMma);
      mma_commit_warp(drain);                       // every MMA issued by the elected lane has retired ...
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
      gemm_epilogue_tile<BN>(pr, tbase, m, n0);
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
  static std::atomic<unsigned long long> attr_done{0};   // one per tile width: the attribute is per function
  const cudaError_t ea = once_per_device(attr_done, [] {
    return cudaFuncSetAttribute(gemm_bf16_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                C::SMEM_BYTES);
  });
  if (ea != cudaSuccess) return ea;
  const int grid = P.total_tiles < num_sms ? P.total_tiles : num_sms;
  count_launch();
  launch_kernel(gemm_bf16_tc_kernel<BN>, grid, 192, C::SMEM_BYTES, stream, P);
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
  if (bn != 128) return cudaErrorInvalidValue;      // 256-wide tiles run on the CTA-pair kernel
  return launch_bn<128>(P, num_sms, stream);
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
