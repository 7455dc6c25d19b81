// Persistent tcgen05 GEMM on CTA pairs (cta_group::2): C = A W^T (+ fused epilogue), 256 x 256 tiles.
//
// A cluster of two CTAs on two SMs computes one 256 x 256 output tile per step.  CTA r loads
// rows [m0 + 128r, +128) of A and rows [n0 + 128r, +128) of W (its half of the N columns) with
// plain (non-multicast) TMA loads whose completion is counted on the leader CTA's barrier; one
// thread of the leader issues tcgen05.mma.cta_group::2 with M = 256, N = 256, which reads A
// from each CTA's own shared memory and the two W halves from both, and writes rows 128r.. of
// the accumulator into CTA r's tensor memory.  Compared with one CTA per 128 x 256 tile, every
// instruction does twice the work and each SM stages half as many W bytes per FLOP.
//
// Roles per CTA (10 warps): warp 0 TMA producer, warp 1 MMA issuer (leader CTA only, one elected
// lane of a convergent warp) and TMEM allocator, warps 2..9 epilogue of this CTA's 128 accumulator
// rows: two warps per TMEM lane quarter, each draining half of the tile's 256 columns (one 128-wide
// head for the fused QK-RMSNorm, half of the a/b pairs for SwiGLU).  With 8-bit operands a tile's
// MMAs take half as long, and four epilogue warps could not empty an accumulator before the other
// one was full.
// Barrier protocol:
//   full[s]      leader only: 2 arrivals (one expect_tx from each CTA's producer) + the bytes
//   empty[s]     both CTAs: the leader's MMA commit multicasts one arrival to each
//   acc_full[a]  both CTAs: multicast commit after a tile's last MMA
//   acc_empty[a] leader only: 16 arrivals (8 epilogue warps of each CTA)
// The epilogue modes are those of the one-CTA kernel (gemm_tc.cu).
#include "common.cuh"
#include "fluxdit_internal.h"
#include "gemm_epilogue.cuh"
#include "pair.cuh"

namespace fdit {

__device__ int g_gemm2_error;

namespace {

constexpr int BM = 256;          // rows per CTA pair (128 per CTA)
constexpr int BN = 256;          // output columns per tile (128 W rows staged per CTA)
constexpr int BK = 64;
constexpr int STAGES = 6;
constexpr int A_BYTES = 128 * BK * 2;          // 16 KB
constexpr int B_BYTES = 128 * BK * 2;          // 16 KB (this CTA's half of W)
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int TMEM_COLS = 2 * BN;              // double-buffered 128 x 256 fp32 accumulator per CTA
constexpr int kEpiWarps = 8;                   // two per TMEM lane quarter
constexpr int kThreads2 = 32 * (2 + kEpiWarps);
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 512;

__device__ __forceinline__ int find_problem(const GemmParams& P, int tile) {
  int p = 0;
#pragma unroll 1
  for (int i = 1; i < P.num_problems; ++i)
    if (tile >= P.prob[i].tile_begin) p = i;
  return p;
}

// kFp8: e4m3 operands, 128 per 128-byte swizzle row (BK = 128 elements per stage, the same bytes
// as 64 bf16), kind::f8f6f4 MMAs with K = 32, and the epilogue applies the row / column scales.
template <bool kFp8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads2, 1)
    gemm_bf16_tc2_kernel(const __grid_constant__ GemmParams P) {
  constexpr int BKE = kFp8 ? 2 * BK : BK;           // K elements per stage
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();          // 0: leader (issues the MMAs), 1: peer
  const int pair = blockIdx.x >> 1;
  const int num_pairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 2);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 2 * kEpiWarps);
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
    tmem_alloc_pair(tmem_slot, TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();                                   // both CTAs' barriers exist before any remote arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_trigger();                                    // after this CTA's tensor-memory allocation
  pdl_wait();                                       // the previous kernel's writes are visible

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer (both CTAs)
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < P.total_tiles; tile += num_pairs) {
        const int p = find_problem(P, tile);
        const GemmProblem& pr = P.prob[p];
        const int lt = tile - pr.tile_begin;
        const int m0 = (lt % pr.tiles_m) * BM + 128 * static_cast<int>(rank);
        const int n0 = (lt / pr.tiles_m) * BN + 128 * static_cast<int>(rank);
        const int nk = pr.K / BKE;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t fb = map_to_rank(&full[stage], 0);
          mbar_arrive_expect_tx_cluster(fb, STAGE_BYTES);
          tma_load_2d_pair(sA + stage * A_BYTES, &P.mapA[p], fb, kb * BKE, m0);
          tma_load_2d_pair(sB + stage * B_BYTES, &P.mapB[p], fb, kb * BKE, n0);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Without an abort every issued stage is consumed by the leader's MMAs before the final
      // cluster barrier.  After one, their completion is counted on the leader's barrier, so
      // wait a bounded time for them instead.
      if (!ok) {
        atomicExch(&g_gemm2_error, kErrTimeoutProducer);
        settle_inflight_copies();
      }
    }
  } else if (warp == 1) {
    if (rank == 0) {
      // ------------------------------------------------------------ MMA issuer (leader only; whole warp, one elected lane issues)
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      const uint32_t idesc = kFp8 ? idesc_e4m3_f32(BM, BN) : idesc_bf16_f32(BM, BN, 0, 0);
      const uint64_t a_desc0 = sw128_desc(smem_u32(sA), 16, 1024);
      const uint64_t b_desc0 = sw128_desc(smem_u32(sB), 16, 1024);
      for (int tile = pair; ok && tile < P.total_tiles; tile += num_pairs) {
        const int p = find_problem(P, tile);
        const int nk = P.prob[p].K / BKE;
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
          const uint64_t ad = desc_advance(a_desc0, stage * A_BYTES);
          const uint64_t bd = desc_advance(b_desc0, stage * B_BYTES);
#pragma unroll
          for (int k = 0; k < 4; ++k) {                  // 32 bytes of K per MMA: 16 bf16 or 32 e4m3
            if constexpr (kFp8)
              mma_pair_f8_warp(d_tmem, desc_advance(ad, k * 32), desc_advance(bd, k * 32), idesc,
                               (kb | k) != 0 ? 1u : 0u);
            else
              mma_pair_warp(d_tmem, desc_advance(ad, k * 32), desc_advance(bd, k * 32), idesc,
                            (kb | k) != 0 ? 1u : 0u);
          }
          mma_commit_pair_warp(&empty[stage]);            // frees this stage in both CTAs
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit_pair_warp(&acc_full[acc]);             // accumulator halves ready in both CTAs
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (!ok && lane == 0) atomicExch(&g_gemm2_error, kErrTimeoutMma);
      mma_commit_pair_local_warp(drain);
      mbar_drain(drain, 0);
    }
  } else {
    // -------------------------------------------------------------- epilogue warps 2..9 (both CTAs)
    const int quarter = warp & 3;                   // the TMEM lane quarter this warp may read
    const int part = (warp - 2) / 4;                // which half of the tile's columns
    const int row = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t acc_empty_leader[2] = {map_to_rank(&acc_empty[0], 0), map_to_rank(&acc_empty[1], 0)};
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = pair; tile < P.total_tiles; tile += num_pairs) {
      const int p = find_problem(P, tile);
      const GemmProblem& pr = P.prob[p];
      const int lt = tile - pr.tile_begin;
      const int m = (lt % pr.tiles_m) * BM + 128 * static_cast<int>(rank) + row;
      const int n0 = (lt / pr.tiles_m) * BN;
      if (!mbar_wait(&acc_full[acc], acc_phase, abort_flag)) {
        atomicExch(&g_gemm2_error, kErrTimeoutEpilogue);
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem_base + lane_addr + static_cast<uint32_t>(acc * BN);
      gemm_epilogue_tile<BN, kFp8, 2>(pr, tbase, m, n0, part);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty_leader[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  tc_fence_before();
  cluster_sync();                                   // the leader no longer reads the peer's smem or TMEM
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

}  // namespace

cudaError_t gemm2_launch(GemmParams& P, int num_sms, cudaStream_t stream, bool fp8) {
  static std::atomic<unsigned long long> attr_done{0};
  const cudaError_t ea = once_per_device(attr_done, [] {
    cudaError_t e =
        cudaFuncSetAttribute(gemm_bf16_tc2_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gemm_bf16_tc2_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    return e;
  });
  if (ea != cudaSuccess) return ea;
  for (int i = 0; i < P.num_problems; ++i) {        // 8-bit problems: K in whole stages, scales present
    const GemmProblem& pr = P.prob[i];
    if (pr.M > 0 && (pr.K % (fp8 ? 2 * BK : BK) != 0 || (fp8 && (!pr.scale_a || !pr.scale_b))))
      return cudaErrorInvalidValue;
  }
  int w = 0, total = 0;
  for (int i = 0; i < P.num_problems; ++i) {
    GemmProblem pr = P.prob[i];
    if (pr.M <= 0 || pr.N <= 0) continue;
    pr.tiles_m = (pr.M + BM - 1) / BM;
    pr.tiles_n = (pr.N + BN - 1) / BN;
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
  int pairs = num_sms / 2;
  if (pairs > total) pairs = total;
  count_launch();
  if (fp8)
    launch_kernel(gemm_bf16_tc2_kernel<true>, 2 * pairs, kThreads2, SMEM_BYTES, stream, P);
  else
    launch_kernel(gemm_bf16_tc2_kernel<false>, 2 * pairs, kThreads2, SMEM_BYTES, stream, P);
  return cudaGetLastError();
}

int gemm2_read_device_error(cudaStream_t stream) {
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbolAsync(&v, g_gemm2_error, sizeof(int), 0, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return -1;
  cudaMemcpyToSymbolAsync(g_gemm2_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, stream);
  cudaStreamSynchronize(stream);
  return v;
}

}  // namespace fdit
