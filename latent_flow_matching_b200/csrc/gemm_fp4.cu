// Persistent NVFP4 GEMM on CTA pairs: C = A W^T (+ fused epilogue) with A and W as e2m1 codes,
// e4m3 block scales (one per 16 elements along K) and fp32 row scales; 256 x 256 tiles.
//
// Same structure as the bf16 / e4m3 pair kernel (gemm_tc2.cu): CTA r of the pair stages rows
// [m0 + 128r, +128) of A and [n0 + 128r, +128) of W, one elected lane of the leader issues
// tcgen05.mma.cta_group::2 with M = N = 256, and eight epilogue warps per CTA drain the
// accumulator with the fused epilogues (the row scales of A and W applied per element) and write
// through shared memory with TMA stores (epilogue_tma.cuh).
// What the 4-bit path adds:
//   * kind::mxf4nvf4 MMAs with K = 64 (32 bytes of packed codes per row, so the 128-byte swizzle
//     row of a stage holds 256 elements and a stage is four MMAs, as for the 8-bit path);
//   * block scales: per stage each CTA loads the A scales of its 128 rows (2 KB) and the W scales
//     of all 256 tile columns (4 KB, the MMA of each CTA multiplies by every column's scales);
//     before every MMA the issuing lane copies that MMA's scales from shared to tensor memory
//     (tcgen05.cp 32x128b.warpx4: 32 rows of 16 bytes broadcast to the four lane quarters, one
//     copy per 128 rows), into one of two 12-column slots used in turn.  A stage's four MMAs and
//     twelve copies go out from one elected lane in a single block (one election, descriptor
//     offsets added in place): the issuing thread takes about 100 cycles per MMA with its copies
//     against the MMA's 128 tensor cycles, so its issue rate bounds how far it runs ahead;
//   * tensor memory holds two 256-column accumulators and the scale slots in 512 columns only
//     if the accumulators overlap: buffer 0 is columns [0, 256), buffer 1 [224, 480), the scale
//     slots [480, 512).  The epilogue part that owns the 32 shared columns drains them first and
//     arrives on `ovl`; a tile's first MMA waits for that arrival from the previous tile (and, as
//     before, for its own buffer to be fully drained two tiles earlier).
// Barrier protocol (as gemm_tc2.cu, plus):
//   ovl  leader only: 8 arrivals (the four owning epilogue warps of each CTA) per tile
#include "common.cuh"
#include "fluxdit_internal.h"
#include "epilogue_tma.cuh"
#include "pair.cuh"

namespace fdit {

__device__ int g_gemm4_error;

namespace {

constexpr int BM = 256;
constexpr int BN = 256;
constexpr int BKE = 256;                       // K elements per stage (128 bytes of codes per row)
constexpr int STAGES = 5;
constexpr int A_BYTES = 128 * 128;             // 16 KB of codes
constexpr int B_BYTES = 128 * 128;
constexpr int SFA_BYTES = 128 * BKE / 16;      // 2 KB: 128 rows x 16 scales
constexpr int SFB_BYTES = 256 * BKE / 16;      // 4 KB: 256 columns x 16 scales
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
constexpr int TMEM_COLS = 512;
constexpr uint32_t kAcc1Col = 224;             // buffer 1 shares columns [224, 256) with buffer 0
constexpr uint32_t kSfCol = 480;               // two scale slots of 16 columns: SFA 4 | SFB 8
constexpr int kEpiWarps = 8;
constexpr int kThreads4 = 32 * (2 + kEpiWarps);
constexpr int EPI_BYTES = 4096;                // per epilogue warp: two staged 32-row x 64-byte boxes
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + kEpiWarps * EPI_BYTES + 1024 + 512;
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory per CTA");

static_assert(BN - kAcc1Col == 32 && kAcc1Col + BN <= kSfCol && kSfCol + 28 <= TMEM_COLS, "tensor memory plan");
static_assert(STAGE_BYTES % 1024 == 0, "the epilogue staging buffers need 1024-byte alignment");

__device__ __forceinline__ int find_problem(const GemmParams& P, int tile) {
  int p = 0;
#pragma unroll 1
  for (int i = 1; i < P.num_problems; ++i)
    if (tile >= P.prob[i].tile_begin) p = i;
  return p;
}

// Instruction descriptor, kind::mxf4nvf4 with block scales: e2m1 A and B (format 1), ue4m3
// scales (scale format 0), K = 64, both operands K-major, scale-factor ids 0.
__host__ __device__ constexpr uint32_t idesc_nvf4(int M, int N) {
  return (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// Shared-memory descriptor of a 32-row x 16-byte scale block: no swizzle, 8-row core matrices
// 128 bytes apart (K-major, one core matrix along K).
__device__ __forceinline__ uint64_t sf_desc(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(16 >> 4) << 16;        // leading byte offset (unused: one core matrix along K)
  d |= static_cast<uint64_t>(128 >> 4) << 32;       // stride byte offset
  d |= 1ull << 46;                                  // descriptor version for tcgen05
  return d;                                         // layout type 0: no swizzle
}

// One stage's four MMAs and their scale copies, issued by one elected lane in a single block:
// MMA k (K elements 64k..64k+63) takes its A/W descriptors advanced by 32k bytes and its scale
// blocks advanced by 512k bytes (W's second 128 columns 2048 bytes further), and uses scale slot
// k & 1 (sf0 / sf1: SFA at +0, the two SFB halves at +4 and +8 columns).  acc0 = 0 only for the
// first stage of a tile.
__device__ __forceinline__ void stage_issue_nvf4(uint32_t d_tmem, uint64_t ad, uint64_t bd, uint64_t sad, uint64_t sbd,
                                                 uint32_t idesc, uint32_t acc0, uint32_t sf0, uint32_t sf1) {
  asm volatile(
      "{\n\t.reg .pred p, t, e;\n\t"
      ".reg .b64 a, b, sa, sb, sc;\n\t"
      ".reg .b32 f0b, f0c, f1b, f1c;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "setp.eq.b32 t, %6, %6;\n\t"
      "add.u32 f0b, %7, 4;\n\tadd.u32 f0c, %7, 8;\n\tadd.u32 f1b, %8, 4;\n\tadd.u32 f1c, %8, 8;\n\t"
      "add.s64 sc, %4, 128;\n\t"
      "@e tcgen05.cp.cta_group::2.32x128b.warpx4 [%7], %3;\n\t"
      "@e tcgen05.cp.cta_group::2.32x128b.warpx4 [f0b], %4;\n\t"
      "@e tcgen05.cp.cta_group::2.32x128b.warpx4 [f0c], sc;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %5, [%7], [f0b], p;\n\t"
      "add.s64 a, %1, 2;\n\tadd.s64 b, %2, 2;\n\tadd.s64 sa, %3, 32;\n\tadd.s64 sb, %4, 32;\n\tadd.s64 sc, %4, 160;\n\t"
      "@e tcgen05.cp.cta_group::2.32x128b.warpx4 [%8], sa;\n\t"
      "@e tcgen05.cp.cta_group::2.32x128b.warpx4 [f1b], sb;\n\t"
      "@e tcgen05.cp.cta_group::2.32x128b.warpx4 [f1c], sc;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], a, b, %5, [%8], [f1b], t;\n\t"
      "add.s64 a, %1, 4;\n\tadd.s64 b, %2, 4;\n\tadd.s64 sa, %3, 64;\n\tadd.s64 sb, %4, 64;\n\tadd.s64 sc, %4, 192;\n\t"
      "@e tcgen05.cp.cta_group::2.32x128b.warpx4 [%7], sa;\n\t"
      "@e tcgen05.cp.cta_group::2.32x128b.warpx4 [f0b], sb;\n\t"
      "@e tcgen05.cp.cta_group::2.32x128b.warpx4 [f0c], sc;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], a, b, %5, [%7], [f0b], t;\n\t"
      "add.s64 a, %1, 6;\n\tadd.s64 b, %2, 6;\n\tadd.s64 sa, %3, 96;\n\tadd.s64 sb, %4, 96;\n\tadd.s64 sc, %4, 224;\n\t"
      "@e tcgen05.cp.cta_group::2.32x128b.warpx4 [%8], sa;\n\t"
      "@e tcgen05.cp.cta_group::2.32x128b.warpx4 [f1b], sb;\n\t"
      "@e tcgen05.cp.cta_group::2.32x128b.warpx4 [f1c], sc;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], a, b, %5, [%8], [f1b], t;\n\t}" ::"r"(d_tmem),
      "l"(ad), "l"(bd), "l"(sad), "l"(sbd), "r"(idesc), "r"(acc0), "r"(sf0), "r"(sf1)
      : "memory");
}

// The offsets written into stage_issue_nvf4 (in the descriptors' 16-byte units: 2 per MMA for A
// and W, 32 per MMA for a 512-byte scale block, 128 for W's second 128 columns of scales).
static_assert(BKE == 4 * 64 && SFA_BYTES == 4 * 512 && SFB_BYTES == 2 * 2048 && kSfCol % 16 == 0,
              "stage_issue_nvf4 assumes four K = 64 MMAs per stage and 512-byte scale blocks");

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads4, 1)
    gemm_fp4_tc2_kernel(const __grid_constant__ GemmParams4 P4) {
  const GemmParams& P = P4.g;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * A_BYTES;
  uint8_t* sSFA = sB + STAGES * B_BYTES;
  uint8_t* sSFB = sSFA + STAGES * SFA_BYTES;
  uint8_t* sEpi = smem + STAGES * STAGE_BYTES;      // 1024-byte aligned: STAGE_BYTES is a multiple of 1024
  uint64_t* full = reinterpret_cast<uint64_t*>(sEpi + kEpiWarps * EPI_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* ovl = acc_empty + 2;
  uint64_t* drain = ovl + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
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
    mbar_init(ovl, 2 * (kEpiWarps / 2));
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < P.num_problems; ++i) {
      tma_prefetch_map(&P.mapA[i]);
      tma_prefetch_map(&P.mapB[i]);
      tma_prefetch_map(&P4.mapSFA[i]);
      tma_prefetch_map(&P4.mapSFB[i]);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
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
        const int tm0 = (lt % pr.tiles_m) * BM, tn0 = (lt / pr.tiles_m) * BN;
        const int m0 = tm0 + 128 * static_cast<int>(rank);
        const int n0 = tn0 + 128 * static_cast<int>(rank);
        const int nk = pr.K / BKE;
        const int kblk = pr.K / 64;                  // 512-byte scale blocks per 128 rows
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t fb = map_to_rank(&full[stage], 0);
          mbar_arrive_expect_tx_cluster(fb, STAGE_BYTES);
          tma_load_2d_pair(sA + stage * A_BYTES, &P.mapA[p], fb, kb * (BKE / 2), m0);
          tma_load_2d_pair(sB + stage * B_BYTES, &P.mapB[p], fb, kb * (BKE / 2), n0);
          // scale rows of 256 bytes: 4 blocks of 512 bytes per 128 rows and stage
          tma_load_2d_pair(sSFA + stage * SFA_BYTES, &P4.mapSFA[p], fb, 0, ((m0 >> 7) * kblk + 4 * kb) * 2);
          tma_load_2d_pair(sSFB + stage * SFB_BYTES, &P4.mapSFB[p], fb, 0, ((tn0 >> 7) * kblk + 4 * kb) * 2);
          tma_load_2d_pair(sSFB + stage * SFB_BYTES + SFB_BYTES / 2, &P4.mapSFB[p], fb, 0,
                           (((tn0 >> 7) + 1) * kblk + 4 * kb) * 2);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        atomicExch(&g_gemm4_error, kErrTimeoutProducer);
        settle_inflight_copies();
      }
    }
  } else if (warp == 1) {
    if (rank == 0) {
      // ------------------------------------------------------------ MMA issuer (leader only)
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      uint32_t ovl_phase = 0;
      bool ok = true;
      bool first = true;
      const uint32_t idesc = idesc_nvf4(BM, BN);
      const uint64_t a_desc0 = sw128_desc(smem_u32(sA), 16, 1024);
      const uint64_t b_desc0 = sw128_desc(smem_u32(sB), 16, 1024);
      const uint64_t sfa_desc0 = sf_desc(smem_u32(sSFA));
      const uint64_t sfb_desc0 = sf_desc(smem_u32(sSFB));
      for (int tile = pair; ok && tile < P.total_tiles; tile += num_pairs) {
        const int p = find_problem(P, tile);
        const int nk = P.prob[p].K / BKE;
        if (!mbar_wait_warp(&acc_empty[acc], acc_phase ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        if (!first) {                                   // the previous tile's shared columns are drained
          if (!mbar_wait_warp(ovl, ovl_phase, abort_flag)) {
            ok = false;
            break;
          }
          ovl_phase ^= 1u;
        }
        first = false;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (acc ? kAcc1Col : 0u);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait_warp(&full[stage], phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = desc_advance(a_desc0, stage * A_BYTES);
          const uint64_t bd = desc_advance(b_desc0, stage * B_BYTES);
          const uint64_t sad = desc_advance(sfa_desc0, stage * SFA_BYTES);
          const uint64_t sbd = desc_advance(sfb_desc0, stage * SFB_BYTES);
          stage_issue_nvf4(d_tmem, ad, bd, sad, sbd, idesc, kb != 0 ? 1u : 0u, tmem_base + kSfCol,
                           tmem_base + kSfCol + 16);
          mma_commit_pair_warp(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit_pair_warp(&acc_full[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (!ok && lane == 0) atomicExch(&g_gemm4_error, kErrTimeoutMma);
      mma_commit_pair_local_warp(drain);
      mbar_drain(drain, 0);
    }
  } else {
    // -------------------------------------------------------------- epilogue warps 2..9 (both CTAs)
    const int quarter = warp & 3;
    const int part = (warp - 2) / 4;
    const int row = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t acc_empty_leader[2] = {map_to_rank(&acc_empty[0], 0), map_to_rank(&acc_empty[1], 0)};
    const uint32_t ovl_leader = map_to_rank(ovl, 0);
    const uint32_t epi_buf = smem_u32(sEpi + (warp - 2) * EPI_BYTES);
    uint32_t epi_which = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = pair; tile < P.total_tiles; tile += num_pairs) {
      const int p = find_problem(P, tile);
      const GemmProblem& pr = P.prob[p];
      const int lt = tile - pr.tile_begin;
      const int m = (lt % pr.tiles_m) * BM + 128 * static_cast<int>(rank) + row;
      const int n0 = (lt / pr.tiles_m) * BN;
      if (!mbar_wait(&acc_full[acc], acc_phase, abort_flag)) {
        atomicExch(&g_gemm4_error, kErrTimeoutEpilogue);
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem_base + lane_addr + (acc ? kAcc1Col : 0u);
      const EpiTma et{&P4.mapOut[p], epi_buf, m - lane, pr.M, &epi_which};
      gemm_epilogue_tile_tma<BN, true, 2, true>(pr, tbase, m, n0, part, acc, ovl_leader, et);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty_leader[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    epi_tma_drain();                                  // this warp's bulk stores are complete
  }

  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

}  // namespace

cudaError_t gemm_fp4_launch(GemmParams4& P4, int num_sms, cudaStream_t stream) {
  static std::atomic<unsigned long long> attr_done{0};
  const cudaError_t ea = once_per_device(attr_done, [] {
    return cudaFuncSetAttribute(gemm_fp4_tc2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  });
  if (ea != cudaSuccess) return ea;
  GemmParams& P = P4.g;
  for (int i = 0; i < P.num_problems; ++i) {        // K in whole stages, scales present
    const GemmProblem& pr = P.prob[i];
    if (pr.M > 0 && (pr.K % BKE != 0 || !pr.scale_a || !pr.scale_b)) return cudaErrorInvalidValue;
    if (pr.M > 0 && pr.N > 0 && !gemm_out_map(&P4.mapOut[i], pr)) return cudaErrorInvalidValue;
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
      P4.mapSFA[w] = P4.mapSFA[i];
      P4.mapSFB[w] = P4.mapSFB[i];
      P4.mapOut[w] = P4.mapOut[i];
    }
    P.prob[w++] = pr;
  }
  P.num_problems = w;
  P.total_tiles = total;
  if (total == 0) return cudaSuccess;
  int pairs = num_sms / 2;
  if (pairs > total) pairs = total;
  count_launch();
  launch_kernel(gemm_fp4_tc2_kernel, 2 * pairs, kThreads4, SMEM_BYTES, stream, P4);
  return cudaGetLastError();
}

int gemm_fp4_read_device_error(cudaStream_t stream) {
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbolAsync(&v, g_gemm4_error, sizeof(int), 0, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return -1;
  cudaMemcpyToSymbolAsync(g_gemm4_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, stream);
  cudaStreamSynchronize(stream);
  return v;
}

}  // namespace fdit
