// Flash-style joint attention on tcgen05: O = softmax(Q K^T / sqrt(d)) V per head,
// non-causal, no mask, over the whole joint sequence (text | image | reference),
// head_dim 128.  Joint attention and the attended padding follow the FLUX.3 Image
// Klein in Diffusers write-up, "Entkoppelte Vorverarbeitung und gemeinsame
// Attention-Blöcke" and "Verarbeitung einzelner Prompts und Batching-Architektur".
//
// CTA = one 128-row query tile of one head, 6 warps:
//   warp 0      TMA: Q once, then K_j / V_j tiles into a 2-deep ring
//   warp 1      one thread issues tcgen05.mma: S_j = Q K_j^T into TMEM buffer j&1,
//               then O += P_{j-1} V_{j-1} with P read from TMEM (A operand in TMEM)
//   warps 2..5  one thread per query row: read S_j from TMEM, online softmax in
//               the exp2 domain, write P_j as packed bf16 over the S_j columns,
//               rescale the O row in TMEM when the running max moved, and at
//               the end write O / l as bf16.
// The running max is only moved when it grows by more than 8 (log2 units), so
// most iterations skip the O rescale; P stays below 2^8, safe in bf16/fp32.
//
// TMEM columns: S0 [0,128), S1 [128,256), O [256,384) of a 512-column allocation.
#include "common.cuh"
#include "fluxdit_internal.h"

namespace fdit {

__device__ int g_attn_error;

namespace {

constexpr int kTile = 128;          // query rows and key rows per tile
constexpr int kHeadDim = 128;
constexpr int kBox = 64;            // 64 bf16 = 128 bytes: one swizzle row
constexpr int kBoxBytes = kTile * kBox * 2;          // 16 KB
constexpr int kTileBytes = 2 * kBoxBytes;            // 32 KB: 128 rows x 128 dims
constexpr int kStages = 2;
constexpr int kSmemBytes = kTileBytes * (1 + 2 * kStages) + 1024 + 256;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kOCol = 256;
constexpr float kRescaleThreshold = 8.0f;

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__global__ void __launch_bounds__(192, 1) attention_tc_kernel(const __grid_constant__ AttnParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = smem + kTileBytes;                       // kStages tiles
  uint8_t* sV = sK + kStages * kTileBytes;               // kStages tiles
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + kStages * kTileBytes);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;                           // [2]
  uint64_t* v_full = bars + 3;                           // [2]
  uint64_t* kv_empty = bars + 5;                         // [2]
  uint64_t* s_full = bars + 7;                           // [2]
  uint64_t* p_full = bars + 9;                           // [2]
  uint64_t* o_done = bars + 11;                          // [2]: PV_i completes o_done[i & 1]
  uint64_t* drain = bars + 13;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 14);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int q0 = blockIdx.x * kTile;
  const int head = blockIdx.y;
  const int n_kv = (P.n + kTile - 1) / kTile;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&kv_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 4);
      mbar_init(&o_done[i], 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&P.mapQ);
    tma_prefetch_map(&P.mapK);
    tma_prefetch_map(&P.mapV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      const int qc = P.q_col0 + head * kHeadDim;
      const int kc = P.k_col0 + head * kHeadDim;
      const int vc = P.v_col0 + head * kHeadDim;
      mbar_arrive_expect_tx(q_full, kTileBytes);
      tma_load_2d(sQ, &P.mapQ, q_full, qc, q0);
      tma_load_2d(sQ + kBoxBytes, &P.mapQ, q_full, qc + kBox, q0);
      uint32_t armed_k = 0, armed_v = 0, parity = 0;
      bool ok = true;
      for (int j = 0; j < n_kv; ++j) {
        const int st = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (!mbar_wait(&kv_empty[st], ph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        const int r0 = j * kTile;
        mbar_arrive_expect_tx(&k_full[st], kTileBytes);
        tma_load_2d(sK + st * kTileBytes, &P.mapK, &k_full[st], kc, r0);
        tma_load_2d(sK + st * kTileBytes + kBoxBytes, &P.mapK, &k_full[st], kc + kBox, r0);
        mbar_arrive_expect_tx(&v_full[st], kTileBytes);
        tma_load_2d(sV + st * kTileBytes, &P.mapV, &v_full[st], vc, r0);
        tma_load_2d(sV + st * kTileBytes + kBoxBytes, &P.mapV, &v_full[st], vc + kBox, r0);
        armed_k |= 1u << st;
        armed_v |= 1u << st;
        parity = (parity & ~(1u << st)) | (ph << st);
      }
      mbar_drain(q_full, 0);
      if (!ok) {
        atomicExch(&g_attn_error, kErrTimeoutProducer);
        for (int s = 0; s < 2; ++s) {
          if (armed_k & (1u << s)) mbar_drain(&k_full[s], (parity >> s) & 1u);
          if (armed_v & (1u << s)) mbar_drain(&v_full[s], (parity >> s) & 1u);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      const uint32_t idesc_s = idesc_bf16_f32(kTile, kTile, 0, 0);      // Q, K both K-major
      const uint32_t idesc_o = idesc_bf16_f32(kTile, kHeadDim, 0, 1);   // P K-major (TMEM), V MN-major
      bool ok = mbar_wait(q_full, 0, abort_flag);
      const uint32_t q_addr = smem_u32(sQ);
      for (int j = 0; ok && j <= n_kv; ++j) {
        if (j < n_kv) {
          const int st = j & 1;
          if (!mbar_wait(&k_full[st], (j >> 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t k_addr = smem_u32(sK + st * kTileBytes);
          const uint32_t s_tmem = tmem_base + static_cast<uint32_t>(st * kTile);
#pragma unroll
          for (int kk = 0; kk < kHeadDim / 16; ++kk) {
            const uint32_t off = (kk >> 2) * kBoxBytes + (kk & 3) * 32;
            mma_ss(s_tmem, sw128_desc(q_addr + off, 16, 1024), sw128_desc(k_addr + off, 16, 1024), idesc_s,
                   kk != 0 ? 1u : 0u);
          }
          mma_commit(&s_full[st]);
        }
        if (j >= 1) {
          const int jp = j - 1;
          const int st = jp & 1;
          if (!mbar_wait(&p_full[st], (jp >> 1) & 1, abort_flag) ||
              !mbar_wait(&v_full[st], (jp >> 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t v_addr = smem_u32(sV + st * kTileBytes);
          const uint32_t p_tmem = tmem_base + static_cast<uint32_t>(st * kTile);
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk) {
            // A: 16 keys of P = 8 packed columns; B: 16 rows of V (2 x 8-row groups) per step
            mma_ts(tmem_base + kOCol, p_tmem + kk * 8, sw128_desc(v_addr + kk * 2048, kBoxBytes, 1024),
                   idesc_o, (jp > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&o_done[jp & 1]);
          mma_commit(&kv_empty[st]);
        }
      }
      if (!ok) atomicExch(&g_attn_error, kErrTimeoutMma);
      mma_commit(drain);
      mbar_drain(drain, 0);
    }
  } else {
    // -------------------------------------------------------------- softmax warps 2..5
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const float sl2 = P.scale_log2;
    float m_run = -INFINITY;      // running max, log2 domain (scaled)
    float l_run = 0.0f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const int st = j & 1;
      if (!mbar_wait(&s_full[st], (j >> 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t s_addr = tmem_base + lane_addr + static_cast<uint32_t>(st * kTile);
      uint32_t s[kTile];
      tmem_ld32(s_addr + 0, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
      tmem_ld32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
      tmem_ld32(s_addr + 64, *reinterpret_cast<uint32_t(*)[32]>(&s[64]));
      tmem_ld32(s_addr + 96, *reinterpret_cast<uint32_t(*)[32]>(&s[96]));
      tmem_ld_wait();
      const int valid = P.n - j * kTile;          // keys of this tile inside the sequence
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < kTile; ++c) {
        float x = __uint_as_float(s[c]) * sl2;
        if (c >= valid) x = -INFINITY;
        s[c] = __float_as_uint(x);
        mx = fmaxf(mx, x);
      }
      const bool grow = mx > m_run + kRescaleThreshold;
      const bool warp_grow = __any_sync(0xffffffffu, grow);
      float m_use = m_run;
      if (warp_grow) m_use = fmaxf(m_run, mx);
      const float alpha = ex2(m_run - m_use);   // 0 on the first tile, 1 when not moved
      float sum = 0.0f;
      uint32_t pk[kTile / 2];
#pragma unroll
      for (int c = 0; c < kTile; c += 2) {
        const float p0 = ex2(__uint_as_float(s[c]) - m_use);
        const float p1 = ex2(__uint_as_float(s[c + 1]) - m_use);
        sum += p0 + p1;
        pk[c / 2] = pack_bf16x2(p0, p1);
      }
      tmem_st32(s_addr + 0, *reinterpret_cast<const uint32_t(*)[32]>(&pk[0]));
      tmem_st32(s_addr + 32, *reinterpret_cast<const uint32_t(*)[32]>(&pk[32]));
      l_run = l_run * alpha + sum;
      if (warp_grow && j > 0) {
        // O holds sum_{i<j} P_i V_i once PV_{j-1} retired; rescale it by alpha
        // Softmax warps may skip these waits, so PV completions are split over two
        // barriers by parity of the PV index: the wanted phase is then never more
        // than one phase behind the barrier, which a parity wait requires.
        if (!mbar_wait(&o_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t o_addr = tmem_base + lane_addr + kOCol;
#pragma unroll 1
        for (int c = 0; c < kHeadDim; c += 32) {
          uint32_t o[32];
          tmem_ld32(o_addr + c, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(o_addr + c, o);
        }
      }
      m_run = m_use;
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[st]);
    }
    if (ok && mbar_wait(&o_done[(n_kv - 1) & 1], ((n_kv - 1) >> 1) & 1, abort_flag)) {
      tc_fence_after();
      const float inv_l = 1.0f / l_run;
      const int qrow = q0 + row;
      const uint32_t o_addr = tmem_base + lane_addr + kOCol;
#pragma unroll 1
      for (int c = 0; c < kHeadDim; c += 32) {
        uint32_t o[32];
        tmem_ld32(o_addr + c, o);
        tmem_ld_wait();
        if (qrow < P.n) {
          uint4* dst = reinterpret_cast<uint4*>(P.out + static_cast<size_t>(qrow) * P.ldo + head * kHeadDim + c);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              w[e] = pack_bf16x2(__uint_as_float(o[v * 8 + 2 * e]) * inv_l,
                                 __uint_as_float(o[v * 8 + 2 * e + 1]) * inv_l);
            dst[v] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
    } else {
      atomicExch(&g_attn_error, kErrTimeoutSoftmax);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace

cudaError_t attention_launch(const AttnParams& P, cudaStream_t stream) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e =
        cudaFuncSetAttribute(attention_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  if (P.n <= 0 || P.heads <= 0) return cudaSuccess;
  dim3 grid((P.n + kTile - 1) / kTile, P.heads);
  count_launch();
  attention_tc_kernel<<<grid, 192, kSmemBytes, stream>>>(P);
  return cudaGetLastError();
}

int attention_read_device_error(cudaStream_t stream) {
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbolAsync(&v, g_attn_error, sizeof(int), 0, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return -1;
  cudaMemcpyToSymbolAsync(g_attn_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, stream);
  cudaStreamSynchronize(stream);
  return v;
}

}  // namespace fdit
