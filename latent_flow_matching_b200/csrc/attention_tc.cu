// Flash-style joint attention on tcgen05: O = softmax(Q K^T / sqrt(d)) V per head,
// non-causal, no mask, over the whole joint sequence (text | image | reference),
// head_dim 128.  Joint attention and the attended padding follow the FLUX.3 Image
// Klein in Diffusers write-up, "Entkoppelte Vorverarbeitung und gemeinsame
// Attention-Blöcke" and "Verarbeitung einzelner Prompts und Batching-Architektur".
//
// A batch of sequences of equal length n sits row after row in q, k, v and out; grid.z picks
// the sequence and every row coordinate is offset by z * n.  Segments generalise this: segment
// z is rows [seg_row0[z], seg_row0[z] + seg_n[z]) and attends only to itself (the per-mode
// blocks of FLUX.3, where the text, image and reference streams each attend within
// themselves).  Key tiles that run past a sequence's end read the following rows (or the
// tensor map's zero fill) and are masked like the ragged tail; query tiles past a segment's
// end exit before they allocate anything.
//
// CTA = two 128-row query tiles (A, B) of one head that share every K/V tile and
// take turns on the tensor core, 12 warps in three warpgroups:
//   warps 0..3   softmax of tile A   (one thread per query row)
//   warps 4..7   softmax of tile B
//   warp 8       TMA: Q_A, Q_B once, then K_j / V_j into 2- and 3-deep rings
//   warp 9       issues tcgen05.mma (warp-convergent code, one elected lane) in the order
//                  S_A(0) S_B(0) | PV_A(0) S_A(1) PV_B(0) S_B(1) | PV_A(1) S_A(2) ...
//                so the tensor core works on one tile while the other tile's
//                softmax runs, and S_X(j) is issued after PV_X(j-1): when a
//                softmax warpgroup sees S_X(j), O_X already holds every earlier
//                P V and can be rescaled in place without another wait.
// Softmax: read S from TMEM, online softmax in the exp2 domain, rescale the O row
// only when the running max grows by more than 8 (log2 units; P stays below 2^8),
// write P as packed bf16 over the S columns (the PV MMA reads its A operand from
// TMEM), and at the end write O / l as bf16.  Packed f32x2 arithmetic and 3-input
// maxima halve the FMA/ADD/MAX issue slots, and one exponential pair in three is
// evaluated on the FMA pipe so the MUFU unit, which otherwise runs at the tensor
// core's pace, is off the critical path.  setmaxnreg moves registers from the
// control warpgroup to the two softmax warpgroups.
//
// TMEM columns: S_A [0,128), S_B [128,256), O_A [256,384), O_B [384,512).
#include "common.cuh"
#include "fluxdit_internal.h"

namespace fdit {

__device__ int g_attn_error;

namespace {

constexpr int kTile = 128;          // query rows and key rows per tile
constexpr int kHeadDim = 128;
constexpr int kQTiles = 2;          // query tiles per CTA
constexpr int kBox = 64;            // 64 bf16 = 128 bytes: one swizzle row
constexpr int kBoxBytes = kTile * kBox * 2;          // 16 KB
constexpr int kTileBytes = 2 * kBoxBytes;            // 32 KB: 128 rows x 128 dims
constexpr int kStagesK = 2;        // K is released right after its second QK^T, so 2 slots suffice
constexpr int kStagesV = 3;        // V is held until the second PV; a third slot hides the L2 round trip
constexpr int kThreads = 384;
constexpr int kSmemBytes = kTileBytes * (kQTiles + kStagesK + kStagesV) + 1024 + 256;   // 225 KB
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kOCol = 256;
constexpr float kRescaleThreshold = 8.0f;
// 384 threads x 168 registers at launch >= 256 x 200 (softmax) + 128 x 96 (control); the control
// warps (TMA producer, MMA issuer) need 96 to run without spilling
constexpr int kSoftmaxRegs = 200;
constexpr int kControlRegs = 96;

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x on the FMA pipe for two lanes at once (packed f32x2 arithmetic), to take part of the
// exponentials off the MUFU unit: split x = j + f with j the nearest integer (|f| <= 1/2) by
// the 1.5 * 2^23 rounding trick, evaluate 2^f with a cubic minimax polynomial (coefficients
// from a Remez exchange fit of 2^f on [-1/2, 1/2]; max relative error 7.5e-5, well below the
// 2^-9 of the bf16 P it feeds), and add j to the exponent field.  Inputs below -126 are
// clamped (their weight is < 2^-126).
__device__ __forceinline__ float2 ex2_poly2(float2 x) {
  x.x = fmaxf(x.x, -126.0f);
  x.y = fmaxf(x.y, -126.0f);
  const float2 magic = make_float2(12582912.0f, 12582912.0f);
  const float2 t = __fadd2_rn(x, magic);
  const float2 r = __fadd2_rn(t, make_float2(-12582912.0f, -12582912.0f));
  const float2 f = __ffma2_rn(r, make_float2(-1.0f, -1.0f), x);
  float2 p = __ffma2_rn(make_float2(0.0551716685f, 0.0551716685f), f, make_float2(0.2426111251f, 0.2426111251f));
  p = __ffma2_rn(p, f, make_float2(0.6932609677f, 0.6932609677f));
  p = __ffma2_rn(p, f, make_float2(0.9999280572f, 0.9999280572f));
  return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// one score pair in kPolyEvery goes through ex2_poly2, the rest through MUFU ex2
constexpr int kPolyEvery = 3;

// kSegs: grid.z indexes P's segments (lengths read once from the parameter arrays); otherwise
// grid.z is a batch index and the sequence length stays a constant-bank operand.
template <bool kSegs>
__global__ void __launch_bounds__(kThreads, 1) attention_tc_kernel(const __grid_constant__ AttnParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                                    // kQTiles tiles
  uint8_t* sK = sQ + kQTiles * kTileBytes;               // kStagesK tiles
  uint8_t* sV = sK + kStagesK * kTileBytes;              // kStagesV tiles
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + kStagesV * kTileBytes);
  uint64_t* q_full = bars;
  uint64_t* k_full = q_full + 1;                         // [kStagesK]
  uint64_t* k_empty = k_full + kStagesK;                 // [kStagesK]
  uint64_t* v_full = k_empty + kStagesK;                 // [kStagesV]
  uint64_t* v_empty = v_full + kStagesV;                 // [kStagesV]
  uint64_t* s_full = v_empty + kStagesV;                 // [query tile]
  uint64_t* p_full = s_full + 2;                         // [query tile], 128 arrivals (every softmax thread)
  uint64_t* o_final = p_full + 2;                        // [query tile]
  uint64_t* drain = o_final + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int q0 = blockIdx.x * (kQTiles * kTile);      // first query row inside this sequence
  const int head = blockIdx.y;
  const int n = kSegs ? P.seg_n[blockIdx.z] : P.n;   // rows of this sequence
  const int row_base = kSegs ? P.seg_row0[blockIdx.z] : static_cast<int>(blockIdx.z) * P.n;
  if (kSegs && q0 >= n) return;                        // whole CTA: nothing initialised yet
  const int n_kv = (n + kTile - 1) / kTile;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < kStagesK; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < kStagesV; ++i) {
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 128);
      mbar_init(&o_final[i], 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_map(&P.mapQ);
    tma_prefetch_map(&P.mapK);
    tma_prefetch_map(&P.mapV);
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_trigger();                                    // after this CTA's tensor-memory allocation
  pdl_wait();                                       // the previous kernel's writes are visible

  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kControlRegs));
    if (warp == 8 && lane == 0) {
      // ------------------------------------------------------------ TMA producer
      const int qc = P.q_col0 + head * kHeadDim;
      const int kc = P.k_col0 + head * kHeadDim;
      const int vc = P.v_col0 + head * kHeadDim;
      mbar_arrive_expect_tx(q_full, kQTiles * kTileBytes);
      for (int t = 0; t < kQTiles; ++t) {
        tma_load_2d(sQ + t * kTileBytes, &P.mapQ, q_full, qc, row_base + q0 + t * kTile);
        tma_load_2d(sQ + t * kTileBytes + kBoxBytes, &P.mapQ, q_full, qc + kBox, row_base + q0 + t * kTile);
      }
      uint32_t armed_k = 0, armed_v = 0, par_k = 0, par_v = 0;   // per slot: armed once / parity of last arming
      bool ok = true;
      for (int j = 0; j < n_kv; ++j) {
        const int r0 = row_base + j * kTile;   // a tile past the sequence end reads masked rows
        const int sk = j % kStagesK, sv = j % kStagesV;
        const uint32_t pk = (j / kStagesK) & 1, pv = (j / kStagesV) & 1;
        if (!mbar_wait(&k_empty[sk], pk ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&k_full[sk], kTileBytes);
        tma_load_2d(sK + sk * kTileBytes, &P.mapK, &k_full[sk], kc, r0);
        tma_load_2d(sK + sk * kTileBytes + kBoxBytes, &P.mapK, &k_full[sk], kc + kBox, r0);
        armed_k |= 1u << sk;
        par_k = (par_k & ~(1u << sk)) | (pk << sk);
        if (!mbar_wait(&v_empty[sv], pv ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&v_full[sv], kTileBytes);
        tma_load_2d(sV + sv * kTileBytes, &P.mapV, &v_full[sv], vc, r0);
        tma_load_2d(sV + sv * kTileBytes + kBoxBytes, &P.mapV, &v_full[sv], vc + kBox, r0);
        armed_v |= 1u << sv;
        par_v = (par_v & ~(1u << sv)) | (pv << sv);
      }
      mbar_drain(q_full, 0);
      if (!ok) {
        atomicExch(&g_attn_error, kErrTimeoutProducer);
        for (int i = 0; i < kStagesK; ++i)
          if (armed_k & (1u << i)) mbar_drain(&k_full[i], (par_k >> i) & 1u);
        for (int i = 0; i < kStagesV; ++i)
          if (armed_v & (1u << i)) mbar_drain(&v_full[i], (par_v >> i) & 1u);
      }
    } else if (warp == 9) {
      // ------------------------------------------------------------ MMA issuer
      const uint32_t idesc_s = idesc_bf16_f32(kTile, kTile, 0, 0);      // Q, K both K-major
      const uint32_t idesc_o = idesc_bf16_f32(kTile, kHeadDim, 0, 1);   // P K-major (TMEM), V MN-major
      // Base descriptors are built once; each MMA adds a compile-time offset (one 64-bit add),
      // which keeps this single issuing thread ahead of the tensor core.
      const uint64_t q_desc0 = sw128_desc(smem_u32(sQ), 16, 1024);
      const uint64_t k_desc0 = sw128_desc(smem_u32(sK), 16, 1024);
      const uint64_t v_desc0 = sw128_desc(smem_u32(sV), kBoxBytes, 1024);
      auto issue_s = [&](int t, int j) {        // S_t(j) = Q_t K_j^T
        const uint64_t qd = desc_advance(q_desc0, t * kTileBytes);
        const uint64_t kd = desc_advance(k_desc0, (j % kStagesK) * kTileBytes);
        const uint32_t s_tmem = tmem_base + static_cast<uint32_t>(t * kTile);
#pragma unroll
        for (int kk = 0; kk < kHeadDim / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kBoxBytes + (kk & 3) * 32;
          mma_ss_warp(s_tmem, desc_advance(qd, off), desc_advance(kd, off), idesc_s, kk != 0 ? 1u : 0u);
        }
        mma_commit_warp(&s_full[t]);
      };
      auto issue_pv = [&](int t, int j) {       // O_t += P_t(j) V_j, P from TMEM
        const uint64_t vd = desc_advance(v_desc0, (j % kStagesV) * kTileBytes);
        const uint32_t p_tmem = tmem_base + static_cast<uint32_t>(t * kTile);
        const uint32_t o_tmem = tmem_base + kOCol + static_cast<uint32_t>(t * kTile);
        const uint32_t acc0 = j > 0 ? 1u : 0u;
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          mma_ts_warp(o_tmem, p_tmem + kk * 8, desc_advance(vd, kk * 2048), idesc_o, kk > 0 ? 1u : acc0);
      };
      auto wait_issue_pv = [&](int t, int j) -> bool {
        if (!mbar_wait_warp(&p_full[t], j & 1, abort_flag)) return false;
        tc_fence_after();
        issue_pv(t, j);
        return true;
      };
      bool ok = mbar_wait_warp(q_full, 0, abort_flag) && mbar_wait_warp(&k_full[0], 0, abort_flag);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        issue_s(1, 0);
        mma_commit_warp(&k_empty[0]);                 // K_0 is no longer read
      }
      for (int j = 0; ok && j < n_kv; ++j) {
        if (!mbar_wait_warp(&v_full[j % kStagesV], (j / kStagesV) & 1, abort_flag) || !wait_issue_pv(0, j)) {
          ok = false;
          break;
        }
        if (j + 1 < n_kv) {
          if (!mbar_wait_warp(&k_full[(j + 1) % kStagesK], ((j + 1) / kStagesK) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_s(0, j + 1);
        } else {
          mma_commit_warp(&o_final[0]);
        }
        if (!wait_issue_pv(1, j)) {
          ok = false;
          break;
        }
        mma_commit_warp(&v_empty[j % kStagesV]);      // V_j is no longer read
        if (j + 1 < n_kv) {
          issue_s(1, j + 1);
          mma_commit_warp(&k_empty[(j + 1) % kStagesK]);   // K_{j+1} is no longer read
        } else {
          mma_commit_warp(&o_final[1]);
        }
      }
      if (!ok && lane == 0) atomicExch(&g_attn_error, kErrTimeoutMma);
      mma_commit_warp(drain);
      mbar_drain(drain, 0);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
    // -------------------------------------------------------------- softmax, warpgroup t = query tile t
    const int t = warp >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t s_addr = tmem_base + lane_addr + static_cast<uint32_t>(t * kTile);
    const uint32_t o_addr = tmem_base + lane_addr + kOCol + static_cast<uint32_t>(t * kTile);
    const float sl2 = P.scale_log2;
    float m_run = -INFINITY;      // running max of the scaled scores, log2 domain
    float l_run = 0.0f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      if (!mbar_wait(&s_full[t], j & 1, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t s[kTile];
      tmem_ld32(s_addr + 0, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
      tmem_ld32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
      tmem_ld32(s_addr + 64, *reinterpret_cast<uint32_t(*)[32]>(&s[64]));
      tmem_ld32(s_addr + 96, *reinterpret_cast<uint32_t(*)[32]>(&s[96]));
      tmem_ld_wait();
      const int valid = n - j * kTile;            // keys of this tile inside the sequence
      if (valid < kTile) {
#pragma unroll
        for (int c = 0; c < kTile; ++c)
          if (c >= valid) s[c] = __float_as_uint(-INFINITY);
      }
      // row max: 4 independent chains of 3-input maxima (one chain would serialise 64 dependent ops)
      float mp[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) mp[i] = fmaxf(__uint_as_float(s[2 * i]), __uint_as_float(s[2 * i + 1]));
#pragma unroll
      for (int c = 8; c < kTile; c += 2)
        mp[(c >> 1) & 3] = max3f(mp[(c >> 1) & 3], __uint_as_float(s[c]), __uint_as_float(s[c + 1]));
      const float mx = fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3]));
      const float mxs = mx * sl2;
      const bool warp_grow = __any_sync(0xffffffffu, mxs > m_run + kRescaleThreshold);
      const float m_use = warp_grow ? fmaxf(m_run, mxs) : m_run;
      const float alpha = ex2(m_run - m_use);     // 0 on the first tile, 1 when not moved
      if (warp_grow && j > 0) {
        // S_t(j) was issued after PV_t(j-1), so O_t is complete up to tile j-1 here and is
        // rescaled before P_t(j) lets PV_t(j) start
#pragma unroll 1
        for (int c = 0; c < kHeadDim; c += 32) {
          uint32_t o[32];
          tmem_ld32(o_addr + c, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const float2 v = __fmul2_rn(make_float2(__uint_as_float(o[e]), __uint_as_float(o[e + 1])),
                                        make_float2(alpha, alpha));
            o[e] = __float_as_uint(v.x);
            o[e + 1] = __float_as_uint(v.y);
          }
          tmem_st32(o_addr + c, o);
        }
      }
      const float2 sl2_2 = make_float2(sl2, sl2);
      const float2 neg_m2 = make_float2(-m_use, -m_use);
      float2 sp[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int c = 0; c < kTile; c += 2) {        // P packed in place over the first half of s
        const float2 x = __ffma2_rn(make_float2(__uint_as_float(s[c]), __uint_as_float(s[c + 1])), sl2_2, neg_m2);
        float2 p;
        if ((c / 2) % kPolyEvery == kPolyEvery - 1) {
          p = ex2_poly2(x);
        } else {
          p = make_float2(ex2(x.x), ex2(x.y));
        }
        sp[(c >> 1) & 3] = __fadd2_rn(sp[(c >> 1) & 3], p);
        s[c / 2] = pack_bf16x2(p.x, p.y);
      }
      tmem_st32(s_addr + 0, *reinterpret_cast<const uint32_t(*)[32]>(&s[0]));
      tmem_st32(s_addr + 32, *reinterpret_cast<const uint32_t(*)[32]>(&s[32]));
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[t]);
      const float2 s01 = __fadd2_rn(__fadd2_rn(sp[0], sp[1]), __fadd2_rn(sp[2], sp[3]));
      l_run = l_run * alpha + (s01.x + s01.y);
      m_run = m_use;
    }
    if (ok && mbar_wait(&o_final[t], 0, abort_flag)) {
      tc_fence_after();
      const float inv_l = 1.0f / l_run;
      const int qrow = q0 + t * kTile + row;
#pragma unroll 1
      for (int c = 0; c < kHeadDim; c += 32) {
        uint32_t o[32];
        tmem_ld32(o_addr + c, o);
        tmem_ld_wait();
        if (qrow < n) {
          uint4* dst = reinterpret_cast<uint4*>(P.out + static_cast<size_t>(row_base + qrow) * P.ldo +
                                                head * kHeadDim + c);
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
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace

cudaError_t attention_launch(const AttnParams& P, cudaStream_t stream) {
  static std::atomic<unsigned long long> attr_done{0};
  const cudaError_t ea = once_per_device(attr_done, [] {
    cudaError_t e =
        cudaFuncSetAttribute(attention_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(attention_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    return e;
  });
  if (ea != cudaSuccess) return ea;
  int n_max = P.n, nz = P.batch;
  if (P.nseg) {
    if (P.nseg < 0 || P.nseg > kMaxSegs) return cudaErrorInvalidValue;
    n_max = 0;
    nz = P.nseg;
    for (int z = 0; z < P.nseg; ++z) {
      if (P.seg_n[z] < 0 || P.seg_row0[z] < 0) return cudaErrorInvalidValue;
      n_max = P.seg_n[z] > n_max ? P.seg_n[z] : n_max;
    }
  }
  if (n_max <= 0 || P.heads <= 0 || nz <= 0) return cudaSuccess;
  dim3 grid((n_max + kQTiles * kTile - 1) / (kQTiles * kTile), P.heads, nz);
  count_launch();
  if (P.nseg)
    launch_kernel(attention_tc_kernel<true>, grid, kThreads, kSmemBytes, stream, P);
  else
    launch_kernel(attention_tc_kernel<false>, grid, kThreads, kSmemBytes, stream, P);
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
