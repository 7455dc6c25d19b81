// Host-side pieces shared by the model runners (fluxdit.cu: FLUX.2-klein, fluxdit3.cu: FLUX.3
// Image Klein): error recording, the per-launch profiler, the launch macro and grouped-GEMM
// problem set-up.  Internal; not exported.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <nvtx3/nvToolsExt.h>

#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "../../include/fluxdit.h"
#include "fluxdit_internal.h"

namespace fdit {

using bf16 = __nv_bfloat16;

// A named NVTX range over one scope of host code (the launches of one transformer block, the
// modulation, the input or output layers), so a profiler's timeline groups the kernels by block.
// Without a profiler attached a push / pop is a check of one function pointer.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  NvtxRange(const char* fmt, int i) {
    char buf[48];
    snprintf(buf, sizeof(buf), fmt, i);
    nvtxRangePushA(buf);
  }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// printf-style flux_get_error() message for the calling thread; returns `code`.
int fail(int code, const char* fmt, ...);
const char* last_error();
int last_error_code();

#define FD_CUDA(expr)                                                                          \
  do {                                                                                         \
    cudaError_t e_ = (expr);                                                                   \
    if (e_ != cudaSuccess) return fail(FLUX_EIO, "%s: %s", #expr, cudaGetErrorString(e_));     \
  } while (0)

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// ------------------------------------------------------------------ per-kernel profiling
// When enabled, every launch of a forward is bracketed by two CUDA events on its
// stream; settle() (after a device synchronisation) accumulates the elapsed time
// per kernel kind together with the launch's algorithmic FLOPs and HBM bytes.
enum ProfKind { kProfGemm = 0, kProfAttention, kProfLnMod, kProfQkNormRope, kProfGemv, kProfOther, kProfKinds };
struct ProfRec {
  int kind;
  cudaEvent_t a, b;
  double flops, bytes;
};
struct Profiler {
  bool on = false;
  std::vector<cudaEvent_t> pool;
  std::vector<ProfRec> pending;
  double ms[kProfKinds] = {}, flops[kProfKinds] = {}, bytes[kProfKinds] = {};
  long long launches[kProfKinds] = {};
  cudaEvent_t get() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
  }
  void settle() {
    for (const ProfRec& r : pending) {
      float t = 0.f;
      if (cudaEventElapsedTime(&t, r.a, r.b) == cudaSuccess) {
        ms[r.kind] += t;
        flops[r.kind] += r.flops;
        bytes[r.kind] += r.bytes;
        launches[r.kind] += 1;
      }
      pool.push_back(r.a);
      pool.push_back(r.b);
    }
    pending.clear();
  }
  void reset() {
    settle();
    for (int k = 0; k < kProfKinds; ++k) ms[k] = flops[k] = bytes[k] = 0, launches[k] = 0;
  }
  ~Profiler() {
    settle();
    for (cudaEvent_t e : pool) cudaEventDestroy(e);
  }
};

inline double gemm_flops(const GemmParams& P) {
  double f = 0;
  for (int i = 0; i < P.num_problems; ++i)
    if (P.prob[i].M > 0) f += 2.0 * P.prob[i].M * static_cast<double>(P.prob[i].N) * P.prob[i].K;
  return f;
}
// Operand storage of a linear: bf16 (2 bytes per element), e4m3 codes (1 byte) or NVFP4 (half a
// byte of code plus one e4m3 block scale per 16 elements); the quantised formats also read one
// fp32 row scale per row of A and of W.
enum class OpFormat { kBf16, kE4M3, kNvfp4 };
// Algorithmic bytes of a launch: A and W read once, the output written once (bf16 for the bias and
// the fused QK-norm + RoPE modes; the SwiGLU writes half the columns in bf16; fp32; the gated
// residual reads and writes its fp32 rows).
inline double gemm_bytes(const GemmParams& P, OpFormat f = OpFormat::kBf16) {
  const double elt = f == OpFormat::kBf16 ? 2.0 : f == OpFormat::kE4M3 ? 1.0 : 0.5 + 1.0 / 16.0;
  const double row = f == OpFormat::kBf16 ? 0.0 : 4.0;
  double b = 0;
  for (int i = 0; i < P.num_problems; ++i) {
    const GemmProblem& pr = P.prob[i];
    if (pr.M <= 0) continue;
    const double out_elt = pr.mode == kEpiBf16Bias || pr.mode == kEpiQKNormRope ? 2
                           : pr.mode == kEpiSwiGLU                             ? 1
                           : pr.mode == kEpiF32Bias                            ? 4
                                                                               : 8;   // gated residual
    b += elt * (static_cast<double>(pr.M) * pr.K + static_cast<double>(pr.N) * pr.K) + row * (pr.M + pr.N) +
         out_elt * pr.M * static_cast<double>(pr.N);
  }
  return b;
}

// Enqueue `expr` (a launch returning cudaError_t) on stream `s`; bracket it with profiling events
// when (m)->prof is enabled.
#define FD_LAUNCH(m, kind, fl, by, expr)                                                   \
  do {                                                                                     \
    cudaEvent_t ea_ = nullptr, eb_ = nullptr;                                              \
    if ((m)->prof.on) {                                                                    \
      ea_ = (m)->prof.get();                                                               \
      eb_ = (m)->prof.get();                                                               \
      cudaEventRecord(ea_, s);                                                             \
    }                                                                                      \
    FD_CUDA(expr);                                                                         \
    if ((m)->prof.on) {                                                                    \
      cudaEventRecord(eb_, s);                                                             \
      (m)->prof.pending.push_back({(kind), ea_, eb_, (fl), (by)});                         \
    }                                                                                      \
  } while (0)

inline void problem(GemmParams& P, int i, const CUtensorMap& a, const CUtensorMap& b, int M, int N, int K, int mode,
                    void* out, int ldo, const bf16* bias, const float* gate) {
  P.mapA[i] = a;
  P.mapB[i] = b;
  GemmProblem& pr = P.prob[i];
  pr = GemmProblem();
  pr.M = M; pr.N = N; pr.K = K; pr.mode = mode; pr.out = out; pr.ldo = ldo; pr.bias = bias; pr.gate = gate;
}

// Make problem i a fused qkv + QK-RMSNorm + RoPE projection (rows start at token rope_row0).
inline void qk_fuse(GemmParams& P, int i, const bf16* gq, const bf16* gk, const float2* rope, int rope_row0,
                    float eps) {
  GemmProblem& pr = P.prob[i];
  pr.mode = kEpiQKNormRope;
  pr.gain_q = gq;
  pr.gain_k = gk;
  pr.rope = rope;
  pr.rope_row0 = rope_row0;
  pr.eps = eps;
}

// Kernel choice for the linear layers of one grouped GEMM.  The CTA-pair kernel (256 x 256
// tiles) is the faster one per SM, but when its tiles would leave more than half of the 74 pairs
// idle (few token rows and N = hidden, e.g. linear2 and the projections at 256^2) the one-CTA
// kernel with 128 x 128 tiles (four times as many) fills the GPU.  SwiGLU problems and 8-bit
// operands stay on the pair kernel (a SwiGLU tile must hold 128 a-rows and their 128 b-rows).
// `nb`: sequences in the batch; the choice is made per sequence, so a batch and its sequences run
// alone take the same kernel (and produce the same bits).  True: the one-CTA kernel.
inline bool small_linear(const GemmParams& P, int num_sms, bool fp8, int nb) {
  if (fp8) return false;
  long pair_tiles = 0, small_tiles = 0;
  bool swiglu = false;
  for (int i = 0; i < P.num_problems; ++i) {
    const GemmProblem& pr = P.prob[i];
    if (pr.M <= 0 || pr.N <= 0) continue;
    pair_tiles += static_cast<long>((pr.M + 255) / 256) * ((pr.N + 255) / 256);
    small_tiles += static_cast<long>((pr.M + 127) / 128) * ((pr.N + 127) / 128);
    swiglu |= pr.mode == kEpiSwiGLU;
  }
  return !swiglu && pair_tiles > 0 && 4 * pair_tiles <= static_cast<long>(num_sms) * nb &&
         small_tiles <= static_cast<long>(num_sms) * nb;
}

// Launch with a kernel chosen by the caller (small_linear of the problems that fix the choice).
inline cudaError_t launch_linear_as(GemmParams& P, int num_sms, cudaStream_t s, bool fp8, bool small) {
  return small && !fp8 ? gemm_launch(P, 128, num_sms, s) : gemm2_launch(P, num_sms, s, fp8);
}

inline cudaError_t launch_linear(GemmParams& P, int num_sms, cudaStream_t s, bool fp8, int nb = 1) {
  return launch_linear_as(P, num_sms, s, fp8, small_linear(P, num_sms, fp8, nb));
}

// ------------------------------------------------------------------ NVFP4 operands
// One NVFP4 GEMM operand: rows [0, rows) of a codes buffer (row stride ldq bytes), its block scales
// starting at 128-row block blk0 of a scale buffer, and its fp32 row scales.
struct Fp4Op {
  CUtensorMap codes, sf;
  const float* scale = nullptr;
};

inline bool make_fp4_op(Fp4Op* op, const uint8_t* codes, size_t rows, size_t k, size_t ldq, const uint8_t* sf,
                        size_t blk0, const float* scale) {
  op->scale = scale;
  if (rows == 0) {
    memset(&op->codes, 0, sizeof(CUtensorMap));
    memset(&op->sf, 0, sizeof(CUtensorMap));
    return true;
  }
  return make_tmap_u8(&op->codes, codes, rows, k / 2, ldq, 128) &&
         make_tmap_sf(&op->sf, sf + blk0 * (k / 64) * 512, nvfp4_scale_bytes(rows, k));
}

// Problem i of an NVFP4 grouped GEMM takes activation operand a and weight operand w.
inline void fp4_operands(GemmParams4& P4, int i, const Fp4Op& a, const Fp4Op& w) {
  P4.g.mapA[i] = a.codes;
  P4.g.mapB[i] = w.codes;
  P4.mapSFA[i] = a.sf;
  P4.mapSFB[i] = w.sf;
  P4.g.prob[i].scale_a = a.scale;
  P4.g.prob[i].scale_b = w.scale;
}

// Quantise weight matrices (bf16 [rows, cols], row stride cols) to NVFP4 in one device allocation
// (*buf: codes and block scales, *scales: row scales).  Fills each matrix's codes / sf / scale.
struct Fp4Mat {
  const bf16* w;
  size_t rows, cols;
  uint8_t* codes = nullptr;
  uint8_t* sf = nullptr;
  float* scale = nullptr;
};
inline int quantize_weights_nvfp4(std::vector<Fp4Mat>& mats, uint8_t** buf, float** scales, cudaStream_t s) {
  auto up = [](size_t v, size_t a) { return (v + a - 1) / a * a; };
  size_t bytes = 0, rows = 0;
  for (const Fp4Mat& x : mats) {
    bytes += up(x.rows * x.cols / 2, 256) + up(nvfp4_scale_bytes(x.rows, x.cols), 256);
    rows += up(x.rows, 64);
  }
  if (dev_alloc(buf, bytes) != cudaSuccess || dev_alloc(scales, rows * 4) != cudaSuccess) {
    cudaFree(*buf);
    cudaFree(*scales);
    *buf = nullptr;
    *scales = nullptr;
    return fail(FLUX_ENOMEM, "device allocation of the NVFP4 weights (%zu bytes) failed", bytes);
  }
  FD_CUDA(cudaMemsetAsync(*buf, 0, bytes, s));       // block-scale padding rows read as 0
  size_t boff = 0, roff = 0;
  for (Fp4Mat& x : mats) {
    x.codes = *buf + boff;
    boff += up(x.rows * x.cols / 2, 256);
    x.sf = *buf + boff;
    boff += up(nvfp4_scale_bytes(x.rows, x.cols), 256);
    x.scale = *scales + roff;
    roff += up(x.rows, 64);
    const int r0 = 0, nr = static_cast<int>(x.rows);
    FD_CUDA(quantize_nvfp4_launch(x.w, static_cast<int>(x.cols), static_cast<int>(x.cols), x.codes,
                                  static_cast<int>(x.cols / 2), x.sf, x.scale, q4_segments(&r0, &nr, 1), s));
  }
  return FLUX_OK;
}

// Grow a device buffer to `need` elements (contents are not kept).
template <typename T>
cudaError_t grow(T** p, size_t* cap, size_t need) {
  if (need <= *cap) return cudaSuccess;
  cudaFree(*p);
  *p = nullptr;
  *cap = 0;
  cudaError_t e = dev_alloc(p, need * sizeof(T));
  if (e == cudaSuccess) *cap = need;
  return e;
}

inline size_t ref_tokens(const RefGrids& r) {
  size_t n = 0;
  for (int k = 0; k < r.count; ++k) n += static_cast<size_t>(r.h[k]) * r.w[k];
  return n;
}

inline bool same_refs(const RefGrids& a, const RefGrids& b) {
  if (a.count != b.count) return false;
  for (int k = 0; k < a.count; ++k)
    if (a.h[k] != b.h[k] || a.w[k] != b.w[k]) return false;
  return true;
}

// Host -> device copy of SwiGLU rows [a (F rows); b (F rows)] of width `row_bytes` into the GEMM
// order: for each group of 128 output columns, its 128 a-rows then its 128 b-rows.
cudaError_t copy_swiglu(void* dst, const uint8_t* src, size_t F, size_t row_bytes, cudaStream_t s);

// Device error words of the tcgen05 kernels (synchronises `s`): 0, or the first nonzero code.
int device_error_words(cudaStream_t s);

}  // namespace fdit
