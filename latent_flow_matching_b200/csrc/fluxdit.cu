// C ABI of the FLUX.2-klein denoising transformer on B200 and the host-side
// runner that enqueues one forward as a sequence of sm_100a kernels.
//
// Forward (one CUDA stream, no host synchronisation):
//   timestep embedding -> time MLP -> every block's modulation (one GEMV)
//   img_in / txt_in projections (grouped tcgen05 GEMM) into the fp32 residual X
//   5 x double block: LN+mod -> qkv GEMM (text | image problems) -> QK-RMSNorm+RoPE
//                     -> joint attention -> proj GEMM + gate*residual -> LN+mod
//                     -> SwiGLU GEMM -> out GEMM + gate*residual
//   20 x single block: LN+mod -> fused linear1 GEMM (qkv | SwiGLU problems)
//                     -> QK-RMSNorm+RoPE -> joint attention -> linear2 GEMM + gate*residual
//   final LN+mod on the image rows -> output GEMM -> velocity (fp32)
// Block structure: "Flux 2 Klein: Reine C-basierte Inferenz" ("Modellarchitektur
// und Leistung") and the FLUX.3 Image Klein in Diffusers write-up ("Entkoppelte
// Vorverarbeitung und gemeinsame Attention-Blöcke", "Modulation pro Token-Typ,
// Flow-Map-Destillation und 4D-RoPE").
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/fluxdit.h"
#include "fluxdit_internal.h"
#include "runner.h"

using bf16 = __nv_bfloat16;

namespace fdit {

// ------------------------------------------------------------------ errors
static thread_local std::string g_error;
static thread_local int g_error_code = 0;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_error = buf;
  g_error_code = code;
  return code;
}

int record_error(int code, const char* msg) { return fail(code, "%s", msg); }

const char* last_error() { return g_error.c_str(); }
int last_error_code() { return g_error_code; }

// ------------------------------------------------------------------ tensor maps
static PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
static std::once_flag g_encode_once;

static bool encoder_ready() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode != nullptr;
}

// 2D map with a box of 128 bytes along the row (one 128-byte swizzle row) and box_rows rows.
static bool make_tmap_2d(CUtensorMap* map, CUtensorMapDataType type, uint32_t box_cols, const void* base,
                         uint64_t rows, uint64_t cols, uint64_t row_stride_bytes, uint32_t box_rows,
                         CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  if (!encoder_ready() || rows == 0 || cols == 0) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {row_stride_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return g_encode(map, type, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_out(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t row_stride_bytes,
                   bool f32) {
  return make_tmap_2d(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, f32 ? 16 : 32,
                      base, rows, cols, row_stride_bytes, 32, CU_TENSOR_MAP_SWIZZLE_64B);
}

namespace {
struct OutMapEntry {
  const void* base;
  uint64_t rows, cols, stride;
  bool f32;
  CUtensorMap map;
};
}  // namespace

bool gemm_out_map(CUtensorMap* dst, const GemmProblem& pr) {
  static std::vector<OutMapEntry> cache;
  static std::mutex mu;
  const bool f32 = pr.mode == kEpiF32Bias || pr.mode == kEpiResidGate;
  const uint64_t cols = pr.mode == kEpiSwiGLU ? pr.N / 2 : pr.N;
  const uint64_t stride = static_cast<uint64_t>(pr.ldo) * (f32 ? 4 : 2);
  std::lock_guard<std::mutex> lock(mu);
  for (const OutMapEntry& c : cache)
    if (c.base == pr.out && c.rows == static_cast<uint64_t>(pr.M) && c.cols == cols && c.stride == stride &&
        c.f32 == f32) {
      *dst = c.map;
      return true;
    }
  OutMapEntry c{pr.out, static_cast<uint64_t>(pr.M), cols, stride, f32, {}};
  if (!make_tmap_out(&c.map, pr.out, c.rows, cols, stride, f32)) return false;
  if (cache.size() >= 512) cache.erase(cache.begin());
  cache.push_back(c);
  *dst = c.map;
  return true;
}

bool make_tmap_sf(CUtensorMap* map, const void* base, uint64_t bytes) {
  if (bytes % 256) return false;
  return make_tmap_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 256, base, bytes / 256, 256, 256, 8,
                      CU_TENSOR_MAP_SWIZZLE_NONE);
}

bool make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t row_stride_bytes,
                    uint32_t box_rows) {
  return make_tmap_2d(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 64, base, rows, cols, row_stride_bytes, box_rows);
}

bool make_tmap_u8(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t row_stride_bytes,
                  uint32_t box_rows) {
  return make_tmap_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 128, base, rows, cols, row_stride_bytes, box_rows);
}

int num_sms_current() {
  int dev = 0, n = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

// ------------------------------------------------------------------ launch counter
static std::atomic<unsigned long long> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

bool pdl_enabled() {
  const char* v = std::getenv("FLUX_PDL");
  return !(v && v[0] == '0' && v[1] == 0);
}

// Allocations that still succeed before the injected failure (-1: none injected).
static std::atomic<long long> g_fail_alloc_after{-1};

static bool injected_alloc_failure() {
  long long n = g_fail_alloc_after.load();
  while (n >= 0)
    if (g_fail_alloc_after.compare_exchange_weak(n, n - 1)) return n == 0;
  return false;
}

cudaError_t dev_alloc(void** p, size_t bytes) {
  *p = nullptr;
  if (injected_alloc_failure()) return cudaErrorMemoryAllocation;
  const cudaError_t e = cudaMalloc(p, bytes);
  if (e != cudaSuccess) {
    *p = nullptr;
    cudaGetLastError();
  }
  return e;
}

cudaError_t dev_alloc_async(void** p, size_t bytes, cudaStream_t s) {
  *p = nullptr;
  if (injected_alloc_failure()) return cudaErrorMemoryAllocation;
  const cudaError_t e = cudaMallocAsync(p, bytes, s);
  if (e != cudaSuccess) {
    *p = nullptr;
    cudaGetLastError();
  }
  return e;
}

// ------------------------------------------------------------------ blob layout
struct BlobTensor {
  std::string name;
  size_t rows, cols;        // cols = 1 for vectors
  size_t blob_off;          // byte offset in the blob
};

int device_error_words(cudaStream_t s) {
  const int g = gemm_read_device_error(s);
  const int g2 = gemm2_read_device_error(s);
  const int g4 = gemm_fp4_read_device_error(s);
  const int a = attention_read_device_error(s);
  const int t = selftest_read_device_error(s);
  return g ? g : (g2 ? g2 : (g4 ? g4 : (a ? a : t)));
}

static bool valid_cfg(const flux_dit_config& c) {
  return c.n_double >= 0 && c.n_single >= 0 && c.n_double + c.n_single >= 1 && c.head_dim == 128 &&
         c.heads >= 1 && c.hidden == c.heads * c.head_dim && c.mlp_hidden > 0 && c.mlp_hidden % 128 == 0 &&
         c.in_ch == 128 && c.txt_dim > 0 && c.txt_dim % 64 == 0 && c.t_freq_dim > 0 && c.t_freq_dim % 64 == 0 &&
         c.rope_theta > 0 && c.eps_ln > 0 && c.eps_rms > 0;
}

// Tensor order of the blob (documented in fluxdit.h).
static std::vector<BlobTensor> blob_tensors(const flux_dit_config& c, size_t* total) {
  const size_t D = c.hidden, F = c.mlp_hidden, hd = c.head_dim;
  std::vector<BlobTensor> t;
  auto add = [&](const std::string& n, size_t r, size_t k) { t.push_back({n, r, k, 0}); };
  add("time_in.w1", D, c.t_freq_dim); add("time_in.b1", D, 1);
  add("time_in.w2", D, D); add("time_in.b2", D, 1);
  add("img_in.w", D, c.in_ch); add("img_in.b", D, 1);
  add("txt_in.w", D, c.txt_dim); add("txt_in.b", D, 1);
  for (int i = 0; i < c.n_double; ++i)
    for (const char* s : {"img", "txt"}) {
      const std::string p = "double." + std::to_string(i) + "." + s + ".";
      add(p + "mod.w", 6 * D, D); add(p + "mod.b", 6 * D, 1);
      add(p + "qkv.w", 3 * D, D); add(p + "qkv.b", 3 * D, 1);
      add(p + "q_gain", hd, 1); add(p + "k_gain", hd, 1);
      add(p + "proj.w", D, D); add(p + "proj.b", D, 1);
      add(p + "mlp_in.w", 2 * F, D); add(p + "mlp_in.b", 2 * F, 1);
      add(p + "mlp_out.w", D, F); add(p + "mlp_out.b", D, 1);
    }
  for (int i = 0; i < c.n_single; ++i) {
    const std::string p = "single." + std::to_string(i) + ".";
    add(p + "mod.w", 3 * D, D); add(p + "mod.b", 3 * D, 1);
    add(p + "lin1.w", 3 * D + 2 * F, D); add(p + "lin1.b", 3 * D + 2 * F, 1);
    add(p + "q_gain", hd, 1); add(p + "k_gain", hd, 1);
    add(p + "lin2.w", D, D + F); add(p + "lin2.b", D, 1);
  }
  add("final.mod.w", 2 * D, D); add("final.mod.b", 2 * D, 1);
  add("final.out.w", c.in_ch, D); add("final.out.b", c.in_ch, 1);
  size_t off = 256;
  for (auto& x : t) {
    x.blob_off = off;
    off = (off + x.rows * x.cols * 2 + 255) / 256 * 256;
  }
  *total = off;
  return t;
}

struct BlobHeader {
  char magic[8];
  uint32_t version, n_tensors;
  int32_t n_double, n_single, hidden, heads, head_dim, mlp_hidden, in_ch, txt_dim, t_freq_dim;
  float rope_theta, eps_ln, eps_rms;
  uint64_t data_offset, data_bytes;
};
static_assert(sizeof(BlobHeader) == 80, "blob header layout");

// ------------------------------------------------------------------ model
struct StreamW {                       // one stream of a double block
  const bf16 *qkv_b, *q_gain, *k_gain, *proj_b, *mlp_in_b, *mlp_out_b;
  const bf16 *w_qkv, *w_proj, *w_mlp_in, *w_mlp_out;
  size_t mod_off;                      // into the modulation vector (floats)
  CUtensorMap m_qkv, m_proj, m_mlp_in, m_mlp_out;
  // FP8 precision: e4m3 codes of the same matrices (same row order) and their row scales
  CUtensorMap m8_qkv, m8_proj, m8_mlp_in, m8_mlp_out;
  const float *s_qkv, *s_proj, *s_mlp_in, *s_mlp_out;
  // NVFP4 precision: codes, block scales and row scales of the same matrices
  Fp4Op q4_qkv, q4_proj, q4_mlp_in, q4_mlp_out;
};
struct SingleW {
  const bf16 *qkv_b, *mlp_b, *q_gain, *k_gain, *lin2_b;
  const bf16 *w_lin1, *w_lin2;
  size_t mod_off;
  CUtensorMap m_qkv, m_mlp, m_lin2;
  CUtensorMap m8_qkv, m8_mlp, m8_lin2;
  const float *s_qkv, *s_mlp, *s_lin2;
  Fp4Op q4_qkv, q4_mlp, q4_lin2;
};

constexpr int kMaxBatch = 2;            // sequences of one shape per forward (prompt and unconditional text)

// Activations of a batch of nb sequences of one shape (nt text + ni image + nr reference rows
// each), stored sequence after sequence: rows [b n, (b + 1) n) of X, Y, QKV, CC and the RoPE table
// belong to sequence b.
struct Workspace {
  size_t cap_n = 0, cap_tok = 0, cap_txt = 0;
  float* X = nullptr;
  bf16 *Y = nullptr, *QKV = nullptr, *CC = nullptr, *tokb = nullptr, *txtb = nullptr;
  float2* rope = nullptr;
  int nt = -1, gh = -1, gw = -1, nb = -1;               // shape the maps and the RoPE table were built for
  RefGrids refs = {-1, {}, {}};
  CUtensorMap a_tokb, a_Yall, a_CC, qkv;                // shared image input; whole-batch views
  CUtensorMap a_txtb[kMaxBatch], a_Ytxt[kMaxBatch], a_Yimg[kMaxBatch], a_Yout[kMaxBatch], a_Otxt[kMaxBatch],
      a_Oimg[kMaxBatch], a_Htxt[kMaxBatch], a_Himg[kMaxBatch];   // per-sequence views
  // FP8 precision: e4m3 copies of the GEMM A operands (Y8 = LN-mod output, C8 = [O | H]) with one
  // scale per row (sY; sC over [O | H] for linear2, sO and sH over O and H for the double blocks)
  size_t cap8 = 0;
  uint8_t *Y8 = nullptr, *C8 = nullptr;
  float *sY = nullptr, *sC = nullptr, *sO = nullptr, *sH = nullptr;
  bool maps8 = false;
  CUtensorMap a8_Yall, a8_CC, a8_Ytxt[kMaxBatch], a8_Yimg[kMaxBatch], a8_Otxt[kMaxBatch], a8_Oimg[kMaxBatch],
      a8_Htxt[kMaxBatch], a8_Himg[kMaxBatch];
  // NVFP4 precision: codes of the LN-mod output (Y4) and of [O | H] (C4), their block scales
  // (sfY; sfO, sfH for the double blocks' O and H; sfC for linear2) and row scales.  The double
  // blocks quantise per stream segment (seg_dbl: text and image rows of every sequence, each
  // segment's scales starting on a 128-row block), the single blocks the whole batch (seg_all).
  size_t cap4_rows = 0, cap4_blocks = 0;
  uint8_t *Y4 = nullptr, *C4 = nullptr, *sfY = nullptr, *sfO = nullptr, *sfH = nullptr, *sfC = nullptr;
  float *sY4 = nullptr, *sO4 = nullptr, *sH4 = nullptr, *sC4 = nullptr;
  bool maps4 = false;
  Q4Segs seg_dbl, seg_all;
  Fp4Op y4_txt[kMaxBatch], y4_img[kMaxBatch], y4_all, o4_txt[kMaxBatch], o4_img[kMaxBatch], h4_txt[kMaxBatch],
      h4_img[kMaxBatch], c4_all;
};

}  // namespace fdit

struct flux_dit {
  flux_dit_config cfg;
  int device = 0, num_sms = 148;
  void* wbuf = nullptr;                // every tensor except the modulation linears
  bf16* mods_w = nullptr;              // all modulation weights, rows concatenated
  bf16* mods_b = nullptr;
  size_t mods_rows = 0;
  float *temb = nullptr, *th = nullptr, *vec = nullptr, *mods = nullptr;
  // modulation vectors of a sampler's timesteps, computed together by flux_dit_prepare_timesteps
  static constexpr int kMaxCachedT = 64;
  float* mods_cache = nullptr;          // [cache_n][mods_rows]
  float cache_t[kMaxCachedT] = {};
  int cache_n = 0;
  const float* mods_cur = nullptr;      // the vector the current forward uses
  const bf16 *t_w1, *t_b1, *t_w2, *t_b2, *img_b, *txt_b, *fin_b;
  size_t fin_mod_off = 0;
  CUtensorMap m_img_in, m_txt_in, m_fin;
  std::vector<fdit::StreamW> dbl;      // [2 * i + 0] image stream, [2 * i + 1] text stream of block i
  std::vector<fdit::SingleW> sgl;
  int act_double = 0, act_single = 0;
  int precision = FLUX_PRECISION_BF16;
  uint8_t* w8 = nullptr;               // e4m3 block linears (allocated on the first switch to FP8)
  float* w8_scale = nullptr;
  uint8_t* w4 = nullptr;               // NVFP4 block linears: codes and block scales (first switch to NVFP4)
  float* w4_scale = nullptr;
  fdit::Workspace ws;
  fdit::Profiler prof;
};

namespace fdit {

static void free_ws8(Workspace& w) {
  cudaFree(w.Y8); cudaFree(w.C8); cudaFree(w.sY); cudaFree(w.sC); cudaFree(w.sO); cudaFree(w.sH);
  w.Y8 = w.C8 = nullptr;
  w.sY = w.sC = w.sO = w.sH = nullptr;
  w.cap8 = 0;
  w.maps8 = false;
}

static void free_ws4(Workspace& w) {
  cudaFree(w.Y4); cudaFree(w.C4); cudaFree(w.sfY); cudaFree(w.sfO); cudaFree(w.sfH); cudaFree(w.sfC);
  cudaFree(w.sY4); cudaFree(w.sO4); cudaFree(w.sH4); cudaFree(w.sC4);
  w.Y4 = w.C4 = w.sfY = w.sfO = w.sfH = w.sfC = nullptr;
  w.sY4 = w.sO4 = w.sH4 = w.sC4 = nullptr;
  w.cap4_rows = w.cap4_blocks = 0;
  w.maps4 = false;
}

static void free_ws(Workspace& w) {
  free_ws8(w);
  free_ws4(w);
  cudaFree(w.X); cudaFree(w.Y); cudaFree(w.QKV); cudaFree(w.CC); cudaFree(w.tokb); cudaFree(w.txtb);
  cudaFree(w.rope);
  w = Workspace();
}

static void destroy(flux_dit* m) {
  if (!m) return;
  free_ws(m->ws);
  cudaFree(m->wbuf); cudaFree(m->mods_w); cudaFree(m->mods_b);
  cudaFree(m->w8); cudaFree(m->w8_scale);
  cudaFree(m->w4); cudaFree(m->w4_scale);
  cudaFree(m->temb); cudaFree(m->th); cudaFree(m->vec); cudaFree(m->mods); cudaFree(m->mods_cache);
  delete m;
}

cudaError_t copy_swiglu(void* dst, const uint8_t* src, size_t F, size_t row_bytes, cudaStream_t s) {
  const size_t chunk = 128 * row_bytes;
  const size_t groups = F / 128;
  cudaError_t e = cudaMemcpy2DAsync(dst, 2 * chunk, src, chunk, chunk, groups, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return e;
  return cudaMemcpy2DAsync(static_cast<uint8_t*>(dst) + chunk, 2 * chunk, src + F * row_bytes, chunk, chunk, groups,
                           cudaMemcpyHostToDevice, s);
}

static int create_impl(const void* blob, size_t blob_bytes, const flux_dit_config* cfg_in, cudaStream_t s,
                       flux_dit** out) {
  *out = nullptr;
  if (!blob || blob_bytes < sizeof(BlobHeader)) return fail(FLUX_EINVAL, "blob is NULL or too small");
  BlobHeader h;
  memcpy(&h, blob, sizeof(h));
  if (memcmp(h.magic, "FLUXDIT\0", 8) != 0 || h.version != 1 || h.data_offset != 256)
    return fail(FLUX_EINVAL, "not a FLUXDIT v1 blob");
  flux_dit_config c = {h.n_double, h.n_single, h.hidden, h.heads, h.head_dim, h.mlp_hidden,
                       h.in_ch, h.txt_dim, h.t_freq_dim, h.rope_theta, h.eps_ln, h.eps_rms};
  if (cfg_in && memcmp(cfg_in, &c, sizeof(c)) != 0) return fail(FLUX_EINVAL, "config differs from the blob header");
  if (!valid_cfg(c)) return fail(FLUX_EINVAL, "unsupported model config in blob header");
  size_t total = 0;
  const std::vector<BlobTensor> ts = blob_tensors(c, &total);
  if (h.n_tensors != ts.size() || h.data_bytes + 256 != total || blob_bytes < total)
    return fail(FLUX_EINVAL, "blob size / tensor count mismatch (expected %zu bytes, %zu tensors)", total, ts.size());

  flux_dit* m = new flux_dit();
  m->cfg = c;
  cudaGetDevice(&m->device);
  m->num_sms = num_sms_current();
  const size_t D = c.hidden, F = c.mlp_hidden;
  const uint8_t* b8 = static_cast<const uint8_t*>(blob);

  // device layout: non-modulation tensors packed in blob order; modulation rows concatenated
  std::vector<size_t> dev_off(ts.size(), SIZE_MAX);
  size_t wbytes = 0, mrows = 0;
  for (size_t i = 0; i < ts.size(); ++i) {
    const std::string& n = ts[i].name;
    const bool is_mod = n.size() > 5 && (n.compare(n.size() - 5, 5, "mod.w") == 0 || n.compare(n.size() - 5, 5, "mod.b") == 0);
    if (is_mod) {
      if (n.back() == 'w') mrows += ts[i].rows;
      continue;
    }
    dev_off[i] = wbytes;
    wbytes = (wbytes + ts[i].rows * ts[i].cols * 2 + 255) / 256 * 256;
  }
  m->mods_rows = mrows;
  auto cleanup = [&](int code, const char* what) {
    destroy(m);
    return fail(code, "%s", what);
  };
  if (dev_alloc(&m->wbuf, wbytes) != cudaSuccess || dev_alloc(&m->mods_w, mrows * D * 2) != cudaSuccess ||
      dev_alloc(&m->mods_b, mrows * 2) != cudaSuccess || dev_alloc(&m->temb, c.t_freq_dim * 4) != cudaSuccess ||
      dev_alloc(&m->th, D * 4) != cudaSuccess || dev_alloc(&m->vec, D * 4) != cudaSuccess ||
      dev_alloc(&m->mods, mrows * 4) != cudaSuccess)
    return cleanup(FLUX_ENOMEM, "device allocation of the model weights failed");

  uint8_t* wb = static_cast<uint8_t*>(m->wbuf);
  size_t mrow = 0;
  std::vector<size_t> mod_row(ts.size(), 0);
  for (size_t i = 0; i < ts.size(); ++i) {
    const BlobTensor& t = ts[i];
    const uint8_t* src = b8 + t.blob_off;
    const size_t bytes = t.rows * t.cols * 2;
    cudaError_t e = cudaSuccess;
    if (dev_off[i] == SIZE_MAX) {
      if (t.name.back() == 'w') {
        mod_row[i] = mrow;
        e = cudaMemcpyAsync(m->mods_w + mrow * D, src, bytes, cudaMemcpyHostToDevice, s);
      } else {
        mod_row[i] = mrow;                                   // bias follows its weight
        e = cudaMemcpyAsync(m->mods_b + mrow, src, bytes, cudaMemcpyHostToDevice, s);
        mrow += t.rows;
      }
    } else {
      uint8_t* dst = wb + dev_off[i];
      const std::string& n = t.name;
      const bool mlp_in = n.find("mlp_in.") != std::string::npos;
      const bool lin1 = n.find("lin1.") != std::string::npos;
      if (mlp_in) {
        e = copy_swiglu(dst, src, F, t.cols * 2, s);
      } else if (lin1) {
        const size_t qkv_bytes = 3 * D * t.cols * 2;
        e = cudaMemcpyAsync(dst, src, qkv_bytes, cudaMemcpyHostToDevice, s);
        if (e == cudaSuccess) e = copy_swiglu(dst + qkv_bytes, src + qkv_bytes, F, t.cols * 2, s);
      } else {
        e = cudaMemcpyAsync(dst, src, bytes, cudaMemcpyHostToDevice, s);
      }
    }
    if (e != cudaSuccess) return cleanup(FLUX_EIO, "weight upload failed");
  }

  auto find = [&](const std::string& n) -> size_t {
    for (size_t i = 0; i < ts.size(); ++i)
      if (ts[i].name == n) return i;
    return SIZE_MAX;
  };
  auto W = [&](const std::string& n) { return reinterpret_cast<const bf16*>(wb + dev_off[find(n)]); };
  auto MOD = [&](const std::string& n) { return mod_row[find(n)]; };
  bool maps_ok = true;
  auto wmap = [&](CUtensorMap* map, const bf16* base, size_t rows, size_t cols, uint32_t box) {
    maps_ok &= make_tmap_bf16(map, base, rows, cols, cols * 2, box);
  };

  m->t_w1 = W("time_in.w1"); m->t_b1 = W("time_in.b1");
  m->t_w2 = W("time_in.w2"); m->t_b2 = W("time_in.b2");
  m->img_b = W("img_in.b"); m->txt_b = W("txt_in.b"); m->fin_b = W("final.out.b");
  wmap(&m->m_img_in, W("img_in.w"), D, c.in_ch, 128);
  wmap(&m->m_txt_in, W("txt_in.w"), D, c.txt_dim, 128);
  wmap(&m->m_fin, W("final.out.w"), c.in_ch, D, 128);
  m->fin_mod_off = MOD("final.mod.w");
  m->dbl.resize(2 * c.n_double);
  for (int i = 0; i < c.n_double; ++i)
    for (int sidx = 0; sidx < 2; ++sidx) {
      const std::string p = "double." + std::to_string(i) + (sidx == 0 ? ".img." : ".txt.");
      StreamW& sw = m->dbl[2 * i + sidx];
      sw.qkv_b = W(p + "qkv.b"); sw.q_gain = W(p + "q_gain"); sw.k_gain = W(p + "k_gain");
      sw.proj_b = W(p + "proj.b"); sw.mlp_in_b = W(p + "mlp_in.b"); sw.mlp_out_b = W(p + "mlp_out.b");
      sw.mod_off = MOD(p + "mod.w");
      sw.w_qkv = W(p + "qkv.w"); sw.w_proj = W(p + "proj.w");
      sw.w_mlp_in = W(p + "mlp_in.w"); sw.w_mlp_out = W(p + "mlp_out.w");
      wmap(&sw.m_qkv, W(p + "qkv.w"), 3 * D, D, 128);
      wmap(&sw.m_proj, W(p + "proj.w"), D, D, 128);
      wmap(&sw.m_mlp_in, W(p + "mlp_in.w"), 2 * F, D, 128);
      wmap(&sw.m_mlp_out, W(p + "mlp_out.w"), D, F, 128);
    }
  m->sgl.resize(c.n_single);
  for (int i = 0; i < c.n_single; ++i) {
    const std::string p = "single." + std::to_string(i) + ".";
    SingleW& sw = m->sgl[i];
    const bf16* l1 = W(p + "lin1.w");
    const bf16* l1b = W(p + "lin1.b");
    sw.qkv_b = l1b; sw.mlp_b = l1b + 3 * D;
    sw.q_gain = W(p + "q_gain"); sw.k_gain = W(p + "k_gain"); sw.lin2_b = W(p + "lin2.b");
    sw.mod_off = MOD(p + "mod.w");
    sw.w_lin1 = l1; sw.w_lin2 = W(p + "lin2.w");
    wmap(&sw.m_qkv, l1, 3 * D, D, 128);
    wmap(&sw.m_mlp, l1 + 3 * D * D, 2 * F, D, 128);
    wmap(&sw.m_lin2, W(p + "lin2.w"), D, D + F, 128);
  }
  if (!maps_ok) return cleanup(FLUX_EIO, "cuTensorMapEncodeTiled failed for a weight tensor");
  m->act_double = c.n_double;
  m->act_single = c.n_single;
  if (cudaStreamSynchronize(s) != cudaSuccess) return cleanup(FLUX_EIO, "weight upload failed (sync)");
  *out = m;
  return FLUX_OK;
}

// FP8 copies of the GEMM A operands for a batch of nb sequences of n = nt + nimg rows, and their maps.
static int prepare_fp8(flux_dit* m, int nt, int nimg, int nb) {
  Workspace& w = m->ws;
  const flux_dit_config& c = m->cfg;
  const size_t D = c.hidden, F = c.mlp_hidden;
  const size_t n = nt + nimg, rows = n * nb;
  if (rows > w.cap8) {
    free_ws8(w);
    bool ok = dev_alloc(&w.Y8, rows * D) == cudaSuccess && dev_alloc(&w.C8, rows * (D + F)) == cudaSuccess &&
              dev_alloc(&w.sY, rows * 4) == cudaSuccess && dev_alloc(&w.sC, rows * 4) == cudaSuccess &&
              dev_alloc(&w.sO, rows * 4) == cudaSuccess && dev_alloc(&w.sH, rows * 4) == cudaSuccess;
    if (!ok) {
      free_ws8(w);
      return fail(FLUX_ENOMEM, "FP8 workspace allocation for %zu tokens failed", rows);
    }
    w.cap8 = rows;
  }
  if (w.maps8) return FLUX_OK;
  bool ok = true;
  auto amap = [&](CUtensorMap* map, const uint8_t* base, size_t nrows, size_t cols, uint64_t stride) {
    if (nrows == 0) {
      memset(map, 0, sizeof(*map));
      return;
    }
    ok &= make_tmap_u8(map, base, nrows, cols, stride, 128);
  };
  amap(&w.a8_Yall, w.Y8, rows, D, D);
  amap(&w.a8_CC, w.C8, rows, D + F, D + F);
  for (int b = 0; b < nb; ++b) {
    const size_t r0 = b * n;
    amap(&w.a8_Ytxt[b], w.Y8 + r0 * D, nt, D, D);
    amap(&w.a8_Yimg[b], w.Y8 + (r0 + nt) * D, nimg, D, D);
    amap(&w.a8_Otxt[b], w.C8 + r0 * (D + F), nt, D, D + F);
    amap(&w.a8_Oimg[b], w.C8 + (r0 + nt) * (D + F), nimg, D, D + F);
    amap(&w.a8_Htxt[b], w.C8 + r0 * (D + F) + D, nt, F, D + F);
    amap(&w.a8_Himg[b], w.C8 + (r0 + nt) * (D + F) + D, nimg, F, D + F);
  }
  if (!ok) return fail(FLUX_EIO, "cuTensorMapEncodeTiled failed for an FP8 activation buffer");
  w.maps8 = true;
  return FLUX_OK;
}

// NVFP4 copies of the GEMM A operands for a batch of nb sequences of n = nt + nimg rows, and their maps.
static int prepare_fp4(flux_dit* m, int nt, int nimg, int nb) {
  Workspace& w = m->ws;
  const flux_dit_config& c = m->cfg;
  const size_t D = c.hidden, F = c.mlp_hidden;
  const int n = nt + nimg, rows = n * nb;
  int r0[2 * kMaxBatch], rs[2 * kMaxBatch];
  for (int b = 0; b < nb; ++b) {
    r0[2 * b] = b * n;
    rs[2 * b] = nt;
    r0[2 * b + 1] = b * n + nt;
    rs[2 * b + 1] = nimg;
  }
  const int zero = 0;
  w.seg_dbl = q4_segments(r0, rs, 2 * nb);
  w.seg_all = q4_segments(&zero, &rows, 1);
  size_t blk_dbl = 0;
  for (int z = 0; z < 2 * nb; ++z) blk_dbl += (rs[z] + 127) / 128;
  const size_t blk_all = (rows + 127) / 128, blocks = std::max(blk_dbl, blk_all);
  if (static_cast<size_t>(rows) > w.cap4_rows || blocks > w.cap4_blocks) {
    free_ws4(w);
    const size_t R = rows, B = blocks * 128;
    const bool ok = dev_alloc(&w.Y4, R * D / 2) == cudaSuccess && dev_alloc(&w.C4, R * (D + F) / 2) == cudaSuccess &&
                    dev_alloc(&w.sfY, B * D / 16) == cudaSuccess && dev_alloc(&w.sfO, B * D / 16) == cudaSuccess &&
                    dev_alloc(&w.sfH, B * F / 16) == cudaSuccess &&
                    dev_alloc(&w.sfC, B * (D + F) / 16) == cudaSuccess && dev_alloc(&w.sY4, R * 4) == cudaSuccess &&
                    dev_alloc(&w.sO4, R * 4) == cudaSuccess && dev_alloc(&w.sH4, R * 4) == cudaSuccess &&
                    dev_alloc(&w.sC4, R * 4) == cudaSuccess;
    if (!ok) {
      free_ws4(w);
      return fail(FLUX_ENOMEM, "NVFP4 workspace allocation for %d tokens failed", rows);
    }
    w.cap4_rows = R;
    w.cap4_blocks = blocks;
  }
  if (w.maps4) return FLUX_OK;
  bool ok = true;
  const size_t lY = D / 2, lC = (D + F) / 2;
  for (int b = 0; b < nb; ++b) {
    const size_t rt = static_cast<size_t>(b) * n, ri = rt + nt;
    const int zt = 2 * b, zi = 2 * b + 1;
    ok &= make_fp4_op(&w.y4_txt[b], w.Y4 + rt * lY, nt, D, lY, w.sfY, w.seg_dbl.blk0[zt], w.sY4 + rt);
    ok &= make_fp4_op(&w.y4_img[b], w.Y4 + ri * lY, nimg, D, lY, w.sfY, w.seg_dbl.blk0[zi], w.sY4 + ri);
    ok &= make_fp4_op(&w.o4_txt[b], w.C4 + rt * lC, nt, D, lC, w.sfO, w.seg_dbl.blk0[zt], w.sO4 + rt);
    ok &= make_fp4_op(&w.o4_img[b], w.C4 + ri * lC, nimg, D, lC, w.sfO, w.seg_dbl.blk0[zi], w.sO4 + ri);
    ok &= make_fp4_op(&w.h4_txt[b], w.C4 + rt * lC + D / 2, nt, F, lC, w.sfH, w.seg_dbl.blk0[zt], w.sH4 + rt);
    ok &= make_fp4_op(&w.h4_img[b], w.C4 + ri * lC + D / 2, nimg, F, lC, w.sfH, w.seg_dbl.blk0[zi], w.sH4 + ri);
  }
  ok &= make_fp4_op(&w.y4_all, w.Y4, rows, D, lY, w.sfY, 0, w.sY4);
  ok &= make_fp4_op(&w.c4_all, w.C4, rows, D + F, lC, w.sfC, 0, w.sC4);
  if (!ok) return fail(FLUX_EIO, "cuTensorMapEncodeTiled failed for an NVFP4 activation buffer");
  w.maps4 = true;
  return FLUX_OK;
}

static int prepare_quant(flux_dit* m, int nt, int nimg, int nb) {
  if (m->precision == FLUX_PRECISION_FP8) return prepare_fp8(m, nt, nimg, nb);
  if (m->precision == FLUX_PRECISION_NVFP4) return prepare_fp4(m, nt, nimg, nb);
  return FLUX_OK;
}

static int prepare_shape(flux_dit* m, int nt, int gh, int gw, const RefGrids& refs, int nb, cudaStream_t s) {
  Workspace& w = m->ws;
  const flux_dit_config& c = m->cfg;
  const size_t D = c.hidden, F = c.mlp_hidden;
  const size_t ni = static_cast<size_t>(gh) * gw, nr = ref_tokens(refs);
  const size_t n = nt + ni + nr, rows = n * nb;
  if (rows > w.cap_n) {
    float* X = nullptr;
    free_ws(w);
    bool ok = dev_alloc(&X, rows * D * 4) == cudaSuccess;
    w.X = X;
    ok = ok && dev_alloc(&w.Y, rows * D * 2) == cudaSuccess;
    ok = ok && dev_alloc(&w.QKV, rows * 3 * D * 2) == cudaSuccess;
    ok = ok && dev_alloc(&w.CC, rows * (D + F) * 2) == cudaSuccess;
    ok = ok && dev_alloc(&w.rope, rows * 64 * sizeof(float2)) == cudaSuccess;
    if (!ok) {
      free_ws(w);
      return fail(FLUX_ENOMEM, "workspace allocation for %zu tokens failed", rows);
    }
    w.cap_n = rows;
  }
  if (grow(&w.tokb, &w.cap_tok, (ni + nr) * c.in_ch) != cudaSuccess ||
      grow(&w.txtb, &w.cap_txt, std::max<size_t>(nt * nb, 1) * c.txt_dim) != cudaSuccess) {
    w.nt = -1;                                  // the maps may name a buffer grow() released: rebuild them
    return fail(FLUX_ENOMEM, "workspace allocation failed");
  }
  if (w.nt == nt && w.gh == gh && w.gw == gw && w.nb == nb && same_refs(w.refs, refs))
    return prepare_quant(m, nt, static_cast<int>(ni + nr), nb);
  w.maps8 = false;
  w.maps4 = false;

  const size_t nimg = ni + nr;
  const uint64_t ldD = D * 2, ldC = (D + F) * 2;
  bool ok = true;
  auto amap = [&](CUtensorMap* map, const void* base, size_t nrows, size_t cols, uint64_t stride, uint32_t box) {
    if (nrows == 0) {
      memset(map, 0, sizeof(*map));
      return;
    }
    ok &= make_tmap_bf16(map, base, nrows, cols, stride, box);
  };
  amap(&w.a_tokb, w.tokb, nimg, c.in_ch, c.in_ch * 2, 128);
  amap(&w.a_Yall, w.Y, rows, D, ldD, 128);
  amap(&w.a_CC, w.CC, rows, D + F, ldC, 128);
  amap(&w.qkv, w.QKV, rows, 3 * D, 3 * D * 2, 128);
  for (int b = 0; b < nb; ++b) {
    const size_t r0 = b * n;                           // first row of sequence b
    amap(&w.a_txtb[b], w.txtb + b * nt * c.txt_dim, nt, c.txt_dim, c.txt_dim * 2, 128);
    amap(&w.a_Ytxt[b], w.Y + r0 * D, nt, D, ldD, 128);
    amap(&w.a_Yimg[b], w.Y + (r0 + nt) * D, nimg, D, ldD, 128);
    amap(&w.a_Yout[b], w.Y + b * ni * D, ni, D, ldD, 128);   // output layer input: image rows only
    amap(&w.a_Otxt[b], w.CC + r0 * (D + F), nt, D, ldC, 128);
    amap(&w.a_Oimg[b], w.CC + (r0 + nt) * (D + F), nimg, D, ldC, 128);
    amap(&w.a_Htxt[b], w.CC + r0 * (D + F) + D, nt, F, ldC, 128);
    amap(&w.a_Himg[b], w.CC + (r0 + nt) * (D + F) + D, nimg, F, ldC, 128);
  }
  if (!ok) return fail(FLUX_EIO, "cuTensorMapEncodeTiled failed for an activation buffer");
  if (rope_table_launch(w.rope, nt, gh, gw, refs, c.rope_theta, s) != cudaSuccess)
    return fail(FLUX_EIO, "rope table launch failed");
  for (int b = 1; b < nb; ++b)                         // every sequence has the same positions
    if (cudaMemcpyAsync(w.rope + b * n * 64, w.rope, n * 64 * sizeof(float2), cudaMemcpyDeviceToDevice, s) !=
        cudaSuccess)
      return fail(FLUX_EIO, "rope table copy failed");
  w.nt = nt; w.gh = gh; w.gw = gw; w.nb = nb; w.refs = refs;
  return prepare_quant(m, nt, static_cast<int>(nimg), nb);
}

// Quantise every block linear to e4m3 with one scale per output row (done once per model).
static int quantize_block_weights(flux_dit* m, cudaStream_t s) {
  const flux_dit_config& c = m->cfg;
  const size_t D = c.hidden, F = c.mlp_hidden;
  struct Mat {
    const bf16* w;
    size_t rows, cols;
  };
  std::vector<Mat> mats;
  for (const StreamW& sw : m->dbl) {
    mats.push_back({sw.w_qkv, 3 * D, D});
    mats.push_back({sw.w_proj, D, D});
    mats.push_back({sw.w_mlp_in, 2 * F, D});
    mats.push_back({sw.w_mlp_out, D, F});
  }
  for (const SingleW& sw : m->sgl) {
    mats.push_back({sw.w_lin1, 3 * D + 2 * F, D});
    mats.push_back({sw.w_lin2, D, D + F});
  }
  size_t bytes = 0, rows = 0;
  for (const Mat& x : mats) {
    bytes += (x.rows * x.cols + 255) / 256 * 256;
    rows += (x.rows + 63) / 64 * 64;
  }
  if (dev_alloc(&m->w8, bytes) != cudaSuccess || dev_alloc(&m->w8_scale, rows * 4) != cudaSuccess) {
    cudaFree(m->w8);
    cudaFree(m->w8_scale);
    m->w8 = nullptr;
    m->w8_scale = nullptr;
    return fail(FLUX_ENOMEM, "device allocation of the FP8 weights (%zu bytes) failed", bytes);
  }
  std::vector<const uint8_t*> q(mats.size());
  std::vector<const float*> sc(mats.size());
  size_t boff = 0, roff = 0;
  for (size_t i = 0; i < mats.size(); ++i) {
    const Mat& x = mats[i];
    uint8_t* qd = m->w8 + boff;
    float* sd = m->w8_scale + roff;
    FD_CUDA(quantize_rows_launch(x.w, static_cast<int>(x.cols), static_cast<int>(x.rows), static_cast<int>(x.cols),
                                 qd, static_cast<int>(x.cols), sd, s));
    q[i] = qd;
    sc[i] = sd;
    boff += (x.rows * x.cols + 255) / 256 * 256;
    roff += (x.rows + 63) / 64 * 64;
  }
  bool ok = true;
  auto wmap = [&](CUtensorMap* map, const uint8_t* base, size_t r, size_t cols) {
    ok &= make_tmap_u8(map, base, r, cols, cols, 128);
  };
  size_t i = 0;
  for (StreamW& sw : m->dbl) {
    wmap(&sw.m8_qkv, q[i], 3 * D, D); sw.s_qkv = sc[i++];
    wmap(&sw.m8_proj, q[i], D, D); sw.s_proj = sc[i++];
    wmap(&sw.m8_mlp_in, q[i], 2 * F, D); sw.s_mlp_in = sc[i++];
    wmap(&sw.m8_mlp_out, q[i], D, F); sw.s_mlp_out = sc[i++];
  }
  for (SingleW& sw : m->sgl) {
    wmap(&sw.m8_qkv, q[i], 3 * D, D);
    wmap(&sw.m8_mlp, q[i] + 3 * D * D, 2 * F, D);
    sw.s_qkv = sc[i];
    sw.s_mlp = sc[i] + 3 * D;
    ++i;
    wmap(&sw.m8_lin2, q[i], D, D + F); sw.s_lin2 = sc[i++];
  }
  if (!ok) return fail(FLUX_EIO, "cuTensorMapEncodeTiled failed for an FP8 weight tensor");
  FD_CUDA(cudaStreamSynchronize(s));
  return FLUX_OK;
}

// Quantise every block linear to NVFP4 (done once per model, on the first switch to NVFP4).
static int quantize_block_weights_nvfp4(flux_dit* m, cudaStream_t s) {
  const flux_dit_config& c = m->cfg;
  const size_t D = c.hidden, F = c.mlp_hidden;
  std::vector<Fp4Mat> mats;
  for (const StreamW& sw : m->dbl) {
    mats.push_back({sw.w_qkv, 3 * D, D});
    mats.push_back({sw.w_proj, D, D});
    mats.push_back({sw.w_mlp_in, 2 * F, D});
    mats.push_back({sw.w_mlp_out, D, F});
  }
  for (const SingleW& sw : m->sgl) {
    mats.push_back({sw.w_lin1, 3 * D + 2 * F, D});
    mats.push_back({sw.w_lin2, D, D + F});
  }
  int rc = quantize_weights_nvfp4(mats, &m->w4, &m->w4_scale, s);
  if (rc) return rc;
  bool ok = true;
  auto op = [&](Fp4Op* o, const Fp4Mat& x, size_t row0, size_t rows) {
    ok &= make_fp4_op(o, x.codes + row0 * x.cols / 2, rows, x.cols, x.cols / 2, x.sf, row0 / 128, x.scale + row0);
  };
  size_t i = 0;
  for (StreamW& sw : m->dbl) {
    op(&sw.q4_qkv, mats[i], 0, 3 * D); ++i;
    op(&sw.q4_proj, mats[i], 0, D); ++i;
    op(&sw.q4_mlp_in, mats[i], 0, 2 * F); ++i;
    op(&sw.q4_mlp_out, mats[i], 0, D); ++i;
  }
  for (SingleW& sw : m->sgl) {
    op(&sw.q4_qkv, mats[i], 0, 3 * D);
    op(&sw.q4_mlp, mats[i], 3 * D, 2 * F);             // the SwiGLU rows start on a 128-row block (D % 128 == 0)
    ++i;
    op(&sw.q4_lin2, mats[i], 0, D); ++i;
  }
  if (!ok) return fail(FLUX_EIO, "cuTensorMapEncodeTiled failed for an NVFP4 weight tensor");
  FD_CUDA(cudaStreamSynchronize(s));
  return FLUX_OK;
}

static int run_modulation(flux_dit* m, float t, cudaStream_t s) {
  const flux_dit_config& c = m->cfg;
  const int D = c.hidden;
  for (int i = 0; i < m->cache_n; ++i)
    if (m->cache_t[i] == t) {                 // prepared with the other timesteps of the sampler
      m->mods_cur = m->mods_cache + static_cast<size_t>(i) * m->mods_rows;
      return FLUX_OK;
    }
  m->mods_cur = m->mods;
  auto gv = [](double rows, double k) { return rows * k * 2 + rows * 6 + k * 4; };
  FD_LAUNCH(m, kProfOther, 0, c.t_freq_dim * 4.0, timestep_embed_launch(m->temb, t, c.t_freq_dim, s));
  FD_LAUNCH(m, kProfGemv, 2.0 * D * c.t_freq_dim, gv(D, c.t_freq_dim),
            gemv_launch(m->t_w1, m->t_b1, m->temb, m->th, D, c.t_freq_dim, 0, 1, s));
  FD_LAUNCH(m, kProfGemv, 2.0 * D * D, gv(D, D), gemv_launch(m->t_w2, m->t_b2, m->th, m->vec, D, D, 0, 0, s));
  FD_LAUNCH(m, kProfGemv, 2.0 * m->mods_rows * D, gv(static_cast<double>(m->mods_rows), D),
            gemv_launch(m->mods_w, m->mods_b, m->vec, m->mods, static_cast<int>(m->mods_rows), D, 1, 0, s));
  return FLUX_OK;
}

// One forward of nb sequences that share the image tokens, the references and t and differ in
// their text (nb = 2: the prompt and the unconditional text of classifier-free guidance).
// txt[b] and v_out[b] are the text rows and the velocity output of sequence b.
static int forward_impl(flux_dit* m, const float* img_tok, int gh, int gw, const float* const* txt, int nt,
                        const float* ref_tok, const RefGrids& refs, float t, float* const* v_out, int nb,
                        cudaStream_t s) {
  const flux_dit_config& c = m->cfg;
  const int D = c.hidden, F = c.mlp_hidden, H = c.heads;
  if (nb < 1 || nb > kMaxBatch) return fail(FLUX_EINVAL, "batch of %d sequences (1..%d)", nb, kMaxBatch);
  if (!img_tok) return fail(FLUX_EINVAL, "img_tok must be a device pointer");
  for (int b = 0; b < nb; ++b) {
    if (!v_out[b]) return fail(FLUX_EINVAL, "velocity output %d is NULL", b);
    if (nt > 0 && !txt[b]) return fail(FLUX_EINVAL, "text %d is NULL", b);
  }
  if (gh < 4 || gh > 64 || gw < 4 || gw > 64) return fail(FLUX_EINVAL, "image grid %dx%d outside 4..64", gh, gw);
  if (nt < 0 || nt > 4096) return fail(FLUX_EINVAL, "bad text (n_txt=%d)", nt);
  if (refs.count < 0 || refs.count > kMaxRefs)
    return fail(FLUX_EINVAL, "%d reference images (at most %d)", refs.count, kMaxRefs);
  for (int k = 0; k < refs.count; ++k)
    if (refs.h[k] < 4 || refs.h[k] > 64 || refs.w[k] < 4 || refs.w[k] > 64)
      return fail(FLUX_EINVAL, "reference %d grid %dx%d outside 4..64", k, refs.h[k], refs.w[k]);
  if (refs.count > 0 && !ref_tok) return fail(FLUX_EINVAL, "ref_tok is NULL for %d reference(s)", refs.count);
  if (!std::isfinite(t)) return fail(FLUX_EINVAL, "t is not finite");
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev != m->device) return fail(FLUX_EINVAL, "model lives on device %d, current device is %d", m->device, dev);

  int rc = prepare_shape(m, nt, gh, gw, refs, nb, s);
  if (rc) return rc;
  Workspace& w = m->ws;
  const int ni = gh * gw, nr = static_cast<int>(ref_tokens(refs)), nimg = ni + nr, n = nt + nimg;
  const int rows = n * nb;
  const float eps_ln = c.eps_ln, eps_rms = c.eps_rms;
  auto seq_row = [&](int b, int r) { return static_cast<size_t>(b) * n + r; };   // row r of sequence b

  rc = run_modulation(m, t, s);                   // one t, so one modulation vector for every sequence
  if (rc) return rc;
  const float* mods = m->mods_cur;
  FD_LAUNCH(m, kProfOther, 0, 6.0 * ni * c.in_ch,
            cast_bf16_launch(img_tok, w.tokb, static_cast<size_t>(ni) * c.in_ch, s));
  if (nr)
    FD_LAUNCH(m, kProfOther, 0, 6.0 * nr * c.in_ch,
              cast_bf16_launch(ref_tok, w.tokb + static_cast<size_t>(ni) * c.in_ch,
                               static_cast<size_t>(nr) * c.in_ch, s));
  for (int b = 0; b < nb && nt; ++b)
    FD_LAUNCH(m, kProfOther, 0, 6.0 * nt * c.txt_dim,
              cast_bf16_launch(txt[b], w.txtb + static_cast<size_t>(b) * nt * c.txt_dim,
                               static_cast<size_t>(nt) * c.txt_dim, s));
  const double ln_bytes = 6.0 * rows * D + 16.0 * D, ln_bytes_img = 6.0 * ni * D + 8.0 * D;
  const double at_flops = 4.0 * nb * n * static_cast<double>(n) * D, at_bytes = 8.0 * rows * D;

  // input projections: text rows with txt_in, image + reference rows with img_in, per sequence
  GemmParams4 P4;
  GemmParams& P = P4.g;
  P.num_problems = 2 * nb;
  for (int b = 0; b < nb; ++b) {
    problem(P, 2 * b, w.a_txtb[b], m->m_txt_in, nt, D, c.txt_dim, kEpiF32Bias, w.X + seq_row(b, 0) * D, D,
            m->txt_b, nullptr);
    problem(P, 2 * b + 1, w.a_tokb, m->m_img_in, nimg, D, c.in_ch, kEpiF32Bias, w.X + seq_row(b, nt) * D, D,
            m->img_b, nullptr);
  }
  FD_LAUNCH(m, kProfGemm, gemm_flops(P), gemm_bytes(P), launch_linear(P, m->num_sms, s, false, nb));

  AttnParams A;
  A.mapQ = w.qkv; A.mapK = w.qkv; A.mapV = w.qkv;
  A.out = w.CC; A.ldo = D + F; A.n = n; A.heads = H; A.batch = nb;
  A.q_col0 = 0; A.k_col0 = D; A.v_col0 = 2 * D;
  A.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(c.head_dim)));

  // FP8 precision: block linears on e4m3 codes (row-wise scales); LN-mod quantises its output,
  // the attention output and the SwiGLU hidden are quantised before the linears that read them.
  // NVFP4 precision: the same operands as e2m1 codes with block and row scales (LN-mod quantises
  // its output per segment in the same pass).
  const bool fp8 = m->precision == FLUX_PRECISION_FP8;
  const bool fp4 = m->precision == FLUX_PRECISION_NVFP4;
  const OpFormat lin_fmt = fp4 ? OpFormat::kNvfp4 : fp8 ? OpFormat::kE4M3 : OpFormat::kBf16;
  auto f8 = [&](int i, const CUtensorMap& a8, const CUtensorMap& w8, const float* sa, const float* sb) {
    P.mapA[i] = a8;
    P.mapB[i] = w8;
    P.prob[i].scale_a = sa;
    P.prob[i].scale_b = sb;
  };
  auto linear = [&]() -> cudaError_t {
    return fp4 ? gemm_fp4_launch(P4, m->num_sms, s) : launch_linear(P, m->num_sms, s, fp8, nb);
  };
  // NVFP4 codes of bf16 rows (ldx elements apart) into q (ldq bytes apart), one launch over the segments
  auto quant4 = [&](const bf16* x, int ldx, int k, uint8_t* q, int ldq, uint8_t* sf, float* sc,
                    const Q4Segs& segs) -> int {
    FD_LAUNCH(m, kProfOther, 0, 2.5 * rows * k + 4.0 * rows,
              quantize_nvfp4_launch(x, ldx, k, q, ldq, sf, sc, segs, s));
    return FLUX_OK;
  };
  // LN-mod of every row: rows r % n < split use (sh0, sc0), the others (sh1, sc1); NVFP4 then
  // quantises Y over the segments `segs`
  auto ln_mod = [&](int split, const float* sh0, const float* sc0, const float* sh1, const float* sc1,
                    const Q4Segs& segs) -> int {
    if (fp4) {
      const LnModSets ms{split, n, n, sh0, sh1, sh1, sc0, sc1, sc1};
      FD_LAUNCH(m, kProfLnMod, 0, 4.56 * rows * D + 4.0 * rows,
                ln_modulate_nvfp4_launch(w.X, D, w.Y4, w.sfY, w.sY4, segs, ms, eps_ln, s));
      return FLUX_OK;
    }
    if (fp8)
      FD_LAUNCH(m, kProfLnMod, 0, 5.0 * rows * D + 4.0 * rows,
                ln_modulate_fp8_launch(w.X, w.Y8, w.sY, rows, D, split, n, n, sh0, sc0, sh1, sc1, sh1, sc1, eps_ln,
                                       s));
    else
      FD_LAUNCH(m, kProfLnMod, 0, ln_bytes, ln_modulate_launch(w.X, w.Y, rows, D, split, n, sh0, sc0, sh1, sc1,
                                                               eps_ln, s));
    return FLUX_OK;
  };
  // e4m3 codes of CC columns [col0, col0 + cols) into C8, one scale per row
  auto quant_cc = [&](int col0, int cols, float* scale) -> int {
    FD_LAUNCH(m, kProfOther, 0, 3.0 * rows * cols + 4.0 * rows,
              quantize_rows_launch(w.CC + col0, D + F, rows, cols, w.C8 + col0, D + F, scale, s));
    return FLUX_OK;
  };

  for (int i = 0; i < m->act_double; ++i) {
    const NvtxRange range("double block %d", i);
    const StreamW& si = m->dbl[2 * i];
    const StreamW& st = m->dbl[2 * i + 1];
    const float* mi = mods + si.mod_off;          // shift1, scale1, gate1, shift2, scale2, gate2
    const float* mt = mods + st.mod_off;
    rc = ln_mod(nt, mt, mt + D, mi, mi + D, w.seg_dbl);
    if (rc) return rc;
    P.num_problems = 2 * nb;
    for (int b = 0; b < nb; ++b) {
      problem(P, 2 * b, w.a_Ytxt[b], st.m_qkv, nt, 3 * D, D, kEpiBf16Bias, w.QKV + seq_row(b, 0) * 3 * D, 3 * D,
              st.qkv_b, nullptr);
      problem(P, 2 * b + 1, w.a_Yimg[b], si.m_qkv, nimg, 3 * D, D, kEpiBf16Bias, w.QKV + seq_row(b, nt) * 3 * D,
              3 * D, si.qkv_b, nullptr);
      qk_fuse(P, 2 * b, st.q_gain, st.k_gain, w.rope, static_cast<int>(seq_row(b, 0)), eps_rms);
      qk_fuse(P, 2 * b + 1, si.q_gain, si.k_gain, w.rope, static_cast<int>(seq_row(b, nt)), eps_rms);
      if (fp8) {
        f8(2 * b, w.a8_Ytxt[b], st.m8_qkv, w.sY + seq_row(b, 0), st.s_qkv);
        f8(2 * b + 1, w.a8_Yimg[b], si.m8_qkv, w.sY + seq_row(b, nt), si.s_qkv);
      }
      if (fp4) {
        fp4_operands(P4, 2 * b, w.y4_txt[b], st.q4_qkv);
        fp4_operands(P4, 2 * b + 1, w.y4_img[b], si.q4_qkv);
      }
    }
    FD_LAUNCH(m, kProfGemm, gemm_flops(P), gemm_bytes(P, lin_fmt), linear());
    FD_LAUNCH(m, kProfAttention, at_flops, at_bytes, attention_launch(A, s));
    if (fp8 && (rc = quant_cc(0, D, w.sO))) return rc;
    if (fp4 && (rc = quant4(w.CC, D + F, D, w.C4, (D + F) / 2, w.sfO, w.sO4, w.seg_dbl))) return rc;
    P.num_problems = 2 * nb;
    for (int b = 0; b < nb; ++b) {
      problem(P, 2 * b, w.a_Otxt[b], st.m_proj, nt, D, D, kEpiResidGate, w.X + seq_row(b, 0) * D, D, st.proj_b,
              mt + 2 * D);
      problem(P, 2 * b + 1, w.a_Oimg[b], si.m_proj, nimg, D, D, kEpiResidGate, w.X + seq_row(b, nt) * D, D,
              si.proj_b, mi + 2 * D);
      if (fp8) {
        f8(2 * b, w.a8_Otxt[b], st.m8_proj, w.sO + seq_row(b, 0), st.s_proj);
        f8(2 * b + 1, w.a8_Oimg[b], si.m8_proj, w.sO + seq_row(b, nt), si.s_proj);
      }
      if (fp4) {
        fp4_operands(P4, 2 * b, w.o4_txt[b], st.q4_proj);
        fp4_operands(P4, 2 * b + 1, w.o4_img[b], si.q4_proj);
      }
    }
    FD_LAUNCH(m, kProfGemm, gemm_flops(P), gemm_bytes(P, lin_fmt), linear());
    rc = ln_mod(nt, mt + 3 * D, mt + 4 * D, mi + 3 * D, mi + 4 * D, w.seg_dbl);
    if (rc) return rc;
    P.num_problems = 2 * nb;
    for (int b = 0; b < nb; ++b) {
      problem(P, 2 * b, w.a_Ytxt[b], st.m_mlp_in, nt, 2 * F, D, kEpiSwiGLU, w.CC + seq_row(b, 0) * (D + F) + D,
              D + F, st.mlp_in_b, nullptr);
      problem(P, 2 * b + 1, w.a_Yimg[b], si.m_mlp_in, nimg, 2 * F, D, kEpiSwiGLU,
              w.CC + seq_row(b, nt) * (D + F) + D, D + F, si.mlp_in_b, nullptr);
      if (fp8) {
        f8(2 * b, w.a8_Ytxt[b], st.m8_mlp_in, w.sY + seq_row(b, 0), st.s_mlp_in);
        f8(2 * b + 1, w.a8_Yimg[b], si.m8_mlp_in, w.sY + seq_row(b, nt), si.s_mlp_in);
      }
      if (fp4) {
        fp4_operands(P4, 2 * b, w.y4_txt[b], st.q4_mlp_in);
        fp4_operands(P4, 2 * b + 1, w.y4_img[b], si.q4_mlp_in);
      }
    }
    FD_LAUNCH(m, kProfGemm, gemm_flops(P), gemm_bytes(P, lin_fmt), linear());
    if (fp8 && (rc = quant_cc(D, F, w.sH))) return rc;
    if (fp4 && (rc = quant4(w.CC + D, D + F, F, w.C4 + D / 2, (D + F) / 2, w.sfH, w.sH4, w.seg_dbl))) return rc;
    P.num_problems = 2 * nb;
    for (int b = 0; b < nb; ++b) {
      problem(P, 2 * b, w.a_Htxt[b], st.m_mlp_out, nt, D, F, kEpiResidGate, w.X + seq_row(b, 0) * D, D,
              st.mlp_out_b, mt + 5 * D);
      problem(P, 2 * b + 1, w.a_Himg[b], si.m_mlp_out, nimg, D, F, kEpiResidGate, w.X + seq_row(b, nt) * D, D,
              si.mlp_out_b, mi + 5 * D);
      if (fp8) {
        f8(2 * b, w.a8_Htxt[b], st.m8_mlp_out, w.sH + seq_row(b, 0), st.s_mlp_out);
        f8(2 * b + 1, w.a8_Himg[b], si.m8_mlp_out, w.sH + seq_row(b, nt), si.s_mlp_out);
      }
      if (fp4) {
        fp4_operands(P4, 2 * b, w.h4_txt[b], st.q4_mlp_out);
        fp4_operands(P4, 2 * b + 1, w.h4_img[b], si.q4_mlp_out);
      }
    }
    FD_LAUNCH(m, kProfGemm, gemm_flops(P), gemm_bytes(P, lin_fmt), linear());
  }
  // single blocks: one set of weights for every row, so the whole batch is one problem
  for (int i = 0; i < m->act_single; ++i) {
    const NvtxRange range("single block %d", i);
    const SingleW& sw = m->sgl[i];
    const float* ms = mods + sw.mod_off;          // shift, scale, gate
    rc = ln_mod(n, ms, ms + D, ms, ms + D, w.seg_all);
    if (rc) return rc;
    P.num_problems = 2;
    problem(P, 0, w.a_Yall, sw.m_qkv, rows, 3 * D, D, kEpiBf16Bias, w.QKV, 3 * D, sw.qkv_b, nullptr);
    problem(P, 1, w.a_Yall, sw.m_mlp, rows, 2 * F, D, kEpiSwiGLU, w.CC + D, D + F, sw.mlp_b, nullptr);
    qk_fuse(P, 0, sw.q_gain, sw.k_gain, w.rope, 0, eps_rms);
    if (fp8) {
      f8(0, w.a8_Yall, sw.m8_qkv, w.sY, sw.s_qkv);
      f8(1, w.a8_Yall, sw.m8_mlp, w.sY, sw.s_mlp);
    }
    if (fp4) {
      fp4_operands(P4, 0, w.y4_all, sw.q4_qkv);
      fp4_operands(P4, 1, w.y4_all, sw.q4_mlp);
    }
    FD_LAUNCH(m, kProfGemm, gemm_flops(P), gemm_bytes(P, lin_fmt), linear());
    FD_LAUNCH(m, kProfAttention, at_flops, at_bytes, attention_launch(A, s));
    if (fp8 && (rc = quant_cc(0, D + F, w.sC))) return rc;
    if (fp4 && (rc = quant4(w.CC, D + F, D + F, w.C4, (D + F) / 2, w.sfC, w.sC4, w.seg_all))) return rc;
    P.num_problems = 1;
    problem(P, 0, w.a_CC, sw.m_lin2, rows, D, D + F, kEpiResidGate, w.X, D, sw.lin2_b, ms + 2 * D);
    if (fp8) f8(0, w.a8_CC, sw.m8_lin2, w.sC, sw.s_lin2);
    if (fp4) fp4_operands(P4, 0, w.c4_all, sw.q4_lin2);
    FD_LAUNCH(m, kProfGemm, gemm_flops(P), gemm_bytes(P, lin_fmt), linear());
  }
  // output layer on the image rows of each sequence
  const NvtxRange range("output layer");
  const float* mf = mods + m->fin_mod_off;         // shift, scale
  for (int b = 0; b < nb; ++b)
    FD_LAUNCH(m, kProfLnMod, 0, ln_bytes_img,
              ln_modulate_launch(w.X + seq_row(b, nt) * D, w.Y + static_cast<size_t>(b) * ni * D, ni, D, ni, ni, mf,
                                 mf + D, mf, mf + D, eps_ln, s));
  P.num_problems = nb;
  for (int b = 0; b < nb; ++b)
    problem(P, b, w.a_Yout[b], m->m_fin, ni, c.in_ch, D, kEpiF32Bias, v_out[b], c.in_ch, m->fin_b, nullptr);
  FD_LAUNCH(m, kProfGemm, gemm_flops(P), gemm_bytes(P), gemm_launch(P, 128, m->num_sms, s));
  return FLUX_OK;
}

}  // namespace fdit

using namespace fdit;

// ====================================================================== C ABI
extern "C" {

const char* flux_get_error(void) { return last_error(); }

int flux_get_error_code(void) { return last_error_code(); }

size_t flux_blob_expected_bytes(const flux_dit_config* cfg) {
  if (!cfg || !valid_cfg(*cfg)) return 0;
  size_t total = 0;
  blob_tensors(*cfg, &total);
  return total;
}

flux_dit* flux_dit_create(const void* blob, size_t blob_bytes, const flux_dit_config* cfg, void* stream) {
  flux_dit* m = nullptr;
  create_impl(blob, blob_bytes, cfg, static_cast<cudaStream_t>(stream), &m);
  return m;
}

void flux_dit_destroy(flux_dit* m) { destroy(m); }

int flux_dit_forward(flux_dit* m, const float* img_tok, int grid_h, int grid_w, const float* txt, int n_txt,
                     const float* ref_tok, int ref_h, int ref_w, float t, float* v_out, void* stream) {
  if (!m) return fail(FLUX_EINVAL, "model is NULL");
  if (!((ref_h == 0 && ref_w == 0) || (ref_h > 0 && ref_w > 0)))
    return fail(FLUX_EINVAL, "reference grid %dx%d", ref_h, ref_w);
  RefGrids refs = {ref_h > 0 ? 1 : 0, {ref_h}, {ref_w}};
  return forward_impl(m, img_tok, grid_h, grid_w, &txt, n_txt, ref_tok, refs, t, &v_out, 1,
                      static_cast<cudaStream_t>(stream));
}

int flux_dit_forward_refs(flux_dit* m, const float* img_tok, int grid_h, int grid_w, const float* txt, int n_txt,
                          const float* ref_tok, int n_refs, const int* ref_grids, float t, float* v_out,
                          void* stream) {
  if (!m) return fail(FLUX_EINVAL, "model is NULL");
  if (n_refs < 0 || n_refs > kMaxRefs) return fail(FLUX_EINVAL, "%d reference images (at most %d)", n_refs, kMaxRefs);
  if (n_refs > 0 && !ref_grids) return fail(FLUX_EINVAL, "ref_grids is NULL");
  RefGrids refs = {n_refs, {}, {}};
  for (int k = 0; k < n_refs; ++k) {
    refs.h[k] = ref_grids[2 * k];
    refs.w[k] = ref_grids[2 * k + 1];
  }
  return forward_impl(m, img_tok, grid_h, grid_w, &txt, n_txt, ref_tok, refs, t, &v_out, 1,
                      static_cast<cudaStream_t>(stream));
}

int flux_dit_forward_cfg(flux_dit* m, const float* img_tok, int grid_h, int grid_w, const float* txt_cond,
                         const float* txt_uncond, int n_txt, const float* ref_tok, int n_refs, const int* ref_grids,
                         float t, float* v_cond, float* v_uncond, void* stream) {
  if (!m) return fail(FLUX_EINVAL, "model is NULL");
  if (n_refs < 0 || n_refs > kMaxRefs) return fail(FLUX_EINVAL, "%d reference images (at most %d)", n_refs, kMaxRefs);
  if (n_refs > 0 && !ref_grids) return fail(FLUX_EINVAL, "ref_grids is NULL");
  if (v_cond && v_cond == v_uncond) return fail(FLUX_EINVAL, "v_cond and v_uncond must be different buffers");
  RefGrids refs = {n_refs, {}, {}};
  for (int k = 0; k < n_refs; ++k) {
    refs.h[k] = ref_grids[2 * k];
    refs.w[k] = ref_grids[2 * k + 1];
  }
  const float* txt[2] = {txt_cond, txt_uncond};
  float* v[2] = {v_cond, v_uncond};
  return forward_impl(m, img_tok, grid_h, grid_w, txt, n_txt, ref_tok, refs, t, v, 2,
                      static_cast<cudaStream_t>(stream));
}

int flux_cfg_euler_step(float* x, const float* v_cond, const float* v_uncond, size_t n, float guidance, float dt,
                        void* stream) {
  if (n && (!x || !v_cond || !v_uncond)) return fail(FLUX_EINVAL, "NULL argument");
  if (!aligned16(x) || !aligned16(v_cond) || !aligned16(v_uncond))
    return fail(FLUX_EINVAL, "x, v_cond and v_uncond must be 16-byte aligned");
  if (!std::isfinite(guidance) || !std::isfinite(dt)) return fail(FLUX_EINVAL, "guidance and dt must be finite");
  FD_CUDA(cfg_euler_launch(x, v_cond, v_uncond, nullptr, n, guidance, dt, static_cast<cudaStream_t>(stream)));
  return FLUX_OK;
}

int flux_cfg_euler_step_out(float* x, const float* v_cond, const float* v_uncond, float* v_guided, size_t n,
                            float guidance, float dt, void* stream) {
  if (n && (!x || !v_cond || !v_uncond || !v_guided)) return fail(FLUX_EINVAL, "NULL argument");
  if (!aligned16(x) || !aligned16(v_cond) || !aligned16(v_uncond) || !aligned16(v_guided))
    return fail(FLUX_EINVAL, "x, v_cond, v_uncond and v_guided must be 16-byte aligned");
  if (!std::isfinite(guidance) || !std::isfinite(dt)) return fail(FLUX_EINVAL, "guidance and dt must be finite");
  FD_CUDA(cfg_euler_launch(x, v_cond, v_uncond, v_guided, n, guidance, dt, static_cast<cudaStream_t>(stream)));
  return FLUX_OK;
}

int flux_blend_latents(const float* x, const float* noise, float t, float* out, size_t n, void* stream) {
  if (n && (!x || !noise || !out)) return fail(FLUX_EINVAL, "NULL argument");
  if (!std::isfinite(t)) return fail(FLUX_EINVAL, "t is not finite");
  FD_CUDA(blend_launch(x, noise, t, out, n, static_cast<cudaStream_t>(stream)));
  return FLUX_OK;
}

int flux_dit_set_precision(flux_dit* m, int precision) {
  if (!m) return fail(FLUX_EINVAL, "model is NULL");
  if (precision == FLUX_PRECISION_BF16) {
    m->precision = precision;
    return FLUX_OK;
  }
  if (precision != FLUX_PRECISION_FP8 && precision != FLUX_PRECISION_NVFP4)
    return fail(FLUX_EINVAL, "unknown precision %d", precision);
  const flux_dit_config& c = m->cfg;
  if (precision == FLUX_PRECISION_FP8 &&
      (c.hidden % 128 || c.mlp_hidden % 128 || (c.hidden != 1024 && c.hidden != 2048 && c.hidden != 3072 &&
                                                c.hidden != 4096) || c.hidden + c.mlp_hidden > 16384))
    return fail(FLUX_EINVAL, "FP8 needs hidden in {1024, 2048, 3072, 4096} and hidden + mlp_hidden <= 16384");
  if (precision == FLUX_PRECISION_NVFP4 &&
      ((c.hidden != 1024 && c.hidden != 2048 && c.hidden != 3072 && c.hidden != 4096) || c.mlp_hidden % 256 ||
       c.hidden + c.mlp_hidden > 16384))
    return fail(FLUX_EINVAL, "NVFP4 needs hidden in {1024, 2048, 3072, 4096}, mlp_hidden a multiple of 256 and "
                             "hidden + mlp_hidden <= 16384");
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev != m->device) return fail(FLUX_EINVAL, "model lives on device %d, current device is %d", m->device, dev);
  if (precision == FLUX_PRECISION_FP8 && !m->w8) {
    const int rc = quantize_block_weights(m, nullptr);
    if (rc) return rc;
  }
  if (precision == FLUX_PRECISION_NVFP4 && !m->w4) {
    const int rc = quantize_block_weights_nvfp4(m, nullptr);
    if (rc) return rc;
  }
  m->precision = precision;
  return FLUX_OK;
}

int flux_dit_set_active_blocks(flux_dit* m, int n_double, int n_single) {
  if (!m) return fail(FLUX_EINVAL, "model is NULL");
  m->act_double = n_double < 0 ? m->cfg.n_double : std::min(n_double, m->cfg.n_double);
  m->act_single = n_single < 0 ? m->cfg.n_single : std::min(n_single, m->cfg.n_single);
  return FLUX_OK;
}

int flux_dit_prepare_timesteps(flux_dit* m, const float* ts, int n, void* stream) {
  if (!m) return fail(FLUX_EINVAL, "model is NULL");
  if (n < 0 || n > flux_dit::kMaxCachedT || (n > 0 && !ts))
    return fail(FLUX_EINVAL, "%d timesteps (0..%d, host array)", n, flux_dit::kMaxCachedT);
  for (int i = 0; i < n; ++i)
    if (!std::isfinite(ts[i])) return fail(FLUX_EINVAL, "timestep %d is not finite", i);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const flux_dit_config& c = m->cfg;
  const int D = c.hidden, tf = c.t_freq_dim;
  m->cache_n = 0;
  if (n == 0) return FLUX_OK;
  if (!m->mods_cache &&
      dev_alloc(&m->mods_cache, static_cast<size_t>(flux_dit::kMaxCachedT) * m->mods_rows * 4) != cudaSuccess)
    return fail(FLUX_ENOMEM, "device allocation of the modulation cache failed");
  // up to four timesteps per pass: the embeddings, the time MLP and every modulation linear read
  // their weights once for the group (the GEMV takes the group's vectors together)
  float* temb = nullptr;
  float* th = nullptr;
  float* vec = nullptr;
  const size_t scratch = 4 * (static_cast<size_t>(tf) + 2 * D);
  if (dev_alloc_async(&temb, scratch * sizeof(float), s) != cudaSuccess)
    return fail(FLUX_ENOMEM, "device allocation of the timestep scratch failed");
  th = temb + 4 * tf;
  vec = th + 4 * D;
  auto gv = [](double rows, double k, double nvec) { return rows * k * 2 + nvec * (rows * 6 + k * 4); };
  auto group = [&](int g, int k) -> int {
    for (int i = 0; i < k; ++i)
      FD_LAUNCH(m, kProfOther, 0, tf * 4.0, timestep_embed_launch(temb + i * tf, ts[g + i], tf, s));
    FD_LAUNCH(m, kProfGemv, 2.0 * k * D * tf, gv(D, tf, k),
              gemv_multi_launch(m->t_w1, m->t_b1, temb, k, th, nullptr, D, tf, 0, 1, s));
    FD_LAUNCH(m, kProfGemv, 2.0 * k * D * D, gv(D, D, k),
              gemv_multi_launch(m->t_w2, m->t_b2, th, k, vec, nullptr, D, D, 0, 0, s));
    FD_LAUNCH(m, kProfGemv, 2.0 * k * m->mods_rows * D, gv(static_cast<double>(m->mods_rows), D, k),
              gemv_multi_launch(m->mods_w, m->mods_b, vec, k, m->mods_cache + static_cast<size_t>(g) * m->mods_rows,
                                nullptr, static_cast<int>(m->mods_rows), D, 1, 0, s));
    return FLUX_OK;
  };
  int rc = FLUX_OK;
  for (int g = 0; g < n && rc == FLUX_OK; g += 4) rc = group(g, std::min(4, n - g));
  cudaFreeAsync(temb, s);
  if (rc) return rc;
  for (int i = 0; i < n; ++i) m->cache_t[i] = ts[i];
  m->cache_n = n;
  return FLUX_OK;
}

size_t flux_dit_modulation_size(const flux_dit* m) { return m ? m->mods_rows : 0; }

int flux_dit_modulation(flux_dit* m, float t, float* mods_out, void* stream) {
  if (!m || !mods_out) return fail(FLUX_EINVAL, "NULL argument");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int rc = run_modulation(m, t, s);
  if (rc) return rc;
  FD_CUDA(cudaMemcpyAsync(mods_out, m->mods_cur, m->mods_rows * sizeof(float), cudaMemcpyDeviceToDevice, s));
  return FLUX_OK;
}

int flux_euler_step(float* x, const float* v, size_t n, float dt, void* stream) {
  if (n && (!x || !v)) return fail(FLUX_EINVAL, "NULL argument");
  if (!aligned16(x) || !aligned16(v)) return fail(FLUX_EINVAL, "x and v must be 16-byte aligned");
  FD_CUDA(euler_launch(x, v, n, dt, static_cast<cudaStream_t>(stream)));
  return FLUX_OK;
}

int flux_pack_latents(const float* lat, float* tok, int h8, int w8, void* stream) {
  if (!lat || !tok) return fail(FLUX_EINVAL, "NULL argument");
  if (h8 < 2 || w8 < 2 || h8 % 2 || w8 % 2) return fail(FLUX_EINVAL, "latent %dx%d must be even and >= 2", h8, w8);
  if (!aligned16(lat) || !aligned16(tok)) return fail(FLUX_EINVAL, "lat and tok must be 16-byte aligned");
  FD_CUDA(pack_latents_launch(lat, tok, 32, h8, w8, static_cast<cudaStream_t>(stream)));
  return FLUX_OK;
}

int flux_unpack_latents(const float* tok, float* lat, int h8, int w8, void* stream) {
  if (!lat || !tok) return fail(FLUX_EINVAL, "NULL argument");
  if (h8 < 2 || w8 < 2 || h8 % 2 || w8 % 2) return fail(FLUX_EINVAL, "latent %dx%d must be even and >= 2", h8, w8);
  if (!aligned16(lat) || !aligned16(tok)) return fail(FLUX_EINVAL, "lat and tok must be 16-byte aligned");
  FD_CUDA(unpack_latents_launch(tok, lat, 32, h8, w8, static_cast<cudaStream_t>(stream)));
  return FLUX_OK;
}

int flux_joint_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* o, int n, int heads,
                         int head_dim, float scale, void* stream) {
  return flux_joint_attention_batch(q, k, v, o, 1, n, heads, head_dim, scale, stream);
}

int flux_joint_attention_batch(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* o, int batch,
                               int n, int heads, int head_dim, float scale, void* stream) {
  if (!q || !k || !v || !o) return fail(FLUX_EINVAL, "NULL argument");
  if (head_dim != 128) return fail(FLUX_EINVAL, "head_dim must be 128 (got %d)", head_dim);
  if (batch < 1 || batch > 65535) return fail(FLUX_EINVAL, "bad batch=%d", batch);
  if (n < 1 || heads < 1 || heads > 1024) return fail(FLUX_EINVAL, "bad n=%d heads=%d", n, heads);
  if (static_cast<long long>(batch) * n > (1ll << 31) - 1) return fail(FLUX_EINVAL, "batch * n too large");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return fail(FLUX_EINVAL, "q, k, v, o must be 16-byte aligned");
  if (!(scale > 0) || !std::isfinite(scale)) return fail(FLUX_EINVAL, "scale must be positive");
  AttnParams A;
  const uint64_t ld = static_cast<uint64_t>(heads) * 128;
  const size_t rows = static_cast<size_t>(batch) * n;
  if (!make_tmap_bf16(&A.mapQ, q, rows, ld, ld * 2, 128) || !make_tmap_bf16(&A.mapK, k, rows, ld, ld * 2, 128) ||
      !make_tmap_bf16(&A.mapV, v, rows, ld, ld * 2, 128))
    return fail(FLUX_EIO, "cuTensorMapEncodeTiled failed");
  A.out = reinterpret_cast<bf16*>(o);
  A.ldo = static_cast<int>(ld);
  A.n = n;
  A.heads = heads;
  A.batch = batch;
  A.q_col0 = A.k_col0 = A.v_col0 = 0;
  A.scale_log2 = static_cast<float>(scale * 1.4426950408889634);
  FD_CUDA(attention_launch(A, static_cast<cudaStream_t>(stream)));
  return FLUX_OK;
}

int flux_linear(const uint16_t* a, int m, int k, int lda, const uint16_t* w, int n, const uint16_t* bias, int mode,
                void* out, int ldo, const float* gate, void* stream) {
  if (!a || !w || !bias || !out) return fail(FLUX_EINVAL, "NULL argument");
  if (m < 1 || k < 64 || k % 64 || n < 32 || n % 32 || lda < k || lda % 8)
    return fail(FLUX_EINVAL, "bad shape m=%d k=%d n=%d lda=%d", m, k, n, lda);
  if (mode < 0 || mode > 3) return fail(FLUX_EINVAL, "bad mode %d", mode);
  if (mode == kEpiSwiGLU && n % 256) return fail(FLUX_EINVAL, "SwiGLU mode needs n %% 256 == 0");
  if (mode == kEpiResidGate && !gate) return fail(FLUX_EINVAL, "gate is NULL");
  const int out_cols = mode == kEpiSwiGLU ? n / 2 : n;
  if (ldo < out_cols || ldo % 8) return fail(FLUX_EINVAL, "bad ldo=%d", ldo);
  if (!aligned16(a) || !aligned16(w) || !aligned16(bias) || !aligned16(out) || (gate && !aligned16(gate)))
    return fail(FLUX_EINVAL, "pointers must be 16-byte aligned");
  const int bn = mode == kEpiSwiGLU ? 256 : gemm_bn_for(n);
  GemmParams P;
  P.num_problems = 1;
  if (!make_tmap_bf16(&P.mapA[0], a, m, k, static_cast<uint64_t>(lda) * 2, 128) ||
      !make_tmap_bf16(&P.mapB[0], w, n, k, static_cast<uint64_t>(k) * 2, 128))
    return fail(FLUX_EIO, "cuTensorMapEncodeTiled failed");
  GemmProblem& pr = P.prob[0];
  pr = GemmProblem();
  pr.M = m; pr.N = n; pr.K = k; pr.mode = mode; pr.out = out; pr.ldo = ldo;
  pr.bias = reinterpret_cast<const bf16*>(bias);
  pr.gate = gate;
  if (bn == 256)
    FD_CUDA(gemm2_launch(P, num_sms_current(), static_cast<cudaStream_t>(stream)));
  else
    FD_CUDA(gemm_launch(P, bn, num_sms_current(), static_cast<cudaStream_t>(stream)));
  return FLUX_OK;
}

int flux_quantize_rows_e4m3(const uint16_t* x, int rows, int cols, int ldx, uint8_t* q, int ldq, float* scale,
                            void* stream) {
  if (!x || !q || !scale) return fail(FLUX_EINVAL, "NULL argument");
  if (rows < 0 || cols < 8 || cols % 8 || cols > 16384 || ldx < cols || ldx % 8 || ldq < cols || ldq % 8)
    return fail(FLUX_EINVAL, "bad shape rows=%d cols=%d ldx=%d ldq=%d", rows, cols, ldx, ldq);
  if (!aligned16(x) || (reinterpret_cast<uintptr_t>(q) & 7) || (reinterpret_cast<uintptr_t>(scale) & 3))
    return fail(FLUX_EINVAL, "x must be 16-byte and q 8-byte aligned");
  FD_CUDA(quantize_rows_launch(reinterpret_cast<const bf16*>(x), ldx, rows, cols, q, ldq, scale,
                               static_cast<cudaStream_t>(stream)));
  return FLUX_OK;
}

int flux_layernorm_modulate_fp8(const float* x, uint8_t* q, float* q_scale, int rows, int dim, const float* shift,
                                const float* scale, float eps, void* stream) {
  if (!x || !q || !q_scale || !shift || !scale) return fail(FLUX_EINVAL, "NULL argument");
  if (rows < 0 || (dim != 1024 && dim != 2048 && dim != 3072 && dim != 4096))
    return fail(FLUX_EINVAL, "bad shape rows=%d dim=%d (dim in 1024, 2048, 3072, 4096)", rows, dim);
  if (!aligned16(x) || !aligned16(q) || !aligned16(shift) || !aligned16(scale))
    return fail(FLUX_EINVAL, "pointers must be 16-byte aligned");
  FD_CUDA(ln_modulate_fp8_launch(x, q, q_scale, rows, dim, rows, rows, rows, shift, scale, shift, scale, shift, scale,
                                 eps, static_cast<cudaStream_t>(stream)));
  return FLUX_OK;
}

int flux_linear_fp8(const uint8_t* a, const float* a_scale, int m, int k, int lda, const uint8_t* w,
                    const float* w_scale, int n, const uint16_t* bias, int mode, void* out, int ldo, const float* gate,
                    void* stream) {
  if (!a || !a_scale || !w || !w_scale || !bias || !out) return fail(FLUX_EINVAL, "NULL argument");
  if (m < 1 || k < 128 || k % 128 || n < 32 || n % 32 || lda < k || lda % 16)
    return fail(FLUX_EINVAL, "bad shape m=%d k=%d n=%d lda=%d (k %% 128, n %% 32, lda %% 16)", m, k, n, lda);
  if (mode < 0 || mode > 3) return fail(FLUX_EINVAL, "bad mode %d", mode);
  if (mode == kEpiSwiGLU && n % 256) return fail(FLUX_EINVAL, "SwiGLU mode needs n %% 256 == 0");
  if (mode == kEpiResidGate && !gate) return fail(FLUX_EINVAL, "gate is NULL");
  const int out_cols = mode == kEpiSwiGLU ? n / 2 : n;
  if (ldo < out_cols || ldo % 8) return fail(FLUX_EINVAL, "bad ldo=%d", ldo);
  if (!aligned16(a) || !aligned16(w) || !aligned16(bias) || !aligned16(out) || !aligned16(a_scale) ||
      !aligned16(w_scale) || (gate && !aligned16(gate)))
    return fail(FLUX_EINVAL, "pointers must be 16-byte aligned");
  GemmParams P;
  P.num_problems = 1;
  if (!make_tmap_u8(&P.mapA[0], a, m, k, static_cast<uint64_t>(lda), 128) ||
      !make_tmap_u8(&P.mapB[0], w, n, k, static_cast<uint64_t>(k), 128))
    return fail(FLUX_EIO, "cuTensorMapEncodeTiled failed");
  problem(P, 0, P.mapA[0], P.mapB[0], m, n, k, mode, out, ldo, reinterpret_cast<const bf16*>(bias), gate);
  P.prob[0].scale_a = a_scale;
  P.prob[0].scale_b = w_scale;
  FD_CUDA(gemm2_launch(P, num_sms_current(), static_cast<cudaStream_t>(stream), true));
  return FLUX_OK;
}

size_t flux_nvfp4_scale_bytes(int rows, int k) {
  if (rows < 0 || k < 64 || k % 64) return 0;
  return nvfp4_scale_bytes(static_cast<size_t>(rows), static_cast<size_t>(k));
}

int flux_quantize_rows_nvfp4(const uint16_t* x, int rows, int k, int ldx, uint8_t* q, int ldq, uint8_t* sf,
                             float* row_scale, void* stream) {
  if (!x || !q || !sf || !row_scale) return fail(FLUX_EINVAL, "NULL argument");
  if (rows < 0 || k < 64 || k % 64 || k > 16384 || ldx < k || ldx % 8 || ldq < k / 2 || ldq % 16)
    return fail(FLUX_EINVAL, "bad shape rows=%d k=%d ldx=%d ldq=%d (k %% 64, k <= 16384, ldx %% 8, ldq %% 16)", rows,
                k, ldx, ldq);
  if (!aligned16(x) || !aligned16(q) || !aligned16(sf) || !aligned16(row_scale))
    return fail(FLUX_EINVAL, "pointers must be 16-byte aligned");
  const int r0 = 0;
  FD_CUDA(quantize_nvfp4_launch(reinterpret_cast<const bf16*>(x), ldx, k, q, ldq, sf, row_scale,
                                q4_segments(&r0, &rows, 1), static_cast<cudaStream_t>(stream)));
  return FLUX_OK;
}

int flux_layernorm_modulate_nvfp4(const float* x, uint8_t* q, uint8_t* sf, float* row_scale, int rows, int dim,
                                  const float* shift, const float* scale, float eps, void* stream) {
  if (!x || !q || !sf || !row_scale || !shift || !scale) return fail(FLUX_EINVAL, "NULL argument");
  if (rows < 0 || (dim != 1024 && dim != 2048 && dim != 3072 && dim != 4096))
    return fail(FLUX_EINVAL, "bad shape rows=%d dim=%d (dim in {1024, 2048, 3072, 4096})", rows, dim);
  if (!aligned16(x) || !aligned16(q) || !aligned16(sf) || !aligned16(row_scale) || !aligned16(shift) ||
      !aligned16(scale))
    return fail(FLUX_EINVAL, "pointers must be 16-byte aligned");
  const int r0 = 0;
  const LnModSets ms{rows, rows, rows > 0 ? rows : 1, shift, shift, shift, scale, scale, scale};
  FD_CUDA(ln_modulate_nvfp4_launch(x, dim, q, sf, row_scale, q4_segments(&r0, &rows, 1), ms, eps,
                                   static_cast<cudaStream_t>(stream)));
  return FLUX_OK;
}

int flux_linear_nvfp4(const uint8_t* a, const uint8_t* a_sf, const float* a_scale, int m, int k, int lda,
                      const uint8_t* w, const uint8_t* w_sf, const float* w_scale, int n, const uint16_t* bias,
                      int mode, void* out, int ldo, const float* gate, void* stream) {
  if (!a || !a_sf || !a_scale || !w || !w_sf || !w_scale || !bias || !out) return fail(FLUX_EINVAL, "NULL argument");
  if (m < 1 || k < 256 || k % 256 || n < 32 || n % 32 || lda < k / 2 || lda % 16)
    return fail(FLUX_EINVAL, "bad shape m=%d k=%d n=%d lda=%d (k %% 256, n %% 32, lda %% 16 bytes)", m, k, n, lda);
  if (mode < 0 || mode > 3) return fail(FLUX_EINVAL, "bad mode %d", mode);
  if (mode == kEpiSwiGLU && n % 256) return fail(FLUX_EINVAL, "SwiGLU mode needs n %% 256 == 0");
  if (mode == kEpiResidGate && !gate) return fail(FLUX_EINVAL, "gate is NULL");
  const int out_cols = mode == kEpiSwiGLU ? n / 2 : n;
  if (ldo < out_cols || ldo % 8) return fail(FLUX_EINVAL, "bad ldo=%d", ldo);
  if (!aligned16(a) || !aligned16(w) || !aligned16(a_sf) || !aligned16(w_sf) || !aligned16(bias) || !aligned16(out) ||
      !aligned16(a_scale) || !aligned16(w_scale) || (gate && !aligned16(gate)))
    return fail(FLUX_EINVAL, "pointers must be 16-byte aligned");
  GemmParams4 P4;
  GemmParams& P = P4.g;
  P.num_problems = 1;
  if (!make_tmap_u8(&P.mapA[0], a, m, k / 2, static_cast<uint64_t>(lda), 128) ||
      !make_tmap_u8(&P.mapB[0], w, n, k / 2, static_cast<uint64_t>(k / 2), 128) ||
      !make_tmap_sf(&P4.mapSFA[0], a_sf, nvfp4_scale_bytes(m, k)) ||
      !make_tmap_sf(&P4.mapSFB[0], w_sf, nvfp4_scale_bytes(n, k)))
    return fail(FLUX_EIO, "cuTensorMapEncodeTiled failed");
  problem(P, 0, P.mapA[0], P.mapB[0], m, n, k, mode, out, ldo, reinterpret_cast<const bf16*>(bias), gate);
  P.prob[0].scale_a = a_scale;
  P.prob[0].scale_b = w_scale;
  FD_CUDA(gemm_fp4_launch(P4, num_sms_current(), static_cast<cudaStream_t>(stream)));
  return FLUX_OK;
}

int flux_qkv_projection(const uint16_t* a, int m, int k, int lda, const uint16_t* w, const uint16_t* bias, int heads,
                        const uint16_t* q_gain, const uint16_t* k_gain, const float* table, int table_row0, float eps,
                        uint16_t* qkv, void* stream) {
  if (!a || !w || !bias || !q_gain || !k_gain || !table || !qkv) return fail(FLUX_EINVAL, "NULL argument");
  if (m < 1 || k < 64 || k % 64 || lda < k || lda % 8 || heads < 1 || heads % 2 || table_row0 < 0)
    return fail(FLUX_EINVAL, "bad shape m=%d k=%d lda=%d heads=%d (heads must be even)", m, k, lda, heads);
  if (!aligned16(a) || !aligned16(w) || !aligned16(bias) || !aligned16(q_gain) || !aligned16(k_gain) ||
      !aligned16(table) || !aligned16(qkv))
    return fail(FLUX_EINVAL, "pointers must be 16-byte aligned");
  const int n = 3 * heads * 128;
  GemmParams P;
  P.num_problems = 1;
  if (!make_tmap_bf16(&P.mapA[0], a, m, k, static_cast<uint64_t>(lda) * 2, 128) ||
      !make_tmap_bf16(&P.mapB[0], w, n, k, static_cast<uint64_t>(k) * 2, 128))
    return fail(FLUX_EIO, "cuTensorMapEncodeTiled failed");
  problem(P, 0, P.mapA[0], P.mapB[0], m, n, k, kEpiBf16Bias, qkv, n, reinterpret_cast<const bf16*>(bias), nullptr);
  qk_fuse(P, 0, reinterpret_cast<const bf16*>(q_gain), reinterpret_cast<const bf16*>(k_gain),
          reinterpret_cast<const float2*>(table), table_row0, eps);
  FD_CUDA(gemm2_launch(P, num_sms_current(), static_cast<cudaStream_t>(stream)));
  return FLUX_OK;
}

int flux_layernorm_modulate(const float* x, uint16_t* y, int rows, int dim, const float* shift, const float* scale,
                            float eps, void* stream) {
  if (!x || !y || !shift || !scale) return fail(FLUX_EINVAL, "NULL argument");
  if (rows < 0 || dim < 4 || dim % 4) return fail(FLUX_EINVAL, "bad shape rows=%d dim=%d", rows, dim);
  if (!aligned16(x) || !aligned16(y) || !aligned16(shift) || !aligned16(scale))
    return fail(FLUX_EINVAL, "pointers must be 16-byte aligned");
  FD_CUDA(ln_modulate_launch(x, reinterpret_cast<bf16*>(y), rows, dim, rows, rows, shift, scale, shift, scale, eps,
                             static_cast<cudaStream_t>(stream)));
  return FLUX_OK;
}

int flux_rope_table(float* table, int n_txt, int gh, int gw, int rh, int rw, float theta, void* stream) {
  if (!table) return fail(FLUX_EINVAL, "NULL argument");
  if (n_txt < 0 || gh < 0 || gw < 0 || rh < 0 || rw < 0 || !(theta > 0))
    return fail(FLUX_EINVAL, "bad arguments");
  const RefGrids refs = {rh > 0 && rw > 0 ? 1 : 0, {rh}, {rw}};
  FD_CUDA(rope_table_launch(reinterpret_cast<float2*>(table), n_txt, gh, gw, refs, theta,
                            static_cast<cudaStream_t>(stream)));
  return FLUX_OK;
}

int flux_qk_rmsnorm_rope(uint16_t* qkv, int rows, int ld, int k_col, int heads, const uint16_t* q_gain,
                         const uint16_t* k_gain, const float* table, float eps, void* stream) {
  if (!qkv || !q_gain || !k_gain || !table) return fail(FLUX_EINVAL, "NULL argument");
  if (rows < 0 || heads < 1 || ld % 8 || k_col % 8 || ld < heads * 128 || k_col + heads * 128 > ld)
    return fail(FLUX_EINVAL, "bad shape rows=%d ld=%d k_col=%d heads=%d", rows, ld, k_col, heads);
  if (!aligned16(qkv) || !aligned16(q_gain) || !aligned16(k_gain) || !aligned16(table))
    return fail(FLUX_EINVAL, "pointers must be 16-byte aligned");
  const bf16* gq = reinterpret_cast<const bf16*>(q_gain);
  const bf16* gk = reinterpret_cast<const bf16*>(k_gain);
  FD_CUDA(qk_norm_rope_launch(reinterpret_cast<bf16*>(qkv), rows, ld, k_col, heads, rows, gq, gk, gq, gk,
                              reinterpret_cast<const float2*>(table), eps, static_cast<cudaStream_t>(stream)));
  return FLUX_OK;
}

int flux_dit_profile(flux_dit* m, int enable) {
  if (!m) return fail(FLUX_EINVAL, "model is NULL");
  FD_CUDA(cudaDeviceSynchronize());
  m->prof.reset();
  m->prof.on = enable != 0;
  return FLUX_OK;
}

int flux_dit_profile_read(flux_dit* m, int kind, double* ms, double* flops, double* bytes, long long* launches) {
  if (!m || kind < 0 || kind >= kProfKinds) return fail(FLUX_EINVAL, "bad model or kernel kind");
  FD_CUDA(cudaDeviceSynchronize());
  m->prof.settle();
  if (ms) *ms = m->prof.ms[kind];
  if (flops) *flops = m->prof.flops[kind];
  if (bytes) *bytes = m->prof.bytes[kind];
  if (launches) *launches = m->prof.launches[kind];
  return FLUX_OK;
}

unsigned long long flux_kernel_launches(void) { return g_launches.load(); }

void flux_test_fail_alloc_after(long long n) { g_fail_alloc_after.store(n < 0 ? -1 : n); }

int flux_device_error(void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  FD_CUDA(cudaStreamSynchronize(s));
  return device_error_words(s);
}

}  // extern "C"
