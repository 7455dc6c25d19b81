// FLUX.3 Image Klein denoising transformer on B200: host runner and C ABI.
//
// The same sm_100a kernels as the FLUX.2-klein runner, arranged into the FLUX.3 block
// structure ("FLUX.3 Image Klein in Diffusers: Architektur, Layout-Steuerung und
// Systemanforderungen im Überblick", mindverse):
//   * "Zweistufiger Transformer und Tokenisierung": text features are 8 encoder layers of
//     2560 values (20480 per token) projected to the width 3072 by one linear layer;
//   * "Entkoppelte Vorverarbeitung und gemeinsame Attention-Blöcke": 5 per-mode blocks in which
//     the text, noisy-image and reference streams have their own weights and attend only to
//     themselves, then 28 joint blocks with one weight set over text | image | reference; every
//     block runs attention and the SwiGLU MLP in parallel on one normalised input;
//   * "Modulation pro Token-Typ, Flow-Map-Destillation und 4D-RoPE": image tokens are
//     modulated with the current t, text and reference tokens with t = 0; the time-distilled
//     checkpoint adds an embedding of the step's target time to every token's conditioning.
//
// Forward (one CUDA stream, no host synchronisation):
//   time vectors: vec_img = MLP_time(emb(t)) (+ MLP_target(emb(t_target))),
//                 vec_ctx = MLP_time(emb(0)) (+ the same target term)
//   modulation GEMVs: per-mode linears (text and reference from vec_ctx, image from vec_img),
//                 the joint linear on both vectors at once, the output layer's from vec_img
//   txt_in (K = 20480) / img_in projections (one grouped GEMM) into the fp32 residual X
//   5 x per-mode block: LN+mod (three row ranges, three modulation sets)
//        -> linear1 GEMM, 6 problems (qkv with fused QK-RMSNorm + RoPE, SwiGLU; per stream)
//        -> attention over three independent segments (one launch)
//        -> linear2 GEMM, 3 problems (per-stream weights and gates) + gate * residual
//   28 x joint block: LN+mod (image rows: the t set; text and reference rows: the t = 0 set)
//        -> linear1 GEMM (qkv | SwiGLU over all rows) -> joint attention
//        -> linear2 GEMM, 3 row-range problems sharing W, each with its token type's gate
//   final LN+mod on the image rows -> output GEMM -> velocity (fp32)
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <string>
#include <vector>

#include "../../include/fluxdit.h"
#include "fluxdit_internal.h"
#include "runner.h"

namespace fdit {
namespace {

constexpr size_t kHeaderBytes = 256;

struct BlobTensor3 {
  std::string name;
  size_t rows, cols;     // cols = 1 for vectors
  size_t off;            // byte offset in the blob
};

bool valid_cfg3(const flux3_dit_config& c) {
  return c.n_mode >= 0 && c.n_joint >= 0 && c.n_mode + c.n_joint >= 1 && c.head_dim == 128 && c.heads >= 2 &&
         c.heads % 2 == 0 && c.hidden == c.heads * c.head_dim && c.mlp_hidden > 0 && c.mlp_hidden % 128 == 0 &&
         c.in_ch == 128 && c.txt_dim > 0 && c.txt_dim % 64 == 0 && c.t_freq_dim > 0 && c.t_freq_dim % 64 == 0 &&
         c.t_freq_dim <= 6144 && c.hidden <= 6144 && (c.flow_map == 0 || c.flow_map == 1) && c.rope_theta > 0 &&
         c.eps_ln > 0 && c.eps_rms > 0;
}

const char* kStreams[3] = {"txt", "img", "ref"};

// Tensor order of the FLUX.3 blob (documented in fluxdit.h).
std::vector<BlobTensor3> blob_tensors3(const flux3_dit_config& c, size_t* total) {
  const size_t D = c.hidden, F = c.mlp_hidden, hd = c.head_dim;
  std::vector<BlobTensor3> t;
  auto add = [&](const std::string& n, size_t r, size_t k) { t.push_back({n, r, k, 0}); };
  auto block = [&](const std::string& p) {
    add(p + "lin1.w", 3 * D + 2 * F, D); add(p + "lin1.b", 3 * D + 2 * F, 1);
    add(p + "q_gain", hd, 1); add(p + "k_gain", hd, 1);
    add(p + "lin2.w", D, D + F); add(p + "lin2.b", D, 1);
  };
  add("time_in.w1", D, c.t_freq_dim); add("time_in.b1", D, 1);
  add("time_in.w2", D, D); add("time_in.b2", D, 1);
  if (c.flow_map) {
    add("target_in.w1", D, c.t_freq_dim); add("target_in.b1", D, 1);
    add("target_in.w2", D, D); add("target_in.b2", D, 1);
  }
  add("img_in.w", D, c.in_ch); add("img_in.b", D, 1);
  add("txt_in.w", D, c.txt_dim); add("txt_in.b", D, 1);
  for (const char* s : kStreams) {
    add(std::string("mode_mod.") + s + ".w", 3 * D, D);
    add(std::string("mode_mod.") + s + ".b", 3 * D, 1);
  }
  for (int i = 0; i < c.n_mode; ++i)
    for (const char* s : kStreams) block("mode." + std::to_string(i) + "." + s + ".");
  add("joint_mod.w", 3 * D, D); add("joint_mod.b", 3 * D, 1);
  for (int i = 0; i < c.n_joint; ++i) block("joint." + std::to_string(i) + ".");
  add("final.mod.w", 2 * D, D); add("final.mod.b", 2 * D, 1);
  add("final.out.w", c.in_ch, D); add("final.out.b", c.in_ch, 1);
  size_t off = kHeaderBytes;
  for (auto& x : t) {
    x.off = off;
    off = (off + x.rows * x.cols * 2 + 255) / 256 * 256;
  }
  *total = off;
  return t;
}

// Header fields at their byte offsets (little endian, no padding):
// magic[8] | u32 version | u32 n_tensors | i32 x 10 | f32 x 3 | u64 data_offset | u64 data_bytes
struct Header3 {
  uint32_t version, n_tensors;
  flux3_dit_config cfg;
  uint64_t data_offset, data_bytes;
};

bool read_header3(const void* blob, size_t bytes, Header3* h) {
  if (!blob || bytes < kHeaderBytes) return false;
  const uint8_t* b = static_cast<const uint8_t*>(blob);
  if (memcmp(b, "FLUX3DT\0", 8) != 0) return false;
  int32_t iv[10];
  float fv[3];
  memcpy(&h->version, b + 8, 4);
  memcpy(&h->n_tensors, b + 12, 4);
  memcpy(iv, b + 16, 40);
  memcpy(fv, b + 56, 12);
  memcpy(&h->data_offset, b + 68, 8);
  memcpy(&h->data_bytes, b + 76, 8);
  h->cfg = {iv[0], iv[1], iv[2], iv[3], iv[4], iv[5], iv[6], iv[7], iv[8], iv[9], fv[0], fv[1], fv[2]};
  return true;
}

// One parallel block's weights (per-mode stream or joint block).
struct BlockW3 {
  const bf16 *qkv_b, *mlp_b, *q_gain, *k_gain, *lin2_b;
  const bf16 *w_lin1, *w_lin2;
  CUtensorMap m_qkv, m_mlp, m_lin2;
  // FP8 precision: e4m3 codes of linear1 (qkv rows, SwiGLU rows) and linear2, row scales
  CUtensorMap m8_qkv, m8_mlp, m8_lin2;
  const float *s_qkv, *s_mlp, *s_lin2;
  // NVFP4 precision: codes, block scales and row scales of the same matrices
  Fp4Op q4_qkv, q4_mlp, q4_lin2;
};

// Row ranges of the joint sequence: text | image | reference (all references together).
enum Seg { kSegTxt = 0, kSegImg = 1, kSegRef = 2 };

// A forward evaluates up to two sequences that share the image, the references and t and differ
// in their text (classifier-free guidance); sequence b occupies rows [b n, (b + 1) n).
constexpr int kMaxBatch3 = 2;

struct Workspace3 {
  size_t cap_n = 0, cap_tok = 0, cap_txt = 0;
  float* X = nullptr;
  bf16 *Y = nullptr, *QKV = nullptr, *CC = nullptr, *tokb = nullptr, *txtb = nullptr;
  float2* rope = nullptr;        // one sequence's positions (every sequence has the same)
  int nt = -1, gh = -1, gw = -1, nb = -1;
  RefGrids refs = {-1, {}, {}};
  CUtensorMap a_tokb, qkv;
  CUtensorMap a_txtb[kMaxBatch3], a_Yall[kMaxBatch3], a_Yout[kMaxBatch3];
  CUtensorMap a_Yseg[kMaxBatch3][3], a_CCseg[kMaxBatch3][3];
  // FP8 precision: e4m3 LN-mod output (Y8, scale sY) and [O | H] (C8, scale sC per row)
  size_t cap8 = 0;
  uint8_t *Y8 = nullptr, *C8 = nullptr;
  float *sY = nullptr, *sC = nullptr;
  bool maps8 = false;
  CUtensorMap a8_Yall[kMaxBatch3], a8_Yseg[kMaxBatch3][3], a8_CCseg[kMaxBatch3][3];
  // NVFP4 precision: codes of the LN-mod output (Y4) and of [O | H] (C4), block scales (sfY, sfC)
  // and row scales.  Each GEMM problem's rows start on a 128-row block of its scales, so the
  // quantisations follow the problems: per stream segment in the per-mode blocks (seg_pm: text,
  // image, reference of sequence 0, then the other sequences' text), per sequence for the joint
  // linear1 (seg_jy) and per token type and sequence for the joint linear2 (seg_jc).
  size_t cap4_rows = 0, cap4_blocks = 0;
  uint8_t *Y4 = nullptr, *C4 = nullptr, *sfY = nullptr, *sfC = nullptr;
  float *sY4 = nullptr, *sC4 = nullptr;
  bool maps4 = false;
  Q4Segs seg_pm, seg_jy, seg_jc;
  Fp4Op y4_pm[kMaxBatch3][3], c4_pm[kMaxBatch3][3], y4_all[kMaxBatch3], c4_seg[kMaxBatch3][3];
};

// Offsets (in units of D floats) of the modulation vectors in the model's mods buffer.
constexpr int kModTxt = 0, kModImg = 3, kModRef = 6, kModJointImg = 9, kModJointCtx = 12, kModFinal = 15,
              kModRowsD = 17;

}  // namespace
}  // namespace fdit

using fdit::bf16;

struct flux3_dit {
  flux3_dit_config cfg;
  int device = 0, num_sms = 148;
  void* wbuf = nullptr;
  float* scratch = nullptr;      // temb [3][t_freq] | th [3][D] | tt [D] | vec [2][D] | mods [17 D]
  float *temb = nullptr, *th = nullptr, *tt = nullptr, *vec = nullptr, *mods = nullptr;
  const bf16 *t_w1, *t_b1, *t_w2, *t_b2, *g_w1 = nullptr, *g_b1 = nullptr, *g_w2 = nullptr, *g_b2 = nullptr;
  const bf16 *img_b, *txt_b, *fin_b;
  const bf16 *mode_mod_w[3], *mode_mod_b[3], *joint_mod_w, *joint_mod_b, *fin_mod_w, *fin_mod_b;
  CUtensorMap m_img_in, m_txt_in, m_fin;
  std::vector<fdit::BlockW3> mode;    // [3 i + stream], stream 0 text, 1 image, 2 reference
  std::vector<fdit::BlockW3> joint;
  int act_mode = 0, act_joint = 0;
  int precision = FLUX_PRECISION_BF16;
  uint8_t* w8 = nullptr;               // e4m3 block linears (allocated on the first switch to FP8)
  float* w8_scale = nullptr;
  uint8_t* w4 = nullptr;               // NVFP4 block linears (first switch to NVFP4)
  float* w4_scale = nullptr;
  fdit::Workspace3 ws;
  fdit::Profiler prof;
};

namespace fdit {
namespace {

void free_ws3_fp8(Workspace3& w) {
  cudaFree(w.Y8); cudaFree(w.C8); cudaFree(w.sY); cudaFree(w.sC);
  w.Y8 = w.C8 = nullptr;
  w.sY = w.sC = nullptr;
  w.cap8 = 0;
  w.maps8 = false;
}

void free_ws3_fp4(Workspace3& w) {
  cudaFree(w.Y4); cudaFree(w.C4); cudaFree(w.sfY); cudaFree(w.sfC); cudaFree(w.sY4); cudaFree(w.sC4);
  w.Y4 = w.C4 = w.sfY = w.sfC = nullptr;
  w.sY4 = w.sC4 = nullptr;
  w.cap4_rows = w.cap4_blocks = 0;
  w.maps4 = false;
}

void free_ws3(Workspace3& w) {
  free_ws3_fp8(w);
  free_ws3_fp4(w);
  cudaFree(w.X); cudaFree(w.Y); cudaFree(w.QKV); cudaFree(w.CC); cudaFree(w.tokb); cudaFree(w.txtb);
  cudaFree(w.rope);
  w = Workspace3();
}

void destroy3(flux3_dit* m) {
  if (!m) return;
  free_ws3(m->ws);
  cudaFree(m->w8);
  cudaFree(m->w8_scale);
  cudaFree(m->w4);
  cudaFree(m->w4_scale);
  cudaFree(m->wbuf);
  cudaFree(m->scratch);
  delete m;
}

int create3_impl(const void* blob, size_t blob_bytes, const flux3_dit_config* cfg_in, cudaStream_t s,
                 flux3_dit** out) {
  *out = nullptr;
  Header3 h;
  if (!read_header3(blob, blob_bytes, &h) || h.version != 1 || h.data_offset != kHeaderBytes)
    return fail(FLUX_EINVAL, "not a FLUX3DT v1 blob");
  const flux3_dit_config c = h.cfg;
  if (cfg_in && memcmp(cfg_in, &c, sizeof(c)) != 0) return fail(FLUX_EINVAL, "config differs from the blob header");
  if (!valid_cfg3(c)) return fail(FLUX_EINVAL, "unsupported FLUX.3 model config in blob header");
  size_t total = 0;
  const std::vector<BlobTensor3> ts = blob_tensors3(c, &total);
  if (h.n_tensors != ts.size() || h.data_bytes + kHeaderBytes != total || blob_bytes < total)
    return fail(FLUX_EINVAL, "blob size / tensor count mismatch (expected %zu bytes, %zu tensors)", total, ts.size());

  flux3_dit* m = new flux3_dit();
  m->cfg = c;
  cudaGetDevice(&m->device);
  m->num_sms = num_sms_current();
  const size_t D = c.hidden, F = c.mlp_hidden;
  auto cleanup = [&](int code, const char* what) {
    destroy3(m);
    return fail(code, "%s", what);
  };
  // device copy: the blob's tensor area as is (same offsets), SwiGLU rows of linear1 re-interleaved
  const size_t scratch_floats = 3 * c.t_freq_dim + 3 * D + D + 2 * D + kModRowsD * D;
  if (dev_alloc(&m->wbuf, total - kHeaderBytes) != cudaSuccess ||
      dev_alloc(&m->scratch, scratch_floats * sizeof(float)) != cudaSuccess)
    return cleanup(FLUX_ENOMEM, "device allocation of the model weights failed");
  m->temb = m->scratch;
  m->th = m->temb + 3 * c.t_freq_dim;
  m->tt = m->th + 3 * D;
  m->vec = m->tt + D;
  m->mods = m->vec + 2 * D;
  uint8_t* wb = static_cast<uint8_t*>(m->wbuf);
  const uint8_t* b8 = static_cast<const uint8_t*>(blob);
  for (const BlobTensor3& t : ts) {
    uint8_t* dst = wb + (t.off - kHeaderBytes);
    const uint8_t* src = b8 + t.off;
    cudaError_t e;
    if (t.name.find("lin1.") != std::string::npos) {
      const size_t qkv_bytes = 3 * D * t.cols * 2;
      e = cudaMemcpyAsync(dst, src, qkv_bytes, cudaMemcpyHostToDevice, s);
      if (e == cudaSuccess) e = copy_swiglu(dst + qkv_bytes, src + qkv_bytes, F, t.cols * 2, s);
    } else {
      e = cudaMemcpyAsync(dst, src, t.rows * t.cols * 2, cudaMemcpyHostToDevice, s);
    }
    if (e != cudaSuccess) return cleanup(FLUX_EIO, "weight upload failed");
  }

  auto W = [&](const std::string& n) -> const bf16* {
    for (const BlobTensor3& t : ts)
      if (t.name == n) return reinterpret_cast<const bf16*>(wb + (t.off - kHeaderBytes));
    return nullptr;
  };
  bool maps_ok = true;
  auto wmap = [&](CUtensorMap* map, const bf16* base, size_t rows, size_t cols) {
    maps_ok &= make_tmap_bf16(map, base, rows, cols, cols * 2, 128);
  };
  m->t_w1 = W("time_in.w1"); m->t_b1 = W("time_in.b1"); m->t_w2 = W("time_in.w2"); m->t_b2 = W("time_in.b2");
  if (c.flow_map) {
    m->g_w1 = W("target_in.w1"); m->g_b1 = W("target_in.b1");
    m->g_w2 = W("target_in.w2"); m->g_b2 = W("target_in.b2");
  }
  m->img_b = W("img_in.b"); m->txt_b = W("txt_in.b"); m->fin_b = W("final.out.b");
  wmap(&m->m_img_in, W("img_in.w"), D, c.in_ch);
  wmap(&m->m_txt_in, W("txt_in.w"), D, c.txt_dim);
  wmap(&m->m_fin, W("final.out.w"), c.in_ch, D);
  for (int sidx = 0; sidx < 3; ++sidx) {
    m->mode_mod_w[sidx] = W(std::string("mode_mod.") + kStreams[sidx] + ".w");
    m->mode_mod_b[sidx] = W(std::string("mode_mod.") + kStreams[sidx] + ".b");
  }
  m->joint_mod_w = W("joint_mod.w"); m->joint_mod_b = W("joint_mod.b");
  m->fin_mod_w = W("final.mod.w"); m->fin_mod_b = W("final.mod.b");
  auto block = [&](BlockW3& bw, const std::string& p) {
    const bf16* l1 = W(p + "lin1.w");
    const bf16* l1b = W(p + "lin1.b");
    bw.w_lin1 = l1; bw.w_lin2 = W(p + "lin2.w");
    bw.qkv_b = l1b; bw.mlp_b = l1b + 3 * D;
    bw.q_gain = W(p + "q_gain"); bw.k_gain = W(p + "k_gain"); bw.lin2_b = W(p + "lin2.b");
    wmap(&bw.m_qkv, l1, 3 * D, D);
    wmap(&bw.m_mlp, l1 + 3 * D * D, 2 * F, D);
    wmap(&bw.m_lin2, W(p + "lin2.w"), D, D + F);
  };
  m->mode.resize(3 * c.n_mode);
  for (int i = 0; i < c.n_mode; ++i)
    for (int sidx = 0; sidx < 3; ++sidx)
      block(m->mode[3 * i + sidx], "mode." + std::to_string(i) + "." + kStreams[sidx] + ".");
  m->joint.resize(c.n_joint);
  for (int i = 0; i < c.n_joint; ++i) block(m->joint[i], "joint." + std::to_string(i) + ".");
  if (!maps_ok) return cleanup(FLUX_EIO, "cuTensorMapEncodeTiled failed for a weight tensor");
  m->act_mode = c.n_mode;
  m->act_joint = c.n_joint;
  if (cudaStreamSynchronize(s) != cudaSuccess) return cleanup(FLUX_EIO, "weight upload failed (sync)");
  *out = m;
  return FLUX_OK;
}

// FP8 copies of the GEMM A operands (LN-mod output and [O | H]) and their maps.
int prepare3_fp8(flux3_dit* m, int nt, int ni, int nr, int nb) {
  Workspace3& w = m->ws;
  const flux3_dit_config& c = m->cfg;
  const size_t D = c.hidden, F = c.mlp_hidden;
  const size_t n = static_cast<size_t>(nt) + ni + nr, rows = n * nb;
  if (rows > w.cap8) {
    free_ws3_fp8(w);
    const bool ok = dev_alloc(&w.Y8, rows * D) == cudaSuccess &&
                    dev_alloc(&w.C8, rows * (D + F)) == cudaSuccess && dev_alloc(&w.sY, rows * 4) == cudaSuccess &&
                    dev_alloc(&w.sC, rows * 4) == cudaSuccess;
    if (!ok) {
      free_ws3_fp8(w);
      return fail(FLUX_ENOMEM, "FP8 workspace allocation for %zu tokens failed", rows);
    }
    w.cap8 = rows;
  }
  if (w.maps8) return FLUX_OK;
  bool ok = true;
  auto amap = [&](CUtensorMap* map, const uint8_t* base, size_t r, size_t cols, uint64_t stride) {
    if (r == 0) {
      memset(map, 0, sizeof(*map));
      return;
    }
    ok &= make_tmap_u8(map, base, r, cols, stride, 128);
  };
  const size_t row0[3] = {0, static_cast<size_t>(nt), static_cast<size_t>(nt) + ni};
  const size_t seg[3] = {static_cast<size_t>(nt), static_cast<size_t>(ni), static_cast<size_t>(nr)};
  for (int bb = 0; bb < nb; ++bb) {
    const size_t r0 = bb * n;
    amap(&w.a8_Yall[bb], w.Y8 + r0 * D, n, D, D);
    for (int sg = 0; sg < 3; ++sg) {
      amap(&w.a8_Yseg[bb][sg], w.Y8 + (r0 + row0[sg]) * D, seg[sg], D, D);
      amap(&w.a8_CCseg[bb][sg], w.C8 + (r0 + row0[sg]) * (D + F), seg[sg], D + F, D + F);
    }
  }
  if (!ok) return fail(FLUX_EIO, "cuTensorMapEncodeTiled failed for an FP8 activation buffer");
  w.maps8 = true;
  return FLUX_OK;
}

// NVFP4 copies of the GEMM A operands and their maps for nb sequences of nt + ni + nr rows.
int prepare3_fp4(flux3_dit* m, int nt, int ni, int nr, int nb) {
  Workspace3& w = m->ws;
  const flux3_dit_config& c = m->cfg;
  const size_t D = c.hidden, F = c.mlp_hidden;
  const int n = nt + ni + nr, rows = n * nb;
  const int row0[3] = {0, nt, nt + ni}, seg[3] = {nt, ni, nr};
  int r0[2 * kMaxBatch3 * 3], rs[2 * kMaxBatch3 * 3], nz = 0;
  for (int sg = 0; sg < 3; ++sg, ++nz) {               // per-mode: sequence 0's streams, the others' text
    r0[nz] = row0[sg];
    rs[nz] = seg[sg];
  }
  for (int bb = 1; bb < nb; ++bb, ++nz) {
    r0[nz] = bb * n;
    rs[nz] = nt;
  }
  w.seg_pm = q4_segments(r0, rs, nz);
  for (int bb = 0; bb < nb; ++bb) {
    r0[bb] = bb * n;
    rs[bb] = n;
  }
  w.seg_jy = q4_segments(r0, rs, nb);
  for (int bb = 0; bb < nb; ++bb)
    for (int sg = 0; sg < 3; ++sg) {
      r0[3 * bb + sg] = bb * n + row0[sg];
      rs[3 * bb + sg] = seg[sg];
    }
  w.seg_jc = q4_segments(r0, rs, 3 * nb);
  auto blocks_of = [](const Q4Segs& g) {
    size_t b = 0;
    for (int z = 0; z < g.n; ++z) b += (g.rows[z] + 127) / 128;
    return b;
  };
  const size_t blocks = std::max(blocks_of(w.seg_pm), std::max(blocks_of(w.seg_jy), blocks_of(w.seg_jc)));
  if (static_cast<size_t>(rows) > w.cap4_rows || blocks > w.cap4_blocks) {
    free_ws3_fp4(w);
    const size_t R = rows, B = blocks * 128;
    const bool ok = dev_alloc(&w.Y4, R * D / 2) == cudaSuccess && dev_alloc(&w.C4, R * (D + F) / 2) == cudaSuccess &&
                    dev_alloc(&w.sfY, B * D / 16) == cudaSuccess &&
                    dev_alloc(&w.sfC, B * (D + F) / 16) == cudaSuccess && dev_alloc(&w.sY4, R * 4) == cudaSuccess &&
                    dev_alloc(&w.sC4, R * 4) == cudaSuccess;
    if (!ok) {
      free_ws3_fp4(w);
      return fail(FLUX_ENOMEM, "NVFP4 workspace allocation for %d tokens failed", rows);
    }
    w.cap4_rows = R;
    w.cap4_blocks = blocks;
  }
  if (w.maps4) return FLUX_OK;
  bool ok = true;
  const size_t lY = D / 2, lC = (D + F) / 2;
  auto y_op = [&](Fp4Op* o, size_t r, int nrows, int blk0) {
    ok &= make_fp4_op(o, w.Y4 + r * lY, nrows, D, lY, w.sfY, blk0, w.sY4 + r);
  };
  auto c_op = [&](Fp4Op* o, size_t r, int nrows, int blk0) {
    ok &= make_fp4_op(o, w.C4 + r * lC, nrows, D + F, lC, w.sfC, blk0, w.sC4 + r);
  };
  for (int sg = 0; sg < 3; ++sg) {
    y_op(&w.y4_pm[0][sg], row0[sg], seg[sg], w.seg_pm.blk0[sg]);
    c_op(&w.c4_pm[0][sg], row0[sg], seg[sg], w.seg_pm.blk0[sg]);
  }
  for (int bb = 1; bb < nb; ++bb) {
    y_op(&w.y4_pm[bb][0], static_cast<size_t>(bb) * n, nt, w.seg_pm.blk0[2 + bb]);
    c_op(&w.c4_pm[bb][0], static_cast<size_t>(bb) * n, nt, w.seg_pm.blk0[2 + bb]);
  }
  for (int bb = 0; bb < nb; ++bb) {
    y_op(&w.y4_all[bb], static_cast<size_t>(bb) * n, n, w.seg_jy.blk0[bb]);
    for (int sg = 0; sg < 3; ++sg)
      c_op(&w.c4_seg[bb][sg], static_cast<size_t>(bb) * n + row0[sg], seg[sg], w.seg_jc.blk0[3 * bb + sg]);
  }
  if (!ok) return fail(FLUX_EIO, "cuTensorMapEncodeTiled failed for an NVFP4 activation buffer");
  w.maps4 = true;
  return FLUX_OK;
}

int prepare3_quant(flux3_dit* m, int nt, int ni, int nr, int nb) {
  if (m->precision == FLUX_PRECISION_FP8) return prepare3_fp8(m, nt, ni, nr, nb);
  if (m->precision == FLUX_PRECISION_NVFP4) return prepare3_fp4(m, nt, ni, nr, nb);
  return FLUX_OK;
}

int prepare_shape3(flux3_dit* m, int nt, int gh, int gw, const RefGrids& refs, int nb, cudaStream_t s) {
  Workspace3& w = m->ws;
  const flux3_dit_config& c = m->cfg;
  const size_t D = c.hidden, F = c.mlp_hidden;
  const size_t ni = static_cast<size_t>(gh) * gw, nr = ref_tokens(refs);
  const size_t n = nt + ni + nr, rows = n * nb;
  if (rows > w.cap_n) {
    free_ws3(w);
    bool ok = dev_alloc(&w.X, rows * D * 4) == cudaSuccess;
    ok = ok && dev_alloc(&w.Y, rows * D * 2) == cudaSuccess;
    ok = ok && dev_alloc(&w.QKV, rows * 3 * D * 2) == cudaSuccess;
    ok = ok && dev_alloc(&w.CC, rows * (D + F) * 2) == cudaSuccess;
    ok = ok && dev_alloc(&w.rope, rows * 64 * sizeof(float2)) == cudaSuccess;
    if (!ok) {
      free_ws3(w);
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
    return prepare3_quant(m, nt, static_cast<int>(ni), static_cast<int>(nr), nb);
  w.maps8 = false;
  w.maps4 = false;

  const uint64_t ldD = D * 2, ldC = (D + F) * 2;
  bool ok = true;
  auto amap = [&](CUtensorMap* map, const void* base, size_t r, size_t cols, uint64_t stride) {
    if (r == 0) {
      memset(map, 0, sizeof(*map));
      return;
    }
    ok &= make_tmap_bf16(map, base, r, cols, stride, 128);
  };
  const size_t row0[3] = {0, static_cast<size_t>(nt), nt + ni};
  const size_t seg[3] = {static_cast<size_t>(nt), ni, nr};
  amap(&w.a_tokb, w.tokb, ni + nr, c.in_ch, c.in_ch * 2);
  amap(&w.qkv, w.QKV, rows, 3 * D, 3 * D * 2);
  for (int bb = 0; bb < nb; ++bb) {
    const size_t r0 = bb * n;
    amap(&w.a_txtb[bb], w.txtb + bb * nt * static_cast<size_t>(c.txt_dim), nt, c.txt_dim,
         static_cast<uint64_t>(c.txt_dim) * 2);
    amap(&w.a_Yall[bb], w.Y + r0 * D, n, D, ldD);
    amap(&w.a_Yout[bb], w.Y + bb * ni * D, ni, D, ldD);        // output layer input: LN of sequence bb's image rows
    for (int sg = 0; sg < 3; ++sg) {
      amap(&w.a_Yseg[bb][sg], w.Y + (r0 + row0[sg]) * D, seg[sg], D, ldD);
      amap(&w.a_CCseg[bb][sg], w.CC + (r0 + row0[sg]) * (D + F), seg[sg], D + F, ldC);
    }
  }
  if (!ok) return fail(FLUX_EIO, "cuTensorMapEncodeTiled failed for an activation buffer");
  if (rope_table_launch(w.rope, nt, gh, gw, refs, c.rope_theta, s) != cudaSuccess)
    return fail(FLUX_EIO, "rope table launch failed");
  w.nt = nt; w.gh = gh; w.gw = gw; w.nb = nb; w.refs = refs;
  return prepare3_quant(m, nt, static_cast<int>(ni), static_cast<int>(nr), nb);
}

// Quantise every block linear (per-mode streams and joint blocks) to e4m3, one scale per row.
int quantize3_block_weights(flux3_dit* m, cudaStream_t s) {
  const flux3_dit_config& c = m->cfg;
  const size_t D = c.hidden, F = c.mlp_hidden;
  std::vector<BlockW3*> blocks;
  for (BlockW3& b : m->mode) blocks.push_back(&b);
  for (BlockW3& b : m->joint) blocks.push_back(&b);
  const size_t r1 = 3 * D + 2 * F, r2 = D;
  const size_t b1 = (r1 * D + 255) / 256 * 256, b2 = (r2 * (D + F) + 255) / 256 * 256;
  const size_t s1 = (r1 + 63) / 64 * 64, s2 = (r2 + 63) / 64 * 64;
  const size_t nb = blocks.size();
  if (dev_alloc(&m->w8, nb * (b1 + b2)) != cudaSuccess || dev_alloc(&m->w8_scale, nb * (s1 + s2) * 4) != cudaSuccess) {
    cudaFree(m->w8);
    cudaFree(m->w8_scale);
    m->w8 = nullptr;
    m->w8_scale = nullptr;
    return fail(FLUX_ENOMEM, "device allocation of the FP8 weights failed");
  }
  bool ok = true;
  for (size_t i = 0; i < nb; ++i) {
    BlockW3& bw = *blocks[i];
    uint8_t* q1 = m->w8 + i * (b1 + b2);
    uint8_t* q2 = q1 + b1;
    float* sc1 = m->w8_scale + i * (s1 + s2);
    float* sc2 = sc1 + s1;
    FD_CUDA(quantize_rows_launch(bw.w_lin1, static_cast<int>(D), static_cast<int>(r1), static_cast<int>(D), q1,
                                 static_cast<int>(D), sc1, s));
    FD_CUDA(quantize_rows_launch(bw.w_lin2, static_cast<int>(D + F), static_cast<int>(r2), static_cast<int>(D + F),
                                 q2, static_cast<int>(D + F), sc2, s));
    ok &= make_tmap_u8(&bw.m8_qkv, q1, 3 * D, D, D, 128);
    ok &= make_tmap_u8(&bw.m8_mlp, q1 + 3 * D * D, 2 * F, D, D, 128);
    ok &= make_tmap_u8(&bw.m8_lin2, q2, D, D + F, D + F, 128);
    bw.s_qkv = sc1;
    bw.s_mlp = sc1 + 3 * D;
    bw.s_lin2 = sc2;
  }
  if (!ok) return fail(FLUX_EIO, "cuTensorMapEncodeTiled failed for an FP8 weight tensor");
  FD_CUDA(cudaStreamSynchronize(s));
  return FLUX_OK;
}

// Quantise every block linear (per-mode streams and joint blocks) to NVFP4.
int quantize3_block_weights_nvfp4(flux3_dit* m, cudaStream_t s) {
  const flux3_dit_config& c = m->cfg;
  const size_t D = c.hidden, F = c.mlp_hidden;
  std::vector<BlockW3*> blocks;
  for (BlockW3& b : m->mode) blocks.push_back(&b);
  for (BlockW3& b : m->joint) blocks.push_back(&b);
  std::vector<Fp4Mat> mats;
  for (BlockW3* b : blocks) {
    mats.push_back({b->w_lin1, 3 * D + 2 * F, D});
    mats.push_back({b->w_lin2, D, D + F});
  }
  int rc = quantize_weights_nvfp4(mats, &m->w4, &m->w4_scale, s);
  if (rc) return rc;
  bool ok = true;
  auto op = [&](Fp4Op* o, const Fp4Mat& x, size_t row0, size_t rows) {
    ok &= make_fp4_op(o, x.codes + row0 * x.cols / 2, rows, x.cols, x.cols / 2, x.sf, row0 / 128, x.scale + row0);
  };
  for (size_t i = 0; i < blocks.size(); ++i) {
    op(&blocks[i]->q4_qkv, mats[2 * i], 0, 3 * D);
    op(&blocks[i]->q4_mlp, mats[2 * i], 3 * D, 2 * F);  // the SwiGLU rows start on a 128-row block
    op(&blocks[i]->q4_lin2, mats[2 * i + 1], 0, D);
  }
  if (!ok) return fail(FLUX_EIO, "cuTensorMapEncodeTiled failed for an NVFP4 weight tensor");
  FD_CUDA(cudaStreamSynchronize(s));
  return FLUX_OK;
}

// Every modulation vector of one forward into m->mods (layout: kMod* offsets).
int run_modulation3(flux3_dit* m, float t, float t_target, cudaStream_t s) {
  const flux3_dit_config& c = m->cfg;
  const int D = c.hidden, tf = c.t_freq_dim;
  auto gv = [](double rows, double k, double nvec) { return rows * k * 2 + nvec * (rows * 6 + k * 4); };
  float* mods = m->mods;
  // embeddings of t (image tokens) and 0 (text and reference tokens), and of the target time
  FD_LAUNCH(m, kProfOther, 0, tf * 4.0, timestep_embed_launch(m->temb, t, tf, s));
  FD_LAUNCH(m, kProfOther, 0, tf * 4.0, timestep_embed_launch(m->temb + tf, 0.0f, tf, s));
  FD_LAUNCH(m, kProfGemv, 4.0 * D * tf, gv(D, tf, 2),
            gemv_multi_launch(m->t_w1, m->t_b1, m->temb, 2, m->th, nullptr, D, tf, 0, 1, s));
  const float* add = nullptr;
  if (c.flow_map) {
    FD_LAUNCH(m, kProfOther, 0, tf * 4.0, timestep_embed_launch(m->temb + 2 * tf, t_target, tf, s));
    FD_LAUNCH(m, kProfGemv, 2.0 * D * tf, gv(D, tf, 1),
              gemv_multi_launch(m->g_w1, m->g_b1, m->temb + 2 * tf, 1, m->th + 2 * D, nullptr, D, tf, 0, 1, s));
    FD_LAUNCH(m, kProfGemv, 2.0 * D * D, gv(D, D, 1),
              gemv_multi_launch(m->g_w2, m->g_b2, m->th + 2 * D, 1, m->tt, nullptr, D, D, 0, 0, s));
    add = m->tt;
  }
  // vec[0] = vec_img, vec[1] = vec_ctx
  FD_LAUNCH(m, kProfGemv, 4.0 * D * D, gv(D, D, 2),
            gemv_multi_launch(m->t_w2, m->t_b2, m->th, 2, m->vec, add, D, D, 0, 0, s));
  const float* v_img = m->vec;
  const float* v_ctx = m->vec + D;
  const float* src[3] = {v_ctx, v_img, v_ctx};
  const int dst[3] = {kModTxt, kModImg, kModRef};
  for (int sidx = 0; sidx < 3; ++sidx)
    FD_LAUNCH(m, kProfGemv, 6.0 * D * D, gv(3.0 * D, D, 1),
              gemv_multi_launch(m->mode_mod_w[sidx], m->mode_mod_b[sidx], src[sidx], 1,
                                mods + static_cast<size_t>(dst[sidx]) * D, nullptr, 3 * D, D, 1, 0, s));
  // joint modulation on both vectors with one weight read: image set at kModJointImg, context set right after
  FD_LAUNCH(m, kProfGemv, 12.0 * D * D, gv(3.0 * D, D, 2),
            gemv_multi_launch(m->joint_mod_w, m->joint_mod_b, m->vec, 2,
                              mods + static_cast<size_t>(kModJointImg) * D, nullptr, 3 * D, D, 1, 0, s));
  FD_LAUNCH(m, kProfGemv, 4.0 * D * D, gv(2.0 * D, D, 1),
            gemv_multi_launch(m->fin_mod_w, m->fin_mod_b, v_img, 1, mods + static_cast<size_t>(kModFinal) * D,
                              nullptr, 2 * D, D, 1, 0, s));
  return FLUX_OK;
}

// One forward of nb sequences that share the image tokens, the references, t and t_target and
// differ in their text (nb = 2: the prompt and the unconditional text of classifier-free
// guidance).  In the per-mode blocks the image and reference streams attend only to themselves
// and are modulated from t and t = 0 alone, so they are the same for every sequence: they run
// once (in sequence 0's rows) and are copied to the other sequences before the joint blocks.
// Every GEMM takes the kernel a one-sequence forward would take, so each velocity equals, bit
// for bit, that of a forward with its text alone.
int forward3_impl(flux3_dit* m, const float* img_tok, int gh, int gw, const float* const* txt, int nt,
                  const float* ref_tok, const RefGrids& refs, float t, float t_target, float* const* v_out, int nb,
                  cudaStream_t s) {
  const flux3_dit_config& c = m->cfg;
  const int D = c.hidden, F = c.mlp_hidden, H = c.heads;
  if (nb < 1 || nb > kMaxBatch3) return fail(FLUX_EINVAL, "batch of %d sequences (1..%d)", nb, kMaxBatch3);
  if (!img_tok) return fail(FLUX_EINVAL, "img_tok must be a device pointer");
  for (int bb = 0; bb < nb; ++bb) {
    if (!v_out[bb]) return fail(FLUX_EINVAL, "velocity output %d is NULL", bb);
    if (nt > 0 && !txt[bb]) return fail(FLUX_EINVAL, "text %d is NULL for %d text tokens", bb, nt);
    for (int o = 0; o < bb; ++o)
      if (v_out[o] == v_out[bb]) return fail(FLUX_EINVAL, "the velocity outputs must be distinct buffers");
  }
  if (gh < 4 || gh > 64 || gw < 4 || gw > 64) return fail(FLUX_EINVAL, "image grid %dx%d outside 4..64", gh, gw);
  if (nt < 0 || nt > 4096) return fail(FLUX_EINVAL, "bad text (n_txt=%d)", nt);
  if (refs.count < 0 || refs.count > kMaxRefs)
    return fail(FLUX_EINVAL, "%d reference images (at most %d)", refs.count, kMaxRefs);
  for (int k = 0; k < refs.count; ++k)
    if (refs.h[k] < 4 || refs.h[k] > 64 || refs.w[k] < 4 || refs.w[k] > 64)
      return fail(FLUX_EINVAL, "reference %d grid %dx%d outside 4..64", k, refs.h[k], refs.w[k]);
  if (refs.count > 0 && !ref_tok) return fail(FLUX_EINVAL, "ref_tok is NULL for %d reference(s)", refs.count);
  if (!std::isfinite(t) || (c.flow_map && !std::isfinite(t_target)))
    return fail(FLUX_EINVAL, "t (and, for the flow-map model, t_target) must be finite");
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev != m->device) return fail(FLUX_EINVAL, "model lives on device %d, current device is %d", m->device, dev);

  int rc = prepare_shape3(m, nt, gh, gw, refs, nb, s);
  if (rc) return rc;
  Workspace3& w = m->ws;
  const int ni = gh * gw, nr = static_cast<int>(ref_tokens(refs)), n = nt + ni + nr, rows_all = n * nb;
  // rows the per-mode blocks touch: all of sequence 0, the text rows of the others
  const int rows_pm = nb == 1 ? n : (nb - 1) * n + nt;
  const int row0[3] = {0, nt, nt + ni};
  const int seg[3] = {nt, ni, nr};
  const size_t sD = D, sDF = static_cast<size_t>(D) + F;
  const float eps_ln = c.eps_ln, eps_rms = c.eps_rms;
  const float* mods = m->mods;
  auto md = [&](int off) { return mods + static_cast<size_t>(off) * D; };

  rc = run_modulation3(m, t, t_target, s);
  if (rc) return rc;
  FD_LAUNCH(m, kProfOther, 0, 6.0 * ni * c.in_ch,
            cast_bf16_launch(img_tok, w.tokb, static_cast<size_t>(ni) * c.in_ch, s));
  if (nr)
    FD_LAUNCH(m, kProfOther, 0, 6.0 * nr * c.in_ch,
              cast_bf16_launch(ref_tok, w.tokb + static_cast<size_t>(ni) * c.in_ch,
                               static_cast<size_t>(nr) * c.in_ch, s));
  for (int bb = 0; bb < nb && nt; ++bb)
    FD_LAUNCH(m, kProfOther, 0, 6.0 * nt * c.txt_dim,
              cast_bf16_launch(txt[bb], w.txtb + static_cast<size_t>(bb) * nt * c.txt_dim,
                               static_cast<size_t>(nt) * c.txt_dim, s));
  const bool fp8 = m->precision == FLUX_PRECISION_FP8;

  // input projections: every text, the image and reference tokens once (sequence 0's rows)
  GemmParams4 P4;
  GemmParams& P = P4.g;
  P.num_problems = 2;
  problem(P, 0, w.a_txtb[0], m->m_txt_in, nt, D, c.txt_dim, kEpiF32Bias, w.X, D, m->txt_b, nullptr);
  problem(P, 1, w.a_tokb, m->m_img_in, ni + nr, D, c.in_ch, kEpiF32Bias, w.X + nt * sD, D, m->img_b, nullptr);
  const bool small_in = small_linear(P, m->num_sms, false, 1);
  for (int bb = 1; bb < nb; ++bb)
    problem(P, P.num_problems++, w.a_txtb[bb], m->m_txt_in, nt, D, c.txt_dim, kEpiF32Bias, w.X + bb * n * sD, D,
            m->txt_b, nullptr);
  FD_LAUNCH(m, kProfGemm, gemm_flops(P), gemm_bytes(P), launch_linear_as(P, m->num_sms, s, false, small_in));

  AttnParams A;
  A.mapQ = w.qkv; A.mapK = w.qkv; A.mapV = w.qkv;
  A.out = w.CC; A.ldo = D + F; A.heads = H; A.batch = 1;
  A.q_col0 = 0; A.k_col0 = D; A.v_col0 = 2 * D;
  A.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(c.head_dim)));

  // FP8 precision: block linears on e4m3 codes; LN-mod quantises its output, [O | H] is quantised
  // (one scale per row) before linear2
  auto f8 = [&](int i, const CUtensorMap& a8, const CUtensorMap& w8, const float* sa, const float* sb) {
    P.mapA[i] = a8;
    P.mapB[i] = w8;
    P.prob[i].scale_a = sa;
    P.prob[i].scale_b = sb;
  };
  // NVFP4 precision: LN-mod quantises its output per segment (`segs`) in the same pass; [O | H] is
  // quantised per segment before linear2
  const bool fp4 = m->precision == FLUX_PRECISION_NVFP4;
  const OpFormat lin_fmt = fp4 ? OpFormat::kNvfp4 : fp8 ? OpFormat::kE4M3 : OpFormat::kBf16;
  auto linear_as = [&](bool small) -> cudaError_t {
    return fp4 ? gemm_fp4_launch(P4, m->num_sms, s) : launch_linear_as(P, m->num_sms, s, fp8, small);
  };
  auto quant4 = [&](const bf16* x, int k, uint8_t* q, uint8_t* sf, float* sc, const Q4Segs& segs) -> int {
    double r = 0;
    for (int z = 0; z < segs.n; ++z) r += segs.rows[z];
    FD_LAUNCH(m, kProfOther, 0, 2.5 * r * k + 4.0 * r,
              quantize_nvfp4_launch(x, static_cast<int>(k == D ? D : D + F), k, q, k == D ? D / 2 : (D + F) / 2, sf,
                                    sc, segs, s));
    return FLUX_OK;
  };
  // LN + modulation of rows [0, r) (text | image | reference per sequence of n rows)
  auto ln3 = [&](int r, const float* sh0, const float* sc0, const float* sh1, const float* sc1, const float* sh2,
                 const float* sc2) -> int {
    if (fp8)
      FD_LAUNCH(m, kProfLnMod, 0, 5.0 * r * D + 4.0 * r,
                ln_modulate_fp8_launch(w.X, w.Y8, w.sY, r, D, nt, nt + ni, n, sh0, sc0, sh1, sc1, sh2, sc2, eps_ln,
                                       s));
    else
      FD_LAUNCH(m, kProfLnMod, 0, 6.0 * r * D + 16.0 * D,
                ln_modulate3_launch(w.X, w.Y, r, D, nt, nt + ni, n, sh0, sc0, sh1, sc1, sh2, sc2, eps_ln, s));
    return FLUX_OK;
  };
  auto ln3q = [&](int r, const Q4Segs& segs, const float* sh0, const float* sc0, const float* sh1, const float* sc1,
                  const float* sh2, const float* sc2) -> int {
    if (!fp4) return ln3(r, sh0, sc0, sh1, sc1, sh2, sc2);
    const LnModSets ms{nt, nt + ni, n, sh0, sh1, sh2, sc0, sc1, sc2};
    FD_LAUNCH(m, kProfLnMod, 0, 4.56 * r * D + 4.0 * r,
              ln_modulate_nvfp4_launch(w.X, D, w.Y4, w.sfY, w.sY4, segs, ms, eps_ln, s));
    return FLUX_OK;
  };
  auto quant_cc = [&](int r) -> int {
    FD_LAUNCH(m, kProfOther, 0, 3.0 * r * sDF + 4.0 * r, quantize_rows_launch(w.CC, D + F, r, D + F, w.C8, D + F, w.sC, s));
    return FLUX_OK;
  };

  // ---------------- per-mode blocks: each stream with its own weights, attention within the stream.
  // Segments: sequence 0's text, image and reference rows, then the other sequences' text rows.
  AttnParams As = A;
  As.nseg = 2 + nb;
  double seg_flops = 0;
  for (int z = 0; z < As.nseg; ++z) {
    As.seg_row0[z] = z < 3 ? row0[z] : (z - 2) * n;
    As.seg_n[z] = z < 3 ? seg[z] : nt;
    seg_flops += 4.0 * As.seg_n[z] * static_cast<double>(As.seg_n[z]) * D;
  }
  const int mode_set[3] = {kModTxt, kModImg, kModRef};
  for (int i = 0; i < m->act_mode; ++i) {
    const NvtxRange range("per-mode block %d", i);
    rc = ln3q(rows_pm, w.seg_pm, md(kModTxt), md(kModTxt + 1), md(kModImg), md(kModImg + 1), md(kModRef),
              md(kModRef + 1));
    if (rc) return rc;
    // linear1: (qkv + QK-RMSNorm + RoPE, SwiGLU) per stream of sequence 0, then the other texts
    P.num_problems = 0;
    auto lin1 = [&](int sg, size_t r0) {
      const BlockW3& bw = m->mode[3 * i + sg];
      const int bb = static_cast<int>(r0 / n), j = P.num_problems;
      problem(P, j, w.a_Yseg[bb][sg], bw.m_qkv, seg[sg], 3 * D, D, kEpiBf16Bias, w.QKV + (r0 + row0[sg]) * 3 * sD,
              3 * D, bw.qkv_b, nullptr);
      qk_fuse(P, j, bw.q_gain, bw.k_gain, w.rope, row0[sg], eps_rms);
      problem(P, j + 1, w.a_Yseg[bb][sg], bw.m_mlp, seg[sg], 2 * F, D, kEpiSwiGLU, w.CC + (r0 + row0[sg]) * sDF + D,
              D + F, bw.mlp_b, nullptr);
      if (fp8) {
        f8(j, w.a8_Yseg[bb][sg], bw.m8_qkv, w.sY + r0 + row0[sg], bw.s_qkv);
        f8(j + 1, w.a8_Yseg[bb][sg], bw.m8_mlp, w.sY + r0 + row0[sg], bw.s_mlp);
      }
      if (fp4) {
        fp4_operands(P4, j, w.y4_pm[bb][sg], bw.q4_qkv);
        fp4_operands(P4, j + 1, w.y4_pm[bb][sg], bw.q4_mlp);
      }
      P.num_problems += 2;
    };
    for (int sg = 0; sg < 3; ++sg) lin1(sg, 0);
    for (int bb = 1; bb < nb; ++bb) lin1(kSegTxt, static_cast<size_t>(bb) * n);
    FD_LAUNCH(m, kProfGemm, gemm_flops(P), gemm_bytes(P, lin_fmt), linear_as(false));   // SwiGLU: pair kernel
    FD_LAUNCH(m, kProfAttention, seg_flops, 8.0 * rows_pm * D, attention_launch(As, s));
    if (fp8 && (rc = quant_cc(rows_pm))) return rc;
    if (fp4 && (rc = quant4(w.CC, D + F, w.C4, w.sfC, w.sC4, w.seg_pm))) return rc;
    // linear2 with each stream's gate into the residual; the kernel is chosen for sequence 0's streams
    P.num_problems = 0;
    auto lin2 = [&](int sg, size_t r0) {
      const BlockW3& bw = m->mode[3 * i + sg];
      const int bb = static_cast<int>(r0 / n), j = P.num_problems++;
      problem(P, j, w.a_CCseg[bb][sg], bw.m_lin2, seg[sg], D, D + F, kEpiResidGate, w.X + (r0 + row0[sg]) * sD, D,
              bw.lin2_b, md(mode_set[sg] + 2));
      if (fp8) f8(j, w.a8_CCseg[bb][sg], bw.m8_lin2, w.sC + r0 + row0[sg], bw.s_lin2);
      if (fp4) fp4_operands(P4, j, w.c4_pm[bb][sg], bw.q4_lin2);
    };
    for (int sg = 0; sg < 3; ++sg) lin2(sg, 0);
    const bool small = small_linear(P, m->num_sms, fp8, 1);
    for (int bb = 1; bb < nb; ++bb) lin2(kSegTxt, static_cast<size_t>(bb) * n);
    FD_LAUNCH(m, kProfGemm, gemm_flops(P), gemm_bytes(P, lin_fmt), linear_as(small));
  }
  // the image and reference streams of sequence 0 into the other sequences
  for (int bb = 1; bb < nb; ++bb)
    FD_LAUNCH(m, kProfOther, 0, 8.0 * (ni + nr) * D,
              cudaMemcpyAsync(w.X + (static_cast<size_t>(bb) * n + nt) * sD, w.X + nt * sD,
                              static_cast<size_t>(ni + nr) * sD * sizeof(float), cudaMemcpyDeviceToDevice, s));

  // ---------------- joint blocks: one weight set, attention over each whole sequence, modulation per token type
  const int joint_set[3] = {kModJointCtx, kModJointImg, kModJointCtx};
  const double at_flops = 4.0 * nb * n * static_cast<double>(n) * D;
  A.n = n;
  A.batch = nb;
  for (int i = 0; i < m->act_joint; ++i) {
    const NvtxRange range("joint block %d", i);
    const BlockW3& bw = m->joint[i];
    rc = ln3q(rows_all, w.seg_jy, md(kModJointCtx), md(kModJointCtx + 1), md(kModJointImg), md(kModJointImg + 1),
              md(kModJointCtx), md(kModJointCtx + 1));
    if (rc) return rc;
    P.num_problems = 2 * nb;
    for (int bb = 0; bb < nb; ++bb) {
      const size_t r0 = static_cast<size_t>(bb) * n;
      problem(P, 2 * bb, w.a_Yall[bb], bw.m_qkv, n, 3 * D, D, kEpiBf16Bias, w.QKV + r0 * 3 * sD, 3 * D, bw.qkv_b,
              nullptr);
      qk_fuse(P, 2 * bb, bw.q_gain, bw.k_gain, w.rope, 0, eps_rms);
      problem(P, 2 * bb + 1, w.a_Yall[bb], bw.m_mlp, n, 2 * F, D, kEpiSwiGLU, w.CC + r0 * sDF + D, D + F, bw.mlp_b,
              nullptr);
      if (fp8) {
        f8(2 * bb, w.a8_Yall[bb], bw.m8_qkv, w.sY + r0, bw.s_qkv);
        f8(2 * bb + 1, w.a8_Yall[bb], bw.m8_mlp, w.sY + r0, bw.s_mlp);
      }
      if (fp4) {
        fp4_operands(P4, 2 * bb, w.y4_all[bb], bw.q4_qkv);
        fp4_operands(P4, 2 * bb + 1, w.y4_all[bb], bw.q4_mlp);
      }
    }
    FD_LAUNCH(m, kProfGemm, gemm_flops(P), gemm_bytes(P, lin_fmt), linear_as(small_linear(P, m->num_sms, fp8, nb)));
    FD_LAUNCH(m, kProfAttention, at_flops, 8.0 * rows_all * D, attention_launch(A, s));
    if (fp8 && (rc = quant_cc(rows_all))) return rc;
    if (fp4 && (rc = quant4(w.CC, D + F, w.C4, w.sfC, w.sC4, w.seg_jc))) return rc;
    P.num_problems = 3 * nb;
    for (int bb = 0; bb < nb; ++bb)
      for (int sg = 0; sg < 3; ++sg) {
        const size_t r = static_cast<size_t>(bb) * n + row0[sg];
        problem(P, 3 * bb + sg, w.a_CCseg[bb][sg], bw.m_lin2, seg[sg], D, D + F, kEpiResidGate, w.X + r * sD, D,
                bw.lin2_b, md(joint_set[sg] + 2));
        if (fp8) f8(3 * bb + sg, w.a8_CCseg[bb][sg], bw.m8_lin2, w.sC + r, bw.s_lin2);
        if (fp4) fp4_operands(P4, 3 * bb + sg, w.c4_seg[bb][sg], bw.q4_lin2);
      }
    FD_LAUNCH(m, kProfGemm, gemm_flops(P), gemm_bytes(P, lin_fmt), linear_as(small_linear(P, m->num_sms, fp8, nb)));
  }

  // ---------------- output layer on the image rows (text and reference tokens are dropped)
  const NvtxRange range("output layer");
  P.num_problems = nb;
  for (int bb = 0; bb < nb; ++bb) {
    FD_LAUNCH(m, kProfLnMod, 0, 6.0 * ni * D + 8.0 * D,
              ln_modulate_launch(w.X + (static_cast<size_t>(bb) * n + nt) * sD, w.Y + static_cast<size_t>(bb) * ni * sD,
                                 ni, D, ni, ni, md(kModFinal), md(kModFinal + 1), md(kModFinal), md(kModFinal + 1),
                                 eps_ln, s));
    problem(P, bb, w.a_Yout[bb], m->m_fin, ni, c.in_ch, D, kEpiF32Bias, v_out[bb], c.in_ch, m->fin_b, nullptr);
  }
  FD_LAUNCH(m, kProfGemm, gemm_flops(P), gemm_bytes(P), gemm_launch(P, 128, m->num_sms, s));
  return FLUX_OK;
}

int read_ref_grids(int n_refs, const int* ref_grids, RefGrids* refs) {
  if (n_refs < 0 || n_refs > kMaxRefs) return fail(FLUX_EINVAL, "%d reference images (at most %d)", n_refs, kMaxRefs);
  if (n_refs > 0 && !ref_grids) return fail(FLUX_EINVAL, "ref_grids is NULL");
  refs->count = n_refs;
  for (int k = 0; k < n_refs; ++k) {
    refs->h[k] = ref_grids[2 * k];
    refs->w[k] = ref_grids[2 * k + 1];
  }
  return FLUX_OK;
}

}  // namespace
}  // namespace fdit

using namespace fdit;

// ====================================================================== C ABI
extern "C" {

size_t flux3_blob_expected_bytes(const flux3_dit_config* cfg) {
  if (!cfg || !valid_cfg3(*cfg)) return 0;
  size_t total = 0;
  blob_tensors3(*cfg, &total);
  return total;
}

flux3_dit* flux3_dit_create(const void* blob, size_t blob_bytes, const flux3_dit_config* cfg, void* stream) {
  flux3_dit* m = nullptr;
  create3_impl(blob, blob_bytes, cfg, static_cast<cudaStream_t>(stream), &m);
  return m;
}

void flux3_dit_destroy(flux3_dit* m) { destroy3(m); }

int flux3_dit_forward(flux3_dit* m, const float* img_tok, int grid_h, int grid_w, const float* txt, int n_txt,
                      const float* ref_tok, int n_refs, const int* ref_grids, float t, float t_target, float* v_out,
                      void* stream) {
  if (!m) return fail(FLUX_EINVAL, "model is NULL");
  RefGrids refs;
  const int rc = read_ref_grids(n_refs, ref_grids, &refs);
  if (rc) return rc;
  return forward3_impl(m, img_tok, grid_h, grid_w, &txt, n_txt, ref_tok, refs, t, t_target, &v_out, 1,
                       static_cast<cudaStream_t>(stream));
}

int flux3_dit_forward_cfg(flux3_dit* m, const float* img_tok, int grid_h, int grid_w, const float* txt_cond,
                          const float* txt_uncond, int n_txt, const float* ref_tok, int n_refs, const int* ref_grids,
                          float t, float t_target, float* v_cond, float* v_uncond, void* stream) {
  if (!m) return fail(FLUX_EINVAL, "model is NULL");
  RefGrids refs;
  const int rc = read_ref_grids(n_refs, ref_grids, &refs);
  if (rc) return rc;
  const float* txt[2] = {txt_cond, txt_uncond};
  float* out[2] = {v_cond, v_uncond};
  return forward3_impl(m, img_tok, grid_h, grid_w, txt, n_txt, ref_tok, refs, t, t_target, out, 2,
                       static_cast<cudaStream_t>(stream));
}

int flux3_dit_set_precision(flux3_dit* m, int precision) {
  if (!m) return fail(FLUX_EINVAL, "model is NULL");
  if (precision == FLUX_PRECISION_BF16) {
    m->precision = precision;
    return FLUX_OK;
  }
  if (precision != FLUX_PRECISION_FP8 && precision != FLUX_PRECISION_NVFP4)
    return fail(FLUX_EINVAL, "unknown precision %d", precision);
  const flux3_dit_config& c = m->cfg;
  if (precision == FLUX_PRECISION_FP8 &&
      ((c.hidden != 1024 && c.hidden != 2048 && c.hidden != 3072 && c.hidden != 4096) ||
       c.hidden + c.mlp_hidden > 16384))
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
    const int rc = quantize3_block_weights(m, nullptr);
    if (rc) return rc;
  }
  if (precision == FLUX_PRECISION_NVFP4 && !m->w4) {
    const int rc = quantize3_block_weights_nvfp4(m, nullptr);
    if (rc) return rc;
  }
  m->precision = precision;
  return FLUX_OK;
}

int flux3_dit_set_active_blocks(flux3_dit* m, int n_mode, int n_joint) {
  if (!m) return fail(FLUX_EINVAL, "model is NULL");
  m->act_mode = n_mode < 0 ? m->cfg.n_mode : std::min(n_mode, m->cfg.n_mode);
  m->act_joint = n_joint < 0 ? m->cfg.n_joint : std::min(n_joint, m->cfg.n_joint);
  return FLUX_OK;
}

size_t flux3_dit_modulation_size(const flux3_dit* m) {
  return m ? static_cast<size_t>(kModRowsD) * m->cfg.hidden : 0;
}

int flux3_dit_modulation(flux3_dit* m, float t, float t_target, float* mods_out, void* stream) {
  if (!m || !mods_out) return fail(FLUX_EINVAL, "NULL argument");
  if (!std::isfinite(t) || (m->cfg.flow_map && !std::isfinite(t_target)))
    return fail(FLUX_EINVAL, "t (and, for the flow-map model, t_target) must be finite");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int rc = run_modulation3(m, t, t_target, s);
  if (rc) return rc;
  FD_CUDA(cudaMemcpyAsync(mods_out, m->mods, flux3_dit_modulation_size(m) * sizeof(float),
                          cudaMemcpyDeviceToDevice, s));
  return FLUX_OK;
}

int flux3_dit_profile(flux3_dit* m, int enable) {
  if (!m) return fail(FLUX_EINVAL, "model is NULL");
  FD_CUDA(cudaDeviceSynchronize());
  m->prof.reset();
  m->prof.on = enable != 0;
  return FLUX_OK;
}

int flux3_dit_profile_read(flux3_dit* m, int kind, double* ms, double* flops, double* bytes, long long* launches) {
  if (!m || kind < 0 || kind >= kProfKinds) return fail(FLUX_EINVAL, "bad model or kernel kind");
  FD_CUDA(cudaDeviceSynchronize());
  m->prof.settle();
  if (ms) *ms = m->prof.ms[kind];
  if (flops) *flops = m->prof.flops[kind];
  if (bytes) *bytes = m->prof.bytes[kind];
  if (launches) *launches = m->prof.launches[kind];
  return FLUX_OK;
}

int flux_joint_attention_segments(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* o, int n_seg,
                                  const int* seg_len, int heads, int head_dim, float scale, void* stream) {
  if (!q || !k || !v || !o || !seg_len) return fail(FLUX_EINVAL, "NULL argument");
  if (head_dim != 128) return fail(FLUX_EINVAL, "head_dim must be 128 (got %d)", head_dim);
  if (n_seg < 1 || n_seg > kMaxSegs) return fail(FLUX_EINVAL, "n_seg=%d outside 1..%d", n_seg, kMaxSegs);
  if (heads < 1 || heads > 1024) return fail(FLUX_EINVAL, "bad heads=%d", heads);
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return fail(FLUX_EINVAL, "q, k, v, o must be 16-byte aligned");
  if (!(scale > 0) || !std::isfinite(scale)) return fail(FLUX_EINVAL, "scale must be positive");
  AttnParams A;
  A.nseg = n_seg;
  long long rows = 0;
  for (int z = 0; z < n_seg; ++z) {
    if (seg_len[z] < 0) return fail(FLUX_EINVAL, "segment %d has negative length", z);
    A.seg_row0[z] = static_cast<int>(rows);
    A.seg_n[z] = seg_len[z];
    rows += seg_len[z];
    if (rows > (1ll << 31) - 1) return fail(FLUX_EINVAL, "segments too long");
  }
  if (rows == 0) return FLUX_OK;
  const uint64_t ld = static_cast<uint64_t>(heads) * 128;
  if (!make_tmap_bf16(&A.mapQ, q, rows, ld, ld * 2, 128) || !make_tmap_bf16(&A.mapK, k, rows, ld, ld * 2, 128) ||
      !make_tmap_bf16(&A.mapV, v, rows, ld, ld * 2, 128))
    return fail(FLUX_EIO, "cuTensorMapEncodeTiled failed");
  A.out = reinterpret_cast<bf16*>(o);
  A.ldo = static_cast<int>(ld);
  A.n = 0;
  A.heads = heads;
  A.batch = 1;
  A.q_col0 = A.k_col0 = A.v_col0 = 0;
  A.scale_log2 = static_cast<float>(scale * 1.4426950408889634);
  FD_CUDA(attention_launch(A, static_cast<cudaStream_t>(stream)));
  return FLUX_OK;
}

}  // extern "C"
