// Timestep conditioning (timestep embedding -> time MLP -> every modulation
// linear) for callers that may not allocate device memory once they are running:
// runtimes that hand all device memory to a pre-sized pool at start-up, or
// latency-critical loops that cannot afford cudaMalloc / cudaFree (cudaFree can
// synchronise the whole device).  The two hidden-size intermediates and the
// embedding live in a fixed device array that is part of this library's image,
// so a call allocates nothing.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <mutex>

#include "../../include/fluxdit.h"
#include "fluxdit_internal.h"

namespace fdit {
namespace {

constexpr int kNoAllocMaxFreq = 1024;      // t_freq_dim limit
constexpr int kNoAllocMaxHidden = 8192;    // hidden limit
constexpr int kNoAllocFloats = kNoAllocMaxFreq + 2 * kNoAllocMaxHidden;   // 17408 floats = 68 KiB

// Scratch shared by every call on a device: [temb | h | vec].  Every element a
// call reads was written earlier by the same call, so nothing needs clearing.
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocFloats];

// The array's device address differs per CUDA context (each context loads its own copy of
// the library's device image), so the address is looked up once per context and kept under
// the context's process-unique ID: a context created later on the same device (after
// cudaDeviceReset, or a caller-made context) gets a fresh lookup instead of a stale address.
struct ScratchEntry {
  unsigned long long ctx_id;
  float* ptr;
};
constexpr int kMaxContexts = 64;
std::mutex g_noalloc_mutex;
ScratchEntry g_noalloc_cache[kMaxContexts];
int g_noalloc_entries = 0;
PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;
PFN_cuCtxGetId_v12000 g_ctx_id = nullptr;

// ID of the calling thread's current context (0 if none is current yet).
int current_context_id(unsigned long long* id) {
  if (!g_ctx_current || !g_ctx_id) {
    void* f1 = nullptr;
    void* f2 = nullptr;
    cudaDriverEntryPointQueryResult q1, q2;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) != cudaSuccess || !f1 ||
        cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) != cudaSuccess || !f2)
      return FLUX_EIO;
    g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f1);
    g_ctx_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(f2);
  }
  CUcontext ctx = nullptr;
  if (g_ctx_current(&ctx) != CUDA_SUCCESS) return FLUX_EIO;
  *id = 0;
  if (ctx && g_ctx_id(ctx, id) != CUDA_SUCCESS) return FLUX_EIO;
  return FLUX_OK;
}

// Device address of the scratch array in the current context (looked up once per context, with
// the caller's device current).
int scratch_for_current_context(float** out, const char** why) {
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  unsigned long long id = 0;
  if (current_context_id(&id)) {
    *why = "could not read the current CUDA context";
    return FLUX_EIO;
  }
  for (int i = 0; id && i < g_noalloc_entries; ++i)
    if (g_noalloc_cache[i].ctx_id == id) {
      *out = g_noalloc_cache[i].ptr;
      return FLUX_OK;
    }
  void* p = nullptr;
  // With no context current yet this also makes the device's primary context current.
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess || !p) {
    *why = "cudaGetSymbolAddress of the no-allocation scratch failed";
    return FLUX_EIO;
  }
  if (!id && current_context_id(&id)) {
    *why = "could not read the current CUDA context";
    return FLUX_EIO;
  }
  if (id && g_noalloc_entries < kMaxContexts) g_noalloc_cache[g_noalloc_entries++] = {id, static_cast<float*>(p)};
  *out = static_cast<float*>(p);
  return FLUX_OK;
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace
}  // namespace fdit

extern "C" int flux_timestep_modulation_noalloc(const uint16_t* w1, const uint16_t* b1, const uint16_t* w2,
                                                const uint16_t* b2, const uint16_t* wmod, const uint16_t* bmod,
                                                int hidden, int t_freq_dim, int mod_rows, float t, float* mods_out,
                                                void* stream) {
  using namespace fdit;
  if (!w1 || !b1 || !w2 || !b2 || !wmod || !bmod || !mods_out) return record_error(FLUX_EINVAL, "NULL argument");
  if (hidden < 8 || hidden % 8 || hidden > kNoAllocMaxHidden)
    return record_error(FLUX_EINVAL, "hidden must be a multiple of 8 in 8..8192 (the no-allocation scratch limit)");
  if (t_freq_dim < 8 || t_freq_dim % 8 || t_freq_dim > kNoAllocMaxFreq)
    return record_error(FLUX_EINVAL,
                        "t_freq_dim must be a multiple of 8 in 8..1024 (the no-allocation scratch limit)");
  if (mod_rows < 1) return record_error(FLUX_EINVAL, "mod_rows must be >= 1");
  if (!std::isfinite(t)) return record_error(FLUX_EINVAL, "t is not finite");
  if (!al16(w1) || !al16(w2) || !al16(wmod) || !al16(mods_out))
    return record_error(FLUX_EINVAL, "weight and output pointers must be 16-byte aligned");
  float* scratch = nullptr;
  const char* why = "";
  const int rc = scratch_for_current_context(&scratch, &why);
  if (rc) return record_error(rc, why);
  float* temb = scratch;
  float* h = scratch + kNoAllocMaxFreq;
  float* vec = h + kNoAllocMaxHidden;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const __nv_bfloat16* W1 = reinterpret_cast<const __nv_bfloat16*>(w1);
  const __nv_bfloat16* B1 = reinterpret_cast<const __nv_bfloat16*>(b1);
  const __nv_bfloat16* W2 = reinterpret_cast<const __nv_bfloat16*>(w2);
  const __nv_bfloat16* B2 = reinterpret_cast<const __nv_bfloat16*>(b2);
  const __nv_bfloat16* WM = reinterpret_cast<const __nv_bfloat16*>(wmod);
  const __nv_bfloat16* BM = reinterpret_cast<const __nv_bfloat16*>(bmod);
  cudaError_t e = timestep_embed_launch(temb, t, t_freq_dim, s);
  if (e == cudaSuccess) e = gemv_launch(W1, B1, temb, h, hidden, t_freq_dim, 0, 1, s);
  if (e == cudaSuccess) e = gemv_launch(W2, B2, h, vec, hidden, hidden, 0, 0, s);
  if (e == cudaSuccess) e = gemv_launch(WM, BM, vec, mods_out, mod_rows, hidden, 1, 0, s);
  if (e != cudaSuccess) return record_error(FLUX_EIO, cudaGetErrorString(e));
  return FLUX_OK;
}
