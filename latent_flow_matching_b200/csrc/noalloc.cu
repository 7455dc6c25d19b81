// Timestep conditioning (timestep embedding -> time MLP -> every modulation
// linear) for callers that may not allocate device memory once they are running:
// runtimes that hand all device memory to a pre-sized pool at start-up, or
// latency-critical loops that cannot afford cudaMalloc / cudaFree (cudaFree can
// synchronise the whole device).  The two hidden-size intermediates and the
// embedding live in a fixed device array that is part of this library's image,
// so a call allocates nothing.
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

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
float* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array for the current device (looked up once per device).
int scratch_for_current_device(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return FLUX_EIO;
  if (dev < 0 || dev >= kMaxDevices) return FLUX_EINVAL;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) return FLUX_EIO;
    g_noalloc_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_noalloc_ptr[dev];
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
  const int rc = scratch_for_current_device(&scratch);
  if (rc) return record_error(rc, "cudaGetSymbolAddress of the no-allocation scratch failed");
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
