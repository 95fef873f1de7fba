// Decode without a caller-provided workspace: the scratch lives in a
// file-scope device array (KVC_STATIC_SCRATCH_BYTES per GPU, held until the
// process exits).  For callers that cannot allocate device memory -- code
// inside a host framework that owns all device allocations, or a serving loop
// that must not call cudaMalloc.  Nothing here allocates.
#include <mutex>

#include "kvc_internal.h"

namespace {

constexpr size_t kScratchBytes = KVC_STATIC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// One copy per device that loads the library.  In host code this name is only
// a stand-in for the symbol, never a device address: the address is looked up
// with cudaGetSymbolAddress while the device is current.
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices];   // device address of g_scratch, per device

kvc_status scratch_of_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess)
    return kvc::report_error(KVC_ECUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices)
    return kvc::report_error(KVC_EUNSUPPORTED, "device %d beyond %d", dev, kMaxDevices);
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess || !p)
      return kvc::report_error(KVC_ECUDA, "cudaGetSymbolAddress(scratch) on device %d: %s", dev,
                               cudaGetErrorString(e));
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return KVC_OK;
}

}  // namespace

extern "C" kvc_status kvc_decode_attn_static(const kvc_layout* layout, const kvc_cache* cache,
                                             const void* q, void* out, void* stream) {
  if (!layout || !cache)
    return kvc::report_error(KVC_EINVAL, "kvc_decode_attn_static: NULL argument");
  const size_t need = kvc_workspace_bytes(layout, cache->n_tokens);
  if (need > kScratchBytes)
    return kvc::report_error(KVC_EWORKSPACE,
                             "kvc_decode_attn_static: this layout needs %zu bytes of scratch; the "
                             "built-in area holds %zu (use kvc_decode_attn with a workspace)",
                             need, kScratchBytes);
  void* ws = nullptr;
  kvc_status st = scratch_of_current_device(&ws);
  if (st != KVC_OK) return st;
  // Every other check, and the zeroing of the error word where the chosen
  // kernel can set it, happens inside kvc_decode_attn before it enqueues
  // anything, so a call that fails launches nothing.
  return kvc_decode_attn(layout, cache, q, out, ws, kScratchBytes, stream);
}

extern "C" kvc_status kvc_static_error_word(uint32_t* dst, void* stream) {
  if (!dst) return kvc::report_error(KVC_EINVAL, "kvc_static_error_word: NULL dst");
  void* ws = nullptr;
  kvc_status st = scratch_of_current_device(&ws);
  if (st != KVC_OK) return st;
  cudaError_t e = cudaMemcpyAsync(dst, ws, sizeof(uint32_t), cudaMemcpyDefault,
                                  (cudaStream_t)stream);
  if (e != cudaSuccess)
    return kvc::report_error(KVC_ECUDA, "copying the scratch error word: %s",
                             cudaGetErrorString(e));
  return KVC_OK;
}
