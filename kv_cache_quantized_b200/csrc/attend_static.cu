// axr_attend_decode_static: axr_attend_decode for callers that cannot allocate device memory.
//
// Some callers of this library run where nothing may call cudaMalloc or any allocating routine at decode time:
// code that runs inside a memory pool it does not own, plugins handed only input and output pointers, or decode
// steps that must not touch the allocator at all.  For them this entry point keeps the split-T partials in a fixed
// device array owned by the library instead of a caller-provided workspace.  The array is a file-scope __device__
// variable of kStaticScratchBytes: every GPU that loads the library holds it until the process exits.
#include <mutex>

#include "axr_host.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(4) << 20;  // 4 MiB: the split partials of B*Hq*splits*(d+2) floats

static __device__ __align__(256) unsigned char g_attend_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the array on the current device.  In host code `g_attend_scratch` names a host-side stand-in,
// not device memory, so the address has to be looked up once per device with that device current.  The cached
// address belongs to the device's current context: after a cudaDeviceReset in the same process it is stale, and
// this entry point must not be called on that device again.
axr_status scratch_for_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return axr::set_error(AXR_ECUDA, "axr_attend_decode_static: cudaGetDevice: %s",
                                              cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices)
    return axr::set_error(AXR_EUNSUPPORTED, "axr_attend_decode_static: device %d beyond %d", dev, kMaxDevices);
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_attend_scratch);
    if (e != cudaSuccess || !p)
      return axr::set_error(AXR_ECUDA, "axr_attend_decode_static: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return AXR_OK;
}

}  // namespace

extern "C" size_t axr_attend_static_scratch_bytes(void) { return kStaticScratchBytes; }

extern "C" axr_status axr_attend_decode_static(const float* q, const uint8_t* kcodes, const uint16_t* knorms,
                                               axr_vkind vkind, const void* v, const uint16_t* vnorms,
                                               const int32_t* seq_lens, int B, int Hq, int Hkv, int T, int Tcap,
                                               int d, int bits, const int8_t* signs, float scale, float* out,
                                               void* stream) {
  const size_t need = axr_attend_workspace_bytes(B, Hq, Hkv, T, d);
  if (need > kStaticScratchBytes)
    return axr::set_error(AXR_EWORKSPACE,
                          "axr_attend_decode_static: these sizes need %zu bytes of scratch, above the fixed %zu; "
                          "use axr_attend_decode with a caller workspace",
                          need, kStaticScratchBytes);
  void* scratch = nullptr;
  axr_status st = scratch_for_current_device(&scratch);
  if (st != AXR_OK) return st;
  // Every partial slot the merge reads is written by the same call first, so nothing needs clearing.
  return axr_attend_decode(q, kcodes, knorms, vkind, v, vnorms, seq_lens, B, Hq, Hkv, T, Tcap, d, bits, signs,
                           scale, out, scratch, kStaticScratchBytes, stream);
}
