// The device status word: how a kernel whose bounded wait gave up tells the host.
//
// Every spin-wait in the decode and score kernels (on an mbarrier, or on a stage's arming) gives up after a bounded
// number of polls (about a second) so that a copy that never lands cannot hang the GPU.  A block that gave up
// writes NaN into its outputs and sets a bit in this word; axr_device_status reads (and optionally clears) it.  The
// word is a file-scope __device__ variable (zero at module load, one per device); kernels in other translation
// units get its device address through their launch arguments.
#include <mutex>

#include "axr_host.h"
#include "tc.cuh"

namespace {

static __device__ unsigned int g_status_word;

constexpr int kMaxDevices = 64;
std::mutex g_mu;
unsigned int* g_status_ptr[kMaxDevices] = {nullptr};

// One polling wait on an mbarrier that nothing arrives on and no copy completes, with a short poll limit: it gives
// up, records the timeout in the status word and returns (the library's own test of the give-up path).
__global__ void wait_timeout_selftest_kernel(unsigned int* status, int polls) {
  __shared__ __align__(8) uint64_t mbar;
  if (threadIdx.x == 0) axr::tc::mbar_init(&mbar, 1);
  __syncthreads();
  if (threadIdx.x == 0 && !axr::tc::mbar_wait_polls(&mbar, 0u, polls)) atomicOr(status, 1u);
}

}  // namespace

namespace axr {

unsigned int* status_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    g_status_ptr[dev] = static_cast<unsigned int*>(p);
  }
  return g_status_ptr[dev];
}

}  // namespace axr

extern "C" axr_status axr_device_status(unsigned int* flags, int clear) {
  using namespace axr;
  if (!flags) return set_error(AXR_EINVAL, "axr_device_status: null pointer");
  unsigned int* p = status_word();
  if (!p) return set_error(AXR_ECUDA, "axr_device_status: the status word has no device address");
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(flags, p, sizeof(unsigned int), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && clear && *flags) e = cudaMemset(p, 0, sizeof(unsigned int));
  if (e != cudaSuccess) return set_error(AXR_ECUDA, "axr_device_status: %s", cudaGetErrorString(e));
  if (*flags & AXR_STATUS_WAIT_TIMEOUT)
    return set_error(AXR_ECUDA,
                     "axr_device_status: a bounded wait in a kernel gave up (a copy or a stage did not arrive in "
                     "about a second); the outputs of the affected calls hold NaN");
  return set_error(AXR_OK, "");
}

extern "C" axr_status axr_selftest_wait_timeout(int polls, void* stream) {
  using namespace axr;
  if (polls < 1 || polls > (1 << 20)) return set_error(AXR_EINVAL, "axr_selftest_wait_timeout: polls=%d", polls);
  unsigned int* p = status_word();
  if (!p) return set_error(AXR_ECUDA, "axr_selftest_wait_timeout: the status word has no device address");
  wait_timeout_selftest_kernel<<<1, 32, 0, as_stream(stream)>>>(p, polls);
  return check_launch("axr_selftest_wait_timeout");
}
