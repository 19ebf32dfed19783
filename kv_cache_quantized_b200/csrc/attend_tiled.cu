// Launchers of the decode kernels for the tiled value layout (d = 128): the tcgen05 kernel (attend_tcv.cuh) and the
// warp-level MMA kernel (attend_mma.cuh).
#include "attend_mma.cuh"
#include "attend_tcv.cuh"
#include "launch.h"

namespace axr {
namespace {

template <int BITS, int G>
axr_status launch_tcv(const DecodeArgs& a, cudaStream_t st) {
  using S = TcaPlan<BITS, G>;
  auto k1 = attend_tcv_kernel<BITS, G>;
  axr_status rs = ensure_smem(k1, S::bytes, "axr_attend_decode");
  if (rs != AXR_OK) return rs;
  const long items = static_cast<long>(a.B) * a.Hkv * a.splits;  // persistent: one CTA per SM
  const unsigned grid = static_cast<unsigned>(items < kSmCount ? items : kSmCount);
  k1<<<grid, S::THREADS, S::bytes, st>>>(a);
  launch_reduce<128, true>(a, st);
  return check_launch("axr_attend_decode");
}

template <int BITS, int G>
axr_status launch_mma(const DecodeArgs& a, cudaStream_t st) {
  using S = MmaPlan<BITS, G>;
  auto k1 = attend_mma_kernel<BITS, G>;
  axr_status rs = ensure_smem(k1, S::bytes, "axr_attend_decode");
  if (rs != AXR_OK) return rs;
  const long items = static_cast<long>(a.B) * a.Hkv * a.splits;  // persistent blocks loop over the items
  const long resident = static_cast<long>(S::MIN_BLOCKS) * kSmCount;
  k1<<<static_cast<unsigned>(items < resident ? items : resident), kDecThreads, S::bytes, st>>>(a);
  launch_reduce<128, true>(a, st);
  return check_launch("axr_attend_decode");
}

template <int BITS>
axr_status by_g(int G, bool tensor, const DecodeArgs& a, cudaStream_t st) {
  switch (G) {
    case 1: return tensor ? launch_tcv<BITS, 1>(a, st) : launch_mma<BITS, 1>(a, st);
    case 2: return tensor ? launch_tcv<BITS, 2>(a, st) : launch_mma<BITS, 2>(a, st);
    case 4: return tensor ? launch_tcv<BITS, 4>(a, st) : launch_mma<BITS, 4>(a, st);
    case 8: return tensor ? launch_tcv<BITS, 8>(a, st) : launch_mma<BITS, 8>(a, st);
  }
  return set_error(AXR_EUNSUPPORTED, "axr_attend_decode: G=%d", G);
}

}  // namespace

axr_status attend_tiled_launch(int bits, int G, bool tensor, const DecodeArgs& a, cudaStream_t st) {
  switch (bits) {
    case 1: return by_g<1>(G, tensor, a, st);
    case 2: return by_g<2>(G, tensor, a, st);
    case 3: return by_g<3>(G, tensor, a, st);
    case 4: return by_g<4>(G, tensor, a, st);
  }
  return set_error(AXR_EUNSUPPORTED, "axr_attend_decode: bits=%d", bits);
}

}  // namespace axr
