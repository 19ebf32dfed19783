// Launcher of the fused per-warp decode kernel (attend_fused.cuh).
#include "attend_fused.cuh"
#include "launch.h"

namespace axr {
namespace {

template <int D, int BITS, int G, bool VQ>
axr_status launch(const DecodeArgs& a, cudaStream_t st) {
  using S = FusedPlan<D, BITS, G, VQ>;
  auto k1 = attend_fused_kernel<D, BITS, G, VQ>;
  axr_status rs = ensure_smem(k1, S::bytes, "axr_attend_decode");
  if (rs != AXR_OK) return rs;
  const long items = static_cast<long>(a.B) * a.Hkv * a.splits;  // persistent: one block per SM
  k1<<<static_cast<unsigned>(items < kSmCount ? items : kSmCount), S::THREADS, S::bytes, st>>>(a);
  launch_reduce<D, VQ>(a, st);
  return check_launch("axr_attend_decode");
}

template <int D, int BITS>
axr_status by_g(int G, bool vq, const DecodeArgs& a, cudaStream_t st) {
  switch (G) {
    case 1: return vq ? launch<D, BITS, 1, true>(a, st) : launch<D, BITS, 1, false>(a, st);
    case 2: return vq ? launch<D, BITS, 2, true>(a, st) : launch<D, BITS, 2, false>(a, st);
    case 4: return vq ? launch<D, BITS, 4, true>(a, st) : launch<D, BITS, 4, false>(a, st);
    case 8: return vq ? launch<D, BITS, 8, true>(a, st) : launch<D, BITS, 8, false>(a, st);
  }
  return set_error(AXR_EUNSUPPORTED, "axr_attend_decode: G=%d", G);
}

}  // namespace

bool attend_fused_supported(int d, int bits) { return d * bits % 128 == 0; }  // rows of whole 16-byte chunks

axr_status attend_fused_launch(int d, int bits, int G, bool vq, const DecodeArgs& a, cudaStream_t st) {
  if (d == 128) {
    switch (bits) {
      case 1: return by_g<128, 1>(G, vq, a, st);
      case 2: return by_g<128, 2>(G, vq, a, st);
      case 3: return by_g<128, 3>(G, vq, a, st);
      case 4: return by_g<128, 4>(G, vq, a, st);
    }
  } else if (d == 64) {
    switch (bits) {
      case 2: return by_g<64, 2>(G, vq, a, st);
      case 4: return by_g<64, 4>(G, vq, a, st);
    }
  }
  return set_error(AXR_EUNSUPPORTED, "axr_attend_decode: fused kernel for d=%d bits=%d", d, bits);
}

}  // namespace axr
