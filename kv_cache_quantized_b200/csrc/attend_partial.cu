// Launcher of the CUDA-core row-layout decode kernel (attend_partial_kernel in decode.cuh): quantized keys through
// the factored gather.
#include "launch.h"

namespace axr {
namespace {

template <int D, int BITS, int G, bool VQ>
axr_status launch(const DecodeArgs& a, cudaStream_t st, const char* what) {
  using S = DecPlan<D, BITS, G, VQ>;
  auto k1 = attend_partial_kernel<D, BITS, G, VQ>;
  axr_status rs = ensure_smem(k1, S::bytes, what);
  if (rs != AXR_OK) return rs;
  const long items = static_cast<long>(a.B) * a.Hkv * a.splits;  // persistent blocks loop over the items
  const long resident = static_cast<long>(S::MIN_BLOCKS) * kSmCount;
  const unsigned grid = static_cast<unsigned>(items < resident ? items : resident);
  k1<<<grid, kDecThreads, S::bytes, st>>>(a);
  launch_reduce<D, VQ>(a, st);
  return check_launch(what);
}

template <int D, int BITS>
axr_status by_g(int G, bool vq, const DecodeArgs& a, cudaStream_t st, const char* w) {
  switch (G) {
    case 1: return vq ? launch<D, BITS, 1, true>(a, st, w) : launch<D, BITS, 1, false>(a, st, w);
    case 2: return vq ? launch<D, BITS, 2, true>(a, st, w) : launch<D, BITS, 2, false>(a, st, w);
    case 4: return vq ? launch<D, BITS, 4, true>(a, st, w) : launch<D, BITS, 4, false>(a, st, w);
    case 8: return vq ? launch<D, BITS, 8, true>(a, st, w) : launch<D, BITS, 8, false>(a, st, w);
  }
  return set_error(AXR_EUNSUPPORTED, "%s: G=%d", w, G);
}

template <int D>
axr_status by_bits(int bits, int G, bool vq, const DecodeArgs& a, cudaStream_t st, const char* w) {
  switch (bits) {
    case 1: return by_g<D, 1>(G, vq, a, st, w);
    case 2: return by_g<D, 2>(G, vq, a, st, w);
    case 3: return by_g<D, 3>(G, vq, a, st, w);
    case 4: return by_g<D, 4>(G, vq, a, st, w);
  }
  return set_error(AXR_EUNSUPPORTED, "%s: bits=%d", w, bits);
}

}  // namespace

axr_status attend_partial_launch(int d, int bits, int G, bool vq, const DecodeArgs& a, cudaStream_t st,
                                 const char* what) {
  if (d != 64 && d != 128) return set_error(AXR_EUNSUPPORTED, "%s: d=%d", what, d);
  return d == 64 ? by_bits<64>(bits, G, vq, a, st, what) : by_bits<128>(bits, G, vq, a, st, what);
}

}  // namespace axr
