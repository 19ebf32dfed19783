// Launcher of the tcgen05 scores-only kernel (score_tc.cuh).
#include "launch.h"
#include "score_tc.cuh"

namespace axr {
namespace {

template <int D, int BITS, int G>
axr_status launch(const DecodeArgs& a, cudaStream_t st) {
  using S = TcScorePlan<D, BITS, G>;
  auto k = score_tc_kernel<D, BITS, G>;
  axr_status rs = ensure_smem(k, S::launch_bytes, "axr_score");
  if (rs != AXR_OK) return rs;
  // one persistent CTA per SM, each taking a contiguous share of the tiles (at most as many CTAs as tiles)
  const long tiles = static_cast<long>(a.B) * a.Hkv * ((a.T + kTile - 1) / kTile);
  const unsigned grid = static_cast<unsigned>(tiles < kSmCount ? tiles : kSmCount);
  k<<<grid, S::THREADS, S::launch_bytes, st>>>(a);
  return check_launch("axr_score");
}

template <int D, int BITS>
axr_status by_g(int G, const DecodeArgs& a, cudaStream_t st) {
  switch (G) {
    case 1: return launch<D, BITS, 1>(a, st);
    case 2: return launch<D, BITS, 2>(a, st);
    case 4: return launch<D, BITS, 4>(a, st);
    case 8: return launch<D, BITS, 8>(a, st);
  }
  return set_error(AXR_EUNSUPPORTED, "axr_score: G=%d", G);
}

template <int D>
axr_status by_bits(int bits, int G, const DecodeArgs& a, cudaStream_t st) {
  switch (bits) {
    case 1: return by_g<D, 1>(G, a, st);
    case 2: return by_g<D, 2>(G, a, st);
    case 3: return by_g<D, 3>(G, a, st);
    case 4: return by_g<D, 4>(G, a, st);
  }
  return set_error(AXR_EUNSUPPORTED, "axr_score: bits=%d", bits);
}

}  // namespace

axr_status score_tc_launch(int d, int bits, int G, const DecodeArgs& a, cudaStream_t st) {
  if (d == 64) return by_bits<64>(bits, G, a, st);
  if (d == 128) return by_bits<128>(bits, G, a, st);
  return set_error(AXR_EUNSUPPORTED, "axr_score: d=%d", d);
}

}  // namespace axr
