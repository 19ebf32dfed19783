// Dispatch of the row-layout decode kernel (attend_rows.cuh) over its compile-time sizes; included by the two
// translation units that instantiate it, one for contiguous caches and one for paged pools.
#pragma once

#include "attend_rows.cuh"
#include "launch.h"

namespace axr {
namespace rows_detail {

// The C entry point a launch serves, for error messages: decode steps carry the new token.
inline const char* entry_name(const DecodeArgs& a) { return a.knew != nullptr ? "axr_decode_step" : "axr_attend_decode"; }

template <int D, int BITS, int G, bool VQ, bool PAGED>
axr_status launch(const DecodeArgs& a, cudaStream_t st) {
  using S = RowsPlan<D, BITS, G, VQ>;
  auto k1 = attend_rows_kernel<D, BITS, G, VQ, PAGED>;
  const char* what = entry_name(a);
  axr_status rs = ensure_smem(k1, S::bytes, what);
  if (rs != AXR_OK) return rs;
  const long items = static_cast<long>(a.B) * a.Hkv * a.splits;  // persistent blocks loop over the items
  const long resident = static_cast<long>(S::MIN_BLOCKS) * kSmCount;
  k1<<<static_cast<unsigned>(items < resident ? items : resident), kDecThreads, S::bytes, st>>>(a);
  launch_reduce<D, VQ>(a, st);
  return check_launch(what);
}

template <int D, int BITS, bool PAGED>
axr_status by_g(int G, bool vq, const DecodeArgs& a, cudaStream_t st) {
  switch (G) {
    case 1: return vq ? launch<D, BITS, 1, true, PAGED>(a, st) : launch<D, BITS, 1, false, PAGED>(a, st);
    case 2: return vq ? launch<D, BITS, 2, true, PAGED>(a, st) : launch<D, BITS, 2, false, PAGED>(a, st);
    case 4: return vq ? launch<D, BITS, 4, true, PAGED>(a, st) : launch<D, BITS, 4, false, PAGED>(a, st);
    case 8: return vq ? launch<D, BITS, 8, true, PAGED>(a, st) : launch<D, BITS, 8, false, PAGED>(a, st);
  }
  return set_error(AXR_EUNSUPPORTED, "%s: G=%d", entry_name(a), G);
}

template <int D, bool PAGED>
axr_status by_bits(int bits, int G, bool vq, const DecodeArgs& a, cudaStream_t st) {
  switch (bits) {
    case 1: return by_g<D, 1, PAGED>(G, vq, a, st);
    case 2: return by_g<D, 2, PAGED>(G, vq, a, st);
    case 3: return by_g<D, 3, PAGED>(G, vq, a, st);
    case 4: return by_g<D, 4, PAGED>(G, vq, a, st);
  }
  return set_error(AXR_EUNSUPPORTED, "%s: bits=%d", entry_name(a), bits);
}

template <bool PAGED>
axr_status dispatch(int d, int bits, int G, bool vq, const DecodeArgs& a, cudaStream_t st) {
  if (d == 64) return by_bits<64, PAGED>(bits, G, vq, a, st);
  if (d == 128) return by_bits<128, PAGED>(bits, G, vq, a, st);
  return set_error(AXR_EUNSUPPORTED, "%s: d=%d", entry_name(a), d);
}

}  // namespace rows_detail
}  // namespace axr
