// Launcher of the streaming decode kernel for quantized keys over fp16 or quantized values (attend_stream.cuh) and
// its split merge (with the one inverse transform for quantized values).
#include <cstring>

#include "attend_stream.cuh"
#include "launch.h"

namespace axr {
namespace {

template <int D, int BITS, int G, bool VQ, bool PAGED = false>
axr_status launch(const DecodeArgs& a, cudaStream_t st, const char* what) {
  using P = StreamPlan<D, BITS, G, VQ>;
  static_assert(P::WARPS * kSmCount == (VQ ? kAttendStreamWorkersQ : kAttendStreamWorkers) && P::TW == kStreamTile,
                "the split plan's worker model");
  static_assert(!PAGED || VQ, "paged pools with quantized values only");
  auto k = attend_stream_kernel<D, BITS, G, VQ, PAGED>;
  axr_status rs = ensure_smem(k, P::bytes, what);
  if (rs != AXR_OK) return rs;
  const size_t rows = static_cast<size_t>(a.B) * a.Hkv * a.Tcap;  // TMA row coordinates are 32-bit
  if (rows + P::TW >= (static_cast<size_t>(1) << 31))
    return set_error(AXR_EUNSUPPORTED, "%s: %zu cache rows exceed the 2^31 a TMA coordinate addresses", what, rows);
  CUtensorMap vmap;
  memset(&vmap, 0, sizeof(vmap));
  if (!VQ && (rs = encode_cache_map(&vmap, a.v, rows, D, P::TW, what)) != AXR_OK) return rs;
  const long items = static_cast<long>(a.B) * a.Hkv * a.splits;  // one per warp worker, dealt across the blocks
  const unsigned grid = static_cast<unsigned>(items < kSmCount ? items : kSmCount);
  k<<<grid, P::THREADS, P::bytes, st>>>(a, vmap);
  launch_reduce<D, VQ>(a, st);
  return check_launch(what);
}

template <int D, int BITS>
axr_status by_g(int G, bool vq, const DecodeArgs& a, cudaStream_t st, const char* w) {
  if (a.block_table) {  // paged pools (quantized values, blocks of at least kStreamTile tokens)
    if (!vq || (1 << a.block_shift) < kStreamTile)
      return set_error(AXR_EUNSUPPORTED, "%s: the streaming kernel's paged pools take quantized values in blocks of "
                       "at least %d tokens", w, kStreamTile);
    switch (G) {
      case 1: return launch<D, BITS, 1, true, true>(a, st, w);
      case 2: return launch<D, BITS, 2, true, true>(a, st, w);
      case 4: return launch<D, BITS, 4, true, true>(a, st, w);
      case 8: return launch<D, BITS, 8, true, true>(a, st, w);
    }
    return set_error(AXR_EUNSUPPORTED, "%s: G=%d", w, G);
  }
  switch (G) {
    case 1: return vq ? launch<D, BITS, 1, true>(a, st, w) : launch<D, BITS, 1, false>(a, st, w);
    case 2: return vq ? launch<D, BITS, 2, true>(a, st, w) : launch<D, BITS, 2, false>(a, st, w);
    case 4: return vq ? launch<D, BITS, 4, true>(a, st, w) : launch<D, BITS, 4, false>(a, st, w);
    case 8: return vq ? launch<D, BITS, 8, true>(a, st, w) : launch<D, BITS, 8, false>(a, st, w);
  }
  return set_error(AXR_EUNSUPPORTED, "%s: G=%d", w, G);
}

}  // namespace

// Code rows of whole 16-byte chunks, or (d = 64, b = 1, 3: rows of 8 or 24 bytes) an even capacity, so that every
// (batch row, KV head) starts on a 16-byte boundary and a tile's rows, rounded up to an even count, stay inside it.
bool attend_stream_supported(int d, int bits, int Tcap) {
  if (d == 128) return bits >= 1 && bits <= 4;
  return d == 64 && bits >= 1 && bits <= 4 && (d * bits % 128 == 0 || Tcap % 2 == 0);
}

axr_status attend_stream_launch(int d, int bits, int G, bool vq, const DecodeArgs& a, cudaStream_t st,
                                const char* what) {
  if (d == 128) {
    switch (bits) {
      case 1: return by_g<128, 1>(G, vq, a, st, what);
      case 2: return by_g<128, 2>(G, vq, a, st, what);
      case 3: return by_g<128, 3>(G, vq, a, st, what);
      case 4: return by_g<128, 4>(G, vq, a, st, what);
    }
  } else if (d == 64) {
    switch (bits) {
      case 1: return by_g<64, 1>(G, vq, a, st, what);
      case 2: return by_g<64, 2>(G, vq, a, st, what);
      case 3: return by_g<64, 3>(G, vq, a, st, what);
      case 4: return by_g<64, 4>(G, vq, a, st, what);
    }
  }
  return set_error(AXR_EUNSUPPORTED, "%s: d=%d bits=%d", what, d, bits);
}

}  // namespace axr
