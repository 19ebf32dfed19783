// Launchers of the scores-only kernels on CUDA cores and warp-level MMAs (score_kernel in decode.cuh, score_mma.cuh).
#include "launch.h"
#include "score_direct.cuh"
#include "score_mma.cuh"

namespace axr {
namespace {

template <int D, int BITS, int G, int MODE>
axr_status launch_mode(const DecodeArgs& a, cudaStream_t st) {
  using S = ScorePlan<D, BITS, G, MODE>;
  auto k = score_kernel<D, BITS, G, MODE>;
  axr_status rs = ensure_smem(k, S::bytes, "axr_score");
  if (rs != AXR_OK) return rs;
  dim3 grid(a.splits, a.Hkv, a.B);
  k<<<grid, kDecThreads, S::bytes, st>>>(a);
  return check_launch("axr_score");
}

template <int D, int BITS, int G>
axr_status launch_mma(const DecodeArgs& a, cudaStream_t st) {
  using S = ScoreMmaPlan<D, BITS, G>;
  auto k = score_mma_kernel<D, BITS, G>;
  axr_status rs = ensure_smem(k, S::bytes, "axr_score");
  if (rs != AXR_OK) return rs;
  const long items = static_cast<long>(a.B) * a.Hkv * a.splits;  // persistent: two blocks per SM
  const long resident = 2L * kSmCount;
  k<<<static_cast<unsigned>(items < resident ? items : resident), S::THREADS, S::bytes, st>>>(a);
  return check_launch("axr_score");
}

// Chunk of the direct-load scorer's warp items: a multiple of 16 tokens minimising ceil(items / resident warps) x
// (chunk + per-item setup), so that the last round of items keeps most warps busy.
int direct_chunk(int B, int Hkv, int T, long resident_warps) {
  const long units = static_cast<long>(B) * Hkv;
  long best_chunk = 256;
  double best = 1e300;
  for (long chunk = 256; chunk < T + 16; chunk += 16) {
    const long items = units * ((T + chunk - 1) / chunk);
    const long rounds = (items + resident_warps - 1) / resident_warps;
    const double cost = static_cast<double>(rounds) * static_cast<double>(chunk + 96);
    if (cost < best - 1e-9) {
      best = cost;
      best_chunk = chunk;
    }
  }
  return static_cast<int>(best_chunk);
}

template <int D, int BITS, int G>
axr_status launch_direct(DecodeArgs a, cudaStream_t st) {
  using P = DirectPlan<D, BITS, G>;
  auto k = score_direct_kernel<D, BITS, G>;
  axr_status rs = ensure_smem(k, P::bytes, "axr_score");
  if (rs != AXR_OK) return rs;
  const long blocks = 2L * kSmCount;  // two resident blocks of 8 warps per SM
  a.chunk = direct_chunk(a.B, a.Hkv, a.T, blocks * P::WARPS);
  k<<<static_cast<unsigned>(blocks), P::THREADS, P::bytes, st>>>(a);
  return check_launch("axr_score");
}

template <int D, int BITS, int G>
axr_status launch(int mode, const DecodeArgs& a, cudaStream_t st) {
  if (mode == kGatherMma) return launch_mma<D, BITS, G>(a, st);
  if (mode == kGatherDirect) return launch_direct<D, BITS, G>(a, st);
  if (mode == kGatherTable) return launch_mode<D, BITS, G, kGatherTable>(a, st);
  if (mode == kGatherFactored) return launch_mode<D, BITS, G, kGatherFactored>(a, st);
  return set_error(AXR_EINVAL, "axr_score: gather mode %d", mode);
}

template <int D, int BITS>
axr_status by_g(int G, int mode, const DecodeArgs& a, cudaStream_t st) {
  switch (G) {
    case 1: return launch<D, BITS, 1>(mode, a, st);
    case 2: return launch<D, BITS, 2>(mode, a, st);
    case 4: return launch<D, BITS, 4>(mode, a, st);
    case 8: return launch<D, BITS, 8>(mode, a, st);
  }
  return set_error(AXR_EUNSUPPORTED, "axr_score: G=%d", G);
}

template <int D>
axr_status by_bits(int bits, int G, int mode, const DecodeArgs& a, cudaStream_t st) {
  switch (bits) {
    case 1: return by_g<D, 1>(G, mode, a, st);
    case 2: return by_g<D, 2>(G, mode, a, st);
    case 3: return by_g<D, 3>(G, mode, a, st);
    case 4: return by_g<D, 4>(G, mode, a, st);
  }
  return set_error(AXR_EUNSUPPORTED, "axr_score: bits=%d", bits);
}

}  // namespace

axr_status score_launch(int d, int bits, int G, int mode, const DecodeArgs& a, cudaStream_t st) {
  if (d == 64) return by_bits<64>(bits, G, mode, a, st);
  if (d == 128) return by_bits<128>(bits, G, mode, a, st);
  return set_error(AXR_EUNSUPPORTED, "axr_score: d=%d", d);
}

}  // namespace axr
