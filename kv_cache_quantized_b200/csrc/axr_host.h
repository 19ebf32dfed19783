// Host-side argument checks and launch plumbing shared by the axr entry points.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "axr_common.cuh"

namespace axr {

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// Report a launch failure (if any) of the kernels queued just before.
inline axr_status check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(AXR_ECUDA, "%s: %s", what, cudaGetErrorString(e));
  return set_error(AXR_OK, "");
}

inline bool supported_g(int G) { return G == 1 || G == 2 || G == 4 || G == 8; }

// Split of the token axis for the decode kernels: the number of token chunks per (batch, KV head) and the chunk
// length.  Depends only on the sizes, so a workspace sized by axr_attend_workspace_bytes always fits.
struct SplitPlan {
  int splits;
  int chunk;  // tokens per split, a multiple of kTile
};

constexpr int kTile = 256;          // tokens scored per block iteration
constexpr int kSmCount = 148;       // B200
constexpr int kBlocksPerSm = 2;     // resident decode blocks per SM the plan aims to fill twice over
constexpr int kMinChunk = 1024;     // keep the per-block table build amortised

inline SplitPlan plan_splits(int B, int Hkv, int T) {
  SplitPlan p{1, kTile};
  if (T <= 0 || B <= 0 || Hkv <= 0) return p;
  const long units = static_cast<long>(B) * Hkv;
  const long target = 2L * kSmCount * kBlocksPerSm;
  long s = (target + units - 1) / units;
  const long max_s = (T + kMinChunk - 1) / kMinChunk;
  if (s > max_s) s = max_s;
  if (s < 1) s = 1;
  long chunk = (T + s - 1) / s;
  chunk = (chunk + kTile - 1) / kTile * kTile;
  p.chunk = static_cast<int>(chunk);
  p.splits = static_cast<int>((T + chunk - 1) / chunk);
  return p;
}

inline size_t attend_ws_bytes(int B, int Hq, int Hkv, int T, int d) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || T <= 0 || d <= 0) return 0;
  const SplitPlan p = plan_splits(B, Hkv, T);
  const size_t parts = static_cast<size_t>(B) * Hq * p.splits;
  size_t bytes = parts * static_cast<size_t>(d) * sizeof(float) + 2 * parts * sizeof(float);
  return (bytes + 255) / 256 * 256;
}

}  // namespace axr
