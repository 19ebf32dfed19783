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

// Device address of the current device's status word (status.cu), or null if it could not be looked up.
unsigned int* status_word();

// Split of the token axis for the decode kernels: the number of token chunks per (batch, KV head) and the chunk
// length.  Depends only on the sizes, so a workspace sized by axr_attend_workspace_bytes always fits.
struct SplitPlan {
  int splits;
  int chunk;  // tokens per split, a multiple of kTile
};

constexpr int kTile = 128;          // tokens per decode tile; chunks are whole tiles
constexpr int kSmCount = 148;       // B200
constexpr int kResident = 2 * kSmCount;  // decode blocks resident at once (two per SM)
constexpr int kMinTiles = 4;        // smallest chunk, in tiles, so per-item setup stays amortised

// Choose the split count that minimises the makespan of a persistent decode kernel: the items (one per batch row,
// KV head and split) are dealt round-robin to `resident` workers, so the time is about ceil(items / resident) chunks
// of `tile`-token tiles plus a per-item setup of `setup` tiles.  Chunks are whole tiles, at least `min_tiles` long.
inline SplitPlan plan_splits(int B, int Hkv, int T, long resident = kResident, int tile = kTile,
                             int min_tiles = kMinTiles, double setup = 0.5) {
  SplitPlan p{1, tile};
  if (T <= 0 || B <= 0 || Hkv <= 0) return p;
  const long units = static_cast<long>(B) * Hkv;
  const long tiles_total = (T + tile - 1) / tile;
  long max_s = tiles_total / min_tiles;
  if (max_s < 1) max_s = 1;
  if (max_s > 4096) max_s = 4096;
  double best = 1e300;
  for (long s = 1; s <= max_s; ++s) {
    const long tiles = (tiles_total + s - 1) / s;
    const long splits = (tiles_total + tiles - 1) / tiles;
    const long rounds = (units * splits + resident - 1) / resident;
    const double cost = static_cast<double>(rounds) * (static_cast<double>(tiles) + setup);
    if (cost < best - 1e-9) {
      best = cost;
      p.chunk = static_cast<int>(tiles * tile);
      p.splits = static_cast<int>(splits);
    }
  }
  return p;
}

// The dense fp16 kernel's plan: one worker per warp (4 per SM), 32-token tiles, chunks of at least 8 tiles, and a
// setup of about one tile (the worker's copy ring fills before its first tile).
constexpr int kDenseWorkers = 4 * kSmCount;
constexpr int kDenseTile = 32;
inline SplitPlan plan_splits_dense(int B, int Hkv, int T) {
  return plan_splits(B, Hkv, T, kDenseWorkers, kDenseTile, 8, 1.0);
}

inline size_t attend_ws_bytes(int B, int Hq, int Hkv, int T, int d) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || T <= 0 || d <= 0) return 0;
  const SplitPlan p = plan_splits(B, Hkv, T), pd = plan_splits_dense(B, Hkv, T);
  const size_t parts = static_cast<size_t>(B) * Hq * (p.splits > pd.splits ? p.splits : pd.splits);
  size_t bytes = parts * static_cast<size_t>(d) * sizeof(float) + 2 * parts * sizeof(float);
  return (bytes + 255) / 256 * 256;
}

}  // namespace axr
