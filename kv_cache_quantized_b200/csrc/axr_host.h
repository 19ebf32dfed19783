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

// The plan of the streaming kernels (per-warp workers over 32-token tiles): chunks of at least 2 tiles, and a setup
// of about two tiles (a worker transforms its queries and fills its copy ring before its first tile), so that small
// problems spread over many workers.  The dense fp16 kernel runs 4 workers per SM, the kernel for quantized keys
// over fp16 values 8.
constexpr int kStreamTile = 32;
constexpr int kDenseWorkers = 4 * kSmCount;
constexpr int kAttendStreamWorkers = 8 * kSmCount;   // fp16 values
constexpr int kAttendStreamWorkersQ = 16 * kSmCount; // quantized values
inline SplitPlan plan_splits_stream(int B, int Hkv, int T, int workers) {
  return plan_splits(B, Hkv, T, workers, kStreamTile, 2, 2.0);
}

inline size_t attend_ws_bytes(int B, int Hq, int Hkv, int T, int d) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || T <= 0 || d <= 0) return 0;
  // the largest split count of the plans (the kernels that may run on this workspace)
  int splits = plan_splits(B, Hkv, T).splits;
  for (int workers : {kDenseWorkers, kAttendStreamWorkers, kAttendStreamWorkersQ}) {
    const int s = plan_splits_stream(B, Hkv, T, workers).splits;
    splits = s > splits ? s : splits;
  }
  const size_t parts = static_cast<size_t>(B) * Hq * splits;
  size_t bytes = parts * static_cast<size_t>(d) * sizeof(float) + 2 * parts * sizeof(float);
  return (bytes + 255) / 256 * 256;
}

}  // namespace axr
