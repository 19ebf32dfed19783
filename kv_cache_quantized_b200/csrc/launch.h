// Host launchers of the decode kernel families.  Each family is compiled in a translation unit of its own (they
// hold many template instances) and exposes one dispatcher over its runtime sizes; decode.cu validates the
// arguments and picks the family.
#pragma once

#include <cuda.h>

#include "decode.cuh"

namespace axr {

// Raise the dynamic shared-memory limit of `kernel` to `bytes` when it is above the default 48 KB.
template <typename K>
axr_status ensure_smem(K kernel, size_t bytes, const char* what) {
  if (bytes > 48 * 1024) {  // idempotent, and per device: set before every launch
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return set_error(AXR_ECUDA, "%s: cudaFuncSetAttribute: %s", what, cudaGetErrorString(e));
  }
  return AXR_OK;
}

// The split merge after a decode kernel, launched as its programmatic dependent: its blocks are scheduled as the
// decode kernel's blocks retire and wait (griddepcontrol.wait) for that grid's completion and memory flush before
// reading the partials, so the launch latency overlaps the decode kernel's tail.  Without programmatic launches in
// the stream (e.g. an older driver) the wait returns at once and ordinary stream order holds.
template <int D, bool VQ, bool EXACT = false>
void launch_reduce(const DecodeArgs& a, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(a.B * a.Hq));
  cfg.blockDim = dim3(D);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, attend_reduce_kernel<D, VQ, EXACT>, a);
}

// Row-layout cache, quantized keys scored through warp-level MMAs (attend_rows.cu); vq: values quantized.
axr_status attend_rows_launch(int d, int bits, int G, bool vq, const DecodeArgs& a, cudaStream_t st);

// Row-layout cache on CUDA cores (attend_partial.cu): quantized keys through the factored gather.
axr_status attend_partial_launch(int d, int bits, int G, bool vq, const DecodeArgs& a, cudaStream_t st,
                                 const char* what);

// 2-D TMA map over an fp16 cache viewed as [rows, D]: boxes of `box_rows` rows x 64 coordinates, 128-byte swizzle
// (dense.cu).
axr_status encode_cache_map(CUtensorMap* map, const void* base, size_t rows, int D, int box_rows, const char* what);

// Quantized keys over fp16 (vq false) or quantized row-layout values on contiguous caches, as a stream of per-warp
// workers (attend_stream.cu); decode steps included.  Code rows of whole 16-byte chunks, or an even capacity
// (attend_stream_supported); the arguments carry the plan_splits_stream split plan for its worker count.
bool attend_stream_supported(int d, int bits, int Tcap);
axr_status attend_stream_launch(int d, int bits, int G, bool vq, const DecodeArgs& a, cudaStream_t st,
                                const char* what);

// Unquantized fp16 keys and values (dense.cu): the dense bandwidth reference, one streaming worker per warp; the
// arguments carry the plan_splits_stream split plan for kDenseWorkers.
axr_status dense_launch(int d, int G, const DecodeArgs& a, cudaStream_t st, const char* what);

// Tiled value layout, d = 128 (attend_tiled.cu): tcgen05 kernel if tensor, else warp-level MMAs.
axr_status attend_tiled_launch(int bits, int G, bool tensor, const DecodeArgs& a, cudaStream_t st);

// Scores only (score.cu): mode is one of kGatherFactored, kGatherMma, kGatherDirect (kGatherTable: lut.cu).
axr_status score_launch(int d, int bits, int G, int mode, const DecodeArgs& a, cudaStream_t st);

// The literal table in shared memory (lut.cu): multi-coordinate fields, G-wide entries; scores, and attend over
// fp16 values.
axr_status table_score_launch(int d, int bits, int G, const DecodeArgs& a, cudaStream_t st);
axr_status table_attend_launch(int d, int bits, int G, const DecodeArgs& a, cudaStream_t st);

// Scores only on the tcgen05 tensor cores (score_tc.cu).
axr_status score_tc_launch(int d, int bits, int G, const DecodeArgs& a, cudaStream_t st);

}  // namespace axr
