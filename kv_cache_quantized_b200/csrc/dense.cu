// Launcher of the dense fp16 decode kernel (dense_stream.cuh), the bandwidth reference, and its split merge.
#include <cudaTypedefs.h>

#include <mutex>

#include "dense_stream.cuh"
#include "launch.h"

namespace axr {
namespace {

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime (no link against libcuda)
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

}  // namespace

// 2-D map over an fp16 cache viewed as [rows, D]: boxes of `box_rows` rows x 64 coordinates, 128-byte swizzle.
axr_status encode_cache_map(CUtensorMap* map, const void* base, size_t rows, int D, int box_rows, const char* what) {
  auto fn = encode_fn();
  if (!fn) return set_error(AXR_ECUDA, "%s: cuTensorMapEncodeTiled unavailable", what);
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
  const cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1u, 1u};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(AXR_ECUDA, "%s: cuTensorMapEncodeTiled failed (%d)", what, (int)r);
  return AXR_OK;
}

namespace {

template <int D, int G>
axr_status launch(const DecodeArgs& a, cudaStream_t st, const char* what) {
  using P = DenseStreamPlan<D, G>;
  static_assert(P::WARPS * kSmCount == kDenseWorkers && P::TW == kStreamTile, "the split plan's worker model");
  auto k = dense_stream_kernel<D, G>;
  axr_status rs = ensure_smem(k, P::bytes, what);
  if (rs != AXR_OK) return rs;
  const size_t rows = static_cast<size_t>(a.B) * a.Hkv * a.Tcap;  // TMA row coordinates are 32-bit
  if (rows + P::TW >= (static_cast<size_t>(1) << 31))
    return set_error(AXR_EUNSUPPORTED, "%s: %zu cache rows exceed the 2^31 a TMA coordinate addresses", what, rows);
  CUtensorMap kmap, vmap;
  if ((rs = encode_cache_map(&kmap, a.kdense, rows, D, P::TW, what)) != AXR_OK) return rs;
  if ((rs = encode_cache_map(&vmap, a.v, rows, D, P::TW, what)) != AXR_OK) return rs;
  const long items = static_cast<long>(a.B) * a.Hkv * a.splits;  // one per warp worker, dealt across the blocks
  const unsigned grid = static_cast<unsigned>(items < kSmCount ? items : kSmCount);
  k<<<grid, P::THREADS, P::bytes, st>>>(a, kmap, vmap);
  launch_reduce<D, false>(a, st);
  return check_launch(what);
}

template <int D>
axr_status by_g(int G, const DecodeArgs& a, cudaStream_t st, const char* w) {
  switch (G) {
    case 1: return launch<D, 1>(a, st, w);
    case 2: return launch<D, 2>(a, st, w);
    case 4: return launch<D, 4>(a, st, w);
    case 8: return launch<D, 8>(a, st, w);
  }
  return set_error(AXR_EUNSUPPORTED, "%s: G=%d", w, G);
}

}  // namespace

axr_status dense_launch(int d, int G, const DecodeArgs& a, cudaStream_t st, const char* what) {
  if (d == 64) return by_g<64>(G, a, st, what);
  if (d == 128) return by_g<128>(G, a, st, what);
  return set_error(AXR_EUNSUPPORTED, "%s: d=%d", what, d);
}

}  // namespace axr
