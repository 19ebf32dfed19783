// Decode step: the new token's key and value go into the cache through the write path, inside the decode launch.
//
// AXELRAM Key Points (2nd item) and Abstract: each new key (and value, when values are quantized) is transformed on
// write -- sign flip, Walsh-Hadamard rotation, norm, Lloyd-Max indices packed LSB-first -- exactly as the writer
// kernels do (write_vec.cuh); fp16 values are stored as they are.
#pragma once

#include "decode.cuh"
#include "write_vec.cuh"

namespace axr {

// One warp writes the new token's key (which == 0) or value (which == 1) at cache row `row` ([B, Hkv, Tcap]
// numbering): codes and fp16 norm, or the fp16 value.  No fence: the caller orders the writes against the reads that
// follow.
template <int D, int BITS, bool VQ>
__device__ __forceinline__ void append_row(const DecodeArgs& a, int b, int hk, size_t row, int which, int lane,
                                           uint8_t* idx_scratch) {
  constexpr int VPL = WarpVec<D>::VPL, LANES = WarpVec<D>::LANES, L = 1 << BITS, R = D * BITS / 8;
  const __half* src = (which == 0 ? a.knew : a.vnew) + (static_cast<size_t>(b) * a.Hkv + hk) * D;
  if (which == 1 && !VQ) {  // fp16 values are stored as they are
    __half* dst = static_cast<__half*>(const_cast<void*>(a.v)) + row * D;
    for (int j = lane; j < D; j += kWarp) dst[j] = src[j];
    return;
  }
  float sg[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) sg[i] = lane < LANES ? sign_of(a.signs[lane * VPL + i]) : 0.0f;
  float tau[L - 1];
#pragma unroll
  for (int k = 0; k < L - 1; ++k) tau[k] = a.cb.tau[k];
  const float n = quantize_vector<D, BITS, __half>(src, sg, tau, lane, idx_scratch);
  __syncwarp();
  uint8_t* codes = const_cast<uint8_t*>(which == 0 ? a.kcodes : static_cast<const uint8_t*>(a.v));
  __half* norms = const_cast<__half*>(which == 0 ? a.knorms : a.vnorms);
  pack_row<D, BITS>(idx_scratch, codes + row * R, lane);
  if (lane == 0) norms[row] = __float2half_rn(n);
}

}  // namespace axr
