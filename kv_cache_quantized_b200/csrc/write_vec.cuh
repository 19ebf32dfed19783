// The write path for one vector, shared by the writer kernels and the decode-step prologue: rotate + normalise +
// quantize with one warp, then pack.
//
// AXELRAM Key Points (2nd item) and Abstract: "transform on write" into the domain where the fixed design-time
// codebook applies.  Transform here: sign flip s .* x, then the Walsh-Hadamard butterfly (Sylvester order) held in
// registers across the warp; norm ||x|| in fp32; index = number of thresholds at or below the unit coordinate;
// codes packed as an LSB-first bitstream (coordinate j at bits [j b, j b + b)).
#pragma once

#include "axr_common.cuh"

namespace axr {

template <typename TIn, int VPL>
__device__ __forceinline__ void load_lane(const TIn* row, int lane, float (&v)[VPL]);

template <>
__device__ __forceinline__ void load_lane<float, 4>(const float* row, int lane, float (&v)[4]) {
  float4 a = reinterpret_cast<const float4*>(row)[lane];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
}
template <>
__device__ __forceinline__ void load_lane<float, 2>(const float* row, int lane, float (&v)[2]) {
  float2 a = reinterpret_cast<const float2*>(row)[lane];
  v[0] = a.x; v[1] = a.y;
}
template <>
__device__ __forceinline__ void load_lane<float, 1>(const float* row, int lane, float (&v)[1]) {
  v[0] = row[lane];
}
template <>
__device__ __forceinline__ void load_lane<__half, 4>(const __half* row, int lane, float (&v)[4]) {
  uint2 a = reinterpret_cast<const uint2*>(row)[lane];
  float2 lo = __half22float2(*reinterpret_cast<__half2*>(&a.x));
  float2 hi = __half22float2(*reinterpret_cast<__half2*>(&a.y));
  v[0] = lo.x; v[1] = lo.y; v[2] = hi.x; v[3] = hi.y;
}
template <>
__device__ __forceinline__ void load_lane<__half, 2>(const __half* row, int lane, float (&v)[2]) {
  float2 a = __half22float2(reinterpret_cast<const __half2*>(row)[lane]);
  v[0] = a.x; v[1] = a.y;
}
template <>
__device__ __forceinline__ void load_lane<__half, 1>(const __half* row, int lane, float (&v)[1]) {
  v[0] = __half2float(row[lane]);
}

// Codes of one vector into idx (shared memory, one byte per coordinate); returns ||x||.  Whole warp.
template <int D, int BITS, typename TIn>
__device__ __forceinline__ float quantize_vector(const TIn* __restrict__ xrow, const float (&sg)[WarpVec<D>::VPL],
                                                 const float (&tau)[(1 << BITS) - 1], int lane, uint8_t* idx) {
  constexpr int VPL = WarpVec<D>::VPL;
  constexpr int LANES = WarpVec<D>::LANES;
  constexpr int L = 1 << BITS;
  const bool active = lane < LANES;
  float v[VPL];
  if (active) {
    load_lane<TIn, VPL>(xrow, lane, v);
  } else {
#pragma unroll
    for (int i = 0; i < VPL; ++i) v[i] = 0.0f;
  }
  float ss = 0.0f;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    ss = fmaf(v[i], v[i], ss);
    v[i] *= sg[i];
  }
  ss = warp_sum(ss);
  const float n = sqrtf(ss);
  fwht_warp<D>(v, lane);  // v = FWHT(s .* x) = sqrt(D) * H (s .* x)
  if (active) {
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const float w = n > 0.0f ? v[i] / n : 0.0f;  // = sqrt(D) * u
      int q = 0;
#pragma unroll
      for (int k = 0; k < L - 1; ++k) q += (w >= tau[k]) ? 1 : 0;
      idx[lane * VPL + i] = static_cast<uint8_t>(q);
    }
  }
  return n;
}

// Pack the D codes idx[0 .. D) of one vector into its R = D b / 8 bytes at out (LSB-first).  Whole warp.
template <int D, int BITS>
__device__ __forceinline__ void pack_row(const uint8_t* __restrict__ idx, uint8_t* __restrict__ out, int lane) {
  constexpr int R = D * BITS / 8;
  for (int byte = lane; byte < R; byte += kWarp) {
    uint32_t acc = 0;
    const int first = (byte * 8) / BITS, last = (byte * 8 + 7) / BITS;
    for (int j = first; j <= last && j < D; ++j) {
      const int pos = j * BITS - byte * 8;  // bit offset of coordinate j relative to this byte (may be < 0)
      const uint32_t code = idx[j];
      acc |= pos >= 0 ? (code << pos) : (code >> (-pos));
    }
    out[byte] = static_cast<uint8_t>(acc & 0xffu);
  }
}

}  // namespace axr
