// Shared device helpers of the axr library (sm_100a).  Nothing here is shared with the CPU oracle.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "axr.h"

namespace axr {

constexpr int kWarp = 32;
constexpr int kMaxLevels = 16;  // b <= 4

// Codebook constants handed to kernels by value (they land in the constant bank).
//   c[k]   unit-scale centroid gamma_k / sqrt(d), fp32, k < L
//   tau[k] N(0,1)-scale threshold between levels k and k+1 (k < L-1): the writer compares y/n against tau, where
//          y = FWHT(s .* x) is the unnormalised transform, which is the same decision as u = H(s.*x)/n >= tau/sqrt(d).
struct Codebook {
  float c[kMaxLevels];
  float tau[kMaxLevels];
  float gamma[kMaxLevels];  // N(0,1)-scale centroids gamma_k = sqrt(d) * c_k, fp32
};

// ---- host-side status plumbing (defined in api.cu) ----
axr_status set_error(axr_status st, const char* fmt, ...);
const Codebook* codebook_for(int d, int bits);  // cached; nullptr if unsupported

// ---- small device helpers ----
__device__ __forceinline__ float sign_of(int8_t s) { return s < 0 ? -1.0f : 1.0f; }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, m));
  return v;
}

// Packed fp32x2 add / fma (sm_100+): one issue slot for two IEEE round-to-nearest operations.
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  unsigned long long ra = *reinterpret_cast<unsigned long long*>(&a);
  unsigned long long rb = *reinterpret_cast<unsigned long long*>(&b);
  unsigned long long rd;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(rd) : "l"(ra), "l"(rb));
  return *reinterpret_cast<float2*>(&rd);
}

__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  unsigned long long ra = *reinterpret_cast<unsigned long long*>(&a);
  unsigned long long rb = *reinterpret_cast<unsigned long long*>(&b);
  unsigned long long rc = *reinterpret_cast<unsigned long long*>(&c);
  unsigned long long rd;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(rd) : "l"(ra), "l"(rb), "l"(rc));
  return *reinterpret_cast<float2*>(&rd);
}

// In-warp unnormalised Walsh-Hadamard transform (Sylvester order) of a length-D vector held VPL values per lane:
// lane l holds elements [l*VPL, l*VPL + VPL).  For D < 32 only lanes < D take part (VPL = 1); the others carry
// zeros and their results are ignored.  Butterfly (a, b) -> (a + b, a - b), lower index first.
template <int D>
struct WarpVec {
  static constexpr int VPL = D >= kWarp ? D / kWarp : 1;
  static constexpr int LANES = D >= kWarp ? kWarp : D;
};

template <int D>
__device__ __forceinline__ void fwht_warp(float (&v)[WarpVec<D>::VPL], int lane) {
  constexpr int VPL = WarpVec<D>::VPL;
  // stages inside a lane
#pragma unroll
  for (int h = 1; h < VPL; h <<= 1) {
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      if ((i & h) == 0) {
        float a = v[i], b = v[i + h];
        v[i] = a + b;
        v[i + h] = a - b;
      }
    }
  }
  // stages across lanes: element stride h = m * VPL for lane mask m
#pragma unroll
  for (int m = 1; m < WarpVec<D>::LANES; m <<= 1) {
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      float other = __shfl_xor_sync(0xffffffffu, v[i], m);
      v[i] = upper ? (other - v[i]) : (v[i] + other);
    }
  }
}

// Bit field [pos, pos+B) of a little-endian word array (pos, B compile-time after unrolling).
template <int B>
__device__ __forceinline__ uint32_t bits_at(const uint32_t* w, int pos) {
  const int wi = pos >> 5, sh = pos & 31;
  if (sh + B <= 32) return (w[wi] >> sh) & ((1u << B) - 1u);
  return __funnelshift_r(w[wi], w[wi + 1], sh) & ((1u << B) - 1u);
}

}  // namespace axr
