// Write path: rotate + normalise + quantize + pack, one warp per vector.
//
// AXELRAM Key Points (2nd item) and Abstract: "transform on write" into the domain where the fixed design-time
// codebook applies.  Transform here: sign flip s .* x, then the Walsh-Hadamard butterfly (Sylvester order) held in
// registers across the warp; norm ||x|| in fp32; index = number of thresholds at or below the unit coordinate.
#include "axr_host.h"
#include "write_vec.cuh"

namespace axr {
namespace {

constexpr int kWriteWarps = 8;

template <int D, int BITS, typename TIn>
__global__ void __launch_bounds__(kWriteWarps * kWarp)
write_kernel(const TIn* __restrict__ x, int64_t n_vec, const int8_t* __restrict__ signs,
             const int64_t* __restrict__ dst_rows, uint8_t* __restrict__ codes, __half* __restrict__ norms,
             Codebook cb) {
  constexpr int VPL = WarpVec<D>::VPL;
  constexpr int LANES = WarpVec<D>::LANES;
  constexpr int L = 1 << BITS;
  constexpr int R = D * BITS / 8;  // bytes per packed row
  __shared__ uint8_t idx_s[kWriteWarps][D];

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const bool active = lane < LANES;
  float sg[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) sg[i] = active ? sign_of(signs[lane * VPL + i]) : 0.0f;
  float tau[L - 1];
#pragma unroll
  for (int k = 0; k < L - 1; ++k) tau[k] = cb.tau[k];

  for (int64_t vec = static_cast<int64_t>(blockIdx.x) * kWriteWarps + warp; vec < n_vec;
       vec += static_cast<int64_t>(gridDim.x) * kWriteWarps) {
    const float n = quantize_vector<D, BITS, TIn>(x + vec * D, sg, tau, lane, idx_s[warp]);
    __syncwarp();
    const int64_t row = dst_rows ? dst_rows[vec] : vec;
    pack_row<D, BITS>(idx_s[warp], codes + row * R, lane);
    if (lane == 0) norms[row] = __float2half_rn(n);
    __syncwarp();
  }
}

// ---- values in the tiled layout --------------------------------------------------------------------------------
//
// Layout: codes [B*Hkv][Tcap/128][d][16 b bytes]: within each tile of 128 tokens, coordinate j's 128 codes form one
// LSB-first bitstream (token o at bits [o b, o b + b)), so that the read path gathers a coordinate's values for a
// token pair from one byte (b = 4).  The quantization is the write path above, unchanged.
constexpr int kTileTok = 128;

// Whole tiles: vectors [128 i, 128 i + 128) fill tile i; one block of 8 warps per tile, plain stores.
template <int D, int BITS, typename TIn>
__global__ void __launch_bounds__(kWriteWarps * kWarp)
write_tiles_kernel(const TIn* __restrict__ x, const int8_t* __restrict__ signs, uint8_t* __restrict__ codes,
                   __half* __restrict__ norms, Codebook cb) {
  constexpr int VPL = WarpVec<D>::VPL;
  constexpr int L = 1 << BITS;
  constexpr int R = kTileTok * BITS / 8;  // bytes per coordinate per tile
  __shared__ uint8_t idx_t[kTileTok][D];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float sg[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) sg[i] = lane * VPL + i < D ? sign_of(signs[lane * VPL + i]) : 0.0f;
  float tau[L - 1];
#pragma unroll
  for (int k = 0; k < L - 1; ++k) tau[k] = cb.tau[k];
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * kTileTok;
  for (int o = warp; o < kTileTok; o += kWriteWarps) {
    const float n = quantize_vector<D, BITS, TIn>(x + (row0 + o) * D, sg, tau, lane, idx_t[o]);
    if (lane == 0) norms[row0 + o] = __float2half_rn(n);
  }
  __syncthreads();
  uint32_t* out = reinterpret_cast<uint32_t*>(codes + static_cast<int64_t>(blockIdx.x) * D * R);
  for (int e = threadIdx.x; e < D * (R / 4); e += kWriteWarps * kWarp) {
    const int j = e / (R / 4), wi = e % (R / 4);
    uint32_t acc = 0;
    const int first = (32 * wi) / BITS, last = min((32 * wi + 31) / BITS, kTileTok - 1);
    for (int o = first; o <= last; ++o) {
      const int pos = o * BITS - 32 * wi;
      const uint32_t code = idx_t[o][j];
      acc |= pos >= 0 ? (code << pos) : (code >> (-pos));
    }
    out[j * (R / 4) + wi] = acc;
  }
}

// Scattered vectors (dst_rows): each coordinate's field is replaced with two word atomics (clear, then set), so
// vectors of the same tile written by one call never lose each other's bits.  Destination rows must be distinct.
template <int D, int BITS, typename TIn>
__global__ void __launch_bounds__(kWriteWarps * kWarp)
write_tiles_scatter_kernel(const TIn* __restrict__ x, int64_t n_vec, const int8_t* __restrict__ signs,
                           const int64_t* __restrict__ dst_rows, int Tcap, uint8_t* __restrict__ codes,
                           __half* __restrict__ norms, Codebook cb) {
  constexpr int VPL = WarpVec<D>::VPL;
  constexpr int L = 1 << BITS;
  constexpr int R = kTileTok * BITS / 8;
  __shared__ uint8_t idx_s[kWriteWarps][D];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float sg[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) sg[i] = lane * VPL + i < D ? sign_of(signs[lane * VPL + i]) : 0.0f;
  float tau[L - 1];
#pragma unroll
  for (int k = 0; k < L - 1; ++k) tau[k] = cb.tau[k];
  const int64_t tiles_cap = Tcap / kTileTok;
  for (int64_t vec = static_cast<int64_t>(blockIdx.x) * kWriteWarps + warp; vec < n_vec;
       vec += static_cast<int64_t>(gridDim.x) * kWriteWarps) {
    const float n = quantize_vector<D, BITS, TIn>(x + vec * D, sg, tau, lane, idx_s[warp]);
    __syncwarp();
    const int64_t row = dst_rows ? dst_rows[vec] : vec;
    const int64_t bh = row / Tcap;
    const int t = static_cast<int>(row % Tcap);
    const int64_t tile = bh * tiles_cap + t / kTileTok;
    const int o = t % kTileTok;
    unsigned int* base = reinterpret_cast<unsigned int*>(codes + tile * D * R);
    for (int j = lane; j < D; j += kWarp) {
      const uint32_t code = idx_s[warp][j];
      const int bit = j * R * 8 + o * BITS;
      const int wi = bit >> 5, sh = bit & 31;
      constexpr uint32_t M = (1u << BITS) - 1u;
      atomicAnd(base + wi, ~(M << sh));
      atomicOr(base + wi, code << sh);
      if (sh + BITS > 32) {  // the field continues in the next word
        const int lo_bits = 32 - sh;
        atomicAnd(base + wi + 1, ~(M >> lo_bits));
        atomicOr(base + wi + 1, code >> lo_bits);
      }
    }
    if (lane == 0) norms[row] = __float2half_rn(n);
    __syncwarp();
  }
}

template <int BITS>
axr_status launch_write_tiles(const void* x, axr_dtype dt, int64_t n_vec, const int8_t* signs, const int64_t* dst,
                              int Tcap, uint8_t* codes, uint16_t* norms, const Codebook& cb, cudaStream_t st) {
  constexpr int D = 128;
  __half* nh = reinterpret_cast<__half*>(norms);
  if (!dst && n_vec % kTileTok == 0) {
    const unsigned grid = static_cast<unsigned>(n_vec / kTileTok);
    if (dt == AXR_F16)
      write_tiles_kernel<D, BITS, __half><<<grid, kWriteWarps * kWarp, 0, st>>>(static_cast<const __half*>(x), signs,
                                                                                 codes, nh, cb);
    else
      write_tiles_kernel<D, BITS, float><<<grid, kWriteWarps * kWarp, 0, st>>>(static_cast<const float*>(x), signs,
                                                                                codes, nh, cb);
  } else {
    int64_t blocks = (n_vec + kWriteWarps - 1) / kWriteWarps;
    const int64_t cap = static_cast<int64_t>(kSmCount) * 16;
    if (blocks > cap) blocks = cap;
    if (dt == AXR_F16)
      write_tiles_scatter_kernel<D, BITS, __half><<<static_cast<unsigned>(blocks), kWriteWarps * kWarp, 0, st>>>(
          static_cast<const __half*>(x), n_vec, signs, dst, Tcap, codes, nh, cb);
    else
      write_tiles_scatter_kernel<D, BITS, float><<<static_cast<unsigned>(blocks), kWriteWarps * kWarp, 0, st>>>(
          static_cast<const float*>(x), n_vec, signs, dst, Tcap, codes, nh, cb);
  }
  return check_launch("axr_write_values_tiled");
}

template <int D, int BITS>
axr_status launch_write(const void* x, axr_dtype dt, int64_t n_vec, const int8_t* signs, const int64_t* dst,
                        uint8_t* codes, uint16_t* norms, const Codebook& cb, cudaStream_t st) {
  int64_t blocks = (n_vec + kWriteWarps - 1) / kWriteWarps;
  const int64_t cap = static_cast<int64_t>(kSmCount) * 16;
  if (blocks > cap) blocks = cap;
  __half* nh = reinterpret_cast<__half*>(norms);
  if (dt == AXR_F16)
    write_kernel<D, BITS, __half><<<static_cast<unsigned>(blocks), kWriteWarps * kWarp, 0, st>>>(
        static_cast<const __half*>(x), n_vec, signs, dst, codes, nh, cb);
  else
    write_kernel<D, BITS, float><<<static_cast<unsigned>(blocks), kWriteWarps * kWarp, 0, st>>>(
        static_cast<const float*>(x), n_vec, signs, dst, codes, nh, cb);
  return check_launch("axr_write_keys");
}

template <int D>
axr_status dispatch_bits(int bits, const void* x, axr_dtype dt, int64_t n, const int8_t* s, const int64_t* dst,
                         uint8_t* c, uint16_t* nr, const Codebook& cb, cudaStream_t st) {
  switch (bits) {
    case 1: return launch_write<D, 1>(x, dt, n, s, dst, c, nr, cb, st);
    case 2: return launch_write<D, 2>(x, dt, n, s, dst, c, nr, cb, st);
    case 3: return launch_write<D, 3>(x, dt, n, s, dst, c, nr, cb, st);
    case 4: return launch_write<D, 4>(x, dt, n, s, dst, c, nr, cb, st);
  }
  return set_error(AXR_EUNSUPPORTED, "axr_write_keys: bits=%d", bits);
}

}  // namespace
}  // namespace axr

extern "C" axr_status axr_write_keys(const void* x, axr_dtype x_dtype, int64_t n_vec, int d, int bits,
                                     const int8_t* signs, const int64_t* dst_rows, uint8_t* codes, uint16_t* norms,
                                     void* stream) {
  using namespace axr;
  if (n_vec < 0) return set_error(AXR_EINVAL, "axr_write_keys: n_vec=%lld < 0", static_cast<long long>(n_vec));
  if (x_dtype != AXR_F32 && x_dtype != AXR_F16) return set_error(AXR_EINVAL, "axr_write_keys: bad dtype");
  if (d != 8 && d != 64 && d != 128) return set_error(AXR_EUNSUPPORTED, "axr_write_keys: d=%d not in {8,64,128}", d);
  if (bits < 1 || bits > 4) return set_error(AXR_EUNSUPPORTED, "axr_write_keys: bits=%d outside 1..4", bits);
  if (n_vec == 0) return set_error(AXR_OK, "");
  if (!x || !signs || !codes || !norms) return set_error(AXR_EINVAL, "axr_write_keys: null pointer");
  const uintptr_t xa = (x_dtype == AXR_F32 ? 4u : 2u) * (d >= 32 ? d / 32 : 1);
  if (!aligned(x, xa)) return set_error(AXR_EINVAL, "axr_write_keys: x not %u-byte aligned", (unsigned)xa);
  if (!aligned(norms, 2)) return set_error(AXR_EINVAL, "axr_write_keys: norms not 2-byte aligned");
  if (dst_rows && !aligned(dst_rows, 8)) return set_error(AXR_EINVAL, "axr_write_keys: dst_rows not 8-byte aligned");
  const Codebook* cb = codebook_for(d, bits);
  if (!cb) return set_error(AXR_EINVAL, "axr_write_keys: codebook unavailable");
  cudaStream_t st = as_stream(stream);
  switch (d) {
    case 8: return dispatch_bits<8>(bits, x, x_dtype, n_vec, signs, dst_rows, codes, norms, *cb, st);
    case 64: return dispatch_bits<64>(bits, x, x_dtype, n_vec, signs, dst_rows, codes, norms, *cb, st);
    default: return dispatch_bits<128>(bits, x, x_dtype, n_vec, signs, dst_rows, codes, norms, *cb, st);
  }
}

extern "C" axr_status axr_write_values_tiled(const void* x, axr_dtype x_dtype, int64_t n_vec, int d, int bits,
                                             const int8_t* signs, const int64_t* dst_rows, int Tcap, uint8_t* codes,
                                             uint16_t* norms, void* stream) {
  using namespace axr;
  const char* w = "axr_write_values_tiled";
  if (n_vec < 0) return set_error(AXR_EINVAL, "%s: n_vec=%lld < 0", w, static_cast<long long>(n_vec));
  if (x_dtype != AXR_F32 && x_dtype != AXR_F16) return set_error(AXR_EINVAL, "%s: bad dtype", w);
  if (d != 128) return set_error(AXR_EUNSUPPORTED, "%s: d=%d (the tiled layout is built for d = 128)", w, d);
  if (bits < 1 || bits > 4) return set_error(AXR_EUNSUPPORTED, "%s: bits=%d outside 1..4", w, bits);
  if (Tcap <= 0 || Tcap % kTileTok) return set_error(AXR_EINVAL, "%s: Tcap=%d is not a positive multiple of 128", w, Tcap);
  if (n_vec == 0) return set_error(AXR_OK, "");
  if (!x || !signs || !codes || !norms) return set_error(AXR_EINVAL, "%s: null pointer", w);
  const uintptr_t xa = (x_dtype == AXR_F32 ? 4u : 2u) * (d / 32);
  if (!aligned(x, xa) || !aligned(codes, 4) || !aligned(norms, 2) || (dst_rows && !aligned(dst_rows, 8)))
    return set_error(AXR_EINVAL, "%s: misaligned pointer", w);
  const Codebook* cb = codebook_for(d, bits);
  if (!cb) return set_error(AXR_EINVAL, "%s: codebook unavailable", w);
  cudaStream_t st = as_stream(stream);
  switch (bits) {
    case 1: return launch_write_tiles<1>(x, x_dtype, n_vec, signs, dst_rows, Tcap, codes, norms, *cb, st);
    case 2: return launch_write_tiles<2>(x, x_dtype, n_vec, signs, dst_rows, Tcap, codes, norms, *cb, st);
    case 3: return launch_write_tiles<3>(x, x_dtype, n_vec, signs, dst_rows, Tcap, codes, norms, *cb, st);
    default: return launch_write_tiles<4>(x, x_dtype, n_vec, signs, dst_rows, Tcap, codes, norms, *cb, st);
  }
}
