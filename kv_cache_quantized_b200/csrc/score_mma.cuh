// Scores through warp-level MMAs (mma.sync.m16n8k16, fp16 operands, fp32 accumulation).
//
// AXELRAM Key Points (1st, 2nd items): every cached token's score is the gather-sum of the query's table entries at
// the token's stored indices, times its stored norm.  The table is read in factored form, as on the tensor cores
// (tc.cuh): each token's centroids, split into hi and lo fp16 planes (about 22 bits), form a row of A; the query's
// hi/lo planes form B (column 2h: hi(q~_h) against both planes, column 2h+1: lo(q~_h) against the hi plane); one
// M = 16 tokens x N = 8 x K = 16 MMA per 8 coordinate pairs and plane.  Here the operands live in registers:
//   A fragment of lane (g, t): pairs 8 kk + t and 8 kk + t + 4 of tokens g and g + 8 -- one byte-indexed lookup in
//                              the hi/lo pair table gives the hi register (K-tile kk) and the lo register (K-tile
//                              kk + d/16) of a pair;
//   B fragment: built once per (batch, KV head) from the transformed query and kept in registers;
//   C fragment: lane (g, t) ends with head t's score of tokens g and g + 8 (columns 2t, 2t+1 summed).
// There is no shuffle reduction and no cross-warp hand-off inside a tile: warp w owns tokens [16 w, 16 w + 16) of
// each 128-token tile; key codes are staged by cp.async, five tiles deep, one block barrier per tile.  Blocks are
// persistent (two per SM) over (batch, KV head, split) items and build the pair table once.
#pragma once

#include "decode.cuh"

namespace axr {

template <int D, int BITS, int G>
struct ScoreMmaPlan {
  static constexpr int TT = 128;
  static constexpr int WARPS = 8, THREADS = 32 * WARPS;
  static constexpr int R = D * BITS / 8;
  static constexpr int KCH = (R % 16 == 0) ? 16 : 8;
  static constexpr int KT = D / 16;               // K-tiles per plane
  static constexpr int NT = G <= 4 ? 1 : 2;       // n-tiles of 8 columns (2 per head)
  static constexpr int STAGE = TT * R;
  static constexpr int NST = 5;                   // code stages: four tiles in flight per block
  static constexpr size_t OFF_STAGE = 0;
  static constexpr size_t OFF_NRM = (size_t)NST * STAGE;                    // [NST][TT] fp16 key norms
  static constexpr size_t OFF_TAB = (OFF_NRM + (size_t)NST * TT * 2 + 255) / 256 * 256;
  static constexpr size_t OFF_QS = OFF_TAB + tc::PairTable16<BITS>::BYTES;
  static constexpr size_t OFF_CENT = OFF_QS + (size_t)G * D * 4;
  static constexpr size_t bytes = OFF_CENT + 16 * 4;
};

__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

template <int D, int BITS, int G>
__global__ void __launch_bounds__(256, 2) score_mma_kernel(const __grid_constant__ DecodeArgs a) {
  using P = ScoreMmaPlan<D, BITS, G>;
  constexpr int R = P::R, KT = P::KT, NT = P::NT, TT = P::TT, NST = P::NST;
  extern __shared__ __align__(16) uint8_t smem[];
  const uint8_t* tab = smem + P::OFF_TAB;
  float* qs = reinterpret_cast<float*>(smem + P::OFF_QS);
  float* cent = reinterpret_cast<float*>(smem + P::OFF_CENT);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, tq = lane & 3;
  const uint32_t repw = static_cast<uint32_t>(lane) << 3;
  const float rd = rsqrtf(static_cast<float>(D));
  // this lane's two rows (tokens 16 w + gq and + 8 of every tile): swizzled chunk offsets, fixed for the kernel
  const int r0 = 16 * warp + gq, r1 = r0 + 8;
  constexpr int NCH = R % 16 == 0 ? R / 16 : R / 8;
  int off0[NCH], off1[NCH];
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    const int cb = R % 16 == 0 ? 16 : 8;
    off0[c] = stage_swizzle<R>(r0 * R + c * cb);
    off1[c] = stage_swizzle<R>(r1 * R + c * cb);
  }

  if (tid < 16) cent[tid] = a.cb.gamma[tid];
  __syncthreads();
  tc::build_table<BITS>(cent, reinterpret_cast<uint2*>(smem + P::OFF_TAB));  // once per block

  const int items = a.B * a.Hkv * a.splits;
  for (int item = blockIdx.x; item < items; item += gridDim.x) {
    const int split = item % a.splits;
    const int hk = (item / a.splits) % a.Hkv;
    const int b = item / (a.splits * a.Hkv);
    const int len = row_len(a, b);
    const int start = split * a.chunk;
    const int end = min(start + a.chunk, a.T);
    const int vend = min(end, len);  // tokens with codes
    const size_t kv_row0 = (static_cast<size_t>(b) * a.Hkv + hk) * a.Tcap;
    const float* qg = a.q + (static_cast<size_t>(b) * a.Hq + hk * G) * D;
    float* out = a.scores + (static_cast<size_t>(b) * a.Hq + hk * G) * a.T;
    for (int t = max(start, len) + tid; t < end; t += P::THREADS)  // masked positions
#pragma unroll
      for (int g = 0; g < G; ++g) out[static_cast<size_t>(g) * a.T + t] = -INFINITY;
    const int ntiles = vend > start ? (vend - start + TT - 1) / TT : 0;

    __syncthreads();  // the previous item is finished with the stages and the row factors
    // key norms ride with the codes when the item's norm row starts 16-byte aligned, else each lane loads its two
    const __half* kn_src = a.knorms + kv_row0;
    const bool nrm_async = (reinterpret_cast<uintptr_t>(kn_src + start) & 15) == 0;
    __half* nst = reinterpret_cast<__half*>(smem + P::OFF_NRM);
    auto issue_tile = [&](int tile) {
      if (tile < ntiles) {
        uint8_t* st = smem + P::OFF_STAGE + static_cast<size_t>(tile % NST) * P::STAGE;
        const int t0 = start + tile * TT;
        const int n = min(TT, vend - t0);
        const int bytes = n * R;
        const uint8_t* src = a.kcodes + (kv_row0 + t0) * R;
        for (int o = tid * P::KCH; o < bytes; o += P::THREADS * P::KCH) cp_async<P::KCH>(st + stage_swizzle<R>(o), src + o);
        if (nrm_async && tid < 16) stage_norms(nst + (tile % NST) * TT, kn_src + t0, n, tid);
      }
      cp_async_commit();
    };
    for (int s = 0; s < NST - 1; ++s) issue_tile(s);
    transform_queries<D, G>(qg, a.signs, a.mult, qs);
    // head scales (each warp computes every head's; warp reductions): 2^(14 - e), |mult| ||q|| in [2^(e-1), 2^e)
    float scl[G];
#pragma unroll
    for (int g = 0; g < G; ++g) scl[g] = tc::head_scale<D>(qg + g * D, a.mult);
    __syncthreads();
    // B fragments: column n = gq of n-tile nt is head 4 nt + gq / 2, hi plane of q~ if gq is even, lo if odd;
    // against the lo plane of the centroids only the hi columns count (bl = 0 in the lo columns)
    uint32_t bh[NT][KT][2], bl[NT][KT][2];
    float inv[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int h = 4 * nt + (gq >> 1);
      const bool hi_col = (gq & 1) == 0;
      float sc = 1.f;
#pragma unroll
      for (int g = 0; g < G; ++g) sc = g == h ? scl[g] : sc;
#pragma unroll
      for (int kk = 0; kk < KT; ++kk) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          float v[2];
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const int j = 16 * kk + 2 * tq + 8 * r + i;
            const float q = h < G ? qs[h * D + j] * sc : 0.f;
            const float qh = __half2float(__float2half_rn(q));
            v[i] = hi_col ? qh : q - qh;
          }
          bh[nt][kk][r] = pack_half2(v[0], v[1]);
          bl[nt][kk][r] = hi_col ? bh[nt][kk][r] : 0u;
        }
      }
      float sc2 = 1.f;  // the scale of head 4 nt + tq, whose two columns this lane's accumulators hold
#pragma unroll
      for (int g = 0; g < G; ++g) sc2 = g == 4 * nt + tq ? scl[g] : sc2;
      inv[nt] = 1.f / sc2;
    }

    for (int tile = 0; tile < ntiles; ++tile) {
      const int t0 = start + tile * TT;
      const int nt_tok = min(TT, vend - t0);
      cp_async_wait<NST - 2>();
      __syncthreads();  // tile complete everywhere; the previous tile's stage is free
      issue_tile(tile + NST - 1);
      const uint8_t* st = smem + P::OFF_STAGE + static_cast<size_t>(tile % NST) * P::STAGE;
      uint32_t w0[R / 4 + 1], w1[R / 4 + 1];
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
        if constexpr (R % 16 == 0) {
          const uint4 u0 = *reinterpret_cast<const uint4*>(st + off0[c]);
          const uint4 u1 = *reinterpret_cast<const uint4*>(st + off1[c]);
          w0[4 * c] = u0.x; w0[4 * c + 1] = u0.y; w0[4 * c + 2] = u0.z; w0[4 * c + 3] = u0.w;
          w1[4 * c] = u1.x; w1[4 * c + 1] = u1.y; w1[4 * c + 2] = u1.z; w1[4 * c + 3] = u1.w;
        } else {
          const uint2 u0 = *reinterpret_cast<const uint2*>(st + off0[c]);
          const uint2 u1 = *reinterpret_cast<const uint2*>(st + off1[c]);
          w0[2 * c] = u0.x; w0[2 * c + 1] = u0.y;
          w1[2 * c] = u1.x; w1[2 * c + 1] = u1.y;
        }
      }
      w0[R / 4] = w1[R / 4] = 0u;
      float kn0, kn1;
      if (nrm_async) {
        kn0 = __half2float(nst[(tile % NST) * TT + r0]);
        kn1 = __half2float(nst[(tile % NST) * TT + r1]);
      } else {
        kn0 = r0 < nt_tok ? __half2float(kn_src[t0 + r0]) : 0.f;
        kn1 = r1 < nt_tok ? __half2float(kn_src[t0 + r1]) : 0.f;
      }
      float c[2][NT][4];  // two accumulator chains (even / odd K-tiles)
#pragma unroll
      for (int x = 0; x < 2; ++x)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int i = 0; i < 4; ++i) c[x][nt][i] = 0.f;
#pragma unroll
      for (int kk = 0; kk < KT; ++kk) {
        const uint2 e00 = *reinterpret_cast<const uint2*>(tab + tc::pair_off<BITS>(w0, 8 * kk + tq, repw));
        const uint2 e10 = *reinterpret_cast<const uint2*>(tab + tc::pair_off<BITS>(w1, 8 * kk + tq, repw));
        const uint2 e01 = *reinterpret_cast<const uint2*>(tab + tc::pair_off<BITS>(w0, 8 * kk + tq + 4, repw));
        const uint2 e11 = *reinterpret_cast<const uint2*>(tab + tc::pair_off<BITS>(w1, 8 * kk + tq + 4, repw));
        const uint32_t ahi[4] = {e00.x, e10.x, e01.x, e11.x};
        const uint32_t alo[4] = {e00.y, e10.y, e01.y, e11.y};
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          mma16816(c[kk & 1][nt], ahi, bh[nt][kk][0], bh[nt][kk][1]);  // hi plane x (hi | lo) q
          mma16816(c[kk & 1][nt], alo, bl[nt][kk][0], bl[nt][kk][1]);  // lo plane x hi q
        }
      }
      const float f0 = kn0 * rd, f1 = kn1 * rd;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int h = 4 * nt + tq;
        if (h < G) {
          float* o = out + static_cast<size_t>(h) * a.T + t0;
          const float s0 = (c[0][nt][0] + c[1][nt][0]) + (c[0][nt][1] + c[1][nt][1]);
          const float s1 = (c[0][nt][2] + c[1][nt][2]) + (c[0][nt][3] + c[1][nt][3]);
          if (r0 < nt_tok) o[r0] = s0 * inv[nt] * f0;
          if (r1 < nt_tok) o[r1] = s1 * inv[nt] * f1;
        }
      }
    }
    cp_async_wait<0>();
  }
}

}  // namespace axr
