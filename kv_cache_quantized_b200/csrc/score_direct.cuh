// Scores through warp-level MMAs with the key codes loaded straight into registers.
//
// AXELRAM Key Points (1st, 2nd items): every cached token's score is the gather-sum of the query's table entries at
// its stored indices, times its stored norm.  The table is read in factored form exactly as in score_mma.cuh (a
// token's centroids split into hi and lo fp16 planes form rows g and g + 8 of the A operand, looked up from the
// conflict-free hi/lo pair table; the query's planes form B; mma.sync.m16n8k16 with fp32 accumulation).  What
// differs is how the codes arrive: lane (g, t) needs only its slice [t R/4, (t + 1) R/4) of the rows of tokens g and
// g + 8 of a 16-token group, and the eight lanes of a t read eight consecutive slices, so a warp's load of a group
// is two fully coalesced requests of 8 whole rows each.  The codes therefore go from global memory into registers
// directly -- no staging tile, no copy engine, no block barrier -- and shared memory serves only the table lookups
// (four wavefronts per token at b = 4, the floor of the hi/lo factored form).  Each warp streams its own token ranges
// with PF groups of codes and norms in flight; warps are independent.
#pragma once

#include "mma_score.cuh"

namespace axr {

template <int D, int BITS, int G>
struct DirectPlan {
  static constexpr int WARPS = 8, THREADS = 32 * WARPS;
  static constexpr int R = D * BITS / 8;        // bytes of a row
  static constexpr int NB = R / 4;              // bytes of a lane's slice of a row
  static constexpr int NWS = (NB + 3) / 4;      // its 32-bit words
  static constexpr int PF = 4;                  // 16-token groups in flight per warp, in registers
  static constexpr int PD = 16;                 // groups ahead that are prefetched into L2
  static constexpr int LINES = (16 * R + 127) / 128;  // 128-byte lines of a group's codes
  static constexpr size_t TAB = (size_t)HiLoTable16<BITS>::BYTES;
  static constexpr size_t OFF_QS = (TAB + 127) / 128 * 128;          // [WARPS][G][D] row factors
  static constexpr size_t OFF_CENT = OFF_QS + (size_t)WARPS * G * D * 4;
  static constexpr size_t bytes = OFF_CENT + 16 * 4;
};

// A lane's NB-byte slice of a row in global memory into words (the slice is NB-aligned within a 4-aligned row for
// NB >= 4, 2-aligned for NB = 2, 6; byte-wise otherwise).
template <int NB, int NWS>
__device__ __forceinline__ void load_slice(const uint8_t* __restrict__ p, uint32_t (&w)[NWS]) {
  if constexpr (NB == 16) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    w[0] = u.x; w[1] = u.y; w[2] = u.z; w[3] = u.w;
  } else if constexpr (NB == 12) {
    const uint32_t* q = reinterpret_cast<const uint32_t*>(p);
    w[0] = __ldg(q); w[1] = __ldg(q + 1); w[2] = __ldg(q + 2);
  } else if constexpr (NB == 8) {
    const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
    w[0] = u.x; w[1] = u.y;
  } else if constexpr (NB == 6) {
    const unsigned short* h = reinterpret_cast<const unsigned short*>(p);
    w[0] = __ldg(h) | (static_cast<uint32_t>(__ldg(h + 1)) << 16);
    w[1] = __ldg(h + 2);
  } else if constexpr (NB == 4) {
    w[0] = __ldg(reinterpret_cast<const uint32_t*>(p));
  } else if constexpr (NB == 3) {
    w[0] = __ldg(p) | (static_cast<uint32_t>(__ldg(p + 1)) << 8) | (static_cast<uint32_t>(__ldg(p + 2)) << 16);
  } else if constexpr (NB == 2) {
    w[0] = __ldg(reinterpret_cast<const unsigned short*>(p));
  } else {
    static_assert(NB == 1, "slice length");
    w[0] = __ldg(p);
  }
}

// Scaled scores (times s_h) of the two tokens whose slices are w0 (token g) and w1 (token g + 8); the MMA loop of
// mma_scores16 with the codes in registers.
template <int D, int BITS, int G, int NWS>
__device__ __forceinline__ void direct_scores16(const uint32_t (&c0)[NWS], const uint32_t (&c1)[NWS],
                                                const uint8_t* tab, uint32_t rep16, const MmaB<D, G>& B,
                                                float (&out)[MmaB<D, G>::NT][2]) {
  constexpr int KT = MmaB<D, G>::KT, NT = MmaB<D, G>::NT;
  uint32_t w0[NWS + 1], w1[NWS + 1];
#pragma unroll
  for (int i = 0; i < NWS; ++i) { w0[i] = c0[i]; w1[i] = c1[i]; }
  w0[NWS] = w1[NWS] = 0u;
  float c[2][NT][4];
#pragma unroll
  for (int x = 0; x < 2; ++x)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) c[x][nt][i] = 0.f;
#pragma unroll
  for (int kk = 0; kk < KT; ++kk) {
    const uint2 e00 = *reinterpret_cast<const uint2*>(tab + hilo_off16<BITS>(w0, 2 * kk, rep16));
    const uint2 e01 = *reinterpret_cast<const uint2*>(tab + hilo_off16<BITS>(w0, 2 * kk + 1, rep16));
    const uint2 e10 = *reinterpret_cast<const uint2*>(tab + hilo_off16<BITS>(w1, 2 * kk, rep16));
    const uint2 e11 = *reinterpret_cast<const uint2*>(tab + hilo_off16<BITS>(w1, 2 * kk + 1, rep16));
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      mma_m16n8k16(c[0][nt], e00.x, e00.y, e01.x, e01.y, B.bh[nt][kk][0], B.bh[nt][kk][1]);
      mma_m16n8k16(c[1][nt], e10.x, e10.y, e11.x, e11.y, B.bh[nt][kk][0], B.bh[nt][kk][1]);
    }
  }
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    out[nt][0] = (c[0][nt][0] + c[0][nt][1]) + (c[0][nt][2] + c[0][nt][3]);
    out[nt][1] = (c[1][nt][0] + c[1][nt][1]) + (c[1][nt][2] + c[1][nt][3]);
  }
}

// Prefetch the 128-byte line at p into L2 (no register, nothing to wait for).
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// Work items: (batch row, KV head, chunk of a.chunk tokens), a multiple of 16; warp w of the grid takes items
// w, w + (all warps), ...
template <int D, int BITS, int G>
__global__ void __launch_bounds__(256, 2) score_direct_kernel(const __grid_constant__ DecodeArgs a) {
  using P = DirectPlan<D, BITS, G>;
  constexpr int NT = MmaB<D, G>::NT, NB = P::NB, NWS = P::NWS, PF = P::PF, VPL = D / kWarp;
  extern __shared__ __align__(16) uint8_t smem[];
  const uint8_t* tab = smem;
  float* cent = reinterpret_cast<float*>(smem + P::OFF_CENT);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float* qs = reinterpret_cast<float*>(smem + P::OFF_QS) + warp * G * D;  // this warp's row factors
  const int gq = lane >> 2, tq = lane & 3;
  const uint32_t rep16 = static_cast<uint32_t>(lane & 15) << 4;
  const float rd = rsqrtf(static_cast<float>(D));
  if (threadIdx.x < 16) cent[threadIdx.x] = a.cb.gamma[threadIdx.x];
  __syncthreads();
  build_hilo_table16<BITS>(cent, smem);
  __syncthreads();  // the table is complete; from here on warps run independently

  const int nchunks = (a.T + a.chunk - 1) / a.chunk;
  const int items = a.B * a.Hkv * nchunks;
  const int nwarps = gridDim.x * P::WARPS;
  float sg[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) sg[i] = sign_of(a.signs[lane * VPL + i]);
  const float qnorm = a.mult * rd;

  for (int item = blockIdx.x * P::WARPS + warp; item < items; item += nwarps) {
    const int ch = item % nchunks;
    const int hk = (item / nchunks) % a.Hkv;
    const int b = item / (nchunks * a.Hkv);
    const int start = ch * a.chunk;
    const int end = min(start + a.chunk, a.T);
    const int vend = min(end, row_len(a, b));
    float* out = a.scores + (static_cast<size_t>(b) * a.Hq + hk * G) * a.T;
    for (int t = max(start, vend) + lane; t < end; t += kWarp)  // masked positions
#pragma unroll
      for (int g = 0; g < G; ++g) out[static_cast<size_t>(g) * a.T + t] = -INFINITY;
    if (vend <= start) continue;
    const size_t row0 = (static_cast<size_t>(b) * a.Hkv + hk) * a.Tcap + start;
    const uint8_t* cbase = a.kcodes + row0 * P::R + tq * NB;
    const __half* nbase = a.knorms + row0;
    const int ngroups = (vend - start + 15) / 16;
    const int last = vend - start - 1;  // rows past it are clamped to it (their scores are dropped)
    // the codes (and norms) of a group travel to L2 PD groups before their registers load them
    // (only lines that start inside the item's valid rows: every prefetched address lies in the cache)
    auto prefetch_group = [&](int j) {
      if (j < ngroups) {
        const uint8_t* g0 = a.kcodes + (row0 + 16 * static_cast<size_t>(j)) * P::R;
        const int bytes = (min(16 * j + 16, last + 1) - 16 * j) * P::R;
        if (lane < P::LINES && 128 * lane < bytes) prefetch_l2(g0 + 128 * lane);
        else if (lane == 31) prefetch_l2(nbase + 16 * j);
      }
    };
    for (int j = 0; j < P::PD; ++j) prefetch_group(j);
    uint32_t c0[PF][NWS], c1[PF][NWS];
    unsigned short nr[PF];
    auto load_group = [&](int j, uint32_t (&x0)[NWS], uint32_t (&x1)[NWS], unsigned short& n) {
      const int r0 = min(16 * j + gq, last), r1 = min(16 * j + gq + 8, last);
      load_slice<NB, NWS>(cbase + static_cast<size_t>(r0) * P::R, x0);
      load_slice<NB, NWS>(cbase + static_cast<size_t>(r1) * P::R, x1);
      n = __ldg(reinterpret_cast<const unsigned short*>(nbase) + min(16 * j + (lane & 15), last));
    };
#pragma unroll
    for (int s = 0; s < PF; ++s) load_group(s, c0[s], c1[s], nr[s]);
    // the item's B operand: q~ = mult H (s .* q) per head by this warp, head scales, hi/lo fragments
    const float* qg = a.q + (static_cast<size_t>(b) * a.Hq + hk * G) * D;
    float scl[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float v[VPL];
#pragma unroll
      for (int i = 0; i < VPL; ++i) v[i] = qg[g * D + lane * VPL + i] * sg[i];
      fwht_warp<D>(v, lane);
#pragma unroll
      for (int i = 0; i < VPL; ++i) qs[g * D + lane * VPL + i] = v[i] * qnorm;
      scl[g] = tc::head_scale<D>(qg + g * D, a.mult);
    }
    __syncwarp();
    MmaB<D, G> B;
    mma_b_build<D, G>(qs, scl, lane, B);
    __syncwarp();  // the row factors are read before the next item overwrites them

    for (int j0 = 0; j0 < ngroups; j0 += PF) {
#pragma unroll
      for (int s = 0; s < PF; ++s) {
        const int j = j0 + s;
        if (j < ngroups) {
          float sc[NT][2];
          direct_scores16<D, BITS, G, NWS>(c0[s], c1[s], tab, rep16, B, sc);
          const unsigned short n0 = __shfl_sync(0xffffffffu, nr[s], gq);
          const unsigned short n1 = __shfl_sync(0xffffffffu, nr[s], gq + 8);
          const float f0 = __half2float(__ushort_as_half(n0)) * rd, f1 = __half2float(__ushort_as_half(n1)) * rd;
          const int t0 = start + 16 * j + gq;
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const int h = 4 * nt + tq;
            if (h < G) {
              if (t0 < vend) out[static_cast<size_t>(h) * a.T + t0] = sc[nt][0] * B.inv[nt] * f0;
              if (t0 + 8 < vend) out[static_cast<size_t>(h) * a.T + t0 + 8] = sc[nt][1] * B.inv[nt] * f1;
            }
          }
          if (j + PF < ngroups) load_group(j + PF, c0[s], c1[s], nr[s]);
          prefetch_group(j + P::PD);
        }
      }
    }
  }
}

}  // namespace axr
