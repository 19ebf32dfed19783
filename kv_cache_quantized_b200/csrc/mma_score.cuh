// Key scores through warp-level MMAs (mma.sync.m16n8k16, fp16 operands, fp32 accumulation), shared by the decode
// kernels.
//
// AXELRAM Key Points (1st, 2nd items): a token's score is the gather-sum of q~_j c_k at its stored indices, times
// its stored norm.  The table is read in factored form with both factors split into hi and lo fp16 planes (about 22
// bits each).  One MMA covers 8 tokens: A row g is token g's hi plane and row g + 8 its lo plane (coordinates along
// K); B column 2h is hi(s_h q~_h) and column 2h + 1 lo(s_h q~_h).  The four products of the two splits then sum to
// s_h times the score: C[g][2h] + C[g][2h + 1] + C[g + 8][2h] + C[g + 8][2h + 1].
//
// K order: the d/2 coordinate pairs are dealt to the four lanes t of a row group in contiguous slices, lane t owning
// pairs [t d/8, (t + 1) d/8) of every token, so that one load fetches a lane's codes of a row.  K-tile kk, k index
// 2t + i + 8 r (i, r in {0, 1}) is coordinate 2 p + i of pair p = t d/8 + 2 kk + r.  Fragments of lane (g, t):
//   A: one lookup in the hi/lo pair table per pair (2 kk + r) of the lane's slice of token g gives two registers,
//      the pair's hi plane (row g) and lo plane (row g + 8): with r = 0 they are A registers 0 and 1, with r = 1
//      registers 2 and 3, so the loads land in the operand as they are;
//   B: registers built once per (batch, KV head) and kept for the item;
//   C: head 4 nt + t's four partial sums for token g (n-tile nt covers heads 4 nt .. 4 nt + 3).
#pragma once

#include "decode.cuh"

namespace axr {

// hi/lo fp16 pair table with 16 copies (128 bytes per entry): entry e of lane l at e * 128 + (l % 16) * 8 holds
// {hi(c_lo), hi(c_hi)} and {lo(c_lo), lo(c_hi)} of the two coordinates of code pair e; a warp's 64-bit lookups take
// their two wavefronts without conflicts (lanes l and l + 16 fall in different halves of the request).
template <int BITS>
struct HiLoTable16 {
  static constexpr int L = 1 << BITS;
  static constexpr int E = L * L;
  static constexpr int BYTES = E * 128;
};

template <int BITS>
__device__ __forceinline__ void build_hilo_table16(const float* __restrict__ gamma, uint8_t* __restrict__ tab) {
  using T = HiLoTable16<BITS>;
  for (int i = threadIdx.x; i < T::E * 16; i += blockDim.x) {
    const int e = i >> 4, l = i & 15;
    const float c0 = gamma[e & (T::L - 1)], c1 = gamma[e >> BITS];
    const __half h0 = __float2half_rn(c0), h1 = __float2half_rn(c1);
    const __half l0 = __float2half_rn(c0 - __half2float(h0)), l1 = __float2half_rn(c1 - __half2float(h1));
    const __half2 hi = __halves2half2(h0, h1), lo = __halves2half2(l0, l1);
    *reinterpret_cast<uint2*>(tab + e * 128 + l * 8) =
        make_uint2(*reinterpret_cast<const uint32_t*>(&hi), *reinterpret_cast<const uint32_t*>(&lo));
  }
}

// Byte offset of this lane's copy of code pair i of a run of packed codes (w: its words, one zero word past the end);
// rep16 = (lane % 16) * 16.
template <int BITS>
__device__ __forceinline__ uint32_t hilo_off16(const uint32_t* w, int i, uint32_t rep16) {
  if constexpr (BITS == 4)  // (pair byte * 256 + rep16) / 2 = pair byte * 128 + (lane % 16) * 8
    return __byte_perm(w[i >> 2], rep16, 0x5504u | (static_cast<uint32_t>(i & 3) << 4)) >> 1;
  else
    return (bits_at<2 * BITS>(w, 2 * BITS * i) << 7) | (rep16 >> 1);
}

// The NB bytes at byte offset `off` of a staged tile (rows swizzled with stage_swizzle<R> if SWZ; the run stays
// inside one 16-byte chunk) into w[0 .. ceil(NB / 4)).
template <int R, int NB, bool SWZ = true>
__device__ __forceinline__ void load_run(const uint8_t* stage, int off, uint32_t* w) {
  const uint8_t* p = stage + (SWZ ? stage_swizzle<R>(off) : off);
  if constexpr (NB == 16) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    w[0] = u.x; w[1] = u.y; w[2] = u.z; w[3] = u.w;
  } else if constexpr (NB == 12) {
    const uint32_t* q = reinterpret_cast<const uint32_t*>(p);
    w[0] = q[0]; w[1] = q[1]; w[2] = q[2];
  } else if constexpr (NB == 8) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    w[0] = u.x; w[1] = u.y;
  } else if constexpr (NB == 6) {
    const uint16_t* h = reinterpret_cast<const uint16_t*>(p);
    w[0] = h[0] | (static_cast<uint32_t>(h[1]) << 16); w[1] = h[2];
  } else if constexpr (NB == 4) {
    w[0] = *reinterpret_cast<const uint32_t*>(p);
  } else if constexpr (NB == 3) {
    w[0] = p[0] | (static_cast<uint32_t>(p[1]) << 8) | (static_cast<uint32_t>(p[2]) << 16);
  } else if constexpr (NB == 2) {
    w[0] = *reinterpret_cast<const uint16_t*>(p);
  } else {
    static_assert(NB == 1, "run length");
    w[0] = *p;
  }
}

// Key/value pair table, 256 bytes per entry e (the 2b-bit code of a coordinate pair): bytes [0, 128) hold 16 copies
// of the hi/lo fp16 pair {hi(c_lo), hi(c_hi)}, {lo(c_lo), lo(c_hi)} (copy c at 8 c), bytes [128, 256) hold 32 copies
// of the hi pair alone (copy c at 128 + 4 c).  The offset of a lookup is one byte permute of the code word (entry
// into byte 1, the lane's copy offset into byte 0): a warp's 64-bit key lookups take two wavefronts and its 32-bit
// value lookups one, whatever the entries.
template <int BITS>
struct PairTableKV {
  static constexpr int L = 1 << BITS;
  static constexpr int E = L * L;
  static constexpr int BYTES = E * 256;
};

template <int BITS>
__device__ __forceinline__ void build_pair_table_kv(const float* __restrict__ gamma, uint8_t* __restrict__ tab) {
  using T = PairTableKV<BITS>;
  for (int i = threadIdx.x; i < T::E * 48; i += blockDim.x) {
    const int e = i / 48, slot = i % 48;
    const float c0 = gamma[e & (T::L - 1)], c1 = gamma[e >> BITS];
    const __half h0 = __float2half_rn(c0), h1 = __float2half_rn(c1);
    const __half2 hi = __halves2half2(h0, h1);
    if (slot < 16) {
      const __half2 lo = __halves2half2(__float2half_rn(c0 - __half2float(h0)), __float2half_rn(c1 - __half2float(h1)));
      *reinterpret_cast<uint2*>(tab + e * 256 + slot * 8) =
          make_uint2(*reinterpret_cast<const uint32_t*>(&hi), *reinterpret_cast<const uint32_t*>(&lo));
    } else {
      *reinterpret_cast<uint32_t*>(tab + e * 256 + 128 + (slot - 16) * 4) = *reinterpret_cast<const uint32_t*>(&hi);
    }
  }
}

// Byte offset in a PairTableKV of code pair i of a run of packed codes (w: its words, one zero word past the end);
// rep = (lane % 16) * 8 for the hi/lo copies, 128 + 4 lane for the hi-only copies.
template <int BITS>
__device__ __forceinline__ uint32_t kv_off(const uint32_t* w, int i, uint32_t rep) {
  if constexpr (BITS == 4)
    return __byte_perm(w[i >> 2], rep, 0x5504u | (static_cast<uint32_t>(i & 3) << 4));
  else
    return (bits_at<2 * BITS>(w, 2 * BITS * i) << 8) | rep;
}

__device__ __forceinline__ void mma_m16n8k16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Power-of-two range scale of one head's B operand from its transformed row q~ (shared memory, one warp):
// 2^(14 - e) with ||q~|| in [2^(e-1), 2^e), so that the fp16 planes stay far from overflow and underflow.  Any
// consistent power of two is exact; the epilogue divides it back out.
template <int D>
__device__ __forceinline__ float head_scale_rows(const float* __restrict__ row) {
  const int lane = threadIdx.x & 31;
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < D / 32; ++i) {
    const float x = row[lane + 32 * i];
    ss = fmaf(x, x, ss);
  }
  const float m = sqrtf(warp_sum(ss));
  if (!(m > 0.f) || !isfinite(m)) return 1.f;
  int e = 0;
  frexpf(m, &e);
  return ldexpf(1.f, 14 - e);
}

template <int D, int G>
struct MmaB {
  static constexpr int KT = D / 16;              // K-tiles
  static constexpr int NT = G <= 4 ? 1 : 2;      // n-tiles of 8 columns
  uint32_t bh[NT][KT][2];                        // columns 2h, 2h + 1: hi and lo plane of s_h q~_h
  float inv[NT];                                 // 1 / scale of head 4 nt + t
};

// B fragments from the transformed query qs [G][D] (smem) and the head scales scl[G]; lane = (g, t).
template <int D, int G>
__device__ __forceinline__ void mma_b_build(const float* __restrict__ qs, const float (&scl)[G], int lane,
                                            MmaB<D, G>& B) {
  constexpr int KT = MmaB<D, G>::KT, NT = MmaB<D, G>::NT;
  const int gq = lane >> 2, tq = lane & 3;
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
          const int j = 2 * (2 * KT * tq + 2 * kk + r) + i;
          const float q = h < G ? qs[h * D + j] * sc : 0.f;
          const float qh = __half2float(__float2half_rn(q));
          v[i] = hi_col ? qh : q - qh;
        }
        const __half2 p = __floats2half2_rn(v[0], v[1]);
        B.bh[nt][kk][r] = *reinterpret_cast<const uint32_t*>(&p);
      }
    }
    float sc2 = 1.f;
#pragma unroll
    for (int g = 0; g < G; ++g) sc2 = g == 4 * nt + tq ? scl[g] : sc2;
    B.inv[nt] = 1.f / sc2;
  }
}

// Block-wide build of the B fragments into shared memory, one 32-bit entry per thread: bs[e][lane] with
// e = (nt KT + kk) 2 + r holds MmaB::bh[nt][kk][r] for that lane (mma_b_build's values); the inverse scales are
// derived on load (mma_b_load).
template <int D, int G>
__device__ __forceinline__ void mma_b_stage(const float* __restrict__ qs, const float* __restrict__ scl,
                                            uint32_t* __restrict__ bs) {
  constexpr int KT = MmaB<D, G>::KT, NT = MmaB<D, G>::NT, NE = NT * KT * 2;
  for (int idx = threadIdx.x; idx < NE * 32; idx += blockDim.x) {
    const int ln = idx & 31, e = idx >> 5;
    const int r = e & 1, kk = (e >> 1) % KT, nt = (e >> 1) / KT;
    const int gq = ln >> 2, tq = ln & 3;
    const int h = 4 * nt + (gq >> 1);
    const bool hi_col = (gq & 1) == 0;
    float v[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int j = 2 * (2 * KT * tq + 2 * kk + r) + i;
      const float q = h < G ? qs[h * D + j] * scl[h] : 0.f;
      const float qh = __half2float(__float2half_rn(q));
      v[i] = hi_col ? qh : q - qh;
    }
    const __half2 p = __floats2half2_rn(v[0], v[1]);
    bs[e * 32 + ln] = *reinterpret_cast<const uint32_t*>(&p);
  }
}

template <int D, int G>
__device__ __forceinline__ void mma_b_load(const uint32_t* __restrict__ bs, const float* __restrict__ scl, int lane,
                                           MmaB<D, G>& B) {
  constexpr int KT = MmaB<D, G>::KT, NT = MmaB<D, G>::NT;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int kk = 0; kk < KT; ++kk)
#pragma unroll
      for (int r = 0; r < 2; ++r) B.bh[nt][kk][r] = bs[((nt * KT + kk) * 2 + r) * 32 + lane];
    const int h = 4 * nt + (lane & 3);
    B.inv[nt] = h < G ? 1.f / scl[h] : 1.f;
  }
}

// Scaled scores (times s_h) of tokens r0 = row0 + g and r1 = r0 + 8 of a staged tile of packed rows (swizzled with
// stage_swizzle<R> if SWZ), for head 4 nt + t: out[nt][0] for r0, out[nt][1] for r1.  The table is a HiLoTable16
// (rep = (lane % 16) * 16), or a PairTableKV if KV (rep = (lane % 16) * 8).
template <int D, int BITS, int G, bool SWZ = true, bool KV = false>
__device__ __forceinline__ void mma_scores16(const uint8_t* st, int row0, const uint8_t* tab, uint32_t rep16,
                                             const MmaB<D, G>& B, int lane, float (&out)[MmaB<D, G>::NT][2]) {
  constexpr int R = D * BITS / 8, KT = MmaB<D, G>::KT, NT = MmaB<D, G>::NT;
  constexpr int NB = R / 4;               // bytes of a lane's slice of a row
  constexpr int NW = (NB + 3) / 4 + 1;    // its words, plus a zero word
  const int gq = lane >> 2, tq = lane & 3;
  uint32_t w0[NW], w1[NW];
  load_run<R, NB, SWZ>(st, (row0 + gq) * R + tq * NB, w0);
  load_run<R, NB, SWZ>(st, (row0 + gq + 8) * R + tq * NB, w1);
#pragma unroll
  for (int i = (NB + 3) / 4; i < NW; ++i) w0[i] = w1[i] = 0u;
  float c[2][NT][4];  // [token g, token g + 8][n-tile]
#pragma unroll
  for (int x = 0; x < 2; ++x)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) c[x][nt][i] = 0.f;
  auto off = [&](const uint32_t* w, int i) {
    if constexpr (KV) return kv_off<BITS>(w, i, rep16);
    else return hilo_off16<BITS>(w, i, rep16);
  };
#pragma unroll
  for (int kk = 0; kk < KT; ++kk) {
    // {hi, lo} of pairs 2 kk (A registers 0, 1) and 2 kk + 1 (registers 2, 3) of token g, then of token g + 8
    const uint2 e00 = *reinterpret_cast<const uint2*>(tab + off(w0, 2 * kk));
    const uint2 e01 = *reinterpret_cast<const uint2*>(tab + off(w0, 2 * kk + 1));
    const uint2 e10 = *reinterpret_cast<const uint2*>(tab + off(w1, 2 * kk));
    const uint2 e11 = *reinterpret_cast<const uint2*>(tab + off(w1, 2 * kk + 1));
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

// mma_scores16 for the two 16-token groups of a 32-token tile (rows row0 .. row0 + 15 into out[0], row0 + 16 ..
// row0 + 31 into out[1]) in one pass over K: the four accumulator chains (two groups x tokens g, g + 8) take turns,
// so that each MMA's successor in its chain issues three MMAs later.  Each chain sums its products in the order
// mma_scores16 does, so the scores are the same bit for bit.
template <int D, int BITS, int G, bool SWZ = true, bool KV = false>
__device__ __forceinline__ void mma_scores16x2(const uint8_t* st, int row0, const uint8_t* tab, uint32_t rep16,
                                               const MmaB<D, G>& B, int lane,
                                               float (&out)[2][MmaB<D, G>::NT][2]) {
  constexpr int R = D * BITS / 8, KT = MmaB<D, G>::KT, NT = MmaB<D, G>::NT;
  constexpr int NB = R / 4;
  constexpr int NW = (NB + 3) / 4 + 1;
  const int gq = lane >> 2, tq = lane & 3;
  uint32_t w[4][NW];  // tokens g, g + 8 of group 0, then of group 1
#pragma unroll
  for (int x = 0; x < 4; ++x) {
    load_run<R, NB, SWZ>(st, (row0 + 16 * (x >> 1) + gq + 8 * (x & 1)) * R + tq * NB, w[x]);
#pragma unroll
    for (int i = (NB + 3) / 4; i < NW; ++i) w[x][i] = 0u;
  }
  float c[4][NT][4];
#pragma unroll
  for (int x = 0; x < 4; ++x)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) c[x][nt][i] = 0.f;
  auto off = [&](const uint32_t* wr, int i) {
    if constexpr (KV) return kv_off<BITS>(wr, i, rep16);
    else return hilo_off16<BITS>(wr, i, rep16);
  };
#pragma unroll
  for (int kk = 0; kk < KT; ++kk) {
    uint2 e[4][2];
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      e[x][0] = *reinterpret_cast<const uint2*>(tab + off(w[x], 2 * kk));
      e[x][1] = *reinterpret_cast<const uint2*>(tab + off(w[x], 2 * kk + 1));
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int x = 0; x < 4; ++x)
        mma_m16n8k16(c[x][nt], e[x][0].x, e[x][0].y, e[x][1].x, e[x][1].y, B.bh[nt][kk][0], B.bh[nt][kk][1]);
  }
#pragma unroll
  for (int m = 0; m < 2; ++m)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const float* cc = c[2 * m + i][nt];
        out[m][nt][i] = (cc[0] + cc[1]) + (cc[2] + cc[3]);
      }
}

}  // namespace axr
