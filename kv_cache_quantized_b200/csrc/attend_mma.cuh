// Decode attention over tiled values (d = 128) with the value product as warp-level MMAs.
//
// The scores are the factored gather of the row-layout kernel (AXELRAM Key Points, 1st and 2nd items: gather-sum of
// q~_j c_k at the stored indices, times the stored norm; packed fp32 FMAs on the CUDA cores).  The value product
// of each 128-token tile, in the rotated domain, is a small matrix product
//   O^T[j][h] += sum_t  c[idx^V_{t,j}] * P'[h][t],   P'[h][t] = p_{h,t} n^V_t (fp16),  fp32 accumulation,
// computed with mma.sync.m16n8k16 (M = 16 coordinates, N = 8 heads, K = 16 tokens): in the tiled value layout a byte
// of a coordinate's row holds two consecutive tokens (b = 4), so every A-fragment register (two fp16 values of one
// coordinate at two consecutive tokens) is one lookup in a byte-indexed table of fp16 centroid pairs, and every
// B-fragment register is two consecutive fp16 weights of one head.
//
// Block structure (256 threads, persistent over (batch, KV head, split) items, two blocks per SM), as the row
// kernel: scoring warps 0..3 own tokens [32 w, 32 w + 32) of every tile and keep the running max and sum of their
// tokens (online softmax); value warp 4 + w consumes the same tokens one tile later against the same running max:
// 8 M-tiles (128 coordinates) x 2 K-tiles, accumulators in registers.  One block barrier per tile.
#pragma once

#include "decode.cuh"

namespace axr {

template <int BITS, int G>
struct MmaPlan {
  static constexpr int D = 128, TT = 128;
  static constexpr int KW = 4;                   // scoring warps; value warps follow them
  static constexpr int WT = TT / KW;             // tokens per scoring warp per tile
  static constexpr int L = 1 << BITS;
  static constexpr int R = D * BITS / 8;         // key bytes per token = value bytes per coordinate per tile
  static constexpr int J = D / 8;                // key coordinates per scoring lane
  static constexpr int HG = G < 4 ? G : 4, PASSES = G / HG;
  static constexpr int STAGE = TT * R;
  static constexpr int E = L * L;
  static constexpr int SW = 4 * BITS;            // bytes of a coordinate row that hold one value warp's 32 tokens
  static constexpr size_t OFF_K = 0;                                          // [kStages][STAGE]
  static constexpr size_t OFF_V = OFF_K + kStages * (size_t)STAGE;           // [kStages][STAGE], rows swizzled
  static constexpr size_t STAGES_END = OFF_V + kStages * (size_t)STAGE;
  static constexpr size_t REDUCE_BYTES = (size_t)KW * 8 * D * 4;             // final sum, reuses the stages
  static constexpr size_t OFF_KTAB = ((STAGES_END > REDUCE_BYTES ? STAGES_END : REDUCE_BYTES) + 15) / 16 * 16;
  static constexpr size_t OFF_QS = OFF_KTAB + (size_t)E * kDecReps * 8;     // (table: fp32 pairs, 16 copies)
  static constexpr size_t OFF_P = OFF_QS + (size_t)G * D * 4;               // [2][8 heads][TT] fp16 weights
  static constexpr size_t OFF_AL = OFF_P + 2 * 8 * (size_t)TT * 2;          // [2][KW][G] rescale factors
  static constexpr size_t OFF_GR = OFF_AL + 2 * (size_t)KW * G * 4;         // [2][KW] rescale flags
  static constexpr size_t OFF_RM = OFF_GR + 2 * (size_t)KW * 4;             // [KW][G] running max
  static constexpr size_t OFF_RL = OFF_RM + (size_t)KW * G * 4;             // [KW][G] running sum
  static constexpr size_t OFF_CENT = OFF_RL + (size_t)KW * G * 4;
  static constexpr size_t bytes = OFF_CENT + 16 * 4;
  static constexpr int MIN_BLOCKS = bytes <= 110 * 1024 ? 2 : 1;
};

__device__ __forceinline__ void mma_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int BITS, int G>
__global__ void __launch_bounds__(kDecThreads, MmaPlan<BITS, G>::MIN_BLOCKS)
attend_mma_kernel(const __grid_constant__ DecodeArgs a) {
  using P = MmaPlan<BITS, G>;
  constexpr int D = P::D, J = P::J, HG = P::HG, TT = P::TT, WT = P::WT, KW = P::KW, R = P::R;
  extern __shared__ __align__(16) uint8_t smem[];
  float* ktab = reinterpret_cast<float*>(smem + P::OFF_KTAB);
  float* qs = reinterpret_cast<float*>(smem + P::OFF_QS);
  __half* pbuf = reinterpret_cast<__half*>(smem + P::OFF_P);
  float* alpha_s = reinterpret_cast<float*>(smem + P::OFF_AL);
  int* grew_s = reinterpret_cast<int*>(smem + P::OFF_GR);
  float* red_m = reinterpret_cast<float*>(smem + P::OFF_RM);
  float* red_l = reinterpret_cast<float*>(smem + P::OFF_RL);
  float* cent = reinterpret_cast<float*>(smem + P::OFF_CENT);
  float* region = reinterpret_cast<float*>(smem);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool scorer = warp < KW;
  const int rtid = scorer ? tid : tid - 128;  // thread index within the role

  if (tid < 16) cent[tid] = a.cb.c[tid];
  for (int i = tid; i < 2 * 8 * TT / 2; i += kDecThreads) reinterpret_cast<uint32_t*>(pbuf)[i] = 0u;  // heads >= G: 0
  __syncthreads();
  build_pair_table<BITS, kDecReps>(cent, ktab);

  const int items = a.B * a.Hkv * a.splits;
  const size_t tiles_cap = static_cast<size_t>(a.Tcap / TT);
  for (int item = blockIdx.x; item < items; item += gridDim.x) {
    const int split = item % a.splits;
    const int hk = (item / a.splits) % a.Hkv;
    const int b = item / (a.splits * a.Hkv);
    const int len = row_len(a, b);
    const int start = split * a.chunk;
    const int end = min(start + a.chunk, len);
    const int ntiles = end > start ? (end - start + TT - 1) / TT : 0;
    const size_t kv_row0 = (static_cast<size_t>(b) * a.Hkv + hk) * a.Tcap;
    const float* qg = a.q + (static_cast<size_t>(b) * a.Hq + hk * G) * D;

    __syncthreads();  // the previous item is finished with the row factors, the stages and the merge region
    transform_queries<D, G>(qg, a.signs, a.mult, qs);
    __syncthreads();

    if (scorer) {
      // ================================= scoring role =================================
      const int sl = tid & 7, kord = sl >> 1;
      const int tk0 = warp * WT + ((tid >> 3) & 3) * 4;  // first token of this lane group, round 0
      const bool writer_lo = (sl & 1) == 0;
      const uint32_t rep_off = rep_offset<BITS, kDecReps>(lane);
      float2 qp[HG][J / 2];
      if constexpr (P::PASSES == 1) {
#pragma unroll
        for (int h = 0; h < HG; ++h)
#pragma unroll
          for (int i = 0; i < J / 2; ++i)
            qp[h][i] = make_float2(qs[h * D + J * sl + 2 * i], qs[h * D + J * sl + 2 * i + 1]);
      }
      float m_run[G], l_lane[G];
#pragma unroll
      for (int g = 0; g < G; ++g) { m_run[g] = -INFINITY; l_lane[g] = 0.f; }
      float kn_next[2], vn_next[2];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int t = start + tk0 + 16 * r + kord;
        kn_next[r] = (ntiles > 0 && t < end) ? __half2float(a.knorms[kv_row0 + t]) : 1.f;
        vn_next[r] = (ntiles > 0 && t < end) ? __half2float(a.vnorms[kv_row0 + t]) : 1.f;
      }
      auto issue_k = [&](int tile) {
        if (tile < ntiles) {
          const int t0 = start + tile * TT;
          role_copy_async<16>(smem + P::OFF_K + (tile % kStages) * P::STAGE, a.kcodes + (kv_row0 + t0) * R,
                              min(TT, end - t0) * R, rtid);
        }
        cp_async_commit();
      };
      issue_k(0);
      issue_k(1);
      for (int it = 0; it <= ntiles; ++it) {
        cp_async_wait<1>();  // tile it has landed; tile it + 1 may still be in flight
        roles_sync();
        issue_k(it + 2);     // into the stage tile it - 1 used
        if (it == ntiles) continue;
        const int t0 = start + it * TT;
        const int nt = min(TT, end - t0);
        const uint8_t* st = smem + P::OFF_K + (it % kStages) * P::STAGE;
        float kn_cur[2], vn_cur[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          kn_cur[r] = kn_next[r];
          vn_cur[r] = vn_next[r];
          const int t = t0 + TT + tk0 + 16 * r + kord;  // my tokens of the next tile
          if (it + 1 < ntiles && t < end) {
            kn_next[r] = __half2float(a.knorms[kv_row0 + t]);
            vn_next[r] = __half2float(a.vnorms[kv_row0 + t]);
          }
        }
        float z[2][G];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int tk = tk0 + 16 * r;
#pragma unroll
          for (int pass = 0; pass < P::PASSES; ++pass) {
            if constexpr (P::PASSES > 1) {
#pragma unroll
              for (int h = 0; h < HG; ++h)
#pragma unroll
                for (int i = 0; i < J / 2; ++i) {
                  const float* qrow = qs + (pass * HG + h) * D + J * sl + 2 * i;
                  qp[h][i] = make_float2(qrow[0], qrow[1]);
                }
            }
            float v[4][HG];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint64_t bits = load_slice<D, BITS, J>(st + (tk + (k ^ kord)) * R, sl);
              factored_slice<BITS, J, HG, kDecReps>(bits, reinterpret_cast<const uint8_t*>(ktab), rep_off, qp, v[k]);
            }
#pragma unroll
            for (int h = 0; h < HG; ++h) {
              v[0][h] += __shfl_xor_sync(0xffffffffu, v[2][h], 4);
              v[1][h] += __shfl_xor_sync(0xffffffffu, v[3][h], 4);
              v[0][h] += __shfl_xor_sync(0xffffffffu, v[1][h], 2);
              v[0][h] += __shfl_xor_sync(0xffffffffu, v[0][h], 1);
              z[r][pass * HG + h] = v[0][h];
            }
          }
        }
        // online softmax over this warp's 32 tokens of the tile
        bool grew = false;
        __half* pt = pbuf + (it & 1) * 8 * TT;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          float mx = -INFINITY;
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const bool valid = tk0 + 16 * r + kord < nt;
            z[r][g] = valid ? z[r][g] * kn_cur[r] : -INFINITY;
            mx = fmaxf(mx, z[r][g]);
          }
#pragma unroll
          for (int msk = 2; msk < 32; msk <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, msk));
          const float m_new = fmaxf(m_run[g], mx);
          const float alpha = (m_new == -INFINITY) ? 1.f : exp2f(m_run[g] - m_new);
          float psum = 0.f;
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const float p = (z[r][g] == -INFINITY) ? 0.f : exp2f(z[r][g] - m_new);
            psum += p;
            // weights P'[g][token] for the value MMAs (lanes 2m and 2m+1 hold the same token: split the heads)
            if ((g & 1) == (sl & 1) || G == 1) {
              if (G > 1 || writer_lo) pt[g * TT + tk0 + 16 * r + kord] = __float2half_rn(p * vn_cur[r]);
            }
          }
          l_lane[g] = l_lane[g] * alpha + (writer_lo ? psum : 0.f);
          grew |= m_new != m_run[g];
          m_run[g] = m_new;
          if (lane == 0) alpha_s[((it & 1) * KW + warp) * G + g] = alpha;
        }
        if (lane == 0) grew_s[(it & 1) * KW + warp] = grew ? 1 : 0;
      }
      cp_async_wait<0>();
      // merge, step 1: publish this warp's running max
      if (lane == 0) {
#pragma unroll
        for (int g = 0; g < G; ++g) red_m[warp * G + g] = m_run[g];
      }
      roles_sync();
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float M = red_m[g];
#pragma unroll
        for (int w2 = 1; w2 < KW; ++w2) M = fmaxf(M, red_m[w2 * G + g]);
        const float scl = (m_run[g] == -INFINITY) ? 0.f : exp2f(m_run[g] - M);
        const float l = warp_sum(l_lane[g]) * scl;
        if (lane == 0) red_l[warp * G + g] = l;
      }
    } else {
      // ================================== value role ==================================
      // value warp vw: tokens [32 vw, 32 vw + 32) of every tile; lane (gq, tq) = (lane / 4, lane % 4) holds the
      // accumulators of coordinates 16 m + gq (+ 8) and heads 2 tq (+ 1) for the 8 M-tiles m
      const int vw = warp - KW;
      const int gq = lane >> 2, tq = lane & 3;
      const uint32_t rep16 = static_cast<uint32_t>(lane & 15) << 4, rep8 = static_cast<uint32_t>(lane & 15) << 3;
      float acc[8][4];
#pragma unroll
      for (int m = 0; m < 8; ++m)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[m][c] = 0.f;
      auto issue_v = [&](int tile) {
        if (tile < ntiles) {
          const size_t tl = static_cast<size_t>(start / TT + tile);
          const uint8_t* src = static_cast<const uint8_t*>(a.v) + ((static_cast<size_t>(b) * a.Hkv + hk) * tiles_cap + tl) * P::STAGE;
          uint8_t* dst = smem + P::OFF_V + (tile % kStages) * P::STAGE;
          for (int o = rtid * 16; o < P::STAGE; o += 128 * 16) cp_async<16>(dst + stage_swizzle<R>(o), src + o);
        }
        cp_async_commit();
      };
      // the fp16 centroid pair of one coordinate at tokens 2p, 2p + 1 of this warp's slice (w: the slice's words)
      // (the scoring role's fp32 pair table, 16 copies at 128 B per entry, rounded to fp16 here)
      auto a_reg = [&](const uint32_t* w, int p) -> uint32_t {
        uint32_t off;
        if constexpr (BITS == 4)  // (byte * 256 + 16 (lane % 16)) / 2 = byte * 128 + 8 (lane % 16)
          off = __byte_perm(w[p >> 2], rep16, 0x5504u | (static_cast<uint32_t>(p & 3) << 4)) >> 1;
        else
          off = (bits_at<2 * BITS>(w, 2 * BITS * p) << 7) | rep8;
        const __half2 h = __float22half2_rn(*reinterpret_cast<const float2*>(reinterpret_cast<const uint8_t*>(ktab) + off));
        return *reinterpret_cast<const uint32_t*>(&h);
      };
      issue_v(0);
      for (int it = 0; it <= ntiles; ++it) {
        cp_async_wait<1>();  // tile it - 1 has landed; tile it may still be in flight
        roles_sync();
        issue_v(it + 1);     // into the stage tile it - 2 used
        if (it == 0) continue;
        const int j = it - 1;  // the tile scored in the previous step
        const int pb = j & 1;
        if (grew_s[pb * KW + vw]) {
          const float al0 = 2 * tq < G ? alpha_s[(pb * KW + vw) * G + 2 * tq] : 1.f;
          const float al1 = 2 * tq + 1 < G ? alpha_s[(pb * KW + vw) * G + 2 * tq + 1] : 1.f;
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            acc[m][0] *= al0; acc[m][1] *= al1; acc[m][2] *= al0; acc[m][3] *= al1;
          }
        }
        const uint8_t* vst = smem + P::OFF_V + (j % kStages) * P::STAGE;
        const __half* pt = pbuf + pb * 8 * TT + vw * WT;
        // B fragments: weights of head gq at tokens (2 tq, 2 tq + 1) and (+8) of each K-tile
        uint32_t bfr[2][2];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          bfr[k][0] = *reinterpret_cast<const uint32_t*>(pt + gq * TT + 16 * k + 2 * tq);
          bfr[k][1] = *reinterpret_cast<const uint32_t*>(pt + gq * TT + 16 * k + 2 * tq + 8);
        }
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          uint32_t w0[BITS + 1], w1[BITS + 1];  // this warp's slice of coordinate rows 16 m + gq and + 8
#pragma unroll
          for (int i = 0; i < BITS; ++i) {
            w0[i] = *reinterpret_cast<const uint32_t*>(vst + stage_swizzle<R>((16 * m + gq) * R + vw * P::SW + 4 * i));
            w1[i] = *reinterpret_cast<const uint32_t*>(vst + stage_swizzle<R>((16 * m + gq + 8) * R + vw * P::SW + 4 * i));
          }
          w0[BITS] = w1[BITS] = 0u;
#pragma unroll
          for (int k = 0; k < 2; ++k)
            mma_16816(acc[m], a_reg(w0, 8 * k + tq), a_reg(w1, 8 * k + tq), a_reg(w0, 8 * k + tq + 4),
                      a_reg(w1, 8 * k + tq + 4), bfr[k][0], bfr[k][1]);
        }
      }
      cp_async_wait<0>();
      roles_sync();  // merge, step 1 (the scoring warps publish their running max)
      // this warp's partial sums, rescaled to the common maximum, into the merge region [vw][head][coordinate]
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int g = 2 * tq + hh;
        if (g < G) {
          float M = red_m[g];
#pragma unroll
          for (int w2 = 1; w2 < KW; ++w2) M = fmaxf(M, red_m[w2 * G + g]);
          const float mw = red_m[vw * G + g];
          const float scl = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            region[(vw * 8 + g) * D + 16 * m + gq] = acc[m][hh] * scl;
            region[(vw * 8 + g) * D + 16 * m + gq + 8] = acc[m][2 + hh] * scl;
          }
        }
      }
    }
    __syncthreads();  // merge, step 2: every value warp's sums and every warp sum are in shared memory
    const size_t part0 = (static_cast<size_t>(b) * a.Hq + hk * G) * a.splits + split;  // head g adds g * splits
    for (int e = tid; e < G * D; e += kDecThreads) {
      const int g = e / D, jj = e % D;
      float s = 0.f;
#pragma unroll
      for (int r = 0; r < KW; ++r) s += region[(r * 8 + g) * D + jj];
      a.ws_o[(part0 + static_cast<size_t>(g) * a.splits) * D + jj] = s;
    }
    if (tid < G) {
      float M = red_m[tid], s = 0.f;
#pragma unroll
      for (int w2 = 1; w2 < KW; ++w2) M = fmaxf(M, red_m[w2 * G + tid]);
#pragma unroll
      for (int w2 = 0; w2 < KW; ++w2) s += red_l[w2 * G + tid];
      a.ws_l[part0 + static_cast<size_t>(tid) * a.splits] = s;
      a.ws_m[part0 + static_cast<size_t>(tid) * a.splits] = M;
    }
  }
}

}  // namespace axr
