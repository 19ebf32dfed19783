// Literal-table gather-sum kernels: the query's table itself sits in shared memory and every index of a token is one
// lookup in it, with no arithmetic on the key side beyond the adds.
//
// A token's packed index row is read as NI fields of W bits (an LSB-first bitstream); field i selects entry e of its
// own table of 2^W entries, and the token's score is the sum of the selected entries.  Each entry holds G fp32
// values, one per query head of a KV group, so one 16-byte load serves four heads that share the code stream.
//
//  * AXELRAM ("table lookup on read", Key Points, 2nd item): LUT[j][k] = q~_j c_k.  A field covers W / b
//    consecutive coordinates, and its entry e is the sum over those coordinates of q~_j c_(their indices in e):
//    W = 8 at b <= 2 (multi-coordinate byte-indexed tables: one byte covers 4 coordinates at b = 2, 8 at b = 1),
//    W = 6 at b = 3 (two coordinates), W = 4 at b = 4 (one), or smaller when the tables would not fit.  The score
//    is then times the stored norm.
//  * LOOKAT (product quantization with asymmetric distance computation): W = 8 and one field per subspace; entry k
//    of table i is q^(i) . C_i[k], C_i the subspace's codebook (K <= 256 centroids).
//
// Kernels: scores only (lut_score_kernel), and decode attention over fp16 values (table_attend_kernel with the
// LutScorer policy: the scores feed a per-warp online softmax and the value product on the CUDA cores; the splits
// are merged by attend_reduce_kernel).
#pragma once

#include <type_traits>

#include "decode.cuh"

namespace axr {

constexpr int kLutThreads = 256;

enum LutKind { kLutAxelram = 0, kLutPq = 1 };

struct LutArgs {
  const float* q;          // [B, Hq, D] f32
  const uint8_t* codes;    // [B, Hkv, Tcap, RB] index rows
  const __half* norms;     // [B, Hkv, Tcap] fp16 (AXELRAM) or null
  const int8_t* signs;     // [D] (AXELRAM)
  const float* pq_cb;      // [Hkv, NI, K, D / NI] f32 (LOOKAT)
  const __half* v;         // [B, Hkv, Tcap, D] fp16 (attend)
  const int32_t* seq_lens;  // [B] or null
  float* scores;           // [B, Hq, T] (scores)
  float* ws_o;             // [B, Hq, S, D] (attend partials, the layout of attend_reduce_kernel)
  float* ws_m;             // [B, Hq, S] running max, log2 units
  float* ws_l;             // [B, Hq, S]
  int B, Hq, Hkv, T, Tcap;
  int K;                   // LOOKAT: centroids per subspace
  int splits, chunk;
  float mult;              // folded into the table: scale (scores) or scale * log2(e) (attend)
  Codebook cb;             // AXELRAM
};

template <int D, int W, int NI, int G>
struct LutPlan {
  static constexpr int E = 1 << W;                       // entries per table
  static constexpr int RB = NI * W / 8;                  // bytes of a token's index row
  static_assert(NI * W % 8 == 0, "whole bytes per row");
  static constexpr int NW = (RB + 3) / 4 + 1;             // its 32-bit words, plus a zero word
  static constexpr size_t TAB = (size_t)NI * E * G * 4;
  static constexpr size_t OFF_QS = TAB;                  // [G][D] row factors
  static constexpr size_t OFF_CENT = OFF_QS + (size_t)G * D * 4;
  static constexpr size_t OFF_MERGE = OFF_CENT + 16 * 4;  // attend: [8 warps][G][D + 2]
  static constexpr size_t score_bytes = OFF_MERGE;
  static constexpr size_t attend_bytes = OFF_MERGE + (size_t)(kLutThreads / kWarp) * G * (D + 2) * 4;
};

// Cache row of token t: [B, Hkv, Tcap] numbering.
__device__ __forceinline__ size_t lut_row(const LutArgs& a, int b, int hk, int t) {
  return (static_cast<size_t>(b) * a.Hkv + hk) * a.Tcap + t;
}

__device__ __forceinline__ int lut_len(const LutArgs& a, int b) {
  if (!a.seq_lens) return a.T;
  const int n = a.seq_lens[b];
  return n < 0 ? 0 : (n > a.T ? a.T : n);
}

// The RB bytes of an index row into words w[0 .. NW) (the last word zero).
template <int RB, int NW>
__device__ __forceinline__ void lut_load_row(const uint8_t* p, uint32_t (&w)[NW]) {
#pragma unroll
  for (int i = 0; i < NW; ++i) w[i] = 0u;
  if constexpr (RB % 16 == 0) {
#pragma unroll
    for (int i = 0; i < RB / 16; ++i) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(p) + i);
      w[4 * i] = u.x; w[4 * i + 1] = u.y; w[4 * i + 2] = u.z; w[4 * i + 3] = u.w;
    }
  } else if constexpr (RB % 8 == 0) {
#pragma unroll
    for (int i = 0; i < RB / 8; ++i) {
      const uint2 u = __ldg(reinterpret_cast<const uint2*>(p) + i);
      w[2 * i] = u.x; w[2 * i + 1] = u.y;
    }
  } else if constexpr (RB % 4 == 0) {
#pragma unroll
    for (int i = 0; i < RB / 4; ++i) w[i] = __ldg(reinterpret_cast<const uint32_t*>(p) + i);
  } else {
    static_assert(RB == 2, "index rows of 2, 4k bytes");
    w[0] = __ldg(reinterpret_cast<const unsigned short*>(p));
  }
}

// Sum over the row's fields of the G-wide table entries they select.
template <int W, int NI, int G, int NW>
__device__ __forceinline__ void lut_gather(const float* __restrict__ tab, const uint32_t (&w)[NW], float (&acc)[G]) {
  constexpr int E = 1 << W;
#pragma unroll
  for (int h = 0; h < G; ++h) acc[h] = 0.f;
#pragma unroll
  for (int i = 0; i < NI; ++i) {
    const uint32_t e = bits_at<W>(w, i * W);
    const float* ent = tab + (static_cast<size_t>(i) * E + e) * G;
    if constexpr (G == 1) {
      acc[0] += ent[0];
    } else if constexpr (G == 2) {
      const float2 x = *reinterpret_cast<const float2*>(ent);
      acc[0] += x.x; acc[1] += x.y;
    } else {
#pragma unroll
      for (int c = 0; c < G / 4; ++c) {
        const float4 x = reinterpret_cast<const float4*>(ent)[c];
        acc[4 * c] += x.x; acc[4 * c + 1] += x.y; acc[4 * c + 2] += x.z; acc[4 * c + 3] += x.w;
      }
    }
  }
}

// AXELRAM tables: entry e of field i = sum over the field's W / b coordinates j of qs[h][j] c[index of j in e],
// qs = mult * q~ (transform_queries), c the unit-scale centroids.
template <int D, int BITS, int W, int NI, int G>
__device__ __forceinline__ void lut_build_axelram(const float* __restrict__ qs, const float* __restrict__ cent,
                                                  float* __restrict__ tab) {
  constexpr int CPF = W / BITS, L = 1 << BITS, E = 1 << W;
  static_assert(W % BITS == 0 && CPF * NI == D, "fields cover the coordinates");
  for (int idx = threadIdx.x; idx < NI * E; idx += blockDim.x) {
    const int i = idx / E, e = idx % E;
    float acc[G];
#pragma unroll
    for (int h = 0; h < G; ++h) acc[h] = 0.f;
#pragma unroll
    for (int c = 0; c < CPF; ++c) {
      const float cv = cent[(e >> (BITS * c)) & (L - 1)];
#pragma unroll
      for (int h = 0; h < G; ++h) acc[h] = fmaf(qs[h * D + i * CPF + c], cv, acc[h]);
    }
#pragma unroll
    for (int h = 0; h < G; ++h) tab[static_cast<size_t>(idx) * G + h] = acc[h];
  }
}

// LOOKAT tables: entry k of table i = qs[h]^(i) . C_i[k] for k < K (0 beyond), qs = mult * q.
template <int D, int NI, int G>
__device__ __forceinline__ void lut_build_pq(const float* __restrict__ qs, const float* __restrict__ cb, int K,
                                             float* __restrict__ tab) {
  constexpr int DS = D / NI, E = 256;
  for (int idx = threadIdx.x; idx < NI * E; idx += blockDim.x) {
    const int i = idx / E, e = idx % E;
    float acc[G];
#pragma unroll
    for (int h = 0; h < G; ++h) acc[h] = 0.f;
    if (e < K) {
      const float* c = cb + (static_cast<size_t>(i) * K + e) * DS;
#pragma unroll 4
      for (int j = 0; j < DS; ++j) {
        const float cv = __ldg(c + j);
#pragma unroll
        for (int h = 0; h < G; ++h) acc[h] = fmaf(qs[h * D + i * DS + j], cv, acc[h]);
      }
    }
#pragma unroll
    for (int h = 0; h < G; ++h) tab[static_cast<size_t>(idx) * G + h] = acc[h];
  }
}

// The item's table: row factors into shared memory, then the entries.
template <int D, int BITS, int W, int NI, int G, int KIND>
__device__ __forceinline__ void lut_build(const LutArgs& a, int b, int hk, uint8_t* smem) {
  using P = LutPlan<D, W, NI, G>;
  float* qs = reinterpret_cast<float*>(smem + P::OFF_QS);
  float* cent = reinterpret_cast<float*>(smem + P::OFF_CENT);
  float* tab = reinterpret_cast<float*>(smem);
  const float* qg = a.q + (static_cast<size_t>(b) * a.Hq + hk * G) * D;
  __syncthreads();  // the previous item is done with the table
  if constexpr (KIND == kLutAxelram) {
    if (threadIdx.x < 16) cent[threadIdx.x] = a.cb.c[threadIdx.x];
    transform_queries<D, G>(qg, a.signs, a.mult, qs);
  } else {
    for (int e = threadIdx.x; e < G * D; e += blockDim.x) qs[e] = qg[e] * a.mult;
  }
  __syncthreads();
  if constexpr (KIND == kLutAxelram)
    lut_build_axelram<D, BITS, W, NI, G>(qs, cent, tab);
  else
    lut_build_pq<D, NI, G>(qs, a.pq_cb + static_cast<size_t>(hk) * NI * a.K * (D / NI), a.K, tab);
  __syncthreads();
}

// Scores [B, Hq, T]: one block per (batch row, KV head, split), one token per thread per step (two in flight).
template <int D, int BITS, int W, int NI, int G, int KIND>
__global__ void __launch_bounds__(kLutThreads) lut_score_kernel(const __grid_constant__ LutArgs a) {
  using P = LutPlan<D, W, NI, G>;
  extern __shared__ __align__(16) uint8_t smem[];
  const float* tab = reinterpret_cast<const float*>(smem);
  const int items = a.B * a.Hkv * a.splits;
  for (int item = blockIdx.x; item < items; item += gridDim.x) {
    const int split = item % a.splits;
    const int hk = (item / a.splits) % a.Hkv;
    const int b = item / (a.splits * a.Hkv);
    const int start = split * a.chunk;
    const int end = min(start + a.chunk, a.T);
    const int vend = min(end, lut_len(a, b));
    float* out = a.scores + (static_cast<size_t>(b) * a.Hq + hk * G) * a.T;
    for (int t = max(start, vend) + threadIdx.x; t < end; t += kLutThreads)
#pragma unroll
      for (int h = 0; h < G; ++h) out[static_cast<size_t>(h) * a.T + t] = -INFINITY;
    if (vend <= start) continue;
    lut_build<D, BITS, W, NI, G, KIND>(a, b, hk, smem);
    const uint8_t* rows = a.codes + lut_row(a, b, hk, 0) * P::RB;
    const __half* nrm = KIND == kLutAxelram ? a.norms + lut_row(a, b, hk, 0) : nullptr;
    for (int t0 = start + threadIdx.x; t0 < vend; t0 += 2 * kLutThreads) {
      const int t1 = t0 + kLutThreads;
      uint32_t w0[P::NW], w1[P::NW];
      lut_load_row<P::RB>(rows + static_cast<size_t>(t0) * P::RB, w0);
      if (t1 < vend) lut_load_row<P::RB>(rows + static_cast<size_t>(t1) * P::RB, w1);
      else lut_load_row<P::RB>(rows + static_cast<size_t>(t0) * P::RB, w1);
      float n0 = 1.f, n1 = 1.f;
      if constexpr (KIND == kLutAxelram) {
        n0 = __half2float(nrm[t0]);
        n1 = t1 < vend ? __half2float(nrm[t1]) : 0.f;
      }
      float s0[G], s1[G];
      lut_gather<W, NI, G>(tab, w0, s0);
      lut_gather<W, NI, G>(tab, w1, s1);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        out[static_cast<size_t>(h) * a.T + t0] = s0[h] * n0;
        if (t1 < vend) out[static_cast<size_t>(h) * a.T + t1] = s1[h] * n1;
      }
    }
  }
}

// The literal-table scorer as a policy of table_attend_kernel: the item's table is built in shared memory, a token's
// scores are the gathered entries times its norm (AXELRAM), in log2 units (mult holds scale * log2(e)).
template <int D, int BITS, int W, int NI, int G, int KIND>
struct LutScorer {
  using P = LutPlan<D, W, NI, G>;
  static constexpr bool EXACT = false;           // scores are real numbers; rescales through exp2
  static constexpr size_t SMEM = P::OFF_MERGE;   // bytes before the merge region
  __device__ static void build(const LutArgs& a, int b, int hk, uint8_t* smem) {
    lut_build<D, BITS, W, NI, G, KIND>(a, b, hk, smem);
  }
  struct Row {  // a token's index row and norm, loaded a tile ahead of its scoring
    uint32_t w[P::NW];
    unsigned short n;
  };
  __device__ static void load(const LutArgs& a, size_t row0, int t, Row& r) {
    lut_load_row<P::RB>(a.codes + (row0 + t) * P::RB, r.w);
    r.n = KIND == kLutAxelram ? __ldg(reinterpret_cast<const unsigned short*>(a.norms) + row0 + t) : 0;
  }
  __device__ static void score(const LutArgs& a, const uint8_t* smem, const Row& r, bool valid, float (&z)[G]) {
    lut_gather<W, NI, G>(reinterpret_cast<const float*>(smem), r.w, z);
    const float n = KIND == kLutAxelram ? __half2float(__ushort_as_half(r.n)) : 1.f;
#pragma unroll
    for (int h = 0; h < G; ++h) z[h] = valid ? z[h] * n : -INFINITY;
  }
};

// Decode attention over fp16 values: tiles of 256 tokens, thread t scores token t of the tile through the scorer S;
// warp w keeps the online softmax of its 32 tokens of every tile (max in log2 units) and the value product over
// them, each lane holding D / 32 coordinates of every head.  At the end of an item the warps merge into the split's
// partial (the layout of attend_reduce_kernel).  With S::EXACT the scores are integers in the log2 domain: every
// weight and every rescale is an exact power of two (ldexp), never a rounded exponential.
template <int D, int G, class S>
__global__ void __launch_bounds__(kLutThreads) table_attend_kernel(const __grid_constant__ LutArgs a) {
  constexpr int DPL = D / kWarp;  // coordinates per lane
  constexpr int WARPS = kLutThreads / kWarp;
  static_assert(DPL == 2 || DPL == 4, "d = 64 or 128");
  extern __shared__ __align__(16) uint8_t smem[];
  float* merge = reinterpret_cast<float*>(smem + S::SMEM);  // [warp][G][D + 2]: o, then m, l
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int items = a.B * a.Hkv * a.splits;
  auto pow2 = [](float x) { return S::EXACT ? ldexpf(1.f, static_cast<int>(x)) : exp2f(x); };
  for (int item = blockIdx.x; item < items; item += gridDim.x) {
    const int split = item % a.splits;
    const int hk = (item / a.splits) % a.Hkv;
    const int b = item / (a.splits * a.Hkv);
    const int start = split * a.chunk;
    const int end = min(min(start + a.chunk, a.T), lut_len(a, b));
    const size_t part0 = (static_cast<size_t>(b) * a.Hq + hk * G) * a.splits + split;  // head g adds g * splits
    if (end <= start) {  // an empty split: nothing to merge
      for (int e = tid; e < G * D; e += kLutThreads)
        a.ws_o[(part0 + static_cast<size_t>(e / D) * a.splits) * D + e % D] = 0.f;
      if (tid < G) {
        a.ws_m[part0 + static_cast<size_t>(tid) * a.splits] = -INFINITY;
        a.ws_l[part0 + static_cast<size_t>(tid) * a.splits] = 0.f;
      }
      continue;
    }
    const size_t row0 = lut_row(a, b, hk, 0);
    const __half* vrow = a.v + row0 * D + lane * DPL;
    // value rows of the warp's 32 tokens of a tile travel in batches of 8 through two register buffers: each is
    // refilled as soon as it is consumed, with the tile's next batch or the first batches of the warp's next tile
    // (which do not wait for that tile's scores), so 16 rows stay in flight
    using VRaw = typename std::conditional<DPL == 4, uint2, unsigned int>::type;
    VRaw va[8], vb[8];
    auto load8 = [&](VRaw (&buf)[8], int wt0, int nw, int k0) {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int tok = wt0 + min(k0 + k, nw - 1);
        buf[k] = __ldg(reinterpret_cast<const VRaw*>(vrow + static_cast<size_t>(tok) * D));
      }
    };
    float m_run[G], l_lane[G], o[G][DPL];
    auto pv8 = [&](const VRaw (&buf)[8], int k0, int nw, const float (&p)[G]) {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        if (k0 + k >= nw) break;
        float2 vv[DPL / 2];
        if constexpr (DPL == 4) {
          const uint2 u = reinterpret_cast<const uint2&>(buf[k]);
          vv[0] = __half22float2(*reinterpret_cast<const __half2*>(&u.x));
          vv[1] = __half22float2(*reinterpret_cast<const __half2*>(&u.y));
        } else {
          const unsigned int u = reinterpret_cast<const unsigned int&>(buf[k]);
          vv[0] = __half22float2(*reinterpret_cast<const __half2*>(&u));
        }
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float pk = __shfl_sync(0xffffffffu, p[h], k0 + k);
#pragma unroll
          for (int c = 0; c < DPL / 2; ++c) {
            o[h][2 * c] = fmaf(pk, vv[c].x, o[h][2 * c]);
            o[h][2 * c + 1] = fmaf(pk, vv[c].y, o[h][2 * c + 1]);
          }
        }
      }
    };
    {
      const int wt0 = start + warp * kWarp, nw = min(kWarp, end - wt0);
      if (nw > 0) load8(va, wt0, nw, 0);
      if (nw > 8) load8(vb, wt0, nw, 8);
    }
    typename S::Row row;  // this thread's token of the current tile, loaded one tile ahead
    S::load(a, row0, min(start + tid, end - 1), row);
    S::build(a, b, hk, smem);
#pragma unroll
    for (int h = 0; h < G; ++h) {
      m_run[h] = -INFINITY;
      l_lane[h] = 0.f;
#pragma unroll
      for (int c = 0; c < DPL; ++c) o[h][c] = 0.f;
    }
    for (int t0 = start; t0 < end; t0 += kLutThreads) {
      const int t = t0 + tid;
      float z[G];
      S::score(a, smem, row, t < end, z);
      if (t0 + kLutThreads < end) S::load(a, row0, min(t + kLutThreads, end - 1), row);  // the next tile's
      float p[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float mx = warp_max(z[h]);
        const float m_new = fmaxf(m_run[h], mx);
        // nothing has accumulated while the running max is -inf; otherwise m_new >= m_run is finite
        const float alpha = (m_run[h] == -INFINITY) ? 0.f : pow2(m_run[h] - m_new);
        p[h] = (z[h] == -INFINITY) ? 0.f : pow2(z[h] - m_new);
        l_lane[h] = l_lane[h] * alpha + p[h];
        m_run[h] = m_new;
#pragma unroll
        for (int c = 0; c < DPL; ++c) o[h][c] *= alpha;
      }
      // a tile with a successor is full (every warp has 32 tokens); only the last tile can be partial
      const int wt0 = t0 + warp * kWarp, nw = min(kWarp, end - wt0);
      const int nx0 = wt0 + kLutThreads, nxw = min(kWarp, end - nx0);
      if (nw > 0) pv8(va, 0, nw, p);
      if (nw > 16) load8(va, wt0, nw, 16);
      else if (nxw > 0) load8(va, nx0, nxw, 0);
      if (nw > 8) pv8(vb, 8, nw, p);
      if (nw > 24) load8(vb, wt0, nw, 24);
      else if (nxw > 8) load8(vb, nx0, nxw, 8);
      if (nw > 16) {
        pv8(va, 16, nw, p);
        if (nxw > 0) load8(va, nx0, nxw, 0);
      }
      if (nw > 24) {
        pv8(vb, 24, nw, p);
        if (nxw > 8) load8(vb, nx0, nxw, 8);
      }
    }
    // merge the warps: each publishes o, m and its l; then every (head, coordinate) sums the rescaled parts
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float* mw = merge + (static_cast<size_t>(warp) * G + h) * (D + 2);
#pragma unroll
      for (int c = 0; c < DPL; ++c) mw[lane * DPL + c] = o[h][c];
      const float l = warp_sum(l_lane[h]);
      if (lane == 0) { mw[D] = m_run[h]; mw[D + 1] = l; }
    }
    __syncthreads();
    for (int e = tid; e < G * D; e += kLutThreads) {
      const int h = e / D, j = e % D;
      float M = -INFINITY;
#pragma unroll
      for (int w2 = 0; w2 < WARPS; ++w2) M = fmaxf(M, merge[(w2 * G + h) * (D + 2) + D]);
      float sum = 0.f, ls = 0.f;
#pragma unroll
      for (int w2 = 0; w2 < WARPS; ++w2) {
        const float* mw = merge + (w2 * G + h) * (D + 2);
        const float f = (mw[D] == -INFINITY) ? 0.f : pow2(mw[D] - M);
        sum = fmaf(f, mw[j], sum);
        ls = fmaf(f, mw[D + 1], ls);
      }
      const size_t part = part0 + static_cast<size_t>(h) * a.splits;
      a.ws_o[part * D + j] = sum;
      if (j == 0) {
        a.ws_m[part] = M;
        a.ws_l[part] = ls;
      }
    }
    __syncthreads();  // the merge region is free again
  }
}

}  // namespace axr
