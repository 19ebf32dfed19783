// Decode-time read path: table scorer, split-T online-softmax . V partial kernel, split merge.
//
// AXELRAM Key Points (1st, 2nd items) and Abstract: the query is transformed once, a d x 2^b table of
// q~_j * c_k is built, and each cached token's score is the gather-sum of table entries at its stored indices times
// its stored norm -- no per-token inverse transform and no key reconstruction.  Softmax and the value product are
// not on the pages; they follow the standard split-T ("flash-decoding") formulation: each block owns a token range,
// keeps a running max and sum per query head, and a second kernel merges the ranges.
//
// Two ways to read the table are implemented (both give the table's values up to fp32 rounding):
//   * TABLE    -- the table LUT[j][k][h] = q~_{h,j} c_k is materialised in shared memory and each token gathers
//                 one G-wide entry per coordinate (one thread per token).
//   * FACTORED -- the table is kept in factored form: its row factor q~_{h,j} sits in registers of the thread that
//                 owns coordinate j, its column factor is gathered from a byte-indexed table of centroid pairs
//                 (c_{k1}, c_{k2}) -- two coordinates per lookup, replicated across banks -- and the product is
//                 formed by a packed fp32x2 FMA that also accumulates it.  On B200 this needs half the shared-memory
//                 wavefronts of TABLE per score (a 16-entry row of G-wide entries spans 2 wavefronts per warp
//                 request, a replicated pair table 1 per coordinate pair), which is what bounds the gather.
#pragma once

#include "axr_host.h"

namespace axr {

constexpr int kDecThreads = 256;
constexpr int kDecWarps = kDecThreads / kWarp;
constexpr float kLog2e = 1.4426950408889634f;

enum Gather { kGatherFactored = 0, kGatherTable = 1 };

struct DecodeArgs {
  const float* q;            // [B, Hq, D]
  const uint8_t* kcodes;     // [B, Hkv, Tcap, R]
  const __half* knorms;      // [B, Hkv, Tcap]
  const __half* kdense;      // [B, Hkv, Tcap, D] (dense reference only)
  const void* v;             // fp16 [B, Hkv, Tcap, D] or codes [B, Hkv, Tcap, R]
  const __half* vnorms;      // [B, Hkv, Tcap] (quantized V)
  const int32_t* seq_lens;   // [B] or null
  const int8_t* signs;       // [D]
  float* scores;             // [B, Hq, T] (scorer)
  float* ws_o;               // [B, Hq, S, D]
  float* ws_m;               // [B, Hq, S]  running max, log2 units
  float* ws_l;               // [B, Hq, S]  running sum
  float* out;                // [B, Hq, D]
  int B, Hq, Hkv, T, Tcap;
  int splits, chunk;
  float mult;                // factor folded into the table (score: scale; attend: scale * log2(e))
  Codebook cb;
};

__device__ __forceinline__ int row_len(const DecodeArgs& a, int b) {
  if (!a.seq_lens) return a.T;
  int n = a.seq_lens[b];
  return n < 0 ? 0 : (n > a.T ? a.T : n);
}

// ---- asynchronous global -> shared copies ------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

template <int BYTES>
__device__ __forceinline__ void cp_async(void* dst, const void* src) {
  if constexpr (BYTES == 16)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(dst)), "l"(src));
  else
    asm volatile("cp.async.ca.shared.global [%0], [%1], %2;\n" ::"r"(smem_u32(dst)), "l"(src), "n"(BYTES));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

// Copy `bytes` (a multiple of CH) from global to shared, spread over the block.
template <int CH>
__device__ __forceinline__ void block_copy_async(uint8_t* dst, const uint8_t* src, int bytes) {
  for (int o = threadIdx.x * CH; o < bytes; o += kDecThreads * CH) cp_async<CH>(dst + o, src + o);
}

// ---- query transform ---------------------------------------------------------------------------------------------

// qs[g][j] = mult * (H (s .* q_g))_j for the G query heads of this KV head (warp g transforms head g).
template <int D, int G>
__device__ __forceinline__ void transform_queries(const float* __restrict__ q, const int8_t* __restrict__ signs,
                                                  float mult, float* __restrict__ qs) {
  constexpr int VPL = WarpVec<D>::VPL;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float norm = mult * rsqrtf(static_cast<float>(D));
  for (int g = warp; g < G; g += kDecWarps) {
    float v[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int j = lane * VPL + i;
      v[i] = q[g * D + j] * sign_of(signs[j]);
    }
    fwht_warp<D>(v, lane);
#pragma unroll
    for (int i = 0; i < VPL; ++i) qs[g * D + lane * VPL + i] = v[i] * norm;
  }
}

// ---- factored gather: byte-indexed centroid-pair table -------------------------------------------------------------

// Entry e (the 2b-bit code of two consecutive coordinates, low coordinate in the low bits) holds (c[e & (L-1)],
// c[e >> b]).  The table is replicated once per lane, entry-major with a 256-byte entry stride: lane l reads copy
// l at byte offset e * 256 + 8 l, so a warp's 32 lookups never share a bank with a different address beyond the
// two wavefronts a 64-bit warp load needs, and the offset of a pair is one byte permute of the packed code word
// (entry index into byte 1, the lane's copy offset into byte 0).
template <int BITS>
struct PairTable {
  static constexpr int L = 1 << BITS;
  static constexpr int E = L * L;
  static constexpr int REPS = 32;
  static constexpr int FLOATS = E * REPS * 2;
};

template <int BITS>
__device__ __forceinline__ void build_pair_table(const float* __restrict__ cent, float* __restrict__ tab) {
  using P = PairTable<BITS>;
  for (int i = threadIdx.x; i < P::E * P::REPS; i += kDecThreads) {
    const int e = i / P::REPS;
    tab[2 * i] = cent[e & (P::L - 1)];
    tab[2 * i + 1] = cent[e >> BITS];
  }
}

// Byte offset of this lane's copy of pair i (coordinates 2i, 2i+1) of a packed slice.  repw = 8 * lane.
template <int BITS>
__device__ __forceinline__ uint32_t pair_addr(uint64_t bits, int i, uint32_t repw) {
  if constexpr (BITS == 4) {
    const uint32_t w = i < 4 ? static_cast<uint32_t>(bits) : static_cast<uint32_t>(bits >> 32);
    return __byte_perm(w, repw, 0x5504u | (static_cast<uint32_t>(i & 3) << 4));
  } else {
    constexpr uint32_t MASK = (1u << (2 * BITS)) - 1u;
    return ((static_cast<uint32_t>(bits >> (2 * BITS * i)) & MASK) << 8) | repw;
  }
}

// The J*b bits of coordinates [J*sl, J*sl + J) of one packed row held in shared memory, as a 64-bit value.
template <int D, int BITS, int J>
__device__ __forceinline__ uint64_t load_slice(const uint8_t* row, int sl) {
  constexpr int NB = J * BITS / 8;  // bytes, <= 8
  const uint8_t* p = row + sl * NB;
  if constexpr (NB == 8) return *reinterpret_cast<const uint64_t*>(p);
  else if constexpr (NB == 4) return *reinterpret_cast<const uint32_t*>(p);
  else if constexpr (NB == 2) return *reinterpret_cast<const uint16_t*>(p);
  else if constexpr (NB == 1) return *p;
  else if constexpr (NB == 6) {
    const uint16_t* h = reinterpret_cast<const uint16_t*>(p);
    return static_cast<uint64_t>(h[0]) | (static_cast<uint64_t>(h[1]) << 16) | (static_cast<uint64_t>(h[2]) << 32);
  } else {  // NB == 3
    return static_cast<uint64_t>(p[0]) | (static_cast<uint64_t>(p[1]) << 8) | (static_cast<uint64_t>(p[2]) << 16);
  }
}

// Partial dot products of one token's slice with the HG heads' row factors: acc[h] = sum over the slice's coordinate
// pairs of (q~_{h,2i}, q~_{h,2i+1}) . (c, c') -- the packed FMA keeps even and odd coordinates in the two halves.
template <int BITS, int J, int HG>
__device__ __forceinline__ void factored_slice(uint64_t bits, const uint8_t* tab, uint32_t rep_off,
                                               const float2 (&qp)[HG][J / 2], float (&acc)[HG]) {
  float2 a[HG];
#pragma unroll
  for (int h = 0; h < HG; ++h) a[h] = make_float2(0.f, 0.f);
#pragma unroll
  for (int i = 0; i < J / 2; ++i) {
    const float2 c = *reinterpret_cast<const float2*>(tab + pair_addr<BITS>(bits, i, rep_off));
#pragma unroll
    for (int h = 0; h < HG; ++h) a[h] = fma2(qp[h][i], c, a[h]);
  }
#pragma unroll
  for (int h = 0; h < HG; ++h) acc[h] = a[h].x + a[h].y;
}

// ---- shared-memory plan of the decode kernels ---------------------------------------------------------------------

constexpr int kTT = 256;     // tokens per tile of the scorer
constexpr int kStages = 2;   // cp.async pipeline depth of the scorer

// Decode tiles are 128 tokens (one key-phase round): two stages of quantized keys and values plus the pair table
// leave room for two blocks per SM; fp16 values take three stages and one block per SM.
template <int D, int BITS, int G, bool VQ, bool DENSE>
struct DecPlan {
  static constexpr int TT = 128;
  static constexpr int NST = (!VQ && !DENSE) ? 3 : 2;     // cp.async pipeline depth
  static constexpr int L = 1 << BITS;
  static constexpr int R = D * BITS / 8;
  static constexpr int KROW = DENSE ? 2 * D : R;          // bytes per key row in the stage
  static constexpr int VROW = VQ ? R : 2 * D;             // bytes per value row
  static constexpr int KCH = (KROW % 16 == 0) ? 16 : 8;   // cp.async chunk for key rows
  static constexpr int VCH = (VROW % 16 == 0) ? 16 : 8;
  static constexpr int STAGE_K = TT * KROW;
  static constexpr int STAGE_V = TT * VROW;
  static constexpr int STAGE = STAGE_K + STAGE_V;
  static constexpr int LPT = 8;                           // key-phase lanes per token
  static constexpr int J = D / LPT;                       // coordinates per lane
  static constexpr int HG = G < 4 ? G : 4;                // heads per key-phase pass
  static constexpr int PASSES = G / HG;
  static constexpr int TPR = D / 8;                       // value-phase threads per token row (8 coordinates each)
  static constexpr int NG = kDecThreads / TPR;            // value-phase token groups
  static constexpr int TAB = DENSE ? 0 : PairTable<BITS>::FLOATS;
  static constexpr int REDUCE = NG * G * D;               // final cross-group sum (reuses the stages)
  // byte offsets
  static constexpr size_t OFF_STAGE = 0;
  static constexpr size_t STAGES_BYTES = (size_t)NST * STAGE;
  static constexpr size_t OFF_TAB = ((STAGES_BYTES > REDUCE * 4 ? STAGES_BYTES : REDUCE * 4) + 15) / 16 * 16;
  static constexpr size_t OFF_QS = OFF_TAB + (size_t)TAB * 4;
  static constexpr size_t OFF_PS = OFF_QS + (size_t)G * D * 4;          // weights [TT][G] float2
  static constexpr size_t OFF_RED = OFF_PS + (size_t)TT * G * 8;
  static constexpr size_t OFF_CENT = OFF_RED + (size_t)kDecWarps * G * 4;
  static constexpr size_t bytes = OFF_CENT + 16 * 4;
};

// ---- the partial kernel ------------------------------------------------------------------------------------------
//
// Per tile of TT = 128 tokens (cp.async staging of key codes and values, norms prefetched to registers), each warp
// w owns tokens [16w, 16w + 16) of the tile end to end, so the softmax state is warp-local:
//   key phase   -- 8 lanes per token, each lane owning D/8 coordinates and the matching row factors in registers;
//                  a lane group of 8 scores 4 tokens; the 8 partial sums of a token are combined by a select-free
//                  butterfly (lane sl processes token k ^ (sl >> 1) at step k), after which lanes 2m, 2m+1 hold
//                  token m of the group;
//   softmax     -- the warp's running max per head is updated from its 16 new scores (shuffles over the warp); the
//                  weights p (times the value norm for quantized values) go to shared memory for the warp only;
//   value phase -- the same warp accumulates coordinates [8vc, 8vc+8) of its 16 tokens, D/8 lanes per token row.
// The warps' (max, sum, accumulator) triples are merged once in the epilogue.
template <int D, int BITS, int G, bool VQ, bool DENSE>
__global__ void __launch_bounds__(kDecThreads, (VQ && G <= 4) ? 2 : 1)
attend_partial_kernel(const __grid_constant__ DecodeArgs a) {
  using P = DecPlan<D, BITS, G, VQ, DENSE>;
  constexpr int J = P::J, HG = P::HG, TPR = P::TPR, NG = P::NG;
  constexpr int TT = P::TT;
  constexpr int RPW = kWarp / TPR;          // value rows a warp reads at once
  constexpr int WT = 16;                    // tokens per warp per tile
  static_assert(TT == kDecWarps * WT, "each warp owns 16 tokens of a tile");
  extern __shared__ __align__(16) uint8_t smem[];
  float* tab = reinterpret_cast<float*>(smem + P::OFF_TAB);
  float* qs = reinterpret_cast<float*>(smem + P::OFF_QS);
  float2* ps = reinterpret_cast<float2*>(smem + P::OFF_PS);
  float* red = reinterpret_cast<float*>(smem + P::OFF_RED);
  float* cent = reinterpret_cast<float*>(smem + P::OFF_CENT);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = blockIdx.z, hk = blockIdx.y, split = blockIdx.x;
  const int len = row_len(a, b);
  const int start = split * a.chunk;
  const int end = min(start + a.chunk, len);
  const int ntiles = end > start ? (end - start + TT - 1) / TT : 0;
  const size_t kv_row0 = (static_cast<size_t>(b) * a.Hkv + hk) * a.Tcap;
  const float* qg = a.q + (static_cast<size_t>(b) * a.Hq + hk * G) * D;
  const uint8_t* ksrc = DENSE ? reinterpret_cast<const uint8_t*>(a.kdense) : a.kcodes;
  const uint8_t* vsrc = static_cast<const uint8_t*>(a.v);

  auto issue_tile = [&](int tile) {
    if (tile < ntiles) {
      uint8_t* st = smem + P::OFF_STAGE + static_cast<size_t>(tile % P::NST) * P::STAGE;
      const int t0 = start + tile * TT;
      const int n = min(TT, end - t0);
      block_copy_async<P::KCH>(st, ksrc + (kv_row0 + t0) * P::KROW, n * P::KROW);
      block_copy_async<P::VCH>(st + P::STAGE_K, vsrc + (kv_row0 + t0) * P::VROW, n * P::VROW);
    }
    cp_async_commit();
  };

  // prologue: start the copies, then build the per-block tables while they fly
  for (int s = 0; s < P::NST - 1; ++s) issue_tile(s);
  if (tid < 16) cent[tid] = a.cb.c[tid];
  if constexpr (DENSE) {
    for (int e = tid; e < G * D; e += kDecThreads) qs[e] = qg[e] * a.mult;  // fp16 keys: untransformed query
  } else {
    transform_queries<D, G>(qg, a.signs, a.mult, qs);
  }
  __syncthreads();
  if constexpr (!DENSE) build_pair_table<BITS>(cent, tab);

  // key-phase lane roles: the token this lane's pair holds after the butterfly is fixed for every tile
  const int sl = tid & 7;                            // slice of coordinates [J*sl, J*sl + J)
  const int kord = sl >> 1;                          // token order xor for the butterfly
  const int tk = warp * WT + ((tid >> 3) & 3) * 4;   // first token of this lane group
  const int my_t = tk + kord;                        // token held after the butterfly
  const bool writer_lo = (sl & 1) == 0;              // the pair's even lane writes heads [0, G/2)
  const uint32_t rep_off = static_cast<uint32_t>(lane) << 3;
  float2 qp[HG][J / 2];
  if constexpr (P::PASSES == 1) {
#pragma unroll
    for (int h = 0; h < HG; ++h)
#pragma unroll
      for (int i = 0; i < J / 2; ++i) qp[h][i] = make_float2(qs[h * D + J * sl + 2 * i], qs[h * D + J * sl + 2 * i + 1]);
  }

  // norms of my token in the first tile
  float kn_next = 1.f, vn_next = 1.f;
  if (ntiles > 0 && start + my_t < end) {
    if constexpr (!DENSE) kn_next = __half2float(a.knorms[kv_row0 + start + my_t]);
    if constexpr (VQ) vn_next = __half2float(a.vnorms[kv_row0 + start + my_t]);
  }

  // value-phase roles and state (warp-local)
  const int vrow = lane / TPR, vc = lane % TPR;
  float2 acc[G][4];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[g][c] = make_float2(0.f, 0.f);
  float m_run[G], l_lane[G];
#pragma unroll
  for (int g = 0; g < G; ++g) { m_run[g] = -INFINITY; l_lane[g] = 0.f; }

  for (int tile = 0; tile < ntiles; ++tile) {
    const int t0 = start + tile * TT;
    const int nt = min(TT, end - t0);
    cp_async_wait<P::NST - 2>();
    __syncthreads();  // this tile's stage is complete, and every thread is done with the previous tile
    issue_tile(tile + P::NST - 1);  // refills the stage the previous tile used
    const uint8_t* st = smem + P::OFF_STAGE + static_cast<size_t>(tile % P::NST) * P::STAGE;
    const float kn_cur = kn_next, vn_cur = vn_next;
    if (tile + 1 < ntiles && t0 + TT + my_t < end) {  // prefetch my token's norms of the next tile
      if constexpr (!DENSE) kn_next = __half2float(a.knorms[kv_row0 + t0 + TT + my_t]);
      if constexpr (VQ) vn_next = __half2float(a.vnorms[kv_row0 + t0 + TT + my_t]);
    }

    // ---- key phase ----
    float z[G];
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
        const int tt = tk + (k ^ kord);
        if constexpr (DENSE) {
          const __half2* kh = reinterpret_cast<const __half2*>(st + tt * P::KROW + 2 * J * sl);
          float2 s2[HG];
#pragma unroll
          for (int h = 0; h < HG; ++h) s2[h] = make_float2(0.f, 0.f);
#pragma unroll
          for (int i = 0; i < J / 2; ++i) {
            const float2 kf = __half22float2(kh[i]);
#pragma unroll
            for (int h = 0; h < HG; ++h) s2[h] = fma2(qp[h][i], kf, s2[h]);
          }
#pragma unroll
          for (int h = 0; h < HG; ++h) v[k][h] = s2[h].x + s2[h].y;
        } else {
          const uint64_t bits = load_slice<D, BITS, J>(st + tt * P::KROW, sl);
          factored_slice<BITS, J, HG>(bits, reinterpret_cast<const uint8_t*>(tab), rep_off, qp, v[k]);
        }
      }
#pragma unroll
      for (int h = 0; h < HG; ++h) {
        v[0][h] += __shfl_xor_sync(0xffffffffu, v[2][h], 4);
        v[1][h] += __shfl_xor_sync(0xffffffffu, v[3][h], 4);
        v[0][h] += __shfl_xor_sync(0xffffffffu, v[1][h], 2);
        v[0][h] += __shfl_xor_sync(0xffffffffu, v[0][h], 1);
        z[pass * HG + h] = v[0][h];
      }
    }

    // ---- warp-local online softmax over this warp's 16 tokens ----
    const bool valid = my_t < nt;
    bool grew = false;
    float alpha[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      z[g] = valid ? z[g] * kn_cur : -INFINITY;
      float mx = z[g];
#pragma unroll
      for (int msk = 2; msk < 32; msk <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, msk));
      const float m_new = fmaxf(m_run[g], mx);
      alpha[g] = (m_new == -INFINITY) ? 1.f : exp2f(m_run[g] - m_new);
      const float p = valid ? exp2f(z[g] - m_new) : 0.f;
      l_lane[g] = l_lane[g] * alpha[g] + (writer_lo ? p : 0.f);
      grew |= m_new != m_run[g];
      m_run[g] = m_new;
      z[g] = p * (VQ ? vn_cur : 1.f);
    }
    {
      float2* row = ps + static_cast<size_t>(my_t) * G;
      constexpr int HALF = G > 1 ? G / 2 : 1;
      if (G > 1 || writer_lo) {
#pragma unroll
        for (int h = 0; h < HALF; ++h) {
          const int g = (writer_lo ? 0 : HALF) + h;
          row[g] = make_float2(z[g], z[g]);
        }
      }
    }
    if (grew) {  // warp-uniform
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int c = 0; c < 4; ++c) { acc[g][c].x *= alpha[g]; acc[g][c].y *= alpha[g]; }
    }
    __syncwarp();

    // ---- value phase: this warp's 16 tokens ----
    const uint8_t* vst = st + P::STAGE_K;
#pragma unroll 2
    for (int i = 0; i < WT / RPW; ++i) {
      const int tt = warp * WT + vrow + RPW * i;
      if (tt >= nt) break;
      float2 pw[G];
#pragma unroll
      for (int g = 0; g < G; ++g) pw[g] = ps[tt * G + g];
      float2 val[4];
      if constexpr (VQ) {
        const uint64_t bits = load_slice<D, BITS, 8>(vst + tt * P::VROW, vc);
#pragma unroll
        for (int c = 0; c < 4; ++c)
          val[c] = *reinterpret_cast<const float2*>(reinterpret_cast<const uint8_t*>(tab) +
                                                    pair_addr<BITS>(bits, c, rep_off));
      } else {
        const uint4 u = *reinterpret_cast<const uint4*>(vst + tt * P::VROW + 16 * vc);
        val[0] = __half22float2(*reinterpret_cast<const __half2*>(&u.x));
        val[1] = __half22float2(*reinterpret_cast<const __half2*>(&u.y));
        val[2] = __half22float2(*reinterpret_cast<const __half2*>(&u.z));
        val[3] = __half22float2(*reinterpret_cast<const __half2*>(&u.w));
      }
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[g][c] = fma2(pw[g], val[c], acc[g][c]);
    }
  }
  cp_async_wait<0>();
  __syncthreads();  // every stage is idle: reuse it for the cross-warp merge

  // ---- epilogue: merge the warps' (max, sum, accumulator) ----
  float* region = reinterpret_cast<float*>(smem + P::OFF_STAGE);
  if (lane == 0) {
#pragma unroll
    for (int g = 0; g < G; ++g) red[warp * G + g] = m_run[g];
  }
  __syncthreads();
  float scl[G], Mblk[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float M = red[g];
#pragma unroll
    for (int w2 = 1; w2 < kDecWarps; ++w2) M = fmaxf(M, red[w2 * G + g]);
    scl[g] = (m_run[g] == -INFINITY) ? 0.f : exp2f(m_run[g] - M);
    const float l = warp_sum(l_lane[g]) * scl[g];
    l_lane[g] = l;  // this warp's rescaled sum (uniform over the warp)
    Mblk[g] = M;
  }
  __syncthreads();  // red is rewritten below
  if (lane == 0) {
#pragma unroll
    for (int g = 0; g < G; ++g) red[warp * G + g] = l_lane[g];
  }
  const int vg = warp * RPW + vrow;  // value group: one per (warp, row slot)
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int c = 0; c < 4; ++c)
      *reinterpret_cast<float2*>(region + (vg * G + g) * D + vc * 8 + 2 * c) =
          make_float2(acc[g][c].x * scl[g], acc[g][c].y * scl[g]);
  __syncthreads();
  const size_t part0 = (static_cast<size_t>(b) * a.Hq + hk * G) * a.splits + split;  // head g adds g * splits
  for (int e = tid; e < G * D; e += kDecThreads) {
    const int g = e / D, j = e % D;
    float s = 0.f;
#pragma unroll 4
    for (int r = 0; r < NG; ++r) s += region[(r * G + g) * D + j];
    a.ws_o[(part0 + static_cast<size_t>(g) * a.splits) * D + j] = s;
  }
  if (tid < G) {
    float s = 0.f;
#pragma unroll
    for (int w2 = 0; w2 < kDecWarps; ++w2) s += red[w2 * G + tid];
    float mv = Mblk[0];  // the block max (uniform); pick head tid without dynamic register indexing
#pragma unroll
    for (int g = 1; g < G; ++g)
      if (g == tid) mv = Mblk[g];
    a.ws_l[part0 + static_cast<size_t>(tid) * a.splits] = s;
    a.ws_m[part0 + static_cast<size_t>(tid) * a.splits] = mv;
  }
}

// Merge of the splits for one (batch, query head) per block, D threads.  With quantized values the merged vector
// is still in the rotated domain and is mapped back once: out = s .* H(o).
template <int D, bool VQ>
__global__ void __launch_bounds__(D) attend_reduce_kernel(const __grid_constant__ DecodeArgs a) {
  __shared__ float vec[D];
  const int bh = blockIdx.x, j = threadIdx.x;
  const float* m = a.ws_m + static_cast<size_t>(bh) * a.splits;
  const float* l = a.ws_l + static_cast<size_t>(bh) * a.splits;
  const float* o = a.ws_o + static_cast<size_t>(bh) * a.splits * D;
  float M = -INFINITY;
  for (int s = 0; s < a.splits; ++s) M = fmaxf(M, m[s]);
  float Ls = 0.f, acc = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < a.splits; ++s) {
      const float w = (m[s] == -INFINITY) ? 0.f : exp2f(m[s] - M);
      Ls = fmaf(w, l[s], Ls);
      acc = fmaf(w, o[static_cast<size_t>(s) * D + j], acc);
    }
  }
  const float r = Ls > 0.f ? acc / Ls : 0.f;
  if constexpr (!VQ) {
    a.out[static_cast<size_t>(bh) * D + j] = r;
  } else {
    constexpr int VPL = WarpVec<D>::VPL;
    vec[j] = r;
    __syncthreads();
    if (j < kWarp) {
      float v[VPL];
#pragma unroll
      for (int i = 0; i < VPL; ++i) v[i] = vec[j * VPL + i];
      fwht_warp<D>(v, j);
      const float nrm = rsqrtf(static_cast<float>(D));
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        const int jj = j * VPL + i;
        a.out[static_cast<size_t>(bh) * D + jj] = v[i] * nrm * sign_of(a.signs[jj]);
      }
    }
  }
}

// ---- scores only ---------------------------------------------------------------------------------------------------

// Shared-memory plan of the scorer: the factored form stages key codes (cp.async, double-buffered) and holds the
// pair table; the table form holds the materialised G-wide table and reads rows straight from global memory.
template <int D, int BITS, int G, int MODE>
struct ScorePlan {
  static constexpr int L = 1 << BITS;
  static constexpr int R = D * BITS / 8;
  static constexpr int KCH = (R % 16 == 0) ? 16 : 8;
  static constexpr int STAGE = kTT * R;
  static constexpr int LPT = 8, J = D / LPT;
  static constexpr int HG = G < 4 ? G : 4, PASSES = G / HG;
  static constexpr size_t OFF_STAGE = 0;
  static constexpr size_t OFF_TAB = MODE == kGatherFactored ? (size_t)kStages * STAGE : 0;
  static constexpr int TAB = MODE == kGatherFactored ? PairTable<BITS>::FLOATS : D * L * G;
  static constexpr size_t OFF_QS = OFF_TAB + (size_t)TAB * 4;
  static constexpr size_t OFF_CENT = OFF_QS + (size_t)G * D * 4;
  static constexpr size_t bytes = OFF_CENT + 16 * 4;
};

template <int R>
__device__ __forceinline__ void load_row(const uint8_t* __restrict__ p, uint32_t (&w)[R / 4 + 1]) {
  if constexpr (R % 16 == 0) {
#pragma unroll
    for (int i = 0; i < R / 16; ++i) {
      uint4 u = __ldg(reinterpret_cast<const uint4*>(p) + i);
      w[4 * i] = u.x; w[4 * i + 1] = u.y; w[4 * i + 2] = u.z; w[4 * i + 3] = u.w;
    }
  } else {
    static_assert(R % 8 == 0, "rows are a multiple of 8 bytes for d >= 64");
#pragma unroll
    for (int i = 0; i < R / 8; ++i) {
      uint2 u = __ldg(reinterpret_cast<const uint2*>(p) + i);
      w[2 * i] = u.x; w[2 * i + 1] = u.y;
    }
  }
  w[R / 4] = 0u;
}

// Gather-sum over the D coordinates of one token row from the materialised table: acc[g] = sum_j lut[j][idx_j][g].
template <int D, int BITS, int G>
__device__ __forceinline__ void table_gather(const uint32_t* w, const float* __restrict__ lut, float (&acc)[G]) {
  constexpr int L = 1 << BITS;
  if constexpr (G == 1) {
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int j = 0; j < D; j += 2) {
      a0 += lut[j * L + bits_at<BITS>(w, j * BITS)];
      a1 += lut[(j + 1) * L + bits_at<BITS>(w, (j + 1) * BITS)];
    }
    acc[0] = a0 + a1;
  } else if constexpr (G == 2) {
    float2 s = make_float2(0.f, 0.f);
#pragma unroll
    for (int j = 0; j < D; ++j) s = add2(s, reinterpret_cast<const float2*>(lut)[j * L + bits_at<BITS>(w, j * BITS)]);
    acc[0] = s.x; acc[1] = s.y;
  } else {
    float2 s[G / 2];
#pragma unroll
    for (int i = 0; i < G / 2; ++i) s[i] = make_float2(0.f, 0.f);
#pragma unroll
    for (int j = 0; j < D; ++j) {
      const float4* e = reinterpret_cast<const float4*>(lut + (j * L + bits_at<BITS>(w, j * BITS)) * G);
#pragma unroll
      for (int i = 0; i < G / 4; ++i) {
        const float4 x = e[i];
        s[2 * i] = add2(s[2 * i], make_float2(x.x, x.y));
        s[2 * i + 1] = add2(s[2 * i + 1], make_float2(x.z, x.w));
      }
    }
#pragma unroll
    for (int i = 0; i < G / 2; ++i) { acc[2 * i] = s[i].x; acc[2 * i + 1] = s[i].y; }
  }
}

template <int D, int BITS, int G, int MODE>
__global__ void __launch_bounds__(kDecThreads) score_kernel(const __grid_constant__ DecodeArgs a) {
  using P = ScorePlan<D, BITS, G, MODE>;
  constexpr int L = 1 << BITS, R = P::R, J = P::J, HG = P::HG;
  extern __shared__ __align__(16) uint8_t smem[];
  float* tab = reinterpret_cast<float*>(smem + P::OFF_TAB);
  float* qs = reinterpret_cast<float*>(smem + P::OFF_QS);
  float* cent = reinterpret_cast<float*>(smem + P::OFF_CENT);
  const int tid = threadIdx.x, lane = tid & 31;
  const int b = blockIdx.z, hk = blockIdx.y;
  const int len = row_len(a, b);
  const int start = blockIdx.x * a.chunk;
  const int end = min(start + a.chunk, a.T);
  const int vend = min(end, len);  // tokens with codes
  const size_t kv_row0 = (static_cast<size_t>(b) * a.Hkv + hk) * a.Tcap;
  float* out = a.scores + (static_cast<size_t>(b) * a.Hq + hk * G) * a.T;
  // tokens in [max(len, start), end) are masked
  for (int t = max(start, len) + tid; t < end; t += kDecThreads)
#pragma unroll
    for (int g = 0; g < G; ++g) out[static_cast<size_t>(g) * a.T + t] = -INFINITY;
  const int ntiles = vend > start ? (vend - start + kTT - 1) / kTT : 0;

  auto issue_tile = [&](int tile) {
    if constexpr (MODE == kGatherFactored) {
      if (tile < ntiles) {
        uint8_t* st = smem + P::OFF_STAGE + static_cast<size_t>(tile % kStages) * P::STAGE;
        const int t0 = start + tile * kTT;
        block_copy_async<P::KCH>(st, a.kcodes + (kv_row0 + t0) * R, min(kTT, vend - t0) * R);
      }
      cp_async_commit();
    }
  };
  for (int s = 0; s < kStages - 1; ++s) issue_tile(s);
  if (tid < 16) cent[tid] = a.cb.c[tid];
  transform_queries<D, G>(a.q + (static_cast<size_t>(b) * a.Hq + hk * G) * D, a.signs, a.mult, qs);
  __syncthreads();

  if constexpr (MODE == kGatherTable) {
    for (int e = tid; e < D * L * G; e += kDecThreads) {
      const int g = e % G, k = (e / G) % L, j = e / (G * L);
      tab[e] = qs[g * D + j] * cent[k];
    }
    __syncthreads();
    for (int t = start + tid; t < vend; t += kDecThreads) {
      uint32_t w[R / 4 + 1];
      load_row<R>(a.kcodes + (kv_row0 + t) * R, w);
      float s[G];
      table_gather<D, BITS, G>(w, tab, s);
      const float n = __half2float(a.knorms[kv_row0 + t]);
#pragma unroll
      for (int g = 0; g < G; ++g) out[static_cast<size_t>(g) * a.T + t] = s[g] * n;
    }
  } else {
    build_pair_table<BITS>(cent, tab);
    const int sl = tid & 7, grp = tid >> 3, kord = sl >> 1;
    const uint32_t rep_off = static_cast<uint32_t>(lane) << 3;
    float2 qp[HG][J / 2];
    if constexpr (P::PASSES == 1) {
#pragma unroll
      for (int h = 0; h < HG; ++h)
#pragma unroll
        for (int i = 0; i < J / 2; ++i) qp[h][i] = make_float2(qs[h * D + J * sl + 2 * i], qs[h * D + J * sl + 2 * i + 1]);
    }
    constexpr int ROUNDS = kTT / 128;
    float kn_next[ROUNDS];
#pragma unroll
    for (int r = 0; r < ROUNDS; ++r) {
      const int t = start + r * 128 + grp * 4 + kord;
      kn_next[r] = (ntiles > 0 && t < vend) ? __half2float(a.knorms[kv_row0 + t]) : 0.f;
    }
    for (int tile = 0; tile < ntiles; ++tile) {
      const int t0 = start + tile * kTT;
      const int nt = min(kTT, vend - t0);
      cp_async_wait<kStages - 2>();
      __syncthreads();  // tile complete; previous tile's stage free
      issue_tile(tile + kStages - 1);
      float kn_cur[ROUNDS];
#pragma unroll
      for (int r = 0; r < ROUNDS; ++r) {
        kn_cur[r] = kn_next[r];
        const int t = t0 + kTT + r * 128 + grp * 4 + kord;  // my token of the next tile
        if (tile + 1 < ntiles && t < vend) kn_next[r] = __half2float(a.knorms[kv_row0 + t]);
      }
      const uint8_t* st = smem + P::OFF_STAGE + static_cast<size_t>(tile % kStages) * P::STAGE;
#pragma unroll
      for (int round = 0; round < ROUNDS; ++round) {
        const int tbase = round * 128 + grp * 4;
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
            const uint64_t bits = load_slice<D, BITS, J>(st + (tbase + (k ^ kord)) * R, sl);
            factored_slice<BITS, J, HG>(bits, reinterpret_cast<const uint8_t*>(tab), rep_off, qp, v[k]);
          }
#pragma unroll
          for (int h = 0; h < HG; ++h) {
            v[0][h] += __shfl_xor_sync(0xffffffffu, v[2][h], 4);
            v[1][h] += __shfl_xor_sync(0xffffffffu, v[3][h], 4);
            v[0][h] += __shfl_xor_sync(0xffffffffu, v[1][h], 2);
            v[0][h] += __shfl_xor_sync(0xffffffffu, v[0][h], 1);
          }
          const int tt = tbase + kord;
          if (tt < nt) {
            const float n = kn_cur[round];
            // lanes 2m and 2m+1 hold the same sums; each writes half of the heads
#pragma unroll
            for (int h = 0; h < HG; ++h)
              if ((h & 1) == (sl & 1))
                out[static_cast<size_t>(pass * HG + h) * a.T + t0 + tt] = v[0][h] * n;
          }
        }
      }
    }
    cp_async_wait<0>();
  }
}

}  // namespace axr
