// Decode attention on the tensor cores (d = 128, values quantized and stored in 128-token tiles).
//
// Scores (AXELRAM Key Points, 1st and 2nd items): the query is transformed once and each token's score is the
// gather-sum of q~_j * c_k at its stored indices times its stored norm.  Here the table is read in factored form on
// the tensor cores, as in the scorer: the gathered centroids of 128 tokens (hi and lo fp16 planes, about 22 bits)
// form the A operand in TMEM, the query's hi/lo planes form B, and S = A B (M = 128 tokens, N = 16, K = 2 d) gives
// the tile's scores in fp32.  The softmax and the value product are the standard split-T formulation; with
// quantized values the product stays in the rotated domain (one inverse transform per output, in the merge):
//   O^T[j][n] = sum_t  c[idx^V_{t,j}] * P'[n][t],   P'[G q + g][t] = p_{g,t} n^V_t for the tokens of stream q,
// an M = 128 (coordinates) x N (4 softmax streams x G heads) x K = 128 (tokens) MMA per tile, whose A operand --
// coordinate j in TMEM lane j, token pairs in the columns -- comes from a byte-indexed table of fp16 centroid pairs
// (one byte of a coordinate's tiled row holds two tokens at b = 4).
//
// Roles (416 threads, one CTA per SM, persistent over (batch, KV head, split) items):
//   key warps 0..3      -- lane = token (TMEM lane): gather the tile's hi/lo centroid pairs into the key A buffer,
//                          and stage key codes (cp.async, completion on the stage's mbarrier);
//   softmax warps 4..7  -- lane = token: read the tile's scores, run the online softmax of their 32 tokens (four
//                          independent streams, no barrier between them), write the fp16 weights into rows
//                          [G q, G q + G) of the block-diagonal B operand of the value MMA and a record (alpha,
//                          m, l) per head; warp 4 also builds the query operand of the next row;
//   value warps 8..11   -- lane = coordinate: gather the value A operand, fold the value MMA result of the tile two
//                          back into registers (o_q = o_q * alpha_q + O[:, G q + g]), stage value codes, and merge
//                          the four streams into the item's partial output;
//   MMA warp 12         -- issues the key MMAs of tile i, then the value MMAs of tile i - 1.
// Tile-indexed mbarriers carry every hand-off (phases follow a per-CTA tile counter); there is no named barrier.
// Every wait is bounded; a failed wait makes the CTA write NaN partials.
#pragma once

#include "score_tc.cuh"

namespace axr {

template <int BITS, int G>
struct TcaPlan {
  static constexpr int D = 128, TT = 128;
  static constexpr int KGW = 4;                 // key gather warps (one per TMEM quarter)
  static constexpr int SW0 = 4, VW0 = 8;        // softmax and value warps (multiples of 4: warp % 4 = TMEM quarter)
  static constexpr int MW = 12;                 // MMA issuer; 13 warps keep 128 registers per thread
  static constexpr int THREADS = 32 * (MW + 1);
  static constexpr int KGT = 32 * KGW;
  static constexpr int L = 1 << BITS;
  static constexpr int R = D * BITS / 8;        // key bytes per token = value bytes per coordinate per tile
  static constexpr int PAIRS = D / 2;
  static constexpr int NSK = G == 8 ? 3 : 4;    // key code stages (lookahead NSK - 2 tiles)
  static constexpr int NSV = G == 8 ? 3 : 4;    // value code stages (lookahead NSV - 2 tiles)
  static constexpr int STAGE = TT * R;
  static constexpr int E = L * L;
  static constexpr int NP = 4 * G < 16 ? 16 : 4 * G;  // value MMA N: stream q's heads in columns [G q, G q + G)
  static constexpr int BQ_BYTES = tc::Layout<D>::B_BYTES;
  static constexpr int BP_BYTES = NP * TT * 2;
  static constexpr uint32_t BP_SBO = TT / 8 * 128;
  static constexpr int RING = 4;                // softmax records (alpha, m, l) per tile, stream and head
  // TMEM columns
  static constexpr int KA0 = 0, KASTRIDE = D;                    // key A: 2 x 128
  static constexpr int VA0 = 2 * D, VASTRIDE = TT / 2;           // value A: 2 x 64
  static constexpr int DS0 = VA0 + 2 * VASTRIDE, DSSTRIDE = 16;  // scores: 2 x 16
  static constexpr int DO0 = DS0 + 2 * DSSTRIDE, DOSTRIDE = NP;  // value product: 2 x NP
  static constexpr int TMEM_COLS = 512;
  static_assert(DO0 + 2 * DOSTRIDE <= TMEM_COLS, "TMEM budget");
  // shared memory
  static constexpr size_t OFF_KTAB = 0;                                   // hi/lo fp16 pairs, 32 copies, 256 B / entry
  static constexpr size_t OFF_VTAB = OFF_KTAB + (size_t)E * 256;          // hi fp16 pairs, 32 copies, 256 B / entry
  static constexpr size_t OFF_KST = OFF_VTAB + (size_t)E * 256;
  static constexpr size_t OFF_VST = OFF_KST + (size_t)NSK * STAGE;
  static constexpr size_t OFF_BQ = OFF_VST + (size_t)NSV * STAGE;        // [2][BQ_BYTES]
  static constexpr size_t OFF_BP = OFF_BQ + 2 * (size_t)BQ_BYTES;         // [2][BP_BYTES]
  static constexpr size_t OFF_REC = OFF_BP + 2 * (size_t)BP_BYTES;        // [RING][4][G][3]
  static constexpr size_t OFF_CENT = OFF_REC + (size_t)RING * 4 * G * 3 * 4;  // gamma[16], c[16]
  static constexpr size_t OFF_MBAR = (OFF_CENT + 32 * 4 + 7) / 8 * 8;
  static constexpr int NMBAR = NSK + NSV + 7 * 2 + RING;
  static constexpr size_t OFF_MISC = OFF_MBAR + (size_t)NMBAR * 8;
  static constexpr size_t bytes = OFF_MISC + 16;
  static_assert(bytes <= 227 * 1024, "shared memory");
};

// Item geometry: (batch, KV head, split) -> token range and tile count.
struct ItemGeo {
  int b, hk, split, start, end, ntiles;
};

__device__ __forceinline__ ItemGeo item_geo(const DecodeArgs& a, int item) {
  ItemGeo g;
  g.split = item % a.splits;
  g.hk = (item / a.splits) % a.Hkv;
  g.b = item / (a.splits * a.Hkv);
  g.start = g.split * a.chunk;
  g.end = min(g.start + a.chunk, row_len(a, g.b));
  g.ntiles = g.end > g.start ? (g.end - g.start + kTile - 1) / kTile : 0;
  return g;
}

// Walks the tiles of this CTA's items (blockIdx.x, + gridDim.x, ...) in order, skipping empty items.
struct TileStream {
  int item, ti;
  ItemGeo g;
  __device__ __forceinline__ void init(const DecodeArgs& a, int items) {
    item = blockIdx.x;
    ti = 0;
    if (item < items) g = item_geo(a, item);
    settle(a, items);
  }
  __device__ __forceinline__ void settle(const DecodeArgs& a, int items) {
    while (item < items && ti >= g.ntiles) {
      item += gridDim.x;
      ti = 0;
      if (item < items) g = item_geo(a, item);
    }
  }
  __device__ __forceinline__ void next(const DecodeArgs& a, int items) {
    ++ti;
    settle(a, items);
  }
};

template <int BITS, int G>
__global__ void __launch_bounds__(TcaPlan<BITS, G>::THREADS, 1)
attend_tcv_kernel(const __grid_constant__ DecodeArgs a) {
  using P = TcaPlan<BITS, G>;
  constexpr int D = P::D, TT = P::TT, R = P::R, NSK = P::NSK, NSV = P::NSV, RING = P::RING;
  extern __shared__ __align__(16) uint8_t smem[];
  const uint8_t* ktab = smem + P::OFF_KTAB;
  const uint8_t* vtab = smem + P::OFF_VTAB;
  uint8_t* kst = smem + P::OFF_KST;
  uint8_t* vst = smem + P::OFF_VST;
  uint8_t* bp = smem + P::OFF_BP;
  float* rec = reinterpret_cast<float*>(smem + P::OFF_REC);  // [RING][stream][G][alpha, m, l]
  float* gam = reinterpret_cast<float*>(smem + P::OFF_CENT);
  float* cen = gam + 16;
  uint64_t* mb = reinterpret_cast<uint64_t*>(smem + P::OFF_MBAR);
  uint64_t* kfull = mb;                 // key stage landed             (count KGT, cp.async arrivals)
  uint64_t* vfull = kfull + NSK;        // value stage landed           (count 128, cp.async arrivals)
  uint64_t* ka_full = vfull + NSV;      // key A gathered               (count 4 warps)
  uint64_t* s_done = ka_full + 2;       // key MMAs done                (commit)
  uint64_t* s_free = s_done + 2;        // scores read                  (count 4 warps)
  uint64_t* p_full = s_free + 2;        // weights written              (count 4 warps)
  uint64_t* av_full = p_full + 2;       // value A gathered             (count 4 warps)
  uint64_t* o_done = av_full + 2;       // value MMAs done              (commit)
  uint64_t* b_full = o_done + 2;        // query operand of a row built (count 1)
  uint64_t* rec_full = b_full + 2;      // softmax records written      (count 4 warps)
  uint32_t* tmem_s = reinterpret_cast<uint32_t*>(smem + P::OFF_MISC);
  volatile int* failed = reinterpret_cast<volatile int*>(smem + P::OFF_MISC + 4);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int items = a.B * a.Hkv * a.splits;

  // ---- setup: tables, zero value B operand, barriers, TMEM ----
  if (tid < 16) {
    gam[tid] = a.cb.gamma[tid];
    cen[tid] = a.cb.c[tid];
  }
  if (warp == P::MW) tc::tmem_alloc(tmem_s, P::TMEM_COLS);
  if (tid == 0) {
    for (int i = 0; i < NSK; ++i) tc::mbar_init(kfull + i, P::KGT);
    for (int i = 0; i < NSV; ++i) tc::mbar_init(vfull + i, 128);
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(ka_full + i, P::KGW);
      tc::mbar_init(s_done + i, 1);
      tc::mbar_init(s_free + i, 4);
      tc::mbar_init(p_full + i, 4);
      tc::mbar_init(av_full + i, 4);
      tc::mbar_init(o_done + i, 1);
      tc::mbar_init(b_full + i, 1);
    }
    for (int i = 0; i < RING; ++i) tc::mbar_init(rec_full + i, 4);
    *failed = 0;
  }
  for (int i = tid; i < 2 * P::BP_BYTES / 4; i += P::THREADS) reinterpret_cast<uint32_t*>(bp)[i] = 0u;
  for (int i = tid; i < 2 * P::BQ_BYTES / 4; i += P::THREADS)  // entries the row builder never writes stay 0
    reinterpret_cast<uint32_t*>(smem + P::OFF_BQ)[i] = 0u;
  __syncthreads();
  tc::build_table<BITS>(gam, reinterpret_cast<uint2*>(smem + P::OFF_KTAB));
  for (int i = tid; i < P::E * 32; i += P::THREADS) {
    const int e = i >> 5, l = i & 31;
    const __half2 h = __halves2half2(__float2half_rn(cen[e & (P::L - 1)]), __float2half_rn(cen[e >> BITS]));
    *reinterpret_cast<__half2*>(smem + P::OFF_VTAB + e * 256 + l * 4) = h;
  }
  tc::fence_async_smem();  // the zeroed value B operand is read by the tensor cores
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *tmem_s;

  if (warp < P::KGW) {
    // ==================================== key gather ====================================
    const int tt = warp * 32 + lane;  // token = TMEM lane
    const uint32_t repw = static_cast<uint32_t>(lane) << 3;
    const uint32_t tl = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    TileStream ahead;
    ahead.init(a, items);
    int ia = 0;
    auto issue = [&]() {
      if (ahead.item >= items) return;
      const ItemGeo& g = ahead.g;
      const int t0 = g.start + ahead.ti * TT;
      const int bytes = min(TT, g.end - t0) * R;
      const uint8_t* src = a.kcodes + ((static_cast<size_t>(g.b) * a.Hkv + g.hk) * a.Tcap + t0) * R;
      uint8_t* dst = kst + static_cast<size_t>(ia % NSK) * P::STAGE;
      for (int o = tid * 16; o < bytes; o += P::KGT * 16) cp_async<16>(dst + stage_swizzle<R>(o), src + o);
      tc::cp_async_mbar_arrive(kfull + ia % NSK);
      ++ia;
      ahead.next(a, items);
    };
    for (int s = 0; s < NSK - 2; ++s) issue();
    int it = 0;
    bool bad = false;
    for (int item = blockIdx.x; item < items && !bad; item += gridDim.x) {
      const ItemGeo g = item_geo(a, item);
      for (int ti = 0; ti < g.ntiles; ++ti, ++it) {
        if (it >= 2 && !warp_wait(s_done + (it & 1), ((it - 2) >> 1) & 1)) { bad = true; break; }
        if (warp_failed(failed)) { bad = true; break; }
        issue();  // into the stage of tile it - 2: its key MMAs have run, so every key warp has read it
        if (!warp_wait(kfull + it % NSK, (it / NSK) & 1)) { bad = true; break; }
        tc::fence_after();
        const int nt = min(TT, g.end - (g.start + ti * TT));
        uint32_t w[R / 4 + 1];
        load_swizzled_row<R>(kst + static_cast<size_t>(it % NSK) * P::STAGE, tt, w);
        w[R / 4] = 0u;
        if (tt >= nt) {
#pragma unroll
          for (int c = 0; c < R / 4; ++c) w[c] = 0u;
        }
        const uint32_t acol = tl + static_cast<uint32_t>(P::KA0 + (it & 1) * P::KASTRIDE);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t hi[32], lo[32];
#pragma unroll
          for (int p = 0; p < 32; ++p) {
            const uint2 e = *reinterpret_cast<const uint2*>(ktab + tc::pair_off<BITS>(w, half * 32 + p, repw));
            hi[p] = e.x;
            lo[p] = e.y;
          }
          tc::st_x32(acol + half * 32, hi);
          tc::st_x32(acol + P::PAIRS + half * 32, lo);
        }
        tc::wait_st();
        tc::fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(ka_full + (it & 1));
      }
    }
    if (bad) *failed = 1;
    cp_async_wait<0>();
  } else if (warp < P::VW0) {
    // ===================================== softmax =====================================
    const int q = warp & 3, tt = q * 32 + lane;  // stream q = this warp's 32 tokens of every tile
    const uint32_t tl = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const float rd = rsqrtf(static_cast<float>(D));
    const bool builder = warp == P::SW0;
    auto build_row_b = [&](const ItemGeo& g, int slot) {  // query operand of row (b, hk), one warp
      tc::build_b_warp<D, G>(a.q + (static_cast<size_t>(g.b) * a.Hq + g.hk * G) * D, a.signs, a.mult,
                             reinterpret_cast<__half*>(smem + P::OFF_BQ + slot * P::BQ_BYTES));
      tc::fence_async_smem();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(b_full + slot);
    };
    auto next_with_tiles = [&](int item) {  // the next item of this CTA that has tiles (or >= items)
      for (item += gridDim.x; item < items; item += gridDim.x)
        if (item_geo(a, item).ntiles > 0) break;
      return item;
    };
    int it = 0, kq = 0;  // tiles and rows-with-tiles so far
    bool bad = false;
    {
      const int first = (blockIdx.x < items && item_geo(a, blockIdx.x).ntiles > 0) ? static_cast<int>(blockIdx.x)
                                                                                   : next_with_tiles(blockIdx.x);
      if (builder && first < items) build_row_b(item_geo(a, first), 0);
    }
    for (int item = blockIdx.x; item < items && !bad; item += gridDim.x) {
      const ItemGeo g = item_geo(a, item);
      const size_t part0 = (static_cast<size_t>(g.b) * a.Hq + g.hk * G) * a.splits + g.split;
      if (g.ntiles == 0) {  // an empty partial (the value warps write o = 0)
        if (builder && lane < G) {
          a.ws_l[part0 + static_cast<size_t>(lane) * a.splits] = 0.f;
          a.ws_m[part0 + static_cast<size_t>(lane) * a.splits] = -INFINITY;
        }
        continue;
      }
      const size_t row0 = (static_cast<size_t>(g.b) * a.Hkv + g.hk) * a.Tcap;
      const float* qg = a.q + (static_cast<size_t>(g.b) * a.Hq + g.hk * G) * D;
      float inv[G], m_run[G], l_run[G];
#pragma unroll
      for (int gg = 0; gg < G; ++gg) {
        inv[gg] = 1.f / tc::head_scale<D>(qg + gg * D, a.mult);  // the builder's scale, recomputed identically
        m_run[gg] = -INFINITY;
        l_run[gg] = 0.f;
      }
      float kn_next = 0.f, vn_next = 0.f;
      if (g.start + tt < g.end) {
        kn_next = __half2float(a.knorms[row0 + g.start + tt]);
        vn_next = __half2float(a.vnorms[row0 + g.start + tt]);
      }
      for (int ti = 0; ti < g.ntiles; ++ti, ++it) {
        const int t0 = g.start + ti * TT;
        const float kn = kn_next, vn = vn_next;
        if (ti + 1 < g.ntiles && t0 + TT + tt < g.end) {
          kn_next = __half2float(a.knorms[row0 + t0 + TT + tt]);
          vn_next = __half2float(a.vnorms[row0 + t0 + TT + tt]);
        }
        if (!warp_wait(s_done + (it & 1), (it >> 1) & 1)) { bad = true; break; }
        tc::fence_after();
        uint32_t d[16];
        tc::ld_x16(tl + static_cast<uint32_t>(P::DS0 + (it & 1) * P::DSSTRIDE), d);
        tc::wait_ld();
        tc::fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(s_free + (it & 1));
        // on the first tile of a row, the next row's query operand (its slot was last read by key MMAs that
        // have completed: s_done of this tile covers every earlier MMA)
        if (builder && ti == 0) {
          const int nxt = next_with_tiles(item);
          if (nxt < items) build_row_b(item_geo(a, nxt), (kq + 1) & 1);
        }
        const bool valid = t0 + tt < g.end;
        float alpha[G], pw[G];
#pragma unroll
        for (int gg = 0; gg < G; ++gg) {
          const float z = valid ? (__uint_as_float(d[2 * gg]) + __uint_as_float(d[2 * gg + 1])) * inv[gg] * kn * rd
                                : -INFINITY;
          const float mx = warp_max(z);
          const float m_new = fmaxf(m_run[gg], mx);
          alpha[gg] = (m_new == -INFINITY) ? 1.f : exp2f(m_run[gg] - m_new);
          const float p = (z == -INFINITY) ? 0.f : exp2f(z - m_new);
          l_run[gg] = l_run[gg] * alpha[gg] + p;
          m_run[gg] = m_new;
          pw[gg] = p * vn;
        }
        // value B buffer it % 2 and record slot it % RING are free once the value MMAs of tile it - 2 have run
        if (it >= 2 && !warp_wait(o_done + (it & 1), ((it - 2) >> 1) & 1)) { bad = true; break; }
        __half* pb = reinterpret_cast<__half*>(bp + (it & 1) * P::BP_BYTES);
#pragma unroll
        for (int gg = 0; gg < G; ++gg) {
          const int n = q * G + gg;
          pb[(n >> 3) * (P::BP_SBO / 2) + (tt >> 3) * 64 + (n & 7) * 8 + (tt & 7)] = __float2half_rn(pw[gg]);
        }
        const bool last = ti + 1 == g.ntiles;
        float lsum[G];
#pragma unroll
        for (int gg = 0; gg < G; ++gg) lsum[gg] = last ? warp_sum(l_run[gg]) : 0.f;
        if (lane == 0) {
          float* r = rec + ((it % RING) * 4 + q) * G * 3;
#pragma unroll
          for (int gg = 0; gg < G; ++gg) {
            r[3 * gg] = alpha[gg];
            r[3 * gg + 1] = m_run[gg];
            r[3 * gg + 2] = lsum[gg];
          }
        }
        tc::fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          tc::mbar_arrive(p_full + (it & 1));
          tc::mbar_arrive(rec_full + (it % RING));
        }
      }
      ++kq;
    }
    if (bad) *failed = 1;
  } else if (warp < P::MW) {
    // ====================================== values ======================================
    const int q4 = warp & 3, j = q4 * 32 + lane;  // coordinate = TMEM lane
    const uint32_t tl = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const uint32_t rep_v = static_cast<uint32_t>(lane) << 2;
    const int vtid = tid - P::VW0 * 32;
    const size_t tiles_cap = static_cast<size_t>(a.Tcap / TT);
    TileStream ahead;
    ahead.init(a, items);
    int ia = 0;
    auto issue_v = [&]() {
      if (ahead.item >= items) return;
      const ItemGeo& g = ahead.g;
      const size_t tile = static_cast<size_t>(g.start / TT + ahead.ti);
      const uint8_t* src = static_cast<const uint8_t*>(a.v) +
                           ((static_cast<size_t>(g.b) * a.Hkv + g.hk) * tiles_cap + tile) * P::STAGE;
      uint8_t* dst = vst + static_cast<size_t>(ia % NSV) * P::STAGE;
      for (int o = vtid * 16; o < P::STAGE; o += 128 * 16) cp_async<16>(dst + stage_swizzle<R>(o), src + o);
      tc::cp_async_mbar_arrive(vfull + ia % NSV);
      ++ia;
      ahead.next(a, items);
    };
    for (int s = 0; s < NSV - 2; ++s) issue_v();
    int it = 0;
    bool bad = false;
    float o[4][G];  // one accumulator per softmax stream and head
    auto fold = [&](int t) {  // o_q = o_q * alpha_q(t) + O(t)[:, G q + g]
      if (!warp_wait(o_done + (t & 1), (t >> 1) & 1) || !warp_wait(rec_full + (t % RING), (t / RING) & 1)) {
        bad = true;
        return;
      }
      tc::fence_after();
      const float* r = rec + (t % RING) * 4 * G * 3;
#pragma unroll
      for (int c0 = 0; c0 < 4 * G; c0 += 16) {
        uint32_t d[16];
        tc::ld_x16(tl + static_cast<uint32_t>(P::DO0 + (t & 1) * P::DOSTRIDE + c0), d);
        tc::wait_ld();
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          if (c0 + c < 4 * G) {
            const int s = (c0 + c) / G, gg = (c0 + c) % G;
            o[s][gg] = fmaf(o[s][gg], r[(s * G + gg) * 3], __uint_as_float(d[c]));
          }
        }
      }
    };
    for (int item = blockIdx.x; item < items; item += gridDim.x) {
      const ItemGeo g = item_geo(a, item);
      const size_t part0 = (static_cast<size_t>(g.b) * a.Hq + g.hk * G) * a.splits + g.split;
#pragma unroll
      for (int s = 0; s < 4; ++s)
#pragma unroll
        for (int gg = 0; gg < G; ++gg) o[s][gg] = 0.f;
      if (!bad) {
        for (int ti = 0; ti < g.ntiles; ++ti, ++it) {
          // value A buffer it % 2 and the stage of tile it - 2 are free once the value MMAs of tile it - 2 have
          // run; that tile is folded here, two tiles behind, so no value MMA waits for a fold
          if (it >= 2 && !warp_wait(o_done + (it & 1), ((it - 2) >> 1) & 1)) { bad = true; break; }
          if (warp_failed(failed)) { bad = true; break; }
          if (ti >= 2) {
            fold(it - 2);
            if (bad) break;
          }
          issue_v();
          if (!warp_wait(vfull + it % NSV, (it / NSV) & 1)) { bad = true; break; }
          tc::fence_after();
          uint32_t w4[R / 4 + 1];
          load_swizzled_row<R>(vst + static_cast<size_t>(it % NSV) * P::STAGE, j, w4);
          w4[R / 4] = 0u;
          const uint32_t acol = tl + static_cast<uint32_t>(P::VA0 + (it & 1) * P::VASTRIDE);
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            uint32_t hv[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              const int cc = half * 32 + c;
              uint32_t off;
              if constexpr (BITS == 4) off = __byte_perm(w4[cc >> 2], rep_v, 0x5504u | (static_cast<uint32_t>(cc & 3) << 4));
              else off = (bits_at<2 * BITS>(w4, 2 * BITS * cc) << 8) | rep_v;
              hv[c] = *reinterpret_cast<const uint32_t*>(vtab + off);
            }
            tc::st_x32(acol + half * 32, hv);
          }
          tc::wait_st();
          tc::fence_before();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(av_full + (it & 1));
        }
        if (!bad && g.ntiles >= 2) fold(it - 2);
        if (!bad && g.ntiles >= 1) fold(it - 1);
        tc::fence_before();
      }
      // merge the streams with the records of the item's last tile
      const float* r = rec + ((it - 1 + RING) % RING) * 4 * G * 3;
#pragma unroll
      for (int gg = 0; gg < G; ++gg) {
        float M = -INFINITY;
        if (g.ntiles > 0 && !bad) {
#pragma unroll
          for (int s = 0; s < 4; ++s) M = fmaxf(M, r[(s * G + gg) * 3 + 1]);
        }
        float ov = 0.f, lv = 0.f;
        if (M != -INFINITY) {
#pragma unroll
          for (int s = 0; s < 4; ++s) {
            const float ms = r[(s * G + gg) * 3 + 1];
            const float sc = ms == -INFINITY ? 0.f : exp2f(ms - M);
            ov = fmaf(o[s][gg], sc, ov);
            lv = fmaf(r[(s * G + gg) * 3 + 2], sc, lv);
          }
        }
        if (g.ntiles > 0) {
          a.ws_o[(part0 + static_cast<size_t>(gg) * a.splits) * D + j] = bad ? __int_as_float(0x7fc00000) : ov;
          if (j == 0) {
            a.ws_l[part0 + static_cast<size_t>(gg) * a.splits] = lv;
            a.ws_m[part0 + static_cast<size_t>(gg) * a.splits] = bad ? __int_as_float(0x7fc00000) : M;
          }
        } else {
          a.ws_o[(part0 + static_cast<size_t>(gg) * a.splits) * D + j] = 0.f;
        }
      }
    }
    if (bad) *failed = 1;
    cp_async_wait<0>();
  } else if (lane == 0) {
    // ======================================== MMA ========================================
    const uint32_t bq0 = smem_u32(smem + P::OFF_BQ), bp0 = smem_u32(bp);
    const uint32_t idesc_p = (1u << 4) | (static_cast<uint32_t>(P::NP >> 3) << 17) | (static_cast<uint32_t>(128 >> 4) << 24);
    int it = 0, kq = 0, last_v = -1;
    bool bad = false;
    auto value_mma = [&](int t) {
      if (!tc::mbar_wait(p_full + (t & 1), (t >> 1) & 1) || !tc::mbar_wait(av_full + (t & 1), (t >> 1) & 1)) {
        bad = true;
        return;
      }
      tc::fence_after();
      const uint32_t a_t = tmem + static_cast<uint32_t>(P::VA0 + (t & 1) * P::VASTRIDE);
      const uint32_t d_t = tmem + static_cast<uint32_t>(P::DO0 + (t & 1) * P::DOSTRIDE);
#pragma unroll
      for (int s = 0; s < TT / 16; ++s) {
        const uint64_t desc = tc::smem_desc(bp0 + static_cast<uint32_t>((t & 1) * P::BP_BYTES + s * 256), P::BP_SBO);
        const uint32_t acc = s > 0 ? 1u : 0u;
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_t),
            "r"(a_t + static_cast<uint32_t>(s * 8)), "l"(desc), "r"(idesc_p), "r"(acc)
            : "memory");
      }
      asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                       smem_u32(o_done + (t & 1)))
                   : "memory");
      last_v = t;
    };
    for (int item = blockIdx.x; item < items && !bad; item += gridDim.x) {
      const ItemGeo g = item_geo(a, item);
      if (g.ntiles == 0) continue;
      for (int ti = 0; ti < g.ntiles; ++ti, ++it) {
        if (*failed) { bad = true; break; }
        if (ti == 0 && !tc::mbar_wait(b_full + (kq & 1), (kq >> 1) & 1)) { bad = true; break; }
        if (it >= 2 && !tc::mbar_wait(s_free + (it & 1), ((it - 2) >> 1) & 1)) { bad = true; break; }
        if (!tc::mbar_wait(ka_full + (it & 1), (it >> 1) & 1)) { bad = true; break; }
        tc::fence_after();
        tc::issue_mma<D>(tmem + static_cast<uint32_t>(P::KA0 + (it & 1) * P::KASTRIDE),
                         tmem + static_cast<uint32_t>(P::DS0 + (it & 1) * P::DSSTRIDE),
                         bq0 + static_cast<uint32_t>((kq & 1) * P::BQ_BYTES), s_done + (it & 1));
        if (it >= 1) {
          value_mma(it - 1);
          if (bad) break;
        }
      }
      ++kq;
    }
    if (!bad && it >= 1) value_mma(it - 1);
    if (bad) *failed = 1;
    // nothing may be in flight when the columns are released
    if (last_v >= 0 && !tc::mbar_wait(o_done + (last_v & 1), (last_v >> 1) & 1)) *failed = 1;
    if (it >= 1 && !tc::mbar_wait(s_done + ((it - 1) & 1), ((it - 1) >> 1) & 1)) *failed = 1;
  }

  tc::fence_before();
  __syncthreads();
  report_wait_failure(a, failed);
  if (*failed) {  // make this CTA's partials NaN so that the merged output shows the failure
    for (int item = blockIdx.x; item < items; item += gridDim.x) {
      const ItemGeo g = item_geo(a, item);
      const size_t part0 = (static_cast<size_t>(g.b) * a.Hq + g.hk * G) * a.splits + g.split;
      if (tid < G) a.ws_m[part0 + static_cast<size_t>(tid) * a.splits] = __int_as_float(0x7fc00000);
    }
  }
  if (warp == P::MW) {
    tc::fence_after();
    tc::tmem_dealloc(tmem, P::TMEM_COLS);
  }
}

}  // namespace axr
