// Scores through warp-level MMAs (mma.sync.m16n8k16, fp16 operands, fp32 accumulation).
//
// AXELRAM Key Points (1st, 2nd items): every cached token's score is the gather-sum of the query's table entries at
// the token's stored indices, times its stored norm.  The table is read in factored form (mma_score.cuh): each
// token's centroids, split into hi and lo fp16 planes (about 22 bits), form two rows of A (one MMA covers 8
// tokens); the query's hi/lo planes form B, built once per (batch, KV head) and kept in registers; lane (g, t) ends
// with head t's score of tokens g and g + 8 of a 16-token group.  There is no shuffle reduction and no cross-warp
// hand-off inside a tile: warp w owns tokens [32 w, 32 w + 32) of each 256-token tile (two 16-token groups).  Code
// tiles arrive as one bulk copy each (completing on a per-stage mbarrier), norms as 16-byte cp.async chunks, four
// stages deep, issued by warp 0 alone, with one block barrier per tile.  Blocks are persistent (two per SM) over
// (batch, KV head, split) items and build the pair table once; the tile pipeline runs on from one item into the
// next (slots past an item's end carry the next item's first tiles), the next item's queries are fetched one item
// ahead, and the B fragments are built once per block.
#pragma once

#include "mma_score.cuh"

namespace axr {

template <int D, int BITS, int G>
struct ScoreMmaPlan {
  static constexpr int TT = 256;                  // tokens per tile
  static constexpr int WARPS = 8, THREADS = 32 * WARPS;
  static constexpr int WT = TT / WARPS;           // tokens per warp per tile (two M = 16 tiles)
  static constexpr int R = D * BITS / 8;
  static constexpr int NT = MmaB<D, G>::NT;
  static constexpr int STAGE = TT * R;
  static constexpr bool BULK = R % 16 == 0;       // codes as one bulk copy per tile, else 8-byte cp.async chunks
  static constexpr size_t QB = (size_t)G * D * 4;  // one item's queries
  static constexpr size_t BS = (size_t)NT * MmaB<D, G>::KT * 2 * 32 * 4;  // staged B fragments
  static constexpr size_t FIXED = (size_t)HiLoTable16<BITS>::BYTES + 3 * QB + BS + 16 * 4 + 16 * 4 + D + 8 * 8 + 8 + 512;
  static constexpr int NST = FIXED + 4 * (size_t)(STAGE + TT * 2) <= 113 * 1024 ? 4 : 3;  // stages
  static constexpr size_t OFF_STAGE = 0;
  static constexpr size_t OFF_NRM = (size_t)NST * STAGE;                    // [NST][TT] fp16 key norms
  static constexpr size_t OFF_TAB = (OFF_NRM + (size_t)NST * TT * 2 + 127) / 128 * 128;
  static constexpr size_t OFF_QS = OFF_TAB + (size_t)HiLoTable16<BITS>::BYTES;  // [G][D] row factors
  static constexpr size_t OFF_QB = OFF_QS + QB;                             // [2][G][D] raw queries
  static constexpr size_t OFF_BS = OFF_QB + 2 * QB;                         // [NT KT 2][32] B fragments
  static constexpr size_t OFF_SCL = OFF_BS + BS;                            // [G] head scales (16 slots)
  static constexpr size_t OFF_CENT = OFF_SCL + 16 * 4;
  static constexpr size_t OFF_SGN = OFF_CENT + 16 * 4;                      // [D] sign vector
  static constexpr size_t OFF_MB = (OFF_SGN + D + 15) / 16 * 16;            // [NST] stages, [2] queries, flag
  static constexpr size_t bytes = OFF_MB + (NST + 2) * 8 + 8;
  static_assert(bytes <= 113 * 1024, "two blocks per SM");
};

template <int D, int BITS, int G>
__global__ void __launch_bounds__(256, 2) score_mma_kernel(const __grid_constant__ DecodeArgs a) {
  using P = ScoreMmaPlan<D, BITS, G>;
  constexpr int NT = P::NT, TT = P::TT, WT = P::WT, NST = P::NST;
  extern __shared__ __align__(16) uint8_t smem[];
  const uint8_t* tab = smem + P::OFF_TAB;
  float* qs = reinterpret_cast<float*>(smem + P::OFF_QS);
  float* qbuf = reinterpret_cast<float*>(smem + P::OFF_QB);
  uint32_t* bs = reinterpret_cast<uint32_t*>(smem + P::OFF_BS);
  float* sclv = reinterpret_cast<float*>(smem + P::OFF_SCL);
  float* cent = reinterpret_cast<float*>(smem + P::OFF_CENT);
  int8_t* sgn = reinterpret_cast<int8_t*>(smem + P::OFF_SGN);
  __half* nst = reinterpret_cast<__half*>(smem + P::OFF_NRM);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + P::OFF_MB);  // stage s holds its code tile
  uint64_t* qfull = full + NST;                                     // [2]: item k's queries land in buffer k % 2
  volatile int* failed = reinterpret_cast<volatile int*>(qfull + 2);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, tq = lane & 3;
  const uint32_t rep16 = static_cast<uint32_t>(lane & 15) << 4;
  const float rd = rsqrtf(static_cast<float>(D));

  if (tid < 16) cent[tid] = a.cb.gamma[tid];
  for (int j = tid; j < D; j += P::THREADS) sgn[j] = a.signs[j];
  if (tid == 0) {
    for (int s = 0; s < NST + 2; ++s) tc::mbar_init(full + s, 1);
    *failed = 0;
  }
  __syncthreads();
  build_hilo_table16<BITS>(cent, smem + P::OFF_TAB);  // once per block

  const int items = a.B * a.Hkv * a.splits;
  struct Geo {  // one item: (batch row, KV head, split), its token range and the part of it holding codes
    int b, hk, start, end, vend, ntiles;
    size_t kv_row0;
    bool nrm_async;  // the norm row starts 16-byte aligned: norms ride with the codes
  };
  auto geo = [&](int item) {
    Geo x;
    const int split = item % a.splits;
    x.hk = (item / a.splits) % a.Hkv;
    x.b = item / (a.splits * a.Hkv);
    x.start = split * a.chunk;
    x.end = min(x.start + a.chunk, a.T);
    x.vend = min(x.end, row_len(a, x.b));
    x.ntiles = x.vend > x.start ? (x.vend - x.start + TT - 1) / TT : 0;
    x.kv_row0 = (static_cast<size_t>(x.b) * a.Hkv + x.hk) * a.Tcap;
    x.nrm_async = (reinterpret_cast<uintptr_t>(a.knorms + x.kv_row0 + x.start) & 15) == 0;
    return x;
  };
  // the block's next item after `item` that has tiles (-1: none); tiles run on from one such item to the next
  auto next_with_tiles = [&](int item) {
    for (int it = item + gridDim.x; it < items; it += gridDim.x)
      if (geo(it).ntiles > 0) return it;
    return -1;
  };
  // Tiles form one sequence over the block's items.  Slot u of item x (block tile seq0 + u, stage (seq0 + u) % NST)
  // is x's tile u, or past x's end the next item with tiles' tile u - x.ntiles; every call commits one cp.async
  // group (norms), so that a wait for "all but the newest NST - 2" finds the slot issued NST - 1 calls earlier.
  auto issue_slot = [&](const Geo& x, const Geo& xn, bool has_n, int seq0, int u) {
    const bool cur = u < x.ntiles;
    const bool nxt = !cur && has_n && u - x.ntiles < xn.ntiles;
    if (cur || nxt) {  // selects rather than a pointer, so that neither item's fields leave registers
      const int tile = cur ? u : u - x.ntiles;
      const int ystart = cur ? x.start : xn.start, yvend = cur ? x.vend : xn.vend;
      const size_t yrow0 = cur ? x.kv_row0 : xn.kv_row0;
      const bool ynrm = cur ? x.nrm_async : xn.nrm_async;
      const int s = (seq0 + u) % NST;
      uint8_t* st = smem + P::OFF_STAGE + static_cast<size_t>(s) * P::STAGE;
      const int t0 = ystart + tile * TT;
      const int n = min(TT, yvend - t0);
      const int nbytes = n * P::R;
      const uint8_t* src = a.kcodes + (yrow0 + t0) * P::R;
      if constexpr (P::BULK) {
        if (tid == 0) {
          mbar_arrive_expect_tx(full + s, nbytes);
          bulk_copy_g2s(st, src, nbytes, full + s);
        }
      } else {
        for (int o = tid * 8; o < nbytes; o += P::THREADS * 8) cp_async<8>(st + o, src + o);
      }
      if (ynrm && tid < TT / 8) {  // 16-byte chunks of 8 tokens, 16 per 128-token half
        const int h0 = 128 * (tid >> 4);
        stage_norms(nst + s * TT + h0, a.knorms + yrow0 + t0 + h0, n - h0, tid & 15);
      }
    }
    cp_async_commit();
  };
  auto fetch_queries = [&](int item, int k) {  // one thread: item's raw queries into buffer k % 2
    const Geo x = geo(item);
    const uint32_t qb = static_cast<uint32_t>(P::QB);
    mbar_arrive_expect_tx(qfull + (k & 1), qb);
    bulk_copy_g2s(qbuf + (k & 1) * G * D, a.q + (static_cast<size_t>(x.b) * a.Hq + x.hk * G) * D, qb,
                  qfull + (k & 1));
  };

  if (static_cast<int>(blockIdx.x) < items) {  // the first item's queries and first slots
    if (tid == 0) fetch_queries(blockIdx.x, 0);
    const Geo x0 = geo(blockIdx.x);
    const int n0 = next_with_tiles(blockIdx.x);
    const Geo x1 = n0 >= 0 ? geo(n0) : x0;
    // bulk copies: warp 0 alone issues (thread 0 the codes, its lanes the norms); the other warps skip the slot
    // arithmetic, and their cp.async waits find no groups
    if (!P::BULK || warp == 0)
      for (int u = 0; u < NST - 1; ++u) issue_slot(x0, x1, n0 >= 0, 0, u);
  }

  int done = 0;  // tiles of this block's earlier items
  int k = 0;     // items of this block so far
  for (int item = blockIdx.x; item < items; item += gridDim.x, ++k) {
    const Geo x = geo(item);
    float* out = a.scores + (static_cast<size_t>(x.b) * a.Hq + x.hk * G) * a.T;
    for (int t = max(x.start, x.vend) + tid; t < x.end; t += P::THREADS)  // masked positions
#pragma unroll
      for (int g = 0; g < G; ++g) out[static_cast<size_t>(g) * a.T + t] = -INFINITY;

    fence_proxy_async();
    __syncthreads();  // the previous item is finished with the row factors and the B fragments
    if (tid == 0 && item + static_cast<int>(gridDim.x) < items) fetch_queries(item + gridDim.x, k + 1);
    if (!tc::mbar_wait(qfull + (k & 1), static_cast<uint32_t>((k >> 1) & 1))) *failed = 1;
    if (x.ntiles == 0) continue;  // its slots carried the next item's tiles
    const int nn = next_with_tiles(item);
    const Geo xn = nn >= 0 ? geo(nn) : x;
    transform_queries<D, G>(qbuf + (k & 1) * G * D, sgn, a.mult, qs);
    __syncthreads();
    if (warp < G) {  // one warp per head
      const float sc = head_scale_rows<D>(qs + warp * D);
      if (lane == 0) sclv[warp] = sc;
    }
    __syncthreads();
    mma_b_stage<D, G>(qs, sclv, bs);  // the block builds the B fragments once
    __syncthreads();
    MmaB<D, G> B;
    mma_b_load<D, G>(bs, sclv, lane, B);
    const __half* kn_src = a.knorms + x.kv_row0;

    for (int tile = 0; tile < x.ntiles; ++tile) {
      const int s = (done + tile) % NST;
      const int t0 = x.start + tile * TT;
      const int nt_tok = min(TT, x.vend - t0);
      cp_async_wait<NST - 2>();
      __syncthreads();  // the tile's norms (and cp.async codes) are complete everywhere; the previous stage is free
      if (!P::BULK || warp == 0) issue_slot(x, xn, nn >= 0, done, tile + NST - 1);
      const uint8_t* st = smem + P::OFF_STAGE + static_cast<size_t>(s) * P::STAGE;
      if constexpr (P::BULK) {
        if (!tc::mbar_wait(full + s, static_cast<uint32_t>(((done + tile) / NST) & 1))) *failed = 1;
      }
      // a code tile that never arrived (a copy that did not complete in about a second) poisons the scores
      const float poison = *failed ? __int_as_float(0x7fc00000) : rd;
      // both M tiles unconditionally (rows past the tile's end hold stale codes -- any byte is a valid table
      // index -- whose scores are dropped), so that their lookup and MMA chains interleave
      float sc[2][NT][2];
#pragma unroll
      for (int m = 0; m < 2; ++m) mma_scores16<D, BITS, G, false>(st, warp * WT + 16 * m, tab, rep16, B, lane, sc[m]);
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        const int row0 = warp * WT + 16 * m;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int r = row0 + gq + 8 * i;
          if (r < nt_tok) {
            const float f = __half2float(x.nrm_async ? nst[s * TT + r] : kn_src[t0 + r]) * poison;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              const int h = 4 * nt + tq;
              if (h < G) out[static_cast<size_t>(h) * a.T + t0 + r] = sc[m][nt][i] * B.inv[nt] * f;
            }
          }
        }
      }
    }
    done += x.ntiles;
  }
  cp_async_wait<0>();
  __syncthreads();
  report_wait_failure(a, failed);
}

}  // namespace axr
