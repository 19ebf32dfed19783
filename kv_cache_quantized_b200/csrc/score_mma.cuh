// Scores through warp-level MMAs (mma.sync.m16n8k16, fp16 operands, fp32 accumulation).
//
// AXELRAM Key Points (1st, 2nd items): every cached token's score is the gather-sum of the query's table entries at
// the token's stored indices, times its stored norm.  The table is read in factored form (mma_score.cuh): each
// token's centroids, split into hi and lo fp16 planes (about 22 bits), form a row of A; the query's hi/lo planes
// form B, built once per (batch, KV head) and kept in registers; lane (g, t) ends with head t's score of tokens g
// and g + 8 of an M = 16 tile.  There is no shuffle reduction and no cross-warp hand-off inside a tile: warp w owns
// tokens [32 w, 32 w + 32) of each 256-token tile (two M = 16 tiles).  Code tiles arrive as one bulk copy each
// (completing on a per-stage mbarrier), norms as 16-byte cp.async chunks, four stages deep, with one block barrier
// per tile.  Blocks are persistent (two per SM) over (batch, KV head, split) items and build the pair table once.
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
  static constexpr int NST = 4;                   // stages: three tiles in flight per block
  static constexpr bool BULK = R % 16 == 0;       // codes as one bulk copy per tile, else 8-byte cp.async chunks
  static constexpr size_t OFF_STAGE = 0;
  static constexpr size_t OFF_NRM = (size_t)NST * STAGE;                    // [NST][TT] fp16 key norms
  static constexpr size_t OFF_TAB = (OFF_NRM + (size_t)NST * TT * 2 + 127) / 128 * 128;
  static constexpr size_t OFF_QS = OFF_TAB + (size_t)HiLoTable16<BITS>::BYTES;  // [G][D] row factors
  static constexpr size_t OFF_CENT = OFF_QS + (size_t)G * D * 4;
  static constexpr size_t OFF_MB = OFF_CENT + 16 * 4;                       // [NST] stage barriers, flag
  static constexpr size_t bytes = OFF_MB + NST * 8 + 8;
  static_assert(bytes <= 113 * 1024, "two blocks per SM");
};

template <int D, int BITS, int G>
__global__ void __launch_bounds__(256, 2) score_mma_kernel(const __grid_constant__ DecodeArgs a) {
  using P = ScoreMmaPlan<D, BITS, G>;
  constexpr int NT = P::NT, TT = P::TT, WT = P::WT, NST = P::NST;
  extern __shared__ __align__(16) uint8_t smem[];
  const uint8_t* tab = smem + P::OFF_TAB;
  float* qs = reinterpret_cast<float*>(smem + P::OFF_QS);
  float* cent = reinterpret_cast<float*>(smem + P::OFF_CENT);
  __half* nst = reinterpret_cast<__half*>(smem + P::OFF_NRM);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + P::OFF_MB);  // stage s holds its code tile
  volatile int* failed = reinterpret_cast<volatile int*>(full + NST);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, tq = lane & 3;
  const uint32_t rep16 = static_cast<uint32_t>(lane & 15) << 4;
  const float rd = rsqrtf(static_cast<float>(D));

  if (tid < 16) cent[tid] = a.cb.gamma[tid];
  if (tid == 0) {
    for (int s = 0; s < NST; ++s) tc::mbar_init(full + s, 1);
    *failed = 0;
  }
  __syncthreads();
  build_hilo_table16<BITS>(cent, smem + P::OFF_TAB);  // once per block
  // tile t of an item uses stage (done + t) % NST and its barrier phase of parity ((done + t) / NST) & 1
  int done = 0;
  auto stg = [&](int tile) { return (done + tile) % NST; };
  auto par = [&](int tile) { return static_cast<uint32_t>(((done + tile) / NST) & 1); };

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

    fence_proxy_async();
    __syncthreads();  // the previous item is finished with the stages and the row factors
    // key norms ride with the codes when the item's norm row starts 16-byte aligned, else each lane loads its own
    const __half* kn_src = a.knorms + kv_row0;
    const bool nrm_async = (reinterpret_cast<uintptr_t>(kn_src + start) & 15) == 0;
    auto issue_tile = [&](int tile) {
      if (tile < ntiles) {
        uint8_t* st = smem + P::OFF_STAGE + static_cast<size_t>(stg(tile)) * P::STAGE;
        const int t0 = start + tile * TT;
        const int n = min(TT, vend - t0);
        const int nbytes = n * P::R;
        const uint8_t* src = a.kcodes + (kv_row0 + t0) * P::R;
        if constexpr (P::BULK) {
          if (tid == 0) {
            mbar_arrive_expect_tx(full + stg(tile), nbytes);
            bulk_copy_g2s(st, src, nbytes, full + stg(tile));
          }
        } else {
          for (int o = tid * 8; o < nbytes; o += P::THREADS * 8) cp_async<8>(st + o, src + o);
        }
        if (nrm_async && tid < TT / 8) {  // 16-byte chunks of 8 tokens, 16 per 128-token half
          const int h0 = 128 * (tid >> 4);
          stage_norms(nst + stg(tile) * TT + h0, kn_src + t0 + h0, n - h0, tid & 15);
        }
      }
      cp_async_commit();
    };
    for (int s = 0; s < NST - 1; ++s) issue_tile(s);
    transform_queries<D, G>(qg, a.signs, a.mult, qs);
    float scl[G];
#pragma unroll
    for (int g = 0; g < G; ++g) scl[g] = tc::head_scale<D>(qg + g * D, a.mult);
    __syncthreads();
    MmaB<D, G> B;
    mma_b_build<D, G>(qs, scl, lane, B);

    for (int tile = 0; tile < ntiles; ++tile) {
      const int t0 = start + tile * TT;
      const int nt_tok = min(TT, vend - t0);
      cp_async_wait<NST - 2>();
      __syncthreads();  // the tile's norms (and cp.async codes) are complete everywhere; the previous stage is free
      issue_tile(tile + NST - 1);
      const uint8_t* st = smem + P::OFF_STAGE + static_cast<size_t>(stg(tile)) * P::STAGE;
      if constexpr (P::BULK) {
        if (!tc::mbar_wait(full + stg(tile), par(tile))) *failed = 1;
      }
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        const int row0 = warp * WT + 16 * m;
        if (row0 >= nt_tok) break;
        float s[NT][2];
        mma_scores16<D, BITS, G, false>(st, row0, tab, rep16, B, lane, s);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int r = row0 + gq + 8 * i;
          if (r < nt_tok) {
            const float kn = nrm_async ? __half2float(nst[stg(tile) * TT + r]) : __half2float(kn_src[t0 + r]);
            // a code tile that never arrived (a copy that did not complete in about a second) poisons the scores
            const float f = *failed ? __int_as_float(0x7fc00000) : kn * rd;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              const int h = 4 * nt + tq;
              if (h < G) out[static_cast<size_t>(h) * a.T + t0 + r] = s[nt][i] * B.inv[nt] * f;
            }
          }
        }
      }
    }
    cp_async_wait<0>();
    done += ntiles;
  }
}

}  // namespace axr
