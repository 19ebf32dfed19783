// Scores on the tensor cores: a warp-specialised, mbarrier-pipelined persistent kernel (one CTA per SM).
//
// AXELRAM Key Points (1st, 2nd items): every cached token's score is the gather-sum of the query's table entries
// at the token's stored indices, times its stored norm.  Here the table is kept in factored form (tc.cuh): the
// gathered centroids of 128 tokens form the A operand of one M = 128, N = 16 MMA chain in tensor memory, the
// query's hi/lo planes form B in shared memory, and the fp32 accumulator holds the tile's scores for every head of
// the KV head.
//
// Roles (416 threads):
//   gather warps 0..7   -- warp w owns TMEM lanes 32 (w % 4) .. + 31 (tokens of the tile) and coordinate-pair
//                          group w / 4 (half of each row's pairs); per tile it reads its half rows of codes from
//                          the staged tile, looks up the hi/lo centroid pairs and stores them into A buffer i % 3
//                          with tcgen05.st, then arrives on a_full.  The same threads stage the key codes: each
//                          copies its share of the tile five ahead with cp.async and arrives (on completion) on
//                          that stage's code_full barrier.
//   epilogue warps 8..11 -- read the accumulator of tile i once mma_done fires, release it (d_empty), scale by the
//                          norms and store the scores; they also build the query operand B of the next row
//                          (double-buffered) while the current one is in use.
//   MMA warp 12 (lane 0) -- waits for a_full (and d_empty, b_full), issues the d/8 MMAs of the tile and commits
//                          them to mma_done, which also frees the A buffer for the gather warps.
// The tile list of the whole problem (rows (b, kv head) in order, ceil(len_b / 128) tiles each) is cut into one
// contiguous range per CTA, so the pipeline runs across row boundaries without draining.  Every wait is bounded;
// a wait that runs out sets a block-wide failure flag, every role leaves its loop, and the CTA's scores are set to
// NaN.
#pragma once

#include <type_traits>

#include "decode.cuh"

namespace axr {

// Position in a CTA's tile range: row (b, hk), tile j of the row's ntr tiles, and k = rows entered so far.
struct TileCursor {
  int b, hk, j, ntr, k;
};

__device__ __forceinline__ int row_tiles(const DecodeArgs& a, int b) { return (row_len(a, b) + kTile - 1) / kTile; }

__device__ inline long long total_tiles(const DecodeArgs& a) {
  long long t = 0;
  for (int b = 0; b < a.B; ++b) t += static_cast<long long>(row_tiles(a, b)) * a.Hkv;
  return t;
}

__device__ inline void cursor_init(const DecodeArgs& a, long long g, TileCursor& c) {
  c.k = 0;
  for (int b = 0; b < a.B; ++b) {
    const int nt = row_tiles(a, b);
    const long long nb = static_cast<long long>(nt) * a.Hkv;
    if (g < nb) {
      c.b = b;
      c.hk = static_cast<int>(g / nt);
      c.j = static_cast<int>(g % nt);
      c.ntr = nt;
      return;
    }
    g -= nb;
  }
  c.b = a.B;
  c.hk = c.j = c.ntr = 0;
}

__device__ inline void cursor_next(const DecodeArgs& a, TileCursor& c) {
  if (++c.j < c.ntr) return;
  c.j = 0;
  ++c.k;
  if (++c.hk < a.Hkv) return;
  c.hk = 0;
  do {
    ++c.b;
  } while (c.b < a.B && row_tiles(a, c.b) == 0);
  c.ntr = c.b < a.B ? row_tiles(a, c.b) : 0;
}

// A wait whose outcome is the same in every lane of the warp (the tcgen05 loads and stores that follow are
// warp-collective).
__device__ __forceinline__ bool warp_wait(uint64_t* mbar, uint32_t parity) {
  const bool ok = tc::mbar_wait(mbar, parity);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ bool warp_failed(volatile int* failed) {
  return __shfl_sync(0xffffffffu, *failed, 0) != 0;
}

template <int D, int BITS, int G>
struct TcScorePlan {
  static constexpr int TT = tc::kM;            // tokens per tile = TMEM lanes
  static constexpr int R = D * BITS / 8;       // code bytes per token
  static constexpr int KCH = (R % 16 == 0) ? 16 : 8;
  static constexpr int NGRP = 2;               // coordinate-pair groups (4 gather warps each)
  static constexpr int GW = 4 * NGRP;          // gather warps
  static constexpr int GT = 32 * GW;           // gather threads
  static constexpr int EW0 = GW;               // first epilogue warp (a multiple of 4: warp % 4 = TMEM lane quarter)
  static constexpr int MW = GW + 4;            // MMA warp
  static constexpr int THREADS = 32 * (MW + 1);
  static constexpr int PAIRS = D / 2;
  static constexpr int PG = PAIRS / NGRP;      // pairs per group
  static constexpr int GBYTES = R / NGRP;      // code bytes per group
  static constexpr bool HALF_ROWS = GBYTES % 16 == 0;  // a group reads only its own 16-byte chunks
  static constexpr int NB = 3;                 // A / accumulator buffers in TMEM
  static constexpr int NS = 8;                 // code stages
  static constexpr int LA = NS - NB;           // tiles of copy lookahead
  static constexpr int ACOLS = D;              // TMEM columns of one A buffer (2 D fp16)
  static constexpr int DCOL0 = NB * ACOLS;     // first accumulator column
  static constexpr int DSTRIDE = 32;
  static constexpr int TMEM_COLS = 512;
  static_assert(DCOL0 + NB * DSTRIDE <= TMEM_COLS, "TMEM budget");
  static_assert(G <= tc::kN / 2, "two accumulator columns per head");
  static constexpr int STAGE = TT * R;
  static constexpr int B_BYTES = tc::Layout<D>::B_BYTES;
  static constexpr size_t OFF_STAGE = 0;
  static constexpr size_t OFF_TAB = ((size_t)NS * STAGE + 1023) / 1024 * 1024;
  static constexpr size_t OFF_B = OFF_TAB + ((size_t)tc::PairTable16<BITS>::BYTES + 1023) / 1024 * 1024;
  static constexpr size_t OFF_CENT = OFF_B + 2 * (size_t)B_BYTES;
  static constexpr size_t OFF_MBAR = OFF_CENT + 16 * 4;               // a_full, mma_done, d_empty, code_full, b_full
  static constexpr int NMBAR = 3 * NB + NS + 2;
  static constexpr size_t OFF_MISC = OFF_MBAR + (size_t)NMBAR * 8;    // TMEM base, failure flag
  static constexpr size_t bytes = OFF_MISC + 16;
  // at least 120 KB so that two CTAs never share an SM (each holds all 512 TMEM columns)
  static constexpr size_t launch_bytes = bytes > 120 * 1024 ? bytes : 120 * 1024;
};

template <int D, int BITS, int G>
__global__ void __launch_bounds__(TcScorePlan<D, BITS, G>::THREADS, 1)
score_tc_kernel(const __grid_constant__ DecodeArgs a) {
  using P = TcScorePlan<D, BITS, G>;
  constexpr int R = P::R, TT = P::TT, NB = P::NB, NS = P::NS, LA = P::LA, PG = P::PG;
  extern __shared__ __align__(16) uint8_t smem[];
  uint8_t* stage = smem + P::OFF_STAGE;
  const uint8_t* tab = smem + P::OFF_TAB;
  float* cent = reinterpret_cast<float*>(smem + P::OFF_CENT);
  uint64_t* mbar = reinterpret_cast<uint64_t*>(smem + P::OFF_MBAR);
  uint64_t* a_full = mbar;
  uint64_t* mma_done = mbar + NB;
  uint64_t* d_empty = mbar + 2 * NB;
  uint64_t* code_full = mbar + 3 * NB;
  uint64_t* b_full = mbar + 3 * NB + NS;
  uint32_t* tmem_s = reinterpret_cast<uint32_t*>(smem + P::OFF_MISC);
  volatile int* failed = reinterpret_cast<volatile int*>(smem + P::OFF_MISC + 4);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  // this CTA's share of the tile list
  const long long total = total_tiles(a);
  const long long g0 = total * blockIdx.x / gridDim.x;
  const int n = static_cast<int>(total * (blockIdx.x + 1) / gridDim.x - g0);

  // positions past a row's length score -inf: rows (b, h) dealt round-robin over the CTAs
  for (long long rh = blockIdx.x; rh < static_cast<long long>(a.B) * a.Hq; rh += gridDim.x) {
    const int len = row_len(a, static_cast<int>(rh / a.Hq));
    float* o = a.scores + rh * a.T;
    for (int t = len + tid; t < a.T; t += P::THREADS) o[t] = -INFINITY;
  }
  if (n <= 0) return;  // uniform over the block, before any barrier or TMEM use

  if (tid < 16) cent[tid] = a.cb.gamma[tid];
  if (warp == 0) tc::tmem_alloc(tmem_s, P::TMEM_COLS);
  if (tid == 0) {
    for (int i = 0; i < NB; ++i) {
      tc::mbar_init(a_full + i, P::GW);
      tc::mbar_init(mma_done + i, 1);
      tc::mbar_init(d_empty + i, 4);
    }
    for (int i = 0; i < NS; ++i) tc::mbar_init(code_full + i, P::GT);
    for (int i = 0; i < 2; ++i) tc::mbar_init(b_full + i, 1);
    *failed = 0;
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *tmem_s;
  tc::build_table<BITS>(cent, reinterpret_cast<uint2*>(smem + P::OFF_TAB));
  for (int i = tid; i < 2 * P::B_BYTES / 4; i += P::THREADS)  // entries the row builder never writes stay 0
    reinterpret_cast<uint32_t*>(smem + P::OFF_B)[i] = 0u;
  tc::fence_async_smem();
  __syncthreads();

  if (warp < P::GW) {
    // ===================================== gather =====================================
    const int grp = warp / 4, quarter = warp & 3, tt = quarter * 32 + lane;
    const uint32_t repw = static_cast<uint32_t>(lane) << 3;
    const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    TileCursor cur, ahead;
    cursor_init(a, g0, cur);
    cursor_init(a, g0, ahead);
    auto issue = [&](int ia) {  // stage tile ia (the `ahead` cursor) into stage ia % NS
      if (ia >= n) return;
      const int t0 = ahead.j * TT;
      const int bytes = min(TT, row_len(a, ahead.b) - t0) * R;
      const uint8_t* src = a.kcodes + ((static_cast<size_t>(ahead.b) * a.Hkv + ahead.hk) * a.Tcap + t0) * R;
      uint8_t* dst = stage + static_cast<size_t>(ia % NS) * P::STAGE;
      for (int o = tid * P::KCH; o < bytes; o += P::GT * P::KCH) cp_async<P::KCH>(dst + stage_swizzle<R>(o), src + o);
      tc::cp_async_mbar_arrive(code_full + ia % NS);
      cursor_next(a, ahead);
    };
    for (int i = 0; i < LA; ++i) issue(i);
    for (int i = 0; i < n; ++i) {
      const int s = i % NB;
      if (i >= NB && !warp_wait(mma_done + s, ((i / NB) - 1) & 1)) { *failed = 1; break; }
      if (warp_failed(failed)) break;
      issue(i + LA);  // into the stage tile i - NB used: every gather thread is past it (MMA i - NB has run)
      if (!warp_wait(code_full + i % NS, (i / NS) & 1)) { *failed = 1; break; }
      tc::fence_after();
      const int nt = min(TT, row_len(a, cur.b) - cur.j * TT);
      const uint8_t* st = stage + static_cast<size_t>(i % NS) * P::STAGE;
      uint32_t hi[PG], lo[PG];
      if constexpr (P::HALF_ROWS) {
        constexpr int NW = P::GBYTES / 4;
        uint32_t w[NW + 1];
#pragma unroll
        for (int c = 0; c < P::GBYTES / 16; ++c) {
          const uint4 u = *reinterpret_cast<const uint4*>(st + stage_swizzle<R>(tt * R + grp * P::GBYTES + c * 16));
          w[4 * c] = u.x; w[4 * c + 1] = u.y; w[4 * c + 2] = u.z; w[4 * c + 3] = u.w;
        }
        w[NW] = 0u;
        if (tt >= nt) {
#pragma unroll
          for (int c = 0; c < NW; ++c) w[c] = 0u;
        }
#pragma unroll
        for (int p = 0; p < PG; ++p) {
          const uint2 e = *reinterpret_cast<const uint2*>(tab + tc::pair_off<BITS>(w, p, repw));
          hi[p] = e.x;
          lo[p] = e.y;
        }
      } else {
        uint32_t w[R / 4 + 1];
        load_swizzled_row<R>(st, tt, w);
        w[R / 4] = 0u;
        if (tt >= nt) {
#pragma unroll
          for (int c = 0; c < R / 4; ++c) w[c] = 0u;
        }
        // the group's first pair as a compile-time constant keeps w[] in registers
        auto lookup = [&](auto first) {
#pragma unroll
          for (int p = 0; p < PG; ++p) {
            const uint2 e = *reinterpret_cast<const uint2*>(tab + tc::pair_off<BITS>(w, decltype(first)::value + p, repw));
            hi[p] = e.x;
            lo[p] = e.y;
          }
        };
        static_assert(P::NGRP == 2, "two pair groups");
        if (grp == 0) lookup(std::integral_constant<int, 0>{});
        else lookup(std::integral_constant<int, PG>{});
      }
      const uint32_t acol = tl + static_cast<uint32_t>(s * P::ACOLS + grp * PG);
      if constexpr (PG == 32) {
        tc::st_x32(acol, hi);
        tc::st_x32(acol + P::PAIRS, lo);
      } else {
        static_assert(PG == 16, "16 or 32 pairs per group");
        tc::st_x16(acol, hi);
        tc::st_x16(acol + P::PAIRS, lo);
      }
      tc::wait_st();
      tc::fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(a_full + s);
      cursor_next(a, cur);
    }
    cp_async_wait<0>();
  } else if (warp < P::MW) {
    // ==================================== epilogue ====================================
    const int quarter = warp & 3, tt = quarter * 32 + lane;
    const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const float rd = rsqrtf(static_cast<float>(D));
    const bool builder = warp == P::EW0;
    // B of row (b, hk) into slot `slot`, by the builder warp alone (no cross-warp barrier)
    auto build_row_b = [&](int b, int hk, int slot) {
      tc::build_b_warp<D, G>(a.q + (static_cast<size_t>(b) * a.Hq + hk * G) * D, a.signs, a.mult,
                             reinterpret_cast<__half*>(smem + P::OFF_B + slot * P::B_BYTES));
      tc::fence_async_smem();  // B is read by the tensor cores (async proxy)
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(b_full + slot);
    };
    TileCursor cur;
    cursor_init(a, g0, cur);
    if (builder) build_row_b(cur.b, cur.hk, 0);
    auto norm_of = [&](const TileCursor& c) {
      const int t = c.j * TT + tt;
      return t < row_len(a, c.b) ? __half2float(a.knorms[(static_cast<size_t>(c.b) * a.Hkv + c.hk) * a.Tcap + t])
                                 : 0.f;
    };
    float kn_next = norm_of(cur);
    float inv[G];
    for (int i = 0; i < n; ++i) {
      const int s = i % NB;
      const bool first = i == 0 || cur.j == 0;
      if (first) {  // the row's head scales (the same computation as the builder's)
        const float* qg = a.q + (static_cast<size_t>(cur.b) * a.Hq + cur.hk * G) * D;
#pragma unroll
        for (int g = 0; g < G; ++g) inv[g] = 1.f / tc::head_scale<D>(qg + g * D, a.mult);
      }
      const float kn = kn_next;
      TileCursor nxt = cur;
      cursor_next(a, nxt);
      if (i + 1 < n) kn_next = norm_of(nxt);
      if (!warp_wait(mma_done + s, (i / NB) & 1)) { *failed = 1; break; }
      tc::fence_after();
      uint32_t d[16];
      tc::ld_x16(tl + static_cast<uint32_t>(P::DCOL0 + s * P::DSTRIDE), d);
      tc::wait_ld();
      tc::fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(d_empty + s);
      const int t0 = cur.j * TT;
      if (t0 + tt < row_len(a, cur.b)) {
        float* out = a.scores + (static_cast<size_t>(cur.b) * a.Hq + cur.hk * G) * a.T + t0 + tt;
        const float f = kn * rd;
#pragma unroll
        for (int g = 0; g < G; ++g)
          out[static_cast<size_t>(g) * a.T] = (__uint_as_float(d[2 * g]) + __uint_as_float(d[2 * g + 1])) * inv[g] * f;
      }
      // on the first tile of a row, prepare B of the next row: its slot was last read by MMAs of the row before,
      // which have completed (mma_done of this tile covers every earlier MMA)
      if (builder && first && i + (cur.ntr - cur.j) < n) {
        TileCursor nr = cur;
        nr.j = nr.ntr - 1;
        cursor_next(a, nr);
        build_row_b(nr.b, nr.hk, (cur.k + 1) & 1);
      }
      if (warp_failed(failed)) break;
      cur = nxt;
    }
  } else if (lane == 0) {
    // ====================================== MMA ======================================
    const uint32_t b0 = smem_u32(smem + P::OFF_B);
    TileCursor cur;
    cursor_init(a, g0, cur);
    int last = -1;
    for (int i = 0; i < n; ++i) {
      const int s = i % NB;
      if (*failed) break;
      if ((i == 0 || cur.j == 0) && !tc::mbar_wait(b_full + (cur.k & 1), (cur.k >> 1) & 1)) { *failed = 1; break; }
      if (i >= NB && !tc::mbar_wait(d_empty + s, ((i / NB) - 1) & 1)) { *failed = 1; break; }
      if (!tc::mbar_wait(a_full + s, (i / NB) & 1)) { *failed = 1; break; }
      tc::fence_after();
      tc::issue_mma<D>(tmem + static_cast<uint32_t>(s * P::ACOLS), tmem + static_cast<uint32_t>(P::DCOL0 + s * P::DSTRIDE),
                       b0 + static_cast<uint32_t>((cur.k & 1) * P::B_BYTES), mma_done + s);
      last = i;
      cursor_next(a, cur);
    }
    // nothing may be in flight when the columns are released
    if (last >= 0 && !tc::mbar_wait(mma_done + last % NB, (last / NB) & 1)) *failed = 1;
  }

  tc::fence_before();
  __syncthreads();
  report_wait_failure(a, failed);
  if (*failed) {  // the scores of this CTA's tiles are not valid
    TileCursor cur;
    cursor_init(a, g0, cur);
    for (int i = 0; i < n; ++i) {
      const int len = row_len(a, cur.b);
      float* out = a.scores + (static_cast<size_t>(cur.b) * a.Hq + cur.hk * G) * a.T;
      for (int e = tid; e < G * TT; e += P::THREADS) {
        const int t = cur.j * TT + e % TT;
        if (t < len) out[static_cast<size_t>(e / TT) * a.T + t] = __int_as_float(0x7fc00000);
      }
      cursor_next(a, cur);
    }
  }
  if (warp == 0) {
    tc::fence_after();
    tc::tmem_dealloc(tmem, P::TMEM_COLS);
  }
}

}  // namespace axr
