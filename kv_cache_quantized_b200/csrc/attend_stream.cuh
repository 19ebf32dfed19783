// Decode attention over quantized keys, and fp16 or quantized values, as a pure stream: the dense kernel's skeleton
// (dense_stream.cuh) with the keys scored from their codes.
//
// AXELRAM Key Points (1st, 2nd items): a token's score is the gather-sum of q~_j c_k at its stored indices times its
// stored norm; the table is read in factored form on mma.sync exactly as mma_score.cuh does it (one MMA per 8 tokens
// and 16 coordinates carries the four products of the hi/lo fp16 planes of both factors; fp32 accumulation).  Lane
// (g, t) then holds head t's scores of tokens g and g + 8 of each 16-token group.  The value product is
//   O^T (d x heads) += V^T (d x tokens) P^T (tokens x heads):
//   fp16 values: A = V^T, read with ldmatrix.trans from the 128-byte-swizzled TMA boxes of the value rows; B = P^T
//       as hi and lo fp16 planes (fp32-level weights, so that the result does not depend on where the splits fall),
//       gathered from the score lanes with four shuffles per 16 tokens;
//   quantized values: the contraction runs over (token t, half s) and the columns over (head h, half s'), with
//       A[p][(t, s)] = v_t,2p+s and B[(t, s)][(h, s')] = [s = s'] p_t,h n^V_t / sqrt(D), so that
//       C[p][(h, s')] = O^T[2 p + s'][h]: one lookup in the hi-only copies of the key/value pair table (the fp16
//       pair (v_2p, v_2p+1) of a token's code byte) is one A register as it is, and B is P^T with a zero beside
//       every weight.  An MMA covers 16 coordinate pairs x 8 tokens x 4 heads; fp16 weights (the table's hi plane
//       holds the centroids to 2^-11); the product stays in the rotated domain and the merge applies the one
//       inverse transform.
//
// Every warp is an independent worker over (batch row, KV head, split) items with a ring of NS stages of its own: a
// stage holds TW tokens' value rows (fp16: D / 64 tiled TMA boxes; quantized: one bulk copy of code rows) and key
// code rows (one bulk copy).  No barrier spans two
// warps.  A decode step's new token is written by the warp whose item holds it, before that item's copies.
#pragma once

#include <cuda.h>

#include "append.cuh"
#include "dense_stream.cuh"
#include "mma_score.cuh"

namespace axr {

template <int D, int BITS, int G, bool VQ>
struct StreamPlan {
  static constexpr int TW = 32;                          // tokens per warp tile
  static constexpr int NS = 2;                           // stages per warp
  static constexpr int WARPS = VQ ? 16 : 8;              // warps per block (one block per SM)
  static constexpr int THREADS = 32 * WARPS;
  static constexpr int R = D * BITS / 8;                 // bytes of a key code row
  static constexpr int BOXC = 64;                        // value coordinates per TMA box
  static constexpr int NBX = D / BOXC;                   // value boxes per row
  static constexpr size_t BOX = (size_t)TW * 128;
  static constexpr size_t VPLANE = VQ ? (size_t)TW * R : NBX * BOX;  // value rows of a stage (first: 1024-aligned)
  static constexpr size_t KPLANE = (size_t)TW * R;       // key code rows of a stage
  static constexpr size_t STAGE = (VPLANE + KPLANE + 1023) / 1024 * 1024;
  static constexpr size_t SCRATCH = ((size_t)G * D * 4 + D + 1023) / 1024 * 1024;  // queries + index scratch
  static constexpr size_t WARP_BYTES = NS * STAGE > SCRATCH ? NS * STAGE : SCRATCH;
  static constexpr size_t OFF_TAB = WARPS * WARP_BYTES;
  static constexpr size_t TAB_BYTES = VQ ? (size_t)PairTableKV<BITS>::BYTES : (size_t)HiLoTable16<BITS>::BYTES;
  static constexpr size_t OFF_MBAR = OFF_TAB + TAB_BYTES;
  static constexpr size_t bytes = 1024 + OFF_MBAR + (size_t)WARPS * NS * 8;  // + the alignment slack
  static constexpr int NT = MmaB<D, G>::NT;              // n-tiles of heads (2: heads 4..7)
  static constexpr int MTV = D / 16;                     // m-tiles of the value product (16 coordinates)
  static constexpr int MPQ = D / 32;                     // quantized values: m-tiles of 16 coordinate pairs
  static constexpr int NBV = R / 8;                      // bytes of lane g's run of a row: pairs D/16 g .. + D/16
  static constexpr int NWV = (NBV + 3) / 4 + 1;          // its words, plus a zero word
  static_assert(R % 8 == 0 && (TW * R) % 16 == 0, "tiles of code rows in whole 16-byte chunks");
  static_assert(TW == 32, "two 16-token groups per tile");
  static_assert(bytes <= 227 * 1024, "shared memory of one block");
};

// vmap: the TMA map of the fp16 value cache (fp16 values only).  PAGED: the rows of each (batch row, KV head) come
// through the block table (RowMap); blocks of at least TW tokens, so that a tile (its first token a multiple of TW)
// never spans two blocks and stays one run of rows.
template <int D, int BITS, int G, bool VQ, bool PAGED = false>
__global__ void __launch_bounds__(StreamPlan<D, BITS, G, VQ>::THREADS, 1)
attend_stream_kernel(const __grid_constant__ DecodeArgs a, const __grid_constant__ CUtensorMap vmap) {
  using P = StreamPlan<D, BITS, G, VQ>;
  constexpr int TW = P::TW, NS = P::NS, R = P::R, NT = P::NT, MTV = P::MTV, VPL = WarpVec<D>::VPL;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  uint8_t* ring = smem + static_cast<size_t>(warp) * P::WARP_BYTES;
  const uint8_t* tab = smem + P::OFF_TAB;
  uint64_t* mbar = reinterpret_cast<uint64_t*>(smem + P::OFF_MBAR) + warp * NS;

  {  // the pair table, once per block: hi/lo key copies (and hi-only value copies with quantized values)
    __shared__ float gamma_s[16];
    if (threadIdx.x < 16) gamma_s[threadIdx.x] = a.cb.gamma[threadIdx.x];
    if (lane == 0)
      for (int s = 0; s < NS; ++s) tc::mbar_init(mbar + s, 1);
    __syncthreads();
    if constexpr (VQ) build_pair_table_kv<BITS>(gamma_s, smem + P::OFF_TAB);
    else build_hilo_table16<BITS>(gamma_s, smem + P::OFF_TAB);
    __syncthreads();
  }
  // the split merge, launched as this grid's programmatic dependent, may be scheduled from now on
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");

  // the lane's key copy in the pair table, and (quantized values) its hi-only value copy
  const uint32_t repk = static_cast<uint32_t>(lane & 15) << (VQ ? 3 : 4);
  const uint32_t repv = 128u + (static_cast<uint32_t>(lane) << 2);
  const int a_row = (lane & 7) + 8 * (lane >> 4), a_col = 8 * ((lane >> 3) & 1);  // ldmatrix.trans rows of V^T
  const float rd = rsqrtf(static_cast<float>(D));
  // items are dealt across the blocks first (item blockIdx.x + gridDim.x (warp + WARPS k)), so that a launch with
  // fewer items than workers still spreads them over every SM
  const int workers = gridDim.x * P::WARPS;
  const int first = blockIdx.x + gridDim.x * warp;
  const int items = a.B * a.Hkv * a.splits;
  uint32_t seq = 0;  // tiles this warp has consumed: stage seq % NS, phase parity (seq / NS) & 1
  bool failed = false;

  for (int item = first; item < items && !failed; item += workers) {
    const int split = item % a.splits;
    const int hk = (item / a.splits) % a.Hkv;
    const int b = item / (a.splits * a.Hkv);
    const int len = row_len(a, b);
    const int start = split * a.chunk;
    const int end = min(start + a.chunk, len);
    const int ntiles = end > start ? (end - start + TW - 1) / TW : 0;
    const RowMap<PAGED> rm = row_map<PAGED>(a, b, hk);  // cache row of each token (contiguous or paged)
    const float* qg = a.q + (static_cast<size_t>(b) * a.Hq + hk * G) * D;
    // the ring is idle between items: it holds the transformed queries and the write path's index scratch
    float* qs = reinterpret_cast<float*>(ring);
    uint8_t* scratch = ring + static_cast<size_t>(G) * D * 4;

    if (a.knew != nullptr && len > 0 && start <= len - 1 && len - 1 < end) {
      // decode step: this item holds the new token (position len - 1): write its key and value through the write
      // path before any of the item's copies is issued
      append_row<D, BITS, VQ>(a, b, hk, rm(len - 1), 0, lane, scratch);
      append_row<D, BITS, VQ>(a, b, hk, rm(len - 1), 1, lane, scratch);
      __threadfence();                                           // the stores reach the device-wide view ...
      asm volatile("fence.proxy.async.global;\n" ::: "memory");  // ... and the async proxy of the copies
    }

    // q~_h = mult H (s .* q_h) / sqrt(D) for the G heads, then the key MMA's B fragments (head-scaled hi/lo planes)
    for (int h = 0; h < G; ++h) {
      float v[VPL];
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        const int j = lane * VPL + i;
        v[i] = qg[h * D + j] * sign_of(a.signs[j]);
      }
      fwht_warp<D>(v, lane);
#pragma unroll
      for (int i = 0; i < VPL; ++i) qs[h * D + lane * VPL + i] = v[i] * (a.mult * rd);
    }
    MmaB<D, G> QB;
    {
      float scl[G];
#pragma unroll
      for (int h = 0; h < G; ++h) scl[h] = tc::head_scale<D>(qg + h * D, a.mult);
      __syncwarp();
      mma_b_build<D, G>(qs, scl, lane, QB);
    }
    // this lane's scratch accesses come before the async proxy's copies into the ring, for every lane
    fence_proxy_async();
    __syncwarp();

    auto issue = [&](int i) {
      if (lane == 0) {
        const int s = static_cast<int>((seq + i) % NS);
        uint8_t* st = ring + static_cast<size_t>(s) * P::STAGE;
        const int t0 = start + i * TW;
        const size_t r0 = rm(t0);  // the tile's first row; its rows are consecutive
        // the tile's code rows, rounded up to whole 16-byte chunks: with rows of 8 or 24 bytes (d = 64, b = 1, 3)
        // an odd row count takes one row more, which lies inside the row's capacity (the launcher requires Tcap
        // even, and a tile that ends at Tcap has an even row count) or inside the tile's block (paged pools)
        const uint32_t cb = static_cast<uint32_t>((min(TW, end - t0) * R + 15) / 16 * 16);
        if constexpr (VQ) {
          mbar_arrive_expect_tx(mbar + s, 2 * cb);
          bulk_copy_g2s(st, static_cast<const uint8_t*>(a.v) + r0 * R, cb, mbar + s);
        } else {
          mbar_arrive_expect_tx(mbar + s, static_cast<uint32_t>(P::VPLANE) + cb);
#pragma unroll
          for (int bx = 0; bx < P::NBX; ++bx)
            tma_load_2d(st + bx * P::BOX, &vmap, bx * P::BOXC, static_cast<int>(r0), mbar + s);
        }
        bulk_copy_g2s(st + P::VPLANE, a.kcodes + r0 * R, cb, mbar + s);
      }
    };
    for (int i = 0; i < NS && i < ntiles; ++i) issue(i);

    // fp16 values: O^T (coordinate 16 mt + g (+ 8), head 2 t (+ 1)); quantized values: head 4 nt + t, coordinates
    // D/8 g + 4 mt + e
    float acc[MTV][4], accq[NT][P::MPQ][4];
#pragma unroll
    for (int mt = 0; mt < MTV; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mt][e] = 0.f;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int mt = 0; mt < P::MPQ; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) accq[nt][mt][e] = 0.f;
    float m_run[NT], l_lane[NT];  // head 4 nt + t
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) { m_run[nt] = -INFINITY; l_lane[nt] = 0.f; }

    // key (and value) norms of this lane's tokens (16 m + g + 8 i of a tile), one tile ahead, kept as raw fp16 bits
    // (key | value << 16) until the tile that uses them, so that the loads have a whole tile to land; L2-only
    // loads, since a decode step writes one of them in this launch
    auto load_norms = [&](int i, uint32_t (&nr)[2][2]) {
      const int t0 = start + i * TW;
      const size_t r0 = i < ntiles ? rm(t0) : 0;
#pragma unroll
      for (int m = 0; m < 2; ++m)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int tok = t0 + 16 * m + g + 8 * e;
          uint32_t r = 0u;  // norms 0 past the end (fp16 +0)
          if (i < ntiles && tok < end) {
            const size_t row = r0 + static_cast<size_t>(tok - t0);
            r = __half_as_ushort(__ldcg(a.knorms + row));
            if constexpr (VQ) r |= static_cast<uint32_t>(__half_as_ushort(__ldcg(a.vnorms + row))) << 16;
          }
          nr[m][e] = r;
        }
    };
    uint32_t nr_next[2][2];
    load_norms(0, nr_next);

    for (int i = 0; i < ntiles; ++i) {
      const int s = static_cast<int>((seq + i) % NS);
      if (!__all_sync(0xffffffffu, tc::mbar_wait(mbar + s, ((seq + i) / NS) & 1))) {
        // a wait gave up: stop issuing and let this warp's copies in flight land (bounded again) before exiting
        failed = true;
        for (int j = i; j < i + NS && j < ntiles; ++j) tc::mbar_wait(mbar + (seq + j) % NS, ((seq + j) / NS) & 1);
        break;
      }
      uint8_t* st = ring + static_cast<size_t>(s) * P::STAGE;
      const uint32_t sV = smem_u32(st);
      const int t0 = start + i * TW;
      float kn[2][2], vn[2][2];  // times the centroid scale 1 / sqrt(D)
#pragma unroll
      for (int m = 0; m < 2; ++m)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const uint32_t r = nr_next[m][e];
          kn[m][e] = __half2float(__ushort_as_half(static_cast<unsigned short>(r & 0xffffu))) * rd;
          vn[m][e] = VQ ? __half2float(__ushort_as_half(static_cast<unsigned short>(r >> 16))) * rd : 1.f;
        }
      load_norms(i + 1, nr_next);
      if (!VQ && t0 + TW > end) {
        // the row ends inside this tile: zero the value rows past it (whatever the cache holds there); the key
        // rows past it are stale codes, valid table indices, whose scores are masked
        uint4* vz = reinterpret_cast<uint4*>(st);
        const int r0 = end - t0;
        for (int e = lane; e < (TW - r0) * 8 * P::NBX; e += 32) {
          const int bx = e / ((TW - r0) * 8), rem = e % ((TW - r0) * 8);
          vz[(bx * P::BOX + (r0 + rem / 8) * 128) / 16 + rem % 8] = make_uint4(0u, 0u, 0u, 0u);
        }
        __syncwarp();
      }

      // ---- scores of the tile's two 16-token groups (times s_h): z[m][nt][i] is token 16 m + g + 8 i, head 4 nt + t
      float z[2][NT][2];
      if constexpr (D == 128 && BITS == 4) {
        // both groups in one pass over K, their four accumulator chains taking turns (measured ahead here: 103.4
        // -> 99.3 us for the long-context step; at d = 64 and at b = 2 the two passes below measured ahead)
        mma_scores16x2<D, BITS, G, false, VQ>(st + P::VPLANE, 0, tab, repk, QB, lane, z);
      } else {
#pragma unroll
        for (int m = 0; m < 2; ++m)
          mma_scores16<D, BITS, G, false, VQ>(st + P::VPLANE, 16 * m, tab, repk, QB, lane, z[m]);
      }

      // ---- online softmax per head (log2 units), over the lanes g of each t
      float alpha[NT];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const bool head = 4 * nt + t < G;
        float mx = -INFINITY;
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const bool valid = head && t0 + 16 * m + g + 8 * e < end;
            z[m][nt][e] = valid ? z[m][nt][e] * QB.inv[nt] * kn[m][e] : -INFINITY;
            mx = fmaxf(mx, z[m][nt][e]);
          }
#pragma unroll
        for (int msk = 4; msk < 32; msk <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, msk));
        const float m_new = fmaxf(m_run[nt], mx);
        alpha[nt] = (m_new == -INFINITY) ? 1.f : exp2f(m_run[nt] - m_new);
        float ps = 0.f;
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float p = (z[m][nt][e] == -INFINITY) ? 0.f : exp2f(z[m][nt][e] - m_new);
            z[m][nt][e] = p;
            ps += p;
          }
        l_lane[nt] = l_lane[nt] * alpha[nt] + ps;
        m_run[nt] = m_new;
      }
      // rescale the accumulators (columns: heads 2 t and 2 t + 1) when some head's running max moved
      bool moved = false;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) moved |= alpha[nt] != 1.f;
      if (VQ && __any_sync(0xffffffffu, moved)) {  // this lane's columns are its own heads 4 nt + t
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int mt = 0; mt < P::MPQ; ++mt)
#pragma unroll
            for (int e = 0; e < 4; ++e) accq[nt][mt][e] *= alpha[nt];
      } else if (!VQ && __any_sync(0xffffffffu, moved)) {
        float al[2];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int h = 2 * t + c;  // held by lanes t' = h % 4 in n-tile h / 4
          float x = __shfl_sync(0xffffffffu, alpha[0], h & 3);
          if constexpr (NT > 1) {
            const float y = __shfl_sync(0xffffffffu, alpha[NT - 1], h & 3);
            x = h >= 4 ? y : x;
          }
          al[c] = x;
        }
#pragma unroll
        for (int mt = 0; mt < MTV; ++mt) {
          acc[mt][0] *= al[0]; acc[mt][1] *= al[1];
          acc[mt][2] *= al[0]; acc[mt][3] *= al[1];
        }
      }

      if constexpr (VQ) {
        // ---- O^T += V^T P^T per 8 tokens: lane (g, t) takes tokens t and t + 4 of the step (A columns 2 t, 2 t + 1
        // and 2 t + 8, 2 t + 9) and pairs D/16 g + 2 mt (A row g) and + 1 (row g + 8) of m-tile mt
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
          for (int ks = 0; ks < 2; ++ks) {
            const int ta = 16 * m + 8 * ks + t;  // the step's token t; token t + 4 is ta + 4
            uint32_t b0[NT], b1[NT];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              // weights of tokens ta, ta + 4 for head 4 nt + g / 2: held by lanes (t, g / 2) and (t + 4, g / 2) as
              // their token 16 m + g' + 8 ks
              const float w = z[m][nt][ks] * vn[m][ks];
              const float xa = __shfl_sync(0xffffffffu, w, 4 * t + (g >> 1));
              const float xb = __shfl_sync(0xffffffffu, w, 4 * (t + 4) + (g >> 1));
              b0[nt] = (g & 1) ? pack_h2(0.f, xa) : pack_h2(xa, 0.f);
              b1[nt] = (g & 1) ? pack_h2(0.f, xb) : pack_h2(xb, 0.f);
            }
            uint32_t wa[P::NWV], wb[P::NWV];
            load_run<R, P::NBV, false>(st, ta * R + g * P::NBV, wa);
            load_run<R, P::NBV, false>(st, (ta + 4) * R + g * P::NBV, wb);
#pragma unroll
            for (int x = (P::NBV + 3) / 4; x < P::NWV; ++x) wa[x] = wb[x] = 0u;
#pragma unroll
            for (int mt = 0; mt < P::MPQ; ++mt) {
              const uint32_t a0 = *reinterpret_cast<const uint32_t*>(tab + kv_off<BITS>(wa, 2 * mt, repv));
              const uint32_t a1 = *reinterpret_cast<const uint32_t*>(tab + kv_off<BITS>(wa, 2 * mt + 1, repv));
              const uint32_t a2 = *reinterpret_cast<const uint32_t*>(tab + kv_off<BITS>(wb, 2 * mt, repv));
              const uint32_t a3 = *reinterpret_cast<const uint32_t*>(tab + kv_off<BITS>(wb, 2 * mt + 1, repv));
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) mma16816(accq[nt][mt], a0, a1, a2, a3, b0[nt], b1[nt]);
            }
          }
      } else {
      // ---- O^T += V^T P^T per 16-token group: B = P^T (tokens 2 t, 2 t + 1 | + 8, + 9; head g)
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        float pv[2][2];  // [b register][token of the pair]
#pragma unroll
        for (int e = 0; e < 2; ++e)
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int src = 4 * (2 * t + u) + (g & 3);  // the lane holding token 2 t + u (+ 8 e) of head g % 4 (+ 4)
            float x = __shfl_sync(0xffffffffu, z[m][0][e], src);
            if constexpr (NT > 1) {
              const float y = __shfl_sync(0xffffffffu, z[m][NT - 1][e], src);
              x = g >= 4 ? y : x;
            } else {
              x = g < G ? x : 0.f;
            }
            pv[e][u] = x;
          }
        uint32_t bh0, bl0, bh1, bl1;
        split_h2(pv[0][0], pv[0][1], bh0, bl0);
        split_h2(pv[1][0], pv[1][1], bh1, bl1);
#pragma unroll
        for (int mt = 0; mt < MTV; ++mt) {
          uint32_t va[4];
          ldsm_x4_t(sV + swz<TW>(16 * m + a_row, 16 * mt + a_col), va[0], va[1], va[2], va[3]);
          mma16816(acc[mt], va[0], va[1], va[2], va[3], bh0, bh1);
          mma16816(acc[mt], va[0], va[1], va[2], va[3], bl0, bl1);
        }
      }
      }

      // the stage is free once every lane's reads (and zeroing writes) of it are done: each lane orders its own
      // accesses before the async proxy's, then the warp syncs, then lane 0 refills it with tile i + NS
      fence_proxy_async();
      __syncwarp();
      if (i + NS < ntiles) issue(i + NS);
    }
    if (failed) break;
    seq += static_cast<uint32_t>(ntiles);

    // ---- the item's partials
    const size_t part0 = (static_cast<size_t>(b) * a.Hq + hk * G) * a.splits + split;  // head h adds h * splits
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float l = l_lane[nt];
#pragma unroll
      for (int msk = 4; msk < 32; msk <<= 1) l += __shfl_xor_sync(0xffffffffu, l, msk);
      const int h = 4 * nt + t;
      if (g == 0 && h < G) {
        a.ws_m[part0 + static_cast<size_t>(h) * a.splits] = m_run[nt];
        a.ws_l[part0 + static_cast<size_t>(h) * a.splits] = l;
      }
    }
    if constexpr (VQ) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int h = 4 * nt + t;
        if (h < G) {
          float* dst = a.ws_o + (part0 + static_cast<size_t>(h) * a.splits) * D + (D / 8) * g;
#pragma unroll
          for (int mt = 0; mt < P::MPQ; ++mt)
            *reinterpret_cast<float4*>(dst + 4 * mt) =
                make_float4(accq[nt][mt][0], accq[nt][mt][1], accq[nt][mt][2], accq[nt][mt][3]);
        }
      }
    } else {
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int h = 2 * t + c;
        if (h < G) {
          float* dst = a.ws_o + (part0 + static_cast<size_t>(h) * a.splits) * D;
#pragma unroll
          for (int mt = 0; mt < MTV; ++mt) {
            dst[16 * mt + g] = acc[mt][c];
            dst[16 * mt + g + 8] = acc[mt][2 + c];
          }
        }
      }
    }
    __syncwarp();  // every lane is done with this item's ring before the next item's scratch writes
  }

  if (failed) {
    // poison every partial this warp owns (the merge then yields NaN) and record the failure in the status word
    for (int item = first; item < items; item += workers) {
      const int split = item % a.splits;
      const int hk = (item / a.splits) % a.Hkv;
      const int b = item / (a.splits * a.Hkv);
      if (lane < G) a.ws_m[(static_cast<size_t>(b) * a.Hq + hk * G + lane) * a.splits + split] =
          __int_as_float(0x7fc00000);
    }
    if (lane == 0 && a.status) atomicOr(a.status, 1u);
  }
}

}  // namespace axr
