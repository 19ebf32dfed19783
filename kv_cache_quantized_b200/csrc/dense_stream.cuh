// The dense fp16 decode kernel: the bandwidth reference beside the quantized read path.  Same split-T online-softmax
// formulation and partial format as the quantized kernels (merged by attend_reduce_kernel), over an unquantized
// [B, Hkv, Tcap, D] fp16 cache.
//
// Built as a pure stream: every warp is an independent worker over (batch row, KV head, split) items, with a ring of
// NS stages of its own.  A stage holds TW key rows and TW value rows, landed by tiled TMA copies (one box of TW rows
// x 64 coordinates per copy, D / 64 boxes per plane) with the 128-byte swizzle, so the ldmatrix reads of 8 rows fall
// in 8 different 16-byte bank groups, and completes on the stage's mbarrier.  No barrier spans more than one warp,
// so a warp waiting on its copies never holds up another.
//
// The arithmetic is the flash-attention register form on mma.sync.m16n8k16 with the query heads of a KV group as
// the M rows (rows G..15 zero):
//   S[h, t] = q_h . k_t     A = Q (hi and lo fp16 planes of the fp32 query, times scale log2 e), B = K^T (ldmatrix);
//   P = 2^(S - m)           the S accumulators of two 8-token n-tiles are the A fragment of one 16-token k-step;
//   O[h, :] += P V          A = P (hi and lo fp16 planes), B = V (ldmatrix.trans).
// fp32 accumulation; the fp16 cache entries enter the products exactly.
#pragma once

#include <cuda.h>

#include "decode.cuh"
#include "warp_mma.cuh"

namespace axr {

template <int D, int G>
struct DenseStreamPlan {
  static constexpr int TW = 32;                          // tokens per warp tile
  static constexpr int NS = 3;                           // stages per warp
  static constexpr int WARPS = 4;                        // warps per block (one block per SM)
  static constexpr int THREADS = 32 * WARPS;
  static constexpr int ROW = 2 * D;                      // bytes of one fp16 row
  static constexpr int BOXC = 64;                        // coordinates per TMA box (128 bytes: the swizzle span)
  static constexpr int NB = D / BOXC;                    // boxes per row
  static constexpr size_t BOX = (size_t)TW * 128;        // one box in shared memory: TW rows of 128 bytes
  static constexpr size_t PLANE = NB * BOX;              // the K (or V) rows of one stage
  static constexpr size_t STAGE = 2 * PLANE;
  static constexpr size_t WARP_BYTES = NS * STAGE;
  static constexpr size_t OFF_MBAR = WARPS * WARP_BYTES;  // [WARPS][NS] mbarriers, after the 1024-aligned rings
  static constexpr size_t bytes = 1024 + OFF_MBAR + (size_t)WARPS * NS * 8;  // + the alignment slack
  static constexpr int KT = D / 16;                      // k-steps of the score MMA
  static constexpr int NT = TW / 8;                      // 8-token n-tiles of a tile
  static constexpr int NO = D / 8;                       // 8-coordinate n-tiles of the output
  static constexpr uint32_t TX = 2u * TW * ROW;          // bytes that complete one stage
  static_assert(G >= 1 && G <= 8, "the query heads of a group fill rows 0..G-1 of one m16 tile");
  static_assert(TW % 16 == 0 && TW <= 256, "whole 16-token k-steps; a TMA box is at most 256 rows");
  static_assert(D % BOXC == 0 && BOX % 1024 == 0, "whole boxes, each aligned for the 128-byte swizzle");
};

// Tiled TMA load of box (x = first coordinate, y = first cache row) of `map` into shared memory, completing on mbar.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* mbar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n" ::
          "r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(mbar))
      : "memory");
}

// Byte offset, inside a plane, of the 16-byte chunk holding coordinates [col, col + 8) of row r (r < TW): box
// col / 64, row r of it, chunk (col % 64) / 8 swizzled by r % 8 (the 128-byte pattern on a 1024-aligned box).
template <int TW>
__device__ __forceinline__ uint32_t swz(int r, int col) {
  return static_cast<uint32_t>((col >> 6) * TW * 128 + r * 128 + ((((col & 63) >> 3) ^ (r & 7)) << 4));
}

// kmap, vmap: 2-D maps over the fp16 caches viewed as [B Hkv Tcap rows, D coordinates], box TW rows x 64
// coordinates, 128-byte swizzle.
template <int D, int G>
__global__ void __launch_bounds__(DenseStreamPlan<D, G>::THREADS, 1)
dense_stream_kernel(const __grid_constant__ DecodeArgs a, const __grid_constant__ CUtensorMap kmap,
                    const __grid_constant__ CUtensorMap vmap) {
  using P = DenseStreamPlan<D, G>;
  constexpr int TW = P::TW, NS = P::NS, KT = P::KT, NT = P::NT, NO = P::NO;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);  // the swizzle wants 1024-aligned boxes
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  uint8_t* ring = smem + static_cast<size_t>(warp) * P::WARP_BYTES;
  uint64_t* mbar = reinterpret_cast<uint64_t*>(smem + P::OFF_MBAR) + warp * NS;
  if (lane == 0)
    for (int s = 0; s < NS; ++s) tc::mbar_init(mbar + s, 1);
  __syncwarp();

  // ldmatrix lane rows: keys (non-transposed, B of the score MMA) and values (transposed, B of the value MMA)
  const int b_row = 8 * (lane >> 4) + (lane & 7), b_col = ((lane >> 3) & 1) * 8;
  const int v_row = 8 * ((lane >> 3) & 1) + (lane & 7), v_col = (lane >> 4) * 8;
  const __half2 zero2 = __float2half2_rn(0.f);
  const uint32_t zero = *reinterpret_cast<const uint32_t*>(&zero2);

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
    const size_t row0 = (static_cast<size_t>(b) * a.Hkv + hk) * a.Tcap;

    // tile i of the item into stage (seq + i) % NS: the boxes of TW key rows and TW value rows, issued by lane 0
    // (rows past the row's length are cache rows of other positions, or zero past the cache's end: masked below)
    auto issue = [&](int i) {
      if (lane == 0) {
        const int s = static_cast<int>((seq + i) % NS);
        uint8_t* st = ring + static_cast<size_t>(s) * P::STAGE;
        mbar_arrive_expect_tx(mbar + s, P::TX);
        const int y = static_cast<int>(row0) + start + i * TW;
#pragma unroll
        for (int bx = 0; bx < P::NB; ++bx) {
          tma_load_2d(st + bx * P::BOX, &kmap, bx * P::BOXC, y, mbar + s);
          tma_load_2d(st + P::PLANE + bx * P::BOX, &vmap, bx * P::BOXC, y, mbar + s);
        }
      }
    };
    for (int i = 0; i < NS && i < ntiles; ++i) issue(i);

    // the query rows of the group as A fragments (rows g < G; rows g + 8 are zero), hi and lo fp16 planes
    uint32_t qh[KT][2], ql[KT][2];
    {
      const float* qrow = a.q + (static_cast<size_t>(b) * a.Hq + hk * G + (g < G ? g : 0)) * D;
#pragma unroll
      for (int kk = 0; kk < KT; ++kk)
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          float2 x = make_float2(0.f, 0.f);
          if (g < G) x = *reinterpret_cast<const float2*>(qrow + 16 * kk + 8 * half + 2 * t);
          split_h2(x.x * a.mult, x.y * a.mult, qh[kk][half], ql[kk][half]);
        }
    }

    float o[NO][4];
#pragma unroll
    for (int n = 0; n < NO; ++n)
#pragma unroll
      for (int i = 0; i < 4; ++i) o[n][i] = 0.f;
    float m_run = -INFINITY, l_part = 0.f;  // row g: running max (log2 units), this lane's share of the sum

    for (int i = 0; i < ntiles; ++i) {
      const int s = static_cast<int>((seq + i) % NS);
      if (!__all_sync(0xffffffffu, tc::mbar_wait(mbar + s, ((seq + i) / NS) & 1))) {  // warp-uniform decision
        // A wait gave up: stop issuing, let this warp's copies in flight (tiles i .. i + NS - 1) land, bounded
        // again, before the block may exit; the partials are poisoned below.
        failed = true;
        for (int j = i; j < i + NS && j < ntiles; ++j) tc::mbar_wait(mbar + (seq + j) % NS, ((seq + j) / NS) & 1);
        break;
      }
      uint8_t* st = ring + static_cast<size_t>(s) * P::STAGE;
      const uint32_t sK = smem_addr(st), sV = sK + static_cast<uint32_t>(P::PLANE);
      const int t0 = start + i * TW;
      if (t0 + TW > end) {
        // the row ends inside this tile: zero the value rows past it, whatever the cache holds there, so that the
        // zero weights of the masked tokens meet finite values (the key rows' scores are masked to -inf)
        uint4* vz = reinterpret_cast<uint4*>(st + P::PLANE);
        const int r0 = end - t0;
        for (int e = lane; e < (TW - r0) * 8 * P::NB; e += 32) {
          const int bx = e / ((TW - r0) * 8), rem = e % ((TW - r0) * 8);
          vz[(bx * P::BOX + (r0 + rem / 8) * 128) / 16 + rem % 8] = make_uint4(0u, 0u, 0u, 0u);
        }
        __syncwarp();
      }

      // ---- S = Q K^T: 16 rows x TW tokens
      float sc[NT][4];
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) sc[n][e] = 0.f;
#pragma unroll
      for (int kk = 0; kk < KT; ++kk)
#pragma unroll
        for (int np = 0; np < NT / 2; ++np) {
          uint32_t kb[4];
          ldsm_x4(sK + swz<TW>(16 * np + b_row, 16 * kk + b_col), kb[0], kb[1], kb[2], kb[3]);
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            mma16816(sc[2 * np + j], qh[kk][0], zero, qh[kk][1], zero, kb[2 * j], kb[2 * j + 1]);
            mma16816(sc[2 * np + j], ql[kk][0], zero, ql[kk][1], zero, kb[2 * j], kb[2 * j + 1]);
          }
        }

      // ---- online softmax of row g over the tile (lane holds tokens 8 n + 2 t + {0, 1})
      float mx = -INFINITY;
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const bool valid = t0 + 8 * n + 2 * t + e < end;
          sc[n][e] = valid ? sc[n][e] : -INFINITY;
          mx = fmaxf(mx, sc[n][e]);
        }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float m_new = fmaxf(m_run, mx);  // finite: every tile holds at least one valid token
      const float alpha = exp2f(m_run - m_new);
      m_run = m_new;
      float ps = 0.f;
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float p = exp2f(sc[n][e] - m_new);
          sc[n][e] = p;
          ps += p;
        }
      l_part = l_part * alpha + ps;
#pragma unroll
      for (int n = 0; n < NO; ++n) {
        o[n][0] *= alpha;
        o[n][1] *= alpha;
      }

      // ---- O += P V, 16 tokens per k-step
#pragma unroll
      for (int kq = 0; kq < TW / 16; ++kq) {
        uint32_t ph0, pl0, ph2, pl2;
        split_h2(sc[2 * kq][0], sc[2 * kq][1], ph0, pl0);
        split_h2(sc[2 * kq + 1][0], sc[2 * kq + 1][1], ph2, pl2);
#pragma unroll
        for (int np = 0; np < NO / 2; ++np) {
          uint32_t vb[4];
          ldsm_x4_t(sV + swz<TW>(16 * kq + v_row, 16 * np + v_col), vb[0], vb[1], vb[2], vb[3]);
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            mma16816(o[2 * np + j], ph0, zero, ph2, zero, vb[2 * j], vb[2 * j + 1]);
            mma16816(o[2 * np + j], pl0, zero, pl2, zero, vb[2 * j], vb[2 * j + 1]);
          }
        }
      }

      // the stage is free once every lane's reads (and zeroing writes) of it are done: each lane orders its own
      // accesses before the async proxy's, then the warp syncs, then lane 0 refills the stage with tile i + NS
      fence_proxy_async();
      __syncwarp();
      if (i + NS < ntiles) issue(i + NS);
    }
    if (failed) break;
    seq += static_cast<uint32_t>(ntiles);

    // ---- the item's partials: rows g < G (lanes 4 g .. 4 g + 3)
    l_part += __shfl_xor_sync(0xffffffffu, l_part, 1);
    l_part += __shfl_xor_sync(0xffffffffu, l_part, 2);
    if (g < G) {
      const size_t part = (static_cast<size_t>(b) * a.Hq + hk * G + g) * a.splits + split;
      float* dst = a.ws_o + part * D + 2 * t;
#pragma unroll
      for (int n = 0; n < NO; ++n) *reinterpret_cast<float2*>(dst + 8 * n) = make_float2(o[n][0], o[n][1]);
      if (t == 0) {
        a.ws_m[part] = m_run;
        a.ws_l[part] = l_part;
      }
    }
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
