// Candidate attention of the sign selector on the tensor cores (mma.sync.m16n8k16, fp16 operands, fp32 accumulation).
//
// The objective (AXELRAM Key Points, 4th item; Abstract) is the MSE of quantized-K attention against fp64 unquantized
// attention, so every candidate needs a full causal attention over the calibration set: a dense contraction, and the
// selector's whole cost.  Its products must be accurate well beyond fp16 (the MSE differences between sign patterns
// are small), so both factors of each product are split into hi and lo fp16 planes:
//   S = Q K^T  as  Qhi Khi^T + Qhi Klo^T + Qlo Khi^T   (the lo x lo term is below 2^-22 of the product),
//   O = P V    as  Phi V + Plo V                        (the values are fp16 inputs, exact),
// with fp32 accumulation, the online softmax in fp32 (FA2 order: rows held by quads of lanes) and the squared error
// against the fp64 reference summed in fp64.
//
// Block: 4 warps, 16 query rows each (64 rows); key tiles of 32, double-buffered: the cp.async copies of tile k + 1
// are in flight while tile k is computed.  Q (hi, lo), K^ (hi, lo) and V tiles sit in shared memory with rows padded
// by 16 bytes, so the ldmatrix reads of 8 rows fall in 8 different 16-byte bank groups.
#pragma once

#include "axr_common.cuh"
#include "warp_mma.cuh"

namespace axr {

template <int D>
struct SelTcPlan {
  static constexpr int BQ = 64, BK = 32, WARPS = 4, THREADS = 32 * WARPS;
  static constexpr int RS = D * 2 + 16;                // padded row stride in bytes (fp16 rows)
  static constexpr size_t QTILE = (size_t)BQ * RS;     // the 64-row query tile (one plane)
  static constexpr size_t KTILE = (size_t)BK * RS;     // a 32-row key or value tile (one plane)
  static constexpr size_t STAGE = 3 * KTILE;           // K^ hi, K^ lo, V
  static constexpr size_t OFF_QH = 0, OFF_QL = QTILE, OFF_ST = 2 * QTILE;  // [2] stages follow the queries
  static constexpr size_t bytes = 2 * QTILE + 2 * STAGE;
  static constexpr int KT = D / 16;                    // k-tiles of the score MMA
  static constexpr int NO = D / 8;                     // n-tiles of the output
  static constexpr int NS = BK / 8;                    // n-tiles of the scores (keys)
};

// One block: query rows [q0, q0 + 64) of head h of (layer, sequence) ls for candidate ci of the chunk.
//   q     [Ly, S, Hq, N, D] f32;  kh, kl [chunk][Ly, S, Hkv, N, D] fp16 hi / lo planes of the reconstructed keys;
//   v     [Ly, S, Hkv, N, D] fp16;  oref [Ly, S, Hq, N, D] f64;  acc [C, Ly, S] f64 squared-error sums.
template <int D>
__global__ void __launch_bounds__(128, 2)
select_attn_tc_kernel(const float* __restrict__ q, const __half* __restrict__ kh, const __half* __restrict__ kl,
                      const __half* __restrict__ v, const double* __restrict__ oref, double* __restrict__ acc,
                      int Ly, int S, int Hq, int Hkv, int N, int c0, int causal) {
  using P = SelTcPlan<D>;
  constexpr int BQ = P::BQ, BK = P::BK, RS = P::RS, KT = P::KT, NO = P::NO;
  static_assert(BK % 16 == 0, "key tiles of whole 16-key MMA steps");
  extern __shared__ __align__(16) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int q0 = blockIdx.x * BQ, h = blockIdx.y;
  const int ls = blockIdx.z % (Ly * S);
  const int ci = blockIdx.z / (Ly * S);
  const int G = Hq / Hkv, hk = h / G;
  const size_t qrow0 = (static_cast<size_t>(ls) * Hq + h) * N;
  const size_t krow0 = (static_cast<size_t>(ls) * Hkv + hk) * N;
  const size_t kcand = static_cast<size_t>(ci) * Ly * S * Hkv * N;
  const float scale_log2 = rsqrtf(static_cast<float>(D)) * 1.4426950408889634f;

  // ---- the Q tile, split into hi / lo fp16 rows (rows past N are zero)
  for (int e = tid; e < BQ * D / 2; e += P::THREADS) {
    const int r = e / (D / 2), c2 = e % (D / 2);
    float x0 = 0.f, x1 = 0.f;
    if (q0 + r < N) {
      const float2 x = *reinterpret_cast<const float2*>(q + (qrow0 + q0 + r) * D + 2 * c2);
      x0 = x.x; x1 = x.y;
    }
    uint32_t hi, lo;
    split_h2(x0, x1, hi, lo);
    *reinterpret_cast<uint32_t*>(smem + P::OFF_QH + r * RS + 4 * c2) = hi;
    *reinterpret_cast<uint32_t*>(smem + P::OFF_QL + r * RS + 4 * c2) = lo;
  }

  // ldmatrix lane addresses: A fragments (rows 16 w + (lane % 16), column half lane / 16), B fragments of the keys
  // (key rows 8 (lane / 16) + (lane % 8), column half (lane / 8) % 2), B fragments of V (.trans: key rows
  // 8 ((lane / 8) % 2) + lane % 8, coordinate half lane / 16)
  const int a_row = 16 * warp + (lane & 15), a_col = (lane >> 4) * 8;
  const int b_row = 8 * (lane >> 4) + (lane & 7), b_col = ((lane >> 3) & 1) * 8;
  const int v_row = 8 * ((lane >> 3) & 1) + (lane & 7), v_col = (lane >> 4) * 8;
  const uint32_t sQH = smem_addr(smem + P::OFF_QH), sQL = smem_addr(smem + P::OFF_QL);

  float o[NO][4];
#pragma unroll
  for (int n = 0; n < NO; ++n)
#pragma unroll
    for (int i = 0; i < 4; ++i) o[n][i] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};  // rows g and g + 8 of the warp
  const int row_lo = q0 + 16 * warp + g, row_hi = row_lo + 8;

  const int kend = causal ? min(N, q0 + BQ) : N;
  const int ntiles = (kend + BK - 1) / BK;
  // cp.async copies of key tile `kt` (rows past N zero-filled) into stage kt % 2; one commit group per tile
  auto issue = [&](int kt) {
    if (kt < ntiles) {
      uint8_t* st = smem + P::OFF_ST + static_cast<size_t>(kt & 1) * P::STAGE;
      for (int e = tid; e < BK * D / 8; e += P::THREADS) {
        const int r = e / (D / 8), c8 = e % (D / 8);
        const int row = min(kt * BK + r, N - 1);
        const int nb = kt * BK + r < N ? 16 : 0;
        const size_t off = (krow0 + row) * D + 8 * c8;
        cp16(st + r * RS + 16 * c8, kh + kcand * D + off, nb);
        cp16(st + P::KTILE + r * RS + 16 * c8, kl + kcand * D + off, nb);
        cp16(st + 2 * P::KTILE + r * RS + 16 * c8, v + off, nb);
      }
    }
    asm volatile("cp.async.commit_group;\n" ::);
  };
  issue(0);
  for (int kt = 0; kt < ntiles; ++kt) {
    const int k0 = kt * BK;
    issue(kt + 1);
    asm volatile("cp.async.wait_group 1;\n" ::);  // tile kt has landed (tile kt + 1 may be in flight)
    __syncthreads();  // ... for every thread's copies; and, the first time, the Q tile is written
    const uint32_t sKH = smem_addr(smem + P::OFF_ST + static_cast<size_t>(kt & 1) * P::STAGE);
    const uint32_t sKL = sKH + P::KTILE, sV = sKH + 2 * P::KTILE;

    // ---- S = Q K^T for the warp's 16 rows x 32 keys (4 n-tiles), three products per step
    float s[P::NS][4];
#pragma unroll
    for (int n = 0; n < P::NS; ++n)
#pragma unroll
      for (int i = 0; i < 4; ++i) s[n][i] = 0.f;
#pragma unroll
    for (int kk = 0; kk < KT; ++kk) {
      uint32_t ah[4], al[4];
      const uint32_t aoff = a_row * RS + (16 * kk + a_col) * 2;
      ldsm_x4(sQH + aoff, ah[0], ah[1], ah[2], ah[3]);
      ldsm_x4(sQL + aoff, al[0], al[1], al[2], al[3]);
#pragma unroll
      for (int np = 0; np < P::NS / 2; ++np) {  // pairs of n-tiles (16 keys)
        uint32_t bh[4], bl[4];
        const uint32_t boff = (16 * np + b_row) * RS + (16 * kk + b_col) * 2;
        ldsm_x4(sKH + boff, bh[0], bh[1], bh[2], bh[3]);
        ldsm_x4(sKL + boff, bl[0], bl[1], bl[2], bl[3]);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          float (&c)[4] = s[2 * np + j];
          mma16816(c, ah[0], ah[1], ah[2], ah[3], bh[2 * j], bh[2 * j + 1]);
          mma16816(c, ah[0], ah[1], ah[2], ah[3], bl[2 * j], bl[2 * j + 1]);
          mma16816(c, al[0], al[1], al[2], al[3], bh[2 * j], bh[2 * j + 1]);
        }
      }
    }

    // ---- online softmax (log2 units): lane (g, t) holds rows g, g + 8, keys 8 n + 2 t + {0, 1}
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int n = 0; n < P::NS; ++n)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int key = k0 + 8 * n + 2 * t + (i & 1);
        const int row = (i < 2) ? row_lo : row_hi;
        const bool valid = key < N && (!causal || key <= row);
        s[n][i] = valid ? s[n][i] * scale_log2 : -INFINITY;
        mx[i >> 1] = fmaxf(mx[i >> 1], s[n][i]);
      }
    float alpha[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
      const float m_new = fmaxf(m_run[r], mx[r]);
      alpha[r] = (m_run[r] == -INFINITY) ? 0.f : exp2f(m_run[r] - m_new);
      m_run[r] = m_new;
    }
    float rs[2] = {0.f, 0.f};
#pragma unroll
    for (int n = 0; n < P::NS; ++n)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float mm = m_run[i >> 1];
        const float p = (s[n][i] == -INFINITY) ? 0.f : exp2f(s[n][i] - mm);
        s[n][i] = p;
        rs[i >> 1] += p;
      }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      rs[r] += __shfl_xor_sync(0xffffffffu, rs[r], 1);
      rs[r] += __shfl_xor_sync(0xffffffffu, rs[r], 2);
      l_run[r] = l_run[r] * alpha[r] + rs[r];
    }
#pragma unroll
    for (int n = 0; n < NO; ++n) {
      o[n][0] *= alpha[0]; o[n][1] *= alpha[0]; o[n][2] *= alpha[1]; o[n][3] *= alpha[1];
    }

    // ---- O += P V: P from the score accumulators (keys 16 kq + {0..15}), split hi / lo; V by ldmatrix.trans
#pragma unroll
    for (int kq = 0; kq < BK / 16; ++kq) {
      uint32_t ph[4], pl[4];
      split_h2(s[2 * kq][0], s[2 * kq][1], ph[0], pl[0]);
      split_h2(s[2 * kq][2], s[2 * kq][3], ph[1], pl[1]);
      split_h2(s[2 * kq + 1][0], s[2 * kq + 1][1], ph[2], pl[2]);
      split_h2(s[2 * kq + 1][2], s[2 * kq + 1][3], ph[3], pl[3]);
#pragma unroll
      for (int np = 0; np < NO / 2; ++np) {  // pairs of output n-tiles (16 coordinates)
        uint32_t b[4];
        ldsm_x4_t(sV + (16 * kq + v_row) * RS + (16 * np + v_col) * 2, b[0], b[1], b[2], b[3]);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          mma16816(o[2 * np + j], ph[0], ph[1], ph[2], ph[3], b[2 * j], b[2 * j + 1]);
          mma16816(o[2 * np + j], pl[0], pl[1], pl[2], pl[3], b[2 * j], b[2 * j + 1]);
        }
      }
    }
    __syncthreads();  // every warp is done with this stage before tile kt + 2 is copied into it
  }
  asm volatile("cp.async.wait_group 0;\n" ::);

  // ---- squared error against the fp64 reference: lane (g, t) holds rows g, g + 8, coordinates 8 n + 2 t + {0, 1}
  double err = 0.0;
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int row = r == 0 ? row_lo : row_hi;
    if (row < N) {
      const float inv = l_run[r] > 0.f ? 1.f / l_run[r] : 0.f;
      const double* ref = oref + (qrow0 + row) * D;
#pragma unroll
      for (int n = 0; n < NO; ++n)
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const double dlt = static_cast<double>(o[n][2 * r + i] * inv) - ref[8 * n + 2 * t + i];
          err += dlt * dlt;
        }
    }
  }
#pragma unroll
  for (int msk = 16; msk > 0; msk >>= 1) err += __shfl_xor_sync(0xffffffffu, err, msk);
  __syncthreads();
  double* werr = reinterpret_cast<double*>(smem);
  if (lane == 0) werr[warp] = err;
  __syncthreads();
  if (tid == 0) atomicAdd(acc + static_cast<size_t>(c0 + ci) * Ly * S + ls, (werr[0] + werr[1]) + (werr[2] + werr[3]));
}

}  // namespace axr
