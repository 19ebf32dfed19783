// Decode attention over a quantized key cache, one warp carrying its tokens through the whole chain: key scores,
// online softmax and the value product, all as warp-level MMAs, with no block barrier inside an item.
//
// AXELRAM Key Points (1st, 2nd items): every token's score is the gather-sum of q~_j c_k at its stored indices times
// its stored norm, read from the factored pair table through mma.sync (mma_score.cuh: hi/lo fp16 operands, fp32
// accumulation); the softmax and the value product follow the standard split-T formulation, and with quantized
// values the product stays in the rotated domain (one inverse transform per output, in the merge kernel).
//
// Block structure: one block of NW warps per SM, persistent over (batch, KV head, split) items.  Tiles of 128 tokens
// (codes, values and norms: one bulk copy each, completing on the stage's mbarrier) stream through NS stages; warp w
// takes the two 16-token groups [32 (w % 4), 32 (w % 4) + 32) of every (NW / 4)-th tile.  Per visit the warp scores its
// 32 tokens (lane (g, t) holds head t's scores of tokens g and g + 8 of each group), updates its own running max and
// sum, moves the weights p n^V / sqrt(d) into the B-operand layout of the value MMA with warp shuffles (heads as
// columns, token pairs along K) and accumulates O^T (d x heads) += V^T P^T, the A operand (V^T) coming from the same
// pair table (hi fp16 copies) with two byte permutes per register.  The last of the four warps to leave a stage
// refills it with the tile NS ahead.  At the end of an item the NW partial (max, sum, O) triples are merged in shared
// memory and written as the item's split partial.
#pragma once

#include "mma_score.cuh"

namespace axr {

template <int D, int BITS, int G, bool VQ>
struct FusedPlan {
  static constexpr int TT = 128;                         // tokens per tile
  static constexpr int MPW = 2;                          // 16-token groups per warp per visit
  static constexpr int WPT = TT / (16 * MPW);            // warps sharing one tile
  static constexpr int NW = G <= 4 ? 16 : 8;             // warps per block (G = 8 needs more registers)
  static constexpr int THREADS = 32 * NW;
  static constexpr int NG = NW / WPT;                    // tiles in work at once
  static constexpr int R = D * BITS / 8;
  static constexpr int VROW = VQ ? R : 2 * D;
  static constexpr int STAGE_K = TT * R;
  static constexpr int STAGE_V = TT * VROW;
  static constexpr int STAGE_N = 2 * TT * 2;             // key norms, then value norms (fp16)
  static constexpr int STAGE = STAGE_K + STAGE_V + STAGE_N;
  static constexpr int MT = D / 16;                      // value m-tiles (16 coordinates each)
  static constexpr size_t TAB = (size_t)PairTableKV<BITS>::BYTES;
  static constexpr size_t REGION = (size_t)NW * G * D * 4;  // O partials at the end of an item; row factors at its start
  static constexpr size_t QB = (size_t)G * D * 4;        // one item's raw queries
  static constexpr size_t BS = (size_t)MmaB<D, G>::NT * MmaB<D, G>::KT * 2 * 32 * 4;  // staged B fragments
  static constexpr size_t SMALL = 2 * (size_t)NW * G * 4 + 16 * 4 + 16 * 4 + 16 * 4 + 18 * 8 + 16 + 2 * QB + BS + D + 64;
  static constexpr size_t kBudget = 227 * 1024;
  static constexpr int NS_FIT = static_cast<int>((kBudget - TAB - REGION - SMALL - 256) / STAGE);
  static constexpr int NS = NS_FIT > 8 ? 8 : NS_FIT;     // stages
  static constexpr size_t OFF_STAGE = 0;
  static constexpr size_t OFF_TAB = (size_t)NS * STAGE;
  static constexpr size_t OFF_REGION = OFF_TAB + TAB;
  static constexpr size_t OFF_RM = OFF_REGION + REGION;  // [NW][G] running max per warp
  static constexpr size_t OFF_RL = OFF_RM + (size_t)NW * G * 4;  // [NW][G] running sum per warp
  static constexpr size_t OFF_CENT = OFF_RL + (size_t)NW * G * 4;
  static constexpr size_t OFF_CNT = OFF_CENT + 16 * 4;   // [NS] warps done with the stage's tile
  static constexpr size_t OFF_ARM = OFF_CNT + 16 * 4;    // [NS] the tile (block-wide sequence number) last issued
  static constexpr size_t OFF_QB = (OFF_ARM + 16 * 4 + 15) / 16 * 16;  // [2][G][D] raw queries, double-buffered
  static constexpr size_t OFF_BS = OFF_QB + 2 * QB;      // [NT KT 2][32] B fragments of the item
  static constexpr size_t OFF_SCL = OFF_BS + BS;         // [G] head scales (16 slots)
  static constexpr size_t OFF_SGN = OFF_SCL + 16 * 4;    // [D] sign vector
  static constexpr size_t OFF_MB = (OFF_SGN + D + 15) / 16 * 16;  // [16] stage barriers, [2] query barriers, flag
  static constexpr size_t bytes = OFF_MB + 18 * 8 + 8;
  static_assert(NS >= 2, "at least two stages");
  static_assert(bytes <= kBudget, "shared memory of one block");
  static_assert(R % 16 == 0 && VROW % 16 == 0, "rows of whole 16-byte chunks (bulk copies)");
  static_assert(REGION >= (size_t)G * D * 4, "row factors fit the merge region");
};

template <int D, int BITS, int G, bool VQ>
__global__ void __launch_bounds__(FusedPlan<D, BITS, G, VQ>::THREADS, 1)
attend_fused_kernel(const __grid_constant__ DecodeArgs a) {
  using P = FusedPlan<D, BITS, G, VQ>;
  constexpr int TT = P::TT, NW = P::NW, WPT = P::WPT, NG = P::NG, NS = P::NS, MT = P::MT, MPW = P::MPW;
  constexpr int R = P::R, VROW = P::VROW;
  constexpr int NT = MmaB<D, G>::NT;
  extern __shared__ __align__(16) uint8_t smem[];
  const uint8_t* tab = smem + P::OFF_TAB;
  float* region = reinterpret_cast<float*>(smem + P::OFF_REGION);
  float* qs = region;  // [G][D] row factors while an item starts
  float* red_m = reinterpret_cast<float*>(smem + P::OFF_RM);
  float* red_l = reinterpret_cast<float*>(smem + P::OFF_RL);
  float* cent = reinterpret_cast<float*>(smem + P::OFF_CENT);
  int* cnt = reinterpret_cast<int*>(smem + P::OFF_CNT);
  volatile int* armed = reinterpret_cast<volatile int*>(smem + P::OFF_ARM);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + P::OFF_MB);
  uint64_t* qfull = full + 16;  // [2]: the queries of the block's k-th item land in buffer k % 2
  volatile int* failed = reinterpret_cast<volatile int*>(full + 18);
  float* qbuf = reinterpret_cast<float*>(smem + P::OFF_QB);
  uint32_t* bs = reinterpret_cast<uint32_t*>(smem + P::OFF_BS);
  float* sclv = reinterpret_cast<float*>(smem + P::OFF_SCL);
  int8_t* sgn = reinterpret_cast<int8_t*>(smem + P::OFF_SGN);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;  // fragment coordinates: row group and column pair of the MMAs
  const uint32_t repk = static_cast<uint32_t>(lane & 15) << 3;      // the lane's hi/lo copy in the pair table
  const uint32_t repv = 128u + (static_cast<uint32_t>(lane) << 2);  // its hi-only copy
  const float rd = rsqrtf(static_cast<float>(D));
  const int tf = t & 1;  // value rows are fetched k + 1 before k on odd t (no bank conflicts)
  // position of coordinate c of head h in a warp's row of the merge region: the C fragments put coordinates
  // 2 (MT g + mt) + {0, 1} of heads 2t + {0, 1} in lane (g, t); XOR-ing in g and t spreads a store's 32 lanes over
  // 32 banks (the plain layout puts them on two)
  constexpr int GS = D == 128 ? 4 : 3;  // log2 of the coordinates per row group g
  auto rswz = [](int h, int c) { return c ^ ((c >> GS) & 7) ^ (((h >> 1) & 3) << 3); };
  const uint32_t sel_lo = tf ? 0x1054u : 0x5410u, sel_hi = tf ? 0x3276u : 0x7632u;

  if (tid < 16) cent[tid] = a.cb.gamma[tid];
  for (int j = tid; j < D; j += P::THREADS) sgn[j] = a.signs[j];
  if (tid < NS) {
    cnt[tid] = 0;
    armed[tid] = -1;
  }
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) tc::mbar_init(full + s, 1);
    tc::mbar_init(qfull, 1);
    tc::mbar_init(qfull + 1, 1);
    *failed = 0;
  }
  __syncthreads();
  build_pair_table_kv<BITS>(cent, smem + P::OFF_TAB);
  // tile t of an item is tile done + t of the block: it uses stage (done + t) % NS and that barrier's phase of parity
  // ((done + t) / NS) & 1.  The warp groups take different tiles, so one group can reach a stage two fills ahead of
  // another; a group therefore first waits until the stage is armed with its own tile (armed[s] == done + t), and
  // only then on the barrier's parity.
  int done = 0;

  const int items = a.B * a.Hkv * a.splits;
  struct Geo {  // one item: (batch row, KV head, split) and its token range
    int b, hk, split, start, end, ntiles;
    size_t kv_row0;
    bool nrm_bulk;
  };
  auto geo = [&](int item) {
    Geo q;
    q.split = item % a.splits;
    q.hk = (item / a.splits) % a.Hkv;
    q.b = item / (a.splits * a.Hkv);
    q.start = q.split * a.chunk;
    q.end = min(q.start + a.chunk, row_len(a, q.b));
    q.ntiles = q.end > q.start ? (q.end - q.start + TT - 1) / TT : 0;
    q.kv_row0 = (static_cast<size_t>(q.b) * a.Hkv + q.hk) * a.Tcap;
    // norms travel with the tile when every norm row is whole 16-byte chunks (the last tile's copy then stays
    // inside the row), else the lanes read them from global memory
    q.nrm_bulk = (a.Tcap % 8) == 0 &&
                 (reinterpret_cast<uintptr_t>(a.knorms + q.kv_row0 + q.start) & 15) == 0 &&
                 (!VQ || (reinterpret_cast<uintptr_t>(a.vnorms + q.kv_row0 + q.start) & 15) == 0);
    return q;
  };
  // lanes 0..3 of one warp: tile `tile` (block sequence number seq0 + tile) of item x -- codes, values and the two
  // norm rows, one bulk copy per lane -- into its stage; the caller's other lanes pass lane >= 4
  auto issue = [&](const Geo& x, int seq0, int tile, int ln) {
    const int s = (seq0 + tile) % NS;
    uint8_t* st = smem + P::OFF_STAGE + static_cast<size_t>(s) * P::STAGE;
    const int t0 = x.start + tile * TT;
    const int n = min(TT, x.end - t0);
    const uint32_t kb = n * R, vb = n * VROW, nb = x.nrm_bulk ? ((n + 7) & ~7) * 2 : 0;
    if (ln == 0) mbar_arrive_expect_tx(full + s, kb + vb + (VQ ? 2 : 1) * nb);
    __syncwarp(0xfu);
    if (ln == 0) bulk_copy_g2s(st, a.kcodes + (x.kv_row0 + t0) * R, kb, full + s);
    else if (ln == 1) bulk_copy_g2s(st + P::STAGE_K, static_cast<const uint8_t*>(a.v) + (x.kv_row0 + t0) * VROW, vb, full + s);
    else if (ln == 2 && nb) bulk_copy_g2s(st + P::STAGE_K + P::STAGE_V, a.knorms + x.kv_row0 + t0, nb, full + s);
    else if (ln == 3 && VQ && nb)
      bulk_copy_g2s(st + P::STAGE_K + P::STAGE_V + 2 * TT, a.vnorms + x.kv_row0 + t0, nb, full + s);
    if (ln == 0) {
      __threadfence_block();  // the stage's reset counter is visible before the stage reads as armed
      armed[s] = seq0 + tile;
    }
  };
  // every thread: the block's k-th item's queries (lane 0 of the last warp) and first tiles (warp w < NS takes tile w)
  auto start_item = [&](int item, int k, int seq0) {
    const Geo x = geo(item);
    if (warp < NS && warp < x.ntiles && lane < 4) issue(x, seq0, warp, lane);
    if (warp == NW - 1 && lane == 4) {
      const uint32_t qb = static_cast<uint32_t>(P::QB);
      mbar_arrive_expect_tx(qfull + (k & 1), qb);
      bulk_copy_g2s(qbuf + (k & 1) * G * D, a.q + (static_cast<size_t>(x.b) * a.Hq + x.hk * G) * D, qb,
                    qfull + (k & 1));
    }
  };
  if (static_cast<int>(blockIdx.x) < items) start_item(blockIdx.x, 0, 0);

  int k = 0;  // items done by this block
  for (int item = blockIdx.x; item < items; item += gridDim.x, ++k) {
    const Geo x = geo(item);
    const int b = x.b, hk = x.hk, split = x.split, start = x.start, end = x.end, ntiles = x.ntiles;
    const size_t kv_row0 = x.kv_row0;
    const bool nrm_bulk = x.nrm_bulk;
    const __half* kn_src = a.knorms + kv_row0;
    const __half* vn_src = VQ ? a.vnorms + kv_row0 : nullptr;

    __syncthreads();  // the previous item is finished with the region (the row factors go there)
    if (!tc::mbar_wait(qfull + (k & 1), static_cast<uint32_t>((k >> 1) & 1))) *failed = 1;
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
    float m_run[NT], l_lane[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) { m_run[nt] = -INFINITY; l_lane[nt] = 0.f; }
    float acc[MT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[mt][c] = 0.f;

    for (int i = warp / WPT; i < ntiles; i += NG) {
      const int s = (done + i) % NS;
      {
        int polls = 0;  // bounded: about a second at most
        while (armed[s] != done + i && ++polls < (1 << 24)) {
        }
        if (armed[s] != done + i) *failed = 1;
      }
      if (!tc::mbar_wait(full + s, static_cast<uint32_t>(((done + i) / NS) & 1))) *failed = 1;
      const uint8_t* st = smem + P::OFF_STAGE + static_cast<size_t>(s) * P::STAGE;
      const uint8_t* vst = st + P::STAGE_K;
      const __half* nst = reinterpret_cast<const __half*>(st + P::STAGE_K + P::STAGE_V);
      const int t0 = start + i * TT;
      const int nt_tok = min(TT, end - t0);
      const int row_w = (warp % WPT) * 16 * MPW;  // first of this warp's tokens in the tile

      // ---- key scores of the warp's MPW x 16 tokens; lane (g, t) holds tokens g, g + 8 of each group, head 4 nt + t
      float z[MPW][NT][2];
#pragma unroll
      for (int m = 0; m < MPW; ++m) mma_scores16<D, BITS, G, false, true>(st, row_w + 16 * m, tab, repk, B, lane, z[m]);
      float vn[MPW][2];
#pragma unroll
      for (int m = 0; m < MPW; ++m)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int r = row_w + 16 * m + g + 8 * j;
          const bool valid = r < nt_tok;
          float kn = 0.f;
          vn[m][j] = 1.f;
          if (valid) {
            kn = __half2float(nrm_bulk ? nst[r] : kn_src[t0 + r]);
            if constexpr (VQ) vn[m][j] = __half2float(nrm_bulk ? nst[TT + r] : vn_src[t0 + r]);
          }
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
            z[m][nt][j] = valid && 4 * nt + t < G ? z[m][nt][j] * B.inv[nt] * kn * rd : -INFINITY;
        }

      // ---- online softmax over the warp's tokens (per head: lanes with the same t)
      float alpha[NT];
      bool grew = false;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        float mx = -INFINITY;
#pragma unroll
        for (int m = 0; m < MPW; ++m) mx = fmaxf(mx, fmaxf(z[m][nt][0], z[m][nt][1]));
#pragma unroll
        for (int msk = 4; msk < 32; msk <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, msk));
        const float m_new = fmaxf(m_run[nt], mx);
        alpha[nt] = (m_new == -INFINITY) ? 1.f : exp2f(m_run[nt] - m_new);
        grew |= m_new != m_run[nt];
        float psum = 0.f;
#pragma unroll
        for (int m = 0; m < MPW; ++m)
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const float p = (z[m][nt][j] == -INFINITY) ? 0.f : exp2f(z[m][nt][j] - m_new);
            psum += p;
            z[m][nt][j] = p > 0.f ? p * (VQ ? vn[m][j] * rd : 1.f) : 0.f;  // the value product's weight
          }
        l_lane[nt] = l_lane[nt] * alpha[nt] + psum;
        m_run[nt] = m_new;
      }
      // rescale the accumulators (columns 2t, 2t + 1 are heads 2t, 2t + 1) when a running max moved
      if (__any_sync(0xffffffffu, grew)) {
        float al[2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int h = 2 * t + hh;
          const int src = (lane & ~3) | (h & 3);
          float x = __shfl_sync(0xffffffffu, alpha[0], src);
          if constexpr (NT == 2) {
            const float y = __shfl_sync(0xffffffffu, alpha[NT - 1], src);
            x = h >= 4 ? y : x;
          }
          al[hh] = x;
        }
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          acc[mt][0] *= al[0]; acc[mt][1] *= al[1]; acc[mt][2] *= al[0]; acc[mt][3] *= al[1];
        }
      }

      // ---- value product: for each M tile of keys, one K = 16 step of O^T += V^T P^T
#pragma unroll
      for (int m = 0; m < MPW; ++m) {
        const int base = row_w + 16 * m;
        if (base >= nt_tok) break;
        // B operand: weights of tokens base + 2t, + 1 and base + 2t + 8, + 9 for head g (lane (g', t') holds tokens
        // g' and g' + 8 of head 4 nt + t')
        const int s0 = 8 * t + (g & 3), s1 = s0 + 4;
        float w00 = __shfl_sync(0xffffffffu, z[m][0][0], s0), w01 = __shfl_sync(0xffffffffu, z[m][0][0], s1);
        float w10 = __shfl_sync(0xffffffffu, z[m][0][1], s0), w11 = __shfl_sync(0xffffffffu, z[m][0][1], s1);
        if constexpr (NT == 2) {
          const float y00 = __shfl_sync(0xffffffffu, z[m][NT - 1][0], s0);
          const float y01 = __shfl_sync(0xffffffffu, z[m][NT - 1][0], s1);
          const float y10 = __shfl_sync(0xffffffffu, z[m][NT - 1][1], s0);
          const float y11 = __shfl_sync(0xffffffffu, z[m][NT - 1][1], s1);
          if (g >= 4) { w00 = y00; w01 = y01; w10 = y10; w11 = y11; }
        }
        uint32_t b0 = 0u, b1 = 0u;
        if (g < G) {
          const __half2 h0 = __floats2half2_rn(w00, w01), h1 = __floats2half2_rn(w10, w11);
          b0 = *reinterpret_cast<const uint32_t*>(&h0);
          b1 = *reinterpret_cast<const uint32_t*>(&h1);
        }
        // A operand: lane g's coordinate pairs MT g .. MT g + MT - 1 of tokens k0, k0 + 1, k0 + 8, k0 + 9
        const int k0 = base + 2 * t;
        const int rows[4] = {k0 + tf, k0 + 1 - tf, k0 + 8 + tf, k0 + 9 - tf};
        if constexpr (VQ) {
          constexpr int NBV = R / 8;
          constexpr int NWV = (NBV + 3) / 4 + 1;
          uint32_t w[4][NWV];
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            load_run<R, NBV, false>(vst, rows[r] * R + g * NBV, w[r]);
#pragma unroll
            for (int k = (NBV + 3) / 4; k < NWV; ++k) w[r][k] = 0u;
          }
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            uint32_t x[4];  // hi fp16 pairs (v_2p, v_2p+1) of the four tokens, p = MT g + mt
#pragma unroll
            for (int r = 0; r < 4; ++r) x[r] = *reinterpret_cast<const uint32_t*>(tab + kv_off<BITS>(w[r], mt, repv));
            mma_m16n8k16(acc[mt], __byte_perm(x[0], x[1], sel_lo), __byte_perm(x[0], x[1], sel_hi),
                         __byte_perm(x[2], x[3], sel_lo), __byte_perm(x[2], x[3], sel_hi), b0, b1);
          }
        } else {
          // fp16 values: the pairs (v_2p, v_2p+1) are the row's own half2 words, MT of them per lane
          uint32_t w[4][MT];
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const uint4* src = reinterpret_cast<const uint4*>(vst + rows[r] * VROW + g * MT * 4);
            const bool live = rows[r] < nt_tok;  // rows past the tile's end hold stale bytes, weighted 0 but maybe NaN
#pragma unroll
            for (int q = 0; q < MT / 4; ++q) {
              const uint4 u = live ? src[q] : make_uint4(0u, 0u, 0u, 0u);
              w[r][4 * q] = u.x; w[r][4 * q + 1] = u.y; w[r][4 * q + 2] = u.z; w[r][4 * q + 3] = u.w;
            }
          }
#pragma unroll
          for (int mt = 0; mt < MT; ++mt)
            mma_m16n8k16(acc[mt], __byte_perm(w[0][mt], w[1][mt], sel_lo), __byte_perm(w[0][mt], w[1][mt], sel_hi),
                         __byte_perm(w[2][mt], w[3][mt], sel_lo), __byte_perm(w[2][mt], w[3][mt], sel_hi), b0, b1);
        }
      }

      // ---- leave the stage; the last of its warps refills it with the tile NS ahead
      __syncwarp();
      int last = 0;
      if (lane == 0) {
        last = atomicAdd(cnt + s, 1) == WPT - 1;
        if (last) cnt[s] = 0;
      }
      if (__shfl_sync(0xffffffffu, last, 0) && i + NS < ntiles && lane < 4) {
        fence_proxy_async();
        issue(x, done, i + NS, lane);
      }
    }

    // ---- merge of the NW warps' partials
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float l = l_lane[nt];
#pragma unroll
      for (int msk = 4; msk < 32; msk <<= 1) l += __shfl_xor_sync(0xffffffffu, l, msk);
      const int h = 4 * nt + t;
      if (g == 0 && h < G) {
        red_m[warp * G + h] = m_run[nt];
        red_l[warp * G + h] = l;
      }
    }
    __syncthreads();  // every warp's tiles are done (no copy in flight) and its max and sum are published
    if (item + static_cast<int>(gridDim.x) < items) {
      fence_proxy_async();  // the stages' generic reads come before the next item's bulk copies
      start_item(item + gridDim.x, k + 1, done + ntiles);
    }
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int h = 2 * t + hh;
      if (h < G) {
        float M = red_m[h];
#pragma unroll
        for (int w2 = 1; w2 < NW; ++w2) M = fmaxf(M, red_m[w2 * G + h]);
        const float mw = red_m[warp * G + h];
        const float scl = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
        float* dst = region + (warp * G + h) * D;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          const int c = 2 * (MT * g + mt);  // A rows g and g + 8 of m-tile mt
          dst[rswz(h, c)] = acc[mt][hh] * scl;
          dst[rswz(h, c + 1)] = acc[mt][2 + hh] * scl;
        }
      }
    }
    __syncthreads();  // merge, step 2: every warp's scaled partial is in shared memory (swizzled, rswz)
    const size_t part0 = (static_cast<size_t>(b) * a.Hq + hk * G) * a.splits + split;  // head h adds h * splits
    for (int e = tid; e < G * D; e += P::THREADS) {
      const int h = e / D, jj = e % D;
      float sum = 0.f;
#pragma unroll 4
      for (int w2 = 0; w2 < NW; ++w2) sum += region[(w2 * G + h) * D + rswz(h, jj)];
      a.ws_o[(part0 + static_cast<size_t>(h) * a.splits) * D + jj] = sum;
    }
    if (warp < G) {  // one warp per head: lane w2 < NW takes warp w2's (max, sum)
      const float mw = lane < NW ? red_m[lane * G + warp] : -INFINITY;
      float M = mw;
#pragma unroll
      for (int msk = 16; msk > 0; msk >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, msk));
      const float lw = (mw == -INFINITY) ? 0.f : red_l[lane * G + warp] * exp2f(mw - M);
      const float sum = warp_sum(lw);
      if (lane == 0) {
        a.ws_l[part0 + static_cast<size_t>(warp) * a.splits] = sum;
        // a stage that never arrived (a copy that did not complete in about a second) poisons the output
        a.ws_m[part0 + static_cast<size_t>(warp) * a.splits] = *failed ? __int_as_float(0x7fc00000) : M;
      }
    }
    done += ntiles;
  }
  __syncthreads();
  report_wait_failure(a, failed);
}

}  // namespace axr
