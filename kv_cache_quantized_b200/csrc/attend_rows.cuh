// Decode attention over a quantized key cache with the key scores as warp-level MMAs (values: fp16 rows or rows of
// codes in the keys' layout).
//
// AXELRAM Key Points (1st, 2nd items): every token's score is the gather-sum of q~_j c_k at its stored indices times
// its stored norm; here the table is read in factored form through mma.sync (mma_score.cuh: hi/lo fp16 operands,
// fp32 accumulation).  The softmax and the value product follow the standard split-T formulation; with quantized
// values the product stays in the rotated domain (one inverse transform per output, in the merge kernel).
//
// Block structure (256 threads, persistent over (batch, KV head, split) items): scoring warps 0..3 own tokens
// [32 w, 32 w + 32) of every 128-token tile, score them as two 16-token groups (lane (g, t) gets head t's scores of
// tokens g, g + 8, 16 + g, 24 + g) and keep the running max and sum of their tokens (online softmax); value warp
// 4 + w consumes the same tokens one tile later against the same running max.  One block barrier per tile; the
// streams of the four warps are merged at the end of an item.
//
// Quantized values: the value product is an MMA too, O^T (d x heads) += V^T (d x tokens) P^T (tokens x heads).  The
// A operand (V^T) comes from the same pair table: a lookup of one code byte gives the fp16 pair (v_2p, v_2p+1) of a
// token, and two byte permutes of the pairs of tokens k and k + 1 give the two A registers (coordinate 2p and 2p + 1,
// tokens k, k + 1).  Lane g's A rows are coordinates 2 (d/16 g + mt) and 2 (d/16 g + mt) + 1 of m-tile mt, so one
// load fetches its codes of a token for all m-tiles.  The weights p n^V / sqrt(d) travel as fp16 in the B-operand
// layout (heads x tokens); the hi fp16 plane of the table holds the centroids to 2^-11.  fp16 values keep the packed
// fp32 FMA product (value lanes own 8 coordinates of a row).
#pragma once

#include "append.cuh"
#include "mma_score.cuh"

namespace axr {

template <int D, int BITS, int G, bool VQ>
struct RowsPlan {
  static constexpr int TT = 128;
  static constexpr int KW = 4;                            // scoring warps; value warps follow them
  static constexpr int WT = TT / KW;                      // tokens per scoring warp per tile
  static constexpr int R = D * BITS / 8;
  static constexpr int VROW = VQ ? R : 2 * D;             // bytes per value row
  static constexpr int VCH = (VROW % 16 == 0) ? 16 : 8;
  static constexpr int KCH = (R % 16 == 0) ? 16 : 8;
  static constexpr int STAGE_K = TT * R;
  static constexpr int STAGE_V = TT * VROW;
  static constexpr int STAGE_N = 2 * TT * 2;              // key norms, then value norms (fp16), with the key tile
  static constexpr int NT = MmaB<D, G>::NT;
  static constexpr int TPR = D / 8;                       // fp16 values: value lanes per token row (8 coordinates)
  static constexpr int RPW = kWarp / TPR;                 // fp16 values: value rows per warp step
  static constexpr int NVG = VQ ? KW : KW * RPW;          // value partial sums, summed at the end
  static constexpr int PST = TT + 8;                      // quantized values: weight row stride (halves), padded
  static constexpr size_t PBUF = VQ ? 2 * 8 * (size_t)PST * 2 : 2 * (size_t)TT * G * 8;
  static constexpr size_t TAB = (size_t)PairTableKV<BITS>::BYTES;
  // everything but the stages
  static constexpr size_t FIXED = TAB + PBUF + 2 * 8 * 8 + 8 + 2 * (size_t)KW * G * 4 +
                                  2 * (size_t)KW * 4 + 2 * (size_t)KW * G * 4 + 16 * 4 + 128;
  static constexpr size_t kTwoBlocks = 113 * 1024;       // per-block budget for two resident blocks per SM
  static constexpr size_t need(int nk, int nv) {
    return FIXED + (size_t)nk * (STAGE_K + STAGE_N) + (size_t)nv * STAGE_V;
  }
  // stage depths (key tiles with their norms, value tiles): NSK - 1 key tiles in flight ahead of the scoring warps
  // and NSV - 1 value tiles ahead of the value warps; the deepest pair that keeps two blocks per SM, else a single
  // block per SM (fp16 values) with deeper stages
  static constexpr int PICK = need(4, 3) <= kTwoBlocks   ? 43
                              : need(3, 3) <= kTwoBlocks ? 33
                              : need(3, 2) <= kTwoBlocks ? 32
                              : need(5, 4) <= 220 * 1024 ? 54
                              : need(4, 3) <= 220 * 1024 ? 43
                                                         : 32;
  static constexpr int NSK = PICK / 10, NSV = PICK % 10;
  static constexpr size_t OFF_K = 0;                                         // [NSK][STAGE_K]
  static constexpr size_t OFF_V = OFF_K + NSK * (size_t)STAGE_K;             // [NSV][STAGE_V]
  static constexpr size_t OFF_N = OFF_V + NSV * (size_t)STAGE_V;             // [NSK][2][TT] fp16 norms
  static constexpr size_t STAGES_END = OFF_N + NSK * (size_t)STAGE_N;
  static constexpr size_t REDUCE_BYTES = (size_t)NVG * G * D * 4;            // final sum, reuses the stages
  static constexpr size_t OFF_TAB = ((STAGES_END > REDUCE_BYTES ? STAGES_END : REDUCE_BYTES) + 127) / 128 * 128;
  // [G][D] row factors: read only while an item starts, before the first value tile is issued into the stages
  static constexpr size_t OFF_QS = OFF_V;
  static_assert((size_t)NSV * STAGE_V >= (size_t)G * D * 4, "row factors fit the value stages");
  static constexpr size_t OFF_P = OFF_TAB + TAB;                             // [2][8][PST] fp16 or [2][TT][G] float2
  static constexpr size_t OFF_AL = OFF_P + PBUF;                             // [2][KW][G] rescale factors
  static constexpr size_t OFF_GR = OFF_AL + 2 * (size_t)KW * G * 4;         // [2][KW] rescale flags
  static constexpr size_t OFF_RM = OFF_GR + 2 * (size_t)KW * 4;             // [KW][G] running max
  static constexpr size_t OFF_RL = OFF_RM + (size_t)KW * G * 4;             // [KW][G] running sum
  static constexpr size_t OFF_CENT = OFF_RL + (size_t)KW * G * 4;
  static constexpr size_t OFF_MB = (OFF_CENT + 16 * 4 + 7) / 8 * 8;          // [NSK + NSV] stage barriers, flag
  static constexpr size_t bytes = OFF_MB + (NSK + NSV) * 8 + 8;
  // code and value tiles travel as one bulk copy each when rows are a multiple of 16 bytes (then nothing is
  // swizzled), else as 8-byte cp.async chunks
  static constexpr bool BULK = R % 16 == 0 && VROW % 16 == 0;
  static constexpr int MIN_BLOCKS = bytes <= kTwoBlocks ? 2 : 1;
  static_assert(bytes <= 227 * 1024, "shared memory of one block");
};

template <int D, int BITS, int G, bool VQ, bool PAGED>
__global__ void __launch_bounds__(kDecThreads, RowsPlan<D, BITS, G, VQ>::MIN_BLOCKS)
attend_rows_kernel(const __grid_constant__ DecodeArgs a) {
  using P = RowsPlan<D, BITS, G, VQ>;
  constexpr int TT = P::TT, WT = P::WT, KW = P::KW, RPW = P::RPW, TPR = P::TPR, NT = P::NT, R = P::R;
  extern __shared__ __align__(16) uint8_t smem[];
  const uint8_t* tab = smem + P::OFF_TAB;
  float* qs = reinterpret_cast<float*>(smem + P::OFF_QS);
  float2* pbuf = reinterpret_cast<float2*>(smem + P::OFF_P);   // fp16 values: [2][TT][G] (p, p)
  __half* pbuf16 = reinterpret_cast<__half*>(smem + P::OFF_P);  // quantized values: [2][8][PST] heads x tokens
  float* alpha_s = reinterpret_cast<float*>(smem + P::OFF_AL);
  int* grew_s = reinterpret_cast<int*>(smem + P::OFF_GR);
  float* red_m = reinterpret_cast<float*>(smem + P::OFF_RM);
  float* red_l = reinterpret_cast<float*>(smem + P::OFF_RL);
  float* cent = reinterpret_cast<float*>(smem + P::OFF_CENT);
  float* region = reinterpret_cast<float*>(smem);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool scorer = warp < KW;
  const int rtid = scorer ? tid : tid - 128;  // thread index within the role
  const uint32_t repk = static_cast<uint32_t>(lane & 15) << 3;  // the lane's hi/lo copy in the pair table
  const uint32_t repv = 128u + (static_cast<uint32_t>(lane) << 2);  // its hi-only copy
  const float rd = rsqrtf(static_cast<float>(D));

  uint64_t* kfull = reinterpret_cast<uint64_t*>(smem + P::OFF_MB);  // key stage s holds its tile
  uint64_t* vfull = kfull + P::NSK;                                   // value stage s holds its tile
  volatile int* failed = reinterpret_cast<volatile int*>(vfull + P::NSV);
  if (tid < 16) cent[tid] = a.cb.gamma[tid];
  if (tid == 0) {
    for (int s = 0; s < P::NSK + P::NSV; ++s) tc::mbar_init(kfull + s, 1);
    *failed = 0;
  }
  __syncthreads();
  build_pair_table_kv<BITS>(cent, smem + P::OFF_TAB);
  // the split merge, launched as this grid's programmatic dependent, may be scheduled from now on (its blocks wait
  // for this grid's completion before reading anything)
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  // tiles of earlier items of this block: tile t of an item uses key stage (done + t) % NSK and value stage
  // (done + t) % NSV, and barrier phases of parity ((done + t) / NS) & 1
  int done = 0;
  auto kstg = [&](int tile) { return (done + tile) % P::NSK; };
  auto kpar = [&](int tile) { return static_cast<uint32_t>(((done + tile) / P::NSK) & 1); };
  auto vstg = [&](int tile) { return (done + tile) % P::NSV; };
  auto vpar = [&](int tile) { return static_cast<uint32_t>(((done + tile) / P::NSV) & 1); };

  const int items = a.B * a.Hkv * a.splits;
  for (int item = blockIdx.x; item < items; item += gridDim.x) {
    const int split = item % a.splits;
    const int hk = (item / a.splits) % a.Hkv;
    const int b = item / (a.splits * a.Hkv);
    const int len = row_len(a, b);
    const int start = split * a.chunk;
    const int end = min(start + a.chunk, len);
    const int ntiles = end > start ? (end - start + TT - 1) / TT : 0;
    const RowMap<PAGED> rm = row_map<PAGED>(a, b, hk);  // cache row of each token (contiguous or paged)
    const float* qg = a.q + (static_cast<size_t>(b) * a.Hq + hk * G) * D;

    fence_proxy_async();  // the merge region's generic writes come before the bulk copies that reuse it
    __syncthreads();      // the previous item is finished with the row factors, the stages and the merge region
    if (a.knew != nullptr && len > 0 && start <= len - 1 && len - 1 < end) {
      // decode step: this item holds the new token (position len - 1): warp 0 writes its key and warp 1 its value
      // through the write path, before any of the item's tiles is copied
      if (warp < 2) {
        append_row<D, BITS, VQ>(a, b, hk, rm(len - 1), warp, lane,
                                reinterpret_cast<uint8_t*>(smem + P::OFF_P) + warp * D);
        __threadfence();  // the stores reach the device-wide view ...
        asm volatile("fence.proxy.async.global;\n" ::: "memory");  // ... and the async proxy of the bulk copies
      }
    }
    transform_queries<D, G>(qg, a.signs, a.mult, qs);
    fence_proxy_async();  // the row factors share memory with the value stages, refilled by bulk copies
    __syncthreads();

    if (scorer) {
      // ================================= scoring role =================================
      const int gq = lane >> 2, tq = lane & 3;
      MmaB<D, G> B;
      {
        float scl[G];
#pragma unroll
        for (int g = 0; g < G; ++g) scl[g] = tc::head_scale<D>(qg + g * D, a.mult);
        mma_b_build<D, G>(qs, scl, lane, B);
      }
      // this lane's tokens of a tile (within the warp's 32): 16 m + gq + 8 i
      float m_run[NT], l_lane[NT];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) { m_run[nt] = -INFINITY; l_lane[nt] = 0.f; }
      // norms: staged with the codes when both norm rows start 16-byte aligned (cp.async), else raw fp16 values of
      // token `lane` of the warp's share of a tile (key norm | value norm << 16) loaded one tile ahead into registers
      // and converted only when used
      // (a paged pool's blocks hold >= 16 tokens, so its norm chunks are aligned whenever the pool's base is)
      const bool nrm_async = (reinterpret_cast<uintptr_t>(a.knorms + rm(start)) & 15) == 0 &&
                             (!VQ || (reinterpret_cast<uintptr_t>(a.vnorms + rm(start)) & 15) == 0);
      __half* nst = reinterpret_cast<__half*>(smem + P::OFF_N);
      auto load_norms = [&](int tile) -> uint32_t {
        const int t = start + tile * TT + warp * WT + lane;
        uint32_t r = 0x3c00u << 16;  // value norm 1 for fp16 values
        if (!nrm_async && tile < ntiles && t < end) {
          // loads cached in L2 only: a decode step writes the new token's norms in this launch
          const size_t row = rm(t);
          r = __half_as_ushort(__ldcg(a.knorms + row));
          if constexpr (VQ) r |= static_cast<uint32_t>(__half_as_ushort(__ldcg(a.vnorms + row))) << 16;
          else r |= 0x3c00u << 16;
        }
        return r;
      };
      uint32_t nrm_next = load_norms(0);
      auto issue_k = [&](int tile) {
        if (tile < ntiles) {
          const int t0 = start + tile * TT;
          const int n = min(TT, end - t0);
          const int bytes = n * R;
          uint8_t* dst = smem + P::OFF_K + kstg(tile) * P::STAGE_K;
          if constexpr (P::BULK) {
            if (rtid == 0) {
              mbar_arrive_expect_tx(kfull + kstg(tile), bytes);
              copy_rows_bulk<R>(dst, a.kcodes, rm, t0, n, kfull + kstg(tile));
            }
          } else {
            copy_rows_async<P::KCH, R>(dst, a.kcodes, rm, t0, n, rtid);
          }
          if (nrm_async) {
            __half* nd = nst + kstg(tile) * 2 * TT;
            if (rtid < 16) stage_norms_map(nd, a.knorms, rm, t0, n, rtid);
            else if (VQ && rtid < 32) stage_norms_map(nd + TT, a.vnorms, rm, t0, n, rtid - 16);
          }
        }
        cp_async_commit();
      };
      for (int s = 0; s < P::NSK - 1; ++s) issue_k(s);
      for (int it = 0; it <= ntiles; ++it) {
        cp_async_wait<P::NSK - 2>();  // tile it's norms have landed; the next NSK - 2 may still be in flight
        roles_sync();
        issue_k(it + P::NSK - 1);     // into the stage tile it - 1 used
        if (it == ntiles) continue;
        const int t0 = start + it * TT;
        const int nt_tok = min(TT, end - t0);
        const uint8_t* st = smem + P::OFF_K + kstg(it) * P::STAGE_K;
        if constexpr (P::BULK) {
          if (!tc::mbar_wait(kfull + kstg(it), kpar(it))) *failed = 1;
        }
        float kn[2][2], vn[2][2];
        if (nrm_async) {
          const __half* nk = nst + kstg(it) * 2 * TT + warp * WT + gq;
#pragma unroll
          for (int m = 0; m < 2; ++m)
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              kn[m][i] = __half2float(nk[16 * m + 8 * i]);
              vn[m][i] = VQ ? __half2float(nk[TT + 16 * m + 8 * i]) : 1.f;
            }
        } else {
          const uint32_t nrm = nrm_next;
          nrm_next = load_norms(it + 1);
#pragma unroll
          for (int m = 0; m < 2; ++m)
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              const uint32_t x = __shfl_sync(0xffffffffu, nrm, 16 * m + gq + 8 * i);
              kn[m][i] = __half2float(__ushort_as_half(static_cast<unsigned short>(x & 0xffffu)));
              vn[m][i] = __half2float(__ushort_as_half(static_cast<unsigned short>(x >> 16)));
            }
        }
        float z[2][NT][2];
#pragma unroll
        for (int m = 0; m < 2; ++m) mma_scores16<D, BITS, G, false, true>(st, warp * WT + 16 * m, tab, repk, B, lane, z[m]);
        // online softmax over this warp's 32 tokens; lane (gq, tq) holds head 4 nt + tq
        bool grew = false;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int h = 4 * nt + tq;
          float mx = -INFINITY;
#pragma unroll
          for (int m = 0; m < 2; ++m)
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              const bool valid = h < G && warp * WT + 16 * m + gq + 8 * i < nt_tok;
              z[m][nt][i] = valid ? z[m][nt][i] * B.inv[nt] * kn[m][i] * rd : -INFINITY;
              mx = fmaxf(mx, z[m][nt][i]);
            }
#pragma unroll
          for (int msk = 4; msk < 32; msk <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, msk));
          const float m_new = fmaxf(m_run[nt], mx);
          const float alpha = (m_new == -INFINITY) ? 1.f : exp2f(m_run[nt] - m_new);
          float psum = 0.f;
#pragma unroll
          for (int m = 0; m < 2; ++m)
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              const float p = (z[m][nt][i] == -INFINITY) ? 0.f : exp2f(z[m][nt][i] - m_new);
              psum += p;
              // weight of the value product: p n^V (quantized values also carry the centroid scale 1/sqrt(d));
              // tokens past the end get 0 whatever their staged norm holds
              const float pv = p > 0.f ? p * (VQ ? vn[m][i] * rd : 1.f) : 0.f;
              if (h < G) {
                const int tok = warp * WT + 16 * m + gq + 8 * i;
                if constexpr (VQ) pbuf16[((it & 1) * 8 + h) * P::PST + tok] = __float2half_rn(pv);
                else pbuf[(static_cast<size_t>(it & 1) * TT + tok) * G + h] = make_float2(pv, pv);
              }
            }
          l_lane[nt] = l_lane[nt] * alpha + psum;
          grew |= m_new != m_run[nt];
          m_run[nt] = m_new;
          if (gq == 0 && h < G) alpha_s[((it & 1) * KW + warp) * G + h] = alpha;
        }
        grew = __any_sync(0xffffffffu, grew);
        if (lane == 0) grew_s[(it & 1) * KW + warp] = grew ? 1 : 0;
      }
      cp_async_wait<0>();
      // merge, step 1: publish this warp's running max
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        if (gq == 0 && 4 * nt + tq < G) red_m[warp * G + 4 * nt + tq] = m_run[nt];
      roles_sync();
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int h = 4 * nt + tq;
        float l = l_lane[nt];
#pragma unroll
        for (int msk = 4; msk < 32; msk <<= 1) l += __shfl_xor_sync(0xffffffffu, l, msk);
        if (h < G) {
          float M = red_m[h];
#pragma unroll
          for (int w2 = 1; w2 < KW; ++w2) M = fmaxf(M, red_m[w2 * G + h]);
          const float scl = (m_run[nt] == -INFINITY) ? 0.f : exp2f(m_run[nt] - M);
          if (gq == 0) red_l[warp * G + h] = l * scl;
        }
      }
    } else if constexpr (VQ) {
      // ========================= value role, quantized values: P V as MMAs =========================
      constexpr int MT = D / 16;            // m-tiles of 16 coordinates
      constexpr int NBV = R / 8;            // bytes of a lane's run of a value row (MT coordinate pairs)
      constexpr int NWV = (NBV + 3) / 4 + 1;
      const int vw = warp - KW;
      const int g = lane >> 2, t = lane & 3, tf = t & 1;
      // lanes with odd t fetch tokens k + 1 before k (rows of both parities in every half-warp: no bank conflicts),
      // so their byte permutes take the two pairs the other way round
      const uint32_t sel_lo = tf ? 0x1054u : 0x5410u, sel_hi = tf ? 0x3276u : 0x7632u;
      const uint8_t* vsrc = static_cast<const uint8_t*>(a.v);
      float acc[MT][4];
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[mt][c] = 0.f;
      auto issue_v = [&](int tile) {
        if (tile < ntiles) {
          const int t0 = start + tile * TT;
          const int n = min(TT, end - t0);
          uint8_t* dst = smem + P::OFF_V + vstg(tile) * P::STAGE_V;
          if constexpr (P::BULK) {
            if (rtid == 0) {
              mbar_arrive_expect_tx(vfull + vstg(tile), n * R);
              copy_rows_bulk<R>(dst, vsrc, rm, t0, n, vfull + vstg(tile));
            }
          } else {
            copy_rows_async<P::KCH, R>(dst, vsrc, rm, t0, n, rtid);
          }
        }
        cp_async_commit();
      };
      for (int it = 0; it <= ntiles; ++it) {
        cp_async_wait<P::NSV - 2>();  // tile it - 1 has landed; the next NSV - 2 may still be in flight
        roles_sync();
        // into the stage tile it - 2 used; the first tiles only now, once the scoring warps have read the row
        // factors that share memory with the value stages
        if (it == 0) {
          for (int s = 0; s <= P::NSV - 2; ++s) issue_v(s);
        } else {
          issue_v(it + P::NSV - 2);
        }
        if (it == 0) continue;
        const int j = it - 1;  // the tile scored in the previous step
        const int nt_tok = min(TT, end - (start + j * TT));
        const int pb = j & 1;
        if (grew_s[pb * KW + vw]) {  // this lane's columns are heads 2t and 2t + 1
          const float al0 = 2 * t < G ? alpha_s[(pb * KW + vw) * G + 2 * t] : 1.f;
          const float al1 = 2 * t + 1 < G ? alpha_s[(pb * KW + vw) * G + 2 * t + 1] : 1.f;
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            acc[mt][0] *= al0; acc[mt][1] *= al1; acc[mt][2] *= al0; acc[mt][3] *= al1;
          }
        }
        const uint8_t* vst = smem + P::OFF_V + vstg(j) * P::STAGE_V;
        if constexpr (P::BULK) {
          if (!tc::mbar_wait(vfull + vstg(j), vpar(j))) *failed = 1;
        }
        const __half* pw = pbuf16 + pb * 8 * P::PST;
#pragma unroll
        for (int kt = 0; kt < WT / 16; ++kt) {
          const int base = vw * WT + 16 * kt;  // the 16 tokens of this k-tile (weights beyond the tile's end are 0)
          if (base >= nt_tok) break;
          const int k0 = base + 2 * t;
          uint32_t b0 = 0u, b1 = 0u;  // B: weights of tokens k0, k0 + 1 and k0 + 8, k0 + 9 for head g
          if (g < G) {
            b0 = *reinterpret_cast<const uint32_t*>(pw + g * P::PST + k0);
            b1 = *reinterpret_cast<const uint32_t*>(pw + g * P::PST + k0 + 8);
          }
          uint32_t w[4][NWV];
          load_run<R, NBV, false>(vst, (k0 + tf) * R + g * NBV, w[0]);
          load_run<R, NBV, false>(vst, (k0 + 1 - tf) * R + g * NBV, w[1]);
          load_run<R, NBV, false>(vst, (k0 + 8 + tf) * R + g * NBV, w[2]);
          load_run<R, NBV, false>(vst, (k0 + 9 - tf) * R + g * NBV, w[3]);
#pragma unroll
          for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int i = (NBV + 3) / 4; i < NWV; ++i) w[r][i] = 0u;
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            uint32_t x[4];  // hi fp16 pairs (v_2p, v_2p+1) of the four tokens, p = MT g + mt
#pragma unroll
            for (int r = 0; r < 4; ++r) x[r] = *reinterpret_cast<const uint32_t*>(tab + kv_off<BITS>(w[r], mt, repv));
            mma_m16n8k16(acc[mt], __byte_perm(x[0], x[1], sel_lo), __byte_perm(x[0], x[1], sel_hi),
                         __byte_perm(x[2], x[3], sel_lo), __byte_perm(x[2], x[3], sel_hi), b0, b1);
          }
        }
      }
      cp_async_wait<0>();
      roles_sync();  // merge, step 1 (the scoring warps publish their running max)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int h = 2 * t + hh;
        if (h < G) {
          float M = red_m[h];
#pragma unroll
          for (int w2 = 1; w2 < KW; ++w2) M = fmaxf(M, red_m[w2 * G + h]);
          const float mw = red_m[vw * G + h];
          const float scl = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
          float* dst = region + (vw * G + h) * D;
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            const int c = 2 * (MT * g + mt);  // A rows g and g + 8 of m-tile mt
            dst[c] = acc[mt][hh] * scl;
            dst[c + 1] = acc[mt][2 + hh] * scl;
          }
        }
      }
    } else {
      // ========================= value role, fp16 values: packed fp32 FMAs =========================
      const int vw = warp - KW;
      const int vrow = lane / TPR, vc = lane % TPR;
      const uint8_t* vsrc = static_cast<const uint8_t*>(a.v);
      float2 acc[G][4];
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[g][c] = make_float2(0.f, 0.f);
      auto issue_v = [&](int tile) {
        if (tile < ntiles) {
          const int t0 = start + tile * TT;
          const int n = min(TT, end - t0);
          uint8_t* dst = smem + P::OFF_V + vstg(tile) * P::STAGE_V;
          if constexpr (P::BULK) {
            if (rtid == 0) {
              mbar_arrive_expect_tx(vfull + vstg(tile), n * P::VROW);
              copy_rows_bulk<P::VROW>(dst, vsrc, rm, t0, n, vfull + vstg(tile));
            }
          } else {
            copy_rows_async<P::VCH, P::VROW>(dst, vsrc, rm, t0, n, rtid);
          }
        }
        cp_async_commit();
      };
      for (int it = 0; it <= ntiles; ++it) {
        cp_async_wait<P::NSV - 2>();  // tile it - 1 has landed; the next NSV - 2 may still be in flight
        roles_sync();
        // into the stage tile it - 2 used; the first tiles only now, once the scoring warps have read the row
        // factors that share memory with the value stages
        if (it == 0) {
          for (int s = 0; s <= P::NSV - 2; ++s) issue_v(s);
        } else {
          issue_v(it + P::NSV - 2);
        }
        if (it == 0) continue;
        const int j = it - 1;  // the tile scored in the previous step
        const int nt_tok = min(TT, end - (start + j * TT));
        const int pb = j & 1;
        if (grew_s[pb * KW + vw]) {
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float al = alpha_s[(pb * KW + vw) * G + g];
#pragma unroll
            for (int c = 0; c < 4; ++c) { acc[g][c].x *= al; acc[g][c].y *= al; }
          }
        }
        const uint8_t* vst = smem + P::OFF_V + vstg(j) * P::STAGE_V;
        if constexpr (P::BULK) {
          if (!tc::mbar_wait(vfull + vstg(j), vpar(j))) *failed = 1;
        }
        const float2* prow = pbuf + static_cast<size_t>(pb) * TT * G;
#pragma unroll 2
        for (int i = 0; i < WT / RPW; ++i) {
          const int tt = vw * WT + vrow + RPW * i;
          if (tt >= nt_tok) break;
          float2 pw[G];
#pragma unroll
          for (int g = 0; g < G; ++g) pw[g] = prow[tt * G + g];
          float2 val[4];
          const uint4 u = *reinterpret_cast<const uint4*>(vst + tt * P::VROW + 16 * vc);
          val[0] = __half22float2(*reinterpret_cast<const __half2*>(&u.x));
          val[1] = __half22float2(*reinterpret_cast<const __half2*>(&u.y));
          val[2] = __half22float2(*reinterpret_cast<const __half2*>(&u.z));
          val[3] = __half22float2(*reinterpret_cast<const __half2*>(&u.w));
#pragma unroll
          for (int g = 0; g < G; ++g)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[g][c] = fma2(pw[g], val[c], acc[g][c]);
        }
      }
      cp_async_wait<0>();
      roles_sync();  // merge, step 1 (the scoring warps publish their running max)
      const int vg = vw * RPW + vrow;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float M = red_m[g];
#pragma unroll
        for (int w2 = 1; w2 < KW; ++w2) M = fmaxf(M, red_m[w2 * G + g]);
        const float mw = red_m[vw * G + g];
        const float scl = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
#pragma unroll
        for (int c = 0; c < 4; ++c)
          *reinterpret_cast<float2*>(region + (vg * G + g) * D + vc * 8 + 2 * c) =
              make_float2(acc[g][c].x * scl, acc[g][c].y * scl);
      }
    }
    __syncthreads();  // merge, step 2: every value group and every warp sum is in shared memory
    const size_t part0 = (static_cast<size_t>(b) * a.Hq + hk * G) * a.splits + split;  // head g adds g * splits
    for (int e = tid; e < G * D; e += kDecThreads) {
      const int g = e / D, jj = e % D;
      float s = 0.f;
#pragma unroll 4
      for (int r = 0; r < P::NVG; ++r) s += region[(r * G + g) * D + jj];
      a.ws_o[(part0 + static_cast<size_t>(g) * a.splits) * D + jj] = s;
    }
    if (tid < G) {
      float M = red_m[tid], s = 0.f;
#pragma unroll
      for (int w2 = 1; w2 < KW; ++w2) M = fmaxf(M, red_m[w2 * G + tid]);
#pragma unroll
      for (int w2 = 0; w2 < KW; ++w2) s += red_l[w2 * G + tid];
      a.ws_l[part0 + static_cast<size_t>(tid) * a.splits] = s;
      // a stage that never arrived (a copy that did not complete in about a second) poisons the output
      a.ws_m[part0 + static_cast<size_t>(tid) * a.splits] = *failed ? __int_as_float(0x7fc00000) : M;
    }
    done += ntiles;
  }
  __syncthreads();
  report_wait_failure(a, failed);
}

}  // namespace axr
