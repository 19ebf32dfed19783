// Power-of-two (PoT) shift-accumulate key codec: writer, integer scores and decode attention with an integer-log2
// softmax.
//
// Source: the arxivdaily page of the shift-accumulate attention paper (English abstract).  Keys are stored as signed
// power-of-two fixed-point codes, so every product of QK^T is a sign flip, a shift and an integer accumulation; a
// fixed-point head-room F >= e_max makes every shift non-negative and the accumulation exact; a sub-power mantissa
// term adds one shift-add; the softmax keeps its running maximum in an integer log2 domain so that every rescale is
// an exact shift; the attention-value product is log-quantized.  The page gives no formulas; the reading here:
//   key row k (fp16): alpha = max_j |k_j| (exact in fp16); u_j = k_j / alpha (fp32); |u_j| to the nearest magnitude
//   level 2^-e (1 + mu / 2^M) in linear value (a value on a midpoint goes up), rank l = (e_max - e) 2^M + mu from the
//   smallest level; code = sign << (E + M) | l, 1 + E + M bits packed LSB-first, e_max = 2^E - 1;
//   query: Q_j = rint(q_j / s_q), s_q = max_j |q_j| / 32767 (fp32);
//   score: S = sum_j sigma_j Q_j (2^M + mu_j) 2^(l_j >> M)  [= sigma_j (Q_j << (F - e_j)) + mu_j (Q_j << (F - e_j - M)),
//   F = e_max + M], an exact int32; the real score is s_q alpha 2^-F S;
//   softmax: r_t = rint(float(S) * (s_q * mult * alpha_t) * 2^-F), mult = scale * log2(e) (fp32, in that order);
//   weights 2^(r_t - max r), exact powers of two; out = sum 2^(r_t - R) v_t / sum 2^(r_t - R).
// On B200 the sign flip and the shift of one coordinate are one integer multiply by +-(2^M + mu) 2^(l >> M) (an
// IMAD issues at the rate of a shift or an add, and the integer is the same).
#include <cmath>

#include "launch.h"
#include "lut.cuh"
#include "write_vec.cuh"

namespace axr {
namespace {

constexpr int kPotMaxLevels = 8;  // 2^(E + M) with 1 + E + M <= 4

struct PotThresholds {
  float t[kPotMaxLevels];  // midpoints between consecutive magnitude levels, ascending (exact dyadic numbers)
};

// ---- writer: one warp per vector ------------------------------------------------------------------------------------

template <int D, int E, int M>
__global__ void __launch_bounds__(256) pot_write_kernel(const __half* __restrict__ x, int64_t n_vec,
                                                        const int64_t* __restrict__ dst_rows,
                                                        uint8_t* __restrict__ codes, __half* __restrict__ alpha,
                                                        const PotThresholds th) {
  constexpr int BITS = 1 + E + M, NL = 1 << (E + M), VPL = D / kWarp, R = D * BITS / 8;
  __shared__ uint8_t idx[256 / kWarp][D];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t wstride = static_cast<int64_t>(gridDim.x) * (blockDim.x / kWarp);
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * (blockDim.x / kWarp) + warp; r < n_vec; r += wstride) {
    float v[VPL];
    load_lane<__half, VPL>(x + r * D, lane, v);
    float mx = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) mx = fmaxf(mx, fabsf(v[i]));
    mx = warp_max(mx);
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const float u = mx > 0.f ? __fdiv_rn(v[i], mx) : 0.f;
      const float mag = fabsf(u);
      int rank = 0;
#pragma unroll
      for (int k = 0; k < NL - 1; ++k) rank += mag >= th.t[k] ? 1 : 0;
      idx[warp][lane * VPL + i] = static_cast<uint8_t>(((u < 0.f ? 1 : 0) << (E + M)) | rank);
    }
    __syncwarp();
    const int64_t row = dst_rows ? dst_rows[r] : r;
    pack_row<D, BITS>(idx[warp], codes + row * R, lane);
    if (lane == 0) alpha[row] = __float2half_rn(mx);  // exact: the max of fp16 magnitudes
    __syncwarp();
  }
}

// ---- scorer policy: the integer shift-accumulate ----------------------------------------------------------------------

template <int D, int E, int M, int G>
struct PotScorer {
  static constexpr int BITS = 1 + E + M, RB = D * BITS / 8, NW = (RB + 3) / 4 + 1, F = (1 << E) - 1 + M;
  static constexpr bool EXACT = true;                // integer log2 weights: exact powers of two
  static constexpr size_t OFF_Q = 0;                 // [G][D] int32 fixed-point queries
  static constexpr size_t OFF_C = (size_t)G * D * 4;  // [G] s_q * mult
  static constexpr size_t SMEM = OFF_C + 16 * 4;

  __device__ static void build(const LutArgs& a, int b, int hk, uint8_t* smem) {
    int* Qs = reinterpret_cast<int*>(smem + OFF_Q);
    float* cq = reinterpret_cast<float*>(smem + OFF_C);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const float* qg = a.q + (static_cast<size_t>(b) * a.Hq + hk * G) * D;
    __syncthreads();  // the previous item is done with the queries
    for (int g = warp; g < G; g += blockDim.x / kWarp) {
      float mx = 0.f;
      for (int j = lane; j < D; j += kWarp) mx = fmaxf(mx, fabsf(qg[g * D + j]));
      mx = warp_max(mx);
      const float s = __fdiv_rn(mx, 32767.f);
      for (int j = lane; j < D; j += kWarp) Qs[g * D + j] = s > 0.f ? __float2int_rn(__fdiv_rn(qg[g * D + j], s)) : 0;
      if (lane == 0) cq[g] = __fmul_rn(s, a.mult);
    }
    __syncthreads();
  }

  struct Row {  // a token's code row and alpha, loaded a tile ahead of its scoring
    uint32_t w[NW];
    unsigned short alpha;
  };
  __device__ static void load(const LutArgs& a, size_t row0, int t, Row& r) {
    lut_load_row<RB>(a.codes + (row0 + t) * RB, r.w);
    r.alpha = __ldg(reinterpret_cast<const unsigned short*>(a.norms) + row0 + t);
  }

  // S[h] = sum_j sigma_j Q[h][j] (2^M + mu_j) 2^(l_j >> M) for the token whose code words are w
  __device__ static void integer_scores(const uint8_t* smem, const uint32_t (&w)[NW], int (&S)[G]) {
    const int* Qs = reinterpret_cast<const int*>(smem + OFF_Q);
#pragma unroll
    for (int h = 0; h < G; ++h) S[h] = 0;
#pragma unroll
    for (int j0 = 0; j0 < D; j0 += 4) {
      int4 qv[G];
#pragma unroll
      for (int h = 0; h < G; ++h) qv[h] = *reinterpret_cast<const int4*>(Qs + h * D + j0);  // one broadcast load
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint32_t code = bits_at<BITS>(w, (j0 + c) * BITS);
        const uint32_t rank = code & ((1u << (E + M)) - 1u);
        const int mag = ((1 << M) + static_cast<int>(rank & ((1u << M) - 1u))) << (rank >> M);
        const int f = (code >> (E + M)) ? -mag : mag;  // the sign flip and the shift
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const int qj = c == 0 ? qv[h].x : c == 1 ? qv[h].y : c == 2 ? qv[h].z : qv[h].w;
          S[h] += qj * f;
        }
      }
    }
  }

  // exponent r_t (integer, as a float) in the log2 domain, -inf for an invalid token
  __device__ static void score(const LutArgs& a, const uint8_t* smem, const Row& r, bool valid, float (&z)[G]) {
    const float* cq = reinterpret_cast<const float*>(smem + OFF_C);
    int S[G];
    integer_scores(smem, r.w, S);
    const float al = __half2float(__ushort_as_half(r.alpha));
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float c = __fmul_rn(cq[h], al);
      const float w = __fmul_rn(__fmul_rn(__int2float_rn(S[h]), c), ldexpf(1.f, -F));
      z[h] = valid ? rintf(w) : -INFINITY;
    }
  }
};

// Scores only: S as int32 (S_out) and the real scores scale * s_q * alpha * 2^-F * S (scores), -inf and 0 past the
// row's length.  a.mult holds the scale.
template <int D, int E, int M, int G>
__global__ void __launch_bounds__(kLutThreads) pot_score_kernel(const __grid_constant__ LutArgs a, int* S_out) {
  using Sc = PotScorer<D, E, M, G>;
  extern __shared__ __align__(16) uint8_t smem[];
  const float* cq = reinterpret_cast<const float*>(smem + Sc::OFF_C);
  const int items = a.B * a.Hkv * a.splits;
  for (int item = blockIdx.x; item < items; item += gridDim.x) {
    const int split = item % a.splits;
    const int hk = (item / a.splits) % a.Hkv;
    const int b = item / (a.splits * a.Hkv);
    const int start = split * a.chunk;
    const int end = min(start + a.chunk, a.T);
    const int vend = min(end, lut_len(a, b));
    const size_t o0 = (static_cast<size_t>(b) * a.Hq + hk * G) * a.T;
    for (int t = max(start, vend) + threadIdx.x; t < end; t += kLutThreads)
#pragma unroll
      for (int h = 0; h < G; ++h) {
        if (a.scores) a.scores[o0 + static_cast<size_t>(h) * a.T + t] = -INFINITY;
        if (S_out) S_out[o0 + static_cast<size_t>(h) * a.T + t] = 0;
      }
    if (vend <= start) continue;
    Sc::build(a, b, hk, smem);
    const size_t row0 = lut_row(a, b, hk, 0);
    for (int t = start + threadIdx.x; t < vend; t += kLutThreads) {
      int S[G];
      typename Sc::Row r;
      Sc::load(a, row0, t, r);
      Sc::integer_scores(smem, r.w, S);
      const float al = __half2float(__ushort_as_half(r.alpha));
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const size_t o = o0 + static_cast<size_t>(h) * a.T + t;
        if (S_out) S_out[o] = S[h];
        if (a.scores)
          a.scores[o] = __fmul_rn(__fmul_rn(__int2float_rn(S[h]), __fmul_rn(cq[h], al)), ldexpf(1.f, -Sc::F));
      }
    }
  }
}

// ---- launchers ----------------------------------------------------------------------------------------------------------

PotThresholds pot_thresholds(int E, int M) {
  PotThresholds th;
  memset(&th, 0, sizeof(th));
  const int n = 1 << (E + M), e_max = (1 << E) - 1;
  double prev = 0.0;
  for (int l = 0; l < n; ++l) {
    const int e = e_max - (l >> M), mu = l & ((1 << M) - 1);
    const double lv = std::ldexp(1.0 + static_cast<double>(mu) / (1 << M), -e);
    if (l > 0) th.t[l - 1] = static_cast<float>((prev + lv) / 2);  // dyadic: exact in fp32
    prev = lv;
  }
  return th;
}

// Split plan for the small-table PoT kernels (several blocks per SM), never more splits than the workspace holds.
SplitPlan pot_plan(int B, int Hkv, int T) {
  SplitPlan p{1, T};
  const long resident = 4L * kSmCount;
  const long units = static_cast<long>(B) * Hkv;
  const int max_s = plan_splits(B, Hkv, T).splits;
  double best = 1e300;
  for (int s = 1; s <= max_s; ++s) {
    const long chunk = ((T + s - 1) / s + 255) / 256 * 256;
    const long splits = (T + chunk - 1) / chunk;
    const long rounds = (units * splits + resident - 1) / resident;
    const double cost = static_cast<double>(rounds) * static_cast<double>(chunk + 512);
    if (cost < best - 1e-9) {
      best = cost;
      p.splits = static_cast<int>(splits);
      p.chunk = static_cast<int>(chunk);
    }
  }
  return p;
}

template <int D, int E, int M, int G>
axr_status pot_launch(bool attend, LutArgs a, int* S_out, float* out, cudaStream_t st, const char* w) {
  using Sc = PotScorer<D, E, M, G>;
  const SplitPlan sp = pot_plan(a.B, a.Hkv, a.T);
  a.splits = sp.splits;
  a.chunk = sp.chunk;
  const unsigned items = static_cast<unsigned>(static_cast<long>(a.B) * a.Hkv * a.splits);
  if (!attend) {
    pot_score_kernel<D, E, M, G><<<items, kLutThreads, Sc::SMEM, st>>>(a, S_out);
    return check_launch(w);
  }
  constexpr size_t bytes = Sc::SMEM + (size_t)(kLutThreads / kWarp) * G * (D + 2) * 4;
  auto k = table_attend_kernel<D, G, Sc>;
  axr_status rs = ensure_smem(k, bytes, w);
  if (rs != AXR_OK) return rs;
  k<<<items, kLutThreads, bytes, st>>>(a);
  rs = check_launch(w);
  if (rs != AXR_OK) return rs;
  DecodeArgs r;
  memset(&r, 0, sizeof(r));
  r.B = a.B; r.Hq = a.Hq; r.Hkv = a.Hkv; r.T = a.T; r.splits = a.splits;
  r.ws_o = a.ws_o; r.ws_m = a.ws_m; r.ws_l = a.ws_l; r.out = out;
  launch_reduce<D, false, true>(r, st);
  return check_launch(w);
}

template <int D, int E, int M>
axr_status pot_by_g(int G, bool attend, const LutArgs& a, int* S_out, float* out, cudaStream_t st, const char* w) {
  switch (G) {
    case 1: return pot_launch<D, E, M, 1>(attend, a, S_out, out, st, w);
    case 2: return pot_launch<D, E, M, 2>(attend, a, S_out, out, st, w);
    case 4: return pot_launch<D, E, M, 4>(attend, a, S_out, out, st, w);
    case 8: return pot_launch<D, E, M, 8>(attend, a, S_out, out, st, w);
  }
  return set_error(AXR_EUNSUPPORTED, "%s: G=%d", w, G);
}

template <int D>
axr_status pot_by_fmt(int E, int M, int G, bool attend, const LutArgs& a, int* S_out, float* out, cudaStream_t st,
                      const char* w) {
  if (E == 1 && M == 0) return pot_by_g<D, 1, 0>(G, attend, a, S_out, out, st, w);
  if (E == 2 && M == 0) return pot_by_g<D, 2, 0>(G, attend, a, S_out, out, st, w);
  if (E == 3 && M == 0) return pot_by_g<D, 3, 0>(G, attend, a, S_out, out, st, w);
  if (E == 1 && M == 1) return pot_by_g<D, 1, 1>(G, attend, a, S_out, out, st, w);
  if (E == 2 && M == 1) return pot_by_g<D, 2, 1>(G, attend, a, S_out, out, st, w);
  return set_error(AXR_EUNSUPPORTED, "%s: (E, M) = (%d, %d)", w, E, M);
}

bool pot_fmt_ok(int E, int M) { return E >= 1 && M >= 0 && M <= 1 && 1 + E + M <= 4; }

axr_status pot_check(const char* w, int B, int Hq, int Hkv, int T, int Tcap, int d, int E, int M) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || T < 0 || Tcap < T)
    return set_error(AXR_EINVAL, "%s: bad sizes B=%d Hq=%d Hkv=%d T=%d Tcap=%d", w, B, Hq, Hkv, T, Tcap);
  if (Hq % Hkv) return set_error(AXR_EINVAL, "%s: Hq=%d is not a multiple of Hkv=%d", w, Hq, Hkv);
  if (d != 64 && d != 128) return set_error(AXR_EUNSUPPORTED, "%s: d=%d not in {64,128}", w, d);
  if (!pot_fmt_ok(E, M)) return set_error(AXR_EUNSUPPORTED, "%s: (E, M) = (%d, %d)", w, E, M);
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return set_error(AXR_EUNSUPPORTED, "%s: G=%d not in {1,2,4,8}", w, G);
  return AXR_OK;
}

template <int D, int E, int M>
axr_status write_fmt(const __half* x, int64_t n, const int64_t* dst, uint8_t* codes, __half* alpha, cudaStream_t st) {
  long blocks = static_cast<long>((n + 7) / 8);
  if (blocks > 16L * kSmCount) blocks = 16L * kSmCount;
  pot_write_kernel<D, E, M><<<static_cast<unsigned>(blocks), 256, 0, st>>>(x, n, dst, codes, alpha,
                                                                           pot_thresholds(E, M));
  return check_launch("axr_pot_write");
}

template <int D>
axr_status write_d(int E, int M, const __half* x, int64_t n, const int64_t* dst, uint8_t* codes, __half* alpha,
                   cudaStream_t st) {
  if (E == 1 && M == 0) return write_fmt<D, 1, 0>(x, n, dst, codes, alpha, st);
  if (E == 2 && M == 0) return write_fmt<D, 2, 0>(x, n, dst, codes, alpha, st);
  if (E == 3 && M == 0) return write_fmt<D, 3, 0>(x, n, dst, codes, alpha, st);
  if (E == 1 && M == 1) return write_fmt<D, 1, 1>(x, n, dst, codes, alpha, st);
  if (E == 2 && M == 1) return write_fmt<D, 2, 1>(x, n, dst, codes, alpha, st);
  return set_error(AXR_EUNSUPPORTED, "axr_pot_write: (E, M) = (%d, %d)", E, M);
}

}  // namespace
}  // namespace axr

extern "C" axr_status axr_pot_write(const uint16_t* x, int64_t n_vec, int d, int E, int M, const int64_t* dst_rows,
                                    uint8_t* codes, uint16_t* alpha, void* stream) {
  using namespace axr;
  const char* w = "axr_pot_write";
  if (d != 64 && d != 128) return set_error(AXR_EUNSUPPORTED, "%s: d=%d not in {64,128}", w, d);
  if (!pot_fmt_ok(E, M)) return set_error(AXR_EUNSUPPORTED, "%s: (E, M) = (%d, %d)", w, E, M);
  if (n_vec < 0) return set_error(AXR_EINVAL, "%s: n_vec < 0", w);
  if (n_vec == 0) return set_error(AXR_OK, "");
  if (!x || !codes || !alpha) return set_error(AXR_EINVAL, "%s: null pointer", w);
  if (!aligned(x, 8) || !aligned(alpha, 2) || (dst_rows && !aligned(dst_rows, 8)))
    return set_error(AXR_EINVAL, "%s: misaligned pointer", w);
  const __half* xh = reinterpret_cast<const __half*>(x);
  __half* ah = reinterpret_cast<__half*>(alpha);
  cudaStream_t st = as_stream(stream);
  if (d == 64) return write_d<64>(E, M, xh, n_vec, dst_rows, codes, ah, st);
  return write_d<128>(E, M, xh, n_vec, dst_rows, codes, ah, st);
}

extern "C" axr_status axr_pot_score(const float* q, const uint8_t* codes, const uint16_t* alpha,
                                    const int32_t* seq_lens, int B, int Hq, int Hkv, int T, int Tcap, int d, int E,
                                    int M, float scale, int32_t* S_out, float* scores, void* stream) {
  using namespace axr;
  const char* w = "axr_pot_score";
  axr_status st = pot_check(w, B, Hq, Hkv, T, Tcap, d, E, M);
  if (st != AXR_OK) return st;
  if (B == 0 || T == 0) return set_error(AXR_OK, "");
  if (!q || !codes || !alpha || (!S_out && !scores)) return set_error(AXR_EINVAL, "%s: null pointer", w);
  if (!aligned(q, 16) || !aligned(codes, 16) || !aligned(alpha, 2) || (S_out && !aligned(S_out, 4)) ||
      (scores && !aligned(scores, 4)) || (seq_lens && !aligned(seq_lens, 4)))
    return set_error(AXR_EINVAL, "%s: misaligned pointer", w);
  if (!std::isfinite(scale)) return set_error(AXR_EINVAL, "%s: scale is not finite", w);
  LutArgs a;
  memset(&a, 0, sizeof(a));
  a.q = q; a.codes = codes; a.norms = reinterpret_cast<const __half*>(alpha); a.seq_lens = seq_lens;
  a.scores = scores; a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.T = T; a.Tcap = Tcap; a.mult = scale;
  const int G = Hq / Hkv;
  if (d == 64) return pot_by_fmt<64>(E, M, G, false, a, S_out, nullptr, as_stream(stream), w);
  return pot_by_fmt<128>(E, M, G, false, a, S_out, nullptr, as_stream(stream), w);
}

extern "C" axr_status axr_pot_attend_decode(const float* q, const uint8_t* codes, const uint16_t* alpha,
                                            const uint16_t* v, const int32_t* seq_lens, int B, int Hq, int Hkv,
                                            int T, int Tcap, int d, int E, int M, float scale, float* out,
                                            void* workspace, size_t ws_bytes, void* stream) {
  using namespace axr;
  const char* w = "axr_pot_attend_decode";
  axr_status st = pot_check(w, B, Hq, Hkv, T, Tcap, d, E, M);
  if (st != AXR_OK) return st;
  if (B == 0) return set_error(AXR_OK, "");
  if (!q || !codes || !alpha || !v || !out) return set_error(AXR_EINVAL, "%s: null pointer", w);
  if (!aligned(q, 16) || !aligned(codes, 16) || !aligned(alpha, 2) || !aligned(v, 16) || !aligned(out, 16) ||
      (seq_lens && !aligned(seq_lens, 4)))
    return set_error(AXR_EINVAL, "%s: misaligned pointer", w);
  if (!std::isfinite(scale)) return set_error(AXR_EINVAL, "%s: scale is not finite", w);
  if (T == 0) {
    cudaError_t e = cudaMemsetAsync(out, 0, sizeof(float) * (size_t)B * Hq * d, as_stream(stream));
    return e == cudaSuccess ? set_error(AXR_OK, "") : set_error(AXR_ECUDA, "%s: %s", w, cudaGetErrorString(e));
  }
  const size_t need = attend_ws_bytes(B, Hq, Hkv, T, d);
  if (!workspace || ws_bytes < need)
    return set_error(AXR_EWORKSPACE, "%s: workspace of %zu bytes, need %zu", w, workspace ? ws_bytes : 0, need);
  if (!aligned(workspace, 16)) return set_error(AXR_EINVAL, "%s: workspace not 16-byte aligned", w);
  LutArgs a;
  memset(&a, 0, sizeof(a));
  a.q = q; a.codes = codes; a.norms = reinterpret_cast<const __half*>(alpha); a.seq_lens = seq_lens;
  a.v = reinterpret_cast<const __half*>(v);
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.T = T; a.Tcap = Tcap; a.mult = scale * kLog2e;
  const int smax = plan_splits(B, Hkv, T).splits;  // the workspace's split count (the PoT plan uses no more)
  const size_t parts = static_cast<size_t>(B) * Hq * smax;
  a.ws_o = static_cast<float*>(workspace);
  a.ws_m = a.ws_o + parts * d;
  a.ws_l = a.ws_m + parts;
  const int G = Hq / Hkv;
  if (d == 64) return pot_by_fmt<64>(E, M, G, true, a, nullptr, out, as_stream(stream), w);
  return pot_by_fmt<128>(E, M, G, true, a, nullptr, out, as_stream(stream), w);
}
