// Launchers of the literal-table kernels (lut.cuh) and the LOOKAT read-path entry points.
#include <cmath>

#include "launch.h"
#include "lut.cuh"

namespace axr {
namespace {

// Split of the token axis for the table kernels: every item builds its (batch row, KV head) table first, so items
// are made long -- the count minimises ceil(items / resident) x (chunk + setup), setup the build's cost in tokens --
// and never more splits than the workspace of axr_attend_workspace_bytes holds.
SplitPlan lut_plan(int B, int Hkv, int T, size_t smem) {
  SplitPlan p{1, T};
  if (T <= 0) return p;
  const long resident = static_cast<long>(kSmCount) * (smem <= 110 * 1024 ? 2 : 1);
  const long units = static_cast<long>(B) * Hkv;
  const int max_s = plan_splits(B, Hkv, T).splits;  // the workspace's split count
  const long setup = 2048;
  double best = 1e300;
  for (int s = 1; s <= max_s; ++s) {
    const long chunk = ((T + s - 1) / s + 255) / 256 * 256;
    const long splits = (T + chunk - 1) / chunk;
    const long rounds = (units * splits + resident - 1) / resident;
    const double cost = static_cast<double>(rounds) * static_cast<double>(chunk + setup);
    if (cost < best - 1e-9) {
      best = cost;
      p.splits = static_cast<int>(splits);
      p.chunk = static_cast<int>(chunk);
    }
  }
  return p;
}

template <typename K>
axr_status lut_smem(K kernel, size_t bytes, const char* what) {
  return ensure_smem(kernel, bytes, what);
}

template <int D, int BITS, int W, int NI, int G, int KIND>
axr_status launch_score(LutArgs a, cudaStream_t st, const char* what) {
  using P = LutPlan<D, W, NI, G>;
  auto k = lut_score_kernel<D, BITS, W, NI, G, KIND>;
  axr_status rs = lut_smem(k, P::score_bytes, what);
  if (rs != AXR_OK) return rs;
  const SplitPlan sp = lut_plan(a.B, a.Hkv, a.T, P::score_bytes);
  a.splits = sp.splits;
  a.chunk = sp.chunk;
  const long items = static_cast<long>(a.B) * a.Hkv * a.splits;
  k<<<static_cast<unsigned>(items), kLutThreads, P::score_bytes, st>>>(a);
  return check_launch(what);
}

template <int D, int BITS, int W, int NI, int G, int KIND>
axr_status launch_attend(LutArgs a, float* out, const int8_t* signs, cudaStream_t st, const char* what) {
  using P = LutPlan<D, W, NI, G>;
  auto k = table_attend_kernel<D, G, LutScorer<D, BITS, W, NI, G, KIND>>;
  axr_status rs = lut_smem(k, P::attend_bytes, what);
  if (rs != AXR_OK) return rs;
  const SplitPlan sp = lut_plan(a.B, a.Hkv, a.T, P::attend_bytes);
  a.splits = sp.splits;
  a.chunk = sp.chunk;
  const long items = static_cast<long>(a.B) * a.Hkv * a.splits;
  k<<<static_cast<unsigned>(items), kLutThreads, P::attend_bytes, st>>>(a);
  rs = check_launch(what);
  if (rs != AXR_OK) return rs;
  DecodeArgs r;
  memset(&r, 0, sizeof(r));
  r.B = a.B; r.Hq = a.Hq; r.Hkv = a.Hkv; r.T = a.T; r.splits = a.splits;
  r.ws_o = a.ws_o; r.ws_m = a.ws_m; r.ws_l = a.ws_l; r.out = out; r.signs = signs;
  launch_reduce<D, false>(r, st);
  return check_launch(what);
}

// ---- AXELRAM: field width per (d, b, G) ----------------------------------------------------------------------------
//
// The widest field (a multiple of b, at most 8 bits) whose tables fit in 160 KB of shared memory: 8 bits at b <= 2
// (4 or 8 coordinates per table), 6 at b = 3, 8 or 4 at b = 4 by the number of heads.
template <int D, int BITS, int G>
struct AxrField {
  static constexpr size_t bytes(int w) { return (size_t)(D * BITS / w) * (size_t(1) << w) * G * 4; }
  // a field holds whole coordinates and the fields tile the row
  static constexpr bool fits(int w) { return w % BITS == 0 && (D * BITS) % w == 0 && bytes(w) <= 160 * 1024; }
  static constexpr int pick() { return fits(8) ? 8 : fits(6) ? 6 : fits(4) ? 4 : BITS == 3 ? 3 : 2; }
  static constexpr int W = pick();
  static constexpr int NI = D * BITS / W;
};

template <int D, int BITS, int G>
axr_status axr_score_g(const LutArgs& a, cudaStream_t st) {
  using F = AxrField<D, BITS, G>;
  return launch_score<D, BITS, F::W, F::NI, G, kLutAxelram>(a, st, "axr_score");
}

template <int D, int BITS, int G>
axr_status axr_attend_g(const LutArgs& a, float* out, const int8_t* signs, cudaStream_t st) {
  using F = AxrField<D, BITS, G>;
  return launch_attend<D, BITS, F::W, F::NI, G, kLutAxelram>(a, out, signs, st, "axr_attend_decode");
}

template <int D, int BITS>
axr_status axr_by_g(int G, bool attend, const LutArgs& a, float* out, const int8_t* signs, cudaStream_t st) {
  switch (G) {
    case 1: return attend ? axr_attend_g<D, BITS, 1>(a, out, signs, st) : axr_score_g<D, BITS, 1>(a, st);
    case 2: return attend ? axr_attend_g<D, BITS, 2>(a, out, signs, st) : axr_score_g<D, BITS, 2>(a, st);
    case 4: return attend ? axr_attend_g<D, BITS, 4>(a, out, signs, st) : axr_score_g<D, BITS, 4>(a, st);
    case 8: return attend ? axr_attend_g<D, BITS, 8>(a, out, signs, st) : axr_score_g<D, BITS, 8>(a, st);
  }
  return set_error(AXR_EUNSUPPORTED, "table kernels: G=%d", G);
}

template <int D>
axr_status axr_by_bits(int bits, int G, bool attend, const LutArgs& a, float* out, const int8_t* signs,
                       cudaStream_t st) {
  switch (bits) {
    case 1: return axr_by_g<D, 1>(G, attend, a, out, signs, st);
    case 2: return axr_by_g<D, 2>(G, attend, a, out, signs, st);
    case 3: return axr_by_g<D, 3>(G, attend, a, out, signs, st);
    case 4: return axr_by_g<D, 4>(G, attend, a, out, signs, st);
  }
  return set_error(AXR_EUNSUPPORTED, "table kernels: bits=%d", bits);
}

LutArgs lut_from_decode(const DecodeArgs& d) {
  LutArgs a;
  memset(&a, 0, sizeof(a));
  a.q = d.q; a.codes = d.kcodes; a.norms = d.knorms; a.signs = d.signs; a.v = static_cast<const __half*>(d.v);
  a.seq_lens = d.seq_lens; a.scores = d.scores; a.ws_o = d.ws_o; a.ws_m = d.ws_m; a.ws_l = d.ws_l;
  a.B = d.B; a.Hq = d.Hq; a.Hkv = d.Hkv; a.T = d.T; a.Tcap = d.Tcap; a.mult = d.mult; a.cb = d.cb;
  return a;
}

// ---- LOOKAT ------------------------------------------------------------------------------------------------------------

template <int D, int NI, int G>
axr_status pq_g(bool attend, const LutArgs& a, float* out, cudaStream_t st) {
  if (attend) return launch_attend<D, 1, 8, NI, G, kLutPq>(a, out, nullptr, st, "axr_pq_attend_decode");
  return launch_score<D, 1, 8, NI, G, kLutPq>(a, st, "axr_pq_score");
}

template <int D, int NI>
axr_status pq_by_g(int G, bool attend, const LutArgs& a, float* out, cudaStream_t st) {
  switch (G) {
    case 1: return pq_g<D, NI, 1>(attend, a, out, st);
    case 2: return pq_g<D, NI, 2>(attend, a, out, st);
    case 4: return pq_g<D, NI, 4>(attend, a, out, st);
    case 8: return pq_g<D, NI, 8>(attend, a, out, st);
  }
  return set_error(AXR_EUNSUPPORTED, "pq: G=%d", G);
}

template <int D>
axr_status pq_by_m(int m, int G, bool attend, const LutArgs& a, float* out, cudaStream_t st) {
  switch (m) {
    case 2: return pq_by_g<D, 2>(G, attend, a, out, st);
    case 4: return pq_by_g<D, 4>(G, attend, a, out, st);
    case 8: return pq_by_g<D, 8>(G, attend, a, out, st);
    case 16: return pq_by_g<D, 16>(G, attend, a, out, st);
  }
  return set_error(AXR_EUNSUPPORTED, "pq: m=%d not in {2, 4, 8, 16}", m);
}

axr_status pq_check(const char* w, int B, int Hq, int Hkv, int T, int Tcap, int d, int m, int K) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || T < 0 || Tcap < T)
    return set_error(AXR_EINVAL, "%s: bad sizes B=%d Hq=%d Hkv=%d T=%d Tcap=%d", w, B, Hq, Hkv, T, Tcap);
  if (Hq % Hkv) return set_error(AXR_EINVAL, "%s: Hq=%d is not a multiple of Hkv=%d", w, Hq, Hkv);
  if (d != 64 && d != 128) return set_error(AXR_EUNSUPPORTED, "%s: d=%d not in {64,128}", w, d);
  if (m != 2 && m != 4 && m != 8 && m != 16) return set_error(AXR_EUNSUPPORTED, "%s: m=%d not in {2,4,8,16}", w, m);
  if (K < 1 || K > 256) return set_error(AXR_EUNSUPPORTED, "%s: K=%d outside 1..256", w, K);
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return set_error(AXR_EUNSUPPORTED, "%s: G=%d not in {1,2,4,8}", w, G);
  return AXR_OK;
}

}  // namespace

// AXELRAM table mode of axr_score (AXR_GATHER_TABLE) and of axr_attend_decode over fp16 values.
axr_status table_score_launch(int d, int bits, int G, const DecodeArgs& da, cudaStream_t st) {
  const LutArgs a = lut_from_decode(da);
  if (d == 64) return axr_by_bits<64>(bits, G, false, a, nullptr, nullptr, st);
  return axr_by_bits<128>(bits, G, false, a, nullptr, nullptr, st);
}

axr_status table_attend_launch(int d, int bits, int G, const DecodeArgs& da, cudaStream_t st) {
  const LutArgs a = lut_from_decode(da);
  if (d == 64) return axr_by_bits<64>(bits, G, true, a, da.out, da.signs, st);
  return axr_by_bits<128>(bits, G, true, a, da.out, da.signs, st);
}

}  // namespace axr

extern "C" axr_status axr_pq_score(const float* q, const uint8_t* codes, const float* codebooks,
                                   const int32_t* seq_lens, int B, int Hq, int Hkv, int T, int Tcap, int d, int m,
                                   int K, float scale, float* scores, void* stream) {
  using namespace axr;
  const char* w = "axr_pq_score";
  axr_status st = pq_check(w, B, Hq, Hkv, T, Tcap, d, m, K);
  if (st != AXR_OK) return st;
  if (B == 0 || T == 0) return set_error(AXR_OK, "");
  if (!q || !codes || !codebooks || !scores) return set_error(AXR_EINVAL, "%s: null pointer", w);
  if (!aligned(q, 16) || !aligned(codes, m >= 4 ? 4 : 2) || !aligned(codebooks, 4) || !aligned(scores, 4) ||
      (seq_lens && !aligned(seq_lens, 4)))
    return set_error(AXR_EINVAL, "%s: misaligned pointer", w);
  if (!std::isfinite(scale)) return set_error(AXR_EINVAL, "%s: scale is not finite", w);
  LutArgs a;
  memset(&a, 0, sizeof(a));
  a.q = q; a.codes = codes; a.pq_cb = codebooks; a.seq_lens = seq_lens; a.scores = scores;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.T = T; a.Tcap = Tcap; a.K = K; a.mult = scale;
  const int G = Hq / Hkv;
  if (d == 64) return pq_by_m<64>(m, G, false, a, nullptr, as_stream(stream));
  return pq_by_m<128>(m, G, false, a, nullptr, as_stream(stream));
}

extern "C" axr_status axr_pq_attend_decode(const float* q, const uint8_t* codes, const float* codebooks,
                                           const uint16_t* v, const int32_t* seq_lens, int B, int Hq, int Hkv, int T,
                                           int Tcap, int d, int m, int K, float scale, float* out, void* workspace,
                                           size_t ws_bytes, void* stream) {
  using namespace axr;
  const char* w = "axr_pq_attend_decode";
  axr_status st = pq_check(w, B, Hq, Hkv, T, Tcap, d, m, K);
  if (st != AXR_OK) return st;
  if (B == 0) return set_error(AXR_OK, "");
  if (!q || !codes || !codebooks || !v || !out) return set_error(AXR_EINVAL, "%s: null pointer", w);
  if (!aligned(q, 16) || !aligned(codes, m >= 4 ? 4 : 2) || !aligned(codebooks, 4) || !aligned(v, 16) ||
      !aligned(out, 16) || (seq_lens && !aligned(seq_lens, 4)))
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
  a.q = q; a.codes = codes; a.pq_cb = codebooks; a.seq_lens = seq_lens; a.v = reinterpret_cast<const __half*>(v);
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.T = T; a.Tcap = Tcap; a.K = K; a.mult = scale * kLog2e;
  // the partials take the layout of axr_attend_workspace_bytes' largest split count (the table plan uses fewer)
  const int smax = plan_splits(B, Hkv, T).splits;
  const size_t parts = static_cast<size_t>(B) * Hq * smax;
  a.ws_o = static_cast<float*>(workspace);
  a.ws_m = a.ws_o + parts * d;
  a.ws_l = a.ws_m + parts;
  const int G = Hq / Hkv;
  if (d == 64) return pq_by_m<64>(m, G, true, a, out, as_stream(stream));
  return pq_by_m<128>(m, G, true, a, out, as_stream(stream));
}
