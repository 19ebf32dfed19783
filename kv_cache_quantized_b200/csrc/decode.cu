// Host entry points of the decode read path: axr_score, axr_attend_decode, axr_dense_decode.
#include <atomic>
#include <cmath>

#include "decode.cuh"
#include "score_tc.cuh"
#include "attend_tcv.cuh"
#include "attend_mma.cuh"
#include "score_mma.cuh"

namespace axr {
namespace {

template <typename K>
axr_status ensure_smem(K kernel, size_t bytes, const char* what) {
  if (bytes > 48 * 1024) {  // idempotent, and per device: set before every launch
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return set_error(AXR_ECUDA, "%s: cudaFuncSetAttribute: %s", what, cudaGetErrorString(e));
  }
  return AXR_OK;
}

// ---- common validation -----------------------------------------------------------------------------------------

axr_status check_decode_sizes(const char* what, int B, int Hq, int Hkv, int T, int Tcap, int d) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || T < 0 || Tcap < T)
    return set_error(AXR_EINVAL, "%s: bad sizes B=%d Hq=%d Hkv=%d T=%d Tcap=%d", what, B, Hq, Hkv, T, Tcap);
  if (Hq % Hkv) return set_error(AXR_EINVAL, "%s: Hq=%d is not a multiple of Hkv=%d", what, Hq, Hkv);
  if (d != 64 && d != 128) return set_error(AXR_EUNSUPPORTED, "%s: d=%d not in {64,128}", what, d);
  if (!supported_g(Hq / Hkv)) return set_error(AXR_EUNSUPPORTED, "%s: G=%d not in {1,2,4,8}", what, Hq / Hkv);
  return AXR_OK;
}

// ---- launchers -------------------------------------------------------------------------------------------------

template <int D, int BITS, int G, bool VQ, bool DENSE>
axr_status launch_attend(const DecodeArgs& a, cudaStream_t st, const char* what) {
  using S = DecPlan<D, BITS, G, VQ, DENSE>;
  auto k1 = attend_partial_kernel<D, BITS, G, VQ, DENSE>;
  axr_status rs = ensure_smem(k1, S::bytes, what);
  if (rs != AXR_OK) return rs;
  const long items = static_cast<long>(a.B) * a.Hkv * a.splits;  // persistent blocks loop over the items
  const long resident = static_cast<long>(S::MIN_BLOCKS) * kSmCount;
  const unsigned grid = static_cast<unsigned>(items < resident ? items : resident);
  k1<<<grid, kDecThreads, S::bytes, st>>>(a);
  attend_reduce_kernel<D, VQ><<<a.B * a.Hq, D, 0, st>>>(a);
  return check_launch(what);
}

template <int BITS, int G>
axr_status launch_attend_tcv(const DecodeArgs& a, cudaStream_t st) {
  using S = TcaPlan<BITS, G>;
  auto k1 = attend_tcv_kernel<BITS, G>;
  axr_status rs = ensure_smem(k1, S::bytes, "axr_attend_decode");
  if (rs != AXR_OK) return rs;
  const long items = static_cast<long>(a.B) * a.Hkv * a.splits;  // persistent: one CTA per SM
  const unsigned grid = static_cast<unsigned>(items < kSmCount ? items : kSmCount);
  k1<<<grid, S::THREADS, S::bytes, st>>>(a);
  attend_reduce_kernel<128, true><<<a.B * a.Hq, 128, 0, st>>>(a);
  return check_launch("axr_attend_decode");
}

template <int BITS, int G>
axr_status launch_attend_mma(const DecodeArgs& a, cudaStream_t st) {
  using S = MmaPlan<BITS, G>;
  auto k1 = attend_mma_kernel<BITS, G>;
  axr_status rs = ensure_smem(k1, S::bytes, "axr_attend_decode");
  if (rs != AXR_OK) return rs;
  const long items = static_cast<long>(a.B) * a.Hkv * a.splits;  // persistent blocks loop over the items
  const long resident = static_cast<long>(S::MIN_BLOCKS) * kSmCount;
  k1<<<static_cast<unsigned>(items < resident ? items : resident), kDecThreads, S::bytes, st>>>(a);
  attend_reduce_kernel<128, true><<<a.B * a.Hq, 128, 0, st>>>(a);
  return check_launch("axr_attend_decode");
}

template <int BITS, int G>
axr_status launch_attend_tiled(const DecodeArgs& a, cudaStream_t st);

template <int BITS>
axr_status attend_tcv_g(int G, const DecodeArgs& a, cudaStream_t st) {
  switch (G) {
    case 1: return launch_attend_tiled<BITS, 1>(a, st);
    case 2: return launch_attend_tiled<BITS, 2>(a, st);
    case 4: return launch_attend_tiled<BITS, 4>(a, st);
    case 8: return launch_attend_tiled<BITS, 8>(a, st);
  }
  return set_error(AXR_EUNSUPPORTED, "axr_attend_decode: G=%d", G);
}

std::atomic<int> g_gather{kGatherMma};

// Tiled values: the tensor-core (tcgen05) kernel in AXR_GATHER_TENSOR mode, else warp-level MMAs for the values.
template <int BITS, int G>
axr_status launch_attend_tiled(const DecodeArgs& a, cudaStream_t st) {
  if (g_gather.load() == kGatherTensor) return launch_attend_tcv<BITS, G>(a, st);
  return launch_attend_mma<BITS, G>(a, st);
}

axr_status attend_tcv_bits(int bits, int G, const DecodeArgs& a, cudaStream_t st) {
  switch (bits) {
    case 1: return attend_tcv_g<1>(G, a, st);
    case 2: return attend_tcv_g<2>(G, a, st);
    case 3: return attend_tcv_g<3>(G, a, st);
    case 4: return attend_tcv_g<4>(G, a, st);
  }
  return set_error(AXR_EUNSUPPORTED, "axr_attend_decode: bits=%d", bits);
}


template <int D, int BITS, int G>
axr_status launch_score_tc(const DecodeArgs& a, cudaStream_t st) {
  using S = TcScorePlan<D, BITS, G>;
  auto k = score_tc_kernel<D, BITS, G>;
  axr_status rs = ensure_smem(k, S::launch_bytes, "axr_score");
  if (rs != AXR_OK) return rs;
  // one persistent CTA per SM, each taking a contiguous share of the tiles (at most as many CTAs as tiles)
  const long tiles = static_cast<long>(a.B) * a.Hkv * ((a.T + kTile - 1) / kTile);
  const unsigned grid = static_cast<unsigned>(tiles < kSmCount ? tiles : kSmCount);
  k<<<grid, S::THREADS, S::launch_bytes, st>>>(a);
  return check_launch("axr_score");
}

template <int D, int BITS, int G, int MODE>
axr_status launch_score_mode(const DecodeArgs& a, cudaStream_t st) {
  using S = ScorePlan<D, BITS, G, MODE>;
  auto k = score_kernel<D, BITS, G, MODE>;
  axr_status rs = ensure_smem(k, S::bytes, "axr_score");
  if (rs != AXR_OK) return rs;
  dim3 grid(a.splits, a.Hkv, a.B);
  k<<<grid, kDecThreads, S::bytes, st>>>(a);
  return check_launch("axr_score");
}

template <int D, int BITS, int G>
axr_status launch_score_mma(const DecodeArgs& a, cudaStream_t st) {
  using S = ScoreMmaPlan<D, BITS, G>;
  auto k = score_mma_kernel<D, BITS, G>;
  axr_status rs = ensure_smem(k, S::bytes, "axr_score");
  if (rs != AXR_OK) return rs;
  const long items = static_cast<long>(a.B) * a.Hkv * a.splits;  // persistent: two blocks per SM
  const long resident = 2L * kSmCount;
  k<<<static_cast<unsigned>(items < resident ? items : resident), S::THREADS, S::bytes, st>>>(a);
  return check_launch("axr_score");
}

template <int D, int BITS, int G>
axr_status launch_score(const DecodeArgs& a, cudaStream_t st) {
  const int mode = g_gather.load();
  if (mode == kGatherMma) return launch_score_mma<D, BITS, G>(a, st);
  if (mode == kGatherTable) return launch_score_mode<D, BITS, G, kGatherTable>(a, st);
  if (mode == kGatherFactored) return launch_score_mode<D, BITS, G, kGatherFactored>(a, st);
  return launch_score_tc<D, BITS, G>(a, st);
}

template <int D, int BITS>
axr_status attend_g(int G, bool vq, const DecodeArgs& a, cudaStream_t st) {
  const char* w = "axr_attend_decode";
  switch (G) {
    case 1: return vq ? launch_attend<D, BITS, 1, true, false>(a, st, w) : launch_attend<D, BITS, 1, false, false>(a, st, w);
    case 2: return vq ? launch_attend<D, BITS, 2, true, false>(a, st, w) : launch_attend<D, BITS, 2, false, false>(a, st, w);
    case 4: return vq ? launch_attend<D, BITS, 4, true, false>(a, st, w) : launch_attend<D, BITS, 4, false, false>(a, st, w);
    case 8: return vq ? launch_attend<D, BITS, 8, true, false>(a, st, w) : launch_attend<D, BITS, 8, false, false>(a, st, w);
  }
  return set_error(AXR_EUNSUPPORTED, "axr_attend_decode: G=%d", G);
}

template <int D>
axr_status attend_bits(int bits, int G, bool vq, const DecodeArgs& a, cudaStream_t st) {
  switch (bits) {
    case 1: return attend_g<D, 1>(G, vq, a, st);
    case 2: return attend_g<D, 2>(G, vq, a, st);
    case 3: return attend_g<D, 3>(G, vq, a, st);
    case 4: return attend_g<D, 4>(G, vq, a, st);
  }
  return set_error(AXR_EUNSUPPORTED, "axr_attend_decode: bits=%d", bits);
}

template <int D, int BITS>
axr_status score_g(int G, const DecodeArgs& a, cudaStream_t st) {
  switch (G) {
    case 1: return launch_score<D, BITS, 1>(a, st);
    case 2: return launch_score<D, BITS, 2>(a, st);
    case 4: return launch_score<D, BITS, 4>(a, st);
    case 8: return launch_score<D, BITS, 8>(a, st);
  }
  return set_error(AXR_EUNSUPPORTED, "axr_score: G=%d", G);
}

template <int D>
axr_status score_bits(int bits, int G, const DecodeArgs& a, cudaStream_t st) {
  switch (bits) {
    case 1: return score_g<D, 1>(G, a, st);
    case 2: return score_g<D, 2>(G, a, st);
    case 3: return score_g<D, 3>(G, a, st);
    case 4: return score_g<D, 4>(G, a, st);
  }
  return set_error(AXR_EUNSUPPORTED, "axr_score: bits=%d", bits);
}

template <int D>
axr_status dense_g(int G, const DecodeArgs& a, cudaStream_t st) {
  const char* w = "axr_dense_decode";
  switch (G) {
    case 1: return launch_attend<D, 1, 1, false, true>(a, st, w);
    case 2: return launch_attend<D, 1, 2, false, true>(a, st, w);
    case 4: return launch_attend<D, 1, 4, false, true>(a, st, w);
    case 8: return launch_attend<D, 1, 8, false, true>(a, st, w);
  }
  return set_error(AXR_EUNSUPPORTED, "axr_dense_decode: G=%d", G);
}

DecodeArgs base_args(int B, int Hq, int Hkv, int T, int Tcap, const int32_t* seq_lens, const float* q,
                     float mult) {
  DecodeArgs a;
  memset(&a, 0, sizeof(a));
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.T = T; a.Tcap = Tcap;
  a.seq_lens = seq_lens; a.q = q; a.mult = mult;
  const SplitPlan p = plan_splits(B, Hkv, T);
  a.splits = p.splits; a.chunk = p.chunk;
  return a;
}

}  // namespace
}  // namespace axr

extern "C" axr_status axr_score(const float* q, const uint8_t* kcodes, const uint16_t* knorms,
                                const int32_t* seq_lens, int B, int Hq, int Hkv, int T, int Tcap, int d, int bits,
                                const int8_t* signs, float scale, float* scores, void* stream) {
  using namespace axr;
  axr_status st = check_decode_sizes("axr_score", B, Hq, Hkv, T, Tcap, d);
  if (st != AXR_OK) return st;
  if (bits < 1 || bits > 4) return set_error(AXR_EUNSUPPORTED, "axr_score: bits=%d outside 1..4", bits);
  if (B == 0 || T == 0) return set_error(AXR_OK, "");
  if (!q || !kcodes || !knorms || !signs || !scores) return set_error(AXR_EINVAL, "axr_score: null pointer");
  if (!aligned(q, 16) || !aligned(kcodes, 16) || !aligned(knorms, 4) || !aligned(scores, 16) ||
      (seq_lens && !aligned(seq_lens, 4)))
    return set_error(AXR_EINVAL, "axr_score: misaligned pointer");
  if (!std::isfinite(scale)) return set_error(AXR_EINVAL, "axr_score: scale is not finite");
  const Codebook* cb = codebook_for(d, bits);
  if (!cb) return set_error(AXR_EINVAL, "axr_score: codebook unavailable");
  DecodeArgs a = base_args(B, Hq, Hkv, T, Tcap, seq_lens, q, scale);
  a.kcodes = kcodes; a.knorms = reinterpret_cast<const __half*>(knorms); a.signs = signs; a.scores = scores;
  a.cb = *cb;
  const int G = Hq / Hkv;
  return d == 64 ? score_bits<64>(bits, G, a, as_stream(stream)) : score_bits<128>(bits, G, a, as_stream(stream));
}

extern "C" size_t axr_attend_workspace_bytes(int B, int Hq, int Hkv, int T, int d) {
  return axr::attend_ws_bytes(B, Hq, Hkv, T, d);
}

namespace {
axr_status carve_workspace(axr::DecodeArgs& a, int d, void* ws, size_t ws_bytes, const char* what) {
  using namespace axr;
  const size_t need = attend_ws_bytes(a.B, a.Hq, a.Hkv, a.T, d);
  if (!ws || ws_bytes < need)
    return set_error(AXR_EWORKSPACE, "%s: workspace of %zu bytes, need %zu", what, ws ? ws_bytes : 0, need);
  if (!aligned(ws, 16)) return set_error(AXR_EINVAL, "%s: workspace not 16-byte aligned", what);
  const size_t parts = static_cast<size_t>(a.B) * a.Hq * a.splits;
  a.ws_o = static_cast<float*>(ws);
  a.ws_m = a.ws_o + parts * d;
  a.ws_l = a.ws_m + parts;
  return AXR_OK;
}
}  // namespace

extern "C" axr_status axr_attend_decode(const float* q, const uint8_t* kcodes, const uint16_t* knorms,
                                        axr_vkind vkind, const void* v, const uint16_t* vnorms,
                                        const int32_t* seq_lens, int B, int Hq, int Hkv, int T, int Tcap, int d,
                                        int bits, const int8_t* signs, float scale, float* out, void* workspace,
                                        size_t ws_bytes, void* stream) {
  using namespace axr;
  const char* w = "axr_attend_decode";
  axr_status st = check_decode_sizes(w, B, Hq, Hkv, T, Tcap, d);
  if (st != AXR_OK) return st;
  if (bits < 1 || bits > 4) return set_error(AXR_EUNSUPPORTED, "%s: bits=%d outside 1..4", w, bits);
  if (vkind != AXR_V_F16 && vkind != AXR_V_QUANT && vkind != AXR_V_QUANT_TILED)
    return set_error(AXR_EINVAL, "%s: bad vkind", w);
  if (vkind == AXR_V_QUANT_TILED && d != 128)
    return set_error(AXR_EUNSUPPORTED, "%s: tiled values need d = 128 (d=%d)", w, d);
  if (vkind == AXR_V_QUANT_TILED && Tcap % 128)
    return set_error(AXR_EINVAL, "%s: tiled values need Tcap a multiple of 128 (Tcap=%d)", w, Tcap);
  if (B == 0) return set_error(AXR_OK, "");
  if (!q || !kcodes || !knorms || !signs || !v || !out || (vkind != AXR_V_F16 && !vnorms))
    return set_error(AXR_EINVAL, "%s: null pointer", w);
  if (!aligned(q, 16) || !aligned(kcodes, 16) || !aligned(knorms, 4) || !aligned(out, 16) || !aligned(v, 16) ||
      (vnorms && !aligned(vnorms, 4)) || (seq_lens && !aligned(seq_lens, 4)))
    return set_error(AXR_EINVAL, "%s: misaligned pointer", w);
  if (!std::isfinite(scale)) return set_error(AXR_EINVAL, "%s: scale is not finite", w);
  if (T == 0) {
    cudaError_t e = cudaMemsetAsync(out, 0, sizeof(float) * (size_t)B * Hq * d, as_stream(stream));
    return e == cudaSuccess ? set_error(AXR_OK, "") : set_error(AXR_ECUDA, "%s: %s", w, cudaGetErrorString(e));
  }
  const Codebook* cb = codebook_for(d, bits);
  if (!cb) return set_error(AXR_EINVAL, "%s: codebook unavailable", w);
  DecodeArgs a = base_args(B, Hq, Hkv, T, Tcap, seq_lens, q, scale * kLog2e);
  st = carve_workspace(a, d, workspace, ws_bytes, w);
  if (st != AXR_OK) return st;
  a.kcodes = kcodes; a.knorms = reinterpret_cast<const __half*>(knorms); a.signs = signs; a.out = out;
  a.v = v; a.vnorms = reinterpret_cast<const __half*>(vnorms); a.cb = *cb;
  const int G = Hq / Hkv;
  if (vkind == AXR_V_QUANT_TILED) return attend_tcv_bits(bits, G, a, as_stream(stream));
  const bool vq = vkind == AXR_V_QUANT;
  return d == 64 ? attend_bits<64>(bits, G, vq, a, as_stream(stream))
                 : attend_bits<128>(bits, G, vq, a, as_stream(stream));
}

extern "C" axr_status axr_dense_decode(const float* q, const uint16_t* k, const uint16_t* v,
                                       const int32_t* seq_lens, int B, int Hq, int Hkv, int T, int Tcap, int d,
                                       float scale, float* out, void* workspace, size_t ws_bytes, void* stream) {
  using namespace axr;
  const char* w = "axr_dense_decode";
  axr_status st = check_decode_sizes(w, B, Hq, Hkv, T, Tcap, d);
  if (st != AXR_OK) return st;
  if (B == 0) return set_error(AXR_OK, "");
  if (!q || !k || !v || !out) return set_error(AXR_EINVAL, "%s: null pointer", w);
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
      (seq_lens && !aligned(seq_lens, 4)))
    return set_error(AXR_EINVAL, "%s: misaligned pointer", w);
  if (!std::isfinite(scale)) return set_error(AXR_EINVAL, "%s: scale is not finite", w);
  if (T == 0) {
    cudaError_t e = cudaMemsetAsync(out, 0, sizeof(float) * (size_t)B * Hq * d, as_stream(stream));
    return e == cudaSuccess ? set_error(AXR_OK, "") : set_error(AXR_ECUDA, "%s: %s", w, cudaGetErrorString(e));
  }
  DecodeArgs a = base_args(B, Hq, Hkv, T, Tcap, seq_lens, q, scale * kLog2e);
  st = carve_workspace(a, d, workspace, ws_bytes, w);
  if (st != AXR_OK) return st;
  a.kdense = reinterpret_cast<const __half*>(k); a.v = v; a.out = out;
  const int G = Hq / Hkv;
  return d == 64 ? dense_g<64>(G, a, as_stream(stream)) : dense_g<128>(G, a, as_stream(stream));
}

extern "C" axr_status axr_set_gather(axr_gather mode) {
  using namespace axr;
  if (mode == AXR_GATHER_FACTORED) g_gather.store(kGatherFactored);
  else if (mode == AXR_GATHER_TABLE) g_gather.store(kGatherTable);
  else if (mode == AXR_GATHER_TENSOR) g_gather.store(kGatherTensor);
  else if (mode == AXR_GATHER_MMA) g_gather.store(kGatherMma);
  else return set_error(AXR_EINVAL, "axr_set_gather: unknown mode %d", (int)mode);
  return set_error(AXR_OK, "");
}

extern "C" axr_gather axr_get_gather(void) {
  const int m = axr::g_gather.load();
  return m == axr::kGatherTable      ? AXR_GATHER_TABLE
         : m == axr::kGatherFactored ? AXR_GATHER_FACTORED
         : m == axr::kGatherMma      ? AXR_GATHER_MMA
                                     : AXR_GATHER_TENSOR;
}
