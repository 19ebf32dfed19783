// Host entry points of the decode read path: axr_score, axr_attend_decode, axr_dense_decode.
#include <atomic>
#include <cmath>

#include "launch.h"

namespace axr {
namespace {

// ---- common validation -----------------------------------------------------------------------------------------

axr_status check_decode_sizes(const char* what, int B, int Hq, int Hkv, int T, int Tcap, int d) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || T < 0 || Tcap < T)
    return set_error(AXR_EINVAL, "%s: bad sizes B=%d Hq=%d Hkv=%d T=%d Tcap=%d", what, B, Hq, Hkv, T, Tcap);
  if (Hq % Hkv) return set_error(AXR_EINVAL, "%s: Hq=%d is not a multiple of Hkv=%d", what, Hq, Hkv);
  if (d != 64 && d != 128) return set_error(AXR_EUNSUPPORTED, "%s: d=%d not in {64,128}", what, d);
  if (!supported_g(Hq / Hkv)) return set_error(AXR_EUNSUPPORTED, "%s: G=%d not in {1,2,4,8}", what, Hq / Hkv);
  return AXR_OK;
}

std::atomic<int> g_gather{kGatherMma};

DecodeArgs base_args(int B, int Hq, int Hkv, int T, int Tcap, const int32_t* seq_lens, const float* q,
                     float mult) {
  DecodeArgs a;
  memset(&a, 0, sizeof(a));
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.T = T; a.Tcap = Tcap;
  a.seq_lens = seq_lens; a.q = q; a.mult = mult;
  a.status = status_word();
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
  const int mode = g_gather.load();
  if (mode == kGatherTensor) return score_tc_launch(d, bits, G, a, as_stream(stream));
  if (mode == kGatherTable) return table_score_launch(d, bits, G, a, as_stream(stream));
  return score_launch(d, bits, G, mode, a, as_stream(stream));
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

namespace {
// axr_attend_decode, and axr_decode_step when knew / vnew are given (the new token written by the decode launch)
axr_status attend_impl(const char* w, const float* q, const uint8_t* kcodes, const uint16_t* knorms,
                       axr_vkind vkind, const void* v, const uint16_t* vnorms, const int32_t* seq_lens, int B, int Hq,
                       int Hkv, int T, int Tcap, int d, int bits, const int8_t* signs, float scale, float* out,
                       void* workspace, size_t ws_bytes, void* stream, const uint16_t* knew, const uint16_t* vnew,
                       const int32_t* block_table = nullptr, int max_blocks = 0, int block_tokens = 0) {
  using namespace axr;
  const bool step = knew != nullptr || vnew != nullptr;
  const bool paged = block_table != nullptr;
  int shift = 0;
  if (paged) {
    while (shift < 31 && (1 << shift) < block_tokens) ++shift;
    if (block_tokens < 16 || block_tokens > (1 << 20) || (1 << shift) != block_tokens)
      return set_error(AXR_EINVAL, "%s: block_tokens=%d is not a power of two in [16, 2^20]", w, block_tokens);
    if (max_blocks <= 0 || static_cast<long>(T) > static_cast<long>(max_blocks) * block_tokens)
      return set_error(AXR_EINVAL, "%s: T=%d exceeds max_blocks=%d x block_tokens=%d", w, T, max_blocks,
                       block_tokens);
    if (!aligned(block_table, 4)) return set_error(AXR_EINVAL, "%s: misaligned block table", w);
    if (vkind == AXR_V_QUANT_TILED) return set_error(AXR_EINVAL, "%s: paged pools take the row value layouts", w);
    Tcap = T;  // no capacity stride: rows come through the block table
  }
  axr_status st = check_decode_sizes(w, B, Hq, Hkv, T, Tcap, d);
  if (st != AXR_OK) return st;
  if (bits < 1 || bits > 4) return set_error(AXR_EUNSUPPORTED, "%s: bits=%d outside 1..4", w, bits);
  if (vkind != AXR_V_F16 && vkind != AXR_V_QUANT && vkind != AXR_V_QUANT_TILED)
    return set_error(AXR_EINVAL, "%s: bad vkind", w);
  if (vkind == AXR_V_QUANT_TILED && d != 128)
    return set_error(AXR_EUNSUPPORTED, "%s: tiled values need d = 128 (d=%d)", w, d);
  if (vkind == AXR_V_QUANT_TILED && Tcap % 128)
    return set_error(AXR_EINVAL, "%s: tiled values need Tcap a multiple of 128 (Tcap=%d)", w, Tcap);
  if (step && vkind == AXR_V_QUANT_TILED) return set_error(AXR_EINVAL, "%s: the row value layouts only", w);
  if (B == 0) return set_error(AXR_OK, "");
  if (step && (!knew || !vnew)) return set_error(AXR_EINVAL, "%s: null pointer", w);
  if (step && (!aligned(knew, 16) || !aligned(vnew, 16))) return set_error(AXR_EINVAL, "%s: misaligned pointer", w);
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
  const int mode = g_gather.load();
  // row-layout values on a contiguous cache, keys through warp-level MMAs (attend and decode step): the streaming
  // kernel; for quantized values only from 2^18 (token, KV head) units or at eight query heads per KV head, since
  // below that the row kernel's shorter setup measured ahead (B = 1, T = 4096: 21.5 against 25.6 us; the
  // long-context step: 107 against 122 us the other way)
  const bool stream_vq = vkind == AXR_V_QUANT &&
                         (Hq / Hkv == 8 || static_cast<long>(B) * Hkv * T >= (1L << 18));
  // paged pools too, with quantized values in blocks of at least one streaming tile (a tile never spans two blocks)
  const bool stream_path = (vkind == AXR_V_F16 || stream_vq) &&
                           (!paged || (stream_vq && block_tokens >= kStreamTile)) &&
                           attend_stream_supported(d, bits, Tcap) &&
                           (step || mode == kGatherMma || mode == kGatherDirect);
  if (stream_path) {
    const SplitPlan p =
        plan_splits_stream(B, Hkv, T, vkind == AXR_V_QUANT ? kAttendStreamWorkersQ : kAttendStreamWorkers);
    a.splits = p.splits; a.chunk = p.chunk;
  }
  st = carve_workspace(a, d, workspace, ws_bytes, w);
  if (st != AXR_OK) return st;
  a.kcodes = kcodes; a.knorms = reinterpret_cast<const __half*>(knorms); a.signs = signs; a.out = out;
  a.v = v; a.vnorms = reinterpret_cast<const __half*>(vnorms); a.cb = *cb;
  a.knew = reinterpret_cast<const __half*>(knew); a.vnew = reinterpret_cast<const __half*>(vnew);
  const int G = Hq / Hkv;
  const bool vq = vkind == AXR_V_QUANT;
  if (paged) {
    a.block_table = block_table; a.max_blocks = max_blocks; a.block_shift = shift;
  }
  if (stream_path) return attend_stream_launch(d, bits, G, vq, a, as_stream(stream), w);
  // decode step and paged pools: the kernel that writes the new token in its prologue and reads rows through the
  // block table (scores through warp-level MMAs)
  if (step || paged) return attend_rows_launch(d, bits, G, vq, a, as_stream(stream));
  // tiled values: the tcgen05 kernel in AXR_GATHER_TENSOR mode, else warp-level MMAs for keys and values
  if (vkind == AXR_V_QUANT_TILED) return attend_tiled_launch(bits, G, mode == kGatherTensor, a, as_stream(stream));
  // fp16 values in AXR_GATHER_TABLE mode: the literal table in shared memory, values on the CUDA cores
  if (mode == kGatherTable && !vq) return table_attend_launch(d, bits, G, a, as_stream(stream));
  // row-layout values the streaming kernel does not take: keys scored through warp-level MMAs in AXR_GATHER_MMA
  // mode (scoring and value warps one tile apart), else on CUDA cores
  if (mode == kGatherMma || mode == kGatherDirect) return attend_rows_launch(d, bits, G, vq, a, as_stream(stream));
  return attend_partial_launch(d, bits, G, vq, a, as_stream(stream), w);
}
}  // namespace

extern "C" axr_status axr_attend_decode(const float* q, const uint8_t* kcodes, const uint16_t* knorms,
                                        axr_vkind vkind, const void* v, const uint16_t* vnorms,
                                        const int32_t* seq_lens, int B, int Hq, int Hkv, int T, int Tcap, int d,
                                        int bits, const int8_t* signs, float scale, float* out, void* workspace,
                                        size_t ws_bytes, void* stream) {
  return attend_impl("axr_attend_decode", q, kcodes, knorms, vkind, v, vnorms, seq_lens, B, Hq, Hkv, T, Tcap, d,
                     bits, signs, scale, out, workspace, ws_bytes, stream, nullptr, nullptr);
}

extern "C" axr_status axr_decode_step(const float* q, const uint16_t* k_new, const uint16_t* v_new, uint8_t* kcodes,
                                      uint16_t* knorms, axr_vkind vkind, void* v, uint16_t* vnorms,
                                      const int32_t* seq_lens, int B, int Hq, int Hkv, int T, int Tcap, int d,
                                      int bits, const int8_t* signs, float scale, float* out, void* workspace,
                                      size_t ws_bytes, void* stream) {
  if (!k_new || !v_new) return axr::set_error(AXR_EINVAL, "axr_decode_step: null pointer");
  return attend_impl("axr_decode_step", q, kcodes, knorms, vkind, v, vnorms, seq_lens, B, Hq, Hkv, T, Tcap, d, bits,
                     signs, scale, out, workspace, ws_bytes, stream, k_new, v_new);
}

extern "C" axr_status axr_attend_decode_paged(const float* q, const uint8_t* kcodes, const uint16_t* knorms,
                                              axr_vkind vkind, const void* v, const uint16_t* vnorms,
                                              const int32_t* block_table, int max_blocks, int block_tokens,
                                              const int32_t* seq_lens, int B, int Hq, int Hkv, int T, int d,
                                              int bits, const int8_t* signs, float scale, float* out,
                                              void* workspace, size_t ws_bytes, void* stream) {
  if (!block_table) return axr::set_error(AXR_EINVAL, "axr_attend_decode_paged: null block table");
  return attend_impl("axr_attend_decode_paged", q, kcodes, knorms, vkind, v, vnorms, seq_lens, B, Hq, Hkv, T, T, d,
                     bits, signs, scale, out, workspace, ws_bytes, stream, nullptr, nullptr, block_table, max_blocks,
                     block_tokens);
}

extern "C" axr_status axr_decode_step_paged(const float* q, const uint16_t* k_new, const uint16_t* v_new,
                                            uint8_t* kcodes, uint16_t* knorms, axr_vkind vkind, void* v,
                                            uint16_t* vnorms, const int32_t* block_table, int max_blocks,
                                            int block_tokens, const int32_t* seq_lens, int B, int Hq, int Hkv, int T,
                                            int d, int bits, const int8_t* signs, float scale, float* out,
                                            void* workspace, size_t ws_bytes, void* stream) {
  if (!k_new || !v_new) return axr::set_error(AXR_EINVAL, "axr_decode_step_paged: null pointer");
  if (!block_table) return axr::set_error(AXR_EINVAL, "axr_decode_step_paged: null block table");
  return attend_impl("axr_decode_step_paged", q, kcodes, knorms, vkind, v, vnorms, seq_lens, B, Hq, Hkv, T, T, d,
                     bits, signs, scale, out, workspace, ws_bytes, stream, k_new, v_new, block_table, max_blocks,
                     block_tokens);
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
  const SplitPlan p = plan_splits_stream(B, Hkv, T, kDenseWorkers);
  a.splits = p.splits; a.chunk = p.chunk;
  st = carve_workspace(a, d, workspace, ws_bytes, w);
  if (st != AXR_OK) return st;
  a.kdense = reinterpret_cast<const __half*>(k); a.v = v; a.out = out;
  return dense_launch(d, Hq / Hkv, a, as_stream(stream), w);
}

extern "C" axr_status axr_set_gather(axr_gather mode) {
  using namespace axr;
  if (mode == AXR_GATHER_FACTORED) g_gather.store(kGatherFactored);
  else if (mode == AXR_GATHER_TABLE) g_gather.store(kGatherTable);
  else if (mode == AXR_GATHER_TENSOR) g_gather.store(kGatherTensor);
  else if (mode == AXR_GATHER_MMA) g_gather.store(kGatherMma);
  else if (mode == AXR_GATHER_DIRECT) g_gather.store(kGatherDirect);
  else return set_error(AXR_EINVAL, "axr_set_gather: unknown mode %d", (int)mode);
  return set_error(AXR_OK, "");
}

extern "C" axr_gather axr_get_gather(void) {
  const int m = axr::g_gather.load();
  return m == axr::kGatherTable      ? AXR_GATHER_TABLE
         : m == axr::kGatherFactored ? AXR_GATHER_FACTORED
         : m == axr::kGatherMma      ? AXR_GATHER_MMA
         : m == axr::kGatherDirect   ? AXR_GATHER_DIRECT
                                     : AXR_GATHER_TENSOR;
}
