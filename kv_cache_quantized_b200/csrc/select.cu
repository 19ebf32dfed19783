// Sign-pattern selection (AXELRAM Key Points, 4th item; Abstract): a one-time, gradient-free choice among candidate
// sign vectors on a few calibration sequences.  Objective per candidate: attention-output MSE of quantized-K
// attention against fp64 unquantized attention, over every (layer, sequence, query head, position, coordinate).
//
// Pipeline per call:
//   1. reference: causal (or full) softmax attention of the calibration Q/K/V in fp64 -> o_ref (workspace);
//   2. for each chunk of candidates: every key row goes through the same write path as axr_write_keys (fp32 norm,
//      sign flip, Walsh-Hadamard, threshold count, fp16 norm) and is reconstructed in the original domain,
//      k^ = s .* H(n16 * c[idx]) -- for a prefill-shaped calibration set this is the cheap direction (one transform
//      per key instead of one per query), and q . k^ equals the table score exactly up to rounding;
//   3. attention with k^, squared error against o_ref accumulated in fp64 per (candidate, layer, sequence): on the
//      tensor cores for d = 64 and 128 (select_tc.cuh: hi/lo fp16 planes of q and k^, three products per step, fp32
//      accumulation), on the CUDA cores in fp32 for d = 8;
//   4. mse = sum / count, best = first index of the minimum: over every layer (one sign vector for the model), or
//      per layer (one sign vector per layer, axr_select_signs_per_layer).
#include <cmath>

#include "axr_host.h"
#include "select_tc.cuh"

namespace axr {
namespace {

constexpr int kSelThreads = 256;
constexpr int kCandChunk = 8;

struct SelArgs {
  const float* q;       // [Ly, S, Hq, N, D]
  const __half* k;      // [Ly, S, Hkv, N, D]
  const __half* v;      // [Ly, S, Hkv, N, D]
  const int8_t* cand;   // [C, D]
  double* oref;         // [Ly, S, Hq, N, D]
  float* khat;          // [chunk, Ly, S, Hkv, N, D] f32 (d = 8), or the hi then lo fp16 planes of it (d >= 64)
  double* acc;          // [C, Ly, S] squared-error sums
  double* mse;          // [C], or [Ly, C] per layer
  int32_t* best;        // [1], or [Ly] per layer
  double* parts;        // [Ly, S, C] per-(layer, sequence) MSEs, or null
  int Ly, S, Hq, Hkv, N, C;
  int c0, nc;           // candidate chunk [c0, c0 + nc)
  int D_;               // head dim (for the finalize kernel)
  int causal;
  Codebook cb;
};

// ---- step 2: write path + reconstruction, one warp per key row ----------------------------------------------------

template <int D, int BITS, bool PLANES>
__global__ void __launch_bounds__(256) requantize_kernel(const __grid_constant__ SelArgs a) {
  constexpr int VPL = WarpVec<D>::VPL;
  constexpr int LANES = WarpVec<D>::LANES;
  constexpr int L = 1 << BITS;
  const int lane = threadIdx.x & 31;
  const size_t rows_per_cand = static_cast<size_t>(a.Ly) * a.S * a.Hkv * a.N;
  const size_t total = rows_per_cand * a.nc;
  const bool active = lane < LANES;
  const float nrm = rsqrtf(static_cast<float>(D));
  for (size_t r = (static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x) / kWarp; r < total;
       r += static_cast<size_t>(gridDim.x) * blockDim.x / kWarp) {
    const size_t ci = r / rows_per_cand, row = r % rows_per_cand;
    const int8_t* s = a.cand + static_cast<size_t>(a.c0 + ci) * D;
    float v[VPL], sg[VPL];
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int j = lane * VPL + i;
      v[i] = active ? __half2float(a.k[row * D + j]) : 0.f;
      sg[i] = active ? sign_of(s[j]) : 0.f;
      ss = fmaf(v[i], v[i], ss);
      v[i] *= sg[i];
    }
    ss = warp_sum(ss);
    const float n = sqrtf(ss);
    const float n16 = __half2float(__float2half_rn(n));
    fwht_warp<D>(v, lane);
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const float w = n > 0.f ? v[i] / n : 0.f;
      int q = 0;
#pragma unroll
      for (int kk = 0; kk < L - 1; ++kk) q += (w >= a.cb.tau[kk]) ? 1 : 0;
      v[i] = n16 * a.cb.c[q];
    }
    fwht_warp<D>(v, lane);
    if (active) {
      if constexpr (PLANES) {  // hi and lo fp16 planes for the tensor-core attention
        __half* kh = reinterpret_cast<__half*>(a.khat);
        __half* kl = kh + total * D;
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
          const float x = v[i] * nrm * sg[i];
          const __half hi = __float2half_rn(x);
          kh[r * D + lane * VPL + i] = hi;
          kl[r * D + lane * VPL + i] = __float2half_rn(x - __half2float(hi));
        }
      } else {
#pragma unroll
        for (int i = 0; i < VPL; ++i) a.khat[r * D + lane * VPL + i] = v[i] * nrm * sg[i];
      }
    }
  }
}

// ---- steps 1 and 3: tiled softmax attention (SIMT), one block per (query tile, query head, layer*seq[*cand]) ------
//
// 256 threads as a 16 x 16 grid: thread (ty, tx) owns score rows [4ty, 4ty+4) x columns [4tx, 4tx+4) of each
// BQ x BK tile and output rows [4ty, 4ty+4) x coordinates [tx*OC, tx*OC+OC).  Rows of one query are held by 16
// consecutive lanes (a half warp), so the row max and sum are half-warp shuffles.

template <typename T> __device__ __forceinline__ T ex(T x);
template <> __device__ __forceinline__ float ex<float>(float x) { return expf(x); }
template <> __device__ __forceinline__ double ex<double>(double x) { return exp(x); }

template <typename T>
__device__ __forceinline__ T half_warp_max(T v) {
#pragma unroll
  for (int m = 8; m > 0; m >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, m));
  return v;
}
template <typename T>
__device__ __forceinline__ T half_warp_sum(T v) {
#pragma unroll
  for (int m = 8; m > 0; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
  return v;
}

template <int D, typename Acc, bool REF>
struct AttnCfg {
  static constexpr int BQ = 64, BK = 64;
  static constexpr int OC = D >= 16 ? D / 16 : 1;
  static constexpr size_t smem = sizeof(Acc) * (size_t)(D * BQ + D * BK + BK * D + BQ * (BK + 1));
};

template <int D, typename Acc, bool REF>
__global__ void __launch_bounds__(kSelThreads) select_attention_kernel(const __grid_constant__ SelArgs a) {
  using C = AttnCfg<D, Acc, REF>;
  constexpr int BQ = C::BQ, BK = C::BK, OC = C::OC;
  extern __shared__ float4 sel_smem[];
  Acc* Qt = reinterpret_cast<Acc*>(sel_smem);  // [D][BQ]
  Acc* Kt = Qt + D * BQ;                       // [D][BK]
  Acc* Vs = Kt + D * BK;                       // [BK][D]
  Acc* Ps = Vs + BK * D;                       // [BQ][BK + 1]

  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int q0 = blockIdx.x * BQ, h = blockIdx.y;
  const int ls = blockIdx.z % (a.Ly * a.S);
  const int ci = blockIdx.z / (a.Ly * a.S);  // candidate within the chunk (0 for the reference)
  const int G = a.Hq / a.Hkv, hk = h / G;
  const size_t qrow0 = (static_cast<size_t>(ls) * a.Hq + h) * a.N;
  const size_t krow0 = (static_cast<size_t>(ls) * a.Hkv + hk) * a.N;
  const size_t rows_per_cand = static_cast<size_t>(a.Ly) * a.S * a.Hkv * a.N;
  const Acc scale = Acc(1) / sqrt(Acc(D));

  for (int e = tid; e < BQ * D; e += kSelThreads) {
    const int r = e / D, j = e % D;
    Qt[j * BQ + r] = (q0 + r < a.N) ? Acc(a.q[(qrow0 + q0 + r) * D + j]) : Acc(0);
  }
  Acc o[4][OC], m[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m[i] = -INFINITY;
    l[i] = 0;
#pragma unroll
    for (int c = 0; c < OC; ++c) o[i][c] = 0;
  }
  const int kend = a.causal ? min(a.N, q0 + BQ) : a.N;
  for (int k0 = 0; k0 < kend; k0 += BK) {
    __syncthreads();
    for (int e = tid; e < BK * D; e += kSelThreads) {
      const int r = e / D, j = e % D;
      const bool in = k0 + r < a.N;
      Acc kv;
      if constexpr (REF) kv = in ? Acc(__half2float(a.k[(krow0 + k0 + r) * D + j])) : Acc(0);
      else kv = in ? Acc(a.khat[(static_cast<size_t>(ci) * rows_per_cand + krow0 + k0 + r) * D + j]) : Acc(0);
      Kt[j * BK + r] = kv;
      Vs[r * D + j] = in ? Acc(__half2float(a.v[(krow0 + k0 + r) * D + j])) : Acc(0);
    }
    __syncthreads();
    Acc s[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) s[i][jj] = 0;
#pragma unroll 4
    for (int j = 0; j < D; ++j) {
      Acc qa[4], ka[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { qa[i] = Qt[j * BQ + 4 * ty + i]; ka[i] = Kt[j * BK + 4 * tx + i]; }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) s[i][jj] = fma(qa[i], ka[jj], s[i][jj]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int qi = q0 + 4 * ty + i;
      Acc mx = -INFINITY;
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int kj = k0 + 4 * tx + jj;
        const bool valid = kj < a.N && (!a.causal || kj <= qi);
        s[i][jj] = valid ? s[i][jj] * scale : Acc(-INFINITY);
        mx = fmax(mx, s[i][jj]);
      }
      mx = half_warp_max(mx);
      const Acc m_new = fmax(m[i], mx);
      const Acc alpha = (m_new == Acc(-INFINITY)) ? Acc(1) : ex<Acc>(m[i] - m_new);
      Acc rs = 0;
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const Acc p = (s[i][jj] == Acc(-INFINITY)) ? Acc(0) : ex<Acc>(s[i][jj] - m_new);
        Ps[(4 * ty + i) * (BK + 1) + 4 * tx + jj] = p;
        rs += p;
      }
      rs = half_warp_sum(rs);
      l[i] = l[i] * alpha + rs;
      m[i] = m_new;
#pragma unroll
      for (int c = 0; c < OC; ++c) o[i][c] *= alpha;
    }
    __syncthreads();
#pragma unroll 4
    for (int kk = 0; kk < BK; ++kk) {
      Acc pv[4], vv[OC];
#pragma unroll
      for (int i = 0; i < 4; ++i) pv[i] = Ps[(4 * ty + i) * (BK + 1) + kk];
#pragma unroll
      for (int c = 0; c < OC; ++c) {
        const int col = tx * OC + c;
        vv[c] = col < D ? Vs[kk * D + col] : Acc(0);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int c = 0; c < OC; ++c) o[i][c] = fma(pv[i], vv[c], o[i][c]);
    }
  }
  // epilogue
  double err = 0.0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int qi = q0 + 4 * ty + i;
    if (qi >= a.N) continue;
    const Acc inv = l[i] > Acc(0) ? Acc(1) / l[i] : Acc(0);
#pragma unroll
    for (int c = 0; c < OC; ++c) {
      const int col = tx * OC + c;
      if (col >= D) continue;
      const size_t idx = (qrow0 + qi) * D + col;
      if constexpr (REF) {
        a.oref[idx] = static_cast<double>(o[i][c] * inv);
      } else {
        const double dlt = static_cast<double>(o[i][c] * inv) - a.oref[idx];
        err += dlt * dlt;
      }
    }
  }
  if constexpr (!REF) {
#pragma unroll
    for (int msk = 16; msk > 0; msk >>= 1) err += __shfl_xor_sync(0xffffffffu, err, msk);
    __shared__ double werr[kSelThreads / kWarp];
    if ((tid & 31) == 0) werr[tid >> 5] = err;
    __syncthreads();
    if (tid == 0) {
      double t = 0.0;
      for (int w = 0; w < kSelThreads / kWarp; ++w) t += werr[w];
      atomicAdd(a.acc + static_cast<size_t>(a.c0 + ci) * a.Ly * a.S + ls, t);
    }
  }
}

// MSEs from the per-(candidate, layer, sequence) sums (each over Hq * N * D elements), summed in a fixed order.
// per_layer: mse [Ly, C] and best [Ly] (one pick per layer); else mse [C] over every layer and best [1].
__global__ void select_finalize_kernel(const __grid_constant__ SelArgs a, int per_layer) {
  const double per_part = static_cast<double>(a.Hq) * a.N * a.D_;
  const int groups = per_layer ? a.Ly : 1;
  const int lpg = per_layer ? 1 : a.Ly;  // layers per group
  for (int i = threadIdx.x; i < groups * a.C; i += blockDim.x) {
    const int g = i / a.C, c = i % a.C;
    const double* acc = a.acc + static_cast<size_t>(c) * a.Ly * a.S;
    double t = 0.0;
    for (int l = g * lpg; l < (g + 1) * lpg; ++l)
      for (int sq = 0; sq < a.S; ++sq) t += acc[l * a.S + sq];
    a.mse[i] = t / (per_part * lpg * a.S);
  }
  if (a.parts)
    for (int i = threadIdx.x; i < a.Ly * a.S * a.C; i += blockDim.x) {
      const int c = i % a.C, ls = i / a.C;
      a.parts[i] = a.acc[static_cast<size_t>(c) * a.Ly * a.S + ls] / per_part;
    }
  __syncthreads();
  for (int g = threadIdx.x; g < groups; g += blockDim.x) {
    int best = 0;
    double bv = INFINITY;
    for (int c = 0; c < a.C; ++c) {
      const double m = a.mse[g * a.C + c];
      if (m < bv) { bv = m; best = c; }
    }
    a.best[g] = best;
  }
}

struct SelLayout {
  size_t oref, khat, acc, total;
};

SelLayout sel_layout(int Ly, int S, int N, int Hq, int Hkv, int d, int C) {
  SelLayout L{};
  const size_t qn = static_cast<size_t>(Ly) * S * Hq * N * d;
  const size_t kn = static_cast<size_t>(Ly) * S * Hkv * N * d;
  const int chunk = C < kCandChunk ? C : kCandChunk;
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  L.oref = 0;
  L.khat = up(qn * sizeof(double));
  L.acc = L.khat + up(kn * chunk * sizeof(float));
  L.total = L.acc + up(static_cast<size_t>(C) * Ly * S * sizeof(double));
  return L;
}

template <int D, int BITS>
axr_status run_select(SelArgs a, int per_layer, cudaStream_t st) {
  using RC = AttnCfg<D, double, true>;
  using FC = AttnCfg<D, float, false>;
  auto kref = select_attention_kernel<D, double, true>;
  auto kq = select_attention_kernel<D, float, false>;
  cudaError_t e = cudaFuncSetAttribute(kref, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)RC::smem);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)FC::smem);
  if (e != cudaSuccess) return set_error(AXR_ECUDA, "axr_select_signs: %s", cudaGetErrorString(e));
  if (e == cudaSuccess && D >= 64)
    e = cudaFuncSetAttribute(select_attn_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)SelTcPlan<D>::bytes);
  if (e != cudaSuccess) return set_error(AXR_ECUDA, "axr_select_signs: %s", cudaGetErrorString(e));
  e = cudaMemsetAsync(a.acc, 0, sizeof(double) * a.C * a.Ly * a.S, st);
  if (e != cudaSuccess) return set_error(AXR_ECUDA, "axr_select_signs: %s", cudaGetErrorString(e));
  const int qtiles = (a.N + RC::BQ - 1) / RC::BQ;
  a.c0 = 0;
  a.nc = 1;
  kref<<<dim3(qtiles, a.Hq, a.Ly * a.S), kSelThreads, RC::smem, st>>>(a);
  axr_status rs = check_launch("axr_select_signs (reference)");
  if (rs != AXR_OK) return rs;
  const size_t rows = static_cast<size_t>(a.Ly) * a.S * a.Hkv * a.N;
  for (int c0 = 0; c0 < a.C; c0 += kCandChunk) {
    a.c0 = c0;
    a.nc = (a.C - c0) < kCandChunk ? (a.C - c0) : kCandChunk;
    size_t warps = rows * a.nc;
    size_t blocks = (warps + 7) / 8;
    if (blocks > static_cast<size_t>(kSmCount) * 32) blocks = static_cast<size_t>(kSmCount) * 32;
    if constexpr (D >= 64) {
      requantize_kernel<D, BITS, true><<<static_cast<unsigned>(blocks), 256, 0, st>>>(a);
      const __half* kh = reinterpret_cast<const __half*>(a.khat);
      const __half* kl = kh + rows * a.nc * D;
      select_attn_tc_kernel<D><<<dim3(qtiles, a.Hq, a.Ly * a.S * a.nc), SelTcPlan<D>::THREADS,
                                  SelTcPlan<D>::bytes, st>>>(a.q, kh, kl, a.v, a.oref, a.acc, a.Ly, a.S, a.Hq,
                                                             a.Hkv, a.N, a.c0, a.causal);
    } else {
      requantize_kernel<D, BITS, false><<<static_cast<unsigned>(blocks), 256, 0, st>>>(a);
      kq<<<dim3(qtiles, a.Hq, a.Ly * a.S * a.nc), kSelThreads, FC::smem, st>>>(a);
    }
    rs = check_launch("axr_select_signs (candidates)");
    if (rs != AXR_OK) return rs;
  }
  a.D_ = D;
  select_finalize_kernel<<<1, 256, 0, st>>>(a, per_layer);
  return check_launch("axr_select_signs (finalize)");
}

template <int D>
axr_status select_bits(int bits, const SelArgs& a, int per_layer, cudaStream_t st) {
  switch (bits) {
    case 1: return run_select<D, 1>(a, per_layer, st);
    case 2: return run_select<D, 2>(a, per_layer, st);
    case 3: return run_select<D, 3>(a, per_layer, st);
    case 4: return run_select<D, 4>(a, per_layer, st);
  }
  return set_error(AXR_EUNSUPPORTED, "axr_select_signs: bits=%d", bits);
}

axr_status select_impl(const char* w, const float* q, const uint16_t* k, const uint16_t* v, int n_layers, int n_seq,
                       int n_tok, int Hq, int Hkv, int d, int bits, const int8_t* candidates, int n_cand, int causal,
                       double* mse_out, int32_t* best_out, double* parts_out, int per_layer, void* workspace,
                       size_t ws_bytes, void* stream) {
  if (n_layers <= 0 || n_seq <= 0 || n_tok <= 0 || Hq <= 0 || Hkv <= 0 || n_cand <= 0)
    return set_error(AXR_EINVAL, "%s: sizes must be positive", w);
  if (Hq % Hkv) return set_error(AXR_EINVAL, "%s: Hq=%d not a multiple of Hkv=%d", w, Hq, Hkv);
  if (d != 8 && d != 64 && d != 128) return set_error(AXR_EUNSUPPORTED, "%s: d=%d not in {8,64,128}", w, d);
  if (bits < 1 || bits > 4) return set_error(AXR_EUNSUPPORTED, "%s: bits=%d outside 1..4", w, bits);
  if (!q || !k || !v || !candidates || !mse_out || !best_out) return set_error(AXR_EINVAL, "%s: null pointer", w);
  if (!aligned(q, d >= 64 ? 16 : 4) || !aligned(k, 2) || !aligned(v, d >= 64 ? 16 : 2) || !aligned(mse_out, 8) ||
      !aligned(best_out, 4) || (parts_out && !aligned(parts_out, 8)))
    return set_error(AXR_EINVAL, "%s: misaligned pointer", w);
  const SelLayout L = sel_layout(n_layers, n_seq, n_tok, Hq, Hkv, d, n_cand);
  if (!workspace || ws_bytes < L.total)
    return set_error(AXR_EWORKSPACE, "%s: workspace of %zu bytes, need %zu", w, workspace ? ws_bytes : 0, L.total);
  if (!aligned(workspace, 16)) return set_error(AXR_EINVAL, "%s: workspace not 16-byte aligned", w);
  const Codebook* cb = codebook_for(d, bits);
  if (!cb) return set_error(AXR_EINVAL, "%s: codebook unavailable", w);
  SelArgs a;
  memset(&a, 0, sizeof(a));
  char* base = static_cast<char*>(workspace);
  a.q = q; a.k = reinterpret_cast<const __half*>(k); a.v = reinterpret_cast<const __half*>(v);
  a.cand = candidates; a.mse = mse_out; a.best = best_out; a.parts = parts_out;
  a.oref = reinterpret_cast<double*>(base + L.oref);
  a.khat = reinterpret_cast<float*>(base + L.khat);
  a.acc = reinterpret_cast<double*>(base + L.acc);
  a.Ly = n_layers; a.S = n_seq; a.Hq = Hq; a.Hkv = Hkv; a.N = n_tok; a.C = n_cand; a.causal = causal ? 1 : 0;
  a.cb = *cb;
  cudaStream_t st = as_stream(stream);
  switch (d) {
    case 8: return select_bits<8>(bits, a, per_layer, st);
    case 64: return select_bits<64>(bits, a, per_layer, st);
    default: return select_bits<128>(bits, a, per_layer, st);
  }
}

}  // namespace
}  // namespace axr

extern "C" size_t axr_select_workspace_bytes(int n_layers, int n_seq, int n_tok, int Hq, int Hkv, int d,
                                             int n_cand) {
  if (n_layers <= 0 || n_seq <= 0 || n_tok <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || n_cand <= 0) return 0;
  return axr::sel_layout(n_layers, n_seq, n_tok, Hq, Hkv, d, n_cand).total;
}

extern "C" axr_status axr_select_signs(const float* q, const uint16_t* k, const uint16_t* v, int n_layers, int n_seq,
                                       int n_tok, int Hq, int Hkv, int d, int bits, const int8_t* candidates,
                                       int n_cand, int causal, double* mse_out, int32_t* best_out, void* workspace,
                                       size_t ws_bytes, void* stream) {
  return axr::select_impl("axr_select_signs", q, k, v, n_layers, n_seq, n_tok, Hq, Hkv, d, bits, candidates, n_cand,
                          causal, mse_out, best_out, nullptr, 0, workspace, ws_bytes, stream);
}

extern "C" axr_status axr_select_signs_per_layer(const float* q, const uint16_t* k, const uint16_t* v, int n_layers,
                                                 int n_seq, int n_tok, int Hq, int Hkv, int d, int bits,
                                                 const int8_t* candidates, int n_cand, int causal,
                                                 double* mse_layers_out, int32_t* best_layers_out,
                                                 double* mse_parts_out, void* workspace, size_t ws_bytes,
                                                 void* stream) {
  return axr::select_impl("axr_select_signs_per_layer", q, k, v, n_layers, n_seq, n_tok, Hq, Hkv, d, bits,
                          candidates, n_cand, causal, mse_layers_out, best_layers_out, mse_parts_out, 1, workspace,
                          ws_bytes, stream);
}
