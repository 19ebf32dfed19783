// LOOKAT write path: product-quantization encoding of keys and the k-means that learns the codebooks.
//
// Source: the newx.sg summary and abstract of "LOOKAT: Lookup-Optimized Key-Attention for Memory-Efficient
// Transformers" -- keys are decomposed into subspaces, a codebook is learned per subspace, and keys are stored as
// codebook indices.  A key's subspace i is its coordinates [i d/m, (i+1) d/m); its index there is the nearest
// centroid by squared Euclidean distance, lowest index on a tie.  The distance is formed in fp32 in a fixed order:
// sum over j = 0, 1, ... of (x_j - c_j)^2 with every subtraction, product and sum rounded separately (no fused
// multiply-add), so that the integer it decides is reproducible.  k-means: Lloyd's iterations, each an assignment
// by that rule, then every centroid with members moved to their mean (summed in fp64, rounded to fp32); a centroid
// without members stays.
#include <cmath>

#include "axr_host.h"

namespace axr {
namespace {

constexpr int kPqThreads = 256;

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__half>(__half x) { return __half2float(x); }

// Nearest centroid of the DS-long subvector xs among cb [K][DS] (global, read through the cache), and its distance.
template <int DS>
__device__ __forceinline__ int pq_nearest(const float (&xs)[DS], const float* __restrict__ cb, int K) {
  int best = 0;
  float bd = INFINITY;
  for (int k = 0; k < K; ++k) {
    const float* c = cb + static_cast<size_t>(k) * DS;
    float acc = 0.f;
#pragma unroll
    for (int j = 0; j < DS; ++j) {
      const float diff = __fsub_rn(xs[j], __ldg(c + j));
      acc = __fadd_rn(acc, __fmul_rn(diff, diff));
    }
    if (acc < bd) {
      bd = acc;
      best = k;
    }
  }
  return best;
}

struct PqEncArgs {
  const void* x;
  int64_t n_vec;
  int m, K;
  const float* cb;        // [H, m, K, DS]
  int head_period, heads;  // vector r uses codebook set (r / head_period) % heads
  const int64_t* dst_rows;
  uint8_t* codes;         // [rows, m]
  // training
  double* sums;           // [m, K, DS]
  unsigned int* counts;   // [m, K]
};

// One thread per (vector, subspace): grid.y = subspace.
template <int DS, typename T, bool TRAIN>
__global__ void __launch_bounds__(kPqThreads) pq_encode_kernel(const __grid_constant__ PqEncArgs a) {
  const int i = blockIdx.y;
  const int d = DS * a.m;
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * kPqThreads + threadIdx.x; r < a.n_vec;
       r += static_cast<int64_t>(gridDim.x) * kPqThreads) {
    const T* src = static_cast<const T*>(a.x) + r * d + i * DS;
    float xs[DS];
#pragma unroll
    for (int j = 0; j < DS; ++j) xs[j] = to_f32<T>(src[j]);
    const int head = static_cast<int>((r / a.head_period) % a.heads);
    const float* cb = a.cb + (static_cast<size_t>(head) * a.m + i) * a.K * DS;
    const int k = pq_nearest<DS>(xs, cb, a.K);
    if constexpr (TRAIN) {
      double* s = a.sums + (static_cast<size_t>(i) * a.K + k) * DS;
#pragma unroll
      for (int j = 0; j < DS; ++j) atomicAdd(s + j, static_cast<double>(xs[j]));
      atomicAdd(a.counts + static_cast<size_t>(i) * a.K + k, 1u);
    } else {
      const int64_t row = a.dst_rows ? a.dst_rows[r] : r;
      a.codes[row * a.m + i] = static_cast<uint8_t>(k);
    }
  }
}

// Lloyd update: every centroid with members moves to their mean; the others stay.
__global__ void pq_update_kernel(float* cb, const double* sums, const unsigned int* counts, int m, int K, int DS) {
  const int n = m * K * DS;
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < n; e += gridDim.x * blockDim.x) {
    const unsigned int c = counts[e / DS];
    if (c) cb[e] = static_cast<float>(sums[e] / static_cast<double>(c));
  }
}

template <int DS, typename T, bool TRAIN>
axr_status launch_encode(const PqEncArgs& a, cudaStream_t st, const char* what) {
  long blocks = static_cast<long>((a.n_vec + kPqThreads - 1) / kPqThreads);
  if (blocks > 4L * kSmCount * 8) blocks = 4L * kSmCount * 8;
  if (blocks < 1) blocks = 1;
  pq_encode_kernel<DS, T, TRAIN><<<dim3(static_cast<unsigned>(blocks), a.m), kPqThreads, 0, st>>>(a);
  return check_launch(what);
}

template <typename T, bool TRAIN>
axr_status encode_ds(int ds, const PqEncArgs& a, cudaStream_t st, const char* what) {
  switch (ds) {
    case 4: return launch_encode<4, T, TRAIN>(a, st, what);
    case 8: return launch_encode<8, T, TRAIN>(a, st, what);
    case 16: return launch_encode<16, T, TRAIN>(a, st, what);
    case 32: return launch_encode<32, T, TRAIN>(a, st, what);
    case 64: return launch_encode<64, T, TRAIN>(a, st, what);
  }
  return set_error(AXR_EUNSUPPORTED, "%s: subspace width %d not in {4, 8, 16, 32, 64}", what, ds);
}

axr_status pq_sizes(const char* w, int d, int m, int K) {
  if (d != 64 && d != 128) return set_error(AXR_EUNSUPPORTED, "%s: d=%d not in {64,128}", w, d);
  if (m != 2 && m != 4 && m != 8 && m != 16) return set_error(AXR_EUNSUPPORTED, "%s: m=%d not in {2,4,8,16}", w, m);
  if (K < 1 || K > 256) return set_error(AXR_EUNSUPPORTED, "%s: K=%d outside 1..256", w, K);
  return AXR_OK;
}

}  // namespace
}  // namespace axr

extern "C" axr_status axr_pq_encode(const void* x, axr_dtype x_dtype, int64_t n_vec, int d, int m, int K,
                                    const float* codebooks, int heads, int head_period, const int64_t* dst_rows,
                                    uint8_t* codes, void* stream) {
  using namespace axr;
  const char* w = "axr_pq_encode";
  axr_status st = pq_sizes(w, d, m, K);
  if (st != AXR_OK) return st;
  if (n_vec < 0 || heads < 1 || head_period < 1) return set_error(AXR_EINVAL, "%s: bad sizes", w);
  if (x_dtype != AXR_F32 && x_dtype != AXR_F16) return set_error(AXR_EINVAL, "%s: bad dtype", w);
  if (n_vec == 0) return set_error(AXR_OK, "");
  if (!x || !codebooks || !codes) return set_error(AXR_EINVAL, "%s: null pointer", w);
  if (!aligned(x, x_dtype == AXR_F32 ? 4 : 2) || !aligned(codebooks, 4) || (dst_rows && !aligned(dst_rows, 8)))
    return set_error(AXR_EINVAL, "%s: misaligned pointer", w);
  PqEncArgs a;
  memset(&a, 0, sizeof(a));
  a.x = x; a.n_vec = n_vec; a.m = m; a.K = K; a.cb = codebooks; a.heads = heads; a.head_period = head_period;
  a.dst_rows = dst_rows; a.codes = codes;
  cudaStream_t s = as_stream(stream);
  if (x_dtype == AXR_F16) return encode_ds<__half, false>(d / m, a, s, w);
  return encode_ds<float, false>(d / m, a, s, w);
}

extern "C" size_t axr_pq_train_workspace_bytes(int d, int m, int K) {
  if (d <= 0 || m <= 0 || K <= 0 || d % m) return 0;
  const size_t sums = static_cast<size_t>(d) * K * sizeof(double);  // m * K * (d / m)
  const size_t counts = static_cast<size_t>(m) * K * sizeof(unsigned int);
  return (sums + 255) / 256 * 256 + (counts + 255) / 256 * 256;
}

extern "C" axr_status axr_pq_train(const void* x, axr_dtype x_dtype, int64_t n_vec, int d, int m, int K, int iters,
                                   float* codebooks, void* workspace, size_t ws_bytes, void* stream) {
  using namespace axr;
  const char* w = "axr_pq_train";
  axr_status st = pq_sizes(w, d, m, K);
  if (st != AXR_OK) return st;
  if (n_vec < 1 || iters < 0) return set_error(AXR_EINVAL, "%s: bad sizes", w);
  if (x_dtype != AXR_F32 && x_dtype != AXR_F16) return set_error(AXR_EINVAL, "%s: bad dtype", w);
  if (!x || !codebooks) return set_error(AXR_EINVAL, "%s: null pointer", w);
  if (!aligned(x, x_dtype == AXR_F32 ? 4 : 2) || !aligned(codebooks, 4))
    return set_error(AXR_EINVAL, "%s: misaligned pointer", w);
  const size_t need = axr_pq_train_workspace_bytes(d, m, K);
  if (!workspace || ws_bytes < need)
    return set_error(AXR_EWORKSPACE, "%s: workspace of %zu bytes, need %zu", w, workspace ? ws_bytes : 0, need);
  if (!aligned(workspace, 16)) return set_error(AXR_EINVAL, "%s: workspace not 16-byte aligned", w);
  const size_t sums_bytes = (static_cast<size_t>(d) * K * sizeof(double) + 255) / 256 * 256;
  PqEncArgs a;
  memset(&a, 0, sizeof(a));
  a.x = x; a.n_vec = n_vec; a.m = m; a.K = K; a.cb = codebooks; a.heads = 1; a.head_period = 1;
  a.sums = static_cast<double*>(workspace);
  a.counts = reinterpret_cast<unsigned int*>(static_cast<char*>(workspace) + sums_bytes);
  cudaStream_t s = as_stream(stream);
  const int ds = d / m;
  for (int it = 0; it < iters; ++it) {
    cudaError_t e = cudaMemsetAsync(workspace, 0, need, s);
    if (e != cudaSuccess) return set_error(AXR_ECUDA, "%s: %s", w, cudaGetErrorString(e));
    st = x_dtype == AXR_F16 ? encode_ds<__half, true>(ds, a, s, w) : encode_ds<float, true>(ds, a, s, w);
    if (st != AXR_OK) return st;
    const int n = d * K;
    pq_update_kernel<<<(n + 255) / 256, 256, 0, s>>>(codebooks, a.sums, a.counts, m, K, ds);
    st = check_launch(w);
    if (st != AXR_OK) return st;
  }
  return set_error(AXR_OK, "");
}
