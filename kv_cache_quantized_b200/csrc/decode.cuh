// Decode-time read path: table scorer, split-T online-softmax . V partial kernel, split merge.
//
// AXELRAM Key Points (1st, 2nd items) and Abstract: the query is transformed once, a d x 2^b table of
// q~_j * c_k is built, and each cached token's score is the gather-sum of table entries at its stored indices times
// its stored norm -- no per-token inverse transform and no key reconstruction.  Softmax and the value product are
// not on the pages; they follow the standard split-T ("flash-decoding") formulation: each block owns a token range,
// keeps a running max and sum per query head, and a second kernel merges the ranges.
//
// Two ways to read the table are implemented (both give the table's values up to fp32 rounding):
//   * TABLE    -- the table LUT[j][k][h] = q~_{h,j} c_k is materialised in shared memory and each token gathers
//                 one G-wide entry per coordinate (one thread per token).
//   * FACTORED -- the table is kept in factored form: its row factor q~_{h,j} sits in registers of the thread that
//                 owns coordinate j, its column factor is gathered from a byte-indexed table of centroid pairs
//                 (c_{k1}, c_{k2}) -- two coordinates per lookup, replicated across banks -- and the product is
//                 formed by a packed fp32x2 FMA that also accumulates it.  On B200 this needs half the shared-memory
//                 wavefronts of TABLE per score (a 16-entry row of G-wide entries spans 2 wavefronts per warp
//                 request, a replicated pair table 1 per coordinate pair), which is what bounds the gather.
#pragma once

#include "axr_host.h"
#include "tc.cuh"

namespace axr {

constexpr int kDecThreads = 256;
constexpr int kDecWarps = kDecThreads / kWarp;
constexpr float kLog2e = 1.4426950408889634f;

enum Gather { kGatherFactored = 0, kGatherTable = 1, kGatherTensor = 2, kGatherMma = 3, kGatherDirect = 4 };

struct DecodeArgs {
  const float* q;            // [B, Hq, D]
  const uint8_t* kcodes;     // [B, Hkv, Tcap, R]
  const __half* knorms;      // [B, Hkv, Tcap]
  const __half* kdense;      // [B, Hkv, Tcap, D] fp16 keys (the dense kernel only)
  const void* v;             // fp16 [B, Hkv, Tcap, D] or codes [B, Hkv, Tcap, R]
  const __half* vnorms;      // [B, Hkv, Tcap] (quantized V)
  const int32_t* seq_lens;   // [B] or null
  const int8_t* signs;       // [D]
  const __half* knew;        // [B, Hkv, D] fp16: decode step, the new token's key, written at position len - 1
  const __half* vnew;        // [B, Hkv, D] fp16: its value (both null outside a decode step)
  float* scores;             // [B, Hq, T] (scorer)
  float* ws_o;               // [B, Hq, S, D]
  float* ws_m;               // [B, Hq, S]  running max, log2 units
  float* ws_l;               // [B, Hq, S]  running sum
  float* out;                // [B, Hq, D]
  int B, Hq, Hkv, T, Tcap;
  int splits, chunk;
  float mult;                // factor folded into the table (score: scale; attend: scale * log2(e))
  Codebook cb;
  unsigned int* status;      // the device's status word (axr_device_status), or null
  const int32_t* block_table;  // paged caches: [B, max_blocks] pool block of each logical block; null: contiguous
  int max_blocks;            // paged: entries per block-table row
  int block_shift;           // paged: log2 of the tokens per block
};

// Cache row of token t of one (batch row, KV head).  Contiguous caches [B, Hkv, Tcap] number the rows
// (b Hkv + hk) Tcap + t; paged pools [num_blocks, Hkv, bt] number them (block_table[b][t / bt] Hkv + hk) bt + t % bt,
// so the bt tokens of one (block, KV head) are contiguous.  PAGED is a compile-time choice, so the contiguous
// kernels carry none of the paging arithmetic.
template <bool PAGED>
struct RowMap {
  const int32_t* table;  // paged: the batch row's block table
  size_t base;           // contiguous: (b Hkv + hk) Tcap; paged: hk bt
  size_t stride;         // paged: Hkv bt, the rows of one block
  int shift;             // paged: log2 bt
  __device__ __forceinline__ size_t operator()(int t) const {
    if constexpr (!PAGED) return base + static_cast<size_t>(t);
    else
      return static_cast<size_t>(__ldg(table + (t >> shift))) * stride + base +
             static_cast<size_t>(t & ((1 << shift) - 1));
  }
  // rows from t to the end of t's block (contiguous caches: unbounded)
  __device__ __forceinline__ int run(int t) const {
    if constexpr (!PAGED) return 1 << 30;
    else return (1 << shift) - (t & ((1 << shift) - 1));
  }
};

template <bool PAGED>
__device__ __forceinline__ RowMap<PAGED> row_map(const DecodeArgs& a, int b, int hk) {
  RowMap<PAGED> m;
  if constexpr (PAGED) {
    m.table = a.block_table + static_cast<size_t>(b) * a.max_blocks;
    m.shift = a.block_shift;
    m.base = static_cast<size_t>(hk) << a.block_shift;
    m.stride = static_cast<size_t>(a.Hkv) << a.block_shift;
  } else {
    m.table = nullptr;
    m.shift = 0;
    m.base = (static_cast<size_t>(b) * a.Hkv + hk) * a.Tcap;
    m.stride = 0;
  }
  return m;
}

// A block whose bounded wait gave up (its `failed` flag set) records it in the device's status word, beside the
// NaN it writes into its outputs.  Called by every thread at the kernel's end; thread 0 reports.
__device__ __forceinline__ void report_wait_failure(const DecodeArgs& a, volatile int* failed) {
  if (threadIdx.x == 0 && *failed && a.status) atomicOr(a.status, 1u);
}

__device__ __forceinline__ int row_len(const DecodeArgs& a, int b) {
  if (!a.seq_lens) return a.T;
  int n = a.seq_lens[b];
  return n < 0 ? 0 : (n > a.T ? a.T : n);
}

// ---- asynchronous global -> shared copies ------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

template <int BYTES>
__device__ __forceinline__ void cp_async(void* dst, const void* src) {
  if constexpr (BYTES == 16)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(dst)), "l"(src));
  else
    asm volatile("cp.async.ca.shared.global [%0], [%1], %2;\n" ::"r"(smem_u32(dst)), "l"(src), "n"(BYTES));
}
// 16-byte copy that reads only the first src_bytes (1..16) of src and zero-fills the rest of dst.
__device__ __forceinline__ void cp_async16_zfill(void* dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes));
}

// Stage the fp16 norms of tokens [0, n) of a tile (n <= 128, src 16-byte aligned) as 16-byte chunks of 8 tokens,
// the last one zero-filled past n: the chunk of thread c (c < 16) of the copying group.
__device__ __forceinline__ void stage_norms(__half* dst, const __half* src, int n, int c) {
  const int tok0 = 8 * c;
  if (c < 16 && tok0 < n) cp_async16_zfill(dst + tok0, src + tok0, min(16, 2 * (n - tok0)));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
// stage_norms for rows [t0, t0 + n) of one (batch row, KV head) through its row map (blocks hold >= 8 tokens, so an
// 8-token chunk never straddles two)
template <class Map>
__device__ __forceinline__ void stage_norms_map(__half* dst, const __half* norms, const Map& rm, int t0, int n,
                                                int c) {
  const int tok0 = 8 * c;
  if (c < 16 && tok0 < n) cp_async16_zfill(dst + tok0, norms + rm(t0 + tok0), min(16, 2 * (n - tok0)));
}

// Bulk (TMA engine) copy of `bytes` (a multiple of 16; both addresses 16-byte aligned) from global to this CTA's
// shared memory, completing on `mbar` as transaction bytes; the caller has armed the barrier with expect_tx.
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* mbar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(mbar))
               : "memory");
}

// Arrive once on `mbar` and add `bytes` to the transaction count of its current phase.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* mbar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(mbar)), "r"(bytes)
               : "memory");
}

// Bulk copies of the rows [t0, t0 + n) of one (batch row, KV head), RB bytes each (a multiple of 16), into dst: one
// copy per run of rows contiguous in global memory (one for a contiguous cache, one per block for a paged pool),
// all completing on `mbar`, which the caller has armed with the total.
template <int RB, class Map>
__device__ __forceinline__ void copy_rows_bulk(uint8_t* dst, const uint8_t* src, const Map& rm, int t0, int n,
                                               uint64_t* mbar) {
  for (int o = 0; o < n;) {
    const int seg = min(n - o, rm.run(t0 + o));
    bulk_copy_g2s(dst + static_cast<size_t>(o) * RB, src + rm(t0 + o) * RB, static_cast<uint32_t>(seg * RB), mbar);
    o += seg;
  }
}

// The same rows as CH-byte cp.async chunks spread over a role's 128 threads (RB a multiple of CH).
template <int CH, int RB, class Map>
__device__ __forceinline__ void copy_rows_async(uint8_t* dst, const uint8_t* src, const Map& rm, int t0, int n,
                                                int rtid) {
  const int bytes = n * RB;
  if (rm.run(t0) >= n) {  // one contiguous run
    const uint8_t* s = src + rm(t0) * RB;
    for (int o = rtid * CH; o < bytes; o += 128 * CH) cp_async<CH>(dst + o, s + o);
  } else {
    for (int o = rtid * CH; o < bytes; o += 128 * CH) cp_async<CH>(dst + o, src + rm(t0 + o / RB) * RB + o % RB);
  }
}

// Order this thread's generic-proxy accesses to shared memory before later async-proxy (bulk copy) accesses.
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

// Copy `bytes` (a multiple of CH) from global to shared, spread over the block.
template <int CH>
__device__ __forceinline__ void block_copy_async(uint8_t* dst, const uint8_t* src, int bytes) {
  for (int o = threadIdx.x * CH; o < bytes; o += kDecThreads * CH) cp_async<CH>(dst + o, src + o);
}

// ---- query transform ---------------------------------------------------------------------------------------------

// qs[g][j] = mult * (H (s .* q_g))_j for the G query heads of this KV head (warp g transforms head g).
template <int D, int G>
__device__ __forceinline__ void transform_queries(const float* __restrict__ q, const int8_t* __restrict__ signs,
                                                  float mult, float* __restrict__ qs) {
  constexpr int VPL = WarpVec<D>::VPL;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float norm = mult * rsqrtf(static_cast<float>(D));
  for (int g = warp; g < G; g += blockDim.x / kWarp) {
    float v[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int j = lane * VPL + i;
      v[i] = q[g * D + j] * sign_of(signs[j]);
    }
    fwht_warp<D>(v, lane);
#pragma unroll
    for (int i = 0; i < VPL; ++i) qs[g * D + lane * VPL + i] = v[i] * norm;
  }
}

// ---- factored gather: byte-indexed centroid-pair table -------------------------------------------------------------

// Entry e (the 2b-bit code of two consecutive coordinates, low coordinate in the low bits) holds (c[e & (L-1)],
// c[e >> b]).  The table is replicated once per lane, entry-major with a 256-byte entry stride: lane l reads copy
// l at byte offset e * 256 + 8 l, so a warp's 32 lookups never share a bank with a different address beyond the
// two wavefronts a 64-bit warp load needs, and the offset of a pair is one byte permute of the packed code word
// (entry index into byte 1, the lane's copy offset into byte 0).
//
// With 16 copies (REPS = 16, 128-byte entry stride) lanes l and l + 16 share a copy; they sit in different halves
// of the warp's 64-bit request, so the request still takes its two wavefronts, at half the shared memory, but the
// offset then needs a shift and a mask instead of one byte permute.
template <int BITS, int REPS_ = 32>
struct PairTable {
  static constexpr int L = 1 << BITS;
  static constexpr int E = L * L;
  static constexpr int REPS = REPS_;
  static constexpr int SHIFT = REPS == 32 ? 8 : 7;   // log2 of the entry stride in bytes
  static constexpr int FLOATS = E * REPS * 2;
};

template <int BITS, int REPS = 32>
__device__ __forceinline__ uint32_t rep_offset(int lane) {
  return static_cast<uint32_t>(lane & (REPS - 1)) << 3;
}

template <int BITS, int REPS = 32>
__device__ __forceinline__ void build_pair_table(const float* __restrict__ cent, float* __restrict__ tab) {
  using P = PairTable<BITS, REPS>;
  for (int i = threadIdx.x; i < P::E * P::REPS; i += kDecThreads) {
    const int e = i / P::REPS;
    tab[2 * i] = cent[e & (P::L - 1)];
    tab[2 * i + 1] = cent[e >> BITS];
  }
}

// Byte offset of this lane's copy of pair i (coordinates 2i, 2i+1) of a packed slice; repw = rep_offset(lane).
template <int BITS, int REPS = 32>
__device__ __forceinline__ uint32_t pair_addr(uint64_t bits, int i, uint32_t repw) {
  if constexpr (BITS == 4 && REPS == 32) {
    const uint32_t w = i < 4 ? static_cast<uint32_t>(bits) : static_cast<uint32_t>(bits >> 32);
    return __byte_perm(w, repw, 0x5504u | (static_cast<uint32_t>(i & 3) << 4));
  } else {
    constexpr uint32_t MASK = (1u << (2 * BITS)) - 1u;
    return ((static_cast<uint32_t>(bits >> (2 * BITS * i)) & MASK) << PairTable<BITS, REPS>::SHIFT) | repw;
  }
}

// The J*b bits of coordinates [J*sl, J*sl + J) of one packed row held in shared memory, as a 64-bit value.
template <int D, int BITS, int J>
__device__ __forceinline__ uint64_t load_slice(const uint8_t* row, int sl) {
  constexpr int NB = J * BITS / 8;  // bytes, <= 8
  const uint8_t* p = row + sl * NB;
  if constexpr (NB == 8) return *reinterpret_cast<const uint64_t*>(p);
  else if constexpr (NB == 4) return *reinterpret_cast<const uint32_t*>(p);
  else if constexpr (NB == 2) return *reinterpret_cast<const uint16_t*>(p);
  else if constexpr (NB == 1) return *p;
  else if constexpr (NB == 6) {
    const uint16_t* h = reinterpret_cast<const uint16_t*>(p);
    return static_cast<uint64_t>(h[0]) | (static_cast<uint64_t>(h[1]) << 16) | (static_cast<uint64_t>(h[2]) << 32);
  } else {  // NB == 3
    return static_cast<uint64_t>(p[0]) | (static_cast<uint64_t>(p[1]) << 8) | (static_cast<uint64_t>(p[2]) << 16);
  }
}

// Partial dot products of one token's slice with the HG heads' row factors: acc[h] = sum over the slice's coordinate
// pairs of (q~_{h,2i}, q~_{h,2i+1}) . (c, c') -- the packed FMA keeps even and odd coordinates in the two halves.
template <int BITS, int J, int HG, int REPS = 32>
__device__ __forceinline__ void factored_slice(uint64_t bits, const uint8_t* tab, uint32_t rep_off,
                                               const float2 (&qp)[HG][J / 2], float (&acc)[HG]) {
  // two accumulators per head (even and odd pairs) halve the dependent FMA chain
  float2 a[2][HG];
#pragma unroll
  for (int h = 0; h < HG; ++h) a[0][h] = a[1][h] = make_float2(0.f, 0.f);
  float2 c[J / 2];
#pragma unroll
  for (int i = 0; i < J / 2; ++i) c[i] = *reinterpret_cast<const float2*>(tab + pair_addr<BITS, REPS>(bits, i, rep_off));
#pragma unroll
  for (int i = 0; i < J / 2; ++i)
#pragma unroll
    for (int h = 0; h < HG; ++h) a[i & 1][h] = fma2(qp[h][i], c[i], a[i & 1][h]);
#pragma unroll
  for (int h = 0; h < HG; ++h) {
    const float2 t = add2(a[0][h], a[1][h]);
    acc[h] = t.x + t.y;
  }
}

// ---- the decode partial kernel: persistent and warp-specialised ---------------------------------------------------
//
// A block of 256 threads runs as two roles, one tile of TT = 128 tokens apart, with one block barrier per tile:
//   scoring warps 0..3 -- hold the query row factors in registers and score the tile's tokens (8 lanes per token,
//                         each lane owning D/8 coordinates; a lane group of 8 scores 4 tokens per round and combines
//                         its partial sums with a select-free butterfly: lane sl processes token k ^ (sl >> 1) at step
//                         k, after which lanes 2m, 2m+1 hold token m); scoring warp w owns tokens [32w, 32w + 32) of
//                         every tile and keeps the running max and sum of its tokens (online softmax); it writes the
//                         weights p (times the value norm for quantized values) and its rescale factor to shared
//                         memory;
//   value warps 4..7   -- hold the value accumulators and consume the previous tile: value warp 4 + w accumulates the
//                         tokens of scoring warp w against the same running max, D/8 lanes per token row.
// Keeping the two register sets in different warps is what lets each role run without spilling.  The roles never
// wait on each other except at the shared per-tile barrier (bar.sync 1 with all 256 threads, which both roles execute
// the same number of times).  Blocks are persistent: each loops over (batch, KV head, split) items, and builds the
// pair table once.

constexpr int kTT = 128;     // tokens per tile of the scorer
constexpr int kStages = 3;   // cp.async pipeline depth (two tiles in flight while one is processed)
constexpr int kDecReps = 16; // pair-table copies in the decode kernel

template <int D, int BITS, int G, bool VQ>
struct DecPlan {
  static constexpr int TT = 128;                          // tokens per tile
  static constexpr int KW = 4;                            // scoring warps; value warps follow them
  static constexpr int RT = 128;                          // role threads
  static constexpr int WT = TT / KW;                      // tokens per scoring warp per tile
  static constexpr int L = 1 << BITS;
  static constexpr int R = D * BITS / 8;
  static constexpr int KROW = R;                          // bytes per key row
  static constexpr int VROW = VQ ? R : 2 * D;             // bytes per value row
  static constexpr int KCH = (KROW % 16 == 0) ? 16 : 8;   // cp.async chunk sizes
  static constexpr int VCH = (VROW % 16 == 0) ? 16 : 8;
  static constexpr int STAGE_K = TT * KROW;
  static constexpr int STAGE_V = TT * VROW;
  static constexpr int J = D / 8;                         // key coordinates per lane
  static constexpr int HG = G < 4 ? G : 4;                // heads per scoring pass
  static constexpr int PASSES = G / HG;
  static constexpr int TPR = D / 8;                       // value lanes per token row (8 coordinates each)
  static constexpr int RPW = kWarp / TPR;                 // value rows per warp step
  static constexpr int NVG = KW * RPW;                    // value lane groups, summed at the end
  static constexpr int TAB = PairTable<BITS, kDecReps>::FLOATS;
  static constexpr size_t OFF_K = 0;                                         // [kStages][STAGE_K]
  static constexpr size_t OFF_V = OFF_K + kStages * (size_t)STAGE_K;         // [kStages][STAGE_V]
  static constexpr size_t STAGES_END = OFF_V + kStages * (size_t)STAGE_V;
  static constexpr size_t REDUCE_BYTES = (size_t)NVG * G * D * 4;            // final sum, reuses the stages
  static constexpr size_t OFF_TAB = ((STAGES_END > REDUCE_BYTES ? STAGES_END : REDUCE_BYTES) + 15) / 16 * 16;
  static constexpr size_t OFF_QS = OFF_TAB + (size_t)TAB * 4;               // [G][D] row factors
  static constexpr size_t OFF_P = OFF_QS + (size_t)G * D * 4;               // [2][TT][G] float2 weights
  static constexpr size_t OFF_AL = OFF_P + 2 * (size_t)TT * G * 8;          // [2][KW][G] rescale factors
  static constexpr size_t OFF_GR = OFF_AL + 2 * (size_t)KW * G * 4;         // [2][KW] rescale flags
  static constexpr size_t OFF_RM = OFF_GR + 2 * (size_t)KW * 4;             // [KW][G] running max
  static constexpr size_t OFF_RL = OFF_RM + (size_t)KW * G * 4;             // [KW][G] running sum
  static constexpr size_t OFF_CENT = OFF_RL + (size_t)KW * G * 4;
  static constexpr size_t bytes = OFF_CENT + 16 * 4;
  static constexpr int MIN_BLOCKS = bytes <= 110 * 1024 ? 2 : 1;
};

__device__ __forceinline__ void roles_sync() { asm volatile("bar.sync 1, 256;\n" ::: "memory"); }

// Copy `bytes` (a multiple of CH) from global to shared with the 128 threads of one role.
template <int CH>
__device__ __forceinline__ void role_copy_async(uint8_t* dst, const uint8_t* src, int bytes, int rtid) {
  for (int o = rtid * CH; o < bytes; o += 128 * CH) cp_async<CH>(dst + o, src + o);
}

template <int D, int BITS, int G, bool VQ>
__global__ void __launch_bounds__(kDecThreads, DecPlan<D, BITS, G, VQ>::MIN_BLOCKS)
attend_partial_kernel(const __grid_constant__ DecodeArgs a) {
  using P = DecPlan<D, BITS, G, VQ>;
  constexpr int J = P::J, HG = P::HG, TT = P::TT, WT = P::WT, KW = P::KW, RPW = P::RPW, TPR = P::TPR;
  extern __shared__ __align__(16) uint8_t smem[];
  float* tab = reinterpret_cast<float*>(smem + P::OFF_TAB);
  float* qs = reinterpret_cast<float*>(smem + P::OFF_QS);
  float2* pbuf = reinterpret_cast<float2*>(smem + P::OFF_P);
  float* alpha_s = reinterpret_cast<float*>(smem + P::OFF_AL);
  int* grew_s = reinterpret_cast<int*>(smem + P::OFF_GR);
  float* red_m = reinterpret_cast<float*>(smem + P::OFF_RM);
  float* red_l = reinterpret_cast<float*>(smem + P::OFF_RL);
  float* cent = reinterpret_cast<float*>(smem + P::OFF_CENT);
  float* region = reinterpret_cast<float*>(smem);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool scorer = warp < KW;
  const int rtid = scorer ? tid : tid - P::RT;  // thread index within the role

  if (tid < 16) cent[tid] = a.cb.c[tid];
  __syncthreads();
  build_pair_table<BITS, kDecReps>(cent, tab);

  const int items = a.B * a.Hkv * a.splits;
  for (int item = blockIdx.x; item < items; item += gridDim.x) {
    const int split = item % a.splits;
    const int hk = (item / a.splits) % a.Hkv;
    const int b = item / (a.splits * a.Hkv);
    const int len = row_len(a, b);
    const int start = split * a.chunk;
    const int end = min(start + a.chunk, len);
    const int ntiles = end > start ? (end - start + TT - 1) / TT : 0;
    const size_t kv_row0 = (static_cast<size_t>(b) * a.Hkv + hk) * a.Tcap;
    const float* qg = a.q + (static_cast<size_t>(b) * a.Hq + hk * G) * D;

    __syncthreads();  // the previous item is finished with the row factors, the stages and the merge region
    transform_queries<D, G>(qg, a.signs, a.mult, qs);
    __syncthreads();

    if (scorer) {
      // ================================= scoring role =================================
      const int sl = tid & 7, kord = sl >> 1;
      const int tk0 = warp * WT + ((tid >> 3) & 3) * 4;  // first token of this lane group, round 0
      const bool writer_lo = (sl & 1) == 0;
      const uint32_t rep_off = rep_offset<BITS, kDecReps>(lane);
      const uint8_t* ksrc = a.kcodes;
      float2 qp[HG][J / 2];
      if constexpr (P::PASSES == 1) {
#pragma unroll
        for (int h = 0; h < HG; ++h)
#pragma unroll
          for (int i = 0; i < J / 2; ++i)
            qp[h][i] = make_float2(qs[h * D + J * sl + 2 * i], qs[h * D + J * sl + 2 * i + 1]);
      }
      float m_run[G], l_lane[G];
#pragma unroll
      for (int g = 0; g < G; ++g) { m_run[g] = -INFINITY; l_lane[g] = 0.f; }
      float kn_next[2], vn_next[2];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int t = start + tk0 + 16 * r + kord;
        kn_next[r] = (ntiles > 0 && t < end) ? __half2float(a.knorms[kv_row0 + t]) : 1.f;
        vn_next[r] = (VQ && ntiles > 0 && t < end) ? __half2float(a.vnorms[kv_row0 + t]) : 1.f;
      }
      auto issue_k = [&](int tile) {
        if (tile < ntiles) {
          const int t0 = start + tile * TT;
          role_copy_async<P::KCH>(smem + P::OFF_K + (tile % kStages) * P::STAGE_K,
                                  ksrc + (kv_row0 + t0) * P::KROW, min(TT, end - t0) * P::KROW, rtid);
        }
        cp_async_commit();
      };
      issue_k(0);
      issue_k(1);
      for (int it = 0; it <= ntiles; ++it) {
        cp_async_wait<1>();  // tile it has landed; tile it + 1 may still be in flight
        roles_sync();
        issue_k(it + 2);     // into the stage tile it - 1 used
        if (it == ntiles) continue;
        const int t0 = start + it * TT;
        const int nt = min(TT, end - t0);
        const uint8_t* st = smem + P::OFF_K + (it % kStages) * P::STAGE_K;
        float kn_cur[2], vn_cur[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          kn_cur[r] = kn_next[r];
          vn_cur[r] = vn_next[r];
          const int t = t0 + TT + tk0 + 16 * r + kord;  // my tokens of the next tile
          if (it + 1 < ntiles && t < end) {
            kn_next[r] = __half2float(a.knorms[kv_row0 + t]);
            if constexpr (VQ) vn_next[r] = __half2float(a.vnorms[kv_row0 + t]);
          }
        }
        float z[2][G];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int tk = tk0 + 16 * r;
#pragma unroll
          for (int pass = 0; pass < P::PASSES; ++pass) {
            if constexpr (P::PASSES > 1) {
#pragma unroll
              for (int h = 0; h < HG; ++h)
#pragma unroll
                for (int i = 0; i < J / 2; ++i) {
                  const float* qrow = qs + (pass * HG + h) * D + J * sl + 2 * i;
                  qp[h][i] = make_float2(qrow[0], qrow[1]);
                }
            }
            float v[4][HG];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int tt = tk + (k ^ kord);
              const uint64_t bits = load_slice<D, BITS, J>(st + tt * P::KROW, sl);
              factored_slice<BITS, J, HG, kDecReps>(bits, reinterpret_cast<const uint8_t*>(tab), rep_off, qp, v[k]);
            }
#pragma unroll
            for (int h = 0; h < HG; ++h) {
              v[0][h] += __shfl_xor_sync(0xffffffffu, v[2][h], 4);
              v[1][h] += __shfl_xor_sync(0xffffffffu, v[3][h], 4);
              v[0][h] += __shfl_xor_sync(0xffffffffu, v[1][h], 2);
              v[0][h] += __shfl_xor_sync(0xffffffffu, v[0][h], 1);
              z[r][pass * HG + h] = v[0][h];
            }
          }
        }
        // online softmax over this warp's 32 tokens of the tile
        bool grew = false;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          float mx = -INFINITY;
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const bool valid = tk0 + 16 * r + kord < nt;
            z[r][g] = valid ? z[r][g] * kn_cur[r] : -INFINITY;
            mx = fmaxf(mx, z[r][g]);
          }
#pragma unroll
          for (int msk = 2; msk < 32; msk <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, msk));
          const float m_new = fmaxf(m_run[g], mx);
          const float alpha = (m_new == -INFINITY) ? 1.f : exp2f(m_run[g] - m_new);
          float psum = 0.f;
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const float p = (z[r][g] == -INFINITY) ? 0.f : exp2f(z[r][g] - m_new);
            psum += p;
            z[r][g] = p * (VQ ? vn_cur[r] : 1.f);
          }
          l_lane[g] = l_lane[g] * alpha + (writer_lo ? psum : 0.f);
          grew |= m_new != m_run[g];
          m_run[g] = m_new;
          if (lane == 0) alpha_s[((it & 1) * KW + warp) * G + g] = alpha;
        }
        if (lane == 0) grew_s[(it & 1) * KW + warp] = grew ? 1 : 0;
        constexpr int HALF = G > 1 ? G / 2 : 1;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          float2* row = pbuf + (static_cast<size_t>(it & 1) * TT + tk0 + 16 * r + kord) * G;
          if (G > 1 || writer_lo) {
#pragma unroll
            for (int h = 0; h < HALF; ++h) {
              const int g = (writer_lo ? 0 : HALF) + h;
              row[g] = make_float2(z[r][g], z[r][g]);
            }
          }
        }
      }
      cp_async_wait<0>();
      // merge, step 1: publish this warp's running max
      if (lane == 0) {
#pragma unroll
        for (int g = 0; g < G; ++g) red_m[warp * G + g] = m_run[g];
      }
      roles_sync();
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float M = red_m[g];
#pragma unroll
        for (int w2 = 1; w2 < KW; ++w2) M = fmaxf(M, red_m[w2 * G + g]);
        const float scl = (m_run[g] == -INFINITY) ? 0.f : exp2f(m_run[g] - M);
        const float l = warp_sum(l_lane[g]) * scl;
        if (lane == 0) red_l[warp * G + g] = l;
      }
    } else {
      // ================================= value role =================================
      const int vw = warp - KW;
      const int vrow = lane / TPR, vc = lane % TPR;
      const uint32_t rep_off = rep_offset<BITS, kDecReps>(lane);
      const uint8_t* vsrc = static_cast<const uint8_t*>(a.v);
      float2 acc[G][4];
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[g][c] = make_float2(0.f, 0.f);
      auto issue_v = [&](int tile) {
        if (tile < ntiles) {
          const int t0 = start + tile * TT;
          role_copy_async<P::VCH>(smem + P::OFF_V + (tile % kStages) * P::STAGE_V,
                                  vsrc + (kv_row0 + t0) * P::VROW, min(TT, end - t0) * P::VROW, rtid);
        }
        cp_async_commit();
      };
      issue_v(0);
      for (int it = 0; it <= ntiles; ++it) {
        cp_async_wait<1>();  // tile it - 1 has landed; tile it may still be in flight
        roles_sync();
        issue_v(it + 1);     // into the stage tile it - 2 used
        if (it == 0) continue;
        const int j = it - 1;  // the tile scored in the previous step
        const int nt = min(TT, end - (start + j * TT));
        const int pb = j & 1;
        if (grew_s[pb * KW + vw]) {
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float al = alpha_s[(pb * KW + vw) * G + g];
#pragma unroll
            for (int c = 0; c < 4; ++c) { acc[g][c].x *= al; acc[g][c].y *= al; }
          }
        }
        const uint8_t* vst = smem + P::OFF_V + (j % kStages) * P::STAGE_V;
        const float2* prow = pbuf + static_cast<size_t>(pb) * TT * G;
#pragma unroll 2
        for (int i = 0; i < WT / RPW; ++i) {
          const int tt = vw * WT + vrow + RPW * i;
          if (tt >= nt) break;
          float2 pw[G];
#pragma unroll
          for (int g = 0; g < G; ++g) pw[g] = prow[tt * G + g];
          float2 val[4];
          if constexpr (VQ) {
            const uint64_t bits = load_slice<D, BITS, 8>(vst + tt * P::VROW, vc);
#pragma unroll
            for (int c = 0; c < 4; ++c)
              val[c] = *reinterpret_cast<const float2*>(reinterpret_cast<const uint8_t*>(tab) +
                                                        pair_addr<BITS, kDecReps>(bits, c, rep_off));
          } else {
            const uint4 u = *reinterpret_cast<const uint4*>(vst + tt * P::VROW + 16 * vc);
            val[0] = __half22float2(*reinterpret_cast<const __half2*>(&u.x));
            val[1] = __half22float2(*reinterpret_cast<const __half2*>(&u.y));
            val[2] = __half22float2(*reinterpret_cast<const __half2*>(&u.z));
            val[3] = __half22float2(*reinterpret_cast<const __half2*>(&u.w));
          }
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
      a.ws_m[part0 + static_cast<size_t>(tid) * a.splits] = M;
    }
  }
}

// Merge of the splits for one (batch, query head) per block, D threads.  With quantized values the merged vector
// is still in the rotated domain and is mapped back once: out = s .* H(o).  EXACT: the splits' maxima are integers
// (a log2 domain of integers), and every rescale is the exact power of two 2^(m_s - M).
// The maximum over the splits and the weight of each split are computed once, in parallel across the block (the
// weights into shared memory, a chunk at a time), so that thread j's sum over the splits of coordinate j is a run of
// independent loads rather than a chain through m and l.
template <int D, bool VQ, bool EXACT = false>
__global__ void __launch_bounds__(D) attend_reduce_kernel(const __grid_constant__ DecodeArgs a) {
  constexpr int CH = 512;  // splits per chunk of weights
  __shared__ float vec[D];
  __shared__ float wsh[CH];
  __shared__ float red[D / kWarp];
  const int bh = blockIdx.x, j = threadIdx.x, lane = j & (kWarp - 1), warp = j / kWarp;
  // launched as a programmatic dependent of the decode kernel: its partials are complete and visible after this
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  const int S = a.splits;
  const float* m = a.ws_m + static_cast<size_t>(bh) * S;
  const float* l = a.ws_l + static_cast<size_t>(bh) * S;
  const float* o = a.ws_o + static_cast<size_t>(bh) * S * D;
  float M = -INFINITY;
  for (int s = j; s < S; s += D) M = fmaxf(M, m[s]);
  M = warp_max(M);
  if (lane == 0) red[warp] = M;
  __syncthreads();
  M = red[0];
#pragma unroll
  for (int w = 1; w < D / kWarp; ++w) M = fmaxf(M, red[w]);
  __syncthreads();  // every thread has read red before it is reused for the sum
  float Ls = 0.f, acc = 0.f;
  if (M != -INFINITY) {  // uniform over the block
    for (int c0 = 0; c0 < S; c0 += CH) {
      const int n = min(CH, S - c0);
      for (int s = j; s < n; s += D) {
        const float ms = m[c0 + s];
        const float w = (ms == -INFINITY) ? 0.f
                        : EXACT           ? ldexpf(1.f, static_cast<int>(ms - M))
                                          : exp2f(ms - M);
        wsh[s] = w;
        Ls = fmaf(w, l[c0 + s], Ls);
      }
      __syncthreads();
      const float* oc = o + static_cast<size_t>(c0) * D + j;
      int s = 0;
      for (; s + 4 <= n; s += 4) {
        const float o0 = oc[static_cast<size_t>(s) * D], o1 = oc[static_cast<size_t>(s + 1) * D];
        const float o2 = oc[static_cast<size_t>(s + 2) * D], o3 = oc[static_cast<size_t>(s + 3) * D];
        acc = fmaf(wsh[s], o0, acc);
        acc = fmaf(wsh[s + 1], o1, acc);
        acc = fmaf(wsh[s + 2], o2, acc);
        acc = fmaf(wsh[s + 3], o3, acc);
      }
      for (; s < n; ++s) acc = fmaf(wsh[s], oc[static_cast<size_t>(s) * D], acc);
      __syncthreads();  // the chunk's weights are read before the next chunk writes them
    }
  }
  Ls = warp_sum(Ls);
  if (lane == 0) red[warp] = Ls;
  __syncthreads();
  Ls = red[0];
#pragma unroll
  for (int w = 1; w < D / kWarp; ++w) Ls += red[w];
  const float r = Ls > 0.f ? acc / Ls : 0.f;
  if constexpr (!VQ) {
    a.out[static_cast<size_t>(bh) * D + j] = r;
  } else {
    constexpr int VPL = WarpVec<D>::VPL;
    vec[j] = r;
    __syncthreads();
    if (j < kWarp) {
      float v[VPL];
#pragma unroll
      for (int i = 0; i < VPL; ++i) v[i] = vec[j * VPL + i];
      fwht_warp<D>(v, j);
      const float nrm = rsqrtf(static_cast<float>(D));
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        const int jj = j * VPL + i;
        a.out[static_cast<size_t>(bh) * D + jj] = v[i] * nrm * sign_of(a.signs[jj]);
      }
    }
  }
}

// ---- scores only ---------------------------------------------------------------------------------------------------

// Shared-memory plan of the scorer: the factored form stages key codes (cp.async, double-buffered) and holds the
// pair table; the table form holds the materialised G-wide table and reads rows straight from global memory.
template <int D, int BITS, int G, int MODE>
struct ScorePlan {
  static constexpr int L = 1 << BITS;
  static constexpr int R = D * BITS / 8;
  static constexpr int KCH = (R % 16 == 0) ? 16 : 8;
  static constexpr int STAGE = kTT * R;
  static constexpr int LPT = 8, J = D / LPT;
  static constexpr int HG = G < 4 ? G : 4, PASSES = G / HG;
  static constexpr size_t OFF_STAGE = 0;
  static constexpr size_t OFF_TAB = MODE == kGatherFactored ? (size_t)kStages * STAGE : 0;
  static constexpr int TAB = MODE == kGatherFactored ? PairTable<BITS>::FLOATS : D * L * G;
  static constexpr size_t OFF_QS = OFF_TAB + (size_t)TAB * 4;
  static constexpr size_t OFF_CENT = OFF_QS + (size_t)G * D * 4;
  static constexpr size_t bytes = OFF_CENT + 16 * 4;
};

template <int R>
__device__ __forceinline__ void load_row(const uint8_t* __restrict__ p, uint32_t (&w)[R / 4 + 1]) {
  if constexpr (R % 16 == 0) {
#pragma unroll
    for (int i = 0; i < R / 16; ++i) {
      uint4 u = __ldg(reinterpret_cast<const uint4*>(p) + i);
      w[4 * i] = u.x; w[4 * i + 1] = u.y; w[4 * i + 2] = u.z; w[4 * i + 3] = u.w;
    }
  } else {
    static_assert(R % 8 == 0, "rows are a multiple of 8 bytes for d >= 64");
#pragma unroll
    for (int i = 0; i < R / 8; ++i) {
      uint2 u = __ldg(reinterpret_cast<const uint2*>(p) + i);
      w[2 * i] = u.x; w[2 * i + 1] = u.y;
    }
  }
  w[R / 4] = 0u;
}

// Gather-sum over the D coordinates of one token row from the materialised table: acc[g] = sum_j lut[j][idx_j][g].
template <int D, int BITS, int G>
__device__ __forceinline__ void table_gather(const uint32_t* w, const float* __restrict__ lut, float (&acc)[G]) {
  constexpr int L = 1 << BITS;
  if constexpr (G == 1) {
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int j = 0; j < D; j += 2) {
      a0 += lut[j * L + bits_at<BITS>(w, j * BITS)];
      a1 += lut[(j + 1) * L + bits_at<BITS>(w, (j + 1) * BITS)];
    }
    acc[0] = a0 + a1;
  } else if constexpr (G == 2) {
    float2 s = make_float2(0.f, 0.f);
#pragma unroll
    for (int j = 0; j < D; ++j) s = add2(s, reinterpret_cast<const float2*>(lut)[j * L + bits_at<BITS>(w, j * BITS)]);
    acc[0] = s.x; acc[1] = s.y;
  } else {
    float2 s[G / 2];
#pragma unroll
    for (int i = 0; i < G / 2; ++i) s[i] = make_float2(0.f, 0.f);
#pragma unroll
    for (int j = 0; j < D; ++j) {
      const float4* e = reinterpret_cast<const float4*>(lut + (j * L + bits_at<BITS>(w, j * BITS)) * G);
#pragma unroll
      for (int i = 0; i < G / 4; ++i) {
        const float4 x = e[i];
        s[2 * i] = add2(s[2 * i], make_float2(x.x, x.y));
        s[2 * i + 1] = add2(s[2 * i + 1], make_float2(x.z, x.w));
      }
    }
#pragma unroll
    for (int i = 0; i < G / 2; ++i) { acc[2 * i] = s[i].x; acc[2 * i + 1] = s[i].y; }
  }
}

template <int D, int BITS, int G, int MODE>
__global__ void __launch_bounds__(kDecThreads) score_kernel(const __grid_constant__ DecodeArgs a) {
  using P = ScorePlan<D, BITS, G, MODE>;
  constexpr int L = 1 << BITS, R = P::R, J = P::J, HG = P::HG;
  extern __shared__ __align__(16) uint8_t smem[];
  float* tab = reinterpret_cast<float*>(smem + P::OFF_TAB);
  float* qs = reinterpret_cast<float*>(smem + P::OFF_QS);
  float* cent = reinterpret_cast<float*>(smem + P::OFF_CENT);
  const int tid = threadIdx.x, lane = tid & 31;
  const int b = blockIdx.z, hk = blockIdx.y;
  const int len = row_len(a, b);
  const int start = blockIdx.x * a.chunk;
  const int end = min(start + a.chunk, a.T);
  const int vend = min(end, len);  // tokens with codes
  const size_t kv_row0 = (static_cast<size_t>(b) * a.Hkv + hk) * a.Tcap;
  float* out = a.scores + (static_cast<size_t>(b) * a.Hq + hk * G) * a.T;
  // tokens in [max(len, start), end) are masked
  for (int t = max(start, len) + tid; t < end; t += kDecThreads)
#pragma unroll
    for (int g = 0; g < G; ++g) out[static_cast<size_t>(g) * a.T + t] = -INFINITY;
  const int ntiles = vend > start ? (vend - start + kTT - 1) / kTT : 0;

  auto issue_tile = [&](int tile) {
    if constexpr (MODE == kGatherFactored) {
      if (tile < ntiles) {
        uint8_t* st = smem + P::OFF_STAGE + static_cast<size_t>(tile % kStages) * P::STAGE;
        const int t0 = start + tile * kTT;
        block_copy_async<P::KCH>(st, a.kcodes + (kv_row0 + t0) * R, min(kTT, vend - t0) * R);
      }
      cp_async_commit();
    }
  };
  for (int s = 0; s < kStages - 1; ++s) issue_tile(s);
  if (tid < 16) cent[tid] = a.cb.c[tid];
  transform_queries<D, G>(a.q + (static_cast<size_t>(b) * a.Hq + hk * G) * D, a.signs, a.mult, qs);
  __syncthreads();

  if constexpr (MODE == kGatherTable) {
    for (int e = tid; e < D * L * G; e += kDecThreads) {
      const int g = e % G, k = (e / G) % L, j = e / (G * L);
      tab[e] = qs[g * D + j] * cent[k];
    }
    __syncthreads();
    for (int t = start + tid; t < vend; t += kDecThreads) {
      uint32_t w[R / 4 + 1];
      load_row<R>(a.kcodes + (kv_row0 + t) * R, w);
      float s[G];
      table_gather<D, BITS, G>(w, tab, s);
      const float n = __half2float(a.knorms[kv_row0 + t]);
#pragma unroll
      for (int g = 0; g < G; ++g) out[static_cast<size_t>(g) * a.T + t] = s[g] * n;
    }
  } else {
    build_pair_table<BITS>(cent, tab);
    const int sl = tid & 7, grp = tid >> 3, kord = sl >> 1;
    const uint32_t rep_off = static_cast<uint32_t>(lane) << 3;
    float2 qp[HG][J / 2];
    if constexpr (P::PASSES == 1) {
#pragma unroll
      for (int h = 0; h < HG; ++h)
#pragma unroll
        for (int i = 0; i < J / 2; ++i) qp[h][i] = make_float2(qs[h * D + J * sl + 2 * i], qs[h * D + J * sl + 2 * i + 1]);
    }
    constexpr int ROUNDS = kTT / 128;
    float kn_next[ROUNDS];
#pragma unroll
    for (int r = 0; r < ROUNDS; ++r) {
      const int t = start + r * 128 + grp * 4 + kord;
      kn_next[r] = (ntiles > 0 && t < vend) ? __half2float(a.knorms[kv_row0 + t]) : 0.f;
    }
    for (int tile = 0; tile < ntiles; ++tile) {
      const int t0 = start + tile * kTT;
      const int nt = min(kTT, vend - t0);
      cp_async_wait<kStages - 2>();
      __syncthreads();  // tile complete; previous tile's stage free
      issue_tile(tile + kStages - 1);
      float kn_cur[ROUNDS];
#pragma unroll
      for (int r = 0; r < ROUNDS; ++r) {
        kn_cur[r] = kn_next[r];
        const int t = t0 + kTT + r * 128 + grp * 4 + kord;  // my token of the next tile
        if (tile + 1 < ntiles && t < vend) kn_next[r] = __half2float(a.knorms[kv_row0 + t]);
      }
      const uint8_t* st = smem + P::OFF_STAGE + static_cast<size_t>(tile % kStages) * P::STAGE;
#pragma unroll
      for (int round = 0; round < ROUNDS; ++round) {
        const int tbase = round * 128 + grp * 4;
#pragma unroll
        for (int pass = 0; pass < P::PASSES; ++pass) {
          if constexpr (P::PASSES > 1) {
#pragma unroll
            for (int h = 0; h < HG; ++h)
#pragma unroll
              for (int i = 0; i < J / 2; ++i) {
                const float* qrow = qs + (pass * HG + h) * D + J * sl + 2 * i;
                qp[h][i] = make_float2(qrow[0], qrow[1]);
              }
          }
          float v[4][HG];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t bits = load_slice<D, BITS, J>(st + (tbase + (k ^ kord)) * R, sl);
            factored_slice<BITS, J, HG>(bits, reinterpret_cast<const uint8_t*>(tab), rep_off, qp, v[k]);
          }
#pragma unroll
          for (int h = 0; h < HG; ++h) {
            v[0][h] += __shfl_xor_sync(0xffffffffu, v[2][h], 4);
            v[1][h] += __shfl_xor_sync(0xffffffffu, v[3][h], 4);
            v[0][h] += __shfl_xor_sync(0xffffffffu, v[1][h], 2);
            v[0][h] += __shfl_xor_sync(0xffffffffu, v[0][h], 1);
          }
          const int tt = tbase + kord;
          if (tt < nt) {
            const float n = kn_cur[round];
            // lanes 2m and 2m+1 hold the same sums; each writes half of the heads
#pragma unroll
            for (int h = 0; h < HG; ++h)
              if ((h & 1) == (sl & 1))
                out[static_cast<size_t>(pass * HG + h) * a.T + t0 + tt] = v[0][h] * n;
          }
        }
      }
    }
    cp_async_wait<0>();
  }
}

// ---- staging layout for one-thread-per-row reads ---------------------------------------------------------------
//
// Staging layout for one-thread-per-row reads: the 16-byte chunk c of row t sits at chunk position c ^ f(t), so
// that the 8 threads of a quarter warp reading chunk c of 8 consecutive rows hit 8 different bank groups.
// Rows of 64 bytes use f(t) = (t >> 1) & 3, rows of 32 bytes f(t) = (t >> 2) & 1; other rows are unswizzled.
template <int R>
__device__ __forceinline__ int stage_swizzle(int o) {
  if constexpr (R == 64) {
    const int t = o >> 6, c = (o >> 4) & 3;
    return (t << 6) | ((c ^ ((t >> 1) & 3)) << 4) | (o & 15);
  } else if constexpr (R == 32) {
    const int t = o >> 5, c = (o >> 4) & 1;
    return (t << 5) | ((c ^ ((t >> 2) & 1)) << 4) | (o & 15);
  } else {
    return o;
  }
}

template <int R>
__device__ __forceinline__ void load_swizzled_row(const uint8_t* stage, int t, uint32_t* w) {
  if constexpr (R % 16 == 0) {
#pragma unroll
    for (int c = 0; c < R / 16; ++c) {
      const uint4 u = *reinterpret_cast<const uint4*>(stage + stage_swizzle<R>(t * R + c * 16));
      w[4 * c] = u.x; w[4 * c + 1] = u.y; w[4 * c + 2] = u.z; w[4 * c + 3] = u.w;
    }
  } else {
#pragma unroll
    for (int c = 0; c < R / 8; ++c) {
      const uint2 u = *reinterpret_cast<const uint2*>(stage + t * R + c * 8);
      w[2 * c] = u.x; w[2 * c + 1] = u.y;
    }
  }
}

}  // namespace axr
