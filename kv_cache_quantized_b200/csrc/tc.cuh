// Tensor-core scoring of 128-token tiles (sm_100a tcgen05): the key side of the read path as one small MMA.
//
// The scores of a tile are D[t][n] = sum_k A[t][k] B[k][n] with
//   A[t][k]  the token's centroids in the rotated domain, split into two fp16 planes: k < d holds hi(c) and
//            k >= d holds lo(c) = c - hi(c) for coordinate k mod d (so A carries about 22 bits of each centroid);
//   B[k][n]  the query's row factors split the same way: column 2h holds hi(q~_h) against both planes, column 2h+1
//            holds lo(q~_h) against the hi plane only, so that D[t][2h] + D[t][2h+1] = sum_j c_j q~_{h,j} up to the
//            product of the two lo parts (relative 2^-22).
// A lives in tensor memory (TMEM lane t = token t of the tile, column k/2, two fp16 per column) and is written by
// the 128 scoring threads with tcgen05.st; B lives in shared memory in the K-major, no-swizzle canonical layout
// (8-row x 16-byte core matrices, 128 B apart along K, 8 rows of N apart by the whole K extent); the accumulator D
// (fp32, N = 16 columns) lives in TMEM next to A.  One thread issues d/8 MMAs of K = 16 (M = 128, N = 16) and commits
// them to an mbarrier that the scoring threads wait on (bounded).
//
// The centroid pairs come from a byte-indexed table like the factored gather's: entry e (two coordinates' codes)
// holds (hi(c_lo), hi(c_hi)) and (lo(c_lo), lo(c_hi)) as two half2 -- eight bytes -- replicated once per lane
// (256-byte entry stride) so that one byte permute gives the lane's offset.
#pragma once

#include <cuda_fp16.h>

#include <type_traits>

#include "axr_common.cuh"

namespace axr {
namespace tc {

constexpr int kM = 128;  // tokens per tile = TMEM lanes
constexpr int kN = 16;   // accumulator columns: 2 per head, up to 8 heads

template <int D>
struct Layout {
  static constexpr int ACOLS = D;                 // 2*D fp16 per row = D columns (hi plane, then lo plane)
  static constexpr int DCOL = ACOLS;              // accumulator columns start after A
  static constexpr int NCOLS = (ACOLS + kN) <= 32 ? 32 : (ACOLS + kN) <= 64 ? 64 : (ACOLS + kN) <= 128 ? 128 : 256;
  static constexpr int KSTEPS = 2 * D / 16;       // MMAs of K = 16
  static constexpr int B_BYTES = kN * 2 * D * 2;  // N x K fp16
  static constexpr uint32_t SBO = 2 * D / 8 * 128;  // bytes between 8-row groups of N
};

// ---- PTX wrappers ----------------------------------------------------------------------------------------------

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, int ncols) {  // one full warp
  const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(dst_smem));
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst), "r"(ncols));
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, int ncols) {  // the allocating warp
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols));
}
__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void st_x32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]),
      "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]),
      "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void ld_x16(uint32_t taddr, uint32_t (&d)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3]), "=r"(d[4]), "=r"(d[5]), "=r"(d[6]), "=r"(d[7]),
        "=r"(d[8]), "=r"(d[9]), "=r"(d[10]), "=r"(d[11]), "=r"(d[12]), "=r"(d[13]), "=r"(d[14]), "=r"(d[15])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void st_x16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* mbar) {
  const uint32_t mb = static_cast<uint32_t>(__cvta_generic_to_shared(mbar));
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(mb) : "memory");
}

// The mbarrier counts one arrival once every cp.async this thread issued so far has landed (the arrival is part of
// the barrier's expected count: no pending-count increment).
__device__ __forceinline__ void cp_async_mbar_arrive(uint64_t* mbar) {
  const uint32_t mb = static_cast<uint32_t>(__cvta_generic_to_shared(mbar));
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(mb) : "memory");
}

// Instruction descriptor of kind::f16: fp16 A and B (K-major), fp32 accumulator, M = 128, N = 16.
__host__ __device__ constexpr uint32_t idesc_f16_m128_n16() {
  return (1u << 4) | (static_cast<uint32_t>(kN >> 3) << 17) | (static_cast<uint32_t>(kM >> 4) << 24);
}

// Shared-memory matrix descriptor: no swizzle, leading (K) byte offset 128, stride (N) byte offset sbo, version 1.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t sbo) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(128u >> 4) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

// The d/8 MMAs of one tile: D (TMEM, fp32, N columns at d_taddr) = A (TMEM, hi/lo planes from column a_taddr) x B
// (shared memory at b_saddr), committed to mbar once they have all completed.
template <int D>
__device__ __forceinline__ void issue_mma(uint32_t a_taddr, uint32_t d_taddr, uint32_t b_saddr, uint64_t* mbar) {
  using LY = Layout<D>;
  const uint32_t idesc = idesc_f16_m128_n16();
#pragma unroll
  for (int s = 0; s < LY::KSTEPS; ++s) {
    const uint64_t desc = smem_desc(b_saddr + static_cast<uint32_t>(s) * 256u, LY::SBO);
    const uint32_t acc = s > 0 ? 1u : 0u;
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_taddr),
        "r"(a_taddr + static_cast<uint32_t>(s * 8)), "l"(desc), "r"(idesc), "r"(acc)
        : "memory");
  }
  const uint32_t mb = static_cast<uint32_t>(__cvta_generic_to_shared(mbar));
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mb) : "memory");
}

__device__ __forceinline__ void mbar_init(uint64_t* mbar, uint32_t count) {
  const uint32_t mb = static_cast<uint32_t>(__cvta_generic_to_shared(mbar));
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(mb), "r"(count));
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Wait for the phase of parity `parity` to complete; gives up after `polls` try_wait polls and returns false.
__device__ __forceinline__ bool mbar_wait_polls(uint64_t* mbar, uint32_t parity, int polls) {
  const uint32_t mb = static_cast<uint32_t>(__cvta_generic_to_shared(mbar));
  for (int it = 0; it < polls; ++it) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(mb), "r"(parity)
        : "memory");
    if (done) return true;
  }
  return false;
}

// Wait for the phase of parity `parity` to complete; gives up after a bounded number of polls (about a second)
// and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t* mbar, uint32_t parity) {
  return mbar_wait_polls(mbar, parity, 1 << 20);
}

// ---- tables and operands ----------------------------------------------------------------------------------------

template <int BITS>
struct PairTable16 {
  static constexpr int L = 1 << BITS;
  static constexpr int E = L * L;
  static constexpr int BYTES = E * 32 * 8;  // 32 copies of 8 bytes per entry
};

// hi/lo fp16 planes of the unit-scale (N(0,1)) centroids gamma_k
template <int BITS>
__device__ __forceinline__ void build_table(const float* __restrict__ gamma, uint2* __restrict__ tab) {
  using P = PairTable16<BITS>;
  for (int i = threadIdx.x; i < P::E * 32; i += blockDim.x) {
    const int e = i >> 5;
    const float c0 = gamma[e & (P::L - 1)], c1 = gamma[e >> BITS];
    const __half h0 = __float2half_rn(c0), h1 = __float2half_rn(c1);
    const __half l0 = __float2half_rn(c0 - __half2float(h0)), l1 = __float2half_rn(c1 - __half2float(h1));
    const __half2 hi = __halves2half2(h0, h1), lo = __halves2half2(l0, l1);
    tab[i] = make_uint2(*reinterpret_cast<const uint32_t*>(&hi), *reinterpret_cast<const uint32_t*>(&lo));
  }
}

// Byte offset of this lane's copy of the pair at byte/field i of a packed row; repw = 8 * lane.
template <int BITS>
__device__ __forceinline__ uint32_t pair_off(const uint32_t* w, int i, uint32_t repw) {
  if constexpr (BITS == 4) {
    return __byte_perm(w[i >> 2], repw, 0x5504u | (static_cast<uint32_t>(i & 3) << 4));
  } else {
    return (bits_at<2 * BITS>(w, 2 * BITS * i) << 8) | repw;
  }
}

// Power-of-two range scale of one head's query operand: 2^(14 - e) with |mult| * ||q|| in [2^(e-1), 2^e).  Every
// |q~_j| is at most |mult| * ||q|| (the transform is orthonormal), so the scaled factors stay below 2^14 in fp16
// while keeping fp16's relative precision; the epilogue divides it out.  Computed by a whole warp from the query in
// global memory, identically wherever it is needed.
template <int D>
__device__ __forceinline__ float head_scale(const float* __restrict__ qh, float mult) {
  const int lane = threadIdx.x & 31;
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < (D + 31) / 32; ++i) {
    const int j = lane + 32 * i;
    const float x = j < D ? qh[j] : 0.f;
    ss = fmaf(x, x, ss);
  }
  const float m = sqrtf(warp_sum(ss)) * fabsf(mult);
  if (!(m > 0.f) || !isfinite(m)) return 1.f;
  int e = 0;
  frexpf(m, &e);
  return ldexpf(1.f, 14 - e);
}

// B operand of the G heads of one KV head, built by one warp from the raw queries: q~_h = mult * H (s .* q_h) in
// registers (lane l holds coordinates 4l .. 4l + 3 for d = 128), scaled by head_scale, split into hi/lo fp16.
// Column 2h holds hi against both A planes, column 2h+1 holds lo against the hi plane; every other entry of the
// operand is zero and is written once (zero_b) -- only the 3 G d live entries are stored per row.
template <int D>
__device__ __forceinline__ int b_off(int n, int k) {  // K-major, no-swizzle canonical layout, in halves
  return (n >> 3) * (Layout<D>::SBO / 2) + (k >> 3) * 64 + (n & 7) * 8 + (k & 7);
}

template <int D, int G>
__device__ __forceinline__ void build_b_warp(const float* __restrict__ qg, const int8_t* __restrict__ signs,
                                             float mult, __half* __restrict__ bs) {
  constexpr int VPL = D / 32;  // coordinates per lane, consecutive: they share one 16-byte core-matrix row
  static_assert(VPL == 2 || VPL == 4, "d = 64 or 128");
  using Vec = typename std::conditional<VPL == 4, uint2, uint32_t>::type;
  const int lane = threadIdx.x & 31;
  const float norm = mult * rsqrtf(static_cast<float>(D));
  float sg[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) sg[i] = signs[VPL * lane + i] < 0 ? -1.f : 1.f;
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float v[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) v[i] = qg[h * D + VPL * lane + i] * sg[i];
    fwht_warp<D>(v, lane);
    const float sc = head_scale<D>(qg + h * D, mult);
    uint32_t hw[VPL / 2], lw[VPL / 2];
#pragma unroll
    for (int i = 0; i < VPL; i += 2) {
      const float q0 = v[i] * norm * sc, q1 = v[i + 1] * norm * sc;
      const __half h0 = __float2half_rn(q0), h1 = __float2half_rn(q1);
      const __half2 hh = __halves2half2(h0, h1);
      const __half2 ll = __halves2half2(__float2half_rn(q0 - __half2float(h0)), __float2half_rn(q1 - __half2float(h1)));
      hw[i / 2] = *reinterpret_cast<const uint32_t*>(&hh);
      lw[i / 2] = *reinterpret_cast<const uint32_t*>(&ll);
    }
    *reinterpret_cast<Vec*>(bs + b_off<D>(2 * h, VPL * lane)) = *reinterpret_cast<const Vec*>(hw);
    *reinterpret_cast<Vec*>(bs + b_off<D>(2 * h, D + VPL * lane)) = *reinterpret_cast<const Vec*>(hw);
    *reinterpret_cast<Vec*>(bs + b_off<D>(2 * h + 1, VPL * lane)) = *reinterpret_cast<const Vec*>(lw);
  }
}

}  // namespace tc
}  // namespace axr
