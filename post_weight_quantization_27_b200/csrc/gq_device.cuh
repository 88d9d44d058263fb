// Device-side helpers shared by the libgq kernels (sm_100a only):
// mbarrier waits with a time limit, TMA tile loads (no multicast), tcgen05
// tensor-memory allocation / MMA / loads, and the 4-bit grid arithmetic.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gq {

// Any single device-side wait gives up after this long and reports
// GQ_ERR_TIMEOUT instead of spinning forever.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// Status words live at the start of each workspace (256 bytes reserved).
constexpr size_t kWsHeader = 256;
enum : int { kDevOk = 0, kDevTimeout = 7, kDevNotPd = 5 };

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Wait until the phase with the given parity has completed.  Returns false
// (without waiting further) once limit_ns has passed.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity,
                                          uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
}

// Cluster of CTAs: rank of this CTA, the shared::cluster address of a
// shared-memory word of another CTA, arrivals on a barrier of another CTA
// and waits that observe them, and the barrier of all threads of the
// cluster.
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
// Arrive (release at cluster scope) on the barrier at the same offset in
// CTA `rank` of the cluster.
__device__ __forceinline__ void mbar_arrive_cluster(uint64_t *bar, uint32_t rank) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(
                   mapa_shared(smem_u32(bar), rank))
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// mbar_wait for a barrier that threads of other CTAs arrive on.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t *bar, uint32_t parity,
                                                  uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
// 2-D tiled load of one box into shared memory; completion is signalled on
// `bar` as transaction bytes.  x is the inner (contiguous) coordinate.
__device__ __forceinline__ void tma_load_2d(void *smem_dst, const CUtensorMap *map, uint64_t *bar,
                                            int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// 2-D tiled store of one box from shared memory (bulk-group completion).
// The box is clipped to the tensor's bounds.  Writes to the box made with
// ordinary stores must be fenced (fence_proxy_async_smem) before the store.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, const void *smem_src,
                                             int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(smem_src)), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void bulk_commit_group() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until every committed bulk store of this thread has finished reading
// shared memory (the source may then be overwritten).
__device__ __forceinline__ void bulk_wait_group_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Wait until every committed bulk store of this thread has completed.
__device__ __forceinline__ void bulk_wait_group0() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (TMA, tensor cores).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// Barrier over `count` threads (a multiple of 32) on hardware barrier `id`.
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t *smem_dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(smem_dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
// The same for a CTA pair (cta_group::2): executed by one warp in each of
// the two CTAs; every tcgen05 operation of such a kernel uses cta_group::2.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t *smem_dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(smem_dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
// Arrive once on the barrier at this offset in each CTA of `cta_mask` when
// every tcgen05.mma (cta_group::2) issued so far by this thread has completed.
__device__ __forceinline__ void mma_commit_pair(uint64_t *bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)),
      "h"(cta_mask)
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor for a 128-byte-swizzled operand tile
// (layout type 2 in bits 61..63, descriptor version 1 in bits 46..47).
// lbo / sbo are byte strides: for an MN-major tile, lbo is the stride
// between 64-element chunks along M (or N) and sbo the stride between
// groups of 8 rows along K; for a K-major tile sbo is the stride between
// groups of 8 rows along M (or N) and lbo is unused (one swizzle atom
// spans the whole 64-element K extent).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo,
                                                    uint32_t layout = 2) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)layout << 61;
  return d;
}
// Layout type 1: 128-byte swizzle with 32-byte atoms, the one layout the
// tensor core accepts for MN-major 32-bit (TF32) operands; atoms are 4 rows
// of 128 bytes, so sbo is the stride between groups of 4 K rows.
constexpr uint32_t kLayoutSw128Atom32 = 1;

// Instruction descriptor of tcgen05.mma kind::f16 with bf16 A and B and an
// fp32 accumulator; a_mn / b_mn select MN-major operands.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4)                         // D format f32
         | (1u << 7)                       // A format bf16
         | (1u << 10)                      // B format bf16
         | ((a_mn ? 1u : 0u) << 15)        // A major
         | ((b_mn ? 1u : 0u) << 16)        // B major
         | ((uint32_t)(N >> 3) << 17)      // N / 8
         | ((uint32_t)(M >> 4) << 24);     // M / 16
}

// D[tmem] (+)= A[smem] * B[smem]^T, issued by one thread.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// The same MMA of a CTA pair (cta_group::2, issued by one thread of CTA 0):
// M = 256 rows, the A rows and B columns of each CTA's half read from that
// CTA's shared memory at the descriptors' offsets.
__device__ __forceinline__ void mma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                              uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on `bar` when every tcgen05.mma issued so far by this thread
// has completed.
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane, with the wait
// for completion in the same statement so the registers are valid after.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Record a device-side failure in a workspace status word (first one wins).
__device__ __forceinline__ void set_status(int *status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// ---------------------------------------------------------------- 4-bit grid
// One group's 16-bit scale and integer zero-point, in IEEE fp32 with
// round-to-nearest-even, identical op order for RTN and GPTQ.
struct GridParams {
  float s;     // the fp16-rounded scale, as float
  float z;     // zero-point (0 for symmetric)
  uint16_t s_bits, z_bits;
};

__device__ __forceinline__ GridParams grid_from_scale(float s32, float mn) {
  // s32: raw scale; mn: min' of the group (0 for symmetric).
  GridParams g;
  __half h = __float2half_rn(fminf(s32, 65504.0f));
  bool degenerate = __half2float(h) == 0.0f;
  if (degenerate) h = __float2half_rn(1.0f);
  g.s = __half2float(h);
  g.s_bits = __half_as_ushort(h);
  float z = rintf(__fdiv_rn(-mn, g.s));
  z = fminf(fmaxf(z, 0.0f), 15.0f);
  if (degenerate) z = 0.0f;
  z = __fadd_rn(z, 0.0f);  // -0 -> +0
  g.z = z;
  g.z_bits = __half_as_ushort(__float2half_rn(z));
  return g;
}
__device__ __forceinline__ GridParams grid_sym(float absmax) {
  return grid_from_scale(__fdiv_rn(absmax, 7.0f), 0.0f);
}
__device__ __forceinline__ GridParams grid_affine(float vmin, float vmax) {
  const float mn = fminf(vmin, 0.0f), mx = fmaxf(vmax, 0.0f);
  return grid_from_scale(__fdiv_rn(__fsub_rn(mx, mn), 15.0f), mn);
}
// Integer code of w (sym: -7..7, affine: 0..15).
__device__ __forceinline__ float grid_code(float w, const GridParams &g, bool sym) {
  float c = __fadd_rn(rintf(__fdiv_rn(w, g.s)), g.z);
  return sym ? fminf(fmaxf(c, -7.0f), 7.0f) : fminf(fmaxf(c, 0.0f), 15.0f);
}
// Correctly rounded fp32 quotient a / b given r = RN(1 / b): q0 = RN(a r) is
// within one ulp of a / b, and one FMA correction q0 + r (a - b q0) gives the
// round-to-nearest quotient (P. Markstein, "Computation of elementary
// functions on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1),
// 1990).  Used where the divisor is fixed for many quotients; checked
// against __fdiv_rn by the GPTQ == RTN tests on diagonal Hessians.
__device__ __forceinline__ float div_by_recip(float a, float b, float r) {
  const float q0 = __fmul_rn(a, r);
  const float e = __fmaf_rn(-q0, b, a);
  return __fmaf_rn(e, r, q0);
}
// Integer code of w and its stored nibble, with rs = RN(1 / s).  The
// quotient is clamped to the code range first (equivalent, since the bounds
// are integers), then rounded half-to-even exactly by adding 1.5 * 2^23: for
// |q| <= 16 the sum lies in [2^23, 2^24), where the spacing is 1 and the
// constant is even, so the rounded sum is C + rint(q) and its low mantissa
// bits are the code.  No float-to-int conversion is needed.
__device__ __forceinline__ float grid_code_fast(float w, const GridParams &g, float rs, bool sym,
                                                uint32_t &nib) {
  constexpr float C = 12582912.0f;  // 1.5 * 2^23
  const float q = div_by_recip(w, g.s, rs);
  if (sym) {
    const float t = __fadd_rn(fminf(fmaxf(q, -7.0f), 7.0f), C);
    nib = (__float_as_uint(t) + 8u) & 0xFu;  // c + 8
    return __fsub_rn(t, C);
  }
  const float r = __fsub_rn(__fadd_rn(fminf(fmaxf(q, -16.0f), 16.0f), C), C);  // rint(q)
  const float c = fminf(fmaxf(__fadd_rn(r, g.z), 0.0f), 15.0f);
  nib = __float_as_uint(__fadd_rn(c, C)) & 0xFu;
  return c;
}
// Code of w with the group's reciprocal scale rs = RN(1 / s).
__device__ __forceinline__ float grid_code_r(float w, const GridParams &g, float rs, bool sym) {
  float c = __fadd_rn(rintf(div_by_recip(w, g.s, rs)), g.z);
  return sym ? fminf(fmaxf(c, -7.0f), 7.0f) : fminf(fmaxf(c, 0.0f), 15.0f);
}
// Stored nibble of a code.
__device__ __forceinline__ uint32_t grid_nibble(float c, bool sym) {
  return static_cast<uint32_t>(static_cast<int>(c) + (sym ? 8 : 0)) & 0xFu;
}

// ---------------------------------------------------------------- any width
// The same grid with BITS-bit codes: symmetric -q..q with q = 2^(BITS-1) - 1,
// s = absmax / q, stored as c + 2^(BITS-1); affine 0..m with m = 2^BITS - 1,
// s = (max' - min') / m, z = rint(-min' / s) clamped to 0..m.  IEEE fp32
// with round-to-nearest-even throughout, the operation order of the 4-bit
// functions above (which they reproduce at BITS = 4).
template <int BITS>
struct BitGrid {
  static constexpr int kQ = (1 << (BITS - 1)) - 1;   // symmetric end code
  static constexpr int kM = (1 << BITS) - 1;         // affine end code
  static constexpr uint32_t kMask = (1u << BITS) - 1u;
  static constexpr uint32_t kOffset = 1u << (BITS - 1);
};

template <int BITS>
__device__ __forceinline__ GridParams grid_from_scale_b(float s32, float mn) {
  GridParams g;
  __half h = __float2half_rn(fminf(s32, 65504.0f));
  const bool degenerate = __half2float(h) == 0.0f;
  if (degenerate) h = __float2half_rn(1.0f);
  g.s = __half2float(h);
  g.s_bits = __half_as_ushort(h);
  float z = rintf(__fdiv_rn(-mn, g.s));
  z = fminf(fmaxf(z, 0.0f), static_cast<float>(BitGrid<BITS>::kM));
  if (degenerate) z = 0.0f;
  z = __fadd_rn(z, 0.0f);  // -0 -> +0
  g.z = z;
  g.z_bits = __half_as_ushort(__float2half_rn(z));
  return g;
}
template <int BITS>
__device__ __forceinline__ GridParams grid_sym_b(float absmax) {
  return grid_from_scale_b<BITS>(__fdiv_rn(absmax, static_cast<float>(BitGrid<BITS>::kQ)), 0.0f);
}
template <int BITS>
__device__ __forceinline__ GridParams grid_affine_b(float vmin, float vmax) {
  const float mn = fminf(vmin, 0.0f), mx = fmaxf(vmax, 0.0f);
  return grid_from_scale_b<BITS>(
      __fdiv_rn(__fsub_rn(mx, mn), static_cast<float>(BitGrid<BITS>::kM)), mn);
}
// Integer code of w (as float) and its stored value, with rs = RN(1 / s):
// c = clamp(rint(w / s) + z) in IEEE fp32.
template <int BITS>
__device__ __forceinline__ float grid_code_b(float w, const GridParams &g, float rs, bool sym,
                                             uint32_t &stored) {
  const float r = rintf(div_by_recip(w, g.s, rs));
  float c;
  if (sym) {
    c = fminf(fmaxf(r, -static_cast<float>(BitGrid<BITS>::kQ)),
              static_cast<float>(BitGrid<BITS>::kQ));
    stored = static_cast<uint32_t>(static_cast<int>(c) + static_cast<int>(BitGrid<BITS>::kOffset));
  } else {
    c = fminf(fmaxf(__fadd_rn(r, g.z), 0.0f), static_cast<float>(BitGrid<BITS>::kM));
    stored = static_cast<uint32_t>(static_cast<int>(c));
  }
  return c;
}
// OR the stored value of column k (of a run of columns starting on a word
// boundary) into its place in the little-endian bit stream held in words[].
template <int BITS, int K, int NW>
__device__ __forceinline__ void put_code(uint32_t (&words)[NW], uint32_t stored) {
  constexpr int bit = BITS * K, w = bit / 32, off = bit % 32;
  words[w] |= stored << off;
  if constexpr (off + BITS > 32) words[w + 1] |= stored >> (32 - off);
}
// put_code with a run-time column index.
__device__ __forceinline__ void put_code_rt(uint32_t *words, int bits, int k, uint32_t stored) {
  const int bit = bits * k, w = bit >> 5, off = bit & 31;
  words[w] |= stored << off;
  if (off + bits > 32) words[w + 1] |= stored >> (32 - off);
}
// Stored value of column k of a run of columns starting on a word boundary.
__device__ __forceinline__ uint32_t get_code(const uint32_t *words, int bits, int k) {
  const int bit = bits * k, w = bit >> 5, off = bit & 31;
  uint32_t v = words[w] >> off;
  if (off + bits > 32) v |= words[w + 1] << (32 - off);
  return v & ((1u << bits) - 1u);
}

}  // namespace gq
