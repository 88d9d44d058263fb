// fp32 GEMM on the tensor cores: C = beta C + alpha A B with fp32 A, B, C.
//
// Used for the GPTQ lazy trailing update W[:, end:] -= Err U[blk, end:]
// ("GPTQ: Post-Training INT4" -- "The GPTQ Algorithm", block-wise
// processing) and for the blocked Cholesky's panel solves and trailing
// updates.  Those updates decide later rounding decisions, so they need
// fp32-level accuracy: each operand element a is split into a TF32-exact
// high part h = a with the low 13 mantissa bits cleared and the remainder
// l = a - h (exact in fp32), and the product is h_a h_b + h_a l_b + l_a h_b
// (three tcgen05.mma kind::tf32; the dropped l_a l_b and the TF32 rounding
// of l are ~2^-20 relative).  The tensor core reads only the high 19 bits of
// each 32-bit TF32 operand (results are bit-identical whether the low 13
// bits are cleared or not), so the staged fp32 tile itself serves as h and
// only l is written.
//
// Persistent kernel, one CTA per SM, 128 x 128 output tiles, K in steps of
// 32 (one 128-byte swizzle row of fp32):
//   warp 0     TMA loads of the fp32 A and B tiles (no multicast)
//   warps 2-5  write l = a - h of each staged element into a second buffer,
//              then make the writes visible to the async proxy before
//              releasing the stage to the MMA warp
//   warp 1     three MMAs per 8-wide K step into one of two TMEM
//              accumulators (the epilogue of one tile overlaps the next)
//   warps 6-9  epilogue: the C tile passes through two staging buffers in
//              chunks of 32 columns -- the next chunk is fetched by TMA
//              while each thread (one accumulator row) forms beta C + alpha
//              acc of the current one, which TMA stores (clipped at the
//              matrix edge).  Global memory is only touched by TMA copies.
// Large products run on CTA pairs instead (gemm_pair_kernel, below: 256 x
// 256 tiles, tcgen05 cta_group::2), as does the bf16 SYRK of the error
// from the Hessian.
// A is K-major (A(m, k) = A[m lda + k]); B is either K-major (B(k, n) =
// B[n ldb + k]) or N-major (B(k, n) = B[k ldb + n]); an N-major TF32 operand
// must be staged with the 32-byte-atom variant of the 128-byte swizzle.  With `lower` only
// tiles and elements with n <= m are computed and stored.
#include "gq_device.cuh"
#include "gq_internal.h"

namespace gq {
namespace {

constexpr int TM = 128, TN = 128, TK = 32, STAGES = 3;
constexpr int TILE_BYTES = TM * TK * 4;         // 16 KB, A or B tile
constexpr int STAGE_BYTES = 4 * TILE_BYTES;     // A_h, A_l, B_h, B_l
constexpr int C_BYTES = TM * TN * 4;            // a C tile: 4 boxes [128 rows][32 fp32]
constexpr int C_STAGE_BYTES = C_BYTES / 2;      // two staging buffers of 32 columns each
constexpr int C_BUF_BYTES = C_BYTES / 4;        // one buffer: [128 rows][32 fp32], one TMA box
constexpr int NUM_THREADS = 320;
constexpr uint32_t TMEM_COLS = 256;
constexpr size_t SMEM_BYTES = STAGES * STAGE_BYTES + C_STAGE_BYTES + 1024 + 256;

struct TcArgs {
  int M, N, K;
  float alpha, beta;
  float *C;
  int64_t ldc;
  int n_mt, n_nt, nkb, n_tiles;
  int b_kmajor, lower;
  int *status;
  double *dot;  // dot mode: [n_tiles] sum over the tile of (alpha A B) * C; C not written
                // (with lower: the strictly lower elements counted twice, the diagonal
                // once, the rest not at all -- the full sum for symmetric A B and C)
};

__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N, bool b_mn) {
  return (1u << 4)                     // D f32
         | (2u << 7)                   // A tf32
         | (2u << 10)                  // B tf32
         | ((b_mn ? 1u : 0u) << 16)    // B major
         | ((uint32_t)(N >> 3) << 17)
         | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_tf32(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_tf32_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                              uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Tile t -> (mt, nt).  General: groups of RASTER_GM row tiles, row tile
// fastest inside a group, so that the tiles in flight at one time share a
// few operand slabs in L2 (a long K makes each slab larger than L2 can hold
// for all row tiles at once).  lower: only nt <= mt, enumerated row by row.
constexpr int RASTER_GM = 16;
__device__ __forceinline__ void tile_of(const TcArgs &a, int t, int &mt, int &nt) {
  if (!a.lower) {
    const int per_group = RASTER_GM * a.n_nt;
    const int g = t / per_group;
    const int r = t - g * per_group;
    const int rows = min(RASTER_GM, a.n_mt - g * RASTER_GM);
    mt = g * RASTER_GM + r % rows;
    nt = r / rows;
    return;
  }
  int r = static_cast<int>((sqrtf(8.0f * t + 1.0f) - 1.0f) * 0.5f);
  while (r * (r + 1) / 2 > t) --r;
  while ((r + 1) * (r + 2) / 2 <= t) ++r;
  mt = r;
  nt = t - r * (r + 1) / 2;
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_tf32x3_kernel(const __grid_constant__ CUtensorMap tmA,
                       const __grid_constant__ CUtensorMap tmB,
                       const __grid_constant__ CUtensorMap tmC, TcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *cs = smem + STAGES * STAGE_BYTES;  // C staging (half a tile), 1024-byte aligned
  uint64_t *bars = reinterpret_cast<uint64_t *>(cs + C_STAGE_BYTES);
  uint64_t *full = bars;                  // TMA landed
  uint64_t *split = bars + STAGES;        // h / l split done
  uint64_t *empty = bars + 2 * STAGES;    // MMAs done with the stage
  uint64_t *acc_full = bars + 3 * STAGES;
  uint64_t *acc_empty = acc_full + 2;
  uint64_t *drain = acc_empty + 2;
  uint64_t *c_full = drain + 1;           // [2]: a C chunk landed in staging buffer b
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(c_full + 2);
  double *red = reinterpret_cast<double *>(bars + 17);  // dot mode: one per epilogue warp

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&split[s], 4);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    mbar_init(drain, 1);
    mbar_init(&c_full[0], 1);
    mbar_init(&c_full[1], 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmC);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      bool ok = true;
      uint32_t it = 0;
      for (int t = blockIdx.x; t < a.n_tiles && ok; t += gridDim.x) {
        int mt, nt;
        tile_of(a, t, mt, nt);
        for (int kb = 0; kb < a.nkb; ++kb, ++it) {
          const uint32_t s = it % STAGES, r = it / STAGES;
          if (!mbar_wait(&empty[s], (r & 1) ^ 1)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[s], 2 * TILE_BYTES);
          uint8_t *st = smem + s * STAGE_BYTES;
          tma_load_2d(st, &tmA, &full[s], kb * TK, mt * TM);
          if (a.b_kmajor) {
            tma_load_2d(st + 2 * TILE_BYTES, &tmB, &full[s], kb * TK, nt * TN);
          } else {
#pragma unroll
            for (int q = 0; q < 4; ++q)
              tma_load_2d(st + 2 * TILE_BYTES + q * (TILE_BYTES / 4), &tmB, &full[s],
                          nt * TN + 32 * q, kb * TK);
          }
        }
      }
      const uint32_t n_wait = it < STAGES ? it : STAGES;
      for (uint32_t k = 0; k < n_wait; ++k) {
        const uint32_t j = it - 1 - k;
        if (!mbar_wait(&full[j % STAGES], (j / STAGES) & 1)) ok = false;
      }
      if (!ok) set_status(a.status, kDevTimeout);
    }
  } else if (warp >= 2 && warp <= 5) {
    // ---------------- h / l split of each staged tile
    const int ct = threadIdx.x - 64;  // 0..127
    bool ok = true;
    uint32_t it = 0;
    for (int t = blockIdx.x; t < a.n_tiles && ok; t += gridDim.x) {
      for (int kb = 0; kb < a.nkb; ++kb, ++it) {
        const uint32_t s = it % STAGES, r = it / STAGES;
        ok = __all_sync(0xffffffffu, mbar_wait(&full[s], r & 1));
        if (!ok) break;
        uint8_t *st = smem + s * STAGE_BYTES;
#pragma unroll
        for (int op = 0; op < 2; ++op) {
          float4 *hp = reinterpret_cast<float4 *>(st + op * 2 * TILE_BYTES);
          float4 *lp = reinterpret_cast<float4 *>(st + op * 2 * TILE_BYTES + TILE_BYTES);
#pragma unroll
          for (int i = 0; i < TILE_BYTES / 16 / 128; ++i) {
            const int idx = ct + 128 * i;
            const float4 v = hp[idx];
            float4 h, l;
            h.x = __uint_as_float(__float_as_uint(v.x) & 0xFFFFE000u);
            h.y = __uint_as_float(__float_as_uint(v.y) & 0xFFFFE000u);
            h.z = __uint_as_float(__float_as_uint(v.z) & 0xFFFFE000u);
            h.w = __uint_as_float(__float_as_uint(v.w) & 0xFFFFE000u);
            l.x = v.x - h.x;
            l.y = v.y - h.y;
            l.z = v.z - h.z;
            l.w = v.w - h.w;
            lp[idx] = l;
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&split[s]);
      }
    }
    if (!ok && lane == 0) set_status(a.status, kDevTimeout);
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      bool ok = true;
      uint32_t it = 0, ch = 0;
      const uint32_t idesc = idesc_tf32(TM, TN, a.b_kmajor == 0);
      for (int t = blockIdx.x; t < a.n_tiles && ok; t += gridDim.x, ++ch) {
        const uint32_t buf = ch & 1, use = ch >> 1;
        if (!mbar_wait(&acc_empty[buf], (use & 1) ^ 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem + buf * TN;
        for (int kb = 0; kb < a.nkb; ++kb, ++it) {
          const uint32_t s = it % STAGES, r = it / STAGES;
          if (!mbar_wait(&split[s], r & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t ah = smem_u32(smem + s * STAGE_BYTES);
          const uint32_t al = ah + TILE_BYTES;
          const uint32_t bh = ah + 2 * TILE_BYTES;
          const uint32_t bl = ah + 3 * TILE_BYTES;
#pragma unroll
          for (int kk = 0; kk < TK / 8; ++kk) {
            // A: K-major, 8 fp32 = 32 bytes along the swizzled row
            const uint64_t dah = smem_desc_sw128(ah + kk * 32, 16, 1024);
            const uint64_t dal = smem_desc_sw128(al + kk * 32, 16, 1024);
            uint64_t dbh, dbl;
            if (a.b_kmajor) {
              dbh = smem_desc_sw128(bh + kk * 32, 16, 1024);
              dbl = smem_desc_sw128(bl + kk * 32, 16, 1024);
            } else {
              // N-major: 32-wide N chunks of 4 KB, 32-byte-atom swizzle,
              // 4-row atoms of 512 bytes; 8 K rows per MMA = 1 KB
              dbh = smem_desc_sw128(bh + kk * 1024, TILE_BYTES / 4, 512, kLayoutSw128Atom32);
              dbl = smem_desc_sw128(bl + kk * 1024, TILE_BYTES / 4, 512, kLayoutSw128Atom32);
            }
            mma_tf32(d_tmem, dal, dbh, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
            mma_tf32(d_tmem, dah, dbl, idesc, 1u);
            mma_tf32(d_tmem, dah, dbh, idesc, 1u);
          }
          mma_commit(&empty[s]);
        }
        if (!ok) break;
        mma_commit(&acc_full[buf]);
      }
      mma_commit(drain);
      if (!mbar_wait(drain, 0)) ok = false;
      if (!ok) set_status(a.status, kDevTimeout);
    }
  } else {
    // ---------------- epilogue: warps 6..9 (thread = accumulator row).  The
    // C tile passes through two staging buffers in chunks of 32 columns:
    // while chunk k is combined with the accumulator in buffer k % 2 and
    // stored by TMA, chunk k + 1 (of this tile or of the next) is already
    // being fetched into the other buffer.  After a failed wait the warps
    // skip the work but keep meeting the named barrier, so none is left
    // waiting.
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;               // row within the tile
    const bool leader = threadIdx.x == 192;          // issues the C copies
    const bool dot = a.dot != nullptr;
    const bool need_c = a.beta != 0.0f || a.lower != 0 || dot;
    constexpr int NCH = TN / 32;                     // chunks per tile
    uint32_t ch = 0, cc = 0;                         // tiles done, chunks done
    bool ok = true;
    auto load_chunk = [&](int t, int h, uint32_t b) {
      int mt, nt;
      tile_of(a, t, mt, nt);
      mbar_arrive_expect_tx(&c_full[b], C_BUF_BYTES);
      tma_load_2d(cs + b * C_BUF_BYTES, &tmC, &c_full[b], nt * TN + 32 * h, mt * TM);
    };
    if (leader && need_c && static_cast<int>(blockIdx.x) < a.n_tiles) load_chunk(blockIdx.x, 0, 0);
    for (int t = blockIdx.x; t < a.n_tiles; t += gridDim.x, ++ch) {
      int mt, nt;
      tile_of(a, t, mt, nt);
      const uint32_t buf = ch & 1, use = ch >> 1;
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[buf], use & 1));
      tc_fence_after();
      const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + buf * TN;
      const int m = mt * TM + r;
      const bool diag = a.lower && mt == nt;
      double rs = 0.0;  // dot mode: this row's sum
#pragma unroll 1
      for (int h = 0; h < NCH; ++h, ++cc) {
        const uint32_t b = cc & 1;
        if (need_c && ok) ok = __all_sync(0xffffffffu, mbar_wait(&c_full[b], (cc >> 1) & 1));
        if (leader && ok && need_c) {
          // the other buffer's last store has been read out: fetch the next chunk into it
          if (!dot) bulk_wait_group_read0();
          if (h + 1 < NCH) {
            load_chunk(t, h + 1, b ^ 1u);
          } else {
            const int tn = t + static_cast<int>(gridDim.x);
            if (tn < a.n_tiles) load_chunk(tn, 0, b ^ 1u);
          }
        }
        if (ok) {
          float v[32];
          tmem_ld32(taddr + h * 32, v);
          uint8_t *row = cs + b * C_BUF_BYTES + r * 128;
          if (dot) {
            // (alpha acc) * C over the row (fp32 over 32 columns, fp64 across)
            float part = 0.0f, pdiag = 0.0f;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              float4 cv = *reinterpret_cast<const float4 *>(row + ((c ^ (r & 7)) << 4));
              if (diag) {  // lower: keep n < m (counted twice below), the diagonal once
                const int n = nt * TN + 32 * h + 4 * c;
                if (n == m) pdiag = fmaf(a.alpha * v[4 * c], cv.x, pdiag);
                if (n + 1 == m) pdiag = fmaf(a.alpha * v[4 * c + 1], cv.y, pdiag);
                if (n + 2 == m) pdiag = fmaf(a.alpha * v[4 * c + 2], cv.z, pdiag);
                if (n + 3 == m) pdiag = fmaf(a.alpha * v[4 * c + 3], cv.w, pdiag);
                if (n >= m) cv.x = 0.0f;
                if (n + 1 >= m) cv.y = 0.0f;
                if (n + 2 >= m) cv.z = 0.0f;
                if (n + 3 >= m) cv.w = 0.0f;
              }
              part = fmaf(a.alpha * v[4 * c], cv.x, part);
              part = fmaf(a.alpha * v[4 * c + 1], cv.y, part);
              part = fmaf(a.alpha * v[4 * c + 2], cv.z, part);
              part = fmaf(a.alpha * v[4 * c + 3], cv.w, part);
            }
            rs += (a.lower ? 2.0 : 1.0) * static_cast<double>(part) + static_cast<double>(pdiag);
          } else {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              // 128-byte swizzle: 16-byte chunk c of row r sits at chunk c ^ (r % 8)
              float4 *p = reinterpret_cast<float4 *>(row + ((c ^ (r & 7)) << 4));
              const float4 old = need_c ? *p : make_float4(0.f, 0.f, 0.f, 0.f);
              float4 o;
              o.x = fmaf(a.beta, old.x, a.alpha * v[4 * c]);
              o.y = fmaf(a.beta, old.y, a.alpha * v[4 * c + 1]);
              o.z = fmaf(a.beta, old.z, a.alpha * v[4 * c + 2]);
              o.w = fmaf(a.beta, old.w, a.alpha * v[4 * c + 3]);
              if (diag) {  // keep the strict upper part of a diagonal tile
                const int n = nt * TN + 32 * h + 4 * c;
                if (n > m) o.x = old.x;
                if (n + 1 > m) o.y = old.y;
                if (n + 2 > m) o.z = old.z;
                if (n + 3 > m) o.w = old.w;
              }
              *p = o;
            }
          }
        }
        if (h == NCH - 1) {
          // the accumulator buffer is free once its columns are in registers
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[buf]);
        }
        if (!dot) fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (leader && ok && !dot) {
          tma_store_2d(&tmC, cs + b * C_BUF_BYTES, nt * TN + 32 * h, mt * TM);
          bulk_commit_group();
          // without C loads nothing else orders the buffer's reuse two chunks on
          if (!need_c) bulk_wait_group_read0();
        }
      }
      if (dot) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) rs += __shfl_xor_sync(0xffffffffu, rs, off);
        if (lane == 0) red[quarter] = rs;
        named_bar_sync(1, 128);
        if (leader && ok) a.dot[t] = ((red[0] + red[1]) + red[2]) + red[3];
        named_bar_sync(1, 128);
      }
    }
    if (leader) bulk_wait_group0();
    if (!ok && lane == 0) set_status(a.status, kDevTimeout);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ---------------------------------------------------------------- CTA pairs
// The same product on 256 x 256 output tiles, each computed by a pair of
// CTAs on two SMs (a cluster of two; tcgen05 cta_group::2).  CTA r of the
// pair stages rows 128 r .. 128 r + 127 of the tile's A slab and columns
// 128 r .. 128 r + 127 of its B slab, in the one-CTA kernel's stage layout;
// CTA 0 issues MMAs of M = 256, N = 256 that read both CTAs' tiles, and each
// CTA's TMEM receives its 128 rows x 256 columns.  Per SM and MMA flop that
// is half the B operand reads from shared memory: the fill, the split and
// the MMA operand reads share the SM's shared-memory bandwidth, which bounds
// the one-CTA kernel's tensor pipe at about half of its rate.
//   full[s]       per CTA: its own TMA loads landed
//   split[s]      CTA 0: the split of stage s done in both CTAs (8 warps)
//   empty[s]      per CTA: the MMAs reading stage s completed (multicast commit)
//   acc_full[b]   per CTA: the tile's MMAs completed (multicast commit)
//   acc_empty[b]  CTA 0: both CTAs' epilogues read accumulator b (8 warps)
// The epilogue passes the C tile through the staging buffer in four chunks
// of 64 columns.  Dot mode writes a partial per (tile, CTA): dot[2 t + r].
//
// BF16 = true: the product A A^T of a matrix given as two bf16 parts A =
// A_h + A_l (tmA maps A_h, tmB maps A_l; rows K-major), as h h^T + h l^T +
// l h^T (the dropped l l^T and the parts' rounding are ~2^-16 relative):
// three tcgen05.mma kind::f16 per 16-wide K slice, at twice the TF32 rate
// and with no split pass (the stage holds A_h, A_l, B_h, B_l of 64 K
// elements each, loaded by TMA).  For the Hessian-route reconstruction error,
// whose 1e-3 tolerance needs far less than fp32 accuracy.
constexpr int PM = 256, PN = 256;
constexpr int TK_BF16 = 64;  // K per stage in bf16 mode (one 128-byte row)
constexpr uint32_t PAIR_TMEM_COLS = 512;

template <bool BF16>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                     const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmC, TcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *cs = smem + STAGES * STAGE_BYTES;
  uint64_t *bars = reinterpret_cast<uint64_t *>(cs + C_STAGE_BYTES);
  uint64_t *full = bars;
  uint64_t *split = bars + STAGES;
  uint64_t *empty = bars + 2 * STAGES;
  uint64_t *acc_full = bars + 3 * STAGES;
  uint64_t *acc_empty = acc_full + 2;
  uint64_t *drain = acc_empty + 2;
  uint64_t *c_full = drain + 1;           // [2]: a C chunk landed in staging buffer b
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(c_full + 2);
  double *red = reinterpret_cast<double *>(bars + 17);  // dot mode: one per epilogue warp

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = static_cast<int>(blockIdx.x >> 1), n_pairs = static_cast<int>(gridDim.x >> 1);
  if (threadIdx.x == 0) {
    for (int st = 0; st < STAGES; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&split[st], 8);
      mbar_init(&empty[st], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 8);
    }
    mbar_init(drain, 1);
    mbar_init(&c_full[0], 1);
    mbar_init(&c_full[1], 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, PAIR_TMEM_COLS);
    tmem_relinquish_pair();
  }
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmC);
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers initialised and TMEM allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int row0 = static_cast<int>(rank) * TM;  // this CTA's rows (and B columns) in a tile

  if (warp == 0) {
    if (lane == 0) {
      bool ok = true;
      uint32_t it = 0;
      for (int t = pair; t < a.n_tiles && ok; t += n_pairs) {
        int mt, nt;
        tile_of(a, t, mt, nt);
        for (int kb = 0; kb < a.nkb; ++kb, ++it) {
          const uint32_t s = it % STAGES, r = it / STAGES;
          if (!mbar_wait(&empty[s], (r & 1) ^ 1)) { ok = false; break; }
          uint8_t *st = smem + s * STAGE_BYTES;
          if constexpr (BF16) {
            // A_h, A_l (rows of the tile's M half), B_h, B_l (rows of its N half)
            mbar_arrive_expect_tx(&full[s], 4 * TILE_BYTES);
            tma_load_2d(st, &tmA, &full[s], kb * TK_BF16, mt * PM + row0);
            tma_load_2d(st + TILE_BYTES, &tmB, &full[s], kb * TK_BF16, mt * PM + row0);
            tma_load_2d(st + 2 * TILE_BYTES, &tmA, &full[s], kb * TK_BF16, nt * PN + row0);
            tma_load_2d(st + 3 * TILE_BYTES, &tmB, &full[s], kb * TK_BF16, nt * PN + row0);
            continue;
          }
          mbar_arrive_expect_tx(&full[s], 2 * TILE_BYTES);
          tma_load_2d(st, &tmA, &full[s], kb * TK, mt * PM + row0);
          if (a.b_kmajor) {
            tma_load_2d(st + 2 * TILE_BYTES, &tmB, &full[s], kb * TK, nt * PN + row0);
          } else {
#pragma unroll
            for (int q = 0; q < 4; ++q)
              tma_load_2d(st + 2 * TILE_BYTES + q * (TILE_BYTES / 4), &tmB, &full[s],
                          nt * PN + row0 + 32 * q, kb * TK);
          }
        }
      }
      const uint32_t n_wait = it < STAGES ? it : STAGES;
      for (uint32_t k = 0; k < n_wait; ++k) {
        const uint32_t j = it - 1 - k;
        if (!mbar_wait(&full[j % STAGES], (j / STAGES) & 1)) ok = false;
      }
      if (!ok) set_status(a.status, kDevTimeout);
    }
  } else if (warp >= 2 && warp <= 5) {
    // ---------------- h / l split of this CTA's staged tiles
    const int ct = threadIdx.x - 64;
    bool ok = true;
    uint32_t it = 0;
    for (int t = pair; t < a.n_tiles && ok; t += n_pairs) {
      for (int kb = 0; kb < a.nkb; ++kb, ++it) {
        const uint32_t s = it % STAGES, r = it / STAGES;
        ok = __all_sync(0xffffffffu, mbar_wait(&full[s], r & 1));
        if (!ok) break;
        if constexpr (!BF16) {
          uint8_t *st = smem + s * STAGE_BYTES;
#pragma unroll
          for (int op = 0; op < 2; ++op) {
            float4 *hp = reinterpret_cast<float4 *>(st + op * 2 * TILE_BYTES);
            float4 *lp = reinterpret_cast<float4 *>(st + op * 2 * TILE_BYTES + TILE_BYTES);
#pragma unroll
            for (int i = 0; i < TILE_BYTES / 16 / 128; ++i) {
              const int idx = ct + 128 * i;
              const float4 v = hp[idx];
              float4 l;
              l.x = v.x - __uint_as_float(__float_as_uint(v.x) & 0xFFFFE000u);
              l.y = v.y - __uint_as_float(__float_as_uint(v.y) & 0xFFFFE000u);
              l.z = v.z - __uint_as_float(__float_as_uint(v.z) & 0xFFFFE000u);
              l.w = v.w - __uint_as_float(__float_as_uint(v.w) & 0xFFFFE000u);
              lp[idx] = l;
            }
          }
          fence_proxy_async_smem();
        }
        // (bf16 mode: the stage is TMA-written only; this forwards its landing)
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(&split[s], 0);
      }
    }
    if (!ok && lane == 0) set_status(a.status, kDevTimeout);
  } else if (warp == 1) {
    // ---------------- MMA issuer (CTA 0 of the pair)
    if (lane == 0 && rank == 0) {
      bool ok = true;
      uint32_t it = 0, ch = 0;
      const uint32_t idesc =
          BF16 ? idesc_bf16_f32(PM, PN, false, false) : idesc_tf32(PM, PN, a.b_kmajor == 0);
      for (int t = pair; t < a.n_tiles && ok; t += n_pairs, ++ch) {
        const uint32_t buf = ch & 1, use = ch >> 1;
        if (!mbar_wait_cluster(&acc_empty[buf], (use & 1) ^ 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem + buf * PN;
        for (int kb = 0; kb < a.nkb; ++kb, ++it) {
          const uint32_t s = it % STAGES, r = it / STAGES;
          if (!mbar_wait_cluster(&split[s], r & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t ah = smem_u32(smem + s * STAGE_BYTES);
          const uint32_t al = ah + TILE_BYTES;
          const uint32_t bh = ah + 2 * TILE_BYTES;
          const uint32_t bl = ah + 3 * TILE_BYTES;
          if constexpr (BF16) {
            // K-major bf16: 16 elements = 32 bytes along the swizzled row
#pragma unroll
            for (int kk = 0; kk < TK_BF16 / 16; ++kk) {
              const uint64_t dah = smem_desc_sw128(ah + kk * 32, 16, 1024);
              const uint64_t dal = smem_desc_sw128(al + kk * 32, 16, 1024);
              const uint64_t dbh = smem_desc_sw128(bh + kk * 32, 16, 1024);
              const uint64_t dbl = smem_desc_sw128(bl + kk * 32, 16, 1024);
              mma_bf16_pair(d_tmem, dal, dbh, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
              mma_bf16_pair(d_tmem, dah, dbl, idesc, 1u);
              mma_bf16_pair(d_tmem, dah, dbh, idesc, 1u);
            }
          } else {
#pragma unroll
            for (int kk = 0; kk < TK / 8; ++kk) {
              const uint64_t dah = smem_desc_sw128(ah + kk * 32, 16, 1024);
              const uint64_t dal = smem_desc_sw128(al + kk * 32, 16, 1024);
              uint64_t dbh, dbl;
              if (a.b_kmajor) {
                dbh = smem_desc_sw128(bh + kk * 32, 16, 1024);
                dbl = smem_desc_sw128(bl + kk * 32, 16, 1024);
              } else {
                dbh = smem_desc_sw128(bh + kk * 1024, TILE_BYTES / 4, 512, kLayoutSw128Atom32);
                dbl = smem_desc_sw128(bl + kk * 1024, TILE_BYTES / 4, 512, kLayoutSw128Atom32);
              }
              mma_tf32_pair(d_tmem, dal, dbh, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
              mma_tf32_pair(d_tmem, dah, dbl, idesc, 1u);
              mma_tf32_pair(d_tmem, dah, dbh, idesc, 1u);
            }
          }
          mma_commit_pair(&empty[s], 3);
        }
        if (!ok) break;
        mma_commit_pair(&acc_full[buf], 3);
      }
      mma_commit_pair(drain, 1);
      if (!mbar_wait(drain, 0)) ok = false;
      if (!ok) set_status(a.status, kDevTimeout);
    }
  } else {
    // ---------------- epilogue: warps 6..9 of each CTA, its 128 rows; the C
    // tile in chunks of 32 columns through two staging buffers, as in the
    // one-CTA kernel
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const bool leader = threadIdx.x == 192;
    const bool dot = a.dot != nullptr;
    const bool need_c = a.beta != 0.0f || a.lower != 0 || dot;
    constexpr int NCH = PN / 32;
    uint32_t ch = 0, cc = 0;
    bool ok = true;
    auto load_chunk = [&](int t, int h, uint32_t b) {
      int mt, nt;
      tile_of(a, t, mt, nt);
      mbar_arrive_expect_tx(&c_full[b], C_BUF_BYTES);
      tma_load_2d(cs + b * C_BUF_BYTES, &tmC, &c_full[b], nt * PN + 32 * h, mt * PM + row0);
    };
    if (leader && need_c && pair < a.n_tiles) load_chunk(pair, 0, 0);
    for (int t = pair; t < a.n_tiles; t += n_pairs, ++ch) {
      int mt, nt;
      tile_of(a, t, mt, nt);
      const uint32_t buf = ch & 1, use = ch >> 1;
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[buf], use & 1));
      tc_fence_after();
      const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + buf * PN;
      const int m = mt * PM + row0 + r;
      const bool diag = a.lower && mt == nt;
      double rs = 0.0;
#pragma unroll 1
      for (int h = 0; h < NCH; ++h, ++cc) {
        const uint32_t b = cc & 1;
        if (need_c && ok) ok = __all_sync(0xffffffffu, mbar_wait(&c_full[b], (cc >> 1) & 1));
        if (leader && ok && need_c) {
          if (!dot) bulk_wait_group_read0();
          if (h + 1 < NCH) {
            load_chunk(t, h + 1, b ^ 1u);
          } else {
            const int tn = t + n_pairs;
            if (tn < a.n_tiles) load_chunk(tn, 0, b ^ 1u);
          }
        }
        if (ok) {
          float v[32];
          tmem_ld32(taddr + h * 32, v);
          uint8_t *row = cs + b * C_BUF_BYTES + r * 128;
          if (dot) {
            float part = 0.0f, pdiag = 0.0f;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              float4 cv = *reinterpret_cast<const float4 *>(row + ((c ^ (r & 7)) << 4));
              if (diag) {
                const int n = nt * PN + 32 * h + 4 * c;
                if (n == m) pdiag = fmaf(a.alpha * v[4 * c], cv.x, pdiag);
                if (n + 1 == m) pdiag = fmaf(a.alpha * v[4 * c + 1], cv.y, pdiag);
                if (n + 2 == m) pdiag = fmaf(a.alpha * v[4 * c + 2], cv.z, pdiag);
                if (n + 3 == m) pdiag = fmaf(a.alpha * v[4 * c + 3], cv.w, pdiag);
                if (n >= m) cv.x = 0.0f;
                if (n + 1 >= m) cv.y = 0.0f;
                if (n + 2 >= m) cv.z = 0.0f;
                if (n + 3 >= m) cv.w = 0.0f;
              }
              part = fmaf(a.alpha * v[4 * c], cv.x, part);
              part = fmaf(a.alpha * v[4 * c + 1], cv.y, part);
              part = fmaf(a.alpha * v[4 * c + 2], cv.z, part);
              part = fmaf(a.alpha * v[4 * c + 3], cv.w, part);
            }
            rs += (a.lower ? 2.0 : 1.0) * static_cast<double>(part) + static_cast<double>(pdiag);
          } else {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              float4 *p = reinterpret_cast<float4 *>(row + ((c ^ (r & 7)) << 4));
              const float4 old = need_c ? *p : make_float4(0.f, 0.f, 0.f, 0.f);
              float4 o;
              o.x = fmaf(a.beta, old.x, a.alpha * v[4 * c]);
              o.y = fmaf(a.beta, old.y, a.alpha * v[4 * c + 1]);
              o.z = fmaf(a.beta, old.z, a.alpha * v[4 * c + 2]);
              o.w = fmaf(a.beta, old.w, a.alpha * v[4 * c + 3]);
              if (diag) {
                const int n = nt * PN + 32 * h + 4 * c;
                if (n > m) o.x = old.x;
                if (n + 1 > m) o.y = old.y;
                if (n + 2 > m) o.z = old.z;
                if (n + 3 > m) o.w = old.w;
              }
              *p = o;
            }
          }
        }
        if (h == NCH - 1) {
          // both CTAs' epilogues free the accumulator on CTA 0's barrier
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(&acc_empty[buf], 0);
        }
        if (!dot) fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (leader && ok && !dot) {
          tma_store_2d(&tmC, cs + b * C_BUF_BYTES, nt * PN + 32 * h, mt * PM + row0);
          bulk_commit_group();
          if (!need_c) bulk_wait_group_read0();
        }
      }
      if (dot) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) rs += __shfl_xor_sync(0xffffffffu, rs, off);
        if (lane == 0) red[quarter] = rs;
        named_bar_sync(1, 128);
        if (leader && ok) a.dot[2 * t + static_cast<int>(rank)] = ((red[0] + red[1]) + red[2]) + red[3];
        named_bar_sync(1, 128);
      }
    }
    if (leader) bulk_wait_group0();
    if (!ok && lane == 0) set_status(a.status, kDevTimeout);
  }

  // every MMA of the pair has completed (CTA 0 waited for them) and both
  // CTAs are done with their TMEM and shared memory before either frees it
  tc_fence_before();
  __syncwarp();
  cluster_sync();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem, PAIR_TMEM_COLS);
  }
}

}  // namespace

// C (M x N, ldc) = beta C + alpha A B; see the file comment for layouts.
// All pointers 16-byte aligned, lda / ldb / ldc multiples of 4.  C may
// overlap A or B only when beta == 0 and every C tile is the B tile of its
// own columns (an in-place left multiplication); tiles of C are read (beta
// != 0 or lower) and written whole, so with `lower` the strict upper part of
// a diagonal tile is written back unchanged.
// Dot mode (dot_partials non-NULL): nothing is written to C; instead
// dot_partials[t] = sum over output tile t of (alpha A B) .* C (fp32 within
// a row of the tile, fp64 across rows), for t < gemm_tf32x3_tiles(M, N,
// lower).  With lower (M == N, A B and C symmetric) the tiles of the lower
// triangle give the sum over the whole matrix: strictly lower elements
// count twice, diagonal ones once.
namespace {
int tile_count(int M, int N, bool lower, int tm, int tn) {
  const int mt = (M + tm - 1) / tm, nt = (N + tn - 1) / tn;
  return lower ? mt * (mt + 1) / 2 : mt * nt;
}
// CTA pairs when they occupy about as many SMs as single CTAs would: then
// each SM moves half the B operand per flop.
bool use_pairs(int M, int N, bool lower) {
  if (M < PM || N < PN) return false;
  const int sms = num_sms();
  const int pairs = tile_count(M, N, lower, PM, PN);
  const int singles = tile_count(M, N, lower, TM, TN);
  const int ctas_pair = 2 * (pairs < sms / 2 ? pairs : sms / 2);
  const int ctas_single = singles < sms ? singles : sms;
  return 10 * ctas_pair >= 9 * ctas_single;
}
}  // namespace

int gemm_tf32x3_tiles(int M, int N, bool lower) {
  if (use_pairs(M, N, lower)) return 2 * tile_count(M, N, lower, PM, PN);
  return tile_count(M, N, lower, TM, TN);
}

gq_status launch_gemm_tf32x3(int M, int N, int K, float alpha, const float *A, int64_t lda,
                             const float *B, int64_t ldb, bool b_kmajor, float beta, float *C,
                             int64_t ldc, bool lower, int *status, cudaStream_t st,
                             double *dot_partials) {
  if (M <= 0 || N <= 0 || K <= 0) return GQ_OK;
  CUtensorMap tA, tB;
  gq_status s = make_tmap_2d(&tA, A, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, K, M, lda, TK, TM);
  if (s != GQ_OK) return s;
  if (b_kmajor)
    s = make_tmap_2d(&tB, B, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, K, N, ldb, TK, TN);
  else
    s = make_tmap_2d(&tB, B, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, N, K, ldb, 32, TK,
                     CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B);
  if (s != GQ_OK) return s;
  CUtensorMap tC;
  s = make_tmap_2d(&tC, C, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, N, M, ldc, 32, TM);
  if (s != GQ_OK) return s;
  const bool pairs = use_pairs(M, N, lower);
  const int tm = pairs ? PM : TM, tn = pairs ? PN : TN;
  TcArgs a{};
  a.M = M;
  a.N = N;
  a.K = K;
  a.alpha = alpha;
  a.beta = beta;
  a.C = C;
  a.ldc = ldc;
  a.n_mt = (M + tm - 1) / tm;
  a.n_nt = (N + tn - 1) / tn;
  a.nkb = (K + TK - 1) / TK;
  a.b_kmajor = b_kmajor ? 1 : 0;
  a.lower = lower ? 1 : 0;
  a.n_tiles = lower ? a.n_mt * (a.n_mt + 1) / 2 : a.n_mt * a.n_nt;
  a.status = status;
  a.dot = dot_partials;
  const int sms = num_sms();
  const int slot = timer_begin(GQ_KERNEL_GEMM_TF32X3, st);
  if (pairs) {
    cudaFuncSetAttribute(gemm_pair_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(SMEM_BYTES));
    const int n_pairs = a.n_tiles < sms / 2 ? a.n_tiles : sms / 2;
    gemm_pair_kernel<false><<<2 * n_pairs, NUM_THREADS, SMEM_BYTES, st>>>(tA, tB, tC, a);
  } else {
    cudaFuncSetAttribute(gemm_tf32x3_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(SMEM_BYTES));
    const int grid = a.n_tiles < sms ? a.n_tiles : sms;
    gemm_tf32x3_kernel<<<grid, NUM_THREADS, SMEM_BYTES, st>>>(tA, tB, tC, a);
  }
  count_launch();
  // the fp32 product: 2 M N K flops, M (M + 1) K for the lower triangle
  timer_end(slot, st,
            lower ? static_cast<double>(M) * (M + 1) * K : 2.0 * M * static_cast<double>(N) * K);
  return check_launch("gemm_tf32x3_kernel");
}

// sum over the lower triangle of (A A^T) .* C, A = A_h + A_l given as bf16
// parts [M][lda] (K = the row length, contiguous; lda a multiple of 8, the
// pad zero), C [M][ldc] fp32 symmetric: dot_partials[i] for i <
// syrk_dot_bf16x3_partials(M) (strictly lower elements counted twice, the
// diagonal once), on CTA pairs.
int syrk_dot_bf16x3_partials(int M) { return 2 * tile_count(M, M, true, PM, PN); }

gq_status launch_syrk_dot_bf16x3(int M, int K, const uint16_t *A_h, const uint16_t *A_l,
                                 int64_t lda, const float *C, int64_t ldc, double *dot_partials,
                                 int *status, cudaStream_t st) {
  if (M <= 0 || K <= 0) return GQ_OK;
  CUtensorMap tH, tL, tC;
  gq_status s = make_tmap_2d(&tH, A_h, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K, M, lda, TK_BF16, TM);
  if (s == GQ_OK)
    s = make_tmap_2d(&tL, A_l, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K, M, lda, TK_BF16, TM);
  if (s == GQ_OK)
    s = make_tmap_2d(&tC, C, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, M, M, ldc, 32, TM);
  if (s != GQ_OK) return s;
  TcArgs a{};
  a.M = M;
  a.N = M;
  a.K = K;
  a.alpha = 1.0f;
  a.beta = 0.0f;
  a.C = const_cast<float *>(C);
  a.ldc = ldc;
  a.n_mt = a.n_nt = (M + PM - 1) / PM;
  a.nkb = (K + TK_BF16 - 1) / TK_BF16;
  a.b_kmajor = 1;
  a.lower = 1;
  a.n_tiles = a.n_mt * (a.n_mt + 1) / 2;
  a.status = status;
  a.dot = dot_partials;
  const int sms = num_sms();
  cudaFuncSetAttribute(gemm_pair_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       static_cast<int>(SMEM_BYTES));
  const int n_pairs = a.n_tiles < sms / 2 ? a.n_tiles : sms / 2;
  const int slot = timer_begin(GQ_KERNEL_SYRK_BF16, st);
  gemm_pair_kernel<true><<<2 * n_pairs, NUM_THREADS, SMEM_BYTES, st>>>(tH, tL, tC, a);
  count_launch();
  timer_end(slot, st, static_cast<double>(M) * (M + 1) * K);
  return check_launch("gemm_pair_kernel<bf16>");
}

}  // namespace gq
