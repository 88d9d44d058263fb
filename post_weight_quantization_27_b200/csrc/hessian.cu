// H += 2 X^T X on the 5th-generation tensor cores.
//
// "GPTQ: Post-Training INT4" -- "Hessian-Based Weight Update": the layer
// Hessian is H = 2 X X^T (X as d_in x tokens), the same for every output
// row; with X stored tokens x d_in it is 2 X^T X.
//
// Design (sm_100a, one CTA per SM, persistent):
//   * H is symmetric, so only 128 x 256 output tiles that touch the upper
//     triangle are computed (about half the dense work).
//   * warp 0 issues TMA loads of X boxes (64 columns x 64 tokens, 128-byte
//     swizzle, no multicast) into a 4-stage shared-memory ring; A = X^T and
//     B = X^T are both "MN-major" operands of tcgen05.mma (columns of X
//     are contiguous), so no transpose is ever materialised.
//   * warp 1 (one elected thread) issues tcgen05.mma kind::f16 bf16 x bf16
//     -> fp32 into one of two 256-column TMEM accumulators.  Every 512
//     tokens the accumulator is handed to the epilogue and the other one
//     is used, so the tensor pipe never waits for the drain.
//   * warps 2..9 add each 512-token partial into fp32 registers (one TMEM
//     lane = one tile row per thread).  Short accumulation chains inside
//     the tensor core keep the fp32 error small at 262144 tokens.
//   * the producers of a wave of tiles stay within a few token steps of
//     each other (see ALIGN_G), so the L2 keeps serving the X slabs they
//     share.
//   * tiles are split over token ranges when there are too few tiles for
//     the SMs, or when a split makes the last wave of tiles less ragged;
//     each (split, tile) writes its raw partial tile to the workspace and
//     a second kernel adds the splits in a fixed order, scales by 2, adds
//     the incoming H and mirrors the upper triangle: the result is
//     deterministic and exactly symmetric.
//   * tiles are taken in groups of 8 row blocks, column block by column
//     block inside a group, so that the tiles in flight at one time share
//     few X column slabs (the L2 then serves most of the operand traffic;
//     row-major order would stream a new 256-column slab per tile).
#include "gq_device.cuh"
#include "gq_internal.h"

namespace gq {
namespace {

#ifndef GQ_HESS_CHUNK_KB
#define GQ_HESS_CHUNK_KB 8
#endif
// K-blocks (of 64 tokens) accumulated inside TMEM before the partial is
// drained into fp32 registers.  The tensor core's fp32 accumulation error
// grows with the length of this chain (measured against 128-token chains:
// 7.9e-7 relative at 512 tokens, 1.8e-6 at 1024), the drain's cost shrinks
// with it: 8 (512 tokens) ran the 8192-wide layer 25% faster than 2.
constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4, CHUNK_KB = GQ_HESS_CHUNK_KB;
constexpr int A_BYTES = BM * BK * 2;  // two 64x64 boxes
constexpr int B_BYTES = BN * BK * 2;  // four 64x64 boxes
constexpr int BOX_BYTES = 64 * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int NUM_THREADS = 320;
constexpr uint32_t TMEM_COLS = 512;
constexpr size_t SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;

struct HessArgs {
  int n_bi, n_bj, n_tiles, n_split, kb_per_split, nkb_total;
  float *P;
  int *status;
  int *align;        // token-alignment counters [waves][align_groups], zeroed; or NULL
  int align_groups;
};

// Token alignment of the tiles in flight.  All tiles of a wave of the
// persistent grid read the same token rows of X at about the same time, so
// the L2 serves the X slabs they share -- as long as the CTAs stay close in
// the token dimension.  Over many waves they drift apart (a CTA that misses
// in L2 slows down and misses more), and at d = 28672 the tiles re-read X
// from DRAM ~120 times.  So the producers of a wave count the groups of
// ALIGN_G k-blocks they have issued, and a producer does not run more than
// ALIGN_LEAD groups ahead of the slowest CTA of its wave.  The wait is
// short and soft: after ALIGN_WAIT_NS without progress (a CTA of the wave
// is not resident, e.g. while another kernel holds SMs) the producer stops
// waiting for the rest of the launch; it still counts its groups, so the
// others are never held up by it.  Only the timing depends on this.
#ifndef GQ_HESS_ALIGN
#define GQ_HESS_ALIGN 1
#endif
constexpr int ALIGN_G = 8, ALIGN_LEAD = 4;
constexpr uint64_t ALIGN_WAIT_NS = 20000;

__device__ __forceinline__ int ld_acquire_gpu(const int *p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ bool wait_count(const int *p, int target) {
  if (ld_acquire_gpu(p) >= target) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    __nanosleep(100);
    if (ld_acquire_gpu(p) >= target) return true;
    if (globaltimer_ns() - t0 > ALIGN_WAIT_NS) return false;
  }
}

// Tiles of row-block b are the column blocks b/2 .. n_bj-1 (a 128-row block
// starting at 128b meets the diagonal in column block floor(128b/256)).
__host__ __device__ __forceinline__ int64_t tile_row_start(int64_t b, int64_t n_bj) {
  const int64_t k = b >> 1;
  return b * n_bj - (k * (k - 1) + (b & 1) * k);
}
constexpr int RASTER_G = 8;  // row blocks per raster group

// Processing position r -> tile (bi, bj): groups of RASTER_G row blocks;
// inside a group, column block j holds the group's row blocks b with
// b <= 2j + 1 (the tiles of j that touch the upper triangle).
__device__ __forceinline__ void raster_tile(int r, int n_bi, int n_bj, int &bi, int &bj) {
  for (int b0 = 0; b0 < n_bi; b0 += RASTER_G) {
    const int b1 = min(b0 + RASTER_G, n_bi);
    const int jlo = b0 >> 1;
    // column blocks jlo .. jm-1 hold 2j + 2 - b0 row blocks, jm .. n_bj-1 all b1 - b0
    const int jm = max(jlo, min(n_bj, (b1 - 1) >> 1));
    const int count = (jm - jlo) * (2 - b0) + (jm - jlo) * (jm + jlo - 1) + (n_bj - jm) * (b1 - b0);
    if (r >= count) {
      r -= count;
      continue;
    }
    for (int j = jlo; j < n_bj; ++j) {
      const int c = min(b1, 2 * j + 2) - b0;
      if (r < c) {
        bi = b0 + r;
        bj = j;
        return;
      }
      r -= c;
    }
  }
  bi = 0;
  bj = 0;
}

// Index of tile (bi, bj) in row-major order over the upper tiles (the
// layout of the partial tiles in the workspace).
__device__ __forceinline__ int natural_tile(int bi, int bj, int n_bj) {
  return static_cast<int>(tile_row_start(bi, n_bj)) + (bj - (bi >> 1));
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    hessian_mma_kernel(const __grid_constant__ CUtensorMap tmX, HessArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE_BYTES);
  uint64_t *full = bars;
  uint64_t *empty = bars + STAGES;
  uint64_t *acc_full = bars + 2 * STAGES;
  uint64_t *acc_empty = acc_full + 2;
  uint64_t *drain = acc_empty + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 8);
    }
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) tma_prefetch_desc(&tmX);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_items = a.n_tiles * a.n_split;

  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0) {
      bool ok = true;
      bool align = a.align != nullptr;  // (only with one token range per tile)
      uint32_t it = 0;
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
        const int split = item / a.n_tiles, t = item % a.n_tiles;
        int bi, bj;
        raster_tile(t, a.n_bi, a.n_bj, bi, bj);
        const int kb0 = split * a.kb_per_split;
        const int kb1 = min(kb0 + a.kb_per_split, a.nkb_total);
        const int wave = (item - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x);
        const int in_wave = min(static_cast<int>(gridDim.x), n_items - wave * static_cast<int>(gridDim.x));
        int *cnt = a.align ? a.align + static_cast<size_t>(wave) * a.align_groups : nullptr;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int g = (kb - kb0) / ALIGN_G;
          if (align && (kb - kb0) % ALIGN_G == 0 && g >= ALIGN_LEAD)
            align = wait_count(cnt + g - ALIGN_LEAD, in_wave);
          const uint32_t s = it % STAGES, r = it / STAGES;
          if (!mbar_wait(&empty[s], (r & 1) ^ 1)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
          uint8_t *sa = smem + s * STAGE_BYTES;
          uint8_t *sb = sa + A_BYTES;
          const int tok = kb * BK;
          tma_load_2d(sa, &tmX, &full[s], bi * BM, tok);
          tma_load_2d(sa + BOX_BYTES, &tmX, &full[s], bi * BM + 64, tok);
#pragma unroll
          for (int q = 0; q < 4; ++q) tma_load_2d(sb + q * BOX_BYTES, &tmX, &full[s], bj * BN + 64 * q, tok);
          if (cnt && ((kb - kb0) % ALIGN_G == ALIGN_G - 1 || kb == kb1 - 1)) atomicAdd(cnt + g, 1);
        }
      }
      // every load issued must have landed before the CTA may exit
      const uint32_t n_wait = it < STAGES ? it : STAGES;
      for (uint32_t k = 0; k < n_wait; ++k) {
        const uint32_t j = it - 1 - k;
        if (!mbar_wait(&full[j % STAGES], (j / STAGES) & 1)) ok = false;
      }
      if (!ok) set_status(a.status, kDevTimeout);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      bool ok = true;
      uint32_t it = 0, ch = 0;
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, true, true);
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
        const int split = item / a.n_tiles;
        const int kb0 = split * a.kb_per_split;
        const int kb1 = min(kb0 + a.kb_per_split, a.nkb_total);
        for (int c0 = kb0; c0 < kb1 && ok; c0 += CHUNK_KB, ++ch) {
          const int c1 = min(c0 + CHUNK_KB, kb1);
          const uint32_t buf = ch & 1, use = ch >> 1;
          if (!mbar_wait(&acc_empty[buf], (use & 1) ^ 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d_tmem = tmem + buf * BN;
          for (int kb = c0; kb < c1; ++kb, ++it) {
            const uint32_t s = it % STAGES, r = it / STAGES;
            if (!mbar_wait(&full[s], r & 1)) { ok = false; break; }
            tc_fence_after();
            const uint32_t sa = smem_u32(smem + s * STAGE_BYTES);
            const uint32_t sb = sa + A_BYTES;
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              // 16 tokens = two 8-row swizzle atoms of 1024 bytes
              const uint64_t ad = smem_desc_sw128(sa + kk * 2048, BOX_BYTES, 1024);
              const uint64_t bd = smem_desc_sw128(sb + kk * 2048, BOX_BYTES, 1024);
              mma_bf16(d_tmem, ad, bd, idesc, (kb > c0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(&empty[s]);
          }
          if (!ok) break;
          mma_commit(&acc_full[buf]);
        }
      }
      mma_commit(drain);
      if (!mbar_wait(drain, 0)) ok = false;
      if (!ok) set_status(a.status, kDevTimeout);
    }
  } else {
    // ---------------- epilogue: warps 2..9
    const int quarter = warp & 3;        // TMEM lanes this warp may access
    const int half = (warp - 2) >> 2;    // which 128 of the 256 columns
    const int row = quarter * 32 + lane;
    uint32_t ch = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
      const int split = item / a.n_tiles;
      const int kb0 = split * a.kb_per_split;
      const int kb1 = min(kb0 + a.kb_per_split, a.nkb_total);
      float m[128];
#pragma unroll
      for (int i = 0; i < 128; ++i) m[i] = 0.0f;
      for (int c0 = kb0; c0 < kb1; c0 += CHUNK_KB, ++ch) {
        const uint32_t buf = ch & 1, use = ch >> 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[buf], use & 1));
        if (!ok) break;
        tc_fence_after();
        const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + buf * BN + half * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float v[32];
          tmem_ld32(taddr + c * 32, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) m[c * 32 + i] += v[i];
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[buf]);
      }
      if (!ok) break;
      int bi, bj;
      raster_tile(item % a.n_tiles, a.n_bi, a.n_bj, bi, bj);
      const size_t slot = static_cast<size_t>(split) * a.n_tiles + natural_tile(bi, bj, a.n_bj);
      float *dst = a.P + (slot * BM + row) * BN + half * 128;
#pragma unroll
      for (int c = 0; c < 128; c += 4)
        *reinterpret_cast<float4 *>(dst + c) = make_float4(m[c], m[c + 1], m[c + 2], m[c + 3]);
    }
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

// H[i][j] (i <= j) := H[i][j] + 2 * sum_s P_s(i, j) (without the H term
// when !accumulate); H[j][i] := H[i][j].
// Tiles of 64 x 64 on or above the diagonal, enumerated column by column
// (t -> (bi, bj), bi <= bj) so that no block is spent on the lower half;
// each thread moves 4 consecutive columns of a row (float4; d is a
// multiple of 8 and a tile's 64 columns never straddle two 256-column
// partial tiles).
__global__ void __launch_bounds__(256) hessian_finish_kernel(float *__restrict__ H, int d,
                                                             const float *__restrict__ P,
                                                             int n_tiles, int n_bj, int n_split,
                                                             const int *status, int accumulate) {
  constexpr int FT = 64;
  __shared__ float tile[FT][FT + 1];
  const bool bad = status != nullptr && *status != 0;
  const int cx = (threadIdx.x & 15) * 4, ry = threadIdx.x >> 4;  // 4 columns, 16 rows per pass
  const int nb = (d + FT - 1) / FT;
  const int64_t n_up = static_cast<int64_t>(nb) * (nb + 1) / 2;
  for (int64_t t = blockIdx.x; t < n_up; t += gridDim.x) {
    int bj = static_cast<int>((sqrt(8.0 * static_cast<double>(t) + 1.0) - 1.0) * 0.5);
    while (static_cast<int64_t>(bj) * (bj + 1) / 2 > t) --bj;
    while (static_cast<int64_t>(bj + 1) * (bj + 2) / 2 <= t) ++bj;
    const int bi = static_cast<int>(t - static_cast<int64_t>(bj) * (bj + 1) / 2);
    const int j = bj * FT + cx;
    for (int r = ry; r < FT; r += 16) {
      const int i = bi * FT + r;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (i < d && j < d && i <= j + 3) {
        const int tb = i / BM, tj = j / BN;
        const int tt = static_cast<int>(tile_row_start(tb, n_bj)) + (tj - (tb >> 1));
        float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s = 0; s < n_split; ++s) {
          const float4 p = *reinterpret_cast<const float4 *>(
              P + (static_cast<size_t>(s * n_tiles + tt) * BM + (i - tb * BM)) * BN + (j - tj * BN));
          sum.x += p.x; sum.y += p.y; sum.z += p.z; sum.w += p.w;
        }
        float *h = H + static_cast<size_t>(i) * d + j;
        const float4 old = accumulate ? *reinterpret_cast<const float4 *>(h)
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
        v = make_float4(old.x + 2.0f * sum.x, old.y + 2.0f * sum.y, old.z + 2.0f * sum.z,
                        old.w + 2.0f * sum.w);
        if (!accumulate) v = make_float4(2.0f * sum.x, 2.0f * sum.y, 2.0f * sum.z, 2.0f * sum.w);
        if (bad) v = make_float4(__int_as_float(0x7fc00000), __int_as_float(0x7fc00000),
                                 __int_as_float(0x7fc00000), __int_as_float(0x7fc00000));
        // only the elements with i <= j belong to this triangle
        if (i <= j) {
          *reinterpret_cast<float4 *>(h) = v;
        } else {
          if (i <= j + 1) h[1] = v.y;
          if (i <= j + 2) h[2] = v.z;
          h[3] = v.w;
        }
      }
      tile[r][cx] = v.x;
      tile[r][cx + 1] = v.y;
      tile[r][cx + 2] = v.z;
      tile[r][cx + 3] = v.w;
    }
    __syncthreads();
    // the mirror: H[j'][i'] = H[i'][j'] for i' < j', rows j' of the tile's columns
    for (int r = ry; r < FT; r += 16) {
      const int jr = bj * FT + r, ic = bi * FT + cx;
      if (jr >= d || ic >= d) continue;
      float *h = H + static_cast<size_t>(jr) * d + ic;
      if (ic + 3 < jr) {
        *reinterpret_cast<float4 *>(h) =
            make_float4(tile[cx][r], tile[cx + 1][r], tile[cx + 2][r], tile[cx + 3][r]);
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (ic + q < jr) h[q] = tile[cx + q][r];
      }
    }
    __syncthreads();
  }
}

}  // namespace

HessPlan hessian_plan(int64_t n_tok, int64_t d_in) {
  HessPlan p{};
  p.n_bi = static_cast<int>((d_in + BM - 1) / BM);
  p.n_bj = static_cast<int>((d_in + BN - 1) / BN);
  p.n_tiles = static_cast<int>(tile_row_start(p.n_bi, p.n_bj));
  p.nkb_total = static_cast<int>((n_tok + BK - 1) / BK);
  int split = 1;
  const int sms = num_sms();
  const int target = 2 * sms;
  if (p.nkb_total > 0 && p.n_tiles < target) {
    const int want = (target + p.n_tiles - 1) / p.n_tiles;
    const int most = p.nkb_total / 4 > 1 ? p.nkb_total / 4 : 1;
    split = want < most ? want : most;
  } else if (p.nkb_total > 0) {
    // enough tiles: split (2..4 ways, each split >= 256 k-blocks) only when
    // that fills the last wave of the persistent grid noticeably better
    auto fill = [&](int sp) {
      const int64_t items = static_cast<int64_t>(p.n_tiles) * sp;
      const int64_t waves = (items + sms - 1) / sms;
      return static_cast<double>(items) / static_cast<double>(waves * sms);
    };
    double best = fill(1);
    for (int sp = 2; sp <= 4; ++sp)
      if (p.nkb_total / sp >= 256 && fill(sp) > best + 0.02) {
        best = fill(sp);
        split = sp;
      }
  }
  if (p.nkb_total == 0) {
    p.n_split = 0;
    p.kb_per_split = 0;
  } else {
    p.kb_per_split = (p.nkb_total + split - 1) / split;
    p.n_split = (p.nkb_total + p.kb_per_split - 1) / p.kb_per_split;
  }
  p.off_align = kWsHeader + static_cast<size_t>(p.n_split) * p.n_tiles * BM * BN * sizeof(float);
  if (GQ_HESS_ALIGN && p.n_split == 1 && p.n_tiles > sms) {
    const int grid = p.n_tiles < sms ? p.n_tiles : sms;
    p.align_waves = (p.n_tiles + grid - 1) / grid;
    p.align_groups = (p.nkb_total + ALIGN_G - 1) / ALIGN_G;
  }
  p.ws_bytes = p.off_align + round_up(static_cast<size_t>(p.align_waves) * p.align_groups *
                                          sizeof(int), 256);
  return p;
}

gq_status launch_hessian(const void *X, int64_t n_tok, int64_t d_in, float *H, void *ws,
                         const HessPlan &p, cudaStream_t st, bool accumulate) {
  int *status = static_cast<int *>(ws);
  float *P = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + kWsHeader);
  if (cudaMemsetAsync(status, 0, kWsHeader, st) != cudaSuccess) return check_launch("memset");
  const int n_items = p.n_tiles * p.n_split;
  if (n_items > 0) {
    CUtensorMap tm;
    gq_status s = make_tmap_2d(&tm, X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d_in, n_tok, d_in,
                               64, BK);
    if (s != GQ_OK) return s;
    int *align = nullptr;
    if (p.align_groups > 0) {
      align = reinterpret_cast<int *>(static_cast<uint8_t *>(ws) + p.off_align);
      if (cudaMemsetAsync(align, 0,
                          static_cast<size_t>(p.align_waves) * p.align_groups * sizeof(int),
                          st) != cudaSuccess)
        return check_launch("memset");
    }
    HessArgs a{p.n_bi, p.n_bj, p.n_tiles, p.n_split, p.kb_per_split, p.nkb_total, P, status,
               align, p.align_groups};
    const int sms = num_sms();
    const int slot = timer_begin(GQ_KERNEL_HESSIAN_MMA, st);
    cudaFuncSetAttribute(hessian_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(SMEM_BYTES));
    const int grid = n_items < sms ? n_items : sms;
    hessian_mma_kernel<<<grid, NUM_THREADS, SMEM_BYTES, st>>>(tm, a);
    count_launch();
    // symmetric half of X^T X: n_tok d_in (d_in + 1) flops
    timer_end(slot, st, static_cast<double>(n_tok) * d_in * (d_in + 1));
    s = check_launch("hessian_mma_kernel");
    if (s != GQ_OK) return s;
  }
  const int64_t nb = (d_in + 63) / 64, n_up = nb * (nb + 1) / 2;
  const int64_t fcap = static_cast<int64_t>(num_sms()) * 16;
  hessian_finish_kernel<<<static_cast<unsigned>(n_up < fcap ? n_up : fcap), 256, 0, st>>>(
      H, static_cast<int>(d_in), P, p.n_tiles, p.n_bj, p.n_split, status, accumulate ? 1 : 0);
  count_launch();
  return check_launch("hessian_finish_kernel");
}

}  // namespace gq
