// Layer reconstruction error SSE = ||(W - W^) X^T||_F^2 on the tensor cores.
//
// "Model Quantization Mechanics", section 2.1 and "GPTQ: Post-Training
// INT4", "OBQ Foundation": the layer-wise objective ||W X - W^ X||^2;
// "GPT-2 Quantization Reconstruction Error" reports it per layer as an MSE.
//
// 1. dW = W - W^ in fp32 from the packed codes and the 16-bit scales, split
//    into bf16 hi + lo (dW = hi + lo to ~2^-17 relative); X is exactly bf16.
// 2. A persistent tcgen05 GEMM over 128 (rows) x 256 (tokens) output tiles:
//    TMA loads hi, lo and X boxes (K-major, 128-byte swizzle, no
//    multicast); two MMAs per K step (hi and lo) accumulate into one of two
//    TMEM accumulators; the epilogue warps square and sum their rows while
//    the next tile is already being multiplied.  The d_out x n_tok product
//    never leaves the SM.
// 3. Per-warp fp64 partials are added in a fixed order: deterministic.
#include "gq_device.cuh"
#include "gq_internal.h"

namespace gq {
namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 3;
constexpr int A_BYTES = BM * BK * 2;  // 16 KB (one box of 64 x 128)
constexpr int B_BYTES = BN * BK * 2;  // 32 KB (one box of 64 x 256)
constexpr int STAGE_BYTES = 2 * A_BYTES + B_BYTES;
constexpr int NUM_THREADS = 320;
constexpr uint32_t TMEM_COLS = 512;
constexpr size_t SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;

struct ReconArgs {
  int n_mt, n_nt, nkb;
  double *partials;  // [n_tiles][8]
  int *status;
  float *Y;          // store mode (W4A16 product): Y [M][ldy] = the GEMM itself, else NULL
  int64_t ldy;
  int M, N;
};

// Tile t -> (row tile, token tile) in groups of 16 row tiles, token tile by
// token tile inside a group: the tiles in flight at one time share a few
// slabs of W - W^ and of X (row-tile-first order cycled all of W - W^
// through the L2 for every couple of token tiles).
constexpr int RASTER_GM = 16;
__device__ __forceinline__ void recon_tile(int t, int n_mt, int n_nt, int &mt, int &nt) {
  const int per_group = RASTER_GM * n_nt;
  const int g = t / per_group;
  const int r = t - g * per_group;
  const int rows = min(RASTER_GM, n_mt - g * RASTER_GM);
  mt = g * RASTER_GM + r % rows;
  nt = r / rows;
}

// dW = W - s (c - z) (times col_inv[c] when given: the codes quantise
// W diag(s_col) and col_inv = 1 / s_col), split into bf16 hi + lo.
template <typename T>
__device__ __forceinline__ float ld_w(const T *p);
template <>
__device__ __forceinline__ float ld_w<float>(const float *p) { return *p; }
template <>
__device__ __forceinline__ float ld_w<__half>(const __half *p) { return __half2float(*p); }
template <>
__device__ __forceinline__ float ld_w<__nv_bfloat16>(const __nv_bfloat16 *p) {
  return __bfloat162float(*p);
}

template <typename T>
__global__ void __launch_bounds__(256) dequant_diff_kernel(
    const T *__restrict__ W, const uint32_t *__restrict__ q, const uint16_t *__restrict__ scales,
    const uint16_t *__restrict__ zeros, const int32_t *__restrict__ g_idx,
    const float *__restrict__ col_inv, int64_t d_out, int64_t d_in, int group_size, int sym,
    __nv_bfloat16 *__restrict__ hi, __nv_bfloat16 *__restrict__ lo, float *__restrict__ dw32,
    int bits) {
  // a unit is a run of columns that fills whole words of the row's bit
  // stream: 8 columns (one word) at 4 bits, else 32 columns (bits words)
  const int run = bits == 4 ? 8 : 32;
  const int nw = run * bits / 32;
  const int64_t units = d_in / run;
  const int64_t row_words = d_in * bits / 32;
  const int64_t n_groups = group_size <= 0 ? 1 : d_in / group_size;
  const int64_t n = d_out * units;
  const uint32_t mask = (1u << bits) - 1u;
  const int offset = sym ? (1 << (bits - 1)) : 0;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * 256) {
    const int64_t r = e / units, u = e % units;
    uint32_t wv[8];
    for (int i = 0; i < nw; ++i) wv[i] = q[r * row_words + u * nw + i];
    for (int c8 = 0; c8 < run; c8 += 8) {
      __align__(16) __nv_bfloat16 h[8], l[8];
      __align__(16) float f[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int64_t c = u * run + c8 + k;
        int64_t gi = g_idx ? g_idx[c] : (group_size <= 0 ? 0 : c / group_size);
        gi = gi < 0 ? 0 : (gi >= n_groups ? n_groups - 1 : gi);
        const float s = __half2float(__ushort_as_half(scales[r * n_groups + gi]));
        const float z = sym ? 0.0f : __half2float(__ushort_as_half(zeros[r * n_groups + gi]));
        const int stored = static_cast<int>(bits == 4 ? (wv[0] >> (4 * k)) & 0xFu
                                                      : get_code(wv, bits, c8 + k) & mask);
        const float code = static_cast<float>(stored - offset);
        float what = s * (code - z);
        if (col_inv) what *= col_inv[c];  // effective weight of a scaled layer
        const float dw = W ? ld_w(W + r * d_in + c) - what : what;  // W NULL: W^ itself
        f[k] = dw;
        const __nv_bfloat16 hb = __float2bfloat16_rn(dw);
        h[k] = hb;
        l[k] = __float2bfloat16_rn(dw - __bfloat162float(hb));
      }
      const int64_t off = r * d_in + u * run + c8;
      if (dw32) {  // fp32 dW (trace route)
        float4 *dst = reinterpret_cast<float4 *>(dw32 + off);
        dst[0] = *reinterpret_cast<const float4 *>(f);
        dst[1] = *reinterpret_cast<const float4 *>(f + 4);
      } else {
        *reinterpret_cast<uint4 *>(hi + off) = *reinterpret_cast<const uint4 *>(h);
        *reinterpret_cast<uint4 *>(lo + off) = *reinterpret_cast<const uint4 *>(l);
      }
    }
  }
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    recon_mma_kernel(const __grid_constant__ CUtensorMap tmHi,
                     const __grid_constant__ CUtensorMap tmLo,
                     const __grid_constant__ CUtensorMap tmX, ReconArgs a) {
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
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tmHi);
    tma_prefetch_desc(&tmLo);
    tma_prefetch_desc(&tmX);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_tiles = a.n_mt * a.n_nt;

  if (warp == 0) {
    if (lane == 0) {
      bool ok = true;
      uint32_t it = 0;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
        int mt, nt;
        recon_tile(t, a.n_mt, a.n_nt, mt, nt);
        for (int kb = 0; kb < a.nkb; ++kb, ++it) {
          const uint32_t s = it % STAGES, r = it / STAGES;
          if (!mbar_wait(&empty[s], (r & 1) ^ 1)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
          uint8_t *st = smem + s * STAGE_BYTES;
          tma_load_2d(st, &tmHi, &full[s], kb * BK, mt * BM);
          tma_load_2d(st + A_BYTES, &tmLo, &full[s], kb * BK, mt * BM);
          tma_load_2d(st + 2 * A_BYTES, &tmX, &full[s], kb * BK, nt * BN);
        }
      }
      const uint32_t n_wait = it < STAGES ? it : STAGES;
      for (uint32_t k = 0; k < n_wait; ++k) {
        const uint32_t j = it - 1 - k;
        if (!mbar_wait(&full[j % STAGES], (j / STAGES) & 1)) ok = false;
      }
      if (!ok) set_status(a.status, kDevTimeout);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = true;
      uint32_t it = 0, ch = 0;
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, false, false);
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++ch) {
        const uint32_t buf = ch & 1, use = ch >> 1;
        if (!mbar_wait(&acc_empty[buf], (use & 1) ^ 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem + buf * BN;
        for (int kb = 0; kb < a.nkb; ++kb, ++it) {
          const uint32_t s = it % STAGES, r = it / STAGES;
          if (!mbar_wait(&full[s], r & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sh = smem_u32(smem + s * STAGE_BYTES);
          const uint32_t sl = sh + A_BYTES;
          const uint32_t sx = sh + 2 * A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            // K-major: 16 elements = 32 bytes along the swizzled 128-byte row
            const uint64_t bd = smem_desc_sw128(sx + kk * 32, 16, 1024);
            mma_bf16(d_tmem, smem_desc_sw128(sh + kk * 32, 16, 1024), bd, idesc,
                     (kb > 0 || kk > 0) ? 1u : 0u);
            mma_bf16(d_tmem, smem_desc_sw128(sl + kk * 32, 16, 1024), bd, idesc, 1u);
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
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const int ew = warp - 2;
    uint32_t ch = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++ch) {
      const uint32_t buf = ch & 1, use = ch >> 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[buf], use & 1));
      if (!ok) break;
      tc_fence_after();
      const uint32_t taddr =
          tmem + (static_cast<uint32_t>(quarter * 32) << 16) + buf * BN + half * 128;
      if (a.Y) {  // store mode: row m of the tile, 128 of its token columns
        int mt, nt;
        recon_tile(t, a.n_mt, a.n_nt, mt, nt);
        const int m = mt * BM + quarter * 32 + lane;
        const int n0 = nt * BN + half * 128;
        float *yrow = a.Y + static_cast<int64_t>(m) * a.ldy + n0;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          float v[32];
          tmem_ld32(taddr + c * 32, v);
          if (m < a.M) {
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
              const int n = n0 + c * 32 + i;
              if (n + 3 < a.N) {
                *reinterpret_cast<float4 *>(yrow + c * 32 + i) =
                    make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
              } else {
#pragma unroll
                for (int e = 0; e < 4; ++e)
                  if (n + e < a.N) yrow[c * 32 + i + e] = v[i + e];
              }
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[buf]);
        continue;
      }
      float ssq = 0.0f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float v[32];
        tmem_ld32(taddr + c * 32, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) ssq = fmaf(v[i], v[i], ssq);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
      double dsum = static_cast<double>(ssq);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, off);
      if (lane == 0) a.partials[static_cast<size_t>(t) * 8 + ew] = dsum;
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

__global__ void __launch_bounds__(1024) recon_reduce_kernel(const double *__restrict__ partials,
                                                            int64_t n, const int *status,
                                                            double *__restrict__ sse,
                                                            double scale = 1.0) {
  __shared__ double red[1024];
  double s = 0.0;
  for (int64_t i = threadIdx.x; i < n; i += 1024) s += partials[i];
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = 512; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0)
    *sse = (status && *status) ? __longlong_as_double(0x7ff8000000000000ll) : red[0] * scale;
}

struct ReconLayout {
  int n_mt, n_nt, nkb;
  size_t off_partials, off_hi, off_lo, total;
};

ReconLayout recon_layout(int64_t d_out, int64_t d_in, int64_t n_tok) {
  ReconLayout L{};
  L.n_mt = static_cast<int>((d_out + BM - 1) / BM);
  L.n_nt = static_cast<int>((n_tok + BN - 1) / BN);
  L.nkb = static_cast<int>((d_in + BK - 1) / BK);
  L.off_partials = kWsHeader;
  size_t off = L.off_partials + round_up(static_cast<size_t>(L.n_mt) * L.n_nt * 8 * sizeof(double), 256);
  L.off_hi = off;
  off += round_up(static_cast<size_t>(d_out) * d_in * 2, 256);
  L.off_lo = off;
  off += round_up(static_cast<size_t>(d_out) * d_in * 2, 256);
  L.total = off;
  return L;
}

}  // namespace

size_t recon_ws_bytes(int64_t d_out, int64_t d_in, int64_t n_tok) {
  return recon_layout(d_out, d_in, n_tok).total;
}

gq_status launch_recon(const void *W, gq_dtype dt, const uint32_t *qpacked,
                       const uint16_t *scales, const uint16_t *zeros, const int32_t *g_idx,
                       int64_t d_out, int64_t d_in, int group_size, int sym, const void *X,
                       int64_t n_tok, double *sse_dev, void *ws, cudaStream_t st,
                       const float *col_inv, float *Y, int bits) {
  if (group_size == 0) group_size = -1;  // per-tensor scales are stored per row
  const ReconLayout L = recon_layout(d_out, d_in, n_tok);
  uint8_t *base = static_cast<uint8_t *>(ws);
  int *status = reinterpret_cast<int *>(base);
  double *partials = reinterpret_cast<double *>(base + L.off_partials);
  __nv_bfloat16 *hi = reinterpret_cast<__nv_bfloat16 *>(base + L.off_hi);
  __nv_bfloat16 *lo = reinterpret_cast<__nv_bfloat16 *>(base + L.off_lo);
  if (cudaMemsetAsync(status, 0, kWsHeader, st) != cudaSuccess) return check_launch("memset");
  const int64_t n_tiles = static_cast<int64_t>(L.n_mt) * L.n_nt;
  if (Y) {  // W4A16 product: dequantise W^ itself (no W), no reduction
    W = nullptr;
    dt = GQ_F32;
    if (n_tok == 0) return GQ_OK;
  }
  if (n_tok == 0) {
    recon_reduce_kernel<<<1, 1024, 0, st>>>(partials, 0, status, sse_dev);
    count_launch();
    return check_launch("recon_reduce_kernel");
  }
  unsigned g = static_cast<unsigned>((d_out * (d_in / (bits == 4 ? 8 : 32)) + 255) / 256);
  const unsigned cap = static_cast<unsigned>(num_sms()) * 16;
  if (g > cap) g = cap;
  switch (dt) {
    case GQ_F32:
      dequant_diff_kernel<float><<<g, 256, 0, st>>>(static_cast<const float *>(W), qpacked,
                                                    scales, zeros, g_idx, col_inv, d_out, d_in,
                                                    group_size, sym, hi, lo, nullptr, bits);
      break;
    case GQ_F16:
      dequant_diff_kernel<__half><<<g, 256, 0, st>>>(static_cast<const __half *>(W), qpacked,
                                                     scales, zeros, g_idx, col_inv, d_out,
                                                     d_in, group_size, sym, hi, lo, nullptr, bits);
      break;
    case GQ_BF16:
      dequant_diff_kernel<__nv_bfloat16><<<g, 256, 0, st>>>(
          static_cast<const __nv_bfloat16 *>(W), qpacked, scales, zeros, g_idx, col_inv, d_out,
          d_in, group_size, sym, hi, lo, nullptr, bits);
      break;
  }
  count_launch();
  CUtensorMap tHi, tLo, tX;
  gq_status s = make_tmap_2d(&tHi, hi, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d_in, d_out, d_in, BK, BM);
  if (s == GQ_OK) s = make_tmap_2d(&tLo, lo, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d_in, d_out, d_in, BK, BM);
  if (s == GQ_OK) s = make_tmap_2d(&tX, X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d_in, n_tok, d_in, BK, BN);
  if (s != GQ_OK) return s;
  cudaFuncSetAttribute(recon_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       static_cast<int>(SMEM_BYTES));
  ReconArgs a{L.n_mt, L.n_nt, L.nkb, partials, status, Y, n_tok, static_cast<int>(d_out),
              static_cast<int>(n_tok)};
  const int grid = static_cast<int>(n_tiles < num_sms() ? n_tiles : num_sms());
  const int slot = timer_begin(GQ_KERNEL_RECON_MMA, st);
  recon_mma_kernel<<<grid, NUM_THREADS, SMEM_BYTES, st>>>(tHi, tLo, tX, a);
  count_launch();
  // one product (W - W^) X^T: 2 n_tok d_out d_in flops (the hi + lo split
  // runs it twice on the tensor cores)
  timer_end(slot, st, 2.0 * static_cast<double>(n_tok) * d_out * d_in);
  s = check_launch("recon_mma_kernel");
  if (s != GQ_OK || Y) return s;
  recon_reduce_kernel<<<1, 1024, 0, st>>>(partials, n_tiles * 8, status, sse_dev);
  count_launch();
  return check_launch("recon_reduce_kernel");
}

// ---------------------------------------------------------------------------
// The same SSE by the trace route: ||dW X^T||_F^2 = tr(dW X^T X dW^T) =
// tr(dW H0 dW^T) / 2 = <H0, G>_F / 2 with G = dW^T dW and the undamped
// H0 = 2 X^T X.  dW^T is formed as a bf16 pair hi + lo (16 significant
// bits), then G's lower triangle on the tensor cores (a SYRK of three bf16
// products, ~2^-16 relative per term) whose epilogue sums G .* H0 over each
// tile instead of storing G (off-diagonal elements twice); fp64 tile
// partials added in a fixed order.  d_out d_in^2 flops instead of 2 n_tok
// d_out d_in.
namespace {

// dW^T as bf16 hi + lo, [d_in][ldt] each (ldt = d_out rounded up to 8,
// zero-padded): a block takes 32 rows x 64 columns of dW, forms them in
// shared memory and writes them transposed, 32 consecutive values per
// column.
template <typename T>
__global__ void __launch_bounds__(256) dequant_diff_t_kernel(
    const T *__restrict__ W, const uint32_t *__restrict__ q, const uint16_t *__restrict__ scales,
    const uint16_t *__restrict__ zeros, const int32_t *__restrict__ g_idx, int64_t d_out,
    int64_t d_in, int group_size, int sym, int bits, __nv_bfloat16 *__restrict__ dth,
    __nv_bfloat16 *__restrict__ dtl, int64_t ldt) {
  __shared__ float tile[64][33];
  const int64_t n_groups = group_size <= 0 ? 1 : d_in / group_size;
  const int64_t row_words = d_in * bits / 32;
  const int offset = sym ? (1 << (bits - 1)) : 0;
  const int64_t tiles_r = (d_out + 31) / 32, tiles_c = (d_in + 63) / 64;
  for (int64_t t = blockIdx.x; t < tiles_r * tiles_c; t += gridDim.x) {
    const int64_t r0 = (t % tiles_r) * 32, c0 = (t / tiles_r) * 64;
    // read: thread -> (row r0 + i, 8 columns)
    {
      const int i = threadIdx.x >> 3, j0 = (threadIdx.x & 7) * 8;
      const int64_t r = r0 + i;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int64_t c = c0 + j0 + k;
        float dw = 0.0f;
        if (r < d_out && c < d_in) {
          int64_t gi = g_idx ? g_idx[c] : (group_size <= 0 ? 0 : c / group_size);
          gi = gi < 0 ? 0 : (gi >= n_groups ? n_groups - 1 : gi);
          const float sc = __half2float(__ushort_as_half(scales[r * n_groups + gi]));
          const float z = sym ? 0.0f : __half2float(__ushort_as_half(zeros[r * n_groups + gi]));
          const uint32_t stored = get_code(q + r * row_words, bits, static_cast<int>(c));
          const float what = sc * (static_cast<float>(static_cast<int>(stored) - offset) - z);
          dw = ld_w(W + r * d_in + c) - what;
        }
        tile[j0 + k][i] = dw;
      }
    }
    __syncthreads();
    // write: warp -> 8 columns, lane -> row
    {
      const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int cc = wp * 8 + k;
        const int64_t c = c0 + cc, r = r0 + lane;
        if (c < d_in && r < ldt) {
          const float v = r < d_out ? tile[cc][lane] : 0.0f;
          const __nv_bfloat16 h = __float2bfloat16_rn(v);
          dth[c * ldt + r] = h;
          dtl[c * ldt + r] = __float2bfloat16_rn(v - __bfloat162float(h));
        }
      }
    }
    __syncthreads();
  }
}

struct TraceLayout {
  int64_t ldt;
  size_t off_partials, off_dth, off_dtl, total;
};
TraceLayout trace_layout(int64_t d_out, int64_t d_in) {
  TraceLayout L{};
  L.ldt = (d_out + 7) / 8 * 8;
  L.off_partials = kWsHeader;
  const int parts = syrk_dot_bf16x3_partials(static_cast<int>(d_in));
  const size_t part = round_up(static_cast<size_t>(d_in) * L.ldt * 2, 256);
  L.off_dth = L.off_partials + round_up(static_cast<size_t>(parts) * sizeof(double), 256);
  L.off_dtl = L.off_dth + part;
  L.total = L.off_dtl + part;
  return L;
}
}  // namespace

size_t recon_hessian_ws_bytes(int64_t d_out, int64_t d_in) {
  return trace_layout(d_out, d_in).total;
}

gq_status launch_recon_hessian(const void *W, gq_dtype dt, const uint32_t *qpacked,
                               const uint16_t *scales, const uint16_t *zeros,
                               const int32_t *g_idx, int64_t d_out, int64_t d_in, int group_size,
                               int sym, const float *H0, double *sse_dev, void *ws,
                               cudaStream_t st, int bits) {
  if (group_size == 0) group_size = -1;  // per-tensor scales are stored per row
  const TraceLayout L = trace_layout(d_out, d_in);
  uint8_t *base = static_cast<uint8_t *>(ws);
  int *status = reinterpret_cast<int *>(base);
  double *partials = reinterpret_cast<double *>(base + L.off_partials);
  auto *dth = reinterpret_cast<__nv_bfloat16 *>(base + L.off_dth);
  auto *dtl = reinterpret_cast<__nv_bfloat16 *>(base + L.off_dtl);
  if (cudaMemsetAsync(status, 0, kWsHeader, st) != cudaSuccess) return check_launch("memset");
  int64_t g = ((L.ldt + 31) / 32) * ((d_in + 63) / 64);
  const int64_t cap = static_cast<int64_t>(num_sms()) * 16;
  if (g > cap) g = cap;
  const unsigned grid = static_cast<unsigned>(g);
  switch (dt) {
    case GQ_F32:
      dequant_diff_t_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float *>(W), qpacked,
                                                         scales, zeros, g_idx, d_out, d_in,
                                                         group_size, sym, bits, dth, dtl, L.ldt);
      break;
    case GQ_F16:
      dequant_diff_t_kernel<__half><<<grid, 256, 0, st>>>(static_cast<const __half *>(W), qpacked,
                                                          scales, zeros, g_idx, d_out, d_in,
                                                          group_size, sym, bits, dth, dtl, L.ldt);
      break;
    case GQ_BF16:
      dequant_diff_t_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
          static_cast<const __nv_bfloat16 *>(W), qpacked, scales, zeros, g_idx, d_out, d_in,
          group_size, sym, bits, dth, dtl, L.ldt);
      break;
  }
  count_launch();
  gq_status s = check_launch("dequant_diff_t_kernel");
  if (s != GQ_OK) return s;
  // G = dW^T dW (lower triangle, K = d_out; rows of dW^T are K-major),
  // each tile summed against H0's
  s = launch_syrk_dot_bf16x3(static_cast<int>(d_in), static_cast<int>(d_out),
                             reinterpret_cast<const uint16_t *>(dth),
                             reinterpret_cast<const uint16_t *>(dtl), L.ldt, H0, d_in, partials,
                             status, st);
  if (s != GQ_OK) return s;
  const int parts = syrk_dot_bf16x3_partials(static_cast<int>(d_in));
  recon_reduce_kernel<<<1, 1024, 0, st>>>(partials, parts, status, sse_dev, 0.5);
  count_launch();
  return check_launch("recon_reduce_kernel");
}

}  // namespace gq
