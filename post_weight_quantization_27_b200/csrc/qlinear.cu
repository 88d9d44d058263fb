// Product of a quantised layer with bf16 activations, dequantising inside
// the GEMM: Y = W^ X^T with W^ = s (c - z) per group, read straight from the
// packed codes and the 16-bit scales ("GPTQ: Post-Training INT4" -- "Group
// Quantization" and "Running GPTQ with AutoGPTQ": the packed 4-bit codes
// with 16-bit scales and zeros are what a quantised model is served from).
//
// Persistent tcgen05 kernel over 128 (output features) x 256 (tokens) tiles,
// K in steps of 64:
//   warp 0      TMA loads of the X box (K-major, 128-byte swizzle, no
//               multicast)
//   warps 2-5   producers: each thread owns one row (output feature) of the
//               tile; per K step it reads that row's 64 codes (2 * bits
//               words) and their scale (and zero), forms W^ in fp32 and
//               writes it as a bf16 hi + lo pair (hi + lo = W^ exactly: an
//               fp16 scale times a small integer has at most 16 significant
//               bits) into the two A tiles, in the 128-byte-swizzled K-major
//               layout the tensor core reads; then makes the writes visible
//               to the async proxy and arrives on the stage's barrier.  In
//               dense mode (no codes) the row's weights are read and split
//               the same way (the layer before quantisation).
//   warp 1      two MMAs per 16-wide K slice (hi and lo against X) into one
//               of two 256-column TMEM accumulators
//   warps 6-13  epilogue: either Y fp32 feature-major [d_out][ldy], or Z
//               bf16 token-major [n_tok][d_out] = act(Y^T) (+ a residual),
//               the input of the next layer.
// The packed codes (bits / 8 bytes per weight) are read once per token
// tile instead of a dequantised copy of W (4 bytes per weight) being
// written and read back.
#include "gq_device.cuh"
#include "gq_internal.h"

namespace gq {
namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 3;
constexpr int A_BYTES = BM * BK * 2;              // 16 KB: one bf16 A tile (hi or lo)
constexpr int X_BYTES = BN * BK * 2;              // 32 KB
constexpr int STAGE_BYTES = 2 * A_BYTES + X_BYTES;
constexpr int NUM_THREADS = 448;
constexpr uint32_t TMEM_COLS = 512;
constexpr size_t SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;

struct QlArgs {
  const uint32_t *q;          // packed codes [d_out][bits d_in / 32], or NULL (dense)
  const uint16_t *scales, *zeros;
  const int32_t *g_idx;
  const void *Wd;             // dense weights [d_out][d_in] (dense mode)
  int w_dtype;
  int64_t d_out, d_in, n_tok;
  int group_size, sym, n_groups;
  int n_mt, n_nt, nkb;
  float *Y;                   // feature-major fp32 output or NULL
  int64_t ldy;
  __nv_bfloat16 *Z;           // token-major bf16 output or NULL
  const __nv_bfloat16 *R;     // residual [n_tok][d_out] added to Z, or NULL
  int act;                    // GQ_ACT_*
  int *status;
};

// Tile t -> (feature tile, token tile) in groups of 16 feature tiles.
__device__ __forceinline__ void ql_tile(int t, int n_mt, int n_nt, int &mt, int &nt) {
  constexpr int G = 16;
  const int per_group = G * n_nt;
  const int g = t / per_group;
  const int r = t - g * per_group;
  const int rows = min(G, n_mt - g * G);
  mt = g * G + r % rows;
  nt = r / rows;
}

__device__ __forceinline__ float activate(float v, int act) {
  if (act == 1) return fmaxf(v, 0.0f);
  if (act == 2) {  // GELU, tanh form: 0.5 v (1 + tanh u) = v / (1 + e^(-2u)), which keeps
                   // its relative accuracy for large negative v (no 1 + tanh cancellation)
    const float u = 0.7978845608028654f * fmaf(0.044715f * v, v * v, v);
    return v / (1.0f + expf(-2.0f * u));
  }
  return v;
}

template <typename T>
__device__ __forceinline__ float ld_dense(const T *p);
template <>
__device__ __forceinline__ float ld_dense<float>(const float *p) { return *p; }
template <>
__device__ __forceinline__ float ld_dense<__half>(const __half *p) { return __half2float(*p); }
template <>
__device__ __forceinline__ float ld_dense<__nv_bfloat16>(const __nv_bfloat16 *p) {
  return __bfloat162float(*p);
}

// Dense mode: the 64 weights of row m, columns k0 .. k0 + 63, in fp32
// (zero past d_in).
template <typename T>
__device__ __forceinline__ void dense_weights(const QlArgs &a, int64_t m, int64_t k0,
                                              float (&w)[64]) {
  const T *src = static_cast<const T *>(a.Wd) + m * a.d_in;
#pragma unroll
  for (int k = 0; k < 64; ++k) w[k] = k0 + k < a.d_in ? ld_dense<T>(src + k0 + k) : 0.0f;
}

// The packed codes of row m for columns k0 .. k0 + 63 (2 BITS words) and,
// when one group covers the whole K step, its scale and zero: loaded one
// K step ahead of their use, so the loads' latency hides behind the
// previous step's work.
template <int BITS>
struct CodeSlot {
  uint32_t wd[2 * BITS];
  float s, z;
};

template <int BITS>
__device__ __forceinline__ void load_slot(const QlArgs &a, int64_t m, int64_t k0, bool uniform,
                                          CodeSlot<BITS> &c) {
  constexpr int NW = 2 * BITS;
  c.s = 0.0f;
  c.z = 0.0f;
  if (m >= a.d_out) {
#pragma unroll
    for (int i = 0; i < NW; ++i) c.wd[i] = 0u;
    return;
  }
  const int64_t row_words = a.d_in * BITS / 32;
  const uint32_t *src = a.q + m * row_words + (k0 * BITS) / 32;
  const int64_t left = row_words - (k0 * BITS) / 32;
#pragma unroll
  for (int i = 0; i < NW; ++i) c.wd[i] = i < left ? __ldg(src + i) : 0u;
  if (uniform) {
    const int64_t gi = a.group_size <= 0 ? 0 : k0 / a.group_size;
    c.s = __half2float(__ushort_as_half(a.scales[m * a.n_groups + gi]));
    c.z = a.sym ? 0.0f : __half2float(__ushort_as_half(a.zeros[m * a.n_groups + gi]));
  }
}

// W^ of the 8 columns k0 + 8 cb .. k0 + 8 cb + 7 of row m from its codes.
template <int BITS>
__device__ __forceinline__ void slot_chunk(const QlArgs &a, int64_t m, int64_t k0, bool uniform,
                                           const CodeSlot<BITS> &c, int cb, float (&w)[8]) {
  const int offset = a.sym ? (1 << (BITS - 1)) : 0;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int k = 8 * cb + e;
    const int bit = BITS * k, wi = bit >> 5, off = bit & 31;
    uint32_t v = c.wd[wi] >> off;
    if (off + BITS > 32) v |= c.wd[wi + 1] << (32 - off);
    v &= (1u << BITS) - 1u;
    float sk = c.s, zk = c.z;
    if (!uniform && m < a.d_out) {
      const int64_t col = k0 + k < a.d_in ? k0 + k : a.d_in - 1;
      int64_t gi = a.g_idx ? a.g_idx[col] : (a.group_size <= 0 ? 0 : col / a.group_size);
      gi = gi < 0 ? 0 : (gi >= a.n_groups ? a.n_groups - 1 : gi);
      sk = __half2float(__ushort_as_half(a.scales[m * a.n_groups + gi]));
      zk = a.sym ? 0.0f : __half2float(__ushort_as_half(a.zeros[m * a.n_groups + gi]));
    }
    const float code = static_cast<float>(static_cast<int>(v) - offset);
    w[e] = (k0 + k < a.d_in && m < a.d_out) ? sk * (code - zk) : 0.0f;
  }
}

// 8 fp32 weights as bf16 hi + lo into chunk cb of row r of the stage's A
// tiles (128-byte swizzle: 16-byte chunk cb of row r sits at cb ^ (r % 8)).
__device__ __forceinline__ void store_chunk(uint8_t *hi_row, uint8_t *lo_row, int r, int cb,
                                            const float (&w)[8]) {
  __align__(16) __nv_bfloat16 h[8], l[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const __nv_bfloat16 hb = __float2bfloat16_rn(w[e]);
    h[e] = hb;
    l[e] = __float2bfloat16_rn(w[e] - __bfloat162float(hb));
  }
  const int pc = (cb ^ (r & 7)) << 4;
  *reinterpret_cast<uint4 *>(hi_row + pc) = *reinterpret_cast<const uint4 *>(h);
  *reinterpret_cast<uint4 *>(lo_row + pc) = *reinterpret_cast<const uint4 *>(l);
}

template <int BITS, typename T>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    qlinear_kernel(const __grid_constant__ CUtensorMap tmX, QlArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE_BYTES);
  uint64_t *x_full = bars;                 // TMA of X landed
  uint64_t *a_full = bars + STAGES;        // the four producer warps wrote A
  uint64_t *empty = bars + 2 * STAGES;     // MMAs done with the stage
  uint64_t *acc_full = bars + 3 * STAGES;
  uint64_t *acc_empty = acc_full + 2;
  uint64_t *drain = acc_empty + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&x_full[s], 1);
      mbar_init(&a_full[s], 4);
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
  const int n_tiles = a.n_mt * a.n_nt;

  if (warp == 0) {
    // ---------------- TMA of X
    if (lane == 0) {
      bool ok = true;
      uint32_t it = 0;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
        int mt, nt;
        ql_tile(t, a.n_mt, a.n_nt, mt, nt);
        for (int kb = 0; kb < a.nkb; ++kb, ++it) {
          const uint32_t s = it % STAGES, r = it / STAGES;
          if (!mbar_wait(&empty[s], (r & 1) ^ 1)) { ok = false; break; }
          mbar_arrive_expect_tx(&x_full[s], X_BYTES);
          tma_load_2d(smem + s * STAGE_BYTES + 2 * A_BYTES, &tmX, &x_full[s], kb * BK, nt * BN);
        }
      }
      const uint32_t n_wait = it < STAGES ? it : STAGES;
      for (uint32_t k = 0; k < n_wait; ++k) {
        const uint32_t j = it - 1 - k;
        if (!mbar_wait(&x_full[j % STAGES], (j / STAGES) & 1)) ok = false;
      }
      if (!ok) set_status(a.status, kDevTimeout);
    }
  } else if (warp >= 2 && warp <= 5) {
    // ---------------- producers: W^ rows as bf16 hi + lo
    const int r = threadIdx.x - 64;  // row of the tile, 0..127
    bool ok = true;
    uint32_t it = 0;
    if constexpr (BITS == 0) {
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
        int mt, nt;
        ql_tile(t, a.n_mt, a.n_nt, mt, nt);
        const int64_t m = static_cast<int64_t>(mt) * BM + r;
        for (int kb = 0; kb < a.nkb; ++kb, ++it) {
          const uint32_t s = it % STAGES, ph = it / STAGES;
          ok = __all_sync(0xffffffffu, mbar_wait(&empty[s], (ph & 1) ^ 1));
          if (!ok) break;
          float w[64];
          if (m < a.d_out) {
            dense_weights<T>(a, m, static_cast<int64_t>(kb) * BK, w);
          } else {
#pragma unroll
            for (int k = 0; k < 64; ++k) w[k] = 0.0f;
          }
          uint8_t *hi_row = smem + s * STAGE_BYTES + r * 128;
#pragma unroll
          for (int cb = 0; cb < 8; ++cb) {
            float w8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) w8[e] = w[8 * cb + e];
            store_chunk(hi_row, hi_row + A_BYTES, r, cb, w8);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&a_full[s]);
        }
      }
    } else {
      const bool uniform = a.g_idx == nullptr && (a.group_size <= 0 || a.group_size % 64 == 0);
      // (t, kb) in processing order; the codes of the next step are loaded
      // before waiting for this step's stage
      int t = blockIdx.x, kb = 0;
      CodeSlot<BITS> nxt;
      auto row_of = [&](int tt) {
        int mt, nt;
        ql_tile(tt, a.n_mt, a.n_nt, mt, nt);
        return static_cast<int64_t>(mt) * BM + r;
      };
      if (t < n_tiles) load_slot<BITS>(a, row_of(t), 0, uniform, nxt);
      while (t < n_tiles && ok) {
        const CodeSlot<BITS> cur = nxt;
        const int64_t m = row_of(t);
        const int64_t k0 = static_cast<int64_t>(kb) * BK;
        int t2 = t, kb2 = kb + 1;
        if (kb2 == a.nkb) {
          t2 = t + static_cast<int>(gridDim.x);
          kb2 = 0;
        }
        if (t2 < n_tiles) load_slot<BITS>(a, row_of(t2), static_cast<int64_t>(kb2) * BK, uniform, nxt);
        const uint32_t s = it % STAGES, ph = it / STAGES;
        ok = __all_sync(0xffffffffu, mbar_wait(&empty[s], (ph & 1) ^ 1));
        if (!ok) break;
        uint8_t *hi_row = smem + s * STAGE_BYTES + r * 128;
#pragma unroll
        for (int cb = 0; cb < 8; ++cb) {
          float w8[8];
          slot_chunk<BITS>(a, m, k0, uniform, cur, cb, w8);
          store_chunk(hi_row, hi_row + A_BYTES, r, cb, w8);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&a_full[s]);
        ++it;
        t = t2;
        kb = kb2;
      }
    }
    if (!ok && lane == 0) set_status(a.status, kDevTimeout);
  } else if (warp == 1) {
    // ---------------- MMA issuer
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
          if (!mbar_wait(&x_full[s], r & 1) || !mbar_wait(&a_full[s], r & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sh = smem_u32(smem + s * STAGE_BYTES);
          const uint32_t sl = sh + A_BYTES;
          const uint32_t sx = sh + 2 * A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
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
    // ---------------- epilogue: warps 6..13, thread = output feature
    const int ew = warp - 6;
    const int quarter = warp & 3;
    const int half = ew >> 2;
    uint32_t ch = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++ch) {
      const uint32_t buf = ch & 1, use = ch >> 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[buf], use & 1));
      if (!ok) break;
      tc_fence_after();
      int mt, nt;
      ql_tile(t, a.n_mt, a.n_nt, mt, nt);
      const int64_t m = static_cast<int64_t>(mt) * BM + quarter * 32 + lane;
      const int64_t n0 = static_cast<int64_t>(nt) * BN + half * 128;
      const uint32_t taddr =
          tmem + (static_cast<uint32_t>(quarter * 32) << 16) + buf * BN + half * 128;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float v[32];
        tmem_ld32(taddr + c * 32, v);
        if (m >= a.d_out) continue;
        if (a.Y) {
          float *yrow = a.Y + m * a.ldy + n0 + c * 32;
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            const int64_t n = n0 + c * 32 + i;
            if (n + 3 < a.n_tok) {
              *reinterpret_cast<float4 *>(yrow + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
            } else {
#pragma unroll
              for (int e = 0; e < 4; ++e)
                if (n + e < a.n_tok) yrow[i + e] = v[i + e];
            }
          }
        }
        if (a.Z) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int64_t n = n0 + c * 32 + i;
            if (n < a.n_tok) {
              float o = activate(v[i], a.act);
              if (a.R) o += __bfloat162float(a.R[n * a.d_out + m]);
              a.Z[n * a.d_out + m] = __float2bfloat16_rn(o);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
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

template <int BITS, typename T>
gq_status launch_typed(const CUtensorMap &tmX, const QlArgs &a, cudaStream_t st) {
  cudaFuncSetAttribute(qlinear_kernel<BITS, T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       static_cast<int>(SMEM_BYTES));
  const int n_tiles = a.n_mt * a.n_nt;
  const int grid = n_tiles < num_sms() ? n_tiles : num_sms();
  const int slot = timer_begin(GQ_KERNEL_QLINEAR, st);
  qlinear_kernel<BITS, T><<<grid, NUM_THREADS, SMEM_BYTES, st>>>(tmX, a);
  count_launch();
  // the product: 2 n_tok d_out d_in flops (two bf16 passes, hi and lo)
  timer_end(slot, st, 2.0 * static_cast<double>(a.n_tok) * a.d_out * a.d_in);
  return check_launch("qlinear_kernel");
}

}  // namespace

gq_status launch_qlinear(const uint32_t *qpacked, const uint16_t *scales, const uint16_t *zeros,
                         const int32_t *g_idx, const void *W_dense, gq_dtype w_dtype,
                         int64_t d_out, int64_t d_in, int bits, int group_size, int sym,
                         const void *X, int64_t n_tok, float *Y, void *Z, const void *R,
                         int act, int *status, cudaStream_t st) {
  if (status && cudaMemsetAsync(status, 0, sizeof(int), st) != cudaSuccess)
    return check_launch("memset");
  if (n_tok == 0) return GQ_OK;
  QlArgs a{};
  a.q = qpacked;
  a.scales = scales;
  a.zeros = zeros;
  a.g_idx = g_idx;
  a.Wd = W_dense;
  a.w_dtype = w_dtype;
  a.d_out = d_out;
  a.d_in = d_in;
  a.n_tok = n_tok;
  a.group_size = group_size == 0 ? -1 : group_size;  // per tensor is stored per row
  a.sym = sym;
  a.n_groups = group_size <= 0 ? 1 : static_cast<int>(d_in / group_size);
  a.n_mt = static_cast<int>((d_out + BM - 1) / BM);
  a.n_nt = static_cast<int>((n_tok + BN - 1) / BN);
  a.nkb = static_cast<int>((d_in + BK - 1) / BK);
  a.Y = Y;
  a.ldy = n_tok;
  a.Z = static_cast<__nv_bfloat16 *>(Z);
  a.R = static_cast<const __nv_bfloat16 *>(R);
  a.act = act;
  a.status = status;
  CUtensorMap tmX;
  const gq_status s =
      make_tmap_2d(&tmX, X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d_in, n_tok, d_in, BK, BN);
  if (s != GQ_OK) return s;
  if (qpacked == nullptr) {
    switch (w_dtype) {
      case GQ_F32: return launch_typed<0, float>(tmX, a, st);
      case GQ_F16: return launch_typed<0, __half>(tmX, a, st);
      case GQ_BF16: return launch_typed<0, __nv_bfloat16>(tmX, a, st);
    }
    return fail(GQ_ERR_DTYPE, "unknown w_dtype");
  }
  switch (bits) {
    case 2: return launch_typed<2, float>(tmX, a, st);
    case 3: return launch_typed<3, float>(tmX, a, st);
    case 4: return launch_typed<4, float>(tmX, a, st);
    case 8: return launch_typed<8, float>(tmX, a, st);
  }
  return fail(GQ_ERR_ARG, "bits must be 2, 3, 4 or 8");
}

}  // namespace gq
