// GPTQ on one layer: the column-block kernel and the lazy trailing update.
//
// "GPTQ: Post-Training INT4" -- "The GPTQ Algorithm": columns in a fixed
// order, blocks of B columns; inside a block, for each column j the code of
// the current weight, delta = (w - q) / U_jj and w[j+1:end] -= delta *
// U[j, j+1:end]; after the block one batched update W[:, end:] -= Err *
// U[blk, end:].  "Group Quantization": a group's scale (and zero) comes
// from its current weights when its first column is reached.
//
// Layout: W is copied once to an fp32 working matrix Wk [d_out][d_in] in
// processing order (act-order gather and dead-column zeroing fused into the
// copy).  The block kernel keeps the B x B block of U in shared memory and
// gives every output row to one thread, whose B weights live in registers
// for the whole block: the in-block update is register FMAs against
// broadcast shared-memory reads, with no shuffles and no synchronisation.
// A processed weight's register is reused for its scaled error delta, so
// the Err block leaves the kernel in one contiguous store per row.
//
// The lazy trailing update is done on two levels.  Columns are grouped in
// super-blocks of S columns (S a power-of-two multiple of B near
// sqrt(B d_in)); after each block only the rest of its super-block is
// updated (K = B), and after each super-block the columns beyond it get
// the whole super-block's update in one GEMM (K = S) from the scaled errors
// of all its blocks.  Every update the single-level scheme applies is
// applied, only summed in another order; the traffic over the trailing
// weights drops from about d_in / 2B to about S / 2B + d_in / 2S fp32
// read-writes per weight.  Both GEMMs are fp32 on the tensor cores
// (gemm_tc.cu).
#include <cmath>

#include "gptq_block.cuh"

namespace gq {

GQ_GPTQ_BLOCK_INSTANCES(GQ_DECLARE_BLOCK)

namespace {

// Super-block width: B times the power of two nearest (on a log scale)
// sqrt(d_in / B), at most the block-rounded width of the layer.
int64_t super_cols(int64_t d_in, int B) {
  const double target = std::sqrt(static_cast<double>(B) * static_cast<double>(d_in));
  int64_t S = B;
  while (static_cast<double>(2 * S) <= target * 1.4142135623730951) S *= 2;
  const int64_t full = (d_in + B - 1) / B * B;
  return S < full ? S : full;
}

struct GptqWs {
  float *Wk;        // [d_out][d_in] fp32 working copy, processing order
  float *Err;       // [d_out][S] scaled errors of the current super-block
  uint8_t *codes;   // [d_out][d_in] codes in processing order (act-order only)
  int32_t *inv;     // [d_in] processing position of each original column
};

GptqWs carve(void *ws, int64_t d_out, int64_t d_in, int B, bool with_perm) {
  uint8_t *p = static_cast<uint8_t *>(ws) + kWsHeader;
  GptqWs w{};
  w.Wk = reinterpret_cast<float *>(p);
  p += round_up(static_cast<size_t>(d_out) * d_in * sizeof(float), 256);
  w.Err = reinterpret_cast<float *>(p);
  p += round_up(static_cast<size_t>(d_out) * super_cols(d_in, B) * sizeof(float), 256);
  if (with_perm) {
    w.codes = p;
    p += round_up(static_cast<size_t>(d_out) * d_in, 256);
    w.inv = reinterpret_cast<int32_t *>(p);
  }
  return w;
}

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__half>(__half v) { return __half2float(v); }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}

// Wk[r][p] = dead[src] ? 0 : W[r][src], src = perm ? perm[p] : p.  One
// warp per row, lanes over columns: no division per element; without a
// permutation each lane converts 4 consecutive columns (d_in is a
// multiple of 8) with one 16-byte store.
template <typename T>
__global__ void __launch_bounds__(256) prep_kernel(const T *__restrict__ W, int64_t d_out,
                                                   int64_t d_in, const int32_t *__restrict__ perm,
                                                   const uint8_t *__restrict__ dead,
                                                   float *__restrict__ Wk) {
  const int lane = threadIdx.x & 31;
  const int64_t nw = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       r < d_out; r += nw) {
    const T *wr = W + r * d_in;
    float *dst = Wk + r * d_in;
    if (perm) {
      for (int64_t p = lane; p < d_in; p += 32) {
        int64_t src = perm[p];
        src = src < 0 ? 0 : (src >= d_in ? d_in - 1 : src);  // never read outside the row
        float v = to_f32(wr[src]);
        if (dead && dead[src]) v = 0.0f;
        dst[p] = v;
      }
    } else {
      for (int64_t p = 4 * lane; p < d_in; p += 128) {
        float4 v = make_float4(to_f32(wr[p]), to_f32(wr[p + 1]), to_f32(wr[p + 2]),
                               to_f32(wr[p + 3]));
        if (dead) {
          if (dead[p]) v.x = 0.0f;
          if (dead[p + 1]) v.y = 0.0f;
          if (dead[p + 2]) v.z = 0.0f;
          if (dead[p + 3]) v.w = 0.0f;
        }
        *reinterpret_cast<float4 *>(dst + p) = v;
      }
    }
  }
}

// Per-channel grid from the initial (working) row: one warp per row.
template <int BITS>
__global__ void __launch_bounds__(256) row_params_kernel(const float *__restrict__ Wk,
                                                         int64_t d_out, int64_t d_in, int sym,
                                                         uint16_t *__restrict__ scales,
                                                         uint16_t *__restrict__ zeros) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t r = warp; r < d_out; r += n_warps) {
    float amax = 0.0f, mn = 0.0f, mx = 0.0f;
    for (int64_t c = lane; c < d_in; c += 32) {
      const float v = Wk[r * d_in + c];
      amax = fmaxf(amax, fabsf(v));
      mn = fminf(mn, v);
      mx = fmaxf(mx, v);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    }
    if (lane == 0) {
      const GridParams g = sym ? grid_sym_b<BITS>(amax) : grid_affine_b<BITS>(mn, mx);
      scales[r] = g.s_bits;
      if (zeros) zeros[r] = sym ? 0 : g.z_bits;
    }
  }
}

__global__ void invert_perm_kernel(const int32_t *__restrict__ perm, int64_t d,
                                   int32_t *__restrict__ inv) {
  for (int64_t p = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; p < d;
       p += static_cast<int64_t>(gridDim.x) * 256)
  {
    const int32_t q = perm[p];
    if (q >= 0 && q < d) inv[q] = static_cast<int32_t>(p);
  }
}

// qpacked from the processing-order stored codes: column c of row r takes
// codes[r][inv[c]].  Each thread packs one run of columns that fills whole
// words: 8 columns (one word) at 4 bits, else 32 columns (bits words).
__global__ void __launch_bounds__(256) pack_perm_kernel(const uint8_t *__restrict__ codes,
                                                        int64_t d_out, int64_t d_in,
                                                        const int32_t *__restrict__ inv,
                                                        uint32_t *__restrict__ qpacked,
                                                        int bits) {
  const int run = bits == 4 ? 8 : 32;          // columns per unit
  const int nw = run * bits / 32;              // words per unit
  const int64_t units = d_in / run;
  const int64_t n = d_out * units;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * 256) {
    const int64_t r = e / units, u = e % units;
    uint32_t v[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int k = 0; k < run; ++k) {
      int64_t pos = inv[u * run + k];
      pos = pos < 0 ? 0 : (pos >= d_in ? d_in - 1 : pos);
      put_code_rt(v, bits, k, static_cast<uint32_t>(codes[r * d_in + pos]));
    }
    uint32_t *dst = qpacked + r * (d_in * bits / 32) + u * nw;
    for (int i = 0; i < nw; ++i) dst[i] = v[i];
  }
}

__global__ void g_idx_kernel(const int32_t *__restrict__ inv, int64_t d, int g,
                             int32_t *__restrict__ g_idx) {
  for (int64_t c = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; c < d;
       c += static_cast<int64_t>(gridDim.x) * 256) {
    const int64_t pos = inv ? inv[c] : c;
    g_idx[c] = g < 0 ? 0 : static_cast<int32_t>(pos / g);
  }
}

GptqBlockLaunch pick_block(int B, int G, int bits) {
#define GQ_PICK(b, g, n) \
  if (B == b && G == g && bits == n) return launch_gptq_block<b, g, n>;
  GQ_GPTQ_BLOCK_INSTANCES(GQ_PICK)
#undef GQ_PICK
  return nullptr;
}

}  // namespace

size_t gptq_ws_bytes(int64_t d_out, int64_t d_in, int block_size) {
  return kWsHeader + round_up(static_cast<size_t>(d_out) * d_in * sizeof(float), 256) +
         round_up(static_cast<size_t>(d_out) * super_cols(d_in, block_size) * sizeof(float),
                  256) +
         round_up(static_cast<size_t>(d_out) * d_in, 256) +
         round_up(static_cast<size_t>(d_in) * sizeof(int32_t), 256);
}

gq_status launch_gptq(const void *W, gq_dtype dt, int64_t d_out, int64_t d_in, const float *U,
                      int group_size, int block_size, int sym, const int32_t *perm,
                      const uint8_t *dead, uint32_t *qpacked, uint16_t *scales, uint16_t *zeros,
                      int32_t *g_idx, void *ws, cudaStream_t st, int bits) {
  const int B = block_size;
  const bool per_tensor = group_size == 0;  // one scale for the matrix, stored per row
  if (per_tensor) group_size = -1;
  GptqBlockLaunch blk = pick_block(B, group_size, bits);
  if (!blk) return fail(GQ_ERR_ARG, "unsupported (block_size, group_size, bits) combination");
  GptqWs w = carve(ws, d_out, d_in, B, perm != nullptr);
  const unsigned cap = static_cast<unsigned>(num_sms()) * 16;
  unsigned grid = static_cast<unsigned>((d_out + 7) / 8);  // a warp per row
  if (grid > cap) grid = cap;
  switch (dt) {
    case GQ_F32:
      prep_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float *>(W), d_out, d_in, perm,
                                               dead, w.Wk);
      break;
    case GQ_F16:
      prep_kernel<__half><<<grid, 256, 0, st>>>(static_cast<const __half *>(W), d_out, d_in,
                                                perm, dead, w.Wk);
      break;
    case GQ_BF16:
      prep_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16 *>(W),
                                                       d_out, d_in, perm, dead, w.Wk);
      break;
  }
  count_launch();
  const int64_t n_groups = group_size == -1 ? 1 : d_in / group_size;
  if (per_tensor) {
    const gq_status s = launch_tensor_params_f32(
        w.Wk, d_out, d_in, sym, scales, zeros, w.Err,
        d_out * super_cols(d_in, B), st, bits);
    if (s != GQ_OK) return s;
  } else if (group_size == -1) {
    unsigned g2 = static_cast<unsigned>((d_out + 7) / 8);
    if (g2 > cap) g2 = cap;
    switch (bits) {
      case 2: row_params_kernel<2><<<g2, 256, 0, st>>>(w.Wk, d_out, d_in, sym, scales, zeros); break;
      case 3: row_params_kernel<3><<<g2, 256, 0, st>>>(w.Wk, d_out, d_in, sym, scales, zeros); break;
      case 8: row_params_kernel<8><<<g2, 256, 0, st>>>(w.Wk, d_out, d_in, sym, scales, zeros); break;
      default: row_params_kernel<4><<<g2, 256, 0, st>>>(w.Wk, d_out, d_in, sym, scales, zeros);
    }
    count_launch();
  }
  int *status = static_cast<int *>(ws);
  if (cudaMemsetAsync(status, 0, kWsHeader, st) != cudaSuccess) return check_launch("memset");
  CUtensorMap tmU;
  {
    const gq_status s = make_tmap_2d(&tmU, U, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, d_in, d_in,
                                     d_in, B, B, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (s != GQ_OK) return s;
  }
  const int64_t S = super_cols(d_in, B);
  for (int64_t s0 = 0; s0 < d_in; s0 += S) {
    const int64_t s1 = s0 + S < d_in ? s0 + S : d_in;
    for (int64_t c0 = s0; c0 < s1; c0 += B) {
      const int bw = static_cast<int>(s1 - c0 < B ? s1 - c0 : B);
      float *err = w.Err + (c0 - s0);
      blk(tmU, w.Wk, d_out, d_in, c0, bw, sym, err, S, perm ? nullptr : qpacked, w.codes,
          scales, zeros, n_groups, status, st);
      const int64_t c1 = c0 + bw;
      if (c1 < s1) {
        // W[:, c1:s1] -= Err_blk U[c0:c1, c1:s1]
        const gq_status s = launch_gemm_tf32x3(
            static_cast<int>(d_out), static_cast<int>(s1 - c1), bw, -1.0f, err, S,
            U + c0 * d_in + c1, d_in, false, 1.0f, w.Wk + c1, d_in, false, status, st);
        if (s != GQ_OK) return s;
      }
    }
    if (s1 < d_in) {
      // W[:, s1:] -= Err_super U[s0:s1, s1:]
      const gq_status s = launch_gemm_tf32x3(
          static_cast<int>(d_out), static_cast<int>(d_in - s1), static_cast<int>(s1 - s0), -1.0f,
          w.Err, S, U + s0 * d_in + s1, d_in, false, 1.0f, w.Wk + s1, d_in, false, status, st);
      if (s != GQ_OK) return s;
    }
  }
  const unsigned gd = static_cast<unsigned>((d_in + 255) / 256);
  if (perm) {
    invert_perm_kernel<<<gd, 256, 0, st>>>(perm, d_in, w.inv);
    count_launch();
    unsigned gp = static_cast<unsigned>((d_out * (d_in / (bits == 4 ? 8 : 32)) + 255) / 256);
    if (gp > cap) gp = cap;
    pack_perm_kernel<<<gp, 256, 0, st>>>(w.codes, d_out, d_in, w.inv, qpacked, bits);
    count_launch();
  }
  if (g_idx) {
    g_idx_kernel<<<gd, 256, 0, st>>>(perm ? w.inv : nullptr, d_in, group_size, g_idx);
    count_launch();
  }
  return check_launch("gptq_quantize_layer");
}

}  // namespace gq
