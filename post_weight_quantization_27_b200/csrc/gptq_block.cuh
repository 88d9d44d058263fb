// The GPTQ column-block kernel ("GPTQ: Post-Training INT4", "The GPTQ
// Algorithm": the loop over the columns of one block of B columns).
//
// One output row per thread.  The row's B weights stay in registers for the
// whole block; the B x B block of U is in shared memory and every thread
// reads the same element at the same time (broadcast, no bank conflicts).
// The column loop is unrolled by template recursion so that every register
// index is a compile-time constant (a plain loop of this size is not fully
// unrolled and would put the weights in local memory).
//
// Column j:  group start -> scale (and zero) from the current weights of
//            the group (a warp-free register reduction over G values);
//            c = code(w_j), q = s (c - z), delta = (w_j - q) / U_jj;
//            w_k -= delta * U_jk for k > j;  w_j := delta (the Err entry).
#pragma once

#include "gq_device.cuh"
#include "gq_internal.h"

namespace gq {

constexpr int GPTQ_ROWS_PER_CTA = 64;

template <int B, int G>
struct BlockCtx {
  const float *Ub;
  int bw;
  bool sym;
  int64_t row, c0, n_groups;
  uint16_t *scales, *zeros;
};

template <int B, int G, int J>
__device__ __forceinline__ void gptq_column(float (&w)[B], uint32_t (&packed)[B / 8],
                                            GridParams &gp, const BlockCtx<B, G> &cx) {
  if constexpr (J < B) {
    if (J < cx.bw) {
      if constexpr (G > 0 && J % G == 0) {
        float amax = 0.0f, mn = 0.0f, mx = 0.0f;
#pragma unroll
        for (int k = J; k < J + G; ++k) {
          amax = fmaxf(amax, fabsf(w[k]));
          mn = fminf(mn, w[k]);
          mx = fmaxf(mx, w[k]);
        }
        gp = cx.sym ? grid_sym(amax) : grid_affine(mn, mx);
        const int64_t gi = (cx.c0 + J) / G;
        cx.scales[cx.row * cx.n_groups + gi] = gp.s_bits;
        if (cx.zeros) cx.zeros[cx.row * cx.n_groups + gi] = cx.sym ? 0 : gp.z_bits;
      }
      const float c = grid_code(w[J], gp, cx.sym);
      const float q = gp.s * (c - gp.z);
      const float delta = __fdiv_rn(w[J] - q, cx.Ub[J * B + J]);
      packed[J / 8] |= grid_nibble(c, cx.sym) << (4 * (J % 8));
#pragma unroll
      for (int k = J + 1; k < B; ++k) w[k] = fmaf(-delta, cx.Ub[J * B + k], w[k]);
      w[J] = delta;
    }
    gptq_column<B, G, J + 1>(w, packed, gp, cx);
  }
}

// Wk: fp32 working weights [d_out][d_in] (processing order); the block is
// columns c0 .. c0+bw-1.  Writes Err [d_out][B], and either the packed
// codes (qpacked, no act-order) or one code byte per column (codes).
template <int B, int G>
__global__ void __launch_bounds__(GPTQ_ROWS_PER_CTA) gptq_block_kernel(
    const float *__restrict__ Wk, int64_t d_out, int64_t d_in, int64_t c0, int bw,
    const float *__restrict__ U, int sym, float *__restrict__ Err,
    uint32_t *__restrict__ qpacked, uint8_t *__restrict__ codes, uint16_t *__restrict__ scales,
    uint16_t *__restrict__ zeros, int64_t n_groups) {
  extern __shared__ __align__(16) float Ub[];  // [B][B], upper triangle of the block
  for (int e = threadIdx.x; e < B * B; e += blockDim.x) {
    const int r = e / B, c = e % B;
    Ub[e] = (r < bw && c < bw && c >= r) ? U[(c0 + r) * d_in + c0 + c] : 0.0f;
  }
  __syncthreads();
  const int64_t row = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (row >= d_out) return;

  float w[B];
  const float *src = Wk + row * d_in + c0;
#pragma unroll
  for (int k = 0; k < B; k += 4) {
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (k < bw) v = *reinterpret_cast<const float4 *>(src + k);
    w[k] = v.x; w[k + 1] = v.y; w[k + 2] = v.z; w[k + 3] = v.w;
  }
  const bool s = sym != 0;
  GridParams gp{};
  if (G < 0) {  // per-channel scale, computed once from the initial row
    gp.s = __half2float(__ushort_as_half(scales[row]));
    gp.z = s ? 0.0f : __half2float(__ushort_as_half(zeros[row]));
  }
  uint32_t packed[B / 8];
#pragma unroll
  for (int i = 0; i < B / 8; ++i) packed[i] = 0;
  const BlockCtx<B, G> cx{Ub, bw, s, row, c0, n_groups, scales, zeros};
  gptq_column<B, G, 0>(w, packed, gp, cx);

  float *err = Err + row * B;
#pragma unroll
  for (int k = 0; k < B; k += 4)
    *reinterpret_cast<float4 *>(err + k) = make_float4(w[k], w[k + 1], w[k + 2], w[k + 3]);
  if (qpacked) {
    uint32_t *dst = qpacked + row * (d_in / 8) + c0 / 8;
#pragma unroll
    for (int i = 0; i < B / 8; ++i)
      if (i * 8 < bw) dst[i] = packed[i];
  } else {
    uint8_t *dst = codes + row * d_in + c0;
#pragma unroll
    for (int i = 0; i < B / 8; ++i)
      if (i * 8 < bw) {
        uint2 v;
        v.x = (packed[i] & 0xFu) | ((packed[i] >> 4) & 0xFu) << 8 |
              ((packed[i] >> 8) & 0xFu) << 16 | ((packed[i] >> 12) & 0xFu) << 24;
        v.y = ((packed[i] >> 16) & 0xFu) | ((packed[i] >> 20) & 0xFu) << 8 |
              ((packed[i] >> 24) & 0xFu) << 16 | ((packed[i] >> 28) & 0xFu) << 24;
        *reinterpret_cast<uint2 *>(dst + i * 8) = v;
      }
  }
}

typedef void (*GptqBlockLaunch)(const float *, int64_t, int64_t, int64_t, int, const float *,
                                int, float *, uint32_t *, uint8_t *, uint16_t *, uint16_t *,
                                int64_t, cudaStream_t);

template <int B, int G>
void launch_gptq_block(const float *Wk, int64_t d_out, int64_t d_in, int64_t c0, int bw,
                       const float *U, int sym, float *Err, uint32_t *qp, uint8_t *codes,
                       uint16_t *scales, uint16_t *zeros, int64_t n_groups, cudaStream_t st) {
  const size_t smem = static_cast<size_t>(B) * B * sizeof(float);
  cudaFuncSetAttribute(gptq_block_kernel<B, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       static_cast<int>(smem));
  const unsigned grid =
      static_cast<unsigned>((d_out + GPTQ_ROWS_PER_CTA - 1) / GPTQ_ROWS_PER_CTA);
  gptq_block_kernel<B, G><<<grid, GPTQ_ROWS_PER_CTA, smem, st>>>(
      Wk, d_out, d_in, c0, bw, U, sym, Err, qp, codes, scales, zeros, n_groups);
  count_launch();
}

// Instantiated in gptq_b*.cu (one translation unit each, compiled in parallel).
#define GQ_GPTQ_BLOCK_INSTANCES(X) \
  X(128, -1) X(128, 128) X(128, 64) X(128, 32) X(64, -1) X(64, 64) X(64, 32) X(32, -1) X(32, 32)

#define GQ_DECLARE_BLOCK(b, g)                                                               \
  extern template void launch_gptq_block<b, g>(const float *, int64_t, int64_t, int64_t, int, \
                                               const float *, int, float *, uint32_t *,       \
                                               uint8_t *, uint16_t *, uint16_t *, int64_t,    \
                                               cudaStream_t);
#define GQ_DEFINE_BLOCK(b, g)                                                         \
  template void launch_gptq_block<b, g>(const float *, int64_t, int64_t, int64_t, int, \
                                        const float *, int, float *, uint32_t *,       \
                                        uint8_t *, uint16_t *, uint16_t *, int64_t,    \
                                        cudaStream_t);

}  // namespace gq
