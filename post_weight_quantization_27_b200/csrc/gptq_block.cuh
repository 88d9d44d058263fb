// The GPTQ column-block kernel ("GPTQ: Post-Training INT4", "The GPTQ
// Algorithm": the loop over the columns of one block of B columns).
//
// One output row per thread.  The block's columns are taken in sub-blocks
// of SB (32, or 64 when the group size is 64): the SB current weights of the
// row live in registers; the updates that the block's earlier columns owe
// them are applied first by a compact loop over those columns (their scaled
// errors delta are kept in shared memory, one column of a [B][rows] array
// per thread, so the accesses are conflict free); then the SB columns are
// quantised one after another with the in-sub-block updates in registers.
// Only the SB-step loop is unrolled (by template recursion, so every
// register index is a constant): the kernel's code stays small enough for
// the instruction cache, which a fully unrolled 128-step loop is not.
// The B x B block of U is in shared memory (one TMA copy); every thread
// reads the same element at the same time (broadcast).
//
// Column j:  group start -> scale (and zero) from the current weights of
//            the group; c = code(w_j), q = s (c - z), delta = (w_j - q) /
//            U_jj; w_k -= delta * U_jk for k > j;  w_j := delta (the Err
//            entry).  Divisions use a correctly rounded reciprocal and one
//            FMA correction.
#pragma once

#include "gq_device.cuh"
#include "gq_internal.h"

namespace gq {

struct SubCtx {
  const float *Ub;   // [B][B]
  const float *rU;   // [B]  RN(1 / U_jj)
  float *D;          // [B][rows] scaled errors of this block
  int B, rows, tid, bw;
  bool sym;
  int64_t row, c0, n_groups;
  uint16_t *scales, *zeros;
};

template <int SB, int G, int BITS, int J>
__device__ __forceinline__ void gptq_column(float (&w)[SB], uint32_t (&packed)[SB * BITS / 32],
                                            GridParams &gp, float &rs, const SubCtx &cx,
                                            int jb) {
  if constexpr (J < SB) {
    const int j = jb + J;  // column within the block
    if (j < cx.bw) {
      if constexpr (G > 0 && G <= SB && J % G == 0) {
        float amax = 0.0f, mn = 0.0f, mx = 0.0f;
#pragma unroll
        for (int k = J; k < J + G; ++k) {
          amax = fmaxf(amax, fabsf(w[k]));
          mn = fminf(mn, w[k]);
          mx = fmaxf(mx, w[k]);
        }
        gp = cx.sym ? grid_sym_b<BITS>(amax) : grid_affine_b<BITS>(mn, mx);
        rs = __fdiv_rn(1.0f, gp.s);
        const int64_t gi = (cx.c0 + j) / G;
        cx.scales[cx.row * cx.n_groups + gi] = gp.s_bits;
        if (cx.zeros) cx.zeros[cx.row * cx.n_groups + gi] = cx.sym ? 0 : gp.z_bits;
      }
      const float *urow = cx.Ub + j * cx.B + jb;
      uint32_t nib;
      float c;
      if constexpr (BITS == 4) {
        c = grid_code_fast(w[J], gp, rs, cx.sym, nib);
        packed[J / 8] |= nib << (4 * (J % 8));
      } else {
        c = grid_code_b<BITS>(w[J], gp, rs, cx.sym, nib);
        put_code<BITS, J>(packed, nib);
      }
      const float q = gp.s * (c - gp.z);
      const float delta = div_by_recip(w[J] - q, urow[J], cx.rU[j]);
#pragma unroll
      for (int k = J + 1; k < SB; ++k) w[k] = fmaf(-delta, urow[k], w[k]);
      w[J] = delta;
      cx.D[j * cx.rows + cx.tid] = delta;
    }
    gptq_column<SB, G, BITS, J + 1>(w, packed, gp, rs, cx, jb);
  }
}

// Wk: fp32 working weights [d_out][d_in] (processing order); the block is
// columns c0 .. c0+bw-1.  Writes the block's scaled errors to Err (row
// stride err_ld >= B), and either the packed codes (qpacked, no act-order)
// or one code byte per column (codes).
// The B x B block of U arrives by one TMA copy (entries past the matrix
// edge read as zero; only the upper triangle is used).
template <int B, int G, int BITS>
__global__ void __launch_bounds__(128) gptq_block_kernel(
    const __grid_constant__ CUtensorMap tmU, const float *__restrict__ Wk, int64_t d_out,
    int64_t d_in, int64_t c0, int bw, int sym, float *__restrict__ Err, int64_t err_ld,
    uint32_t *__restrict__ qpacked, uint8_t *__restrict__ codes, uint16_t *__restrict__ scales,
    uint16_t *__restrict__ zeros, int64_t n_groups, int *status) {
  constexpr int SB = (G == 64) ? 64 : 32;
  static_assert(B % SB == 0, "sub-block must divide the block");
  extern __shared__ __align__(128) float Ub[];  // [B][B], rU[B], D[B][rows], mbarrier
  const int rows = blockDim.x, tid = threadIdx.x;
  float *rU = Ub + B * B;
  float *D = rU + B;
  uint64_t *bar = reinterpret_cast<uint64_t *>(D + B * rows);
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (tid == 0) {
    mbar_arrive_expect_tx(bar, B * B * sizeof(float));
    tma_load_2d(Ub, &tmU, bar, static_cast<int32_t>(c0), static_cast<int32_t>(c0));
  }
  if (!mbar_wait(bar, 0)) {
    if (tid == 0) set_status(status, kDevTimeout);
    return;
  }
  for (int j = tid; j < B; j += rows) rU[j] = j < bw ? __fdiv_rn(1.0f, Ub[j * B + j]) : 1.0f;
  __syncthreads();
  const int64_t row = static_cast<int64_t>(blockIdx.x) * rows + tid;
  if (row >= d_out) return;

  const bool s = sym != 0;
  const float *src = Wk + row * d_in + c0;
  GridParams gp{};
  float rs = 1.0f;
  if (G < 0) {  // per-channel scale, computed once from the initial row
    gp.s = __half2float(__ushort_as_half(scales[row]));
    gp.z = s ? 0.0f : __half2float(__ushort_as_half(zeros[row]));
    rs = __fdiv_rn(1.0f, gp.s);
  } else if (G == B) {  // one group per block: its first column sees the initial values
    float amax = 0.0f, mn = 0.0f, mx = 0.0f;
    for (int k = 0; k < bw; k += 4) {
      const float4 v = *reinterpret_cast<const float4 *>(src + k);
      amax = fmaxf(fmaxf(amax, fmaxf(fabsf(v.x), fabsf(v.y))), fmaxf(fabsf(v.z), fabsf(v.w)));
      mn = fminf(fminf(mn, fminf(v.x, v.y)), fminf(v.z, v.w));
      mx = fmaxf(fmaxf(mx, fmaxf(v.x, v.y)), fmaxf(v.z, v.w));
    }
    gp = s ? grid_sym_b<BITS>(amax) : grid_affine_b<BITS>(mn, mx);
    rs = __fdiv_rn(1.0f, gp.s);
    scales[row * n_groups + c0 / B] = gp.s_bits;
    if (zeros) zeros[row * n_groups + c0 / B] = s ? 0 : gp.z_bits;
  }
  const SubCtx cx{Ub, rU, D, B, rows, tid, bw, s, row, c0, n_groups, scales, zeros};
  constexpr int GS = (G == B) ? -1 : G;  // group handled above when it spans the block

  for (int jb = 0; jb < bw; jb += SB) {
    float w[SB];
#pragma unroll
    for (int k = 0; k < SB; k += 4) {
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (jb + k < bw) v = *reinterpret_cast<const float4 *>(src + jb + k);
      w[k] = v.x; w[k + 1] = v.y; w[k + 2] = v.z; w[k + 3] = v.w;
    }
    // updates owed by the block's earlier columns
    for (int j = 0; j < jb; ++j) {
      const float dj = D[j * rows + tid];
      const float *u = Ub + j * B + jb;
#pragma unroll
      for (int k = 0; k < SB; k += 4) {
        const float4 uv = *reinterpret_cast<const float4 *>(u + k);
        w[k] = fmaf(-dj, uv.x, w[k]);
        w[k + 1] = fmaf(-dj, uv.y, w[k + 1]);
        w[k + 2] = fmaf(-dj, uv.z, w[k + 2]);
        w[k + 3] = fmaf(-dj, uv.w, w[k + 3]);
      }
    }
    constexpr int NW = SB * BITS / 32;  // packed words of the sub-block
    uint32_t packed[NW];
#pragma unroll
    for (int i = 0; i < NW; ++i) packed[i] = 0;
    gptq_column<SB, GS, BITS, 0>(w, packed, gp, rs, cx, jb);

    float *err = Err + row * err_ld + jb;
#pragma unroll
    for (int k = 0; k < SB; k += 4)
      *reinterpret_cast<float4 *>(err + k) = make_float4(w[k], w[k + 1], w[k + 2], w[k + 3]);
    if (qpacked) {
      // the sub-block starts on a word boundary: column c0 + jb is a
      // multiple of 32; word i holds stream bits 32 i .. 32 i + 31
      uint32_t *dst = qpacked + row * (d_in * BITS / 32) + (c0 + jb) * BITS / 32;
#pragma unroll
      for (int i = 0; i < NW; ++i)
        if (jb + (32 * i) / BITS < bw) dst[i] = packed[i];
    } else {
      uint8_t *dst = codes + row * d_in + c0 + jb;
#pragma unroll
      for (int i = 0; i < SB / 8; ++i)
        if (jb + i * 8 < bw) {
          uint2 v;
          if constexpr (BITS == 4) {
            v.x = (packed[i] & 0xFu) | ((packed[i] >> 4) & 0xFu) << 8 |
                  ((packed[i] >> 8) & 0xFu) << 16 | ((packed[i] >> 12) & 0xFu) << 24;
            v.y = ((packed[i] >> 16) & 0xFu) | ((packed[i] >> 20) & 0xFu) << 8 |
                  ((packed[i] >> 24) & 0xFu) << 16 | ((packed[i] >> 28) & 0xFu) << 24;
          } else {
            v.x = get_code(packed, BITS, 8 * i) | get_code(packed, BITS, 8 * i + 1) << 8 |
                  get_code(packed, BITS, 8 * i + 2) << 16 | get_code(packed, BITS, 8 * i + 3) << 24;
            v.y = get_code(packed, BITS, 8 * i + 4) | get_code(packed, BITS, 8 * i + 5) << 8 |
                  get_code(packed, BITS, 8 * i + 6) << 16 | get_code(packed, BITS, 8 * i + 7) << 24;
          }
          *reinterpret_cast<uint2 *>(dst + i * 8) = v;
        }
    }
  }
}

typedef gq_status (*GptqBlockLaunch)(const CUtensorMap &, const float *, int64_t, int64_t,
                                     int64_t, int, int, float *, int64_t, uint32_t *, uint8_t *,
                                     uint16_t *, uint16_t *, int64_t, int *, cudaStream_t);

// tmU: fp32 tensor map over U with a B x B box and no swizzle.  Rows per
// CTA shrink for short layers so that more SMs take part.
template <int B, int G, int BITS>
gq_status launch_gptq_block(const CUtensorMap &tmU, const float *Wk, int64_t d_out,
                            int64_t d_in, int64_t c0, int bw, int sym, float *Err,
                            int64_t err_ld, uint32_t *qp, uint8_t *codes, uint16_t *scales,
                            uint16_t *zeros, int64_t n_groups, int *status, cudaStream_t st) {
  const int sms = num_sms();
  const int rows = d_out >= 4 * 128 * sms ? 128 : (d_out >= 2 * 64 * sms ? 64 : 32);
  const size_t smem = (static_cast<size_t>(B) * (B + 1) + static_cast<size_t>(B) * rows) *
                          sizeof(float) + 16;
  cudaFuncSetAttribute(gptq_block_kernel<B, G, BITS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       static_cast<int>(smem));
  const unsigned grid = static_cast<unsigned>((d_out + rows - 1) / rows);
  const int slot = timer_begin(GQ_KERNEL_GPTQ_BLOCK, st);
  gptq_block_kernel<B, G, BITS><<<grid, rows, smem, st>>>(tmU, Wk, d_out, d_in, c0, bw, sym, Err,
                                                    err_ld, qp, codes, scales, zeros, n_groups,
                                                    status);
  count_launch();
  // working weights of the block read, Err written (fp32), the U block,
  // codes (packed: BITS / 8 bytes, else one byte per weight), scales (+ zeros)
  const double groups = G < 0 ? 0.0 : static_cast<double>((bw + G - 1) / G);
  timer_end(slot, st,
            static_cast<double>(d_out) * bw * (8.0 + (qp ? BITS / 8.0 : 1.0)) +
                4.0 * static_cast<double>(B) * B + 2.0 * d_out * groups * (sym ? 1 : 2));
  return GQ_OK;
}

// Instantiated in gptq_b*.cu (one translation unit each, compiled in
// parallel): (block, group, bits); widths other than 4 with block 128.
#define GQ_GPTQ_BLOCK_INSTANCES(X)                                                            \
  X(128, -1, 4) X(128, 128, 4) X(128, 64, 4) X(128, 32, 4) X(64, -1, 4) X(64, 64, 4)           \
  X(64, 32, 4) X(32, -1, 4) X(32, 32, 4)                                                       \
  X(128, -1, 8) X(128, 128, 8) X(128, 64, 8) X(128, 32, 8)                                     \
  X(128, -1, 3) X(128, 128, 3) X(128, 64, 3) X(128, 32, 3)                                     \
  X(128, -1, 2) X(128, 128, 2) X(128, 64, 2) X(128, 32, 2)

#define GQ_BLOCK_SIG(b, g, n)                                                               \
  gq_status launch_gptq_block<b, g, n>(const CUtensorMap &, const float *, int64_t, int64_t,   \
                                       int64_t, int, int, float *, int64_t, uint32_t *,        \
                                       uint8_t *, uint16_t *, uint16_t *, int64_t, int *,      \
                                       cudaStream_t);
#define GQ_DECLARE_BLOCK(b, g, n) extern template GQ_BLOCK_SIG(b, g, n)
#define GQ_DEFINE_BLOCK(b, g, n) template GQ_BLOCK_SIG(b, g, n)

}  // namespace gq
