// Round-to-nearest 4-bit quantisation with int4 packing (HBM-bound).
//
// "GPT-2 Quantization Reconstruction Error" -- "What this project does":
// one scale per output row, 15 levels (symmetric); "Model Quantization
// Mechanics" section 1: affine scale/zero-point per group of g consecutive
// weights; "GPTQ: Post-Training INT4" -- "Group Quantization": 4-bit codes
// plus a 16-bit scale (and zero) per group.
//
// A segment is one (row, group) pair, or a whole row for per-channel.  A
// team of TEAM lanes owns a segment; each lane holds WPL packed words (8
// weights each) in registers, so the weights are read from HBM once with
// 16-byte vector loads and every packed word is written by one coalesced
// 4-byte store.  Rows longer than 32 * 8 words stream twice through L2
// instead (second kernel).
#include "gq_device.cuh"
#include "gq_internal.h"

namespace gq {
namespace {

template <typename T>
struct Vec8;
template <>
struct Vec8<float> {
  static __device__ __forceinline__ void load(const float *p, float (&v)[8]) {
    const float4 a = __ldg(reinterpret_cast<const float4 *>(p));
    const float4 b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
};
template <>
struct Vec8<__half> {
  static __device__ __forceinline__ void load(const __half *p, float (&v)[8]) {
    const uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[i]));
      v[2 * i] = f.x;
      v[2 * i + 1] = f.y;
    }
  }
};
template <>
struct Vec8<__nv_bfloat16> {
  static __device__ __forceinline__ void load(const __nv_bfloat16 *p, float (&v)[8]) {
    const uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[i]));
      v[2 * i] = f.x;
      v[2 * i + 1] = f.y;
    }
  }
};

// Code word of 8 weights.  rs = RN(1 / s): the quotient w / s is formed as a
// correctly rounded division from the reciprocal (gq_device.cuh), so the
// decision rint(w / s) is the IEEE one in three instructions; the rest is
// integer arithmetic (round-half-even conversion, clamp, nibble insert).
template <bool SYM>
__device__ __forceinline__ uint32_t pack_word(const float (&v)[8], const GridParams &g,
                                              float rs) {
  const int z = static_cast<int>(g.z);
  uint32_t word = 0;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    int c = __float2int_rn(div_by_recip(v[k], g.s, rs));
    if (SYM) {
      c = min(max(c, -7), 7) + 8;
    } else {
      c = min(max(c, -16), 16) + z;
      c = min(max(c, 0), 15);
    }
    word |= static_cast<uint32_t>(c) << (4 * k);
  }
  return word;
}

// Running statistic of a segment: max |w| (symmetric) or min and max (affine;
// both start at 0, which is what the grid's range widening needs).
template <bool SYM>
struct SegStat {
  float a = 0.0f, b = 0.0f;
  __device__ __forceinline__ void add(float x) {
    if (SYM) {
      a = fmaxf(a, fabsf(x));
    } else {
      a = fminf(a, x);
      b = fmaxf(b, x);
    }
  }
  __device__ __forceinline__ void reduce(int width) {
    for (int off = width / 2; off > 0; off >>= 1) {
      if (SYM) {
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
      } else {
        a = fminf(a, __shfl_xor_sync(0xffffffffu, a, off));
        b = fmaxf(b, __shfl_xor_sync(0xffffffffu, b, off));
      }
    }
  }
  __device__ __forceinline__ GridParams grid() const {
    return SYM ? grid_sym(a) : grid_affine(a, b);
  }
};

// Segments of at most TEAM * WPL words, held in registers.  UNROLL
// segment groups per warp iteration keep enough loads in flight.
template <typename T, int TEAM, int WPL, int UNROLL, bool SYM>
__global__ void __launch_bounds__(256) rtn_reg_kernel(const T *__restrict__ W, int64_t total,
                                                      int64_t seg_words,
                                                      uint32_t *__restrict__ q,
                                                      uint16_t *__restrict__ scales,
                                                      uint16_t *__restrict__ zeros) {
  constexpr int SPW = 32 / TEAM;  // segments per warp per unroll step
  const int lane = threadIdx.x & 31;
  const int tl = lane % TEAM;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;

  // segment s = row * n_groups + group; every segment starts seg_words * 8
  // weights after the previous one, so its address needs no division
  for (int64_t base = warp * SPW * UNROLL; base < total; base += n_warps * SPW * UNROLL) {
    float v[UNROLL][WPL][8];
    int64_t seg[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      seg[u] = base + u * SPW + lane / TEAM;
      const bool act = seg[u] < total;
      const T *src = W + (act ? seg[u] : 0) * seg_words * 8;
#pragma unroll
      for (int k = 0; k < WPL; ++k) {
        const int64_t w = tl + static_cast<int64_t>(k) * TEAM;
        if (act && w < seg_words) {
          Vec8<T>::load(src + w * 8, v[u][k]);
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) v[u][k][e] = 0.0f;  // never changes the statistic
        }
      }
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      SegStat<SYM> st;
#pragma unroll
      for (int k = 0; k < WPL; ++k)
#pragma unroll
        for (int e = 0; e < 8; ++e) st.add(v[u][k][e]);
      st.reduce(TEAM);
      if (seg[u] >= total) continue;
      const GridParams g = st.grid();
      const float rs = __frcp_rn(g.s);
      if (tl == 0) {
        scales[seg[u]] = g.s_bits;
        if (zeros) zeros[seg[u]] = SYM ? 0 : g.z_bits;
      }
      uint32_t *dst = q + seg[u] * seg_words;
#pragma unroll
      for (int k = 0; k < WPL; ++k) {
        const int64_t w = tl + static_cast<int64_t>(k) * TEAM;
        if (w < seg_words) dst[w] = pack_word<SYM>(v[u][k], g, rs);
      }
    }
  }
}

// Long rows (per-channel with a large d_in): one warp per row, two passes.
template <typename T, bool SYM>
__global__ void __launch_bounds__(256) rtn_stream_kernel(const T *__restrict__ W, int64_t d_out,
                                                         int64_t d_in,
                                                         uint32_t *__restrict__ q,
                                                         uint16_t *__restrict__ scales,
                                                         uint16_t *__restrict__ zeros) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int64_t words = d_in / 8;
  for (int64_t row = warp; row < d_out; row += n_warps) {
    const T *src = W + row * d_in;
    SegStat<SYM> st;
#pragma unroll 4
    for (int64_t w = lane; w < words; w += 32) {
      float v[8];
      Vec8<T>::load(src + w * 8, v);
#pragma unroll
      for (int e = 0; e < 8; ++e) st.add(v[e]);
    }
    st.reduce(32);
    const GridParams g = st.grid();
    const float rs = __frcp_rn(g.s);
    if (lane == 0) {
      scales[row] = g.s_bits;
      if (zeros) zeros[row] = SYM ? 0 : g.z_bits;
    }
#pragma unroll 4
    for (int64_t w = lane; w < words; w += 32) {
      float v[8];
      Vec8<T>::load(src + w * 8, v);
      q[row * words + w] = pack_word<SYM>(v, g, rs);
    }
  }
}

template <typename T, int TEAM, int WPL, int UNROLL>
void launch_reg(const void *W, int64_t d_out, int64_t seg_words, int64_t n_groups, int sym,
                uint32_t *q, uint16_t *sc, uint16_t *z, cudaStream_t st) {
  const int64_t total = d_out * n_groups;
  const int64_t per_block = (256 / 32) * (32 / TEAM) * UNROLL;
  int64_t blocks = (total + per_block - 1) / per_block;
  const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
  if (blocks > cap) blocks = cap;
  const T *w = static_cast<const T *>(W);
  if (sym)
    rtn_reg_kernel<T, TEAM, WPL, UNROLL, true><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        w, total, seg_words, q, sc, z);
  else
    rtn_reg_kernel<T, TEAM, WPL, UNROLL, false><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        w, total, seg_words, q, sc, z);
  count_launch();
}

template <typename T>
gq_status launch_typed(const void *W, int64_t d_out, int64_t d_in, int group_size, int sym,
                       uint32_t *q, uint16_t *sc, uint16_t *z, cudaStream_t st) {
  const int64_t seg_len = group_size == -1 ? d_in : group_size;
  const int64_t n_groups = d_in / seg_len;
  const int64_t words = seg_len / 8;
  if (words <= 1) launch_reg<T, 1, 1, 4>(W, d_out, words, n_groups, sym, q, sc, z, st);
  else if (words <= 2) launch_reg<T, 2, 1, 4>(W, d_out, words, n_groups, sym, q, sc, z, st);
  else if (words <= 4) launch_reg<T, 4, 1, 4>(W, d_out, words, n_groups, sym, q, sc, z, st);
  else if (words <= 8) launch_reg<T, 8, 1, 4>(W, d_out, words, n_groups, sym, q, sc, z, st);
  else if (words <= 16) launch_reg<T, 16, 1, 4>(W, d_out, words, n_groups, sym, q, sc, z, st);
  else if (words <= 32) launch_reg<T, 32, 1, 4>(W, d_out, words, n_groups, sym, q, sc, z, st);
  else if (words <= 64) launch_reg<T, 32, 2, 2>(W, d_out, words, n_groups, sym, q, sc, z, st);
  else if (words <= 128) launch_reg<T, 32, 4, 1>(W, d_out, words, n_groups, sym, q, sc, z, st);
  else if (words <= 256) launch_reg<T, 32, 8, 1>(W, d_out, words, n_groups, sym, q, sc, z, st);
  else {
    int64_t blocks = (d_out + 7) / 8;
    const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
    if (blocks > cap) blocks = cap;
    const T *w = static_cast<const T *>(W);
    if (sym)
      rtn_stream_kernel<T, true><<<static_cast<unsigned>(blocks), 256, 0, st>>>(w, d_out, d_in,
                                                                               q, sc, z);
    else
      rtn_stream_kernel<T, false><<<static_cast<unsigned>(blocks), 256, 0, st>>>(w, d_out, d_in,
                                                                                q, sc, z);
    count_launch();
  }
  return check_launch("rtn_quantize_pack");
}

}  // namespace

gq_status launch_rtn(const void *W, gq_dtype dt, int64_t d_out, int64_t d_in, int group_size,
                     int sym, uint32_t *qpacked, uint16_t *scales, uint16_t *zeros,
                     cudaStream_t st) {
  switch (dt) {
    case GQ_F32:
      return launch_typed<float>(W, d_out, d_in, group_size, sym, qpacked, scales, zeros, st);
    case GQ_F16:
      return launch_typed<__half>(W, d_out, d_in, group_size, sym, qpacked, scales, zeros, st);
    case GQ_BF16:
      return launch_typed<__nv_bfloat16>(W, d_out, d_in, group_size, sym, qpacked, scales, zeros,
                                         st);
  }
  return fail(GQ_ERR_DTYPE, "unknown dtype");
}

}  // namespace gq
