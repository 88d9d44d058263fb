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
#include <cstring>
#include <type_traits>

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

// Eight weights as loaded (16-bit types stay packed, 4 registers per word),
// converted to fp32 where used, so that more words can be in flight.
template <typename T>
struct Raw8;
template <>
struct Raw8<float> {
  float4 a, b;
  __device__ __forceinline__ void load(const float *p) {
    a = __ldg(reinterpret_cast<const float4 *>(p));
    b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
  }
  __device__ __forceinline__ void zero() { a = b = make_float4(0.f, 0.f, 0.f, 0.f); }
  __device__ __forceinline__ void get(float (&v)[8]) const {
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
};
template <typename H2>
struct Raw8Half {
  uint4 u;
  __device__ __forceinline__ void zero() { u = make_uint4(0, 0, 0, 0); }
  __device__ __forceinline__ void get(float (&v)[8]) const {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if constexpr (std::is_same<H2, __half2>::value) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[i]));
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
      } else {  // a bf16 value is the upper half of the fp32 with the same value
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
      }
    }
  }
};
template <>
struct Raw8<__half> : Raw8Half<__half2> {
  __device__ __forceinline__ void load(const __half *p) {
    u = __ldg(reinterpret_cast<const uint4 *>(p));
  }
};
template <>
struct Raw8<__nv_bfloat16> : Raw8Half<__nv_bfloat162> {
  __device__ __forceinline__ void load(const __nv_bfloat16 *p) {
    u = __ldg(reinterpret_cast<const uint4 *>(p));
  }
};

// Running min and max of 0 and the weights seen, in the weights' own type
// (min and max are exact in every format, and a 16-bit pair takes one
// instruction for two weights), read out as fp32 once per segment.  NaN is
// passed over, as fminf / fmaxf do.
template <typename T>
struct MinMax;
template <>
struct MinMax<float> {
  float mn = 0.0f, mx = 0.0f;
  __device__ __forceinline__ void add(const Raw8<float> &r) {
    float v[8];
    r.get(v);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      mn = fminf(mn, v[e]);
      mx = fmaxf(mx, v[e]);
    }
  }
  __device__ __forceinline__ void get(float &lo, float &hi) const {
    lo = mn;
    hi = mx;
  }
};
template <typename H2>
struct MinMaxHalf {
  H2 mn, mx;
  __device__ __forceinline__ MinMaxHalf() {
    const uint32_t zero = 0u;
    memcpy(&mn, &zero, 4);
    memcpy(&mx, &zero, 4);
  }
  __device__ __forceinline__ void add(const Raw8Half<H2> &r) {
    const uint32_t w[4] = {r.u.x, r.u.y, r.u.z, r.u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      H2 h;
      memcpy(&h, &w[i], 4);
      mn = __hmin2(mn, h);
      mx = __hmax2(mx, h);
    }
  }
  __device__ __forceinline__ void get(float &lo, float &hi) const {
    lo = fminf(__low2float(mn), __high2float(mn));
    hi = fmaxf(__low2float(mx), __high2float(mx));
  }
};
template <>
struct MinMax<__half> : MinMaxHalf<__half2> {};
template <>
struct MinMax<__nv_bfloat16> : MinMaxHalf<__nv_bfloat162> {};

// Code word of 8 weights.  rs = RN(1 / s): the quotient w / s is formed as a
// correctly rounded division from the reciprocal and rounded exactly with a
// magic-constant addition (gq_device.cuh), so the decision rint(w / s) is the
// IEEE one in a handful of full-rate instructions per weight.
template <bool SYM>
__device__ __forceinline__ uint32_t pack_word(const float (&v)[8], const GridParams &g,
                                              float rs) {
  uint32_t word = 0;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    uint32_t nib;
    grid_code_fast(v[k], g, rs, SYM, nib);
    word |= nib << (4 * k);
  }
  return word;
}

// The same codes for a group whose quotients are known to be small (see
// SegStat::grid: |w / s| < 23), so C + OFF + rint(q) is exact and the code is
// read from the bits of that sum as an integer.
//
// Two weights at a time: the division from the reciprocal and the rounding
// addition run on the paired fp32 pipe (f32x2 mul / fma / add, each half an
// IEEE round-to-nearest operation, so the quotient and its rounding are those
// of the scalar route; OFF is even, so ties still go to the even integer).
// The low halves of the sums' bits (Cb's are 0) of weights k and k + 4 share
// a register.  Symmetric: OFF = 8 and the low half is the stored code
// c + 8 in 1..15 (clamped to 15 as well, which only a NaN weight reaches, so
// that it cannot spill into its neighbours).  Affine: OFF = 2^14, the low
// half is 2^14 + rint(q) and is clamped to [2^14 - z, 2^14 - z + 15], i.e.
// rint(q) + z clamped to 0..15 plus the base 2^14 - z.  Either way each
// half is a base plus its 4-bit code, so the word is sum_j pair_j 16^j minus
// base * 0x11111111 in 32-bit modular arithmetic (linear, and the codes
// themselves do not overlap).
__device__ __forceinline__ uint64_t f32x2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f32x2_unpack(uint64_t r, uint32_t &lo, uint32_t &hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=r"(lo), "=r"(hi) : "l"(r));
}
// RN(RN(w / s) + c) for a pair of weights: rs2 = (RN(1/s), RN(1/s)), ns2 = (-s, -s),
// c2 = (c, c).  The steps of div_by_recip, in pairs.
__device__ __forceinline__ uint64_t quotient_plus_f32x2(uint64_t w, uint64_t rs2, uint64_t ns2,
                                                        uint64_t c2) {
  uint64_t q0, e, q, t;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(q0) : "l"(w), "l"(rs2));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(e) : "l"(q0), "l"(ns2), "l"(w));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(q) : "l"(e), "l"(rs2), "l"(q0));
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(t) : "l"(q), "l"(c2));
  return t;
}
__device__ __forceinline__ uint32_t mad_u32(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("mad.lo.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

template <bool SYM>
__device__ __forceinline__ uint32_t pack_word_small(const float (&v)[8], float s, float rs,
                                                    int zi) {
  constexpr float C = 12582912.0f;  // 1.5 * 2^23; its low 22 mantissa bits are 0
  constexpr float OFF = SYM ? 8.0f : 16384.0f;
  const uint64_t rs2 = f32x2_pack(rs, rs), ns2 = f32x2_pack(-s, -s);
  const uint64_t c2 = f32x2_pack(C + OFF, C + OFF);
  uint32_t t[8];
#pragma unroll
  for (int p = 0; p < 4; ++p)
    f32x2_unpack(quotient_plus_f32x2(f32x2_pack(v[2 * p], v[2 * p + 1]), rs2, ns2, c2),
                 t[2 * p], t[2 * p + 1]);
  // symmetric: base 0 (the low halves are the stored codes themselves); the
  // upper clamp only acts on a NaN weight, whose code it keeps in its nibble
  const uint32_t b16 = SYM ? 0u : 16384u - static_cast<uint32_t>(zi);
  const uint32_t lo2 = b16 * 0x10001u, hi2 = (b16 + 15u) * 0x10001u;
  uint32_t word = 0u - b16 * 0x11111111u;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint32_t pr;  // low half of t_j, then low half of t_{j+4} (nibble j + 4 = 16 bits up)
    asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(pr) : "r"(t[j]), "r"(t[j + 4]));
    if (!SYM) asm("max.u16x2 %0, %0, %1;" : "+r"(pr) : "r"(lo2));
    asm("min.u16x2 %0, %0, %1;" : "+r"(pr) : "r"(hi2));
    word = mad_u32(pr, 1u << (4 * j), word);
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
  // from the min and max of 0 and the weights (lo <= 0 <= hi)
  __device__ __forceinline__ void set(float lo, float hi) {
    if (SYM) {
      a = fmaxf(-lo, hi);
    } else {
      a = lo;
      b = hi;
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
  // Same values as grid_sym / grid_affine, with the divisions by 7 and 15
  // done from their correctly rounded reciprocals.  small: every finite
  // weight of the segment has |w / s| < 7.5 (symmetric: the fp16 scale is
  // a normal number, or the group is all but zero) or < 23 (affine: the
  // scale did not saturate; then |w| <= b - a <= 15 s32 (1 + 2^-22), a
  // normal fp16 s is at least s32 (1 - 2^-11), a subnormal one at least
  // s32 / 1.5, and a zero one is replaced by 1 for weights below
  // 15 * 2^-24), so pack_word_small gives the same codes.
  __device__ __forceinline__ GridParams grid(bool &small) const {
    GridParams g;
    float s32 = SYM ? div_by_recip(a, 7.0f, 1.0f / 7.0f)
                    : div_by_recip(__fsub_rn(b, a), 15.0f, 1.0f / 15.0f);
    small = s32 <= 65504.0f;
    __half h = __float2half_rn(fminf(s32, 65504.0f));
    const bool degenerate = __half2float(h) == 0.0f;
    if (degenerate) h = __float2half_rn(1.0f);
    g.s = __half2float(h);
    g.s_bits = __half_as_ushort(h);
    if (SYM) {
      // a normal fp16 scale is within 2^-11 of s32; a group whose s32 rounds
      // to 0 in fp16 has |w| < 7 * 2^-25 and uses s = 1
      small = small && ((g.s_bits & 0x7C00u) != 0 || degenerate);
      g.z = 0.0f;
      g.z_bits = 0;
    } else {
      float z = rintf(div_by_recip(-a, g.s, __frcp_rn(g.s)));
      z = fminf(fmaxf(z, 0.0f), 15.0f);
      if (degenerate) z = 0.0f;
      g.z = __fadd_rn(z, 0.0f);
      g.z_bits = __half_as_ushort(__float2half_rn(g.z));
    }
    return g;
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
    Raw8<T> raw[UNROLL][WPL];
    int64_t seg[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      seg[u] = base + u * SPW + lane / TEAM;
      const bool act = seg[u] < total;
      const T *src = W + (act ? seg[u] : 0) * seg_words * 8;
#pragma unroll
      for (int k = 0; k < WPL; ++k) {
        const int64_t w = tl + static_cast<int64_t>(k) * TEAM;
        if (act && w < seg_words) raw[u][k].load(src + w * 8);
        else raw[u][k].zero();  // zeros never change the statistic
      }
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      MinMax<T> mm;
#pragma unroll
      for (int k = 0; k < WPL; ++k) mm.add(raw[u][k]);
      float lo, hi;
      mm.get(lo, hi);
      SegStat<SYM> st;
      st.set(lo, hi);
      st.reduce(TEAM);
      if (seg[u] >= total) continue;
      bool small;
      const GridParams g = st.grid(small);
      const float rs = __frcp_rn(g.s);
      const int zi = static_cast<int>(g.z);
      if (tl == 0) {
        scales[seg[u]] = g.s_bits;
        if (zeros) zeros[seg[u]] = SYM ? 0 : g.z_bits;
      }
      uint32_t *dst = q + seg[u] * seg_words;
#pragma unroll
      for (int k = 0; k < WPL; ++k) {
        const int64_t w = tl + static_cast<int64_t>(k) * TEAM;
        if (w < seg_words) {
          float v[8];
          raw[u][k].get(v);
          dst[w] = small ? pack_word_small<SYM>(v, g.s, rs, zi) : pack_word<SYM>(v, g, rs);
        }
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
    bool small;
    const GridParams g = st.grid(small);
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

// ---------------------------------------------------------------- per-tensor
// One scale (and zero) for the whole matrix ("GPT-2 Quantization
// Reconstruction Error", "Possible extensions": per-tensor, a single global
// scale), stored once per row so that the output has the per-channel
// layout.  Statistic of all weights (block partials, then one block), the
// parameters, then the codes.
template <bool SYM>
__device__ __forceinline__ void block_combine(SegStat<SYM> &st, float *sa, float *sb) {
  st.reduce(32);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) {
    sa[warp] = st.a;
    sb[warp] = st.b;
  }
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    st.a = lane < nw ? sa[lane] : 0.0f;
    st.b = lane < nw ? sb[lane] : 0.0f;
    st.reduce(32);
  }
}

template <typename T, bool SYM>
__global__ void __launch_bounds__(256) tensor_stat_kernel(const T *__restrict__ W, int64_t words,
                                                          float *__restrict__ part) {
  __shared__ float sa[8], sb[8];
  SegStat<SYM> st;
  for (int64_t w = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; w < words;
       w += static_cast<int64_t>(gridDim.x) * 256) {
    float v[8];
    Vec8<T>::load(W + w * 8, v);
#pragma unroll
    for (int e = 0; e < 8; ++e) st.add(v[e]);
  }
  block_combine<SYM>(st, sa, sb);
  if (threadIdx.x == 0) {
    part[2 * blockIdx.x] = st.a;
    part[2 * blockIdx.x + 1] = st.b;
  }
}

// part: n_part (a, b) pairs, or W itself (n_part == 0: a small tensor is
// reduced here directly).
template <typename T, bool SYM, int BITS = 4>
__global__ void __launch_bounds__(256) tensor_params_kernel(const float *__restrict__ part,
                                                            int n_part, const T *__restrict__ W,
                                                            int64_t words, int64_t d_out,
                                                            uint16_t *__restrict__ scales,
                                                            uint16_t *__restrict__ zeros) {
  __shared__ float sa[8], sb[8];
  __shared__ uint16_t ps, pz;
  SegStat<SYM> st;
  if (n_part > 0) {
    for (int i = threadIdx.x; i < n_part; i += 256) {
      if (SYM) {
        st.a = fmaxf(st.a, part[2 * i]);
      } else {
        st.a = fminf(st.a, part[2 * i]);
        st.b = fmaxf(st.b, part[2 * i + 1]);
      }
    }
  } else {
    for (int64_t w = threadIdx.x; w < words; w += 256) {
      float v[8];
      Vec8<T>::load(W + w * 8, v);
#pragma unroll
      for (int e = 0; e < 8; ++e) st.add(v[e]);
    }
  }
  block_combine<SYM>(st, sa, sb);
  if (threadIdx.x == 0) {
    bool small;
    GridParams g;
    if constexpr (BITS == 4)
      g = st.grid(small);
    else
      g = SYM ? grid_sym_b<BITS>(st.a) : grid_affine_b<BITS>(st.a, st.b);
    ps = g.s_bits;
    pz = SYM ? 0 : g.z_bits;
  }
  __syncthreads();
  for (int64_t r = threadIdx.x; r < d_out; r += 256) {
    scales[r] = ps;
    if (zeros) zeros[r] = pz;
  }
}

template <typename T, bool SYM>
__global__ void __launch_bounds__(256) tensor_pack_kernel(const T *__restrict__ W, int64_t words,
                                                          const uint16_t *__restrict__ scales,
                                                          const uint16_t *__restrict__ zeros,
                                                          uint32_t *__restrict__ q) {
  GridParams g{};
  g.s = __half2float(__ushort_as_half(scales[0]));
  g.z = SYM ? 0.0f : __half2float(__ushort_as_half(zeros[0]));
  const float rs = __frcp_rn(g.s);
  for (int64_t w = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; w < words;
       w += static_cast<int64_t>(gridDim.x) * 256) {
    float v[8];
    Vec8<T>::load(W + w * 8, v);
    q[w] = pack_word<SYM>(v, g, rs);
  }
}

// ---------------------------------------------------------------- other widths
// Codes of BITS != 4 bits: a row is one little-endian bit stream along d_in
// (column k at bits BITS k ..), so 32 consecutive columns make BITS whole
// words.  One warp per segment (row, group), lanes over 32-column chunks:
// a first pass for the statistic, a second (from L1 / L2) for the codes.
// With params_given the scale (and zero) of each row are read instead
// (per-tensor: one parameter set, stored per row).
template <int BITS, int K = 0>
__device__ __forceinline__ void pack_run(const float (&v)[32], const GridParams &g, float rs,
                                         bool sym, uint32_t (&words)[BITS]) {
  if constexpr (K < 32) {
    uint32_t stored;
    grid_code_b<BITS>(v[K], g, rs, sym, stored);
    put_code<BITS, K>(words, stored);
    pack_run<BITS, K + 1>(v, g, rs, sym, words);
  }
}

template <typename T>
__device__ __forceinline__ void load32(const T *p, float (&v)[32]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float t[8];
    Vec8<T>::load(p + 8 * i, t);
#pragma unroll
    for (int e = 0; e < 8; ++e) v[8 * i + e] = t[e];
  }
}

template <typename T, int BITS, bool SYM>
__global__ void __launch_bounds__(256) rtn_bits_kernel(const T *__restrict__ W, int64_t d_out,
                                                       int64_t d_in, int64_t seg_len,
                                                       uint32_t *__restrict__ q,
                                                       uint16_t *__restrict__ scales,
                                                       uint16_t *__restrict__ zeros,
                                                       int params_given) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int64_t n_groups = d_in / seg_len, total = d_out * n_groups, chunks = seg_len / 32;
  const int64_t row_words = d_in / 32 * BITS;
  for (int64_t seg = warp; seg < total; seg += n_warps) {
    const int64_t row = seg / n_groups, gi = seg - row * n_groups;
    const T *src = W + row * d_in + gi * seg_len;
    GridParams g{};
    if (!params_given) {
      SegStat<SYM> st;
      for (int64_t c = lane; c < chunks; c += 32) {
        float v[32];
        load32(src + c * 32, v);
#pragma unroll
        for (int e = 0; e < 32; ++e) st.add(v[e]);
      }
      st.reduce(32);
      g = SYM ? grid_sym_b<BITS>(st.a) : grid_affine_b<BITS>(st.a, st.b);
      if (lane == 0) {
        scales[seg] = g.s_bits;
        if (zeros) zeros[seg] = SYM ? 0 : g.z_bits;
      }
    } else {
      g.s = __half2float(__ushort_as_half(scales[seg]));
      g.z = SYM ? 0.0f : __half2float(__ushort_as_half(zeros[seg]));
    }
    const float rs = __frcp_rn(g.s);
    uint32_t *dst = q + row * row_words + gi * (seg_len / 32) * BITS;
    for (int64_t c = lane; c < chunks; c += 32) {
      float v[32];
      load32(src + c * 32, v);
      uint32_t words[BITS];
#pragma unroll
      for (int i = 0; i < BITS; ++i) words[i] = 0u;
      pack_run<BITS>(v, g, rs, SYM, words);
#pragma unroll
      for (int i = 0; i < BITS; ++i) dst[c * BITS + i] = words[i];
    }
  }
}

template <typename T, int BITS>
gq_status launch_bits(const void *W, int64_t d_out, int64_t d_in, int group_size, int sym,
                      uint32_t *q, uint16_t *sc, uint16_t *z, cudaStream_t st) {
  const T *w = static_cast<const T *>(W);
  int params_given = 0;
  int64_t seg_len = group_size <= 0 ? d_in : group_size;
  if (group_size == 0) {  // per tensor: one parameter set (from block partials), then the codes
    const int64_t words = d_out * d_in / 8;
    const int64_t cap = static_cast<int64_t>(num_sms()) * 4;
    int64_t nb = (words + 255) / 256;
    if (nb > cap) nb = cap;
    if (nb > d_out * d_in * BITS / 32 / 2) nb = d_out * d_in * BITS / 32 / 2;
    float *part = reinterpret_cast<float *>(q);  // the packed output as scratch
    if (words <= 8192 || nb < 2) {
      if (sym) tensor_params_kernel<T, true, BITS><<<1, 256, 0, st>>>(nullptr, 0, w, words, d_out, sc, z);
      else tensor_params_kernel<T, false, BITS><<<1, 256, 0, st>>>(nullptr, 0, w, words, d_out, sc, z);
      count_launch();
    } else {
      if (sym) {
        tensor_stat_kernel<T, true><<<static_cast<unsigned>(nb), 256, 0, st>>>(w, words, part);
        tensor_params_kernel<T, true, BITS><<<1, 256, 0, st>>>(part, static_cast<int>(nb), w, words, d_out, sc, z);
      } else {
        tensor_stat_kernel<T, false><<<static_cast<unsigned>(nb), 256, 0, st>>>(w, words, part);
        tensor_params_kernel<T, false, BITS><<<1, 256, 0, st>>>(part, static_cast<int>(nb), w, words, d_out, sc, z);
      }
      count_launch(2);
    }
    params_given = 1;
  }
  const int64_t total = d_out * (d_in / seg_len);
  int64_t blocks = (total + 7) / 8;
  const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
  if (blocks > cap) blocks = cap;
  if (sym)
    rtn_bits_kernel<T, BITS, true><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        w, d_out, d_in, seg_len, q, sc, z, params_given);
  else
    rtn_bits_kernel<T, BITS, false><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        w, d_out, d_in, seg_len, q, sc, z, params_given);
  count_launch();
  return check_launch("rtn_quantize_pack");
}

template <typename T>
gq_status launch_typed_bits(const void *W, int64_t d_out, int64_t d_in, int group_size,
                            int sym, int bits, uint32_t *q, uint16_t *sc, uint16_t *z,
                            cudaStream_t st) {
  switch (bits) {
    case 2: return launch_bits<T, 2>(W, d_out, d_in, group_size, sym, q, sc, z, st);
    case 3: return launch_bits<T, 3>(W, d_out, d_in, group_size, sym, q, sc, z, st);
    case 8: return launch_bits<T, 8>(W, d_out, d_in, group_size, sym, q, sc, z, st);
  }
  return fail(GQ_ERR_ARG, "bits must be 2, 3, 4 or 8");
}

template <typename T, bool SYM>
void launch_tensor_typed(const T *W, int64_t d_out, int64_t d_in, uint32_t *q, uint16_t *sc,
                         uint16_t *z, float *scratch, int64_t scratch_floats, cudaStream_t st) {
  const int64_t words = d_out * d_in / 8;
  const int64_t cap = static_cast<int64_t>(num_sms()) * 4;
  int64_t nb = (words + 255) / 256;
  if (nb > cap) nb = cap;
  if (nb > scratch_floats / 2) nb = scratch_floats / 2;
  if (words <= 8192 || nb < 2) {  // small: one block reads the tensor itself
    tensor_params_kernel<T, SYM><<<1, 256, 0, st>>>(nullptr, 0, W, words, d_out, sc, z);
    count_launch();
  } else {
    tensor_stat_kernel<T, SYM><<<static_cast<unsigned>(nb), 256, 0, st>>>(W, words, scratch);
    tensor_params_kernel<T, SYM><<<1, 256, 0, st>>>(scratch, static_cast<int>(nb), W, words,
                                                    d_out, sc, z);
    count_launch(2);
  }
  int64_t gp = (words + 255) / 256;
  const int64_t gcap = static_cast<int64_t>(num_sms()) * 8;
  if (gp > gcap) gp = gcap;
  tensor_pack_kernel<T, SYM><<<static_cast<unsigned>(gp), 256, 0, st>>>(W, words, sc, z, q);
  count_launch();
}

template <typename T, int TEAM, int WPL, int UNROLL>
void launch_reg(const void *W, int64_t d_out, int64_t seg_words, int64_t n_groups, int sym,
                uint32_t *q, uint16_t *sc, uint16_t *z, cudaStream_t st) {
  const int64_t total = d_out * n_groups;
  const int64_t per_block = (256 / 32) * (32 / TEAM) * UNROLL;
  int64_t blocks = (total + per_block - 1) / per_block;
  // 16-bit weights: up to one segment group per warp on the largest layers,
  // so that the block scheduler balances the tail (a grid-stride of 2-3
  // rounds per warp left the last round part-empty: 8192 x 28672 fp16
  // 104 -> 100 us); fp32 rows (lm_head) run better on a capped grid
  const int64_t cap = static_cast<int64_t>(num_sms()) * (sizeof(T) == 2 ? 64 : 8);
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

// Team size and words per lane: as many words per lane as a small register
// budget allows (4 for 16-bit weights, 2 for fp32), so that a warp quantises
// several groups at once and the per-group work is amortised.
template <typename T>
gq_status launch_typed(const void *W, int64_t d_out, int64_t d_in, int group_size, int sym,
                       uint32_t *q, uint16_t *sc, uint16_t *z, cudaStream_t st) {
  if (group_size == 0) {  // per-tensor; the packed output is the block partials' scratch
    const T *w = static_cast<const T *>(W);
    const int64_t scratch = d_out * d_in / 8;
    float *part = reinterpret_cast<float *>(q);
    if (sym)
      launch_tensor_typed<T, true>(w, d_out, d_in, q, sc, z, part, scratch, st);
    else
      launch_tensor_typed<T, false>(w, d_out, d_in, q, sc, z, part, scratch, st);
    return check_launch("rtn per-tensor");
  }
  const int64_t seg_len = group_size == -1 ? d_in : group_size;
  const int64_t n_groups = d_in / seg_len;
  const int64_t words = seg_len / 8;
  constexpr int WL = sizeof(T) == 2 ? 4 : 2;  // target words per lane
#define GQ_R(TEAM, WPL) launch_reg<T, TEAM, WPL, 2>(W, d_out, words, n_groups, sym, q, sc, z, st)
  if (words <= 1) GQ_R(1, 1);
  else if (words <= 2) GQ_R(1, 2);
  else if (words <= WL) GQ_R(1, WL);
  else if (words <= 2 * WL) GQ_R(2, WL);
  else if (words <= 4 * WL) GQ_R(4, WL);
  else if (words <= 8 * WL) GQ_R(8, WL);
  else if (words <= 16 * WL) GQ_R(16, WL);
  else if (words <= 32 * WL) GQ_R(32, WL);
  else if (words <= 128) GQ_R(32, 4);
  else if (words <= 256) GQ_R(32, 8);
#undef GQ_R
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

// Per-tensor grid parameters of an fp32 matrix (the GPTQ working copy),
// written once per row; scratch holds the block partials.
template <int BITS>
void tensor_params_f32_bits(const float *part, int n_part, const float *W, int64_t words,
                            int64_t d_out, int sym, uint16_t *scales, uint16_t *zeros,
                            cudaStream_t st) {
  if (sym)
    tensor_params_kernel<float, true, BITS><<<1, 256, 0, st>>>(part, n_part, W, words, d_out, scales, zeros);
  else
    tensor_params_kernel<float, false, BITS><<<1, 256, 0, st>>>(part, n_part, W, words, d_out, scales, zeros);
}

gq_status launch_tensor_params_f32(const float *W, int64_t d_out, int64_t d_in, int sym,
                                   uint16_t *scales, uint16_t *zeros, float *scratch,
                                   int64_t scratch_floats, cudaStream_t st, int bits) {
  const int64_t words = d_out * d_in / 8;
  const int64_t cap = static_cast<int64_t>(num_sms()) * 4;
  int64_t nb = (words + 255) / 256;
  if (nb > cap) nb = cap;
  if (nb > scratch_floats / 2) nb = scratch_floats / 2;
  const bool small = words <= 8192 || nb < 2;
  if (!small) {
    if (sym)
      tensor_stat_kernel<float, true><<<static_cast<unsigned>(nb), 256, 0, st>>>(W, words, scratch);
    else
      tensor_stat_kernel<float, false><<<static_cast<unsigned>(nb), 256, 0, st>>>(W, words, scratch);
    count_launch();
  }
  const int n_part = small ? 0 : static_cast<int>(nb);
  switch (bits) {
    case 2: tensor_params_f32_bits<2>(scratch, n_part, W, words, d_out, sym, scales, zeros, st); break;
    case 3: tensor_params_f32_bits<3>(scratch, n_part, W, words, d_out, sym, scales, zeros, st); break;
    case 8: tensor_params_f32_bits<8>(scratch, n_part, W, words, d_out, sym, scales, zeros, st); break;
    default: tensor_params_f32_bits<4>(scratch, n_part, W, words, d_out, sym, scales, zeros, st);
  }
  count_launch();
  return check_launch("per-tensor parameters");
}

gq_status launch_rtn(const void *W, gq_dtype dt, int64_t d_out, int64_t d_in, int group_size,
                     int sym, uint32_t *qpacked, uint16_t *scales, uint16_t *zeros,
                     cudaStream_t st, int bits) {
  int wb = 0;
  gq_status s = GQ_OK;
  const int slot = timer_begin(GQ_KERNEL_RTN, st);
  const bool b4 = bits == 4;
  switch (dt) {
    case GQ_F32:
      wb = 4;
      s = b4 ? launch_typed<float>(W, d_out, d_in, group_size, sym, qpacked, scales, zeros, st)
             : launch_typed_bits<float>(W, d_out, d_in, group_size, sym, bits, qpacked, scales,
                                        zeros, st);
      break;
    case GQ_F16:
      wb = 2;
      s = b4 ? launch_typed<__half>(W, d_out, d_in, group_size, sym, qpacked, scales, zeros, st)
             : launch_typed_bits<__half>(W, d_out, d_in, group_size, sym, bits, qpacked, scales,
                                         zeros, st);
      break;
    case GQ_BF16:
      wb = 2;
      s = b4 ? launch_typed<__nv_bfloat16>(W, d_out, d_in, group_size, sym, qpacked, scales,
                                           zeros, st)
             : launch_typed_bits<__nv_bfloat16>(W, d_out, d_in, group_size, sym, bits, qpacked,
                                                scales, zeros, st);
      break;
    default:
      s = fail(GQ_ERR_DTYPE, "unknown dtype");
  }
  // W read; codes (bits / 8 bytes per weight), fp16 scales (and zeros) written
  const double n_groups = group_size <= 0 ? 1.0 : static_cast<double>(d_in / group_size);
  timer_end(slot, st,
            static_cast<double>(d_out) * d_in * (wb + bits / 8.0) +
                2.0 * d_out * n_groups * (sym ? 1 : 2));
  return s;
}

}  // namespace gq
