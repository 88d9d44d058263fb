// Damping, dead columns, act-order, and U with H^-1 = U^T U, all in fp32.
//
// "GPTQ: Post-Training INT4" -- "Running GPTQ with AutoGPTQ": damp_percent
// (H += damp * mean diag H) and desc_act (columns by descending diag H);
// "The GPTQ Algorithm": Cholesky of H, then its inverse; "Model
// Quantization Mechanics", section 2.1: GPTQ uses a Cholesky factor of the
// inverse Hessian.
//
// Instead of inverting H and factoring the inverse, this file uses the
// identity U = J L^-1 J, where J reverses the index order and L is the
// lower Cholesky factor of A = J H J: U is upper triangular with positive
// diagonal and U^T U = J L^-T L^-1 J = J A^-1 J = H^-1, so by uniqueness it
// is the upper Cholesky factor of H^-1.  Two d^3/3 steps instead of three.
//
// Memory: A is gathered (reversed, act-order permuted) into the U buffer
// and factored in place, except that each diagonal block's factor (then its
// inverse) goes to a [NB][NB] slot of the workspace; X = L^-1 is built in
// the H buffer (the caller's H is scratch); the last kernel writes
// U = J X J back into the U buffer.
// Blocked right-looking algorithms with 128-wide panels grouped in
// super-panels (two levels, above a width); each CTA of the panel kernel
// factors the diagonal block in shared memory and solves its panel rows
// against it, one CTA inverts the block for the inverse's chain, and the
// trailing updates and the inverse's block steps are fp32 GEMMs on the
// tensor cores (3 x TF32 split, gemm_tc.cu).
#include <cfloat>
#include <cmath>
#include <climits>
#include <map>
#include <mutex>
#include <string>

#include "gq_device.cuh"
#include "gq_internal.h"

namespace gq {
namespace {

constexpr int NB = 128;  // panel width

struct CholWs {
  int *status;    // [0] device status, [1] info (first bad pivot, INT_MAX if none)
  double *mean;   // scratch for the damping mean
  float *key;     // [d] diag after damping (act-order keys)
  float *linv;    // [n_panels][NB][NB] inverse of each diagonal block of L
};

CholWs carve(void *ws, int64_t d) {
  uint8_t *p = static_cast<uint8_t *>(ws);
  CholWs w;
  w.status = reinterpret_cast<int *>(p);
  w.mean = reinterpret_cast<double *>(p + 64);
  size_t off = kWsHeader;
  w.key = reinterpret_cast<float *>(p + off);
  off += round_up(static_cast<size_t>(d) * sizeof(float), 256);
  w.linv = reinterpret_cast<float *>(p + off);
  return w;
}

// ---------------------------------------------------------------- damping
// One block: dead columns (H_jj == 0 -> 1), the mean of the diagonal in
// fp64 (fixed reduction order), then H_jj += damp * mean.
__global__ void __launch_bounds__(1024) damp_kernel(float *__restrict__ H, int64_t d, float damp,
                                                    uint8_t *__restrict__ dead_out,
                                                    float *__restrict__ key, int *status) {
  __shared__ double red[1024];
  double s = 0.0;
  for (int64_t j = threadIdx.x; j < d; j += blockDim.x) {
    float hjj = H[j * d + j];
    const bool dead = hjj == 0.0f;
    if (dead) hjj = 1.0f;
    if (dead_out) dead_out[j] = dead ? 1 : 0;
    s += static_cast<double>(hjj);
  }
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = 512; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  const double lam = static_cast<double>(damp) * (red[0] / static_cast<double>(d));
  for (int64_t j = threadIdx.x; j < d; j += blockDim.x) {
    float hjj = H[j * d + j];
    if (hjj == 0.0f) hjj = 1.0f;
    const float v = static_cast<float>(static_cast<double>(hjj) + lam);
    H[j * d + j] = v;
    key[j] = v;
  }
  if (threadIdx.x == 0) {
    status[0] = 0;
    status[1] = INT_MAX;
  }
}

// ---------------------------------------------------------------- act-order
// perm[rank(i)] = i with rank(i) = #{j : key_j > key_i} + #{j < i : key_j == key_i},
// i.e. a stable sort by descending key.
__global__ void __launch_bounds__(256) rank_kernel(const float *__restrict__ key, int64_t d,
                                                   int32_t *__restrict__ perm) {
  __shared__ float tile[256];
  // NaN keys count as -FLT_MAX so that the ranks always form a permutation
  const int64_t i = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  float ki = i < d ? key[i] : 0.0f;
  if (!(ki == ki)) ki = -FLT_MAX;
  int64_t rank = 0;
  for (int64_t j0 = 0; j0 < d; j0 += 256) {
    __syncthreads();
    float kt = j0 + threadIdx.x < d ? key[j0 + threadIdx.x] : -FLT_MAX;
    tile[threadIdx.x] = kt == kt ? kt : -FLT_MAX;
    __syncthreads();
    const int n = static_cast<int>(d - j0 < 256 ? d - j0 : 256);
    for (int t = 0; t < n; ++t) {
      const float kj = tile[t];
      rank += (kj > ki) || (kj == ki && j0 + t < i);
    }
  }
  if (i < d) perm[rank] = static_cast<int32_t>(i);
}

// A[a][b] = H[p(d-1-a)][p(d-1-b)] (lower triangle and diagonal only).
__global__ void __launch_bounds__(256) gather_reversed_kernel(const float *__restrict__ H,
                                                              int64_t d,
                                                              const int32_t *__restrict__ perm,
                                                              float *__restrict__ A) {
  // one warp per row; without a permutation a row of A is a row of H read
  // backwards, one aligned float4 per lane (d is a multiple of 4); the
  // float4 that holds the diagonal may also write up to three elements
  // right of it, whose values are the symmetric matrix's own (the strict
  // upper part is never read)
  const int lane = threadIdx.x & 31;
  const int64_t nw = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t a = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       a < d; a += nw) {
    const int64_t sa = d - 1 - a;
    if (perm) {
      const int64_t ra = perm[sa];
      for (int64_t b = lane; b <= a; b += 32) A[a * d + b] = H[ra * d + perm[d - 1 - b]];
    } else {
      const float *hr = H + sa * d;
      for (int64_t b = 4 * lane; b <= a; b += 128) {
        const float4 v = *reinterpret_cast<const float4 *>(hr + (d - 4 - b));
        *reinterpret_cast<float4 *>(A + a * d + b) = make_float4(v.w, v.z, v.y, v.x);
      }
    }
  }
}

// ---------------------------------------------------------------- panel factor
constexpr int SP = NB + 1;  // padded row stride in shared memory (bank-conflict free columns)
constexpr int TT = 2 * NB + 4;  // row stride of the transposed sub-panel (float4 aligned)

// Factor the 32 x 32 piece at (c0, c0) of S in place with one warp (lane =
// row, the row in registers); rd gets the reciprocals of its diagonal.
// Column J: the pivot is broadcast by a shuffle, the column of L goes
// through colbuf (32 floats, read back as broadcast float4s) to every
// row's update.  The column loop runs over J = 8 J8 + E with E unrolled
// (chol32_step<E>), so a column's register is picked among 4 candidates
// and the update needs no per-element test; the 8-step body keeps the code
// small (a fully unrolled factor is large enough that its instruction
// fetches dominate on an SM that has not run it recently).  The pivot step
// is the panel's serial chain -- the other warps wait for it -- so its
// latency is what counts.  Entries right of a lane's diagonal are updated
// too; they are never read; entries left of column J see l_k = 0.  A pivot
// that is not positive and finite is replaced by 1; returns the first such
// column (32 if none).
template <int E>
__device__ __forceinline__ void chol32_step(float (&w)[32], int J8, float *colbuf, int lane,
                                            float &my_rd, int &bad) {
  const int J = 8 * J8 + E;
  const float a0 = (J8 & 1) ? w[8 + E] : w[E];
  const float a1 = (J8 & 1) ? w[24 + E] : w[16 + E];
  const float wj = (J8 & 2) ? a1 : a0;  // w[J]
  float piv = __shfl_sync(0xffffffffu, wj, J);
  const bool ill = !(piv > 0.0f) || !(piv < FLT_MAX);
  bad = (ill && bad == 32) ? J : bad;
  piv = ill ? 1.0f : piv;
  // 1 / sqrt(piv): hardware estimate plus one Newton step r (3 - piv r^2) / 2
  float rj = rsqrtf(piv);
  rj = rj * fmaf(-0.5f * piv, rj * rj, 1.5f);
  const float lij = lane > J ? wj * rj : (lane == J ? piv * rj : 0.0f);
  my_rd = lane == J ? rj : my_rd;
  colbuf[lane] = lij;
  __syncwarp();
#pragma unroll
  for (int k4 = 0; k4 < 8; ++k4) {
    const float4 l4 = reinterpret_cast<const float4 *>(colbuf)[k4];
    const float lk[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int k = 4 * k4 + q;
      const float u = fmaf(-lij, lk[q], w[k]);
      if (k % 8 == E) w[k] = (k / 8 == J8) ? lij : u;
      else w[k] = u;
    }
  }
  __syncwarp();
}

__device__ __forceinline__ int chol32_piece(float *S, float *rd, float *colbuf, int c0,
                                            int lane) {
  float w[32];
#pragma unroll
  for (int k = 0; k < 32; ++k) w[k] = (k <= lane) ? S[(c0 + lane) * SP + c0 + k] : 0.0f;
  float my_rd = 1.0f;
  int bad = 32;
#pragma unroll 1
  for (int J8 = 0; J8 < 4; ++J8) {
    chol32_step<0>(w, J8, colbuf, lane, my_rd, bad);
    chol32_step<1>(w, J8, colbuf, lane, my_rd, bad);
    chol32_step<2>(w, J8, colbuf, lane, my_rd, bad);
    chol32_step<3>(w, J8, colbuf, lane, my_rd, bad);
    chol32_step<4>(w, J8, colbuf, lane, my_rd, bad);
    chol32_step<5>(w, J8, colbuf, lane, my_rd, bad);
    chol32_step<6>(w, J8, colbuf, lane, my_rd, bad);
    chol32_step<7>(w, J8, colbuf, lane, my_rd, bad);
  }
#pragma unroll
  for (int k = 0; k < 32; ++k)
    if (k <= lane) S[(c0 + lane) * SP + c0 + k] = w[k];
  rd[c0 + lane] = my_rd;
  return bad;
}

// One 8 x 8 register tile of the rank-32 update M[i][k] -= sum_j L[i][j] L[k][j]
// from the transposed sub-panel T (T[j][q] = L of source row q, column j):
// target rows are sources qi .. qi+7, target columns sources qk .. qk+7.
__device__ __forceinline__ void update_tile8(const float *__restrict__ T, int qi, int qk,
                                             float *dst, int dst_ld, bool tri, int i0, int k0) {
  float acc[8][8];
#pragma unroll
  for (int x = 0; x < 8; ++x)
#pragma unroll
    for (int y = 0; y < 8; ++y) acc[x][y] = 0.0f;
#pragma unroll 4
  for (int j = 0; j < 32; ++j) {
    const float4 a0 = *reinterpret_cast<const float4 *>(T + j * TT + qi);
    const float4 a1 = *reinterpret_cast<const float4 *>(T + j * TT + qi + 4);
    const float4 b0 = *reinterpret_cast<const float4 *>(T + j * TT + qk);
    const float4 b1 = *reinterpret_cast<const float4 *>(T + j * TT + qk + 4);
    const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
    const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
    for (int x = 0; x < 8; ++x)
#pragma unroll
      for (int y = 0; y < 8; ++y) acc[x][y] = fmaf(av[x], bv[y], acc[x][y]);
  }
#pragma unroll
  for (int x = 0; x < 8; ++x)
#pragma unroll
    for (int y = 0; y < 8; ++y)
      if (!tri || k0 + y <= i0 + x) dst[(i0 + x) * dst_ld + k0 + y] -= acc[x][y];
}

// ---------------------------------------------------------------- panel
// One 128-column panel of the blocked Cholesky: the 128 x 128 diagonal
// block factored in shared memory, and the rows below it solved against
// that factor, in one launch.  CTA t owns the panel rows k0 + 128 t .. +127;
// every CTA factors the diagonal block itself, so the panel solve needs
// neither a separate launch nor the block's inverse.  CTA 0 writes the
// factor to lpp ([NB][NB], identity padded), not back into A: with more
// CTAs than fit on the GPU at once, later CTAs still read the unfactored
// block from A after CTA 0 has finished.
// The 128 columns go in sub-panels of 32 (c0 = 0, 32, 64, 96):
//   (a) one warp factors the 32 x 32 diagonal piece, a row per lane in
//       registers (pivot and column broadcast by shuffles);
//   (b) one thread per row below the piece (in the diagonal block and in
//       the CTA's own rows) solves x L^T = a with the row in registers and
//       also stores it transposed (T[j][q], q < 128: block row, q >= 128:
//       own row q - 128), so that the update reads whole float4 runs;
//   (c) the rank-32 update of the remaining columns in 8 x 8 register
//       tiles, in two parts: first the next sub-panel's 32 columns (all
//       warps), then the rest (warps 1-7) while warp 0 already factors the
//       next diagonal piece, which only needs the first part.
constexpr size_t PANEL_SMEM = (2 * NB * SP + NB + 32 * TT + 32) * sizeof(float);

__global__ void __launch_bounds__(256) potrf_trsm_kernel(float *__restrict__ A, int64_t d,
                                                         int64_t k0, int nb,
                                                         float *__restrict__ lpp, int *status,
                                                         int n_rb) {
  extern __shared__ float sm[];
  float *S = sm;            // [NB][SP]  the diagonal block, then its factor L (lower)
  float *P = S + NB * SP;   // [NB][SP]  this CTA's panel rows (CTA 0: unused)
  float *rd = P + NB * SP;  // [NB]      1 / L_jj
  float *T = rd + NB;       // [32][TT]  the current sub-panel, transposed
  float *colbuf = T + 32 * TT;  // [32]    one column of a 32 x 32 piece
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool own = blockIdx.x > 0;
  const int64_t row0 = k0 + static_cast<int64_t>(blockIdx.x) * NB;
  const int prows = own ? static_cast<int>(d - row0 < NB ? d - row0 : NB) : 0;

  {
    float4 v[NB * NB / 4 / 256];
#pragma unroll
    for (int u = 0; u < NB * NB / 4 / 256; ++u) {
      const int idx = tid + 256 * u;
      const int r = idx >> 5, c = (idx & 31) * 4;
      v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r < nb && c < nb && c <= r)
        v[u] = *reinterpret_cast<const float4 *>(A + (k0 + r) * d + k0 + c);
    }
#pragma unroll
    for (int u = 0; u < NB * NB / 4 / 256; ++u) {
      const int idx = tid + 256 * u;
      const int r = idx >> 5, c = (idx & 31) * 4;
      const float e[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int q = 0; q < 4; ++q)
        S[r * SP + c + q] = r < nb ? e[q] : (r == c + q ? 1.0f : 0.0f);  // identity padding
    }
    if (own) {
#pragma unroll
      for (int u = 0; u < NB * NB / 4 / 256; ++u) {
        const int idx = tid + 256 * u;
        const int r = idx >> 5, c = (idx & 31) * 4;
        v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (r < prows && c < nb)
          v[u] = *reinterpret_cast<const float4 *>(A + (row0 + r) * d + k0 + c);
      }
#pragma unroll
      for (int u = 0; u < NB * NB / 4 / 256; ++u) {
        const int idx = tid + 256 * u;
        const int r = idx >> 5, c = (idx & 31) * 4;
        P[r * SP + c] = v[u].x;
        P[r * SP + c + 1] = v[u].y;
        P[r * SP + c + 2] = v[u].z;
        P[r * SP + c + 3] = v[u].w;
      }
    }
  }
  __syncthreads();

  int bad = 32 * 4;  // first bad pivot column of the block (warp 0 lanes), 128 if none
  if (warp == 0) {
    const int b = chol32_piece(S, rd, colbuf, 0, lane);
    bad = b < 32 ? b : bad;
  }
  for (int c0 = 0; c0 < NB; c0 += 32) {
    __syncthreads();  // piece c0 factored; the previous update finished
    // (b) rows below the piece -- in the block, then the CTA's rows:
    //     x = a L_dd^-T, right-looking within the row; stored back and
    //     transposed into T
    const int base = c0 + 32;
    const int below = NB - base;
    const int n_rows = below + (own ? NB : 0);
    for (int i = tid; i < n_rows; i += 256) {
      const bool in_s = i < below;
      float *row = in_s ? S + (base + i) * SP : P + (i - below) * SP;
      const int q = in_s ? base + i : NB + (i - below);
      float a[32];
#pragma unroll
      for (int k = 0; k < 32; ++k) a[k] = row[c0 + k];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float x = a[j] * rd[c0 + j];
        a[j] = x;
#pragma unroll
        for (int k = j + 1; k < 32; ++k) a[k] = fmaf(-x, S[(c0 + k) * SP + c0 + j], a[k]);
      }
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        row[c0 + k] = a[k];
        T[k * TT + q] = a[k];
      }
    }
    __syncthreads();
    if (base >= NB) break;
    // (c) 8 x 8 tiles over the remaining columns k >= base.  Column tile
    //     tk (columns base + 8 tk ..), row tile ti of the block (rows base +
    //     8 ti .., only tk <= ti) or tp of the own rows.
    const int m8 = below / 8;
    const int p8 = own ? NB / 8 : 0;
    // part 1: the next sub-panel's columns (tk < 4), all warps
    {
      const int n_s = 4 * m8 - 6;       // block tiles with tk < 4 and tk <= ti
      const int n_t = n_s + p8 * 4;
      for (int t = tid; t < n_t; t += 256) {
        int qi, tk;
        bool tri;
        float *dst;
        int dld, i0;
        if (t < n_s) {
          // rows ti = 0..3 hold ti + 1 tiles, the rest 4
          int ti, u = t;
          if (u < 10) {
            ti = u < 1 ? 0 : (u < 3 ? 1 : (u < 6 ? 2 : 3));
            tk = u - ti * (ti + 1) / 2;
          } else {
            ti = 4 + (u - 10) / 4;
            tk = (u - 10) % 4;
          }
          i0 = base + 8 * ti;
          qi = i0;
          dst = S;
          dld = SP;
          tri = ti == tk;
        } else {
          const int u = t - n_s;
          const int tp = u / 4;
          tk = u % 4;
          i0 = 8 * tp;
          qi = NB + i0;
          dst = P;
          dld = SP;
          tri = false;
        }
        update_tile8(T, qi, base + 8 * tk, dst, dld, tri, i0, base + 8 * tk);
      }
    }
    __syncthreads();
    // part 2: columns beyond the next sub-panel (tk >= 4), warps 1-7, while
    //         warp 0 factors the next diagonal piece
    if (warp == 0) {
      const int b = chol32_piece(S, rd, colbuf, base, lane);
      bad = (b < 32 && bad == 128) ? base + b : bad;
    } else if (m8 > 4) {
      const int mr = m8 - 4;                      // column tiles tk = 4 .. m8-1
      const int n_s = mr * (mr + 1) / 2;          // block tiles with 4 <= tk <= ti
      const int n_t = n_s + p8 * mr;
      for (int t = tid - 32; t < n_t; t += 224) {
        int ti, tk;
        if (t < n_s) {
          int r = static_cast<int>((sqrtf(8.0f * t + 1.0f) - 1.0f) * 0.5f);
          while (r * (r + 1) / 2 > t) --r;
          while ((r + 1) * (r + 2) / 2 <= t) ++r;
          ti = 4 + r;
          tk = 4 + (t - r * (r + 1) / 2);
          const int i0 = base + 8 * ti;
          update_tile8(T, i0, base + 8 * tk, S, SP, ti == tk, i0, base + 8 * tk);
        } else {
          const int u = t - n_s;
          const int tp = u / mr;
          tk = 4 + u % mr;
          update_tile8(T, NB + 8 * tp, base + 8 * tk, P, SP, false, 8 * tp, base + 8 * tk);
        }
      }
    }
  }
  if (blockIdx.x == 0 && warp == 0 && lane == 0 && bad < nb)
    atomicMin(&status[1], static_cast<int>(k0 + bad));

  if (!own) {
    for (int e = tid; e < NB * NB; e += 256) {
      const int r = e / NB, c = e % NB;
      lpp[e] = c <= r ? S[r * SP + c] : 0.0f;
    }
  } else {
    for (int e = tid; e < NB * NB / 4; e += 256) {
      const int r = e >> 5, c = (e & 31) * 4;
      if (r < prows && c < nb)
        *reinterpret_cast<float4 *>(A + (row0 + r) * d + k0 + c) =
            make_float4(P[r * SP + c], P[r * SP + c + 1], P[r * SP + c + 2], P[r * SP + c + 3]);
    }
  }

  // Further row blocks (a grid smaller than the panel's n_rb row blocks):
  // the diagonal block's factor stays in S and rd, and each further block
  // of 128 rows is solved against it as the CTA's own rows were above --
  // the same operations in the same order, without factoring the block
  // again.  T's block part is refilled from S for each sub-panel.
  for (int rb = static_cast<int>(blockIdx.x + gridDim.x); rb < n_rb;
       rb += static_cast<int>(gridDim.x)) {
    const int64_t r0 = k0 + static_cast<int64_t>(rb) * NB;
    const int pr = static_cast<int>(d - r0 < NB ? d - r0 : NB);
    __syncthreads();  // the previous rows are written out; P and T are free
    for (int e = tid; e < NB * NB / 4; e += 256) {
      const int r = e >> 5, c = (e & 31) * 4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r < pr && c < nb) v = *reinterpret_cast<const float4 *>(A + (r0 + r) * d + k0 + c);
      P[r * SP + c] = v.x;
      P[r * SP + c + 1] = v.y;
      P[r * SP + c + 2] = v.z;
      P[r * SP + c + 3] = v.w;
    }
    __syncthreads();
    for (int c0 = 0; c0 < NB; c0 += 32) {
      const int base = c0 + 32;
      for (int i = tid; i < NB; i += 256) {
        float *row = P + i * SP;
        float a[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) a[k] = row[c0 + k];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float x = a[j] * rd[c0 + j];
          a[j] = x;
#pragma unroll
          for (int k = j + 1; k < 32; ++k) a[k] = fmaf(-x, S[(c0 + k) * SP + c0 + j], a[k]);
        }
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          row[c0 + k] = a[k];
          T[k * TT + NB + i] = a[k];
        }
      }
      if (base >= NB) break;
      for (int e = tid; e < 32 * (NB - base); e += 256) {
        const int k = e / (NB - base), q = base + e % (NB - base);
        T[k * TT + q] = S[q * SP + c0 + k];
      }
      __syncthreads();
      const int m8 = (NB - base) / 8;
      for (int t = tid; t < (NB / 8) * m8; t += 256) {
        const int tp = t / m8, tk = t % m8;
        update_tile8(T, NB + 8 * tp, base + 8 * tk, P, SP, false, 8 * tp, base + 8 * tk);
      }
      __syncthreads();
    }
    __syncthreads();
    for (int e = tid; e < NB * NB / 4; e += 256) {
      const int r = e >> 5, c = (e & 31) * 4;
      if (r < pr && c < nb)
        *reinterpret_cast<float4 *>(A + (r0 + r) * d + k0 + c) =
            make_float4(P[r * SP + c], P[r * SP + c + 1], P[r * SP + c + 2], P[r * SP + c + 3]);
    }
  }
}

constexpr int TP = 33;      // stride of the 32 x 32 temporaries

// ---------------------------------------------------------------- block inverse
// lp := L_pp^-1, in place, for the factored diagonal block that
// potrf_trsm_kernel left in lp ([NB][NB], lower, identity padded past the
// matrix edge).  Each warp inverts one 32 x 32 diagonal block (a column per
// lane), then X_ij = -X_ii (sum_k L_ik X_kj) fills the blocks below, one
// diagonal band at a time.
constexpr size_t INV_SMEM = (2 * NB * SP + NB + 3 * 32 * TP) * sizeof(float);

__global__ void __launch_bounds__(256) block_inverse_kernel(float *__restrict__ lp) {
  extern __shared__ float sm[];
  float *S = sm;                // [NB][SP]  L (lower)
  float *Li = S + NB * SP;      // [NB][SP]  L^-1 (lower)
  float *rd = Li + NB * SP;     // [NB]
  float *T = rd + NB;           // [3][32][TP]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int e = tid; e < NB * NB / 4; e += 256) {
    const int r = e >> 5, c = (e & 31) * 4;
    const float4 v = *reinterpret_cast<const float4 *>(lp + r * NB + c);
    const float x[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      S[r * SP + c + q] = x[q];
      Li[r * SP + c + q] = 0.0f;
    }
  }
  __syncthreads();
  if (tid < NB) rd[tid] = __frcp_rn(S[tid * SP + tid]);
  __syncthreads();
  if (warp < 4) {
    const int q0 = 32 * warp;
    float v[32];
#pragma unroll
    for (int r = 0; r < 32; ++r) v[r] = (r == lane) ? 1.0f : 0.0f;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const float x = v[j] * rd[q0 + j];
      v[j] = x;
#pragma unroll
      for (int r = j + 1; r < 32; ++r) v[r] = fmaf(-S[(q0 + r) * SP + q0 + j], x, v[r]);
    }
#pragma unroll
    for (int r = 0; r < 32; ++r) Li[(q0 + r) * SP + q0 + lane] = v[r];
  }
  __syncthreads();
  // (each thread: one row r, four consecutive columns)
  for (int lvl = 1; lvl < 4; ++lvl) {
    const int nblk = 4 - lvl;
    for (int e = tid; e < nblk * 256; e += 256) {
      const int b = e >> 8, r = (e >> 3) & 31, c = (e & 7) * 4;
      const int j = b, i = b + lvl;
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
      const float *srow = S + (32 * i + r) * SP;
#pragma unroll 4
      for (int k = 32 * j; k < 32 * i; ++k) {
        const float l = srow[k];
        const float *x = Li + k * SP + 32 * j + c;
        a0 = fmaf(l, x[0], a0);
        a1 = fmaf(l, x[1], a1);
        a2 = fmaf(l, x[2], a2);
        a3 = fmaf(l, x[3], a3);
      }
      float *t = T + (b * 32 + r) * TP + c;
      t[0] = a0; t[1] = a1; t[2] = a2; t[3] = a3;
    }
    __syncthreads();
    for (int e = tid; e < nblk * 256; e += 256) {
      const int b = e >> 8, r = (e >> 3) & 31, c = (e & 7) * 4;
      const int j = b, i = b + lvl;
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
      const float *xrow = Li + (32 * i + r) * SP + 32 * i;
      for (int k = 0; k <= r; ++k) {
        const float xv = xrow[k];
        const float *t = T + (b * 32 + k) * TP + c;
        a0 = fmaf(xv, t[0], a0);
        a1 = fmaf(xv, t[1], a1);
        a2 = fmaf(xv, t[2], a2);
        a3 = fmaf(xv, t[3], a3);
      }
      float *o = Li + (32 * i + r) * SP + 32 * j + c;
      o[0] = -a0; o[1] = -a1; o[2] = -a2; o[3] = -a3;
    }
    __syncthreads();
  }
  __syncthreads();  // every thread has read lp before it is overwritten
  for (int e = tid; e < NB * NB; e += 256) lp[e] = Li[(e / NB) * SP + e % NB];
}

// X := I on the lower triangle and on the whole NB x NB diagonal blocks
// (the right-hand side of L X = I); the rest of the upper part is never read.
// X := I on the lower triangle and on every super-panel's diagonal block
// (the upper part of those blocks is read by the inverse's K = S updates;
// the rest of the upper triangle is never read).
__global__ void __launch_bounds__(256) eye_lower_kernel(float *__restrict__ X, int64_t d,
                                                        int64_t S) {
  // one warp per row, float4 stores (d and S are multiples of 4)
  const int lane = threadIdx.x & 31;
  const int64_t nw = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       r < d; r += nw) {
    int64_t end = (r / S + 1) * S;
    if (end > d) end = d;
    for (int64_t c = 4 * lane; c < end; c += 128) {
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r == c) v.x = 1.0f;
      if (r == c + 1) v.y = 1.0f;
      if (r == c + 2) v.z = 1.0f;
      if (r == c + 3) v.w = 1.0f;
      *reinterpret_cast<float4 *>(X + r * d + c) = v;
    }
  }
}

// U[a][b] = X[d-1-a][d-1-b] for a <= b, 0 below the diagonal: one warp per
// row, a row of X read backwards as aligned float4s.
__global__ void __launch_bounds__(256) reverse_upper_kernel(const float *__restrict__ X,
                                                            int64_t d, float *__restrict__ U) {
  const int lane = threadIdx.x & 31;
  const int64_t nw = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t a = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       a < d; a += nw) {
    const float *xr = X + (d - 1 - a) * d;
    for (int64_t b = 4 * lane; b < d; b += 128) {
      float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
      if (b + 3 >= a) {
        const float4 v = *reinterpret_cast<const float4 *>(xr + (d - 4 - b));
        o = make_float4(b >= a ? v.w : 0.f, b + 1 >= a ? v.z : 0.f, b + 2 >= a ? v.y : 0.f, v.x);
      }
      *reinterpret_cast<float4 *>(U + a * d + b) = o;
    }
  }
}

// The factorisation runs on the reversed matrix: reversed pivot k is column
// d-1-k in processing order.
__global__ void finish_info_kernel(int *status, int64_t d, int32_t *info_dev) {
  const int v = status[1] == INT_MAX ? -1 : static_cast<int>(d - 1 - status[1]);
  status[1] = v;
  if (info_dev) *info_dev = v;
}

}  // namespace

// Super-panel width: NB times the power of two nearest (on a log scale)
// sqrt(d / NB).
#ifndef GQ_CHOL_TWO_LEVEL_MIN_D
#define GQ_CHOL_TWO_LEVEL_MIN_D 4097
#endif
// Super-panel width S: about sqrt(NB d) (a power-of-two multiple of NB);
// below GQ_CHOL_TWO_LEVEL_MIN_D one level (S = d): there the fewer launches
// matter more than the trailing matrix's traffic, which mostly stays in L2
// (the 49-layer GPT-2-small step, widths 768 and 3072: 24.9 -> 23.9 ms).
int64_t chol_super_cols(int64_t d) {
  if (d < GQ_CHOL_TWO_LEVEL_MIN_D) return d;
  const double target = std::sqrt(static_cast<double>(NB) * static_cast<double>(d));
  int64_t S = NB;
  while (static_cast<double>(2 * S) <= target * 1.4142135623730951) S *= 2;
  return S;
}

size_t chol_ws_bytes(int64_t d) {
  const int64_t n_panels = (d + NB - 1) / NB;
  return kWsHeader + round_up(static_cast<size_t>(d) * sizeof(float), 256) +
         static_cast<size_t>(n_panels) * NB * NB * sizeof(float);
}

// A second stream (and two events) per caller stream and device, created on
// first use and kept for the life of the process.  Keyed by the caller's
// stream so that solves issued on different streams keep independent
// inverse chains (one shared helper stream would serialise them).  None is
// created while the caller's stream is being captured into a graph; the
// inverse chain then stays on the caller's stream.
struct AuxStream {
  cudaStream_t s = nullptr;
  cudaEvent_t ev = nullptr, join = nullptr;
};

AuxStream *aux_stream(cudaStream_t caller) {
  static std::mutex mu;
  static std::map<std::pair<int, cudaStream_t>, AuxStream> cache;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_pair(dev, caller);
  auto it = cache.find(key);
  if (it != cache.end()) return &it->second;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(caller, &cap) != cudaSuccess || cap != cudaStreamCaptureStatusNone) {
    cudaGetLastError();
    return nullptr;
  }
  AuxStream a;
  if (cudaStreamCreateWithFlags(&a.s, cudaStreamNonBlocking) != cudaSuccess ||
      cudaEventCreateWithFlags(&a.ev, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&a.join, cudaEventDisableTiming) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return &(cache[key] = a);
}

gq_status launch_damp_chol(float *H, int64_t d, float damp, int act_order, int32_t *perm_out,
                           uint8_t *dead_out, float *U, int32_t *info_dev, void *ws,
                           cudaStream_t st, bool use_aux) {
  CholWs w = carve(ws, d);
  damp_kernel<<<1, 1024, 0, st>>>(H, d, damp, dead_out, w.key, w.status);
  count_launch();
  if (act_order) {
    rank_kernel<<<static_cast<unsigned>((d + 255) / 256), 256, 0, st>>>(w.key, d, perm_out);
    count_launch();
  }
  // row kernels: one warp per row, 8 rows per block
  const int64_t row_blocks = (d + 7) / 8, cap = static_cast<int64_t>(num_sms()) * 16;
  const unsigned gr = static_cast<unsigned>(row_blocks < cap ? row_blocks : cap);
  float *A = U;  // the factorisation lives in the U buffer
  float *X = H;  // L^-1 is built in the H buffer
  gather_reversed_kernel<<<gr, 256, 0, st>>>(H, d, act_order ? perm_out : nullptr, A);
  count_launch();
  {
    const gq_status s = check_launch("damp/gather");
    if (s != GQ_OK) return s;
  }
  cudaFuncSetAttribute(potrf_trsm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       static_cast<int>(PANEL_SMEM));
  cudaFuncSetAttribute(block_inverse_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       static_cast<int>(INV_SMEM));
  const int64_t n_panels = (d + NB - 1) / NB;
  eye_lower_kernel<<<gr, 256, 0, st>>>(X, d, chol_super_cols(d));
  count_launch();
  // The inverse X = L^-1 (blocked forward substitution on the identity) runs
  // as a second chain: its step p needs the panel p of L and step p-1 only,
  // so on a second stream it overlaps the rest of the factorisation.
  cudaStream_t inv_st = st;
  AuxStream *aux = nullptr;
  if (use_aux) {
    aux = aux_stream(st);
    if (aux) inv_st = aux->s;
  }
  // Two levels: panels of NB columns are grouped in super-panels of S
  // columns.  After a panel, only the rest of its super-panel is updated
  // (K = NB: a lower-triangular block and the rectangle below it), and
  // after a super-panel the whole trailing matrix gets the super-panel's
  // update in one SYRK with K = S; the inverse chain does the same with its
  // block rows.  The same terms as the one-level scheme, summed in another
  // order; the trailing matrix is read and written about S / 2 NB + d / 2 S
  // times instead of d / 2 NB times.
  const int64_t S = chol_super_cols(d);
  for (int64_t s0 = 0; s0 < d; s0 += S) {
    const int64_t s1 = s0 + S < d ? s0 + S : d;
    for (int64_t k0 = s0; k0 < s1; k0 += NB) {
      const int64_t p = k0 / NB;
      const int nb = static_cast<int>(d - k0 < NB ? d - k0 : NB);
      const int64_t k1 = k0 + nb;
      const int rest = static_cast<int>(d - k1);
      const int tiles = static_cast<int>(1 + (rest + NB - 1) / NB);
      const int pgrid = tiles < num_sms() ? tiles : num_sms();  // one wave; CTAs loop
      float *lp = w.linv + p * NB * NB;
      int slot = timer_begin(GQ_KERNEL_POTRF_TRSM, st);
      potrf_trsm_kernel<<<pgrid, 256, PANEL_SMEM, st>>>(A, d, k0, nb, lp, w.status, tiles);
      count_launch();
      // Cholesky of the block nb^3 / 3, the panel solve rest nb^2
      timer_end(slot, st, static_cast<double>(nb) * nb * (nb / 3.0 + rest));
      if (aux) {
        if (cudaEventRecord(aux->ev, st) != cudaSuccess ||
            cudaStreamWaitEvent(aux->s, aux->ev, 0) != cudaSuccess)
          return check_launch("stream fork");
      }
      const int in_sp = static_cast<int>(s1 - k1);  // columns left in the super-panel
      if (in_sp > 0) {
        // A[k1:s1, k1:s1] -= P P^T (lower part), P = A[k1:s1, k0:k1]
        gq_status s = launch_gemm_tf32x3(in_sp, in_sp, nb, -1.0f, A + k1 * d + k0, d,
                                         A + k1 * d + k0, d, true, 1.0f, A + k1 * d + k1, d,
                                         true, w.status, st);
        if (s != GQ_OK) return s;
        if (d > s1) {
          // A[s1:, k1:s1] -= A[s1:, k0:k1] A[k1:s1, k0:k1]^T
          s = launch_gemm_tf32x3(static_cast<int>(d - s1), in_sp, nb, -1.0f, A + s1 * d + k0, d,
                                 A + k1 * d + k0, d, true, 1.0f, A + s1 * d + k1, d, false,
                                 w.status, st);
          if (s != GQ_OK) return s;
        }
      }
      // ---- inverse step p (on inv_st): X[k0:k1, 0:k1] := L_pp^-1 X[k0:k1, 0:k1]
      slot = timer_begin(GQ_KERNEL_BLOCK_INVERSE, inv_st);
      block_inverse_kernel<<<1, 256, INV_SMEM, inv_st>>>(lp);
      count_launch();
      timer_end(slot, inv_st, static_cast<double>(nb) * nb * nb / 3.0);
      const int cols = static_cast<int>(k1);
      // (in place: each output tile owns its columns)
      gq_status s = launch_gemm_tf32x3(nb, cols, nb, 1.0f, lp, NB, X + k0 * d, d, false, 0.0f,
                                       X + k0 * d, d, false, w.status, inv_st);
      if (s != GQ_OK) return s;
      if (in_sp > 0) {
        // X[k1:s1, 0:k1] -= L[k1:s1, k0:k1] X[k0:k1, 0:k1]
        s = launch_gemm_tf32x3(in_sp, cols, nb, -1.0f, A + k1 * d + k0, d, X + k0 * d, d, false,
                               1.0f, X + k1 * d, d, false, w.status, inv_st);
        if (s != GQ_OK) return s;
      }
    }
    if (d > s1) {
      const int rest = static_cast<int>(d - s1), sw = static_cast<int>(s1 - s0);
      // A[s1:, s1:] -= L[s1:, s0:s1] L[s1:, s0:s1]^T (lower part)
      gq_status s = launch_gemm_tf32x3(rest, rest, sw, -1.0f, A + s1 * d + s0, d,
                                       A + s1 * d + s0, d, true, 1.0f, A + s1 * d + s1, d, true,
                                       w.status, st);
      if (s != GQ_OK) return s;
      // X[s1:, 0:s1] -= L[s1:, s0:s1] X[s0:s1, 0:s1] (on inv_st, after the
      // super-panel's last inverse step)
      s = launch_gemm_tf32x3(rest, static_cast<int>(s1), sw, -1.0f, A + s1 * d + s0, d,
                             X + s0 * d, d, false, 1.0f, X + s1 * d, d, false, w.status, inv_st);
      if (s != GQ_OK) return s;
    }
  }
  if (aux) {
    if (cudaEventRecord(aux->join, aux->s) != cudaSuccess ||
        cudaStreamWaitEvent(st, aux->join, 0) != cudaSuccess)
      return check_launch("stream join");
  }
  reverse_upper_kernel<<<gr, 256, 0, st>>>(X, d, U);
  count_launch();
  finish_info_kernel<<<1, 1, 0, st>>>(w.status, d, info_dev);
  count_launch();
  return check_launch("damp_cholesky_inverse");
}

}  // namespace gq

// ---------------------------------------------------------------------------
// gq_damp_cholesky_inverse_noalloc: the same computation for callers that
// cannot allocate device memory, so cannot hand in a workspace either.  Its
// scratch is the file-scope array below, a fixed part of every GPU context
// that loads this library (it stays there until the process exits).
namespace gq {
namespace {

constexpr int64_t kNoAllocMaxDin = 4096;
constexpr size_t kNoAllocScratchBytes =
    kWsHeader + ((static_cast<size_t>(kNoAllocMaxDin) * sizeof(float) + 255) / 256) * 256 +
    static_cast<size_t>((kNoAllocMaxDin + NB - 1) / NB) * NB * NB * sizeof(float);

static __device__ __align__(256) uint8_t g_noalloc_chol_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kMaxDevices] = {};

// The array's device address on the current device, looked up once per
// device.  The array's name is only a host-side handle in host code; the
// kernels need this address.
gq_status noalloc_scratch(void **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return fail(GQ_ERR_CUDA, "no current CUDA device (or device index >= 64)");
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_chol_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail(GQ_ERR_CUDA, std::string("cudaGetSymbolAddress failed: ") +
                                   cudaGetErrorString(e));
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return GQ_OK;
}

}  // namespace
}  // namespace gq

extern "C" gq_status gq_damp_cholesky_inverse_noalloc(float *H, int64_t d_in, float damp_percent,
                                                      int act_order, int32_t *perm_out,
                                                      uint8_t *dead_out, float *U,
                                                      int32_t *info_dev, int32_t *info_host,
                                                      void *stream) {
  using namespace gq;
  clear_error();
  if (!H || !U) return fail(GQ_ERR_ARG, "null pointer");
  if ((reinterpret_cast<uintptr_t>(H) | reinterpret_cast<uintptr_t>(U)) % 16 != 0)
    return fail(GQ_ERR_ARG, "H and U must be 16-byte aligned");
  if (act_order != 0 && !perm_out) return fail(GQ_ERR_ARG, "act_order needs perm_out");
  if (!(damp_percent >= 0.0f) || !(damp_percent < 1e30f))
    return fail(GQ_ERR_ARG, "damp_percent must be finite and >= 0");
  if (d_in < 8 || d_in % 8 != 0)
    return fail(GQ_ERR_SHAPE, "d_in must be a positive multiple of 8");
  if (d_in > kNoAllocMaxDin)
    return fail(GQ_ERR_SHAPE, "d_in " + std::to_string(d_in) +
                                  " exceeds the no-allocation limit of " +
                                  std::to_string(kNoAllocMaxDin) +
                                  "; use gq_damp_cholesky_inverse with a workspace");
  void *scratch = nullptr;
  const gq_status s0 = noalloc_scratch(&scratch);
  if (s0 != GQ_OK) return s0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // Every buffer in the scratch is written before it is read within the call
  // (damp_kernel resets the status words), so earlier calls' leftovers are
  // harmless.
  const gq_status s = launch_damp_chol(H, d_in, damp_percent, act_order, perm_out, dead_out, U,
                                       info_dev, scratch, st, false);
  if (s != GQ_OK) return s;
  if (info_host) {
    // words 0 and 1 of the scratch: device status, info; read on the
    // caller's stream only (a synchronous copy could wait on other streams)
    int32_t words[2] = {0, -1};
    if (cudaMemcpyAsync(words, scratch, sizeof(words), cudaMemcpyDeviceToHost, st) !=
            cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
      return check_launch("damp_cholesky_noalloc sync");
    *info_host = words[1];
    if (words[0] == kDevTimeout)
      return fail(GQ_ERR_TIMEOUT, "damp_cholesky_inverse_noalloc: a device-side wait gave up");
    if (words[1] >= 0)
      return fail(GQ_ERR_NOT_PD, "damped Hessian not positive definite at column " +
                                     std::to_string(words[1]));
  }
  return GQ_OK;
}
