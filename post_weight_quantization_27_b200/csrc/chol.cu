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
// and factored in place; X = L^-1 is built in the H buffer (the caller's H
// is scratch); the last kernel writes U = J X J back into the U buffer.
// Blocked right-looking algorithms with 128-wide panels; one CTA factors a
// diagonal block in shared memory (and inverts it), the panel solve, the
// trailing updates and the inverse's block steps are fp32 GEMMs on the
// tensor cores (3 x TF32 split, gemm_tc.cu).
#include <cfloat>
#include <climits>
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
  for (int64_t a = blockIdx.y; a < d; a += gridDim.y) {
    const int64_t sa = d - 1 - a;
    const int64_t ra = perm ? perm[sa] : sa;
    for (int64_t b = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; b <= a;
         b += static_cast<int64_t>(gridDim.x) * 256) {
      const int64_t sb = d - 1 - b;
      const int64_t cb = perm ? perm[sb] : sb;
      A[a * d + b] = H[ra * d + cb];
    }
  }
}

// ---------------------------------------------------------------- panel factor
// Cholesky of the nb x nb diagonal block at (k0, k0) of the lower matrix A
// (in place), and the inverse of that block written to linv [NB][NB].
// The 128 columns are done in sub-panels of 32:
//   (a) one warp factors the 32 x 32 diagonal piece with a row per lane in
//       registers (pivot and column broadcast by shuffles);
//   (b) one thread per row below solves x L^T = a with the row in registers;
//   (c) all threads apply the sub-panel to the rest of the block in 4 x 4
//       register tiles.
// The inverse: each warp inverts one 32 x 32 diagonal block (a column per
// lane), then X_ij = -X_ii (sum_k L_ik X_kj) for the blocks below, one
// diagonal band at a time.
constexpr int SP = NB + 1;  // padded row stride in shared memory (bank-conflict free columns)

// Column J of the warp's 32 x 32 Cholesky (lane = row, w = the row), unrolled
// by template recursion so every register index is a constant.
template <int J>
__device__ __forceinline__ void chol32_column(float (&w)[32], float &my_rd, int lane, int64_t col0,
                                              int nb_left, int *status) {
  if constexpr (J < 32) {
    float piv = __shfl_sync(0xffffffffu, w[J], J);
    if (!(piv > 0.0f) || !(piv < FLT_MAX)) {
      if (lane == 0 && J < nb_left) atomicMin(&status[1], static_cast<int>(col0 + J));
      piv = 1.0f;
    }
    // 1 / sqrt(piv): hardware estimate plus one Newton step r (3 - piv r^2) / 2
    float rj = rsqrtf(piv);
    rj = rj * fmaf(-0.5f * piv, rj * rj, 1.5f);
    const float dj = piv * rj;
    const float lij = lane > J ? w[J] * rj : (lane == J ? dj : 0.0f);
    w[J] = lij;
    if (lane == J) my_rd = rj;
#pragma unroll
    for (int k = J + 1; k < 32; ++k) {
      const float lkj = __shfl_sync(0xffffffffu, lij, k);
      if (k <= lane) w[k] = fmaf(-lij, lkj, w[k]);
    }
    chol32_column<J + 1>(w, my_rd, lane, col0, nb_left, status);
  }
}
constexpr int TP = 33;      // stride of the 32 x 32 temporaries
constexpr size_t POTRF_SMEM = (2 * NB * SP + NB + 3 * 32 * TP) * sizeof(float);

__global__ void __launch_bounds__(256) potrf_panel_kernel(float *__restrict__ A, int64_t d,
                                                          int64_t k0, int nb,
                                                          float *__restrict__ linv,
                                                          int *status) {
  extern __shared__ float sm[];
  float *S = sm;                // [NB][SP]  the block, then L (lower)
  float *Li = S + NB * SP;      // [NB][SP]  L^-1 (lower)
  float *rd = Li + NB * SP;     // [NB]      1 / L_jj
  float *T = rd + NB;           // [3][32][TP] temporaries of the inverse
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // the block's lower part, 16 float4 loads per thread in flight at once;
  // identity padding past the matrix edge (only the lower part is ever read)
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
      for (int q = 0; q < 4; ++q) {
        float x = e[q];
        if (r >= nb) x = (r == c + q) ? 1.0f : 0.0f;
        S[r * SP + c + q] = x;
        Li[r * SP + c + q] = 0.0f;
      }
    }
  }
  __syncthreads();

  for (int c0 = 0; c0 < NB; c0 += 32) {
    // (a) diagonal 32 x 32 piece
    if (warp == 0) {
      float w[32];
#pragma unroll
      for (int k = 0; k < 32; ++k) w[k] = (k <= lane) ? S[(c0 + lane) * SP + c0 + k] : 0.0f;
      float my_rd = 1.0f;
      chol32_column<0>(w, my_rd, lane, k0 + c0, nb - c0, status);
#pragma unroll
      for (int k = 0; k < 32; ++k)
        if (k <= lane) S[(c0 + lane) * SP + c0 + k] = w[k];
      rd[c0 + lane] = my_rd;
    }
    __syncthreads();
    // (b) rows below the piece: x = a L_dd^-T, right-looking within the row
    for (int r = c0 + 32 + tid; r < NB; r += 256) {
      float a[32];
#pragma unroll
      for (int k = 0; k < 32; ++k) a[k] = S[r * SP + c0 + k];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float x = a[j] * rd[c0 + j];
        a[j] = x;
#pragma unroll
        for (int k = j + 1; k < 32; ++k) a[k] = fmaf(-x, S[(c0 + k) * SP + c0 + j], a[k]);
      }
#pragma unroll
      for (int k = 0; k < 32; ++k) S[r * SP + c0 + k] = a[k];
    }
    __syncthreads();
    // (c) rest of the block: S[i][k] -= sum_j S[i][c0+j] S[k][c0+j], base <= k <= i
    const int base = c0 + 32;
    const int mt = (NB - base) / 4;  // 4 x 4 tiles per side
    const int n_tiles = mt * (mt + 1) / 2;
    for (int t = tid; t < n_tiles; t += 256) {
      int ti = 0;
      while ((ti + 1) * (ti + 2) / 2 <= t) ++ti;
      const int tk = t - ti * (ti + 1) / 2;
      const int i0 = base + 4 * ti, kk0 = base + 4 * tk;
      float acc[4][4];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = 0.0f;
#pragma unroll 8
      for (int j = 0; j < 32; ++j) {
        float pi[4], pk[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          pi[a] = S[(i0 + a) * SP + c0 + j];
          pk[a] = S[(kk0 + a) * SP + c0 + j];
        }
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(pi[a], pk[b], acc[a][b]);
      }
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b)
          if (kk0 + b <= i0 + a) S[(i0 + a) * SP + kk0 + b] -= acc[a][b];
    }
    __syncthreads();
  }

  // inverse, diagonal blocks: warp q, lane = column
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
  // bands below the diagonal: X_ij = -X_ii sum_{k=j}^{i-1} L_ik X_kj, i - j = lvl
  // (each thread: one row r, four consecutive columns 4*c4 .. 4*c4+3)
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

  for (int e = tid; e < NB * NB; e += 256) {
    const int r = e / NB, c = e % NB;
    if (r < nb && c <= r) A[(k0 + r) * d + k0 + c] = S[r * SP + c];
    linv[e] = Li[r * SP + c];
  }
}

// X := I on the lower triangle and on the whole NB x NB diagonal blocks
// (the right-hand side of L X = I); the rest of the upper part is never read.
__global__ void __launch_bounds__(256) eye_lower_kernel(float *__restrict__ X, int64_t d) {
  for (int64_t r = blockIdx.y; r < d; r += gridDim.y) {
    int64_t end = (r / NB + 1) * NB;
    if (end > d) end = d;
    for (int64_t c = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; c < end;
         c += static_cast<int64_t>(gridDim.x) * 256)
      X[r * d + c] = r == c ? 1.0f : 0.0f;
  }
}

// U[a][b] = X[d-1-a][d-1-b] for a <= b, 0 below the diagonal; also turns
// the recorded pivot failure into the info value.
__global__ void __launch_bounds__(256) reverse_upper_kernel(const float *__restrict__ X,
                                                            int64_t d, float *__restrict__ U) {
  for (int64_t a = blockIdx.y; a < d; a += gridDim.y)
    for (int64_t b = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; b < d;
         b += static_cast<int64_t>(gridDim.x) * 256)
      U[a * d + b] = b >= a ? X[(d - 1 - a) * d + (d - 1 - b)] : 0.0f;
}

// The factorisation runs on the reversed matrix: reversed pivot k is column
// d-1-k in processing order.
__global__ void finish_info_kernel(int *status, int64_t d, int32_t *info_dev) {
  const int v = status[1] == INT_MAX ? -1 : static_cast<int>(d - 1 - status[1]);
  status[1] = v;
  if (info_dev) *info_dev = v;
}

}  // namespace

size_t chol_ws_bytes(int64_t d) {
  const int64_t n_panels = (d + NB - 1) / NB;
  return kWsHeader + round_up(static_cast<size_t>(d) * sizeof(float), 256) +
         static_cast<size_t>(n_panels) * NB * NB * sizeof(float);
}

gq_status launch_damp_chol(float *H, int64_t d, float damp, int act_order, int32_t *perm_out,
                           uint8_t *dead_out, float *U, int32_t *info_dev, void *ws,
                           cudaStream_t st) {
  CholWs w = carve(ws, d);
  damp_kernel<<<1, 1024, 0, st>>>(H, d, damp, dead_out, w.key, w.status);
  count_launch();
  if (act_order) {
    rank_kernel<<<static_cast<unsigned>((d + 255) / 256), 256, 0, st>>>(w.key, d, perm_out);
    count_launch();
  }
  const unsigned gx = static_cast<unsigned>((d + 255) / 256);
  const unsigned gy = static_cast<unsigned>(d < 65535 ? d : 65535);
  float *A = U;  // the factorisation lives in the U buffer
  float *X = H;  // L^-1 is built in the H buffer
  gather_reversed_kernel<<<dim3(gx, gy), 256, 0, st>>>(
      H, d, act_order ? perm_out : nullptr, A);
  count_launch();
  {
    const gq_status s = check_launch("damp/gather");
    if (s != GQ_OK) return s;
  }
  const size_t pot_smem = POTRF_SMEM;
  cudaFuncSetAttribute(potrf_panel_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       static_cast<int>(pot_smem));
  const int64_t n_panels = (d + NB - 1) / NB;
  // ---- Cholesky, right-looking
  for (int64_t p = 0; p < n_panels; ++p) {
    const int64_t k0 = p * NB;
    const int nb = static_cast<int>(d - k0 < NB ? d - k0 : NB);
    float *lp = w.linv + p * NB * NB;
    potrf_panel_kernel<<<1, 256, pot_smem, st>>>(A, d, k0, nb, lp, w.status);
    count_launch();
    const int64_t k1 = k0 + nb;
    const int rest = static_cast<int>(d - k1);
    if (rest > 0) {
      // panel rows below: A[k1:, k0:k1] := A[k1:, k0:k1] L_pp^-T (in place:
      // each output tile owns its rows)
      gq_status s = launch_gemm_tf32x3(rest, nb, NB, 1.0f, A + k1 * d + k0, d, lp, NB, true,
                                       0.0f, A + k1 * d + k0, d, false, w.status, st);
      if (s != GQ_OK) return s;
      // trailing: A[k1:, k1:] -= P P^T (lower part)
      s = launch_gemm_tf32x3(rest, rest, NB, -1.0f, A + k1 * d + k0, d, A + k1 * d + k0, d,
                             true, 1.0f, A + k1 * d + k1, d, true, w.status, st);
      if (s != GQ_OK) return s;
    }
  }
  // ---- X = L^-1 by blocked forward substitution on the identity
  eye_lower_kernel<<<dim3(gx, gy), 256, 0, st>>>(X, d);
  count_launch();
  for (int64_t p = 0; p < n_panels; ++p) {
    const int64_t r0 = p * NB;
    const int nb = static_cast<int>(d - r0 < NB ? d - r0 : NB);
    const int cols = static_cast<int>(r0 + nb);
    float *lp = w.linv + p * NB * NB;
    // X[r0:r0+nb, 0:cols] := L_pp^-1 X[r0:r0+nb, 0:cols] (in place: each
    // output tile owns its columns)
    gq_status s = launch_gemm_tf32x3(nb, cols, nb, 1.0f, lp, NB, X + r0 * d, d, false, 0.0f,
                                     X + r0 * d, d, false, w.status, st);
    if (s != GQ_OK) return s;
    const int64_t r1 = r0 + nb;
    const int rest = static_cast<int>(d - r1);
    if (rest > 0) {
      // X[r1:, 0:cols] -= L[r1:, r0:r1] X[r0:r1, 0:cols]
      s = launch_gemm_tf32x3(rest, cols, nb, -1.0f, A + r1 * d + r0, d, X + r0 * d, d, false,
                             1.0f, X + r1 * d, d, false, w.status, st);
      if (s != GQ_OK) return s;
    }
  }
  reverse_upper_kernel<<<dim3(gx, gy), 256, 0, st>>>(X, d, U);
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
                                       info_dev, scratch, st);
  if (s != GQ_OK) return s;
  if (info_host) {
    int32_t info = -1;
    const int32_t *src = info_dev ? info_dev : reinterpret_cast<const int32_t *>(scratch) + 1;
    if (cudaStreamSynchronize(st) != cudaSuccess ||
        cudaMemcpy(&info, src, sizeof(int32_t), cudaMemcpyDeviceToHost) != cudaSuccess)
      return check_launch("damp_cholesky_noalloc sync");
    *info_host = info;
    if (info >= 0)
      return fail(GQ_ERR_NOT_PD, "damped Hessian not positive definite at column " +
                                     std::to_string(info));
  }
  return GQ_OK;
}
