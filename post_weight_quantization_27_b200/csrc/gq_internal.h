// Host-side declarations shared by the libgq translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>
#include <string>

#include "../../include/gq.h"

namespace gq {

extern std::atomic<uint64_t> g_launches;
inline void count_launch(uint64_t n = 1) { g_launches.fetch_add(n, std::memory_order_relaxed); }

// Per-launch timing (gq_kernel_timer_*): timer_begin before a launch
// returns a record slot (or -1 when the kernel is not being timed; one
// atomic load on that path), timer_end after it records the closing event
// and the launch's algorithmic work.
extern std::atomic<uint32_t> g_timer_mask;
int timer_begin_slow(gq_kernel k, cudaStream_t st);
void timer_end_slow(int slot, cudaStream_t st, double work);
inline int timer_begin(gq_kernel k, cudaStream_t st) {
  return (g_timer_mask.load(std::memory_order_relaxed) & (1u << k)) ? timer_begin_slow(k, st)
                                                                     : -1;
}
inline void timer_end(int slot, cudaStream_t st, double work) {
  if (slot >= 0) timer_end_slow(slot, st, work);
}

// Clears the thread-local error text (start of every entry point).
void clear_error();
// Sets the thread-local error text and returns `s`.
gq_status fail(gq_status s, const std::string &msg);
// GQ_ERR_CUDA with the text of the pending CUDA error, or GQ_OK.
gq_status check_launch(const char *what);

inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// 2-D bf16 / fp32 tensor map with 128-byte swizzle: inner extent `inner`
// elements (contiguous), outer extent `outer` rows with a row pitch of
// `pitch_elems` elements; box of box_inner x box_outer.
gq_status make_tmap_2d(CUtensorMap *map, const void *base, CUtensorMapDataType dt,
                       size_t elem_bytes, uint64_t inner, uint64_t outer, uint64_t pitch_elems,
                       uint32_t box_inner, uint32_t box_outer,
                       CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B);

int num_sms();

// ---- kernels (each returns GQ_OK or GQ_ERR_CUDA after launching) ----
// group_size: -1 per row, 0 per tensor (one scale, stored once per row), else per group.
// bits: 2, 3, 4 or 8 (codes of other widths than 4 need d_in and the group a
// multiple of 32; rows are little-endian bit streams, see include/gq.h).
gq_status launch_tensor_params_f32(const float *W, int64_t d_out, int64_t d_in, int sym,
                                   uint16_t *scales, uint16_t *zeros, float *scratch,
                                   int64_t scratch_floats, cudaStream_t st, int bits = 4);
gq_status launch_rtn(const void *W, gq_dtype dt, int64_t d_out, int64_t d_in, int group_size,
                     int sym, uint32_t *qpacked, uint16_t *scales, uint16_t *zeros,
                     cudaStream_t st, int bits = 4);

struct HessPlan {
  int n_bi, n_bj, n_tiles, n_split, nkb_total, kb_per_split;
  int align_groups, align_waves;  // token-alignment counters (0: none)
  size_t off_align, ws_bytes;
};
HessPlan hessian_plan(int64_t n_tok, int64_t d_in);
gq_status launch_hessian(const void *X, int64_t n_tok, int64_t d_in, float *H, void *ws,
                         const HessPlan &plan, cudaStream_t st, bool accumulate = true);

size_t chol_ws_bytes(int64_t d);
// use_aux: run the inverse chain on a second stream (forked from and joined
// back to `st` with events).
gq_status launch_damp_chol(float *H, int64_t d, float damp, int act_order, int32_t *perm_out,
                           uint8_t *dead_out, float *U, int32_t *info_dev, void *ws,
                           cudaStream_t st, bool use_aux = true);

// C = beta C + alpha A B in fp32 on the tensor cores (3 x TF32 split); with
// dot_partials, per output tile the sum of (alpha A B) .* C instead (C is
// read, not written; gemm_tf32x3_tiles(M, N, lower) partials; with lower
// the lower-triangle tiles give the full sum of a symmetric product).
gq_status launch_gemm_tf32x3(int M, int N, int K, float alpha, const float *A, int64_t lda,
                             const float *B, int64_t ldb, bool b_kmajor, float beta, float *C,
                             int64_t ldc, bool lower, int *status, cudaStream_t st,
                             double *dot_partials = nullptr);
int gemm_tf32x3_tiles(int M, int N, bool lower = false);
// sum over the lower triangle of (A A^T) .* C with A = A_h + A_l in bf16
// parts [M][lda] (K contiguous, lda a multiple of 8), C symmetric fp32:
// syrk_dot_bf16x3_partials(M) fp64 partials (strictly lower elements
// twice, the diagonal once); ~2^-16 relative per product term.
int syrk_dot_bf16x3_partials(int M);
gq_status launch_syrk_dot_bf16x3(int M, int K, const uint16_t *A_h, const uint16_t *A_l,
                                 int64_t lda, const float *C, int64_t ldc, double *dot_partials,
                                 int *status, cudaStream_t st);

size_t gptq_ws_bytes(int64_t d_out, int64_t d_in, int block_size);
gq_status launch_gptq(const void *W, gq_dtype dt, int64_t d_out, int64_t d_in, const float *U,
                      int group_size, int block_size, int sym, const int32_t *perm,
                      const uint8_t *dead, uint32_t *qpacked, uint16_t *scales, uint16_t *zeros,
                      int32_t *g_idx, void *ws, cudaStream_t st, int bits = 4);

size_t recon_ws_bytes(int64_t d_out, int64_t d_in, int64_t n_tok);
// SSE by the trace route tr(dW H0 dW^T) / 2 (H0 = 2 X^T X undamped).
size_t recon_hessian_ws_bytes(int64_t d_out, int64_t d_in);
gq_status launch_recon_hessian(const void *W, gq_dtype dt, const uint32_t *qpacked,
                               const uint16_t *scales, const uint16_t *zeros,
                               const int32_t *g_idx, int64_t d_out, int64_t d_in, int group_size,
                               int sym, const float *H0, double *sse_dev, void *ws,
                               cudaStream_t st, int bits = 4);
gq_status launch_recon(const void *W, gq_dtype dt, const uint32_t *qpacked,
                       const uint16_t *scales, const uint16_t *zeros, const int32_t *g_idx,
                       int64_t d_out, int64_t d_in, int group_size, int sym, const void *X,
                       int64_t n_tok, double *sse_dev, void *ws, cudaStream_t st,
                       const float *col_inv = nullptr, float *Y = nullptr, int bits = 4);

// Y = W^ X^T with the codes dequantised inside the GEMM (qlinear.cu): Y
// feature-major fp32 and / or Z = act(Y^T) + R token-major bf16; dense
// weights when qpacked is NULL.  status: the call's device status word.
gq_status launch_qlinear(const uint32_t *qpacked, const uint16_t *scales, const uint16_t *zeros,
                         const int32_t *g_idx, const void *W_dense, gq_dtype w_dtype,
                         int64_t d_out, int64_t d_in, int bits, int group_size, int sym,
                         const void *X, int64_t n_tok, float *Y, void *Z, const void *R,
                         int act, int *status, cudaStream_t st);

// Sequential quantisation of a chain of layers (pipeline.cu).
size_t seq_ws_bytes(const gq_seq_layer *layers, int n_layers, int64_t n_tok, int block_size);
gq_status launch_sequential(const void *X0, int64_t n_tok, const gq_seq_layer *layers, int n,
                            int bits, int group_size, int block_size, int sym, float damp,
                            double *sse_dev, void *X_all, void *ws, cudaStream_t st);

// Activation-aware scaling before RTN (awq.cu).
size_t awq_ws_bytes(int64_t d_out, int64_t d_in, int64_t n_tok, int group_size, int sym,
                    int bits = 4);
gq_status launch_awq_rtn_search(const void *W, gq_dtype dt, int64_t d_out, int64_t d_in,
                                const float *H, const void *X, int64_t n_tok, int group_size,
                                int sym, int n_grid, uint32_t *qpacked, uint16_t *scales,
                                uint16_t *zeros, float *col_scale, double *mse_host,
                                int32_t *best_host, void *ws, cudaStream_t st, int bits = 4);

}  // namespace gq
