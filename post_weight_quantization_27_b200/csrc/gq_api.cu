// extern "C" entry points of libgq.so: argument validation, workspace
// sizing, and dispatch to the kernels.  See include/gq.h for the contract.
#include <cstdio>
#include <cstring>
#include <mutex>

#include "gq_device.cuh"
#include "gq_internal.h"

namespace gq {

std::atomic<uint64_t> g_launches{0};
static thread_local std::string t_last_error;

void clear_error() { t_last_error.clear(); }

gq_status fail(gq_status s, const std::string &msg) {
  t_last_error = msg;
  return s;
}

gq_status check_launch(const char *what) {
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) return GQ_OK;
  return fail(GQ_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

gq_status make_tmap_2d(CUtensorMap *map, const void *base, CUtensorMapDataType dt,
                       size_t elem_bytes, uint64_t inner, uint64_t outer, uint64_t pitch_elems,
                       uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(GQ_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {pitch_elems * elem_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(GQ_ERR_CUDA, "cuTensorMapEncodeTiled failed");
  return GQ_OK;
}

}  // namespace gq

using namespace gq;

namespace {

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

gq_status check_dtype(gq_dtype dt) {
  if (dt != GQ_F32 && dt != GQ_F16 && dt != GQ_BF16) return fail(GQ_ERR_DTYPE, "unknown w_dtype");
  return GQ_OK;
}

gq_status check_layer(int64_t d_out, int64_t d_in) {
  if (d_out < 1 || d_in < 8 || d_in % 8 != 0)
    return fail(GQ_ERR_SHAPE, "need d_out >= 1 and d_in a positive multiple of 8");
  if (d_in > (int64_t(1) << 30) || d_out > (int64_t(1) << 31))
    return fail(GQ_ERR_SHAPE, "layer too large");
  return GQ_OK;
}

gq_status check_group(int group_size, int64_t d_in) {
  if (group_size == -1 || group_size == 0) return GQ_OK;
  if (group_size < 8 || group_size % 8 != 0 || d_in % group_size != 0)
    return fail(GQ_ERR_SHAPE, "group_size must be -1, 0 or a multiple of 8 dividing d_in");
  return GQ_OK;
}

// Code widths: 2, 3, 4 or 8 bits.  Rows are bit streams cut into 32-bit
// words, and widths other than 4 are packed in runs of 32 columns: d_in and
// the group size must then be multiples of 32.
gq_status check_bits(int bits, int64_t d_in, int group_size) {
  if (bits != 2 && bits != 3 && bits != 4 && bits != 8)
    return fail(GQ_ERR_ARG, "bits must be 2, 3, 4 or 8");
  if (bits != 4 && (d_in % 32 != 0 || (group_size > 0 && group_size % 32 != 0)))
    return fail(GQ_ERR_SHAPE, "codes of other widths than 4 bits need d_in and group_size "
                              "multiples of 32");
  return GQ_OK;
}

gq_status check_ws(const void *ws, size_t have, size_t need) {
  if (need == 0) return GQ_OK;
  if (!ws || have < need)
    return fail(GQ_ERR_WORKSPACE, "workspace too small: need " + std::to_string(need) +
                                      " bytes, have " + std::to_string(have));
  if (!aligned(ws, 256)) return fail(GQ_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  return GQ_OK;
}

#define GQ_TRY(x)                         \
  do {                                    \
    const gq_status _s = (x);             \
    if (_s != GQ_OK) return _s;           \
  } while (0)

// GQ_ERR_TIMEOUT if a device status word (read after the stream has been
// synchronised) records a wait that gave up, else GQ_OK.
gq_status device_status(int32_t word, const char *what) {
  if (word == kDevTimeout)
    return fail(GQ_ERR_TIMEOUT, std::string(what) + ": a device-side wait gave up");
  if (word != kDevOk)
    return fail(GQ_ERR_CUDA, std::string(what) + ": device status " + std::to_string(word));
  return GQ_OK;
}

// One thread waits on an mbarrier; with `arrive` it arrives on it first.
// The wait gives up after limit_ns and records kDevTimeout in *status.
__global__ void bounded_wait_kernel(int arrive, uint64_t limit_ns, int *status) {
  __shared__ __align__(8) uint64_t bar;
  mbar_init(&bar, 1);
  fence_barrier_init();
  if (arrive) mbar_arrive(&bar);
  if (!mbar_wait(&bar, 0, limit_ns)) set_status(status, kDevTimeout);
}

}  // namespace

extern "C" {

const char *gq_status_string(gq_status s) {
  switch (s) {
    case GQ_OK: return "GQ_OK";
    case GQ_ERR_ARG: return "GQ_ERR_ARG";
    case GQ_ERR_SHAPE: return "GQ_ERR_SHAPE";
    case GQ_ERR_DTYPE: return "GQ_ERR_DTYPE";
    case GQ_ERR_WORKSPACE: return "GQ_ERR_WORKSPACE";
    case GQ_ERR_NOT_PD: return "GQ_ERR_NOT_PD";
    case GQ_ERR_NONFINITE: return "GQ_ERR_NONFINITE";
    case GQ_ERR_TIMEOUT: return "GQ_ERR_TIMEOUT";
    case GQ_ERR_CUDA: return "GQ_ERR_CUDA";
  }
  return "GQ_UNKNOWN_STATUS";
}

const char *gq_last_error(void) { return t_last_error.c_str(); }

uint64_t gq_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

size_t gq_hessian_workspace_size(int64_t n_tok, int64_t d_in) {
  if (n_tok < 0 || d_in < 8 || d_in % 8 != 0) return 0;
  return hessian_plan(n_tok, d_in).ws_bytes;
}

gq_status gq_hessian_accumulate(const void *X_bf16, int64_t n_tok, int64_t d_in, float *H,
                                void *ws, size_t ws_bytes, void *stream) {
  t_last_error.clear();
  if (!H || (n_tok > 0 && !X_bf16)) return fail(GQ_ERR_ARG, "null pointer");
  if (n_tok < 0 || d_in < 8 || d_in % 8 != 0)
    return fail(GQ_ERR_SHAPE, "need n_tok >= 0 and d_in a positive multiple of 8");
  if (d_in > 65536 || n_tok > (int64_t(1) << 31) - 64)
    return fail(GQ_ERR_SHAPE, "d_in or n_tok too large");
  if (n_tok > 0 && !aligned(X_bf16, 16)) return fail(GQ_ERR_ARG, "X must be 16-byte aligned");
  const HessPlan p = hessian_plan(n_tok, d_in);
  GQ_TRY(check_ws(ws, ws_bytes, p.ws_bytes));
  return launch_hessian(X_bf16, n_tok, d_in, H, ws, p, static_cast<cudaStream_t>(stream));
}

gq_status gq_hessian_compute(const void *X_bf16, int64_t n_tok, int64_t d_in, float *H,
                             void *ws, size_t ws_bytes, void *stream) {
  t_last_error.clear();
  if (!H || (n_tok > 0 && !X_bf16)) return fail(GQ_ERR_ARG, "null pointer");
  if (n_tok < 0 || d_in < 8 || d_in % 8 != 0)
    return fail(GQ_ERR_SHAPE, "need n_tok >= 0 and d_in a positive multiple of 8");
  if (d_in > 65536 || n_tok > (int64_t(1) << 31) - 64)
    return fail(GQ_ERR_SHAPE, "d_in or n_tok too large");
  if (n_tok > 0 && !aligned(X_bf16, 16)) return fail(GQ_ERR_ARG, "X must be 16-byte aligned");
  const HessPlan p = hessian_plan(n_tok, d_in);
  GQ_TRY(check_ws(ws, ws_bytes, p.ws_bytes));
  return launch_hessian(X_bf16, n_tok, d_in, H, ws, p, static_cast<cudaStream_t>(stream), false);
}

size_t gq_damp_cholesky_workspace_size(int64_t d_in) {
  if (d_in < 8 || d_in % 8 != 0) return 0;
  return chol_ws_bytes(d_in);
}

gq_status gq_damp_cholesky_inverse(float *H, int64_t d_in, float damp_percent, int act_order,
                                   int32_t *perm_out, uint8_t *dead_out, float *U,
                                   int32_t *info_dev, int32_t *info_host, void *ws,
                                   size_t ws_bytes, void *stream) {
  t_last_error.clear();
  if (!H || !U) return fail(GQ_ERR_ARG, "null pointer");
  if ((reinterpret_cast<uintptr_t>(H) | reinterpret_cast<uintptr_t>(U)) % 16 != 0)
    return fail(GQ_ERR_ARG, "H and U must be 16-byte aligned");
  if (act_order != 0 && !perm_out) return fail(GQ_ERR_ARG, "act_order needs perm_out");
  if (!(damp_percent >= 0.0f) || !(damp_percent < 1e30f))
    return fail(GQ_ERR_ARG, "damp_percent must be finite and >= 0");
  if (d_in < 8 || d_in % 8 != 0 || d_in > 65536)
    return fail(GQ_ERR_SHAPE, "d_in must be a multiple of 8 in [8, 65536]");
  GQ_TRY(check_ws(ws, ws_bytes, chol_ws_bytes(d_in)));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  GQ_TRY(launch_damp_chol(H, d_in, damp_percent, act_order, perm_out, dead_out, U, info_dev, ws,
                          st));
  if (info_host) {
    // words 0 and 1 of the workspace: device status, info
    int32_t words[2] = {0, -1};
    if (cudaMemcpyAsync(words, ws, sizeof(words), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
      return check_launch("damp_cholesky sync");
    *info_host = words[1];
    GQ_TRY(device_status(words[0], "damp_cholesky_inverse"));
    if (words[1] >= 0)
      return fail(GQ_ERR_NOT_PD, "damped Hessian not positive definite at column " +
                                     std::to_string(words[1]));
  }
  return GQ_OK;
}

size_t gq_gptq_workspace_size(int64_t d_out, int64_t d_in, int block_size) {
  if (d_out < 1 || d_in < 8 || d_in % 8 != 0 || block_size < 32 || block_size > 128 ||
      block_size % 32 != 0)
    return 0;
  return gptq_ws_bytes(d_out, d_in, block_size);
}

gq_status gq_gptq_quantize_layer(const void *W, gq_dtype w_dtype, int64_t d_out, int64_t d_in,
                                 const float *U, int bits, int group_size, int block_size,
                                 int sym, const int32_t *perm, const uint8_t *dead,
                                 uint32_t *qpacked, uint16_t *scales, uint16_t *zeros,
                                 int32_t *g_idx, void *ws, size_t ws_bytes, void *stream) {
  t_last_error.clear();
  GQ_TRY(check_dtype(w_dtype));
  if (!W || !U || !qpacked || !scales) return fail(GQ_ERR_ARG, "null pointer");
  if (sym != 0 && sym != 1) return fail(GQ_ERR_ARG, "sym must be 0 or 1");
  if (sym == 0 && !zeros) return fail(GQ_ERR_ARG, "affine quantization needs zeros");
  GQ_TRY(check_layer(d_out, d_in));
  GQ_TRY(check_group(group_size, d_in));
  GQ_TRY(check_bits(bits, d_in, group_size));
  if (block_size != 32 && block_size != 64 && block_size != 128)
    return fail(GQ_ERR_ARG, "block_size must be 32, 64 or 128");
  if (bits != 4 && block_size != 128)
    return fail(GQ_ERR_ARG, "codes of other widths than 4 bits need block_size 128");
  if (group_size > 0 && (group_size < 32 || block_size % group_size != 0))
    return fail(GQ_ERR_ARG, "GPTQ group_size must be -1, 0, 32, 64 or 128 and divide block_size");
  if (!aligned(W, 16) || !aligned(U, 16)) return fail(GQ_ERR_ARG, "W and U must be 16-byte aligned");
  GQ_TRY(check_ws(ws, ws_bytes, gptq_ws_bytes(d_out, d_in, block_size)));
  return launch_gptq(W, w_dtype, d_out, d_in, U, group_size, block_size, sym, perm, dead,
                     qpacked, scales, zeros, g_idx, ws, static_cast<cudaStream_t>(stream), bits);
}

gq_status gq_rtn_quantize_pack(const void *W, gq_dtype w_dtype, int64_t d_out, int64_t d_in,
                               int bits, int group_size, int sym, uint32_t *qpacked,
                               uint16_t *scales, uint16_t *zeros, void *stream) {
  t_last_error.clear();
  GQ_TRY(check_dtype(w_dtype));
  if (!W || !qpacked || !scales) return fail(GQ_ERR_ARG, "null pointer");
  if (sym != 0 && sym != 1) return fail(GQ_ERR_ARG, "sym must be 0 or 1");
  if (sym == 0 && !zeros) return fail(GQ_ERR_ARG, "affine quantization needs zeros");
  GQ_TRY(check_layer(d_out, d_in));
  GQ_TRY(check_group(group_size, d_in));
  GQ_TRY(check_bits(bits, d_in, group_size));
  if (!aligned(W, 16)) return fail(GQ_ERR_ARG, "W must be 16-byte aligned");
  return launch_rtn(W, w_dtype, d_out, d_in, group_size, sym, qpacked, scales, zeros,
                    static_cast<cudaStream_t>(stream), bits);
}

size_t gq_recon_workspace_size(int64_t d_out, int64_t d_in, int64_t n_tok) {
  if (d_out < 1 || d_in < 8 || d_in % 8 != 0 || n_tok < 0) return 0;
  return recon_ws_bytes(d_out, d_in, n_tok);
}

gq_status gq_recon_error(const void *W, gq_dtype w_dtype, const uint32_t *qpacked,
                         const uint16_t *scales, const uint16_t *zeros, const int32_t *g_idx,
                         int64_t d_out, int64_t d_in, int bits, int group_size, int sym,
                         const void *X_bf16, int64_t n_tok, double *sse_dev, double *sse_host,
                         double *mse_host, void *ws, size_t ws_bytes, void *stream) {
  t_last_error.clear();
  GQ_TRY(check_dtype(w_dtype));
  if (!W || !qpacked || !scales || !sse_dev || (n_tok > 0 && !X_bf16))
    return fail(GQ_ERR_ARG, "null pointer");
  if (sym != 0 && sym != 1) return fail(GQ_ERR_ARG, "sym must be 0 or 1");
  if (sym == 0 && !zeros) return fail(GQ_ERR_ARG, "affine quantization needs zeros");
  GQ_TRY(check_layer(d_out, d_in));
  GQ_TRY(check_group(group_size, d_in));
  GQ_TRY(check_bits(bits, d_in, group_size));
  if (n_tok < 0 || n_tok > (int64_t(1) << 31) - 256) return fail(GQ_ERR_SHAPE, "bad n_tok");
  if (!aligned(W, 16) || (n_tok > 0 && !aligned(X_bf16, 16)))
    return fail(GQ_ERR_ARG, "W and X must be 16-byte aligned");
  GQ_TRY(check_ws(ws, ws_bytes, recon_ws_bytes(d_out, d_in, n_tok)));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  GQ_TRY(launch_recon(W, w_dtype, qpacked, scales, zeros, g_idx, d_out, d_in, group_size, sym,
                      X_bf16, n_tok, sse_dev, ws, st, nullptr, nullptr, bits));
  if (sse_host || mse_host) {
    double sse = 0.0;
    int32_t word = 0;
    if (cudaMemcpyAsync(&sse, sse_dev, sizeof(double), cudaMemcpyDeviceToHost, st) !=
            cudaSuccess ||
        cudaMemcpyAsync(&word, ws, sizeof(word), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
      return check_launch("recon_error sync");
    if (sse_host) *sse_host = sse;
    if (mse_host) *mse_host = n_tok > 0 ? sse / (static_cast<double>(n_tok) * d_out) : 0.0;
    GQ_TRY(device_status(word, "recon_error"));
  }
  return GQ_OK;
}

size_t gq_recon_error_hessian_workspace_size(int64_t d_out, int64_t d_in) {
  if (d_out < 1 || d_in < 8 || d_in % 8 != 0) return 0;
  return recon_hessian_ws_bytes(d_out, d_in);
}

gq_status gq_recon_error_hessian(const void *W, gq_dtype w_dtype, const uint32_t *qpacked,
                                 const uint16_t *scales, const uint16_t *zeros,
                                 const int32_t *g_idx, int64_t d_out, int64_t d_in, int bits,
                                 int group_size, int sym, const float *H0, int64_t n_tok,
                                 double *sse_dev, double *sse_host, double *mse_host, void *ws,
                                 size_t ws_bytes, void *stream) {
  t_last_error.clear();
  GQ_TRY(check_dtype(w_dtype));
  if (!W || !qpacked || !scales || !sse_dev || !H0) return fail(GQ_ERR_ARG, "null pointer");
  if (sym != 0 && sym != 1) return fail(GQ_ERR_ARG, "sym must be 0 or 1");
  if (sym == 0 && !zeros) return fail(GQ_ERR_ARG, "affine quantization needs zeros");
  GQ_TRY(check_layer(d_out, d_in));
  GQ_TRY(check_group(group_size, d_in));
  GQ_TRY(check_bits(bits, d_in, group_size));
  if (n_tok < 0) return fail(GQ_ERR_SHAPE, "bad n_tok");
  if (d_out > (int64_t(1) << 30) || d_in > (int64_t(1) << 30))
    return fail(GQ_ERR_SHAPE, "layer too large");
  if (!aligned(W, 16) || !aligned(H0, 16))
    return fail(GQ_ERR_ARG, "W and H0 must be 16-byte aligned");
  GQ_TRY(check_ws(ws, ws_bytes, recon_hessian_ws_bytes(d_out, d_in)));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  GQ_TRY(launch_recon_hessian(W, w_dtype, qpacked, scales, zeros, g_idx, d_out, d_in, group_size,
                              sym, H0, sse_dev, ws, st, bits));
  if (sse_host || mse_host) {
    double sse = 0.0;
    int32_t word = 0;
    if (cudaMemcpyAsync(&sse, sse_dev, sizeof(double), cudaMemcpyDeviceToHost, st) !=
            cudaSuccess ||
        cudaMemcpyAsync(&word, ws, sizeof(word), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
      return check_launch("recon_error_hessian sync");
    if (sse_host) *sse_host = sse;
    if (mse_host) *mse_host = n_tok > 0 ? sse / (static_cast<double>(n_tok) * d_out) : 0.0;
    GQ_TRY(device_status(word, "recon_error_hessian"));
  }
  return GQ_OK;
}

size_t gq_w4a16_workspace_size(int64_t d_out, int64_t d_in, int64_t n_tok) {
  if (d_out < 1 || d_in < 8 || d_in % 8 != 0 || n_tok < 0) return 0;
  return kWsHeader;
}

namespace {
gq_status check_product(const uint32_t *qpacked, const uint16_t *scales, const uint16_t *zeros,
                        int64_t d_out, int64_t d_in, int bits, int group_size, int sym,
                        const void *X_bf16, int64_t n_tok, void *ws, size_t ws_bytes) {
  if (qpacked && !scales) return fail(GQ_ERR_ARG, "null scales");
  if (n_tok > 0 && !X_bf16) return fail(GQ_ERR_ARG, "null X");
  if (sym != 0 && sym != 1) return fail(GQ_ERR_ARG, "sym must be 0 or 1");
  if (qpacked && sym == 0 && !zeros) return fail(GQ_ERR_ARG, "affine quantization needs zeros");
  GQ_TRY(check_layer(d_out, d_in));
  GQ_TRY(check_group(group_size, d_in));
  if (qpacked) GQ_TRY(check_bits(bits, d_in, group_size));
  if (n_tok < 0 || n_tok > (int64_t(1) << 31) - 256) return fail(GQ_ERR_SHAPE, "bad n_tok");
  if (d_out > (int64_t(1) << 31) - 256) return fail(GQ_ERR_SHAPE, "bad d_out");
  if (n_tok > 0 && !aligned(X_bf16, 16)) return fail(GQ_ERR_ARG, "X must be 16-byte aligned");
  return check_ws(ws, ws_bytes, kWsHeader);
}
}  // namespace

gq_status gq_w4a16_matmul(const uint32_t *qpacked, const uint16_t *scales,
                          const uint16_t *zeros, const int32_t *g_idx, int64_t d_out,
                          int64_t d_in, int bits, int group_size, int sym, const void *X_bf16,
                          int64_t n_tok, float *Y, void *ws, size_t ws_bytes, void *stream) {
  t_last_error.clear();
  if (!qpacked || !Y) return fail(GQ_ERR_ARG, "null pointer");
  GQ_TRY(check_product(qpacked, scales, zeros, d_out, d_in, bits, group_size, sym, X_bf16, n_tok,
                       ws, ws_bytes));
  if (!aligned(Y, 16) || n_tok % 4 != 0)
    return fail(GQ_ERR_ARG, "Y must be 16-byte aligned and n_tok a multiple of 4");
  return launch_qlinear(qpacked, scales, zeros, g_idx, nullptr, GQ_F32, d_out, d_in, bits,
                        group_size, sym, X_bf16, n_tok, Y, nullptr, nullptr, GQ_ACT_NONE,
                        static_cast<int *>(ws), static_cast<cudaStream_t>(stream));
}

gq_status gq_qlinear_bf16(const uint32_t *qpacked, const uint16_t *scales,
                          const uint16_t *zeros, const int32_t *g_idx, const void *W_dense,
                          gq_dtype w_dtype, int64_t d_out, int64_t d_in, int bits,
                          int group_size, int sym, const void *X_bf16, int64_t n_tok, int act,
                          const void *R_bf16, void *Z_bf16, void *ws, size_t ws_bytes,
                          void *stream) {
  t_last_error.clear();
  if (!Z_bf16 || (!qpacked && !W_dense)) return fail(GQ_ERR_ARG, "null pointer");
  if (!qpacked) {
    GQ_TRY(check_dtype(w_dtype));
    if (!aligned(W_dense, 16)) return fail(GQ_ERR_ARG, "W must be 16-byte aligned");
  }
  if (act != GQ_ACT_NONE && act != GQ_ACT_RELU && act != GQ_ACT_GELU)
    return fail(GQ_ERR_ARG, "act must be GQ_ACT_NONE, GQ_ACT_RELU or GQ_ACT_GELU");
  GQ_TRY(check_product(qpacked, scales, zeros, d_out, d_in, bits, group_size, sym, X_bf16, n_tok,
                       ws, ws_bytes));
  return launch_qlinear(qpacked, scales, zeros, g_idx, W_dense, w_dtype, d_out, d_in, bits,
                        group_size, sym, X_bf16, n_tok, nullptr, Z_bf16, R_bf16, act,
                        static_cast<int *>(ws), static_cast<cudaStream_t>(stream));
}

size_t gq_gptq_sequential_workspace_size(const gq_seq_layer *layers, int n_layers,
                                         int64_t n_tok, int block_size) {
  if (!layers || n_layers < 1 || n_tok < 0) return 0;
  if (block_size != 32 && block_size != 64 && block_size != 128) return 0;
  for (int l = 0; l < n_layers; ++l)
    if (layers[l].d_in < 8 || layers[l].d_in % 8 != 0 || layers[l].d_out < 1) return 0;
  return seq_ws_bytes(layers, n_layers, n_tok, block_size);
}

gq_status gq_gptq_sequential(const void *X0_bf16, int64_t n_tok, const gq_seq_layer *layers,
                             int n_layers, int bits, int group_size, int block_size, int sym,
                             float damp_percent, double *sse_dev, void *X_all_out_bf16,
                             void *ws, size_t ws_bytes, void *stream) {
  t_last_error.clear();
  if (!layers || n_layers < 1 || !sse_dev || (n_tok > 0 && !X0_bf16))
    return fail(GQ_ERR_ARG, "null pointer or no layers");
  if (n_tok < 1 || n_tok > (int64_t(1) << 31) - 256) return fail(GQ_ERR_SHAPE, "bad n_tok");
  if (sym != 0 && sym != 1) return fail(GQ_ERR_ARG, "sym must be 0 or 1");
  if (block_size != 32 && block_size != 64 && block_size != 128)
    return fail(GQ_ERR_ARG, "block_size must be 32, 64 or 128");
  if (!(damp_percent >= 0.0f) || !(damp_percent < 1e30f))
    return fail(GQ_ERR_ARG, "damp_percent must be finite and >= 0");
  if (!aligned(X0_bf16, 16)) return fail(GQ_ERR_ARG, "X0 must be 16-byte aligned");
  for (int l = 0; l < n_layers; ++l) {
    const gq_seq_layer &y = layers[l];
    GQ_TRY(check_dtype(y.w_dtype));
    if (!y.W || !y.qpacked || !y.scales || (sym == 0 && !y.zeros))
      return fail(GQ_ERR_ARG, "layer " + std::to_string(l) + ": null pointer");
    GQ_TRY(check_layer(y.d_out, y.d_in));
    GQ_TRY(check_group(group_size, y.d_in));
    GQ_TRY(check_bits(bits, y.d_in, group_size));
    if (y.d_in > 65536) return fail(GQ_ERR_SHAPE, "d_in too large");
    if (group_size > 0 && (group_size < 32 || block_size % group_size != 0))
      return fail(GQ_ERR_ARG, "group_size must be -1, 0, 32, 64 or 128 and divide block_size");
    if (bits != 4 && block_size != 128)
      return fail(GQ_ERR_ARG, "codes of other widths than 4 bits need block_size 128");
    if (l > 0 && y.d_in != layers[l - 1].d_out)
      return fail(GQ_ERR_SHAPE, "layer " + std::to_string(l) + ": d_in != previous d_out");
    if (y.act != GQ_ACT_NONE && y.act != GQ_ACT_RELU && y.act != GQ_ACT_GELU)
      return fail(GQ_ERR_ARG, "bad act");
    if (!aligned(y.W, 16)) return fail(GQ_ERR_ARG, "W must be 16-byte aligned");
    if (y.residual_from >= 0) {
      if (y.residual_from > l) return fail(GQ_ERR_ARG, "residual must be an earlier input");
      const int64_t dr = layers[y.residual_from].d_in;
      if (dr != y.d_out) return fail(GQ_ERR_SHAPE, "residual width != d_out");
    }
  }
  GQ_TRY(check_ws(ws, ws_bytes, seq_ws_bytes(layers, n_layers, n_tok, block_size)));
  return launch_sequential(X0_bf16, n_tok, layers, n_layers, bits, group_size, block_size, sym,
                           damp_percent, sse_dev, X_all_out_bf16, ws,
                           static_cast<cudaStream_t>(stream));
}

size_t gq_awq_workspace_size(int64_t d_out, int64_t d_in, int64_t n_tok, int bits,
                             int group_size, int sym) {
  if (d_out < 1 || d_in < 8 || d_in % 8 != 0 || n_tok < 1) return 0;
  if (group_size > 0 && (group_size < 8 || group_size % 8 != 0 || d_in % group_size != 0))
    return 0;
  if (group_size < -1) return 0;
  if (bits != 2 && bits != 3 && bits != 4 && bits != 8) return 0;
  return awq_ws_bytes(d_out, d_in, n_tok, group_size, sym, bits);
}

gq_status gq_awq_rtn_search(const void *W, gq_dtype w_dtype, int64_t d_out, int64_t d_in,
                            const float *H, const void *X_bf16, int64_t n_tok, int bits,
                            int group_size, int sym, int n_grid, uint32_t *qpacked,
                            uint16_t *scales, uint16_t *zeros, float *col_scale,
                            double *mse_host, int32_t *best_host, void *ws, size_t ws_bytes,
                            void *stream) {
  t_last_error.clear();
  GQ_TRY(check_dtype(w_dtype));
  if (!W || !H || !X_bf16 || !qpacked || !scales) return fail(GQ_ERR_ARG, "null pointer");
  if (sym != 0 && sym != 1) return fail(GQ_ERR_ARG, "sym must be 0 or 1");
  if (sym == 0 && !zeros) return fail(GQ_ERR_ARG, "affine quantization needs zeros");
  if (n_grid < 1 || n_grid > 256) return fail(GQ_ERR_ARG, "n_grid must be 1 .. 256");
  GQ_TRY(check_layer(d_out, d_in));
  GQ_TRY(check_group(group_size, d_in));
  GQ_TRY(check_bits(bits, d_in, group_size));
  if (n_tok < 1 || n_tok > (int64_t(1) << 31) - 256) return fail(GQ_ERR_SHAPE, "bad n_tok");
  if (!aligned(W, 16) || !aligned(X_bf16, 16))
    return fail(GQ_ERR_ARG, "W and X must be 16-byte aligned");
  GQ_TRY(check_ws(ws, ws_bytes, awq_ws_bytes(d_out, d_in, n_tok, group_size, sym, bits)));
  return launch_awq_rtn_search(W, w_dtype, d_out, d_in, H, X_bf16, n_tok, group_size, sym,
                               n_grid, qpacked, scales, zeros, col_scale, mse_host, best_host,
                               ws, static_cast<cudaStream_t>(stream), bits);
}

gq_status gq_workspace_status(const void *ws, int32_t *status_host, void *stream) {
  t_last_error.clear();
  if (!ws) return fail(GQ_ERR_ARG, "null workspace");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t word = 0;
  if (cudaMemcpyAsync(&word, ws, sizeof(word), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return check_launch("workspace_status sync");
  if (status_host) *status_host = word;
  return device_status(word, "workspace_status");
}

gq_status gq_selftest_bounded_wait(int arrive, uint64_t limit_ns, void *ws, size_t ws_bytes,
                                   void *stream) {
  t_last_error.clear();
  if (limit_ns > 1000000000ull) return fail(GQ_ERR_ARG, "limit_ns must be at most 1 s");
  GQ_TRY(check_ws(ws, ws_bytes, kWsHeader));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, kWsHeader, st) != cudaSuccess) return check_launch("memset");
  bounded_wait_kernel<<<1, 1, 0, st>>>(arrive ? 1 : 0, limit_ns, static_cast<int *>(ws));
  count_launch();
  GQ_TRY(check_launch("bounded_wait_kernel"));
  return gq_workspace_status(ws, nullptr, stream);
}

}  // extern "C"
