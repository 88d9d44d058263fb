// Activation-aware per-channel scaling before RTN.
//
// "Model Quantization Mechanics", section 2.2: a per-channel factor s
// multiplies the weights of input channels with large activations and
// divides those activations, so that the layer's output is unchanged while
// the salient weights lose less to rounding; "GPT-2 Quantization
// Reconstruction Error", "Possible extensions": scale up important channels,
// chosen by activation magnitude, before quantising.
//
// Channel magnitude from the undamped Hessian H = 2 X^T X already on the
// device: s_c = (H_cc / H_bar)^(alpha / 2) (H_bar the geometric mean of the
// positive H_cc; s_c = 1 for a dead channel), i.e. (RMS_c / its geometric
// mean)^alpha.  For each alpha = k / n_grid the layer is quantised as
// RTN(W diag(s)) and its error ||(W - dequant diag(s)^-1) X^T||^2 measured
// with the reconstruction kernel; the alpha with the smallest error (the
// first on ties) is quantised once more into the caller's buffers.
#include <cfloat>
#include <vector>

#include "gq_device.cuh"
#include "gq_internal.h"

namespace gq {
namespace {

constexpr int kMaxGrid = 256;

// log2 H_cc for positive diagonal entries (-inf marks the others) and the
// mean of those logs, summed in fp64 in a fixed order (one block).
__global__ void __launch_bounds__(1024) awq_logdiag_kernel(const float *__restrict__ H, int64_t d,
                                                           float *__restrict__ logd,
                                                           float *__restrict__ logbar) {
  __shared__ double red[1024];
  __shared__ int cnt[1024];
  double s = 0.0;
  int c = 0;
  for (int64_t j = threadIdx.x; j < d; j += 1024) {
    const float h = H[j * d + j];
    const bool pos = h > 0.0f && h <= FLT_MAX;
    const float l = pos ? log2f(h) : -INFINITY;
    logd[j] = l;
    if (pos) {
      s += static_cast<double>(l);
      ++c;
    }
  }
  red[threadIdx.x] = s;
  cnt[threadIdx.x] = c;
  __syncthreads();
  for (int w = 512; w > 0; w >>= 1) {
    if (threadIdx.x < w) {
      red[threadIdx.x] += red[threadIdx.x + w];
      cnt[threadIdx.x] += cnt[threadIdx.x + w];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) *logbar = cnt[0] > 0 ? static_cast<float>(red[0] / cnt[0]) : 0.0f;
}

__global__ void __launch_bounds__(256) awq_colscale_kernel(const float *__restrict__ logd,
                                                           const float *__restrict__ logbar,
                                                           int64_t d, float alpha,
                                                           float *__restrict__ s,
                                                           float *__restrict__ inv) {
  const float lb = *logbar;
  for (int64_t j = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; j < d;
       j += static_cast<int64_t>(gridDim.x) * 256) {
    const float l = logd[j];
    const float sc = l == -INFINITY ? 1.0f : exp2f(0.5f * alpha * (l - lb));
    s[j] = sc;
    inv[j] = __frcp_rn(sc);
  }
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

// Wp = W diag(s) in fp32, four columns per thread step.
template <typename T>
__global__ void __launch_bounds__(256) awq_apply_kernel(const T *__restrict__ W, int64_t d_out,
                                                        int64_t d_in, const float *__restrict__ s,
                                                        float *__restrict__ Wp) {
  const int64_t n4 = d_out * d_in / 4;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; e < n4;
       e += static_cast<int64_t>(gridDim.x) * 256) {
    const int64_t i = e * 4, c = i % d_in;
    const float4 sc = *reinterpret_cast<const float4 *>(s + c);
    float4 o;
    o.x = __fmul_rn(to_f32(W[i]), sc.x);
    o.y = __fmul_rn(to_f32(W[i + 1]), sc.y);
    o.z = __fmul_rn(to_f32(W[i + 2]), sc.z);
    o.w = __fmul_rn(to_f32(W[i + 3]), sc.w);
    *reinterpret_cast<float4 *>(Wp + i) = o;
  }
}

struct AwqWs {
  float *logd, *logbar, *s, *inv, *Wp;
  uint32_t *q;
  uint16_t *sc, *z;
  double *sse;
  void *recon;
};

AwqWs carve(void *ws, int64_t d_out, int64_t d_in, int group_size, int bits) {
  const int64_t n_groups = group_size <= 0 ? 1 : d_in / group_size;
  uint8_t *p = static_cast<uint8_t *>(ws) + kWsHeader;
  AwqWs w{};
  auto take = [&](size_t bytes) {
    uint8_t *r = p;
    p += round_up(bytes, 256);
    return r;
  };
  w.logd = reinterpret_cast<float *>(take(static_cast<size_t>(d_in) * 4));
  w.logbar = reinterpret_cast<float *>(take(4));
  w.s = reinterpret_cast<float *>(take(static_cast<size_t>(d_in) * 4));
  w.inv = reinterpret_cast<float *>(take(static_cast<size_t>(d_in) * 4));
  w.Wp = reinterpret_cast<float *>(take(static_cast<size_t>(d_out) * d_in * 4));
  w.q = reinterpret_cast<uint32_t *>(take(static_cast<size_t>(d_out) * (d_in * bits / 32) * 4));
  w.sc = reinterpret_cast<uint16_t *>(take(static_cast<size_t>(d_out) * n_groups * 2));
  w.z = reinterpret_cast<uint16_t *>(take(static_cast<size_t>(d_out) * n_groups * 2));
  w.sse = reinterpret_cast<double *>(take(kMaxGrid * sizeof(double)));
  w.recon = p;
  return w;
}

// Bytes that carve() lays out before the reconstruction workspace.
size_t carve_bytes(int64_t d_out, int64_t d_in, int group_size, int bits) {
  const int64_t n_groups = group_size <= 0 ? 1 : d_in / group_size;
  return kWsHeader + 3 * round_up(static_cast<size_t>(d_in) * 4, 256) + round_up(4, 256) +
         round_up(static_cast<size_t>(d_out) * d_in * 4, 256) +
         round_up(static_cast<size_t>(d_out) * (d_in * bits / 32) * 4, 256) +
         2 * round_up(static_cast<size_t>(d_out) * n_groups * 2, 256) +
         round_up(kMaxGrid * sizeof(double), 256);
}

gq_status scale_and_quantize(const void *W, gq_dtype dt, int64_t d_out, int64_t d_in,
                             const AwqWs &w, float alpha, int group_size, int sym, uint32_t *q,
                             uint16_t *sc, uint16_t *z, cudaStream_t st, int bits) {
  const unsigned gd = static_cast<unsigned>((d_in + 255) / 256);
  awq_colscale_kernel<<<gd, 256, 0, st>>>(w.logd, w.logbar, d_in, alpha, w.s, w.inv);
  count_launch();
  int64_t g = (d_out * d_in / 4 + 255) / 256;
  const int64_t cap = static_cast<int64_t>(num_sms()) * 16;
  if (g > cap) g = cap;
  switch (dt) {
    case GQ_F32:
      awq_apply_kernel<float><<<static_cast<unsigned>(g), 256, 0, st>>>(
          static_cast<const float *>(W), d_out, d_in, w.s, w.Wp);
      break;
    case GQ_F16:
      awq_apply_kernel<__half><<<static_cast<unsigned>(g), 256, 0, st>>>(
          static_cast<const __half *>(W), d_out, d_in, w.s, w.Wp);
      break;
    case GQ_BF16:
      awq_apply_kernel<__nv_bfloat16><<<static_cast<unsigned>(g), 256, 0, st>>>(
          static_cast<const __nv_bfloat16 *>(W), d_out, d_in, w.s, w.Wp);
      break;
  }
  count_launch();
  const gq_status s = check_launch("awq scale");
  if (s != GQ_OK) return s;
  return launch_rtn(w.Wp, GQ_F32, d_out, d_in, group_size, sym, q, sc, sym ? nullptr : z, st,
                    bits);
}

}  // namespace

size_t awq_ws_bytes(int64_t d_out, int64_t d_in, int64_t n_tok, int group_size, int,
                    int bits) {
  return carve_bytes(d_out, d_in, group_size, bits) + recon_ws_bytes(d_out, d_in, n_tok);
}

gq_status launch_awq_rtn_search(const void *W, gq_dtype dt, int64_t d_out, int64_t d_in,
                                const float *H, const void *X, int64_t n_tok, int group_size,
                                int sym, int n_grid, uint32_t *qpacked, uint16_t *scales,
                                uint16_t *zeros, float *col_scale, double *mse_host,
                                int32_t *best_host, void *ws, cudaStream_t st, int bits) {
  const AwqWs w = carve(ws, d_out, d_in, group_size, bits);
  awq_logdiag_kernel<<<1, 1024, 0, st>>>(H, d_in, w.logd, w.logbar);
  count_launch();
  for (int k = 0; k < n_grid; ++k) {
    const float alpha = static_cast<float>(k) / static_cast<float>(n_grid);
    gq_status s = scale_and_quantize(W, dt, d_out, d_in, w, alpha, group_size, sym, w.q, w.sc,
                                     w.z, st, bits);
    if (s != GQ_OK) return s;
    s = launch_recon(W, dt, w.q, w.sc, sym ? nullptr : w.z, nullptr, d_out, d_in, group_size,
                     sym, X, n_tok, w.sse + k, w.recon, st, w.inv, nullptr, bits);
    if (s != GQ_OK) return s;
  }
  std::vector<double> sse(static_cast<size_t>(n_grid));
  int32_t word = 0;  // device status of the reconstruction calls
  if (cudaMemcpyAsync(sse.data(), w.sse, sizeof(double) * n_grid, cudaMemcpyDeviceToHost, st) !=
          cudaSuccess ||
      cudaMemcpyAsync(&word, w.recon, sizeof(word), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return check_launch("awq sync");
  if (word == kDevTimeout)
    return fail(GQ_ERR_TIMEOUT, "awq_rtn_search: a device-side wait gave up");
  int best = 0;
  for (int k = 1; k < n_grid; ++k)
    if (sse[k] < sse[best]) best = k;
  for (int k = 0; k < n_grid; ++k)
    if (!(sse[k] == sse[k])) return fail(GQ_ERR_NONFINITE, "non-finite reconstruction error");
  const float alpha = static_cast<float>(best) / static_cast<float>(n_grid);
  gq_status s = scale_and_quantize(W, dt, d_out, d_in, w, alpha, group_size, sym, qpacked,
                                   scales, zeros, st, bits);
  if (s != GQ_OK) return s;
  if (col_scale && cudaMemcpyAsync(col_scale, w.s, sizeof(float) * d_in,
                                   cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return check_launch("awq copy");
  if (mse_host)
    for (int k = 0; k < n_grid; ++k)
      mse_host[k] = sse[k] / (static_cast<double>(n_tok) * static_cast<double>(d_out));
  if (best_host) *best_host = best;
  return check_launch("awq_rtn_search");
}

}  // namespace gq
