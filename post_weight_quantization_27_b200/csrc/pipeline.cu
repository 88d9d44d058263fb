// Layers quantised one after another on the inputs they actually receive.
//
// "GPT-2 Quantization Reconstruction Error" -- "Key findings": the per-layer
// errors were measured with the whole model running, so a layer's input
// already carries the error of the quantised layers before it.  Here layer
// l is calibrated on X_l, the output of the quantised layers 0 .. l-1:
//   H0 = 2 X_l^T X_l; damping and U; GPTQ of W_l; the layer error
//   tr(dW H0 dW^T) / 2 = ||(W_l - W^_l) X_l^T||^2; then
//   X_{l+1} = act(X_l W^_l^T) (+ X_j), computed from the packed codes.
// Host orchestration of the library's own launches, all on one stream; the
// inputs X_0 .. X_n stay in the workspace (a residual may reach back).
#include <algorithm>
#include <vector>

#include "gq_device.cuh"
#include "gq_internal.h"

namespace gq {
namespace {

struct SeqLayout {
  std::vector<size_t> off_x;  // X_0 .. X_n (bf16)
  size_t off_h0, off_h, off_u, off_dead, off_scratch, total;
  size_t scratch;
};

SeqLayout seq_layout(const gq_seq_layer *layers, int n, int64_t n_tok, int block_size) {
  SeqLayout L{};
  size_t off = kWsHeader;
  int64_t d_max = 0;
  size_t scratch = kWsHeader;
  for (int l = 0; l <= n; ++l) {
    const int64_t d = l < n ? layers[l].d_in : layers[n - 1].d_out;
    L.off_x.push_back(off);
    off += round_up(static_cast<size_t>(n_tok) * d * 2, 256);
  }
  for (int l = 0; l < n; ++l) {
    const int64_t di = layers[l].d_in, dout = layers[l].d_out;
    d_max = std::max(d_max, di);
    scratch = std::max({scratch, hessian_plan(n_tok, di).ws_bytes, chol_ws_bytes(di),
                        gptq_ws_bytes(dout, di, block_size), recon_hessian_ws_bytes(dout, di)});
  }
  const size_t dd = round_up(static_cast<size_t>(d_max) * d_max * sizeof(float), 256);
  L.off_h0 = off;
  L.off_h = off + dd;
  L.off_u = off + 2 * dd;
  L.off_dead = off + 3 * dd;
  L.off_scratch = L.off_dead + round_up(static_cast<size_t>(d_max), 256);
  L.scratch = round_up(scratch, 256);
  L.total = L.off_scratch + L.scratch;
  return L;
}

}  // namespace

size_t seq_ws_bytes(const gq_seq_layer *layers, int n_layers, int64_t n_tok, int block_size) {
  return seq_layout(layers, n_layers, n_tok, block_size).total;
}

gq_status launch_sequential(const void *X0, int64_t n_tok, const gq_seq_layer *layers, int n,
                            int bits, int group_size, int block_size, int sym, float damp,
                            double *sse_dev, void *X_all, void *ws, cudaStream_t st) {
  const SeqLayout L = seq_layout(layers, n, n_tok, block_size);
  uint8_t *base = static_cast<uint8_t *>(ws);
  int *status = reinterpret_cast<int *>(base);
  auto xbuf = [&](int l) { return static_cast<void *>(base + L.off_x[l]); };
  float *H0 = reinterpret_cast<float *>(base + L.off_h0);
  float *H = reinterpret_cast<float *>(base + L.off_h);
  float *U = reinterpret_cast<float *>(base + L.off_u);
  void *scr = base + L.off_scratch;
  if (cudaMemsetAsync(status, 0, kWsHeader, st) != cudaSuccess) return check_launch("memset");
  if (cudaMemcpyAsync(xbuf(0), X0, static_cast<size_t>(n_tok) * layers[0].d_in * 2,
                      cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return check_launch("copy X0");
  for (int l = 0; l < n; ++l) {
    const gq_seq_layer &y = layers[l];
    const int64_t di = y.d_in, dout = y.d_out;
    gq_status s = launch_hessian(xbuf(l), n_tok, di, H0, scr, hessian_plan(n_tok, di), st, false);
    if (s != GQ_OK) return s;
    if (cudaMemcpyAsync(H, H0, static_cast<size_t>(di) * di * sizeof(float),
                        cudaMemcpyDeviceToDevice, st) != cudaSuccess)
      return check_launch("copy H");
    // damping, dead columns (an input channel that is zero on every token)
    // and U; GPTQ zeroes the dead columns' weights
    uint8_t *dead = base + L.off_dead;
    s = launch_damp_chol(H, di, damp, 0, nullptr, dead, U, nullptr, scr, st, false);
    if (s != GQ_OK) return s;
    s = launch_gptq(y.W, y.w_dtype, dout, di, U, group_size, block_size, sym, nullptr, dead,
                    y.qpacked, y.scales, sym ? nullptr : y.zeros, nullptr, scr, st, bits);
    if (s != GQ_OK) return s;
    s = launch_recon_hessian(y.W, y.w_dtype, y.qpacked, y.scales, sym ? nullptr : y.zeros,
                             nullptr, dout, di, group_size, sym, H0, sse_dev + l, scr, st, bits);
    if (s != GQ_OK) return s;
    const void *R = y.residual_from >= 0 ? xbuf(y.residual_from) : nullptr;
    s = launch_qlinear(y.qpacked, y.scales, sym ? nullptr : y.zeros, nullptr, nullptr, GQ_F32,
                       dout, di, bits, group_size, sym, xbuf(l), n_tok, nullptr, xbuf(l + 1), R,
                       y.act, reinterpret_cast<int *>(scr), st);
    if (s != GQ_OK) return s;
  }
  if (X_all) {  // every input X_0 .. X_n, one after another (as the workspace holds them)
    size_t off = 0;
    for (int l = 0; l <= n; ++l) {
      const int64_t dl = l < n ? layers[l].d_in : layers[n - 1].d_out;
      const size_t bytes = static_cast<size_t>(n_tok) * dl * 2;
      if (cudaMemcpyAsync(static_cast<uint8_t *>(X_all) + off, xbuf(l), bytes,
                          cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return check_launch("copy X_all");
      off += bytes;
    }
  }
  return check_launch("gptq_sequential");
}

}  // namespace gq
