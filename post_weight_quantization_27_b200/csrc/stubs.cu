// Temporary placeholders for kernels not written yet.
#include "gq_device.cuh"
#include "gq_internal.h"
namespace gq {
size_t chol_ws_bytes(int64_t d) { return kWsHeader + 16; }
gq_status launch_damp_chol(float *, int64_t, float, int, int32_t *, uint8_t *, float *, int32_t *,
                           void *, cudaStream_t) {
  return fail(GQ_ERR_ARG, "not built yet");
}
size_t gptq_ws_bytes(int64_t, int64_t, int) { return kWsHeader; }
gq_status launch_gptq(const void *, gq_dtype, int64_t, int64_t, const float *, int, int, int,
                      const int32_t *, const uint8_t *, uint32_t *, uint16_t *, uint16_t *,
                      int32_t *, void *, cudaStream_t) {
  return fail(GQ_ERR_ARG, "not built yet");
}
size_t recon_ws_bytes(int64_t, int64_t, int64_t) { return kWsHeader; }
gq_status launch_recon(const void *, gq_dtype, const uint32_t *, const uint16_t *,
                       const uint16_t *, const int32_t *, int64_t, int64_t, int, int,
                       const void *, int64_t, double *, void *, cudaStream_t) {
  return fail(GQ_ERR_ARG, "not built yet");
}
}  // namespace gq
