// Instantiations of the GPTQ column-block kernel for block 128 with 8-bit
// codes (per channel, groups of 128, 64 and 32).
#include "gptq_block.cuh"
namespace gq {
GQ_DEFINE_BLOCK(128, -1, 8)
GQ_DEFINE_BLOCK(128, 128, 8)
GQ_DEFINE_BLOCK(128, 64, 8)
GQ_DEFINE_BLOCK(128, 32, 8)
}  // namespace gq
