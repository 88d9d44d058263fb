// Instantiations of the GPTQ column-block kernel for block 128 with 2-bit
// codes (per channel, groups of 128, 64 and 32).
#include "gptq_block.cuh"
namespace gq {
GQ_DEFINE_BLOCK(128, -1, 2)
GQ_DEFINE_BLOCK(128, 128, 2)
GQ_DEFINE_BLOCK(128, 64, 2)
GQ_DEFINE_BLOCK(128, 32, 2)
}  // namespace gq
