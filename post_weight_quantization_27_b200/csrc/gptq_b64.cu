// Instantiations of the GPTQ column-block kernel for block 64, 4-bit codes.
#include "gptq_block.cuh"
namespace gq {
GQ_DEFINE_BLOCK(64, -1, 4)
GQ_DEFINE_BLOCK(64, 64, 4)
GQ_DEFINE_BLOCK(64, 32, 4)
}  // namespace gq
