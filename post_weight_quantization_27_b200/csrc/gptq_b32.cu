// Instantiations of the GPTQ column-block kernel for block 32, 4-bit codes.
#include "gptq_block.cuh"
namespace gq {
GQ_DEFINE_BLOCK(32, -1, 4)
GQ_DEFINE_BLOCK(32, 32, 4)
}  // namespace gq
