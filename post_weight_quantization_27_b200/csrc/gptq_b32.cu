// Instantiations of the GPTQ column-block kernel for block 32.
#include "gptq_block.cuh"
namespace gq {
GQ_DEFINE_BLOCK(32, -1)
GQ_DEFINE_BLOCK(32, 32)
}  // namespace gq
