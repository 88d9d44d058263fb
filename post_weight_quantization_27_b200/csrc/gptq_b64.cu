// Instantiations of the GPTQ column-block kernel for block 64.
#include "gptq_block.cuh"
namespace gq {
GQ_DEFINE_BLOCK(64, -1)
GQ_DEFINE_BLOCK(64, 64)
GQ_DEFINE_BLOCK(64, 32)
}  // namespace gq
