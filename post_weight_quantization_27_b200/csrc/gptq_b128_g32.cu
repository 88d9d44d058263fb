// Instantiation of the GPTQ column-block kernel for block 128, group 32, 4-bit codes.
#include "gptq_block.cuh"
namespace gq {
GQ_DEFINE_BLOCK(128, 32, 4)
}  // namespace gq
