// Instantiation of the GPTQ column-block kernel for block 128, group -1, 4-bit codes.
#include "gptq_block.cuh"
namespace gq {
GQ_DEFINE_BLOCK(128, -1, 4)
}  // namespace gq
