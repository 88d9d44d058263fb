// Instantiation of the GPTQ column-block kernel for block 128, group 64.
#include "gptq_block.cuh"
namespace gq {
GQ_DEFINE_BLOCK(128, 64)
}  // namespace gq
