// Instantiation of the GPTQ column-block kernel for block 128, group 128.
#include "gptq_block.cuh"
namespace gq {
GQ_DEFINE_BLOCK(128, 128)
}  // namespace gq
