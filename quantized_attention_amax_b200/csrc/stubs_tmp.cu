#include "internal.cuh"
namespace faq {
cudaError_t launch_rotate_block_quant(const RotateOperand*, int, int*, cudaStream_t) { return cudaErrorNotSupported; }
}
