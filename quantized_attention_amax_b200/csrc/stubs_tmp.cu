#include "internal.cuh"
namespace faq {
cudaError_t launch_rotate_block_quant(const RotateOperand*, int, int*, cudaStream_t) { return cudaErrorNotSupported; }
size_t decode_workspace_bytes(int B, int Hq, int D, int splits) { return (size_t)B * Hq * splits * (D + 2) * 4; }
int decode_auto_splits(int, int, int) { return 1; }
cudaError_t launch_attention_decode(const AttnArgs&, int, void*, cudaStream_t) { return cudaErrorNotSupported; }
}
