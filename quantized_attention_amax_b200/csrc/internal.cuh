// internal.cuh -- declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "faq.h"

namespace faq {

// One operand of a quantize launch: bf16 input rows -> codes + scales.
struct QuantOperand {
  const void* x;       // bf16 input
  void* codes;         // output codes
  void* scales;        // output scales (fp32 or E8M0 bytes)
  const float* amax;   // INT8 per head: calibration maxima [H]
  long long rows;      // B * H * S
  int B, H, S, D;
  int layout;
  int blk;             // FP8 block: tokens per block
  // row -> head by multiply-high division (filled by the row quantizer's launcher)
  uint32_t mS, mH;     // magic multipliers for S and H
  int lS, lH;          // their shifts
};

// Per-device status word (timeouts recorded by bounded waits; failed index checks in
// FA_DEBUG_BOUNDS builds).
int* device_status_ptr();

// FA_DEBUG_BOUNDS builds: point this translation unit's index checks at the device status word
// (once per device); a no-op otherwise.  Each launcher calls it before its launches.
#ifdef FA_DEBUG_BOUNDS
inline cudaError_t bounds_attach_impl(const void* symbol) {
  static int done[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 64) return e;
  if (done[dev]) return cudaSuccess;
  int* p = device_status_ptr();
  if (!p) return cudaErrorUnknown;
  if ((e = cudaMemcpyToSymbol(symbol, &p, sizeof p)) != cudaSuccess) return e;
  done[dev] = 1;
  return cudaSuccess;
}
#define bounds_attach() bounds_attach_impl(reinterpret_cast<const void*>(&g_bounds_status))
#else
#define bounds_attach() cudaSuccess
#endif

// Driver entry point for tensor-map encoding (resolved once).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled_fn();

// Number of SMs of the current device (cached).
int sm_count();

// Raise a kernel's dynamic shared memory limit to `bytes` on the current device.  The attribute
// belongs to one device, so it is set once per (kernel, device) pair, under a lock.
cudaError_t set_smem_limit(const void* kernel, int bytes);

// Launchers (quant.cu).
cudaError_t launch_calibrate(const QuantOperand& op, float* amax, cudaStream_t s);
cudaError_t launch_quantize_rows(int mode, const QuantOperand* ops, int nops, cudaStream_t s);
cudaError_t launch_quantize_fp8_block(const QuantOperand* ops, int nops, cudaStream_t s);

// Launchers (rotate.cu).
struct RotateOperand {
  const void* x;       // bf16 input [.., D]
  const void* R;       // bf16 [D, D] or nullptr (no rotation, unless hadamard)
  void* codes;         // e4m3
  float* scales;       // [B, H, nblk]
  void* dbg;           // nullable bf16 rotated output
  int B, H, S, D, layout, blk;
  // R = bf16(H_D diag(sigma) / sqrt(D)) generated in shared memory from the signs (R unused)
  int hadamard;
  uint32_t sign_bits[4];  // bit j set: sigma_j = -1
};
cudaError_t launch_rotate_block_quant(const RotateOperand* ops, int nops, int* status, cudaStream_t s);

// Launcher (hadamard.cu): rotation R = bf16(H_D diag(sigma) / sqrt(D)) by a fast Walsh-Hadamard
// transform (rotate = 1) or none (rotate = 0), then FP8 block quantization.
struct HadamardOperand {
  const void* x;          // bf16 input [.., D]
  void* codes;            // e4m3
  float* scales;          // [B, H, nblk]
  void* dbg;              // nullable bf16 rotated output
  uint32_t sign_bits[4];  // bit j set: sigma_j = -1 (D / 32 words used)
  int B, H, S, D, layout, blk, rotate;
};
cudaError_t launch_hadamard_block_quant(const HadamardOperand* ops, int nops, cudaStream_t s);

// Launchers (attn2.cu / decode.cu).
struct AttnArgs {
  const fa_qtensor* q;
  const fa_qtensor* k;
  const fa_qtensor* v;
  int causal;
  float softmax_scale;
  void* out;
  float* lse;
  int* status;
};
// Prefill (E4M3, INT8, MXFP4): V' pre-pass + attention; `ws` holds prefill2_workspace_bytes(), sized for
// key tiles of `tile_keys` keys (prefill_tile_keys(Q's mode): 112 for the MX modes, 128 otherwise).
size_t prefill2_workspace_bytes(int B, int Hkv, int Sk, int D, int tile_keys = 128);
int prefill_tile_keys(int q_mode);
cudaError_t launch_attention_prefill2(const AttnArgs& a, void* ws, cudaStream_t s);
// Mixed branches (modes differ, or a branch is not quantized): bf16 Q / K pair kernel;
// `ws` holds mixed_workspace_bytes(q, k).
size_t mixed_workspace_bytes(const fa_qtensor* q, const fa_qtensor* k);
cudaError_t launch_attention_mixed(const AttnArgs& a, void* ws, cudaStream_t s);

size_t decode_workspace_bytes(int B, int Hq, int D, int splits);
int decode_auto_splits(int B, int Hkv, int Sk);
cudaError_t launch_attention_decode(const AttnArgs& a, int splits, void* ws, cudaStream_t s);

// Decode with the new token appended to an INT8 per-head cache in the same kernel.
struct DecodeAppendArgs {
  const fa_tensor* q;      // bf16 [B, Hq, 1, D]
  const fa_tensor* k_new;  // bf16 [B, Hkv, 1, D]
  const fa_tensor* v_new;
  const float* amax_q;
  const float* amax_k;
  const float* amax_v;
  const fa_qtensor* k_cache;  // S = capacity
  const fa_qtensor* v_cache;
  int pos;
  float softmax_scale;
  void* out;
  float* lse;
  int* status;
};
cudaError_t launch_decode_append(const DecodeAppendArgs& a, int splits, void* ws, cudaStream_t s);

cudaError_t launch_fill_empty_rows(void* out, float* lse, long long rows, int D, cudaStream_t s);

}  // namespace faq
