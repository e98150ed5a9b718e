// attn_common.cuh -- device helpers shared by the prefill attention kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "internal.cuh"
#include "sm100.cuh"

namespace faq {
namespace attn {

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Packed two-lane fp32 arithmetic (sm_100 f32x2 forms): one instruction per pair.
__device__ __forceinline__ void fmul2(float& a0, float& a1, float b0, float b1) {
  asm("{\n\t.reg .b64 x, y;\n\tmov.b64 x, {%0, %1};\n\tmov.b64 y, {%2, %3};\n\t"
      "mul.rn.ftz.f32x2 x, x, y;\n\tmov.b64 {%0, %1}, x;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "f"(b0), "f"(b1));
}
__device__ __forceinline__ void ffma2(float& a0, float& a1, float b0, float b1, float c0, float c1) {
  asm("{\n\t.reg .b64 x, y, z;\n\tmov.b64 x, {%0, %1};\n\tmov.b64 y, {%2, %3};\n\tmov.b64 z, {%4, %5};\n\t"
      "fma.rn.ftz.f32x2 x, x, y, z;\n\tmov.b64 {%0, %1}, x;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
__device__ __forceinline__ void fadd2(float& a0, float& a1, float b0, float b1) {
  asm("{\n\t.reg .b64 x, y;\n\tmov.b64 x, {%0, %1};\n\tmov.b64 y, {%2, %3};\n\t"
      "add.rn.ftz.f32x2 x, x, y;\n\tmov.b64 {%0, %1}, x;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "f"(b0), "f"(b1));
}

// 2^x for a pair on the FMA pipe (takes load off the MUFU unit, which runs ex2
// at a quarter of the FMA rate): x = n + f with n = rint(x), f in [-0.5, 0.5];
// 2^f from a cubic fitted for least maximum relative error on that interval
// (Lawson's iteratively reweighted least squares, C. L. Lawson, "Contributions to
// the theory of linear least maximum approximation", 1961; the fit and its fp32
// error check are fit_ex2_cubic.py beside this file), 7.5e-5 relative error in
// fp32 -- below half an fp16 ulp, the precision P' is stored in; 2^n enters
// through the exponent field.  x is clamped at -126: p(f) >= 2^-0.5 has a biased exponent of
// at least 126, so n >= -126 never borrows past the exponent field (the result
// for x <= -126 is a denormal, read as 0 downstream).
__device__ __forceinline__ void ex2_poly2(float& a, float& b) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23: x + kRound holds rint(x) in its low mantissa bits
  float x0 = fmaxf(a, -126.0f), x1 = fmaxf(b, -126.0f);
  float j0 = x0, j1 = x1;
  fadd2(j0, j1, kRound, kRound);
  float n0 = j0, n1 = j1;
  fadd2(n0, n1, -kRound, -kRound);
  float f0 = x0, f1 = x1;
  fadd2(f0, f1, -n0, -n1);
  float p0 = 5.517132208e-02f, p1 = 5.517132208e-02f;
  ffma2(p0, p1, f0, f1, 2.426105440e-01f, 2.426105440e-01f);
  ffma2(p0, p1, f0, f1, 6.932609677e-01f, 6.932609677e-01f);
  ffma2(p0, p1, f0, f1, 9.999281168e-01f, 9.999281168e-01f);
  a = __int_as_float(__float_as_int(p0) + (__float_as_int(j0) << 23));
  b = __int_as_float(__float_as_int(p1) + (__float_as_int(j1) << 23));
}

// max(a, b, c) in one instruction (sm_100 three-input form).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Every lane waits; the warp proceeds only if all lanes saw the phase complete.
__device__ __forceinline__ bool warp_wait(uint64_t* b, uint32_t parity, volatile int* abort_flag, int* status,
                                          int where) {
  const bool ok = mbar_wait(b, parity, abort_flag, status, where);
  return __all_sync(0xffffffffu, ok);
}

// blk < 0: no scale (operands whose scales are already applied)
__device__ __forceinline__ float scale_at(const float* s, int blk, int nblk, int bh, int h, int tok) {
  return blk < 0 ? 1.0f : blk == 0 ? __ldg(s + h) : __ldg(s + (long long)bh * nblk + tok / blk);
}

// Two E4M3 codes -> two fp16 (exact).  Low byte -> low half.
__device__ __forceinline__ uint32_t e4m3x2_to_h2(uint16_t v) {
  uint32_t r;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(v));
  return r;
}
// Two E2M1 codes (one byte, low nibble first) -> two fp16 (exact).
__device__ __forceinline__ uint32_t e2m1x2_to_h2(uint32_t byte) {
  uint32_t r;
  asm("{ .reg .b8 b; cvt.u8.u32 b, %1; cvt.rn.f16x2.e2m1x2 %0, b; }" : "=r"(r) : "r"(byte));
  return r;
}

// Copy a 128-row x 4-byte scale-factor atom (byte (m % 32) * 16 + (m / 32) * 4
// + k) from shared memory into TMEM lanes m % 32 of every lane quarter,
// column m / 32, byte k -- the layout block-scaled tcgen05.mma reads.
__device__ __forceinline__ void sf_to_tmem(uint32_t taddr, uint32_t saddr) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr),
               "l"(make_sdesc(saddr, 16, 128, kSwzNone))
               : "memory");
}

// 32 lanes write the scale atom of 128 token rows from E8M0 [rows][4];
// rows at or past `valid` get byte 0 (their codes are zero-filled).
__device__ __forceinline__ void write_sf_atom(uint8_t* atom, const uint8_t* e8, long long row0, int valid, int lane) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int m = lane * 4 + q;
    uint32_t v = 0;
    if (m < valid) v = __ldg(reinterpret_cast<const uint32_t*>(e8 + (row0 + m) * 4));
    *reinterpret_cast<uint32_t*>(atom + (m & 31) * 16 + (m >> 5) * 4) = v;
  }
}

// Two int8 codes -> two fp16 (exact): fp16(1024 + u) - 1152 with u = c + 128.
__device__ __forceinline__ uint32_t s8x2_to_h2(uint32_t w_biased, int sel) {
  const uint32_t h = __byte_perm(w_biased, 0x6464u, sel);
  const __half2 v = __hsub2(*reinterpret_cast<const __half2*>(&h), __halves2half2(__ushort_as_half(0x6480), __ushort_as_half(0x6480)));
  return *reinterpret_cast<const uint32_t*>(&v);
}


// 4D tensor map over token rows of D_bytes bytes (8-bit codes, or bf16 rows read as bytes):
// (row bytes, rows of the layout...), boxes of box_bytes (default: the whole row) x box_rows.
inline cudaError_t make_code_map(CUtensorMap* map, const void* base, int B, int H, int S, int D_bytes, int layout,
                          int box_rows, int box_bytes = 0) {
  const int bb = box_bytes > 0 ? box_bytes : D_bytes;
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return cudaErrorNotSupported;
  cuuint64_t dims[4], strides[3];
  cuuint32_t box[4], es[4] = {1, 1, 1, 1};
  if (layout == FA_LAYOUT_BNSD) {
    dims[0] = D_bytes; dims[1] = S; dims[2] = H; dims[3] = B;
    strides[0] = (cuuint64_t)D_bytes; strides[1] = (cuuint64_t)S * D_bytes; strides[2] = (cuuint64_t)H * S * D_bytes;
    box[0] = bb; box[1] = box_rows; box[2] = 1; box[3] = 1;
  } else {
    dims[0] = D_bytes; dims[1] = H; dims[2] = S; dims[3] = B;
    strides[0] = (cuuint64_t)D_bytes; strides[1] = (cuuint64_t)H * D_bytes; strides[2] = (cuuint64_t)S * H * D_bytes;
    box[0] = bb; box[1] = 1; box[2] = box_rows; box[3] = 1;
  }
  const CUtensorMapSwizzle swz = bb == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                 : bb == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                            : CU_TENSOR_MAP_SWIZZLE_32B;
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}


}  // namespace attn
}  // namespace faq
