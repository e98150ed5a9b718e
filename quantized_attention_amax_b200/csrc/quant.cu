// quant.cu -- HBM-bound quantization kernels for FA quantization:
//   calibrate_kernel          running per-head max |x|        (wiki "FA 量化", 组合1)
//   quant_rows_kernel<MODE>   one pass over token rows:
//       INT8 per head   code = sat8(rne(x / s_h)), s_h = amax_h / 127  (组合1)
//       FP8 per token   s = amax_row / 448, code = e4m3(x / s)        (组合2)
//       MXFP4           per 32 elements: e = floor(log2 amax) - 2,
//                       code = e2m1(x * 2^-e), E8M0 byte e + 127      (组合3)
//       FP8 per head    s_h = amax_h / 448 (static, calibrated)       (模式清单: FA PerHead)
//       INT8 per token  s = amax_row / 127                            (模式清单: FA PerToken)
//       MXFP8           as MXFP4 with e = floor(log2 amax) - 8 and E4M3 elements
//                                                                     (模式清单: FA PerBlock)
//   fp8_block_kernel          one scale = amax / 448 per block of tokens
//                             (MindIE SD "量化", FA量化 / 块量化)
// Rows are D contiguous bf16 values in either layout; each row is handled by
// D/32 lanes with four 16-byte loads each.  x / s is rounded as IEEE division
// (div.rn.f32) rounds it, so the codes match a correctly rounded x / s exactly:
// the FMA-corrected reciprocal products of quant_common.cuh (checked against
// IEEE division exhaustively), IEEE division itself for scales below 2^-90.
#include <cuda_bf16.h>

#include "internal.cuh"
#include "quant_common.cuh"
#include "sm100.cuh"

namespace faq {
namespace {

// per half: max(|a|, |b|), its sign the XOR of the inputs' signs (exact; only magnitudes are used)
__device__ __forceinline__ uint32_t bf16x2_absmax(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ void unpack_bf16x8(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// Four fp32 values -> four E4M3 bytes (a in the lowest byte), RNE, saturating.
__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  uint16_t lo, hi;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(b), "f"(a));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(d), "f"(c));
  return (uint32_t)lo | ((uint32_t)hi << 16);
}

// Eight fp32 values -> eight E2M1 nibbles (v[0] in the lowest nibble).
__device__ __forceinline__ uint32_t e2m1x8(const float (&v)[8]) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  return r;
}

// Int8 codes of four quotients, rounded half to even, on the FMA / ALU pipes (a float-to-integer
// conversion would run on the quarter-rate XU pipe): adding 1.5 * 2^23 rounds to an integer in
// the low mantissa bits (exact for |x| < 2^22), whose low byte is the two's-complement code;
// three byte permutes pack the four codes.  SAT (static scales, which data can exceed): NaN -> 0
// as a conversion gives, then a clamp to [-128, 127] (before or after rounding gives the same
// integer, the bounds being integers).  Without SAT (per-token scales) |x / s| <= 127 holds by
// construction, so no clamp is needed.
template <bool SAT>
__device__ __forceinline__ uint32_t s8x4(float a, float b, float c, float d) {
  if (SAT) {
    a = fminf(fmaxf(a == a ? a : 0.0f, -128.0f), 127.0f);
    b = fminf(fmaxf(b == b ? b : 0.0f, -128.0f), 127.0f);
    c = fminf(fmaxf(c == c ? c : 0.0f, -128.0f), 127.0f);
    d = fminf(fmaxf(d == d ? d : 0.0f, -128.0f), 127.0f);
  }
  constexpr float kMagic = 12582912.0f;
  asm("{\n\t.reg .b64 x, y, m;\n\tmov.b64 x, {%0, %1};\n\tmov.b64 y, {%2, %3};\n\tmov.b64 m, {%4, %4};\n\t"
      "add.rn.f32x2 x, x, m;\n\tadd.rn.f32x2 y, y, m;\n\tmov.b64 {%0, %1}, x;\n\tmov.b64 {%2, %3}, y;\n\t}"
      : "+f"(a), "+f"(b), "+f"(c), "+f"(d)
      : "f"(kMagic));
  const uint32_t ab = __byte_perm(__float_as_uint(a), __float_as_uint(b), 0x0040);  // low bytes of a, b
  const uint32_t cd = __byte_perm(__float_as_uint(c), __float_as_uint(d), 0x0040);
  return __byte_perm(ab, cd, 0x5410);
}

// max(|a|, |b|) per half as above, but a NaN in either input gives NaN
__device__ __forceinline__ uint32_t bf16x2_absmax_nan(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// n / d for n < 2^32 by one multiply-high (T. Granlund and P. L. Montgomery, "Division by
// invariant integers using multiplication", PLDI 1994, unsigned case): m and l from fastdiv_magic.
__device__ __forceinline__ uint32_t fast_div(uint32_t n, uint32_t m, int l) {
  return (uint32_t)(((unsigned long long)__umulhi(n, m) + n) >> l);
}

// Canonical [B, H, S] index of token row r of the data layout.
__device__ __forceinline__ long long scale_index(long long r, int layout, int H, int S) {
  if (layout == FA_LAYOUT_BNSD) return r;
  const long long h = r % H, bs = r / H;
  return ((bs / S) * H + h) * S + (bs % S);
}

// Exponent e of the MX shared scale: floor(log2 amax) - EMAX (2 for E2M1, 8 for E4M3 elements),
// clamped to [-127, 127]; amax == 0 or an fp32-subnormal amax gives -127.
template <int EMAX>
__device__ __forceinline__ int mx_exponent(float amax) {
  const int E = (int)((__float_as_uint(amax) >> 23) & 0xFF);
  if (E == 0) return -127;
  return max(-127, min(127, E - 127 - EMAX));
}

// One row = D / 32 lanes; each lane owns 32 consecutive elements (one MX block): four 16-byte
// loads, so the per-row work (the scale, its reciprocal, the lane shuffles, the addresses) is
// shared by 32 elements per lane.
constexpr int kRowThreads = 256;

template <int MODE, int D>
__global__ void __launch_bounds__(kRowThreads) quant_rows_kernel(QuantOperand o0, QuantOperand o1, QuantOperand o2) {
  constexpr int LPR = D / 32;  // lanes per row
  constexpr int RPW = 32 / LPR;  // rows per warp
  const int lane = threadIdx.x & 31;
  const int gl = lane % LPR;   // 32-element chunk of the row
  const int sub = lane / LPR;

  // per-head static modes: one scale per head from the calibration maxima
  constexpr bool PER_HEAD = MODE == FA_MODE_INT8_PER_HEAD || MODE == FA_MODE_FP8_PER_HEAD;
  constexpr bool INT8 = MODE == FA_MODE_INT8_PER_HEAD || MODE == FA_MODE_INT8_PER_TOKEN;
  constexpr bool MX = MODE == FA_MODE_MXFP4_PER_BLOCK || MODE == FA_MODE_MXFP8_PER_BLOCK;
  constexpr float QMAX = INT8 ? 127.0f : 448.0f;
  if (PER_HEAD && blockIdx.x == 0) {
    for (int t = threadIdx.x; t < o0.H && o0.rows > 0; t += blockDim.x)
      static_cast<float*>(o0.scales)[t] = __fdiv_rn(o0.amax[t], QMAX);
    for (int t = threadIdx.x; t < o1.H && o1.rows > 0; t += blockDim.x)
      static_cast<float*>(o1.scales)[t] = __fdiv_rn(o1.amax[t], QMAX);
    for (int t = threadIdx.x; t < o2.H && o2.rows > 0; t += blockDim.x)
      static_cast<float*>(o2.scales)[t] = __fdiv_rn(o2.amax[t], QMAX);
  }

  const long long rows0 = o0.rows, rows01 = o0.rows + o1.rows;
  const long long total = rows01 + o2.rows;
  const long long nwarps = (long long)gridDim.x * (blockDim.x / 32);
  const long long wid = ((long long)blockIdx.x * blockDim.x + threadIdx.x) / 32;

  for (long long r = wid * RPW + sub; r - sub < total; r += nwarps * RPW) {
    const bool valid = r < total;  // the same for every lane of the row
    const int which = r < rows0 ? 0 : (r < rows01 ? 1 : 2);
    const long long rr = which == 0 ? r : (which == 1 ? r - rows0 : r - rows01);
    // the row's operand, field by field (no address of a kernel parameter is taken)
    const void* const op_x = which == 0 ? o0.x : (which == 1 ? o1.x : o2.x);
    void* const op_codes = which == 0 ? o0.codes : (which == 1 ? o1.codes : o2.codes);
    void* const op_scales = which == 0 ? o0.scales : (which == 1 ? o1.scales : o2.scales);
    uint4 raw[4];
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(op_x) + rr * D) + gl * 4;
    const long long op_rows = which == 0 ? o0.rows : (which == 1 ? o1.rows : o2.rows);
    const bool ld_ok = valid && in_bounds(rr * D + (gl + 1) * 32 <= op_rows * D, 101);
#pragma unroll
    for (int c = 0; c < 4; ++c) raw[c] = ld_ok ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
    // max |x| over the lane's 32 elements on the packed bf16 pairs (exact, no unpacking)
    float m = 0.0f;
    if (!PER_HEAD) {
      uint32_t m2 = 0;
#pragma unroll
      for (int c = 0; c < 4; ++c)
        m2 = bf16x2_absmax(bf16x2_absmax(m2, bf16x2_absmax(raw[c].x, raw[c].y)), bf16x2_absmax(raw[c].z, raw[c].w));
      m2 &= 0x7FFF7FFFu;
      m = fmaxf(__uint_as_float(m2 << 16), __uint_as_float(m2 & 0xFFFF0000u));
      if (!MX) {
#pragma unroll
        for (int off = LPR / 2; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
      }
    }
    uint4 out[2];
    if (MX) {
      // one 32-element block per lane: e = floor(log2 amax) - emax, x * 2^-e exact
      const int e = mx_exponent<MODE == FA_MODE_MXFP8_PER_BLOCK ? 8 : 2>(m);
      const float inv = __uint_as_float((uint32_t)(127 - e) << 23);
      if (valid) {
        if (MODE == FA_MODE_MXFP8_PER_BLOCK) {
          uint32_t w[8];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            float f[8];
            unpack_bf16x8(raw[c], f);
            w[2 * c] = e4m3x4(f[0] * inv, f[1] * inv, f[2] * inv, f[3] * inv);
            w[2 * c + 1] = e4m3x4(f[4] * inv, f[5] * inv, f[6] * inv, f[7] * inv);
          }
          uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(op_codes) + rr * D + gl * 32);
          if (in_bounds(rr * D + (gl + 1) * 32 <= op_rows * D, 102)) {
            dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
            dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
          }
        } else {
          uint32_t w[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            float v8[8];
            unpack_bf16x8(raw[i], v8);
#pragma unroll
            for (int k = 0; k < 8; ++k) v8[k] *= inv;
            w[i] = e2m1x8(v8);
          }
          if (in_bounds(rr * (D / 2) + (gl + 1) * 16 <= op_rows * (D / 2), 103))
            *reinterpret_cast<uint4*>(static_cast<uint8_t*>(op_codes) + rr * (D / 2) + gl * 16) =
                make_uint4(w[0], w[1], w[2], w[3]);
        }
        const int op_layout = which == 0 ? o0.layout : (which == 1 ? o1.layout : o2.layout);
        const int op_H = which == 0 ? o0.H : (which == 1 ? o1.H : o2.H);
        const int op_S = which == 0 ? o0.S : (which == 1 ? o1.S : o2.S);
        const long long si = scale_index(rr, op_layout, op_H, op_S) * (D / 32) + gl;
        if (in_bounds(si >= 0 && si < op_rows * (D / 32), 104)) static_cast<uint8_t*>(op_scales)[si] = (uint8_t)(e + 127);
      }
      continue;
    }
    // one scale per row (dynamic modes) or per head (static modes)
    float sc = 0.0f, rc = 0.0f;
    // bounded: every |x| of the warp's rows is within its scale's maximum, so the INT8 quotients
    // need neither the overflow guard nor the clamp (dynamic scales: by construction)
    bool bounded = !PER_HEAD;
    if (PER_HEAD) {
      float lim = -1.0f;
      if (valid) {
        const int op_layout = which == 0 ? o0.layout : (which == 1 ? o1.layout : o2.layout);
        const int op_H = which == 0 ? o0.H : (which == 1 ? o1.H : o2.H);
        // row -> head in 32 bits (rows < 2^32, checked by the launcher)
        const uint32_t r32 = (uint32_t)rr;
        const uint32_t mS = which == 0 ? o0.mS : (which == 1 ? o1.mS : o2.mS);
        const uint32_t mH = which == 0 ? o0.mH : (which == 1 ? o1.mH : o2.mH);
        const int lS = which == 0 ? o0.lS : (which == 1 ? o1.lS : o2.lS);
        const int lH = which == 0 ? o0.lH : (which == 1 ? o1.lH : o2.lH);
        const uint32_t hs = op_layout == FA_LAYOUT_BNSD ? fast_div(r32, mS, lS) : r32;  // row of [B, H] (BNSD)
        const int h = (int)(hs - fast_div(hs, mH, lH) * (uint32_t)op_H);
        // the static scale and its reciprocal, recomputed per row (a per-CTA table behind a
        // barrier measured slower: each CTA handles only a few rows)
        const float a = in_bounds(h >= 0 && h < op_H, 107) ? __ldg((which == 0 ? o0.amax : (which == 1 ? o1.amax : o2.amax)) + h) : 0.0f;
        sc = __fdiv_rn(a, QMAX);
        rc = sc >= kFastDivMin ? __frcp_rn(sc) : 0.0f;
        lim = fabsf(a) < INFINITY ? a : -1.0f;
      }
      if (INT8) {
        // NaN-propagating max |x| of the lane's 32 elements: a NaN fails the comparison
        uint32_t m2 = 0;
#pragma unroll
        for (int c = 0; c < 4; ++c)
          m2 = bf16x2_absmax_nan(bf16x2_absmax_nan(m2, bf16x2_absmax_nan(raw[c].x, raw[c].y)),
                                 bf16x2_absmax_nan(raw[c].z, raw[c].w));
        m2 &= 0x7FFF7FFFu;  // the sign bits are the XOR of the inputs' signs
        const bool in = !valid || (__uint_as_float(m2 << 16) <= lim && __uint_as_float(m2 & 0xFFFF0000u) <= lim);
        bounded = __all_sync(0xffffffffu, in);
      }
    } else {
      sc = __fdiv_rn(m, QMAX);
      rc = sc >= kFastDivMin ? __frcp_rn(sc) : 0.0f;
    }
    // codes, 8 elements at a time straight from the packed row
    uint32_t w[8];
    const bool fast = sc >= kFastDivMin;
    if (INT8 && bounded) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float v[8];
        unpack_bf16x8(raw[c], v);
        if (fast) {
#pragma unroll
          for (int i = 0; i < 8; i += 2) int8_div_bounded_x2(v[i], v[i + 1], sc, rc);
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) v[i] = sc > 0.0f ? __fdiv_rn(v[i], sc) : 0.0f;
        }
        w[2 * c] = s8x4<false>(v[0], v[1], v[2], v[3]);
        w[2 * c + 1] = s8x4<false>(v[4], v[5], v[6], v[7]);
      }
    } else {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float v[8];
        unpack_bf16x8(raw[c], v);
        if (fast) {
          // x / s as IEEE division rounds it where that decides the code (quant_common.cuh)
#pragma unroll
          for (int i = 0; i < 8; ++i)
            v[i] = INT8 ? int8_div(v[i], sc, rc) : (PER_HEAD ? fp8_div_sat(v[i], sc, rc) : fp8_div(v[i], sc, rc));
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) v[i] = sc > 0.0f ? __fdiv_rn(v[i], sc) : 0.0f;
        }
        w[2 * c] = INT8 ? s8x4<true>(v[0], v[1], v[2], v[3]) : e4m3x4(v[0], v[1], v[2], v[3]);
        w[2 * c + 1] = INT8 ? s8x4<true>(v[4], v[5], v[6], v[7]) : e4m3x4(v[4], v[5], v[6], v[7]);
      }
    }
    if (valid) {
      out[0] = make_uint4(w[0], w[1], w[2], w[3]);
      out[1] = make_uint4(w[4], w[5], w[6], w[7]);
      uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(op_codes) + rr * D + gl * 32);
      if (in_bounds(rr * D + (gl + 1) * 32 <= op_rows * D, 105)) {
        dst[0] = out[0];
        dst[1] = out[1];
      }
      if (!PER_HEAD && gl == 0) {
        const int op_layout = which == 0 ? o0.layout : (which == 1 ? o1.layout : o2.layout);
        const int op_H = which == 0 ? o0.H : (which == 1 ? o1.H : o2.H);
        const int op_S = which == 0 ? o0.S : (which == 1 ? o1.S : o2.S);
        const long long si = scale_index(rr, op_layout, op_H, op_S);
        if (in_bounds(si >= 0 && si < op_rows, 106)) static_cast<float*>(op_scales)[si] = sc;
      }
    }
  }
}

// Per-head running max: grid (chunks, H, batches); each CTA reduces a slice of one head's rows of
// one batch and folds it into amax[h] with one atomic max on the float bits (valid because every
// value is >= 0).  Row and chunk indices come from shifts (D / 8 is a power of two).
template <int D>
__global__ void __launch_bounds__(256) calibrate_kernel(const __nv_bfloat16* __restrict__ x, int B, int H, int S,
                                                        int layout, float* amax) {
  constexpr int VPR = D / 8;  // uint4 per row
  constexpr int VSH = D == 128 ? 4 : 3;
  const int h = blockIdx.y;
  const long long nvec = (long long)S * VPR;
  const long long rstride = layout == FA_LAYOUT_BNSD ? D : (long long)H * D;  // elements from token s to s + 1
  float m = 0.0f;
  for (int b = blockIdx.z; b < B; b += gridDim.z) {
    const __nv_bfloat16* xb = layout == FA_LAYOUT_BNSD ? x + ((long long)b * H + h) * S * D
                                                       : x + (long long)b * S * H * D + (long long)h * D;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < nvec;
         i += (long long)gridDim.x * blockDim.x) {
      const long long off = (xb - x) + (i >> VSH) * rstride + (i & (VPR - 1)) * 8;
      if (!in_bounds(off >= 0 && off + 8 <= (long long)B * H * S * D, 108)) continue;
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(xb + (i >> VSH) * rstride) + (i & (VPR - 1)));
      float f[8];
      unpack_bf16x8(u, f);
#pragma unroll
      for (int k = 0; k < 8; ++k) m = fmaxf(m, fabsf(f[k]));
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  __shared__ float wm[8];
  if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float bm = 0.0f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) bm = fmaxf(bm, wm[w]);
    atomicMax(reinterpret_cast<int*>(amax + h), __float_as_int(bm));
  }
}

// FP8 block quantization without rotation: one CTA per (b, h, block).
// Pass 1 finds the block's amax, pass 2 quantizes (the re-read hits L2).
__global__ void __launch_bounds__(256) fp8_block_kernel(QuantOperand op) {
  const int g = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int s0 = g * op.blk;
  const int s1 = min(op.S, s0 + op.blk);
  const int vpr = op.D / 8;
  const int nvec = (s1 - s0) * vpr;
  const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(op.x);
  auto row_of = [&](int s) -> long long {
    return op.layout == FA_LAYOUT_BNSD ? ((long long)b * op.H + h) * op.S + s : ((long long)b * op.S + s) * op.H + h;
  };
  float m = 0.0f;
  for (int i = threadIdx.x; i < nvec; i += blockDim.x) {
    const long long nrows = (long long)op.B * op.H * op.S;
    if (!in_bounds(row_of(s0 + i / vpr) < nrows, 109)) continue;
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(x + row_of(s0 + i / vpr) * op.D) + (i % vpr));
    float f[8];
    unpack_bf16x8(u, f);
#pragma unroll
    for (int k = 0; k < 8; ++k) m = fmaxf(m, fabsf(f[k]));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  __shared__ float wm[8];
  __shared__ float s_sc;
  if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float bm = 0.0f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) bm = fmaxf(bm, wm[w]);
    s_sc = __fdiv_rn(bm, 448.0f);
    const int nblk = (op.S + op.blk - 1) / op.blk;
    if (in_bounds(((long long)b * op.H + h) * nblk + g < (long long)op.B * op.H * nblk, 110))
      static_cast<float*>(op.scales)[((long long)b * op.H + h) * nblk + g] = s_sc;
  }
  __syncthreads();
  const float sc = s_sc;
  const float rc = sc >= kFastDivMin ? __frcp_rn(sc) : 0.0f;
  for (int i = threadIdx.x; i < nvec; i += blockDim.x) {
    const long long row = row_of(s0 + i / vpr);
    if (!in_bounds(row < (long long)op.B * op.H * op.S, 111)) continue;
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(x + row * op.D) + (i % vpr));
    float f[8];
    unpack_bf16x8(u, f);
    float v[8];
    if (sc >= kFastDivMin) {
#pragma unroll
      for (int k = 0; k < 8; ++k) v[k] = fp8_div(f[k], sc, rc);
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) v[k] = sc > 0.0f ? __fdiv_rn(f[k], sc) : 0.0f;
    }
    reinterpret_cast<uint2*>(static_cast<uint8_t*>(op.codes) + row * op.D)[i % vpr] =
        make_uint2(e4m3x4(v[0], v[1], v[2], v[3]), e4m3x4(v[4], v[5], v[6], v[7]));
  }
}

// Magic multiplier and shift of fast_div for a divisor d in [1, 2^31): l = ceil(log2 d),
// m = floor(2^32 (2^l - d) / d) + 1 (below 2^32 for every such d).  d = 0 (an unused operand) -> 1.
void fastdiv_magic(long long d, uint32_t& m, int& l) {
  if (d < 1) d = 1;
  l = 0;
  while ((1LL << l) < d) ++l;
  m = (uint32_t)((((1ULL << l) - (unsigned long long)d) << 32) / (unsigned long long)d + 1);
}

template <int MODE>
cudaError_t launch_rows_mode(const QuantOperand (&oi)[3], int D, cudaStream_t s) {
  if (const cudaError_t be = bounds_attach(); be != cudaSuccess) return be;
  const long long total = oi[0].rows + oi[1].rows + oi[2].rows;
  constexpr bool PER_HEAD = MODE == FA_MODE_INT8_PER_HEAD || MODE == FA_MODE_FP8_PER_HEAD;
  if (total == 0 && !PER_HEAD) return cudaSuccess;
  QuantOperand o[3] = {oi[0], oi[1], oi[2]};
  for (int i = 0; i < 3; ++i) {
    if (PER_HEAD && o[i].rows > 0xFFFFFFFFLL) return cudaErrorInvalidValue;  // heads found in 32 bits
    fastdiv_magic(o[i].S, o[i].mS, o[i].lS);
    fastdiv_magic(o[i].H, o[i].mH, o[i].lH);
  }
  const int rows_per_block = (kRowThreads / 32) * (32 / (D / 32));
  const long long want = (total + rows_per_block - 1) / rows_per_block;
  const long long cap = (long long)sm_count() * 8 * 4;  // enough resident warps, grid-stride beyond
  const int grid = (int)(want < 1 ? 1 : (want > cap ? cap : want));
  if (D == 128)
    quant_rows_kernel<MODE, 128><<<grid, kRowThreads, 0, s>>>(o[0], o[1], o[2]);
  else
    quant_rows_kernel<MODE, 64><<<grid, kRowThreads, 0, s>>>(o[0], o[1], o[2]);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_calibrate(const QuantOperand& op, float* amax, cudaStream_t s) {
  if (const cudaError_t be = bounds_attach(); be != cudaSuccess) return be;
  const long long nvec = (long long)op.B * op.S * (op.D / 8);
  if (nvec == 0) return cudaSuccess;
  if (op.H > 65535) return cudaErrorInvalidValue;
  // about eight resident CTAs per SM in total, spread over heads and batches
  const long long per_b = (long long)op.S * (op.D / 8);
  const int bz = op.B < 65535 ? op.B : 65535;
  long long chunks = ((long long)sm_count() * 8 + (long long)op.H * bz - 1) / ((long long)op.H * bz);
  const long long most = (per_b + 255) / 256;
  if (chunks > most) chunks = most;
  if (chunks < 1) chunks = 1;
  dim3 grid((unsigned)chunks, (unsigned)op.H, (unsigned)bz);
  const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(op.x);
  if (op.D == 128)
    calibrate_kernel<128><<<grid, 256, 0, s>>>(x, op.B, op.H, op.S, op.layout, amax);
  else
    calibrate_kernel<64><<<grid, 256, 0, s>>>(x, op.B, op.H, op.S, op.layout, amax);
  return cudaGetLastError();
}

cudaError_t launch_quantize_rows(int mode, const QuantOperand* ops, int nops, cudaStream_t s) {
  QuantOperand o[3] = {};
  int D = 128;
  for (int i = 0; i < nops && i < 3; ++i) {
    o[i] = ops[i];
    D = ops[i].D;
  }
  switch (mode) {
    case FA_MODE_FP8_PER_TOKEN: return launch_rows_mode<FA_MODE_FP8_PER_TOKEN>(o, D, s);
    case FA_MODE_INT8_PER_HEAD: return launch_rows_mode<FA_MODE_INT8_PER_HEAD>(o, D, s);
    case FA_MODE_MXFP4_PER_BLOCK: return launch_rows_mode<FA_MODE_MXFP4_PER_BLOCK>(o, D, s);
    case FA_MODE_FP8_PER_HEAD: return launch_rows_mode<FA_MODE_FP8_PER_HEAD>(o, D, s);
    case FA_MODE_INT8_PER_TOKEN: return launch_rows_mode<FA_MODE_INT8_PER_TOKEN>(o, D, s);
    case FA_MODE_MXFP8_PER_BLOCK: return launch_rows_mode<FA_MODE_MXFP8_PER_BLOCK>(o, D, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_quantize_fp8_block(const QuantOperand* ops, int nops, cudaStream_t s) {
  if (const cudaError_t be = bounds_attach(); be != cudaSuccess) return be;
  for (int i = 0; i < nops; ++i) {
    const QuantOperand& op = ops[i];
    if (op.rows == 0) continue;
    dim3 grid((unsigned)((op.S + op.blk - 1) / op.blk), (unsigned)op.H, (unsigned)op.B);
    fp8_block_kernel<<<grid, 256, 0, s>>>(op);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace faq
