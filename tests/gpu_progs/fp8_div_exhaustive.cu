// Exhaustive checks of the quantizers' division (quant_common.cuh) against IEEE division, through
// the codes: every positive finite bf16 amax and its scale s = fl(amax / C) (IEEE); scales >=
// kFastDivMin take the fast form, smaller ones IEEE division (as the quantizers do).
//   mode 0: fp8_div,     C = 448, every finite bf16 x with |x| <= amax (dynamic FP8 scales)
//   mode 1: fp8_div_sat, C = 448, every finite bf16 x (static FP8 scales, codes saturate)
//   mode 2: int8_div,    C = 127, every finite bf16 x (INT8, codes saturate)
//   mode 3: int8_div_bounded, C = 127, every finite bf16 x with |x| <= amax
//   mode 4: int8_div_bounded_x2 (the packed pair form), as mode 3
// Prints one line per mode: "mode M fast rows R mismatches N".
#include <cstdint>
#include <cstdio>

#include "quant_common.cuh"

__device__ __forceinline__ uint32_t e4m3_code(float v) {
  uint16_t o;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(o) : "f"(0.0f), "f"(v));
  return o & 0xFF;
}
__device__ __forceinline__ uint32_t s8_code(float v) {
  const int i = __float2int_rn(v);
  return (uint32_t)(max(-128, min(127, i)) & 0xFF);
}

template <int MODE>
__global__ void sweep(unsigned long long* bad, unsigned long long* fast_rows) {
  const uint32_t abits = blockIdx.x + 1;  // 0x0001 .. 0x7F7F: positive finite bf16
  const float amax = __uint_as_float(abits << 16);
  const float s = __fdiv_rn(amax, MODE >= 2 ? 127.0f : 448.0f);
  const bool fast = s >= faq::kFastDivMin;
  const float r = __frcp_rn(s);
  if (threadIdx.x == 0 && fast) atomicAdd(fast_rows, 1ull);
  unsigned long long nb = 0;
  for (uint32_t xb = threadIdx.x; xb < 65536u; xb += blockDim.x) {
    if ((xb & 0x7F80u) == 0x7F80u) continue;  // inf / nan
    const float x = __uint_as_float(xb << 16);
    if ((MODE == 0 || MODE >= 3) && fabsf(x) > amax) continue;
    const float qe = __fdiv_rn(x, s);
    float qf;
    if (!fast) qf = qe;
    else if (MODE == 0) qf = faq::fp8_div(x, s, r);
    else if (MODE == 1) qf = faq::fp8_div_sat(x, s, r);
    else if (MODE == 2) qf = faq::int8_div(x, s, r);
    else if (MODE == 3) qf = faq::int8_div_bounded(x, s, r);
    else {
      float y = -x;  // the pair's second lane: -x must give -q
      qf = x;
      faq::int8_div_bounded_x2(qf, y, s, r);
      if (s8_code(-qe) != s8_code(y)) ++nb;
    }
    const bool diff = MODE >= 2 ? s8_code(qe) != s8_code(qf) : e4m3_code(qe) != e4m3_code(qf);
    if (diff) ++nb;
  }
  if (nb) atomicAdd(bad, nb);
}

int main() {
  unsigned long long *bad, *fr;
  if (cudaMalloc(&bad, 8) != cudaSuccess || cudaMalloc(&fr, 8) != cudaSuccess) return 2;
  for (int mode = 0; mode < 5; ++mode) {
    cudaMemset(bad, 0, 8);
    cudaMemset(fr, 0, 8);
    if (mode == 0) sweep<0><<<0x7F7F, 256>>>(bad, fr);
    else if (mode == 1) sweep<1><<<0x7F7F, 256>>>(bad, fr);
    else if (mode == 2) sweep<2><<<0x7F7F, 256>>>(bad, fr);
    else if (mode == 3) sweep<3><<<0x7F7F, 256>>>(bad, fr);
    else sweep<4><<<0x7F7F, 256>>>(bad, fr);
    if (cudaDeviceSynchronize() != cudaSuccess) return 3;
    unsigned long long hb = 0, hf = 0;
    cudaMemcpy(&hb, bad, 8, cudaMemcpyDeviceToHost);
    cudaMemcpy(&hf, fr, 8, cudaMemcpyDeviceToHost);
    printf("mode %d fast rows %llu mismatches %llu\n", mode, hf, hb);
  }
  return 0;
}
