// Exhaustive check of fp8_div (quant_common.cuh) against IEEE division, through the E4M3 code:
// every positive finite bf16 amax, its scale s = fl(amax / 448) (IEEE), and every finite bf16 x with
// |x| <= amax.  Scales >= kFastDivMin take fp8_div, smaller ones IEEE division (as the quantizers do).
// Prints one line: "fast rows R mismatches M"; exit status 0 when the run itself succeeded.
#include <cstdint>
#include <cstdio>

#include "quant_common.cuh"

__device__ __forceinline__ uint32_t e4m3_code(float v) {
  uint16_t o;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(o) : "f"(0.0f), "f"(v));
  return o & 0xFF;
}

__global__ void sweep(unsigned long long* bad, unsigned long long* fast_rows) {
  const uint32_t abits = blockIdx.x + 1;  // 0x0001 .. 0x7F7F: positive finite bf16
  const float amax = __uint_as_float(abits << 16);
  const float s = __fdiv_rn(amax, 448.0f);
  const bool fast = s >= faq::kFastDivMin;
  const float r = __frcp_rn(s);
  if (threadIdx.x == 0 && fast) atomicAdd(fast_rows, 1ull);
  unsigned long long nb = 0;
  for (uint32_t xb = threadIdx.x; xb < 65536u; xb += blockDim.x) {
    if ((xb & 0x7F80u) == 0x7F80u) continue;  // inf / nan
    const float x = __uint_as_float(xb << 16);
    if (fabsf(x) > amax) continue;
    const float qf = fast ? faq::fp8_div(x, s, r) : __fdiv_rn(x, s);
    if (e4m3_code(__fdiv_rn(x, s)) != e4m3_code(qf)) ++nb;
  }
  if (nb) atomicAdd(bad, nb);
}

int main() {
  unsigned long long *bad, *fr;
  if (cudaMalloc(&bad, 8) != cudaSuccess || cudaMalloc(&fr, 8) != cudaSuccess) return 2;
  cudaMemset(bad, 0, 8);
  cudaMemset(fr, 0, 8);
  sweep<<<0x7F7F, 256>>>(bad, fr);
  if (cudaDeviceSynchronize() != cudaSuccess) return 3;
  unsigned long long hb = 0, hf = 0;
  cudaMemcpy(&hb, bad, 8, cudaMemcpyDeviceToHost);
  cudaMemcpy(&hf, fr, 8, cudaMemcpyDeviceToHost);
  printf("fast rows %llu mismatches %llu\n", hf, hb);
  return 0;
}
