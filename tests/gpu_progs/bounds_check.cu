// The FA_DEBUG_BOUNDS index check of sm100.cuh: 64 threads each guard a store into a 32-entry
// buffer with in_bounds(i < 32, site 9).  Threads 0..31 store; threads 32..63 must fail the
// check, skip the store (the buffer holds no element for them, so nothing is written past it),
// and leave (9 << 8) | kStatusBounds in the status word.  No access leaves the buffer, so the
// check is exercised without any fault.  Prints "status S stored N guard G" and exits 0.
#define FA_DEBUG_BOUNDS
#include <cstdio>

#include "sm100.cuh"

__global__ void guarded(int* buf, int n) {
  const int i = threadIdx.x;
  if (faq::in_bounds(i < n, 9)) buf[i] = i + 1;
}

int main() {
  int *status, *buf;
  // 32 entries for the guarded stores, then 32 guard entries that must stay zero
  if (cudaMalloc(&status, 4) != cudaSuccess || cudaMalloc(&buf, 64 * 4) != cudaSuccess) return 2;
  cudaMemset(status, 0, 4);
  cudaMemset(buf, 0, 64 * 4);
  if (cudaMemcpyToSymbol(faq::g_bounds_status, &status, sizeof status) != cudaSuccess) return 3;
  guarded<<<1, 64>>>(buf, 32);
  if (cudaDeviceSynchronize() != cudaSuccess) return 4;
  int hs = 0, hb[64];
  cudaMemcpy(&hs, status, 4, cudaMemcpyDeviceToHost);
  cudaMemcpy(hb, buf, sizeof hb, cudaMemcpyDeviceToHost);
  int stored = 0, guard = 0;
  for (int i = 0; i < 32; ++i) stored += hb[i] == i + 1;
  for (int i = 32; i < 64; ++i) guard += hb[i] != 0;
  printf("status %d stored %d guard %d\n", hs, stored, guard);
  return 0;
}
