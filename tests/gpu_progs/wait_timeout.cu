// The bounded mbarrier wait of sm100.cuh, made to run out: one CTA waits on an mbarrier that
// nothing arrives at, with the bound set to 2 ms.  Every thread must give up (false), the status
// word must hold (where << 8) | kStatusTimeout, the abort flag must be raised, and a kernel
// launched afterwards must run normally (the context is intact).  No trap, no fault.
// Prints "status S done D after A" and exits 0 on success.
#define FAQ_WAIT_NS 2000000ull  // 2 ms
#include <cstdio>

#include "sm100.cuh"

__global__ void wait_nothing(int* status, int* done) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    faq::mbar_init(&bar, 1);  // expects one arrival; none comes
    abort_flag = 0;
    faq::fence_barrier_init();
  }
  __syncthreads();
  const bool ok = faq::mbar_wait(&bar, 0, &abort_flag, status, 7);
  if (ok) atomicAdd(&done[0], 1);       // must stay 0
  else atomicAdd(&done[1], 1);          // every thread gives up
  __syncthreads();
  if (threadIdx.x == 0) done[2] = abort_flag;
}

__global__ void after(int* out) { out[threadIdx.x] = threadIdx.x * 3; }

int main() {
  int *status, *done, *out;
  if (cudaMalloc(&status, 4) != cudaSuccess || cudaMalloc(&done, 12) != cudaSuccess ||
      cudaMalloc(&out, 64 * 4) != cudaSuccess)
    return 2;
  cudaMemset(status, 0, 4);
  cudaMemset(done, 0, 12);
  wait_nothing<<<1, 64>>>(status, done);
  if (cudaDeviceSynchronize() != cudaSuccess) return 3;
  int hs = 0, hd[3] = {0, 0, 0};
  cudaMemcpy(&hs, status, 4, cudaMemcpyDeviceToHost);
  cudaMemcpy(hd, done, 12, cudaMemcpyDeviceToHost);
  after<<<1, 64>>>(out);
  if (cudaDeviceSynchronize() != cudaSuccess) return 4;
  int ho[64];
  cudaMemcpy(ho, out, sizeof ho, cudaMemcpyDeviceToHost);
  int good = 0;
  for (int i = 0; i < 64; ++i) good += ho[i] == i * 3;
  printf("status %d done %d gaveup %d abort %d after %d\n", hs, hd[0], hd[1], hd[2], good);
  return 0;
}
