// decode_noalloc.cu -- single-token INT8 decode that needs no caller-provided
// workspace and allocates nothing.
//
// fa_attention_quant's split-KV decode writes per-split partial results to a
// workspace the caller must allocate.  Some callers cannot do that at the
// point where they run decode: a serving loop that must never synchronise the
// device (cudaMalloc / cudaFree may), or plain C/C++ host code that links
// libfaq.so and has no device allocator of its own.  This entry point keeps the
// partials in a fixed buffer that lives in the library's own device memory
// instead.
//
// The buffer is a file-scope device array (FA_DECODE_NOALLOC_SCRATCH_BYTES).
// Every GPU that loads the library holds it until the process exits.  All
// calls on a device share it, so two calls whose kernels overlap on the GPU
// (for example on two streams) race on it; issue them in one stream or
// serialise them.  Every call overwrites every partial it later reads, so
// nothing in the buffer has to be cleared between calls.
#include <cuda_runtime.h>

#include <mutex>

#include "internal.cuh"

namespace faq {
namespace {

static __device__ __align__(256) unsigned char g_decode_scratch[FA_DECODE_NOALLOC_SCRATCH_BYTES];

// Device address of the buffer on the current device.  The name of a
// __device__ array in host code is only a host-side stand-in, so the real
// address is looked up once per device (with that device current) and cached.
void* scratch_on_current_device() {
  static void* cache[64] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess) return nullptr;
    cache[dev] = p;
  }
  return cache[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

}  // namespace
}  // namespace faq

using namespace faq;

extern "C" fa_status fa_attention_decode_noalloc(const fa_qtensor* q, const fa_qtensor* k, const fa_qtensor* v,
                                                 float softmax_scale, void* out, float* lse, int num_splits,
                                                 fa_stream_t s) {
  if (!q || !k || !v) return FA_ERR_INVALID_ARG;
  if (q->mode != FA_MODE_INT8_PER_HEAD || k->mode != q->mode || v->mode != q->mode) return FA_ERR_UNSUPPORTED;
  if (q->S != 1 || q->D != 128 || k->D != 128 || v->D != 128) return FA_ERR_UNSUPPORTED;
  if (q->layout != k->layout || q->layout != v->layout ||
      (q->layout != FA_LAYOUT_BNSD && q->layout != FA_LAYOUT_BSND))
    return FA_ERR_INVALID_ARG;
  if (q->B < 0 || k->S < 0 || q->H < 1 || k->H < 1 || q->H % k->H != 0) return FA_ERR_INVALID_ARG;
  if (q->B != k->B || q->B != v->B || k->H != v->H || k->S != v->S) return FA_ERR_INVALID_ARG;
  const int group = q->H / k->H;
  if (!(group == 1 || group == 2 || group == 4 || group == 8 || group == 16)) return FA_ERR_UNSUPPORTED;
  if (num_splits < 0) return FA_ERR_INVALID_ARG;
  // no query rows: nothing to do (as fa_attention_quant)
  if (q->B == 0) return FA_OK;
  if (!q->codes || !q->scales || !aligned16(q->codes) || !aligned4(q->scales)) return FA_ERR_INVALID_ARG;
  if (!out || !aligned16(out)) return FA_ERR_INVALID_ARG;
  if (lse && !aligned4(lse)) return FA_ERR_INVALID_ARG;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(s);
  // no key: every row's output is 0 and its LSE -inf (as fa_attention_quant)
  if (k->S == 0) return launch_fill_empty_rows(out, lse, (long long)q->B * q->H, q->D, cs) == cudaSuccess ? FA_OK : FA_ERR_CUDA;
  if (!k->codes || !k->scales || !v->codes || !v->scales) return FA_ERR_INVALID_ARG;
  if (!aligned16(k->codes) || !aligned16(v->codes) || !aligned4(k->scales) || !aligned4(v->scales))
    return FA_ERR_INVALID_ARG;

  // Split count: the caller's, else the automatic choice reduced until the
  // partials fit the fixed buffer.
  int splits = num_splits;
  if (splits == 0) {
    splits = decode_auto_splits(k->B, k->H, k->S);
    while (splits > 1 && decode_workspace_bytes(q->B, q->H, q->D, splits) > FA_DECODE_NOALLOC_SCRATCH_BYTES)
      --splits;
  }
  if (decode_workspace_bytes(q->B, q->H, q->D, splits) > FA_DECODE_NOALLOC_SCRATCH_BYTES) return FA_ERR_WORKSPACE;

  void* scratch = scratch_on_current_device();
  int* status = device_status_ptr();
  if (!scratch || !status) return FA_ERR_CUDA;
  AttnArgs a = {q, k, v, 0, softmax_scale, out, lse, status};
  const cudaError_t e = launch_attention_decode(a, splits, scratch, cs);
  if (e == cudaErrorNotSupported) return FA_ERR_UNSUPPORTED;
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}
