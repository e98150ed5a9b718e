// faq_api.cu -- the C ABI declared in include/faq.h: host-side argument
// validation, the per-device status word, and dispatch to the kernels.
#include <cuda_runtime.h>
#include <string.h>

#include <mutex>
#include <set>
#include <utility>

#include "internal.cuh"
#include "sm100.cuh"

namespace faq {

// Device status word: bounded waits that run out record (where << 8 | code).
static __device__ int g_status;

int* device_status_ptr() {
  static int* cache[64] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return nullptr;
    cache[dev] = static_cast<int*>(p);
  }
  return cache[dev];
}

EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

int sm_count() {
  static int cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cache[dev]) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cache[dev] = n > 0 ? n : 148;
  }
  return cache[dev];
}

cudaError_t set_smem_limit(const void* kernel, int bytes) {
  static std::mutex mu;
  static std::set<std::pair<const void*, int>> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  if (done.count({kernel, dev})) return cudaSuccess;
  if ((e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes)) != cudaSuccess) return e;
  done.insert({kernel, dev});
  return cudaSuccess;
}

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_layout(int l) { return l == FA_LAYOUT_BNSD || l == FA_LAYOUT_BSND; }

bool quantized_mode(int m) {
  return m == FA_MODE_INT8_PER_HEAD || m == FA_MODE_FP8_PER_TOKEN || m == FA_MODE_MXFP4_PER_BLOCK ||
         m == FA_MODE_FP8_BLOCK || m == FA_MODE_FP8_PER_HEAD || m == FA_MODE_INT8_PER_TOKEN ||
         m == FA_MODE_MXFP8_PER_BLOCK;
}

fa_status check_tensor(const fa_tensor* t) {
  if (!t) return FA_ERR_INVALID_ARG;
  if (t->B < 0 || t->H < 1 || t->S < 0 || !valid_layout(t->layout)) return FA_ERR_INVALID_ARG;
  if (t->D != 64 && t->D != 128) return FA_ERR_UNSUPPORTED;
  if ((long long)t->B * t->S > 0 && (!t->data || !aligned16(t->data))) return FA_ERR_INVALID_ARG;
  return FA_OK;
}

fa_status check_out(const fa_tensor* t, const fa_qtensor* o, fa_mode mode) {
  if (!o) return FA_ERR_INVALID_ARG;
  if (o->mode != mode || o->B != t->B || o->H != t->H || o->S != t->S || o->D != t->D || o->layout != t->layout)
    return FA_ERR_INVALID_ARG;
  if ((long long)t->B * t->S == 0) return FA_OK;
  if (!o->codes || !o->scales || !aligned16(o->codes) || (reinterpret_cast<uintptr_t>(o->scales) & 3u))
    return FA_ERR_INVALID_ARG;
  if (mode == FA_MODE_FP8_BLOCK && o->block_tokens < 1) return FA_ERR_INVALID_ARG;
  if ((mode == FA_MODE_MXFP4_PER_BLOCK || mode == FA_MODE_MXFP8_PER_BLOCK) && o->D % 32 != 0) return FA_ERR_INVALID_ARG;
  return FA_OK;
}

fa_status from_cuda(cudaError_t e) { return e == cudaSuccess ? FA_OK : FA_ERR_CUDA; }

QuantOperand make_op(const fa_tensor* t, const fa_qtensor* o, const float* amax) {
  QuantOperand op = {};
  op.x = t->data;
  op.codes = o->codes;
  op.scales = o->scales;
  op.amax = amax;
  op.rows = (long long)t->B * t->H * t->S;
  op.B = t->B;
  op.H = t->H;
  op.S = t->S;
  op.D = t->D;
  op.layout = t->layout;
  op.blk = o->block_tokens;
  return op;
}

fa_status check_qtensor(const fa_qtensor* t) {
  if (!t) return FA_ERR_INVALID_ARG;
  if (!quantized_mode(t->mode)) return FA_ERR_UNSUPPORTED;
  if (t->B < 0 || t->H < 1 || t->S < 0 || !valid_layout(t->layout)) return FA_ERR_INVALID_ARG;
  if (t->D != 64 && t->D != 128) return FA_ERR_UNSUPPORTED;
  if (t->mode == FA_MODE_FP8_BLOCK && t->block_tokens < 1) return FA_ERR_INVALID_ARG;
  // codes 16-byte aligned (TMA); scales (fp32, or E8M0 bytes read four at a time) 4-byte aligned
  if ((long long)t->B * t->S > 0 &&
      (!t->codes || !t->scales || !aligned16(t->codes) || (reinterpret_cast<uintptr_t>(t->scales) & 3u)))
    return FA_ERR_INVALID_ARG;
  return FA_OK;
}

// An attention operand: a quantized descriptor, or FA_MODE_FLOAT whose codes are the bf16 tensor
// itself (scales unused).
fa_status check_operand(const fa_qtensor* t) {
  if (!t) return FA_ERR_INVALID_ARG;
  if (t->mode != FA_MODE_FLOAT) return check_qtensor(t);
  if (t->B < 0 || t->H < 1 || t->S < 0 || !valid_layout(t->layout)) return FA_ERR_INVALID_ARG;
  if (t->D != 64 && t->D != 128) return FA_ERR_UNSUPPORTED;
  if ((long long)t->B * t->S > 0 && (!t->codes || !aligned16(t->codes))) return FA_ERR_INVALID_ARG;
  return FA_OK;
}

}  // namespace
}  // namespace faq

using namespace faq;

extern "C" {

const char* fa_version(void) { return "faq-b200 0.1 (sm_100a)"; }

const char* fa_status_str(fa_status st) {
  switch (st) {
    case FA_OK: return "ok";
    case FA_ERR_INVALID_ARG: return "invalid argument";
    case FA_ERR_UNSUPPORTED: return "unsupported";
    case FA_ERR_NO_CALIBRATION: return "static mode without calibration data";
    case FA_ERR_CONFIG_CONFLICT: return "qconfig and details are mutually exclusive";
    case FA_ERR_CUDA: return "CUDA error";
    case FA_ERR_TIMEOUT: return "kernel wait timed out";
    case FA_ERR_WORKSPACE: return "workspace missing or too small";
    case FA_ERR_BOUNDS: return "index check failed (bounds-checked build)";
  }
  return "unknown status";
}

fa_status fa_resolve_config(const fa_branch_cfg* qconfig, const fa_branch_cfg* details, fa_mode modes_out[3]) {
  if (!modes_out) return FA_ERR_INVALID_ARG;
  const bool has_q = qconfig && qconfig->set;
  const bool has_d = details && (details[0].set || details[1].set || details[2].set);
  if (has_q && has_d) return FA_ERR_CONFIG_CONFLICT;
  if (has_q) {
    if (qconfig->mode < FA_MODE_FLOAT || qconfig->mode > FA_MODE_MXFP8_PER_BLOCK) return FA_ERR_INVALID_ARG;
    modes_out[0] = modes_out[1] = modes_out[2] = qconfig->mode;
    return FA_OK;
  }
  if (has_d) {
    for (int i = 0; i < 3; ++i) {
      if (details[i].set && (details[i].mode < FA_MODE_FLOAT || details[i].mode > FA_MODE_MXFP8_PER_BLOCK))
        return FA_ERR_INVALID_ARG;
      modes_out[i] = details[i].set ? details[i].mode : FA_MODE_FLOAT;
    }
    return FA_OK;
  }
  modes_out[0] = modes_out[1] = modes_out[2] = FA_MODE_INT8_PER_HEAD;
  return FA_OK;
}

fa_status fa_calibrate_per_head(const fa_tensor* x, float* amax_h, fa_stream_t s) {
  fa_status st = check_tensor(x);
  if (st != FA_OK) return st;
  if (!amax_h) return FA_ERR_INVALID_ARG;
  fa_qtensor dummy = {};
  dummy.B = x->B; dummy.H = x->H; dummy.S = x->S; dummy.D = x->D; dummy.layout = x->layout;
  QuantOperand op = make_op(x, &dummy, nullptr);
  return from_cuda(launch_calibrate(op, amax_h, reinterpret_cast<cudaStream_t>(s)));
}

fa_status fa_quantize(const fa_tensor* q, const fa_tensor* k, const fa_tensor* v, fa_mode mode, const float* amax_q,
                      const float* amax_k, const float* amax_v, fa_qtensor* q_out, fa_qtensor* k_out,
                      fa_qtensor* v_out, fa_stream_t s) {
  if (!quantized_mode(mode)) return mode == FA_MODE_FLOAT ? FA_ERR_INVALID_ARG : FA_ERR_UNSUPPORTED;
  const fa_tensor* in[3] = {q, k, v};
  fa_qtensor* out[3] = {q_out, k_out, v_out};
  const float* am[3] = {amax_q, amax_k, amax_v};
  QuantOperand ops[3];
  int n = 0;
  for (int i = 0; i < 3; ++i) {
    if (!in[i]) continue;
    fa_status st = check_tensor(in[i]);
    if (st != FA_OK) return st;
    st = check_out(in[i], out[i], mode);
    if (st != FA_OK) return st;
    if ((mode == FA_MODE_INT8_PER_HEAD || mode == FA_MODE_FP8_PER_HEAD) && !am[i]) return FA_ERR_NO_CALIBRATION;
    ops[n++] = make_op(in[i], out[i], am[i]);
  }
  if (n == 0) return FA_ERR_INVALID_ARG;
  for (int i = 1; i < n; ++i)
    if (ops[i].D != ops[0].D) return FA_ERR_INVALID_ARG;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(s);
  if (mode == FA_MODE_FP8_BLOCK) return from_cuda(launch_quantize_fp8_block(ops, n, cs));
  return from_cuda(launch_quantize_rows(mode, ops, n, cs));
}

fa_status fa_rotate_quantize(const fa_tensor* q, const fa_tensor* k, const fa_tensor* v, const void* rot_q,
                             const void* rot_k, int q_block, int kv_block, fa_qtensor* q_out, fa_qtensor* k_out,
                             fa_qtensor* v_out, void* rot_q_dbg, void* rot_k_dbg, fa_stream_t s) {
  const fa_tensor* in[3] = {q, k, v};
  fa_qtensor* out[3] = {q_out, k_out, v_out};
  const void* rot[3] = {rot_q, rot_k, nullptr};
  void* dbg[3] = {rot_q_dbg, rot_k_dbg, nullptr};
  const int blk[3] = {q_block, kv_block, kv_block};
  RotateOperand ops[3] = {};
  int n = 0;
  for (int i = 0; i < 3; ++i) {
    if (!in[i]) continue;
    fa_status st = check_tensor(in[i]);
    if (st != FA_OK) return st;
    st = check_out(in[i], out[i], FA_MODE_FP8_BLOCK);
    if (st != FA_OK) return st;
    if (blk[i] < 1 || out[i]->block_tokens != blk[i]) return FA_ERR_INVALID_ARG;
    if (i < 2 && (long long)in[i]->B * in[i]->S > 0) {
      if (!rot[i] || !aligned16(rot[i])) return FA_ERR_INVALID_ARG;
      if (dbg[i] && !aligned16(dbg[i])) return FA_ERR_INVALID_ARG;
    }
    RotateOperand& op = ops[n++];
    op.x = in[i]->data;
    op.R = rot[i];
    op.codes = out[i]->codes;
    op.scales = static_cast<float*>(out[i]->scales);
    op.dbg = dbg[i];
    op.B = in[i]->B; op.H = in[i]->H; op.S = in[i]->S; op.D = in[i]->D; op.layout = in[i]->layout;
    op.blk = blk[i];
  }
  if (n == 0) return FA_ERR_INVALID_ARG;
  int* status = device_status_ptr();
  if (!status) return FA_ERR_CUDA;
  cudaError_t e = launch_rotate_block_quant(ops, n, status, reinterpret_cast<cudaStream_t>(s));
  if (e == cudaErrorNotSupported) return FA_ERR_UNSUPPORTED;
  return from_cuda(e);
}

fa_status fa_rotate_quantize_hadamard(const fa_tensor* q, const fa_tensor* k, const fa_tensor* v,
                                      const uint32_t* sign_bits_q, const uint32_t* sign_bits_k, int q_block,
                                      int kv_block, fa_qtensor* q_out, fa_qtensor* k_out, fa_qtensor* v_out,
                                      void* rot_q_dbg, void* rot_k_dbg, fa_stream_t s) {
  const fa_tensor* in[3] = {q, k, v};
  fa_qtensor* out[3] = {q_out, k_out, v_out};
  const uint32_t* sg[3] = {sign_bits_q, sign_bits_k, nullptr};
  void* dbg[3] = {rot_q_dbg, rot_k_dbg, nullptr};
  const int blk[3] = {q_block, kv_block, kv_block};
  HadamardOperand ops[3];
  int n = 0;
  for (int i = 0; i < 3; ++i) {
    if (!in[i]) continue;
    fa_status st = check_tensor(in[i]);
    if (st != FA_OK) return st;
    st = check_out(in[i], out[i], FA_MODE_FP8_BLOCK);
    if (st != FA_OK) return st;
    if (blk[i] < 1 || out[i]->block_tokens != blk[i]) return FA_ERR_INVALID_ARG;
    if (dbg[i] && !aligned16(dbg[i])) return FA_ERR_INVALID_ARG;
    HadamardOperand& op = ops[n++];
    op.x = in[i]->data;
    op.codes = out[i]->codes;
    op.scales = static_cast<float*>(out[i]->scales);
    op.dbg = dbg[i];
    for (int w = 0; w < 4; ++w) op.sign_bits[w] = (sg[i] && w < in[i]->D / 32) ? sg[i][w] : 0u;
    op.B = in[i]->B; op.H = in[i]->H; op.S = in[i]->S; op.D = in[i]->D; op.layout = in[i]->layout;
    op.blk = blk[i];
    op.rotate = i < 2;
  }
  if (n == 0) return FA_ERR_INVALID_ARG;
  for (int i = 1; i < n; ++i)
    if (ops[i].D != ops[0].D) return FA_ERR_INVALID_ARG;
  // D = 128 with blocks that divide 256 tokens: the tensor-core rotation pipeline with R generated
  // in shared memory from the signs (the rotation is HBM-bound there, so a product costs no more
  // than the transform); otherwise the fast Walsh-Hadamard transform kernel
  bool pipeline = ops[0].D == 128;
  for (int i = 0; i < n; ++i) pipeline = pipeline && ops[i].blk <= 256 && 256 % ops[i].blk == 0;
  if (pipeline) {
    RotateOperand ro[3] = {};
    for (int i = 0; i < n; ++i) {
      const HadamardOperand& h = ops[i];
      ro[i].x = h.x;
      ro[i].R = nullptr;
      ro[i].codes = h.codes;
      ro[i].scales = h.scales;
      ro[i].dbg = h.dbg;
      ro[i].B = h.B; ro[i].H = h.H; ro[i].S = h.S; ro[i].D = h.D; ro[i].layout = h.layout; ro[i].blk = h.blk;
      ro[i].hadamard = h.rotate;
      for (int w = 0; w < 4; ++w) ro[i].sign_bits[w] = h.sign_bits[w];
    }
    int* status = device_status_ptr();
    if (!status) return FA_ERR_CUDA;
    const cudaError_t e = launch_rotate_block_quant(ro, n, status, reinterpret_cast<cudaStream_t>(s));
    if (e == cudaErrorNotSupported) return FA_ERR_UNSUPPORTED;
    return from_cuda(e);
  }
  const cudaError_t e = launch_hadamard_block_quant(ops, n, reinterpret_cast<cudaStream_t>(s));
  if (e == cudaErrorNotSupported) return FA_ERR_UNSUPPORTED;
  return from_cuda(e);
}

// Branches in different modes, or any branch not quantized: the bf16 mixed path.
static bool is_mixed(const fa_qtensor* q, const fa_qtensor* k, const fa_qtensor* v) {
  return q->mode != k->mode || (v && q->mode != v->mode) || q->mode == FA_MODE_FLOAT || k->mode == FA_MODE_FLOAT ||
         (v && v->mode == FA_MODE_FLOAT);
}

static bool is_decode(const fa_qtensor* q, const fa_qtensor* k) {
  if (q->S != 1 || q->mode != FA_MODE_INT8_PER_HEAD || q->D != 128) return false;
  const int group = q->H / k->H;
  return group == 1 || group == 2 || group == 4 || group == 8 || group == 16;
}

static size_t attention_ws(const fa_qtensor* q, const fa_qtensor* k, const fa_qtensor* v, int num_splits) {
  if (!q || !k || k->H < 1 || q->H % k->H || num_splits < 0) return 0;
  if (is_mixed(q, k, v)) {
    if (k->B < 0 || k->S < 0 || q->B < 0 || q->S < 0 || (q->D != 64 && q->D != 128)) return 0;
    return mixed_workspace_bytes(q, k);
  }
  if (is_decode(q, k)) {
    const int splits = num_splits > 0 ? num_splits : decode_auto_splits(k->B, k->H, k->S);
    return decode_workspace_bytes(q->B, q->H, q->D, splits);
  }
  if (q->mode == FA_MODE_INT8_PER_HEAD || q->mode == FA_MODE_FP8_PER_TOKEN || q->mode == FA_MODE_FP8_BLOCK ||
      q->mode == FA_MODE_FP8_PER_HEAD || q->mode == FA_MODE_INT8_PER_TOKEN) {
    if (k->B < 0 || k->S < 0 || (q->D != 64 && q->D != 128)) return 0;
    return prefill2_workspace_bytes(k->B, k->H, k->S, q->D);
  }
  if (q->mode == FA_MODE_MXFP4_PER_BLOCK || q->mode == FA_MODE_MXFP8_PER_BLOCK) {
    if (k->B < 0 || k->S < 0 || q->D != 128) return 0;
    return prefill2_workspace_bytes(k->B, k->H, k->S, q->D, prefill_tile_keys(q->mode));
  }
  return 0;
}

size_t fa_attention_workspace_size(const fa_qtensor* q, const fa_qtensor* k, int num_splits) {
  return attention_ws(q, k, nullptr, num_splits);
}

size_t fa_attention_workspace_size_qkv(const fa_qtensor* q, const fa_qtensor* k, const fa_qtensor* v,
                                       int num_splits) {
  if (!v) return 0;
  return attention_ws(q, k, v, num_splits);
}

fa_status fa_attention_quant(const fa_qtensor* q, const fa_qtensor* k, const fa_qtensor* v, int causal,
                             float softmax_scale, void* out, float* lse, int num_splits, void* workspace,
                             size_t ws_bytes, fa_stream_t s) {
  fa_status st;
  if ((st = check_operand(q)) != FA_OK) return st;
  if ((st = check_operand(k)) != FA_OK) return st;
  if ((st = check_operand(v)) != FA_OK) return st;
  const bool mixed = is_mixed(q, k, v);
  if (q->layout != k->layout || q->layout != v->layout) return FA_ERR_INVALID_ARG;
  if (q->D != k->D || q->D != v->D) return FA_ERR_INVALID_ARG;
  if (q->B != k->B || q->B != v->B) return FA_ERR_INVALID_ARG;
  if (k->H != v->H || k->S != v->S) return FA_ERR_INVALID_ARG;
  if (q->H % k->H != 0) return FA_ERR_INVALID_ARG;
  if (!mixed && q->mode == FA_MODE_FP8_BLOCK && k->block_tokens != v->block_tokens) return FA_ERR_INVALID_ARG;
  if (num_splits < 0) return FA_ERR_INVALID_ARG;
  const long long qrows = (long long)q->B * q->H * q->S;
  if (qrows == 0) return FA_OK;
  if (!out || !aligned16(out)) return FA_ERR_INVALID_ARG;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return FA_ERR_INVALID_ARG;
  const bool decode = !mixed && is_decode(q, k);
  if (!mixed && (q->mode == FA_MODE_MXFP4_PER_BLOCK || q->mode == FA_MODE_MXFP8_PER_BLOCK) && q->D != 128)
    return FA_ERR_UNSUPPORTED;
  if (mixed && (v->mode == FA_MODE_MXFP4_PER_BLOCK || v->mode == FA_MODE_MXFP8_PER_BLOCK) && v->D != 128)
    return FA_ERR_UNSUPPORTED;
  const int splits = decode ? (num_splits > 0 ? num_splits : decode_auto_splits(k->B, k->H, k->S)) : 0;
  if (k->S > 0) {
    const size_t need = mixed    ? mixed_workspace_bytes(q, k)
                        : decode ? decode_workspace_bytes(q->B, q->H, q->D, splits)
                                 : prefill2_workspace_bytes(k->B, k->H, k->S, q->D, prefill_tile_keys(q->mode));
    if (!workspace || ws_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return FA_ERR_WORKSPACE;
  }
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(s);
  if (k->S == 0) return from_cuda(launch_fill_empty_rows(out, lse, qrows, q->D, cs));
  int* status = device_status_ptr();
  if (!status) return FA_ERR_CUDA;
  AttnArgs a = {q, k, v, causal ? 1 : 0, softmax_scale, out, lse, status};
  cudaError_t e;
  if (mixed)
    e = launch_attention_mixed(a, workspace, cs);
  else if (decode)
    e = launch_attention_decode(a, splits, workspace, cs);
  else
    e = launch_attention_prefill2(a, workspace, cs);
  if (e == cudaErrorNotSupported) return FA_ERR_UNSUPPORTED;
  return from_cuda(e);
}

// Shared checks of fa_decode_append's operands; returns the split count through *splits.
static fa_status check_decode_append(const fa_tensor* q, const fa_tensor* k_new, const fa_tensor* v_new,
                                     const fa_qtensor* kc, const fa_qtensor* vc, int pos, int num_splits,
                                     int* splits) {
  if (!q || !k_new || !v_new || !kc || !vc) return FA_ERR_INVALID_ARG;
  if (kc->mode != FA_MODE_INT8_PER_HEAD || vc->mode != FA_MODE_INT8_PER_HEAD) return FA_ERR_UNSUPPORTED;
  if (q->D != 128 || k_new->D != 128 || v_new->D != 128 || kc->D != 128 || vc->D != 128) return FA_ERR_UNSUPPORTED;
  if (!valid_layout(q->layout) || q->layout != k_new->layout || q->layout != v_new->layout ||
      q->layout != kc->layout || q->layout != vc->layout)
    return FA_ERR_INVALID_ARG;
  if (q->S != 1 || k_new->S != 1 || v_new->S != 1) return FA_ERR_INVALID_ARG;
  if (q->B < 1 || kc->H < 1 || q->H % kc->H != 0) return FA_ERR_INVALID_ARG;
  if (k_new->B != q->B || v_new->B != q->B || kc->B != q->B || vc->B != q->B) return FA_ERR_INVALID_ARG;
  if (k_new->H != kc->H || v_new->H != kc->H || vc->H != kc->H || vc->S != kc->S) return FA_ERR_INVALID_ARG;
  const int group = q->H / kc->H;
  if (!(group == 1 || group == 2 || group == 4 || group == 8 || group == 16)) return FA_ERR_UNSUPPORTED;
  if (pos < 0 || pos >= kc->S || num_splits < 0) return FA_ERR_INVALID_ARG;
  if (!q->data || !k_new->data || !v_new->data || !aligned16(q->data) || !aligned16(k_new->data) ||
      !aligned16(v_new->data))
    return FA_ERR_INVALID_ARG;
  if (!kc->codes || !vc->codes || !kc->scales || !vc->scales || !aligned16(kc->codes) || !aligned16(vc->codes) ||
      (reinterpret_cast<uintptr_t>(kc->scales) & 3u) || (reinterpret_cast<uintptr_t>(vc->scales) & 3u))
    return FA_ERR_INVALID_ARG;
  *splits = num_splits > 0 ? num_splits : decode_auto_splits(q->B, kc->H, pos + 1);
  return FA_OK;
}

size_t fa_decode_append_workspace_size(const fa_tensor* q, const fa_qtensor* k_cache, int pos, int num_splits) {
  if (!q || !k_cache || k_cache->H < 1 || q->H % k_cache->H || pos < 0 || num_splits < 0) return 0;
  const int splits = num_splits > 0 ? num_splits : decode_auto_splits(q->B, k_cache->H, pos + 1);
  return decode_workspace_bytes(q->B, q->H, q->D, splits);
}

fa_status fa_decode_append(const fa_tensor* q, const fa_tensor* k_new, const fa_tensor* v_new, const float* amax_q,
                           const float* amax_k, const float* amax_v, fa_qtensor* k_cache, fa_qtensor* v_cache,
                           int pos, float softmax_scale, void* out, float* lse, int num_splits, void* workspace,
                           size_t ws_bytes, fa_stream_t s) {
  int splits = 0;
  fa_status st = check_decode_append(q, k_new, v_new, k_cache, v_cache, pos, num_splits, &splits);
  if (st != FA_OK) return st;
  if (!amax_q || !amax_k || !amax_v) return FA_ERR_NO_CALIBRATION;
  if (!out || !aligned16(out)) return FA_ERR_INVALID_ARG;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return FA_ERR_INVALID_ARG;
  const size_t need = decode_workspace_bytes(q->B, q->H, q->D, splits);
  if (!workspace || ws_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return FA_ERR_WORKSPACE;
  int* status = device_status_ptr();
  if (!status) return FA_ERR_CUDA;
  DecodeAppendArgs a = {q, k_new, v_new, amax_q, amax_k, amax_v, k_cache, v_cache, pos, softmax_scale, out, lse, status};
  const cudaError_t e = launch_decode_append(a, splits, workspace, reinterpret_cast<cudaStream_t>(s));
  if (e == cudaErrorNotSupported) return FA_ERR_UNSUPPORTED;
  return from_cuda(e);
}

fa_status fa_check_device_status(fa_stream_t s) {
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(s);
  if (cudaStreamSynchronize(cs) != cudaSuccess) return FA_ERR_CUDA;
  int* p = device_status_ptr();
  if (!p) return FA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, p, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return FA_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpy(p, &zero, sizeof zero, cudaMemcpyHostToDevice) != cudaSuccess) return FA_ERR_CUDA;
    return (v & 0xFF) == kStatusBounds ? FA_ERR_BOUNDS : FA_ERR_TIMEOUT;
  }
  return FA_OK;
}

}  // extern "C"
