/*
 * faq.h -- C ABI of the B200 (sm_100a) FA-quantization library (libfaq.so).
 *
 * FA quantization quantizes the Q/K/V activations that feed flash attention
 * and then computes attention on the low-bit operands (msModelSlim wiki
 * "FA 量化", section 概述 / overview; MindIE SD "量化", section FA量化).
 * This header declares the whole boundary: calibration, quantization of
 * Q/K/V in the pages' modes, the rotate -> block-quant step, and attention
 * on the quantized operands (prefill, and split-KV decode for Sq = 1).
 *
 * Conventions shared by every entry point
 *   - All data pointers are DEVICE pointers owned by the caller.  The
 *     library never allocates, frees or synchronises on these paths; every
 *     call is asynchronous on the caller's stream `s` (0 = legacy default).
 *   - bf16 tensors use layout BNSD = [B, H, S, D] or BSND = [B, S, H, D]
 *     (MindIE SD "量化", FA量化 / 注意事项: Q/K/V input layouts BNSD and
 *     BSND), dense, D contiguous, 16-byte aligned base pointers.
 *   - D must be 64 or 128.
 *   - Arguments are validated on the host before any launch; a rejected call
 *     launches nothing and returns a non-zero fa_status.
 *   - Kernel-side failures (a bounded wait that ran out) are recorded in a
 *     per-device status word and reported by fa_check_device_status().
 *
 * Quantized tensor (fa_qtensor) storage, per mode -- codes keep the data
 * layout, scale arrays are canonical whatever the layout:
 *   FA_MODE_INT8_PER_HEAD    codes int8 [..D];   scales fp32 [H]
 *   FA_MODE_FP8_PER_TOKEN    codes e4m3 [..D];   scales fp32 [B, H, S]
 *   FA_MODE_FP8_BLOCK        codes e4m3 [..D];   scales fp32 [B, H, ceil(S/block_tokens)]
 *   FA_MODE_MXFP4_PER_BLOCK  codes packed e2m1 [..D/2] (element 2i in the
 *                            low nibble, 2i+1 in the high nibble);
 *                            scales uint8 E8M0 [B, H, S, D/32]
 *   FA_MODE_FP8_PER_HEAD     codes e4m3 [..D];   scales fp32 [H]
 *   FA_MODE_INT8_PER_TOKEN   codes int8 [..D];   scales fp32 [B, H, S]
 *   FA_MODE_MXFP8_PER_BLOCK  codes e4m3 [..D];   scales uint8 E8M0 [B, H, S, D/32]
 */
#ifndef FAQ_H
#define FAQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FAQ_API __attribute__((visibility("default")))
#else
#define FAQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* fa_stream_t; /* a cudaStream_t */

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1,     /* bad pointer, shape, layout, alignment      */
  FA_ERR_UNSUPPORTED = 2,     /* valid request this build does not run      */
  FA_ERR_NO_CALIBRATION = 3,  /* static mode without calibration data       */
  FA_ERR_CONFIG_CONFLICT = 4, /* qconfig and details both given             */
  FA_ERR_CUDA = 5,            /* a CUDA runtime call or launch failed       */
  FA_ERR_TIMEOUT = 6,         /* a kernel's bounded wait ran out            */
  FA_ERR_WORKSPACE = 7,       /* workspace missing or too small             */
  FA_ERR_BOUNDS = 8           /* FA_DEBUG_BOUNDS build: an index check failed */
} fa_status;

typedef enum { FA_LAYOUT_BNSD = 0, FA_LAYOUT_BSND = 1 } fa_layout;

/* The pages' FA modes (msModelSlim wiki "FA 量化", 分支组合 / branch
 * combinations 组合1-3 and 该类下的模式清单 / mode list: FA PerHead INT8/FP8
 * static, FA PerToken INT8/FP8 dynamic; MindIE SD "量化", FA量化 / 块量化). */
typedef enum {
  FA_MODE_FLOAT = 0,           /* not quantized ("float": the branch stays bf16) */
  FA_MODE_INT8_PER_HEAD = 1,   /* 组合1: INT8, per-head static minmax, s = amax/127 */
  FA_MODE_FP8_PER_TOKEN = 2,   /* 组合2: E4M3, per-token dynamic, s = amax/448     */
  FA_MODE_MXFP4_PER_BLOCK = 3, /* 组合3: E2M1 + E8M0 per 32 elements of head_dim   */
  FA_MODE_FP8_BLOCK = 4,       /* 块量化: E4M3, one scale per block of tokens      */
  FA_MODE_FP8_PER_HEAD = 5,    /* FA PerHead, FP8: per-head static, s = amax/448   */
  FA_MODE_INT8_PER_TOKEN = 6,  /* FA PerToken, INT8: per-token dynamic, s = amax/127 */
  FA_MODE_MXFP8_PER_BLOCK = 7  /* FA PerBlock, MXFP8: E4M3 + E8M0 per 32 elements  */
} fa_mode;

/* A bf16 activation tensor. */
typedef struct {
  const void* data; /* device, bf16 */
  int B, H, S, D;
  fa_layout layout;
} fa_tensor;

/* A quantized tensor: codes + scales + mode + layout.  Filled by the caller
 * (pointers to caller-owned device buffers of the sizes listed above; codes
 * 16-byte aligned, scales 4-byte aligned, else FA_ERR_INVALID_ARG). */
typedef struct {
  void* codes;
  void* scales;
  fa_mode mode;
  int B, H, S, D;
  fa_layout layout;
  int block_tokens; /* FA_MODE_FP8_BLOCK only: tokens per scale block */
} fa_qtensor;

/* Per-branch quantization settings (msModelSlim "fa3_quant 配置说明",
 * §2.1 FA3QuantProcessorConfig and §2.3 FA3AttentionDetails). */
typedef struct {
  int set;      /* 0 = not given */
  fa_mode mode; /* FA_MODE_FLOAT = the branch is not quantized */
} fa_branch_cfg;

/*
 * fa_resolve_config -- turn a unified qconfig and/or per-branch details into
 * the mode of each branch (q, k, v).
 *   Source: "fa3_quant 配置说明" §2.1 配置约束 -- qconfig and details are
 *   mutually exclusive; both given is an error; neither given means the
 *   default int8 / per_head / symmetric / minmax.  §2.3 and the wiki's
 *   分支组合 note: a branch that details leaves unset is not quantized.
 *   qconfig: nullable; details: nullable array of 3 (q, k, v).
 *   modes_out: host array of 3.
 *   Returns FA_ERR_CONFIG_CONFLICT when both are set, FA_ERR_INVALID_ARG on
 *   a NULL modes_out or an out-of-range mode.  Host only, no CUDA call.
 */
FAQ_API fa_status fa_resolve_config(const fa_branch_cfg* qconfig, const fa_branch_cfg* details, fa_mode modes_out[3]);

/*
 * fa_calibrate_per_head -- static per-head minmax calibration.
 *   Source: wiki "FA 量化", 组合1 -- one scale per attention head, found
 *   offline (minmax) and then frozen; calibration data is mandatory.
 *   x: bf16 calibration batch.  amax_h: device fp32 [x->H], a RUNNING
 *   maximum: on return amax_h[h] = max(amax_h[h], max |x| over head h).
 *   The caller zero-fills it before the first batch.  Call once per batch.
 */
FAQ_API fa_status fa_calibrate_per_head(const fa_tensor* x, float* amax_h, fa_stream_t s);

/*
 * fa_quantize -- quantize Q, K and V with one unified mode, in one launch.
 *   Sources: wiki "FA 量化" 组合1 (INT8 per-head static: s_h = amax_h/127,
 *   code = int8 round-half-even(x / s_h), saturated to [-128, 127], the
 *   range printed in MindIE SD "量化", Linear量化 / 通用原理), 组合2 (FP8
 *   E4M3 per-token dynamic: s = amax_token/448, code = e4m3(x / s)),
 *   组合3 (MXFP4: per 32 elements of head_dim, e = floor(log2 amax) - 2,
 *   E8M0 byte e + 127, code = e2m1(x / 2^e)); MindIE SD FA量化 / 块量化
 *   (E4M3 with one scale = amax/448 per block of block_tokens tokens);
 *   "FA 量化", 该类下的模式清单: FA PerHead with FP8 (组合1's calibration,
 *   s_h = amax_h/448, values past the calibrated range saturate to +-448) and
 *   FA PerToken with INT8 (组合2's per-token amax, s = amax_token/127) and
 *   FA PerBlock with MXFP8 (组合3's rule with E4M3 elements: per 32 elements
 *   of head_dim, e = floor(log2 amax) - 8, code = e4m3(x / 2^e), saturating).
 *   Rounding is round-half-to-even, saturating; x / s is rounded as one IEEE
 *   fp32 division; a zero scale gives zero codes.
 *   q, k, v: bf16 inputs; any of them may be NULL to skip that operand.
 *   mode: one of the quantized modes.  amax_q/k/v: device fp32 [H] from
 *   fa_calibrate_per_head, required for FA_MODE_INT8_PER_HEAD and
 *   FA_MODE_FP8_PER_HEAD (NULL there -> FA_ERR_NO_CALIBRATION), ignored
 *   otherwise.
 *   q_out/k_out/v_out: caller-filled descriptors whose codes/scales point to
 *   buffers of the sizes above; their dims/layout must equal the input's
 *   and their mode must equal `mode`.  For FA_MODE_FP8_BLOCK,
 *   block_tokens >= 1 (the pages use 128 for Q and 256 for K/V).
 */
FAQ_API fa_status fa_quantize(const fa_tensor* q, const fa_tensor* k, const fa_tensor* v, fa_mode mode,
                      const float* amax_q, const float* amax_k, const float* amax_v, fa_qtensor* q_out,
                      fa_qtensor* k_out, fa_qtensor* v_out, fa_stream_t s);

/*
 * fa_rotate_quantize -- rotate Q and K, then FP8 block-quantize Q, K, V.
 *   Source: MindIE SD "量化", FA量化 / 技术特点: 旋转 (Q and K are
 *   multiplied by trained rotation matrices q_rot / k_rot to spread
 *   outliers; V is not rotated), then 块量化 (E4M3, block 128 for Q and
 *   256 for K/V).  Q' = bf16(Q R_q) (fp32 accumulation, one rounding),
 *   K' = bf16(K R_k), V' = V; then FA_MODE_FP8_BLOCK quantization.
 *   rot_q, rot_k: device bf16 [D, D] row-major (x' = x * R).  q_block,
 *   kv_block: tokens per scale block; must equal q_out->block_tokens and
 *   k_out/v_out->block_tokens.  rot_q_dbg / rot_k_dbg: nullable device bf16
 *   outputs (input layout) receiving Q', K' as rounded before quantization.
 *   Outputs must have mode FA_MODE_FP8_BLOCK.
 */
FAQ_API fa_status fa_rotate_quantize(const fa_tensor* q, const fa_tensor* k, const fa_tensor* v, const void* rot_q,
                             const void* rot_k, int q_block, int kv_block, fa_qtensor* q_out, fa_qtensor* k_out,
                             fa_qtensor* v_out, void* rot_q_dbg, void* rot_k_dbg, fa_stream_t s);

/*
 * fa_rotate_quantize_hadamard -- fa_rotate_quantize for rotations of the
 * Hadamard-times-signs form, given by their signs instead of a D x D matrix
 * in memory (the rotation specialization of the same flow).
 *   Source: MindIE SD "量化", FA量化 / 技术特点: 旋转 (Q and K multiplied by a
 *   rotation before 块量化), with the rotation R = bf16(H_D diag(sigma) /
 *   sqrt(D)): H_D the Sylvester Hadamard matrix, entry (i, j) =
 *   (-1)^popcount(i & j), and sigma a vector of signs.  Every entry of R is
 *   +-c with c = bf16(1 / sqrt(D)), so x R = c * sigma * FWHT(x) elementwise,
 *   FWHT(x)_j = sum_d x_d (-1)^popcount(d & j).  The rotated row is evaluated
 *   in fp32 and rounded once to bf16, then quantized exactly as
 *   fa_rotate_quantize does (FA_MODE_FP8_BLOCK).  With D = 128 and blocks
 *   that divide 256 tokens, the rotation runs in fa_rotate_quantize's
 *   pipeline with R built in shared memory from the signs (results identical
 *   to fa_rotate_quantize given that R); otherwise a fast Walsh-Hadamard
 *   transform computes it (results equal up to the order of the fp32 sums).
 *   sign_bits_q, sign_bits_k: HOST pointers to D / 32 words; bit j % 32 of
 *   word j / 32 set means sigma_j = -1; NULL means every sigma_j = +1.
 *   Everything else (q_block, kv_block, outputs, the nullable rot_*_dbg
 *   outputs, layouts, errors) as fa_rotate_quantize, without R pointers.
 *   Any block size >= 1 is accepted.
 */
FAQ_API fa_status fa_rotate_quantize_hadamard(const fa_tensor* q, const fa_tensor* k, const fa_tensor* v,
                                              const uint32_t* sign_bits_q, const uint32_t* sign_bits_k,
                                              int q_block, int kv_block, fa_qtensor* q_out, fa_qtensor* k_out,
                                              fa_qtensor* v_out, void* rot_q_dbg, void* rot_k_dbg, fa_stream_t s);

/*
 * fa_attention_quant -- flash attention on quantized Q/K/V, bf16 output.
 *   Sources: MindIE SD "量化", FA量化 / FP8 Attention (attention computed
 *   on the low-bit operands, the output dequantized back to the original
 *   precision); FlashAttention (Dao et al. 2022), cited by the wiki's
 *   参考资料: O = softmax(Q K^T * scale) V with an online softmax.
 *   q, k, v: quantized descriptors of one layout and D.  Each branch has its
 *   own mode (msModelSlim "fa3_quant 配置说明" §2.3 FA3AttentionDetails:
 *   fa_q / fa_k / fa_v each take a QConfig; the wiki's 分支组合 note: a branch
 *   left unset is not quantized): FA_MODE_FLOAT marks an unquantized branch,
 *   whose `codes` is the bf16 tensor itself (scales unused).  When the three
 *   modes differ, or any is FA_MODE_FLOAT, the call computes attention on
 *   the dequantized operands (x = code * scale, MX: code * 2^(e - 127)):
 *   Q and K are dequantized to bf16 in the workspace (a float branch is read
 *   in place), V' is made from V's own mode, and QK^T runs on bf16 tensor
 *   cores; all three FLOAT is plain bf16 attention.  A V in an MX mode needs
 *   D == 128 there.
 *   q->B == k->B == v->B, k and v have equal dims, q->H % k->H == 0 (GQA:
 *   query head h reads kv head h / (Hq / Hkv)).  causal: key j is visible
 *   to query i iff j <= i + (Sk - Sq).  softmax_scale <= 0 means 1/sqrt(D).
 *   out: device bf16, q's layout and dims.  lse: nullable device fp32
 *   [B, Hq, Sq], natural-log sum-exp of the scaled scores (-inf for a row
 *   with no visible key, whose output is 0).
 *   workspace: device memory of at least fa_attention_workspace_size_qkv()
 *   bytes, 256-byte aligned, owned by the caller and only used during the
 *   call's kernels (FA_ERR_WORKSPACE if missing, short or misaligned).
 *   Decode (q->S == 1) keeps its split-KV partials there before an LSE
 *   combine.  Prefill keeps there, made once per call by a pre-pass and
 *   read by every query tile: V' = fp16(code * s_v / r_t) (r_t the largest
 *   V scale of each 128-key tile; MXFP4: V' = fp16(e2m1 * 2^(e - E_t)), E_t
 *   the tile's largest UE8M0 exponent), a 16-byte record per tile holding
 *   r_t (E_t), and 512 bytes of K scales per tile (128 per-key floats, or
 *   MXFP4's scale-factor atom).  num_splits (decode only): 0 = automatic.
 *   Modes run here: INT8_PER_HEAD, FP8_PER_TOKEN, FP8_BLOCK, MXFP4_PER_BLOCK,
 *   FP8_PER_HEAD, INT8_PER_TOKEN and MXFP8_PER_BLOCK for prefill (the MX modes
 *   with D == 128); INT8_PER_HEAD for decode (others -> FA_ERR_UNSUPPORTED).
 */
FAQ_API fa_status fa_attention_quant(const fa_qtensor* q, const fa_qtensor* k, const fa_qtensor* v, int causal,
                             float softmax_scale, void* out, float* lse, int num_splits, void* workspace,
                             size_t ws_bytes, fa_stream_t s);

/* Size of the fixed device buffer that fa_attention_decode_noalloc keeps its
 * split-KV partials in (16 MiB per GPU that loads the library). */
#define FA_DECODE_NOALLOC_SCRATCH_BYTES (16u << 20)

/*
 * fa_attention_decode_noalloc -- the INT8 split-KV decode of
 * fa_attention_quant (q->S == 1) for callers that cannot allocate device
 * memory where they run decode: a serving loop that must never synchronise
 * the device (cudaMalloc / cudaFree can), or plain C/C++ host code linking
 * libfaq.so without a device allocator of its own.  The pages have no
 * counterpart to this call; it only changes where the per-split partial
 * results live.
 *   Instead of a caller workspace, the partials live in a buffer of
 *   FA_DECODE_NOALLOC_SCRATCH_BYTES inside the library's own device memory
 *   (one per GPU, held until the process exits).  Nothing is allocated and
 *   no allocating routine is called.
 *   The first call on a device looks the buffer's device address up (with
 *   that device current) and caches it; make that first call before any
 *   stream capture.
 *   All calls on a device share the buffer: calls whose kernels overlap on
 *   the GPU (for example on two streams) race; keep them on one stream or
 *   serialise them.  Each call overwrites every partial it reads, so nothing
 *   needs clearing between calls.
 *   Arguments as for fa_attention_quant, restricted to FA_MODE_INT8_PER_HEAD,
 *   q->S == 1, D == 128 and Hq / Hkv in {1, 2, 4, 8, 16} (FA_ERR_UNSUPPORTED
 *   otherwise).  num_splits: 0 = automatic, reduced until the partials fit;
 *   a split count whose partials, B * Hq * splits * (D + 2) * 4 bytes,
 *   exceed the buffer returns FA_ERR_WORKSPACE before any launch.
 */
FAQ_API fa_status fa_attention_decode_noalloc(const fa_qtensor* q, const fa_qtensor* k, const fa_qtensor* v,
                                              float softmax_scale, void* out, float* lse, int num_splits,
                                              fa_stream_t s);

/*
 * fa_decode_append -- one decode step on an INT8 per-head KV cache: the new
 * token's query is quantized, its key and value are quantized into the cache
 * at position `pos`, and split-KV attention runs over the cache's first
 * pos + 1 tokens, all in the decode kernel (then the LSE combine).
 *   Sources: msModelSlim wiki "FA 量化", 概述 (K/V quantization compresses
 *   the cache for long-context decode; 组合1 INT8 per-head static scales),
 *   "量化模式", 模式索引 (decode); the split-KV decode and combine of
 *   fa_attention_quant.
 *   q: bf16 [B, Hq, 1, D]; k_new, v_new: bf16 [B, Hkv, 1, D]; D == 128,
 *   Hq / Hkv in {1, 2, 4, 8, 16}; one layout for every operand.
 *   amax_q/k/v: device fp32 [Hq] / [Hkv] / [Hkv] calibration maxima
 *   (s = amax / 127 as in fa_quantize; NULL -> FA_ERR_NO_CALIBRATION).
 *   k_cache, v_cache: FA_MODE_INT8_PER_HEAD descriptors whose S is the
 *   cache capacity; codes at positions < pos must already hold the earlier
 *   tokens (quantized with the same amax); position pos is written by this
 *   call, and the scale arrays [Hkv] are (re)written with amax / 127.
 *   0 <= pos < capacity.  out: bf16 [B, Hq, 1, D] in the layout; lse:
 *   nullable [B, Hq].  workspace: fa_decode_append_workspace_size() bytes,
 *   256-byte aligned.  num_splits: 0 = automatic (from pos + 1 keys).
 *   Calls on one cache are ordered by the stream; the cache is read and
 *   written by this call's kernels only.
 */
FAQ_API fa_status fa_decode_append(const fa_tensor* q, const fa_tensor* k_new, const fa_tensor* v_new,
                                   const float* amax_q, const float* amax_k, const float* amax_v,
                                   fa_qtensor* k_cache, fa_qtensor* v_cache, int pos, float softmax_scale,
                                   void* out, float* lse, int num_splits, void* workspace, size_t ws_bytes,
                                   fa_stream_t s);

/* Workspace bytes fa_decode_append needs (its split-KV partials,
 * B*Hq*splits*(D+2)*4).  Returns 0 on invalid arguments. */
FAQ_API size_t fa_decode_append_workspace_size(const fa_tensor* q, const fa_qtensor* k_cache, int pos,
                                               int num_splits);

/* Workspace bytes fa_attention_quant needs for these operands and split
 * count: decode B*Hq*splits*(D+2)*4; prefill (every mode, the MX modes with
 * D == 128 only) B*Hkv*Sk*D*2 + B*Hkv*T*16 + B*Hkv*T*512, each part rounded
 * up to 256, with T the number of key tiles: ceil(Sk/112) for the MX modes
 * (MXFP4, MXFP8), ceil(Sk/128) otherwise.  Returns 0 on invalid arguments. */
FAQ_API size_t fa_attention_workspace_size(const fa_qtensor* q, const fa_qtensor* k, int num_splits);

/* The same for any three branches: equal to fa_attention_workspace_size when
 * q, k and v share one quantized mode; with mixed branches (modes differ, or
 * one is FA_MODE_FLOAT) the prefill parts above plus the bf16 dequantized
 * copies of Q (B*Hq*Sq*D*2) and K (B*Hkv*Sk*D*2) that are not FA_MODE_FLOAT,
 * each rounded up to 256.  fa_attention_workspace_size(q, k) already returns
 * this when q and k differ in mode or one is FA_MODE_FLOAT; when only v
 * differs it cannot know, so size mixed calls with this function.  Returns 0
 * on invalid arguments (v NULL included). */
FAQ_API size_t fa_attention_workspace_size_qkv(const fa_qtensor* q, const fa_qtensor* k, const fa_qtensor* v,
                                               int num_splits);

/* Synchronise `s`, read and clear this device's status word.  Returns
 * FA_ERR_TIMEOUT if a kernel's bounded wait ran out since the last check,
 * FA_ERR_BOUNDS if (in a library built with FA_DEBUG_BOUNDS) an index check
 * failed -- the access was skipped, so the outputs are not valid --,
 * FA_ERR_CUDA if the stream reports an error, FA_OK otherwise.  The first
 * event since the last check is the one reported. */
FAQ_API fa_status fa_check_device_status(fa_stream_t s);

/* Static text for a status code. */
FAQ_API const char* fa_status_str(fa_status st);

/* Library version string. */
FAQ_API const char* fa_version(void);

#ifdef __cplusplus
}
#endif
#endif /* FAQ_H */
