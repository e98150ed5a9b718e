/*
 * faq_oracle.h -- the oracle: a plain, slow, fp64 CPU statement of FA
 * quantization and of attention on the dequantized operands.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  It shares no code,
 * header, table or constant with the CUDA path under
 * quantized_attention_amax_b200/, and it does not include that path's
 * headers.  The product path never calls it.
 *
 * Sources (web pages on FA quantization):
 *   [FA]   msModelSlim wiki "FA 量化" -- sections 概述 (overview),
 *          分支组合 (branch combinations: 组合1 INT8 per-head static,
 *          组合2 FP8 E4M3 per-token dynamic, 组合3 MXFP4 per-block dynamic),
 *          该类下的模式清单 (mode list: FA PerHead INT8/FP8 static, FA PerToken
 *          INT8/FP8 dynamic, FA PerBlock MXFP8/MXFP4).
 *   [MODE] msModelSlim wiki "量化模式" -- 模式索引 (mode index): FakeQuant
 *          means quantize and immediately dequantize.
 *   [SD]   MindIE SD "量化" -- Linear 量化 / 通用原理 (INT8 range figure
 *          [-max, max] -> [-128, 127]); FA量化 / 技术特点 (rotate -> block
 *          quant, Q block 128, K/V block 256 -> FP8 attention, output back
 *          to the original precision); 注意事项 (layouts BNSD and BSND).
 *   FlashAttention (Dao et al., NeurIPS 2022), cited by [FA] 参考资料:
 *          softmax(Q K^T * scale) V, exact.
 *
 * Parity status of each function is stated beside it and in the design
 * notes; every function here is pinned by the "not gpu" tests.
 *
 * Layouts: BNSD = [B, H, S, D], BSND = [B, S, H, D]; D is contiguous in both.
 * Scale arrays are canonical whatever the data layout:
 *   INT8 per head  : fp32 [H]
 *   FP8 per head   : fp32 [H]
 *   FP8 per token  : fp32 [B, H, S]
 *   INT8 per token : fp32 [B, H, S]
 *   FP8 block      : fp32 [B, H, ceil(S / blk)]
 *   MXFP4, MXFP8   : uint8 E8M0 [B, H, S, D / 32]
 * MXFP4 codes are packed [.., D/2] in the data layout, element 2i in the low
 * nibble, 2i+1 in the high nibble.
 */
#ifndef FAQ_ORACLE_H
#define FAQ_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORC_LAYOUT_BNSD = 0, ORC_LAYOUT_BSND = 1 };
enum {
  ORC_MODE_FLOAT = 0,          /* bf16, not quantized                        */
  ORC_MODE_INT8_PER_HEAD = 1,  /* [FA] 组合1                                  */
  ORC_MODE_FP8_PER_TOKEN = 2,  /* [FA] 组合2                                  */
  ORC_MODE_MXFP4 = 3,          /* [FA] 组合3                                  */
  ORC_MODE_FP8_BLOCK = 4,      /* [SD] FA量化 块量化                           */
  ORC_MODE_FP8_PER_HEAD = 5,   /* [FA] 模式清单: FA PerHead, FP8               */
  ORC_MODE_INT8_PER_TOKEN = 6, /* [FA] 模式清单: FA PerToken, INT8             */
  ORC_MODE_MXFP8 = 7           /* [FA] 模式清单: FA PerBlock, MXFP8            */
};

/* A quantized (or bf16) operand as the oracle sees it. */
typedef struct {
  int mode;
  const void* codes;   /* int8 / e4m3 bytes / packed e2m1 / bf16 bits     */
  const void* scales;  /* see the table above; unused for ORC_MODE_FLOAT  */
  int B, H, S, D;
  int layout;
  int blk;             /* tokens per scale block, ORC_MODE_FP8_BLOCK only  */
} orc_qt;

/* ---- scalar codecs (format definitions) ---------------------------------*/
float    orc_bf16_to_f32(uint16_t h);
uint16_t orc_f64_to_bf16(double x);     /* one round-to-nearest-even        */
uint8_t  orc_e4m3_encode(float v);      /* float8_e4m3fn, RNE, sat +-448    */
double   orc_e4m3_decode(uint8_t c);
uint8_t  orc_e2m1_encode(float v);      /* 4-bit E2M1, RNE, sat +-6         */
double   orc_e2m1_decode(uint8_t c);
int8_t   orc_int8_encode(float v);      /* RNE to integer, clamp [-128,127] */
int      orc_mx_exponent(float amax);   /* floor(log2 amax) - 2, [-127,127] */
int      orc_mx_exponent_e4m3(float amax); /* floor(log2 amax) - 8, [-127,127] */

/* ---- quantizers ---------------------------------------------------------*/
void orc_calibrate_per_head(const uint16_t* x, int B, int H, int S, int D,
                            int layout, float* amax /* [H], running max */);
void orc_quantize_int8_per_head(const uint16_t* x, int B, int H, int S, int D,
                                int layout, const float* amax,
                                int8_t* codes, float* scales /* [H] */);
void orc_quantize_fp8_per_token(const uint16_t* x, int B, int H, int S, int D,
                                int layout, uint8_t* codes,
                                float* scales /* [B,H,S] */);
void orc_quantize_fp8_per_head(const uint16_t* x, int B, int H, int S, int D,
                               int layout, const float* amax,
                               uint8_t* codes, float* scales /* [H] */);
void orc_quantize_int8_per_token(const uint16_t* x, int B, int H, int S, int D,
                                 int layout, int8_t* codes,
                                 float* scales /* [B,H,S] */);
void orc_quantize_mxfp4(const uint16_t* x, int B, int H, int S, int D,
                        int layout, uint8_t* codes /* packed */,
                        uint8_t* e8m0 /* [B,H,S,D/32] */);
void orc_quantize_mxfp8(const uint16_t* x, int B, int H, int S, int D,
                        int layout, uint8_t* codes /* e4m3 [..D] */,
                        uint8_t* e8m0 /* [B,H,S,D/32] */);
void orc_rotate_f64(const uint16_t* x, int B, int H, int S, int D, int layout,
                    const uint16_t* R /* [D,D] row-major, x*R */,
                    double* out /* same layout as x */);
void orc_rotate(const uint16_t* x, int B, int H, int S, int D, int layout,
                const uint16_t* R, uint16_t* out /* bf16, same layout */);
void orc_quantize_fp8_block(const uint16_t* x, int B, int H, int S, int D,
                            int layout, int blk, uint8_t* codes,
                            float* scales /* [B,H,ceil(S/blk)] */);

/* ---- dequantization and attention ---------------------------------------*/
double orc_dequant_elem(const orc_qt* t, int b, int h, int s, int d);
void   orc_dequant_head(const orc_qt* t, int b, int h, double* out /* [S,D] */);

/* Exact softmax attention on the dequantized operands, for the query rows
 * listed in `rows` (all Sq rows when rows == NULL).  GQA: query head h reads
 * kv head h / (Hq / Hkv).  Causal: key j is visible to query i iff
 * j <= i + (Sk - Sq).  scale <= 0 means 1/sqrt(D).  out: [B, Hq, nrows, D];
 * lse (nullable): natural-log sum-exp [B, Hq, nrows]; a row with no visible
 * key gets out = 0 and lse = -inf. */
void orc_attention(const orc_qt* q, const orc_qt* k, const orc_qt* v,
                   int causal, double scale, const int* rows, int nrows,
                   double* out, double* lse);

/* Array forms of the scalar codecs. */
void orc_e4m3_encode_n(const float* v, uint8_t* out, size_t n);
void orc_e2m1_encode_n(const float* v, uint8_t* out, size_t n);
void orc_int8_encode_n(const float* v, int8_t* out, size_t n);
void orc_mx_exponent_n(const float* v, int* out, size_t n);
void orc_f64_to_bf16_n(const double* v, uint16_t* out, size_t n);

int orc_num_threads(void);

#ifdef __cplusplus
}
#endif
#endif
