// attn.cu -- flash attention on quantized Q/K/V for sm_100a (prefill).
//
// Computes O = softmax(S) V with S = (Q^ K^T) * s_q * s_k * softmax_scale on
// the low-bit operands (MindIE SD "量化", FA量化 / FP8 Attention: attention
// in the low-precision domain, output dequantized to the original bf16;
// FlashAttention's online softmax, cited by the wiki "FA 量化" 参考资料).
//
// One CTA owns one 128-row Q tile of one (batch, query head) and streams the
// visible 128-key K/V tiles:
//   warp 0      TMA producer: Q once, then K and V code tiles into a 2-stage
//               ring (128B- or 64B-swizzled, zero-filled past the sequence).
//   warp 1      MMA issuer (one thread): S = Q K^T with tcgen05.mma
//               kind::f8f6f4 (E4M3), kind::i8 (INT8) or block-scaled
//               kind::mxf4 (E2M1 with the UE8M0 scales of every 32 elements
//               along head_dim copied into TMEM) into a double-buffered S in
//               TMEM; then O += P' V' with kind::f16 into O in TMEM.
//   warps 2-3   V converters: V code tile -> V' = fp16(code) (exact; for
//               MXFP4 fp16(e2m1 * 2^(e - e_ref)) with e_ref the largest
//               exponent the CTA reads) in the MN-major 128B-swizzled layout
//               the P.V MMA reads.
//   warps 4-7   softmax, one thread per query row: load S from TMEM, apply
//               the K scales, causal / ragged masks, online max and sum in
//               the exp2 domain, P' = fp16(p * s_v / vref) into shared memory.
//               O is rescaled in TMEM only when the row max grows by more
//               than 2^8 (p stays <= 256).  Epilogue: O * vref / l -> bf16.
// V's scales vary along the P.V contraction, so they are folded into P (in
// fp16, 11-bit precision) rather than into an 8-bit P: see the design notes.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>

#include "attn_common.cuh"
#include "internal.cuh"
#include "sm100.cuh"

namespace faq {
namespace {
using namespace attn;

constexpr int BM = 128;  // query rows per tile
constexpr int BN = 128;  // keys per tile
constexpr int NS = 2;    // K/V code stages
constexpr int NTHREADS = 256;

enum { KIND_E4M3 = 0, KIND_S8 = 1, KIND_MXF4 = 2 };

struct AttnParams {
  int B, Hq, Hkv, Sq, Sk, group, causal, layout;
  float scale_log2;  // softmax_scale * log2(e)
  const float* qs;
  const float* ks;
  const float* vs;
  int q_blk, k_blk, v_blk;     // tokens per scale (1 = per token); 0 = one scale per head
  int q_nblk, k_nblk, v_nblk;  // scale blocks per (b, h)
  const uint8_t* qe8;  // MXFP4: E8M0 [B, H, S, D/32]
  const uint8_t* ke8;
  const uint8_t* ve8;
  __nv_bfloat16* out;
  float* lse;
  int* status;
  int n_qtiles;
};

template <int KIND, int D>
struct Smem {
  static constexpr uint32_t RB = KIND == KIND_MXF4 ? D / 2 : D;  // code bytes per token row
  static constexpr uint32_t Q = 0;
  static constexpr uint32_t K = Q + BM * RB;
  static constexpr uint32_t V = K + NS * BN * RB;
  static constexpr uint32_t VH = V + NS * BN * RB;     // 2 x fp16 V' tiles
  static constexpr uint32_t P = VH + 2 * BN * D * 2;   // 2 x fp16 P' tiles
  static constexpr uint32_t SC = P + 2 * BM * BN * 2;  // [2][BN] K scales, [2][BN] V factors
  static constexpr uint32_t SF = SC + 4 * BN * 4;      // MXFP4: Q scale atom + NS K scale atoms (512 B each)
  static constexpr uint32_t BAR = SF + (1 + NS) * 512;
  static constexpr uint32_t TOTAL = BAR + 512;
  static constexpr uint32_t ALLOC = TOTAL + 1024;  // slack for 1024-byte alignment
};

// Barrier slots.
enum {
  B_Q = 0,
  B_KFULL = 1,   // [2]
  B_KEMPTY = 3,  // [2]
  B_VFULL = 5,   // [2]
  B_VEMPTY = 7,  // [2]
  B_VHFULL = 9,  // [2]
  B_SFULL = 11,  // [2]
  B_SEMPTY = 13, // [2]
  B_PFULL = 15,  // [2]
  B_PVDONE = 17, // [2]
  B_FINAL = 19,
  B_SC = 20,     // [2] softmax threads published this tile's per-column scales
  B_RED = 22,    // softmax threads published their V-scale maxima
  B_ERED = 23,   // converter threads published their E8M0 maxima (MXFP4)
  B_COUNT = 24
};

template <int KIND, int D>
__global__ void __launch_bounds__(NTHREADS, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                    const __grid_constant__ CUtensorMap tmv, const AttnParams p) {
  using L = Smem<KIND, D>;
  constexpr uint32_t RB = L::RB;
  constexpr bool MX = KIND == KIND_MXF4;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L::BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + B_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar + B_COUNT + 1);
  float* red = reinterpret_cast<float*>(bar + B_COUNT + 2);
  float* sKsc = reinterpret_cast<float*>(smem + L::SC);           // [2][BN]
  float* sVf = reinterpret_cast<float*>(smem + L::SC + 2 * BN * 4);  // [2][BN]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---- work item
  const int nbh = p.B * p.Hq;
  const int widx = blockIdx.x;
  const int qt = p.causal ? (p.n_qtiles - 1 - widx / nbh) : (widx / nbh);
  const int bh = widx % nbh;
  const int hq = bh % p.Hq, b = bh / p.Hq;
  const int hk = hq / p.group;
  const int bhk = b * p.Hkv + hk;
  const int q0 = qt * BM;
  const int diag = p.Sk - p.Sq;  // key j visible to query i iff j <= i + diag (causal)
  int kv_end = p.Sk;
  if (p.causal) kv_end = min(p.Sk, max(0, q0 + BM - 1 + diag + 1));
  const int n_tiles = (kv_end + BN - 1) / BN;

  if (tid == 0) {
    mbar_init(&bar[B_Q], 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar[B_KFULL + i], 1);
      mbar_init(&bar[B_KEMPTY + i], 1);
      mbar_init(&bar[B_VFULL + i], 1);
      mbar_init(&bar[B_VEMPTY + i], 2);
      mbar_init(&bar[B_VHFULL + i], 2);
      mbar_init(&bar[B_SFULL + i], 1);
      mbar_init(&bar[B_SEMPTY + i], 4);
      mbar_init(&bar[B_PFULL + i], 4);
      mbar_init(&bar[B_PVDONE + i], 1);
    }
    mbar_init(&bar[B_FINAL], 1);
    mbar_init(&bar[B_SC], 128);
    mbar_init(&bar[B_SC + 1], 128);
    mbar_init(&bar[B_RED], 128);
    mbar_init(&bar[B_ERED], 64);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const uint32_t tS[2] = {tbase, tbase + 128};
  const uint32_t tO = tbase + 256;
  const uint32_t tSFA = tbase + 384;                       // MXFP4: Q scale factors
  const uint32_t tSFB[2] = {tbase + 392, tbase + 400};     // MXFP4: K scale factors

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (MX && n_tiles > 0) {
      // Scale-factor atoms (all 32 lanes): Q once, then every K tile in the
      // stage of its codes.  Published with the TMA's barrier arrival below.
      write_sf_atom(smem + L::SF, p.qe8, (long long)(b * p.Hq + hq) * p.Sq + q0, p.Sq - q0, lane);
      fence_async_smem();
      __syncwarp();
    }
    if (lane == 0 && n_tiles > 0) {
      tma_prefetch_desc(&tmq);
      tma_prefetch_desc(&tmk);
      tma_prefetch_desc(&tmv);
      const bool bnsd = p.layout == FA_LAYOUT_BNSD;
      mbar_arrive_expect_tx(&bar[B_Q], BM * RB);
      tma_load_4d(smem + L::Q, &tmq, &bar[B_Q], 0, bnsd ? q0 : hq, bnsd ? hq : q0, b);
    }
    int j = 0;
    const bool bnsd = p.layout == FA_LAYOUT_BNSD;
    for (; j < n_tiles; ++j) {
      const int s = j % NS;
      const int k0 = j * BN;
      bool ok = true;
      if (j >= NS) ok = mbar_wait(&bar[B_KEMPTY + s], ((j / NS) - 1) & 1, abort_flag, p.status, 1);
      if (!__all_sync(0xffffffffu, ok)) break;
      if (MX) {
        write_sf_atom(smem + L::SF + (1 + s) * 512, p.ke8, (long long)bhk * p.Sk + k0, p.Sk - k0, lane);
        fence_async_smem();
        __syncwarp();
      }
      if (lane == 0) {
        mbar_arrive_expect_tx(&bar[B_KFULL + s], BN * RB);
        tma_load_4d(smem + L::K + s * BN * RB, &tmk, &bar[B_KFULL + s], 0, bnsd ? k0 : hk, bnsd ? hk : k0, b);
        if (j >= NS) ok = mbar_wait(&bar[B_VEMPTY + s], ((j / NS) - 1) & 1, abort_flag, p.status, 2);
        if (ok) {
          mbar_arrive_expect_tx(&bar[B_VFULL + s], BN * RB);
          tma_load_4d(smem + L::V + s * BN * RB, &tmv, &bar[B_VFULL + s], 0, bnsd ? k0 : hk, bnsd ? hk : k0, b);
        }
      }
      if (!__all_sync(0xffffffffu, ok)) { ++j; break; }
    }
    if (lane == 0 && *abort_flag) {
      // Let loads already issued land before the CTA can exit.
      for (int t = max(0, j - NS); t < j; ++t) {
        mbar_wait(&bar[B_KFULL + t % NS], (t / NS) & 1, abort_flag, nullptr, 0);
        mbar_wait(&bar[B_VFULL + t % NS], (t / NS) & 1, abort_flag, nullptr, 0);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0 && n_tiles > 0) {
      constexpr uint32_t SW = RB == 128 ? kSwz128 : kSwz64;
      constexpr uint32_t SBO8 = RB == 128 ? 1024 : 512;
      constexpr uint32_t idesc_qk = KIND == KIND_E4M3 ? make_idesc(kAccF32, kFmtE4M3, kFmtE4M3, 0, 0, BN, BM)
                                                      : make_idesc(kAccS32, kFmtS8, kFmtS8, 0, 0, BN, BM);
      constexpr uint32_t idesc_pv = make_idesc(kAccF32, kFmtF16, kFmtF16, 0, 1, D, BM);
      const uint32_t sQ = smem_u32(smem + L::Q);
      bool ok = mbar_wait(&bar[B_Q], 0, abort_flag, p.status, 3);
      if (MX && ok) {
        tc_fence_after();
        sf_to_tmem(tSFA, smem_u32(smem + L::SF));
      }
      for (int j = 0; ok && j <= n_tiles; ++j) {
        if (j < n_tiles) {
          const int s = j % NS, bb = j & 1;
          if (!mbar_wait(&bar[B_KFULL + s], (j / NS) & 1, abort_flag, p.status, 4)) break;
          if (j >= 2 && !mbar_wait(&bar[B_SEMPTY + bb], ((j >> 1) - 1) & 1, abort_flag, p.status, 5)) break;
          tc_fence_after();
          const uint32_t sK = smem_u32(smem + L::K + s * BN * RB);
          if (MX) sf_to_tmem(tSFB[bb], smem_u32(smem + L::SF + (1 + s) * 512));
#pragma unroll
          for (int kk = 0; kk < (int)RB / 32; ++kk) {
            const uint64_t da = make_sdesc(sQ + kk * 32, 16, SBO8, SW);
            const uint64_t db = make_sdesc(sK + kk * 32, 16, SBO8, SW);
            if (KIND == KIND_E4M3)
              mma_f8f6f4(tS[bb], da, db, idesc_qk, kk > 0);
            else if (KIND == KIND_S8)
              mma_i8(tS[bb], da, db, idesc_qk, kk > 0);
            else  // 64 E2M1 per MMA: scale bytes 2kk, 2kk+1 of each row
              mma_mxf4(tS[bb], da, db, make_idesc_bs(kFmtE2M1x, kFmtE2M1x, BN, BM, 2 * kk, 2 * kk), tSFA, tSFB[bb],
                       kk > 0);
          }
          mma_commit(&bar[B_KEMPTY + s]);
          mma_commit(&bar[B_SFULL + bb]);
        }
        if (j >= 1) {
          const int jj = j - 1, bb = jj & 1;
          if (!mbar_wait(&bar[B_PFULL + bb], (jj >> 1) & 1, abort_flag, p.status, 6)) break;
          if (!mbar_wait(&bar[B_VHFULL + bb], (jj >> 1) & 1, abort_flag, p.status, 7)) break;
          tc_fence_after();
          const uint32_t sP = smem_u32(smem + L::P + bb * BM * BN * 2);
          const uint32_t sVh = smem_u32(smem + L::VH + bb * BN * D * 2);
#pragma unroll
          for (int ks = 0; ks < BN / 16; ++ks) {
            const uint64_t da = make_sdesc(sP + (ks >> 2) * (BM * 128) + (ks & 3) * 32, 16, 1024, kSwz128);
            const uint64_t db = make_sdesc(sVh + ks * 16 * 128, BN * 128, 1024, kSwz128);
            mma_f16(tO, da, db, idesc_pv, (jj > 0 || ks > 0) ? 1u : 0u);
          }
          mma_commit(&bar[B_PVDONE + bb]);
        }
      }
      // All tcgen05 work issued by this thread has completed before TMEM is freed.
      mma_commit(&bar[B_FINAL]);
      mbar_wait(&bar[B_FINAL], 0, abort_flag, nullptr, 0);
    }
    __syncwarp();
  } else if (warp < 4) {
    // --------------------------------------------------------- V converter
    const int ct = tid - 64;  // 0..63
    int eref = 0;  // MXFP4: largest E8M0 byte of the V rows this CTA reads
    if (MX) {
      int m = 0;
      for (int t = ct; t < kv_end; t += 64) {
        const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(p.ve8 + ((long long)bhk * p.Sk + t) * 4));
        m = max(m, (int)max(max(w & 0xFF, (w >> 8) & 0xFF), max((w >> 16) & 0xFF, w >> 24)));
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
      int* ered = reinterpret_cast<int*>(red) + 4;
      if (lane == 0) ered[warp - 2] = m;
      mbar_arrive(&bar[B_ERED]);
      warp_wait(&bar[B_ERED], 0, abort_flag, p.status, 16);
      eref = max(ered[0], ered[1]);
    }
    for (int j = 0; j < n_tiles; ++j) {
      const int s = j % NS, bb = j & 1;
      if (!warp_wait(&bar[B_VFULL + s], (j / NS) & 1, abort_flag, p.status, 8)) break;
      if (j >= 2 && !warp_wait(&bar[B_PVDONE + bb], ((j >> 1) - 1) & 1, abort_flag, p.status, 9)) break;
      const uint8_t* src = smem + L::V + s * BN * RB;
      uint8_t* dst = smem + L::VH + bb * BN * D * 2;
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        const int r = ct + rr * 64;
        if (MX) {
          // 16 raw bytes = 32 E2M1 = one 32-element scale block of head_dim.
          const int key = j * BN + r;
          uint32_t e4 = 0;
          if (key < p.Sk) e4 = __ldg(reinterpret_cast<const uint32_t*>(p.ve8 + ((long long)bhk * p.Sk + key) * 4));
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            const uint4 raw = *reinterpret_cast<const uint4*>(src + swz64_offset(r, c));  // D = 128: 64-byte rows
            const int de = (int)((e4 >> (8 * c)) & 0xFF) - eref;  // <= 0
            const __half fs = de >= -24 ? __float2half_rn(ldexpf(1.0f, de)) : __float2half_rn(0.0f);
            const __half2 f2 = __halves2half2(fs, fs);
            const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
            uint32_t h[16];
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
              for (int y = 0; y < 2; ++y) {
                uint32_t v2 = e2m1x2_to_h2((w[q] >> (16 * y)) & 0xFF);
                uint32_t v3 = e2m1x2_to_h2((w[q] >> (16 * y + 8)) & 0xFF);
                __half2 a = __hmul2(*reinterpret_cast<__half2*>(&v2), f2);
                __half2 c2 = __hmul2(*reinterpret_cast<__half2*>(&v3), f2);
                h[q * 4 + y * 2] = *reinterpret_cast<uint32_t*>(&a);
                h[q * 4 + y * 2 + 1] = *reinterpret_cast<uint32_t*>(&c2);
              }
            const int d0 = c * 32;
            const int nb = d0 >> 6, cc = (d0 & 63) >> 3;
            uint8_t* base = dst + nb * (BN * 128);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              *reinterpret_cast<uint4*>(base + swz128_offset(r, cc + q)) =
                  make_uint4(h[4 * q], h[4 * q + 1], h[4 * q + 2], h[4 * q + 3]);
          }
          continue;
        }
#pragma unroll
        for (int c = 0; c < D / 16; ++c) {
          const uint32_t soff = RB == 128 ? swz128_offset(r, c) : swz64_offset(r, c);
          const uint4 raw = *reinterpret_cast<const uint4*>(src + soff);
          const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
          uint32_t h[8];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            if (KIND == KIND_E4M3) {
              h[2 * i] = e4m3x2_to_h2((uint16_t)(w[i] & 0xFFFF));
              h[2 * i + 1] = e4m3x2_to_h2((uint16_t)(w[i] >> 16));
            } else {
              const uint32_t ub = w[i] ^ 0x80808080u;
              h[2 * i] = s8x2_to_h2(ub, 0x4140);      // bytes 0, 1 -> (0x64, b0), (0x64, b1)
              h[2 * i + 1] = s8x2_to_h2(ub, 0x4342);  // bytes 2, 3
            }
          }
          const int d0 = c * 16;
          const int nb = d0 >> 6, cc = (d0 & 63) >> 3;
          uint8_t* base = dst + nb * (BN * 128);
          *reinterpret_cast<uint4*>(base + swz128_offset(r, cc)) = make_uint4(h[0], h[1], h[2], h[3]);
          *reinterpret_cast<uint4*>(base + swz128_offset(r, cc + 1)) = make_uint4(h[4], h[5], h[6], h[7]);
        }
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bar[B_VHFULL + bb]);
        mbar_arrive(&bar[B_VEMPTY + s]);
      }
    }
  } else {
    // ------------------------------------------------------------- softmax
    const int i = tid - 128;          // row within the tile == TMEM lane
    const int wg = warp - 4;          // TMEM lane quarter
    const int row = q0 + i;
    const bool row_ok = row < p.Sq;
    const uint32_t lane_off = (uint32_t)(wg * 32) << 16;
    const int kbh = bhk, qbh = b * p.Hq + hq;

    // Row constant: s_q * softmax_scale * log2(e) (per-head K scale folded in too).
    // MXFP4: the block scales are applied inside the MMA, so only the softmax scale.
    const float sq = MX ? 1.0f : (row_ok ? scale_at(p.qs, p.q_blk, p.q_nblk, qbh, hq, row) : 0.0f);
    float crow = sq * p.scale_log2;
    const bool k_head = MX || p.k_blk == 0;
    const bool k_tile_const = k_head || (p.k_blk % BN == 0);
    if (k_head && !MX) crow *= __ldg(p.ks + hk);
    // V reference: the largest V scale this CTA reads (per-head: the head's
    // scale; MXFP4: 2^(e_ref - 127), the factor the converters divided out).
    float vref;
    if (MX) {
      int m = 0;
      for (int t = i; t < kv_end; t += BM) {
        const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(p.ve8 + ((long long)bhk * p.Sk + t) * 4));
        m = max(m, (int)max(max(w & 0xFF, (w >> 8) & 0xFF), max((w >> 16) & 0xFF, w >> 24)));
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
      if (lane == 0) red[wg] = __int_as_float(m);
      mbar_arrive(&bar[B_RED]);
      warp_wait(&bar[B_RED], 0, abort_flag, p.status, 14);
      const int e = max(max(__float_as_int(red[0]), __float_as_int(red[1])),
                        max(__float_as_int(red[2]), __float_as_int(red[3])));
      vref = ldexpf(1.0f, e - 127);
    } else if (p.v_blk == 0) {
      vref = __ldg(p.vs + hk);
    } else {
      float m = 0.0f;
      const int nb_end = (kv_end + p.v_blk - 1) / p.v_blk;
      for (int t = i; t < nb_end; t += BM) m = fmaxf(m, __ldg(p.vs + (long long)kbh * p.v_nblk + t));
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
      if (lane == 0) red[wg] = m;
      mbar_arrive(&bar[B_RED]);
      warp_wait(&bar[B_RED], 0, abort_flag, p.status, 14);
      vref = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    }
    const float vinv = vref > 0.0f ? 1.0f / vref : 0.0f;

    float m_run = -INFINITY, l_run = 0.0f;
    bool ok = true;
    for (int j = 0; j < n_tiles && ok; ++j) {
      const int bb = j & 1;
      const int k0 = j * BN;
      // Scales of this tile (loaded before waiting so the latency overlaps).
      float ksc_tile = 1.0f, vf_tile = 1.0f;
      float my_k = 0.0f, my_v = 0.0f;
      const int tok = k0 + i;
      if (!k_head && !MX) {
        if (k_tile_const) ksc_tile = __ldg(p.ks + (long long)kbh * p.k_nblk + k0 / p.k_blk);
        else my_k = tok < p.Sk ? __ldg(p.ks + (long long)kbh * p.k_nblk + tok / p.k_blk) : 0.0f;
      }
      const bool v_tile_const = MX || p.v_blk == 0 || (p.v_blk % BN == 0);
      if (!MX && p.v_blk != 0) {
        if (v_tile_const) vf_tile = __ldg(p.vs + (long long)kbh * p.v_nblk + k0 / p.v_blk) * vinv;
        else my_v = tok < p.Sk ? __ldg(p.vs + (long long)kbh * p.v_nblk + tok / p.v_blk) * vinv : 0.0f;
      }
      if (!k_tile_const) sKsc[bb * BN + i] = my_k;
      if (!v_tile_const) sVf[bb * BN + i] = my_v;
      if (!k_tile_const || !v_tile_const) {
        mbar_arrive(&bar[B_SC + bb]);
        if (!warp_wait(&bar[B_SC + bb], (j >> 1) & 1, abort_flag, p.status, 15)) { ok = false; break; }
      }

      if (!warp_wait(&bar[B_SFULL + bb], (j >> 1) & 1, abort_flag, p.status, 10)) { ok = false; break; }
      tc_fence_after();
      float sv[BN];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tS[bb] + lane_off + c * 32, r);
        tmem_ld_wait();
#pragma unroll
        for (int k = 0; k < 32; ++k)
          sv[c * 32 + k] = KIND == KIND_S8 ? (float)(int)r[k] : __uint_as_float(r[k]);  // s32 only for INT8
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[B_SEMPTY + bb]);

      // Scores in the log2 domain, masked.
      const float cr = crow * ksc_tile;
      const bool need_mask = (k0 + BN > p.Sk) || (p.causal && (k0 + BN - 1 > q0 + diag));
      const int lim = p.causal ? min(p.Sk - 1, row + diag) : p.Sk - 1;  // last visible key
      float mt = -INFINITY;
      if (k_tile_const) {
#pragma unroll
        for (int k = 0; k < BN; ++k) sv[k] *= cr;
      } else {
#pragma unroll
        for (int k = 0; k < BN; ++k) sv[k] *= cr * sKsc[bb * BN + k];
      }
      if (need_mask) {
#pragma unroll
        for (int k = 0; k < BN; ++k)
          if (k0 + k > lim) sv[k] = -INFINITY;
      }
#pragma unroll
      for (int k = 0; k < BN; ++k) mt = fmaxf(mt, sv[k]);

      // Online max with a stale threshold: rescale only if the max grows by > 8.
      const float m_new = fmaxf(m_run, mt);
      const bool grow = m_new > m_run + 8.0f;
      const float m_use = grow ? m_new : m_run;
      const float alpha = grow ? ex2(m_run - m_use) : 1.0f;  // 0 when m_run = -inf
      if (j > 0 && __any_sync(0xffffffffu, grow)) {
        // O may be rescaled only after P V of the previous tile has landed.
        if (!warp_wait(&bar[B_PVDONE + ((j - 1) & 1)], ((j - 1) >> 1) & 1, abort_flag, p.status, 11)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 16; ++c) {
          uint32_t r[16];
          tmem_ld16(tO + lane_off + c * 16, r);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 16; ++k) r[k] = __float_as_uint(__uint_as_float(r[k]) * alpha);
          tmem_st16(tO + lane_off + c * 16, r);
        }
        tmem_st_wait();
      }
      l_run *= alpha;
      m_run = m_use;
      const float base = m_use == -INFINITY ? 0.0f : m_use;

      // P' buffer bb is free once P V of tile j-2 has completed.
      if (j >= 2 && !warp_wait(&bar[B_PVDONE + bb], ((j >> 1) - 1) & 1, abort_flag, p.status, 12)) {
        ok = false;
        break;
      }
      uint8_t* sP = smem + L::P + bb * BM * BN * 2;
      float lsum = 0.0f;
#pragma unroll
      for (int c = 0; c < BN / 8; ++c) {
        uint32_t h[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int col = c * 8 + 2 * k;
          const float p0 = ex2(sv[col] - base), p1 = ex2(sv[col + 1] - base);
          lsum += p0 + p1;
          float f0, f1;
          if (v_tile_const) {
            f0 = p0 * vf_tile;
            f1 = p1 * vf_tile;
          } else {
            f0 = p0 * sVf[bb * BN + col];
            f1 = p1 * sVf[bb * BN + col + 1];
          }
          const __half2 hv = __floats2half2_rn(f0, f1);
          h[k] = *reinterpret_cast<const uint32_t*>(&hv);
        }
        *reinterpret_cast<uint4*>(sP + (c >> 3) * (BM * 128) + swz128_offset(i, c & 7)) =
            make_uint4(h[0], h[1], h[2], h[3]);
      }
      l_run += lsum;
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[B_PFULL + bb]);
    }

    // ------------------------------------------------------------ epilogue
    if (ok && n_tiles > 0) {
      ok = warp_wait(&bar[B_PVDONE + ((n_tiles - 1) & 1)], ((n_tiles - 1) >> 1) & 1, abort_flag, p.status, 13);
      tc_fence_after();
    }
    const float ofac = (l_run > 0.0f) ? vref / l_run : 0.0f;
    __nv_bfloat16* orow = nullptr;
    if (row_ok) {
      const long long ridx = p.layout == FA_LAYOUT_BNSD ? ((long long)qbh * p.Sq + row)
                                                        : (((long long)b * p.Sq + row) * p.Hq + hq);
      orow = p.out + ridx * D;
    }
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t r[32];
      if (ok && n_tiles > 0) {
        tmem_ld32(tO + lane_off + c * 32, r);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int k = 0; k < 32; ++k) r[k] = 0u;
      }
      if (row_ok) {
#pragma unroll
        for (int k = 0; k < 32; k += 8) {
          uint32_t o[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 v2 = __floats2bfloat162_rn(__uint_as_float(r[k + 2 * e]) * ofac,
                                                            __uint_as_float(r[k + 2 * e + 1]) * ofac);
            o[e] = *reinterpret_cast<const uint32_t*>(&v2);
          }
          *reinterpret_cast<uint4*>(orow + c * 32 + k) = make_uint4(o[0], o[1], o[2], o[3]);
        }
      }
    }
    if (row_ok && p.lse) {
      const float lse = l_run > 0.0f ? (m_run + __log2f(l_run)) * 0.69314718055994530942f : -INFINITY;
      p.lse[(long long)qbh * p.Sq + row] = lse;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

__global__ void fill_empty_kernel(__nv_bfloat16* out, float* lse, long long rows, int D) {
  const long long n = rows * D;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
    out[i] = __float2bfloat16(0.0f);
  if (lse)
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < rows;
         i += (long long)gridDim.x * blockDim.x)
      lse[i] = -INFINITY;
}

void scale_desc(const fa_qtensor* t, int& blk, int& nblk) {
  switch (t->mode) {
    case FA_MODE_INT8_PER_HEAD: blk = 0; nblk = 1; break;
    case FA_MODE_FP8_PER_TOKEN: blk = 1; nblk = t->S; break;
    case FA_MODE_FP8_BLOCK: blk = t->block_tokens; nblk = (t->S + t->block_tokens - 1) / t->block_tokens; break;
    default: blk = 0; nblk = 1; break;
  }
}

template <int KIND, int D>
cudaError_t launch_kind(const AttnArgs& a, const AttnParams& prm, cudaStream_t s) {
  using L = Smem<KIND, D>;
  CUtensorMap mq, mk, mv;
  cudaError_t e;
  const int RB = (int)L::RB;
  if ((e = make_code_map(&mq, a.q->codes, a.q->B, a.q->H, a.q->S, RB, a.q->layout, BM)) != cudaSuccess) return e;
  if ((e = make_code_map(&mk, a.k->codes, a.k->B, a.k->H, a.k->S, RB, a.k->layout, BN)) != cudaSuccess) return e;
  if ((e = make_code_map(&mv, a.v->codes, a.v->B, a.v->H, a.v->S, RB, a.v->layout, BN)) != cudaSuccess) return e;
  auto kern = attn_fwd_kernel<KIND, D>;
  static bool attr_set = false;  // one attribute call per instantiation (idempotent, benign race)
  if (!attr_set) {
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC)) != cudaSuccess)
      return e;
    attr_set = true;
  }
  const long long grid = (long long)prm.n_qtiles * prm.B * prm.Hq;
  if (grid > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  kern<<<(unsigned)grid, NTHREADS, L::ALLOC, s>>>(mq, mk, mv, prm);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention_prefill(const AttnArgs& a, cudaStream_t s) {
  const fa_qtensor* q = a.q;
  const fa_qtensor* k = a.k;
  AttnParams prm = {};
  prm.B = q->B; prm.Hq = q->H; prm.Hkv = k->H; prm.Sq = q->S; prm.Sk = k->S; prm.group = q->H / k->H;
  prm.causal = a.causal; prm.layout = q->layout;
  const float scale = a.softmax_scale > 0.0f ? a.softmax_scale : 1.0f / sqrtf((float)q->D);
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.qs = static_cast<const float*>(q->scales);
  prm.ks = static_cast<const float*>(k->scales);
  prm.vs = static_cast<const float*>(a.v->scales);
  scale_desc(q, prm.q_blk, prm.q_nblk);
  scale_desc(k, prm.k_blk, prm.k_nblk);
  scale_desc(a.v, prm.v_blk, prm.v_nblk);
  prm.out = static_cast<__nv_bfloat16*>(a.out);
  prm.lse = a.lse;
  prm.status = a.status;
  prm.n_qtiles = (q->S + BM - 1) / BM;
  switch (q->mode) {
    case FA_MODE_FP8_PER_TOKEN:
    case FA_MODE_FP8_BLOCK:
      return q->D == 128 ? launch_kind<KIND_E4M3, 128>(a, prm, s) : launch_kind<KIND_E4M3, 64>(a, prm, s);
    case FA_MODE_INT8_PER_HEAD:
      return q->D == 128 ? launch_kind<KIND_S8, 128>(a, prm, s) : launch_kind<KIND_S8, 64>(a, prm, s);
    case FA_MODE_MXFP4_PER_BLOCK:
      if (q->D != 128) return cudaErrorNotSupported;
      prm.qe8 = static_cast<const uint8_t*>(q->scales);
      prm.ke8 = static_cast<const uint8_t*>(k->scales);
      prm.ve8 = static_cast<const uint8_t*>(a.v->scales);
      return launch_kind<KIND_MXF4, 128>(a, prm, s);
    default:
      return cudaErrorNotSupported;
  }
}

cudaError_t launch_fill_empty_rows(void* out, float* lse, long long rows, int D, cudaStream_t s) {
  const long long n = rows * D;
  int grid = (int)((n + 255) / 256);
  if (grid > 4096) grid = 4096;
  if (grid < 1) grid = 1;
  fill_empty_kernel<<<grid, 256, 0, s>>>(static_cast<__nv_bfloat16*>(out), lse, rows, D);
  return cudaGetLastError();
}

}  // namespace faq
