// attn2.cu -- prefill attention on FP8 (E4M3) and INT8 operands, two query
// tiles per CTA (FlashAttention's online softmax on the low-bit operands:
// MindIE SD "量化", FA量化 / FP8 Attention; wiki "FA 量化" 参考资料).
//
// A CTA owns two 128-row query "slots" that read the same kv head (two query
// heads of one GQA group at the same rows, or two consecutive row tiles of one
// head) and streams their visible 128-key K/V tiles once for both:
//   warpgroup 0 (88 registers per thread after setmaxnreg):
//     warp 0   producer: Q tiles once; per K/V tile the K codes (3-stage ring)
//              and V codes (2-stage ring) by TMA, and the tile's K scales and
//              V factors s_v / v_ref into a 2-stage shared ring.
//     warp 1   MMA issuer (one thread), over the two slots:
//              S_s = Q_s K^T (kind::f8f6f4 / kind::i8) into slot s's TMEM S,
//              and O_s += P'_s V' (kind::f16 with the A operand P'_s in TMEM,
//              where the softmax stored it over S_s).  PV_s(j) and then
//              QK_s(j+1) are issued once slot s's softmax of tile j is done;
//              the tensor pipe runs them in order, so P'_s is read before S_s
//              is overwritten, and the other slot's softmax runs meanwhile.
//     warps 2-3  V codes -> V' = fp16(code) (exact), MN-major, 128B-swizzled,
//              double-buffered.
//   warpgroups 1 and 2 (208 registers per thread): softmax of slot 0 and slot 1, one
//     thread per query row: S from TMEM, K scale, mask, online max in the
//     exp2 domain (O rescaled in TMEM only when the max grows by more than
//     2^8), p = exp2(t * c - m), P' = fp16(p * s_v / v_ref) stored into the
//     first 64 TMEM columns of S_s (tcgen05.st).
// TMEM: S_0/P'_0, S_1/P'_1, O_0, O_1 (4 x 128 columns).  Keeping P' in TMEM
// keeps it off the shared-memory port, which the shared-memory operands of
// Q K^T and the V' operand of P.V already load heavily.  Every wait is bounded.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>

#include "attn_common.cuh"
#include "internal.cuh"
#include "sm100.cuh"

namespace faq {
namespace {
using namespace attn;

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int NT = 384;  // 12 warps
constexpr int NKS = 3;   // K code stages
constexpr int NVS = 2;   // V code stages

enum { K_E4M3 = 0, K_S8 = 1 };
enum { SC_HEAD = 0, SC_COL = 1, SC_TILE = 2 };  // one scale per head / per key / per 128-key tile

struct P2 {
  int B, Hq, Hkv, Sq, Sk, group, causal, layout;
  float scale_log2;
  const float* qs;
  const float* ks;
  const float* vs;
  int q_blk, k_blk, v_blk, q_nblk, k_nblk, v_nblk;
  __nv_bfloat16* out;
  float* lse;
  int* status;
  int n_qtiles;
  int pair_heads;  // 1: the slots are query heads 2p, 2p+1 at one row tile; 0: row tiles 2t, 2t+1 of one head
};

template <int D>
struct L2 {
  static constexpr uint32_t Q = 0;                   // 2 x [128][D]
  static constexpr uint32_t K = Q + 2 * BM * D;        // NKS stages
  static constexpr uint32_t V = K + NKS * BN * D;      // NVS stages
  static constexpr uint32_t VH = V + NVS * BN * D;     // 2 x fp16 V'
  static constexpr uint32_t SC = VH + 2 * BN * D * 2;  // 2 stages x ([128] k scale, [128] v factor)
  static constexpr uint32_t MISC = SC + 2 * 2 * BN * 4;
  static constexpr uint32_t BAR = MISC + 64;
  static constexpr uint32_t TOTAL = BAR + 512;
  static constexpr uint32_t ALLOC = TOTAL + 1024;
};

enum {
  X_Q = 0,
  X_KF = 1,    // [NKS]
  X_KE = 4,    // [NKS]
  X_VF = 7,    // [NVS]
  X_VE = 9,    // [NVS]
  X_VHF = 11,  // [2]
  X_VHE = 13,  // [2]
  X_SF = 15,   // [2 slots]
  X_PF = 17,   // [2 slots]
  X_PVD = 19,  // [2 slots]
  X_SCF = 21,  // [2]
  X_SCE = 23,  // [2 slots][2 stages]
  X_FIN = 27,
  X_COUNT = 28
};

__device__ __forceinline__ void setmaxnreg_inc208() { asm volatile("setmaxnreg.inc.sync.aligned.u32 208;"); }
__device__ __forceinline__ void setmaxnreg_dec88() { asm volatile("setmaxnreg.dec.sync.aligned.u32 88;"); }

template <int KIND, int D, int SC>
__global__ void __launch_bounds__(NT, 1)
    attn2_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                 const __grid_constant__ CUtensorMap tmv, const P2 p) {
  using L = L2<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L::BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + X_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar + X_COUNT + 1);
  float* misc = reinterpret_cast<float*>(smem + L::MISC);  // [0] = v_ref

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---- work item: (b, kv head) and two query slots
  int hqs[2], q0s[2], ns[2], kv_ends[2];
  int b, hk;
  {
    const int widx = blockIdx.x;
    if (p.pair_heads) {
      const int npair = p.Hq / 2;
      const int per_t = p.B * npair;
      const int qt = p.causal ? (p.n_qtiles - 1 - widx / per_t) : (widx / per_t);
      const int r = widx % per_t;
      b = r / npair;
      const int pr = r % npair;
      hqs[0] = 2 * pr;
      hqs[1] = 2 * pr + 1;
      q0s[0] = q0s[1] = qt * BM;
    } else {
      const int npairs_t = (p.n_qtiles + 1) / 2;
      const int per_t = p.B * p.Hq;
      const int tp = p.causal ? (npairs_t - 1 - widx / per_t) : (widx / per_t);
      const int r = widx % per_t;
      b = r / p.Hq;
      hqs[0] = hqs[1] = r % p.Hq;
      q0s[0] = 2 * tp * BM;
      q0s[1] = (2 * tp + 1) * BM;
    }
    hk = hqs[0] / p.group;
    const int diag = p.Sk - p.Sq;
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      int e = 0;
      if (q0s[s] < p.Sq) e = p.causal ? min(p.Sk, max(0, min(q0s[s] + BM, p.Sq) - 1 + diag + 1)) : p.Sk;
      kv_ends[s] = e;
      ns[s] = (e + BN - 1) / BN;
    }
  }
  const int n_tiles = max(ns[0], ns[1]);
  const int kv_end = max(kv_ends[0], kv_ends[1]);
  const int bhk = b * p.Hkv + hk;

  if (tid == 0) {
    mbar_init(&bar[X_Q], 1);
    for (int i = 0; i < NKS; ++i) {
      mbar_init(&bar[X_KF + i], 1);
      mbar_init(&bar[X_KE + i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar[X_VF + i], 1);
      mbar_init(&bar[X_VE + i], 2);
      mbar_init(&bar[X_VHF + i], 2);
      mbar_init(&bar[X_VHE + i], 1);
      mbar_init(&bar[X_SF + i], 1);
      mbar_init(&bar[X_PF + i], 4);
      mbar_init(&bar[X_PVD + i], 1);
      mbar_init(&bar[X_SCF + i], 1);
      mbar_init(&bar[X_SCE + i], 4);
      mbar_init(&bar[X_SCE + 2 + i], 4);
    }
    mbar_init(&bar[X_FIN], 1);
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

  if (warp < 4) {
    setmaxnreg_dec88();
    if (warp == 0) {
      // ------------------------------------------------------------ producer
      if (n_tiles > 0) {
        const bool bnsd = p.layout == FA_LAYOUT_BNSD;
        float vref = 1.0f;
        if (SC != SC_HEAD) {
          float m = 0.0f;
          const int nb_end = (kv_end + p.v_blk - 1) / p.v_blk;
          for (int t = lane; t < nb_end; t += 32) m = fmaxf(m, __ldg(p.vs + (long long)bhk * p.v_nblk + t));
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
          vref = m > 0.0f ? m : 1.0f;
          if (lane == 0) misc[0] = vref;
        }
        const float vinv = 1.0f / vref;
        if (lane == 0) {
          tma_prefetch_desc(&tmq);
          tma_prefetch_desc(&tmk);
          tma_prefetch_desc(&tmv);
          const int nq = (ns[0] > 0 ? 1 : 0) + (ns[1] > 0 ? 1 : 0);
          mbar_arrive_expect_tx(&bar[X_Q], nq * BM * D);
#pragma unroll
          for (int s = 0; s < 2; ++s)
            if (ns[s] > 0)
              tma_load_4d(smem + L::Q + s * BM * D, &tmq, &bar[X_Q], 0, bnsd ? q0s[s] : hqs[s], bnsd ? hqs[s] : q0s[s], b);
        }
        int j = 0;
        for (; j < n_tiles; ++j) {
          const int k0 = j * BN, st = j & 1;
          bool ok = true;
          if (SC != SC_HEAD) {
            // scale ring stage st is free once both slots finished tile j - 2
            for (int s = 0; s < 2 && ok; ++s)
              if (j >= 2 && j - 2 < ns[s]) ok = mbar_wait(&bar[X_SCE + 2 * s + st], ((j >> 1) - 1) & 1, abort_flag, p.status, 60);
            if (!__all_sync(0xffffffffu, ok)) break;
            float* ksc = reinterpret_cast<float*>(smem + L::SC + st * 2 * BN * 4);
            float* vcf = ksc + BN;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int c = lane * 4 + q, tok = k0 + c;
              float kv = 0.0f, vv = 0.0f;
              if (tok < p.Sk) {
                kv = __ldg(p.ks + (long long)bhk * p.k_nblk + tok / p.k_blk);
                vv = __ldg(p.vs + (long long)bhk * p.v_nblk + tok / p.v_blk) * vinv;
              }
              ksc[c] = kv;
              vcf[c] = vv;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar[X_SCF + st]);
          }
          if (lane == 0) {
            const int ks = j % NKS, vs = j % NVS;
            if (j >= NKS) ok = mbar_wait(&bar[X_KE + ks], ((j / NKS) - 1) & 1, abort_flag, p.status, 61);
            if (ok) {
              mbar_arrive_expect_tx(&bar[X_KF + ks], BN * D);
              tma_load_4d(smem + L::K + ks * BN * D, &tmk, &bar[X_KF + ks], 0, bnsd ? k0 : hk, bnsd ? hk : k0, b);
              if (j >= NVS) ok = mbar_wait(&bar[X_VE + vs], ((j / NVS) - 1) & 1, abort_flag, p.status, 62);
              if (ok) {
                mbar_arrive_expect_tx(&bar[X_VF + vs], BN * D);
                tma_load_4d(smem + L::V + vs * BN * D, &tmv, &bar[X_VF + vs], 0, bnsd ? k0 : hk, bnsd ? hk : k0, b);
              }
            }
          }
          if (!__all_sync(0xffffffffu, ok)) { ++j; break; }
        }
        if (lane == 0 && *abort_flag) {
          // let issued loads land before the CTA can exit
          for (int t = max(0, j - NKS); t < j; ++t) mbar_wait(&bar[X_KF + t % NKS], (t / NKS) & 1, abort_flag, nullptr, 0);
          for (int t = max(0, j - NVS); t < j; ++t) mbar_wait(&bar[X_VF + t % NVS], (t / NVS) & 1, abort_flag, nullptr, 0);
        }
      }
      __syncwarp();
    } else if (warp == 1) {
      // ---------------------------------------------------------- MMA issuer
      if (lane == 0 && n_tiles > 0) {
        constexpr uint32_t SW = D == 128 ? kSwz128 : kSwz64;
        constexpr uint32_t SBO8 = D == 128 ? 1024 : 512;
        constexpr uint32_t idesc_qk = KIND == K_E4M3 ? make_idesc(kAccF32, kFmtE4M3, kFmtE4M3, 0, 0, BN, BM)
                                                     : make_idesc(kAccS32, kFmtS8, kFmtS8, 0, 0, BN, BM);
        constexpr uint32_t idesc_pv = make_idesc(kAccF32, kFmtF16, kFmtF16, 0, 1, D, BM);
        auto qk = [&](int s, int j) {
          const uint32_t sQ = smem_u32(smem + L::Q + s * BM * D);
          const uint32_t sK = smem_u32(smem + L::K + (j % NKS) * BN * D);
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk) {
            const uint64_t da = make_sdesc(sQ + kk * 32, 16, SBO8, SW);
            const uint64_t db = make_sdesc(sK + kk * 32, 16, SBO8, SW);
            if (KIND == K_E4M3)
              mma_f8f6f4(tbase + s * 128, da, db, idesc_qk, kk > 0);
            else
              mma_i8(tbase + s * 128, da, db, idesc_qk, kk > 0);
          }
          mma_commit(&bar[X_SF + s]);
        };
        auto pv = [&](int s, int j) {
          // A = P'_s in TMEM: 16 fp16 of K per MMA = 8 columns
          const uint32_t sVh = smem_u32(smem + L::VH + (j & 1) * BN * D * 2);
#pragma unroll
          for (int ks = 0; ks < BN / 16; ++ks) {
            const uint64_t db = make_sdesc(sVh + ks * 16 * 128, BN * 128, 1024, kSwz128);
            mma_f16_ts(tbase + 256 + s * 128, tbase + s * 128 + ks * 8, db, idesc_pv, (j > 0 || ks > 0) ? 1u : 0u);
          }
          mma_commit(&bar[X_PVD + s]);
        };
        bool ok = mbar_wait(&bar[X_Q], 0, abort_flag, p.status, 63);
        if (ok) ok = mbar_wait(&bar[X_KF], 0, abort_flag, p.status, 64);
        if (ok) {
          tc_fence_after();
          if (ns[0] > 0) qk(0, 0);
          if (ns[1] > 0) qk(1, 0);
          mma_commit(&bar[X_KE]);
        }
        for (int j = 0; ok && j < n_tiles; ++j) {
          // slot s: PV_s(j) (reads P'_s over S_s), then QK_s(j+1) (rewrites S_s)
          bool vh = false, k1 = false;
          for (int s = 0; s < 2 && ok; ++s) {
            if (j >= ns[s]) continue;
            ok = mbar_wait(&bar[X_PF + s], j & 1, abort_flag, p.status, 65);
            if (ok && !vh) {
              ok = mbar_wait(&bar[X_VHF + (j & 1)], (j >> 1) & 1, abort_flag, p.status, 66);
              vh = true;
            }
            if (!ok) break;
            tc_fence_after();
            pv(s, j);
            if (j + 1 < ns[s]) {
              if (!k1) {
                ok = mbar_wait(&bar[X_KF + (j + 1) % NKS], ((j + 1) / NKS) & 1, abort_flag, p.status, 67);
                k1 = true;
                if (!ok) break;
                tc_fence_after();
              }
              qk(s, j + 1);
            }
          }
          if (!ok) break;
          mma_commit(&bar[X_VHE + (j & 1)]);
          if (k1) mma_commit(&bar[X_KE + (j + 1) % NKS]);
        }
        mma_commit(&bar[X_FIN]);
        mbar_wait(&bar[X_FIN], 0, abort_flag, nullptr, 0);
      }
      __syncwarp();
    } else {
      // --------------------------------------------------------- V converter
      const int ct = tid - 64;
      for (int j = 0; j < n_tiles; ++j) {
        const int vb = j & 1;
        if (!warp_wait(&bar[X_VF + j % NVS], (j / NVS) & 1, abort_flag, p.status, 68)) break;
        if (j >= 2 && !warp_wait(&bar[X_VHE + vb], ((j >> 1) - 1) & 1, abort_flag, p.status, 69)) break;
        const uint8_t* src = smem + L::V + (j % NVS) * BN * D;
        uint8_t* dst = smem + L::VH + vb * BN * D * 2;
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          const int r = ct + rr * 64;
#pragma unroll
          for (int c = 0; c < D / 16; ++c) {
            const uint32_t soff = D == 128 ? swz128_offset(r, c) : swz64_offset(r, c);
            const uint4 raw = *reinterpret_cast<const uint4*>(src + soff);
            const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
            uint32_t h[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              if (KIND == K_E4M3) {
                h[2 * i] = e4m3x2_to_h2((uint16_t)(w[i] & 0xFFFF));
                h[2 * i + 1] = e4m3x2_to_h2((uint16_t)(w[i] >> 16));
              } else {
                const uint32_t ub = w[i] ^ 0x80808080u;
                h[2 * i] = s8x2_to_h2(ub, 0x4140);
                h[2 * i + 1] = s8x2_to_h2(ub, 0x4342);
              }
            }
            const int d0 = c * 16;
            uint8_t* base = dst + (d0 >> 6) * (BN * 128);
            const int cc = (d0 & 63) >> 3;
            *reinterpret_cast<uint4*>(base + swz128_offset(r, cc)) = make_uint4(h[0], h[1], h[2], h[3]);
            *reinterpret_cast<uint4*>(base + swz128_offset(r, cc + 1)) = make_uint4(h[4], h[5], h[6], h[7]);
          }
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bar[X_VHF + vb]);
          mbar_arrive(&bar[X_VE + j % NVS]);
        }
      }
    }
  } else {
    setmaxnreg_inc208();
    // ------------------------------------------------------------- softmax
    const int s = (warp - 4) >> 2;  // slot
    const int i = tid - 128 - s * 128;
    const uint32_t loff = (uint32_t)(((warp - 4) & 3) * 32) << 16;
    const uint32_t tS = tbase + s * 128, tO = tbase + 256 + s * 128;
    const int hq = hqs[s], q0 = q0s[s], n = ns[s];
    const int row = q0 + i;
    const bool row_ok = row < p.Sq;
    const int qbh = b * p.Hq + hq;
    const int diag = p.Sk - p.Sq;
    const float sq = row_ok ? scale_at(p.qs, p.q_blk, p.q_nblk, qbh, hq, row) : 0.0f;
    float crow = sq * p.scale_log2;
    if (SC == SC_HEAD) crow *= __ldg(p.ks + hk);
    // S8 accumulators arrive biased: t = float(0x4B400000 + acc) = 1.5 * 2^23 + acc (exact, |acc| < 2^22)
    constexpr float kBias = KIND == K_S8 ? 12582912.0f : 0.0f;
    float vref = SC == SC_HEAD ? __ldg(p.vs + hk) : 1.0f;
    float m_run = -INFINITY, l_run = 0.0f;
    bool ok = true;
    for (int j = 0; j < n && ok; ++j) {
      const int k0 = j * BN, st = j & 1;
      const float* ksc = reinterpret_cast<const float*>(smem + L::SC + st * 2 * BN * 4);
      const float* vcf = ksc + BN;
      if (SC != SC_HEAD && !warp_wait(&bar[X_SCF + st], (j >> 1) & 1, abort_flag, p.status, 70)) { ok = false; break; }
      if (SC != SC_HEAD && j == 0) vref = misc[0];
      if (!warp_wait(&bar[X_SF + s], j & 1, abort_flag, p.status, 71)) { ok = false; break; }
      tc_fence_after();
      // All four 32-column loads in flight before one wait; values used in place.
      uint32_t tr[BN];
      tmem_ld32(tS + loff + 0, *reinterpret_cast<uint32_t(*)[32]>(&tr[0]));
      tmem_ld32(tS + loff + 32, *reinterpret_cast<uint32_t(*)[32]>(&tr[32]));
      tmem_ld32(tS + loff + 64, *reinterpret_cast<uint32_t(*)[32]>(&tr[64]));
      tmem_ld32(tS + loff + 96, *reinterpret_cast<uint32_t(*)[32]>(&tr[96]));
      tmem_ld_wait();
      float t[BN];
#pragma unroll
      for (int k = 0; k < BN; ++k) t[k] = KIND == K_S8 ? __uint_as_float(0x4B400000u + tr[k]) : __uint_as_float(tr[k]);
      // per-key K scale; tile-constant K scale folds into the row constant
      float cr = crow;
      if (SC == SC_COL) {
#pragma unroll
        for (int k = 0; k < BN; k += 4) {
          const float4 kk4 = *reinterpret_cast<const float4*>(ksc + k);
          t[k] *= kk4.x; t[k + 1] *= kk4.y; t[k + 2] *= kk4.z; t[k + 3] *= kk4.w;
        }
      } else if (SC == SC_TILE) {
        cr *= ksc[0];
      }
      // masks: keys past the sequence, and causal
      const bool need_mask = (k0 + BN > p.Sk) || (p.causal && (k0 + BN - 1 > q0 + diag));
      if (need_mask) {
        const int lim = p.causal ? min(p.Sk - 1, row + diag) : p.Sk - 1;
#pragma unroll
        for (int k = 0; k < BN; ++k)
          if (k0 + k > lim) t[k] = -INFINITY;
      }
      float mx[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) mx[e] = t[e];
#pragma unroll
      for (int k = 8; k < BN; ++k) mx[k & 7] = fmaxf(mx[k & 7], t[k]);
      const float mt = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
      const float mts = mt == -INFINITY ? -INFINITY : (mt - kBias) * cr;  // tile max of the log2-domain score
      const float m_new = fmaxf(m_run, mts);
      const bool grow = m_new > m_run + 8.0f;
      const float m_use = grow ? m_new : m_run;
      const float alpha = grow ? ex2(m_run - m_use) : 1.0f;
      const bool any_grow = __any_sync(0xffffffffu, grow) && j > 0;
      if (j > 0) {
        // P'_s and O_s are free once P V of tile j-1 has completed.
        if (!warp_wait(&bar[X_PVD + s], (j - 1) & 1, abort_flag, p.status, 72)) { ok = false; break; }
        if (any_grow) {
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < D / 16; ++c) {
            uint32_t r[16];
            tmem_ld16(tO + loff + c * 16, r);
            tmem_ld_wait();
#pragma unroll
            for (int k = 0; k < 16; ++k) r[k] = __float_as_uint(__uint_as_float(r[k]) * alpha);
            tmem_st16(tO + loff + c * 16, r);
          }
          tmem_st_wait();
        }
      }
      l_run *= alpha;
      m_run = m_use;
      // exp2 argument: t * cr - (bias * cr + m)   (the bias term is 0 for E4M3)
      const float nb = m_use == -INFINITY ? 0.0f : -(kBias * cr + m_use);
      float vt = 1.0f, nbv = nb;
      if (SC == SC_TILE) {
        vt = vcf[0];
        nbv = vt > 0.0f ? nb + __log2f(vt) : -INFINITY;  // fold s_v / v_ref into the exponent
      }
      // exp2 of all 128 scores first (independent, keeps the XU pipe fed), then
      // the row sum, then V fold + fp16 packing + stores.
#pragma unroll
      for (int k = 0; k < BN; ++k) t[k] = ex2(fmaf(t[k], cr, SC == SC_COL ? nb : nbv));
      float ls[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) ls[e] = t[e];
#pragma unroll
      for (int k = 8; k < BN; ++k) ls[k & 7] += t[k];
      // P' (fp16 pairs) into the first 64 TMEM columns of S_s: two 32-column stores.
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t h[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int k = half * 64 + 2 * e;
          float a = t[k], c2 = t[k + 1];
          if (SC == SC_COL) {
            a *= vcf[k];
            c2 *= vcf[k + 1];
          }
          const __half2 hv = __floats2half2_rn(a, c2);
          h[e] = *reinterpret_cast<const uint32_t*>(&hv);
        }
        tmem_st32(tS + loff + half * 32, h);
      }
      tmem_st_wait();
      float lsum = ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
      if (SC == SC_TILE) lsum = vt > 0.0f ? lsum / vt : 0.0f;
      l_run += lsum;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bar[X_PF + s]);
        if (SC != SC_HEAD) mbar_arrive(&bar[X_SCE + 2 * s + st]);
      }
    }
    // ---------------------------------------------------------- epilogue
    if (ok && n > 0) {
      ok = warp_wait(&bar[X_PVD + s], (n - 1) & 1, abort_flag, p.status, 73);
      tc_fence_after();
    }
    if (q0 < p.Sq) {
      const float ofac = l_run > 0.0f ? vref / l_run : 0.0f;
      __nv_bfloat16* orow = nullptr;
      if (row_ok) {
        const long long ridx = p.layout == FA_LAYOUT_BNSD ? ((long long)qbh * p.Sq + row)
                                                          : (((long long)b * p.Sq + row) * p.Hq + hq);
        orow = p.out + ridx * D;
      }
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        if (ok && n > 0) {
          tmem_ld32(tO + loff + c * 32, r);
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
      if (row_ok && p.lse)
        p.lse[(long long)qbh * p.Sq + row] =
            l_run > 0.0f ? (m_run + __log2f(l_run)) * 0.69314718055994530942f : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

template <int KIND, int D, int SC>
cudaError_t launch2(const AttnArgs& a, const P2& prm, cudaStream_t s) {
  using L = L2<D>;
  CUtensorMap mq, mk, mv;
  cudaError_t e;
  if ((e = make_code_map(&mq, a.q->codes, a.q->B, a.q->H, a.q->S, D, a.q->layout, BM)) != cudaSuccess) return e;
  if ((e = make_code_map(&mk, a.k->codes, a.k->B, a.k->H, a.k->S, D, a.k->layout, BN)) != cudaSuccess) return e;
  if ((e = make_code_map(&mv, a.v->codes, a.v->B, a.v->H, a.v->S, D, a.v->layout, BN)) != cudaSuccess) return e;
  auto kern = attn2_kernel<KIND, D, SC>;
  static bool attr_set = false;
  if (!attr_set) {
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC)) != cudaSuccess)
      return e;
    attr_set = true;
  }
  long long grid;
  if (prm.pair_heads)
    grid = (long long)prm.n_qtiles * prm.B * (prm.Hq / 2);
  else
    grid = (long long)((prm.n_qtiles + 1) / 2) * prm.B * prm.Hq;
  if (grid > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  kern<<<(unsigned)grid, NT, L::ALLOC, s>>>(mq, mk, mv, prm);
  return cudaGetLastError();
}

template <int KIND, int D>
cudaError_t launch2_sc(const AttnArgs& a, const P2& prm, int sc, cudaStream_t s) {
  switch (sc) {
    case SC_HEAD: return launch2<KIND, D, SC_HEAD>(a, prm, s);
    case SC_COL: return launch2<KIND, D, SC_COL>(a, prm, s);
    default: return launch2<KIND, D, SC_TILE>(a, prm, s);
  }
}

void scale_desc2(const fa_qtensor* t, int& blk, int& nblk) {
  switch (t->mode) {
    case FA_MODE_INT8_PER_HEAD: blk = 0; nblk = 1; break;
    case FA_MODE_FP8_PER_TOKEN: blk = 1; nblk = t->S; break;
    case FA_MODE_FP8_BLOCK: blk = t->block_tokens; nblk = (t->S + t->block_tokens - 1) / t->block_tokens; break;
    default: blk = 0; nblk = 1; break;
  }
}

}  // namespace

// Prefill attention for E4M3 and INT8 operands (two query tiles per CTA).
cudaError_t launch_attention_prefill2(const AttnArgs& a, cudaStream_t s) {
  const fa_qtensor* q = a.q;
  const fa_qtensor* k = a.k;
  P2 prm = {};
  prm.B = q->B; prm.Hq = q->H; prm.Hkv = k->H; prm.Sq = q->S; prm.Sk = k->S; prm.group = q->H / k->H;
  prm.causal = a.causal; prm.layout = q->layout;
  const float scale = a.softmax_scale > 0.0f ? a.softmax_scale : 1.0f / sqrtf((float)q->D);
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.qs = static_cast<const float*>(q->scales);
  prm.ks = static_cast<const float*>(k->scales);
  prm.vs = static_cast<const float*>(a.v->scales);
  scale_desc2(q, prm.q_blk, prm.q_nblk);
  scale_desc2(k, prm.k_blk, prm.k_nblk);
  scale_desc2(a.v, prm.v_blk, prm.v_nblk);
  prm.out = static_cast<__nv_bfloat16*>(a.out);
  prm.lse = a.lse;
  prm.status = a.status;
  prm.n_qtiles = (q->S + BM - 1) / BM;
  prm.pair_heads = (prm.group % 2 == 0) ? 1 : 0;
  int sc = SC_HEAD;
  if (q->mode == FA_MODE_FP8_PER_TOKEN) sc = SC_COL;
  if (q->mode == FA_MODE_FP8_BLOCK) sc = (k->block_tokens % BN == 0) ? SC_TILE : SC_COL;
  switch (q->mode) {
    case FA_MODE_FP8_PER_TOKEN:
    case FA_MODE_FP8_BLOCK:
      return q->D == 128 ? launch2_sc<K_E4M3, 128>(a, prm, sc, s) : launch2_sc<K_E4M3, 64>(a, prm, sc, s);
    case FA_MODE_INT8_PER_HEAD:
      return q->D == 128 ? launch2_sc<K_S8, 128>(a, prm, SC_HEAD, s) : launch2_sc<K_S8, 64>(a, prm, SC_HEAD, s);
    default:
      return cudaErrorNotSupported;
  }
}

}  // namespace faq
