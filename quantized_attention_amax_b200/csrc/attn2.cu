// attn2.cu -- prefill attention on FP8 (E4M3), INT8 and MXFP4 operands
// (FlashAttention's online softmax on low-bit operands: MindIE SD "量化",
// FA量化 / FP8 Attention and MXFP4 Attention; wiki "FA 量化" 参考资料).
//
// Two kernels per call:
//   vprep: V codes -> V' = fp16(code * s_v / r_t) once per call, r_t = the
//     largest V scale of key tile t (INT8: V' = fp16(code), exact; MX:
//     V' = fp16(code * 2^(e - E_t)) with E_t the tile's largest block exponent),
//     into a caller workspace, with r_t beside it.  Every query tile reads the
//     same V tiles, so the conversion is done once instead of once per query
//     tile.  The same pass lays out each K tile's scales for the attention:
//     128 per-key floats (E4M3, INT8 per token) or the tile's UE8M0
//     scale-factor atom (MX).
//   attn_pair: one CTA owns two 128-row query tiles that read the same K / V'
//     tiles (the layout and schedule are described above the kernel).  Key
//     tiles hold 128 keys, or 112 for the MX kinds, whose block-scale factors
//     need TMEM columns beside the two S tiles and two O accumulators.
// Every wait is bounded.
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
constexpr int NKS = 3;      // K code stages
constexpr int NSC = 4;      // scale ring stages

// per half: max(|a|, |b|), its sign the XOR of the inputs' signs (only magnitudes are used)
__device__ __forceinline__ uint32_t bf16x2_absmax(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// A bounded wait on the per-tile chain, polling (test_wait) or suspending (try_wait).
template <bool SPIN>
__device__ __forceinline__ bool chain_wait(uint64_t* b, uint32_t parity, volatile int* abort_flag, int* status,
                                           int where) {
  return SPIN ? mbar_wait_spin(b, parity, abort_flag, status, where) : mbar_wait(b, parity, abort_flag, status, where);
}
// K_BF16: bf16 Q and K (dequantized operands of mixed branches, or unquantized ones)
enum { K_E4M3 = 0, K_S8 = 1, K_MXF4 = 2, K_MXF8 = 3, K_BF16 = 4 };
enum { SC_HEAD = 0, SC_COL = 1, SC_TILE = 2 };  // one scale per head / per key / per 128-key tile

struct P2 {
  int B, Hq, Hkv, Sq, Sk, group, causal, layout;
  float scale_log2;
  const float* qs;
  const float* ks;
  const float* vs;
  const float* ksp;   // [B, Hkv, ntiles] x 512 B: per-key K scales, zero past Sk (E4M3) / UE8M0 atom (MXFP4)
  const float4* fvr;  // [B, Hkv, ntiles] V' tile factor records {r_t, log2 r_t, 0, 0} (E4M3) / {E_t, E_t - 127, 0, 0} (MXFP4)
  const uint8_t* qe8; // MXFP4 UE8M0 scales [B, H, S, D / 32]
  const uint8_t* ke8;
  const uint8_t* ve8;
  int q_blk, k_blk, v_blk, q_nblk, k_nblk, v_nblk;
  int ntiles_k;
  __nv_bfloat16* out;
  float* lse;
  int* status;
  int n_qtiles;
  int pair_heads;  // two-tile kernel: 1 = the two tiles are query heads 2h, 2h+1 at one row block, 0 = row blocks 2t, 2t+1 of one head
};

template <int R>
__device__ __forceinline__ void setmaxnreg_inc() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(R)); }
template <int R>
__device__ __forceinline__ void setmaxnreg_dec() { asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(R)); }

// ---- two query tiles per CTA (E4M3 / INT8 / MX / bf16) ------------------
// One CTA owns two 128-row query tiles A and B that read the same K / V' tiles
// (query heads 2h, 2h+1 of one kv head, or row blocks 2t, 2t+1 of one head),
// with one S and one O accumulator each in TMEM (S_A, S_B, O_A, O_B = 512
// columns for D = 128; the MX kinds' 112-key S tiles leave room for the Q and
// K block-scale factors).  Each tile has its own softmax warpgroup, one thread
// per query row holding the row's scores, so the row maximum needs no
// exchange between threads.  The MMA thread alternates the tiles:
//   QK_A(0) QK_B(0) | PV_A(0) QK_A(1) PV_B(0) QK_B(1) | PV_A(1) QK_A(2) ...
// so while one warpgroup runs the softmax of tile j, the tensor pipe runs the
// other tile's P V and next Q K^T.
// Pairs of exponentials (out of every 8) that the pair kernel computes with the cubic on the
// FMA pipe instead of the MUFU.
#ifndef FAQ_PAIR_POLY
#define FAQ_PAIR_POLY 0
#endif
// The same for the MX kinds (their 112-key tiles leave the MUFU the larger share of the step):
// 0 / 1 / 2 / 3 of every 8 pairs measured at mxfp4 259 / 259 / 261 / 255 us, mxfp8 275 / 267 / 269 /
// 265 us.
#ifndef FAQ_PAIR_POLY_MX
#define FAQ_PAIR_POLY_MX 3
#endif
// Waits of the per-tile chain that poll (test_wait) instead of suspending: bit 0 the MMA
// thread's wait for P', bit 1 the softmax's wait for S, bit 2 the MMA thread's K / V' waits.
// Measured on the 8-bit prefill workloads: bit 0 alone saves 1-1.5 %; bit 1 costs about 2 %
// (eight polling warps take issue slots from the other tile's exponentials).
#ifndef FAQ_PAIR_SPIN
#define FAQ_PAIR_SPIN 1
#endif
constexpr int PNT = 384;  // warpgroup 0 (loads, MMA, scale ring) + two softmax warpgroups
constexpr int PR0 = 56;
constexpr int PRS = 224;
static_assert(128 * PR0 + 256 * PRS <= PNT * ((65536 / PNT) & ~7), "register split exceeds the launch");

template <int KIND, int D>
struct LP {
  // MX kinds: block-scaled Q K^T with the scale factors in TMEM.  Their 16 factor columns leave
  // no room beside two 128-key S tiles and two O accumulators, so their key tiles hold 112 keys.
  static constexpr bool MX = KIND == K_MXF4 || KIND == K_MXF8;
  static constexpr int TN = MX ? 112 : BN;               // keys per tile
  static constexpr int RB = KIND == K_BF16 ? 2 * D : KIND == K_MXF4 ? D / 2 : D;  // Q / K bytes per token row
  static constexpr int NA = RB > 128 ? RB / 128 : 1;     // 128-byte swizzle atoms per row (bf16 at D = 128: 2)
  static constexpr int AB = RB > 128 ? 128 : RB;         // bytes per atom row
  static constexpr int NK = KIND == K_BF16 ? 2 : NKS;    // K stages (bf16 tiles are twice as large)
  // V' stages: three for the 8-bit kinds, so a V' tile is requested two key-tile steps before its
  // P V (a 32 KB tile from L2 takes a good part of one step to land); two fit beside bf16 Q / K
  static constexpr int NV = KIND == K_BF16 ? 2 : 3;
  static constexpr uint32_t Q = 0;                       // 2 x NA x [128][AB]
  static constexpr uint32_t K = Q + 2 * BM * RB;         // NK stages
  static constexpr uint32_t VH = K + NK * TN * RB;       // NV stages of fp16 V'
  static constexpr uint32_t SC = VH + NV * TN * D * 2;   // NSC stages x ([128] K scales or atom, V' factor record)
  static constexpr uint32_t MISC = SC + NSC * 2 * BN * 4;
  static constexpr uint32_t SFA = MISC + 64;             // MX: the two Q tiles' scale-factor atoms
  static constexpr uint32_t BAR = SFA + (MX ? 2 * 512 : 0);
  static constexpr uint32_t TOTAL = BAR + 512;
  static constexpr uint32_t ALLOC = TOTAL + 1024;
  static_assert(ALLOC <= 227 * 1024, "shared memory per CTA");
  static_assert(VH % 1024 == 0, "V' stages need 1024-byte alignment for the 128-byte swizzle");
  static_assert((TN * RB) % 1024 == 0 && (TN * D * 2) % 1024 == 0, "stage sizes keep the swizzle alignment");
  // TMEM columns.  E4M3 / INT8 / bf16: S_A, S_B at 0, 128; O_A, O_B at 256, 256 + D.  MX (D = 128):
  // O_A, O_B at 0, 128; S_A at 256 and S_B at 384 (112 columns each); the Q tiles' factors at 368
  // and 376 and the K tiles' (two slots) at 496 and 504, every block 8-column aligned.
  static constexpr uint32_t TS0 = MX ? 256 : 0;
  static constexpr uint32_t TO0 = MX ? 0 : 256;
  static constexpr uint32_t TO1 = MX ? 128 : 256 + D;
  static constexpr uint32_t TSFQ = 368;
  static constexpr uint32_t TSFK = 496;
  static_assert(!MX || D == 128, "MX paths: head_dim 128");
};

enum {
  Y_Q = 0,
  Y_KF = 1,              // [NKS]
  Y_KE = Y_KF + NKS,     // [NKS]
  Y_VF = Y_KE + NKS,     // [3] (up to three V' stages)
  Y_VE = Y_VF + 3,       // [3]
  Y_SF = Y_VE + 3,       // [2] S_A / S_B full
  Y_PF = Y_SF + 2,       // [2] P'_A / P'_B stored
  Y_PVD = Y_PF + 2,      // [2] P V of tile A / B done
  Y_SCF = Y_PVD + 2,     // [NSC]
  Y_SCE = Y_SCF + NSC,   // [NSC]
  Y_FIN = Y_SCE + NSC,
  Y_COUNT = Y_FIN + 1
};
static_assert(Y_COUNT * 8 + 8 <= 512, "barrier block overflows its region");

template <int KIND, int D, int SC>
__global__ void __launch_bounds__(PNT, 1)
    attn_pair_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                     const __grid_constant__ CUtensorMap tmv, const P2 p) {
  static_assert(KIND == K_E4M3 || KIND == K_BF16 || (KIND == K_S8 && SC != SC_TILE) ||
                    ((KIND == K_MXF4 || KIND == K_MXF8) && SC == SC_HEAD),
                "E4M3, INT8, MX or bf16 operands");
  using L = LP<KIND, D>;
  constexpr bool MX = L::MX;
  constexpr int TN = L::TN;
  constexpr bool RING = MX || SC != SC_HEAD;  // per-tile records (and K scales / atoms) through the scale ring
  constexpr int NKS = L::NK;  // K stages of this kind
  constexpr int NVS = L::NV;  // V' stages of this kind
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L::BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + Y_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar + Y_COUNT + 1);
  float* misc = reinterpret_cast<float*>(smem + L::MISC);  // [0] = v_ref

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---- work item: batch b, the two tiles' query heads and first rows; heaviest first when causal
  int b, hqt[2], q0t[2];
  if (p.pair_heads) {
    const int hp = p.Hq / 2, per_t = p.B * hp;
    const int qt = p.causal ? (p.n_qtiles - 1 - (int)blockIdx.x / per_t) : ((int)blockIdx.x / per_t);
    const int r = blockIdx.x % per_t;
    b = r / hp;
    hqt[0] = 2 * (r % hp);
    hqt[1] = hqt[0] + 1;
    q0t[0] = q0t[1] = qt * BM;
  } else {
    const int np = (p.n_qtiles + 1) / 2, per_t = p.B * p.Hq;
    const int pt = p.causal ? (np - 1 - (int)blockIdx.x / per_t) : ((int)blockIdx.x / per_t);
    const int r = blockIdx.x % per_t;
    b = r / p.Hq;
    hqt[0] = hqt[1] = r % p.Hq;
    q0t[0] = 2 * pt * BM;
    q0t[1] = q0t[0] + BM;
  }
  const int hk = hqt[0] / p.group;
  const int diag = p.Sk - p.Sq;
  int nt[2];
#pragma unroll
  for (int x = 0; x < 2; ++x) {
    int kv_end = 0;
    if (q0t[x] < p.Sq) kv_end = p.causal ? min(p.Sk, max(0, min(q0t[x] + BM, p.Sq) - 1 + diag + 1)) : p.Sk;
    nt[x] = (kv_end + TN - 1) / TN;
  }
  const int n = max(nt[0], nt[1]);
  const int bhk = b * p.Hkv + hk;

  if (tid == 0) {
    mbar_init(&bar[Y_Q], MX ? 2 : 1);  // MX: the Q codes and the Q tiles' scale-factor atoms
    for (int i = 0; i < NKS; ++i) {
      mbar_init(&bar[Y_KF + i], 1);
      mbar_init(&bar[Y_KE + i], 1);
    }
    for (int i = 0; i < NVS; ++i) {
      mbar_init(&bar[Y_VF + i], 1);
      mbar_init(&bar[Y_VE + i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar[Y_SF + i], 1);
      mbar_init(&bar[Y_PF + i], 4);
      mbar_init(&bar[Y_PVD + i], 1);
    }
    for (int i = 0; i < NSC; ++i) {
      mbar_init(&bar[Y_SCF + i], 1);
      mbar_init(&bar[Y_SCE + i], 8);  // both softmax warpgroups
    }
    mbar_init(&bar[Y_FIN], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;  // columns as in LP

  if (warp < 4) {
    setmaxnreg_dec<PR0>();
    const bool bnsd = p.layout == FA_LAYOUT_BNSD;
    if (warp == 0) {
      // ------------------------------------------------------ Q and K loads
      if (lane == 0 && n > 0) {
        tma_prefetch_desc(&tmq);
        tma_prefetch_desc(&tmk);
        mbar_arrive_expect_tx(&bar[Y_Q], ((nt[0] > 0) + (nt[1] > 0)) * BM * L::RB);
#pragma unroll
        for (int x = 0; x < 2; ++x)
          if (nt[x] > 0)
#pragma unroll
            for (int a = 0; a < L::NA; ++a)
              tma_load_4d(smem + L::Q + x * BM * L::RB + a * BM * L::AB, &tmq, &bar[Y_Q], a * L::AB,
                          bnsd ? q0t[x] : hqt[x], bnsd ? hqt[x] : q0t[x], b);
        int j = 0;
        for (; j < n; ++j) {
          const int k0 = j * TN, ks = j % NKS;
          if (j >= NKS && !mbar_wait(&bar[Y_KE + ks], ((j / NKS) - 1) & 1, abort_flag, p.status, 81)) break;
          mbar_arrive_expect_tx(&bar[Y_KF + ks], TN * L::RB);
#pragma unroll
          for (int a = 0; a < L::NA; ++a)
            tma_load_4d(smem + L::K + ks * TN * L::RB + a * TN * L::AB, &tmk, &bar[Y_KF + ks], a * L::AB,
                        bnsd ? k0 : hk, bnsd ? hk : k0, b);
        }
        if (*abort_flag) {
          mbar_drain(&bar[Y_Q], 0);
          for (int t = max(0, j - NKS); t < j; ++t) mbar_drain(&bar[Y_KF + t % NKS], (t / NKS) & 1);
        }
      }
      __syncwarp();
    } else if (warp == 3) {
      // --------------------------------------------------------- V' loads
      if (lane == 0 && n > 0) {
        tma_prefetch_desc(&tmv);
        int j = 0;
        for (; j < n; ++j) {
          const int k0 = j * TN, vs = j % NVS;
          if (j >= NVS && !mbar_wait(&bar[Y_VE + vs], ((j / NVS) - 1) & 1, abort_flag, p.status, 82)) break;
          mbar_arrive_expect_tx(&bar[Y_VF + vs], TN * D * 2);
#pragma unroll
          for (int a2 = 0; a2 < D / 64; ++a2)
            tma_load_4d(smem + L::VH + vs * TN * D * 2 + a2 * TN * 128, &tmv, &bar[Y_VF + vs], 64 * a2, k0, hk, b);
        }
        if (*abort_flag)
          for (int t = max(0, j - NVS); t < j; ++t) mbar_drain(&bar[Y_VF + t % NVS], (t / NVS) & 1);
      }
      __syncwarp();
    } else if (warp == 2) {
      // ------------------------------------------------------- scale ring
      if (MX && n > 0) {
        // the Q tiles' scale-factor atoms, published with the Q codes' barrier (rows past Sq: 0)
#pragma unroll
        for (int x = 0; x < 2; ++x)
          write_sf_atom(smem + L::SFA + x * 512, p.qe8, (long long)(b * p.Hq + hqt[x]) * p.Sq + q0t[x], p.Sq - q0t[x],
                        lane);
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[Y_Q]);
      }
      if (RING && n > 0) {
        const float4* fvh = p.fvr + (long long)bhk * p.ntiles_k;
        float m = 0.0f;
        for (int t = lane; t < n; t += 32) m = fmaxf(m, __ldg(&fvh[t].x));
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        if (lane == 0) {
          // v_ref: the largest V' factor over this CTA's tiles, and its log2.  MX: the records hold
          // {E_t, E_t - 127}, so v_ref = 2^(E_ref - 127) with E_ref the largest E_t.
          misc[0] = MX ? exp2f(m - 127.0f) : (m > 0.0f ? m : 1.0f);
          misc[1] = MX ? m - 127.0f : log2f(misc[0]);
          const float* kph = p.ksp + (long long)bhk * p.ntiles_k * BN;
          int j = 0;
          for (; j < n; ++j) {
            const int st = j % NSC;
            if (j >= NSC && !mbar_wait(&bar[Y_SCE + st], ((j / NSC) - 1) & 1, abort_flag, p.status, 80)) break;
            uint8_t* stage = smem + L::SC + st * 2 * BN * 4;
            mbar_arrive_expect_tx(&bar[Y_SCF + st], BN * 4 + 16);
            bulk_load(stage, kph + (long long)j * BN, BN * 4, &bar[Y_SCF + st]);
            bulk_load(stage + BN * 4, fvh + j, 16, &bar[Y_SCF + st]);
          }
          if (*abort_flag)
            for (int t = max(0, j - NSC); t < j; ++t) mbar_drain(&bar[Y_SCF + t % NSC], (t / NSC) & 1);
        }
      }
      __syncwarp();
    } else {
      // ---------------------------------------------------------- MMA issuer
      if (lane == 0 && n > 0) {
        constexpr uint32_t SW = L::AB == 128 ? kSwz128 : kSwz64;
        constexpr uint32_t SBO8 = L::AB == 128 ? 1024 : 512;
        constexpr uint32_t idesc_qk = KIND == K_E4M3   ? make_idesc(kAccF32, kFmtE4M3, kFmtE4M3, 0, 0, TN, BM)
                                      : KIND == K_BF16 ? make_idesc(kAccF32, kFmtBF16, kFmtBF16, 0, 0, TN, BM)
                                                       : make_idesc(kAccS32, kFmtS8, kFmtS8, 0, 0, TN, BM);
        constexpr uint32_t idesc_pv = make_idesc(kAccF32, kFmtF16, kFmtF16, 0, 1, D, BM);
        // Descriptors as 32-bit halves: the high half (stride, version, swizzle) is constant per
        // tile kind, the low half (start address >> 4 | leading offset) is computed once per tile
        // base, and each MMA adds a compile-time offset (>> 4) to it, which stays inside the 14-bit
        // address field (shared memory is below 256 KB).  The issuing warp shares its SM
        // sub-partition with two softmax warps, so each MMA costs it only a few instructions.
        const uint64_t dq0 = make_sdesc(smem_u32(smem + L::Q), 16, SBO8, SW);
        const uint64_t dv0 = make_sdesc(smem_u32(smem + L::VH), TN * 128, 1024, kSwz128);
        const uint32_t qk_hi = (uint32_t)(dq0 >> 32), v_hi = (uint32_t)(dv0 >> 32);
        const uint32_t q_lo = (uint32_t)dq0, k_lo = (uint32_t)make_sdesc(smem_u32(smem + L::K), 16, SBO8, SW);
        const uint32_t v_lo = (uint32_t)dv0;
        auto qk = [&](int x, int j) {
          const uint32_t ql = q_lo + (x ? (uint32_t)((BM * L::RB) >> 4) : 0u);
          const uint32_t kl = k_lo + (uint32_t)(j % NKS) * (uint32_t)((TN * L::RB) >> 4);
          // one MMA per 32 bytes of the row (K = 32 codes, 64 E2M1, or 16 bf16): atom a = kk * 32 / AB
#pragma unroll
          for (int kk = 0; kk < L::RB / 32; ++kk) {
            const uint32_t off = ((kk * 32 / L::AB) * BM * L::AB + (kk * 32) % L::AB) >> 4;
            if constexpr (MX) {
              // block scales from TMEM: this tile's Q factors, the K tile's (slot j % 2); the
              // factor id picks the row's scale bytes for this MMA's K range
              const uint64_t da = ((uint64_t)qk_hi << 32) | (ql + off), db = ((uint64_t)qk_hi << 32) | (kl + off);
              const uint32_t sfa = tbase + L::TSFQ + 8 * x, sfb = tbase + L::TSFK + 8 * (j & 1);
              if (KIND == K_MXF4)
                mma_mxf4(tbase + L::TS0 + x * 128, da, db,
                         make_idesc_bs(kFmtE2M1x, kFmtE2M1x, TN, BM, 2 * kk, 2 * kk), sfa, sfb, kk > 0);
              else
                mma_mxf8(tbase + L::TS0 + x * 128, da, db, make_idesc_bs(kFmtE4M3, kFmtE4M3, TN, BM, kk, kk), sfa,
                         sfb, kk > 0);
            } else if (KIND == K_E4M3) {
              mma_f8f6f4_lh(tbase + x * 128, ql + off, qk_hi, kl + off, qk_hi, idesc_qk, kk > 0);
            } else if (KIND == K_BF16) {
              mma_f16_lh(tbase + x * 128, ql + off, qk_hi, kl + off, qk_hi, idesc_qk, kk > 0);
            } else {
              mma_i8_lh(tbase + x * 128, ql + off, qk_hi, kl + off, qk_hi, idesc_qk, kk > 0);
            }
          }
          mma_commit(&bar[Y_SF + x]);
        };
        auto pv = [&](int x, int j) {
          // A = P' in TMEM: key k of the tile sits in column k / 2 of S_x (fp16 pairs)
          const uint32_t vl = v_lo + (uint32_t)(j % NVS) * (uint32_t)((TN * D * 2) >> 4);
#pragma unroll
          for (int ks = 0; ks < TN / 16; ++ks)
            mma_f16_ts_lh(tbase + L::TO0 + x * (L::TO1 - L::TO0), tbase + L::TS0 + x * 128 + ks * 8,
                          vl + (uint32_t)((ks * 16 * 128) >> 4), v_hi, idesc_pv, (j > 0 || ks > 0) ? 1u : 0u);
          mma_commit(&bar[Y_PVD + x]);
        };
        // MX: K tile j's scale-factor atom (in its scale ring stage) into TMEM slot j % 2, ordered
        // before the MMAs that read it
        auto k_factors = [&](int j) {
          if constexpr (MX) {
            if (!mbar_wait(&bar[Y_SCF + j % NSC], (j / NSC) & 1, abort_flag, p.status, 88)) return false;
            tc_fence_after();
            sf_to_tmem(tbase + L::TSFK + 8 * (j & 1), smem_u32(smem + L::SC + (j % NSC) * 2 * BN * 4));
          }
          return true;
        };
        bool ok = mbar_wait(&bar[Y_Q], 0, abort_flag, p.status, 83);
        if (MX && ok) {
          tc_fence_after();
          sf_to_tmem(tbase + L::TSFQ, smem_u32(smem + L::SFA));
          sf_to_tmem(tbase + L::TSFQ + 8, smem_u32(smem + L::SFA + 512));
        }
        if (ok) ok = mbar_wait(&bar[Y_KF], 0, abort_flag, p.status, 84) && k_factors(0);
        if (ok) {
          tc_fence_after();
          if (nt[0] > 0) qk(0, 0);
          if (nt[1] > 0) qk(1, 0);
          mma_commit(&bar[Y_KE]);
        }
        for (int j = 0; ok && j < n; ++j) {
          bool v_ready = false, k_ready = false;
#pragma unroll
          for (int x = 0; x < 2 && ok; ++x) {
            if (j >= nt[x]) continue;
            ok = chain_wait<(FAQ_PAIR_SPIN & 1) != 0>(&bar[Y_PF + x], j & 1, abort_flag, p.status, 85);
            if (ok && !v_ready)
              ok = v_ready = chain_wait<(FAQ_PAIR_SPIN & 4) != 0>(&bar[Y_VF + j % NVS], (j / NVS) & 1, abort_flag,
                                                                  p.status, 86);
            if (!ok) break;
            tc_fence_after();
            pv(x, j);
            if (j + 1 < nt[x]) {
              if (!k_ready)
                ok = k_ready = chain_wait<(FAQ_PAIR_SPIN & 4) != 0>(&bar[Y_KF + (j + 1) % NKS], ((j + 1) / NKS) & 1,
                                                                    abort_flag, p.status, 87) &&
                               k_factors(j + 1);
              if (!ok) break;
              tc_fence_after();
              qk(x, j + 1);
            }
          }
          if (!ok) break;
          mma_commit(&bar[Y_VE + j % NVS]);
          if (j + 1 < n) mma_commit(&bar[Y_KE + (j + 1) % NKS]);
        }
        mma_commit(&bar[Y_FIN]);
        mbar_drain(&bar[Y_FIN], 0);
      }
      __syncwarp();
    }
  } else {
    setmaxnreg_inc<PRS>();
    // ------------------------------------------------------------- softmax
    const int x = (warp - 4) >> 2;  // query tile of this warpgroup
    const int i = tid - 128 - x * 128;
    const uint32_t loff = (uint32_t)((warp & 3) * 32) << 16;
    const int hq = x ? hqt[1] : hqt[0], q0 = x ? q0t[1] : q0t[0], nx = x ? nt[1] : nt[0];
    const int row = q0 + i;
    const bool row_ok = row < p.Sq;
    const int qbh = b * p.Hq + hq;
    const uint32_t tS = tbase + L::TS0 + x * 128;
    const uint32_t tO = tbase + L::TO0 + x * (L::TO1 - L::TO0);
    // MX: the block scales are applied inside the MMA, so only the softmax scale
    const float sq = row_ok ? (MX ? 1.0f : scale_at(p.qs, p.q_blk, p.q_nblk, qbh, hq, row)) : 0.0f;
    float crow = sq * p.scale_log2;
    if (!RING) crow *= __ldg(p.ks + hk);
    // S8 accumulators with one K scale per head arrive biased (t = 1.5 * 2^23 + acc, exact for
    // |acc| < 2^22); with per-key K scales they are converted exactly instead
    constexpr bool BIASED = KIND == K_S8 && SC == SC_HEAD;
    constexpr float kBias = BIASED ? 12582912.0f : 0.0f;
    float vref = RING ? 1.0f : __ldg(p.vs + hk);
    float m_run = -INFINITY, l_run = 0.0f;
    float lgref = 0.0f;  // log2(v_ref)
    bool ok = true;
    for (int j = 0; j < n && ok; ++j) {
      const int k0 = j * TN;
      const int sst = j % NSC;
      const float* ksc = reinterpret_cast<const float*>(smem + L::SC + sst * 2 * BN * 4);
      if (RING && !warp_wait(&bar[Y_SCF + sst], (j / NSC) & 1, abort_flag, p.status, 90)) { ok = false; break; }
      if (RING && j == 0) {
        vref = misc[0];
        lgref = misc[1];
      }
      if (j >= nx) {
        // the other tile's key range is longer: release the ring stage and move on
        if (RING) {
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar[Y_SCE + sst]);
        }
        continue;
      }
      float flog = 0.0f, finv = 1.0f, cr = crow;
      if (RING) {
        // the V' factor r_t / v_ref as its log2 (the record holds log2 r_t), floored at -60
        flog = fmaxf(ksc[BN + 1] - lgref, -60.0f);
        finv = ex2(-flog);
      }
      if (SC == SC_TILE) cr *= ksc[0];
      // the tile's per-key K scales into registers while S is still being computed
      float ksr[SC == SC_COL ? BN : 1];
      if (SC == SC_COL) {
#pragma unroll
        for (int k = 0; k < BN; k += 4) *reinterpret_cast<float4*>(&ksr[k]) = *reinterpret_cast<const float4*>(ksc + k);
      }
      if (!__all_sync(0xffffffffu, chain_wait<(FAQ_PAIR_SPIN & 2) != 0>(&bar[Y_SF + x], j & 1, abort_flag, p.status, 91))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float t[TN];
      // S from TMEM (all four 32-column loads, one wait), the per-key K scale, the masks
      auto load_s = [&](bool again) {
        // per-key K scales: two halves of 64 columns, so half of the scales' registers are free
        // before the second half of S lands; otherwise all four loads and one wait
        constexpr int NH = SC == SC_COL ? 2 : 1;
#pragma unroll
        for (int hh = 0; hh < NH; ++hh) {
          constexpr int W = TN / NH;
          static_assert(W % 16 == 0, "S loads of 32 and 16 columns");
          uint32_t tr[W];
#pragma unroll
          for (int c = 0; c < W / 32; ++c)
            tmem_ld32(tS + loff + W * hh + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&tr[32 * c]));
          if constexpr (W % 32 != 0)  // 112-key tiles: the last 16 columns
            tmem_ld16(tS + loff + W * hh + W / 32 * 32, *reinterpret_cast<uint32_t(*)[16]>(&tr[W / 32 * 32]));
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < W; ++k)
            t[W * hh + k] = BIASED ? __uint_as_float(0x4B400000u + tr[k])
                                   : (KIND == K_S8 ? (float)(int)tr[k] : __uint_as_float(tr[k]));
          if (SC == SC_COL) {
            if (!again) {
#pragma unroll
              for (int k = W * hh; k < W * hh + W; k += 2) fmul2(t[k], t[k + 1], ksr[k], ksr[k + 1]);
            } else {
              // a second read: the scales again from the ring stage (still held), not kept in registers
#pragma unroll
              for (int k = W * hh; k < W * hh + W; k += 4) {
                const float4 kv = *reinterpret_cast<const float4*>(ksc + k);
                fmul2(t[k], t[k + 1], kv.x, kv.y);
                fmul2(t[k + 2], t[k + 3], kv.z, kv.w);
              }
            }
          }
        }
        const bool need_mask = (k0 + TN > p.Sk) || (p.causal && (k0 + TN - 1 > q0 + diag));
        if (need_mask) {
          const int lim = p.causal ? min(p.Sk - 1, row + diag) : p.Sk - 1;
#pragma unroll
          for (int k = 0; k < TN; ++k)
            if (k0 + k > lim) t[k] = -INFINITY;
        }
      };
      // p' = 2^(t * cr - (bias * cr + m) + log2(r_t / v_ref)) in place, and their sum
      auto exponentials = [&](float m) -> float {
        const float nb = (m == -INFINITY ? 0.0f : -(kBias * cr + m)) + flog;
#pragma unroll
        for (int k = 0; k < TN; k += 2) {
          ffma2(t[k], t[k + 1], cr, cr, nb, nb);
          if (((k >> 1) & 7) < (MX ? FAQ_PAIR_POLY_MX : FAQ_PAIR_POLY)) {
            ex2_poly2(t[k], t[k + 1]);  // this share of the pairs on the FMA pipe
          } else {
            t[k] = ex2(t[k]);
            t[k + 1] = ex2(t[k + 1]);
          }
        }
        float ls[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) ls[e] = t[e];
#pragma unroll
        for (int k = 8; k < TN; k += 2) fadd2(ls[k & 7], ls[(k & 7) + 1], t[k], t[k + 1]);
        return ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
      };
      load_s(false);
      // Speculative exponentials.  After a row's first tile the running max rarely moves, so
      // the tile is exponentiated against it directly, without its own row maximum.  The sum
      // tells whether that was safe: below 2^15 every p' stays below 2^15 (fp16 holds it) and
      // the max would not have moved by more than 2^8 (the lazy rule below).  Otherwise -- and
      // on a row's first tile -- S is read again (P' has not overwritten it yet), the tile's
      // maximum taken, O rescaled if the maximum moves, and the exponentials redone.
      float l_tile = 0.0f;
      bool exact = __any_sync(0xffffffffu, m_run == -INFINITY);
      bool failed = false;
#pragma unroll 1
      for (int pass = 0; pass < 2; ++pass) {
        if (exact) {
          // row maximum: eight chains of three-input maxima
          float mx[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            mx[e] = t[e];
#pragma unroll
            for (int q = 1; q < TN / 8; q += 2)
              mx[e] = q + 1 < TN / 8 ? fmax3(mx[e], t[e + 8 * q], t[e + 8 * q + 8]) : fmaxf(mx[e], t[e + 8 * q]);
          }
          const float mt = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
          const float mts = mt == -INFINITY ? -INFINITY : (mt - kBias) * cr;  // log2 domain
          // the running max moves only when the tile's max exceeds it by more than 2^8
          const float m_fin = mts > m_run + 8.0f ? mts : m_run;
          const float alpha = m_fin != m_run ? ex2(m_run - m_fin) : 1.0f;
          if (__any_sync(0xffffffffu, m_fin != m_run) && j > 0) {
            // O is free once P V of tile j-1 has completed
            if (!warp_wait(&bar[Y_PVD + x], (j - 1) & 1, abort_flag, p.status, 92)) { failed = true; break; }
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
              uint32_t r[32];
              tmem_ld32(tO + loff + c * 32, r);
              tmem_ld_wait();
#pragma unroll
              for (int k = 0; k < 32; k += 2) {
                float a0 = __uint_as_float(r[k]), a1 = __uint_as_float(r[k + 1]);
                fmul2(a0, a1, alpha, alpha);
                r[k] = __float_as_uint(a0);
                r[k + 1] = __float_as_uint(a1);
              }
              tmem_st32(tO + loff + c * 32, r);
            }
            tmem_st_wait();
          }
          l_run *= alpha;
          m_run = m_fin;
        }
        l_tile = exponentials(m_run);
        if (exact || !__any_sync(0xffffffffu, !(l_tile < 32768.0f))) break;
        exact = true;
        load_s(true);
      }
      if (failed) { ok = false; break; }
      {
        uint32_t hp[TN / 2];
#pragma unroll
        for (int e = 0; e < TN / 2; ++e) {
          const __half2 hv = __floats2half2_rn(t[2 * e], t[2 * e + 1]);
          hp[e] = *reinterpret_cast<const uint32_t*>(&hv);
        }
        tmem_st32(tS + loff, *reinterpret_cast<uint32_t(*)[32]>(&hp[0]));
        if constexpr (TN == 128) {
          tmem_st32(tS + loff + 32, *reinterpret_cast<uint32_t(*)[32]>(&hp[32]));
        } else {  // 112 keys: 56 columns
          static_assert(TN == 112, "P' stores of 32 + 16 + 8 columns");
          tmem_st16(tS + loff + 32, *reinterpret_cast<uint32_t(*)[16]>(&hp[32]));
          tmem_st8(tS + loff + 48, *reinterpret_cast<uint32_t(*)[8]>(&hp[48]));
        }
      }
      tmem_st_wait();
      l_run += l_tile * finv;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bar[Y_PF + x]);
        if (RING) mbar_arrive(&bar[Y_SCE + sst]);
      }
    }
    // ---------------------------------------------------------- epilogue
    if (ok && nx > 0) {
      ok = warp_wait(&bar[Y_PVD + x], (nx - 1) & 1, abort_flag, p.status, 93);
      tc_fence_after();
    }
    if (q0 < p.Sq) {
      const float ofac = l_run > 0.0f ? vref / l_run : 0.0f;
      __nv_bfloat16* orow = nullptr;
      bool out_ok = row_ok;
      if (row_ok) {
        const long long ridx = p.layout == FA_LAYOUT_BNSD ? ((long long)qbh * p.Sq + row)
                                                          : (((long long)b * p.Sq + row) * p.Hq + hq);
        out_ok = in_bounds(ridx >= 0 && ridx < (long long)p.B * p.Hq * p.Sq, 123);
        orow = p.out + ridx * D;
      }
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        if (ok && nx > 0) {
          tmem_ld32(tO + loff + c * 32, r);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) r[k] = 0u;
        }
        if (out_ok) {
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
      if (out_ok && p.lse && in_bounds((long long)qbh * p.Sq + row < (long long)p.B * p.Hq * p.Sq, 124))
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

// ---- V pre-pass: one CTA per (128-token tile, b * Hkv + h).
// V scales per token or per block (VSC): r_t = max s_v over the tile's tokens (1 if all are 0),
//   V' = fp16(code * (s_v / r_t)) (|V'| <= 448 for E4M3, 127 for INT8), r_t in the tile's record and
//   the tile's per-key K scales beside it.
// V scale per head: V' = fp16(code) exactly (the per-head scale stays outside).
// MXFP4: E_t = the largest UE8M0 byte of the tile's tokens, V' = fp16(e2m1 * 2^(e - E_t)), |V'| <= 6.
// V pre-pass: V' fp16 tiles + per-tile factor records (+ the K tile's per-key scales).  MIXED:
// records are linear factors for every kind (the bf16 pair kernel's scale ring) and the per-key K
// scales are 1 (Q and K arrive dequantized).
// TN: keys per tile (112 for the MX pair kernel; 128 otherwise).
template <int KIND, int D, bool VSC, bool MIXED = false, int TN = BN>
__global__ void __launch_bounds__(256) vprep_kernel(const uint8_t* __restrict__ codes, const float* __restrict__ vs,
                                                    int v_blk, int v_nblk, int H, int S, int layout,
                                                    __half* __restrict__ vh, float4* __restrict__ fvr, int ntiles,
                                                    const float* __restrict__ ks, int k_blk, int k_nblk,
                                                    float* __restrict__ ksp, const uint8_t* __restrict__ ve8,
                                                    const uint8_t* __restrict__ ke8) {
  static_assert(TN == BN || KIND == K_MXF4 || KIND == K_MXF8, "112-key tiles: MX kinds only");
  static_assert(TN <= BN && TN % 16 == 0, "a tile fits the CTA's 128 token slots");
  const int t = blockIdx.x, bh = blockIdx.y;
  // the tile's records and V' rows: tile t of ntiles, (b, h) row bh of the launch's B * H
  if (!in_bounds(t < ntiles && (long long)t * TN < (long long)S + TN, 125)) return;
  const int b = bh / H, h = bh % H;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int tok0 = t * TN;
  const int slot = warp * 16 + (lane >> 1);  // token slot of this thread within the tile
  const int tok = tok0 + slot;
  // rows past S stay unwritten: the attention's TMA box reads them as zero
  const bool live = tok < S && slot < TN;
  const long long src_row = layout == FA_LAYOUT_BNSD ? ((long long)bh * S + tok) : (((long long)b * S + tok) * H + h);
  if constexpr (KIND == K_MXF4 || KIND == K_MXF8) {
    static_assert(D == 128, "MX paths: head_dim 128");
    constexpr bool F8 = KIND == K_MXF8;
    // each thread owns half a code row: two 32-element scale blocks of 16 (E2M1) or 32 (E4M3) bytes
    constexpr int NC = F8 ? 4 : 2;  // 16-byte chunks per thread
    const uint8_t* src = codes + src_row * (F8 ? D : D / 2) + (lane & 1) * (F8 ? D / 2 : D / 4);
    uint4 raw[NC];
#pragma unroll
    for (int c = 0; c < NC; ++c) raw[c] = live ? __ldg(reinterpret_cast<const uint4*>(src) + c) : make_uint4(0, 0, 0, 0);
    const uint32_t* ve4 = reinterpret_cast<const uint32_t*>(ve8) + (long long)bh * S;
    int m = 0;  // E_t, reduced by every warp itself
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int tt = tok0 + lane * 4 + q;
      if (tt < S && lane * 4 + q < TN) {
        const uint32_t w = __ldg(ve4 + tt);
        m = max(m, (int)max(max(w & 0xFFu, (w >> 8) & 0xFFu), max((w >> 16) & 0xFFu, w >> 24)));
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
    if (threadIdx.x == 0)
      fvr[(long long)bh * ntiles + t] = make_float4(MIXED ? ldexpf(1.0f, m - 127) : (float)m, (float)(m - 127), 0.0f, 0.0f);
    if (MIXED) {
      if (threadIdx.x < BN) ksp[((long long)bh * ntiles + t) * BN + threadIdx.x] = tok0 + (int)threadIdx.x < S ? 1.0f : 0.0f;
    } else if (threadIdx.x < BN) {
      // the K tile's scale-factor atom: token row r at byte (r % 32) * 16 + (r / 32) * 4, zero past S
      // (and, for 112-key tiles, in the atom's last 16 rows)
      const int key = tok0 + threadIdx.x;
      const uint32_t w = (key < S && (int)threadIdx.x < TN)
                             ? __ldg(reinterpret_cast<const uint32_t*>(ke8) + (long long)bh * S + key)
                             : 0u;
      reinterpret_cast<uint32_t*>(ksp + ((long long)bh * ntiles + t) * BN)[(threadIdx.x & 31) * 4 + (threadIdx.x >> 5)] = w;
    }
    if (!live) return;
    const uint32_t e4 = __ldg(ve4 + tok);
    uint4* dst = reinterpret_cast<uint4*>(vh + ((long long)bh * S + tok) * D + (lane & 1) * (D / 2));
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      const int blk = (lane & 1) * 2 + (F8 ? c / 2 : c);             // 32-element block of the row
      const int de = (int)((e4 >> (8 * blk)) & 0xFFu) - m;  // <= 0
      const __half fs = de >= -24 ? __float2half_rn(ldexpf(1.0f, de)) : __float2half_rn(0.0f);
      const __half2 f2 = __halves2half2(fs, fs);
      const uint32_t w[4] = {raw[c].x, raw[c].y, raw[c].z, raw[c].w};
      if (F8) {  // 16 E4M3 bytes -> 16 fp16
        uint32_t o[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t v2 = e4m3x2_to_h2((uint16_t)(w[i >> 1] >> ((i & 1) * 16)));
          const __half2 y = __hmul2(*reinterpret_cast<const __half2*>(&v2), f2);
          o[i] = *reinterpret_cast<const uint32_t*>(&y);
        }
        dst[2 * c] = make_uint4(o[0], o[1], o[2], o[3]);
        dst[2 * c + 1] = make_uint4(o[4], o[5], o[6], o[7]);
      } else {
        uint32_t o[16];  // byte i holds elements 2i (low nibble) and 2i + 1
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint32_t v2 = e2m1x2_to_h2((w[i >> 2] >> (8 * (i & 3))) & 0xFFu);
          const __half2 y = __hmul2(*reinterpret_cast<const __half2*>(&v2), f2);
          o[i] = *reinterpret_cast<const uint32_t*>(&y);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) dst[4 * c + q] = make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
      }
    }
    return;
  } else if constexpr (KIND == K_BF16) {
    // unquantized V: V' = fp16(v / r_t), r_t the power of two that puts the tile's max |v| in
    // [2^14, 2^15) (exact scaling; fp16 keeps 11 bits), records r_t
    __shared__ float red[8];
    constexpr int NC = D / 16;  // 16-byte chunks (8 bf16) per thread: half a row
    const uint4* src = reinterpret_cast<const uint4*>(codes + (src_row * D + (lane & 1) * (D / 2)) * 2);
    uint4 raw[NC];
    uint32_t m2 = 0;
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      raw[c] = live ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
      m2 = bf16x2_absmax(bf16x2_absmax(m2, raw[c].x), bf16x2_absmax(raw[c].y, raw[c].z));
      m2 = bf16x2_absmax(m2, raw[c].w);
    }
    m2 &= 0x7FFF7FFFu;
    float am = fmaxf(__uint_as_float(m2 << 16), __uint_as_float(m2 & 0xFFFF0000u));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, off));
    if (lane == 0) red[warp] = am;
    __syncthreads();
    am = fmaxf(fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3])), fmaxf(fmaxf(red[4], red[5]), fmaxf(red[6], red[7])));
    int E = (int)((__float_as_uint(am) >> 23) & 0xFFu) - 127;  // floor(log2 am) for a normal am
    E = max(E, -112);
    const float r = am > 0.0f ? __uint_as_float((uint32_t)(E - 14 + 127) << 23) : 1.0f;
    const float inv = am > 0.0f ? __uint_as_float((uint32_t)(14 - E + 127) << 23) : 1.0f;
    if (threadIdx.x == 0) fvr[(long long)bh * ntiles + t] = make_float4(r, am > 0.0f ? (float)(E - 14) : 0.0f, 0.0f, 0.0f);
    if (threadIdx.x < BN) ksp[((long long)bh * ntiles + t) * BN + threadIdx.x] = tok0 + (int)threadIdx.x < S ? 1.0f : 0.0f;
    if (!live) return;
    uint4* dst = reinterpret_cast<uint4*>(vh + ((long long)bh * S + tok) * D + (lane & 1) * (D / 2));
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      const uint32_t w[4] = {raw[c].x, raw[c].y, raw[c].z, raw[c].w};
      uint32_t o[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const __half2 y = __floats2half2_rn(__uint_as_float(w[i] << 16) * inv, __uint_as_float(w[i] & 0xFFFF0000u) * inv);
        o[i] = *reinterpret_cast<const uint32_t*>(&y);
      }
      dst[c] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    return;
  }
  constexpr int CPT = D / 32;  // 16-code chunks per thread: each thread owns half a token row
  const uint8_t* src = codes + src_row * D + (lane & 1) * (D / 2);
  uint4 raw[CPT];
#pragma unroll
  for (int c = 0; c < CPT; ++c) raw[c] = live ? __ldg(reinterpret_cast<const uint4*>(src) + c) : make_uint4(0, 0, 0, 0);
  float f = 1.0f;
  if (VSC) {
    // every warp reduces the tile's 128 scales itself (no block barrier); v_blk 0: one per head
    const float* vsh = vs + (long long)bh * v_nblk;
    float m = 0.0f;
    if (v_blk == 0) {
      m = __ldg(vs + h);
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int tt = tok0 + lane * 4 + q;
        if (tt < S) m = fmaxf(m, __ldg(vsh + tt / v_blk));
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    }
    const float r = m > 0.0f ? m : 1.0f;
    f = live ? (v_blk == 0 ? m : __ldg(vsh + tok / v_blk)) / r : 0.0f;
    if (threadIdx.x == 0) fvr[(long long)bh * ntiles + t] = make_float4(r, log2f(r), 0.0f, 0.0f);
    // the tile's per-key K scales, zero past S, at a 16-byte aligned per-tile slot
    if (threadIdx.x < BN) {
      const int key = tok0 + threadIdx.x;
      ksp[((long long)bh * ntiles + t) * BN + threadIdx.x] =
          key < S ? (MIXED ? 1.0f : __ldg(ks + (long long)bh * k_nblk + key / k_blk)) : 0.0f;
    }
  }
  if (!live) return;
  uint4* dst = reinterpret_cast<uint4*>(vh + ((long long)bh * S + tok) * D + (lane & 1) * (D / 2));
#pragma unroll
  for (int c = 0; c < CPT; ++c) {
    const uint32_t w[4] = {raw[c].x, raw[c].y, raw[c].z, raw[c].w};
    uint32_t o[8];
    if (KIND == K_E4M3) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t h2 = e4m3x2_to_h2((uint16_t)(w[i >> 1] >> ((i & 1) * 16)));
        if (VSC) {
          const float2 x = __half22float2(*reinterpret_cast<const __half2*>(&h2));
          const __half2 y = __floats2half2_rn(x.x * f, x.y * f);
          o[i] = *reinterpret_cast<const uint32_t*>(&y);
        } else {
          o[i] = h2;  // exact
        }
      }
    } else if (VSC) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t pr = w[i >> 1] >> ((i & 1) * 16);
        const __half2 y = __floats2half2_rn((float)(int8_t)(pr & 0xFFu) * f, (float)(int8_t)((pr >> 8) & 0xFFu) * f);
        o[i] = *reinterpret_cast<const uint32_t*>(&y);
      }
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t ub = w[i] ^ 0x80808080u;
        o[2 * i] = s8x2_to_h2(ub, 0x4140);
        o[2 * i + 1] = s8x2_to_h2(ub, 0x4342);
      }
    }
    dst[2 * c] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[2 * c + 1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

// Tensor map over V' [B][H][S][D] fp16: 64-column x `rows`-token boxes, 128-byte swizzle.
cudaError_t make_vh_map(CUtensorMap* map, const void* base, int B, int H, int S, int D, int rows) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return cudaErrorNotSupported;
  const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)S, (cuuint64_t)H, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)S * D * 2, (cuuint64_t)H * S * D * 2};
  const cuuint32_t box[4] = {64, (cuuint32_t)rows, 1, 1};
  const cuuint32_t es[4] = {1, 1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

struct Prefill2Ws {
  __half* vh;
  float4* fvr;
  float* ksp;
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace: V' fp16 [B, Hkv, Sk, D] | V' factor records [B, Hkv, ntiles] | K scales [B, Hkv, ntiles * 128],
// ntiles = the key tiles of `tn` keys.
Prefill2Ws carve_ws(void* ws, int B, int Hkv, int Sk, int D, int tn = BN) {
  const size_t ntiles = ((size_t)Sk + tn - 1) / tn;
  uint8_t* base = static_cast<uint8_t*>(ws);
  Prefill2Ws w;
  w.vh = reinterpret_cast<__half*>(base);
  base += align256((size_t)B * Hkv * Sk * D * 2);
  w.fvr = reinterpret_cast<float4*>(base);
  base += align256((size_t)B * Hkv * ntiles * 16);
  w.ksp = reinterpret_cast<float*>(base);
  return w;
}

template <int KIND, int D, bool VSC, int TN = BN>
cudaError_t prepare2(const AttnArgs& a, const P2& prm, const Prefill2Ws& w, int RB, CUtensorMap* mq, CUtensorMap* mk,
                     CUtensorMap* mv, cudaStream_t s) {
  cudaError_t e;
  if ((e = make_code_map(mq, a.q->codes, a.q->B, a.q->H, a.q->S, RB, a.q->layout, BM)) != cudaSuccess) return e;
  if ((e = make_code_map(mk, a.k->codes, a.k->B, a.k->H, a.k->S, RB, a.k->layout, TN)) != cudaSuccess) return e;
  if ((e = make_vh_map(mv, w.vh, a.v->B, a.v->H, a.v->S, D, TN)) != cudaSuccess) return e;
  const dim3 pgrid((unsigned)prm.ntiles_k, (unsigned)(a.v->B * a.v->H));
  if (pgrid.y > 65535u) return cudaErrorInvalidValue;
  vprep_kernel<KIND, D, VSC, false, TN><<<pgrid, 256, 0, s>>>(static_cast<const uint8_t*>(a.v->codes), prm.vs, prm.v_blk,
                                               prm.v_nblk, a.v->H, a.v->S, a.v->layout, w.vh, w.fvr, prm.ntiles_k,
                                               prm.ks, prm.k_blk, prm.k_nblk, w.ksp, prm.ve8, prm.ke8);
  return cudaGetLastError();
}

template <int KIND, int D, int SC>
cudaError_t run_pair(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, P2 prm, cudaStream_t s) {
  using L = LP<KIND, D>;
  cudaError_t e;
  auto kern = attn_pair_kernel<KIND, D, SC>;
  if ((e = set_smem_limit(reinterpret_cast<const void*>(kern), L::ALLOC)) != cudaSuccess) return e;
  // GQA groups of even size pair two query heads at one row block (equal key ranges); otherwise
  // a head's row blocks pair up.
  prm.pair_heads = prm.group % 2 == 0;
  const long long grid = prm.pair_heads ? (long long)prm.n_qtiles * prm.B * (prm.Hq / 2)
                                        : (long long)((prm.n_qtiles + 1) / 2) * prm.B * prm.Hq;
  if (grid > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  kern<<<(unsigned)grid, PNT, L::ALLOC, s>>>(mq, mk, mv, prm);
  return cudaGetLastError();
}

template <int KIND, int D, int SC>
cudaError_t launch_pair(const AttnArgs& a, P2 prm, const Prefill2Ws& w, cudaStream_t s) {
  using L = LP<KIND, D>;
  CUtensorMap mq, mk, mv;
  cudaError_t e;
  if ((e = prepare2<KIND, D, L::MX || SC != SC_HEAD, L::TN>(a, prm, w, L::RB, &mq, &mk, &mv, s)) != cudaSuccess)
    return e;
  return run_pair<KIND, D, SC>(mq, mk, mv, prm, s);
}

// ------------------------------------------------------------ mixed branches

// Dequantized bf16 copy of a quantized operand, in its own layout: x = code * s (E4M3 / INT8
// codes, per-head, per-token or per-block scales) or code * 2^(e - 127) (MX, E8M0 e per 32
// elements); the product in fp32, then rounded to bf16.  One thread per 8 elements.
__global__ void __launch_bounds__(256) deq_bf16_kernel(const uint8_t* __restrict__ codes, const void* __restrict__ scales,
                                                       int mode, int B, int H, int S, int D, int layout, int blk,
                                                       __nv_bfloat16* __restrict__ out) {
  const int cpr = D / 8;  // 8-element chunks per row
  const long long n = (long long)B * H * S * cpr;
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < n; idx += stride) {
    const long long r = idx / cpr;  // token row in memory order
    const int c0 = (int)(idx - r * cpr) * 8;
    int b, h, t;
    if (layout == FA_LAYOUT_BNSD) {
      t = (int)(r % S);
      const long long bh = r / S;
      h = (int)(bh % H);
      b = (int)(bh / H);
    } else {
      h = (int)(r % H);
      const long long bs = r / H;
      t = (int)(bs % S);
      b = (int)(bs / S);
    }
    const long long bht = ((long long)b * H + h) * S + t;  // scales are [B, H, S, ...] in every layout
    float x[8];
    if (mode == FA_MODE_MXFP4_PER_BLOCK || mode == FA_MODE_MXFP8_PER_BLOCK) {
      const int e = (int)static_cast<const uint8_t*>(scales)[bht * (D / 32) + c0 / 32];
      const float sc = ldexpf(1.0f, e - 127);
      if (mode == FA_MODE_MXFP4_PER_BLOCK) {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(codes + r * (D / 2) + c0 / 2);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t h2 = e2m1x2_to_h2((w >> (8 * i)) & 0xFFu);
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h2));
          x[2 * i] = f.x * sc;
          x[2 * i + 1] = f.y * sc;
        }
      } else {
        const uint2 w = *reinterpret_cast<const uint2*>(codes + r * D + c0);
        const uint32_t ww[2] = {w.x, w.y};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t h2 = e4m3x2_to_h2((uint16_t)(ww[i >> 1] >> ((i & 1) * 16)));
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h2));
          x[2 * i] = f.x * sc;
          x[2 * i + 1] = f.y * sc;
        }
      }
    } else {
      const float* sf = static_cast<const float*>(scales);
      float sc;
      if (mode == FA_MODE_INT8_PER_HEAD || mode == FA_MODE_FP8_PER_HEAD) sc = __ldg(sf + h);
      else if (mode == FA_MODE_FP8_BLOCK) sc = __ldg(sf + ((long long)b * H + h) * ((S + blk - 1) / blk) + t / blk);
      else sc = __ldg(sf + bht);  // per token
      const uint2 w = *reinterpret_cast<const uint2*>(codes + r * D + c0);
      const uint32_t ww[2] = {w.x, w.y};
      const bool s8 = mode == FA_MODE_INT8_PER_HEAD || mode == FA_MODE_INT8_PER_TOKEN;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t pr = ww[i >> 1] >> ((i & 1) * 16);
        if (s8) {
          x[2 * i] = (float)(int8_t)(pr & 0xFFu) * sc;
          x[2 * i + 1] = (float)(int8_t)((pr >> 8) & 0xFFu) * sc;
        } else {
          const uint32_t h2 = e4m3x2_to_h2((uint16_t)pr);
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h2));
          x[2 * i] = f.x * sc;
          x[2 * i + 1] = f.y * sc;
        }
      }
    }
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 y = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
      o[i] = *reinterpret_cast<const uint32_t*>(&y);
    }
    *reinterpret_cast<uint4*>(out + r * D + c0) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

cudaError_t launch_deq_bf16(const fa_qtensor* t, __nv_bfloat16* out, cudaStream_t s) {
  const long long n = (long long)t->B * t->H * t->S * (t->D / 8);
  if (n == 0) return cudaSuccess;
  long long grid = (n + 255) / 256;
  const long long cap = 8LL * sm_count();
  if (grid > cap) grid = cap;
  deq_bf16_kernel<<<(unsigned)grid, 256, 0, s>>>(static_cast<const uint8_t*>(t->codes), t->scales, (int)t->mode, t->B,
                                                 t->H, t->S, t->D, (int)t->layout, t->block_tokens, out);
  return cudaGetLastError();
}

template <int D>
cudaError_t vprep_mixed(const AttnArgs& a, const P2& prm, const Prefill2Ws& w, cudaStream_t s) {
  const dim3 pgrid((unsigned)prm.ntiles_k, (unsigned)(a.v->B * a.v->H));
  if (pgrid.y > 65535u) return cudaErrorInvalidValue;
  const uint8_t* vc = static_cast<const uint8_t*>(a.v->codes);
#define FAQ_VPREP_MIXED(KIND_, D_)                                                                                   \
  vprep_kernel<KIND_, D_, true, true><<<pgrid, 256, 0, s>>>(vc, prm.vs, prm.v_blk, prm.v_nblk, a.v->H, a.v->S,        \
                                                         a.v->layout, w.vh, w.fvr, prm.ntiles_k, nullptr, 0, 1, w.ksp, \
                                                         prm.ve8, nullptr)
  switch (a.v->mode) {
    case FA_MODE_FLOAT: FAQ_VPREP_MIXED(K_BF16, D); break;
    case FA_MODE_FP8_PER_TOKEN:
    case FA_MODE_FP8_BLOCK:
    case FA_MODE_FP8_PER_HEAD: FAQ_VPREP_MIXED(K_E4M3, D); break;
    case FA_MODE_INT8_PER_HEAD:
    case FA_MODE_INT8_PER_TOKEN: FAQ_VPREP_MIXED(K_S8, D); break;
    case FA_MODE_MXFP4_PER_BLOCK:
      if constexpr (D == 128) { FAQ_VPREP_MIXED(K_MXF4, 128); break; }
      return cudaErrorNotSupported;
    case FA_MODE_MXFP8_PER_BLOCK:
      if constexpr (D == 128) { FAQ_VPREP_MIXED(K_MXF8, 128); break; }
      return cudaErrorNotSupported;
    default: return cudaErrorNotSupported;
  }
#undef FAQ_VPREP_MIXED
  return cudaGetLastError();
}

template <int KIND, int D, int SC>
cudaError_t launch_prefill(const AttnArgs& a, const P2& prm, const Prefill2Ws& w, cudaStream_t s) {
  return launch_pair<KIND, D, SC>(a, prm, w, s);
}

template <int KIND, int D>
cudaError_t launch2_sc(const AttnArgs& a, const P2& prm, const Prefill2Ws& w, int sc, cudaStream_t s) {
  switch (sc) {
    case SC_HEAD: return launch_prefill<KIND, D, SC_HEAD>(a, prm, w, s);
    case SC_COL: return launch_prefill<KIND, D, SC_COL>(a, prm, w, s);
    default: return launch_prefill<KIND, D, SC_TILE>(a, prm, w, s);
  }
}

// Rows with no key (Sk == 0): output 0, LSE -inf.
__global__ void fill_empty_kernel(__nv_bfloat16* out, float* lse, long long rows, int D) {
  const long long n = rows * D;
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) out[i] = __float2bfloat16(0.0f);
  if (lse)
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < rows; i += stride) lse[i] = -INFINITY;
}

void scale_desc2(const fa_qtensor* t, int& blk, int& nblk) {
  switch (t->mode) {
    case FA_MODE_INT8_PER_HEAD: blk = 0; nblk = 1; break;
    case FA_MODE_FP8_PER_TOKEN:
    case FA_MODE_INT8_PER_TOKEN: blk = 1; nblk = t->S; break;
    case FA_MODE_FP8_BLOCK: blk = t->block_tokens; nblk = (t->S + t->block_tokens - 1) / t->block_tokens; break;
    default: blk = 0; nblk = 1; break;
  }
}

}  // namespace

// Keys per tile of the prefill kernel for Q's mode: 112 for the MX modes, 128 otherwise.
int prefill_tile_keys(int q_mode) {
  const bool mx = q_mode == FA_MODE_MXFP4_PER_BLOCK || q_mode == FA_MODE_MXFP8_PER_BLOCK;
  return mx ? LP<K_MXF4, 128>::TN : BN;
}

// Prefill attention for E4M3, INT8 and MXFP4 operands.
size_t prefill2_workspace_bytes(int B, int Hkv, int Sk, int D, int tile_keys) {
  const size_t ntiles = ((size_t)Sk + tile_keys - 1) / tile_keys;
  return align256((size_t)B * Hkv * Sk * D * 2) + align256((size_t)B * Hkv * ntiles * 16) +
         align256((size_t)B * Hkv * ntiles * BN * 4);
}

cudaError_t launch_attention_prefill2(const AttnArgs& a, void* ws, cudaStream_t s) {
  if (const cudaError_t be = bounds_attach(); be != cudaSuccess) return be;
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
  const int tn = prefill_tile_keys(q->mode);
  prm.ntiles_k = (k->S + tn - 1) / tn;
  const Prefill2Ws w = carve_ws(ws, k->B, k->H, k->S, q->D, tn);
  prm.fvr = w.fvr;
  prm.ksp = w.ksp;
  int sc = SC_HEAD;
  if (q->mode == FA_MODE_FP8_PER_TOKEN) sc = SC_COL;
  if (q->mode == FA_MODE_FP8_BLOCK) sc = (k->block_tokens % BN == 0) ? SC_TILE : SC_COL;
  switch (q->mode) {
    case FA_MODE_FP8_PER_TOKEN:
    case FA_MODE_FP8_BLOCK:
      return q->D == 128 ? launch2_sc<K_E4M3, 128>(a, prm, w, sc, s) : launch2_sc<K_E4M3, 64>(a, prm, w, sc, s);
    case FA_MODE_INT8_PER_HEAD:
      return q->D == 128 ? launch_prefill<K_S8, 128, SC_HEAD>(a, prm, w, s) : launch_prefill<K_S8, 64, SC_HEAD>(a, prm, w, s);
    case FA_MODE_FP8_PER_HEAD:
      return q->D == 128 ? launch_prefill<K_E4M3, 128, SC_HEAD>(a, prm, w, s)
                         : launch_prefill<K_E4M3, 64, SC_HEAD>(a, prm, w, s);
    case FA_MODE_INT8_PER_TOKEN:
      return q->D == 128 ? launch_prefill<K_S8, 128, SC_COL>(a, prm, w, s) : launch_prefill<K_S8, 64, SC_COL>(a, prm, w, s);
    case FA_MODE_MXFP4_PER_BLOCK:
    case FA_MODE_MXFP8_PER_BLOCK:
      if (q->D != 128) return cudaErrorNotSupported;
      prm.qe8 = static_cast<const uint8_t*>(q->scales);
      prm.ke8 = static_cast<const uint8_t*>(k->scales);
      prm.ve8 = static_cast<const uint8_t*>(a.v->scales);
      return q->mode == FA_MODE_MXFP4_PER_BLOCK ? launch_pair<K_MXF4, 128, SC_HEAD>(a, prm, w, s)
                                                 : launch_pair<K_MXF8, 128, SC_HEAD>(a, prm, w, s);
    default:
      return cudaErrorNotSupported;
  }
}

// Mixed branches: Q and K as bf16 (dequantized into the workspace, or used as they are when not
// quantized), V' from V's own mode, then the bf16 pair kernel with every scale already applied.
size_t mixed_workspace_bytes(const fa_qtensor* q, const fa_qtensor* k) {
  size_t n = prefill2_workspace_bytes(k->B, k->H, k->S, q->D);
  if (q->mode != FA_MODE_FLOAT) n += align256((size_t)q->B * q->H * q->S * q->D * 2);
  if (k->mode != FA_MODE_FLOAT) n += align256((size_t)k->B * k->H * k->S * k->D * 2);
  return n;
}

cudaError_t launch_attention_mixed(const AttnArgs& a, void* ws, cudaStream_t s) {
  if (const cudaError_t be = bounds_attach(); be != cudaSuccess) return be;
  const fa_qtensor* q = a.q;
  const fa_qtensor* k = a.k;
  const int D = q->D;
  if ((a.v->mode == FA_MODE_MXFP4_PER_BLOCK || a.v->mode == FA_MODE_MXFP8_PER_BLOCK) && D != 128)
    return cudaErrorNotSupported;
  P2 prm = {};
  prm.B = q->B; prm.Hq = q->H; prm.Hkv = k->H; prm.Sq = q->S; prm.Sk = k->S; prm.group = q->H / k->H;
  prm.causal = a.causal; prm.layout = q->layout;
  const float scale = a.softmax_scale > 0.0f ? a.softmax_scale : 1.0f / sqrtf((float)D);
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.q_blk = -1;  // Q arrives with its scales applied
  prm.q_nblk = 1;
  prm.vs = static_cast<const float*>(a.v->scales);
  scale_desc2(a.v, prm.v_blk, prm.v_nblk);
  if (a.v->mode == FA_MODE_MXFP4_PER_BLOCK || a.v->mode == FA_MODE_MXFP8_PER_BLOCK)
    prm.ve8 = static_cast<const uint8_t*>(a.v->scales);
  prm.out = static_cast<__nv_bfloat16*>(a.out);
  prm.lse = a.lse;
  prm.status = a.status;
  prm.n_qtiles = (q->S + BM - 1) / BM;
  prm.ntiles_k = (k->S + BN - 1) / BN;
  const Prefill2Ws w = carve_ws(ws, k->B, k->H, k->S, D);
  prm.fvr = w.fvr;
  prm.ksp = w.ksp;
  uint8_t* extra = static_cast<uint8_t*>(ws) + prefill2_workspace_bytes(k->B, k->H, k->S, D);
  const void* qb = q->codes;
  const void* kb = k->codes;
  cudaError_t e;
  if (q->mode != FA_MODE_FLOAT) {
    if ((e = launch_deq_bf16(q, reinterpret_cast<__nv_bfloat16*>(extra), s)) != cudaSuccess) return e;
    qb = extra;
    extra += align256((size_t)q->B * q->H * q->S * D * 2);
  }
  if (k->mode != FA_MODE_FLOAT) {
    if ((e = launch_deq_bf16(k, reinterpret_cast<__nv_bfloat16*>(extra), s)) != cudaSuccess) return e;
    kb = extra;
  }
  CUtensorMap mq, mk, mv;
  const int rb = 2 * D, ab = rb > 128 ? 128 : rb;
  if ((e = make_code_map(&mq, qb, q->B, q->H, q->S, rb, q->layout, BM, ab)) != cudaSuccess) return e;
  if ((e = make_code_map(&mk, kb, k->B, k->H, k->S, rb, k->layout, BN, ab)) != cudaSuccess) return e;
  if ((e = make_vh_map(&mv, w.vh, a.v->B, a.v->H, a.v->S, D, BN)) != cudaSuccess) return e;
  if (D == 128) {
    if ((e = vprep_mixed<128>(a, prm, w, s)) != cudaSuccess) return e;
    return run_pair<K_BF16, 128, SC_TILE>(mq, mk, mv, prm, s);
  }
  if ((e = vprep_mixed<64>(a, prm, w, s)) != cudaSuccess) return e;
  return run_pair<K_BF16, 64, SC_TILE>(mq, mk, mv, prm, s);
}

cudaError_t launch_fill_empty_rows(void* out, float* lse, long long rows, int D, cudaStream_t s) {
  if (const cudaError_t be = bounds_attach(); be != cudaSuccess) return be;
  const long long n = rows * D;
  int grid = (int)((n + 255) / 256);
  if (grid > 4096) grid = 4096;
  if (grid < 1) grid = 1;
  fill_empty_kernel<<<grid, 256, 0, s>>>(static_cast<__nv_bfloat16*>(out), lse, rows, D);
  return cudaGetLastError();
}

}  // namespace faq
