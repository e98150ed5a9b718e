// decode.cu -- split-KV attention for single-token decode on INT8 per-head
// operands, plus the log-sum-exp combine of the splits.
//
// Decode reads every cached K/V code once, so it is bound by HBM bandwidth
// (msModelSlim wiki "量化模式", 模式索引 note: decode is memory-bound; wiki
// "FA 量化", 概述: K/V quantization serves long-context decode).  One CTA
// streams one contiguous chunk of keys of one (batch, kv head) and serves
// all G = Hq / Hkv query heads that read it (GQA), so each code is read once:
//   S^T [128 keys x 16] = K_tile [128 x D] . Q^T      tcgen05 kind::i8, M = 128
//                                                     keys, N = 16 (G heads,
//                                                     zero-padded)
//   softmax per key thread: per-tile head max reduced across the 4 warps,
//   p = exp2(s - m), P = rne(255 p) as u8, running sum L of the quantized P
//   O^T [D x 16] = V_tile^T . P^T                     kind::i8, A = V codes
//                                                     (MN-major), B = P (u8)
//   fold: O_acc = O_acc * 2^(m_prev - m) + O^T (fp32, one thread per dim)
// Each split writes (O_acc, m, L) and takes a ticket; the last CTA of a (b, kv head) merges
// the splits in the same launch:
//   m* = max_c m_c,  O = s_v * sum_c 2^(m_c - m*) O_c / sum_c 2^(m_c - m*) L_c.
#include <cuda_bf16.h>
#include <math.h>

#include <atomic>

#include "internal.cuh"
#include "sm100.cuh"

namespace faq {
namespace {

constexpr int DBN = 128;      // keys per tile
constexpr int DNS = 3;        // K/V stages
constexpr int DTHREADS = 256;
constexpr int DN = 16;        // MMA N (query heads, padded)

struct DecParams {
  int B, Hq, Hkv, Sk, group, layout, splits, chunk;  // chunk: keys per split (multiple of DBN)
  float scale_log2;
  const int8_t* q;
  const float* qs;
  const float* ks;
  const float* vs;
  float* opart;  // [B*Hq][splits][D]
  float* ml;     // [B*Hq][splits][2]  (m in log2 units, L)
  unsigned long long* tickets;  // [B*Hkv] (epoch << 32 | CTAs done), reset to 0 by the last CTA
  unsigned int epoch;           // nonzero, new for every call
  __nv_bfloat16* out;           // [B*Hq][D] (Sq = 1: BNSD and BSND coincide)
  float* lse;                   // nullable [B*Hq]
  int* status;
  // Fused cache append: Q quantized from bf16 in every CTA, and the new token's K / V rows quantized
  // into the cache at position pos by the CTA whose chunk holds it (before its TMA reads).
  int append;
  const __nv_bfloat16* qf;    // [B, Hq, D] bf16 (S = 1 in either layout)
  const __nv_bfloat16* knew;  // [B, Hkv, D] bf16
  const __nv_bfloat16* vnew;
  const float* amax_q;        // per-head calibration maxima: s = amax / 127
  const float* amax_k;
  const float* amax_v;
  int8_t* kc;                 // cache codes, capacity cap tokens
  int8_t* vc;
  float* ks_out;              // cache scales [Hkv]
  float* vs_out;
  int cap, pos;
};

template <int D>
struct DSmem {
  static constexpr uint32_t Q = 0;                  // [16][D] int8, swizzled
  static constexpr uint32_t K = 2048;               // stages of [128][D]
  static constexpr uint32_t V = K + DNS * DBN * D;
  static constexpr uint32_t P = V + DNS * DBN * D;  // 2 x [16][128] u8 (K-major)
  static constexpr uint32_t RED = P + 2 * 2048;     // [2][4 warps][16] floats (tile maxima)
  static constexpr uint32_t LRED = RED + 2 * 4 * 16 * 4;  // [4 warps][16] floats (sums)
  static constexpr uint32_t FLAG = LRED + 4 * 16 * 4;     // the combine's "last CTA" flag
  static constexpr uint32_t BAR = FLAG + 16;
  static constexpr uint32_t TOTAL = BAR + 512;
  static constexpr uint32_t ALLOC = TOTAL + 1024;
};

enum {
  D_Q = 0,
  D_KFULL = 1,    // [3]
  D_KEMPTY = 4,   // [3]
  D_VFULL = 7,    // [3]
  D_VEMPTY = 10,  // [3]
  D_SFULL = 13,   // [2]
  D_SEMPTY = 15,  // [2]
  D_PFULL = 17,   // [2]
  D_ODONE = 19,   // [2]
  D_OEMPTY = 21,  // [2]
  D_RED = 23,     // [2]
  D_FINAL = 25,
  D_LRED = 26,
  D_COUNT = 27
};

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// x / s rounded as IEEE division, then round-half-to-even to an integer, saturated to int8.
__device__ __forceinline__ uint32_t s8_code(float x, float s) {
  if (!(s > 0.0f)) return 0u;
  const int i = max(-128, min(127, __float2int_rn(__fdiv_rn(x, s))));
  return (uint32_t)(i & 0xFF);
}
__device__ __forceinline__ uint32_t s8_codes4(uint2 bf4, float s) {
  const float x0 = __uint_as_float(bf4.x << 16), x1 = __uint_as_float(bf4.x & 0xFFFF0000u);
  const float x2 = __uint_as_float(bf4.y << 16), x3 = __uint_as_float(bf4.y & 0xFFFF0000u);
  return s8_code(x0, s) | (s8_code(x1, s) << 8) | (s8_code(x2, s) << 16) | (s8_code(x3, s) << 24);
}

__device__ __forceinline__ bool wwait(uint64_t* b, uint32_t parity, volatile int* abort_flag, int* status, int where) {
  const bool ok = mbar_wait(b, parity, abort_flag, status, where);
  return __all_sync(0xffffffffu, ok);
}

template <int D, int G>
__global__ void __launch_bounds__(DTHREADS, 2)
    decode_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv, const DecParams p) {
  using L = DSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L::BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + D_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar + D_COUNT + 1);
  float* red = reinterpret_cast<float*>(smem + L::RED);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.y;
  const int bhk = blockIdx.x;
  const int b = bhk / p.Hkv, hk = bhk % p.Hkv;
  const int key0 = split * p.chunk;
  const int key1 = min(p.Sk, key0 + p.chunk);
  const int n_tiles = key1 > key0 ? (key1 - key0 + DBN - 1) / DBN : 0;

  if (tid == 0) {
    mbar_init(&bar[D_Q], 128);
    for (int i = 0; i < DNS; ++i) {
      mbar_init(&bar[D_KFULL + i], 1);
      mbar_init(&bar[D_KEMPTY + i], 1);
      mbar_init(&bar[D_VFULL + i], 1);
      mbar_init(&bar[D_VEMPTY + i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar[D_SFULL + i], 1);
      mbar_init(&bar[D_SEMPTY + i], 4);
      mbar_init(&bar[D_PFULL + i], 4);
      mbar_init(&bar[D_ODONE + i], 1);
      mbar_init(&bar[D_OEMPTY + i], 4);
      mbar_init(&bar[D_RED + i], 128);
    }
    mbar_init(&bar[D_FINAL], 1);
    mbar_init(&bar[D_LRED], 128);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 64);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const uint32_t tS[2] = {tbase, tbase + 16};
  const uint32_t tOT[2] = {tbase + 32, tbase + 48};

  if (warp == 0) {
    if (p.append && key0 <= p.pos && p.pos < key1) {
      // the new token's K / V rows into the cache (lane l: elements 4l .. 4l + 3), visible to the
      // TMA reads below through the async-proxy fence
      static_assert(D == 128, "decode: head_dim 128");
      const float sk = __fdiv_rn(__ldg(p.amax_k + hk), 127.0f), sv = __fdiv_rn(__ldg(p.amax_v + hk), 127.0f);
      const long long src = ((long long)b * p.Hkv + hk) * D;
      const long long dst = p.layout == FA_LAYOUT_BNSD ? (((long long)b * p.Hkv + hk) * p.cap + p.pos) * D
                                                       : (((long long)b * p.cap + p.pos) * p.Hkv + hk) * D;
      reinterpret_cast<uint32_t*>(p.kc + dst)[lane] = s8_codes4(__ldg(reinterpret_cast<const uint2*>(p.knew + src) + lane), sk);
      reinterpret_cast<uint32_t*>(p.vc + dst)[lane] = s8_codes4(__ldg(reinterpret_cast<const uint2*>(p.vnew + src) + lane), sv);
      asm volatile("fence.proxy.async.global;" ::: "memory");
    }
    if (p.append && split == 0 && b == 0 && lane == 0) {
      p.ks_out[hk] = __fdiv_rn(__ldg(p.amax_k + hk), 127.0f);
      p.vs_out[hk] = __fdiv_rn(__ldg(p.amax_v + hk), 127.0f);
    }
    __syncwarp();
    if (lane == 0 && n_tiles > 0) {
      tma_prefetch_desc(&tmk);
      tma_prefetch_desc(&tmv);
      const bool bnsd = p.layout == FA_LAYOUT_BNSD;
      int j = 0;
      int nk = 0;  // K tiles whose loads were issued (one more than V's when the loop stops between them)
      for (; j < n_tiles; ++j) {
        const int s = j % DNS;
        const int k0 = key0 + j * DBN;
        if (j >= DNS && !mbar_wait(&bar[D_KEMPTY + s], ((j / DNS) - 1) & 1, abort_flag, p.status, 21)) break;
        mbar_arrive_expect_tx(&bar[D_KFULL + s], DBN * D);
        tma_load_4d(smem + L::K + s * DBN * D, &tmk, &bar[D_KFULL + s], 0, bnsd ? k0 : hk, bnsd ? hk : k0, b);
        nk = j + 1;
        if (j >= DNS && !mbar_wait(&bar[D_VEMPTY + s], ((j / DNS) - 1) & 1, abort_flag, p.status, 22)) break;
        mbar_arrive_expect_tx(&bar[D_VFULL + s], DBN * D);
        tma_load_4d(smem + L::V + s * DBN * D, &tmv, &bar[D_VFULL + s], 0, bnsd ? k0 : hk, bnsd ? hk : k0, b);
      }
      if (*abort_flag) {
        // let this CTA's issued loads land before it can leave
        for (int t = max(0, nk - DNS); t < nk; ++t) mbar_drain(&bar[D_KFULL + t % DNS], (t / DNS) & 1);
        for (int t = max(0, j - DNS); t < j; ++t) mbar_drain(&bar[D_VFULL + t % DNS], (t / DNS) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && n_tiles > 0) {
      constexpr uint32_t SW = D == 128 ? kSwz128 : kSwz64;
      constexpr uint32_t SBO8 = D == 128 ? 1024 : 512;
      constexpr uint32_t ROWB = D;  // bytes per key row
      constexpr uint32_t idesc_qk = make_idesc(kAccS32, kFmtS8, kFmtS8, 0, 0, DN, 128);
      constexpr uint32_t idesc_pv = make_idesc(kAccS32, kFmtS8, kFmtU8, 1, 0, DN, D);
      const uint32_t sQ = smem_u32(smem + L::Q);
      bool ok = mbar_wait(&bar[D_Q], 0, abort_flag, p.status, 23);
      for (int j = 0; ok && j <= n_tiles; ++j) {
        if (j < n_tiles) {
          const int s = j % DNS, bb = j & 1;
          if (!mbar_wait(&bar[D_KFULL + s], (j / DNS) & 1, abort_flag, p.status, 24)) break;
          if (j >= 2 && !mbar_wait(&bar[D_SEMPTY + bb], ((j >> 1) - 1) & 1, abort_flag, p.status, 25)) break;
          tc_fence_after();
          const uint32_t sK = smem_u32(smem + L::K + s * DBN * D);
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk)
            mma_i8(tS[bb], make_sdesc(sK + kk * 32, 16, SBO8, SW), make_sdesc(sQ + kk * 32, 16, SBO8, SW),
                   idesc_qk, kk > 0);
          mma_commit(&bar[D_KEMPTY + s]);
          mma_commit(&bar[D_SFULL + bb]);
        }
        if (j >= 1) {
          const int jj = j - 1, s = jj % DNS, bb = jj & 1;
          if (!mbar_wait(&bar[D_PFULL + bb], (jj >> 1) & 1, abort_flag, p.status, 26)) break;
          if (!mbar_wait(&bar[D_VFULL + s], (jj / DNS) & 1, abort_flag, p.status, 27)) break;
          if (jj >= 2 && !mbar_wait(&bar[D_OEMPTY + bb], ((jj >> 1) - 1) & 1, abort_flag, p.status, 28)) break;
          tc_fence_after();
          const uint32_t sV = smem_u32(smem + L::V + s * DBN * D);
          const uint32_t sP = smem_u32(smem + L::P + bb * 2048);
#pragma unroll
          for (int kk = 0; kk < DBN / 32; ++kk)
            mma_i8(tOT[bb], make_sdesc(sV + kk * 32 * ROWB, 16384, SBO8, SW), make_sdesc(sP + kk * 32, 16, 1024, kSwz128),
                   idesc_pv, kk > 0);
          mma_commit(&bar[D_VEMPTY + s]);
          mma_commit(&bar[D_ODONE + bb]);
        }
      }
      mma_commit(&bar[D_FINAL]);
      mbar_drain(&bar[D_FINAL], 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    const int i = tid - 128;  // key row of S^T, dim row of O^T
    const int wg = warp - 4;
    const uint32_t loff = (uint32_t)(wg * 32) << 16;
    const int hq0 = hk * G;

    // Q rows (G heads, zero-padded to 16) into the K-major swizzled B operand.
    {
      const int r = i >> 3, c = i & 7;  // 16 rows x 8 chunks of 16 bytes (D = 128)
      if (c < D / 16) {
        uint4 v = make_uint4(0, 0, 0, 0);
        if (r < G) {
          const long long qrow = (long long)b * p.Hq + hq0 + r;  // S = 1: the same row in either layout
          if (p.append) {
            // quantize the new query row here: 16 codes from 16 bf16 values
            const float sq = __fdiv_rn(__ldg(p.amax_q + hq0 + r), 127.0f);
            const uint2* src = reinterpret_cast<const uint2*>(p.qf + qrow * D + c * 16);
            v = make_uint4(s8_codes4(__ldg(src), sq), s8_codes4(__ldg(src + 1), sq), s8_codes4(__ldg(src + 2), sq),
                           s8_codes4(__ldg(src + 3), sq));
          } else {
            v = __ldg(reinterpret_cast<const uint4*>(p.q + qrow * D) + c);
          }
        }
        const uint32_t off = D == 128 ? swz128_offset(r, c) : swz64_offset(r, c);
        *reinterpret_cast<uint4*>(smem + L::Q + off) = v;
      }
      if (i < 16 * 8) {
        // zero the unused head rows of both P^T buffers once
        const int pr = i >> 3, pc = i & 7;
        if (pr >= G) {
          *reinterpret_cast<uint4*>(smem + L::P + swz128_offset(pr, pc)) = make_uint4(0, 0, 0, 0);
          *reinterpret_cast<uint4*>(smem + L::P + 2048 + swz128_offset(pr, pc)) = make_uint4(0, 0, 0, 0);
        }
      }
      fence_async_smem();
      mbar_arrive(&bar[D_Q]);
    }

    float ch[G], m_run[G], alpha_prev[G], Lp[G], Oacc[G];
    const float skv = p.append ? __fdiv_rn(__ldg(p.amax_k + hk), 127.0f) : __ldg(p.ks + hk);
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float sqh = p.append ? __fdiv_rn(__ldg(p.amax_q + hq0 + h), 127.0f) : __ldg(p.qs + hq0 + h);
      ch[h] = sqh * skv * p.scale_log2;
      m_run[h] = -INFINITY;
      alpha_prev[h] = 1.0f;
      Lp[h] = 0.0f;
      Oacc[h] = 0.0f;
    }
    bool ok = true;
    for (int j = 0; j < n_tiles && ok; ++j) {
      const int bb = j & 1;
      const int key = key0 + j * DBN + i;
      if (!wwait(&bar[D_SFULL + bb], (j >> 1) & 1, abort_flag, p.status, 29)) { ok = false; break; }
      tc_fence_after();
      uint32_t r[16];
      tmem_ld16(tS[bb] + loff, r);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[D_SEMPTY + bb]);
      float sc[G];
      const bool valid = key < key1;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        sc[h] = valid ? (float)(int)r[h] * ch[h] : -INFINITY;
        float m = sc[h];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        if (lane == 0) red[(bb * 4 + wg) * 16 + h] = m;
      }
      mbar_arrive(&bar[D_RED + bb]);
      if (!wwait(&bar[D_RED + bb], (j >> 1) & 1, abort_flag, p.status, 30)) { ok = false; break; }
      float alpha[G];
      uint32_t p8[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float mt = fmaxf(fmaxf(red[(bb * 4 + 0) * 16 + h], red[(bb * 4 + 1) * 16 + h]),
                               fmaxf(red[(bb * 4 + 2) * 16 + h], red[(bb * 4 + 3) * 16 + h]));
        const float m_new = fmaxf(m_run[h], mt);
        alpha[h] = m_new == -INFINITY ? 1.0f : ex2f(m_run[h] - m_new);
        const float base = m_new == -INFINITY ? 0.0f : m_new;
        const float pv = ex2f(sc[h] - base);
        p8[h] = (uint32_t)__float2int_rn(fminf(pv * 255.0f, 255.0f));
        Lp[h] = Lp[h] * alpha[h] + (float)p8[h];
        m_run[h] = m_new;
      }
      // P^T buffer bb is free once P V of tile j-2 has completed.
      if (j >= 2 && !wwait(&bar[D_ODONE + bb], ((j >> 1) - 1) & 1, abort_flag, p.status, 31)) { ok = false; break; }
      uint8_t* sP = smem + L::P + bb * 2048;
#pragma unroll
      for (int h = 0; h < G; ++h) sP[h * 128 + ((((i >> 4) ^ (h & 7))) << 4) + (i & 15)] = (uint8_t)p8[h];
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[D_PFULL + bb]);
      // Fold O^T of tile j-1.
      if (j >= 1) {
        const int jb = (j - 1) & 1;
        if (!wwait(&bar[D_ODONE + jb], ((j - 1) >> 1) & 1, abort_flag, p.status, 32)) { ok = false; break; }
        tc_fence_after();
        uint32_t o[16];
        tmem_ld16(tOT[jb] + loff, o);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[D_OEMPTY + jb]);
#pragma unroll
        for (int h = 0; h < G; ++h) Oacc[h] = Oacc[h] * alpha_prev[h] + (float)(int)o[h];
      }
#pragma unroll
      for (int h = 0; h < G; ++h) alpha_prev[h] = alpha[h];
    }
    if (ok && n_tiles > 0) {
      const int jl = n_tiles - 1, jb = jl & 1;
      ok = wwait(&bar[D_ODONE + jb], (jl >> 1) & 1, abort_flag, p.status, 33);
      if (ok) {
        tc_fence_after();
        uint32_t o[16];
        tmem_ld16(tOT[jb] + loff, o);
        tmem_ld_wait();
#pragma unroll
        for (int h = 0; h < G; ++h) Oacc[h] = Oacc[h] * alpha_prev[h] + (float)(int)o[h];
      }
    }
    // L: sum of the per-key partial sums over the 128 threads.
    float* lred = reinterpret_cast<float*>(smem + L::LRED);  // [4 warps][16]
    __syncwarp();
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float v = Lp[h];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
      if (lane == 0) lred[wg * 16 + h] = v;
    }
    mbar_arrive(&bar[D_LRED]);
    wwait(&bar[D_LRED], 0, abort_flag, p.status, 34);
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const long long row = ((long long)b * p.Hq + hq0 + h) * p.splits + split;
      if (!in_bounds(row >= 0 && row < (long long)p.B * p.Hq * p.splits, 131)) continue;
      if (i < D) p.opart[row * D + i] = ok ? Oacc[h] : 0.0f;
      if (i == 0) {
        const float Lt = lred[h] + lred[16 + h] + lred[32 + h] + lred[48 + h];
        p.ml[row * 2 + 0] = (ok && n_tiles > 0) ? m_run[h] : -INFINITY;
        p.ml[row * 2 + 1] = ok ? Lt : 0.0f;
      }
    }
    // ---- LSE combine, fused: the last CTA of this (b, kv head) to finish merges the splits.
    // Every CTA fences its partials and takes a ticket; the CTA that takes the last one reads
    // all of them (no CTA ever waits for another).  A ticket word holds this call's epoch in its
    // high half, so whatever the workspace held before the first call counts as empty; the
    // last CTA resets it to 0.
    __threadfence();
    asm volatile("bar.sync 1, 128;" ::: "memory");  // the four softmax warps
    volatile int* last_flag = reinterpret_cast<volatile int*>(smem + L::FLAG);
    if (i == 0) {
      unsigned long long* tk = p.tickets + bhk;
      unsigned long long old = atomicAdd(tk, 0ull);
      int last = 0;
      for (int it = 0; it < (1 << 20); ++it) {
        const unsigned long long nw =
            (unsigned)(old >> 32) == p.epoch ? old + 1ull : (((unsigned long long)p.epoch << 32) | 1ull);
        const unsigned long long prev = atomicCAS(tk, old, nw);
        if (prev == old) {
          last = (int)(nw & 0xFFFFFFFFull) == p.splits;
          break;
        }
        old = prev;
        if (it == (1 << 20) - 1 && p.status) atomicCAS(p.status, 0, (35 << 8) | kStatusTimeout);
      }
      *last_flag = last;
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (*last_flag) {
      __threadfence();
      const float vsc = p.append ? __fdiv_rn(__ldg(p.amax_v + hk), 127.0f) : __ldg(p.vs + hk);
      for (int idx = i; idx < G * D; idx += 128) {
        const int h = idx / D, d = idx - h * D;
        const long long qrow = (long long)b * p.Hq + hq0 + h;
        if (!in_bounds(qrow >= 0 && qrow < (long long)p.B * p.Hq, 132)) continue;
        const float* mlr = p.ml + qrow * p.splits * 2;
        const float* opr = p.opart + qrow * p.splits * D + d;
        float m = -INFINITY;
        for (int c = 0; c < p.splits; ++c) m = fmaxf(m, __ldcg(mlr + 2 * c));
        float Ls = 0.0f, acc = 0.0f;
        for (int c = 0; c < p.splits; ++c) {
          const float mc = __ldcg(mlr + 2 * c);
          if (mc != -INFINITY) {
            const float wc = ex2f(mc - m);
            Ls += wc * __ldcg(mlr + 2 * c + 1);
            acc += wc * __ldcg(opr + (long long)c * D);
          }
        }
        p.out[qrow * D + d] = __float2bfloat16(Ls > 0.0f ? acc * (vsc / Ls) : 0.0f);
        if (d == 0 && p.lse) p.lse[qrow] = Ls > 0.0f ? (m + __log2f(Ls / 255.0f)) * 0.69314718055994530942f : -INFINITY;
      }
      if (i == 0) atomicExch(p.tickets + bhk, 0ull);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 64);
  }
}

// Tensor map over int8 codes of S visible tokens stored in a buffer of cap >= S tokens.
cudaError_t make_map(CUtensorMap* map, const void* base, int B, int H, int S, int D, int layout, int cap) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return cudaErrorNotSupported;
  cuuint64_t dims[4], strides[3];
  cuuint32_t box[4], es[4] = {1, 1, 1, 1};
  if (layout == FA_LAYOUT_BNSD) {
    dims[0] = D; dims[1] = S; dims[2] = H; dims[3] = B;
    strides[0] = (cuuint64_t)D; strides[1] = (cuuint64_t)cap * D; strides[2] = (cuuint64_t)H * cap * D;
    box[0] = D; box[1] = DBN; box[2] = 1; box[3] = 1;
  } else {
    dims[0] = D; dims[1] = H; dims[2] = S; dims[3] = B;
    strides[0] = (cuuint64_t)D; strides[1] = (cuuint64_t)H * D; strides[2] = (cuuint64_t)cap * H * D;
    box[0] = D; box[1] = 1; box[2] = DBN; box[3] = 1;
  }
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int D, int G>
cudaError_t launch_dec(const CUtensorMap& mk, const CUtensorMap& mv, const DecParams& prm, cudaStream_t s) {
  auto kern = decode_kernel<D, G>;
  cudaError_t e = set_smem_limit(reinterpret_cast<const void*>(kern), DSmem<D>::ALLOC);
  if (e != cudaSuccess) return e;
  // (b, kv head) on x (up to 2^31 - 1), the split on y (at most 256)
  if ((long long)prm.B * prm.Hkv > 0x7FFFFFFFLL || prm.splits > 65535) return cudaErrorNotSupported;
  dim3 grid((unsigned)(prm.B * prm.Hkv), (unsigned)prm.splits);
  kern<<<grid, DTHREADS, DSmem<D>::ALLOC, s>>>(mk, mv, prm);
  return cudaGetLastError();
}

int chunk_of(int Sk, int splits) {
  int c = (Sk + splits - 1) / splits;
  return ((c + DBN - 1) / DBN) * DBN;
}

}  // namespace

int decode_auto_splits(int B, int Hkv, int Sk) {
  // Enough CTAs for about four rounds of two resident CTAs per SM, with at
  // least four key tiles per CTA.
  const int slots = sm_count() * 2;
  const int units = B * Hkv;
  const int tiles = (Sk + DBN - 1) / DBN;
  int best = 1;
  double best_cost = 1e30;
  for (int sp = 1; sp <= 256 && sp <= tiles; ++sp) {
    const int tpc = (chunk_of(Sk, sp)) / DBN;  // tiles per CTA
    const long long ctas = (long long)units * sp;
    const long long rounds = (ctas + slots - 1) / slots;
    const double cost = (double)rounds * (tpc + 2.0);  // +2: per-CTA fill / drain
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best = sp;
    }
  }
  return best;
}

// Partials [B*Hq][splits][D] and [B*Hq][splits][2] fp32, then one 8-byte ticket per
// (b, kv head), B * Hq of them at most, 256-byte aligned.
size_t decode_workspace_bytes(int B, int Hq, int D, int splits) {
  const size_t parts = (size_t)B * Hq * splits * ((size_t)D + 2) * sizeof(float);
  return ((parts + 255) & ~size_t(255)) + (size_t)B * Hq * 8;
}

namespace {

// Decode kernel (one CTA per split and (b, kv head)) then the combine; kv_len visible tokens in
// K / V buffers of cap tokens.
cudaError_t run_decode(DecParams prm, const void* kcodes, const void* vcodes, int D, int kv_len, int cap, int out_layout,
                       void* out, float* lse, cudaStream_t s) {
  if (const cudaError_t be = bounds_attach(); be != cudaSuccess) return be;
  (void)out_layout;  // Sq = 1: row (b, hq) at (b * Hq + hq) * D in either layout
  const int G = prm.group;
  prm.Sk = kv_len;
  prm.chunk = chunk_of(kv_len, prm.splits);
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.lse = lse;
  // a fresh nonzero epoch per call for the combine tickets
  static std::atomic<unsigned int> epochs{0};
  unsigned int ep = epochs.fetch_add(1u) + 1u;
  if (ep == 0u) ep = epochs.fetch_add(1u) + 1u;
  prm.epoch = ep;
  CUtensorMap mk, mv;
  cudaError_t e;
  if ((e = make_map(&mk, kcodes, prm.B, prm.Hkv, kv_len, D, prm.layout, cap)) != cudaSuccess) return e;
  if ((e = make_map(&mv, vcodes, prm.B, prm.Hkv, kv_len, D, prm.layout, cap)) != cudaSuccess) return e;
  if (D == 128) {
    switch (G) {
      case 1: e = launch_dec<128, 1>(mk, mv, prm, s); break;
      case 2: e = launch_dec<128, 2>(mk, mv, prm, s); break;
      case 4: e = launch_dec<128, 4>(mk, mv, prm, s); break;
      case 8: e = launch_dec<128, 8>(mk, mv, prm, s); break;
      case 16: e = launch_dec<128, 16>(mk, mv, prm, s); break;
      default: return cudaErrorNotSupported;
    }
  } else {
    return cudaErrorNotSupported;
  }
  return e;
}

DecParams base_params(int B, int Hq, int Hkv, int D, int layout, int splits, float softmax_scale, void* ws,
                      int* status) {
  DecParams prm = {};
  prm.B = B; prm.Hq = Hq; prm.Hkv = Hkv; prm.group = Hq / Hkv; prm.layout = layout;
  prm.splits = splits;
  const float scale = softmax_scale > 0.0f ? softmax_scale : 1.0f / sqrtf((float)D);
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.opart = static_cast<float*>(ws);
  prm.ml = prm.opart + (size_t)B * Hq * splits * D;
  const size_t parts = (size_t)B * Hq * splits * ((size_t)D + 2) * sizeof(float);
  prm.tickets = reinterpret_cast<unsigned long long*>(static_cast<uint8_t*>(ws) + ((parts + 255) & ~size_t(255)));
  prm.status = status;
  return prm;
}

}  // namespace

cudaError_t launch_attention_decode(const AttnArgs& a, int splits, void* ws, cudaStream_t s) {
  const fa_qtensor* q = a.q;
  const fa_qtensor* k = a.k;
  DecParams prm = base_params(q->B, q->H, k->H, q->D, q->layout, splits, a.softmax_scale, ws, a.status);
  prm.q = static_cast<const int8_t*>(q->codes);
  prm.qs = static_cast<const float*>(q->scales);
  prm.ks = static_cast<const float*>(k->scales);
  prm.vs = static_cast<const float*>(a.v->scales);
  return run_decode(prm, k->codes, a.v->codes, q->D, k->S, k->S, q->layout, a.out, a.lse, s);
}

cudaError_t launch_decode_append(const DecodeAppendArgs& a, int splits, void* ws, cudaStream_t s) {
  DecParams prm = base_params(a.q->B, a.q->H, a.k_cache->H, a.q->D, a.q->layout, splits, a.softmax_scale, ws,
                              a.status);
  prm.append = 1;
  prm.qf = static_cast<const __nv_bfloat16*>(a.q->data);
  prm.knew = static_cast<const __nv_bfloat16*>(a.k_new->data);
  prm.vnew = static_cast<const __nv_bfloat16*>(a.v_new->data);
  prm.amax_q = a.amax_q; prm.amax_k = a.amax_k; prm.amax_v = a.amax_v;
  prm.kc = static_cast<int8_t*>(a.k_cache->codes);
  prm.vc = static_cast<int8_t*>(a.v_cache->codes);
  prm.ks_out = static_cast<float*>(a.k_cache->scales);
  prm.vs_out = static_cast<float*>(a.v_cache->scales);
  prm.vs = prm.vs_out;  // the combine reads the V scales the decode kernel has written
  prm.cap = a.k_cache->S;
  prm.pos = a.pos;
  return run_decode(prm, a.k_cache->codes, a.v_cache->codes, a.q->D, a.pos + 1, a.k_cache->S, a.q->layout, a.out,
                    a.lse, s);
}

}  // namespace faq
