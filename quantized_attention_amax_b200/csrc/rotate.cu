// rotate.cu -- fused rotate -> FP8 block quantization (MindIE SD "量化",
// FA量化 / 技术特点: 旋转 then 块量化).
//
// Q' = bf16(Q R_q), K' = bf16(K R_k) (fp32 accumulation, one rounding), V' = V;
// then one E4M3 scale = amax / 448 per (b, h, block of `blk` tokens) and
// codes e4m3(x' / scale).  A work item is a 256-token chunk of one
// (operand, batch, head); one persistent CTA per SM walks the items
// blockIdx.x, blockIdx.x + gridDim.x, ... in a three-role pipeline:
//   warp 16     TMA: each item as two 128-token bf16 tiles (128B-swizzled,
//               64-element K atoms) into one of two 64 KB input stages; the
//               items come in operand order (Q, K, V), so the one resident
//               rotation is loaded when the operand changes, after the MMAs
//               that read the previous one.  A rotation of the Hadamard-
//               times-signs form is written by this warp from its signs
//               instead, in the same swizzled layout.
//   warp 17     tcgen05.mma kind::f16 (bf16 x bf16 -> fp32): X R into one of
//               two 256-column TMEM buffers, R read as the MN-major B operand
//               exactly as stored ([D, D] row-major, x' = x R).  V items skip it.
//   warps 0-15  the epilogue of the previous item: warp e takes tile e / 8,
//               column half (e / 4) % 2 and TMEM lane quarter e % 4; its bf16
//               half row (rotated in TMEM, or V from the shared tile) stays in
//               registers for half-row maxima -> block maxima (lane
//               butterflies, then one exchange through shared memory) -> scale
//               -> E4M3 codes (division rounded as IEEE), staged in a swizzled
//               shared tile that one TMA store per 128-token tile writes out as
//               whole 128-byte rows (an optional bf16 copy of the rotated rows
//               goes out with plain stores).
// So the loads and MMAs of item k + 1 overlap the epilogue of item k.
// blk must divide 256.
#include <cuda_bf16.h>
#include <math.h>
#include <string.h>

#include "internal.cuh"
#include "quant_common.cuh"
#include "sm100.cuh"

namespace faq {
namespace {

constexpr int CH = 256;          // tokens per work item
constexpr int NCP = 2;                // column parts per row: a thread holds 128 / NCP values of a row
constexpr int CW = 128 / NCP;         // columns per thread
constexpr int REPI = 32 * 8 * NCP;    // epilogue threads: 2 tiles x 4 lane quarters x NCP parts
constexpr int RTHREADS = REPI + 64;   // + the TMA producer and the MMA issuer warps
constexpr int WPROD = REPI / 32, WMMA = WPROD + 1;

// n / d for 0 <= n < 2^31 as one widening multiply and a shift: l = ceil(log2 d),
// m = floor(2^(31 + l) / d) + 1 < 2^32; then n m / 2^(31 + l) = n / d + n (m - 2^(31 + l) / d) / 2^(31 + l)
// and the error term is below 2^-l <= 1 / d, so the floor is exact.
struct FastDiv {
  uint32_t d, m;
  int l;
};

inline FastDiv make_fastdiv(uint32_t d) {
  FastDiv f;
  f.d = d;
  f.l = 0;
  while ((1u << f.l) < d) ++f.l;
  f.m = (uint32_t)((1ull << (31 + f.l)) / d + 1);
  return f;
}

__device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv& f) {
  return (uint32_t)(((unsigned long long)n * f.m) >> (31 + f.l));
}

struct RotOp {
  void* codes;
  float* scales;
  __nv_bfloat16* dbg;
  int B, H, S, layout, blk, rotate;
  int had;               // rotation generated from the signs (Hadamard form) instead of loaded
  uint32_t sgn[4];       // its signs: bit j set, sigma_j = -1
  uint32_t cbits;        // bf16 bits of c = bf16(1 / sqrt(D))
  int lblk;              // log2(blk) (blk divides 256, so it is a power of two)
  long long first_item;  // first work item of this operand
  int chunks;            // 256-token chunks per (b, h)
  FastDiv fd_chunks, fd_h;
};

struct RotParams {
  RotOp op[3];
  int nops;
  long long items;
  int* status;
};

struct RSmem {
  static constexpr uint32_t X = 0;               // 2 stages x [2 tiles][2 K atoms][128 rows][128 B]
  static constexpr uint32_t R = 2 * 65536;       // the current rotation: [2 N atoms][128 d rows][128 B]
  static constexpr uint32_t C = R + 32768;       // E4M3 codes: [2 tiles][128 rows][128 B], 128B-swizzled
  static constexpr uint32_t RED = C + 32768;     // [2 items][epilogue warps][32 lanes] lane-group maxima
  static constexpr uint32_t GM = RED + 2 * REPI * 4;  // [2 items][8 row groups of 32][NCP parts] group maxima
  static constexpr uint32_t BAR = GM + 2 * 8 * NCP * 4;
  static constexpr uint32_t TOTAL = BAR + 256;
  static constexpr uint32_t ALLOC = TOTAL + 1024;
  static_assert(ALLOC <= 227 * 1024, "shared memory per CTA");
};

enum {
  RB_XF = 0,    // [2] input stage full (TMA)
  RB_XE = 2,    // [2] input stage free (every epilogue warp)
  RB_TF = 4,    // [2] TMEM buffer full (MMA commit)
  RB_TE = 6,    // [2] TMEM buffer free (every epilogue warp)
  RB_RF = 8,    // rotation loaded (TMA)
  RB_RE = 9,    // rotation free (MMA commit after its last use)
  RB_FIN = 10,  // every MMA complete
  RB_COUNT = 11
};

// Hardware named barriers among the epilogue warps (0 is __syncthreads).  Every epilogue warp
// reaches each of them once per item, whatever happened before (their mbarrier waits are bounded
// and a failed one only marks the warp), and the decision to stop is the barrier's own OR
// reduction, identical in every warp; so no warp can be left waiting at one.
enum {
  NB_MAX = 1,   // group maxima written (every epilogue thread)
  NB_CODE = 2   // [2] a tile's codes staged (its 8 warps)
};

__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  uint16_t lo, hi;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(b), "f"(a));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(d), "f"(c));
  return (uint32_t)lo | ((uint32_t)hi << 16);
}

// R = bf16(H_D diag(sigma) / sqrt(D)) for D = 128, written by the 32 lanes of one warp straight
// into the shared-memory layout the TMA copy of a stored R produces: [2 column atoms of 64][128
// rows d][128 B], 16-byte chunk q of row d at chunk q ^ (d & 7) (the 128-byte swizzle).  Entry
// (d, j) = +-c, negative when popcount(d & j) + [sigma_j = -1] is odd (the Sylvester Hadamard
// sign times sigma_j; rounding to bf16 commutes with the sign).
__device__ __forceinline__ void write_hadamard_rotation(uint8_t* dst, const uint32_t (&sgn)[4], uint32_t cbits,
                                                        int lane) {
  // a chunk holds j = j0 .. j0 + 7 with j0 a multiple of 8, so popcount(d & j) = popcount(d & j0) +
  // popcount(d & t) for t = j - j0: the chunk's eight sign bits are the parity of d & j0 (all
  // eight), the parities of (d & 7) & t (a pattern per d & 7), and the eight sigma bits
  const uint32_t c2 = cbits | (cbits << 16);
  for (int i = lane; i < 2 * 128 * 8; i += 32) {
    const int nb = i >> 10, d = (i >> 3) & 127, q = i & 7;
    const int j0 = nb * 64 + q * 8;
    uint32_t neg = (sgn[j0 >> 5] >> (j0 & 31)) & 0xFFu;
    if (__popc(d & j0) & 1) neg ^= 0xFFu;
    const int d7 = d & 7;
    // bit t: parity of popcount(d7 & t) (the rows of the 8 x 8 Sylvester matrix)
    const uint32_t pat = ((d7 & 1) ? 0xAAu : 0u) ^ ((d7 & 2) ? 0xCCu : 0u) ^ ((d7 & 4) ? 0xF0u : 0u);
    neg ^= pat;
    uint32_t w[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) w[t] = c2 | (((neg >> (2 * t)) & 1u) << 15) | (((neg >> (2 * t + 1)) & 1u) << 31);
    *reinterpret_cast<uint4*>(dst + nb * 16384 + d * 128 + ((q ^ d7) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// per half: max(|a|, |b|), its sign the XOR of the inputs' signs (exact; only magnitudes are used)
__device__ __forceinline__ uint32_t bf16x2_absmax(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// E4M3 codes of 16 bf16 values (packed pairs in a, b) divided by sc with IEEE division;
// zero codes when sc == 0.
__device__ __noinline__ uint4 codes_ieee(uint4 a, uint4 b, float sc) {
  const uint32_t p[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  uint32_t w[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const uint32_t p0 = p[2 * e], p1 = p[2 * e + 1];
    w[e] = sc > 0.0f ? e4m3x4(__fdiv_rn(__uint_as_float(p0 << 16), sc), __fdiv_rn(__uint_as_float(p0 & 0xFFFF0000u), sc),
                              __fdiv_rn(__uint_as_float(p1 << 16), sc), __fdiv_rn(__uint_as_float(p1 & 0xFFFF0000u), sc))
                     : 0u;
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, const void* src, int c0, int c1, int c2, int c3) {
  asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(map),
               "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// this thread's bulk stores have finished reading shared memory / have completed
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// bar.red.or over `count` threads at named barrier `id`: true in every thread when any
// participant passed true.
__device__ __forceinline__ bool named_barrier_or(int id, int count, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void named_barrier_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

struct RItem {
  int oi, b, h, t0, ntile;
};

__device__ __forceinline__ RItem decode_item(const RotParams& prm, long long g) {
  RItem it;
  it.oi = 0;
  if (prm.nops > 1 && g >= prm.op[1].first_item) it.oi = 1;
  if (prm.nops > 2 && g >= prm.op[2].first_item) it.oi = 2;
  const RotOp& op = prm.op[it.oi];
  const uint32_t local = (uint32_t)(g - op.first_item);  // < 2^31 (checked at launch)
  uint32_t chunk;
  if (op.layout == FA_LAYOUT_BNSD) {
    // (b, h, chunk): a chunk is one contiguous 64 KB stretch
    const uint32_t bh = fdiv(local, op.fd_chunks);
    chunk = local - bh * op.chunks;
    const uint32_t b = fdiv(bh, op.fd_h);
    it.h = (int)(bh - b * op.H);
    it.b = (int)b;
  } else {
    // (b, chunk, h): a token's heads are adjacent in memory, so neighbouring CTAs, taking
    // neighbouring heads of one token range, read and write whole DRAM pages between them
    const uint32_t bc = fdiv(local, op.fd_h);
    it.h = (int)(local - bc * op.H);
    const uint32_t b = fdiv(bc, op.fd_chunks);
    chunk = bc - b * op.chunks;
    it.b = (int)b;
  }
  it.t0 = (int)chunk * CH;
  it.ntile = min(2, (op.S - it.t0 + 127) / 128);
  return it;
}

// One row's part: its block's scale from the exchanged group maxima (rd), the scale itself
// (written by the block's first row), and the row part's E4M3 codes into the staging tile
// (128B-swizzled rows, as the TMA store reads them).
__device__ __forceinline__ float max4(float4 a) { return fmaxf(fmaxf(a.x, a.y), fmaxf(a.z, a.w)); }

__device__ __forceinline__ void stage_codes(const RotOp& op, const RItem& it, const float* rd, const float* gm, int u,
                                            int part, int quarter, int lane, int i, int t,
                                            const uint32_t (&v)[CW / 2], uint8_t* ctile) {
  static_assert(NCP == 2, "the group-max gather below reads 2 parts per 32-row group");
  const int r_in = u * 128 + i;  // row within the chunk
  float m;
  if (op.blk < 32) {
    m = fmaxf(rd[((u * NCP + 0) * 4 + quarter) * 32 + lane], rd[((u * NCP + 1) * 4 + quarter) * 32 + lane]);
  } else {
    // the block's 32-row groups are contiguous in gm: blk / 16 values from group (r_in / blk) * (blk / 32)
    const float* gp = gm + ((r_in & ~(op.blk - 1)) >> 5) * NCP;
    const float4* g4 = reinterpret_cast<const float4*>(gp);
    if (op.lblk == 5) m = fmaxf(gp[0], gp[1]);
    else if (op.lblk == 6) m = max4(g4[0]);
    else if (op.lblk == 7) m = fmaxf(max4(g4[0]), max4(g4[1]));
    else m = fmaxf(fmaxf(max4(g4[0]), max4(g4[1])), fmaxf(max4(g4[2]), max4(g4[3])));
  }
  const float sc = __fdiv_rn(m, 448.0f);
  if (part == 0 && (r_in & (op.blk - 1)) == 0) {
    const int nblk = (op.S + op.blk - 1) >> op.lblk;
    const long long si = ((long long)it.b * op.H + it.h) * nblk + (t >> op.lblk);
    if (in_bounds(si >= 0 && si < (long long)op.B * op.H * nblk, 141)) op.scales[si] = sc;
  }
  if (sc >= kFastDivMin) {
    const float rc = __frcp_rn(sc);
#pragma unroll
    for (int q = 0; q < CW / 16; ++q) {
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t p0 = v[8 * q + 2 * e], p1 = v[8 * q + 2 * e + 1];
        w[e] = e4m3x4(fp8_div(__uint_as_float(p0 << 16), sc, rc), fp8_div(__uint_as_float(p0 & 0xFFFF0000u), sc, rc),
                      fp8_div(__uint_as_float(p1 << 16), sc, rc), fp8_div(__uint_as_float(p1 & 0xFFFF0000u), sc, rc));
      }
      *reinterpret_cast<uint4*>(ctile + swz128_offset(i, part * (CW / 16) + q)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  } else {
    // tiny or zero scale: IEEE division, out of line (rare)
#pragma unroll
    for (int q = 0; q < CW / 16; ++q)
      *reinterpret_cast<uint4*>(ctile + swz128_offset(i, part * (CW / 16) + q)) =
          codes_ieee(make_uint4(v[8 * q], v[8 * q + 1], v[8 * q + 2], v[8 * q + 3]),
                     make_uint4(v[8 * q + 4], v[8 * q + 5], v[8 * q + 6], v[8 * q + 7]), sc);
  }
}

// Persistent: one CTA per SM walks work items g = blockIdx.x, blockIdx.x + gridDim.x, ...
// (operand, batch, head, 256-token chunk).  The producer loads item k + 1's tiles into the other
// input stage and the MMA thread rotates it into the other TMEM buffer while the epilogue warps
// quantize item k.
__global__ void __launch_bounds__(RTHREADS, 1)
    rotate_block_quant_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                              const __grid_constant__ CUtensorMap mv, const __grid_constant__ CUtensorMap mrq,
                              const __grid_constant__ CUtensorMap mrk, const __grid_constant__ CUtensorMap mcq,
                              const __grid_constant__ CUtensorMap mck, const __grid_constant__ CUtensorMap mcv,
                              const RotParams prm) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + RSmem::BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + RB_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar + RB_COUNT + 1);
  float* red = reinterpret_cast<float*>(smem + RSmem::RED);
  float* gmax = reinterpret_cast<float*>(smem + RSmem::GM);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long G = gridDim.x;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar[RB_XF + i], 1);
      mbar_init(&bar[RB_XE + i], REPI / 32);
      mbar_init(&bar[RB_TF + i], 1);
      mbar_init(&bar[RB_TE + i], REPI / 32);
    }
    mbar_init(&bar[RB_RF], 1);
    mbar_init(&bar[RB_RE], 1);
    mbar_init(&bar[RB_FIN], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == WMMA) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;  // TMEM buffer t at columns 256 t: [2 tiles][128]

  if (warp == WPROD) {
    // ------------------------------------------------------------- producer
    // Every lane walks the items (the same sequence); lane 0 issues the barrier operations and
    // the TMA copies, and the whole warp writes a rotation generated from signs.
    long long k = 0;
    int rload = 0, rop = -1;  // rotations loaded so far; the operand whose rotation is resident
    for (long long g = blockIdx.x; g < prm.items; g += G, ++k) {
      const int st = (int)(k & 1);
      bool ok = true;
      if (lane == 0 && k >= 2) ok = mbar_wait(&bar[RB_XE + st], (uint32_t)(((k >> 1) - 1) & 1), abort_flag, prm.status, 45);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      const RItem it = decode_item(prm, g);
      const RotOp& op = prm.op[it.oi];
      if (op.rotate && it.oi != rop) {
        // a CTA meets its items in operand order, so each rotation is loaded once; the next
        // one waits until the MMAs that read the previous one have completed
        if (lane == 0 && rload > 0) ok = mbar_wait(&bar[RB_RE], (uint32_t)((rload - 1) & 1), abort_flag, prm.status, 49);
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
        if (op.had) {
          write_hadamard_rotation(smem + RSmem::R, op.sgn, op.cbits, lane);
          fence_async_smem();  // the MMA reads it through the async proxy
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar[RB_RF]);
        } else if (lane == 0) {
          mbar_arrive_expect_tx(&bar[RB_RF], 32768);
          for (int nb = 0; nb < 2; ++nb)
            tma_load_4d(smem + RSmem::R + nb * 16384, it.oi == 0 ? &mrq : &mrk, &bar[RB_RF], nb * 64, 0, 0, 0);
        }
        ++rload;
        rop = it.oi;
      }
      if (lane == 0) {
        const CUtensorMap* mx = it.oi == 0 ? &mq : (it.oi == 1 ? &mk : &mv);
        const bool bnsd = op.layout == FA_LAYOUT_BNSD;
        mbar_arrive_expect_tx(&bar[RB_XF + st], it.ntile * 2 * 16384);
        for (int u = 0; u < it.ntile; ++u)
          for (int kb = 0; kb < 2; ++kb) {
            const int t = it.t0 + u * 128;
            tma_load_4d(smem + RSmem::X + st * 65536 + (u * 2 + kb) * 16384, mx, &bar[RB_XF + st], kb * 64,
                        bnsd ? t : it.h, bnsd ? it.h : t, it.b);
          }
      }
      __syncwarp();
    }
    if (lane == 0 && *abort_flag) {
      // let loads already issued land before the CTA can exit
      if (rload > 0) mbar_drain(&bar[RB_RF], (uint32_t)((rload - 1) & 1));
      for (long long t = (k >= 2 ? k - 2 : 0); t < k; ++t)
        mbar_drain(&bar[RB_XF + (t & 1)], (uint32_t)((t >> 1) & 1));
    }
    __syncwarp();
  } else if (warp == WMMA) {
    // ----------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = make_idesc(kAccF32, kFmtBF16, kFmtBF16, 0, 1, 128, 128);
      long long k = 0;
      int tuse0 = 0, tuse1 = 0;  // rotate items so far per TMEM buffer
      int rwait = 0, rop = -1;   // rotations waited for; the operand whose rotation is resident
      for (long long g = blockIdx.x; g < prm.items; g += G, ++k) {
        const RItem it = decode_item(prm, g);
        const RotOp& op = prm.op[it.oi];
        if (!op.rotate) continue;
        if (it.oi != rop) {
          if (rop >= 0) mma_commit(&bar[RB_RE]);  // fires once the previous rotation's MMAs complete
          if (!mbar_wait(&bar[RB_RF], (uint32_t)(rwait & 1), abort_flag, prm.status, 46)) break;
          ++rwait;
          rop = it.oi;
        }
        const int st = (int)(k & 1), tb = (int)(k & 1);
        if (!mbar_wait(&bar[RB_XF + st], (uint32_t)((k >> 1) & 1), abort_flag, prm.status, 47)) break;
        const int tu = tb ? tuse1 : tuse0;
        if (tu > 0 && !mbar_wait(&bar[RB_TE + tb], (uint32_t)((tu - 1) & 1), abort_flag, prm.status, 48)) break;
        tc_fence_after();
        const uint32_t sR = smem_u32(smem + RSmem::R);
        for (int u = 0; u < it.ntile; ++u) {
          const uint32_t sX = smem_u32(smem + RSmem::X + st * 65536 + u * 2 * 16384);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint64_t da = make_sdesc(sX + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, kSwz128);
            const uint64_t db = make_sdesc(sR + ks * 16 * 128, 16384, 1024, kSwz128);
            mma_f16(tbase + tb * 256 + u * 128, da, db, idesc, ks > 0);
          }
        }
        mma_commit(&bar[RB_TF + tb]);
        if (tb) ++tuse1; else ++tuse0;
      }
      mma_commit(&bar[RB_FIN]);
      mbar_drain(&bar[RB_FIN], 0);
    }
    __syncwarp();
  } else {
    // -------------------------------------------------------------- epilogue
    // warp e: tile u = e / (4 NCP), column part p = (e / 4) % NCP, TMEM lane quarter e % 4
    const int u = warp / (4 * NCP), part = (warp >> 2) % NCP, quarter = warp & 3;
    const int i = quarter * 32 + lane;  // row within the 128-token tile
    const uint32_t loff = (uint32_t)(quarter * 32) << 16;
    // lane 0 of each tile's first warp stores the tile's staged codes with TMA
    const bool issuer = part == 0 && quarter == 0 && lane == 0;
    long long k = 0;
    int tuse0 = 0, tuse1 = 0;  // rotate items so far per TMEM buffer
    for (long long g = blockIdx.x; g < prm.items; g += G, ++k) {
      const RItem it = decode_item(prm, g);
      const RotOp& op = prm.op[it.oi];
      const int st = (int)(k & 1);
      const bool bnsd = op.layout == FA_LAYOUT_BNSD;
      const bool tile_live = u < it.ntile;  // warp-uniform
      // CW elements of the row as packed bf16x2
      uint32_t v[CW / 2];
      bool wok;  // this warp's wait succeeded (else the item is abandoned at the next barrier)
      if (op.rotate) {
        const int tb = (int)(k & 1);
        const int tu = tb ? tuse1 : tuse0;
        wok = __all_sync(0xffffffffu, mbar_wait(&bar[RB_TF + tb], (uint32_t)(tu & 1), abort_flag, prm.status, 41));
        if (tb) ++tuse1; else ++tuse0;
        if (wok) {
          tc_fence_after();
          if (tile_live) {  // TMEM loads are warp-collective
#pragma unroll
            for (int c = 0; c < CW / 16; ++c) {
              uint32_t r[16];
              tmem_ld16(tbase + tb * 256 + u * 128 + loff + part * CW + c * 16, r);
              tmem_ld_wait();
#pragma unroll
              for (int q = 0; q < 8; ++q) v[c * 8 + q] = bf16x2_rn(__uint_as_float(r[2 * q]), __uint_as_float(r[2 * q + 1]));
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&bar[RB_TE + tb]);
            mbar_arrive(&bar[RB_XE + st]);  // the MMA that read the stage has completed
          }
        }
      } else {
        wok = __all_sync(0xffffffffu, mbar_wait(&bar[RB_XF + st], (uint32_t)((k >> 1) & 1), abort_flag, prm.status, 42));
        if (wok) {
          if (tile_live) {
            // column c of the row sits in K atom c / 64, 16-byte chunk (c % 64) / 8
            const int c0 = part * CW;
#pragma unroll
            for (int q = 0; q < CW / 8; ++q) {
              const int c = c0 + q * 8;
              const uint4 x = *reinterpret_cast<const uint4*>(smem + RSmem::X + st * 65536 + (u * 2 + (c >> 6)) * 16384 +
                                                               swz128_offset(i, (c & 63) >> 3));
              v[4 * q] = x.x; v[4 * q + 1] = x.y; v[4 * q + 2] = x.z; v[4 * q + 3] = x.w;
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar[RB_XE + st]);
        }
      }
      // Block maxima.  blk divides 256, so it is a power of two: a block is either a group of
      // blk < 32 adjacent lanes of one warp (its NCP column parts in warps of the same tile and
      // quarter) or blk / 32 whole 32-row groups, every part.  Butterflies over the group's lanes
      // leave every lane with its group's maximum; one shared exchange (per lane, or per warp
      // into the group array), double-buffered by item parity so a single barrier per item
      // suffices, combines the rest.
      const int t = it.t0 + u * 128 + i;
      const bool live = wok && tile_live && t < op.S;
      float am = 0.0f;
      if (live) {
        uint32_t m2 = 0;  // running max of |x| as packed bf16x2 (signs garbage until masked)
#pragma unroll
        for (int q = 0; q < CW / 2; ++q) m2 = bf16x2_absmax(m2, v[q]);
        m2 &= 0x7FFF7FFFu;
        am = fmaxf(__uint_as_float(m2 << 16), __uint_as_float(m2 & 0xFFFF0000u));
      }
      const long long ridx = bnsd ? (((long long)it.b * op.H + it.h) * op.S + t) : (((long long)it.b * op.S + t) * op.H + it.h);
      if (live && op.dbg && in_bounds(ridx >= 0 && ridx < (long long)op.B * op.H * op.S, 142)) {
        uint4* d = reinterpret_cast<uint4*>(op.dbg + ridx * 128 + part * CW);
#pragma unroll
        for (int q = 0; q < CW / 8; ++q) d[q] = make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
      }
      const int gl = op.blk < 32 ? op.blk : 32;
      for (int off = 1; off < gl; off <<= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, off));
      float* rd = red + (k & 1) * REPI;         // [epilogue warps][32 lanes]
      float* gmx = gmax + (k & 1) * 8 * NCP;    // [32-row group][part]
      if (op.blk < 32) rd[warp * 32 + lane] = am;
      else if (lane == 0) gmx[(u * 4 + quarter) * NCP + part] = am;
      // the previous item's code stores must have read the staging tile before it is rewritten;
      // the barrier below passes that on to every epilogue thread
      if (issuer) bulk_wait_read_all();
      if (named_barrier_or(NB_MAX, REPI, !wok)) break;
      if (!tile_live) continue;
      if (live) stage_codes(op, it, rd, gmx, u, part, quarter, lane, i, t, v, smem + RSmem::C + u * 16384);
      fence_async_smem();  // this thread's staged codes -> visible to the TMA store
      named_barrier_sync(NB_CODE + u, REPI / 2);
      if (issuer) {
        const int tt = it.t0 + u * 128;
        tma_store_4d(it.oi == 0 ? &mcq : (it.oi == 1 ? &mck : &mcv), smem + RSmem::C + u * 16384, 0,
                     bnsd ? tt : it.h, bnsd ? it.h : tt, it.b);
        bulk_commit();
      }
    }
    if (issuer) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == WMMA) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// E4M3 codes [.., D = 128] as a 4D u8 map in the operand's layout, one 128-token box (128B-swizzled).
cudaError_t make_code_map(CUtensorMap* map, void* base, int B, int H, int S, int layout) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return cudaErrorNotSupported;
  const int D = 128;
  cuuint64_t dims[4], strides[3];
  cuuint32_t box[4], es[4] = {1, 1, 1, 1};
  if (layout == FA_LAYOUT_BNSD) {
    dims[0] = D; dims[1] = S; dims[2] = H; dims[3] = B;
    strides[0] = (cuuint64_t)D; strides[1] = (cuuint64_t)S * D; strides[2] = (cuuint64_t)H * S * D;
    box[0] = 128; box[1] = 128; box[2] = 1; box[3] = 1;
  } else {
    dims[0] = D; dims[1] = H; dims[2] = S; dims[3] = B;
    strides[0] = (cuuint64_t)D; strides[1] = (cuuint64_t)H * D; strides[2] = (cuuint64_t)S * H * D;
    box[0] = 128; box[1] = 1; box[2] = 128; box[3] = 1;
  }
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, base, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_bf16_map(CUtensorMap* map, const void* base, int B, int H, int S, int layout) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return cudaErrorNotSupported;
  const int D = 128;
  cuuint64_t dims[4], strides[3];
  cuuint32_t box[4], es[4] = {1, 1, 1, 1};
  if (layout == FA_LAYOUT_BNSD) {
    dims[0] = D; dims[1] = S; dims[2] = H; dims[3] = B;
    strides[0] = (cuuint64_t)D * 2; strides[1] = (cuuint64_t)S * D * 2; strides[2] = (cuuint64_t)H * S * D * 2;
    box[0] = 64; box[1] = 128; box[2] = 1; box[3] = 1;
  } else {
    dims[0] = D; dims[1] = H; dims[2] = S; dims[3] = B;
    strides[0] = (cuuint64_t)D * 2; strides[1] = (cuuint64_t)H * D * 2; strides[2] = (cuuint64_t)S * H * D * 2;
    box[0] = 64; box[1] = 1; box[2] = 128; box[3] = 1;
  }
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// R [D, D] row-major as a 4D map (j, d, 1, 1) with 64-element boxes.
cudaError_t make_rot_map(CUtensorMap* map, const void* R) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return cudaErrorNotSupported;
  cuuint64_t dims[4] = {128, 128, 1, 1}, strides[3] = {256, 256 * 128, 256 * 128};
  cuuint32_t box[4] = {64, 128, 1, 1}, es[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(R), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_rotate_block_quant(const RotateOperand* ops, int nops, int* status, cudaStream_t s) {
  if (const cudaError_t be = bounds_attach(); be != cudaSuccess) return be;
  RotParams prm = {};
  prm.status = status;
  CUtensorMap maps[3], rmaps[2], cmaps[3];
  memset(maps, 0, sizeof maps);
  memset(rmaps, 0, sizeof rmaps);
  memset(cmaps, 0, sizeof cmaps);
  long long total = 0;
  int n = 0;
  for (int i = 0; i < nops; ++i) {
    const RotateOperand& o = ops[i];
    if (o.D != 128) return cudaErrorNotSupported;
    if (CH % o.blk != 0) return cudaErrorNotSupported;
    if ((long long)o.B * o.H * o.S == 0) continue;
    RotOp& r = prm.op[n];
    r.codes = o.codes;
    r.scales = o.scales;
    r.dbg = static_cast<__nv_bfloat16*>(o.dbg);
    r.B = o.B; r.H = o.H; r.S = o.S; r.layout = o.layout; r.blk = o.blk;
    r.rotate = o.R != nullptr || o.hadamard;
    r.had = o.hadamard;
    for (int w = 0; w < 4; ++w) r.sgn[w] = o.hadamard ? o.sign_bits[w] : 0u;
    {
      // c = bf16(1 / sqrt(D)), round to nearest even
      const float c32 = 1.0f / sqrtf((float)o.D);
      uint32_t bits;
      memcpy(&bits, &c32, 4);
      r.cbits = ((bits + 0x7FFFu + ((bits >> 16) & 1u)) >> 16) & 0xFFFFu;
    }
    r.chunks = (o.S + CH - 1) / CH;
    r.lblk = 0;
    while ((1 << r.lblk) < o.blk) ++r.lblk;
    r.fd_chunks = make_fastdiv((uint32_t)r.chunks);
    r.fd_h = make_fastdiv((uint32_t)o.H);
    r.first_item = total;
    total += (long long)o.B * o.H * r.chunks;
    cudaError_t e = make_bf16_map(&maps[n], o.x, o.B, o.H, o.S, o.layout);
    if (e != cudaSuccess) return e;
    e = make_code_map(&cmaps[n], o.codes, o.B, o.H, o.S, o.layout);
    if (e != cudaSuccess) return e;
    if (r.rotate && !r.had) {
      // Q and K each bring their own rotation; slot by operand position.
      e = make_rot_map(&rmaps[n < 2 ? n : 1], o.R);
      if (e != cudaSuccess) return e;
    }
    ++n;
  }
  prm.nops = n;
  prm.items = total;
  if (n == 0) return cudaSuccess;
  if (total > 0x7FFFFFFFLL) return cudaErrorInvalidValue;  // item indices stay below 2^31
  {
    const cudaError_t e = set_smem_limit(reinterpret_cast<const void*>(rotate_block_quant_kernel), RSmem::ALLOC);
    if (e != cudaSuccess) return e;
  }
  const long long grid = total < sm_count() ? total : sm_count();
  rotate_block_quant_kernel<<<(unsigned)grid, RTHREADS, RSmem::ALLOC, s>>>(
      maps[0], maps[1], maps[2], rmaps[0], rmaps[1], cmaps[0], cmaps[1], cmaps[2], prm);
  return cudaGetLastError();
}

}  // namespace faq
