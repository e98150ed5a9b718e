// rotate.cu -- fused rotate -> FP8 block quantization (MindIE SD "量化",
// FA量化 / 技术特点: 旋转 then 块量化).
//
// Q' = bf16(Q R_q), K' = bf16(K R_k) (fp32 accumulation, one rounding), V' = V;
// then one E4M3 scale = amax / 448 per (b, h, block of `blk` tokens) and
// codes e4m3(x' / scale).  One CTA handles a 256-token chunk of one
// (operand, batch, head):
//   warp 0     TMA: the chunk as two 128-token bf16 tiles (128B-swizzled,
//              64-element K atoms) and, for Q and K, the rotation R.
//   warp 1     tcgen05.mma kind::f16 (bf16 x bf16 -> fp32): X R into TMEM,
//              R read as the MN-major B operand exactly as stored ([D, D]
//              row-major, x' = x R).
//   all 8 warps, then, the epilogue: warp w takes TMEM lane quarter w % 4
//              and column half w / 4 of each 128-token tile; its bf16 half
//              rows (rotated in TMEM, or V from the shared tile) stay in
//              registers for half-row maxima -> block maxima (one warp per
//              block, through shared memory) -> scale -> E4M3 codes (IEEE
//              division), with an optional bf16 copy of the rotated rows.
// blk must divide 256.
#include <cuda_bf16.h>
#include <string.h>

#include "internal.cuh"
#include "quant_common.cuh"
#include "sm100.cuh"

namespace faq {
namespace {

constexpr int CH = 256;  // tokens per CTA
constexpr int RTHREADS = 256;

struct RotOp {
  void* codes;
  float* scales;
  __nv_bfloat16* dbg;
  int B, H, S, layout, blk, rotate;
  long long first_cta;  // first CTA index of this operand
  int chunks;           // 256-token chunks per (b, h)
};

struct RotParams {
  RotOp op[3];
  int nops;
  int* status;
};

struct RSmem {
  static constexpr uint32_t X = 0;           // [2 tiles][2 K atoms][128 rows][128 B]
  static constexpr uint32_t R = 65536;       // [2 N atoms][128 d rows][128 B]
  static constexpr uint32_t RMAX = R + 32768;    // [2 tiles][2 halves][128] half-row maxima
  static constexpr uint32_t BMAX = RMAX + 2048;  // [256] per-block scale (up to 256 blocks per chunk)
  static constexpr uint32_t BAR = BMAX + 1024;
  static constexpr uint32_t TOTAL = BAR + 256;
  static constexpr uint32_t ALLOC = TOTAL + 1024;
};

__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  uint16_t lo, hi;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(b), "f"(a));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(d), "f"(c));
  return (uint32_t)lo | ((uint32_t)hi << 16);
}

__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

__global__ void __launch_bounds__(RTHREADS, 2)
    rotate_block_quant_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                              const __grid_constant__ CUtensorMap mv, const __grid_constant__ CUtensorMap mrq,
                              const __grid_constant__ CUtensorMap mrk, const RotParams prm) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + RSmem::BAR);  // 0: loads, 1: mma, 2: row maxima, 3: block scales
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar + 5);
  float* rmax = reinterpret_cast<float*>(smem + RSmem::RMAX);
  float* bsc = reinterpret_cast<float*>(smem + RSmem::BMAX);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long cta = blockIdx.x;
  int oi = 0;
  if (prm.nops > 1 && cta >= prm.op[1].first_cta) oi = 1;
  if (prm.nops > 2 && cta >= prm.op[2].first_cta) oi = 2;
  const RotOp& op = prm.op[oi];
  const CUtensorMap* mx = oi == 0 ? &mq : (oi == 1 ? &mk : &mv);
  const CUtensorMap* mr = oi == 0 ? &mrq : &mrk;
  const long long local = cta - op.first_cta;
  const int chunk = (int)(local % op.chunks);
  const long long bh = local / op.chunks;
  const int h = (int)(bh % op.H), b = (int)(bh / op.H);
  const int t0 = chunk * CH;
  const int ntile = min(2, (op.S - t0 + 127) / 128);
  const bool bnsd = op.layout == FA_LAYOUT_BNSD;

  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    mbar_init(&bar[2], RTHREADS);
    mbar_init(&bar[3], RTHREADS);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      const uint32_t bytes = ntile * 2 * 16384 + (op.rotate ? 32768 : 0);
      mbar_arrive_expect_tx(&bar[0], bytes);
      for (int u = 0; u < ntile; ++u)
        for (int kb = 0; kb < 2; ++kb) {
          const int t = t0 + u * 128;
          tma_load_4d(smem + RSmem::X + (u * 2 + kb) * 16384, mx, &bar[0], kb * 64, bnsd ? t : h, bnsd ? h : t, b);
        }
      if (op.rotate)
        for (int nb = 0; nb < 2; ++nb) tma_load_4d(smem + RSmem::R + nb * 16384, mr, &bar[0], nb * 64, 0, 0, 0);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && op.rotate) {
      constexpr uint32_t idesc = make_idesc(kAccF32, kFmtBF16, kFmtBF16, 0, 1, 128, 128);
      if (mbar_wait(&bar[0], 0, abort_flag, prm.status, 40)) {
        tc_fence_after();
        const uint32_t sR = smem_u32(smem + RSmem::R);
        for (int u = 0; u < ntile; ++u) {
          const uint32_t sX = smem_u32(smem + RSmem::X + u * 2 * 16384);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint64_t da = make_sdesc(sX + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, kSwz128);
            const uint64_t db = make_sdesc(sR + ks * 16 * 128, 16384, 1024, kSwz128);
            mma_f16(tbase + u * 128, da, db, idesc, ks > 0);
          }
        }
      }
      mma_commit(&bar[1]);
      mbar_wait(&bar[1], 0, abort_flag, nullptr, 0);
    }
    __syncwarp();
  }

  // ---------------------------------------------------------------- epilogue
  const int half = warp >> 2;                 // columns [64 * half, 64 * half + 64)
  const int i = (warp & 3) * 32 + lane;       // row within a 128-token tile
  const uint32_t loff = (uint32_t)((warp & 3) * 32) << 16;
  bool ok = mbar_wait(&bar[op.rotate ? 1 : 0], 0, abort_flag, prm.status, op.rotate ? 41 : 42);
  ok = __all_sync(0xffffffffu, ok);
  if (op.rotate) tc_fence_after();
  // 64 elements (half a row) of each tile as 32 packed bf16x2
  uint32_t v[2][32];
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int t = t0 + u * 128 + i;
    const bool live = u < ntile && t < op.S;
    float am = 0.0f;
    if (u < ntile && ok) {  // warp-uniform: TMEM loads are warp-collective
      if (op.rotate) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t r[32];
          tmem_ld32(tbase + u * 128 + loff + half * 64 + c * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 16; ++k) v[u][c * 16 + k] = bf16x2_rn(__uint_as_float(r[2 * k]), __uint_as_float(r[2 * k + 1]));
        }
      } else {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const uint4 x = *reinterpret_cast<const uint4*>(smem + RSmem::X + (u * 2 + half) * 16384 + swz128_offset(i, q));
          v[u][4 * q] = x.x; v[u][4 * q + 1] = x.y; v[u][4 * q + 2] = x.z; v[u][4 * q + 3] = x.w;
        }
      }
#pragma unroll
      for (int k = 0; k < 32; ++k)
        am = fmaxf(am, fmaxf(fabsf(__uint_as_float(v[u][k] << 16)), fabsf(__uint_as_float(v[u][k] & 0xFFFF0000u))));
      if (op.dbg && live) {
        const long long ridx = bnsd ? (((long long)b * op.H + h) * op.S + t) : (((long long)b * op.S + t) * op.H + h);
        uint4* d = reinterpret_cast<uint4*>(op.dbg + ridx * 128 + half * 64);
#pragma unroll
        for (int q = 0; q < 8; ++q) d[q] = make_uint4(v[u][4 * q], v[u][4 * q + 1], v[u][4 * q + 2], v[u][4 * q + 3]);
      }
    }
    rmax[(u * 2 + half) * 128 + i] = live ? am : 0.0f;
  }
  mbar_arrive(&bar[2]);
  ok = __all_sync(0xffffffffu, mbar_wait(&bar[2], 0, abort_flag, prm.status, 43)) && ok;

  // block scales: warp w reduces blocks w, w + 8, ... of the chunk (2 * blk half-row maxima each)
  const int nb_chunk = CH / op.blk;
  const int nblk = (op.S + op.blk - 1) / op.blk;
  for (int bb = warp; bb < nb_chunk; bb += RTHREADS / 32) {
    float m = 0.0f;
    for (int k = lane; k < 2 * op.blk; k += 32) {
      const int row = bb * op.blk + (k >> 1);
      m = fmaxf(m, rmax[((row >> 7) * 2 + (k & 1)) * 128 + (row & 127)]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    const float sc = __fdiv_rn(m, 448.0f);
    if (lane == 0) {
      bsc[bb] = sc;
      const int t = t0 + bb * op.blk;
      if (t < op.S) op.scales[((long long)b * op.H + h) * nblk + t / op.blk] = ok ? sc : 0.0f;
    }
  }
  mbar_arrive(&bar[3]);
  ok = __all_sync(0xffffffffu, mbar_wait(&bar[3], 0, abort_flag, prm.status, 44)) && ok;

  // codes: this thread's 64 values of each tile row
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int r_in = u * 128 + i;
    const int t = t0 + r_in;
    if (!(u < ntile && t < op.S)) continue;
    const float sc = bsc[r_in / op.blk];
    const bool fast = sc >= kFastDivMin;
    const float rc = fast ? __frcp_rn(sc) : 0.0f;
    const long long ridx = bnsd ? (((long long)b * op.H + h) * op.S + t) : (((long long)b * op.S + t) * op.H + h);
    uint32_t w[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const uint32_t p0 = v[u][2 * e], p1 = v[u][2 * e + 1];
      const float x0 = __uint_as_float(p0 << 16), x1 = __uint_as_float(p0 & 0xFFFF0000u);
      const float x2 = __uint_as_float(p1 << 16), x3 = __uint_as_float(p1 & 0xFFFF0000u);
      if (fast)
        w[e] = ok ? e4m3x4(fp8_div(x0, sc, rc), fp8_div(x1, sc, rc), fp8_div(x2, sc, rc), fp8_div(x3, sc, rc)) : 0u;
      else
        w[e] = (sc > 0.0f && ok) ? e4m3x4(__fdiv_rn(x0, sc), __fdiv_rn(x1, sc), __fdiv_rn(x2, sc), __fdiv_rn(x3, sc)) : 0u;
    }
    uint4* crow = reinterpret_cast<uint4*>(static_cast<uint8_t*>(op.codes) + ridx * 128 + half * 64);
#pragma unroll
    for (int q = 0; q < 4; ++q) crow[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 256);
  }
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
  RotParams prm = {};
  prm.status = status;
  CUtensorMap maps[3], rmaps[2];
  memset(maps, 0, sizeof maps);
  memset(rmaps, 0, sizeof rmaps);
  long long total = 0;
  int n = 0;
  for (int i = 0; i < nops; ++i) {
    const RotateOperand& o = ops[i];
    if (o.D != 128) return cudaErrorNotSupported;
    if (CH % o.blk != 0) return cudaErrorNotSupported;
    if ((long long)o.B * o.S == 0) continue;
    RotOp& r = prm.op[n];
    r.codes = o.codes;
    r.scales = o.scales;
    r.dbg = static_cast<__nv_bfloat16*>(o.dbg);
    r.B = o.B; r.H = o.H; r.S = o.S; r.layout = o.layout; r.blk = o.blk;
    r.rotate = o.R != nullptr;
    r.chunks = (o.S + CH - 1) / CH;
    r.first_cta = total;
    total += (long long)o.B * o.H * r.chunks;
    cudaError_t e = make_bf16_map(&maps[n], o.x, o.B, o.H, o.S, o.layout);
    if (e != cudaSuccess) return e;
    if (r.rotate) {
      // Q and K each bring their own rotation; slot by operand position.
      e = make_rot_map(&rmaps[n < 2 ? n : 1], o.R);
      if (e != cudaSuccess) return e;
    }
    ++n;
  }
  prm.nops = n;
  if (n == 0) return cudaSuccess;
  if (total > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(rotate_block_quant_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         RSmem::ALLOC);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  rotate_block_quant_kernel<<<(unsigned)total, RTHREADS, RSmem::ALLOC, s>>>(maps[0], maps[1], maps[2], rmaps[0],
                                                                            rmaps[1], prm);
  return cudaGetLastError();
}

}  // namespace faq
