// hadamard.cu -- rotate + FP8 block quantization for rotations of the Hadamard-times-signs form
// (MindIE SD "量化", FA量化 / 技术特点: 旋转, then 块量化), by a fast Walsh-Hadamard transform.
//
// R = bf16(H_D * diag(sigma) / sqrt(D)), H_D the Sylvester Hadamard matrix (entry (i, j) =
// (-1)^popcount(i & j)), sigma a vector of signs.  Every entry of R is +-c with c = bf16(1 /
// sqrt(D)), so the rotated row is x * R = c * sigma (elementwise) * FWHT(x) with
// FWHT(x)_j = sum_d x_d (-1)^popcount(d & j): D log2 D additions in place of a D x D product.
// As in the general rotation, the rotated row is evaluated in fp32 and rounded once to bf16; the
// block scale is amax / 448 over the block's rotated bf16 values, and the codes are the E4M3
// values of x' / s (rounded as IEEE division rounds it).  V is block-quantized without rotation.
//
// This kernel serves D = 64 and block sizes that do not divide 256 tokens; D = 128 with blocks
// that do goes through the rotation pipeline of rotate.cu with R generated in shared memory from
// the same signs (the rotation is HBM-bound on the tensor cores, so the product costs nothing
// there, and that pipeline streams at close to the copy bandwidth).
//
// One CTA per quantization block (b, h, blk tokens), 256 threads; each token row is shared by
// D / 16 lanes (sixteen elements each, one coalesced read of the row), the transform runs in
// registers with its last log2(D / 16) stages across lanes by shuffles, then the bf16 rounding
// and the amax; the block's amax through shared memory; then the codes, one coalesced store per
// row.  The rotated rows of a block of up to 256 tokens stay in registers between the two
// passes; longer blocks recompute the rows past that.
#include <cuda_bf16.h>
#include <string.h>

#include "internal.cuh"
#include "quant_common.cuh"
#include "sm100.cuh"

namespace faq {
namespace {

constexpr int HT = 256;                  // threads per CTA

// per half: max(|a|, |b|), its sign the XOR of the inputs' signs (exact; only magnitudes are used)
__device__ __forceinline__ uint32_t habsmax(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// (a0, a1) + (b0, b1) and (a0, a1) - (b0, b1), round to nearest, no flush of subnormals
__device__ __forceinline__ void butterfly2(float& a0, float& a1, float& b0, float& b1) {
  asm("{\n\t.reg .b64 x, y, s, d;\n\tmov.b64 x, {%0, %1};\n\tmov.b64 y, {%2, %3};\n\t"
      "add.rn.f32x2 s, x, y;\n\tsub.rn.f32x2 d, x, y;\n\t"
      "mov.b64 {%0, %1}, s;\n\tmov.b64 {%2, %3}, d;\n\t}"
      : "+f"(a0), "+f"(a1), "+f"(b0), "+f"(b1));
}

// 16 bytes global -> shared memory, asynchronously (completes at cp_async_wait_all of this thread)
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ uint32_t e4m3x4h(float a, float b, float c, float d) {
  uint16_t lo, hi;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(b), "f"(a));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(d), "f"(c));
  return (uint32_t)lo | ((uint32_t)hi << 16);
}

struct HadOp {
  const __nv_bfloat16* x;
  uint8_t* codes;
  float* scales;      // [B, H, nblk]
  __nv_bfloat16* dbg; // nullable: the rotated bf16 tensor
  long long cta0;     // first CTA of this operand
  int B, H, S, layout, blk, nblk, rotate;
  uint32_t sign[64];  // per bf16 pair of the rotated row: XOR mask of the two sign bits
};
struct HadParams {
  HadOp op[3];
  int nops;
  float c;  // bf16(1 / sqrt(D))
};

// The row of token s of (b, h): its element offset in the layout.
__device__ __forceinline__ long long row_off(const HadOp& o, int b, int h, int s, int D) {
  return (o.layout == FA_LAYOUT_BNSD ? ((long long)b * o.H + h) * o.S + s : ((long long)b * o.S + s) * o.H + h) * D;
}

// Rows are shared by a group of LPR = D / 16 lanes, sixteen consecutive elements per lane
// (two 16-byte loads, so each row is read by one coalesced access), 32 / LPR rows per warp at a
// time.  The transform's stages with h < 16 pair elements of one lane; the stages h = 16 .. D/2
// pair lanes sub and sub ^ (h / 16) of the row's group, exchanged by shuffles.
template <int D>
struct HadCfg {
  static constexpr int LPR = D / 16;     // lanes per row
  static constexpr int RPW = 32 / LPR;   // rows per warp and step
  static constexpr int RPC = RPW * (HT / 32);  // rows per CTA and step
  static constexpr int KEEP_STEPS = 8;   // steps whose rotated rows stay in registers (8 bf16 pairs each)
};

// Sixteen elements (lane sub of the row) -> rotated and rounded bf16 pairs; returns their abs-max.
template <int D>
__device__ __forceinline__ uint32_t lane_rotated(const HadOp& o, uint4 ra, uint4 rb, int sub, float c, uint32_t (&out)[8]) {
  const uint32_t w[8] = {ra.x, ra.y, ra.z, ra.w, rb.x, rb.y, rb.z, rb.w};
  if (!o.rotate) {
    uint32_t m2 = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      out[e] = w[e];
      m2 = habsmax(m2, w[e]);
    }
    return m2;
  }
  float v[16];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    v[2 * e] = __uint_as_float(w[e] << 16);
    v[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
  }
  // natural-order Walsh-Hadamard transform: stage h pairs element j with j + h (j's bit h clear)
#pragma unroll
  for (int e = 0; e < 16; e += 2) {
    const float a = v[e], b = v[e + 1];
    v[e] = a + b;
    v[e + 1] = a - b;
  }
#pragma unroll
  for (int h = 2; h < 16; h *= 2) {
#pragma unroll
    for (int i = 0; i < 16; i += 2 * h) {
#pragma unroll
      for (int k = i; k < i + h; k += 2) butterfly2(v[k], v[k + 1], v[k + h], v[k + h + 1]);
    }
  }
#pragma unroll
  for (int lb = 1; lb < D / 16; lb *= 2) {
    const bool upper = sub & lb;  // this lane holds the j + h half of each pair
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float other = __shfl_xor_sync(0xffffffffu, v[e], lb);
      v[e] = upper ? other - v[e] : v[e] + other;
    }
  }
  // times c, one rounding to bf16, then the signs (exact on the rounded value)
  uint32_t m2 = 0;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const __nv_bfloat162 r = __floats2bfloat162_rn(v[2 * e] * c, v[2 * e + 1] * c);
    out[e] = *reinterpret_cast<const uint32_t*>(&r) ^ o.sign[sub * 8 + e];
    m2 = habsmax(m2, out[e]);
  }
  return m2;
}

// Sixteen E4M3 codes of one lane's bf16 pairs divided by the block scale sc.
__device__ __forceinline__ uint4 lane_codes(const uint32_t (&p)[8], float sc) {
  uint32_t w[4];
  if (sc >= kFastDivMin) {
    const float rc = __frcp_rn(sc);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t p0 = p[2 * e], p1 = p[2 * e + 1];
      w[e] = e4m3x4h(fp8_div(__uint_as_float(p0 << 16), sc, rc), fp8_div(__uint_as_float(p0 & 0xFFFF0000u), sc, rc),
                     fp8_div(__uint_as_float(p1 << 16), sc, rc), fp8_div(__uint_as_float(p1 & 0xFFFF0000u), sc, rc));
    }
  } else {
    // a tiny or zero scale: IEEE division (rare); zero codes when sc == 0
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t p0 = p[2 * e], p1 = p[2 * e + 1];
      w[e] = sc > 0.0f ? e4m3x4h(__fdiv_rn(__uint_as_float(p0 << 16), sc), __fdiv_rn(__uint_as_float(p0 & 0xFFFF0000u), sc),
                                 __fdiv_rn(__uint_as_float(p1 << 16), sc), __fdiv_rn(__uint_as_float(p1 & 0xFFFF0000u), sc))
                       : 0u;
    }
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// One CTA per quantization block (b, h, blk tokens).  Pass 1 rotates the block's rows and takes
// their amax; the rows of the first KEEP_STEPS steps stay in registers, later ones (long
// blocks only) are recomputed in pass 2, which writes the codes.
template <int D>
__global__ void __launch_bounds__(HT) hadamard_block_quant_kernel(const __grid_constant__ HadParams p) {
  using C = HadCfg<D>;
  __shared__ float wmax[HT / 32];
  const long long cta = blockIdx.x;
  const int which = (p.nops > 2 && cta >= p.op[2].cta0) ? 2 : ((p.nops > 1 && cta >= p.op[1].cta0) ? 1 : 0);
  const HadOp& o = p.op[which];
  const long long local = cta - o.cta0;
  const int g = (int)(local % o.nblk);
  const long long bh = local / o.nblk;
  const int h = (int)(bh % o.H), b = (int)(bh / o.H);
  const int s0 = g * o.blk, rows = min(o.blk, o.S - s0);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int sub = lane % C::LPR;                       // this lane's 16 elements of the row
  const int rsub = warp * C::RPW + lane / C::LPR;      // this lane's row within a step
  const int nsteps = (rows + C::RPC - 1) / C::RPC;

  auto load = [&](int st, uint4& ra, uint4& rb) {
    const int r = st * C::RPC + rsub;
    if (r < rows) {
      const uint4* src = reinterpret_cast<const uint4*>(o.x + row_off(o, b, h, s0 + r, D)) + 2 * sub;
      ra = __ldg(src);
      rb = __ldg(src + 1);
    } else {
      ra = rb = make_uint4(0, 0, 0, 0);
    }
  };
  // The rows of the kept steps land in shared memory first, every copy in flight at once (each
  // lane copies and later reads only its own 32 bytes of a row, so no barrier is needed).
  extern __shared__ __align__(16) uint4 stage[];  // [KEEP_STEPS * RPC rows][D / 8]
#pragma unroll
  for (int k = 0; k < C::KEEP_STEPS; ++k) {
    const int r = k * C::RPC + rsub;
    if (k < nsteps && r < rows) {
      const uint4* src = reinterpret_cast<const uint4*>(o.x + row_off(o, b, h, s0 + r, D)) + 2 * sub;
      uint4* dst = stage + (size_t)r * (D / 8) + 2 * sub;
      cp_async16(dst, src);
      cp_async16(dst + 1, src + 1);
    }
  }
  cp_async_wait_all();
  // pass 1
  uint32_t kept[C::KEEP_STEPS][8];
  uint32_t m2 = 0;
  for (int st = 0; st < nsteps; ++st) {
    uint4 ra = make_uint4(0, 0, 0, 0), rb = ra;
    const int rr = st * C::RPC + rsub;
    if (st < C::KEEP_STEPS) {
      if (rr < rows) {
        ra = stage[(size_t)rr * (D / 8) + 2 * sub];
        rb = stage[(size_t)rr * (D / 8) + 2 * sub + 1];
      }
    } else {
      load(st, ra, rb);
    }
    uint32_t pr[8];
    m2 = habsmax(m2, lane_rotated<D>(o, ra, rb, sub, p.c, pr));
    const int r = st * C::RPC + rsub;
    if (o.dbg && r < rows && in_bounds(row_off(o, b, h, s0 + r, D) < (long long)o.B * o.H * o.S * D, 151)) {
      uint4* dd = reinterpret_cast<uint4*>(o.dbg + row_off(o, b, h, s0 + r, D)) + 2 * sub;
      dd[0] = make_uint4(pr[0], pr[1], pr[2], pr[3]);
      dd[1] = make_uint4(pr[4], pr[5], pr[6], pr[7]);
    }
#pragma unroll
    for (int k = 0; k < C::KEEP_STEPS; ++k)
      if (k == st) {
#pragma unroll
        for (int e = 0; e < 8; ++e) kept[k][e] = pr[e];
      }
  }
  m2 &= 0x7FFF7FFFu;
  float m = fmaxf(__uint_as_float(m2 << 16), __uint_as_float(m2 & 0xFFFF0000u));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  if (lane == 0) wmax[warp] = m;
  __syncthreads();
  m = 0.0f;
#pragma unroll
  for (int w = 0; w < HT / 32; ++w) m = fmaxf(m, wmax[w]);
  const float sc = __fdiv_rn(m, 448.0f);
  if (tid == 0 && in_bounds(bh * o.nblk + g < (long long)o.B * o.H * o.nblk, 152)) o.scales[bh * o.nblk + g] = sc;
  // pass 2: codes, one coalesced 16-byte store per lane and row
  for (int st = 0; st < nsteps; ++st) {
    uint32_t pr[8];
    if (st < C::KEEP_STEPS) {
#pragma unroll
      for (int k = 0; k < C::KEEP_STEPS; ++k)
        if (k == st) {
#pragma unroll
          for (int e = 0; e < 8; ++e) pr[e] = kept[k][e];
        }
    } else {
      uint4 ra, rb;
      load(st, ra, rb);
      lane_rotated<D>(o, ra, rb, sub, p.c, pr);
    }
    const int r = st * C::RPC + rsub;
    if (r < rows && in_bounds(row_off(o, b, h, s0 + r, D) < (long long)o.B * o.H * o.S * D, 153))
      reinterpret_cast<uint4*>(o.codes + row_off(o, b, h, s0 + r, D))[sub] = lane_codes(pr, sc);
  }
}

template <int D>
cudaError_t launch_had(const HadParams& prm, long long ctas, cudaStream_t s) {
  using C = HadCfg<D>;
  constexpr int SM = C::KEEP_STEPS * C::RPC * D * 2;  // staged rows (64 KB for D = 128)
  auto kern = hadamard_block_quant_kernel<D>;
  const cudaError_t e = set_smem_limit(reinterpret_cast<const void*>(kern), SM);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)ctas, HT, SM, s>>>(prm);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_hadamard_block_quant(const HadamardOperand* ops, int nops, cudaStream_t s) {
  if (const cudaError_t be = bounds_attach(); be != cudaSuccess) return be;
  HadParams prm = {};
  long long ctas = 0;
  int D = 0;
  for (int i = 0; i < nops; ++i) {
    const HadamardOperand& a = ops[i];
    HadOp& o = prm.op[prm.nops];
    if ((long long)a.B * a.S == 0) continue;
    if (D && a.D != D) return cudaErrorInvalidValue;
    D = a.D;
    o.x = static_cast<const __nv_bfloat16*>(a.x);
    o.codes = static_cast<uint8_t*>(a.codes);
    o.scales = a.scales;
    o.dbg = static_cast<__nv_bfloat16*>(a.dbg);
    o.B = a.B; o.H = a.H; o.S = a.S; o.layout = a.layout; o.blk = a.blk;
    o.nblk = (a.S + a.blk - 1) / a.blk;
    o.rotate = a.rotate;
    o.cta0 = ctas;
    for (int e = 0; e < a.D / 2; ++e) {
      const uint32_t lo = (a.sign_bits[(2 * e) / 32] >> ((2 * e) % 32)) & 1u;
      const uint32_t hi = (a.sign_bits[(2 * e + 1) / 32] >> ((2 * e + 1) % 32)) & 1u;
      o.sign[e] = a.rotate ? ((lo << 15) | (hi << 31)) : 0u;
    }
    ctas += (long long)a.B * a.H * o.nblk;
    ++prm.nops;
  }
  if (prm.nops == 0) return cudaSuccess;
  if (ctas > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  // c = bf16(1 / sqrt(D)), round to nearest even
  const float c32 = 1.0f / sqrtf((float)D);
  uint32_t bits;
  memcpy(&bits, &c32, 4);
  bits = (bits + 0x7FFFu + ((bits >> 16) & 1u)) & 0xFFFF0000u;
  memcpy(&prm.c, &bits, 4);
  if (D == 128) return launch_had<128>(prm, ctas, s);
  if (D == 64) return launch_had<64>(prm, ctas, s);
  return cudaErrorNotSupported;
}

}  // namespace faq
