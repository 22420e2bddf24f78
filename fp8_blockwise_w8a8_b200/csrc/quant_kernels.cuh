// quant_kernels.cuh -- HBM-streaming quantizers: 128x128 weight blocks and 1x128 token groups
// (optionally fused with RMSNorm).  Both are bit-exact restatements of the block quantization
// rule: s = amax / 448 (fp32 IEEE division; 1 for an all-zero block) or the smallest power of
// two >= fp32(amax / 448) (E8M0), and q = RNE-saturating-E4M3(x / s).
#pragma once
#include "ptx.cuh"

namespace fp8q {

constexpr int kScaleF32 = 0;
constexpr int kScaleE8M0 = 1;

// bf16 halves of a 32-bit word, widened to fp32 (exact).
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint4 ld_stream_v4(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Running maximum of |x| over packed bf16 pairs: max.xorsign.abs compares magnitudes, so the
// magnitude bits of the result are max(|a|, |b|) per half (the sign bit is not used).
__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Both halves of an absmax_bf16x2 accumulator reduced to one fp32 magnitude.
__device__ __forceinline__ float absmax_finish(uint32_t m) {
  return fmaxf(bf16_lo(m & 0x7FFF7FFFu), bf16_hi(m & 0x7FFF7FFFu));
}

__device__ __forceinline__ uint32_t absmax_uint4(uint32_t m, const uint4 &v) {
  return absmax_bf16x2(absmax_bf16x2(m, v.x), absmax_bf16x2(absmax_bf16x2(v.y, v.z), v.w));
}

// Exponent e of the E8M0 scale for a block maximum: the smallest e with 2^e >= fp32(amax/448),
// clamped to [-127, 127]; e = 0 for an all-zero block.
__device__ __forceinline__ int e8m0_exponent(float amax) {
  if (amax == 0.0f) return 0;
  const uint32_t b = __float_as_uint(__fdiv_rn(amax, 448.0f));
  const int ef = static_cast<int>((b >> 23) & 0xFFu);
  const uint32_t mant = b & 0x7FFFFFu;
  int e;
  if (ef == 0) e = (mant > 0x400000u) ? -126 : -127;   // subnormal quotient: 2^-127 = 0x400000
  else e = (ef - 127) + (mant != 0u ? 1 : 0);
  return max(-127, min(127, e));
}

// 2^e as fp32 for e in [-127, 127] (2^-127 is the subnormal 0x00400000).
__device__ __forceinline__ float pow2_f32(int e) {
  return e >= -126 ? __uint_as_float(static_cast<uint32_t>(e + 127) << 23)
                   : __uint_as_float(0x00400000u);
}

__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// Per-block parameters of the fp32-scale quantizer.
//   fast = true : bracket fast path (see quant8_f32), exact fallback where it is ambiguous.
//   fast = false: the exact fp64 quotient for every element (tiny scales, s < 2^-60).
struct QParams {
  float s;       // the scale (divisor)
  float2 lo2;    // RN(r * (1 - 2^-19)) in both lanes, r ~ 1/s
  float2 hi2;    // RN(r * (1 + 2^-19)) in both lanes
  bool fast;
  bool tie;      // amax / 448 is exact (see quant8_f32)
};

__device__ __forceinline__ QParams qparams_f32(float amax) {
  QParams p;
  p.s = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 448.0f);
  // amax is a bf16 value a * 2^E with an integer significand a <= 255; amax / 448 =
  // (a / 7) * 2^(E - 6) is exact iff 7 divides a.
  const uint32_t ab = __float_as_uint(amax);
  const uint32_t a = ((ab >> 16) & 0x7Fu) | (((ab >> 23) & 0xFFu) != 0u ? 0x80u : 0u);
  p.tie = (a % 7u) == 0u;
  p.fast = p.s >= 0x1.0p-60f;
  // r approximates 1/s within one ulp (2^-23 relative, the documented bound of rcp.approx).
  const float r = rcp_approx(p.fast ? p.s : 1.0f);
  const float lo = __fmul_rn(r, 0x1.ffffc0p-1f), hi = __fmul_rn(r, 0x1.000020p+0f);
  p.lo2 = make_float2(lo, lo);
  p.hi2 = make_float2(hi, hi);
  return p;
}

__device__ __forceinline__ float2 unpack_bf16x2(uint32_t w) {
  return make_float2(bf16_lo(w), bf16_hi(w));
}

// Eight E4M3 codes of RN_fp32(x / s) for the eight bf16 values of one uint4 (byte i = element i).
//
// Where the bracket ends disagree there are two cases.  If amax/448 is exact, s = b 2^k with
// b = a/7 <= 36 (at most 6 significant bits), so mid * s has at most 11 significant bits for every
// E4M3 midpoint mid (5 bits): a quotient x/s that is not exactly a midpoint then lies at least
// ~2^-11 (relative) away from it, far outside the bracket -- a disagreement is an exact tie and
// the code is the even one of the two.  Otherwise the eight codes are recomputed through the
// exact fp64 quotient (quant8_fp64).
//
// Bracket: with r = 1/s (1 + e_r), |e_r| <= 2^-23, the rounded products x * RN(r (1 -+ 2^-19))
// are within a relative 2^-23 + 3 * 2^-24 of x/s (1 -+ 2^-19), so they bracket x/s strictly.
// RN_fp32 and the E4M3 conversion are both monotone, hence when the two bracket ends give the
// same code, that code is the code of RN_fp32(x/s).  Otherwise (some x/s within ~2^-19 of an
// E4M3 rounding boundary, exact ties included) the tie rule or the fp64 quotient below decides.
// Eight codes through an fp64 quotient, exact for every element: with r64 = RN64(1/s) the product
// q64 = RN64(x * r64) is within 2^-52 (relative) of x/s.  If x/s is an fp32 number, RN32(q64) is
// that number.  Otherwise x/s is at least ~2^-49 (relative) away from every fp32 rounding
// boundary B -- B has 25 significant bits ending in a one, so B * s has at least 24 and can never
// equal the 8-bit x -- and RN32(q64) = RN32(x/s).  Used only where the fp32 bracket is ambiguous.
__device__ __forceinline__ uint2 quant8_fp64(const uint4 v, float s) {
  const double r64 = __drcp_rn(static_cast<double>(s));
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t c[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 x = unpack_bf16x2(w[j]);
    c[j] = cvt_e4m3x2(__double2float_rn(__dmul_rn(static_cast<double>(x.x), r64)),
                      __double2float_rn(__dmul_rn(static_cast<double>(x.y), r64)));
  }
  return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

__device__ __forceinline__ uint2 quant8_f32(const uint4 v, const QParams &p) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  if (p.fast) {
    uint32_t lo[4], hi[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 x = unpack_bf16x2(w[j]);
      const float2 a = __fmul2_rn(x, p.lo2), b = __fmul2_rn(x, p.hi2);
      lo[j] = cvt_e4m3x2(a.x, a.y);
      hi[j] = cvt_e4m3x2(b.x, b.y);
    }
    const uint32_t l0 = lo[0] | (lo[1] << 16), l1 = lo[2] | (lo[3] << 16);
    const uint32_t h0 = hi[0] | (hi[1] << 16), h1 = hi[2] | (hi[3] << 16);
    const uint32_t d0 = l0 ^ h0, d1 = l1 ^ h1;
    if (__builtin_expect((d0 | d1) == 0u, 1)) return make_uint2(l0, l1);
    if (p.tie) {
      // exact ties: per byte, keep the lower end's code if it is even, else take the other
      // (the two magnitudes are adjacent and share the sign)
      return make_uint2(l0 ^ (d0 & ((l0 & 0x01010101u) * 0xFFu)),
                        l1 ^ (d1 & ((l1 & 0x01010101u) * 0xFFu)));
    }
  }
  return quant8_fp64(v, p.s);  // ambiguous bracket, or a tiny scale (s < 2^-60)
}

// Eight codes for a power-of-two scale 2^e: x * 2^-e is exact (inv2 = {2^-e, 2^-e}).
__device__ __forceinline__ uint2 quant8_pow2(const uint4 v, const float2 inv2) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t c[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 t = __fmul2_rn(unpack_bf16x2(w[j]), inv2);
    c[j] = cvt_e4m3x2(t.x, t.y);
  }
  return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

// ---------------------------------------------------------------------------------------------
// 128x128 weight blocks.  One CTA (256 threads) per block: thread t owns the 16-byte column
// chunk (t % 16) of rows (t / 16) + 16 i, i = 0..7, so every load and store instruction of a
// warp covers two full 256-byte (load) / 128-byte (store) row segments.
// ---------------------------------------------------------------------------------------------
// One 128x128 block: quantize w[128][ldw] (the block's top-left element) into q[128][ldq] and write
// its scale to *scale (fp32 or one E8M0 byte).  All 256 threads of the CTA take part; red is 8
// floats of shared memory.
template <int FMT>
__device__ __forceinline__ void quant_weight_one_block(const uint16_t *__restrict__ w, int64_t ldw,
                                                       uint8_t *__restrict__ q, int64_t ldq,
                                                       void *scale, float *red) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int r0 = tid >> 4;
  const int c8 = (tid & 15) * 8;
  const uint16_t *src = w + r0 * ldw + c8;
  uint4 v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = ld_stream_v4(src + static_cast<int64_t>(i) * 16 * ldw);
  uint32_t m2 = 0u;
#pragma unroll
  for (int i = 0; i < 8; ++i) m2 = absmax_uint4(m2, v[i]);
  float amax = absmax_finish(m2);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (lane == 0) red[warp] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) amax = fmaxf(amax, red[i]);
  __syncthreads();  // red[] is rewritten by the next block
  uint8_t *dst = q + r0 * ldq + c8;
  if (FMT == kScaleF32) {
    const QParams p = qparams_f32(amax);
    if (tid == 0) *static_cast<float *>(scale) = p.s;
#pragma unroll
    for (int i = 0; i < 8; ++i)
      *reinterpret_cast<uint2 *>(dst + static_cast<int64_t>(i) * 16 * ldq) = quant8_f32(v[i], p);
  } else {
    const int e = e8m0_exponent(amax);
    if (tid == 0) *static_cast<uint8_t *>(scale) = static_cast<uint8_t>(e + 127);
    const float inv = pow2_f32(-e);
    const float2 inv2 = make_float2(inv, inv);
#pragma unroll
    for (int i = 0; i < 8; ++i)
      *reinterpret_cast<uint2 *>(dst + static_cast<int64_t>(i) * 16 * ldq) = quant8_pow2(v[i], inv2);
  }
}

template <int FMT>
__global__ void __launch_bounds__(256, 4) k_quant_weight_block(const uint16_t *__restrict__ w,
                                                            int64_t ldw, uint8_t *__restrict__ q,
                                                            int64_t ldq, void *__restrict__ sw,
                                                            int KB, int64_t nblocks) {
  __shared__ float red[8];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int r0 = tid >> 4;
  const int c8 = (tid & 15) * 8;
  for (int64_t blk = blockIdx.x; blk < nblocks; blk += gridDim.x) {
    const int64_t nb = blk / KB, kb = blk - nb * KB;
    const uint16_t *src = w + (nb * 128 + r0) * ldw + kb * 128 + c8;
    uint4 v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = ld_stream_v4(src + static_cast<int64_t>(i) * 16 * ldw);
    uint32_t m2 = 0u;
#pragma unroll
    for (int i = 0; i < 8; ++i) m2 = absmax_uint4(m2, v[i]);
    float amax = absmax_finish(m2);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if (lane == 0) red[warp] = amax;
    __syncthreads();
    amax = red[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) amax = fmaxf(amax, red[i]);
    __syncthreads();  // red[] is rewritten by the next block
    uint8_t *dst = q + (nb * 128 + r0) * ldq + kb * 128 + c8;
    if (FMT == kScaleF32) {
      const QParams p = qparams_f32(amax);
      if (tid == 0) static_cast<float *>(sw)[blk] = p.s;
#pragma unroll
      for (int i = 0; i < 8; ++i)
        *reinterpret_cast<uint2 *>(dst + static_cast<int64_t>(i) * 16 * ldq) = quant8_f32(v[i], p);
    } else {
      const int e = e8m0_exponent(amax);
      if (tid == 0) static_cast<uint8_t *>(sw)[blk] = static_cast<uint8_t>(e + 127);
      const float inv = pow2_f32(-e);
      const float2 inv2 = make_float2(inv, inv);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        *reinterpret_cast<uint2 *>(dst + static_cast<int64_t>(i) * 16 * ldq) = quant8_pow2(v[i], inv2);
    }
  }
}

// ---------------------------------------------------------------------------------------------
// All the weights of a step in one launch.  Matrix i of the batch owns the blocks
// [block_offset_i, block_offset_{i+1}) of one global numbering; persistent CTAs walk that
// numbering with a stride of the grid, keeping the current matrix (the offsets are held in shared
// memory and only ever move forward).  A descriptor that breaks the shape or alignment rules, or a
// block outside its matrix, records FP8Q_ERR_SHAPE and is skipped.
// ---------------------------------------------------------------------------------------------
struct WeightDesc {
  const uint16_t *w;
  uint8_t *q;
  void *s;
  int64_t N, K, ldw, ldq, block_offset;
};
constexpr int kMaxBatchMatrices = 2048;
constexpr int kErrShapeDev = 2;  // FP8Q_ERR_SHAPE

template <int FMT>
__global__ void __launch_bounds__(256, 4) k_quant_weight_block_batched(
    const WeightDesc *__restrict__ d, int count, int64_t total) {
  __shared__ float red[8];
  __shared__ int64_t s_off[kMaxBatchMatrices + 1];
  for (int i = threadIdx.x; i < count; i += blockDim.x) s_off[i] = d[i].block_offset;
  if (threadIdx.x == 0) s_off[count] = total;
  __syncthreads();
  int cur = 0;
  for (int64_t g = blockIdx.x; g < total; g += gridDim.x) {
    while (cur + 1 < count && g >= s_off[cur + 1]) ++cur;
    const WeightDesc md = d[cur];
    const int64_t local = g - s_off[cur];
    const bool shape_ok = md.N > 0 && md.K > 0 && md.N % 128 == 0 && md.K % 128 == 0 &&
                          md.ldw >= md.K && md.ldq >= md.K && md.ldw % 8 == 0 && md.ldq % 16 == 0 &&
                          (reinterpret_cast<uintptr_t>(md.w) & 15u) == 0 &&
                          (reinterpret_cast<uintptr_t>(md.q) & 15u) == 0 && md.s != nullptr &&
                          (FMT != kScaleF32 || (reinterpret_cast<uintptr_t>(md.s) & 3u) == 0);
    const int64_t KB = md.K / 128;
    if (!shape_ok || local < 0 || local >= (md.N / 128) * KB) {
      if (threadIdx.x == 0) record_error(kErrShapeDev);
      continue;
    }
    const int64_t nb = local / KB, kb = local - nb * KB;
    void *scale = FMT == kScaleF32 ? static_cast<void *>(static_cast<float *>(md.s) + local)
                                   : static_cast<void *>(static_cast<uint8_t *>(md.s) + local);
    quant_weight_one_block<FMT>(md.w + nb * 128 * md.ldw + kb * 128, md.ldw,
                                md.q + nb * 128 * md.ldq + kb * 128, md.ldq, scale, red);
  }
}

// ---------------------------------------------------------------------------------------------
// Scale parameters from a table, for the token kernel (one scale per 128 elements, so the
// per-block arithmetic matters).  amax = a * 2^(ef - 134) with a = 128 + (7 mantissa bits) the
// bf16 significand; s = RN(amax / 448) = RN(a / 7) * 2^(ef - 140) exactly while the result is a
// normal number, and 1/s ~ RN(7 / a) * 2^(140 - ef) within 2^-23 (two roundings of 2^-24).
// The table holds, per a: RN(a/7), RN(RN(7/a) (1 - 2^-19)), RN(RN(7/a) (1 + 2^-19)); it is
// built with IEEE divisions when the kernel starts.
// ---------------------------------------------------------------------------------------------
struct ScaleTab {
  float s[128], lo[128], hi[128];
};

__device__ __forceinline__ void build_scale_tab(ScaleTab *t, int tid, int nthreads) {
  for (int i = tid; i < 128; i += nthreads) {
    const float a = static_cast<float>(128 + i);
    t->s[i] = __fdiv_rn(a, 7.0f);
    const float r = __fdiv_rn(7.0f, a);
    t->lo[i] = __fmul_rn(r, 0x1.ffffc0p-1f);
    t->hi[i] = __fmul_rn(r, 0x1.000020p+0f);
  }
}

// x * 2^k for a normal x and a result in the normal range (exact: exponent arithmetic).
__device__ __forceinline__ float scale_pow2(float x, int k) {
  return __uint_as_float(__float_as_uint(x) + (static_cast<uint32_t>(k) << 23));
}

__device__ __forceinline__ QParams qparams_tab(float amax, const ScaleTab *t) {
  const uint32_t ab = __float_as_uint(amax);
  const int ef = static_cast<int>(ab >> 23);
  if (ef < 75) return qparams_f32(amax);  // zero or tiny blocks: s < 2^-60
  const int i = static_cast<int>((ab >> 16) & 0x7Fu);
  QParams p;
  p.s = scale_pow2(t->s[i], ef - 140);
  const float lo = scale_pow2(t->lo[i], 140 - ef), hi = scale_pow2(t->hi[i], 140 - ef);
  p.lo2 = make_float2(lo, lo);
  p.hi2 = make_float2(hi, hi);
  p.fast = true;
  p.tie = ((128u + static_cast<uint32_t>(i)) % 7u) == 0u;
  return p;
}

// Scale and codes of one 1x128 activation group in either format: fp32 amax/448 with the exact
// bracket quantizer, or the E8M0 power of two 2^e (the least with 2^e >= fp32(amax/448), clamped
// to [-127, 127]) stored as its fp32 value, where x * 2^-e is exact and one product per element
// gives the code.
template <int FMT>
struct TokScale {
  QParams p;       // FMT == kScaleF32
  float2 inv2;     // FMT == kScaleE8M0: {2^-e, 2^-e}
  float s;         // the scale written to sa
  __device__ __forceinline__ TokScale(float amax, const ScaleTab *tab) {
    if constexpr (FMT == kScaleF32) {
      p = qparams_tab(amax, tab);
      s = p.s;
    } else {
      const int e = e8m0_exponent(amax);
      s = pow2_f32(e);
      const float inv = pow2_f32(-e);
      inv2 = make_float2(inv, inv);
    }
  }
  __device__ __forceinline__ uint2 codes(const uint4 v) const {
    if constexpr (FMT == kScaleF32) return quant8_f32(v, p);
    else return quant8_pow2(v, inv2);
  }
};

// ---------------------------------------------------------------------------------------------
// 1x128 token groups, optionally preceded by RMSNorm.  One warp per row at a time.
//
// RMSNorm, phase 1: lane l owns the 128-blocks l, l + 32, ... of the row and reads each one from
// global memory (L1-cached; the row was prefetched into L2 while the previous row was processed)
// to form the fp64 sum of squares of the block in ascending k.  The block sums go through a small
// per-warp shared-memory area and lane 0 adds them in ascending block order, then forms r.
// Phase 2 re-reads the row (now in L1/L2) for the quantization.  gamma is held once per CTA as
// fp32, split per 16-byte chunk j into gA[j] (elements 8j..8j+3) and gB[j] (8j+4..8j+7).
//
// Quantization: LPB lanes per 128-block (8 with RMSNorm, so that the gamma reads are free of bank
// conflicts; 4 without), 32 / LPB blocks per warp step; lane `sub` of a block owns the 16-byte
// chunks sub + LPB c, c = 0 .. 16 / LPB - 1.  The loads of the next step are issued before the
// current step is processed.
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ void prefetch_l2(const void *p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&v);
}

// y = bf16( (x * r) * gamma ), two fp32 roundings, for the 8 elements of one uint4; ga and gb
// hold gamma of those elements as fp32.
__device__ __forceinline__ uint4 rms_apply8(const uint4 v, float r, const float4 ga,
                                            const float4 gb) {
  const float2 r2 = make_float2(r, r);
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  const float2 gg[4] = {make_float2(ga.x, ga.y), make_float2(ga.z, ga.w), make_float2(gb.x, gb.y),
                        make_float2(gb.z, gb.w)};
  uint32_t y[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 u = __fmul2_rn(__fmul2_rn(unpack_bf16x2(w[j]), r2), gg[j]);
    y[j] = pack_bf16x2(u.x, u.y);
  }
  return make_uint4(y[0], y[1], y[2], y[3]);
}

// fp64 sum of squares of one 128-element bf16 block, in ascending k.
__device__ __forceinline__ double block_sumsq(const uint16_t *blk) {
  const uint4 *p = reinterpret_cast<const uint4 *>(blk);
  uint4 v[16];
#pragma unroll
  for (int c = 0; c < 16; ++c) v[c] = p[c];
  double acc = 0.0;
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    const uint32_t wv[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const double a = static_cast<double>(bf16_lo(wv[j]));
      acc = __fma_rn(a, a, acc);  // a*a is exact in fp64, so this is RN(acc + a*a)
      const double b2 = static_cast<double>(bf16_hi(wv[j]));
      acc = __fma_rn(b2, b2, acc);
    }
  }
  return acc;
}

// Residual add of one row, coalesced (lane l takes 16-byte chunks l, l + 32, ...):
// res <- h = bf16_RNE(fp32(x) + fp32(res)).  The res lines just read stay in L1 for the passes
// over h that follow (after a __syncwarp).
__device__ __forceinline__ void row_add_residual(const uint16_t *xr, uint16_t *rr, int K, int lane) {
  const int KC = K >> 3;
#pragma unroll 2
  for (int j = lane; j < KC; j += 32) {
    const uint4 a = *reinterpret_cast<const uint4 *>(xr + j * 8);
    const uint4 b = *reinterpret_cast<const uint4 *>(rr + j * 8);
    const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
    uint32_t h[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 s2 = f2_add_rn(unpack_bf16x2(wa[i]), unpack_bf16x2(wb[i]));
      h[i] = pack_bf16x2(s2.x, s2.y);
    }
    *reinterpret_cast<uint4 *>(rr + j * 8) = make_uint4(h[0], h[1], h[2], h[3]);
  }
}

// Shared-memory bytes of the token kernel.
__host__ __device__ constexpr int token_smem_bytes(int K, bool norm, int wpc) {
  return static_cast<int>(sizeof(ScaleTab)) + (norm ? K * 4 + wpc * (K / 128) * 8 : 0);
}

// 1x128 token quant, optionally after RMSNorm.  Instantiations:
//   NORM    one warp per row: fp64 sums of squares (lane per 128-block, ascending k), lane 0 adds
//           them in block order and forms r; then the normalised row is quantized, 8 lanes per block;
//   ADD     (with NORM) each row is first replaced by h = bf16(fp32(x) + fp32(res)) in res (row
//           stride ldr), and h is what gets normalised and quantized;
//   !NORM   plain quant, 4 lanes per block, over (row, step) units with the next unit's loads in
//           flight: whole rows per warp; SPREAD (fewer rows than warps) spreads the units over all
//           warps; PACKED (K/128 not a multiple of the 8 blocks of a step) packs each step with
//           consecutive blocks of the flattened (row, block) sequence.
// FMT selects the group scale: fp32 amax/448 or the E8M0 power of two (TokScale).
template <bool NORM, bool SPREAD = false, bool ADD = false, bool PACKED = false,
          int FMT = kScaleF32>
__global__ void __launch_bounds__(512) k_rmsnorm_quant_token(
    const uint16_t *__restrict__ x, int64_t ldx, const uint16_t *__restrict__ gamma, float eps,
    int64_t M, int K, uint8_t *__restrict__ q, int64_t ldq, float *__restrict__ sa, int64_t lds,
    uint16_t *res, int64_t ldr) {
  constexpr int LPB = NORM ? 8 : 4;        // lanes per 128-block
  constexpr int CPL = 16 / LPB;            // 16-byte chunks per lane
  constexpr int BPS = 32 / LPB;            // blocks per warp step
  extern __shared__ __align__(16) uint8_t smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int wpc = blockDim.x >> 5;
  const int KB = K >> 7;
  ScaleTab *tab = reinterpret_cast<ScaleTab *>(smem);
  float4 *gA = reinterpret_cast<float4 *>(smem + sizeof(ScaleTab));
  float4 *gB = gA + (K >> 3);
  double *wsum = reinterpret_cast<double *>(smem + sizeof(ScaleTab) + K * 4) + warp * KB;  // NORM
  const int grp = lane / LPB, sub = lane % LPB;

  build_scale_tab(tab, threadIdx.x, blockDim.x);
  if (NORM) {
    for (int j = threadIdx.x; j < (K >> 3); j += blockDim.x) {
      const uint4 g = *reinterpret_cast<const uint4 *>(gamma + j * 8);
      gA[j] = make_float4(bf16_lo(g.x), bf16_hi(g.x), bf16_lo(g.y), bf16_hi(g.y));
      gB[j] = make_float4(bf16_lo(g.z), bf16_hi(g.z), bf16_lo(g.w), bf16_hi(g.w));
    }
  }
  __syncthreads();

  const int64_t stride = static_cast<int64_t>(gridDim.x) * wpc;
  if constexpr (!NORM && PACKED) {
    // Plain 1x128 quant, packed walk: the warp's BPS lane groups take BPS consecutive blocks of the
    // flattened (row, block) sequence, so a step may finish one row and start the next and no group
    // idles when K/128 is not a multiple of BPS.  Group g of warp w starts at flat block
    // BPS w + g and advances by BPS stride blocks (dm rows and db blocks, with a carry); its next
    // block's loads are in flight while the current one is converted.
    const int64_t f0 = (static_cast<int64_t>(blockIdx.x) * wpc + warp) * BPS + grp;
    int64_t m = f0 / KB;
    int b = static_cast<int>(f0 - m * KB);
    const int64_t df = stride * BPS;
    const int64_t dm = df / KB;
    const int db = static_cast<int>(df - dm * KB);
    uint4 v0[CPL], v1[CPL];
    auto load_blk = [&](int64_t mm, int bb, uint4 (&dst)[CPL]) {
      if (mm < M) {
        const uint16_t *src = x + mm * ldx + bb * 128;
#pragma unroll
        for (int c = 0; c < CPL; ++c) dst[c] = ld_stream_v4(src + (sub + LPB * c) * 8);
      }
    };
    load_blk(m, b, v0);
    while (__any_sync(0xffffffffu, m < M)) {
      int64_t m1 = m + dm;
      int b1 = b + db;
      if (b1 >= KB) {
        b1 -= KB;
        ++m1;
      }
      load_blk(m1, b1, v1);
      const bool active = m < M;
      uint32_t mx = 0u;
#pragma unroll
      for (int c = 0; c < CPL; ++c) mx = absmax_uint4(mx, v0[c]);
#pragma unroll
      for (int o = LPB / 2; o > 0; o >>= 1)
        mx = absmax_bf16x2(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      if (active) {
        const TokScale<FMT> p(absmax_finish(mx), tab);
        uint8_t *qb = q + m * ldq + b * 128;
#pragma unroll
        for (int c = 0; c < CPL; ++c)
          *reinterpret_cast<uint2 *>(qb + (sub + LPB * c) * 8) = p.codes(v0[c]);
        if (sub == 0) sa[static_cast<int64_t>(b) * lds + m] = p.s;
      }
#pragma unroll
      for (int c = 0; c < CPL; ++c) v0[c] = v1[c];
      m = m1;
      b = b1;
    }
    return;
  }
  if (!NORM) {
    // Plain 1x128 quant over (row, step) units, a step being BPS blocks of one row; the next
    // unit's loads are in flight while the current one is converted.  With at least as many rows
    // as warps, a warp takes whole rows (its steps in order, then the row `stride` further on).
    // With fewer rows (SPREAD, which the launch picks when M < stride), the warps take every
    // stride-th unit, so a few rows still occupy them all.
    const int S = (KB + BPS - 1) / BPS;  // steps per row
    const int64_t u0 = static_cast<int64_t>(blockIdx.x) * wpc + warp;
    int64_t m = u0, Sq = 0;              // SPREAD: the unit stride is Sq rows and Sr steps
    int b0 = 0, Sr = 0;
    if constexpr (SPREAD) {
      m = u0 / S;
      b0 = static_cast<int>(u0 - m * S) * BPS;
      Sq = stride / S;
      Sr = static_cast<int>(stride - Sq * S);
    }
    uint4 v0[CPL], v1[CPL];
    auto load_unit = [&](int64_t mm, int bb0, uint4 (&dst)[CPL]) {
      if (mm < M) {
        const int bb = bb0 + grp < KB ? bb0 + grp : bb0;
        const uint16_t *src = x + mm * ldx + bb * 128;
#pragma unroll
        for (int c = 0; c < CPL; ++c) dst[c] = ld_stream_v4(src + (sub + LPB * c) * 8);
      }
    };
    load_unit(m, b0, v0);
    while (m < M) {
      int64_t m1 = m;
      int b1 = b0 + BPS;
      if constexpr (SPREAD) {
        m1 = m + Sq;
        b1 = b0 + Sr * BPS;
        if (b1 >= S * BPS) {
          b1 -= S * BPS;
          ++m1;
        }
      } else if (b1 >= KB) {
        b1 = 0;
        m1 += stride;
      }
      load_unit(m1, b1, v1);
      const int b = b0 + grp;
      const bool active = b < KB;
      uint32_t mx = 0u;
#pragma unroll
      for (int c = 0; c < CPL; ++c) mx = absmax_uint4(mx, v0[c]);
#pragma unroll
      for (int o = LPB / 2; o > 0; o >>= 1)
        mx = absmax_bf16x2(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const TokScale<FMT> p(absmax_finish(mx), tab);
      uint8_t *qb = q + m * ldq + b * 128;
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        const uint2 codes = p.codes(v0[c]);
        if (active) *reinterpret_cast<uint2 *>(qb + (sub + LPB * c) * 8) = codes;
      }
      if (active && sub == 0) sa[static_cast<int64_t>(b) * lds + m] = p.s;
#pragma unroll
      for (int c = 0; c < CPL; ++c) v0[c] = v1[c];
      m = m1;
      b0 = b1;
    }
    return;
  }
  for (int64_t m = static_cast<int64_t>(blockIdx.x) * wpc + warp; m < M; m += stride) {
    uint16_t *rr = ADD ? res + m * ldr : nullptr;
    // the row that is normalised and quantized: x, or h (written over res in the first pass)
    const uint16_t *xr = ADD ? rr : x + m * ldx;
    const int64_t next = m + stride;
    if (next < M) {
      const char *nr = reinterpret_cast<const char *>(x + next * ldx);
      for (int off = lane * 128; off < K * 2; off += 32 * 128) prefetch_l2(nr + off);
      if (ADD) {
        const char *nh = reinterpret_cast<const char *>(res + next * ldr);
        for (int off = lane * 128; off < K * 2; off += 32 * 128) prefetch_l2(nh + off);
      }
    }

    float r = 1.0f;
    if (NORM) {
      // Sum of squares in fp64: each lane takes its own 128-blocks in ascending k ...
      if (ADD) {
        row_add_residual(x + m * ldx, rr, K, lane);
        __syncwarp();  // every lane's h stores before the reads below
      }
      for (int b = lane; b < KB; b += 32) wsum[b] = block_sumsq(xr + b * 128);
      __syncwarp();
      // ... then lane 0 adds the block sums in ascending block order.
      if (lane == 0) {
        double S = 0.0;
        for (int b = 0; b < KB; ++b) S = __dadd_rn(S, wsum[b]);
        const double var = __dadd_rn(__ddiv_rn(S, static_cast<double>(K)), static_cast<double>(eps));
        r = __double2float_rn(__ddiv_rn(1.0, __dsqrt_rn(var)));
      }
      r = __shfl_sync(0xffffffffu, r, 0);
    }

    // The loads of the next step are issued before the current step is processed.
    uint4 vn[CPL];
    {
      const int bb = grp < KB ? grp : 0;
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        const uint16_t *src = xr + bb * 128 + (sub + LPB * c) * 8;
        vn[c] = NORM ? *reinterpret_cast<const uint4 *>(src) : ld_stream_v4(src);
      }
    }
#pragma unroll 2
    for (int b0 = 0; b0 < KB; b0 += BPS) {
      const int b = b0 + grp;
      const bool active = b < KB;
      const int bb = active ? b : b0;
      uint4 v[CPL];
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        const int chunk = sub + LPB * c;
        v[c] = NORM ? rms_apply8(vn[c], r, gA[bb * 16 + chunk], gB[bb * 16 + chunk]) : vn[c];
      }
      if (b0 + BPS < KB) {
        const int bn = b0 + BPS + grp < KB ? b0 + BPS + grp : b0 + BPS;
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
          const uint16_t *src = xr + bn * 128 + (sub + LPB * c) * 8;
          vn[c] = NORM ? *reinterpret_cast<const uint4 *>(src) : ld_stream_v4(src);
        }
      }
      uint32_t m2 = 0u;
#pragma unroll
      for (int c = 0; c < CPL; ++c) m2 = absmax_uint4(m2, v[c]);
#pragma unroll
      for (int o = LPB / 2; o > 0; o >>= 1) m2 = absmax_bf16x2(m2, __shfl_xor_sync(0xffffffffu, m2, o));
      const TokScale<FMT> p(absmax_finish(m2), tab);
      uint8_t *qb = q + m * ldq + b * 128;
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        const uint2 codes = p.codes(v[c]);
        if (active) *reinterpret_cast<uint2 *>(qb + (sub + LPB * c) * 8) = codes;
      }
      if (active && sub == 0) sa[static_cast<int64_t>(b) * lds + m] = p.s;
    }
    __syncwarp();  // lane 0 has read every block sum before they are overwritten
  }
}

// ---------------------------------------------------------------------------------------------
// Per-token (full-row) quantization, optionally after RMSNorm: one scale per row of K (the
// "group size 0" per-token mode; applied to a weight it gives per-output-channel scales).  One
// warp per row.  With RMSNorm, r is formed exactly as in k_rmsnorm_quant_token; then one pass
// over the row finds its absolute maximum (of y with RMSNorm) and a second pass writes the codes.
// Both passes read the row through L1 (the row was prefetched into L2 during the previous one).
// ---------------------------------------------------------------------------------------------
// ADD (with NORM): as in k_rmsnorm_quant_token, each row is first replaced by
// h = bf16(fp32(x) + fp32(res)) in res, and h is normalised and quantized.
// Per-row quantization without RMSNorm for rows of up to 32 C 16-byte chunks (K <= 256 C): the warp
// loads the whole row into registers at once (lane l holds chunks l, l + 32, ...), takes its amax
// and writes the codes from the same registers -- one pass over memory with C loads in flight per
// lane.  Same arithmetic as k_quant_rowwise<false>.
template <int C>
__global__ void __launch_bounds__(256) k_quant_rowwise_regs(const uint16_t *__restrict__ x, int64_t ldx,
                                                            int64_t M, int K, uint8_t *__restrict__ q,
                                                            int64_t ldq, float *__restrict__ s_out) {
  __shared__ ScaleTab tab;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int wpc = blockDim.x >> 5;
  const int KC = K >> 3;
  build_scale_tab(&tab, threadIdx.x, blockDim.x);
  __syncthreads();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * wpc;
  for (int64_t m = static_cast<int64_t>(blockIdx.x) * wpc + warp; m < M; m += stride) {
    const uint16_t *xr = x + m * ldx;
    uint4 v[C];
#pragma unroll
    for (int i = 0; i < C; ++i) {
      const int j = lane + 32 * i;
      v[i] = j < KC ? ld_stream_v4(xr + j * 8) : make_uint4(0u, 0u, 0u, 0u);  // zeros: no effect on amax
    }
    uint32_t m2 = 0u;
#pragma unroll
    for (int i = 0; i < C; ++i) m2 = absmax_uint4(m2, v[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m2 = absmax_bf16x2(m2, __shfl_xor_sync(0xffffffffu, m2, o));
    const QParams p = qparams_tab(absmax_finish(m2), &tab);
    uint8_t *qr = q + m * ldq;
#pragma unroll
    for (int i = 0; i < C; ++i) {
      const int j = lane + 32 * i;
      if (j < KC) *reinterpret_cast<uint2 *>(qr + j * 8) = quant8_f32(v[i], p);
    }
    if (lane == 0) s_out[m] = p.s;
  }
}

template <bool NORM, bool ADD = false>
__global__ void __launch_bounds__(512) k_quant_rowwise(
    const uint16_t *__restrict__ x, int64_t ldx, const uint16_t *__restrict__ gamma, float eps,
    int64_t M, int K, uint8_t *__restrict__ q, int64_t ldq, float *__restrict__ s_out,
    uint16_t *res, int64_t ldr) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int wpc = blockDim.x >> 5;
  const int KB = K >> 7, KC = K >> 3;   // 128-blocks and 16-byte chunks per row
  ScaleTab *tab = reinterpret_cast<ScaleTab *>(smem);
  float4 *gA = reinterpret_cast<float4 *>(smem + sizeof(ScaleTab));
  float4 *gB = gA + KC;
  double *wsum = reinterpret_cast<double *>(smem + sizeof(ScaleTab) + K * 4) + warp * KB;  // NORM

  build_scale_tab(tab, threadIdx.x, blockDim.x);
  if (NORM) {
    for (int j = threadIdx.x; j < KC; j += blockDim.x) {
      const uint4 g = *reinterpret_cast<const uint4 *>(gamma + j * 8);
      gA[j] = make_float4(bf16_lo(g.x), bf16_hi(g.x), bf16_lo(g.y), bf16_hi(g.y));
      gB[j] = make_float4(bf16_lo(g.z), bf16_hi(g.z), bf16_lo(g.w), bf16_hi(g.w));
    }
  }
  __syncthreads();

  const int64_t stride = static_cast<int64_t>(gridDim.x) * wpc;
  for (int64_t m = static_cast<int64_t>(blockIdx.x) * wpc + warp; m < M; m += stride) {
    uint16_t *rr = ADD ? res + m * ldr : nullptr;
    const uint16_t *xr = ADD ? rr : x + m * ldx;   // the row that is normalised and quantized
    const int64_t next = m + stride;
    if (next < M) {
      const char *nr = reinterpret_cast<const char *>(x + next * ldx);
      for (int off = lane * 128; off < K * 2; off += 32 * 128) prefetch_l2(nr + off);
      if (ADD) {
        const char *nh = reinterpret_cast<const char *>(res + next * ldr);
        for (int off = lane * 128; off < K * 2; off += 32 * 128) prefetch_l2(nh + off);
      }
    }
    float r = 1.0f;
    if (NORM) {
      if (ADD) {
        row_add_residual(x + m * ldx, rr, K, lane);
        __syncwarp();  // every lane's h stores before the reads below
      }
      for (int b = lane; b < KB; b += 32) wsum[b] = block_sumsq(xr + b * 128);
      __syncwarp();
      if (lane == 0) {
        double S = 0.0;
        for (int b = 0; b < KB; ++b) S = __dadd_rn(S, wsum[b]);
        const double var = __dadd_rn(__ddiv_rn(S, static_cast<double>(K)), static_cast<double>(eps));
        r = __double2float_rn(__ddiv_rn(1.0, __dsqrt_rn(var)));
      }
      r = __shfl_sync(0xffffffffu, r, 0);
    }
    // the row's absolute maximum
    uint32_t m2 = 0u;
#pragma unroll 4
    for (int j = lane; j < KC; j += 32) {
      uint4 v = *reinterpret_cast<const uint4 *>(xr + j * 8);
      if (NORM) v = rms_apply8(v, r, gA[j], gB[j]);
      m2 = absmax_uint4(m2, v);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m2 = absmax_bf16x2(m2, __shfl_xor_sync(0xffffffffu, m2, o));
    const QParams p = qparams_tab(absmax_finish(m2), tab);
    // the codes
    uint8_t *qr = q + m * ldq;
#pragma unroll 4
    for (int j = lane; j < KC; j += 32) {
      uint4 v = *reinterpret_cast<const uint4 *>(xr + j * 8);
      if (NORM) v = rms_apply8(v, r, gA[j], gB[j]);
      *reinterpret_cast<uint2 *>(qr + j * 8) = quant8_f32(v, p);
    }
    if (lane == 0) s_out[m] = p.s;
    __syncwarp();  // lane 0 has read every block sum before they are overwritten
  }
}

// ---------------------------------------------------------------------------------------------
// SiLU-and-mul + 1x128 quant, the front end of an MoE down projection: h = [gate | up] bf16
// [R, 2I] -> codes of y = bf16(silu(gate) * up) [R, I] and fp32 scales sa[kb * lds + m].
//
// e^x is computed by the method of Cody and Waite (1980): k = rint(x / ln 2), r = (x - k c1) -
// k c2 with ln 2 = c1 + c2 split so that k c1 is exact, e^r from its degree-7 Taylor polynomial
// by Horner's rule (|r| <= ln2 / 2: truncation below 2^-27 relative), scaled by 2^k exactly.
// Every step is an explicit IEEE round-to-nearest fp32 operation (no contraction), so y is
// reproducible bit for bit; silu(g) = g / (1 + e^-g) with an IEEE division.  The kernel uses the
// two-element form exp_cw2 (packed fp32x2 operations round each lane as the scalar ones do).
// ---------------------------------------------------------------------------------------------
// e^x for two elements at once (packed fp32x2 operations with explicit rounding: each lane
// rounds as a scalar IEEE operation would, and no multiply and add are fused).  Branch-free: the polynomial runs on x clamped into range, then the results
// out of range (inf above ln(FLT_MAX), 0 below half the least subnormal) are selected; the
// scaling by 2^k always takes two exact steps 2^k1 * 2^(k - k1) with k1 = clamp(k, -126, 127).
__device__ __forceinline__ float2 exp_cw2(float2 x) {
  const float2 xc = make_float2(fminf(fmaxf(x.x, -104.0f), 0x1.62e430p+6f),
                                fminf(fmaxf(x.y, -104.0f), 0x1.62e430p+6f));
  const float2 t = f2_mul_rn(xc, make_float2(0x1.715476p+0f, 0x1.715476p+0f));
  const float2 kf = make_float2(rintf(t.x), rintf(t.y));
  const float2 nk = make_float2(-kf.x, -kf.y);
  float2 r = f2_add_rn(xc, f2_mul_rn(nk, make_float2(0x1.62e400p-1f, 0x1.62e400p-1f)));
  r = f2_add_rn(r, f2_mul_rn(nk, make_float2(0x1.7f7d1cp-20f, 0x1.7f7d1cp-20f)));
  float2 p = make_float2(0x1.a01a02p-13f, 0x1.a01a02p-13f);
  p = f2_add_rn(f2_mul_rn(p, r), make_float2(0x1.6c16c2p-10f, 0x1.6c16c2p-10f));
  p = f2_add_rn(f2_mul_rn(p, r), make_float2(0x1.111112p-7f, 0x1.111112p-7f));
  p = f2_add_rn(f2_mul_rn(p, r), make_float2(0x1.555556p-5f, 0x1.555556p-5f));
  p = f2_add_rn(f2_mul_rn(p, r), make_float2(0x1.555556p-3f, 0x1.555556p-3f));
  p = f2_add_rn(f2_mul_rn(p, r), make_float2(0.5f, 0.5f));
  p = f2_add_rn(f2_mul_rn(p, r), make_float2(1.0f, 1.0f));
  p = f2_add_rn(f2_mul_rn(p, r), make_float2(1.0f, 1.0f));
  const int ka = static_cast<int>(kf.x), kb = static_cast<int>(kf.y);
  const int ka1 = min(max(ka, -126), 127), kb1 = min(max(kb, -126), 127);
  p = f2_mul_rn(p, make_float2(__int_as_float((ka1 + 127) << 23), __int_as_float((kb1 + 127) << 23)));
  p = f2_mul_rn(p, make_float2(__int_as_float((ka - ka1 + 127) << 23),
                                __int_as_float((kb - kb1 + 127) << 23)));
  const float inf = __int_as_float(0x7f800000);
  p.x = x.x > 0x1.62e430p+6f ? inf : (x.x < -104.0f ? 0.0f : p.x);
  p.y = x.y > 0x1.62e430p+6f ? inf : (x.y < -104.0f ? 0.0f : p.y);
  return p;
}

// silu(g) = g / (1 + e^-g) given e = e^-g.  Where 1 + e^-g is infinite the quotient is a zero
// with g's sign, selected after dividing by 1 instead (an infinite divisor would take the
// division's slow path).
__device__ __forceinline__ float silu_from_exp(float g, float e) {
  const float d = __fadd_rn(1.0f, e);
  const bool big = d == __int_as_float(0x7f800000);
  return big ? __int_as_float(__float_as_int(g) & 0x80000000) : __fdiv_rn(g, big ? 1.0f : d);
}

// y = bf16(silu(g) * u) for the 8 elements of one uint4 of gate and the matching uint4 of up.
__device__ __forceinline__ uint4 silu_mul8(const uint4 g, const uint4 u) {
  const uint32_t gw[4] = {g.x, g.y, g.z, g.w}, uw[4] = {u.x, u.y, u.z, u.w};
  uint32_t y[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 gg = make_float2(bf16_lo(gw[j]), bf16_hi(gw[j]));
    const float2 e = exp_cw2(make_float2(-gg.x, -gg.y));
    const float2 sl = make_float2(silu_from_exp(gg.x, e.x), silu_from_exp(gg.y, e.y));
    const float2 v = __fmul2_rn(sl, make_float2(bf16_lo(uw[j]), bf16_hi(uw[j])));
    y[j] = pack_bf16x2(v.x, v.y);
  }
  return make_uint4(y[0], y[1], y[2], y[3]);
}

// One warp per row at a time; 8 lanes per 128-block (4 blocks per warp step), lane `sub` of a
// block owns the 16-byte chunks sub + 8 c, c = 0, 1.  The gate and up loads of the next step
// are issued before the current step is processed.
// PACKED (I/128 not a multiple of the 4 blocks of a warp step): the warp's 4 lane groups take 4
// consecutive blocks of the flattened (row, block) sequence, so a step may finish one row and
// start the next and no group computes exponentials for nothing; each group advances by a
// precomputed (rows, blocks) stride with a carry, its next block's loads in flight.
template <bool PACKED = false, int FMT = kScaleF32>
__global__ void __launch_bounds__(512) k_silu_mul_quant(
    const uint16_t *__restrict__ h, int64_t ldh, int64_t R, int I, uint8_t *__restrict__ q,
    int64_t ldq, float *__restrict__ sa, int64_t lds) {
  constexpr int LPB = 8, CPL = 2, BPS = 4;
  extern __shared__ __align__(16) uint8_t smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int wpc = blockDim.x >> 5;
  const int IB = I >> 7;
  ScaleTab *tab = reinterpret_cast<ScaleTab *>(smem);
  const int grp = lane / LPB, sub = lane % LPB;
  build_scale_tab(tab, threadIdx.x, blockDim.x);
  __syncthreads();

  const int64_t stride = static_cast<int64_t>(gridDim.x) * wpc;
  if constexpr (PACKED) {
    const int64_t f0 = (static_cast<int64_t>(blockIdx.x) * wpc + warp) * BPS + grp;
    int64_t m = f0 / IB;
    int b = static_cast<int>(f0 - m * IB);
    const int64_t df = stride * BPS;
    const int64_t dm = df / IB;
    const int db = static_cast<int>(df - dm * IB);
    uint4 gn[CPL], un[CPL];
    auto load_blk = [&](int64_t mm, int bb) {
      if (mm < R) {
        const uint16_t *gr = h + mm * ldh + bb * 128, *ur = gr + I;
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
          gn[c] = ld_stream_v4(gr + (sub + LPB * c) * 8);
          un[c] = ld_stream_v4(ur + (sub + LPB * c) * 8);
        }
      }
    };
    load_blk(m, b);
    while (__any_sync(0xffffffffu, m < R)) {
      const bool active = m < R;
      uint4 v[CPL];
#pragma unroll
      for (int c = 0; c < CPL; ++c) v[c] = silu_mul8(gn[c], un[c]);
      int64_t m1 = m + dm;
      int b1 = b + db;
      if (b1 >= IB) {
        b1 -= IB;
        ++m1;
      }
      load_blk(m1, b1);
      uint32_t m2 = 0u;
#pragma unroll
      for (int c = 0; c < CPL; ++c) m2 = absmax_uint4(m2, v[c]);
#pragma unroll
      for (int o = LPB / 2; o > 0; o >>= 1) m2 = absmax_bf16x2(m2, __shfl_xor_sync(0xffffffffu, m2, o));
      if (active) {
        const TokScale<FMT> p(absmax_finish(m2), tab);
        uint8_t *qb = q + m * ldq + b * 128;
#pragma unroll
        for (int c = 0; c < CPL; ++c)
          *reinterpret_cast<uint2 *>(qb + (sub + LPB * c) * 8) = p.codes(v[c]);
        if (sub == 0) sa[static_cast<int64_t>(b) * lds + m] = p.s;
      }
      m = m1;
      b = b1;
    }
    return;
  }
  for (int64_t m = static_cast<int64_t>(blockIdx.x) * wpc + warp; m < R; m += stride) {
    const uint16_t *gr = h + m * ldh, *ur = gr + I;
    uint4 gn[CPL], un[CPL];
    {
      const int bb = grp < IB ? grp : 0;
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        gn[c] = ld_stream_v4(gr + bb * 128 + (sub + LPB * c) * 8);
        un[c] = ld_stream_v4(ur + bb * 128 + (sub + LPB * c) * 8);
      }
    }
    for (int b0 = 0; b0 < IB; b0 += BPS) {
      const int b = b0 + grp;
      const bool active = b < IB;
      uint4 v[CPL];
#pragma unroll
      for (int c = 0; c < CPL; ++c) v[c] = silu_mul8(gn[c], un[c]);
      if (b0 + BPS < IB) {
        const int bn = b0 + BPS + grp < IB ? b0 + BPS + grp : b0 + BPS;
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
          gn[c] = ld_stream_v4(gr + bn * 128 + (sub + LPB * c) * 8);
          un[c] = ld_stream_v4(ur + bn * 128 + (sub + LPB * c) * 8);
        }
      }
      uint32_t m2 = 0u;
#pragma unroll
      for (int c = 0; c < CPL; ++c) m2 = absmax_uint4(m2, v[c]);
#pragma unroll
      for (int o = LPB / 2; o > 0; o >>= 1) m2 = absmax_bf16x2(m2, __shfl_xor_sync(0xffffffffu, m2, o));
      const TokScale<FMT> p(absmax_finish(m2), tab);
      uint8_t *qb = q + m * ldq + b * 128;
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        const uint2 codes = p.codes(v[c]);
        if (active) *reinterpret_cast<uint2 *>(qb + (sub + LPB * c) * 8) = codes;
      }
      if (active && sub == 0) sa[static_cast<int64_t>(b) * lds + m] = p.s;
    }
  }
}

// ---------------------------------------------------------------------------------------------
// Inverse RoPE + 1x128 quant: the front end of the attention output projection (wo_a).  o is
// [T][H][D] bf16 with token stride ldo; the last R dims of each head are rotated by -theta_i in
// pairs (a, b) = (2i, 2i + 1) (INTERLEAVED) or (i, i + R/2), with c = cos[p][i], s = sin[p][i]:
//   y_a = bf16( fp32(x_a c) + fp32(x_b s) ),   y_b = bf16( fp32(x_b c) - fp32(x_a s) ),
// every product and sum one IEEE fp32 rounding; the first D - R dims pass through.  The result is
// quantized in 1x128 groups along the token's H*D row.  The host guarantees D % 8 == 0 and
// R % 8 == 0 (R % 16 == 0 for half-split pairs), so every 16-byte chunk lies inside one head and
// is all rotary or all pass-through, and the cache entries a chunk needs are 16-byte aligned.
// ---------------------------------------------------------------------------------------------
constexpr int kErrRange = 9;  // FP8Q_ERR_RANGE: a position outside [0, max_pos)

__device__ __forceinline__ float4 ldg_f4(const float *p) {
  return __ldg(reinterpret_cast<const float4 *>(p));
}

// Products and sums here use the scalar IEEE intrinsics, which are never merged into a fused
// multiply-add: the rotation must round x_a c and x_b s separately, and a pair of packed
// multiply and add intrinsics was measured to be contracted (a tie rounded the other way).

// Four interleaved pairs (x_2i, x_2i+1), i = i0 .. i0 + 3, with their cos / sin entries.
__device__ __forceinline__ uint4 inv_rope8_pairs(const uint4 x, const float4 c, const float4 s) {
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
  const float cc[4] = {c.x, c.y, c.z, c.w}, ss[4] = {s.x, s.y, s.z, s.w};
  uint32_t y[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float xa = bf16_lo(w[j]), xb = bf16_hi(w[j]);
    const float ya = __fadd_rn(__fmul_rn(xa, cc[j]), __fmul_rn(xb, ss[j]));
    const float yb = __fsub_rn(__fmul_rn(xb, cc[j]), __fmul_rn(xa, ss[j]));
    y[j] = pack_bf16x2(ya, yb);
  }
  return make_uint4(y[0], y[1], y[2], y[3]);
}

// Eight elements of one half of the rotary part (x) with their partners in the other half (z):
// y = fp32(x c) + fp32(z s) for the first half, fp32(x c) - fp32(z s) for the second.
__device__ __forceinline__ uint4 inv_rope8_halves(const uint4 x, const uint4 z, bool second,
                                                  const float *cs, const float *sn) {
  const float4 c0 = ldg_f4(cs), c1 = ldg_f4(cs + 4), s0 = ldg_f4(sn), s1 = ldg_f4(sn + 4);
  const float cc[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
  const float ss[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
  const uint32_t wx[4] = {x.x, x.y, x.z, x.w}, wz[4] = {z.x, z.y, z.z, z.w};
  uint32_t y[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    float v[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float xv = h ? bf16_hi(wx[j]) : bf16_lo(wx[j]);
      const float zv = h ? bf16_hi(wz[j]) : bf16_lo(wz[j]);
      const float pc = __fmul_rn(xv, cc[2 * j + h]), ps = __fmul_rn(zv, ss[2 * j + h]);
      v[h] = second ? __fsub_rn(pc, ps) : __fadd_rn(pc, ps);
    }
    y[j] = pack_bf16x2(v[0], v[1]);
  }
  return make_uint4(y[0], y[1], y[2], y[3]);
}

// One warp per token at a time; 8 lanes per 128-block (4 blocks per warp step), lane `sub` of a
// block owns the 16-byte chunks sub + 8 c, c = 0, 1; the next step's chunks are loaded before
// the current step is processed.  A token whose position is outside [0, max_pos) is not written
// and records kErrRange in the device error word.
template <int FMT, bool INTERLEAVED>
__global__ void __launch_bounds__(512) k_inverse_rope_quant(
    const uint16_t *__restrict__ o, int64_t ldo, const int64_t *__restrict__ pos,
    const float *__restrict__ cosc, const float *__restrict__ sinc, int64_t max_pos, int64_t T,
    int D, int R, int K, uint8_t *__restrict__ q, int64_t ldq, float *__restrict__ sa,
    int64_t lds) {
  constexpr int LPB = 8, CPL = 2, BPS = 4;
  extern __shared__ __align__(16) uint8_t smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int wpc = blockDim.x >> 5;
  const int KB = K >> 7, half = R >> 1, pass = D - R;
  ScaleTab *tab = reinterpret_cast<ScaleTab *>(smem);
  const int grp = lane / LPB, sub = lane % LPB;
  if (FMT == kScaleF32) build_scale_tab(tab, threadIdx.x, blockDim.x);
  __syncthreads();
  // Offset inside its head of each chunk this lane owns at the first step, and the advance per
  // step (BPS blocks) modulo D: the offsets then follow without a division per step.
  int d_first[CPL];
#pragma unroll
  for (int c = 0; c < CPL; ++c) d_first[c] = (grp * 128 + (sub + LPB * c) * 8) % D;
  const int d_step = (BPS * 128) % D;

  const int64_t stride = static_cast<int64_t>(gridDim.x) * wpc;
  for (int64_t m = static_cast<int64_t>(blockIdx.x) * wpc + warp; m < T; m += stride) {
    int64_t p = 0;
    if (R > 0) {
      p = __ldg(pos + m);
      if (p < 0 || p >= max_pos) {
        if (lane == 0) record_error(kErrRange);
        continue;
      }
    }
    const float *cs = cosc + p * half, *sn = sinc + p * half;
    const uint16_t *xr = o + m * ldo;
    int bl = grp < KB ? grp : 0;  // the block whose chunks xn holds
    uint4 xn[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) xn[c] = ld_stream_v4(xr + bl * 128 + (sub + LPB * c) * 8);
    int d0c[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) d0c[c] = d_first[c];
    for (int b0 = 0; b0 < KB; b0 += BPS) {
      const int b = b0 + grp;
      const bool active = b < KB;
      uint4 v[CPL];
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        // while active, xn[c] holds block b and d0 is its chunk's offset inside the head
        const int k0 = b * 128 + (sub + LPB * c) * 8;
        const int d0 = d0c[c];
        d0c[c] = d0 + d_step >= D ? d0 + d_step - D : d0 + d_step;
        v[c] = xn[c];
        if (active && d0 >= pass) {
          const int j0 = d0 - pass;
          if (INTERLEAVED) {
            v[c] = inv_rope8_pairs(xn[c], ldg_f4(cs + j0 / 2), ldg_f4(sn + j0 / 2));
          } else {
            const bool second = j0 >= half;
            const int i0 = second ? j0 - half : j0;
            const uint4 z = ld_stream_v4(xr + (second ? k0 - half : k0 + half));
            v[c] = inv_rope8_halves(xn[c], z, second, cs + i0, sn + i0);
          }
        }
      }
      if (b0 + BPS < KB) {
        bl = b0 + BPS + grp < KB ? b0 + BPS + grp : b0 + BPS;
#pragma unroll
        for (int c = 0; c < CPL; ++c) xn[c] = ld_stream_v4(xr + bl * 128 + (sub + LPB * c) * 8);
      }
      uint32_t m2 = 0u;
#pragma unroll
      for (int c = 0; c < CPL; ++c) m2 = absmax_uint4(m2, v[c]);
#pragma unroll
      for (int s = LPB / 2; s > 0; s >>= 1)
        m2 = absmax_bf16x2(m2, __shfl_xor_sync(0xffffffffu, m2, s));
      const float amax = absmax_finish(m2);
      uint8_t *qb = q + m * ldq + b * 128;
      float scale;
      if (FMT == kScaleF32) {
        const QParams qp = qparams_tab(amax, tab);
        scale = qp.s;
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
          const uint2 codes = quant8_f32(v[c], qp);
          if (active) *reinterpret_cast<uint2 *>(qb + (sub + LPB * c) * 8) = codes;
        }
      } else {
        const int e = e8m0_exponent(amax);
        scale = pow2_f32(e);
        const float inv = pow2_f32(-e);
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
          const uint2 codes = quant8_pow2(v[c], make_float2(inv, inv));
          if (active) *reinterpret_cast<uint2 *>(qb + (sub + LPB * c) * 8) = codes;
        }
      }
      if (active && sub == 0) sa[static_cast<int64_t>(b) * lds + m] = scale;
    }
  }
}

// ---------------------------------------------------------------------------------------------
// FP8 KV cache with per-step QKV scale recalibration.  A token's QKV row holds Hq heads of Q, then
// Hkv of K, then Hkv of V (D values each).  k_qkv_amax reduces |x| over each of the three parts
// (warp, then CTA, then one atomicMax per part on the fp32 bit pattern, which orders non-negative
// floats like their values); k_qkv_finalize turns the maxima into s = amax / 448 (1 for zero).
// k_kv_cache_write quantizes Q into a dense buffer and K, V into the cache rows named by the
// token's slot, with the bracket quantizer for an arbitrary fp32 scale (no tie shortcut: every
// ambiguous bracket takes the exact fp64 quotient).
// ---------------------------------------------------------------------------------------------
constexpr int kErrRangeKv = 9;  // FP8Q_ERR_RANGE

__device__ __forceinline__ QParams qparams_scale(float s) {
  QParams p;
  p.s = s;
  p.tie = false;
  p.fast = s >= 0x1.0p-60f && s <= 0x1.0p+100f;
  const float r = rcp_approx(p.fast ? s : 1.0f);
  const float lo = __fmul_rn(r, 0x1.ffffc0p-1f), hi = __fmul_rn(r, 0x1.000020p+0f);
  p.lo2 = make_float2(lo, lo);
  p.hi2 = make_float2(hi, hi);
  return p;
}

// Grid: any number of CTAs of 256 threads; warps take rows, lanes 16-byte chunks of a row.
__global__ void __launch_bounds__(256) k_qkv_amax(const uint16_t *__restrict__ qkv, int64_t ld,
                                                  int64_t T, int cq, int ck, int cv,
                                                  uint32_t *__restrict__ amax3) {
  __shared__ float red[8][3];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int cw = cq + ck + cv;  // 16-byte chunks per row; Q chunks [0, cq), K [cq, cq + ck)
  uint32_t m[3] = {0u, 0u, 0u};
  const int64_t wstride = static_cast<int64_t>(gridDim.x) * 8;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * 8 + warp; t < T; t += wstride) {
    const uint16_t *row = qkv + t * ld;
#pragma unroll 8
    for (int c = lane; c < cw; c += 32) {
      const uint4 v = ld_stream_v4(row + c * 8);
      const int part = c < cq ? 0 : (c < cq + ck ? 1 : 2);
      const uint32_t a = absmax_uint4(0u, v);
      m[0] = part == 0 ? absmax_bf16x2(m[0], a) : m[0];
      m[1] = part == 1 ? absmax_bf16x2(m[1], a) : m[1];
      m[2] = part == 2 ? absmax_bf16x2(m[2], a) : m[2];
    }
  }
  float f[3];
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    f[i] = absmax_finish(m[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) f[i] = fmaxf(f[i], __shfl_xor_sync(0xffffffffu, f[i], o));
  }
  if (lane == 0) {
#pragma unroll
    for (int i = 0; i < 3; ++i) red[warp][i] = f[i];
  }
  __syncthreads();
  if (threadIdx.x < 3) {
    float v = red[0][threadIdx.x];
    for (int w = 1; w < 8; ++w) v = fmaxf(v, red[w][threadIdx.x]);
    atomicMax(amax3 + threadIdx.x, __float_as_uint(v));
  }
}

__global__ void k_qkv_finalize(const uint32_t *__restrict__ amax3, float *__restrict__ scale3) {
  if (threadIdx.x < 3) {
    const float a = __uint_as_float(amax3[threadIdx.x]);
    scale3[threadIdx.x] = a == 0.0f ? 1.0f : __fdiv_rn(a, 448.0f);
  }
}

// Grid: CTAs of 128 threads, one token at a time per CTA; each thread loads up to 8 of the
// token's 16-byte chunks before it converts any, so a token's loads are all in flight together.
// A slot outside [0, num_slots) other than a negative one, or a scale that is not positive and
// finite, records FP8Q_ERR_RANGE; the token's cache rows (for a bad scale: that part) are not
// written.
constexpr int kKvThreads = 128, kKvBatch = 8;
__global__ void __launch_bounds__(kKvThreads) k_kv_cache_write(
    const uint16_t *__restrict__ qkv, int64_t ld, int64_t T, int cq, int ckv,
    const int64_t *__restrict__ slots, int64_t num_slots, const float *__restrict__ scale3,
    uint8_t *__restrict__ q_out, int64_t ldq, uint8_t *__restrict__ k_cache,
    uint8_t *__restrict__ v_cache) {
  const float sq = __ldg(scale3), sk = __ldg(scale3 + 1), sv = __ldg(scale3 + 2);
  const bool okq = sq > 0.0f && sq <= 0x1.fffffep+127f, okk = sk > 0.0f && sk <= 0x1.fffffep+127f,
             okv = sv > 0.0f && sv <= 0x1.fffffep+127f;
  const QParams pq = qparams_scale(okq ? sq : 1.0f), pk = qparams_scale(okk ? sk : 1.0f),
                pv = qparams_scale(okv ? sv : 1.0f);
  if (!(okq && okk && okv) && blockIdx.x == 0 && threadIdx.x == 0) record_error(kErrRangeKv);
  const int cw = cq + 2 * ckv;
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    const uint16_t *row = qkv + t * ld;
    const int64_t slot = __ldg(slots + t);
    const bool cached = slot >= 0 && slot < num_slots;
    if (slot >= num_slots && threadIdx.x == 0) record_error(kErrRangeKv);
    const bool do_q = q_out != nullptr && okq, do_k = cached && okk, do_v = cached && okv;
    for (int base = 0; base < cw; base += kKvBatch * kKvThreads) {
      uint4 v[kKvBatch];
#pragma unroll
      for (int j = 0; j < kKvBatch; ++j) {
        const int c = base + j * kKvThreads + threadIdx.x;
        const bool want = c < cq ? do_q : (c < cq + ckv ? do_k : do_v);
        if (c < cw && want) v[j] = ld_stream_v4(row + c * 8);
      }
#pragma unroll
      for (int j = 0; j < kKvBatch; ++j) {
        const int c = base + j * kKvThreads + threadIdx.x;
        if (c >= cw) continue;
        if (c < cq) {
          if (do_q) *reinterpret_cast<uint2 *>(q_out + t * ldq + c * 8) = quant8_f32(v[j], pq);
        } else if (c < cq + ckv) {
          if (do_k)
            *reinterpret_cast<uint2 *>(k_cache + slot * (ckv * 8) + (c - cq) * 8) =
                quant8_f32(v[j], pk);
        } else if (do_v) {
          *reinterpret_cast<uint2 *>(v_cache + slot * (ckv * 8) + (c - cq - ckv) * 8) =
              quant8_f32(v[j], pv);
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------------------------
// Self-test of the bounded-wait teardown: the GEMM kernels' roles and helpers, run against a
// barrier that nothing ever arrives on.  Warp 1 allocates TMEM; thread 0 waits on the barrier
// with a short limit, gives up, records FP8Q_ERR_TIMEOUT and raises the abort flag; warps 2-3
// wait (warp-wide) on another barrier that nothing arrives on and leave on the abort flag; TMEM
// is released and the kernel returns.  No fault, no trap: the context stays usable.
// ---------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(128, 1) k_selftest_timeout(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bars[2];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort_store;
  volatile int *s_abort = &s_abort_store;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t b0 = smem_u32(&bars[0]), b1 = smem_u32(&bars[1]);
  if (threadIdx.x == 0) {
    mbar_init(b0, 1);
    mbar_init(b1, 1);
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&s_tmem), 32);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = s_tmem;
  if (warp == 0) {
    if (lane == 0) wait_one(b0, 0, s_abort, limit_ns);   // never completes: times out
    __syncwarp();
  } else if (warp >= 2) {
    // a longer limit: these warps leave because of the abort flag, not their own limit
    wait_warp(b1, 0, s_abort, 10 * limit_ns);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 32);
  }
}

}  // namespace fp8q
