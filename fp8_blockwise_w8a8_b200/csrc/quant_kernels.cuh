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

__device__ __forceinline__ float amax_word(float m, uint32_t w) {
  return fmaxf(m, fmaxf(fabsf(bf16_lo(w)), fabsf(bf16_hi(w))));
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

// Per-block quantization parameters.  mode 0: codes = cvt(x * inv) exactly (power-of-two
// scale); mode 1: fast path x * rcp with a bracket check, exact division when the bracket
// straddles a rounding boundary; mode 2: exact division for every element.
struct QParams {
  float s;     // the scale (divisor)
  float mul;   // 1/s: exact for powers of two, RN(1/s) otherwise
  int mode;
};

__device__ __forceinline__ QParams qparams_f32(float amax) {
  QParams p;
  p.s = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 448.0f);
  p.mul = __fdiv_rn(1.0f, p.s);
  // The bracket argument needs 1/s finite and products far from the subnormal range.
  p.mode = (p.s >= 0x1.0p-100f) ? 1 : 2;
  return p;
}

__device__ __forceinline__ QParams qparams_pow2(int e) {
  QParams p;
  p.s = pow2_f32(e);
  p.mul = pow2_f32(-e);  // exact: x * 2^-e == x / 2^e, each rounded once
  p.mode = 0;
  return p;
}

// Two E4M3 codes for RN_fp32(x0 / s), RN_fp32(x1 / s) (low byte = x0).
//
// Fast path: t = RN(x * RN(1/s)) is within (1 + 2^-24)^2 of x/s; t * (1 -+ 2^-20) (rounded)
// then bracket x/s strictly, and RN_fp32 and the E4M3 conversion are both monotone, so when
// both bracket ends give the same code that code is the exact one.  Otherwise (x/s within about
// 2^-20 of an E4M3 rounding boundary) the pair is redone with IEEE divisions.
__device__ __forceinline__ uint16_t quant_pair(float x0, float x1, const QParams &p) {
  if (p.mode == 0) return cvt_e4m3x2(__fmul_rn(x0, p.mul), __fmul_rn(x1, p.mul));
  if (p.mode == 1) {
    const float t0 = __fmul_rn(x0, p.mul), t1 = __fmul_rn(x1, p.mul);
    const uint16_t lo = cvt_e4m3x2(__fmul_rn(t0, 0x1.ffffe0p-1f), __fmul_rn(t1, 0x1.ffffe0p-1f));
    const uint16_t hi = cvt_e4m3x2(__fmul_rn(t0, 0x1.000010p+0f), __fmul_rn(t1, 0x1.000010p+0f));
    if (lo == hi) return lo;
  }
  return cvt_e4m3x2(__fdiv_rn(x0, p.s), __fdiv_rn(x1, p.s));
}

// 8 bf16 values (one uint4) -> 8 codes (one uint2).
__device__ __forceinline__ uint2 quant8_bf16(const uint4 v, const QParams &p) {
  const uint32_t c0 = quant_pair(bf16_lo(v.x), bf16_hi(v.x), p);
  const uint32_t c1 = quant_pair(bf16_lo(v.y), bf16_hi(v.y), p);
  const uint32_t c2 = quant_pair(bf16_lo(v.z), bf16_hi(v.z), p);
  const uint32_t c3 = quant_pair(bf16_lo(v.w), bf16_hi(v.w), p);
  return make_uint2(c0 | (c1 << 16), c2 | (c3 << 16));
}

// ---------------------------------------------------------------------------------------------
// 128x128 weight blocks.  One CTA (256 threads) per block: thread t owns the 16-byte column
// chunk (t % 16) of rows (t / 16) + 16 i, i = 0..7, so every load and store instruction of a
// warp covers two full 256-byte (load) / 128-byte (store) row segments.
// ---------------------------------------------------------------------------------------------
template <int FMT>
__global__ void __launch_bounds__(256) k_quant_weight_block(const uint16_t *__restrict__ w,
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
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      amax = amax_word(amax, v[i].x);
      amax = amax_word(amax, v[i].y);
      amax = amax_word(amax, v[i].z);
      amax = amax_word(amax, v[i].w);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if (lane == 0) red[warp] = amax;
    __syncthreads();
    amax = red[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) amax = fmaxf(amax, red[i]);
    __syncthreads();  // red[] is rewritten by the next block
    QParams p;
    if (FMT == kScaleF32) {
      p = qparams_f32(amax);
      if (tid == 0) static_cast<float *>(sw)[blk] = p.s;
    } else {
      const int e = e8m0_exponent(amax);
      p = qparams_pow2(e);
      if (tid == 0) static_cast<uint8_t *>(sw)[blk] = static_cast<uint8_t>(e + 127);
    }
    uint8_t *dst = q + (nb * 128 + r0) * ldq + kb * 128 + c8;
#pragma unroll
    for (int i = 0; i < 8; ++i)
      *reinterpret_cast<uint2 *>(dst + static_cast<int64_t>(i) * 16 * ldq) = quant8_bf16(v[i], p);
  }
}

// ---------------------------------------------------------------------------------------------
// 1x128 token groups, optionally preceded by RMSNorm.  One warp per row at a time; rows are
// double-buffered in shared memory with cp.async so the next row streams in while the current
// one is processed.  Shared layout of a row: 128-element blocks at a 272-byte stride (256 bytes
// of data + 16 bytes of padding), so that lane b reading its own block b sequentially (the RMS
// sum of squares) hits distinct banks.  gamma uses the same layout, once per CTA.
// ---------------------------------------------------------------------------------------------
constexpr int kRowBlockStride = 272;

__device__ __forceinline__ void cp_async_16(uint32_t dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_1() {
  asm volatile("cp.async.wait_group 1;" ::: "memory");
}

__device__ __forceinline__ void load_row_async(uint32_t dst, const uint16_t *src, int K,
                                               int lane) {
  const int chunks = K >> 3;  // 16-byte chunks
  for (int j = lane; j < chunks; j += 32)
    cp_async_16(dst + (j >> 4) * kRowBlockStride + (j & 15) * 16, src + j * 8);
}

template <bool NORM>
__global__ void __launch_bounds__(128) k_rmsnorm_quant_token(
    const uint16_t *__restrict__ x, int64_t ldx, const uint16_t *__restrict__ gamma, float eps,
    int64_t M, int K, uint8_t *__restrict__ q, int64_t ldq, float *__restrict__ sa, int64_t lds) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int wpc = blockDim.x >> 5;
  const int KB = K >> 7;
  const int row_bytes = KB * kRowBlockStride;
  uint8_t *g_s = smem;                                     // gamma (NORM only)
  uint8_t *buf0 = smem + (NORM ? row_bytes : 0) + warp * 2 * row_bytes;
  const uint32_t buf_u32[2] = {smem_u32(buf0), smem_u32(buf0 + row_bytes)};

  if (NORM) {
    const int chunks = K >> 3;
    for (int j = threadIdx.x; j < chunks; j += blockDim.x)
      *reinterpret_cast<uint4 *>(g_s + (j >> 4) * kRowBlockStride + (j & 15) * 16) =
          *reinterpret_cast<const uint4 *>(gamma + j * 8);
    __syncthreads();
  }

  const int64_t stride = static_cast<int64_t>(gridDim.x) * wpc;
  int64_t m = static_cast<int64_t>(blockIdx.x) * wpc + warp;
  if (m < M) load_row_async(buf_u32[0], x + m * ldx, K, lane);
  cp_async_commit();
  const int half = lane >> 4, hl = lane & 15;
  for (int it = 0; m < M; m += stride, ++it) {
    const int cur = it & 1;
    const int64_t next = m + stride;
    if (next < M) load_row_async(buf_u32[cur ^ 1], x + next * ldx, K, lane);
    cp_async_commit();
    cp_async_wait_1();
    __syncwarp();
    const uint8_t *row = cur ? buf0 + row_bytes : buf0;

    float r = 1.0f;
    if (NORM) {
      // Sum of squares in fp64: each lane walks its own 128-blocks in ascending k ...
      double P[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        P[i] = 0.0;
        const int b = lane + 32 * i;
        if (b < KB) {
          const uint4 *blk = reinterpret_cast<const uint4 *>(row + b * kRowBlockStride);
          double acc = 0.0;
#pragma unroll 4
          for (int c = 0; c < 16; ++c) {
            const uint4 v = blk[c];
            const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const double a = static_cast<double>(bf16_lo(wv[j]));
              acc = __fma_rn(a, a, acc);  // a*a is exact in fp64, so this is RN(acc + a*a)
              const double b2 = static_cast<double>(bf16_hi(wv[j]));
              acc = __fma_rn(b2, b2, acc);
            }
          }
          P[i] = acc;
        }
      }
      // ... then the block sums are added in ascending block order.
      double S = 0.0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (32 * i >= KB) break;
        for (int j = 0; j < 32; ++j) {
          const double pj = __shfl_sync(0xffffffffu, P[i], j);
          if (32 * i + j < KB) S = __dadd_rn(S, pj);
        }
      }
      const double var = __dadd_rn(__ddiv_rn(S, static_cast<double>(K)), static_cast<double>(eps));
      r = __double2float_rn(__ddiv_rn(1.0, __dsqrt_rn(var)));
    }

    // Quantize two 128-blocks per step: lanes 0-15 take block 2j, lanes 16-31 block 2j + 1;
    // each lane owns 8 consecutive elements.
    for (int b0 = 0; b0 < KB; b0 += 2) {
      const int b = b0 + half;
      const bool active = b < KB;
      const int bb = active ? b : b0;
      uint4 v = *reinterpret_cast<const uint4 *>(row + bb * kRowBlockStride + hl * 16);
      if (NORM) {
        const uint4 g = *reinterpret_cast<const uint4 *>(g_s + bb * kRowBlockStride + hl * 16);
        const uint32_t xv[4] = {v.x, v.y, v.z, v.w};
        const uint32_t gv[4] = {g.x, g.y, g.z, g.w};
        uint32_t yv[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float y0 = __fmul_rn(__fmul_rn(bf16_lo(xv[j]), r), bf16_lo(gv[j]));
          const float y1 = __fmul_rn(__fmul_rn(bf16_hi(xv[j]), r), bf16_hi(gv[j]));
          const __nv_bfloat162 yy = __floats2bfloat162_rn(y0, y1);
          yv[j] = *reinterpret_cast<const uint32_t *>(&yy);
        }
        v = make_uint4(yv[0], yv[1], yv[2], yv[3]);
      }
      float amax = 0.0f;
      amax = amax_word(amax, v.x);
      amax = amax_word(amax, v.y);
      amax = amax_word(amax, v.z);
      amax = amax_word(amax, v.w);
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      const QParams p = qparams_f32(amax);
      const uint2 codes = quant8_bf16(v, p);
      if (active) {
        *reinterpret_cast<uint2 *>(q + m * ldq + b * 128 + hl * 8) = codes;
        if (hl == 0) sa[static_cast<int64_t>(b) * lds + m] = p.s;
      }
    }
    __syncwarp();  // every lane is done with this buffer before it is refilled
  }
}

}  // namespace fp8q
