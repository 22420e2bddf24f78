// attn_kernels.cuh -- decode attention over the FP8 (E4M3) KV cache, for sm_100a.
//
// For sequence b (one query token) and query head h, kv head g = h / G (G = Hq / Hkv query heads
// share one kv head), over the sequence's L cached positions j (slot = block_table[b][j / bs] * bs
// + j % bs of a paged cache whose rows hold Hkv heads of D codes):
//   z_j = c * sum_d dec(q[h][d]) dec(k_j[g][d]),   c = sm_scale * s_q * s_k
//   o[h][d] = s_v * sum_j softmax(z)_j dec(v_j[g][d])   -> bf16
// (scaled dot-product attention on the dequantized tensors; FP8-RL abstract, item (ii): the FP8
// KV cache written with per-tensor scales by fp8q_kv_cache_write).
//
// Two kernels ("split-KV"):
//   k_attn_decode_split   one CTA per (chunk of C positions, kv head g, sequence b), 128 threads,
//                         the G query heads of g together so every K and V row is read once.  The
//                         cache slots of the chunk's positions are resolved once into shared
//                         memory; the K and V rows of each tile of 64 positions are copied into
//                         shared memory by cp.async, two tiles deep (the next tile's copies run
//                         under this tile's arithmetic).  Per tile:
//                           scores  8 lanes per position, lane `sub` holding dims 16 sub .. 16 sub
//                                   + 15 of the G query rows in registers; each lane dequantizes
//                                   its 16 bytes of the K row (cvt e4m3x2 -> f16x2 -> f32), takes
//                                   G partial dot products in fp32 and the 8 lanes add them;
//                           softmax running maximum and sum per head (online softmax): the tile's
//                                   weights exp(z - m) and the rescale exp(m_old - m_new), expf;
//                           values  thread t owns dim t of the G heads' fp32 accumulators and adds
//                                   p_j dec(v_j[g][t]) for the tile's positions.
//                         The chunk's (m, l, o) per head go to the workspace in fp32.
//   k_attn_decode_combine one CTA per (kv head, sequence): o = s_v sum_s e^(m_s - M) o_s /
//                         sum_s e^(m_s - M) l_s over the sequence's chunks (in chunk order), bf16.
// A block id outside the cache, or a sequence length outside [0, max_seq_len], records
// FP8Q_ERR_RANGE (9) in the device error word; such positions are skipped and such lengths are
// clamped, so no access leaves the buffers.
#pragma once
#include <cstdint>
#include <cstring>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include "ptx.cuh"

namespace fp8q {

constexpr int kAttnD = 128;         // head dimension handled
constexpr int kAttnThreads = 128;   // one thread per output dim in the value pass
constexpr int kAttnTile = 64;       // positions per tile
constexpr int kAttnMaxChunk = 4096; // positions per split at most
constexpr int kAttnLPP = kAttnD / 16;                 // lanes per position in the score pass
constexpr int kAttnPPR = (kAttnThreads / 32) * (32 / kAttnLPP);  // positions per score round

struct AttnArgs {
  const uint8_t *q;          // [B][ldq] codes
  int64_t ldq;
  const uint8_t *k_cache;    // [num_slots][Hkv * D]
  const uint8_t *v_cache;
  int64_t num_slots;
  const float *scale3;       // s_q, s_k, s_v (device)
  const int32_t *block_table;  // [B][max_blocks]
  int64_t max_blocks;
  const int32_t *seq_lens;   // [B]
  int Hq, Hkv, block_size;
  int max_seq_len;
  int chunk;                 // positions per split (a multiple of kAttnTile)
  int nsplit;                // splits per sequence, ceil(max_seq_len / chunk)
  float sm_scale;
  float *ws;                 // [B][Hkv][nsplit][G][D + 2] fp32: o, then m, l
  uint16_t *out;             // [B][ldo] bf16
  int64_t ldo;
};

// Two E4M3 codes (low byte first) -> two fp32 values, exactly (E4M3 is a subset of fp16).
__device__ __forceinline__ float2 e4m3x2_to_f32x2(uint16_t c2) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(c2));
  __half2 hv;
  memcpy(&hv, &h2, 4);
  return __half22float2(hv);
}

__device__ __forceinline__ int attn_seq_len(const AttnArgs &a, int b) {
  int L = a.seq_lens[b];
  if (L < 0 || L > a.max_seq_len) {
    record_error(9 /* FP8Q_ERR_RANGE */);
    L = L < 0 ? 0 : a.max_seq_len;
  }
  return L;
}

// Dynamic shared memory of k_attn_decode_split: two stages of a tile's K and V rows, then the
// cache slot of every position of the chunk.
constexpr int kAttnStageBytes = 2 * kAttnTile * kAttnD;
constexpr int kAttnSmem = 2 * kAttnStageBytes + kAttnMaxChunk * 4;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}

template <int G>
__global__ void __launch_bounds__(kAttnThreads) k_attn_decode_split(const AttnArgs a) {
  constexpr int D = kAttnD;
  extern __shared__ __align__(128) uint8_t s_kv[];   // [stage][K | V][position][D] codes
  int32_t *s_slot = reinterpret_cast<int32_t *>(s_kv + 2 * kAttnStageBytes);  // or -1
  __shared__ float s_z[G][kAttnTile];
  __shared__ __align__(16) float s_p[kAttnTile][G];
  __shared__ float s_red[4][G];
  const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int L = attn_seq_len(a, b);
  const int j_begin = s * a.chunk;
  if (j_begin >= L) return;                      // an empty chunk: the combine does not read it
  const int j_end = min(L, j_begin + a.chunk);
  const int ntiles = (j_end - j_begin + kAttnTile - 1) / kAttnTile;
  const int64_t row = static_cast<int64_t>(a.Hkv) * D;
  static_assert(kAttnThreads == 2 * kAttnTile, "one thread per K row and one per V row");
  const float c = a.sm_scale * a.scale3[0] * a.scale3[1];
  const int64_t nslot_blocks = a.num_slots / a.block_size;

  // this lane's 16 dims of the G query rows, decoded
  const int sub = lane % kAttnLPP;
  float2 qr[G][8];  // dims (2i, 2i + 1) of this lane's 16
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const uint4 qc = *reinterpret_cast<const uint4 *>(a.q + static_cast<int64_t>(b) * a.ldq +
                                                      (g * G + h) * D + 16 * sub);
    const uint32_t w[4] = {qc.x, qc.y, qc.z, qc.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      qr[h][2 * i] = e4m3x2_to_f32x2(static_cast<uint16_t>(w[i] & 0xFFFFu));
      qr[h][2 * i + 1] = e4m3x2_to_f32x2(static_cast<uint16_t>(w[i] >> 16));
    }
  }

  // The cache slot of every position of the chunk (-1 where the block id is bad).
  for (int i = tid; i < j_end - j_begin; i += kAttnThreads) {
    const int j = j_begin + i;
    const int64_t blk = a.block_table[static_cast<int64_t>(b) * a.max_blocks + j / a.block_size];
    int32_t slot = -1;
    if (blk >= 0 && blk < nslot_blocks)
      slot = static_cast<int32_t>(blk * a.block_size + j % a.block_size);
    else
      record_error(9 /* FP8Q_ERR_RANGE */);
    s_slot[i] = slot;
  }
  __syncthreads();
  // Tile t's K rows (threads 0..63, one position each) and V rows (threads 64..127) into stage
  // t & 1 by 16-byte cp.async, zero-filled for a position that is not read.
  auto stage_tile = [&](int t) {
    const int p = tid & (kAttnTile - 1), half = tid / kAttnTile;
    const int i = t * kAttnTile + p;
    const int32_t slot = i < j_end - j_begin ? s_slot[i] : -1;
    const uint32_t dst = smem_u32(s_kv + (t & 1) * kAttnStageBytes + half * kAttnTile * D + p * D);
    const uint8_t *src = (half ? a.v_cache : a.k_cache) + (slot >= 0 ? slot * row : 0) + g * D;
    const uint32_t nb = slot >= 0 ? 16u : 0u;
#pragma unroll
    for (int c = 0; c < D / 16; ++c) cp_async16(dst + 16 * c, src + 16 * c, nb);
    asm volatile("cp.async.commit_group;" ::: "memory");
  };

  float m_run[G], l_run[G], acc[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m_run[h] = -INFINITY;
    l_run[h] = 0.0f;
    acc[h] = 0.0f;
  }

  stage_tile(0);
  for (int t = 0; t < ntiles; ++t) {
    const int n = min(kAttnTile, j_end - (j_begin + t * kAttnTile));
    const int32_t *slots_t = s_slot + t * kAttnTile;
    if (t + 1 < ntiles) {
      stage_tile(t + 1);                                          // in flight during tile t
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();                                              // tile t's rows are in place
    const uint8_t *sk = s_kv + (t & 1) * kAttnStageBytes;
    const uint8_t *sv = sk + kAttnTile * D;
    // scores: round r, warp w, lane group -> tile position r * PPR + w * (32 / LPP) + lane / LPP
    for (int r = 0; r < kAttnTile / kAttnPPR; ++r) {
      const int jt = r * kAttnPPR + warp * (32 / kAttnLPP) + lane / kAttnLPP;
      const bool valid = jt < n && slots_t[jt] >= 0;
      float2 z2[G];  // even and odd dims summed apart (packed fp32x2 FMAs)
#pragma unroll
      for (int h = 0; h < G; ++h) z2[h] = make_float2(0.0f, 0.0f);
      const uint4 kc = *reinterpret_cast<const uint4 *>(sk + jt * D + 16 * sub);
      const uint32_t w[4] = {kc.x, kc.y, kc.z, kc.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 lo = e4m3x2_to_f32x2(static_cast<uint16_t>(w[i] & 0xFFFFu));
        const float2 hi = e4m3x2_to_f32x2(static_cast<uint16_t>(w[i] >> 16));
#pragma unroll
        for (int h = 0; h < G; ++h) {
          z2[h] = __ffma2_rn(qr[h][2 * i], lo, z2[h]);
          z2[h] = __ffma2_rn(qr[h][2 * i + 1], hi, z2[h]);
        }
      }
      float z[G];
#pragma unroll
      for (int h = 0; h < G; ++h) z[h] = z2[h].x + z2[h].y;
#pragma unroll
      for (int o = kAttnLPP / 2; o > 0; o >>= 1)
#pragma unroll
        for (int h = 0; h < G; ++h) z[h] += __shfl_xor_sync(0xffffffffu, z[h], o);
      if (sub == 0)
#pragma unroll
        for (int h = 0; h < G; ++h) s_z[h][jt] = valid ? c * z[h] : -INFINITY;
    }
    __syncthreads();
    // online softmax: the tile's maximum per head, its weights, the rescale of the running state
    float zt[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      zt[h] = tid < kAttnTile ? s_z[h][tid] : -INFINITY;
      float v = zt[h];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
      if (lane == 0) s_red[warp][h] = v;
    }
    __syncthreads();
    float alpha[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float mt = fmaxf(fmaxf(s_red[0][h], s_red[1][h]), fmaxf(s_red[2][h], s_red[3][h]));
      const float m_new = fmaxf(m_run[h], mt);
      // no finite score yet: nothing to weigh or rescale
      alpha[h] = m_new == -INFINITY ? 1.0f : expf(m_run[h] - m_new);
      if (tid < kAttnTile) s_p[tid][h] = zt[h] == -INFINITY ? 0.0f : expf(zt[h] - m_new);
      m_run[h] = m_new;
    }
    __syncthreads();  // s_red is reused below; s_p complete
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float v = tid < kAttnTile ? s_p[tid][h] : 0.0f;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) s_red[warp][h] = v;
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float tsum = (s_red[0][h] + s_red[1][h]) + (s_red[2][h] + s_red[3][h]);
      l_run[h] = fmaf(l_run[h], alpha[h], tsum);
      acc[h] *= alpha[h];
    }
    // values: this thread's dim of the tile's positions, two positions per step (their two
    // bytes converted together).  Positions past n hold zero rows and zero weights.
    const int n2 = (n + 1) & ~1;
#pragma unroll 4
    for (int jt = 0; jt < n2; jt += 2) {
      const uint16_t c2 = static_cast<uint16_t>(sv[jt * D + tid]) |
                          static_cast<uint16_t>(static_cast<uint16_t>(sv[(jt + 1) * D + tid]) << 8);
      const float2 v = e4m3x2_to_f32x2(c2);
      if constexpr (G == 1) {
        acc[0] = fmaf(s_p[jt][0], v.x, acc[0]);
        acc[0] = fmaf(s_p[jt + 1][0], v.y, acc[0]);
      } else {
#pragma unroll
        for (int h = 0; h < G; h += 2) {
          float2 a2 = make_float2(acc[h], acc[h + 1]);
          a2 = __ffma2_rn(make_float2(s_p[jt][h], s_p[jt][h + 1]), make_float2(v.x, v.x), a2);
          a2 = __ffma2_rn(make_float2(s_p[jt + 1][h], s_p[jt + 1][h + 1]), make_float2(v.y, v.y),
                          a2);
          acc[h] = a2.x;
          acc[h + 1] = a2.y;
        }
      }
    }
    __syncthreads();  // the stage, s_z, s_p and s_red are rewritten by the next tiles
  }
  // the chunk's partial state
  float *part = a.ws + ((static_cast<int64_t>(b) * a.Hkv + g) * a.nsplit + s) * (G * (D + 2));
#pragma unroll
  for (int h = 0; h < G; ++h) {
    part[h * (D + 2) + tid] = acc[h];
    if (tid == 0) {
      part[h * (D + 2) + D] = m_run[h];
      part[h * (D + 2) + D + 1] = l_run[h];
    }
  }
}

template <int G>
__global__ void __launch_bounds__(kAttnThreads) k_attn_decode_combine(const AttnArgs a) {
  constexpr int D = kAttnD;
  const int g = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int L = min(max(a.seq_lens[b], 0), a.max_seq_len);  // the split kernel recorded errors
  const int ns = (L + a.chunk - 1) / a.chunk;
  const float sv = a.scale3[2];
  const float *base = a.ws + (static_cast<int64_t>(b) * a.Hkv + g) * a.nsplit * (G * (D + 2));
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float M = -INFINITY;
    for (int s = 0; s < ns; ++s) M = fmaxf(M, base[s * (G * (D + 2)) + h * (D + 2) + D]);
    float num = 0.0f, den = 0.0f;
    if (M != -INFINITY) {
      for (int s = 0; s < ns; ++s) {
        const float *p = base + s * (G * (D + 2)) + h * (D + 2);
        if (p[D] == -INFINITY) continue;
        const float w = expf(p[D] - M);
        num = fmaf(w, p[tid], num);
        den = fmaf(w, p[D + 1], den);
      }
    }
    const float o = den > 0.0f ? sv * (num / den) : 0.0f;
    const __nv_bfloat16 ob = __float2bfloat16_rn(o);
    a.out[static_cast<int64_t>(b) * a.ldo + (g * G + h) * D + tid] =
        *reinterpret_cast<const uint16_t *>(&ob);
  }
}

}  // namespace fp8q
