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
//   k_attn_decode_split   one CTA per (chunk of positions, kv head g, sequence b), 128 threads,
//                         the G query heads of g together so every K and V row is read once.  The
//                         cache slots of the chunk's positions are resolved once into shared
//                         memory; the K and V rows of each tile of 64 positions are copied into
//                         shared memory by cp.async, two tiles deep (the next tile's copies run
//                         under this tile's arithmetic).  Each warp takes 16 positions of every
//                         tile with its own online-softmax state:
//                           scores  mma.sync m16n8k16 (fp16 operands, exact for E4M3 codes,
//                                   fp32 accumulation): rows = the G query heads (the rest of the
//                                   16 zero), columns = positions, k = dims in an order that lets
//                                   each lane read whole 32-bit words of a K row;
//                           softmax per head in log2 units: the warp's maximum, weights
//                                   2^(z - m) (exp2f), the rescale of the running state;
//                           values  a second m16n8k16 whose A fragment is the score accumulators
//                                   turned into fp16 weights, B = V (two positions' bytes of one
//                                   dim paired by byte_perm), columns = dims (again permuted).
//                         The four warps' states are merged in shared memory and the chunk's
//                         (m, l, o) per head go to the workspace in fp32.
//   k_attn_decode_combine one CTA per (kv head, sequence): the chunks' states merged in chunk
//                         order, o = s_v num / den, bf16.
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
constexpr int kAttnThreads = 128;   // four warps; also one thread per dim in the merge
constexpr int kAttnTile = 64;       // positions per tile (16 per warp)
constexpr int kAttnMaxChunk = 4096; // positions per split at most

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

// Two E4M3 codes (low byte first) -> f16x2 (low half first), exactly.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t c2) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(static_cast<uint16_t>(c2 & 0xFFFFu)));
  return h2;
}

__device__ __forceinline__ uint32_t f32x2_to_f16x2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  uint32_t r;
  memcpy(&r, &h, 4);
  return r;
}

// d += A B for one m16n8k16 tile: A row-major fp16 (a0: row g, cols 2t..2t+1; a1: row g + 8;
// a2: row g, cols 2t + 8..; a3: row g + 8, cols 2t + 8..), B column-major fp16 (b0: rows 2t..2t+1
// of col g; b1: rows 2t + 8..), fp32 accumulators d (d0, d1: row g, cols 2t, 2t + 1; d2, d3: row
// g + 8), g = lane / 4, t = lane % 4.
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                              uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int G>
__global__ void __launch_bounds__(kAttnThreads) k_attn_decode_split(const AttnArgs a) {
  constexpr int D = kAttnD;
  static_assert(G >= 1 && G <= 8, "the query heads of a group fill at most 8 of the 16 MMA rows");
  extern __shared__ __align__(128) uint8_t s_kv[];   // [stage][K | V][position][D] codes
  int32_t *s_slot = reinterpret_cast<int32_t *>(s_kv + 2 * kAttnStageBytes);  // or -1
  const int s = blockIdx.x, gk = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;               // MMA fragment row group and column pair
  const int L = attn_seq_len(a, b);
  const int j_begin = s * a.chunk;
  if (j_begin >= L) return;                      // an empty chunk: the combine does not read it
  const int j_end = min(L, j_begin + a.chunk);
  const int ntiles = (j_end - j_begin + kAttnTile - 1) / kAttnTile;
  const int64_t row = static_cast<int64_t>(a.Hkv) * D;
  static_assert(kAttnThreads == 2 * kAttnTile, "one thread per K row and one per V row");
  // scores in log2 units: z = c log2(e) q.k, weights 2^(z - m)
  const float c2 = a.sm_scale * a.scale3[0] * a.scale3[1] * 1.4426950408889634f;
  const int64_t nslot_blocks = a.num_slots / a.block_size;

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
  auto stage_tile = [&](int tt) {
    const int p = tid & (kAttnTile - 1), half = tid / kAttnTile;
    const int i = tt * kAttnTile + p;
    const int32_t slot = i < j_end - j_begin ? s_slot[i] : -1;
    const uint32_t dst = smem_u32(s_kv + (tt & 1) * kAttnStageBytes + half * kAttnTile * D + p * D);
    const uint8_t *src = (half ? a.v_cache : a.k_cache) + (slot >= 0 ? slot * row : 0) + gk * D;
    const uint32_t nb = slot >= 0 ? 16u : 0u;
#pragma unroll
    for (int c = 0; c < D / 16; ++c) cp_async16(dst + 16 * c, src + 16 * c, nb);
    asm volatile("cp.async.commit_group;" ::: "memory");
  };

  // Query fragments (A of the score MMAs): row g = query head g of the group (rows >= G and the
  // rows g + 8 are zero).  The 128 dims are taken in an order of our choosing (the sum does not
  // depend on it): in k-step ks, columns 2t, 2t + 1 are dims 16 ks + 4t, + 1 and columns 2t + 8,
  // 2t + 9 are dims 16 ks + 4t + 2, + 3, so each lane reads 4 consecutive codes per row.
  uint32_t qa0[8], qa2[8];
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    uint32_t w = 0u;
    if (g < G)
      w = *reinterpret_cast<const uint32_t *>(a.q + static_cast<int64_t>(b) * a.ldq +
                                              (gk * G + g) * D + 16 * ks + 4 * t);
    qa0[ks] = e4m3x2_to_f16x2(w & 0xFFFFu);
    qa2[ks] = e4m3x2_to_f16x2(w >> 16);
  }

  // Output accumulators (row g = head g): n-tile J = 4 aa + cc, its columns 2t and 2t + 1 are
  // dims 32 aa + 8t + cc and 32 aa + 8t + 4 + cc (again an order that makes each lane's V reads
  // whole 32-bit words).
  float o[16][2];
#pragma unroll
  for (int J = 0; J < 16; ++J) o[J][0] = o[J][1] = 0.0f;
  float m_run = -INFINITY, l_run = 0.0f;               // this lane's part of head g's sum
  const int p0 = 16 * warp;                            // the warp's positions in each tile

  stage_tile(0);
  for (int tt = 0; tt < ntiles; ++tt) {
    const int n = min(kAttnTile, j_end - (j_begin + tt * kAttnTile));
    const int32_t *slots_t = s_slot + tt * kAttnTile;
    if (tt + 1 < ntiles) {
      stage_tile(tt + 1);                                          // in flight during tile tt
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();                                               // tile tt's rows are in place
    const uint8_t *sk = s_kv + (tt & 1) * kAttnStageBytes + p0 * D;
    const uint8_t *sv = sk + kAttnTile * D;
    // scores S[head][position] for the warp's 16 positions (two n-tiles of 8)
    float sc[2][4];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      sc[j][0] = sc[j][1] = sc[j][2] = sc[j][3] = 0.0f;
      const uint8_t *krow = sk + (8 * j + g) * D + 4 * t;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t w = *reinterpret_cast<const uint32_t *>(krow + 16 * ks);
        mma_f16_16816(sc[j], qa0[ks], 0u, qa2[ks], 0u, e4m3x2_to_f16x2(w & 0xFFFFu),
                      e4m3x2_to_f16x2(w >> 16));
      }
    }
    // online softmax for head g over the warp's positions 8j + 2t + e
    float z[2][2], mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int ip = p0 + 8 * j + 2 * t + e;
        const bool valid = g < G && ip < n && slots_t[ip] >= 0;
        z[j][e] = valid ? sc[j][e] * c2 : -INFINITY;
        mx = fmaxf(mx, z[j][e]);
      }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float m_new = fmaxf(m_run, mx);
    const float alpha = m_new == -INFINITY ? 1.0f : exp2f(m_run - m_new);
    float pw[2][2], psum = 0.0f;
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        pw[j][e] = z[j][e] == -INFINITY ? 0.0f : exp2f(z[j][e] - m_new);
        psum += pw[j][e];
      }
    l_run = fmaf(l_run, alpha, psum);
    m_run = m_new;
#pragma unroll
    for (int J = 0; J < 16; ++J) {
      o[J][0] *= alpha;
      o[J][1] *= alpha;
    }
    // weights as the A fragment of the value MMA (k = the warp's 16 positions): columns 2t, 2t + 1
    // are positions 2t, 2t + 1 (n-tile 0 of the scores), columns 2t + 8, 2t + 9 are 8 + 2t, 9 + 2t
    const uint32_t pa0 = f32x2_to_f16x2(pw[0][0], pw[0][1]);
    const uint32_t pa2 = f32x2_to_f16x2(pw[1][0], pw[1][1]);
    // values: B[position][dim], four dims of two positions per pair of 32-bit reads
#pragma unroll
    for (int aa = 0; aa < 4; ++aa) {
      const uint8_t *vcol = sv + 32 * aa + 4 * g;
      const uint32_t w0 = *reinterpret_cast<const uint32_t *>(vcol + (2 * t) * D);
      const uint32_t w1 = *reinterpret_cast<const uint32_t *>(vcol + (2 * t + 1) * D);
      const uint32_t w2 = *reinterpret_cast<const uint32_t *>(vcol + (2 * t + 8) * D);
      const uint32_t w3 = *reinterpret_cast<const uint32_t *>(vcol + (2 * t + 9) * D);
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        const uint32_t sel = static_cast<uint32_t>(cc | ((cc + 4) << 4));
        float d[4] = {o[4 * aa + cc][0], o[4 * aa + cc][1], 0.0f, 0.0f};
        mma_f16_16816(d, pa0, 0u, pa2, 0u, e4m3x2_to_f16x2(__byte_perm(w0, w1, sel)),
                      e4m3x2_to_f16x2(__byte_perm(w2, w3, sel)));
        o[4 * aa + cc][0] = d[0];
        o[4 * aa + cc][1] = d[1];
      }
    }
    __syncthreads();  // the stage is rewritten by the copies of tile tt + 2
  }

  // merge the four warps' states (the stage memory is free now) and write the chunk's partial
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
  float *s_m = reinterpret_cast<float *>(s_kv);                // [4][8]
  float *s_l = s_m + 32;                                        // [4][8]
  float *s_o = s_l + 32;                                        // [4][8][D]
  if (g < G) {
    if (t == 0) {
      s_m[warp * 8 + g] = m_run;
      s_l[warp * 8 + g] = l_run;
    }
#pragma unroll
    for (int aa = 0; aa < 4; ++aa)
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        s_o[(warp * 8 + g) * D + 32 * aa + 8 * t + cc] = o[4 * aa + cc][0];
        s_o[(warp * 8 + g) * D + 32 * aa + 8 * t + 4 + cc] = o[4 * aa + cc][1];
      }
  }
  __syncthreads();
  float *part = a.ws + ((static_cast<int64_t>(b) * a.Hkv + gk) * a.nsplit + s) * (G * (D + 2));
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, s_m[w * 8 + h]);
    float acc = 0.0f, lsum = 0.0f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float mw = s_m[w * 8 + h];
        if (mw == -INFINITY) continue;
        const float f = exp2f(mw - M);
        acc = fmaf(f, s_o[(w * 8 + h) * D + tid], acc);
        lsum = fmaf(f, s_l[w * 8 + h], lsum);
      }
    }
    part[h * (D + 2) + tid] = acc;
    if (tid == 0) {
      part[h * (D + 2) + D] = M;
      part[h * (D + 2) + D + 1] = lsum;
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
  // one pass over the chunks in order, merging each into a running (M, num, den); m is in log2
  // units (the split kernel's scores)
  float M[G], num[G], den[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    M[h] = -INFINITY;
    num[h] = den[h] = 0.0f;
  }
#pragma unroll 2
  for (int s = 0; s < ns; ++s) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float *p = base + s * (G * (D + 2)) + h * (D + 2);
      const float ms = p[D], ls = p[D + 1], os = p[tid];
      if (ms == -INFINITY) continue;
      if (ms > M[h]) {
        const float f = exp2f(M[h] - ms);                  // 0 while M is still -inf
        num[h] *= f;
        den[h] *= f;
        M[h] = ms;
      }
      const float f = exp2f(ms - M[h]);
      num[h] = fmaf(f, os, num[h]);
      den[h] = fmaf(f, ls, den[h]);
    }
  }
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const float o = den[h] > 0.0f ? sv * (num[h] / den[h]) : 0.0f;
    const __nv_bfloat16 ob = __float2bfloat16_rn(o);
    a.out[static_cast<int64_t>(b) * a.ldo + (g * G + h) * D + tid] =
        *reinterpret_cast<const uint16_t *>(&ob);
  }
}

}  // namespace fp8q
