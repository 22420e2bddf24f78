// gemm_kernel.cuh -- block-scaled FP8 (E4M3) W8A8 GEMM for sm_100a, dense and grouped (MoE).
//
//   out[m, n] = bf16( sum_kb sa[m, kb] * sw[n / 128, kb] * P_kb[m, n] )
//
// P_kb, the dot product of the E4M3 codes over one 128-wide K-block, is computed by tcgen05.mma
// (kind::f8f6f4, fp32 accumulate) into tensor memory; the scale product is applied and the
// partials are accumulated in fp32 registers ("promotion") by the epilogue warps.
//
// Structure (one persistent CTA per SM, 384 threads = 3 warpgroups):
//   warp 0      TMA producer (lane 0): A tile 128 x 128 B and B tile 256 x 128 B per K-block into
//               a 4-stage shared-memory ring, 128-byte swizzled
//   warps 1, 3  MMA issuers (lane 0 of each): 4 MMAs (K = 32 each) per K-block into one of two
//               256-column TMEM buffers, so the MMAs of K-block kb + 1 run while the epilogue
//               promotes K-block kb.  Warp 1 issues the even K-blocks (buffer 0), warp 3 the odd
//               ones (buffer 1): one thread's issue cost plus its barrier waits exceed the slack
//               the tensor pipe leaves between K-blocks.  Warp 1 also allocates TMEM.
//   warp 2      scale producer: stages the weight scales of each tile (both 128-column halves,
//               all K-blocks) in shared memory, double-buffered across tiles; grouped: also
//               streams the activation scales of each K-block into a shared ring with cp.async
//               (8 K-blocks ahead)
//   warps 4-11  epilogue/promotion: warp w reads TMEM lanes 32 * (w % 4) (its 32 rows of the
//               tile) and column half (w - 4) / 4; each thread keeps 128 fp32 accumulators and
//               (dense) loads its own row's activation scales from global memory two K-blocks
//               ahead.
//               Per K-block it reads its 128 columns as eight 16-column TMEM loads, promoting
//               each chunk while the next load is in flight (the last chunk under the first load
//               of the next K-block)
// Registers: launched at 168 per thread (384 x 168 = 64512); warpgroup 0 drops to 64 and the two
// epilogue warpgroups rise to 216 (128 x 64 + 256 x 216 = 63488 <= 64512; per sub-partition
// 64 x 32 + 2 x 216 x 32 = 15872 <= 16128).
// Every wait is bounded: on expiry a kernel records FP8Q_ERR_TIMEOUT in the device error word,
// all roles leave their loops, in-flight copies and MMAs are drained, and TMEM is released.
#pragma once
#include <cuda.h>
#include "ptx.cuh"

namespace fp8q {

constexpr int kBM = 128, kBN = 256, kBK = 128;
constexpr int kStages = 4;
constexpr int kGemmThreads = 384;
constexpr int kProducerRegs = 64, kEpilogueRegs = 216;
constexpr int kTileABytes = kBM * kBK;            // 16 KB
constexpr int kTileBBytes = kBN * kBK;            // 32 KB
constexpr int kStageBytes = kTileABytes + kTileBBytes;
constexpr int kStagingBytesPerWarp = 32 * 64;     // 32 rows x 32 bf16 columns
constexpr int kMaxExperts = 1024;

// Shared-memory layout (offsets from a 1024-byte aligned base).
constexpr int kOffA = 0;
constexpr int kOffB = kOffA + kStages * kTileABytes;
constexpr int kOffStaging = kOffB + kStages * kTileBBytes;
constexpr int kSaStages = 8;                      // grouped: K-blocks of activation scales in flight
constexpr int kMaxKB = 256;                       // K <= 32768
constexpr int kOffSa = kOffStaging + 8 * kStagingBytesPerWarp;      // [kSaStages][128] fp32
constexpr int kOffSw = kOffSa + kSaStages * kBM * 4;                // [2 tiles][2 halves][kMaxKB]
constexpr int kOffBar = kOffSw + 2 * 2 * kMaxKB * 4;
// full, empty, tmem_full[2], tmem_empty[2], done, sa_full/empty[kSaStages], sw_full/empty[2]
constexpr int kNumBars = 2 * kStages + 4 + 1 + 2 * kSaStages + 4;
constexpr int kOffMisc = kOffBar + kNumBars * 8;  // tmem base, abort flag
constexpr int kOffGroups = kOffMisc + 16;          // grouped: offsets[E+1], tile prefix[E+1]
constexpr int kGemmSmemDense = kOffGroups + 1024;  // + alignment slack
constexpr int kGemmSmemGrouped = kOffGroups + 2 * (kMaxExperts + 1) * 4 + 1024;

// Shared-memory layout of k_gemm_w8a8_block.  With TS (tile stores by TMA) the operand ring has 3
// stages and each epilogue warp a whole 8 KB output slot (its 32 rows x 128 columns of bf16), so
// a finished tile leaves through the TMA engine while the warps promote the next one.
template <bool TS> struct BlockLayout {
  static constexpr int stages = TS ? 3 : kStages;
  static constexpr int offA = 0;
  static constexpr int offB = offA + stages * kTileABytes;
  static constexpr int offStaging = offB + stages * kTileBBytes;
  static constexpr int stagingPerWarp = TS ? 8192 : kStagingBytesPerWarp;
  static constexpr int offSa = offStaging + 8 * stagingPerWarp;
  static constexpr int offSw = offSa + kSaStages * kBM * 4;
  static constexpr int offBar = offSw + 2 * 2 * kMaxKB * 4;
  static constexpr int numBars = 2 * stages + 4 + 1 + 2 * kSaStages + 4;
  static constexpr int offMisc = offBar + numBars * 8;
  static constexpr int offGroups = offMisc + 16;
  static constexpr int smemDense = offGroups + 1024;
  static constexpr int smemGrouped = offGroups + 2 * (kMaxExperts + 1) * 4 + 1024;
};
static_assert(BlockLayout<true>::smemGrouped <= 227 * 1024, "TMA-store layout exceeds shared memory");
static_assert(BlockLayout<false>::smemGrouped == kGemmSmemGrouped, "layouts differ");

// Instruction descriptor, kind::f8f6f4: D fp32 (bits 4-5 = 1), A and B E4M3 (bits 7-9, 10-12
// = 0), both K-major (bits 15, 16 = 0), N >> 3 in bits 17-22, M >> 4 in bits 24-28.
constexpr uint32_t kIdesc = (1u << 4) | (static_cast<uint32_t>(kBN >> 3) << 17) |
                            (static_cast<uint32_t>(kBM >> 4) << 24);

// Shared-memory matrix descriptor for a K-major tile written by TMA with 128-byte swizzle:
// rows of 128 bytes, 8-row core groups 1024 bytes apart (stride byte offset), descriptor
// version 1 (bit 46), swizzle mode 2 = 128B (bits 61-63).  Start address in 16-byte units.
__device__ __forceinline__ uint64_t sdesc_k128(uint32_t saddr) {
  return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (static_cast<uint64_t>(1) << 16) |
         (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
         (static_cast<uint64_t>(2) << 61);
}

struct GemmArgs {
  const float *sa;
  int64_t lds;
  const void *sw;       // fp32 or E8M0 bytes
  int sw_fmt;
  const int32_t *group_offsets;  // nullptr: dense
  int E;
  int M, N, K;
  uint16_t *out;
  int64_t ldo;
  int num_n;            // ceil(N / 256)
  int num_m;            // dense: ceil(M / 128)
  int group_m;          // dense rasterization: m-blocks per group (>= 1)
  int splits;           // K-splits per tile (1: no split)
  float *ws;            // splits > 1: fp32 partials, [tile][split][2][32][128] float4
  int n_tiles_per_group;  // block-diagonal: 256-column tiles per group (0: plain dense); group
                          // g of the output reads A's K-blocks [g K/128, (g + 1) K/128)
};

// Work unit u covers tile u / splits and the K-blocks [kb0, kb1) of split u % splits.
struct Unit {
  int t, j, kb0, kb1;
};

__device__ __forceinline__ Unit unit_of(const GemmArgs &a, int u, int KB) {
  Unit w;
  w.t = u / a.splits;
  w.j = u - w.t * a.splits;
  w.kb0 = (w.j * KB) / a.splits;
  w.kb1 = ((w.j + 1) * KB) / a.splits;
  return w;
}

struct Tile {
  int m0;        // first row of the tile in A / out
  int row_end;   // rows >= row_end are not stored (M, or the expert's end)
  int n0;        // first column
  int b_row;     // first row of the tile in the B tensor map (expert * N + n0)
  int e;         // expert (0 when dense)
  int a_kb;      // first K-block of the tile's slice of A (block-diagonal groups; else 0)
};

// Dense rasterization: groups of group_m m-blocks, m fastest inside a group, so that the CTAs
// running at the same time share B tiles and the group's A rows stay in L2 while B streams past
// once per group (the host sizes a group's A slice to a fraction of L2).
__device__ __forceinline__ Tile dense_tile(const GemmArgs &a, int t) {
  const int per_group = a.group_m * a.num_n;
  const int g = t / per_group;
  const int first_m = g * a.group_m;
  const int gm = min(a.num_m - first_m, a.group_m);
  const int r = t - g * per_group;
  Tile tl;
  tl.m0 = (first_m + r % gm) * kBM;
  tl.n0 = (r / gm) * kBN;
  tl.row_end = a.M;
  tl.b_row = tl.n0;
  tl.e = 0;
  tl.a_kb = a.n_tiles_per_group ? (tl.n0 / kBN) / a.n_tiles_per_group * (a.K / kBK) : 0;
  return tl;
}

// Grouped: expert e owns m-tiles [prefix[e], prefix[e+1]); n fastest so the CTAs of one expert
// share its weight in L2.
__device__ __forceinline__ Tile grouped_tile(const GemmArgs &a, const int *s_off,
                                             const int *s_prefix, int t) {
  const int gm = t / a.num_n;
  const int nb = t - gm * a.num_n;
  int lo = 0, hi = a.E - 1;  // largest e with prefix[e] <= gm
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_prefix[mid] <= gm) lo = mid; else hi = mid - 1;
  }
  Tile tl;
  tl.e = lo;
  tl.m0 = s_off[lo] + (gm - s_prefix[lo]) * kBM;
  tl.row_end = s_off[lo + 1];
  tl.n0 = nb * kBN;
  tl.b_row = lo * a.N + tl.n0;
  tl.a_kb = 0;
  return tl;
}

__device__ __forceinline__ float load_sw(const GemmArgs &a, const uint8_t *sw_row, int kb) {
  if (a.sw_fmt == 0) return __ldg(reinterpret_cast<const float *>(sw_row) + kb);
  const int b = __ldg(sw_row + kb);
  return b >= 1 ? __uint_as_float(static_cast<uint32_t>(b) << 23) : __uint_as_float(0x00400000u);
}

__device__ __forceinline__ void cp_async_4(uint32_t dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_16_zfill(uint32_t dst, const void *src,
                                                  uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
// Arrive on `bar` once every cp.async this thread issued so far has landed (no count increment).
__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

// acc[j] += sc * (r[2j], r[2j + 1]) for j < 8: packed fp32x2 FMAs, round to nearest (the fp32
// promotion of one 16-column chunk of a K-block partial).
__device__ __forceinline__ void promote8(float2 *acc, const uint32_t (&r)[16], float sc) {
  const float2 sc2 = make_float2(sc, sc);
#pragma unroll
  for (int j = 0; j < 8; ++j)
    acc[j] = __ffma2_rn(make_float2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1])), sc2,
                        acc[j]);
}

// bf16 conversion and store of 32 columns (v[j] = columns 2j, 2j + 1 of chunk c4) of this
// thread's row, through the warp's swizzled staging buffer so that each global store
// instruction writes 64-byte row segments.
__device__ __forceinline__ void store_packed32(const uint32_t (&pk)[16], uint32_t stage_u32,
                                               int lane, uint16_t *out_base, const Tile &tl, int q,
                                               int c4, bool col_ok, int64_t ldo) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int phys = j ^ ((lane >> 1) & 3);
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(stage_u32 + lane * 64 + phys * 16),
                 "r"(pk[4 * j]), "r"(pk[4 * j + 1]), "r"(pk[4 * j + 2]), "r"(pk[4 * j + 3])
                 : "memory");
  }
  __syncwarp();
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const int r = p * 8 + (lane >> 2), c = lane & 3;
    const int phys = c ^ ((r >> 1) & 3);
    uint4 w;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(w.x), "=r"(w.y), "=r"(w.z), "=r"(w.w)
                 : "r"(stage_u32 + r * 64 + phys * 16)
                 : "memory");
    const int grow = tl.m0 + 32 * q + r;
    if (col_ok && grow < tl.row_end)
      *reinterpret_cast<uint4 *>(out_base + static_cast<int64_t>(grow) * ldo + 32 * c4 + 8 * c) = w;
  }
  __syncwarp();
}

__device__ __forceinline__ void store_chunk32(const float2 (&v)[16], uint32_t stage_u32, int lane,
                                              uint16_t *out_base, const Tile &tl, int q, int c4,
                                              bool col_ok, int64_t ldo) {
  uint32_t pk[16];
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    const __nv_bfloat162 v2 = __floats2bfloat162_rn(v[u].x, v[u].y);
    pk[u] = *reinterpret_cast<const uint32_t *>(&v2);
  }
  store_packed32(pk, stage_u32, lane, out_base, tl, q, c4, col_ok, ldo);
}

template <bool GROUPED, bool TS>
__global__ void __launch_bounds__(kGemmThreads, 1)
    k_gemm_w8a8_block(const __grid_constant__ CUtensorMap tm_a,
                      const __grid_constant__ CUtensorMap tm_b,
                      const __grid_constant__ CUtensorMap tm_out, const GemmArgs args) {
  using L = BlockLayout<TS>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar_full = sbase + L::offBar;              // [L::stages]
  const uint32_t bar_empty = bar_full + 8 * L::stages;      // [L::stages]
  const uint32_t bar_tfull = bar_empty + 8 * L::stages;     // [2]
  const uint32_t bar_tempty = bar_tfull + 16;             // [2]
  const uint32_t bar_done = bar_tempty + 16;
  const uint32_t bar_safull = bar_done + 8;                   // [kSaStages]
  const uint32_t bar_saempty = bar_safull + 8 * kSaStages;    // [kSaStages]
  const uint32_t bar_swfull = bar_saempty + 8 * kSaStages;    // [2]
  const uint32_t bar_swempty = bar_swfull + 16;               // [2]
  float *s_sa = reinterpret_cast<float *>(smem + L::offSa);
  float *s_sw = reinterpret_cast<float *>(smem + L::offSw);
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(smem + L::offMisc);
  volatile int *s_abort = reinterpret_cast<volatile int *>(smem + L::offMisc + 4);
  int *s_off = reinterpret_cast<int *>(smem + L::offGroups);
  int *s_prefix = s_off + (kMaxExperts + 1);

  const int KB = args.K / kBK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < L::stages; ++i) {
      mbar_init(bar_full + 8 * i, 1);
      mbar_init(bar_empty + 8 * i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_tfull + 8 * i, 1);
      mbar_init(bar_tempty + 8 * i, 8);
    }
    mbar_init(bar_done, 2);
    for (int i = 0; i < kSaStages; ++i) {
      mbar_init(bar_safull + 8 * i, 32);
      mbar_init(bar_saempty + 8 * i, 8);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_swfull + 8 * i, 32);
      mbar_init(bar_swempty + 8 * i, 8);
    }
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(s_tmem), 512);
    tmem_relinquish();
  }
  int total_tiles, total_units;
  if (GROUPED) {
    // Clamp the offsets into [previous, M] and count m-tiles per expert.
    for (int i = threadIdx.x; i <= args.E; i += blockDim.x) s_off[i] = args.group_offsets[i];
    __syncthreads();
    if (threadIdx.x == 0) {
      int prev = 0, acc = 0;
      for (int e = 0; e <= args.E; ++e) {
        int v = s_off[e];
        v = v < prev ? prev : (v > args.M ? args.M : v);
        if (e == 0) v = v < 0 ? 0 : v;
        s_off[e] = v;
        prev = v;
      }
      for (int e = 0; e < args.E; ++e) {
        s_prefix[e] = acc;
        acc += (s_off[e + 1] - s_off[e] + kBM - 1) / kBM;
      }
      s_prefix[args.E] = acc;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  total_tiles = GROUPED ? s_prefix[args.E] * args.num_n : args.num_m * args.num_n;
  total_units = total_tiles * args.splits;

  if (warp < 4) {
    reg_dealloc<kProducerRegs>();
    if (warp == 0) {
      // ------------------------------------------------------------------ TMA producer
      if (lane == 0) {
        tma_prefetch_desc(&tm_a);
        tma_prefetch_desc(&tm_b);
        uint32_t it = 0;
        for (int u = blockIdx.x; u < total_units; u += gridDim.x) {
          const Unit un = unit_of(args, u, KB);
          const Tile tl = GROUPED ? grouped_tile(args, s_off, s_prefix, un.t) : dense_tile(args, un.t);
          bool ok = true;
          for (int kb = un.kb0; kb < un.kb1; ++kb, ++it) {
            const uint32_t s = it % L::stages, ph = (it / L::stages) & 1u;
            if (!wait_one(bar_empty + 8 * s, ph ^ 1u, s_abort)) { ok = false; break; }
            mbar_arrive_expect_tx(bar_full + 8 * s, kStageBytes);
            tma_load_2d(sbase + L::offA + s * kTileABytes, &tm_a, (tl.a_kb + kb) * kBK, tl.m0,
                        bar_full + 8 * s);
            tma_load_2d(sbase + L::offB + s * kTileBBytes, &tm_b, kb * kBK, tl.b_row,
                        bar_full + 8 * s);
          }
          if (!ok) break;
        }
        // Drain: every issued load has landed before the CTA can exit.
        for (uint32_t s = 0; s < L::stages && s < it; ++s) {
          const uint32_t last = s + ((it - 1 - s) / L::stages) * L::stages;  // last fill of stage s
          wait_drain(bar_full + 8 * s, (last / L::stages) & 1u);
        }
      }
      __syncwarp();
    } else if (warp == 2) {
      // ---------------------------------------------------------------- scale producer
      const int NB = args.N / 128;
      const size_t sw_elem = args.sw_fmt == 0 ? 4 : 1;
      uint32_t it = 0, tile_it = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x, ++tile_it) {
        const Unit un = unit_of(args, u, KB);
        const Tile tl = GROUPED ? grouped_tile(args, s_off, s_prefix, un.t) : dense_tile(args, un.t);
        // weight scales of the tile's two 128-column halves, all K-blocks, as fp32
        const uint32_t tp = tile_it & 1u;
        if (!wait_warp(bar_swempty + 8 * tp, ((tile_it >> 1) & 1u) ^ 1u, s_abort)) break;
        for (int j = lane; j < 2 * KB; j += 32) {
          const int hh = j >= KB ? 1 : 0, kb = j - hh * KB;
          const int nb = tl.n0 / 128 + hh;
          float v = 0.0f;
          if (nb < NB) {
            const uint8_t *row = static_cast<const uint8_t *>(args.sw) +
                                 (static_cast<size_t>(tl.e) * NB + nb) * KB * sw_elem;
            v = load_sw(args, row, kb);
          }
          s_sw[(tp * 2 + hh) * kMaxKB + kb] = v;
        }
        mbar_arrive(bar_swfull + 8 * tp);
        if constexpr (GROUPED) {
          // activation scales: one 128-row column of sa per K-block, zero-filled past row_end
          const int rows_here = tl.row_end - tl.m0;
          for (int kb = un.kb0; kb < un.kb1; ++kb, ++it) {
            const uint32_t s2 = it % kSaStages, ph2 = (it / kSaStages) & 1u;
            if (!wait_warp(bar_saempty + 8 * s2, ph2 ^ 1u, s_abort)) { ok = false; break; }
            const float *src = args.sa + static_cast<int64_t>(kb) * args.lds + tl.m0 + 4 * lane;
            const uint32_t dst = smem_u32(s_sa + s2 * kBM + 4 * lane);
            const int valid = max(0, min(4, rows_here - 4 * lane));
            if ((reinterpret_cast<uintptr_t>(src) & 15u) == 0) {
              cp_async_16_zfill(dst, valid > 0 ? src : args.sa, 4u * valid);
            } else {
#pragma unroll
              for (int i = 0; i < 4; ++i)
                cp_async_4(dst + 4 * i, i < valid ? src + i : args.sa, i < valid ? 4u : 0u);
            }
            cp_async_arrive_noinc(bar_safull + 8 * s2);
          }
        }
      }
      cp_async_wait_all();
      __syncwarp();
    } else if (warp == 1 || warp == 3) {
      // ------------------------------------------------------------------ MMA issuers
      // Two issuing threads: warp 1 takes the even K-blocks (TMEM buffer 0), warp 3 the odd ones
      // (buffer 1), so each has two K-blocks of tensor-pipe time to cover its waits and issue.
      if (lane == 0) {
        const uint32_t mine = warp == 3 ? 1u : 0u;
        uint32_t it = 0;
        for (int u = blockIdx.x; u < total_units; u += gridDim.x) {
          const Unit un = unit_of(args, u, KB);
          bool ok = true;
          for (int kb = un.kb0; kb < un.kb1; ++kb, ++it) {
            if ((it & 1u) != mine) continue;
            const uint32_t s = it % L::stages, ph = (it / L::stages) & 1u;
            const uint32_t b = it & 1u, bph = (it >> 1) & 1u;
            if (!wait_one(bar_tempty + 8 * b, bph ^ 1u, s_abort)) { ok = false; break; }
            if (!wait_one(bar_full + 8 * s, ph, s_abort)) { ok = false; break; }
            tc_fence_after();
            const uint64_t ad = sdesc_k128(sbase + L::offA + s * kTileABytes);
            const uint64_t bd = sdesc_k128(sbase + L::offB + s * kTileBBytes);
            const uint32_t d = tmem_base + b * kBN;
#pragma unroll
            for (int kk = 0; kk < kBK / 32; ++kk)  // 32-byte steps inside the 128-byte row
              mma_f8f6f4(d, ad + 2 * kk, bd + 2 * kk, kIdesc, kk > 0 ? 1u : 0u);
            mma_commit(bar_empty + 8 * s);
            mma_commit(bar_tfull + 8 * b);
          }
          if (!ok) break;
        }
        // Every MMA has completed before TMEM is released.
        mma_commit(bar_done);
        wait_drain(bar_done, 0);
      }
      __syncwarp();
    }
  } else {
    reg_alloc<kEpilogueRegs>();
    // ------------------------------------------------------------------ epilogue / promotion
    const int q = warp & 3;         // TMEM lane quarter = rows 32q .. 32q + 31 of the tile
    const int h = (warp - 4) >> 2;  // column half of the 256-wide tile
    const int NB = args.N / 128;
    uint8_t *stage = smem + L::offStaging + (warp - 4) * L::stagingPerWarp;
    const uint32_t stage_u32 = smem_u32(stage);
    uint32_t it = 0, tile_it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x, ++tile_it) {
      const Unit un = unit_of(args, u, KB);
      const Tile tl = GROUPED ? grouped_tile(args, s_off, s_prefix, un.t) : dense_tile(args, un.t);
      const int nbh = tl.n0 / 128 + h;
      const bool col_ok = nbh < NB;
      const uint32_t tp = tile_it & 1u;
      if (!wait_warp(bar_swfull + 8 * tp, (tile_it >> 1) & 1u, s_abort)) { ok = false; break; }
      const float *sw_tile = s_sw + (tp * 2 + h) * kMaxKB;
      float2 acc[64];  // columns 2j, 2j + 1 of this thread's row
#pragma unroll
      for (int j = 0; j < 64; ++j) acc[j] = make_float2(0.0f, 0.0f);
      // Activation scales.  Dense: this thread loads its own row's scales from global memory
      // two K-blocks ahead.  Grouped: the scale producer streams them through a shared ring
      // (measured faster for the short, many-tile grouped problems).
      const int row = tl.m0 + 32 * q + lane;
      const bool row_ok = row < tl.row_end;
      const float *sa_row = args.sa + row + static_cast<int64_t>(tl.a_kb) * args.lds;
      float sa0 = 0.0f, sa1 = 0.0f;
      if constexpr (!GROUPED) {
        sa0 = (row_ok && un.kb0 < un.kb1)
                  ? __ldg(sa_row + static_cast<int64_t>(un.kb0) * args.lds) : 0.0f;
        sa1 = (row_ok && un.kb0 + 1 < un.kb1)
                  ? __ldg(sa_row + static_cast<int64_t>(un.kb0 + 1) * args.lds) : 0.0f;
      }
      uint32_t rb[16];  // the last chunk of the previous K-block, promoted under the next load
      float sc_prev = 0.0f;
      bool have_prev = false;
      for (int kb = un.kb0; kb < un.kb1; ++kb, ++it) {
        float sa_cur;
        if constexpr (GROUPED) {
          const uint32_t s2 = it % kSaStages, ph2 = (it / kSaStages) & 1u;
          if (!wait_warp(bar_safull + 8 * s2, ph2, s_abort)) { ok = false; break; }
          sa_cur = s_sa[s2 * kBM + 32 * q + lane];
          __syncwarp();
          if (lane == 0) mbar_arrive(bar_saempty + 8 * s2);
        } else {
          sa_cur = sa0;
          sa0 = sa1;
          sa1 = (row_ok && kb + 2 < un.kb1)
                    ? __ldg(sa_row + static_cast<int64_t>(kb + 2) * args.lds) : 0.0f;
        }
        const float sc = __fmul_rn(sa_cur, sw_tile[kb]);
        const uint32_t b = it & 1u, bph = (it >> 1) & 1u;
        if (!wait_warp(bar_tfull + 8 * b, bph, s_abort)) { ok = false; break; }
        tc_fence_after();
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + b * kBN + h * 128;
        // Eight 16-column chunks; the load of chunk c + 1 is in flight while chunk c is promoted.
        // The buffer goes back to the MMA as soon as the last chunk is in registers.
        uint32_t ra[16];
        tmem_ld_32x32b_x16(taddr, ra);
        if (have_prev) promote8(acc + 56, rb, sc_prev);
        tmem_ld_wait(ra);
#pragma unroll
        for (int c = 0; c < 3; ++c) {
          tmem_ld_32x32b_x16(taddr + 32 * c + 16, rb);
          promote8(acc + 16 * c, ra, sc);
          tmem_ld_wait(rb);
          tmem_ld_32x32b_x16(taddr + 32 * c + 32, ra);
          promote8(acc + 16 * c + 8, rb, sc);
          tmem_ld_wait(ra);
        }
        tmem_ld_32x32b_x16(taddr + 112, rb);
        promote8(acc + 48, ra, sc);
        tmem_ld_wait(rb);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_tempty + 8 * b);
        sc_prev = sc;
        have_prev = true;
      }
      if (have_prev) promote8(acc + 56, rb, sc_prev);
      if (!ok) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_swempty + 8 * tp);
      uint16_t *out_base = args.out + static_cast<int64_t>(tl.n0 + 128 * h);
      if (args.splits > 1) {
        // Split K: this unit's fp32 partial goes to the workspace (coalesced: lane = row); the
        // partials of a tile are added in split order by k_splitk_reduce, launched next.
        const int rl = 32 * q + lane;
        float4 *mine = reinterpret_cast<float4 *>(args.ws) +
                       (static_cast<size_t>(un.t) * args.splits + un.j) * (2 * 32 * 128) +
                       (h * 32) * 128 + rl;
#pragma unroll
        for (int c = 0; c < 32; ++c)
          __stcg(mine + c * 128, make_float4(acc[2 * c].x, acc[2 * c].y, acc[2 * c + 1].x,
                                             acc[2 * c + 1].y));
        continue;
      }
      if constexpr (TS) {
        if (!GROUPED || tl.row_end >= tl.m0 + 32 * q + 32) {  // this warp's 32 rows are all in
          // This warp's bf16 rows go to its slot as two 32 x 64 boxes (128-byte swizzle) and out
          // through the TMA engine; the warp goes on to the next tile.  Grouped: a warp whose rows
          // an expert's end cuts takes the masked path below.
          if (lane == 0) bulk_wait_read0();  // the slot's previous stores have read it
          __syncwarp();
#pragma unroll
          for (int cc = 0; cc < 16; ++cc) {
            uint32_t pk[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const __nv_bfloat162 v2 = __floats2bfloat162_rn(acc[4 * cc + u].x, acc[4 * cc + u].y);
              pk[u] = *reinterpret_cast<const uint32_t *>(&v2);
            }
            const uint32_t addr = stage_u32 + (cc >> 3) * 4096 + lane * 128 +
                                  ((static_cast<uint32_t>(cc & 7) ^ static_cast<uint32_t>(lane & 7)) << 4);
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(pk[0]),
                         "r"(pk[1]), "r"(pk[2]), "r"(pk[3])
                         : "memory");
          }
          fence_proxy_async_shared();
          __syncwarp();
          if (lane == 0) {
            const int y = tl.m0 + 32 * q;
#pragma unroll
            for (int bx = 0; bx < 2; ++bx) {
              const int x = tl.n0 + 128 * h + 64 * bx;
              if (x < args.N && y < args.M) tma_store_2d(&tm_out, x, y, stage_u32 + bx * 4096);
            }
            bulk_commit();
          }
          continue;
        }
        if (lane == 0) bulk_wait_read0();  // the masked path below reuses the slot
        __syncwarp();
      }
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4)
        store_chunk32(*reinterpret_cast<const float2(*)[16]>(acc + 16 * c4), stage_u32, lane,
                      out_base, tl, q, c4, col_ok, args.ldo);
    }
    if constexpr (TS) {
      if (lane == 0) bulk_wait0();  // every tile store of this warp has completed
      __syncwarp();
    }
    tc_fence_before();
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// ---------------------------------------------------------------------------------------------
// Per-token x per-channel ("PTPC") W8A8 GEMM: out[m, n] = bf16( P[m, n] * fp32(sa[m] * sw[n]) )
// with P the fp32 tensor-core dot product over all of K.  With no per-K-block promotion the MMA
// accumulates a whole tile in one TMEM buffer; the epilogue drains a buffer once per tile while
// the MMA fills the other.  Same persistent structure, shared-memory layout and barriers as
// k_gemm_w8a8_block:
//   warp 0      TMA producer (A 128 x 128 B, B 256 x 128 B per K-block, 4-stage ring)
//   warp 1      TMEM allocator and MMA issuer: per tile, all K-blocks into buffer tile % 2
//   warp 2      scale producer: the tile's 256 weight scales, double-buffered across tiles
//   warps 4-11  epilogue: warp w reads TMEM lanes 32 (w % 4), column half (w - 4) / 4
// ---------------------------------------------------------------------------------------------
struct RowwiseArgs {
  const float *sa;      // [M] per-token scales
  const float *sw;      // [N] per-channel scales
  int M, N, K;
  uint16_t *out;
  int64_t ldo;
  int num_n, num_m;
  int group_m;          // dense rasterization: m-blocks per group
};

__global__ void __launch_bounds__(kGemmThreads, 1)
    k_gemm_w8a8_rowwise(const __grid_constant__ CUtensorMap tm_a,
                        const __grid_constant__ CUtensorMap tm_b, const RowwiseArgs args) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar_full = sbase + kOffBar;              // [kStages]
  const uint32_t bar_empty = bar_full + 8 * kStages;      // [kStages]
  const uint32_t bar_tfull = bar_empty + 8 * kStages;     // [2]
  const uint32_t bar_tempty = bar_tfull + 16;             // [2]
  const uint32_t bar_done = bar_tempty + 16;
  const uint32_t bar_swfull = bar_done + 8;               // [2]
  const uint32_t bar_swempty = bar_swfull + 16;           // [2]
  float *s_sw = reinterpret_cast<float *>(smem + kOffSw);  // [2][256]
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(smem + kOffMisc);
  volatile int *s_abort = reinterpret_cast<volatile int *>(smem + kOffMisc + 4);
  const int KB = args.K / kBK;
  GemmArgs ga{};
  ga.num_m = args.num_m;
  ga.num_n = args.num_n;
  ga.group_m = args.group_m;
  ga.M = args.M;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(bar_full + 8 * i, 1);
      mbar_init(bar_empty + 8 * i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_tfull + 8 * i, 1);
      mbar_init(bar_tempty + 8 * i, 8);
      mbar_init(bar_swfull + 8 * i, 32);
      mbar_init(bar_swempty + 8 * i, 8);
    }
    mbar_init(bar_done, 1);
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(s_tmem), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  const int total_tiles = args.num_m * args.num_n;

  if (warp < 4) {
    reg_dealloc<kProducerRegs>();
    if (warp == 0) {
      // ------------------------------------------------------------------ TMA producer
      if (lane == 0) {
        tma_prefetch_desc(&tm_a);
        tma_prefetch_desc(&tm_b);
        uint32_t it = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
          const Tile tl = dense_tile(ga, t);
          for (int kb = 0; kb < KB; ++kb, ++it) {
            const uint32_t s = it % kStages, ph = (it / kStages) & 1u;
            if (!wait_one(bar_empty + 8 * s, ph ^ 1u, s_abort)) { ok = false; break; }
            mbar_arrive_expect_tx(bar_full + 8 * s, kStageBytes);
            tma_load_2d(sbase + kOffA + s * kTileABytes, &tm_a, kb * kBK, tl.m0, bar_full + 8 * s);
            tma_load_2d(sbase + kOffB + s * kTileBBytes, &tm_b, kb * kBK, tl.b_row,
                        bar_full + 8 * s);
          }
        }
        for (uint32_t s = 0; s < kStages && s < it; ++s) {
          const uint32_t last = s + ((it - 1 - s) / kStages) * kStages;  // last fill of stage s
          wait_drain(bar_full + 8 * s, (last / kStages) & 1u);
        }
      }
      __syncwarp();
    } else if (warp == 2) {
      // ---------------------------------------------------------------- scale producer
      uint32_t tile_it = 0;
      for (int t = blockIdx.x; t < total_tiles; t += gridDim.x, ++tile_it) {
        const Tile tl = dense_tile(ga, t);
        const uint32_t tp = tile_it & 1u;
        if (!wait_warp(bar_swempty + 8 * tp, ((tile_it >> 1) & 1u) ^ 1u, s_abort)) break;
        for (int j = lane; j < kBN; j += 32) {
          const int n = tl.n0 + j;
          s_sw[tp * kBN + j] = n < args.N ? __ldg(args.sw + n) : 0.0f;
        }
        mbar_arrive(bar_swfull + 8 * tp);
      }
      __syncwarp();
    } else if (warp == 1) {
      // ------------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        uint32_t it = 0, tile_it = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++tile_it) {
          const uint32_t b = tile_it & 1u, bph = (tile_it >> 1) & 1u;
          if (!wait_one(bar_tempty + 8 * b, bph ^ 1u, s_abort)) { ok = false; break; }
          const uint32_t d = tmem_base + b * kBN;
          for (int kb = 0; kb < KB; ++kb, ++it) {
            const uint32_t s = it % kStages, ph = (it / kStages) & 1u;
            if (!wait_one(bar_full + 8 * s, ph, s_abort)) { ok = false; break; }
            tc_fence_after();
            const uint64_t ad = sdesc_k128(sbase + kOffA + s * kTileABytes);
            const uint64_t bd = sdesc_k128(sbase + kOffB + s * kTileBBytes);
#pragma unroll
            for (int kk = 0; kk < kBK / 32; ++kk)
              mma_f8f6f4(d, ad + 2 * kk, bd + 2 * kk, kIdesc, (kb > 0 || kk > 0) ? 1u : 0u);
            mma_commit(bar_empty + 8 * s);
          }
          if (!ok) break;
          mma_commit(bar_tfull + 8 * b);
        }
        // Every MMA has completed before TMEM is released.
        mma_commit(bar_done);
        wait_drain(bar_done, 0);
      }
      __syncwarp();
    }
  } else {
    reg_alloc<kEpilogueRegs>();
    // ------------------------------------------------------------------ epilogue
    const int q = warp & 3;         // TMEM lane quarter = rows 32q .. 32q + 31 of the tile
    const int h = (warp - 4) >> 2;  // column half of the 256-wide tile
    const int NB = args.N / 128;
    uint8_t *stage = smem + kOffStaging + (warp - 4) * kStagingBytesPerWarp;
    const uint32_t stage_u32 = smem_u32(stage);
    uint32_t tile_it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++tile_it) {
      const Tile tl = dense_tile(ga, t);
      const int row = tl.m0 + 32 * q + lane;
      const float sa_row = row < tl.row_end ? __ldg(args.sa + row) : 0.0f;
      const bool col_ok = tl.n0 / 128 + h < NB;
      const uint32_t tp = tile_it & 1u, b = tile_it & 1u, bph = (tile_it >> 1) & 1u;
      if (!wait_warp(bar_swfull + 8 * tp, bph, s_abort)) { ok = false; break; }
      if (!wait_warp(bar_tfull + 8 * b, bph, s_abort)) { ok = false; break; }
      tc_fence_after();
      const float *swh = s_sw + tp * kBN + 128 * h;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + b * kBN + h * 128;
      uint16_t *out_base = args.out + static_cast<int64_t>(tl.n0 + 128 * h);
#pragma unroll 1
      for (int c4 = 0; c4 < 4; ++c4) {
        uint32_t r0[16], r1[16];
        tmem_ld_32x32b_x16(taddr + 32 * c4, r0);
        tmem_ld_32x32b_x16(taddr + 32 * c4 + 16, r1);
        tmem_ld_wait(r0);
        tmem_ld_wait(r1);
        if (c4 == 3) {
          // the whole buffer is in registers: hand it back to the MMA before the last stores
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar_tempty + 8 * b);
        }
        float2 v[16];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int c = 32 * c4 + 2 * j;
          v[j] = make_float2(__fmul_rn(__uint_as_float(r0[2 * j]), __fmul_rn(sa_row, swh[c])),
                             __fmul_rn(__uint_as_float(r0[2 * j + 1]), __fmul_rn(sa_row, swh[c + 1])));
          v[8 + j] = make_float2(
              __fmul_rn(__uint_as_float(r1[2 * j]), __fmul_rn(sa_row, swh[c + 16])),
              __fmul_rn(__uint_as_float(r1[2 * j + 1]), __fmul_rn(sa_row, swh[c + 17])));
        }
        store_chunk32(v, stage_u32, lane, out_base, tl, q, c4, col_ok, args.ldo);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_swempty + 8 * tp);  // done with this tile's weight scales
    }
    tc_fence_before();
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// ---------------------------------------------------------------------------------------------
// Hardware block-scaled GEMM for power-of-two (E8M0) scales:
//   out[m, n] = bf16( sum_kb 2^ea[m, kb] * 2^ew[n / 128, kb] * P_kb[m, n] )
// tcgen05.mma kind::mxf8f6f4.block_scale applies one UE8M0 scale per 32 K-elements of each row of
// A and each column of B inside the tensor core; the 128-group scale of a K-block is given to all
// four of its 32-element sub-blocks.  All of K accumulates in one 256-column TMEM buffer, so the
// epilogue only converts: it moves the whole tile to registers, hands the buffer back to the MMA
// and then writes bf16 while the next tile accumulates.
// Scale factors in TMEM: SFA in 4 columns (row m at lane m % 32 of every sub-partition, column
// m / 32), SFB in 8 (column n at lane n % 32, column n / 32).  Each 32-bit cell holds the scales
// of four consecutive K-blocks, one per byte; the instruction's scale-factor ID picks the byte.
// So one group of three tcgen05.cp (SFA, SFB 0-127, SFB 128-255) serves four K-blocks; two such
// slots (TMEM columns 256 + 16 j) alternate between groups.  Roles:
//   warp 0      TMA producer, as in k_gemm_w8a8_block
//   warp 1      MMA issuer: at the first K-block of a group the three copies from the group's
//               shared scale tiles, then per K-block 4 block-scaled MMAs; after the group's last
//               MMA a commit frees the group's slot (shared tiles and TMEM columns)
//   warp 2      scale producer: per group converts the activation scales (fp32 powers of two;
//               anything else records FP8Q_ERR_NOT_POW2) and the tile's weight-scale bytes into
//               the 32 x 16-byte shared tiles tcgen05.cp reads; the next group's global loads are
//               issued as soon as the current group is written
//   warps 4-11  epilogue
// Block-diagonal head groups work as in k_gemm_w8a8_block (Tile::a_kb).
// ---------------------------------------------------------------------------------------------
struct MxArgs {
  const float *sa;       // K-block-major fp32 powers of two, sa[kb * lds + m]
  int64_t lds;
  const uint8_t *sw;     // E8M0 bytes [N/128][K/128]
  int M, N, K;           // K: per group when n_tiles_per_group > 0
  uint16_t *out;
  int64_t ldo;
  int num_n, num_m;
  int group_m;          // dense rasterization: m-blocks per group
  int n_tiles_per_group;
};

constexpr int kErrNotPow2 = 10;  // FP8Q_ERR_NOT_POW2
constexpr int kSfGroup = 4;                            // K-blocks per scale-factor group
constexpr int kSfTileBytes = 32 * 16;                  // one tcgen05.cp source: 32 rows x 16 B
constexpr int kSfSlotBytes = 3 * kSfTileBytes;         // SFA, SFB columns 0-127, SFB 128-255
constexpr int kOffSf = kOffSa;                         // [2 slots][3][32][16] B
static_assert(kOffSf + 2 * kSfSlotBytes <= kOffBar, "scale-factor tiles overlap barriers");
// Block-scaled instruction descriptor: A, B E4M3 (bits 7-9, 10-12 = 0), K-major, N >> 3 in bits
// 17-22, scale format UE8M0 (bit 23), M >> 4 in bits 24-28, K = 32 (bit 31 = 0); the scale-factor
// IDs (bits 4-5 for B, 29-30 for A) are set per K-block by mx_idesc.
constexpr uint32_t kIdescMx = (static_cast<uint32_t>(kBN >> 3) << 17) | (1u << 23) |
                              (static_cast<uint32_t>(kBM >> 4) << 24);

__device__ __forceinline__ uint32_t mx_idesc(uint32_t sf_id) {
  return kIdescMx | (sf_id << 4) | (sf_id << 29);
}

// Shared-memory descriptor of a 32-row x 16-byte tile, rows contiguous, no swizzle: 8-row core
// groups 128 bytes apart (stride byte offset), leading byte offset 16 (a single 16-byte column),
// descriptor version 1 (bit 46), layout 0.
__device__ __forceinline__ uint64_t sdesc_sf(uint32_t saddr) {
  return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (static_cast<uint64_t>(16 >> 4) << 16) |
         (static_cast<uint64_t>(128 >> 4) << 32) | (static_cast<uint64_t>(1) << 46);
}

// E8M0 byte of an fp32 power of two (2^-127 .. 2^127); other values record kErrNotPow2.
__device__ __forceinline__ uint32_t e8m0_of_pow2(float v) {
  const uint32_t b = __float_as_uint(v);
  const uint32_t ex = (b >> 23) & 0xFFu, mant = b & 0x7FFFFFu;
  if (b >> 31 || ex == 0xFFu || (ex != 0u && mant != 0u) || (ex == 0u && mant != 0x400000u)) {
    record_error(kErrNotPow2);
    return 127u;
  }
  return ex;  // 2^-127 (0x00400000) has exponent field 0, its E8M0 byte
}

__global__ void __launch_bounds__(kGemmThreads, 1)
    k_gemm_w8a8_mx(const __grid_constant__ CUtensorMap tm_a,
                   const __grid_constant__ CUtensorMap tm_b, const MxArgs args) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar_full = sbase + kOffBar;              // [kStages]
  const uint32_t bar_empty = bar_full + 8 * kStages;      // [kStages]
  const uint32_t bar_tfull = bar_empty + 8 * kStages;
  const uint32_t bar_tempty = bar_tfull + 16;
  const uint32_t bar_done = bar_tempty + 16;
  const uint32_t bar_sffull = bar_done + 8;               // [2]
  const uint32_t bar_sfempty = bar_sffull + 16;           // [2]
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(smem + kOffMisc);
  volatile int *s_abort = reinterpret_cast<volatile int *>(smem + kOffMisc + 4);
  const int KB = args.K / kBK;
  const int NB = args.N / 128;
  GemmArgs ga{};
  ga.num_m = args.num_m;
  ga.num_n = args.num_n;
  ga.group_m = args.group_m;
  ga.M = args.M;
  ga.K = args.K;
  ga.n_tiles_per_group = args.n_tiles_per_group;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(bar_full + 8 * i, 1);
      mbar_init(bar_empty + 8 * i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_sffull + 8 * i, 1);
      mbar_init(bar_sfempty + 8 * i, 1);
    }
    mbar_init(bar_tfull, 1);
    mbar_init(bar_tempty, 8);
    mbar_init(bar_done, 1);
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(s_tmem), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  const int total_tiles = args.num_m * args.num_n;

  if (warp < 4) {
    reg_dealloc<kProducerRegs>();
    if (warp == 0) {
      // ------------------------------------------------------------------ TMA producer
      if (lane == 0) {
        tma_prefetch_desc(&tm_a);
        tma_prefetch_desc(&tm_b);
        uint32_t it = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
          const Tile tl = dense_tile(ga, t);
          for (int kb = 0; kb < KB; ++kb, ++it) {
            const uint32_t s = it % kStages, ph = (it / kStages) & 1u;
            if (!wait_one(bar_empty + 8 * s, ph ^ 1u, s_abort)) { ok = false; break; }
            mbar_arrive_expect_tx(bar_full + 8 * s, kStageBytes);
            tma_load_2d(sbase + kOffA + s * kTileABytes, &tm_a, (tl.a_kb + kb) * kBK, tl.m0,
                        bar_full + 8 * s);
            tma_load_2d(sbase + kOffB + s * kTileBBytes, &tm_b, kb * kBK, tl.b_row,
                        bar_full + 8 * s);
          }
        }
        for (uint32_t s = 0; s < kStages && s < it; ++s) {
          const uint32_t last = s + ((it - 1 - s) / kStages) * kStages;  // last fill of stage s
          wait_drain(bar_full + 8 * s, (last / kStages) & 1u);
        }
      }
      __syncwarp();
    } else if (warp == 2) {
      // ---------------------------------------------------------------- scale producer
      float qa[kSfGroup][4];        // the next group's activation scales (rows lane + 32 c)
      uint32_t qb[kSfGroup][2];     // and weight-scale bytes of the tile's two 128-column halves
      int lt = blockIdx.x, lg = 0;  // the next group to load: tile, first K-block
      auto load_group = [&]() {
        if (lt >= total_tiles) return;
        const Tile tl = dense_tile(ga, lt);
#pragma unroll
        for (int j = 0; j < kSfGroup; ++j) {
          const bool in = lg + j < KB;
          const float *sa_kb = args.sa + static_cast<int64_t>(tl.a_kb + lg + j) * args.lds;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int m = tl.m0 + lane + 32 * c;
            qa[j][c] = (in && m < args.M) ? __ldg(sa_kb + m) : 1.0f;
          }
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int nb = tl.n0 / 128 + hh;
            qb[j][hh] = (in && nb < NB) ? __ldg(args.sw + static_cast<int64_t>(nb) * KB + lg + j)
                                        : 127u;
          }
        }
        lg += kSfGroup;
        if (lg >= KB) {
          lg = 0;
          lt += gridDim.x;
        }
      };
      load_group();
      uint32_t gi = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
        for (int g0 = 0; g0 < KB; g0 += kSfGroup, ++gi) {
          const uint32_t j = gi & 1u, ph = (gi >> 1) & 1u;
          // the MMAs of the group that last used this slot have completed
          if (!wait_warp(bar_sfempty + 8 * j, ph ^ 1u, s_abort)) { ok = false; break; }
          uint8_t *tile = smem + kOffSf + j * kSfSlotBytes;
          uint32_t w[4];
#pragma unroll
          for (int c = 0; c < 4; ++c)
            w[c] = e8m0_of_pow2(qa[0][c]) | (e8m0_of_pow2(qa[1][c]) << 8) |
                   (e8m0_of_pow2(qa[2][c]) << 16) | (e8m0_of_pow2(qa[3][c]) << 24);
          *reinterpret_cast<uint4 *>(tile + lane * 16) = make_uint4(w[0], w[1], w[2], w[3]);
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const uint32_t bw =
                qb[0][hh] | (qb[1][hh] << 8) | (qb[2][hh] << 16) | (qb[3][hh] << 24);
            *reinterpret_cast<uint4 *>(tile + (1 + hh) * kSfTileBytes + lane * 16) =
                make_uint4(bw, bw, bw, bw);
          }
          fence_proxy_async_shared();  // generic-proxy writes -> the tensor core's reads
          __syncwarp();
          if (lane == 0) mbar_arrive(bar_sffull + 8 * j);
          load_group();
        }
      }
      __syncwarp();
    } else if (warp == 1) {
      // ------------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        uint32_t it = 0, tile_it = 0, gi = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++tile_it) {
          // the epilogue has moved the previous tile out of the accumulator
          if (!wait_one(bar_tempty, (tile_it & 1u) ^ 1u, s_abort)) { ok = false; break; }
          tc_fence_after();
          uint32_t tsf = 0;
          for (int kb = 0; kb < KB; ++kb, ++it) {
            const uint32_t sfj = static_cast<uint32_t>(kb % kSfGroup);
            if (sfj == 0) {
              const uint32_t j = gi & 1u, ph = (gi >> 1) & 1u;
              if (!wait_one(bar_sffull + 8 * j, ph, s_abort)) { ok = false; break; }
              tc_fence_after();
              tsf = tmem_base + 256 + 16 * j;
              const uint32_t sft = sbase + kOffSf + j * kSfSlotBytes;
              tmem_cp_32x128b_x4(tsf, sdesc_sf(sft));
              tmem_cp_32x128b_x4(tsf + 4, sdesc_sf(sft + kSfTileBytes));
              tmem_cp_32x128b_x4(tsf + 8, sdesc_sf(sft + 2 * kSfTileBytes));
            }
            const uint32_t s = it % kStages, ph = (it / kStages) & 1u;
            if (!wait_one(bar_full + 8 * s, ph, s_abort)) { ok = false; break; }
            tc_fence_after();
            const uint64_t ad = sdesc_k128(sbase + kOffA + s * kTileABytes);
            const uint64_t bd = sdesc_k128(sbase + kOffB + s * kTileBBytes);
            const uint32_t idesc = mx_idesc(sfj);
            const uint32_t tsfa = tsf | (sfj << 30), tsfb = (tsf + 4) | (sfj << 30);
#pragma unroll
            for (int kk = 0; kk < kBK / 32; ++kk)
              mma_mxf8f6f4(tmem_base, ad + 2 * kk, bd + 2 * kk, idesc, tsfa, tsfb,
                           (kb > 0 || kk > 0) ? 1u : 0u);
            mma_commit(bar_empty + 8 * s);
            if (sfj == kSfGroup - 1 || kb == KB - 1) {
              mma_commit(bar_sfempty + 8 * (gi & 1u));  // the group's scale slot is free
              ++gi;
            }
          }
          if (!ok) break;
          mma_commit(bar_tfull);
        }
        // Every MMA and copy has completed before TMEM is released.
        mma_commit(bar_done);
        wait_drain(bar_done, 0);
      }
      __syncwarp();
    }
  } else {
    reg_alloc<kEpilogueRegs>();
    // ------------------------------------------------------------------ epilogue
    const int q = warp & 3;         // TMEM lane quarter = rows 32q .. 32q + 31 of the tile
    const int h = (warp - 4) >> 2;  // column half of the 256-wide tile
    uint8_t *stage = smem + kOffStaging + (warp - 4) * kStagingBytesPerWarp;
    const uint32_t stage_u32 = smem_u32(stage);
    uint32_t tile_it = 0;
    for (int t = blockIdx.x; t < total_tiles; t += gridDim.x, ++tile_it) {
      const Tile tl = dense_tile(ga, t);
      const bool col_ok = tl.n0 / 128 + h < NB;
      if (!wait_warp(bar_tfull, tile_it & 1u, s_abort)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + h * 128;
      // the tile's 128 columns: eight 16-column loads in flight together, one wait
      uint32_t r[8][16];
#pragma unroll
      for (int c = 0; c < 8; ++c) tmem_ld_32x32b_x16(taddr + 16 * c, r[c]);
#pragma unroll
      for (int c = 0; c < 8; ++c) tmem_ld_wait(r[c]);
      // the whole tile is in registers: the accumulator goes back to the MMA
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_tempty);
      uint32_t pk[4][16];
#pragma unroll
      for (int c = 0; c < 8; ++c)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const __nv_bfloat162 v2 = __floats2bfloat162_rn(__uint_as_float(r[c][2 * j]),
                                                          __uint_as_float(r[c][2 * j + 1]));
          pk[c / 2][8 * (c & 1) + j] = *reinterpret_cast<const uint32_t *>(&v2);
        }
      uint16_t *out_base = args.out + static_cast<int64_t>(tl.n0 + 128 * h);
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4)
        store_packed32(pk[c4], stage_u32, lane, out_base, tl, q, c4, col_ok, args.ldo);
    }
    tc_fence_before();
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// Split-K reduction: out[m, n] = bf16( sum over j = 0 .. S - 1, in that order, of partial_j ).

// Partials: [tile][split][half h][chunk c][row r] float4 = columns 128 h + 4 c .. + 3 of row r.
// Grid: 8 CTAs of 256 threads per dense tile; thread (r, g) adds row r, columns 16 g .. 16 g + 15
// (4 float4 per split, read coalesced across rows) and writes 32 contiguous output bytes.
constexpr int kReduceThreads = 256;
__global__ void __launch_bounds__(kReduceThreads)
    k_splitk_reduce(const float4 *__restrict__ ws, int splits, int num_m, int num_n, int group_m,
                    int M, int N, uint16_t *__restrict__ out, int64_t ldo) {
  const int t = blockIdx.x >> 3;                  // dense tile, same order as dense_tile()
  const int r = threadIdx.x & 127;
  const int g = ((blockIdx.x & 7) << 1) | (threadIdx.x >> 7);  // 16-column group, 0 .. 15
  GemmArgs a{};
  a.num_m = num_m;
  a.num_n = num_n;
  a.group_m = group_m;
  a.M = M;
  const Tile tl = dense_tile(a, t);
  const int row = tl.m0 + r, col = tl.n0 + 16 * g;
  // Launched as a programmatic dependent of the GEMM (its launch overlaps the GEMM's tail): wait
  // until the GEMM grid has completed and its partials are visible.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (row >= M || col >= N) return;
  const int h = g >> 3, c0 = (g & 7) * 4;
  const float4 *p = ws + static_cast<size_t>(t) * splits * (2 * 32 * 128) + (h * 32 + c0) * 128 + r;
  // The partials of up to four splits are loaded together, then added in split order.
  float4 sum[4];
  for (int j0 = 0; j0 < splits; j0 += 4) {
    float4 v[4][4];
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      if (j0 + jj < splits) {
        const float4 *pj = p + static_cast<size_t>(j0 + jj) * (2 * 32 * 128);
#pragma unroll
        for (int i = 0; i < 4; ++i) v[jj][i] = __ldcg(pj + i * 128);
      }
    }
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      if (j0 + jj < splits) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          sum[i] = j0 + jj == 0
                       ? v[jj][i]
                       : make_float4(__fadd_rn(sum[i].x, v[jj][i].x), __fadd_rn(sum[i].y, v[jj][i].y),
                                     __fadd_rn(sum[i].z, v[jj][i].z), __fadd_rn(sum[i].w, v[jj][i].w));
      }
    }
  }
  uint32_t pk[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 lo = __floats2bfloat162_rn(sum[i].x, sum[i].y);
    const __nv_bfloat162 hi = __floats2bfloat162_rn(sum[i].z, sum[i].w);
    pk[2 * i] = *reinterpret_cast<const uint32_t *>(&lo);
    pk[2 * i + 1] = *reinterpret_cast<const uint32_t *>(&hi);
  }
  uint4 *dst = reinterpret_cast<uint4 *>(out + static_cast<int64_t>(row) * ldo + col);
  dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
}

}  // namespace fp8q
