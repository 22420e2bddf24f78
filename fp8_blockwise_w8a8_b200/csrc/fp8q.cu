// fp8q.cu -- the C ABI of libfp8q.so: argument checks, TMA descriptors and kernel launches.
// The declarations and the contract of every entry point are in include/fp8q.h.
#include "fp8q.h"

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "gemm_kernel.cuh"
#include "ptx.cuh"
#include "quant_kernels.cuh"
#include "attn_kernels.cuh"

namespace {

constexpr int kMaxDevices = 64;
constexpr int kMaxTokenK = 16384;

struct DeviceState {
  bool probed = false;
  bool is_sm100 = false;
  int sms = 0;
  bool attrs_set = false;
  void *static_scratch = nullptr;  // this device's address of g_splitk_static_scratch
};

// Split-K scratch owned by the library, for fp8q_gemm_w8a8_block_splitk_noalloc: 24 MiB of
// fp32 partials (192 tile-splits of 128 x 256).
constexpr int64_t kStaticScratchBytes = int64_t{24} << 20;
__device__ __align__(256) uint8_t g_splitk_static_scratch[kStaticScratchBytes];

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int device_state(DeviceState **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FP8Q_ERR_ARCH;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState &st = g_dev[dev];
  if (!st.probed) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return FP8Q_ERR_ARCH;
    st.is_sm100 = (major == 10 && minor == 0);
    st.sms = sms;
    st.probed = true;
  }
  if (!st.is_sm100) return FP8Q_ERR_ARCH;
  if (!st.attrs_set) {
    if (cudaFuncSetAttribute(fp8q::k_gemm_w8a8_block<false, false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             fp8q::kGemmSmemDense) != cudaSuccess ||
        cudaFuncSetAttribute(fp8q::k_gemm_w8a8_block<true, false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             fp8q::kGemmSmemGrouped) != cudaSuccess ||
        cudaFuncSetAttribute(fp8q::k_gemm_w8a8_block<false, true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             fp8q::BlockLayout<true>::smemDense) != cudaSuccess ||
        cudaFuncSetAttribute(fp8q::k_gemm_w8a8_block<true, true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             fp8q::BlockLayout<true>::smemGrouped) != cudaSuccess ||
        cudaFuncSetAttribute(fp8q::k_rmsnorm_quant_token<true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) !=
            cudaSuccess ||
        cudaFuncSetAttribute(fp8q::k_attn_decode_split<1>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, fp8q::kAttnSmem) !=
            cudaSuccess ||
        cudaFuncSetAttribute(fp8q::k_attn_decode_split<2>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, fp8q::kAttnSmem) !=
            cudaSuccess ||
        cudaFuncSetAttribute(fp8q::k_attn_decode_split<4>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, fp8q::kAttnSmem) !=
            cudaSuccess ||
        cudaFuncSetAttribute(fp8q::k_attn_decode_split<8>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, fp8q::kAttnSmem) !=
            cudaSuccess ||
        cudaFuncSetAttribute(fp8q::k_rmsnorm_quant_token<false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) !=
            cudaSuccess ||
        cudaFuncSetAttribute(fp8q::k_quant_rowwise<true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) !=
            cudaSuccess ||
        cudaFuncSetAttribute(fp8q::k_quant_rowwise<false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) !=
            cudaSuccess ||
        cudaFuncSetAttribute(fp8q::k_rmsnorm_quant_token<true, false, true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) !=
            cudaSuccess ||
        cudaFuncSetAttribute(fp8q::k_quant_rowwise<true, true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) !=
            cudaSuccess ||
        cudaFuncSetAttribute(fp8q::k_gemm_w8a8_rowwise,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             fp8q::kGemmSmemDense) != cudaSuccess ||
        cudaFuncSetAttribute(fp8q::k_gemm_w8a8_mx, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             fp8q::kGemmSmemDense) != cudaSuccess ||
        cudaFuncSetAttribute(fp8q::k_rmsnorm_quant_token<true, false, false, false,
                                                         fp8q::kScaleE8M0>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) !=
            cudaSuccess ||
        cudaFuncSetAttribute(fp8q::k_rmsnorm_quant_token<false, false, false, false,
                                                         fp8q::kScaleE8M0>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) !=
            cudaSuccess ||
        cudaFuncSetAttribute(fp8q::k_rmsnorm_quant_token<true, false, true, false,
                                                         fp8q::kScaleE8M0>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) !=
            cudaSuccess)
      return FP8Q_ERR_LAUNCH;
    st.attrs_set = true;
  }
  *out = &st;
  return FP8Q_OK;
}

int get_encoder() {
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_encode) return FP8Q_OK;
  void *fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
          cudaSuccess ||
      q != cudaDriverEntryPointSuccess || fn == nullptr)
    return FP8Q_ERR_LAUNCH;
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return FP8Q_OK;
}

// 2-D uint8 tensor map over a row-major [rows][ld] matrix, box = box_rows x 128 bytes, 128-byte
// swizzle, out-of-bounds elements read as zero.
int make_u8_map(CUtensorMap *map, const void *base, int64_t rows, int64_t cols, int64_t ld,
                uint32_t box_rows) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld)};
  const cuuint32_t box[2] = {128, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base),
                              dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FP8Q_OK : FP8Q_ERR_LAUNCH;
}

// 2-D bf16 tensor map over a row-major [rows][ld] output, box = 32 rows x 64 columns (128 bytes),
// 128-byte swizzle: the tile-store target of the block GEMM.
int make_bf16_out_map(CUtensorMap *map, void *base, int64_t rows, int64_t cols, int64_t ld) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld * 2)};
  const cuuint32_t box[2] = {64, 32};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box,
                              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FP8Q_OK : FP8Q_ERR_LAUNCH;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int launch_status() {
  return cudaGetLastError() == cudaSuccess ? FP8Q_OK : FP8Q_ERR_LAUNCH;
}

// Rasterization of the dense GEMMs: m-blocks per group, sized so that a group's rows of A
// (group_m x 128 rows x K codes) take at most 48 MiB of the 126 MB L2.  Each group streams the
// whole of B once, so larger groups read B fewer times: on the 8192 x 24576 x 4096 prefill GEMM one
// group of all 64 m-blocks reads 183 MB from DRAM against 437 MB with groups of 16 (1.04 x the
// algorithmic bytes instead of 1.50 x), and runs 2 % faster.
int raster_group_m(int64_t M, int64_t K) {
  const int64_t num_m = (M + fp8q::kBM - 1) / fp8q::kBM;
  int64_t g = (int64_t{48} << 20) / (int64_t{fp8q::kBM} * (K > 0 ? K : 1));
  if (g < 8) g = 8;
  if (g > num_m) g = num_m;
  return static_cast<int>(g < 1 ? 1 : g);
}

int check_gemm_common(const void *aq, int64_t lda, const float *sa, int64_t lds, const void *wq,
                      int64_t ldw, const void *sw, int sw_fmt, int64_t M, int64_t N, int64_t K,
                      const void *out, int64_t ldo) {
  if (sw_fmt != FP8Q_SCALE_F32 && sw_fmt != FP8Q_SCALE_E8M0) return FP8Q_ERR_ARG;
  if (M < 0 || N <= 0 || K <= 0 || N % 128 || K % 128) return FP8Q_ERR_SHAPE;
  if (M > INT32_MAX - 256 || N > (1 << 30) || K > 128 * fp8q::kMaxKB) return FP8Q_ERR_SHAPE;
  if (lda < K || ldw < K || ldo < N || lds < M) return FP8Q_ERR_SHAPE;
  if (M == 0) return FP8Q_OK;
  if (!aq || !sa || !wq || !sw || !out) return FP8Q_ERR_NULL;
  if (!aligned16(aq) || !aligned16(wq) || !aligned16(out) || !aligned16(sa) || !aligned16(sw) ||
      lda % 16 || ldw % 16 || ldo % 8 || lds % 4)
    return FP8Q_ERR_ALIGN;
  return FP8Q_OK;
}

// Split-K workspace: fp32 partials of one 128 x 256 tile per (tile, split).
constexpr int64_t kSplitPartialBytes = int64_t{fp8q::kBM} * fp8q::kBN * 4;

int64_t splitk_tiles(int64_t M, int64_t N) {
  return ((M + fp8q::kBM - 1) / fp8q::kBM) * ((N + fp8q::kBN - 1) / fp8q::kBN);
}

int64_t splitk_workspace_bytes(int64_t M, int64_t N, int splits) {
  if (splits <= 1) return 0;
  return splitk_tiles(M, N) * splits * kSplitPartialBytes;
}

// splits = 0 picks the K-split count from a cost model fitted to B200 measurements of this
// kernel (decode-sized M): time(S) ~ KB / S * t_kb + (S > 1 ? t_red + t_part * tiles * S : 0),
// with t_kb = 0.6 us per K-block of one CTA, t_red = 4.6 us for the reduction launch and
// t_part = 0.064 us per 128 x 256 fp32 partial written and re-read.  S is limited to one wave
// (tiles * S <= SMs).  Returns a count in [1, K/128] or 0 on error.
int resolve_splits(int64_t M, int64_t N, int64_t K, int splits, int sms) {
  const int64_t KB = K / fp8q::kBK;
  if (splits < 0 || splits > KB) return 0;
  if (splits > 0) return splits;
  const int64_t tiles = splitk_tiles(M, N);
  if (tiles <= 0 || tiles * 2 > sms) return 1;
  constexpr double t_kb = 0.6, t_red = 4.6, t_part = 0.064;
  int best = 1;
  double best_t = static_cast<double>(KB) * t_kb;
  for (int64_t s = 2; s <= KB && tiles * s <= sms; ++s) {
    const double t = static_cast<double>((KB + s - 1) / s) * t_kb + t_red +
                     t_part * static_cast<double>(tiles * s);
    if (t < best_t) {
      best_t = t;
      best = static_cast<int>(s);
    }
  }
  return best;
}

int launch_gemm(bool grouped, const void *aq, int64_t lda, const float *sa, int64_t lds,
                const void *wq, int64_t ldw, const void *sw, int sw_fmt,
                const int32_t *group_offsets, int64_t E, int64_t M, int64_t N, int64_t K,
                void *out, int64_t ldo, cudaStream_t stream, int splits = 1,
                void *workspace = nullptr, int64_t groups = 0) {
  DeviceState *st = nullptr;
  int rc = device_state(&st);
  if (rc != FP8Q_OK) return rc;
  if ((rc = get_encoder()) != FP8Q_OK) return rc;
  CUtensorMap tm_a, tm_b;
  // block-diagonal (groups > 0): A holds the groups' K-slices side by side, [M][groups * K]
  const int64_t a_cols = groups > 0 ? groups * K : K;
  if ((rc = make_u8_map(&tm_a, aq, M, a_cols, lda, fp8q::kBM)) != FP8Q_OK) return rc;
  const int64_t b_rows = grouped ? E * N : N;
  if ((rc = make_u8_map(&tm_b, wq, b_rows, K, ldw, fp8q::kBN)) != FP8Q_OK) return rc;
  fp8q::GemmArgs a;
  a.sa = sa;
  a.lds = lds;
  a.sw = sw;
  a.sw_fmt = sw_fmt;
  a.group_offsets = group_offsets;
  a.E = static_cast<int>(E);
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(N);
  a.K = static_cast<int>(K);
  a.out = static_cast<uint16_t *>(out);
  a.ldo = ldo;
  a.num_n = static_cast<int>((N + fp8q::kBN - 1) / fp8q::kBN);
  a.num_m = static_cast<int>((M + fp8q::kBM - 1) / fp8q::kBM);
  a.group_m = raster_group_m(M, K);
  a.splits = splits;
  a.ws = static_cast<float *>(workspace);
  a.n_tiles_per_group = groups > 0 ? static_cast<int>(N / groups / fp8q::kBN) : 0;
  // Upper bound of the tile count (grouped: every expert may add one partial m-tile).
  const int64_t tiles = (static_cast<int64_t>(a.num_m) + (grouped ? E : 0)) * a.num_n;
  const int64_t units = tiles * splits;
  const int grid = static_cast<int>(units < st->sms ? units : st->sms);
  // Tile stores by TMA when a CTA runs several tiles (the store then overlaps the next tile); one
  // tile per CTA keeps the deeper 4-stage operand ring instead.
  const bool ts = splits == 1 && tiles > st->sms;
  CUtensorMap tm_out;
  if (ts && (rc = make_bf16_out_map(&tm_out, out, M, N, ldo)) != FP8Q_OK) return rc;
  if (!ts) tm_out = tm_a;  // unused
  if (grouped && ts)
    fp8q::k_gemm_w8a8_block<true, true><<<grid, fp8q::kGemmThreads,
                                          fp8q::BlockLayout<true>::smemGrouped, stream>>>(
        tm_a, tm_b, tm_out, a);
  else if (grouped)
    fp8q::k_gemm_w8a8_block<true, false><<<grid, fp8q::kGemmThreads, fp8q::kGemmSmemGrouped,
                                           stream>>>(tm_a, tm_b, tm_out, a);
  else if (ts)
    fp8q::k_gemm_w8a8_block<false, true><<<grid, fp8q::kGemmThreads,
                                           fp8q::BlockLayout<true>::smemDense, stream>>>(
        tm_a, tm_b, tm_out, a);
  else
    fp8q::k_gemm_w8a8_block<false, false><<<grid, fp8q::kGemmThreads, fp8q::kGemmSmemDense,
                                            stream>>>(tm_a, tm_b, tm_out, a);
  if (splits > 1 && !grouped) {
    if ((rc = launch_status()) != FP8Q_OK) return rc;
    // the reduction as a programmatic dependent launch: it is scheduled while the GEMM drains and
    // waits in-kernel (griddepcontrol.wait) for the GEMM's partials
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(tiles * 8));
    cfg.blockDim = dim3(fp8q::kReduceThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, fp8q::k_splitk_reduce, static_cast<const float4 *>(workspace),
                           splits, a.num_m, a.num_n, a.group_m, a.M, a.N, a.out, ldo) !=
        cudaSuccess) {
      cudaGetLastError();
      return FP8Q_ERR_LAUNCH;
    }
  }
  return launch_status();
}

// Launch shape of the one-warp-per-row kernels: the warps per CTA (16, 12, 8, 4, 2 or 1) that keep
// the most warps resident per SM within the shared-memory budget; wpc == 0 if none fits.
struct RowLaunch {
  int wpc = 0, ctas = 0, smem = 0;
};
template <typename Kern>
RowLaunch pick_row_launch(Kern kern, int K, bool norm) {
  RowLaunch best;
  for (int wpc : {16, 12, 8, 4, 2, 1}) {
    const int smem = fp8q::token_smem_bytes(K, norm, wpc);
    if (smem > 227 * 1024) continue;
    int per_sm = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 32 * wpc, smem);
    if (per_sm * wpc > best.ctas * best.wpc) {
      best.wpc = wpc;
      best.ctas = per_sm;
      best.smem = smem;
    }
  }
  return best;
}

// Decode attention: positions per split, chosen so that B * Hkv * splits is about 2048 CTAs (a
// multiple of the tile, at least one tile, at most kAttnMaxChunk positions); depends on the sizes
// only, so the workspace query needs no device.
int attn_chunk(int64_t B, int64_t Hkv, int64_t max_seq_len) {
  const int64_t work = (max_seq_len > 0 ? max_seq_len : 1) * (B > 0 ? B : 1) * Hkv;
  int64_t c = (work + 2047) / 2048;
  c = (c + fp8q::kAttnTile - 1) / fp8q::kAttnTile * fp8q::kAttnTile;
  if (c < fp8q::kAttnTile) c = fp8q::kAttnTile;
  if (c > fp8q::kAttnMaxChunk) c = fp8q::kAttnMaxChunk;
  return static_cast<int>(c);
}

int attn_shape_status(int64_t B, int64_t Hq, int64_t Hkv, int64_t D, int64_t block_size,
                      int64_t max_seq_len) {
  // B and Hkv are grid dimensions (z, y)
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || D != fp8q::kAttnD || block_size <= 0 ||
      max_seq_len < 0 || max_seq_len > (1 << 30) || B > 65535 || Hkv > 1024)
    return FP8Q_ERR_SHAPE;
  const int64_t G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return FP8Q_ERR_SHAPE;
  return FP8Q_OK;
}

int64_t attn_workspace_bytes(int64_t B, int64_t Hq, int64_t Hkv, int64_t max_seq_len) {
  const int64_t chunk = attn_chunk(B, Hkv, max_seq_len);
  const int64_t nsplit = max_seq_len > 0 ? (max_seq_len + chunk - 1) / chunk : 1;
  return B * Hkv * nsplit * (Hq / Hkv) * (fp8q::kAttnD + 2) * 4;
}

}  // namespace

extern "C" {

int fp8q_abi_version(void) { return (1 << 16) | 6; }

const char *fp8q_status_string(int status) {
  switch (status) {
    case FP8Q_OK: return "ok";
    case FP8Q_ERR_NULL: return "null pointer argument";
    case FP8Q_ERR_SHAPE: return "unsupported shape (K and N must be multiples of 128; sizes >= 0; ld >= extent)";
    case FP8Q_ERR_ALIGN: return "pointer or leading dimension not 16-byte aligned";
    case FP8Q_ERR_ARCH: return "current device is not sm_100 (B200)";
    case FP8Q_ERR_LAUNCH: return "CUDA runtime or launch failure";
    case FP8Q_ERR_TIMEOUT: return "a kernel gave up on a bounded wait (outputs incomplete)";
    case FP8Q_ERR_ARG: return "enum argument out of range";
    case FP8Q_ERR_NOT_POW2: return "a scale given to the hardware block-scaled GEMM is not a power of two (outputs invalid)";
    case FP8Q_ERR_RANGE: return "an index or scale input was outside its valid range (a RoPE position, a cache slot, a non-positive or non-finite scale); the affected rows were not written";
    case FP8Q_ERR_TOO_LARGE: return "problem needs more split-K scratch than the library's static 24 MiB buffer (use fp8q_gemm_w8a8_block_splitk with a workspace, or fewer splits)";
    default: return "unknown status";
  }
}

int fp8q_quant_weight_block(const void *w_bf16, int64_t N, int64_t K, int64_t ldw,
                            void *wq_e4m3, int64_t ldq, void *sw, int sw_fmt,
                            cudaStream_t stream) {
  if (sw_fmt != FP8Q_SCALE_F32 && sw_fmt != FP8Q_SCALE_E8M0) return FP8Q_ERR_ARG;
  if (N < 0 || K < 0 || N % 128 || K % 128) return FP8Q_ERR_SHAPE;
  if (ldw < K || ldq < K) return FP8Q_ERR_SHAPE;
  if (N == 0 || K == 0) return FP8Q_OK;
  if (!w_bf16 || !wq_e4m3 || !sw) return FP8Q_ERR_NULL;
  if (!aligned16(w_bf16) || !aligned16(wq_e4m3) || ldw % 8 || ldq % 16) return FP8Q_ERR_ALIGN;
  if (sw_fmt == FP8Q_SCALE_F32 && (reinterpret_cast<uintptr_t>(sw) & 3u)) return FP8Q_ERR_ALIGN;
  DeviceState *st = nullptr;
  const int rc = device_state(&st);
  if (rc != FP8Q_OK) return rc;
  const int KB = static_cast<int>(K / 128);
  const int64_t nblocks = (N / 128) * (K / 128);
  const int64_t grid = nblocks < (1ll << 30) ? nblocks : (1ll << 30);
  const auto *w = static_cast<const uint16_t *>(w_bf16);
  auto *q = static_cast<uint8_t *>(wq_e4m3);
  if (sw_fmt == FP8Q_SCALE_F32)
    fp8q::k_quant_weight_block<fp8q::kScaleF32><<<static_cast<unsigned>(grid), 256, 0, stream>>>(
        w, ldw, q, ldq, sw, KB, nblocks);
  else
    fp8q::k_quant_weight_block<fp8q::kScaleE8M0><<<static_cast<unsigned>(grid), 256, 0, stream>>>(
        w, ldw, q, ldq, sw, KB, nblocks);
  return launch_status();
}

static_assert(sizeof(fp8q_weight_desc) == sizeof(fp8q::WeightDesc),
              "fp8q_weight_desc and the kernel's descriptor must match");

int fp8q_quant_weight_block_batched(const fp8q_weight_desc *descs, int64_t count,
                                    int64_t total_blocks, int sw_fmt, cudaStream_t stream) {
  if (sw_fmt != FP8Q_SCALE_F32 && sw_fmt != FP8Q_SCALE_E8M0) return FP8Q_ERR_ARG;
  if (count < 0 || count > fp8q::kMaxBatchMatrices || total_blocks < 0) return FP8Q_ERR_SHAPE;
  if (count == 0 || total_blocks == 0) return FP8Q_OK;
  if (!descs) return FP8Q_ERR_NULL;
  if (reinterpret_cast<uintptr_t>(descs) & 7u) return FP8Q_ERR_ALIGN;
  DeviceState *st = nullptr;
  const int rc = device_state(&st);
  if (rc != FP8Q_OK) return rc;
  const int64_t cap = static_cast<int64_t>(st->sms) * 4;
  const int grid = static_cast<int>(total_blocks < cap ? total_blocks : cap);
  const auto *d = reinterpret_cast<const fp8q::WeightDesc *>(descs);
  if (sw_fmt == FP8Q_SCALE_F32)
    fp8q::k_quant_weight_block_batched<fp8q::kScaleF32><<<grid, 256, 0, stream>>>(
        d, static_cast<int>(count), total_blocks);
  else
    fp8q::k_quant_weight_block_batched<fp8q::kScaleE8M0><<<grid, 256, 0, stream>>>(
        d, static_cast<int>(count), total_blocks);
  return launch_status();
}

}  // extern "C"

namespace {

template <int FMT>
int rmsnorm_quant_token_impl(const void *x_bf16, const void *gamma_bf16, float eps, int64_t M,
                             int64_t K, int64_t ldx, void *xq_e4m3, int64_t ldq, float *sa,
                             int64_t lds, cudaStream_t stream) {
  if (M < 0 || K <= 0 || K % 128 || K > kMaxTokenK) return FP8Q_ERR_SHAPE;
  if (ldx < K || ldq < K || lds < M) return FP8Q_ERR_SHAPE;
  if (M == 0) return FP8Q_OK;
  if (!x_bf16 || !xq_e4m3 || !sa) return FP8Q_ERR_NULL;
  if (!aligned16(x_bf16) || !aligned16(xq_e4m3) || !aligned16(sa) || ldx % 8 || ldq % 16 ||
      lds % 4 || (gamma_bf16 && !aligned16(gamma_bf16)))
    return FP8Q_ERR_ALIGN;
  DeviceState *st = nullptr;
  const int rc = device_state(&st);
  if (rc != FP8Q_OK) return rc;
  const bool norm = gamma_bf16 != nullptr;
  const RowLaunch L =
      norm ? pick_row_launch(fp8q::k_rmsnorm_quant_token<true, false, false, false, FMT>,
                             static_cast<int>(K), true)
           : pick_row_launch(fp8q::k_rmsnorm_quant_token<false, false, false, false, FMT>,
                             static_cast<int>(K), false);
  if (L.wpc == 0) return FP8Q_ERR_SHAPE;
  const int wpc = L.wpc, smem = L.smem;
  // the plain kernel spreads (row, step) units over the warps, the fused one whole rows
  const int64_t units = norm ? M : M * ((K / 128 + 7) / 8);
  // plain, K/128 not a multiple of the 8 blocks of a warp step: the packed walk (8 consecutive
  // blocks of the flattened (row, block) sequence per warp step)
  const bool packed = !norm && (K / 128) % 8 != 0;
  const int64_t need = (units + wpc - 1) / wpc;
  const int64_t cap = static_cast<int64_t>(st->sms) * L.ctas;
  const int grid = static_cast<int>(need < cap ? need : cap);
  const auto *x = static_cast<const uint16_t *>(x_bf16);
  const auto *g = static_cast<const uint16_t *>(gamma_bf16);
  auto *q = static_cast<uint8_t *>(xq_e4m3);
  if (norm)
    fp8q::k_rmsnorm_quant_token<true, false, false, false, FMT><<<grid, 32 * wpc, smem, stream>>>(
        x, ldx, g, eps, M, static_cast<int>(K), q, ldq, sa, lds, nullptr, 0);
  else if (packed) {
    const int64_t pneed = ((M * (K / 128) + 7) / 8 + wpc - 1) / wpc;
    const int pgrid = static_cast<int>(pneed < cap ? pneed : cap);
    fp8q::k_rmsnorm_quant_token<false, false, false, true, FMT><<<pgrid, 32 * wpc, smem, stream>>>(
        x, ldx, nullptr, eps, M, static_cast<int>(K), q, ldq, sa, lds, nullptr, 0);
  } else if (M < static_cast<int64_t>(grid) * wpc)  // fewer rows than warps: spread the steps
    fp8q::k_rmsnorm_quant_token<false, true, false, false, FMT><<<grid, 32 * wpc, smem, stream>>>(
        x, ldx, nullptr, eps, M, static_cast<int>(K), q, ldq, sa, lds, nullptr, 0);
  else
    fp8q::k_rmsnorm_quant_token<false, false, false, false, FMT><<<grid, 32 * wpc, smem, stream>>>(
        x, ldx, nullptr, eps, M, static_cast<int>(K), q, ldq, sa, lds, nullptr, 0);
  return launch_status();
}

}  // namespace

extern "C" {

int fp8q_rmsnorm_quant_token(const void *x_bf16, const void *gamma_bf16, float eps, int64_t M,
                             int64_t K, int64_t ldx, void *xq_e4m3, int64_t ldq, float *sa,
                             int64_t lds, cudaStream_t stream) {
  return rmsnorm_quant_token_impl<fp8q::kScaleF32>(x_bf16, gamma_bf16, eps, M, K, ldx, xq_e4m3,
                                                   ldq, sa, lds, stream);
}

int fp8q_rmsnorm_quant_token_fmt(const void *x_bf16, const void *gamma_bf16, float eps,
                                 int64_t M, int64_t K, int64_t ldx, void *xq_e4m3, int64_t ldq,
                                 float *sa, int64_t lds, int sa_fmt, cudaStream_t stream) {
  if (sa_fmt == FP8Q_SCALE_F32)
    return rmsnorm_quant_token_impl<fp8q::kScaleF32>(x_bf16, gamma_bf16, eps, M, K, ldx,
                                                     xq_e4m3, ldq, sa, lds, stream);
  if (sa_fmt == FP8Q_SCALE_E8M0)
    return rmsnorm_quant_token_impl<fp8q::kScaleE8M0>(x_bf16, gamma_bf16, eps, M, K, ldx,
                                                      xq_e4m3, ldq, sa, lds, stream);
  return FP8Q_ERR_ARG;
}

int fp8q_gemm_w8a8_block(const void *aq, int64_t lda, const float *sa, int64_t lds,
                         const void *wq, int64_t ldw, const void *sw, int sw_fmt, int64_t M,
                         int64_t N, int64_t K, void *out_bf16, int64_t ldo,
                         cudaStream_t stream) {
  int rc = check_gemm_common(aq, lda, sa, lds, wq, ldw, sw, sw_fmt, M, N, K, out_bf16, ldo);
  if (rc != FP8Q_OK || M == 0) return rc;
  if (sw_fmt == FP8Q_SCALE_F32 && (reinterpret_cast<uintptr_t>(sw) & 3u)) return FP8Q_ERR_ALIGN;
  return launch_gemm(false, aq, lda, sa, lds, wq, ldw, sw, sw_fmt, nullptr, 1, M, N, K, out_bf16,
                     ldo, stream);
}

int fp8q_gemm_w8a8_block_diag(const void *aq, int64_t lda, const float *sa, int64_t lds,
                              const void *wq, int64_t ldw, const void *sw, int sw_fmt,
                              int64_t G, int64_t M, int64_t N_g, int64_t K_g, void *out_bf16,
                              int64_t ldo, cudaStream_t stream) {
  if (G <= 0 || G > (1 << 16) || N_g <= 0 || N_g % fp8q::kBN) return FP8Q_ERR_SHAPE;
  if (N_g > (1 << 30) / G || K_g > (1 << 30) / G) return FP8Q_ERR_SHAPE;
  int rc = check_gemm_common(aq, lda, sa, lds, wq, ldw, sw, sw_fmt, M, G * N_g, K_g, out_bf16,
                             ldo);
  if (rc != FP8Q_OK || M == 0) return rc;
  if (lda < G * K_g) return FP8Q_ERR_SHAPE;
  if (sw_fmt == FP8Q_SCALE_F32 && (reinterpret_cast<uintptr_t>(sw) & 3u)) return FP8Q_ERR_ALIGN;
  return launch_gemm(false, aq, lda, sa, lds, wq, ldw, sw, sw_fmt, nullptr, 1, M, G * N_g, K_g,
                     out_bf16, ldo, stream, 1, nullptr, G);
}

int fp8q_gemm_splitk_workspace_bytes(int64_t M, int64_t N, int64_t K, int splits,
                                     int64_t *bytes) {
  if (!bytes) return FP8Q_ERR_NULL;
  *bytes = 0;
  if (M < 0 || N <= 0 || K <= 0 || N % 128 || K % 128) return FP8Q_ERR_SHAPE;
  if (M > INT32_MAX - 256 || N > (1 << 30) || K > 128 * fp8q::kMaxKB) return FP8Q_ERR_SHAPE;
  if (splits < 0 || splits > K / 128) return FP8Q_ERR_ARG;
  int sms = 0;
  if (splits == 0) {
    DeviceState *st = nullptr;
    const int rc = device_state(&st);
    if (rc != FP8Q_OK) return rc;
    sms = st->sms;
  }
  const int s = resolve_splits(M, N, K, splits, sms);
  if (s <= 0) return FP8Q_ERR_ARG;
  if (splitk_tiles(M, N) * s > INT32_MAX) return FP8Q_ERR_SHAPE;
  *bytes = splitk_workspace_bytes(M, N, s);
  return FP8Q_OK;
}

int fp8q_gemm_w8a8_block_splitk(const void *aq, int64_t lda, const float *sa, int64_t lds,
                                const void *wq, int64_t ldw, const void *sw, int sw_fmt,
                                int64_t M, int64_t N, int64_t K, void *out_bf16, int64_t ldo,
                                int splits, void *workspace, int64_t workspace_bytes,
                                cudaStream_t stream) {
  int rc = check_gemm_common(aq, lda, sa, lds, wq, ldw, sw, sw_fmt, M, N, K, out_bf16, ldo);
  if (rc != FP8Q_OK) return rc;
  if (splits < 0 || splits > K / 128) return FP8Q_ERR_ARG;
  if (M == 0) return FP8Q_OK;
  if (sw_fmt == FP8Q_SCALE_F32 && (reinterpret_cast<uintptr_t>(sw) & 3u)) return FP8Q_ERR_ALIGN;
  DeviceState *st = nullptr;
  if ((rc = device_state(&st)) != FP8Q_OK) return rc;
  const int s = resolve_splits(M, N, K, splits, st->sms);
  if (s <= 0) return FP8Q_ERR_ARG;
  if (splitk_tiles(M, N) * s > INT32_MAX) return FP8Q_ERR_SHAPE;
  if (s > 1) {
    if (!workspace) return FP8Q_ERR_NULL;
    if (!aligned16(workspace)) return FP8Q_ERR_ALIGN;
    if (workspace_bytes < splitk_workspace_bytes(M, N, s)) return FP8Q_ERR_SHAPE;
  }
  return launch_gemm(false, aq, lda, sa, lds, wq, ldw, sw, sw_fmt, nullptr, 1, M, N, K, out_bf16,
                     ldo, stream, s, s > 1 ? workspace : nullptr);
}

int fp8q_gemm_w8a8_block_splitk_noalloc(const void *aq, int64_t lda, const float *sa,
                                        int64_t lds, const void *wq, int64_t ldw, const void *sw,
                                        int sw_fmt, int64_t M, int64_t N, int64_t K,
                                        void *out_bf16, int64_t ldo, int splits,
                                        cudaStream_t stream) {
  int rc = check_gemm_common(aq, lda, sa, lds, wq, ldw, sw, sw_fmt, M, N, K, out_bf16, ldo);
  if (rc != FP8Q_OK) return rc;
  if (splits < 0 || splits > K / 128) return FP8Q_ERR_ARG;
  if (M == 0) return FP8Q_OK;
  if (sw_fmt == FP8Q_SCALE_F32 && (reinterpret_cast<uintptr_t>(sw) & 3u)) return FP8Q_ERR_ALIGN;
  DeviceState *st = nullptr;
  if ((rc = device_state(&st)) != FP8Q_OK) return rc;
  const int s = resolve_splits(M, N, K, splits, st->sms);
  if (s <= 0) return FP8Q_ERR_ARG;
  const int64_t tiles = splitk_tiles(M, N);
  if (tiles * s > INT32_MAX) return FP8Q_ERR_SHAPE;
  if (s == 1)
    return launch_gemm(false, aq, lda, sa, lds, wq, ldw, sw, sw_fmt, nullptr, 1, M, N, K,
                       out_bf16, ldo, stream);
  if (tiles * s * kSplitPartialBytes > kStaticScratchBytes) return FP8Q_ERR_TOO_LARGE;
  void *scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!st->static_scratch) {
      // once per device, with that device current (device_state resolved the current device)
      if (cudaGetSymbolAddress(&st->static_scratch, g_splitk_static_scratch) != cudaSuccess) {
        st->static_scratch = nullptr;
        return FP8Q_ERR_LAUNCH;
      }
    }
    scratch = st->static_scratch;
  }
  return launch_gemm(false, aq, lda, sa, lds, wq, ldw, sw, sw_fmt, nullptr, 1, M, N, K, out_bf16,
                     ldo, stream, s, scratch);
}

int fp8q_grouped_gemm_w8a8_block(const void *aq, int64_t lda, const float *sa, int64_t lds,
                                 const void *wq, int64_t ldw, const void *sw, int sw_fmt,
                                 const int32_t *group_offsets, int64_t E, int64_t M, int64_t N,
                                 int64_t K, void *out_bf16, int64_t ldo, cudaStream_t stream) {
  if (E <= 0 || E > fp8q::kMaxExperts) return FP8Q_ERR_SHAPE;
  int rc = check_gemm_common(aq, lda, sa, lds, wq, ldw, sw, sw_fmt, M, N, K, out_bf16, ldo);
  if (rc != FP8Q_OK || M == 0) return rc;
  if (!group_offsets) return FP8Q_ERR_NULL;
  if (E * N > INT32_MAX) return FP8Q_ERR_SHAPE;
  return launch_gemm(true, aq, lda, sa, lds, wq, ldw, sw, sw_fmt, group_offsets, E, M, N, K,
                     out_bf16, ldo, stream);
}

int fp8q_quant_rowwise(const void *x_bf16, const void *gamma_bf16, float eps, int64_t M,
                       int64_t K, int64_t ldx, void *q_e4m3, int64_t ldq, float *s,
                       cudaStream_t stream) {
  if (M < 0 || K <= 0 || K % 128 || K > kMaxTokenK) return FP8Q_ERR_SHAPE;
  if (ldx < K || ldq < K) return FP8Q_ERR_SHAPE;
  if (M == 0) return FP8Q_OK;
  if (!x_bf16 || !q_e4m3 || !s) return FP8Q_ERR_NULL;
  if (!aligned16(x_bf16) || !aligned16(q_e4m3) || (reinterpret_cast<uintptr_t>(s) & 3u) ||
      ldx % 8 || ldq % 16 || (gamma_bf16 && !aligned16(gamma_bf16)))
    return FP8Q_ERR_ALIGN;
  DeviceState *st = nullptr;
  const int rc = device_state(&st);
  if (rc != FP8Q_OK) return rc;
  const bool norm = gamma_bf16 != nullptr;
  if (!norm && K <= 4096) {  // the row fits in registers: one pass over memory
    const auto *x = static_cast<const uint16_t *>(x_bf16);
    auto *q = static_cast<uint8_t *>(q_e4m3);
    const int Ki = static_cast<int>(K);
    int per_sm = 0;
    auto launch = [&](auto kern) {
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, 0);
      const int64_t need = (M + 7) / 8, cap = static_cast<int64_t>(st->sms) * (per_sm > 0 ? per_sm : 1);
      kern<<<static_cast<int>(need < cap ? need : cap), 256, 0, stream>>>(x, ldx, M, Ki, q, ldq, s);
    };
    if (K <= 1024) launch(fp8q::k_quant_rowwise_regs<4>);
    else if (K <= 2048) launch(fp8q::k_quant_rowwise_regs<8>);
    else launch(fp8q::k_quant_rowwise_regs<16>);
    return launch_status();
  }
  const RowLaunch L = norm
                           ? pick_row_launch(fp8q::k_quant_rowwise<true>, static_cast<int>(K), true)
                           : pick_row_launch(fp8q::k_quant_rowwise<false>, static_cast<int>(K), false);
  if (L.wpc == 0) return FP8Q_ERR_SHAPE;
  const int wpc = L.wpc, smem = L.smem;
  const int64_t need = (M + wpc - 1) / wpc;
  const int64_t cap = static_cast<int64_t>(st->sms) * L.ctas;
  const int grid = static_cast<int>(need < cap ? need : cap);
  const auto *x = static_cast<const uint16_t *>(x_bf16);
  const auto *g = static_cast<const uint16_t *>(gamma_bf16);
  auto *q = static_cast<uint8_t *>(q_e4m3);
  if (norm)
    fp8q::k_quant_rowwise<true><<<grid, 32 * wpc, smem, stream>>>(
        x, ldx, g, eps, M, static_cast<int>(K), q, ldq, s, nullptr, 0);
  else
    fp8q::k_quant_rowwise<false><<<grid, 32 * wpc, smem, stream>>>(
        x, ldx, nullptr, eps, M, static_cast<int>(K), q, ldq, s, nullptr, 0);
  return launch_status();
}

int fp8q_add_rmsnorm_quant(const void *x_bf16, int64_t ldx, void *residual_bf16, int64_t ldr,
                           const void *gamma_bf16, float eps, int64_t M, int64_t K, int per_token,
                           int sa_fmt, void *q_e4m3, int64_t ldq, float *sa, int64_t lds,
                           cudaStream_t stream) {
  if (M < 0 || K <= 0 || K % 128 || K > kMaxTokenK) return FP8Q_ERR_SHAPE;
  if (per_token != 0 && per_token != 1) return FP8Q_ERR_ARG;
  if (sa_fmt != FP8Q_SCALE_F32 && sa_fmt != FP8Q_SCALE_E8M0) return FP8Q_ERR_ARG;
  if (per_token && sa_fmt != FP8Q_SCALE_F32) return FP8Q_ERR_ARG;
  if (ldx < K || ldr < K || ldq < K || (!per_token && lds < M)) return FP8Q_ERR_SHAPE;
  if (M == 0) return FP8Q_OK;
  if (!x_bf16 || !residual_bf16 || !gamma_bf16 || !q_e4m3 || !sa) return FP8Q_ERR_NULL;
  if (!aligned16(x_bf16) || !aligned16(residual_bf16) || !aligned16(gamma_bf16) ||
      !aligned16(q_e4m3) || ldx % 8 || ldr % 8 || ldq % 16 ||
      (per_token ? (reinterpret_cast<uintptr_t>(sa) & 3u) != 0 : (!aligned16(sa) || lds % 4)))
    return FP8Q_ERR_ALIGN;
  {  // x is read while the residual is written: the two row ranges must not overlap
    const auto xb = reinterpret_cast<uintptr_t>(x_bf16), rb = reinterpret_cast<uintptr_t>(residual_bf16);
    const uintptr_t xe = xb + static_cast<uintptr_t>(((M - 1) * ldx + K) * 2);
    const uintptr_t re = rb + static_cast<uintptr_t>(((M - 1) * ldr + K) * 2);
    if (xb < re && rb < xe) return FP8Q_ERR_ARG;
  }
  DeviceState *st = nullptr;
  const int rc = device_state(&st);
  if (rc != FP8Q_OK) return rc;
  const RowLaunch L =
      per_token
          ? pick_row_launch(fp8q::k_quant_rowwise<true, true>, static_cast<int>(K), true)
          : pick_row_launch(fp8q::k_rmsnorm_quant_token<true, false, true>, static_cast<int>(K), true);
  if (L.wpc == 0) return FP8Q_ERR_SHAPE;
  const int wpc = L.wpc, smem = L.smem;
  const int64_t need = (M + wpc - 1) / wpc;
  const int64_t cap = static_cast<int64_t>(st->sms) * L.ctas;
  const int grid = static_cast<int>(need < cap ? need : cap);
  const auto *x = static_cast<const uint16_t *>(x_bf16);
  auto *res = static_cast<uint16_t *>(residual_bf16);
  const auto *g = static_cast<const uint16_t *>(gamma_bf16);
  auto *q = static_cast<uint8_t *>(q_e4m3);
  if (per_token)
    fp8q::k_quant_rowwise<true, true><<<grid, 32 * wpc, smem, stream>>>(
        x, ldx, g, eps, M, static_cast<int>(K), q, ldq, sa, res, ldr);
  else if (sa_fmt == FP8Q_SCALE_E8M0)
    fp8q::k_rmsnorm_quant_token<true, false, true, false, fp8q::kScaleE8M0>
        <<<grid, 32 * wpc, smem, stream>>>(x, ldx, g, eps, M, static_cast<int>(K), q, ldq, sa,
                                           lds, res, ldr);
  else
    fp8q::k_rmsnorm_quant_token<true, false, true><<<grid, 32 * wpc, smem, stream>>>(
        x, ldx, g, eps, M, static_cast<int>(K), q, ldq, sa, lds, res, ldr);
  return launch_status();
}

int fp8q_silu_mul_quant(const void *h_bf16, int64_t R, int64_t I, int64_t ldh, void *q_e4m3,
                        int64_t ldq, float *sa, int64_t lds, int sa_fmt, cudaStream_t stream) {
  if (R < 0 || I <= 0 || I % 128 || I > kMaxTokenK) return FP8Q_ERR_SHAPE;
  if (sa_fmt != FP8Q_SCALE_F32 && sa_fmt != FP8Q_SCALE_E8M0) return FP8Q_ERR_ARG;
  if (ldh < 2 * I || ldq < I || lds < R) return FP8Q_ERR_SHAPE;
  if (R == 0) return FP8Q_OK;
  if (!h_bf16 || !q_e4m3 || !sa) return FP8Q_ERR_NULL;
  if (!aligned16(h_bf16) || !aligned16(q_e4m3) || !aligned16(sa) || ldh % 8 || ldq % 16 ||
      lds % 4)
    return FP8Q_ERR_ALIGN;
  DeviceState *st = nullptr;
  const int rc = device_state(&st);
  if (rc != FP8Q_OK) return rc;
  const int smem = static_cast<int>(sizeof(fp8q::ScaleTab));
  int best_wpc = 0, best_ctas = 0;
  for (int wpc : {16, 8, 4}) {
    int per_sm = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fp8q::k_silu_mul_quant<false>,
                                                  32 * wpc, smem);
    if (per_sm * wpc > best_ctas * best_wpc) {
      best_wpc = wpc;
      best_ctas = per_sm;
    }
  }
  if (best_wpc == 0) return FP8Q_ERR_LAUNCH;
  const int64_t cap = static_cast<int64_t>(st->sms) * best_ctas;
  if ((I / 128) % 4 != 0) {  // packed walk: 4 consecutive blocks of the flattened (row, block) order
    const int64_t need = ((R * (I / 128) + 3) / 4 + best_wpc - 1) / best_wpc;
    const int grid = static_cast<int>(need < cap ? need : cap);
    if (sa_fmt == FP8Q_SCALE_E8M0)
      fp8q::k_silu_mul_quant<true, fp8q::kScaleE8M0><<<grid, 32 * best_wpc, smem, stream>>>(
          static_cast<const uint16_t *>(h_bf16), ldh, R, static_cast<int>(I),
          static_cast<uint8_t *>(q_e4m3), ldq, sa, lds);
    else
      fp8q::k_silu_mul_quant<true><<<grid, 32 * best_wpc, smem, stream>>>(
          static_cast<const uint16_t *>(h_bf16), ldh, R, static_cast<int>(I),
          static_cast<uint8_t *>(q_e4m3), ldq, sa, lds);
    return launch_status();
  }
  const int64_t need = (R + best_wpc - 1) / best_wpc;
  const int grid = static_cast<int>(need < cap ? need : cap);
  if (sa_fmt == FP8Q_SCALE_E8M0)
    fp8q::k_silu_mul_quant<false, fp8q::kScaleE8M0><<<grid, 32 * best_wpc, smem, stream>>>(
        static_cast<const uint16_t *>(h_bf16), ldh, R, static_cast<int>(I),
        static_cast<uint8_t *>(q_e4m3), ldq, sa, lds);
  else
    fp8q::k_silu_mul_quant<false><<<grid, 32 * best_wpc, smem, stream>>>(
        static_cast<const uint16_t *>(h_bf16), ldh, R, static_cast<int>(I),
        static_cast<uint8_t *>(q_e4m3), ldq, sa, lds);
  return launch_status();
}

int fp8q_inverse_rope_quant(const void *o_bf16, int64_t ldo, const int64_t *positions,
                            const float *cos_cache, const float *sin_cache, int64_t max_pos,
                            int64_t T, int64_t H, int64_t D, int64_t rope_dim, int interleaved,
                            int scale_fmt, void *q_e4m3, int64_t ldq, float *sa, int64_t lds,
                            cudaStream_t stream) {
  if (scale_fmt != FP8Q_SCALE_F32 && scale_fmt != FP8Q_SCALE_E8M0) return FP8Q_ERR_ARG;
  if (interleaved != 0 && interleaved != 1) return FP8Q_ERR_ARG;
  if (T < 0 || H <= 0 || D <= 0 || D % 8 || rope_dim < 0 || rope_dim > D || rope_dim % 8)
    return FP8Q_ERR_SHAPE;
  if (!interleaved && rope_dim % 16) return FP8Q_ERR_SHAPE;
  if (H > (1 << 24) / D) return FP8Q_ERR_SHAPE;
  const int64_t K = H * D;
  if (K % 128 || ldo < K || ldq < K || lds < T) return FP8Q_ERR_SHAPE;
  if (rope_dim > 0 && max_pos <= 0) return FP8Q_ERR_SHAPE;
  if (T == 0) return FP8Q_OK;
  if (!o_bf16 || !q_e4m3 || !sa) return FP8Q_ERR_NULL;
  if (rope_dim > 0 && (!positions || !cos_cache || !sin_cache)) return FP8Q_ERR_NULL;
  if (!aligned16(o_bf16) || !aligned16(q_e4m3) || !aligned16(sa) || ldo % 8 || ldq % 16 ||
      lds % 4)
    return FP8Q_ERR_ALIGN;
  if (rope_dim > 0 && (!aligned16(cos_cache) || !aligned16(sin_cache) ||
                       reinterpret_cast<uintptr_t>(positions) % 8))
    return FP8Q_ERR_ALIGN;
  DeviceState *st = nullptr;
  const int rc = device_state(&st);
  if (rc != FP8Q_OK) return rc;
  using Kernel = void (*)(const uint16_t *, int64_t, const int64_t *, const float *,
                          const float *, int64_t, int64_t, int, int, int, uint8_t *, int64_t,
                          float *, int64_t);
  const Kernel k = scale_fmt == FP8Q_SCALE_F32
                       ? (interleaved ? fp8q::k_inverse_rope_quant<fp8q::kScaleF32, true>
                                      : fp8q::k_inverse_rope_quant<fp8q::kScaleF32, false>)
                       : (interleaved ? fp8q::k_inverse_rope_quant<fp8q::kScaleE8M0, true>
                                      : fp8q::k_inverse_rope_quant<fp8q::kScaleE8M0, false>);
  const int smem = static_cast<int>(sizeof(fp8q::ScaleTab));
  const int wpc = 16;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, 32 * wpc, smem) != cudaSuccess ||
      per_sm == 0)
    return FP8Q_ERR_LAUNCH;
  const int64_t need = (T + wpc - 1) / wpc;
  const int64_t cap = static_cast<int64_t>(st->sms) * per_sm;
  const int grid = static_cast<int>(need < cap ? need : cap);
  k<<<grid, 32 * wpc, smem, stream>>>(static_cast<const uint16_t *>(o_bf16), ldo, positions,
                                     cos_cache, sin_cache, max_pos, T, static_cast<int>(D),
                                     static_cast<int>(rope_dim), static_cast<int>(K),
                                     static_cast<uint8_t *>(q_e4m3), ldq, sa, lds);
  return launch_status();
}

int fp8q_qkv_scales(const void *qkv_bf16, int64_t T, int64_t ld, int64_t Hq, int64_t Hkv,
                    int64_t D, float *amax3, float *scale3, cudaStream_t stream) {
  if (T < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || D % 8) return FP8Q_ERR_SHAPE;
  if ((Hq + 2 * Hkv) * D > (1 << 24) || ld < (Hq + 2 * Hkv) * D) return FP8Q_ERR_SHAPE;
  if (!amax3 || !scale3 || (T > 0 && !qkv_bf16)) return FP8Q_ERR_NULL;
  if ((T > 0 && !aligned16(qkv_bf16)) || ld % 8 || (reinterpret_cast<uintptr_t>(amax3) & 3u) ||
      (reinterpret_cast<uintptr_t>(scale3) & 3u))
    return FP8Q_ERR_ALIGN;
  DeviceState *st = nullptr;
  const int rc = device_state(&st);
  if (rc != FP8Q_OK) return rc;
  if (cudaMemsetAsync(amax3, 0, 3 * sizeof(float), stream) != cudaSuccess) return FP8Q_ERR_LAUNCH;
  if (T > 0) {
    const int64_t need = (T + 7) / 8;
    const int64_t cap = static_cast<int64_t>(st->sms) * 8;
    const int grid = static_cast<int>(need < cap ? need : cap);
    fp8q::k_qkv_amax<<<grid, 256, 0, stream>>>(
        static_cast<const uint16_t *>(qkv_bf16), ld, T, static_cast<int>(Hq * D / 8),
        static_cast<int>(Hkv * D / 8), static_cast<int>(Hkv * D / 8),
        reinterpret_cast<uint32_t *>(amax3));
    const int lrc = launch_status();
    if (lrc != FP8Q_OK) return lrc;
  }
  fp8q::k_qkv_finalize<<<1, 32, 0, stream>>>(reinterpret_cast<const uint32_t *>(amax3), scale3);
  return launch_status();
}

int fp8q_kv_cache_write(const void *qkv_bf16, int64_t T, int64_t ld, int64_t Hq, int64_t Hkv,
                        int64_t D, const int64_t *slots, int64_t num_slots, const float *scale3,
                        void *q_e4m3, int64_t ldq, void *k_cache, void *v_cache,
                        cudaStream_t stream) {
  if (T < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || D % 16 || num_slots < 0) return FP8Q_ERR_SHAPE;
  if ((Hq + 2 * Hkv) * D > (1 << 24) || ld < (Hq + 2 * Hkv) * D) return FP8Q_ERR_SHAPE;
  if (q_e4m3 && ldq < Hq * D) return FP8Q_ERR_SHAPE;
  if (T == 0) return FP8Q_OK;
  if (!qkv_bf16 || !slots || !scale3 || !k_cache || !v_cache) return FP8Q_ERR_NULL;
  if (!aligned16(qkv_bf16) || ld % 8 || (reinterpret_cast<uintptr_t>(slots) & 7u) ||
      (reinterpret_cast<uintptr_t>(scale3) & 3u) || (reinterpret_cast<uintptr_t>(k_cache) & 7u) ||
      (reinterpret_cast<uintptr_t>(v_cache) & 7u) ||
      (q_e4m3 && ((reinterpret_cast<uintptr_t>(q_e4m3) & 7u) || ldq % 8)))
    return FP8Q_ERR_ALIGN;
  DeviceState *st = nullptr;
  const int rc = device_state(&st);
  if (rc != FP8Q_OK) return rc;
  const int64_t cap = static_cast<int64_t>(st->sms) * 16;
  const int grid = static_cast<int>(T < cap ? T : cap);
  fp8q::k_kv_cache_write<<<grid, fp8q::kKvThreads, 0, stream>>>(
      static_cast<const uint16_t *>(qkv_bf16), ld, T, static_cast<int>(Hq * D / 8),
      static_cast<int>(Hkv * D / 8), slots, num_slots, scale3, static_cast<uint8_t *>(q_e4m3),
      ldq, static_cast<uint8_t *>(k_cache), static_cast<uint8_t *>(v_cache));
  return launch_status();
}

int fp8q_attention_decode_workspace_bytes(int64_t B, int64_t Hq, int64_t Hkv, int64_t D,
                                          int64_t max_seq_len, int64_t *bytes) {
  if (!bytes) return FP8Q_ERR_NULL;
  *bytes = 0;
  const int rc = attn_shape_status(B, Hq, Hkv, D, 1, max_seq_len);
  if (rc != FP8Q_OK) return rc;
  *bytes = attn_workspace_bytes(B, Hq, Hkv, max_seq_len);
  return FP8Q_OK;
}

int fp8q_attention_decode(const void *q_e4m3, int64_t ldq, const void *k_cache,
                          const void *v_cache, int64_t num_slots, const float *scale3,
                          const int32_t *block_table, int64_t max_blocks,
                          const int32_t *seq_lens, int64_t B, int64_t Hq, int64_t Hkv, int64_t D,
                          int64_t block_size, int64_t max_seq_len, float sm_scale,
                          void *out_bf16, int64_t ldo, void *workspace, int64_t workspace_bytes,
                          cudaStream_t stream) {
  int rc = attn_shape_status(B, Hq, Hkv, D, block_size, max_seq_len);
  if (rc != FP8Q_OK) return rc;
  // slots are int32 in the kernel
  if (num_slots < 0 || num_slots > INT32_MAX || max_blocks < 0 ||
      max_blocks * block_size < max_seq_len || ldq < Hq * D || ldo < Hq * D)
    return FP8Q_ERR_SHAPE;
  if (B == 0) return FP8Q_OK;
  if (!q_e4m3 || !k_cache || !v_cache || !scale3 || !block_table || !seq_lens || !out_bf16 ||
      !workspace)
    return FP8Q_ERR_NULL;
  if (!aligned16(q_e4m3) || ldq % 16 || !aligned16(k_cache) || !aligned16(v_cache) ||
      !aligned16(workspace) || (reinterpret_cast<uintptr_t>(scale3) & 3u) ||
      (reinterpret_cast<uintptr_t>(block_table) & 3u) ||
      (reinterpret_cast<uintptr_t>(seq_lens) & 3u) || (reinterpret_cast<uintptr_t>(out_bf16) & 1u))
    return FP8Q_ERR_ALIGN;
  if (workspace_bytes < attn_workspace_bytes(B, Hq, Hkv, max_seq_len)) return FP8Q_ERR_SHAPE;
  DeviceState *st = nullptr;
  if ((rc = device_state(&st)) != FP8Q_OK) return rc;
  fp8q::AttnArgs a;
  a.q = static_cast<const uint8_t *>(q_e4m3);
  a.ldq = ldq;
  a.k_cache = static_cast<const uint8_t *>(k_cache);
  a.v_cache = static_cast<const uint8_t *>(v_cache);
  a.num_slots = num_slots;
  a.scale3 = scale3;
  a.block_table = block_table;
  a.max_blocks = max_blocks;
  a.seq_lens = seq_lens;
  a.Hq = static_cast<int>(Hq);
  a.Hkv = static_cast<int>(Hkv);
  a.block_size = static_cast<int>(block_size);
  a.max_seq_len = static_cast<int>(max_seq_len);
  a.chunk = attn_chunk(B, Hkv, max_seq_len);
  a.nsplit = max_seq_len > 0 ? static_cast<int>((max_seq_len + a.chunk - 1) / a.chunk) : 1;
  a.sm_scale = sm_scale;
  a.ws = static_cast<float *>(workspace);
  a.out = static_cast<uint16_t *>(out_bf16);
  a.ldo = ldo;
  const dim3 gs(static_cast<unsigned>(a.nsplit), static_cast<unsigned>(Hkv),
                static_cast<unsigned>(B));
  const dim3 gc(static_cast<unsigned>(Hkv), static_cast<unsigned>(B));
  const int64_t G = Hq / Hkv;
  if (max_seq_len > 0) {
    if (G == 1) fp8q::k_attn_decode_split<1><<<gs, fp8q::kAttnThreads, fp8q::kAttnSmem, stream>>>(a);
    else if (G == 2) fp8q::k_attn_decode_split<2><<<gs, fp8q::kAttnThreads, fp8q::kAttnSmem, stream>>>(a);
    else if (G == 4) fp8q::k_attn_decode_split<4><<<gs, fp8q::kAttnThreads, fp8q::kAttnSmem, stream>>>(a);
    else fp8q::k_attn_decode_split<8><<<gs, fp8q::kAttnThreads, fp8q::kAttnSmem, stream>>>(a);
    if ((rc = launch_status()) != FP8Q_OK) return rc;
  }
  if (G == 1) fp8q::k_attn_decode_combine<1><<<gc, fp8q::kAttnThreads, 0, stream>>>(a);
  else if (G == 2) fp8q::k_attn_decode_combine<2><<<gc, fp8q::kAttnThreads, 0, stream>>>(a);
  else if (G == 4) fp8q::k_attn_decode_combine<4><<<gc, fp8q::kAttnThreads, 0, stream>>>(a);
  else fp8q::k_attn_decode_combine<8><<<gc, fp8q::kAttnThreads, 0, stream>>>(a);
  return launch_status();
}

int fp8q_gemm_w8a8_rowwise(const void *aq, int64_t lda, const float *sa, const void *wq,
                           int64_t ldw, const float *sw, int64_t M, int64_t N, int64_t K,
                           void *out_bf16, int64_t ldo, cudaStream_t stream) {
  if (M < 0 || N <= 0 || K <= 0 || N % 128 || K % 128) return FP8Q_ERR_SHAPE;
  if (M > INT32_MAX - 256 || N > (1 << 30) || K > (1 << 30)) return FP8Q_ERR_SHAPE;
  if (lda < K || ldw < K || ldo < N) return FP8Q_ERR_SHAPE;
  if (M == 0) return FP8Q_OK;
  if (!aq || !sa || !wq || !sw || !out_bf16) return FP8Q_ERR_NULL;
  if (!aligned16(aq) || !aligned16(wq) || !aligned16(out_bf16) ||
      (reinterpret_cast<uintptr_t>(sa) & 3u) || (reinterpret_cast<uintptr_t>(sw) & 3u) ||
      lda % 16 || ldw % 16 || ldo % 8)
    return FP8Q_ERR_ALIGN;
  DeviceState *st = nullptr;
  int rc = device_state(&st);
  if (rc != FP8Q_OK) return rc;
  if ((rc = get_encoder()) != FP8Q_OK) return rc;
  CUtensorMap tm_a, tm_b;
  if ((rc = make_u8_map(&tm_a, aq, M, K, lda, fp8q::kBM)) != FP8Q_OK) return rc;
  if ((rc = make_u8_map(&tm_b, wq, N, K, ldw, fp8q::kBN)) != FP8Q_OK) return rc;
  fp8q::RowwiseArgs a;
  a.sa = sa;
  a.sw = sw;
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(N);
  a.K = static_cast<int>(K);
  a.out = static_cast<uint16_t *>(out_bf16);
  a.ldo = ldo;
  a.num_n = static_cast<int>((N + fp8q::kBN - 1) / fp8q::kBN);
  a.num_m = static_cast<int>((M + fp8q::kBM - 1) / fp8q::kBM);
  a.group_m = raster_group_m(M, K);
  const int64_t tiles = static_cast<int64_t>(a.num_m) * a.num_n;
  const int grid = static_cast<int>(tiles < st->sms ? tiles : st->sms);
  fp8q::k_gemm_w8a8_rowwise<<<grid, fp8q::kGemmThreads, fp8q::kGemmSmemDense, stream>>>(tm_a,
                                                                                       tm_b, a);
  return launch_status();
}

int fp8q_gemm_w8a8_mx(const void *aq, int64_t lda, const float *sa, int64_t lds,
                      const void *wq, int64_t ldw, const void *sw_e8m0, int64_t G, int64_t M,
                      int64_t N_g, int64_t K_g, void *out_bf16, int64_t ldo,
                      cudaStream_t stream) {
  if (G <= 0 || G > (1 << 16) || N_g <= 0 || N_g % 128 || K_g <= 0 || K_g % 128)
    return FP8Q_ERR_SHAPE;
  if (G > 1 && N_g % fp8q::kBN) return FP8Q_ERR_SHAPE;
  if (N_g > (1 << 30) / G || K_g > (1 << 30) / G || M < 0 || M > INT32_MAX - 256)
    return FP8Q_ERR_SHAPE;
  const int64_t N = G * N_g;
  if (lda < G * K_g || ldw < K_g || ldo < N || lds < M) return FP8Q_ERR_SHAPE;
  if (M == 0) return FP8Q_OK;
  if (!aq || !sa || !wq || !sw_e8m0 || !out_bf16) return FP8Q_ERR_NULL;
  if (!aligned16(aq) || !aligned16(wq) || !aligned16(out_bf16) ||
      (reinterpret_cast<uintptr_t>(sa) & 3u) || lda % 16 || ldw % 16 || ldo % 8)
    return FP8Q_ERR_ALIGN;
  DeviceState *st = nullptr;
  int rc = device_state(&st);
  if (rc != FP8Q_OK) return rc;
  if ((rc = get_encoder()) != FP8Q_OK) return rc;
  CUtensorMap tm_a, tm_b;
  if ((rc = make_u8_map(&tm_a, aq, M, G * K_g, lda, fp8q::kBM)) != FP8Q_OK) return rc;
  if ((rc = make_u8_map(&tm_b, wq, N, K_g, ldw, fp8q::kBN)) != FP8Q_OK) return rc;
  fp8q::MxArgs a;
  a.sa = sa;
  a.lds = lds;
  a.sw = static_cast<const uint8_t *>(sw_e8m0);
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(N);
  a.K = static_cast<int>(K_g);
  a.out = static_cast<uint16_t *>(out_bf16);
  a.ldo = ldo;
  a.num_n = static_cast<int>((N + fp8q::kBN - 1) / fp8q::kBN);
  a.num_m = static_cast<int>((M + fp8q::kBM - 1) / fp8q::kBM);
  a.group_m = raster_group_m(M, K_g);
  a.n_tiles_per_group = G > 1 ? static_cast<int>(N_g / fp8q::kBN) : 0;
  const int64_t tiles = static_cast<int64_t>(a.num_m) * a.num_n;
  const int grid = static_cast<int>(tiles < st->sms ? tiles : st->sms);
  fp8q::k_gemm_w8a8_mx<<<grid, fp8q::kGemmThreads, fp8q::kGemmSmemDense, stream>>>(tm_a, tm_b,
                                                                                  a);
  return launch_status();
}

int fp8q_selftest_timeout(int64_t limit_ns, cudaStream_t stream) {
  if (limit_ns <= 0 || limit_ns > 100000000) return FP8Q_ERR_ARG;  // (0, 100 ms]
  DeviceState *st = nullptr;
  const int rc = device_state(&st);
  if (rc != FP8Q_OK) return rc;
  fp8q::k_selftest_timeout<<<1, 128, 0, stream>>>(static_cast<uint64_t>(limit_ns));
  return launch_status();
}

int fp8q_check_device_error(cudaStream_t stream) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return FP8Q_ERR_LAUNCH;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, fp8q::g_device_error, sizeof v) != cudaSuccess)
    return FP8Q_ERR_LAUNCH;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(fp8q::g_device_error, &zero, sizeof zero) != cudaSuccess)
      return FP8Q_ERR_LAUNCH;
  }
  return v == 0 ? FP8Q_OK : v;
}

}  // extern "C"
