/*
 * fp8q.h -- C ABI of libfp8q.so, the blockwise FP8 (E4M3) W8A8 linear layer on B200 (sm_100a).
 *
 * Four operations make up the hot path of an FP8 linear layer whose bf16 weights change every
 * step ("FP8-RL: A Practical and Stable Low-Precision Stack for LLM Reinforcement Learning",
 * abstract, item (i): W8A8 linear layers with blockwise FP8 quantization, weights requantized
 * after every policy update):
 *
 *   fp8q_quant_weight_block       bf16 W -> E4M3 codes + one scale per 128x128 block
 *   fp8q_rmsnorm_quant_token      bf16 X -> [RMSNorm] -> E4M3 codes + one scale per 1x128 group
 *   fp8q_gemm_w8a8_block          codes x codes -> bf16, per-K-block fp32 promotion
 *   fp8q_grouped_gemm_w8a8_block  the same GEMM per expert over row groups (MoE)
 *
 * Numerics (shared by all entry points):
 *   - E4M3 is the OCP FP8 E4M3 format (bias 7, max 448, no infinities, 0x7F/0xFF NaN).
 *   - A block scale is s = amax / 448 in fp32 (IEEE division), or 1 for an all-zero block; the
 *     codes are q = RNE-saturating-E4M3(x / s), x / s an IEEE fp32 division.  The sign of zero
 *     is kept (a negative value that rounds to zero gives 0x80).
 *   - E8M0 scales (FP8Q_SCALE_E8M0): one byte b, value 2^(b - 127); the quantizer picks the
 *     smallest power of two >= fp32(amax / 448), exponent clamped to [-127, 127], so every
 *     scale it writes is exactly representable ("DeepSeek V4 performance: FP8 WO_A output
 *     projection (vLLM PR 54894 analysis)", section 1: unsigned exponent, bias 127, lossless
 *     only for exact powers of two).
 *   - Outputs of the two quantizers are bit-exact against the CPU oracle; GEMM outputs satisfy
 *     |out - ref| <= 8e-3 * sum_k |dec(a) sa dec(w) sw| + 1 bf16 ulp of |ref|.
 *
 * Conventions:
 *   - Every pointer argument is a DEVICE pointer on the current CUDA device, except where a
 *     comment says otherwise.  The caller owns all buffers; the library never allocates device
 *     memory at call time (its one buffer of its own is the fixed 24 MiB split-K scratch of
 *     fp8q_gemm_w8a8_block_splitk_noalloc, a __device__ array reserved on each device when the
 *     library's module loads there) and never synchronizes, except fp8q_check_device_error.  Work is enqueued on
 *     `stream` (0 = legacy default stream).
 *   - Leading dimensions are in ELEMENTS of the buffer's type.  Matrices are row-major.
 *   - Shapes: K and N must be multiples of 128 ("... vLLM PR 54894 analysis", section 2: the
 *     FP8 path requires out % 128 == 0 and in % 128 == 0).  Unlike the page, which falls back
 *     to bf16, this library returns FP8Q_ERR_SHAPE.  M may be any value >= 0; M == 0 is a
 *     successful no-op.
 *   - Activation scales sa are fp32 in K-block-major layout: the scale of row m, K-block kb is
 *     sa[kb * lds + m], lds >= M, lds % 4 == 0.  Weight scales sw are a row-major
 *     [N/128][K/128] grid ("... vLLM PR 54894 analysis", section 2: scale viewed as
 *     [groups, out/128, in/128]); the grouped GEMM takes [E][N/128][K/128].
 *   - Alignment: every base pointer 16-byte aligned; leading dimensions such that each row
 *     starts 16-byte aligned (bf16: ld % 8 == 0; u8: ld % 16 == 0; fp32: ld % 4 == 0).
 *     Otherwise FP8Q_ERR_ALIGN.
 *   - The current device must be sm_100 (B200); otherwise FP8Q_ERR_ARCH.
 *   - Return value: an fp8q_status.  Only argument and launch errors are returned; a kernel
 *     that gives up on a bounded internal wait records FP8Q_ERR_TIMEOUT in a device-side
 *     error word, read (and cleared) by fp8q_check_device_error.
 *   - Thread safety: the entry points keep no host state apart from per-device caches filled
 *     on first use; concurrent calls on different streams are safe.
 */
#ifndef FP8Q_H
#define FP8Q_H

#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FP8Q_OK = 0,
  FP8Q_ERR_NULL = 1,    /* a required pointer is NULL */
  FP8Q_ERR_SHAPE = 2,   /* K or N not a multiple of 128, negative size, ld too small, K too large */
  FP8Q_ERR_ALIGN = 3,   /* a pointer or leading dimension breaks the 16-byte rule */
  FP8Q_ERR_ARCH = 4,    /* current device is not sm_100, or no device */
  FP8Q_ERR_LAUNCH = 5,  /* a CUDA runtime call or kernel launch failed */
  FP8Q_ERR_TIMEOUT = 6, /* (device error word) a kernel gave up on a bounded wait */
  FP8Q_ERR_ARG = 7,     /* an enum argument is out of range */
  FP8Q_ERR_TOO_LARGE = 8, /* the problem does not fit the library's static split-K scratch */
  FP8Q_ERR_RANGE = 9,     /* (device error word) a position, cache slot or scale out of range */
  FP8Q_ERR_NOT_POW2 = 10  /* (device error word) an MX-GEMM activation scale is not 2^e */
} fp8q_status;

typedef enum {
  FP8Q_SCALE_F32 = 0,   /* fp32 scales */
  FP8Q_SCALE_E8M0 = 1   /* one unsigned-exponent byte per scale, value 2^(b - 127) */
} fp8q_scale_fmt;

/* Requantize a bf16 weight into 128x128-block FP8 (a1 with fp32 scales, a2 with E8M0 scales).
 *   w_bf16   [N][ldw] bf16, read                        (N, K multiples of 128; ldw >= K)
 *   wq_e4m3  [N][ldq] uint8 E4M3 codes, written         (ldq >= K)
 *   sw       [N/128][K/128] fp32 (sw_fmt = FP8Q_SCALE_F32) or uint8 (FP8Q_SCALE_E8M0), written
 * Source: FP8-RL abstract (i) (per-step requantization of changed policy weights);
 * vLLM PR 54894 analysis, sections 1 and 2 (E8M0 bytes, the [out/128, in/128] scale grid). */
int fp8q_quant_weight_block(const void *w_bf16, int64_t N, int64_t K, int64_t ldw,
                            void *wq_e4m3, int64_t ldq, void *sw, int sw_fmt,
                            cudaStream_t stream);

/* One matrix of a batched weight requantization (fp8q_quant_weight_block_batched): the arguments
 * of fp8q_quant_weight_block for that matrix, plus the index of its first 128x128 block in the
 * batch's block numbering (the sum of (N/128)(K/128) over the matrices before it). */
typedef struct {
  const void *w;          /* bf16 [N][ldw], read */
  void *q;                /* uint8 [N][ldq], written */
  void *s;                /* [N/128][K/128] fp32 or E8M0 scales, written */
  int64_t N, K, ldw, ldq; /* as fp8q_quant_weight_block */
  int64_t block_offset;   /* first block of this matrix in the batch numbering */
} fp8q_weight_desc;

/* Batched a1 / a2: every matrix of `descs` (DEVICE memory, count <= 2048, block_offset ascending,
 * total_blocks = the sum of all matrices' blocks) requantized in one launch, with the arithmetic
 * and outputs of fp8q_quant_weight_block.  The descriptors are read on the device: one that
 * breaks that call's shape or alignment rules (or block numbering that does not match the
 * matrices) records FP8Q_ERR_SHAPE in the device error word and its blocks are skipped.
 * Source: FP8-RL abstract, item (i) (the policy's weights change every step, so all of them are
 * requantized every step). */
int fp8q_quant_weight_block_batched(const fp8q_weight_desc *descs, int64_t count,
                                    int64_t total_blocks, int sw_fmt, cudaStream_t stream);


/* Per-token 1x128 activation quantization, optionally fused with RMSNorm (a3 / a4).
 *   x_bf16      [M][ldx] bf16, read
 *   gamma_bf16  [K] bf16 RMSNorm weight, or NULL for plain token quant (no normalisation)
 *   eps         RMSNorm epsilon (fp32; ignored when gamma_bf16 is NULL)
 *   xq_e4m3     [M][ldq] uint8 codes, written
 *   sa          fp32 scales, sa[kb * lds + m], written for m < M only
 * With gamma: r = fp32(1 / sqrt(S / K + eps)) where S is the fp64 sum of x^2 taken in ascending
 * k within each 128-block and then over blocks in ascending order; y = bf16_RNE((x * r) * gamma)
 * with two fp32 roundings; the 1x128 quant then runs on y, which is never written to memory.
 * K <= 16384.  Source: SGLang PR 21403 analysis, section 1 (RMSNorm with weight and epsilon
 * fused with FP8 quant so the normalised tensor makes no round trip through memory); vLLM PR
 * 54894 analysis, section 3 (quant_group_size = 128). */
int fp8q_rmsnorm_quant_token(const void *x_bf16, const void *gamma_bf16, float eps, int64_t M,
                             int64_t K, int64_t ldx, void *xq_e4m3, int64_t ldq, float *sa,
                             int64_t lds, cudaStream_t stream);

/* fp8q_rmsnorm_quant_token with a choice of activation scale (sa_fmt):
 *   FP8Q_SCALE_F32   s = fp32(amax / 448) (1 for an all-zero group): the call above;
 *   FP8Q_SCALE_E8M0  s = 2^e, e the smallest integer with 2^e >= fp32(amax / 448), clamped to
 *                    [-127, 127] (1 for an all-zero group), written to sa as its fp32 value; the
 *                    codes are RNEsat(y / 2^e), a division that is exact.  These scales feed
 *                    fp8q_gemm_w8a8_mx (hardware block scaling) as well as the other GEMMs.
 * Other arguments, rules and errors as fp8q_rmsnorm_quant_token; another sa_fmt is FP8Q_ERR_ARG.
 * Source: vLLM PR 54894 analysis, sections 1 and 3 (E8M0 scales with bias 127; the group-128
 * quant feeds a GEMM that takes MX scales on both operands); SGLang PR 21403 analysis, section 1. */
int fp8q_rmsnorm_quant_token_fmt(const void *x_bf16, const void *gamma_bf16, float eps,
                                 int64_t M, int64_t K, int64_t ldx, void *xq_e4m3, int64_t ldq,
                                 float *sa, int64_t lds, int sa_fmt, cudaStream_t stream);

/* Block-scaled W8A8 GEMM (a5): out[m, n] = bf16( sum_kb sa[m, kb] * sw[n/128, kb] * P_kb[m, n] )
 * where P_kb is the fp32 tensor-core dot product of the E4M3 codes over K-block kb and each
 * K-block partial is promoted (scaled and accumulated) in fp32.  K <= 32768.
 *   aq   [M][lda] uint8 activation codes     sa  fp32, sa[kb * lds + m]
 *   wq   [N][ldw] uint8 weight codes         sw  [N/128][K/128], fp32 or E8M0 per sw_fmt
 *   out  [M][ldo] bf16, written (rows < M, columns < N)
 * Source: SGLang PR 21403 analysis, section 3 (the GEMM consumes the pre-quantized (codes,
 * scale) pair and writes bf16); FP8-RL abstract (i). */
int fp8q_gemm_w8a8_block(const void *aq, int64_t lda, const float *sa, int64_t lds,
                         const void *wq, int64_t ldw, const void *sw, int sw_fmt, int64_t M,
                         int64_t N, int64_t K, void *out_bf16, int64_t ldo, cudaStream_t stream);

/* The block-scaled GEMM above with its K dimension split over several CTAs per output tile, for
 * shapes with too few 128 x 256 output tiles to occupy every SM (decode: M <= 128).  Split j of
 * S takes the K-blocks [j * KB / S, (j + 1) * KB / S) (KB = K / 128), promotes them exactly as
 * fp8q_gemm_w8a8_block does and writes its fp32 partial to `workspace`; a second kernel on the
 * same stream then adds the S partials of each tile in the order j = 0, 1, ..., S - 1
 * (deterministic) and writes bf16.  The result differs from fp8q_gemm_w8a8_block only in the
 * fp32 summation order of the K-block terms and meets the same error bound.
 *   splits           S in [1, K / 128]; 0 = chosen by the library (1 when the tiles already fill
 *                    the SMs)
 *   workspace        DEVICE memory of at least fp8q_gemm_splitk_workspace_bytes(M, N, K, splits)
 *                    bytes, 16-byte aligned, owned by the caller; unused (may be NULL) when the
 *                    resolved S is 1.  Its contents need no initialisation.  Two calls that
 *                    share a workspace must be ordered (same stream, or synchronized):
 *                    concurrent calls on one workspace race.
 * Other arguments, layouts and errors as fp8q_gemm_w8a8_block; splits out of range gives
 * FP8Q_ERR_ARG, a workspace smaller than required FP8Q_ERR_SHAPE.  Source: the same passages as
 * fp8q_gemm_w8a8_block (the split only reorders the fp32 promotion sum over K-blocks). */
int fp8q_gemm_w8a8_block_splitk(const void *aq, int64_t lda, const float *sa, int64_t lds,
                                const void *wq, int64_t ldw, const void *sw, int sw_fmt,
                                int64_t M, int64_t N, int64_t K, void *out_bf16, int64_t ldo,
                                int splits, void *workspace, int64_t workspace_bytes,
                                cudaStream_t stream);

/* Workspace size in bytes for fp8q_gemm_w8a8_block_splitk with these sizes and `splits` (0 =
 * the library's choice on the current device), written to *bytes (a HOST pointer); 0 when the
 * resolved split count is 1. */
int fp8q_gemm_splitk_workspace_bytes(int64_t M, int64_t N, int64_t K, int splits,
                                     int64_t *bytes);

/* fp8q_gemm_w8a8_block_splitk without a caller workspace: the split-K partials live in a fixed
 * 24 MiB buffer that the library declares in its own device memory (reserved
 * when the library's device code is loaded), so the call allocates nothing.  It serves callers
 * that cannot allocate device memory at call time: an inference engine that hands all free HBM
 * to its KV-cache pool at start-up and has no room left for per-call workspaces, or a caller that
 * must not call cudaMalloc/cudaFree on its hot path because they can synchronize the device.
 * The pages define no such variant; it computes exactly what fp8q_gemm_w8a8_block_splitk does
 * (same kernel, same split order, bit-identical results for the same splits).
 *   Limit: tiles * S <= 192 (tiles = ceil(M / 128) * ceil(N / 256), S the resolved split
 *   count); beyond it FP8Q_ERR_TOO_LARGE.  Decode (M <= 128, N <= 12288) with
 *   S <= 4 fits.  A resolved S of 1 runs fp8q_gemm_w8a8_block and touches no scratch.
 *   Nothing in the buffer needs to start at zero: each call writes every partial it reads.
 *   The first call on each device looks the buffer's address up (cudaGetSymbolAddress, with
 *   that device current); make that first call before any stream capture.  The address and
 *   the kernels' function attributes are cached per device for the life of the process and
 *   are not refreshed after cudaDeviceReset: do not call this entry point on a device after
 *   resetting it.
 *   Each device has one such buffer (per process), shared by every caller: two calls on one
 *   device that are not ordered with respect to each other (unsynchronized streams, host
 *   threads) race on it and give wrong results.  Order them.
 * Other arguments and errors as fp8q_gemm_w8a8_block_splitk. */
int fp8q_gemm_w8a8_block_splitk_noalloc(const void *aq, int64_t lda, const float *sa,
                                        int64_t lds, const void *wq, int64_t ldw, const void *sw,
                                        int sw_fmt, int64_t M, int64_t N, int64_t K,
                                        void *out_bf16, int64_t ldo, int splits,
                                        cudaStream_t stream);

/* Block-diagonal W8A8 GEMM over G head groups: the batched projection that follows
 * fp8q_inverse_rope_quant.  Group g multiplies its own K-slice of each token's row by its own
 * weight and writes its own column range:
 *   out[m][g N_g + n] = sum over kb of fp32(sa[(g KB_g + kb) lds + m] * sw[g][n/128][kb])
 *                       * (fp32 dot product of the 128 codes of A[m][g K_g + 128 kb ...] and
 *                          W[g][n][128 kb ...]),  KB_g = K_g / 128
 *   aq      [M][lda] uint8 codes, lda >= G K_g (the groups' K-slices side by side)
 *   sa      fp32 activation scales, K-block-major over all G K_g columns
 *   wq      [G][N_g][ldw] uint8 codes (group stride N_g ldw), i.e. G N_g rows of K_g codes
 *   sw      [G][N_g/128][K_g/128] fp32 or E8M0
 *   out     [M][ldo] bf16, ldo >= G N_g: the [M, G, N_g] result flattened over (G, N_g)
 * N_g % 256 == 0 (a 128 x 256 output tile never straddles two groups), K_g % 128 == 0; the other
 * rules, the arithmetic and the tolerance are those of fp8q_gemm_w8a8_block.  Source: vLLM PR
 * 54894 analysis, sections 2-3 (weights viewed as [groups, out_per_group, in_features] with
 * scales [groups, out/128, in/128]; a batched FP8 GEMM over the groups, flattened over
 * (groups, out) afterwards). */
int fp8q_gemm_w8a8_block_diag(const void *aq, int64_t lda, const float *sa, int64_t lds,
                              const void *wq, int64_t ldw, const void *sw, int sw_fmt,
                              int64_t G, int64_t M, int64_t N_g, int64_t K_g, void *out_bf16,
                              int64_t ldo, cudaStream_t stream);

/* W8A8 GEMM with hardware block scaling for power-of-two (E8M0) scales, dense (G = 1) or
 * block-diagonal over G head groups (as fp8q_gemm_w8a8_block_diag):
 *   out[m][g N_g + n] = sum over kb of sa[(g KB_g + kb) lds + m] * 2^(sw[g][n/128][kb] - 127)
 *                       * (dot product of the 128 codes of K-block kb)
 * The tensor core applies both scales (tcgen05.mma kind::mxf8f6f4.block_scale, the 128-group
 * scale given to each of its four 32-element sub-blocks) and accumulates all of K in fp32; no
 * software promotion.  The sum is the one fp8q_gemm_w8a8_block computes, within the same
 * tolerance.
 *   aq       [M][lda] uint8 codes, lda >= G K_g
 *   sa       fp32 activation scales, K-block-major sa[kb * lds + m]; every value must be a power
 *            of two in [2^-127, 2^127] (what FP8Q_SCALE_E8M0 quantizers write); any other value
 *            records FP8Q_ERR_NOT_POW2 in the device error word and the outputs are invalid
 *   wq       [G][N_g][ldw] uint8 codes; sw_e8m0 [G][N_g/128][K_g/128] E8M0 bytes
 *   out      [M][ldo] bf16, ldo >= G N_g
 * N_g % 128 == 0 (% 256 when G > 1), K_g % 128 == 0.  Source: vLLM PR 54894 analysis, sections 1-3
 * (E8M0 scales; batched_gemm_a8w8_mxscale(o_fp8, weight, o_scale, e8m0_scale) consumes the
 * inverse-RoPE quant's output with MX scales on both operands). */
int fp8q_gemm_w8a8_mx(const void *aq, int64_t lda, const float *sa, int64_t lds,
                      const void *wq, int64_t ldw, const void *sw_e8m0, int64_t G, int64_t M,
                      int64_t N_g, int64_t K_g, void *out_bf16, int64_t ldo,
                      cudaStream_t stream);

/* FP8 KV cache, step 1: per-step recalibration of the per-tensor QKV scales.
 *   qkv_bf16  [T][ld] bf16, read: each token's row holds Hq heads of Q, then Hkv heads of K, then
 *             Hkv heads of V, D values per head (D % 8 == 0)
 *   amax3     [3] fp32, DEVICE memory, written: max |x| over all of Q, of K, of V
 *   scale3    [3] fp32, DEVICE memory, written: s = amax / 448 (IEEE fp32), 1 for an all-zero part
 * Three stream operations: a memset of amax3, the reduction (one atomicMax per CTA and part on
 * the fp32 bit pattern: the result does not depend on the order), and a one-warp finalize.  T may
 * be 0 (scales 1).  Bit-exact against the CPU oracle.  Source: FP8-RL abstract, item (ii) (FP8
 * KV cache with per-step QKV scale recalibration). */
int fp8q_qkv_scales(const void *qkv_bf16, int64_t T, int64_t ld, int64_t Hq, int64_t Hkv,
                    int64_t D, float *amax3, float *scale3, cudaStream_t stream);

/* FP8 KV cache, step 2: quantize Q and write K and V into the cache.
 *   qkv_bf16  as fp8q_qkv_scales (D % 16 == 0)
 *   slots     [T] int64, DEVICE memory: the cache row of each token; a negative slot means the
 *             token is not cached (padding); a slot >= num_slots records FP8Q_ERR_RANGE and the
 *             token's cache rows are not written
 *   scale3    [3] fp32, DEVICE memory: the per-tensor scales (from fp8q_qkv_scales, or the
 *             caller's); a scale that is not positive and finite records FP8Q_ERR_RANGE and that
 *             part is not written
 *   q_e4m3    [T][ldq] uint8 codes of Q, written; may be NULL (Q not quantized)
 *   k_cache, v_cache
 *             [num_slots][Hkv * D] uint8 each (a paged cache [blocks][block_size][Hkv][D] seen
 *             as slot-major rows), rows slots[t] written, all others untouched
 * Codes are RNE-saturating E4M3 of x / s (one IEEE fp32 division), bit-exact against the CPU
 * oracle.  Source: FP8-RL abstract, item (ii). */
int fp8q_kv_cache_write(const void *qkv_bf16, int64_t T, int64_t ld, int64_t Hq, int64_t Hkv,
                        int64_t D, const int64_t *slots, int64_t num_slots, const float *scale3,
                        void *q_e4m3, int64_t ldq, void *k_cache, void *v_cache,
                        cudaStream_t stream);

/* FP8 KV cache, step 3: decode attention that reads the cache (one query token per sequence).
 * For sequence b and query head h (kv head g = h / (Hq / Hkv), grouped-query attention), over the
 * sequence's L = seq_lens[b] positions j, cached at slot block_table[b][j / block_size] *
 * block_size + j % block_size:
 *   z_j = sm_scale * s_q * s_k * sum_d dec(q[b][h D + d]) * dec(k_cache[slot_j][g D + d])
 *   out[b][h D + d] = bf16( s_v * sum_j softmax(z)_j * dec(v_cache[slot_j][g D + d]) )
 * with (s_q, s_k, s_v) = scale3 (as fp8q_kv_cache_write uses them); L = 0 gives 0.  The dot
 * products run on the tensor cores (fp16 operands, exact for E4M3 codes, fp32 accumulation), the
 * softmax in fp32 (exp2), the weights enter the value sums as fp16; results within
 * |out - ref| <= ulp_bf16(|ref|)/2 + absref * (2^-11 + 2 (D + 2) 2^-24 zabs + (L + 16) 2^-23)
 * of the fp64 reference (absref = s_v sum_j p_j |dec(v_j)|, zabs = the largest
 * |sm_scale s_q s_k| sum_d |dec(q) dec(k_j)|).  Two launches: the positions of each (sequence,
 * kv head) are split into chunks whose partial softmax states go to `workspace`, then combined
 * in chunk order.
 *   q_e4m3       [B][ldq] uint8 codes (Hq heads of D; from fp8q_kv_cache_write), 16-byte aligned,
 *                ldq % 16 == 0
 *   k_cache, v_cache
 *                [num_slots][Hkv * D] uint8, 16-byte aligned (the paged cache of
 *                fp8q_kv_cache_write)
 *   scale3       [3] fp32, DEVICE memory
 *   block_table  [B][max_blocks] int32, DEVICE memory: block ids; an id outside [0, num_slots /
 *                block_size) records FP8Q_ERR_RANGE and its positions are skipped
 *   seq_lens     [B] int32, DEVICE memory; a length outside [0, max_seq_len] records
 *                FP8Q_ERR_RANGE and is clamped
 *   max_seq_len  a HOST bound on seq_lens (it sizes the split), <= max_blocks * block_size
 *   out_bf16     [B][ldo] bf16, written (Hq * D values per row)
 *   workspace    DEVICE memory of fp8q_attention_decode_workspace_bytes(...) bytes, 16-byte
 *                aligned, caller-owned, reusable in stream order
 * D == 128 and Hq / Hkv in {1, 2, 4, 8} (else FP8Q_ERR_SHAPE).  Source: FP8-RL abstract, item (ii)
 * (the FP8 KV cache serves the attention of the rollout's decode steps; the page gives no
 * attention arithmetic: plain scaled dot-product attention on the dequantized tensors). */
int fp8q_attention_decode(const void *q_e4m3, int64_t ldq, const void *k_cache,
                          const void *v_cache, int64_t num_slots, const float *scale3,
                          const int32_t *block_table, int64_t max_blocks,
                          const int32_t *seq_lens, int64_t B, int64_t Hq, int64_t Hkv, int64_t D,
                          int64_t block_size, int64_t max_seq_len, float sm_scale,
                          void *out_bf16, int64_t ldo, void *workspace, int64_t workspace_bytes,
                          cudaStream_t stream);

/* Workspace bytes of fp8q_attention_decode for these sizes, written to *bytes (HOST pointer);
 * depends on the sizes only. */
int fp8q_attention_decode_workspace_bytes(int64_t B, int64_t Hq, int64_t Hkv, int64_t D,
                                          int64_t max_seq_len, int64_t *bytes);

/* Grouped W8A8 GEMM for MoE experts (a6): for each expert e the rows
 * [group_offsets[e], group_offsets[e+1]) of aq/sa/out are multiplied by expert e's weight.
 *   wq             [E][N][ldw] uint8 codes (expert stride N * ldw)
 *   sw             [E][N/128][K/128] fp32 or E8M0
 *   group_offsets  [E + 1] int32, DEVICE memory, nondecreasing, [0] = 0, [E] = M.  The kernel
 *                  clamps each offset into [previous offset, M]; rows not covered by any
 *                  expert are left unwritten.
 * E <= 1024.  Source: vLLM PR 54894 analysis, section 3 (batched FP8 GEMM over [groups, out,
 * in] weights with per-group block scales); FP8-RL abstract (dense and MoE models). */
int fp8q_grouped_gemm_w8a8_block(const void *aq, int64_t lda, const float *sa, int64_t lds,
                                 const void *wq, int64_t ldw, const void *sw, int sw_fmt,
                                 const int32_t *group_offsets, int64_t E, int64_t M, int64_t N,
                                 int64_t K, void *out_bf16, int64_t ldo, cudaStream_t stream);

/* SiLU-and-mul + 1x128 quant: the front end of an MoE down projection, fed by the gate/up GEMM.
 *   h_bf16   [R][ldh] bf16 = [gate | up]: gate in columns [0, I), up in [I, 2I), read
 *   q_e4m3   [R][ldq] uint8 codes of y = bf16_RNE( fp32(silu(gate) * up) ), written
 *   sa       fp32 scales, sa[kb * lds + r] (1x128 groups of y), written for r < R only
 * silu(g) = g / (1 + e^-g) in fp32 with an IEEE division; e^x in fp32 by Cody-Waite range
 * reduction and a degree-7 Taylor polynomial with every step an IEEE fp32 rounding (reproducible
 * bit for bit; within 2 ulp of the true e^x).  Scales (per sa_fmt, FP8Q_SCALE_F32 or
 * FP8Q_SCALE_E8M0) and codes as fp8q_rmsnorm_quant_token_fmt.
 * I % 128 == 0, I <= 16384, ldh >= 2 I.  Bit-exact against the CPU oracle.  Source: FP8-RL
 * abstract, item (i) (W8A8 linear layers of MoE models: the down projection's input is the
 * activated gate/up output, quantized 1x128 like every activation here). */
int fp8q_silu_mul_quant(const void *h_bf16, int64_t R, int64_t I, int64_t ldh, void *q_e4m3,
                        int64_t ldq, float *sa, int64_t lds, int sa_fmt, cudaStream_t stream);

/* Inverse RoPE + 1x128 quant: the front end of the attention output projection (wo_a), whose
 * output feeds the per-head-group GEMM fp8q_gemm_w8a8_block_diag.
 *   o_bf16     [T][H][D] bf16, heads contiguous, token stride ldo (elements), read
 *   positions  [T] int64, DEVICE memory: each token's position, read when rope_dim > 0
 *   cos_cache, sin_cache
 *              [max_pos][rope_dim / 2] fp32, DEVICE memory (16-byte aligned), read
 *   q_e4m3     [T][ldq] uint8 codes of y (below) along the flattened H*D row, written
 *   sa         fp32 scales sa[kb * lds + t], one per 128-group of y, written for t < T only
 * y: the last rope_dim dims of each head are rotated by -theta_i in pairs (a, b) = (2i, 2i + 1)
 * (interleaved = 1) or (i, i + rope_dim / 2) (interleaved = 0), with c = cos[p][i] and
 * s = sin[p][i]: y_a = bf16(fp32(x_a c) + fp32(x_b s)), y_b = bf16(fp32(x_b c) - fp32(x_a s)),
 * each product and sum one IEEE fp32 rounding; the first D - rope_dim dims pass through.
 * scale_fmt FP8Q_SCALE_F32: s = fp32(amax / 448) (1 for an all-zero group); FP8Q_SCALE_E8M0:
 * s = the smallest power of two >= fp32(amax / 448) (the MX scale of the GEMM that follows),
 * stored as its fp32 value.  Codes are RNE-saturating E4M3 of y / s.
 * D % 8 == 0, rope_dim % 8 == 0 (% 16 when interleaved == 0), rope_dim <= D, H*D % 128 == 0,
 * H*D <= 2^24.  A token whose position is outside [0, max_pos) is not written and records
 * FP8Q_ERR_RANGE in the device error word (fp8q_check_device_error).  Bit-exact against the
 * CPU oracle.  Source: vLLM PR 54894 analysis, section 3 (inverse_rope_group_quant(o [T, heads,
 * head_dim], positions, cos cache, sin cache, num_groups, quant_group_size=128) fuses the
 * inverse RoPE with the FP8 quantization so that the rotated bf16 values never reach memory). */
int fp8q_inverse_rope_quant(const void *o_bf16, int64_t ldo, const int64_t *positions,
                            const float *cos_cache, const float *sin_cache, int64_t max_pos,
                            int64_t T, int64_t H, int64_t D, int64_t rope_dim, int interleaved,
                            int scale_fmt, void *q_e4m3, int64_t ldq, float *sa, int64_t lds,
                            cudaStream_t stream);

/* Per-token (full-row) quantization, optionally fused with RMSNorm: one fp32 scale per row of K
 * (the "group size 0 = per token" mode).  Applied to a weight W [N, K] it gives the
 * per-output-channel codes and scales the per-channel GEMM below takes.
 *   x_bf16      [M][ldx] bf16, read
 *   gamma_bf16  [K] bf16 RMSNorm weight, or NULL (no normalisation); eps as fp8q_rmsnorm_quant_token
 *   q_e4m3      [M][ldq] uint8 codes, written
 *   s           [M] fp32 scales, written (4-byte aligned)
 * s = amax / 448 over the whole (normalised) row, IEEE division, 1 for an all-zero row; codes
 * q = RNEsat(y / s).  RMSNorm arithmetic as fp8q_rmsnorm_quant_token.  K % 128 == 0, K <= 16384.
 * Bit-exact against the CPU oracle.  Source: SGLang PR 21403 analysis, section 1 (RMSNorm with
 * weight and epsilon fused with FP8 quant, group_size 0 = per token) and section 2 (CHANNEL
 * weight strategy -> per-token path). */
int fp8q_quant_rowwise(const void *x_bf16, const void *gamma_bf16, float eps, int64_t M,
                       int64_t K, int64_t ldx, void *q_e4m3, int64_t ldq, float *s,
                       cudaStream_t stream);

/* Residual add + RMSNorm + quantization in one pass over each row (the fused add-RMSNorm-quant of
 * a pre-norm block; the updated residual stream is written back):
 *   x_bf16        [M][ldx] bf16, read (the sub-layer output)
 *   residual_bf16 [M][ldr] bf16, read and overwritten with h = bf16_RNE(fp32(x) + fp32(residual))
 *   gamma_bf16    [K] bf16 RMSNorm weight (required); eps as fp8q_rmsnorm_quant_token
 *   per_token     0: 1x128 groups, sa [K/128][lds] K-block-major as fp8q_rmsnorm_quant_token
 *                 (lds >= M, lds % 4 == 0, 16-byte aligned); 1: one scale per row, sa [M]
 *                 (4-byte aligned; lds unused), as fp8q_quant_rowwise
 *   sa_fmt        FP8Q_SCALE_F32, or FP8Q_SCALE_E8M0 with per_token == 0 (the power-of-two
 *                 scales of fp8q_rmsnorm_quant_token_fmt); anything else is FP8Q_ERR_ARG
 *   q_e4m3        [M][ldq] uint8 codes of RMSNorm(h), written
 * The norm and quant arithmetic are those of fp8q_rmsnorm_quant_token / fp8q_quant_rowwise, on h.
 * The x and residual row ranges must not overlap (FP8Q_ERR_ARG otherwise); ldx, ldr % 8 == 0,
 * ldq % 16 == 0, K % 128 == 0, K <= 16384; per_token other than 0 or 1 is FP8Q_ERR_ARG.
 * Bit-exact (codes, scales and the new residual) against the CPU oracle.  Source: SGLang PR 21403
 * analysis, section 1 (the fused kernel it calls is the AMD library's add_rmsnorm_quant, with
 * weight, epsilon and group_size 0 = per token; the call it prints passes no residual, so the
 * residual add is the reading above: what an unfused bf16 add writes). */
int fp8q_add_rmsnorm_quant(const void *x_bf16, int64_t ldx, void *residual_bf16, int64_t ldr,
                           const void *gamma_bf16, float eps, int64_t M, int64_t K, int per_token,
                           int sa_fmt, void *q_e4m3, int64_t ldq, float *sa, int64_t lds,
                           cudaStream_t stream);

/* Per-token x per-channel W8A8 GEMM:
 *   out[m, n] = bf16( P[m, n] * fp32(sa[m] * sw[n]) ),  P = fp32 tensor-core dot product over K
 * with no per-K-block promotion (the scales are constant along K).
 *   aq [M][lda] uint8 codes, sa [M] fp32; wq [N][ldw] uint8 codes, sw [N] fp32
 *   out [M][ldo] bf16, written (rows < M, columns < N)
 * Shapes and alignment as fp8q_gemm_w8a8_block (sa and sw 4-byte aligned).  Error bound as the
 * block-scaled GEMM: |out - ref| <= 8e-3 sum_k |dec(a) dec(w)| sa sw + 1 bf16 ulp.  Source: SGLang
 * PR 21403 analysis, section 3 (the PTPC GEMM takes the (codes, x_scale) tuple and the per-channel
 * weight scale, no bias, bf16 out). */
int fp8q_gemm_w8a8_rowwise(const void *aq, int64_t lda, const float *sa, const void *wq,
                           int64_t ldw, const float *sw, int64_t M, int64_t N, int64_t K,
                           void *out_bf16, int64_t ldo, cudaStream_t stream);

/* Self-test of the bounded-wait path: launches one small kernel that allocates TMEM, waits on a
 * barrier nothing arrives on with the limit limit_ns (0 < limit_ns <= 100 ms), gives up, records
 * FP8Q_ERR_TIMEOUT in the device error word, stops its other warps through the abort flag and
 * releases TMEM, as the GEMM kernels do on a timeout.  A following fp8q_check_device_error
 * returns FP8Q_ERR_TIMEOUT; the context stays usable.  For tests. */
int fp8q_selftest_timeout(int64_t limit_ns, cudaStream_t stream);

/* Synchronize `stream`, then read and clear the device error word of the current device.
 * Returns FP8Q_OK, FP8Q_ERR_TIMEOUT (a kernel gave up on a bounded wait since the last call;
 * its outputs are incomplete) or FP8Q_ERR_LAUNCH (the synchronize failed). */
int fp8q_check_device_error(cudaStream_t stream);

/* Static, NUL-terminated description of a status code.  Never NULL. */
const char *fp8q_status_string(int status);

/* ABI version: (major << 16) | minor. */
int fp8q_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FP8Q_H */
