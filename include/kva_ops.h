/*
 * kva_ops.h -- per-step entry points of libkva.
 *
 * Each call runs exactly one step of the path (one kernel) on caller buffers.
 * They exist so every step can be checked on its own against the float64
 * oracle, and for callers that compose the path themselves.  Conventions
 * (device pointers, row-major, async on `stream`, host-side validation,
 * kva_status return) are those of kva.h.  `err` is an optional device int
 * that receives device status bits (KVA_DEV_*); NULL disables reporting.
 */
#ifndef KVA_OPS_H_
#define KVA_OPS_H_

#include <stdint.h>

#include "kva.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef enum kva_epilogue {
  KVA_EPI_STORE_BF16 = 0,  /* D = A B^T, in the operands' 16-bit format */
  KVA_EPI_STORE_F32 = 1,   /* D = A B^T, fp32 */
  KVA_EPI_ADD_F32 = 2,     /* D += A B^T, fp32 (the projector's residual stream) */
  KVA_EPI_SWIGLU_BF16 = 3  /* D = silu(A Bg^T) * (A Bu^T), 16-bit (SwiGLU FFN, model card table) */
} kva_epilogue;

typedef enum kva_b_mode {
  KVA_B_SINGLE = 0,   /* B[0] is [N, K] */
  KVA_B_SEGMENTS = 1, /* B[0..2] each [seg_rows, K], stacked along N (q | k | v) */
  KVA_B_PAIRED = 2    /* B[0] gate, B[1] up, each [N, K]; only with KVA_EPI_SWIGLU_BF16 */
} kva_b_mode;

/* The same with q8_0 weights ("Qwen3.8-27B-KVA" model card, projector quantization: q8_0
 * projector weights at about the quality of 16-bit ones).  Each B matrix [rows, K] is given
 * as int8 codes Bq[i] [rows, K] (row stride K) and fp16 scales Bs[i] [K / 32, rows] (the
 * scales of one 32-wide K block for all rows contiguous); its weight (r, k) is
 * Bs[i][k / 32][r] * Bq[i][r][k], rounded once to dtype for the tensor cores.
 * CTA pairs only; epilogue KVA_EPI_STORE_BF16, KVA_EPI_ADD_F32 or KVA_EPI_SWIGLU_BF16; no
 * output split.  K a multiple of 64, rows (N, or seg_rows) a multiple of 8, seg_rows a
 * multiple of 256; pointers 16-byte aligned. */
int kva_op_gemm_q8_0(int32_t dtype, const void* A, int64_t lda, const void* const* Bq,
                     const void* const* Bs, int32_t b_mode, int64_t seg_rows, void* D, int64_t ldd,
                     int32_t M, int32_t N, int32_t K, int32_t epilogue, int32_t* err, void* stream);

/* The same with q4_0 weights (the same section's q4_0 projector, about half the bytes of
 * q8_0).  Each B matrix [rows, K] is given as packed codes Bq[i], uint8 [rows, K / 2] (row
 * stride K / 2): per 32-wide K block of a row 16 bytes, byte j holding the code c (0..15)
 * of element j in its low nibble and that of element j + 16 in its high nibble; scales
 * Bs[i] as above.  Its weight (r, k) is Bs[i][k / 32][r] * (c(r, k) - 8), rounded once to
 * dtype for the tensor cores.  Same modes, sizes and errors as kva_op_gemm_q8_0. */
int kva_op_gemm_q4_0(int32_t dtype, const void* A, int64_t lda, const void* const* Bq,
                     const void* const* Bs, int32_t b_mode, int64_t seg_rows, void* D, int64_t ldd,
                     int32_t M, int32_t N, int32_t K, int32_t epilogue, int32_t* err, void* stream);

/* Test of the failure path of the pipelined kernels; the method has no counterpart to it.
 * Runs kva_op_gemm's CTA-pair kernel (epilogue KVA_EPI_STORE_BF16, A [M, K], B [N, K], D
 * [M, N], all row-major with the K or N dimension contiguous) with the MMA issuer of the
 * first work item waiting on a barrier that nothing arrives on.  That wait runs out after
 * about a millisecond; the kernel then raises its abort flag, lets every copy and MMA it
 * issued land, and returns with KVA_DEV_WAIT_TIMEOUT set in the device int *err.  D is left
 * partly written.  Other blocks may wait out their own limit (2 s) before they see the
 * abort, so the call can take a few seconds.  Same size rules as kva_op_gemm. */
int kva_test_gemm_wait_timeout(int32_t dtype, const void* A, const void* B, void* D, int32_t M,
                               int32_t N, int32_t K, int32_t* err, void* stream);

/* RMSNorm of `rows` rows of width n ("Qwen3.8-27B-KVA" model card, architecture):
 * out[r] = x[r] / sqrt(mean(x[r]^2) + eps) * g, out [rows, ldo] in out_dtype (bf16 / fp16).
 * x is [rows, ldx] in x_dtype.  n, ldx, ldo multiples of 4; pointers 16-byte aligned. */
int kva_op_rmsnorm(const void* x, int32_t x_dtype, int64_t ldx, const float* g, void* out,
                   int32_t out_dtype, int64_t ldo, int32_t rows, int32_t n, float eps,
                   void* stream);

/* D = A B^T with an epilogue on tcgen05 tensor cores (the projector's linears).
 *   dtype 16-bit format of A, B and of 16-bit outputs: KVA_BF16 or KVA_F16
 *   A     [M, K], row stride lda
 *   B     HOST array of 1..3 device pointers per b_mode, each with row stride ldb
 *   D     output [M, ldd] (bf16 or fp32 per epilogue); with n_split > 0 columns
 *         >= n_split go to D1 [M, ldd1] at column - n_split (n_split % 32 == 0)
 *   block_n 0 (choose), 128 or 256 (one CTA per tile of that width), 512 (a CTA pair on
 *           a 256 x 256 tile, the default when the B layout allows it)
 * K, lda, ldb multiples of 8; seg_rows a multiple of the tile width (256 for the pair). */
int kva_op_gemm(int32_t dtype, const void* A, int64_t lda, const void* const* B, int32_t b_mode,
                int64_t ldb, int64_t seg_rows, void* D, int64_t ldd, void* D1, int64_t ldd1,
                int64_t n_split, int32_t M, int32_t N, int32_t K, int32_t epilogue,
                int32_t block_n, int32_t* err, void* stream);

/* Block-causal multi-head attention of the projector (model card table row
 * "attention"): qkv [T, ldq] holds q | k | v, each n_heads x 128 wide;
 * out [T, ldo] gets the n_heads x 128 head outputs, both in dtype (bf16 / fp16).
 * Key j is visible to query i iff j <= i and i / window == j / window (window 0:
 * plain causal). */
int kva_op_attention(int32_t dtype, const void* qkv, int64_t ldq, void* out, int64_t ldo,
                     int32_t T, int32_t n_heads, int32_t window, void* stream);

/* Gated delta-rule scan alone, for n_seq x n_layers independent problems of T tokens:
 *   k     fp16 [n_seq*n_layers, T, n_k*d]  (unit-norm keys)
 *   v     fp16 [n_seq*n_layers, T, n_v*d]
 *   gb    fp32 [n_seq*n_layers, 2, n_v, T] (g then beta per v head)
 *   state fp32 [n_seq*n_layers, n_v, d, d] read and updated in place
 * v head h reads k head h / (n_v / n_k).  d = 64 or 128.  With d = 128 the call
 * stages per-chunk intermediates in stream-ordered scratch (cudaMallocAsync and
 * cudaFreeAsync on `stream`); KVA_ERR_NO_MEMORY if that fails. */
int kva_op_gdn_scan(const void* k, const void* v, const float* gb, float* state, int32_t n_seq,
                    int32_t n_layers, int32_t T, int32_t n_k, int32_t n_v, int32_t d,
                    void* stream);

/* Limits of kva_gdn_layer_update_noalloc's fixed scratch (about 6.5 MB per GPU). */
#define KVA_NOALLOC_MAX_T 256    /* tokens per call */
#define KVA_NOALLOC_MAX_QK 2048  /* n_k * d */
#define KVA_NOALLOC_MAX_V 6144   /* n_v * d */
#define KVA_NOALLOC_MAX_NV 64    /* n_v */

/* State update of ONE gated-DeltaNet layer of one sequence that allocates nothing.
 *
 * For callers that may not call cudaMalloc (or create a kva_handle, which does): an
 * engine that has reserved nearly all device memory for its own cache pool and
 * routes every allocation through its own allocator, or a plugin whose host program
 * owns device memory.  The method described by the model card has no counterpart to
 * this entry point; it exists only so such callers can run the layer update.
 *
 * It runs the same kernels as kva_update_states for that layer (conv + SiLU,
 * L2 norms, gates, chunked scan, tail shift), keeping the intermediates in a
 * fixed array compiled into the library (every GPU that loads the library holds it
 * until the process exits).  The caller still passes every input and output:
 *   mixer_in   bf16 [T, mixer_ld]: this layer's columns [q | k | v | a | b] from column 0
 *   conv_w     fp32 [C, 4], A_log / dt_bias fp32 [n_v]
 *   state      fp32 [n_v, d, d], conv_state bf16 [3, C]: read and updated in place
 * mixer_in and conv_state are always bf16 (this call has no handle that would name
 * another format).  Sizes beyond the KVA_NOALLOC_* limits return KVA_ERR_TOO_LARGE
 * before any launch.  The first call on a device looks up the device addresses of the
 * array and of a status word beside it (once per device, with that device current);
 * make that first call before any stream capture.  The addresses are kept for the life
 * of the device's primary context: do not use this entry point across a
 * cudaDeviceReset.  All calls share the one array: calls whose work overlaps on the
 * GPU (different streams, or different host threads) race on it and must be
 * serialised by the caller.  A pipeline wait that gave up inside the scan sets
 * KVA_DEV_WAIT_TIMEOUT in the status word (read it with
 * kva_gdn_layer_update_noalloc_status).  Returns kva_status. */
int kva_gdn_layer_update_noalloc(const void* mixer_in, int64_t mixer_ld, int32_t T, int32_t n_k,
                                 int32_t n_v, int32_t d, const float* conv_w, const float* A_log,
                                 const float* dt_bias, float* state, void* conv_state, float eps,
                                 void* stream);

/* Device status bits (KVA_DEV_*) that kva_gdn_layer_update_noalloc calls on the current
 * device have set since the last read.  Synchronises `stream`, stores the bits in *status
 * (0 = clean), clears them, and returns KVA_ERR_DEVICE when bits were set.  Allocates
 * nothing. */
int kva_gdn_layer_update_noalloc_status(void* stream, int32_t* status);

#ifdef __cplusplus
}
#endif
#endif /* KVA_OPS_H_ */
