/*
 * kva.h -- C ABI of the KVA (late-layer KV approximation) prefill path on B200.
 *
 * What the path computes ("Qwen3.8-27B-KVA: late-layer KV approximation" model
 * card, sections "What the hell?" and the architecture table):
 *   for one ubatch of T tokens, a projector predicts from the layer-31
 *   residual (H = 5120 per token) the input of every late layer's token mixer:
 *       RMSNorm, Linear{H -> d}, n_blocks causal transformer blocks
 *       (MHA at head dim 128, causal within the ubatch / within `attn_window`
 *       blocks, SwiGLU FFN), RMSNorm, then a linear head for each late layer
 *       (+ optional drafter heads);
 *   then the cheap state updates run on those mixer inputs:
 *       gated-DeltaNet layers: causal depthwise conv1d (kernel 4) + SiLU,
 *       L2-norm of q and k, g = -exp(A_log) * softplus(a + dt_bias),
 *       beta = sigmoid(b), and the gated delta rule
 *       S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *       carried across ubatches;
 *       full-attention layers: RMSNorm of each k head, RoPE on the first
 *       `rope_dims` dims (theta 1e7, pairs (i, i + rope_dims/2)), K/V cache write.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers unless the argument says "host".
 *     The caller owns every tensor; the library owns only the workspace it
 *     allocates in kva_init and frees in kva_free.
 *   - Matrices are row-major.  Weights are [out, in] (the `in` dim contiguous).
 *     bf16 means IEEE bfloat16 stored in 2 bytes.
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL is
 *     the legacy default stream).  They never synchronise and never allocate (the per-step
 *     test entry point kva_op_gdn_scan of kva_ops.h, which has no handle, is the one call
 *     that takes stream-ordered scratch).
 *   - Every call returns a kva_status.  Arguments are validated on the host
 *     before anything is enqueued; on an error nothing is launched.  Errors that
 *     only the device can see (page-table entry out of range, an internal wait
 *     that timed out) skip the offending write and set a device status word,
 *     read back by kva_get_device_status.
 *   - A handle serves one stream at a time.  Different handles are independent.
 */
#ifndef KVA_H_
#define KVA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KVA_MAX_LATE 64   /* late layers per handle */
#define KVA_MAX_BLOCKS 8  /* projector blocks */

typedef enum kva_status {
  KVA_OK = 0,
  KVA_ERR_INVALID_ARG = -1,   /* null pointer, negative size, inconsistent dims */
  KVA_ERR_UNSUPPORTED = -2,   /* dims outside what the kernels implement */
  KVA_ERR_TOO_LARGE = -3,     /* T > max_T, n_seq > max_seq, pos beyond the cache */
  KVA_ERR_ALIGNMENT = -4,     /* a pointer or leading dimension is not 16-byte aligned */
  KVA_ERR_CUDA = -5,          /* a CUDA runtime call or launch failed */
  KVA_ERR_NO_MEMORY = -6,     /* workspace allocation failed in kva_init */
  KVA_ERR_DEVICE = -7         /* device status word is set (kva_get_device_status) */
} kva_status;

/* device status bits (kva_get_device_status) */
#define KVA_DEV_PAGE_OOB 0x1      /* a page-table entry or page index was out of range */
#define KVA_DEV_WAIT_TIMEOUT 0x2  /* a pipeline wait inside a kernel gave up */

typedef enum kva_layer_type { KVA_LAYER_GDN = 0, KVA_LAYER_ATTN = 1 } kva_layer_type;
/* KVA_Q8_0 is a KV-cache format only: see kva_kv_cache. */
typedef enum kva_dtype { KVA_BF16 = 0, KVA_F32 = 1, KVA_F16 = 2, KVA_Q8_0 = 3 } kva_dtype;
typedef enum kva_kv_layout { KVA_KV_CONTIGUOUS = 0, KVA_KV_PAGED = 1 } kva_kv_layout;

/* Geometry.  The r3 projector of the model card is
 * {hidden 5120, d_model 3072, n_heads 24, head_dim 128, ffn 8448, n_blocks 3,
 *  attn_window 1024, n_late 32 (24 GDN + 8 attention), gdn 16/48 heads of 128,
 *  attention 4 KV heads of 256 with 64 rotary dims, n_draft_cols 4 x 5120}. */
typedef struct kva_dims {
  int32_t hidden;       /* H: residual width */
  int32_t d_model;      /* d: projector width = n_heads * head_dim */
  int32_t n_heads;      /* projector attention heads */
  int32_t head_dim;     /* projector head dim; must be 128 */
  int32_t ffn;          /* SwiGLU hidden width */
  int32_t n_blocks;     /* transformer blocks, <= KVA_MAX_BLOCKS */
  int32_t attn_window;  /* projector block-causal window in tokens; 0 = causal over the ubatch */
  int32_t n_late;       /* late layers, <= KVA_MAX_LATE */
  int32_t layer_type[KVA_MAX_LATE]; /* kva_layer_type per late layer, in layer order */
  int32_t gdn_n_k;      /* q/k heads per GDN layer */
  int32_t gdn_n_v;      /* v heads per GDN layer (multiple of gdn_n_k) */
  int32_t gdn_d_k;      /* q/k head dim (64 or 128) */
  int32_t gdn_d_v;      /* v head dim (must equal gdn_d_k) */
  int32_t conv_k;       /* conv kernel size; must be 4 */
  int32_t attn_n_kv;    /* KV heads per attention layer */
  int32_t attn_d_h;     /* KV head dim (128 or 256) */
  int32_t rope_dims;    /* rotary dims at the start of each KV head (even, <= attn_d_h) */
  double rope_theta;    /* RoPE base (1e7 for the model card's base model) */
  float norm_eps;       /* epsilon of every RMSNorm / L2 norm (1e-6) */
  int32_t n_draft_cols; /* drafter output columns after the mixer columns (0 if none) */
  int32_t max_T;        /* largest ubatch the handle accepts */
  int32_t max_seq;      /* largest n_seq for kva_update_states */
  int32_t compute_dtype;/* 16-bit operand format of the projector: KVA_BF16 or KVA_F16.  The
                           projector matrices, every activation fed to a GEMM, the mixer
                           inputs (mixer_out / mixer_in), the drafter outputs and the conv
                           state are in this format; accumulation is fp32 throughout. */
} kva_dims;

/* Weights of one projector block (device pointers). */
typedef struct kva_block_weights {
  const float* g_attn;  /* [d] RMSNorm gain before attention (effective gain, no +1) */
  const void* Wq;       /* [d, d] in compute_dtype (bf16 or fp16), like every matrix below */
  const void* Wk;       /* [d, d] */
  const void* Wv;       /* [d, d] */
  const void* Wo;       /* [d, d] */
  const float* g_ffn;   /* [d] RMSNorm gain before the FFN */
  const void* Wg;       /* [ffn, d] gate */
  const void* Wu;       /* [ffn, d] up */
  const void* Wd;       /* [d, ffn] down */
} kva_block_weights;

/* Projector weights and the late layers' own parameters (device pointers). */
typedef struct kva_weights {
  const float* g_in;    /* [H] input RMSNorm gain */
  const void* W_in;     /* [d, H], compute_dtype */
  kva_block_weights blocks[KVA_MAX_BLOCKS];
  const float* g_out;   /* [d] output RMSNorm gain */
  const void* W_heads;  /* [n_mix + n_draft_cols, d], compute_dtype: the heads of all late layers
                           concatenated in layer order, then the drafter heads.  Per GDN
                           layer the rows are [q (n_k*d_k) | k (n_k*d_k) | v (n_v*d_v) |
                           a (n_v) | b (n_v)], per attention layer [k (n_kv*d_h) | v (n_kv*d_h)]. */
  const float* conv_w;  /* [n_gdn, C, conv_k], C = 2*n_k*d_k + n_v*d_v; tap conv_k-1 = current token */
  const float* A_log;   /* [n_gdn, n_v] */
  const float* dt_bias; /* [n_gdn, n_v] */
  const float* k_norm_g;/* [n_attn, d_h] k RMSNorm gain */
  /* Projector weight format (the model card's projector quantization: q8_0 projectors at
   * about the quality of 16-bit ones).  KVA_W_16: the matrices above are compute_dtype.
   * KVA_W_Q8_0: every projector matrix pointer above (W_in, each block's Wq..Wd, W_heads)
   * holds int8 codes [N, K] row-major instead, and the matching *_scale pointer below
   * fp16 scales [K / 32, N] (one 32-wide K block of all N rows contiguous); the weight
   * (n, k) is scale[k / 32][n] * code[n][k].  KVA_W_Q4_0: the same with packed 4-bit
   * codes, uint8 [N, K / 2]: per 32-wide K block of a row 16 bytes, byte j holding the code
   * c (0..15) of element j in its low nibble and that of element j + 16 in its high
   * nibble; the weight is scale[k / 32][n] * (c - 8).  Every K (H, d, ffn) must be a
   * multiple of 64.  The prefill then runs the heads GEMM without the fused state-update
   * epilogue. */
  int32_t weight_format;
  const void* W_in_scale;
  const void* W_heads_scale;
  const void* block_scale[KVA_MAX_BLOCKS][7]; /* Wq, Wk, Wv, Wo, Wg, Wu, Wd */
} kva_weights;

typedef enum kva_weight_format { KVA_W_16 = 0, KVA_W_Q8_0 = 1, KVA_W_Q4_0 = 2 } kva_weight_format;

/* KV caches of the attention layers (device pointers, written in place).
 * CONTIGUOUS: k[l], v[l] are [n_seq, n_kv, max_pos, row]; token p of sequence s
 *             goes to row p.
 * PAGED:      k[l], v[l] are [n_pages, n_kv, page_size, row]; token p of sequence s
 *             goes to page page_table[s * pages_per_seq + p / page_size], row
 *             p % page_size.  page_table is int32 on the device.
 * A row is d_h values in bf16 or fp16 (dtype KVA_BF16 / KVA_F16), or, for KVA_Q8_0,
 * the quantized-cache form of the model card's other notes (with q8_0 caches the
 * approximated rows are rotated by the exact layers' Hadamard transform): the row (K after k
 * RMSNorm + RoPE, V as predicted) times the orthonormal Walsh-Hadamard matrix
 * H_{d_h} / sqrt(d_h) in Sylvester order, stored as d_h / 32 blocks of 34 bytes, each
 * an fp16 scale d = max|x| / 127 followed by 32 int8 codes round(x / d) (half away
 * from zero); a value reads back as d * code.  Row size d_h * 34 / 32 bytes. */
typedef struct kva_kv_cache {
  int32_t layout;            /* kva_kv_layout */
  int32_t n_layers;          /* must equal the number of attention layers */
  void* k[KVA_MAX_LATE];
  void* v[KVA_MAX_LATE];
  int64_t max_pos;           /* CONTIGUOUS: rows per (sequence, head) */
  int32_t page_size;         /* PAGED: tokens per page */
  int32_t n_pages;           /* PAGED: pages in each layer's pool */
  int32_t pages_per_seq;     /* PAGED: columns of page_table */
  const int32_t* page_table; /* PAGED: [n_seq, pages_per_seq] */
  int32_t dtype;             /* row format of the caches: KVA_BF16, KVA_F16 or KVA_Q8_0 */
} kva_kv_cache;

typedef struct kva_handle kva_handle;

/* Validate dims, select the current CUDA device, allocate the workspace for
 * max_T tokens x max_seq sequences.  *out receives the handle (NULL on error). */
int kva_init(const kva_dims* dims, kva_handle** out);

/* Bytes of device workspace kva_init allocates for these dims (0 if invalid). */
size_t kva_workspace_bytes(const kva_dims* dims);

/* One ubatch of one sequence: projector + all state updates.
 *   residual       [T, H] in residual_dtype (KVA_BF16, KVA_F16 or KVA_F32)
 *   T              1..max_T tokens
 *   deltanet_state fp32 [n_gdn, n_v, d_v, d_k], read and updated in place
 *   conv_state     compute_dtype [n_gdn, conv_k-1, C], the last raw conv inputs (oldest
 *                  first), read and updated in place
 *   kv             caches written at positions pos .. pos+T-1 (sequence 0)
 *   pos            absolute position of the first token (RoPE angle and cache row)
 *   draft_out      compute_dtype [T, n_draft_cols] or NULL (drafter outputs)
 *   mixer_out      compute_dtype [T, n_mix] or NULL: when given, the mixer inputs are written
 *                  there (and read back by the state updates) instead of the workspace */
int kva_prefill_ubatch(kva_handle* h, const void* residual, int32_t residual_dtype,
                       int32_t T, const kva_weights* w, float* deltanet_state,
                       void* conv_state, const kva_kv_cache* kv, int64_t pos,
                       void* draft_out, void* mixer_out, void* stream);

/* State updates only, for n_seq independent sequences of T tokens each.
 *   mixer_in  compute_dtype [n_seq, T, mixer_ld] (the first n_mix columns are used)
 *   pos       HOST int64 [n_seq], first position of each sequence's ubatch
 *   state     fp32 [n_seq, n_gdn, n_v, d_v, d_k], in place
 *   conv_state compute_dtype [n_seq, n_gdn, conv_k-1, C], in place
 *   debug_qkv bf16 [n_seq, n_gdn, T, 2*n_k*d_k + n_v*d_v] or NULL: when given,
 *             receives [q_hat | k_hat | v] after conv, SiLU and the L2 norms
 *   debug_gb  fp32 [n_seq, n_gdn, 2, n_v, T] or NULL: receives g then beta */
int kva_update_states(kva_handle* h, const void* mixer_in, int64_t mixer_ld, int32_t n_seq,
                      int32_t T, const int64_t* pos, const kva_weights* w, float* state,
                      void* conv_state, const kva_kv_cache* kv, void* debug_qkv,
                      void* debug_gb, void* stream);

/* Parameters of the exact last-token pass that the projector path does not need. */
typedef struct kva_last_params {
  int32_t attn_n_q;          /* query heads of an attention layer: a multiple of attn_n_kv, at
                                most 8 per KV head (24 over 4 in the model card's base model) */
  const float* gdn_norm_w;   /* [n_gdn, d_v] weight of the gated RMSNorm at each gated-DeltaNet
                                layer's output (device) */
  const float* q_norm_g;     /* [n_attn, d_h] q RMSNorm gain of each attention layer (device) */
} kva_last_params;

/* The exact last-token pass through ONE late layer's token mixer, for n_seq sequences
 * ("Qwen3.8-27B-KVA" model card, "What the hell?": after the cheap state updates the engine
 * runs the last token of each ubatch through the late layers exactly, on top of the
 * approximated context).  When this pass follows, kva_prefill_ubatch covers tokens
 * 0..T-2 of the ubatch and the last token reaches each late layer's state / cache here,
 * with that layer's exact inputs; the caller runs the layers in order, since each layer's
 * inputs come from the base model's projections of the previous layer's output (those
 * projections, the o-projection and the FFN are the caller's).
 *   layer      index among the n_late late layers (0-based)
 *   x          compute_dtype [n_seq, x_ld], the token's exact inputs of that layer:
 *              gated-DeltaNet: [q | k | v | a | b] as in the mixer, then the output gate
 *              z (n_v * d_v); attention: [k | v] as in the mixer, then q (n_q * d_h) and
 *              its gate (n_q * d_h)
 *   pos        HOST int64 [n_seq], the token's position (RoPE angle and cache row)
 *   w          the late layers' parameters (conv_w, A_log, dt_bias, k_norm_g)
 *   lp         the pass's own parameters (above)
 *   state, conv_state, kv   as in kva_update_states (all layers; this layer's part is
 *              read and updated: the state and conv tail take the token, the caches
 *              get its K and V rows at pos)
 *   out        [n_seq, out_ld] in out_dtype (KVA_F32 or compute_dtype): the mixer output,
 *              n_v * d_v values o = RMSNorm(S q) * w * silu(z) per value head for a
 *              gated-DeltaNet layer, n_q * d_h values softmax(q K^T / sqrt(d_h)) V *
 *              sigmoid(gate) per query head over cache rows 0..pos for an attention layer
 * KV caches must be KVA_BF16 or KVA_F16 (KVA_ERR_UNSUPPORTED for q8_0 caches). */
int kva_last_token_layer(kva_handle* h, int32_t layer, int32_t n_seq, const void* x, int64_t x_ld,
                         const int64_t* pos, const kva_weights* w, const kva_last_params* lp,
                         float* state, void* conv_state, const kva_kv_cache* kv, void* out,
                         int32_t out_dtype, int64_t out_ld, void* stream);

/* Synchronise the handle's last stream, return the device status bits in
 * *status (0 = clean) and clear them.  Returns KVA_ERR_DEVICE when bits were set. */
int kva_get_device_status(kva_handle* h, int32_t* status);

/* Tokens sent through the approximated path since kva_init (host counter). */
int kva_stats(kva_handle* h, int64_t* tokens_approximated);

/* *fused = 1 when kva_prefill_ubatch runs the state updates' inputs (conv + SiLU, L2 norms,
 * gates, k RMSNorm + RoPE + KV cache rows) in the epilogue of the heads GEMM, so the mixer
 * inputs never reach HBM; 0 when it writes the mixer and runs them as separate kernels.
 * The dims decide (128-dim DeltaNet heads, key/value widths in whole 256-column tiles,
 * 256-dim attention heads with 64 rotary dims); both give the same results.
 * KVA_ERR_INVALID_ARG for a null argument. */
int kva_heads_fused(kva_handle* h, int32_t* fused);

/* Stage kinds of the launch plan (for profiling and launch counts). */
typedef enum kva_stage {
  KVA_ST_RMSNORM = 0,     /* every RMSNorm */
  KVA_ST_GEMM_TRUNK = 1,  /* input linear and the blocks' q/k/v, o, gate/up and down GEMMs */
  KVA_ST_ATTENTION = 2,   /* block-causal attention */
  KVA_ST_GEMM_HEADS = 3,  /* the wide GEMM over all per-layer (and drafter) heads */
  KVA_ST_GDN_PREPARE = 4, /* conv + SiLU + L2 norms + gates */
  KVA_ST_GDN_TAIL = 5,    /* conv tail shift */
  KVA_ST_GDN_SCAN = 6,    /* chunked gated delta-rule scan */
  KVA_ST_KV_WRITE = 7,    /* k norm + RoPE + KV cache write */
  KVA_ST_LAST_TOKEN = 8,  /* the exact last-token pass of a late layer */
  KVA_ST_COUNT = 9
} kva_stage;

/* Device-time profile of the stages, summed since the last read. */
typedef struct kva_profile {
  float ms[KVA_ST_COUNT];        /* summed device time between the events around each launch */
  int32_t timed[KVA_ST_COUNT];   /* launches that were timed */
  int64_t launches[KVA_ST_COUNT];/* kernel launches enqueued (counted whether or not timed) */
} kva_profile;

/* capacity > 0: create `capacity` CUDA event pairs and from now on record one pair
 * around every kernel launch on the call's stream (launches beyond the capacity are
 * counted but not timed until the next read).  capacity == 0: stop and release the
 * events.  This is a set-up call (it creates events); the timed calls do not allocate. */
int kva_profile_enable(kva_handle* h, int32_t capacity);

/* Synchronise the handle's stream, fill *out with the summed stage times and launch
 * counts since the last read (or enable), and reset them. */
int kva_profile_read(kva_handle* h, kva_profile* out);

void kva_free(kva_handle* h);
const char* kva_strerror(int32_t status);

#ifdef __cplusplus
}
#endif
#endif /* KVA_H_ */
