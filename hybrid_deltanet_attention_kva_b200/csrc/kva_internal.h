// Internal launchers shared by the translation units of libkva.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kva.h"

namespace kva {

// Every kernel of the library is launched with programmatic stream serialization: it may
// be scheduled while the kernel before it on the stream is finishing.  Each kernel runs
// only set-up work that touches no global memory (barrier init, TMEM allocation, tensor
// map prefetch) before griddepcontrol.wait, which returns once the previous grid has
// completed and its writes are visible; right after it, the kernel lets the next one be
// scheduled.  So at most two grids are in flight and each one sees all earlier results.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
}

enum GemmEpilogue {
  EPI_STORE_BF16 = 0,   // D = acc (in the 16-bit operand format)
  EPI_STORE_F32 = 1,    // D = acc (fp32)
  EPI_ADD_F32 = 2,      // D += acc (fp32 residual stream)
  EPI_SWIGLU_BF16 = 3,  // D[:, j] = silu(gate_j) * up_j (16-bit), gate/up rows from B0/B1
  EPI_MIXER = 4,        // heads GEMM with the state-update epilogue (internal: MixParams)
};

enum GemmBMode {
  B_SINGLE = 0,    // B0 is [N, K]
  B_SEGMENTS = 1,  // B0,B1,B2 stacked along N, each [seg_rows, K] (q, k, v projections)
  B_PAIRED = 2,    // B0 (gate) and B1 (up), each [N, K]; output N columns
};

struct GemmArgs {
  const void* A = nullptr;  // bf16 [M, K], row stride lda elements
  int64_t lda = 0;
  const void* B[3] = {nullptr, nullptr, nullptr};
  int b_mode = B_SINGLE;
  int64_t ldb = 0;          // row stride of every B matrix (elements)
  int64_t seg_rows = 0;     // rows of each segment (B_SEGMENTS)
  void* D = nullptr;        // output columns [0, n_split)
  int64_t ldd = 0;
  void* D1 = nullptr;       // output columns [n_split, N), column index shifted by n_split
  int64_t ldd1 = 0;
  int64_t n_split = 0;      // 0: everything goes to D
  int M = 0, N = 0, K = 0;
  int epilogue = EPI_STORE_BF16;
  int block_n = 0;          // 0: choose
  int dtype = KVA_BF16;     // 16-bit format of A, B and 16-bit outputs: KVA_BF16 or KVA_F16
  int splits = 0;           // ADD_F32 only: K ranges per tile (0: choose)
  int* err = nullptr;       // device status word
  bool b_const = false;     // B is never written by kernels on the stream (weights): the
                            // first stages' B tiles may be loaded before the previous kernel ends
  int wq = 0;               // 0: 16-bit B; 1: B[i] are q8_0 codes (int8 [rows, K]); 2: q4_0
                            //   codes (uint8 [rows, K / 2], two per byte); fp16 scales Bs[i]
  const void* Bs[3] = {nullptr, nullptr, nullptr};  //   [K / 32, rows]
  int64_t lds = 0;          // wq: row stride of Bs in scales (0: the matrix's rows)
  int stall_item1 = 0;      // CTA pairs, test of the failure path (kva_test_gemm_wait_timeout):
                            //   1 + the work item whose MMA issuer waits on a barrier that
                            //   nothing arrives on until the wait runs out (0: never)
};

int num_sms();
// Tiled TMA descriptor (128-byte swizzle, zero fill out of range) of a 16-bit
// array with three dimensions: d0 contiguous, d1 rows of d0 elements, d2 blocks of
// d1 rows; box [box1 rows][box0 elements], one block deep.  False when the driver
// entry point is missing or rejects the arguments.
bool make_map_3d_16bit(void* map, const void* base, bool fp16, int64_t d0, int64_t d1,
                       int64_t d2, int box0, int box1);
int launch_gemm(const GemmArgs& a, cudaStream_t s);
// `zero` (optional): also clear the first nz fp32 values of each row of zero (row stride ldz)
int launch_rmsnorm(const void* x, int x_dtype, int64_t ldx, const float* g, void* out,
                   int64_t ldo, int rows, int n, float eps, cudaStream_t s,
                   int out_dtype = KVA_BF16, float* zero = nullptr, int64_t ldz = 0, int nz = 0);
// err (optional): device status word for a wait that timed out
int launch_attention(const void* qkv, int64_t ldq, void* out, int64_t ldo, int T, int n_heads,
                     int window, cudaStream_t s, int dtype = KVA_BF16, int* err = nullptr);
// 16-bit row-major [rows, inner] (row stride ld elements) for TMA, box [box_rows, box_inner],
// 128-byte swizzle (box_inner x 2 bytes must be 128)
bool make_map_2d_16bit(void* map, const void* base, bool fp16, int64_t inner, int64_t rows,
                       int64_t ld, int box_inner, int box_rows);

struct GdnLaunch {
  int mix_dtype = KVA_BF16;     // format of the mixer inputs and of the conv tail
  const void* mix = nullptr;    // 16-bit [n_seq, T, mix_ld]
  int64_t mix_ld = 0;
  int64_t mix_seq_stride = 0;   // elements between sequences
  int n_seq = 0, T = 0;
  int n_gdn = 0;
  int layer_col[KVA_MAX_LATE] = {0};
  int n_k = 0, n_v = 0, d_k = 0, d_v = 0, C = 0;
  const float* conv_w = nullptr;
  const float* A_log = nullptr;
  const float* dt_bias = nullptr;
  void* conv_state = nullptr;   // 16-bit [n_seq, n_gdn, 3, C]
  float* state = nullptr;       // fp32 [n_seq, n_gdn, n_v, d_v, d_k]
  void* kbuf = nullptr;         // fp16 [n_seq, n_gdn, T, n_k*d_k]
  void* vbuf = nullptr;         // fp16 [n_seq, n_gdn, T, n_v*d_v]
  float* gbuf = nullptr;        // fp32 [n_seq, n_gdn, 2, n_v, T] (g then beta)
  void* b1buf = nullptr;        // d_k = 128: fp16 [n_seq, n_gdn, n_v, chunks, 64, 64]
  float* scbuf = nullptr;       // d_k = 128: fp32 [n_seq, n_gdn, n_v, chunks, 80]
  void* debug_qkv = nullptr;    // bf16 [n_seq, n_gdn, T, C] or null
  float eps = 1e-6f;
  int* err = nullptr;
};
int launch_gdn_prepare(const GdnLaunch& g, cudaStream_t s);
int launch_gdn_tail(const GdnLaunch& g, cudaStream_t s);
int launch_gdn_scan(const GdnLaunch& g, cudaStream_t s);
int launch_gdn_scan_tc(const GdnLaunch& g, cudaStream_t s);  // d_k = d_v = 128
// the two halves of launch_gdn_scan_tc for the layers [l0, l0 + nl): B1 and scalars
// (no state), then the state chain (reads what the first wrote for those layers)
int launch_gdn_chunk_prep(const GdnLaunch& g, int l0, int nl, cudaStream_t s);
int launch_gdn_chain(const GdnLaunch& g, int l0, int nl, cudaStream_t s);
// bytes of the per-chunk buffers (b1buf, then scbuf) the 128-dimensional scan needs
size_t gdn_chunk_bytes(int n_seq, int n_gdn, int n_v, int T);
// b1buf and scbuf inside a region of gdn_chunk_bytes(...) bytes at `base`
void gdn_chunk_split(void* base, int n_seq, int n_gdn, int n_v, int T, void** b1, float** sc);

constexpr int kMaxSeqPos = 256;
struct KvLaunch {
  int mix_dtype = KVA_BF16;
  const void* mix = nullptr;
  int64_t mix_ld = 0;
  int64_t mix_seq_stride = 0;
  int n_seq = 0, T = 0;
  int n_attn = 0;
  int layer_col[KVA_MAX_LATE] = {0};
  int n_kv = 0, d_h = 0, rope_dims = 0;
  double rope_theta = 1e7;
  double inv_freq[128] = {0};     // theta^(-2i / rope_dims), i < rope_dims / 2 (fp64, host)
  const float* k_gain = nullptr;  // [n_attn, d_h]
  int64_t pos[kMaxSeqPos] = {0};
  kva_kv_cache cache;
  float eps = 1e-6f;
  int* err = nullptr;
};
int launch_kv_write(const KvLaunch& k, cudaStream_t s);

// ---------------------------------------------------------------------------
// Exact last-token pass of one late layer (kva_last_token_layer).
struct GdnDecodeLaunch {
  const void* x = nullptr;        // 16-bit [n_seq, x_ld]: [q | k | v | a | b | z] of the token
  int64_t x_ld = 0;
  int x_dtype = KVA_BF16;         // also the conv tail's format
  int n_seq = 0, n_k = 0, n_v = 0, d = 0, C = 0;
  const float* conv_w = nullptr;  // this layer's [C, 4]
  const float* A_log = nullptr;   // [n_v]
  const float* dt_bias = nullptr; // [n_v]
  const float* norm_w = nullptr;  // [d] gated RMSNorm weight
  float* state = nullptr;         // this layer's [n_v, d, d] of sequence 0
  int64_t state_seq_stride = 0;   // floats between sequences
  void* conv_state = nullptr;     // this layer's [3, C] of sequence 0
  int64_t conv_seq_stride = 0;    // elements between sequences
  void* out = nullptr;            // [n_seq, out_ld]
  int64_t out_ld = 0;
  int out_dtype = KVA_BF16;       // KVA_F32 or x_dtype
  float eps = 1e-6f;
};
int launch_gdn_decode(const GdnDecodeLaunch& g, cudaStream_t s);

constexpr int kDecodeMaxSplit = 64;    // cache-row splits per (sequence, KV head)
constexpr int kDecodeSlots = 2048;     // partial states (sequence x KV head x split) in the workspace
constexpr int kDecodeMaxGroup = 8;     // query heads per KV head
struct AttnDecodeLaunch {
  const void* x = nullptr;        // 16-bit [n_seq, x_ld]: [k | v | q | gate] of the token
  int64_t x_ld = 0;
  int x_dtype = KVA_BF16;
  int n_seq = 0, n_kv = 0, n_q = 0, G = 0, d_h = 0, rope_dims = 0;
  double inv_freq[128] = {0};     // theta^(-2i / rope_dims) (fp64, host)
  const float* k_gain = nullptr;  // this layer's [d_h]
  const float* q_gain = nullptr;  // [d_h]
  int64_t pos[kMaxSeqPos] = {0};  // position of each sequence's token
  void* kc = nullptr;             // this layer's K and V caches
  void* vc = nullptr;
  int layout = KVA_KV_CONTIGUOUS;
  int64_t max_pos = 0;
  int page_size = 0, n_pages = 0, pages_per_seq = 0;
  const int32_t* page_table = nullptr;
  int cache_dtype = KVA_BF16;
  int n_split = 1;
  int64_t rows_per_split = 0;     // a multiple of the 64-row tile
  float* part = nullptr;          // [n_seq, n_kv, n_split, G, d_h + 2] partial O, max, sum
  void* out = nullptr;            // [n_seq, out_ld]
  int64_t out_ld = 0;
  int out_dtype = KVA_BF16;
  float eps = 1e-6f;
  int* err = nullptr;
};
// splits of the longest sequence's max_rows cache rows for n_seq x n_kv CTAs on `sms` SMs
int attn_decode_splits(int n_seq, int n_kv, int64_t max_rows, int sms, int64_t* rows_per_split);
int launch_attn_decode(const AttnDecodeLaunch& a, cudaStream_t s);

// ---------------------------------------------------------------------------
// Heads GEMM with the state-update epilogue (the wide head GEMM writes the scan's
// inputs, the gates and the KV-cache rows directly instead of the mixer).
// The N dimension is tiled per layer segment: every tile lies inside one segment.
enum MixKind {
  MIX_RAW = 0,      // q columns of a gated-DeltaNet layer: only conv-tail / halo / debug copies
  MIX_GDN_K = 1,    // k columns: conv + SiLU + per-head L2 norm -> kbuf
  MIX_GDN_V = 2,    // v columns: conv + SiLU -> vbuf
  MIX_GDN_AB = 3,   // a | b columns of two layers (one per tile half): gates g, beta -> gbuf
  MIX_ATT_K = 4,    // one attention key head: RMSNorm x gain, RoPE -> K cache
  MIX_ATT_V = 5,    // one attention value head -> V cache
  MIX_DRAFT = 6,    // drafter columns -> draft_out
};
struct MixTile {
  int col0;    // first row of W_heads (column of the mixer) of the tile's columns 0-127
  int col1;    // first row of its columns 128-255 (col0 + 128, except for gate tiles)
  int ncols;   // valid columns (<= 256; per half for gate tiles)
  int kind;    // MixKind
  int layer;   // index among the gated-DeltaNet layers (GDN kinds) or the attention layers
  int sub;     // offset inside the segment: conv channel of column 0 (GDN kinds), value
               // channel (GDN V), key channel (GDN K), head (ATT kinds), drafter column;
               // for a gate tile the layer of its second half (-1: none)
};
constexpr int kMixHaloRows = 6;  // rows 0, 1, 2, 125, 126, 127 of every 128-token block
struct MixParams {
  const MixTile* tiles = nullptr;
  int T = 0;
  int64_t pos = 0;
  // gated-DeltaNet layers
  int n_k = 0, n_v = 0, C = 0;    // C = conv channels (q | k | v)
  const float* conv_w = nullptr;  // [n_gdn, C, 4]
  const float* A_log = nullptr;   // [n_gdn, n_v]
  const float* dt_bias = nullptr; // [n_gdn, n_v]
  void* kbuf = nullptr;           // fp16 [n_gdn, T, n_k*128]
  void* vbuf = nullptr;           // fp16 [n_gdn, T, n_v*128]
  float* gbuf = nullptr;          // fp32 [n_gdn, 2, n_v, T]
  void* halo = nullptr;           // 16-bit [n_gdn, nblk, 6, C] raw rows around block edges
  void* tail_new = nullptr;       // 16-bit [n_gdn, 3, C] raw rows T-3 .. T-1
  int nblk = 0;                   // 128-token blocks of the workspace (max_T / 128)
  float eps = 1e-6f;
  // attention layers
  int n_kv = 0;                   // KV heads per attention layer (head dim 256)
  const float* k_gain = nullptr;  // [n_attn, 256]
  int rope_dims = 64;
  double rope_theta = 1e7;
  double inv_freq[32] = {0};      // theta^(-2i / 64), i < 32 (fp64, host)
  kva_kv_cache cache;
  // outputs kept from the plain path
  void* draft = nullptr;          // [T, n_draft_cols] or null
  int64_t ld_draft = 0;
  void* mixer_out = nullptr;      // [T, n_mix] debug copy of the raw mixer, or null
  int64_t ld_mix = 0;
  void* att_raw = nullptr;        // [T, ld_att_raw] at mixer columns: attention k/v stay raw here
  int64_t ld_att_raw = 0;         //   (a q8_0 cache is written by the plain KV writer after)
  int* err = nullptr;
};
// The heads GEMM over `num_tiles` tiles of the table, A = z [M, K] (16-bit, lda), B = W_heads.
int launch_heads_fused(int dtype, const void* A, int64_t lda, const void* W, int64_t n_rows_w,
                       int M, int K, int num_tiles, const MixParams& mp, cudaStream_t s);
// After the fused heads GEMM: the conv outputs of the first 3 rows of every 128-token block
// (from the halo rows and the old conv tail), then the new conv tail.
int launch_gdn_halo_fix(const MixParams& mp, int n_gdn, cudaStream_t s, int dtype,
                        const void* conv_state);
int launch_gdn_tail_fused(const MixParams& mp, int n_gdn, void* conv_state, cudaStream_t s);

}  // namespace kva
