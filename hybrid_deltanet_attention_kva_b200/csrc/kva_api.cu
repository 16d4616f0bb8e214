// C ABI of libkva: argument validation, workspace ownership and the launch plan
// of one KVA ubatch ("Qwen3.8-27B-KVA" model card, "What the hell?": from each
// token's layer-31 residual the projector predicts what every late layer's token
// mixer takes as input, and the cheap state updates then consume those predictions).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>
#include <vector>

#include "../../include/kva.h"
#include "../../include/kva_ops.h"
#include "kva_internal.h"

using namespace kva;

struct kva_handle {
  kva_dims d;
  int device = 0;
  int n_gdn = 0, n_attn = 0;
  int C = 0, gdn_width = 0, attn_width = 0;
  int64_t n_mix = 0;
  int gdn_col[KVA_MAX_LATE] = {0};
  int attn_col[KVA_MAX_LATE] = {0};
  // workspace (one allocation)
  void* ws = nullptr;
  size_t ws_bytes = 0;
  __nv_bfloat16* u_in = nullptr;  // [max_T, H]
  __nv_bfloat16* u = nullptr;     // [max_T, d]
  float* x = nullptr;             // [max_T, d]
  __nv_bfloat16* qkv = nullptr;   // [max_T, max(3d, ffn)]: q|k|v, then the FFN hidden
  __nv_bfloat16* o = nullptr;     // [max_T, d]
  __nv_bfloat16* mixer = nullptr; // [max_T, n_mix]
  __nv_bfloat16* kbuf = nullptr;  // [max_seq, n_gdn, max_T, n_k d_k]
  __nv_bfloat16* vbuf = nullptr;  // [max_seq, n_gdn, max_T, n_v d_v]
  float* gbuf = nullptr;          // [max_seq, n_gdn, 2, n_v, max_T]
  float* dec_part = nullptr;      // last-token attention partials [kDecodeSlots, 8, d_h + 2]
  int* status = nullptr;          // device status word
  void* chunk = nullptr;          // per-chunk B1 and scalars of the 128-dimensional scan
  // heads GEMM with the state-update epilogue (kva_prefill_ubatch), when the dims allow it
  bool fused = false;
  MixTile* tiles = nullptr;       // device table: [n_tiles], drafter tiles last
  int n_tiles = 0, n_tiles_draft = 0;
  void* halo = nullptr;           // raw rows around 128-token block edges
  void* tail_new = nullptr;       // raw last 3 rows of the ubatch
  int nblk = 0;
  cudaStream_t last_stream = nullptr;
  int64_t tokens = 0;
  // profiling: event pairs around launches, launch counters per stage kind
  cudaEvent_t* ev = nullptr;
  int* ev_kind = nullptr;
  int ev_cap = 0, ev_used = 0;
  int64_t launches[KVA_ST_COUNT] = {0};
};

namespace {
// Runs one launcher between the stage's events (when profiling) and counts it.
template <typename F>
int staged(kva_handle* h, int kind, cudaStream_t s, F&& launch) {
  const bool timed = h->ev_cap > 0 && h->ev_used < h->ev_cap;
  if (timed) cudaEventRecord(h->ev[2 * h->ev_used], s);
  const int e = launch();
  if (timed) {
    cudaEventRecord(h->ev[2 * h->ev_used + 1], s);
    h->ev_kind[h->ev_used++] = kind;
  }
  if (!e) ++h->launches[kind];
  return e;
}
}  // namespace

namespace {

struct Layout {
  size_t off[16];
  size_t total;
};

size_t align_up(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

int derive(const kva_dims* d, int* n_gdn, int* n_attn, int64_t* n_mix) {
  if (!d) return KVA_ERR_INVALID_ARG;
  if (d->hidden <= 0 || d->d_model <= 0 || d->n_heads <= 0 || d->ffn <= 0 || d->n_blocks < 0 ||
      d->n_blocks > KVA_MAX_BLOCKS || d->n_late <= 0 || d->n_late > KVA_MAX_LATE ||
      d->max_T <= 0 || d->max_seq <= 0 || d->attn_window < 0 || d->n_draft_cols < 0 ||
      !(d->norm_eps >= 0.f))
    return KVA_ERR_INVALID_ARG;
  if (d->head_dim != 128 || d->n_heads * d->head_dim != d->d_model) return KVA_ERR_UNSUPPORTED;
  if (d->hidden % 64 || d->d_model % 256 || d->ffn % 64) return KVA_ERR_UNSUPPORTED;
  if (d->conv_k != 4) return KVA_ERR_UNSUPPORTED;
  if (d->max_seq > kMaxSeqPos) return KVA_ERR_UNSUPPORTED;
  if (d->compute_dtype != KVA_BF16 && d->compute_dtype != KVA_F16) return KVA_ERR_INVALID_ARG;
  int ng = 0, na = 0;
  for (int i = 0; i < d->n_late; ++i) {
    if (d->layer_type[i] == KVA_LAYER_GDN) ++ng;
    else if (d->layer_type[i] == KVA_LAYER_ATTN) ++na;
    else return KVA_ERR_INVALID_ARG;
  }
  if (ng) {
    if (d->gdn_n_k <= 0 || d->gdn_n_v <= 0 || d->gdn_n_v % d->gdn_n_k) return KVA_ERR_INVALID_ARG;
    if (d->gdn_d_k != d->gdn_d_v || (d->gdn_d_k != 64 && d->gdn_d_k != 128))
      return KVA_ERR_UNSUPPORTED;
    if ((d->gdn_n_k * d->gdn_d_k) % 128) return KVA_ERR_UNSUPPORTED;
  }
  if (na) {
    if (d->attn_n_kv <= 0 || (d->attn_d_h != 128 && d->attn_d_h != 256)) return KVA_ERR_UNSUPPORTED;
    if (d->rope_dims < 0 || d->rope_dims % 2 || d->rope_dims > d->attn_d_h)
      return KVA_ERR_UNSUPPORTED;
    if (!(d->rope_theta > 1.0)) return KVA_ERR_INVALID_ARG;
  }
  const int64_t C = 2LL * d->gdn_n_k * d->gdn_d_k + (int64_t)d->gdn_n_v * d->gdn_d_v;
  const int64_t gw = C + 2LL * d->gdn_n_v;
  const int64_t aw = 2LL * d->attn_n_kv * d->attn_d_h;
  const int64_t nm = ng * gw + na * aw;
  // every row of the mixer and its per-layer blocks must stay 16-byte aligned for the
  // vector loads of the state-update kernels
  if ((ng && gw % 8) || nm % 8 || d->n_draft_cols % 32) return KVA_ERR_UNSUPPORTED;
  *n_gdn = ng;
  *n_attn = na;
  *n_mix = nm;
  return KVA_OK;
}

// The fused heads epilogue needs 128-dim DeltaNet heads, key/value widths in whole
// 256-column tiles, a layer's gates in half a tile, 256-dim attention heads with 64
// rotary dims.
bool fused_ok(const kva_dims* d, int ng, int na) {
  if (ng) {
    if (d->gdn_d_k != 128 || d->gdn_d_v != 128) return false;
    if ((d->gdn_n_k * 128) % 256 || (d->gdn_n_v * 128) % 256 || 2 * d->gdn_n_v > 128) return false;
  }
  if (na && (d->attn_d_h != 256 || d->rope_dims != 64)) return false;
  return d->n_draft_cols % 8 == 0;
}

int fused_tiles(const kva_dims* d, int ng, int na, int* n_draft_tiles) {
  const int per_gdn = 2 * (d->gdn_n_k * 128 / 256) + d->gdn_n_v * 128 / 256;
  *n_draft_tiles = (d->n_draft_cols + 255) / 256;
  return ng * per_gdn + (ng + 1) / 2 + na * 2 * d->attn_n_kv + *n_draft_tiles;  // gates: 2 layers a tile
}

Layout layout_of(const kva_dims* d, int ng, int64_t n_mix) {
  const size_t T = d->max_T, S = d->max_seq;
  const size_t dm = d->d_model;
  const size_t C = 2ull * d->gdn_n_k * d->gdn_d_k + (size_t)d->gdn_n_v * d->gdn_d_v;
  size_t sz[15];
  sz[0] = T * d->hidden * 2;                                          // u_in
  sz[1] = T * dm * 2;                                                 // u
  sz[2] = T * dm * 4;                                                 // x
  sz[3] = T * (3 * dm > (size_t)d->ffn ? 3 * dm : (size_t)d->ffn) * 2; // qkv / FFN hidden
  sz[4] = T * dm * 2;                                                 // o
  sz[5] = T * (size_t)n_mix * 2;                                      // mixer
  sz[6] = S * ng * T * (size_t)d->gdn_n_k * d->gdn_d_k * 2;           // kbuf
  sz[7] = S * ng * T * (size_t)d->gdn_n_v * d->gdn_d_v * 2;           // vbuf
  sz[8] = S * ng * 2 * (size_t)d->gdn_n_v * T * 4;                    // gbuf
  sz[9] = 256;                                                        // status
  sz[10] = d->gdn_d_k == 128 ? gdn_chunk_bytes((int)S, ng, d->gdn_n_v, (int)T) : 0;  // B1, scalars
  int na = 0;
  for (int i = 0; i < d->n_late; ++i) na += d->layer_type[i] == KVA_LAYER_ATTN;
  const bool fz = fused_ok(d, ng, na);
  int ndt = 0;
  const size_t nblk = (T + 127) / 128;
  sz[11] = fz ? ng * nblk * kMixHaloRows * C * 2 : 0;                      // halo rows
  sz[12] = fz ? ng * 3 * C * 2 : 0;                                         // last rows
  sz[13] = fz ? fused_tiles(d, ng, na, &ndt) * sizeof(MixTile) : 0;         // tile table
  // partial states of the last-token attention (sequence x KV head x split slots)
  sz[14] = na ? (size_t)kDecodeSlots * kDecodeMaxGroup * (d->attn_d_h + 2) * 4 : 0;
  Layout L;
  size_t o = 0;
  for (int i = 0; i < 15; ++i) {
    L.off[i] = o;
    o += align_up(sz[i]);
  }
  L.total = o;
  return L;
}

bool a16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int cuda_ok(cudaError_t e) { return e == cudaSuccess ? KVA_OK : KVA_ERR_CUDA; }

int check_weights(const kva_handle* h, const kva_weights* w, bool projector) {
  if (!w) return KVA_ERR_INVALID_ARG;
  if (h->n_gdn && (!w->conv_w || !w->A_log || !w->dt_bias)) return KVA_ERR_INVALID_ARG;
  if (h->n_attn && !w->k_norm_g) return KVA_ERR_INVALID_ARG;
  if (!projector) return KVA_OK;
  if (!w->g_in || !w->W_in || !w->g_out || !w->W_heads) return KVA_ERR_INVALID_ARG;
  if (!a16(w->g_in) || !a16(w->W_in) || !a16(w->g_out) || !a16(w->W_heads)) return KVA_ERR_ALIGNMENT;
  for (int b = 0; b < h->d.n_blocks; ++b) {
    const kva_block_weights& B = w->blocks[b];
    const void* ps[9] = {B.g_attn, B.Wq, B.Wk, B.Wv, B.Wo, B.g_ffn, B.Wg, B.Wu, B.Wd};
    for (const void* p : ps) {
      if (!p) return KVA_ERR_INVALID_ARG;
      if (!a16(p)) return KVA_ERR_ALIGNMENT;
    }
  }
  if (w->weight_format == KVA_W_Q8_0 || w->weight_format == KVA_W_Q4_0) {
    const kva_dims& d = h->d;
    if (d.hidden % 64 || d.d_model % 64 || d.ffn % 64) return KVA_ERR_UNSUPPORTED;
    if (!w->W_in_scale || !w->W_heads_scale) return KVA_ERR_INVALID_ARG;
    if (!a16(w->W_in_scale) || !a16(w->W_heads_scale)) return KVA_ERR_ALIGNMENT;
    for (int b = 0; b < d.n_blocks; ++b)
      for (int i = 0; i < 7; ++i) {
        if (!w->block_scale[b][i]) return KVA_ERR_INVALID_ARG;
        if (!a16(w->block_scale[b][i])) return KVA_ERR_ALIGNMENT;
      }
  } else if (w->weight_format != KVA_W_16) {
    return KVA_ERR_INVALID_ARG;
  }
  return KVA_OK;
}

int check_cache(const kva_handle* h, const kva_kv_cache* kv, int n_seq, const int64_t* pos, int T) {
  if (!h->n_attn) return KVA_OK;
  if (!kv || kv->n_layers != h->n_attn) return KVA_ERR_INVALID_ARG;
  for (int i = 0; i < h->n_attn; ++i) {
    if (!kv->k[i] || !kv->v[i]) return KVA_ERR_INVALID_ARG;
    if (!a16(kv->k[i]) || !a16(kv->v[i])) return KVA_ERR_ALIGNMENT;
  }
  for (int s = 0; s < n_seq; ++s)
    if (pos[s] < 0) return KVA_ERR_INVALID_ARG;
  if (kv->layout == KVA_KV_CONTIGUOUS) {
    if (kv->max_pos <= 0) return KVA_ERR_INVALID_ARG;
    for (int s = 0; s < n_seq; ++s)
      if (pos[s] + T > kv->max_pos) return KVA_ERR_TOO_LARGE;
  } else if (kv->layout == KVA_KV_PAGED) {
    if (kv->page_size <= 0 || kv->n_pages <= 0 || kv->pages_per_seq <= 0 || !kv->page_table)
      return KVA_ERR_INVALID_ARG;
    for (int s = 0; s < n_seq; ++s)
      if (pos[s] + T > (int64_t)kv->pages_per_seq * kv->page_size) return KVA_ERR_TOO_LARGE;
  } else {
    return KVA_ERR_INVALID_ARG;
  }
  return KVA_OK;
}

// fz: the heads GEMM already ran the fused epilogue (conv outputs except block edges,
// gates, KV rows); only the edge fix-up, the conv tail and the scan remain, and the KV
// writer when the epilogue left the attention k/v raw (fz->att_raw, a q8_0 cache).
int update_states_impl(kva_handle* h, const void* mix, int64_t mix_ld, int n_seq, int T,
                       const int64_t* pos, const kva_weights* w, float* state, void* conv_state,
                       const kva_kv_cache* kv, void* debug_qkv, void* debug_gb, cudaStream_t s,
                       const MixParams* fz = nullptr) {
  const kva_dims& d = h->d;
  int e = KVA_OK;
  if (h->n_gdn) {
    GdnLaunch g;
    g.mix = fz ? static_cast<const void*>(h->kbuf) : mix;  // (unread when fused)
    g.mix_ld = mix_ld;
    g.mix_seq_stride = (int64_t)T * mix_ld;
    g.n_seq = n_seq;
    g.T = T;
    g.n_gdn = h->n_gdn;
    for (int i = 0; i < h->n_gdn; ++i) g.layer_col[i] = h->gdn_col[i];
    g.n_k = d.gdn_n_k;
    g.n_v = d.gdn_n_v;
    g.d_k = d.gdn_d_k;
    g.d_v = d.gdn_d_v;
    g.C = h->C;
    g.conv_w = w->conv_w;
    g.A_log = w->A_log;
    g.dt_bias = w->dt_bias;
    g.conv_state = conv_state;
    g.state = state;
    g.kbuf = h->kbuf;
    g.vbuf = h->vbuf;
    g.gbuf = debug_gb ? static_cast<float*>(debug_gb) : h->gbuf;
    gdn_chunk_split(h->chunk, n_seq, h->n_gdn, d.gdn_n_v, T, &g.b1buf, &g.scbuf);
    g.debug_qkv = debug_qkv;
    g.eps = d.norm_eps;
    g.err = h->status;
    g.mix_dtype = d.compute_dtype;
    if (fz) {
      if ((e = staged(h, KVA_ST_GDN_PREPARE, s, [&] {
             return launch_gdn_halo_fix(*fz, h->n_gdn, s, d.compute_dtype, conv_state);
           })))
        return e;
      if ((e = staged(h, KVA_ST_GDN_TAIL, s,
                      [&] { return launch_gdn_tail_fused(*fz, h->n_gdn, conv_state, s); })))
        return e;
    } else {
      if ((e = staged(h, KVA_ST_GDN_PREPARE, s, [&] { return launch_gdn_prepare(g, s); }))) return e;
      if ((e = staged(h, KVA_ST_GDN_TAIL, s, [&] { return launch_gdn_tail(g, s); }))) return e;
    }
    if ((e = staged(h, KVA_ST_GDN_SCAN, s, [&] { return launch_gdn_scan(g, s); }))) return e;
    if (d.gdn_d_k == 128) ++h->launches[KVA_ST_GDN_SCAN];  // two kernels
  }
  if (h->n_attn && (!fz || fz->att_raw)) {
    KvLaunch k;
    k.mix = fz ? fz->att_raw : mix;
    k.mix_ld = fz ? fz->ld_att_raw : mix_ld;
    k.mix_seq_stride = (int64_t)T * k.mix_ld;
    k.n_seq = n_seq;
    k.T = T;
    k.n_attn = h->n_attn;
    for (int i = 0; i < h->n_attn; ++i) k.layer_col[i] = h->attn_col[i];
    k.n_kv = d.attn_n_kv;
    k.d_h = d.attn_d_h;
    k.rope_dims = d.rope_dims;
    k.rope_theta = d.rope_theta;
    for (int i = 0; i < d.rope_dims / 2 && i < 128; ++i)
      k.inv_freq[i] = std::pow(d.rope_theta, -2.0 * i / d.rope_dims);
    k.k_gain = w->k_norm_g;
    for (int i = 0; i < n_seq; ++i) k.pos[i] = pos[i];
    k.cache = *kv;
    k.eps = d.norm_eps;
    k.err = h->status;
    k.mix_dtype = d.compute_dtype;
    if ((e = staged(h, KVA_ST_KV_WRITE, s, [&] { return launch_kv_write(k, s); }))) return e;
  }
  return KVA_OK;
}

}  // namespace

extern "C" {

size_t kva_workspace_bytes(const kva_dims* dims) {
  int ng, na;
  int64_t nm;
  if (derive(dims, &ng, &na, &nm)) return 0;
  return layout_of(dims, ng, nm).total;
}

int kva_init(const kva_dims* dims, kva_handle** out) {
  if (!out) return KVA_ERR_INVALID_ARG;
  *out = nullptr;
  int ng, na;
  int64_t nm;
  int e = derive(dims, &ng, &na, &nm);
  if (e) return e;
  kva_handle* h = new (std::nothrow) kva_handle();
  if (!h) return KVA_ERR_NO_MEMORY;
  h->d = *dims;
  h->n_gdn = ng;
  h->n_attn = na;
  h->n_mix = nm;
  h->C = 2 * dims->gdn_n_k * dims->gdn_d_k + dims->gdn_n_v * dims->gdn_d_v;
  h->gdn_width = h->C + 2 * dims->gdn_n_v;
  h->attn_width = 2 * dims->attn_n_kv * dims->attn_d_h;
  int col = 0, gi = 0, ai = 0;
  for (int i = 0; i < dims->n_late; ++i) {
    if (dims->layer_type[i] == KVA_LAYER_GDN) {
      h->gdn_col[gi++] = col;
      col += h->gdn_width;
    } else {
      h->attn_col[ai++] = col;
      col += h->attn_width;
    }
  }
  if (cudaGetDevice(&h->device) != cudaSuccess) {
    delete h;
    return KVA_ERR_CUDA;
  }
  Layout L = layout_of(dims, ng, nm);
  if (cudaMalloc(&h->ws, L.total) != cudaSuccess) {
    cudaGetLastError();
    delete h;
    return KVA_ERR_NO_MEMORY;
  }
  h->ws_bytes = L.total;
  uint8_t* b = static_cast<uint8_t*>(h->ws);
  h->u_in = reinterpret_cast<__nv_bfloat16*>(b + L.off[0]);
  h->u = reinterpret_cast<__nv_bfloat16*>(b + L.off[1]);
  h->x = reinterpret_cast<float*>(b + L.off[2]);
  h->qkv = reinterpret_cast<__nv_bfloat16*>(b + L.off[3]);
  h->o = reinterpret_cast<__nv_bfloat16*>(b + L.off[4]);
  h->mixer = reinterpret_cast<__nv_bfloat16*>(b + L.off[5]);
  h->kbuf = reinterpret_cast<__nv_bfloat16*>(b + L.off[6]);
  h->vbuf = reinterpret_cast<__nv_bfloat16*>(b + L.off[7]);
  h->gbuf = reinterpret_cast<float*>(b + L.off[8]);
  h->status = reinterpret_cast<int*>(b + L.off[9]);
  h->chunk = b + L.off[10];
  h->dec_part = na ? reinterpret_cast<float*>(b + L.off[14]) : nullptr;
  h->fused = fused_ok(dims, ng, na);
  if (h->fused) {
    h->halo = b + L.off[11];
    h->tail_new = b + L.off[12];
    h->tiles = reinterpret_cast<MixTile*>(b + L.off[13]);
    h->nblk = (dims->max_T + 127) / 128;
    // the tile table: every tile inside one layer segment, drafter tiles last
    std::vector<MixTile> tab;
    const int nkdk = dims->gdn_n_k * 128, nvdv = dims->gdn_n_v * 128;
    int gi = 0, ai = 0;
    auto tile = [](int col0, int ncols, int kind, int layer, int sub) {
      return MixTile{col0, col0 + 128, ncols, kind, layer, sub};
    };
    for (int i = 0; i < dims->n_late; ++i) {
      if (dims->layer_type[i] == KVA_LAYER_GDN) {
        const int c = h->gdn_col[gi];
        for (int j = 0; j < nkdk; j += 256) tab.push_back(tile(c + j, 256, MIX_RAW, gi, j));
        for (int j = 0; j < nkdk; j += 256) tab.push_back(tile(c + nkdk + j, 256, MIX_GDN_K, gi, nkdk + j));
        for (int j = 0; j < nvdv; j += 256)
          tab.push_back(tile(c + 2 * nkdk + j, 256, MIX_GDN_V, gi, 2 * nkdk + j));
        // the gates of layers 2m and 2m + 1 share one tile, one layer per half
        if (gi % 2 == 1)
          tab.push_back({h->gdn_col[gi - 1] + h->C, c + h->C, 2 * dims->gdn_n_v, MIX_GDN_AB, gi - 1, gi});
        else if (gi == h->n_gdn - 1)
          tab.push_back({c + h->C, c + h->C, 2 * dims->gdn_n_v, MIX_GDN_AB, gi, -1});
        ++gi;
      } else {
        const int c = h->attn_col[ai];
        for (int j = 0; j < dims->attn_n_kv; ++j) tab.push_back(tile(c + 256 * j, 256, MIX_ATT_K, ai, j));
        for (int j = 0; j < dims->attn_n_kv; ++j)
          tab.push_back(tile(c + 256 * (dims->attn_n_kv + j), 256, MIX_ATT_V, ai, j));
        ++ai;
      }
    }
    h->n_tiles = static_cast<int>(tab.size());
    for (int j = 0; j < dims->n_draft_cols; j += 256) {
      const int w = dims->n_draft_cols - j < 256 ? dims->n_draft_cols - j : 256;
      tab.push_back(tile(static_cast<int>(nm) + j, w, MIX_DRAFT, 0, j));
    }
    h->n_tiles_draft = static_cast<int>(tab.size()) - h->n_tiles;
    if (cudaMemcpy(h->tiles, tab.data(), tab.size() * sizeof(MixTile), cudaMemcpyHostToDevice) !=
        cudaSuccess) {
      cudaGetLastError();
      cudaFree(h->ws);
      delete h;
      return KVA_ERR_CUDA;
    }
  }
  if (cudaMemset(h->status, 0, 256) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) {
    cudaGetLastError();
    cudaFree(h->ws);
    delete h;
    return KVA_ERR_CUDA;
  }
  *out = h;
  return KVA_OK;
}

int kva_profile_enable(kva_handle* h, int32_t capacity) {
  if (!h || capacity < 0) return KVA_ERR_INVALID_ARG;
  int cur = 0;
  cudaGetDevice(&cur);
  if (cur != h->device) cudaSetDevice(h->device);
  int e = KVA_OK;
  if (h->ev) {
    cudaStreamSynchronize(h->last_stream);
    for (int i = 0; i < 2 * h->ev_cap; ++i) cudaEventDestroy(h->ev[i]);
    delete[] h->ev;
    delete[] h->ev_kind;
    h->ev = nullptr;
    h->ev_kind = nullptr;
    h->ev_cap = h->ev_used = 0;
  }
  if (capacity > 0) {
    h->ev = new (std::nothrow) cudaEvent_t[2 * capacity];
    h->ev_kind = new (std::nothrow) int[capacity];
    if (!h->ev || !h->ev_kind) {
      delete[] h->ev;
      delete[] h->ev_kind;
      h->ev = nullptr;
      h->ev_kind = nullptr;
      e = KVA_ERR_NO_MEMORY;
    } else {
      int made = 0;
      for (; made < 2 * capacity; ++made)
        if (cudaEventCreate(&h->ev[made]) != cudaSuccess) break;
      if (made < 2 * capacity) {
        for (int i = 0; i < made; ++i) cudaEventDestroy(h->ev[i]);
        delete[] h->ev;
        delete[] h->ev_kind;
        h->ev = nullptr;
        h->ev_kind = nullptr;
        e = KVA_ERR_CUDA;
      } else {
        h->ev_cap = capacity;
      }
    }
  }
  for (int k = 0; k < KVA_ST_COUNT; ++k) h->launches[k] = 0;
  if (cur != h->device) cudaSetDevice(cur);
  return e;
}

int kva_profile_read(kva_handle* h, kva_profile* out) {
  if (!h || !out) return KVA_ERR_INVALID_ARG;
  int cur = 0;
  cudaGetDevice(&cur);
  if (cur != h->device) cudaSetDevice(h->device);
  int e = cuda_ok(cudaStreamSynchronize(h->last_stream));
  for (int k = 0; k < KVA_ST_COUNT; ++k) {
    out->ms[k] = 0.f;
    out->timed[k] = 0;
    out->launches[k] = h->launches[k];
    h->launches[k] = 0;
  }
  for (int i = 0; i < h->ev_used && !e; ++i) {
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, h->ev[2 * i], h->ev[2 * i + 1]) != cudaSuccess) {
      e = KVA_ERR_CUDA;
      break;
    }
    out->ms[h->ev_kind[i]] += ms;
    out->timed[h->ev_kind[i]] += 1;
  }
  h->ev_used = 0;
  if (cur != h->device) cudaSetDevice(cur);
  return e;
}

void kva_free(kva_handle* h) {
  if (!h) return;
  if (h->ev) kva_profile_enable(h, 0);
  if (h->ws) {
    int cur = 0;
    cudaGetDevice(&cur);
    cudaSetDevice(h->device);
    cudaDeviceSynchronize();
    cudaFree(h->ws);
    cudaSetDevice(cur);
  }
  delete h;
}

int kva_prefill_ubatch(kva_handle* h, const void* residual, int32_t residual_dtype, int32_t T,
                       const kva_weights* w, float* deltanet_state, void* conv_state,
                       const kva_kv_cache* kv, int64_t pos, void* draft_out, void* mixer_out,
                       void* stream) {
  if (!h) return KVA_ERR_INVALID_ARG;
  const kva_dims& d = h->d;
  if (T < 0) return KVA_ERR_INVALID_ARG;
  if (T > d.max_T) return KVA_ERR_TOO_LARGE;
  if (T == 0) return KVA_OK;
  if (!residual ||
      (residual_dtype != KVA_BF16 && residual_dtype != KVA_F32 && residual_dtype != KVA_F16))
    return KVA_ERR_INVALID_ARG;
  if (!a16(residual)) return KVA_ERR_ALIGNMENT;
  int e = check_weights(h, w, true);
  if (e) return e;
  if (h->n_gdn && (!deltanet_state || !conv_state)) return KVA_ERR_INVALID_ARG;
  if ((deltanet_state && !a16(deltanet_state)) || (conv_state && !a16(conv_state)))
    return KVA_ERR_ALIGNMENT;
  if ((e = check_cache(h, kv, 1, &pos, T))) return e;
  if (mixer_out && !a16(mixer_out)) return KVA_ERR_ALIGNMENT;
  if (draft_out && (!a16(draft_out) || d.n_draft_cols == 0)) return KVA_ERR_INVALID_ARG;
  // the plain path splits the heads GEMM's output at n_mix (a multiple of its 32-column
  // epilogue chunks); the fused path writes the drafter tiles on their own
  if (!h->fused && h->n_mix % 32 && draft_out) return KVA_ERR_UNSUPPORTED;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int cur = 0;
  if (cudaGetDevice(&cur) != cudaSuccess) return KVA_ERR_CUDA;
  if (cur != h->device && cudaSetDevice(h->device) != cudaSuccess) return KVA_ERR_CUDA;
  h->last_stream = s;

  const int H = d.hidden, dm = d.d_model, F = d.ffn;
  // quantized projector weights (codes + scales): GemmArgs::wq is the weight format
  const int wq = w->weight_format;
  const bool qw = wq != KVA_W_16;
  const int cd = d.compute_dtype;
  const float eps = d.norm_eps;
  // 1. RMSNorm(residual) (which also clears x) -> Linear{H -> d} into the fp32 residual stream x
  if ((e = staged(h, KVA_ST_RMSNORM, s, [&] {
         return launch_rmsnorm(residual, residual_dtype, H, w->g_in, h->u_in, H, T, H, eps, s, cd,
                               h->x, dm, dm);
       })))
    goto done;
  {
    GemmArgs a;
    a.b_const = true;  // weights
    a.A = h->u_in;
    a.lda = H;
    a.B[0] = w->W_in;
    a.ldb = H;
    a.D = h->x;
    a.ldd = dm;
    a.M = T;
    a.N = dm;
    a.K = H;
    a.epilogue = EPI_ADD_F32;  // into a zeroed x, so the K range can be split
    a.err = h->status;
    a.dtype = cd;
    if (qw) {
      a.wq = wq;
      a.Bs[0] = w->W_in_scale;
    }
    if ((e = staged(h, KVA_ST_GEMM_TRUNK, s, [&] { return launch_gemm(a, s); }))) goto done;
  }
  // 2. the causal transformer blocks (pre-norm, residual adds fused in the GEMM epilogues)
  for (int b = 0; b < d.n_blocks; ++b) {
    const kva_block_weights& B = w->blocks[b];
    if ((e = staged(h, KVA_ST_RMSNORM, s, [&] {
           return launch_rmsnorm(h->x, KVA_F32, dm, B.g_attn, h->u, dm, T, dm, eps, s, cd);
         })))
      goto done;
    GemmArgs q;
    q.b_const = true;  // weights
    q.A = h->u;
    q.lda = dm;
    q.B[0] = B.Wq;
    q.B[1] = B.Wk;
    q.B[2] = B.Wv;
    q.b_mode = B_SEGMENTS;
    q.seg_rows = dm;
    q.ldb = dm;
    q.D = h->qkv;
    q.ldd = 3 * dm;
    q.M = T;
    q.N = 3 * dm;
    q.K = dm;
    q.epilogue = EPI_STORE_BF16;
    q.err = h->status;
    q.dtype = cd;
    if (qw) {
      q.wq = wq;
      for (int i = 0; i < 3; ++i) q.Bs[i] = w->block_scale[b][i];
    }
    if ((e = staged(h, KVA_ST_GEMM_TRUNK, s, [&] { return launch_gemm(q, s); }))) goto done;
    if ((e = staged(h, KVA_ST_ATTENTION, s, [&] {
           return launch_attention(h->qkv, 3 * dm, h->o, dm, T, d.n_heads, d.attn_window, s, cd,
                                   h->status);
         })))
      goto done;
    GemmArgs o;
    o.b_const = true;  // weights
    o.A = h->o;
    o.lda = dm;
    o.B[0] = B.Wo;
    o.ldb = dm;
    o.D = h->x;
    o.ldd = dm;
    o.M = T;
    o.N = dm;
    o.K = dm;
    o.epilogue = EPI_ADD_F32;
    o.err = h->status;
    o.dtype = cd;
    if (qw) {
      o.wq = wq;
      o.Bs[0] = w->block_scale[b][3];
    }
    if ((e = staged(h, KVA_ST_GEMM_TRUNK, s, [&] { return launch_gemm(o, s); }))) goto done;
    if ((e = staged(h, KVA_ST_RMSNORM, s, [&] {
           return launch_rmsnorm(h->x, KVA_F32, dm, B.g_ffn, h->u, dm, T, dm, eps, s, cd);
         })))
      goto done;
    GemmArgs gu;
    gu.b_const = true;  // weights
    gu.A = h->u;
    gu.lda = dm;
    gu.B[0] = B.Wg;
    gu.B[1] = B.Wu;
    gu.b_mode = B_PAIRED;
    gu.ldb = dm;
    gu.D = h->qkv;  // FFN hidden [T, F] reuses the q|k|v buffer region
    gu.ldd = F;
    gu.M = T;
    gu.N = F;
    gu.K = dm;
    gu.epilogue = EPI_SWIGLU_BF16;
    gu.err = h->status;
    gu.dtype = cd;
    if (qw) {
      gu.wq = wq;
      gu.Bs[0] = w->block_scale[b][4];
      gu.Bs[1] = w->block_scale[b][5];
    }
    if ((e = staged(h, KVA_ST_GEMM_TRUNK, s, [&] { return launch_gemm(gu, s); }))) goto done;
    GemmArgs dn;
    dn.b_const = true;  // weights
    dn.A = h->qkv;
    dn.lda = F;
    dn.B[0] = B.Wd;
    dn.ldb = F;
    dn.D = h->x;
    dn.ldd = dm;
    dn.M = T;
    dn.N = dm;
    dn.K = F;
    dn.epilogue = EPI_ADD_F32;
    dn.err = h->status;
    dn.dtype = cd;
    if (qw) {
      dn.wq = wq;
      dn.Bs[0] = w->block_scale[b][6];
    }
    if ((e = staged(h, KVA_ST_GEMM_TRUNK, s, [&] { return launch_gemm(dn, s); }))) goto done;
  }
  // 3. RMSNorm -> all per-layer heads (+ drafter heads) in one wide GEMM
  if ((e = staged(h, KVA_ST_RMSNORM, s, [&] {
         return launch_rmsnorm(h->x, KVA_F32, dm, w->g_out, h->u, dm, T, dm, eps, s, cd);
       })))
    goto done;
  if (h->fused && !qw) {
    // the heads GEMM writes the state updates' inputs directly (no mixer round trip)
    MixParams mp;
    mp.tiles = h->tiles;
    mp.T = T;
    mp.pos = pos;
    mp.n_k = d.gdn_n_k;
    mp.n_v = d.gdn_n_v;
    mp.C = h->C;
    mp.conv_w = w->conv_w;
    mp.A_log = w->A_log;
    mp.dt_bias = w->dt_bias;
    mp.kbuf = h->kbuf;
    mp.vbuf = h->vbuf;
    mp.gbuf = h->gbuf;
    mp.halo = h->halo;
    mp.tail_new = h->tail_new;
    mp.nblk = h->nblk;
    mp.eps = eps;
    mp.n_kv = d.attn_n_kv;
    mp.k_gain = w->k_norm_g;
    mp.rope_dims = d.rope_dims;
    mp.rope_theta = d.rope_theta;
    for (int i = 0; i < 32; ++i) mp.inv_freq[i] = std::pow(d.rope_theta, -2.0 * i / 64);
    if (h->n_attn) mp.cache = *kv;
    mp.draft = draft_out;
    mp.ld_draft = d.n_draft_cols;
    mp.mixer_out = mixer_out;
    mp.ld_mix = h->n_mix;
    if (h->n_attn && kv->dtype == KVA_Q8_0) {  // the rotated q8_0 rows come from the KV writer
      mp.att_raw = h->mixer;
      mp.ld_att_raw = h->n_mix;
    }
    mp.err = h->status;
    const int nt = h->n_tiles + (draft_out ? h->n_tiles_draft : 0);
    if ((e = staged(h, KVA_ST_GEMM_HEADS, s, [&] {
           return launch_heads_fused(cd, h->u, dm, w->W_heads, h->n_mix + d.n_draft_cols, T, dm, nt,
                                     mp, s);
         })))
      goto done;
    e = update_states_impl(h, nullptr, 0, 1, T, &pos, w, deltanet_state, conv_state, kv, nullptr,
                           nullptr, s, &mp);
  } else {
    __nv_bfloat16* mix = mixer_out ? static_cast<__nv_bfloat16*>(mixer_out) : h->mixer;
    GemmArgs hd;
    hd.b_const = true;  // weights
    hd.A = h->u;
    hd.lda = dm;
    hd.B[0] = w->W_heads;
    hd.ldb = dm;
    hd.D = mix;
    hd.ldd = h->n_mix;
    hd.M = T;
    hd.N = static_cast<int>(h->n_mix + (draft_out ? d.n_draft_cols : 0));
    hd.K = dm;
    hd.epilogue = EPI_STORE_BF16;
    if (draft_out) {
      hd.D1 = draft_out;
      hd.ldd1 = d.n_draft_cols;
      hd.n_split = h->n_mix;
    }
    hd.err = h->status;
    hd.dtype = cd;
    if (qw) {  // the mixer rows; the drafter rows follow as a GEMM of their own
      hd.wq = wq;
      hd.Bs[0] = w->W_heads_scale;
      hd.lds = h->n_mix + d.n_draft_cols;
      hd.N = static_cast<int>(h->n_mix);
      hd.D1 = nullptr;
      hd.n_split = 0;
    }
    if ((e = staged(h, KVA_ST_GEMM_HEADS, s, [&] { return launch_gemm(hd, s); }))) goto done;
    if (qw && draft_out) {
      GemmArgs dr = hd;
      dr.B[0] = static_cast<const uint8_t*>(w->W_heads) +
                h->n_mix * static_cast<int64_t>(wq == KVA_W_Q4_0 ? dm / 2 : dm);
      dr.Bs[0] = static_cast<const __half*>(w->W_heads_scale) + h->n_mix;
      dr.D = draft_out;
      dr.ldd = d.n_draft_cols;
      dr.N = d.n_draft_cols;
      if ((e = staged(h, KVA_ST_GEMM_HEADS, s, [&] { return launch_gemm(dr, s); }))) goto done;
    }
    // 4. state updates on the mixer inputs
    e = update_states_impl(h, mix, h->n_mix, 1, T, &pos, w, deltanet_state, conv_state, kv,
                           nullptr, nullptr, s);
  }
  if (!e) h->tokens += T;
done:
  if (cur != h->device) cudaSetDevice(cur);
  return e;
}

int kva_update_states(kva_handle* h, const void* mixer_in, int64_t mixer_ld, int32_t n_seq,
                      int32_t T, const int64_t* pos, const kva_weights* w, float* state,
                      void* conv_state, const kva_kv_cache* kv, void* debug_qkv, void* debug_gb,
                      void* stream) {
  if (!h) return KVA_ERR_INVALID_ARG;
  const kva_dims& d = h->d;
  if (T < 0 || n_seq < 0) return KVA_ERR_INVALID_ARG;
  if (T > d.max_T || n_seq > d.max_seq) return KVA_ERR_TOO_LARGE;
  if (T == 0 || n_seq == 0) return KVA_OK;
  if (!mixer_in || !pos || mixer_ld < h->n_mix) return KVA_ERR_INVALID_ARG;
  if (!a16(mixer_in) || mixer_ld % 8) return KVA_ERR_ALIGNMENT;
  int e = check_weights(h, w, false);
  if (e) return e;
  if (h->n_gdn && (!state || !conv_state)) return KVA_ERR_INVALID_ARG;
  if ((state && !a16(state)) || (conv_state && !a16(conv_state))) return KVA_ERR_ALIGNMENT;
  if ((e = check_cache(h, kv, n_seq, pos, T))) return e;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int cur = 0;
  if (cudaGetDevice(&cur) != cudaSuccess) return KVA_ERR_CUDA;
  if (cur != h->device && cudaSetDevice(h->device) != cudaSuccess) return KVA_ERR_CUDA;
  h->last_stream = s;
  e = update_states_impl(h, mixer_in, mixer_ld, n_seq, T, pos, w, state, conv_state, kv, debug_qkv,
                         debug_gb, s);
  if (!e) h->tokens += (int64_t)n_seq * T;
  if (cur != h->device) cudaSetDevice(cur);
  return e;
}

int kva_last_token_layer(kva_handle* h, int32_t layer, int32_t n_seq, const void* x, int64_t x_ld,
                         const int64_t* pos, const kva_weights* w, const kva_last_params* lp,
                         float* state, void* conv_state, const kva_kv_cache* kv, void* out,
                         int32_t out_dtype, int64_t out_ld, void* stream) {
  if (!h || !w || !lp) return KVA_ERR_INVALID_ARG;
  const kva_dims& d = h->d;
  if (layer < 0 || layer >= d.n_late || n_seq < 0) return KVA_ERR_INVALID_ARG;
  if (n_seq > d.max_seq) return KVA_ERR_TOO_LARGE;
  if (n_seq == 0) return KVA_OK;
  if (!x || !pos || !out) return KVA_ERR_INVALID_ARG;
  if (out_dtype != KVA_F32 && out_dtype != d.compute_dtype) return KVA_ERR_INVALID_ARG;
  if (!a16(x) || x_ld % 8 || !a16(out) || out_ld % 4) return KVA_ERR_ALIGNMENT;
  for (int i = 0; i < n_seq; ++i)
    if (pos[i] < 0) return KVA_ERR_INVALID_ARG;
  const bool gdn = d.layer_type[layer] == KVA_LAYER_GDN;
  int li = 0;  // index among the layers of this type
  for (int i = 0; i < layer; ++i) li += d.layer_type[i] == d.layer_type[layer];
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int cur = 0;
  if (cudaGetDevice(&cur) != cudaSuccess) return KVA_ERR_CUDA;
  if (cur != h->device && cudaSetDevice(h->device) != cudaSuccess) return KVA_ERR_CUDA;
  int e = KVA_OK;
  if (gdn) {
    const int nvdv = d.gdn_n_v * d.gdn_d_v;
    if (x_ld < h->gdn_width + nvdv || out_ld < nvdv) e = KVA_ERR_INVALID_ARG;
    else if (!w->conv_w || !w->A_log || !w->dt_bias || !lp->gdn_norm_w || !state || !conv_state)
      e = KVA_ERR_INVALID_ARG;
    else if (!a16(w->conv_w) || !a16(state) || !a16(conv_state)) e = KVA_ERR_ALIGNMENT;
    if (!e) {
      GdnDecodeLaunch g;
      g.x = x;
      g.x_ld = x_ld;
      g.x_dtype = d.compute_dtype;
      g.n_seq = n_seq;
      g.n_k = d.gdn_n_k;
      g.n_v = d.gdn_n_v;
      g.d = d.gdn_d_k;
      g.C = h->C;
      g.conv_w = w->conv_w + (int64_t)li * h->C * 4;
      g.A_log = w->A_log + (int64_t)li * d.gdn_n_v;
      g.dt_bias = w->dt_bias + (int64_t)li * d.gdn_n_v;
      g.norm_w = lp->gdn_norm_w + (int64_t)li * d.gdn_d_v;
      const int64_t sstate = (int64_t)d.gdn_n_v * d.gdn_d_v * d.gdn_d_k;
      g.state = state + (int64_t)li * sstate;
      g.state_seq_stride = (int64_t)h->n_gdn * sstate;
      g.conv_state = static_cast<uint16_t*>(conv_state) + (int64_t)li * 3 * h->C;
      g.conv_seq_stride = (int64_t)h->n_gdn * 3 * h->C;
      g.out = out;
      g.out_ld = out_ld;
      g.out_dtype = out_dtype;
      g.eps = d.norm_eps;
      h->last_stream = s;
      e = staged(h, KVA_ST_LAST_TOKEN, s, [&] { return launch_gdn_decode(g, s); });
    }
  } else {
    const int n_q = lp->attn_n_q, dh = d.attn_d_h;
    if (n_q <= 0 || n_q % d.attn_n_kv || n_q / d.attn_n_kv > kDecodeMaxGroup) e = KVA_ERR_UNSUPPORTED;
    else if (x_ld < h->attn_width + 2LL * n_q * dh || out_ld < (int64_t)n_q * dh) e = KVA_ERR_INVALID_ARG;
    else if (!w->k_norm_g || !lp->q_norm_g) e = KVA_ERR_INVALID_ARG;
    else if (!(e = check_cache(h, kv, n_seq, pos, 1)) && kv->dtype != KVA_BF16 && kv->dtype != KVA_F16)
      e = KVA_ERR_UNSUPPORTED;
    if (!e && (int64_t)n_seq * d.attn_n_kv > kDecodeSlots) e = KVA_ERR_UNSUPPORTED;
    if (!e) {
      AttnDecodeLaunch a;
      a.x = x;
      a.x_ld = x_ld;
      a.x_dtype = d.compute_dtype;
      a.n_seq = n_seq;
      a.n_kv = d.attn_n_kv;
      a.n_q = n_q;
      a.G = n_q / d.attn_n_kv;
      a.d_h = dh;
      a.rope_dims = d.rope_dims;
      for (int i = 0; i < d.rope_dims / 2 && i < 128; ++i)
        a.inv_freq[i] = std::pow(d.rope_theta, -2.0 * i / d.rope_dims);
      a.k_gain = w->k_norm_g + (int64_t)li * dh;
      a.q_gain = lp->q_norm_g + (int64_t)li * dh;
      int64_t max_rows = 0;
      for (int i = 0; i < n_seq; ++i) {
        a.pos[i] = pos[i];
        if (pos[i] + 1 > max_rows) max_rows = pos[i] + 1;
      }
      a.kc = kv->k[li];
      a.vc = kv->v[li];
      a.layout = kv->layout;
      a.max_pos = kv->max_pos;
      a.page_size = kv->page_size;
      a.n_pages = kv->n_pages;
      a.pages_per_seq = kv->pages_per_seq;
      a.page_table = kv->page_table;
      a.cache_dtype = kv->dtype;
      const int slots_per = kDecodeSlots / (n_seq * d.attn_n_kv);
      a.n_split = attn_decode_splits(n_seq, d.attn_n_kv, max_rows, num_sms(), &a.rows_per_split);
      if (a.n_split > slots_per) {  // fewer, longer splits so the partials fit the workspace
        const int64_t tiles = (max_rows + 63) / 64;
        a.rows_per_split = (tiles + slots_per - 1) / slots_per * 64;
        a.n_split = (int)((max_rows + a.rows_per_split - 1) / a.rows_per_split);
      }
      a.part = h->dec_part;
      a.out = out;
      a.out_ld = out_ld;
      a.out_dtype = out_dtype;
      a.eps = d.norm_eps;
      a.err = h->status;
      h->last_stream = s;
      e = staged(h, KVA_ST_LAST_TOKEN, s, [&] { return launch_attn_decode(a, s); });
      if (!e) ++h->launches[KVA_ST_LAST_TOKEN];  // two kernels
    }
  }
  if (cur != h->device) cudaSetDevice(cur);
  return e;
}

int kva_get_device_status(kva_handle* h, int32_t* status) {
  if (!h || !status) return KVA_ERR_INVALID_ARG;
  int cur = 0;
  cudaGetDevice(&cur);
  if (cur != h->device) cudaSetDevice(h->device);
  int v = 0;
  int e = cuda_ok(cudaStreamSynchronize(h->last_stream));
  if (!e) e = cuda_ok(cudaMemcpy(&v, h->status, sizeof(int), cudaMemcpyDeviceToHost));
  if (!e) e = cuda_ok(cudaMemset(h->status, 0, sizeof(int)));
  if (!e) e = cuda_ok(cudaDeviceSynchronize());
  if (cur != h->device) cudaSetDevice(cur);
  *status = v;
  if (e) return e;
  return v ? KVA_ERR_DEVICE : KVA_OK;
}

int kva_stats(kva_handle* h, int64_t* tokens_approximated) {
  if (!h || !tokens_approximated) return KVA_ERR_INVALID_ARG;
  *tokens_approximated = h->tokens;
  return KVA_OK;
}

int kva_heads_fused(kva_handle* h, int32_t* fused) {
  if (!h || !fused) return KVA_ERR_INVALID_ARG;
  *fused = h->fused ? 1 : 0;
  return KVA_OK;
}

const char* kva_strerror(int32_t status) {
  switch (status) {
    case KVA_OK: return "ok";
    case KVA_ERR_INVALID_ARG: return "invalid argument";
    case KVA_ERR_UNSUPPORTED: return "dimensions not supported by the kernels";
    case KVA_ERR_TOO_LARGE: return "size beyond the handle's or cache's capacity";
    case KVA_ERR_ALIGNMENT: return "pointer or leading dimension not 16-byte aligned";
    case KVA_ERR_CUDA: return "CUDA runtime or launch error";
    case KVA_ERR_NO_MEMORY: return "device workspace allocation failed";
    case KVA_ERR_DEVICE: return "device reported an error (see device status bits)";
    default: return "unknown status";
  }
}

// ------------------------------------------------------------ per-step ops
int kva_op_rmsnorm(const void* x, int32_t x_dtype, int64_t ldx, const float* g, void* out,
                   int32_t out_dtype, int64_t ldo, int32_t rows, int32_t n, float eps,
                   void* stream) {
  return launch_rmsnorm(x, x_dtype, ldx, g, out, ldo, rows, n, eps,
                        static_cast<cudaStream_t>(stream), out_dtype);
}

int kva_op_gemm(int32_t dtype, const void* A, int64_t lda, const void* const* B, int32_t b_mode,
                int64_t ldb, int64_t seg_rows, void* D, int64_t ldd, void* D1, int64_t ldd1,
                int64_t n_split, int32_t M, int32_t N, int32_t K, int32_t epilogue,
                int32_t block_n, int32_t* err, void* stream) {
  if (!B) return KVA_ERR_INVALID_ARG;
  if (b_mode < KVA_B_SINGLE || b_mode > KVA_B_PAIRED) return KVA_ERR_INVALID_ARG;
  GemmArgs a;
  a.A = A;
  a.lda = lda;
  const int nb = b_mode == KVA_B_SINGLE ? 1 : (b_mode == KVA_B_PAIRED ? 2 : 3);
  for (int i = 0; i < nb; ++i) a.B[i] = B[i];
  a.b_mode = b_mode;
  a.ldb = ldb;
  a.seg_rows = seg_rows;
  a.D = D;
  a.ldd = ldd;
  a.D1 = D1;
  a.ldd1 = ldd1;
  a.n_split = n_split;
  a.M = M;
  a.N = N;
  a.K = K;
  a.epilogue = epilogue;
  a.block_n = block_n;
  a.err = err;
  a.dtype = dtype;
  if (M < 0 || N < 0 || K < 0) return KVA_ERR_INVALID_ARG;
  return launch_gemm(a, static_cast<cudaStream_t>(stream));
}

int kva_test_gemm_wait_timeout(int32_t dtype, const void* A, const void* B, void* D, int32_t M,
                               int32_t N, int32_t K, int32_t* err, void* stream) {
  if (!A || !B || !D || !err) return KVA_ERR_INVALID_ARG;
  if (M <= 0 || N <= 0 || K <= 0) return KVA_ERR_INVALID_ARG;
  GemmArgs a;
  a.A = A;
  a.lda = K;
  a.B[0] = B;
  a.b_mode = KVA_B_SINGLE;
  a.ldb = K;
  a.D = D;
  a.ldd = N;
  a.M = M;
  a.N = N;
  a.K = K;
  a.epilogue = KVA_EPI_STORE_BF16;
  a.block_n = 512;  // the CTA-pair kernel
  a.err = err;
  a.dtype = dtype;
  a.stall_item1 = 1;  // the first work item
  return launch_gemm(a, static_cast<cudaStream_t>(stream));
}

static int op_gemm_quant(int wq, int32_t dtype, const void* A, int64_t lda, const void* const* Bq,
                         const void* const* Bs, int32_t b_mode, int64_t seg_rows, void* D, int64_t ldd,
                         int32_t M, int32_t N, int32_t K, int32_t epilogue, int32_t* err, void* stream) {
  if (!Bq || !Bs) return KVA_ERR_INVALID_ARG;
  if (b_mode < KVA_B_SINGLE || b_mode > KVA_B_PAIRED) return KVA_ERR_INVALID_ARG;
  GemmArgs a;
  a.A = A;
  a.lda = lda;
  const int nb = b_mode == KVA_B_SINGLE ? 1 : (b_mode == KVA_B_PAIRED ? 2 : 3);
  for (int i = 0; i < nb; ++i) {
    a.B[i] = Bq[i];
    a.Bs[i] = Bs[i];
  }
  a.wq = wq;
  a.b_mode = b_mode;
  a.ldb = K;
  a.seg_rows = seg_rows;
  a.D = D;
  a.ldd = ldd;
  a.M = M;
  a.N = N;
  a.K = K;
  a.epilogue = epilogue;
  a.block_n = 512;
  a.err = err;
  a.dtype = dtype;
  if (M < 0 || N < 0 || K < 0) return KVA_ERR_INVALID_ARG;
  return launch_gemm(a, static_cast<cudaStream_t>(stream));
}

int kva_op_gemm_q8_0(int32_t dtype, const void* A, int64_t lda, const void* const* Bq,
                     const void* const* Bs, int32_t b_mode, int64_t seg_rows, void* D, int64_t ldd,
                     int32_t M, int32_t N, int32_t K, int32_t epilogue, int32_t* err, void* stream) {
  return op_gemm_quant(KVA_W_Q8_0, dtype, A, lda, Bq, Bs, b_mode, seg_rows, D, ldd, M, N, K, epilogue,
                       err, stream);
}

int kva_op_gemm_q4_0(int32_t dtype, const void* A, int64_t lda, const void* const* Bq,
                     const void* const* Bs, int32_t b_mode, int64_t seg_rows, void* D, int64_t ldd,
                     int32_t M, int32_t N, int32_t K, int32_t epilogue, int32_t* err, void* stream) {
  return op_gemm_quant(KVA_W_Q4_0, dtype, A, lda, Bq, Bs, b_mode, seg_rows, D, ldd, M, N, K, epilogue,
                       err, stream);
}

int kva_op_attention(int32_t dtype, const void* qkv, int64_t ldq, void* out, int64_t ldo,
                     int32_t T, int32_t n_heads, int32_t window, void* stream) {
  return launch_attention(qkv, ldq, out, ldo, T, n_heads, window,
                          static_cast<cudaStream_t>(stream), dtype);
}

int kva_op_gdn_scan(const void* k, const void* v, const float* gb, float* state, int32_t n_seq,
                    int32_t n_layers, int32_t T, int32_t n_k, int32_t n_v, int32_t d,
                    void* stream) {
  if (!k || !v || !gb || !state || n_seq < 0 || n_layers < 0 || T < 0 || n_k <= 0 || n_v <= 0)
    return KVA_ERR_INVALID_ARG;
  if (n_layers > KVA_MAX_LATE) return KVA_ERR_UNSUPPORTED;
  if (!a16(k) || !a16(v) || !a16(gb) || !a16(state)) return KVA_ERR_ALIGNMENT;
  GdnLaunch g;
  g.n_seq = n_seq;
  g.n_gdn = n_layers;
  g.T = T;
  g.n_k = n_k;
  g.n_v = n_v;
  g.d_k = g.d_v = d;
  g.C = 2 * n_k * d + n_v * d;
  g.kbuf = const_cast<void*>(k);
  g.vbuf = const_cast<void*>(v);
  g.gbuf = const_cast<float*>(gb);
  g.state = state;
  // fields the scan does not read, set so the shared argument check passes
  g.mix = k;
  g.conv_state = const_cast<void*>(k);
  g.conv_w = gb;
  g.A_log = gb;
  g.dt_bias = gb;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the 128-dimensional scan stages B1 and the chunk scalars in stream-ordered scratch
  void* chunk = nullptr;
  if (d == 128 && T > 0 && n_seq > 0 && n_layers > 0) {
    if (cudaMallocAsync(&chunk, gdn_chunk_bytes(n_seq, n_layers, n_v, T), st) != cudaSuccess)
      return KVA_ERR_NO_MEMORY;
    gdn_chunk_split(chunk, n_seq, n_layers, n_v, T, &g.b1buf, &g.scbuf);
  }
  const int e = launch_gdn_scan(g, st);
  if (chunk && cudaFreeAsync(chunk, st) != cudaSuccess) return KVA_ERR_CUDA;
  return e;
}

}  // extern "C"
