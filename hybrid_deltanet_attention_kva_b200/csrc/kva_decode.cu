// Exact last-token pass: one token of each sequence through one late layer's token mixer
// ("Qwen3.8-27B-KVA" model card, "What the hell?": after the cheap state updates the engine
// runs the last token of each ubatch through the late layers exactly, on top of the
// approximated context).  The layer's exact inputs for the token come from the caller (the
// base model's projections of the previous layer's output); this file turns them into the
// mixer output and updates the layer's state or cache with the token.
//
// Gated-DeltaNet layer (one CTA of 4 warps per (value head, sequence)):
//   conv over the carried 3-row tail + SiLU on the head's q, k and v channels, L2 norms,
//   g = -exp(A_log) softplus(a + dt_bias), beta = sigmoid(b), then per state row v
//       S[v,:] <- e^g S[v,:] + beta (v_v - e^g S[v,:].k) k,   o_v = S[v,:].q
//   (the delta rule of one token), each row read and written once as 512-byte warp
//   vectors (all of a warp's rows in flight before the first is used); then the gated
//   RMSNorm o = RMSNorm(o) * w * silu(z).  The value heads of one key head form a cluster:
//   each block shifts its own value channels of the conv tail once it has read them, and
//   block 0 shifts the shared q and k channels after the cluster barrier.
// Full-attention layer (split-K flash decoding):
//   every CTA forms the token's k (RMSNorm + RoPE) and its query group (the n_q / n_kv
//   query heads that read one KV head, RMSNorm + RoPE) in shared memory; split 0 writes
//   the token's K and V rows to the cache.  Each CTA streams its range of the sequence's
//   cache rows through a 3-stage cp.async ring (64 rows, 16-byte chunks XOR-swizzled by
//   row so ldmatrix is conflict free; paged rows through the page table, rows past the
//   range zero-filled) and runs S^T = Q K^T and O^T += V^T P^T on mma.sync: the query
//   group is the M side of the first product (padded to 16), so the score fragments are
//   already the B fragments of the second.  Online softmax in the exp2 domain; the four
//   warps' partial states merge in shared memory, the splits in a combine kernel that
//   also applies the output gate sigmoid(gate).
#include <type_traits>

#include "kva_common.cuh"

namespace kva {
namespace {

constexpr int DEC_TILE = 64;   // cache rows per tile (16 per warp)
constexpr int DEC_STAGES = 3;
constexpr int DEC_THREADS = 128;

// byte offset of 16-bit element (row, col) in a [rows][D] tile whose 16-byte chunks are
// XOR-swizzled by the row's low 3 bits
template <int D>
__device__ __forceinline__ uint32_t dsw(int row, int col) {
  return static_cast<uint32_t>(row * D * 2 + ((((col >> 3) ^ (row & 7)) << 4) | ((col & 7) * 2)));
}

// byte offset of (row, col) in a K or V tile of 64 rows: with TMA, D / 64 boxes of
// [64 rows][64 dims] in the 128-byte swizzle the copy engine writes; with cp.async, rows of
// D values whose 16-byte chunks are XOR-swizzled by the row (dsw)
template <int D, bool TMA>
__device__ __forceinline__ uint32_t toff(int row, int col) {
  if constexpr (TMA)
    return static_cast<uint32_t>((col >> 6) * 8192 + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4) +
                                 (col & 7) * 2);
  else
    return dsw<D>(row, col);
}

// RoPE on this lane's EPL consecutive dims (dims lane * EPL + i): pairs (i, i + half)
// meet through one xor shuffle; the angle pos * inv_freq is formed and range-reduced in
// fp64 (exact at long positions), then sincosf.
template <int EPL>
__device__ __forceinline__ void rope_lane(float (&v)[EPL], int lane, int64_t pos, const double* inv_freq,
                                          int rope_dims) {
  const int half = rope_dims / 2;
  if (half == 0) return;
  const int off = half / EPL;
  const int dim0 = lane * EPL;
  float partner[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) partner[i] = __shfl_xor_sync(0xffffffffu, v[i], off);
  if (dim0 < rope_dims) {
    const double two_pi = 6.283185307179586476925286766559;
    const double inv_two_pi = 0.15915494309189533576888376337251;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int d = dim0 + i;
      const int pi = d < half ? d : d - half;
      const double ang = static_cast<double>(pos) * inv_freq[pi];
      const double q = rint(ang * inv_two_pi);
      const float red = static_cast<float>(fma(-q, two_pi, ang));
      float sn, cs;
      sincosf(red, &sn, &cs);
      v[i] = d < half ? v[i] * cs - partner[i] * sn : v[i] * cs + partner[i] * sn;
    }
  }
}

template <typename T>
__device__ __forceinline__ float to_f(T x) {
  if constexpr (std::is_same<T, float>::value) return x;
  else return F16<T>::to(x);
}
template <typename T>
__device__ __forceinline__ T from_f(float x) {
  if constexpr (std::is_same<T, float>::value) return x;
  else return F16<T>::from(x);
}

// ============================================================================
// gated-DeltaNet layer
// ============================================================================
template <int D, typename TX, typename TO>
__global__ void __launch_bounds__(256) gdn_decode_kernel(const GdnDecodeLaunch p) {
  constexpr int EPL = D / 32;
  constexpr int NW = 8;
  constexpr int RPW = D / NW;  // state rows per warp, all loaded before any is used
  using V = typename std::conditional<EPL == 4, float4, float2>::type;
  __shared__ float qv[D], kv[D], vv[D], zz[D], ov[D];
  __shared__ float sc[4];
  griddep_wait_and_release();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x, s = blockIdx.y;
  const int n_k = p.n_k, n_v = p.n_v, C = p.C;
  const int kh = h / (n_v / n_k);
  const TX* x = static_cast<const TX*>(p.x) + s * p.x_ld;
  TX* tail = static_cast<TX*>(p.conv_state) + s * p.conv_seq_stride;  // [3][C]
  const float4* w4 = reinterpret_cast<const float4*>(p.conv_w);
  float* S = p.state + s * p.state_seq_stride + static_cast<int64_t>(h) * D * D;

  // this warp's state rows start streaming in before anything else
  V rows[RPW];
#pragma unroll
  for (int j = 0; j < RPW; ++j) rows[j] = reinterpret_cast<const V*>(S + (warp * RPW + j) * D)[lane];

  // causal conv over [tail; x] (tap 3 = this token) + SiLU on the head's q, k, v channels.
  // Thread t takes channel t of [q | k] and, for t < D, channel t of v; the raw values it
  // reads are also the new conv tail [rows 1, 2; x] of those channels, written below.
  TX qk_keep[3], v_keep[3];
  int qk_ch = -1, v_ch = -1;
#pragma unroll
  for (int pass = 0; pass < 2; ++pass) {
    const int c = tid + pass * 256;
    if (c >= 3 * D) break;
    const int part = c / D, i = c - part * D;
    const int ch = part == 0 ? kh * D + i : part == 1 ? n_k * D + kh * D + i : 2 * n_k * D + h * D + i;
    const float4 w = w4[ch];
    const TX t0 = tail[ch], t1 = tail[C + ch], t2 = tail[2 * C + ch], xc = x[ch];
    const float a = w.x * to_f(t0) + w.y * to_f(t1) + w.z * to_f(t2) + w.w * to_f(xc);
    const float act = a / (1.f + expf(-a));
    (part == 0 ? qv : part == 1 ? kv : vv)[i] = act;
    if (part == 2) {
      v_ch = ch;
      v_keep[0] = t1, v_keep[1] = t2, v_keep[2] = xc;
    } else {
      qk_ch = ch;
      qk_keep[0] = t1, qk_keep[1] = t2, qk_keep[2] = xc;
    }
  }
  for (int i = tid; i < D; i += 256) zz[i] = to_f(x[C + 2 * n_v + h * D + i]);
  if (tid == 0) {
    const float a = to_f(x[C + h]) + p.dt_bias[h];
    const float b = to_f(x[C + n_v + h]);
    const float sp = a > 20.f ? a : log1pf(expf(a));
    sc[0] = expf(-expf(p.A_log[h]) * sp);  // e^g
    sc[1] = 1.f / (1.f + expf(-b));        // beta
  }
  // the new conv tail: this head's value channels (read by this block only) at once; the key
  // head's q and k channels, which the cluster's other blocks read too, by block 0 of the
  // cluster after the cluster barrier
  if (v_ch >= 0) {
    tail[v_ch] = v_keep[0];
    tail[C + v_ch] = v_keep[1];
    tail[2 * C + v_ch] = v_keep[2];
  }
  __syncthreads();
  cluster_sync();
  if (cluster_ctarank() == 0 && qk_ch >= 0) {
    tail[qk_ch] = qk_keep[0];
    tail[C + qk_ch] = qk_keep[1];
    tail[2 * C + qk_ch] = qk_keep[2];
  }
  if (warp < 2) {  // L2 norms of q (warp 0) and k (warp 1)
    float* arr = warp == 0 ? qv : kv;
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < EPL; ++i) ss += arr[lane + 32 * i] * arr[lane + 32 * i];
    ss = warp_sum(ss);
    const float r = rsqrtf(ss + p.eps);
#pragma unroll
    for (int i = 0; i < EPL; ++i) arr[lane + 32 * i] *= r;
  }
  __syncthreads();

  // the one-token delta rule on this lane's EPL consecutive columns of each row
  float kr[EPL], qr[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    kr[i] = kv[lane * EPL + i];
    qr[i] = qv[lane * EPL + i];
  }
  const float eg = sc[0], beta = sc[1];
#pragma unroll
  for (int j = 0; j < RPW; ++j) {
    const int r = warp * RPW + j;
    float* e = reinterpret_cast<float*>(&rows[j]);
    float sk = 0.f;
#pragma unroll
    for (int i = 0; i < EPL; ++i) sk += e[i] * kr[i];
    sk = warp_sum(sk);
    const float coef = beta * (vv[r] - eg * sk);
    float o = 0.f;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      e[i] = eg * e[i] + coef * kr[i];
      o += e[i] * qr[i];
    }
    o = warp_sum(o);
    reinterpret_cast<V*>(S + r * D)[lane] = rows[j];
    if (lane == 0) ov[r] = o;
  }
  __syncthreads();
  if (warp == 0) {
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < EPL; ++i) ss += ov[lane + 32 * i] * ov[lane + 32 * i];
    ss = warp_sum(ss);
    if (lane == 0) sc[2] = rsqrtf(ss / static_cast<float>(D) + p.eps);
  }
  __syncthreads();
  TO* out = static_cast<TO*>(p.out) + s * p.out_ld + h * D;
  const float rr = sc[2];
  for (int i = tid; i < D; i += 256) {
    const float z = zz[i];
    out[i] = from_f<TO>(ov[i] * rr * p.norm_w[i] * (z / (1.f + expf(-z))));
  }
}

// ============================================================================
// full-attention layer
// ============================================================================
template <int D>
struct DecSmem {
  static constexpr int TILE_BYTES = DEC_TILE * D * 2;
  static constexpr int K = 0;                                     // [stage] K tiles
  static constexpr int V = K + DEC_STAGES * TILE_BYTES;          // [stage] V tiles
  static constexpr int Q = V + DEC_STAGES * TILE_BYTES;          // [16][D] query group
  static constexpr int KN = Q + 16 * D * 2;                      // the token's k row
  static constexpr int VN = KN + D * 2;                          // and v row
  static constexpr int BAR = VN + D * 2;                         // [stage] tile landed (TMA path)
  static constexpr int MISC = BAR + DEC_STAGES * 8;              // abort flag
  static constexpr int BYTES = MISC + 16;
  static constexpr int ALLOC = BYTES + 1024;                     // slack for 1024-byte alignment
  // after the row loop, per warp: m[8], l[8], O[8][D] fp32 (inside the K tiles)
  static constexpr int MERGE_WARP = (16 + 8 * D) * 4;
  static_assert(4 * MERGE_WARP <= DEC_STAGES * TILE_BYTES, "merge area fits the tiles");
};

// element offset of cache row j of (sequence s, KV head kvh) in the K and the V array (the
// same for both), or -1 for a page-table entry out of range (which sets the device status word)
__device__ __forceinline__ int64_t dec_row(const AttnDecodeLaunch& p, int s, int kvh, int64_t j) {
  if (p.layout == KVA_KV_PAGED) {
    const int64_t pi = j / p.page_size;
    const int page = pi < p.pages_per_seq ? p.page_table[static_cast<int64_t>(s) * p.pages_per_seq + pi] : -1;
    if (page < 0 || page >= p.n_pages) {
      set_device_error(p.err, KVA_DEV_PAGE_OOB);
      return -1;
    }
    return ((static_cast<int64_t>(page) * p.n_kv + kvh) * p.page_size + j % p.page_size) * p.d_h;
  }
  return ((static_cast<int64_t>(s) * p.n_kv + kvh) * p.max_pos + j) * p.d_h;
}

template <int D, typename TX, typename TC, bool TMA>
__global__ void __launch_bounds__(DEC_THREADS) attn_decode_kernel(const __grid_constant__ CUtensorMap mKc,
                                                                  const __grid_constant__ CUtensorMap mVc,
                                                                  const AttnDecodeLaunch p) {
  using L = DecSmem<D>;
  constexpr int EPL = D / 32;
  constexpr int CH = D / 8;  // 16-byte chunks per row
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* dsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, kvh = blockIdx.y, s = blockIdx.z;
  const int G = p.G;
  const int64_t pos = p.pos[s];
  const int64_t rows = pos + 1;  // cache rows 0..pos (pos is this token)
  const int64_t r_begin = static_cast<int64_t>(split) * p.rows_per_split;
  const int64_t r_end = r_begin + p.rows_per_split < rows ? r_begin + p.rows_per_split : rows;
  const uint32_t sbase = smem_u32(dsm);
  TC* qsm = reinterpret_cast<TC*>(dsm + L::Q);
  TC* knew = reinterpret_cast<TC*>(dsm + L::KN);
  TC* vnew = reinterpret_cast<TC*>(dsm + L::VN);
  uint64_t* full = reinterpret_cast<uint64_t*>(dsm + L::BAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(dsm + L::MISC);
  if (TMA && tid == 0) {
    for (int i = 0; i < DEC_STAGES; ++i) mbar_init(&full[i], 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&mKc);
    tma_prefetch_desc(&mVc);
  }
  griddep_wait_and_release();

  // ---- the row ring: rows r_begin .. r_end - 1 in 64-row tiles; the first tiles are
  // requested before anything else, this token's own row goes in from shared memory later
  const int64_t n_rows = r_end > r_begin ? r_end - r_begin : 0;
  const int n_tiles = static_cast<int>((n_rows + DEC_TILE - 1) / DEC_TILE);
  int issued = 0, last_ok = -1;  // thread 0 (TMA path): tiles requested, last tile seen landed
  auto issue = [&](int t) {
    const int st = t % DEC_STAGES;
    const uint32_t kb = sbase + L::K + st * L::TILE_BYTES, vb = sbase + L::V + st * L::TILE_BYTES;
    const int64_t j0 = r_begin + static_cast<int64_t>(t) * DEC_TILE;
    if constexpr (TMA) {  // thread 0: the tile's D / 64 boxes of K and of V
      int64_t y = j0, z = static_cast<int64_t>(s) * p.n_kv + kvh;
      if (p.layout == KVA_KV_PAGED) {  // a tile lies inside one page (page_size % 64 == 0)
        const int64_t pi = j0 / p.page_size;
        int page = pi < p.pages_per_seq ? p.page_table[static_cast<int64_t>(s) * p.pages_per_seq + pi] : -1;
        if (page < 0 || page >= p.n_pages) {
          set_device_error(p.err, KVA_DEV_PAGE_OOB);
          page = 0;  // read a valid page; the result is flagged
        }
        y = j0 % p.page_size;
        z = static_cast<int64_t>(page) * p.n_kv + kvh;
      }
      mbar_arrive_expect_tx(&full[st], 2 * L::TILE_BYTES);
#pragma unroll
      for (int q = 0; q < D / 64; ++q) {
        tma_load_3d(dsm + L::K + st * L::TILE_BYTES + q * 8192, &mKc, &full[st], 64 * q,
                    static_cast<int>(y), static_cast<int>(z), l2_policy_evict_first());
        tma_load_3d(dsm + L::V + st * L::TILE_BYTES + q * 8192, &mVc, &full[st], 64 * q,
                    static_cast<int>(y), static_cast<int>(z), l2_policy_evict_first());
      }
      issued = t + 1;
    } else {
      const int c = tid % CH;
      for (int r = tid / CH; r < DEC_TILE; r += DEC_THREADS / CH) {
        const int64_t j = j0 + r;
        if (j == pos) continue;
        const uint32_t off = dsw<D>(r, 8 * c);
        const int64_t o = j < r_end ? dec_row(p, s, kvh, j) : -1;
        cp_async16(kb + off, static_cast<const TC*>(p.kc) + (o >= 0 ? o + 8 * c : 0), o >= 0 ? 16u : 0u);
        cp_async16(vb + off, static_cast<const TC*>(p.vc) + (o >= 0 ? o + 8 * c : 0), o >= 0 ? 16u : 0u);
      }
    }
  };
  // this token's own row from shared memory; with TMA also zero V rows past the split's end
  // (the copy engine read whatever the cache holds there, and 0 x NaN would poison the sum)
  auto put_pos = [&](int t) {
    const int st = t % DEC_STAGES;
    const int64_t j0 = r_begin + static_cast<int64_t>(t) * DEC_TILE;
    const int64_t r = pos - j0;
    if (r >= 0 && r < DEC_TILE)
      for (int c = tid; c < CH; c += DEC_THREADS) {
        const uint32_t off = toff<D, TMA>(static_cast<int>(r), 8 * c);
        *reinterpret_cast<uint4*>(dsm + L::K + st * L::TILE_BYTES + off) = reinterpret_cast<const uint4*>(knew)[c];
        *reinterpret_cast<uint4*>(dsm + L::V + st * L::TILE_BYTES + off) = reinterpret_cast<const uint4*>(vnew)[c];
      }
    if (TMA && j0 + DEC_TILE > r_end)
      for (int i = tid; i < DEC_TILE * CH; i += DEC_THREADS) {
        const int rr = i / CH, c = i - rr * CH;
        if (j0 + rr >= r_end)
          *reinterpret_cast<uint4*>(dsm + L::V + st * L::TILE_BYTES + toff<D, TMA>(rr, 8 * c)) =
              make_uint4(0u, 0u, 0u, 0u);
      }
  };
  if constexpr (TMA) {
    if (tid == 0)
      for (int t = 0; t < DEC_STAGES - 1 && t < n_tiles; ++t) issue(t);
  } else {
#pragma unroll
    for (int t = 0; t < DEC_STAGES - 1; ++t) {
      if (t < n_tiles) issue(t);
      cp_async_commit();
    }
  }

  // ---- the token's k (RMSNorm + RoPE), v, and the query group (RMSNorm + RoPE)
  const TX* x = static_cast<const TX*>(p.x) + s * p.x_ld;
  for (int i = tid; i < 16 * D / 8; i += DEC_THREADS)
    reinterpret_cast<uint4*>(qsm)[i] = make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();
  for (int item = warp; item <= G; item += 4) {
    const bool is_k = item == G;
    const TX* src = is_k ? x + kvh * D : x + 2 * p.n_kv * D + (kvh * G + item) * D;
    const float* gain = is_k ? p.k_gain : p.q_gain;
    float v[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) v[i] = to_f(src[lane * EPL + i]);
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < EPL; ++i) ss += v[i] * v[i];
    ss = warp_sum(ss);
    const float r = rsqrtf(ss / static_cast<float>(D) + p.eps);
#pragma unroll
    for (int i = 0; i < EPL; ++i) v[i] *= r * gain[lane * EPL + i];
    rope_lane<EPL>(v, lane, pos, p.inv_freq, p.rope_dims);
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int col = lane * EPL + i;
      if (is_k) knew[col] = F16<TC>::from(v[i]);
      else *reinterpret_cast<TC*>(dsm + L::Q + dsw<D>(item, col)) = F16<TC>::from(v[i]);
    }
  }
  for (int i = tid; i < D; i += DEC_THREADS) vnew[i] = F16<TC>::from(to_f(x[p.n_kv * D + kvh * D + i]));
  __syncthreads();
  if (split == 0) {  // the token's K and V rows go to the cache (no CTA reads them back)
    const int64_t o = dec_row(p, s, kvh, pos);
    if (o >= 0)
      for (int i = tid; i < CH; i += DEC_THREADS) {
        reinterpret_cast<uint4*>(static_cast<TC*>(p.kc) + o)[i] = reinterpret_cast<const uint4*>(knew)[i];
        reinterpret_cast<uint4*>(static_cast<TC*>(p.vc) + o)[i] = reinterpret_cast<const uint4*>(vnew)[i];
      }
  }

  // query fragments (A of S^T = Q K^T; query heads on M, rows 8-15 are zero)
  uint32_t qa0[D / 16], qa2[D / 16];
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    qa0[kk] = *reinterpret_cast<const uint32_t*>(dsm + L::Q + dsw<D>(lane >> 2, 16 * kk + 2 * (lane & 3)));
    qa2[kk] = *reinterpret_cast<const uint32_t*>(dsm + L::Q + dsw<D>(lane >> 2, 16 * kk + 8 + 2 * (lane & 3)));
  }

  // the cp.async tiles of the prologue hold every row but this token's (put_pos, below); TMA
  // tiles get theirs once they have landed
  if constexpr (!TMA) {
#pragma unroll
    for (int t = 0; t < DEC_STAGES - 1; ++t)
      if (t < n_tiles) put_pos(t);
  }

  const float kNegInf = -__int_as_float(0x7f800000);
  const float scale_log2 = 1.4426950408889634f * rsqrtf(static_cast<float>(D));
  float m_run = kNegInf, l_run = 0.f;  // head lane / 4
  float o[D / 16][4];
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
  const int mi = lane >> 3, lr = lane & 7;

#pragma unroll 1
  for (int t = 0; t < n_tiles; ++t) {
    const int st = t % DEC_STAGES;
    if constexpr (TMA) {
      if (tid == 0 && !*abort_flag && t + DEC_STAGES - 1 < n_tiles) issue(t + DEC_STAGES - 1);
      if (!*abort_flag) {
        if (mbar_wait(&full[st], (t / DEC_STAGES) & 1, abort_flag)) {
          if (tid == 0) last_ok = t;
        } else {
          *abort_flag = 1;
          set_device_error(p.err, KVA_DEV_WAIT_TIMEOUT);
        }
      }
      put_pos(t);
      fence_proxy_async_smem();  // generic writes into a tile the copy engine refills later
    } else {
      if (t + DEC_STAGES - 1 < n_tiles) {
        issue(t + DEC_STAGES - 1);
        put_pos(t + DEC_STAGES - 1);
      }
      cp_async_commit();
      cp_async_wait<DEC_STAGES - 1>();
    }
    __syncthreads();
    const uint32_t kb = sbase + L::K + st * L::TILE_BYTES, vb = sbase + L::V + st * L::TILE_BYTES;
    const int rw = 16 * warp;  // this warp's first row of the tile

    // S^T = Q K^T over this warp's 16 rows (two n-tiles of 8)
    float sacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t b[4];
      ldmatrix_x4(b, kb + toff<D, TMA>(rw + (mi >> 1) * 8 + lr, 16 * kk + (mi & 1) * 8));
      const uint32_t a[4] = {qa0[kk], 0u, qa2[kk], 0u};
      const uint32_t b0[2] = {b[0], b[1]}, b1[2] = {b[2], b[3]};
      F16<TC>::mma(sacc[0], a, b0);
      F16<TC>::mma(sacc[1], a, b1);
    }
    // online softmax of head lane / 4 over rows (2 (lane & 3) + j) + 8 nt
    const int64_t row0 = r_begin + static_cast<int64_t>(t) * DEC_TILE + rw + 2 * (lane & 3);
    float sv[2][2];
    float mt_ = kNegInf;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const bool ok = row0 + 8 * nt + j < r_end;
        sv[nt][j] = ok ? sacc[nt][j] * scale_log2 : kNegInf;
        mt_ = fmaxf(mt_, sv[nt][j]);
      }
    mt_ = fmaxf(mt_, __shfl_xor_sync(0xffffffffu, mt_, 1));
    mt_ = fmaxf(mt_, __shfl_xor_sync(0xffffffffu, mt_, 2));
    const float m_new = fmaxf(m_run, mt_);
    const float alpha = m_new == kNegInf ? 1.f : exp2f(m_run - m_new);
    float pv[2][2];
    float ps = 0.f;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        pv[nt][j] = m_new == kNegInf ? 0.f : exp2f(sv[nt][j] - m_new);
        ps += pv[nt][j];
      }
    l_run = l_run * alpha + ps;
    m_run = m_new;
    // O^T columns are heads 2 (lane & 3) and 2 (lane & 3) + 1
    const float al0 = __shfl_sync(0xffffffffu, alpha, 8 * (lane & 3));
    const float al1 = __shfl_sync(0xffffffffu, alpha, 8 * (lane & 3) + 4);
    const uint32_t pb[2] = {F16<TC>::pack(pv[0][0], pv[0][1]), F16<TC>::pack(pv[1][0], pv[1][1])};
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
      o[mt][0] *= al0;
      o[mt][1] *= al1;
      o[mt][2] *= al0;
      o[mt][3] *= al1;
      uint32_t a[4];
      ldmatrix_x4_trans(a, vb + toff<D, TMA>(rw + (mi >> 1) * 8 + lr, 16 * mt + (mi & 1) * 8));
      const uint32_t av[4] = {a[0], a[1], a[2], a[3]};
      F16<TC>::mma(o[mt], av, pb);
    }
    __syncthreads();  // the stage is free for the next issue
  }
  if constexpr (TMA) {
    // every tile this block requested has landed before its shared memory is reused
    if (tid == 0)
      for (int t = last_ok + 1; t < issued; ++t)
        if (!mbar_wait_limit(&full[t % DEC_STAGES], (t / DEC_STAGES) & 1))
          set_device_error(p.err, KVA_DEV_WAIT_TIMEOUT);
  } else {
    cp_async_wait<0>();
  }
  __syncthreads();

  // ---- merge the four warps' states, then write this split's partial
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
  float* mw = reinterpret_cast<float*>(dsm + L::K + warp * L::MERGE_WARP);
  if ((lane & 3) == 0) {
    mw[lane >> 2] = m_run;
    mw[8 + (lane >> 2)] = l_run;
  }
  float* Ow = mw + 16;
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt) {
    const int d0 = 16 * mt + (lane >> 2), h0 = 2 * (lane & 3);
    Ow[h0 * D + d0] = o[mt][0];
    Ow[(h0 + 1) * D + d0] = o[mt][1];
    Ow[h0 * D + d0 + 8] = o[mt][2];
    Ow[(h0 + 1) * D + d0 + 8] = o[mt][3];
  }
  __syncthreads();
  float* part = p.part + ((static_cast<int64_t>(s) * p.n_kv + kvh) * p.n_split + split) * G * (D + 2);
  for (int i = tid; i < G * D; i += DEC_THREADS) {
    const int g = i / D, d = i - g * D;
    float M = kNegInf;
#pragma unroll
    for (int w = 0; w < 4; ++w)
      M = fmaxf(M, reinterpret_cast<const float*>(dsm + L::K + w * L::MERGE_WARP)[g]);
    float Osum = 0.f, Lsum = 0.f;
    if (M != kNegInf) {
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float* b = reinterpret_cast<const float*>(dsm + L::K + w * L::MERGE_WARP);
        const float f = b[g] == kNegInf ? 0.f : exp2f(b[g] - M);
        Osum += f * b[16 + g * D + d];
        Lsum += f * b[8 + g];
      }
    }
    part[g * (D + 2) + d] = Osum;
    if (d == 0) {
      part[g * (D + 2) + D] = M;
      part[g * (D + 2) + D + 1] = Lsum;
    }
  }
}

// every query head: merge the splits, divide by the softmax sum, apply sigmoid(gate).  The
// splits' maxima and sums are staged in shared memory first, so each thread's sum over the
// splits is a run of independent loads.
template <int D, typename TX, typename TO>
__global__ void __launch_bounds__(D) attn_decode_combine_kernel(const AttnDecodeLaunch p) {
  __shared__ float wsm[kDecodeMaxSplit];  // per split: weight 2^(m - M)
  __shared__ float lsum;
  griddep_wait_and_release();
  const int h = blockIdx.x, s = blockIdx.y, d = threadIdx.x;
  const int G = p.G, kvh = h / G, g = h - kvh * G;
  const float kNegInf = -__int_as_float(0x7f800000);
  const int64_t stride = static_cast<int64_t>(G) * (D + 2);
  const float* base = p.part + (static_cast<int64_t>(s) * p.n_kv + kvh) * p.n_split * stride + g * (D + 2);
  const int64_t rows = p.pos[s] + 1;
  const int ns = static_cast<int>((rows + p.rows_per_split - 1) / p.rows_per_split);
  if (d < 32) {  // one warp: the maxima, the weights, the softmax sum
    float M = kNegInf;
    for (int i = d; i < ns; i += 32) M = fmaxf(M, base[i * stride + D]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float L = 0.f;
    for (int i = d; i < ns; i += 32) {
      const float m = base[i * stride + D];
      const float f = m == kNegInf ? 0.f : exp2f(m - M);
      wsm[i] = f;
      L += f * base[i * stride + D + 1];
    }
    L = warp_sum(L);
    if (d == 0) lsum = L;
  }
  __syncthreads();
  float O = 0.f;
#pragma unroll 8
  for (int i = 0; i < ns; ++i) O += wsm[i] * base[i * stride + d];
  const TX* x = static_cast<const TX*>(p.x) + s * p.x_ld;
  const float gate = to_f(x[2 * p.n_kv * D + p.n_q * D + h * D + d]);
  TO* out = static_cast<TO*>(p.out) + s * p.out_ld + h * D;
  out[d] = from_f<TO>(O / lsum * (1.f / (1.f + expf(-gate))));
}

template <typename TX, typename TO>
int launch_gdn_decode_t(const GdnDecodeLaunch& g, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(g.n_v, g.n_seq);
  cfg.blockDim = dim3(256);
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = g.n_v / g.n_k;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t r = g.d == 128 ? cudaLaunchKernelEx(&cfg, gdn_decode_kernel<128, TX, TO>, g)
                                   : cudaLaunchKernelEx(&cfg, gdn_decode_kernel<64, TX, TO>, g);
  return r == cudaSuccess ? KVA_OK : KVA_ERR_CUDA;
}

template <int D, typename TX, typename TC, typename TO>
int launch_attn_decode_t(const AttnDecodeLaunch& a, cudaStream_t s) {
  const size_t smem = DecSmem<D>::ALLOC;
  // TMA boxes of 64 rows need the rows of a tile in one page (page_size % 64 == 0)
  const bool tma = a.layout == KVA_KV_CONTIGUOUS || a.page_size % DEC_TILE == 0;
  CUtensorMap mK{}, mV{};
  if (tma) {
    const int64_t rows = a.layout == KVA_KV_CONTIGUOUS ? a.max_pos : a.page_size;
    const int64_t planes = a.layout == KVA_KV_CONTIGUOUS ? static_cast<int64_t>(a.n_seq) * a.n_kv
                                                         : static_cast<int64_t>(a.n_pages) * a.n_kv;
    const bool f16 = a.cache_dtype == KVA_F16;
    if (!make_map_3d_16bit(&mK, a.kc, f16, D, rows, planes, 64, DEC_TILE) ||
        !make_map_3d_16bit(&mV, a.vc, f16, D, rows, planes, 64, DEC_TILE))
      return KVA_ERR_CUDA;
  }
  auto kern = tma ? attn_decode_kernel<D, TX, TC, true> : attn_decode_kernel<D, TX, TC, false>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
      cudaSuccess)
    return KVA_ERR_CUDA;
  cudaError_t r = launch_pdl(kern, dim3(a.n_split, a.n_kv, a.n_seq), dim3(DEC_THREADS), smem, s, mK, mV, a);
  if (r != cudaSuccess) return KVA_ERR_CUDA;
  r = launch_pdl(attn_decode_combine_kernel<D, TX, TO>, dim3(a.n_q, a.n_seq), dim3(D), 0, s, a);
  return r == cudaSuccess ? KVA_OK : KVA_ERR_CUDA;
}

template <typename TX, typename TC>
int launch_attn_decode_tc(const AttnDecodeLaunch& a, cudaStream_t s) {
  const bool f32 = a.out_dtype == KVA_F32;
  if (a.d_h == 256)
    return f32 ? launch_attn_decode_t<256, TX, TC, float>(a, s) : launch_attn_decode_t<256, TX, TC, TX>(a, s);
  return f32 ? launch_attn_decode_t<128, TX, TC, float>(a, s) : launch_attn_decode_t<128, TX, TC, TX>(a, s);
}

}  // namespace

int launch_gdn_decode(const GdnDecodeLaunch& g, cudaStream_t s) {
  if (g.n_seq == 0) return KVA_OK;
  if (g.d != 64 && g.d != 128) return KVA_ERR_UNSUPPORTED;
  if (g.n_v % g.n_k || g.n_v / g.n_k > 8) return KVA_ERR_UNSUPPORTED;  // portable cluster size
  const bool xf = g.x_dtype == KVA_F16, of32 = g.out_dtype == KVA_F32;
  if (xf) return of32 ? launch_gdn_decode_t<__half, float>(g, s) : launch_gdn_decode_t<__half, __half>(g, s);
  return of32 ? launch_gdn_decode_t<__nv_bfloat16, float>(g, s)
              : launch_gdn_decode_t<__nv_bfloat16, __nv_bfloat16>(g, s);
}

int attn_decode_splits(int n_seq, int n_kv, int64_t max_rows, int sms, int64_t* rows_per_split) {
  const int64_t tiles = (max_rows + DEC_TILE - 1) / DEC_TILE;
  // one CTA per SM (three 64-row stages fill its shared memory): one wave of equal splits
  int64_t want = sms / (static_cast<int64_t>(n_seq) * n_kv);
  if (want > kDecodeMaxSplit) want = kDecodeMaxSplit;
  if (want > tiles) want = tiles;
  if (want < 1) want = 1;
  const int64_t tiles_per = (tiles + want - 1) / want;
  *rows_per_split = tiles_per * DEC_TILE;
  return static_cast<int>((max_rows + *rows_per_split - 1) / *rows_per_split);
}

int launch_attn_decode(const AttnDecodeLaunch& a, cudaStream_t s) {
  if (a.n_seq == 0) return KVA_OK;
  if (a.d_h != 128 && a.d_h != 256) return KVA_ERR_UNSUPPORTED;
  if (a.G < 1 || a.G > 8 || a.n_q != a.G * a.n_kv) return KVA_ERR_UNSUPPORTED;
  if (a.n_split < 1 || a.n_split > kDecodeMaxSplit) return KVA_ERR_INVALID_ARG;
  const int epl = a.d_h / 32;
  if (a.rope_dims < 0 || a.rope_dims % 2 || a.rope_dims > a.d_h) return KVA_ERR_UNSUPPORTED;
  if (a.rope_dims > 0) {
    const int half = a.rope_dims / 2;
    if (half % epl || ((half / epl) & (half / epl - 1))) return KVA_ERR_UNSUPPORTED;
  }
  const bool xf = a.x_dtype == KVA_F16, cf = a.cache_dtype == KVA_F16;
  if (a.cache_dtype != KVA_BF16 && a.cache_dtype != KVA_F16) return KVA_ERR_UNSUPPORTED;
  if (xf) return cf ? launch_attn_decode_tc<__half, __half>(a, s) : launch_attn_decode_tc<__half, __nv_bfloat16>(a, s);
  return cf ? launch_attn_decode_tc<__nv_bfloat16, __half>(a, s)
            : launch_attn_decode_tc<__nv_bfloat16, __nv_bfloat16>(a, s);
}

}  // namespace kva
