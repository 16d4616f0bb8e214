// Gated-DeltaNet state updates of the late layers ("Qwen3.8-27B-KVA" model card,
// section "What the hell?": conv + silu, l2-norm and the deltanet scan run on the
// approximated in_proj_qkv / in_proj_a / in_proj_b outputs).
//
// 1. gdn_prepare_kernel: causal depthwise conv1d (kernel 4, carried tail of the
//    last 3 raw rows) + SiLU over the q/k/v channels, per-head L2 norm of q and k,
//    and the gates g = -exp(A_log) softplus(a + dt_bias), beta = sigmoid(b).
// 2. gdn_tail_kernel: the new conv tail = last 3 raw rows of [tail; X] (bit copy).
// 3. gdn_scan_kernel: the gated delta rule
//        S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
//    over the ubatch in chunks of 64 tokens, emitting only the final state.
//    Per chunk (local cumulative decay gam_t = sum_{s<=t} g_s):
//        L[t,s] = beta_t e^(gam_t-gam_s) k_t.k_s (s < t),  Tm = (I + L)^-1,
//        U      = Tm diag(beta) V - Tm diag(beta e^gam) K S^T,
//        S     <- e^gam_last S + (diag(e^(gam_last-gam)) U)^T K.
//    One CTA per (sequence, layer, v head); state warp w owns state rows
//    [16w, 16w+16) as mma.sync accumulators, so the state-dependent products
//    (U and the update) are warp-local, while 4 prep warps build the chunk-local
//    K K^T, Tm and W = Tm diag(beta e^gam) K one chunk ahead.  Chunk
//    contractions run on tensor cores with fp16
//    operands (every operand is bounded: unit keys, SiLU values, the inverse,
//    the state) and fp32 accumulation; the state stays fp32.
#include "kva_common.cuh"

namespace kva {

// ------------------------------------------------------------------ prepare
// Each thread owns 8 consecutive channels (one 16-byte vector per token row) and
// streams PREP_TT tokens: a window of the 3 previous rows (unpacked) and
// PREP_AHEAD raw rows in flight, so every input row is loaded and unpacked once
// and the loads of later rows overlap the arithmetic of earlier ones.  The L2 norm
// of a q/k head is a shuffle reduction over the d_k/8 lanes that hold it.  Blocks
// along x cover 2048 channels of the token range, the last x-block computes the
// gates.
constexpr int PREP_TT = 64;
constexpr int PREP_AHEAD = 8;
constexpr int PREP_THREADS = 256;
constexpr int PREP_CH = PREP_THREADS * 8;

template <typename TM>
__device__ __forceinline__ void unpack8(const uint4& v, float (&x)[8]) {
  const uint32_t* u = &v.x;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = F16<TM>::unpack(u[i]);
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
}

template <typename TM>
__global__ void __launch_bounds__(PREP_THREADS, 2) gdn_prepare_kernel(const GdnLaunch p) {
  griddep_wait_and_release();
  const int slot = blockIdx.z;  // seq * n_gdn + layer
  const int seq = slot / p.n_gdn, layer = slot % p.n_gdn;
  const int T = p.T;
  const int t0 = blockIdx.y * PREP_TT;
  const int tend = min(T, t0 + PREP_TT);
  const int nt = tend - t0;
  const int C = p.C;
  const int nkdk = p.n_k * p.d_k;
  const TM* mix = static_cast<const TM*>(p.mix) + seq * p.mix_seq_stride + p.layer_col[layer];
  const int64_t ld = p.mix_ld;
  const int n_cblk = (C + PREP_CH - 1) / PREP_CH;

  if (static_cast<int>(blockIdx.x) < n_cblk) {
    // q is only an optional debug output (the state update reads k, v and the gates):
    // without a debug buffer, blocks whose channels are all q have nothing to do
    if (!p.debug_qkv && (blockIdx.x + 1) * PREP_CH <= nkdk) return;
    const int c0 = blockIdx.x * PREP_CH + threadIdx.x * 8;
    const bool active = c0 < C;
    const int cc = active ? c0 : 0;
    const TM* tail = static_cast<const TM*>(p.conv_state) + static_cast<int64_t>(slot) * 3 * C + cc;
    // raw row t of [tail; X] for these 8 channels (t >= -3; rows past T re-read row
    // T - 1, whose values are then not used)
    auto row = [&](int t) {
      const TM* src = t < 0 ? tail + (t + 3) * C : mix + static_cast<int64_t>(min(t, T - 1)) * ld + cc;
      return __ldg(reinterpret_cast<const uint4*>(src));
    };
    uint4 q[PREP_AHEAD];
#pragma unroll
    for (int j = 0; j < PREP_AHEAD; ++j) q[j] = row(t0 + j);
    float win[3][8];
#pragma unroll
    for (int r = 0; r < 3; ++r) unpack8<TM>(row(t0 - 3 + r), win[r]);
    float w[8][4];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float4 wv = *reinterpret_cast<const float4*>(p.conv_w + (static_cast<int64_t>(layer) * C + cc + e) * 4);
      w[e][0] = wv.x;
      w[e][1] = wv.y;
      w[e][2] = wv.z;
      w[e][3] = wv.w;
    }
    const bool is_qk = c0 < 2 * nkdk;
    const int hl = p.d_k / 8;  // lanes per q/k head
    const int64_t tbase = static_cast<int64_t>(slot) * T;
    __nv_bfloat16* dbg = static_cast<__nv_bfloat16*>(p.debug_qkv);
    // the token loop is uniform over the block (the norm shuffles need every lane)
    for (int tb = 0; tb < nt; tb += PREP_AHEAD) {
#pragma unroll
      for (int j = 0; j < PREP_AHEAD; ++j) {
        const int i = tb + j;
        float x[8];
        unpack8<TM>(q[j], x);
        q[j] = row(t0 + i + PREP_AHEAD);
        float z[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
          z[e] = silu_tanh(w[e][0] * win[0][e] + w[e][1] * win[1][e] + w[e][2] * win[2][e] +
                           w[e][3] * x[e]);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          win[0][e] = win[1][e];
          win[1][e] = win[2][e];
          win[2][e] = x[e];
        }
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) ss += z[e] * z[e];
        for (int o = 1; o < hl; o <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if (is_qk) {
          const float sc = rsqrtf(ss + p.eps);
#pragma unroll
          for (int e = 0; e < 8; ++e) z[e] *= sc;
        }
        if (active && i < nt) {
          const int64_t t = tbase + t0 + i;
          uint4 hv;
          hv.x = pack_f16(z[0], z[1]);
          hv.y = pack_f16(z[2], z[3]);
          hv.z = pack_f16(z[4], z[5]);
          hv.w = pack_f16(z[6], z[7]);
          if (c0 >= 2 * nkdk) {
            const int nvdv = C - 2 * nkdk;
            *reinterpret_cast<uint4*>(static_cast<__half*>(p.vbuf) + t * nvdv + (c0 - 2 * nkdk)) = hv;
          } else if (c0 >= nkdk) {
            *reinterpret_cast<uint4*>(static_cast<__half*>(p.kbuf) + t * nkdk + (c0 - nkdk)) = hv;
          }
          if (dbg) {
            uint4 bv;
            bv.x = pack_bf16(z[0], z[1]);
            bv.y = pack_bf16(z[2], z[3]);
            bv.z = pack_bf16(z[4], z[5]);
            bv.w = pack_bf16(z[6], z[7]);
            *reinterpret_cast<uint4*>(dbg + t * C + c0) = bv;
          }
        }
      }
    }
  } else {
    // gates for nt tokens x n_v heads
    const int n_v = p.n_v;
    const float* A_log = p.A_log + layer * n_v;
    const float* dt_bias = p.dt_bias + layer * n_v;
    float* gb = p.gbuf + static_cast<int64_t>(slot) * 2 * n_v * T;
    for (int idx = threadIdx.x; idx < nt * n_v; idx += PREP_THREADS) {
      const int i = idx / n_v, h = idx - i * n_v;
      const int t = t0 + i;
      const float a = F16<TM>::to(mix[t * ld + C + h]);
      const float b = F16<TM>::to(mix[t * ld + C + n_v + h]);
      const float x = a + dt_bias[h];
      const float sp = x > 20.f ? x : log1pf(expf(x));
      gb[h * T + t] = -expf(A_log[h]) * sp;
      gb[(n_v + h) * T + t] = 1.f / (1.f + expf(-b));
    }
  }
}

// The tail holds raw 16-bit values: a bit copy, whatever their format.
__global__ void gdn_tail_kernel(const GdnLaunch p) {
  griddep_wait_and_release();
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= p.C) return;
  const int slot = blockIdx.y;
  const int seq = slot / p.n_gdn, layer = slot % p.n_gdn;
  const uint16_t* mix = static_cast<const uint16_t*>(p.mix) + seq * p.mix_seq_stride +
                        p.layer_col[layer] + c;
  uint16_t* tail = static_cast<uint16_t*>(p.conv_state) + static_cast<int64_t>(slot) * 3 * p.C + c;
  // new tail row i is row T+i of [old tail; X]; ascending i reads only rows > i
  for (int i = 0; i < 3; ++i) {
    const int src = p.T + i;
    const uint16_t v = src >= 3 ? mix[static_cast<int64_t>(src - 3) * p.mix_ld] : tail[src * p.C];
    tail[i * p.C] = v;
  }
}

// ------------------------------------------------------------------ scan
constexpr int SCAN_CH = 64;
constexpr int SCAN_PREP_WARPS = 4;
constexpr int SCAN_PREP_THREADS = SCAN_PREP_WARPS * 32;
constexpr uint64_t kScanWaitNs = 200000000ull;  // a chunk hand-off takes microseconds

// byte offset of (row, 16-byte chunk) in a 16-bit tile whose rows are `rb` bytes
__device__ __forceinline__ uint32_t sw_off(int row, int chunk, int rb) {
  return static_cast<uint32_t>(row * rb + ((chunk ^ (row & 7)) << 4));
}

// Bounded wait; the clock is read only every 64 polls (a %globaltimer read is slow).
__device__ __forceinline__ bool mbar_wait_ns(uint64_t* bar, uint32_t parity, uint64_t limit) {
  uint64_t t0 = 0;
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63u) == 0) {
      const uint64_t t = globaltimer_ns();
      if (t0 == 0) t0 = t;
      else if (t - t0 > limit) return false;
    }
  }
}

__device__ __forceinline__ void prep_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(SCAN_PREP_THREADS) : "memory");
}

template <int D>
struct ScanLayout {
  static constexpr int NSW = D / 16;  // state warps: 16 state rows each
  static constexpr int NT = (NSW + SCAN_PREP_WARPS) * 32;
  static constexpr int KVB = SCAN_CH * D * 2;        // one [64][D] fp16 tile
  static constexpr int TBB = SCAN_CH * SCAN_CH * 2;  // one [64][64] fp16 tile
  // one chunk buffer (prep -> state): -W = -Tm diag(beta e^gam) K, U0 = Tm diag(beta) V,
  // decay vector and e^(gam_last)
  static constexpr int B_W = 0;
  static constexpr int B_U = KVB;
  static constexpr int B_DEC = 2 * KVB;
  static constexpr int BUF = ((B_DEC + SCAN_CH * 4 + 16) + 127) / 128 * 128;
  // K ring of 3 slots: the state warps read chunk c's slot while the prep warps
  // solve chunk c+1 and prefetch chunk c+2
  static constexpr int OFF_K = 2 * BUF;
  // prep-private
  static constexpr int OFF_V = OFF_K + 3 * KVB;               // V, double buffered
  static constexpr int OFF_GB = OFF_V + 2 * KVB;              // raw g, beta, double buffered
  static constexpr int OFF_LN = OFF_GB + 2 * 2 * SCAN_CH * 4;  // -L, fp16 [64][64]
  static constexpr int OFF_TD = OFF_LN + TBB;          // diagonal blocks of Tm, fp16 [64][64]
  static constexpr int OFF_LD = OFF_TD + TBB;          // diagonal blocks of L, fp32 [4][16][17]
  static constexpr int OFF_G = OFF_LD + 4 * 16 * 17 * 4;  // gam, e^gam
  static constexpr int OFF_BAR = OFF_G + 2 * SCAN_CH * 4;
  static constexpr int BYTES = OFF_BAR + 64;
};

__device__ __forceinline__ uint32_t ld_smem_u32(const uint8_t* p) {
  return *reinterpret_cast<const uint32_t*>(p);
}

// One CTA per (sequence, layer, v head).  Warps [0, NSW) are state warps: warp w
// holds state rows [16w, 16w+16) as mma.sync accumulators and, per chunk, forms
// U = U0 + (-W) S^T for its rows and the update S <- e^gam_last S + (dec U)^T K.
// The 4 prep warps run one chunk ahead: cumulative decays, L = beta e^(gam_t -
// gam_s) K K^T (s < t), the 16x16 diagonal blocks of Tm = (I + L)^-1 by substitution
// in registers, and then (I + L) X = [diag(beta) V | diag(beta e^gam) K] by block-row
// forward substitution on tensor cores, each prep warp owning a quarter of the
// columns (so the solve needs no cross-warp synchronisation).  Buffers change
// hands through mbarriers (ready: prep -> state, free: state -> prep) with
// time-bounded waits.
template <int D>
__global__ void __launch_bounds__(ScanLayout<D>::NT, 1) gdn_scan_kernel(const GdnLaunch p) {
  griddep_wait_and_release();
  using L = ScanLayout<D>;
  constexpr int NSW = L::NSW;
  constexpr int RB = 2 * D;
  extern __shared__ __align__(128) uint8_t sm[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::OFF_BAR);  // ready[2], free[2]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c = lane & 3, mi = lane >> 3, lr = lane & 7;
  const int h = blockIdx.x, layer = blockIdx.y, seq = blockIdx.z;
  const int n_v = p.n_v;
  const int kh = h / (n_v / p.n_k);
  const int T = p.T;
  const int slot = seq * p.n_gdn + layer;
  const int nkdk = p.n_k * D, nvdv = n_v * D;
  const int n_chunks = (T + SCAN_CH - 1) / SCAN_CH;

  if (tid == 0) {
    mbar_init(&bars[0], SCAN_PREP_THREADS);
    mbar_init(&bars[1], SCAN_PREP_THREADS);
    mbar_init(&bars[2], NSW * 32);
    mbar_init(&bars[3], NSW * 32);
    fence_mbar_init();
  }
  __syncthreads();

  if (warp < NSW) {
    // ===================================================== state warps
    float* Sg = p.state + (static_cast<int64_t>(slot) * n_v + h) * D * D;
    float S[D / 8][4];
    {
      const float* s0 = Sg + (16 * warp + g) * D + 2 * c;
      const float* s1 = s0 + 8 * D;
#pragma unroll
      for (int nt = 0; nt < D / 8; ++nt) {
        const float2 a = *reinterpret_cast<const float2*>(s0 + 8 * nt);
        const float2 b = *reinterpret_cast<const float2*>(s1 + 8 * nt);
        S[nt][0] = a.x;
        S[nt][1] = a.y;
        S[nt][2] = b.x;
        S[nt][3] = b.y;
      }
    }
    for (int ci = 0; ci < n_chunks; ++ci) {
      const int b = ci & 1;
      if (!mbar_wait_ns(&bars[b], (ci >> 1) & 1, kScanWaitNs)) set_device_error(p.err, KVA_DEV_WAIT_TIMEOUT);
      const uint8_t* buf = sm + b * L::BUF;
      const uint32_t sK = smem_u32(sm + L::OFF_K + (ci % 3) * L::KVB), sW = smem_u32(buf + L::B_W);
      const float* dec = reinterpret_cast<const float*>(buf + L::B_DEC);
      // U starts from U0 = Tm diag(beta) V, this warp's columns [16w, 16w+16)
      float U[4][2][4];
#pragma unroll
      for (int m = 0; m < 4; ++m)
#pragma unroll
        for (int n = 0; n < 2; ++n) {
          const int t = m * 16 + g;
          const float2 u0 = F16<__half>::unpack(ld_smem_u32(buf + L::B_U + sw_off(t, warp * 2 + n, RB) + 4 * c));
          const float2 u1 = F16<__half>::unpack(ld_smem_u32(buf + L::B_U + sw_off(t + 8, warp * 2 + n, RB) + 4 * c));
          U[m][n][0] = u0.x;
          U[m][n][1] = u0.y;
          U[m][n][2] = u1.x;
          U[m][n][3] = u1.y;
        }
      // U += (-W) S^T, the B operand straight from this warp's state rows
      {
        uint32_t sb[D / 8][2];
#pragma unroll
        for (int nt = 0; nt < D / 8; ++nt) {
          sb[nt][0] = pack_f16(S[nt][0], S[nt][1]);
          sb[nt][1] = pack_f16(S[nt][2], S[nt][3]);
        }
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          uint32_t b0[2] = {sb[2 * ks][0], sb[2 * ks + 1][0]};
          uint32_t b1[2] = {sb[2 * ks][1], sb[2 * ks + 1][1]};
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            uint32_t a[4];
            ldmatrix_x4(a, sW + sw_off(m * 16 + (mi & 1) * 8 + lr, ks * 2 + (mi >> 1), RB));
            mma_f16_16816(U[m][0], a, b0);
            mma_f16_16816(U[m][1], a, b1);
          }
        }
      }
      // S <- e^gam_last S + (dec U)^T K
      {
        const float gl = dec[SCAN_CH];
#pragma unroll
        for (int nt = 0; nt < D / 8; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) S[nt][e] *= gl;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const float d0 = dec[m * 16 + g], d1 = dec[m * 16 + 8 + g];
          uint32_t a[4];
          a[0] = movmatrix_trans(pack_f16(U[m][0][0] * d0, U[m][0][1] * d0));
          a[1] = movmatrix_trans(pack_f16(U[m][1][0] * d0, U[m][1][1] * d0));
          a[2] = movmatrix_trans(pack_f16(U[m][0][2] * d1, U[m][0][3] * d1));
          a[3] = movmatrix_trans(pack_f16(U[m][1][2] * d1, U[m][1][3] * d1));
#pragma unroll
          for (int nt = 0; nt < D / 8; nt += 2) {
            uint32_t bk[4];
            ldmatrix_x4_trans(bk, sK + sw_off(m * 16 + (mi & 1) * 8 + lr, nt + (mi >> 1), RB));
            uint32_t b0[2] = {bk[0], bk[1]}, b1[2] = {bk[2], bk[3]};
            mma_f16_16816(S[nt], a, b0);
            mma_f16_16816(S[nt + 1], a, b1);
          }
        }
      }
      mbar_arrive(&bars[2 + b]);
    }
    float* s0 = Sg + (16 * warp + g) * D + 2 * c;
    float* s1 = s0 + 8 * D;
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt) {
      *reinterpret_cast<float2*>(s0 + 8 * nt) = make_float2(S[nt][0], S[nt][1]);
      *reinterpret_cast<float2*>(s1 + 8 * nt) = make_float2(S[nt][2], S[nt][3]);
    }
  } else {
    // ===================================================== prep warps
    constexpr int NTW = D / 16;  // 8-column tiles per prep warp (a quarter of 2D columns)
    const int pt = tid - NSW * 32;  // 0..127
    const int pw = warp - NSW;      // 0..3
    const bool kpart = pw >= 2;     // warps 0,1: U0 columns (V); warps 2,3: -W columns (K)
    const int col0 = (pw & 1) * (D / 2);
    const __half* kg =
        static_cast<const __half*>(p.kbuf) + static_cast<int64_t>(slot) * T * nkdk + kh * D;
    const __half* vg =
        static_cast<const __half*>(p.vbuf) + static_cast<int64_t>(slot) * T * nvdv + h * D;
    const float* gg = p.gbuf + static_cast<int64_t>(slot) * 2 * n_v * T + h * T;
    const float* bg = gg + static_cast<int64_t>(n_v) * T;
    float* Ld = reinterpret_cast<float*>(sm + L::OFF_LD);
    float* gam = reinterpret_cast<float*>(sm + L::OFF_G);
    float* Gam = gam + SCAN_CH;
    const uint32_t sLN = smem_u32(sm + L::OFF_LN);
    const uint32_t sTD = smem_u32(sm + L::OFF_TD);

    // K, V rows of chunk cj into their ring slots and its raw g, beta into the
    // chunk's g/beta slot, all with cp.async (zero past T: identity steps)
    auto issue_chunk = [&](int cj) {
      const uint32_t dK = smem_u32(sm + L::OFF_K + (cj % 3) * L::KVB);
      const uint32_t dV = smem_u32(sm + L::OFF_V + (cj & 1) * L::KVB);
      const uint32_t dG = smem_u32(sm + L::OFF_GB + (cj & 1) * 2 * SCAN_CH * 4);
      const int cb = cj * SCAN_CH;
      for (int i = pt; i < SCAN_CH * (D / 8); i += SCAN_PREP_THREADS) {
        const int r = i / (D / 8), ch = i % (D / 8);
        const int t = cb + r;
        const bool ok = t < T;
        const int64_t tt = ok ? t : 0;
        cp_async16(dK + sw_off(r, ch, RB), kg + tt * nkdk + ch * 8, ok ? 16u : 0u);
        cp_async16(dV + sw_off(r, ch, RB), vg + tt * nvdv + ch * 8, ok ? 16u : 0u);
      }
      if (pt < SCAN_CH) {
        const int t = cb + pt;
        const bool ok = t < T;
        cp_async4(dG + pt * 4, gg + (ok ? t : 0), ok ? 4u : 0u);
        cp_async4(dG + (SCAN_CH + pt) * 4, bg + (ok ? t : 0), ok ? 4u : 0u);
      }
      cp_async_commit();
    };

    issue_chunk(0);
    for (int ci = 0; ci < n_chunks; ++ci) {
      const int b = ci & 1;
      if (ci >= 2 && !mbar_wait_ns(&bars[2 + b], ((ci >> 1) - 1) & 1, kScanWaitNs))
        set_device_error(p.err, KVA_DEV_WAIT_TIMEOUT);
      // chunk ci + 1's K slot was last read by the state warps for chunk ci - 2 (done)
      if (ci + 1 < n_chunks) {
        issue_chunk(ci + 1);
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      uint8_t* buf = sm + b * L::BUF;
      const uint8_t* kp = sm + L::OFF_K + (ci % 3) * L::KVB;
      const uint8_t* vp = sm + L::OFF_V + (ci & 1) * L::KVB;
      const uint32_t sK = smem_u32(kp);
      const uint32_t sV = smem_u32(vp);
      const float* gs = reinterpret_cast<const float*>(sm + L::OFF_GB + (ci & 1) * 2 * SCAN_CH * 4);
      const float* bs = gs + SCAN_CH;
      float* dec = reinterpret_cast<float*>(buf + L::B_DEC);
      prep_sync();
      // (2) cumulative decays (warp 0) and K K^T for m-tile pw
      if (pw == 0) {
        const float v0 = gs[2 * lane], v1 = gs[2 * lane + 1];
        const float pair = v0 + v1;
        float sc = pair;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const float y = __shfl_up_sync(0xffffffffu, sc, o);
          if (lane >= o) sc += y;
        }
        const float ex = sc - pair;
        const float total = __shfl_sync(0xffffffffu, sc, 31);
        const float ga = ex + v0, gb2 = ex + pair;
        gam[2 * lane] = ga;
        gam[2 * lane + 1] = gb2;
        Gam[2 * lane] = expf(ga);
        Gam[2 * lane + 1] = expf(gb2);
        dec[2 * lane] = expf(total - ga);
        dec[2 * lane + 1] = expf(total - gb2);
        if (lane == 0) dec[SCAN_CH] = expf(total);
      }
      {
        float acc[8][4];
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          uint32_t a[4];
          ldmatrix_x4(a, sK + sw_off(pw * 16 + (mi & 1) * 8 + lr, ks * 2 + (mi >> 1), RB));
#pragma unroll
          for (int j = 0; j < 8; j += 2) {
            uint32_t bb[4];
            ldmatrix_x4(bb, sK + sw_off(j * 8 + (mi >> 1) * 8 + lr, ks * 2 + (mi & 1), RB));
            uint32_t b0[2] = {bb[0], bb[1]}, b1[2] = {bb[2], bb[3]};
            mma_f16_16816(acc[j], a, b0);
            mma_f16_16816(acc[j + 1], a, b1);
          }
        }
        prep_sync();  // gam ready
        // -L (fp16, all blocks) and the diagonal blocks of L (fp32)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          float lv[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int t = pw * 16 + g + (e >> 1) * 8;
            const int s2 = j * 8 + 2 * c + (e & 1);
            lv[e] = s2 < t ? bs[t] * expf(gam[t] - gam[s2]) * acc[j][e] : 0.f;
            if ((s2 >> 4) == pw) Ld[(pw * 16 + (t & 15)) * 17 + (s2 & 15)] = lv[e];
          }
          const int t0 = pw * 16 + g;
          const uint32_t o0 = static_cast<uint32_t>(t0 * 128 + ((j ^ (t0 & 7)) << 4) + 4 * c);
          const uint32_t o1 = static_cast<uint32_t>((t0 + 8) * 128 + ((j ^ ((t0 + 8) & 7)) << 4) + 4 * c);
          *reinterpret_cast<uint32_t*>(sm + L::OFF_LN + o0) = pack_f16(-lv[0], -lv[1]);
          *reinterpret_cast<uint32_t*>(sm + L::OFF_LN + o1) = pack_f16(-lv[2], -lv[3]);
        }
      }
      prep_sync();
      // (3) diagonal blocks of Tm = (I + L)^-1, one column per thread, in registers
      if (pt < 64) {
        const int blk = pt >> 4, col = pt & 15;
        const float* Lb = Ld + blk * 16 * 17;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) x[r] = r == col ? 1.f : 0.f;
#pragma unroll
        for (int r = 1; r < 16; ++r) {
          float sacc = 0.f;
#pragma unroll
          for (int q = 0; q < r; ++q) sacc += Lb[r * 17 + q] * x[q];
          if (r > col) x[r] = -sacc;
        }
        // Tm block into the fp16 tile at rows/cols [16 blk, 16 blk + 16)
#pragma unroll
        for (int r = 0; r < 16; ++r) {
          const int t = blk * 16 + r, s2 = blk * 16 + col;
          *reinterpret_cast<__half*>(sm + L::OFF_TD + t * 128 + (((s2 >> 3) ^ (t & 7)) << 4) + (s2 & 7) * 2) =
              __float2half_rn(x[r]);
        }
      }
      prep_sync();
      // (4) block rows i = 0..3: X_i = Tm_ii (B_i - sum_{j<i} L_ij X_j), for this warp's
      //     2D/4 columns of B = [diag(beta) V | diag(beta e^gam) K]
      {
        const uint32_t srcB = kpart ? sK : sV;
        const uint8_t* srcBp = kpart ? kp : vp;
        uint8_t* dst = kpart ? buf + L::B_W : buf + L::B_U;
        const float sgn = kpart ? -1.f : 1.f;
        (void)srcB;
        uint32_t xb[3][NTW][2];  // X_0..X_2 as B fragments (k = rows of the block)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float y[NTW][4];
          const int t0 = i * 16 + g, t1 = t0 + 8;
          const float f0 = bs[t0] * (kpart ? Gam[t0] : 1.f);
          const float f1 = bs[t1] * (kpart ? Gam[t1] : 1.f);
#pragma unroll
          for (int n = 0; n < NTW; ++n) {
            const int ch = (col0 >> 3) + n;
            const float2 v0 = F16<__half>::unpack(ld_smem_u32(srcBp + sw_off(t0, ch, RB) + 4 * c));
            const float2 v1 = F16<__half>::unpack(ld_smem_u32(srcBp + sw_off(t1, ch, RB) + 4 * c));
            y[n][0] = f0 * v0.x;
            y[n][1] = f0 * v0.y;
            y[n][2] = f1 * v1.x;
            y[n][3] = f1 * v1.y;
          }
#pragma unroll
          for (int j = 0; j < i; ++j) {
            uint32_t a[4];
            ldmatrix_x4(a, sLN + sw_off(i * 16 + (mi & 1) * 8 + lr, j * 2 + (mi >> 1), 128));
#pragma unroll
            for (int n = 0; n < NTW; ++n) mma_f16_16816(y[n], a, xb[j][n]);
          }
          uint32_t yb[NTW][2];
#pragma unroll
          for (int n = 0; n < NTW; ++n) {
            yb[n][0] = movmatrix_trans(pack_f16(y[n][0], y[n][1]));
            yb[n][1] = movmatrix_trans(pack_f16(y[n][2], y[n][3]));
          }
          uint32_t a[4];
          ldmatrix_x4(a, sTD + sw_off(i * 16 + (mi & 1) * 8 + lr, i * 2 + (mi >> 1), 128));
#pragma unroll
          for (int n = 0; n < NTW; ++n) {
            float x[4] = {0.f, 0.f, 0.f, 0.f};
            mma_f16_16816(x, a, yb[n]);
            if (i < 3) {
              xb[i < 3 ? i : 0][n][0] = movmatrix_trans(pack_f16(x[0], x[1]));
              xb[i < 3 ? i : 0][n][1] = movmatrix_trans(pack_f16(x[2], x[3]));
            }
            const int ch = (col0 >> 3) + n;
            *reinterpret_cast<uint32_t*>(dst + sw_off(t0, ch, RB) + 4 * c) = pack_f16(sgn * x[0], sgn * x[1]);
            *reinterpret_cast<uint32_t*>(dst + sw_off(t1, ch, RB) + 4 * c) = pack_f16(sgn * x[2], sgn * x[3]);
          }
        }
      }
      mbar_arrive(&bars[b]);
    }
  }
}

// ------------------------------------------------------------------ launchers
static int check_gdn(const GdnLaunch& g) {
  if (!g.mix || !g.conv_state || !g.kbuf || !g.vbuf || !g.gbuf || !g.conv_w || !g.A_log ||
      !g.dt_bias)
    return KVA_ERR_INVALID_ARG;
  if (g.d_k != g.d_v || (g.d_k != 64 && g.d_k != 128)) return KVA_ERR_UNSUPPORTED;
  if (g.n_k <= 0 || g.n_v % g.n_k) return KVA_ERR_UNSUPPORTED;
  if (g.C % 128 || (g.n_k * g.d_k) % 128) return KVA_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(g.mix) | reinterpret_cast<uintptr_t>(g.conv_state) |
       reinterpret_cast<uintptr_t>(g.conv_w)) & 15u)
    return KVA_ERR_ALIGNMENT;
  if (g.mix_ld % 8) return KVA_ERR_ALIGNMENT;
  return KVA_OK;
}

int launch_gdn_prepare(const GdnLaunch& g, cudaStream_t s) {
  if (g.T == 0 || g.n_gdn == 0 || g.n_seq == 0) return KVA_OK;
  int e = check_gdn(g);
  if (e) return e;
  // channel blocks vary fastest, so the blocks in flight read whole row segments
  dim3 grid((g.C + PREP_CH - 1) / PREP_CH + 1, (g.T + PREP_TT - 1) / PREP_TT, g.n_seq * g.n_gdn);
  cudaError_t r;
  if (g.mix_dtype == KVA_F16)
    r = launch_pdl(gdn_prepare_kernel<__half>, grid, dim3(PREP_THREADS), 0, s, g);
  else if (g.mix_dtype == KVA_BF16)
    r = launch_pdl(gdn_prepare_kernel<__nv_bfloat16>, grid, dim3(PREP_THREADS), 0, s, g);
  else
    return KVA_ERR_INVALID_ARG;
  return r == cudaSuccess ? KVA_OK : KVA_ERR_CUDA;
}

int launch_gdn_tail(const GdnLaunch& g, cudaStream_t s) {
  if (g.T == 0 || g.n_gdn == 0 || g.n_seq == 0) return KVA_OK;
  int e = check_gdn(g);
  if (e) return e;
  dim3 grid((g.C + 255) / 256, g.n_seq * g.n_gdn);
  return launch_pdl(gdn_tail_kernel, grid, dim3(256), 0, s, g) == cudaSuccess ? KVA_OK : KVA_ERR_CUDA;
}

// ------------------------------------------------------------------ after the fused heads GEMM
// The heads GEMM's state-update epilogue (kva_gemm.cu) convolves every token whose 3
// predecessors lie in the same 128-token block.  The first 3 tokens of each block are
// done here from the raw rows it kept around block edges (and the old conv tail for
// block 0): the same conv + SiLU + L2 norm as gdn_prepare_kernel.  Grid (block, layer,
// 2048-channel group of the k | v channels), 8 channels per thread.
template <typename TM>
__global__ void __launch_bounds__(256) gdn_halo_fix_kernel(const MixParams mp, const void* conv_state) {
  griddep_wait_and_release();
  const int b = blockIdx.x, layer = blockIdx.y;
  const int nkdk = mp.n_k * 128;
  const int c0 = nkdk + blockIdx.z * 2048 + threadIdx.x * 8;  // conv channel (k or v)
  const int C = mp.C;
  const bool active = c0 < C;
  const int cc = active ? c0 : nkdk;
  const TM* halo = static_cast<const TM*>(mp.halo);
  const TM* tail = static_cast<const TM*>(conv_state) + static_cast<int64_t>(layer) * 3 * C;
  auto raw = [&](int u) {  // raw row u (>= -3) of [old tail; X] for these 8 channels
    const TM* src;
    if (u >= 128 * b) src = halo + ((static_cast<int64_t>(layer) * mp.nblk + b) * kMixHaloRows + (u - 128 * b)) * C;
    else if (u >= 0) src = halo + ((static_cast<int64_t>(layer) * mp.nblk + b - 1) * kMixHaloRows + (u - 128 * b + 6)) * C;
    else src = tail + static_cast<int64_t>(u + 3) * C;
    return *reinterpret_cast<const uint4*>(src + cc);
  };
  float w[8][4];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float4 wv = *reinterpret_cast<const float4*>(mp.conv_w + (static_cast<int64_t>(layer) * C + cc + e) * 4);
    w[e][0] = wv.x;
    w[e][1] = wv.y;
    w[e][2] = wv.z;
    w[e][3] = wv.w;
  }
  const bool is_k = c0 < 2 * nkdk;
#pragma unroll 1
  for (int i = 0; i < 3; ++i) {
    const int t = 128 * b + i;
    if (t >= mp.T) break;  // uniform over the block
    float x[4][8];
#pragma unroll
    for (int j = 0; j < 4; ++j) unpack8<TM>(raw(t - 3 + j), x[j]);
    float z[8];
#pragma unroll
    for (int e = 0; e < 8; ++e)
      z[e] = silu_tanh(w[e][0] * x[0][e] + w[e][1] * x[1][e] + w[e][2] * x[2][e] + w[e][3] * x[3][e]);
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) ss += z[e] * z[e];
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);  // 16 lanes = one head
    if (is_k) {
      const float sc = rsqrtf(ss + mp.eps);
#pragma unroll
      for (int e = 0; e < 8; ++e) z[e] *= sc;
    }
    if (active) {
      uint4 hv;
      hv.x = pack_f16(z[0], z[1]);
      hv.y = pack_f16(z[2], z[3]);
      hv.z = pack_f16(z[4], z[5]);
      hv.w = pack_f16(z[6], z[7]);
      const int64_t row = static_cast<int64_t>(layer) * mp.T + t;
      if (is_k)
        *reinterpret_cast<uint4*>(static_cast<__half*>(mp.kbuf) + row * nkdk + (c0 - nkdk)) = hv;
      else
        *reinterpret_cast<uint4*>(static_cast<__half*>(mp.vbuf) + row * (C - 2 * nkdk) + (c0 - 2 * nkdk)) = hv;
    }
  }
}

// New conv tail from the last raw rows the fused epilogue kept (raw row T-3+i, or old
// tail row T+i when T < 3); ascending i reads only rows not yet overwritten.
__global__ void gdn_tail_fused_kernel(const MixParams mp, void* conv_state) {
  griddep_wait_and_release();
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= mp.C) return;
  const int layer = blockIdx.y;
  const uint16_t* tn = static_cast<const uint16_t*>(mp.tail_new) + static_cast<int64_t>(layer) * 3 * mp.C + c;
  uint16_t* tail = static_cast<uint16_t*>(conv_state) + static_cast<int64_t>(layer) * 3 * mp.C + c;
  for (int i = 0; i < 3; ++i) {
    const int u = mp.T - 3 + i;
    tail[i * mp.C] = u >= 0 ? tn[i * mp.C] : tail[(mp.T + i) * mp.C];
  }
}

int launch_gdn_halo_fix(const MixParams& mp, int n_gdn, cudaStream_t s, int dtype, const void* conv_state) {
  if (mp.T == 0 || n_gdn == 0) return KVA_OK;
  const int nkdk = mp.n_k * 128;
  if ((mp.C - nkdk) % 8 || nkdk % 128) return KVA_ERR_UNSUPPORTED;
  dim3 grid((mp.T + 127) / 128, n_gdn, (mp.C - nkdk + 2047) / 2048);
  const cudaError_t r =
      dtype == KVA_F16 ? launch_pdl(gdn_halo_fix_kernel<__half>, grid, dim3(256), 0, s, mp, conv_state)
                       : launch_pdl(gdn_halo_fix_kernel<__nv_bfloat16>, grid, dim3(256), 0, s, mp, conv_state);
  return r == cudaSuccess ? KVA_OK : KVA_ERR_CUDA;
}

int launch_gdn_tail_fused(const MixParams& mp, int n_gdn, void* conv_state, cudaStream_t s) {
  if (mp.T == 0 || n_gdn == 0) return KVA_OK;
  dim3 grid((mp.C + 255) / 256, n_gdn);
  return launch_pdl(gdn_tail_fused_kernel, grid, dim3(256), 0, s, mp, conv_state) == cudaSuccess
             ? KVA_OK
             : KVA_ERR_CUDA;
}

template <int D>
static int launch_scan_d(const GdnLaunch& g, cudaStream_t s) {
  constexpr int bytes = ScanLayout<D>::BYTES;
  if (cudaFuncSetAttribute(gdn_scan_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           bytes) != cudaSuccess)
    return KVA_ERR_CUDA;
  dim3 grid(g.n_v, g.n_gdn, g.n_seq);
  return launch_pdl(gdn_scan_kernel<D>, grid, dim3(ScanLayout<D>::NT), bytes, s, g) == cudaSuccess
             ? KVA_OK
             : KVA_ERR_CUDA;
}

int launch_gdn_scan(const GdnLaunch& g, cudaStream_t s) {
  if (g.T == 0 || g.n_gdn == 0 || g.n_seq == 0) return KVA_OK;
  int e = check_gdn(g);
  if (e) return e;
  if (!g.state) return KVA_ERR_INVALID_ARG;
  return g.d_k == 128 ? launch_gdn_scan_tc(g, s) : launch_scan_d<64>(g, s);
}

}  // namespace kva
