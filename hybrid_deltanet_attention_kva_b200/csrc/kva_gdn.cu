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
//    One CTA per (sequence, layer, v head); warp w owns state rows
//    [16w, 16w+16) as mma.sync accumulators, so the state-dependent products
//    (U and the update) are warp-local; K K^T, Tm and W = Tm diag(beta e^gam) K
//    are shared per chunk.  Chunk contractions run on tensor cores with fp16
//    operands (every operand is bounded: unit keys, SiLU values, the inverse,
//    the state) and fp32 accumulation; the state stays fp32.
#include "kva_common.cuh"

namespace kva {

// ------------------------------------------------------------------ prepare
// Each thread owns 8 consecutive channels (one 16-byte vector per token row) for
// PREP_TT tokens: all raw rows are loaded up front, the conv runs in registers,
// and the L2 norm of a q/k head is a shuffle reduction over the d_k/8 lanes that
// hold it.  Blocks along x cover 2048 channels of one row, the last x-block of a
// token group computes the gates.
constexpr int PREP_TT = 16;
constexpr int PREP_THREADS = 256;
constexpr int PREP_CH = PREP_THREADS * 8;

template <typename TM>
__global__ void __launch_bounds__(PREP_THREADS) gdn_prepare_kernel(const GdnLaunch p) {
  const int slot = blockIdx.z;  // seq * n_gdn + layer
  const int seq = slot / p.n_gdn, layer = slot % p.n_gdn;
  const int T = p.T;
  const int t0 = blockIdx.y * PREP_TT;
  const int nt = min(PREP_TT, T - t0);
  const int C = p.C;
  const int nkdk = p.n_k * p.d_k;
  const TM* mix = static_cast<const TM*>(p.mix) + seq * p.mix_seq_stride + p.layer_col[layer];
  const int64_t ld = p.mix_ld;
  const int n_cblk = (C + PREP_CH - 1) / PREP_CH;

  if (static_cast<int>(blockIdx.x) < n_cblk) {
    const int c0 = blockIdx.x * PREP_CH + threadIdx.x * 8;
    const bool active = c0 < C;
    const int cc = active ? c0 : 0;
    const TM* tail = static_cast<const TM*>(p.conv_state) + static_cast<int64_t>(slot) * 3 * C + cc;
    // raw rows t0-3 .. t0+PREP_TT-1 of [tail; X] for these 8 channels
    uint4 raw[PREP_TT + 3];
#pragma unroll
    for (int i = 0; i < PREP_TT + 3; ++i) {
      const int t = t0 - 3 + i;
      if (t < 0)
        raw[i] = *reinterpret_cast<const uint4*>(tail + (t + 3) * C);
      else if (t < T)
        raw[i] = *reinterpret_cast<const uint4*>(mix + t * ld + cc);
      else
        raw[i] = make_uint4(0u, 0u, 0u, 0u);
    }
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
#pragma unroll
    for (int i = 0; i < PREP_TT; ++i) {
      float z[8];
#pragma unroll
      for (int e = 0; e < 8; e += 2) {
        float2 x0 = F16<TM>::unpack((&raw[i].x)[e / 2]);
        float2 x1 = F16<TM>::unpack((&raw[i + 1].x)[e / 2]);
        float2 x2 = F16<TM>::unpack((&raw[i + 2].x)[e / 2]);
        float2 x3 = F16<TM>::unpack((&raw[i + 3].x)[e / 2]);
        z[e] = silu_f(w[e][0] * x0.x + w[e][1] * x1.x + w[e][2] * x2.x + w[e][3] * x3.x);
        z[e + 1] = silu_f(w[e + 1][0] * x0.y + w[e + 1][1] * x1.y + w[e + 1][2] * x2.y +
                          w[e + 1][3] * x3.y);
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

// byte offset of (row, 16-byte chunk) in a bf16 tile whose rows are `rb` bytes
__device__ __forceinline__ uint32_t sw_off(int row, int chunk, int rb) {
  return static_cast<uint32_t>(row * rb + ((chunk ^ (row & 7)) << 4));
}

template <int D>
struct ScanSmem {
  static constexpr int KV_BYTES = SCAN_CH * D * 2;
  static constexpr int TB_BYTES = SCAN_CH * SCAN_CH * 2;
  static constexpr int LD = SCAN_CH + 1;
  static constexpr int F_BYTES = SCAN_CH * LD * 4;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + KV_BYTES;
  static constexpr int OFF_W = OFF_V + KV_BYTES;
  static constexpr int OFF_TB = OFF_W + KV_BYTES;
  static constexpr int OFF_TBG = OFF_TB + TB_BYTES;
  static constexpr int OFF_L = OFF_TBG + TB_BYTES;
  static constexpr int OFF_T = OFF_L + F_BYTES;
  static constexpr int OFF_M = OFF_T + F_BYTES;
  static constexpr int OFF_VEC = OFF_M + 3 * 256 * 4;
  static constexpr int BYTES = OFF_VEC + 5 * SCAN_CH * 4;
};

template <int D>
__global__ void __launch_bounds__(2 * D) gdn_scan_kernel(const GdnLaunch p) {
  constexpr int NW = D / 16;
  constexpr int NT = NW * 32;
  constexpr int RB = 2 * D;  // bytes per K/V/W row
  using SM = ScanSmem<D>;
  extern __shared__ __align__(128) uint8_t sm[];
  const uint32_t sK = smem_u32(sm + SM::OFF_K);
  const uint32_t sV = smem_u32(sm + SM::OFF_V);
  const uint32_t sW = smem_u32(sm + SM::OFF_W);
  const uint32_t sTB = smem_u32(sm + SM::OFF_TB);
  const uint32_t sTBG = smem_u32(sm + SM::OFF_TBG);
  float* Lf = reinterpret_cast<float*>(sm + SM::OFF_L);
  float* Tf = reinterpret_cast<float*>(sm + SM::OFF_T);
  float* Mf = reinterpret_cast<float*>(sm + SM::OFF_M);
  float* gs = reinterpret_cast<float*>(sm + SM::OFF_VEC);
  float* bs = gs + SCAN_CH;
  float* gam = bs + SCAN_CH;
  float* Gam = gam + SCAN_CH;
  float* dec = Gam + SCAN_CH;
  constexpr int LD = SM::LD;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c = lane & 3, mi = lane >> 3, lr = lane & 7;
  const int h = blockIdx.x, layer = blockIdx.y, seq = blockIdx.z;
  const int n_v = p.n_v;
  const int kh = h / (n_v / p.n_k);
  const int T = p.T;
  const int slot = seq * p.n_gdn + layer;
  const int nkdk = p.n_k * D, nvdv = n_v * D;
  const __half* kg =
      static_cast<const __half*>(p.kbuf) + static_cast<int64_t>(slot) * T * nkdk + kh * D;
  const __half* vg =
      static_cast<const __half*>(p.vbuf) + static_cast<int64_t>(slot) * T * nvdv + h * D;
  const float* gg = p.gbuf + static_cast<int64_t>(slot) * 2 * n_v * T + h * T;
  const float* bg = gg + static_cast<int64_t>(n_v) * T;
  float* Sg = p.state + (static_cast<int64_t>(slot) * n_v + h) * D * D;

  // state rows r0 = 16w + g and r0 + 8, as m16n8 accumulator fragments
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

  const int n_chunks = (T + SCAN_CH - 1) / SCAN_CH;
  for (int ci = 0; ci < n_chunks; ++ci) {
    const int c0 = ci * SCAN_CH;
    // (1) K, V rows of the chunk (zero past T), g and beta (0 past T: identity steps)
    for (int i = tid; i < SCAN_CH * (D / 8); i += NT) {
      const int r = i / (D / 8), ch = i % (D / 8);
      const int t = c0 + r;
      const bool ok = t < T;
      const int64_t tt = ok ? t : 0;
      cp_async16(sK + sw_off(r, ch, RB), kg + tt * nkdk + ch * 8, ok ? 16u : 0u);
      cp_async16(sV + sw_off(r, ch, RB), vg + tt * nvdv + ch * 8, ok ? 16u : 0u);
    }
    cp_async_commit();
    if (tid < SCAN_CH) {
      const int t = c0 + tid;
      gs[tid] = t < T ? gg[t] : 0.f;
      bs[tid] = t < T ? bg[t] : 0.f;
    }
    cp_async_wait<0>();
    __syncthreads();

    // (2) A = K K^T tiles of this warp; warp 0 also forms the cumulative decays
    constexpr int NPW = 32 / NW;  // n-tiles (of 8) per warp
    const int mt_a = warp & 3;
    const int nb_a = (warp >> 2) * NPW;
    float acc[NPW][4];
#pragma unroll
    for (int j = 0; j < NPW; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      uint32_t a[4];
      ldmatrix_x4(a, sK + sw_off(mt_a * 16 + (mi & 1) * 8 + lr, ks * 2 + (mi >> 1), RB));
#pragma unroll
      for (int j = 0; j < NPW; j += 2) {
        uint32_t b[4];
        ldmatrix_x4(b, sK + sw_off((nb_a + j) * 8 + (mi >> 1) * 8 + lr, ks * 2 + (mi & 1), RB));
        uint32_t b0[2] = {b[0], b[1]}, b1[2] = {b[2], b[3]};
        mma_f16_16816(acc[j], a, b0);
        mma_f16_16816(acc[j + 1], a, b1);
      }
    }
    if (warp == 0) {
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
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < NPW; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int t = mt_a * 16 + g + (e >> 1) * 8;
        const int s = (nb_a + j) * 8 + 2 * c + (e & 1);
        Lf[t * LD + s] = s < t ? bs[t] * expf(gam[t] - gam[s]) * acc[j][e] : 0.f;
      }
    }
    __syncthreads();

    // (3) Tm = (I + L)^-1 by 16x16 blocks: diagonal blocks by substitution ...
    if (tid < 64) {
      const int base = (tid >> 4) * 16, col = tid & 15;
      for (int r = 0; r < 16; ++r) {
        float v;
        if (r < col) {
          v = 0.f;
        } else if (r == col) {
          v = 1.f;
        } else {
          float s = 0.f;
          for (int q = col; q < r; ++q) s += Lf[(base + r) * LD + base + q] * Tf[(base + q) * LD + base + col];
          v = -s;
        }
        Tf[(base + r) * LD + base + col] = v;
      }
    }
    __syncthreads();
    // ... then block rows i = 1..3: T_ij = -T_ii sum_{k=j}^{i-1} L_ik T_kj
    for (int i = 1; i < 4; ++i) {
      for (int o = tid; o < i * 256; o += NT) {
        const int j = o >> 8, e = o & 255, r = e >> 4, cc = e & 15;
        float s = 0.f;
        for (int k = j; k < i; ++k)
#pragma unroll
          for (int q = 0; q < 16; ++q)
            s += Lf[(16 * i + r) * LD + 16 * k + q] * Tf[(16 * k + q) * LD + 16 * j + cc];
        Mf[o] = s;
      }
      __syncthreads();
      for (int o = tid; o < i * 256; o += NT) {
        const int j = o >> 8, e = o & 255, r = e >> 4, cc = e & 15;
        float s = 0.f;
#pragma unroll
        for (int q = 0; q < 16; ++q) s += Tf[(16 * i + r) * LD + 16 * i + q] * Mf[(j << 8) + q * 16 + cc];
        Tf[(16 * i + r) * LD + 16 * j + cc] = -s;
      }
      __syncthreads();
    }

    // (4) TB = Tm diag(beta), TBG = Tm diag(beta e^gam) as bf16 (zero above the block diagonal)
    for (int o = tid; o < SCAN_CH * SCAN_CH / 2; o += NT) {
      const int t = o >> 5, s = (o & 31) * 2;
      const bool upper = (s >> 4) > (t >> 4);
      const float x0 = upper ? 0.f : Tf[t * LD + s];
      const float x1 = upper ? 0.f : Tf[t * LD + s + 1];
      const float b0 = bs[s], b1 = bs[s + 1];
      const uint32_t off = static_cast<uint32_t>(t * 128 + (((s >> 3) ^ (t & 7)) << 4) + (s & 7) * 2);
      *reinterpret_cast<uint32_t*>(sm + SM::OFF_TB + off) = pack_f16(x0 * b0, x1 * b1);
      *reinterpret_cast<uint32_t*>(sm + SM::OFF_TBG + off) =
          pack_f16(x0 * b0 * Gam[s], x1 * b1 * Gam[s + 1]);
    }
    __syncthreads();

    // (5) this warp's columns [16w, 16w+16): U = TB V (initial value of U) and
    //     W = TBG K, stored negated for everyone
    float U[4][2][4];
    {
      float Wt[4][2][4];
#pragma unroll
      for (int m = 0; m < 4; ++m)
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) U[m][n][e] = Wt[m][n][e] = 0.f;
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        uint32_t bv[4], bk[4];
        const int row = ks * 16 + (mi & 1) * 8 + lr;
        const int ch = warp * 2 + (mi >> 1);
        ldmatrix_x4_trans(bv, sV + sw_off(row, ch, RB));
        ldmatrix_x4_trans(bk, sK + sw_off(row, ch, RB));
        uint32_t bv0[2] = {bv[0], bv[1]}, bv1[2] = {bv[2], bv[3]};
        uint32_t bk0[2] = {bk[0], bk[1]}, bk1[2] = {bk[2], bk[3]};
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          uint32_t a[4], ag[4];
          const uint32_t off = sw_off(m * 16 + (mi & 1) * 8 + lr, ks * 2 + (mi >> 1), 128);
          ldmatrix_x4(a, sTB + off);
          ldmatrix_x4(ag, sTBG + off);
          mma_f16_16816(U[m][0], a, bv0);
          mma_f16_16816(U[m][1], a, bv1);
          mma_f16_16816(Wt[m][0], ag, bk0);
          mma_f16_16816(Wt[m][1], ag, bk1);
        }
      }
#pragma unroll
      for (int m = 0; m < 4; ++m)
#pragma unroll
        for (int n = 0; n < 2; ++n) {
          const int ch = warp * 2 + n;
          const int r0 = m * 16 + g;
          *reinterpret_cast<uint32_t*>(sm + SM::OFF_W + sw_off(r0, ch, RB) + 4 * c) =
              pack_f16(-Wt[m][n][0], -Wt[m][n][1]);
          *reinterpret_cast<uint32_t*>(sm + SM::OFF_W + sw_off(r0 + 8, ch, RB) + 4 * c) =
              pack_f16(-Wt[m][n][2], -Wt[m][n][3]);
        }
    }
    __syncthreads();

    // (6) U += (-W) S^T, the B operand taken straight from this warp's state rows
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

    // (7) S <- e^gam_last S + (dec U)^T K
    {
      const float gl = Gam[SCAN_CH - 1];
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
          uint32_t b[4];
          ldmatrix_x4_trans(b, sK + sw_off(m * 16 + (mi & 1) * 8 + lr, nt + (mi >> 1), RB));
          uint32_t b0[2] = {b[0], b[1]}, b1[2] = {b[2], b[3]};
          mma_f16_16816(S[nt], a, b0);
          mma_f16_16816(S[nt + 1], a, b1);
        }
      }
    }
    __syncthreads();
  }

  {
    float* s0 = Sg + (16 * warp + g) * D + 2 * c;
    float* s1 = s0 + 8 * D;
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt) {
      *reinterpret_cast<float2*>(s0 + 8 * nt) = make_float2(S[nt][0], S[nt][1]);
      *reinterpret_cast<float2*>(s1 + 8 * nt) = make_float2(S[nt][2], S[nt][3]);
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
  if (g.mix_dtype == KVA_F16)
    gdn_prepare_kernel<__half><<<grid, PREP_THREADS, 0, s>>>(g);
  else if (g.mix_dtype == KVA_BF16)
    gdn_prepare_kernel<__nv_bfloat16><<<grid, PREP_THREADS, 0, s>>>(g);
  else
    return KVA_ERR_INVALID_ARG;
  return cudaPeekAtLastError() == cudaSuccess ? KVA_OK : KVA_ERR_CUDA;
}

int launch_gdn_tail(const GdnLaunch& g, cudaStream_t s) {
  if (g.T == 0 || g.n_gdn == 0 || g.n_seq == 0) return KVA_OK;
  int e = check_gdn(g);
  if (e) return e;
  dim3 grid((g.C + 255) / 256, g.n_seq * g.n_gdn);
  gdn_tail_kernel<<<grid, 256, 0, s>>>(g);
  return cudaPeekAtLastError() == cudaSuccess ? KVA_OK : KVA_ERR_CUDA;
}

template <int D>
static int launch_scan_d(const GdnLaunch& g, cudaStream_t s) {
  constexpr int bytes = ScanSmem<D>::BYTES;
  if (cudaFuncSetAttribute(gdn_scan_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           bytes) != cudaSuccess)
    return KVA_ERR_CUDA;
  dim3 grid(g.n_v, g.n_gdn, g.n_seq);
  gdn_scan_kernel<D><<<grid, 2 * D, bytes, s>>>(g);
  return cudaPeekAtLastError() == cudaSuccess ? KVA_OK : KVA_ERR_CUDA;
}

int launch_gdn_scan(const GdnLaunch& g, cudaStream_t s) {
  if (g.T == 0 || g.n_gdn == 0 || g.n_seq == 0) return KVA_OK;
  int e = check_gdn(g);
  if (e) return e;
  if (!g.state) return KVA_ERR_INVALID_ARG;
  return g.d_k == 128 ? launch_scan_d<128>(g, s) : launch_scan_d<64>(g, s);
}

}  // namespace kva
