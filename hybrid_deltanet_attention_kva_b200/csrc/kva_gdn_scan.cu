// Gated delta-rule scan for 128-dimensional heads on the fifth-generation tensor
// cores (the deltanet scan of the "Qwen3.8-27B-KVA" model card, section "What the
// hell?", run on the approximated q/k/v and gates):
//     S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
// in chunks of 64 tokens, emitting only the final state.  With the local
// cumulative decay gam_t = sum_{s<=t} g_s of a chunk,
//     L[t,s] = beta_t e^(gam_t-gam_s) k_t.k_s (s < t),   Tm = (I + L)^-1,
//     B1     = diag(e^(gam_last-gam)) Tm diag(beta),
//     D      = (V^T - S K^T diag(e^gam)) B1^T            (= (dec U)^T, v x t),
//     S     <- e^gam_last S + D K.
// (U = Tm diag(beta) (V - diag(e^gam) K S^T) is the chunk's corrected value
// matrix; D folds its row decays and beta into B1.)
//
// Two kernels:
// 1. gdn_chunk_prep_kernel, fully parallel over (value head, chunk, layer): B1 and
//    the chunk's scalars {e^gam[64], e^gam_last}.  Nothing here depends on the
//    state.  K K^T and the 16 x 16 block products run on mma.sync; the diagonal
//    blocks of Tm are solved in fp32.
// 2. gdn_scan_tc_kernel, one CTA per (sequence, layer, value head), two CTAs per
//    SM: the state S (128 x 128 fp32) lives in tensor memory for the whole ubatch,
//    TMEM lane v holding state row v.  Per chunk, eight warps (two per TMEM lane
//    quarter, each owning half of the columns) and one elected lane of warp 0 run
//        pass 1: A <- fp16(S)                            (tcgen05.ld / st)
//        MMA   : Y  = A K^T             | S <- e^gam_last S meanwhile
//        pass 2: A <- fp16(V^T - Y diag(e^gam))          (V rows read from shared memory)
//        MMA   : D  = A B1^T
//        pass 3: A <- fp16(D)
//        MMA   : S += A K                                (K as an MN-major operand)
//    Rounding V^T - Y diag(e^gam) once (the chunk's corrected values before B1) keeps
//    the round to four instructions.  K, V and B1 of the next chunk arrive by TMA,
//    issued by one thread of warp 1 while the tensor cores form Y.  Every wait
//    is bounded; on a timeout the block raises its abort flag, runs the remaining
//    steps without waiting or issuing, drains its own copies and MMAs, and returns
//    with the device status set.
#include "kva_common.cuh"

namespace kva {
namespace {

constexpr int SD = 128;             // d_k = d_v
constexpr int SCH = 64;             // chunk length
constexpr int SC_FLOATS = 80;       // per chunk and head: e^gam[64], e^gam_last, padding
constexpr int B1_BYTES = SCH * SCH * 2;

// byte offset of (row, 16-byte chunk c16 in 0..15) in a K chunk tile held as two
// [64][64] halves with the 128-byte swizzle
__device__ __forceinline__ uint32_t kv_off(int row, int c16) {
  return static_cast<uint32_t>((c16 >> 3) * (SCH * 64 * 2) + row * 128 +
                               (((c16 & 7) ^ (row & 7)) << 4));
}
// byte offset of (row, 16-byte chunk c8 in 0..7) in a [64][64] 16-bit tile
__device__ __forceinline__ uint32_t t64_off(int row, int c8) {
  return static_cast<uint32_t>(row * 128 + ((c8 ^ (row & 7)) << 4));
}
__device__ __forceinline__ uint32_t t64_elem(int row, int col) {
  return t64_off(row, col >> 3) + (col & 7) * 2;
}
__device__ __forceinline__ float u2f(uint32_t x) { return __uint_as_float(x); }

// ============================================================================
// chunk preparation
// ============================================================================
constexpr int LDB = 16 * 16 + 8;  // diagonal-block stride of the fp32 copies (floats)

// Shared-memory views of one chunk's preparation, worked by four warps (threads 0-127):
// warp w owns the 16 rows [16 w, 16 w + 16) of K K^T and L.
struct PrepView {
  uint32_t kb;      // K tile: two 128B-swizzled [64][64] halves (shared address)
  uint32_t sL;      // L below the diagonal blocks, Tm on them: [64][64] fp16, t64 layout
  uint8_t* L;       // the same tile, generic pointer
  uint8_t* B1;      // B1 tile [64][64] fp16, t64 layout; blocks above the diagonal stay zero
  float* Ld;        // the 4 diagonal blocks of L in fp32, stride LDB
  float* ab;        // decay factors a[64], b[1..3][64]
  float* gam;       // cumulative decay gam[64]
  float* dec;       // e^(gam_last - gam)[64]
  const float* gs;  // raw g[64] (0 past T)
  const float* bs;  // beta[64] (0 past T)
};

// (1) K K^T for the blocks on and below the diagonal: warp w, column tiles [0, 2 w + 2) of 8
__device__ __forceinline__ void prep_kkt(const PrepView& v, float (&acc)[8][4], int warp, int lane) {
  const int mi = lane >> 3, lr = lane & 7;
  const int mt = warp;
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
#pragma unroll
  for (int ks = 0; ks < SD / 16; ++ks) {
    uint32_t a[4];
    ldmatrix_x4(a, v.kb + kv_off(mt * 16 + (mi & 1) * 8 + lr, ks * 2 + (mi >> 1)));
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      if (jj > mt) continue;
      uint32_t bb[4];
      ldmatrix_x4(bb, v.kb + kv_off(jj * 16 + (mi >> 1) * 8 + lr, ks * 2 + (mi & 1)));
      const uint32_t b0[2] = {bb[0], bb[1]}, b1[2] = {bb[2], bb[3]};
      mma_f16_16816(acc[2 * jj], a, b0);
      mma_f16_16816(acc[2 * jj + 1], a, b1);
    }
  }
}

// (2) cumulative decays (one warp); the chain's scalars {e^gam[64], e^gam_last, 0...} go to
//     `scg` (SC_FLOATS floats, 8-byte aligned)
__device__ __forceinline__ void prep_decays(const PrepView& v, float* scg, int lane) {
  const float v0 = v.gs[2 * lane], v1 = v.gs[2 * lane + 1];
  const float pair = v0 + v1;
  float incl = pair;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const float ex = incl - pair;
  const float total = __shfl_sync(0xffffffffu, incl, 31);
  const float ga = ex + v0, gb2 = ex + pair;
  v.gam[2 * lane] = ga;
  v.gam[2 * lane + 1] = gb2;
  v.dec[2 * lane] = expf(total - ga);
  v.dec[2 * lane + 1] = expf(total - gb2);
  *reinterpret_cast<float2*>(scg + 2 * lane) = make_float2(expf(ga), expf(gb2));
  if (lane < (SC_FLOATS - SCH) / 2)
    *reinterpret_cast<float2*>(scg + SCH + 2 * lane) = make_float2(lane == 0 ? expf(total) : 0.f, 0.f);
  // below the diagonal blocks e^(gam_t - gam_s) = a_t b_i(s) with the reference
  // r_i = gam at the last token of block i - 1 (t in block i, s < 16 i): both
  // factors are at most 1, so neither overflows however strong the decay
  const int bi = lane >> 3;  // block of tokens 2 lane, 2 lane + 1
  float ref[4];
#pragma unroll
  for (int i = 1; i < 4; ++i) ref[i] = __shfl_sync(0xffffffffu, gb2, 8 * i - 1);
  ref[0] = 0.f;
  float rb = ref[1];
#pragma unroll
  for (int i = 2; i < 4; ++i) rb = bi == i ? ref[i] : rb;
  v.ab[2 * lane] = bi ? __expf(ga - rb) : 1.f;
  v.ab[2 * lane + 1] = bi ? __expf(gb2 - rb) : 1.f;
#pragma unroll
  for (int i = 1; i < 4; ++i) {
    const bool below = 2 * lane < 16 * i;
    v.ab[SCH * i + 2 * lane] = below ? __expf(ref[i] - ga) : 0.f;
    v.ab[SCH * i + 2 * lane + 1] = below ? __expf(ref[i] - gb2) : 0.f;
  }
}

// (3) L = beta_t e^(gam_t - gam_s) k_t.k_s below the diagonal: fp32 copies of the diagonal
//     blocks (direct exponentials), fp16 blocks below them (factored decays)
__device__ __forceinline__ void prep_l(const PrepView& v, const float (&acc)[8][4], int warp, int lane) {
  const int g = lane >> 2, cq = lane & 3, mt = warp;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int sb = j >> 1;
    if (sb > mt) continue;
    const int s0 = j * 8 + 2 * cq;
    if (sb == mt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int t = mt * 16 + g + (e >> 1) * 8;
        const int s = s0 + (e & 1);
        v.Ld[mt * LDB + (t & 15) * 16 + (s & 15)] =
            s < t ? v.bs[t] * __expf(v.gam[t] - v.gam[s]) * acc[j][e] : 0.f;
      }
    } else {
      const int t0 = mt * 16 + g;
      const float r0 = v.bs[t0] * v.ab[t0], r1 = v.bs[t0 + 8] * v.ab[t0 + 8];
      const float c0 = v.ab[SCH * mt + s0], c1 = v.ab[SCH * mt + s0 + 1];
      *reinterpret_cast<uint32_t*>(v.L + t64_elem(t0, s0)) = pack_f16(r0 * c0 * acc[j][0], r0 * c1 * acc[j][1]);
      *reinterpret_cast<uint32_t*>(v.L + t64_elem(t0 + 8, s0)) = pack_f16(r1 * c0 * acc[j][2], r1 * c1 * acc[j][3]);
    }
  }
}

// (4) diagonal blocks of Tm = (I + L)^-1 in fp32, one row per thread (threads 0-63): row r
//     of (I + L_b)^-1 solves x (I + L_b) = e_r; going from the last column down, x_p is
//     final when reached and is eliminated from every earlier column (the FMAs of one step
//     are independent).  Tm's blocks go to L's diagonal, B1's to B1.
__device__ __forceinline__ void prep_diag(const PrepView& v, int tid) {
  const int blk = tid >> 4, r = tid & 15;
  const float* Lb = v.Ld + blk * LDB;
  float x[16];
#pragma unroll
  for (int q = 0; q < 16; ++q) x[q] = q == r ? 1.f : 0.f;
#pragma unroll
  for (int q2 = 15; q2 >= 1; --q2) {
    float lrow[16];
#pragma unroll
    for (int v4 = 0; v4 < (q2 + 3) / 4; ++v4) {
      const float4 l4 = reinterpret_cast<const float4*>(Lb + q2 * 16)[v4];
      lrow[4 * v4] = l4.x;
      lrow[4 * v4 + 1] = l4.y;
      lrow[4 * v4 + 2] = l4.z;
      lrow[4 * v4 + 3] = l4.w;
    }
#pragma unroll
    for (int q = 0; q < q2; ++q) x[q] = fmaf(-x[q2], lrow[q], x[q]);
  }
  const int t = blk * 16 + r;
  const float dt = v.dec[t];
  const float* bb = v.bs + blk * 16;
  uint32_t tm[8], bv[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    tm[q] = pack_f16(x[2 * q], x[2 * q + 1]);
    bv[q] = pack_f16(dt * x[2 * q] * bb[2 * q], dt * x[2 * q + 1] * bb[2 * q + 1]);
  }
  *reinterpret_cast<uint4*>(v.L + t64_off(t, 2 * blk)) = make_uint4(tm[0], tm[1], tm[2], tm[3]);
  *reinterpret_cast<uint4*>(v.L + t64_off(t, 2 * blk + 1)) = make_uint4(tm[4], tm[5], tm[6], tm[7]);
  *reinterpret_cast<uint4*>(v.B1 + t64_off(t, 2 * blk)) = make_uint4(bv[0], bv[1], bv[2], bv[3]);
  *reinterpret_cast<uint4*>(v.B1 + t64_off(t, 2 * blk + 1)) = make_uint4(bv[4], bv[5], bv[6], bv[7]);
}

// (5) blocks below the diagonal by column block jb, 8 columns (half hf) per task:
//     X_ij = -Tm_ii sum_{k=jb}^{i-1} L_ik X_k,jb,  B1_ij = diag(dec) X_ij diag(beta).
//     Warps 0 and 1 take column block 0 (three block rows), warps 2 and 3 column blocks 1
//     then 2 (two and one).
__device__ __forceinline__ void prep_offdiag_task(const PrepView& v, int jb, int hf, int lane) {
  const int g = lane >> 2, cq = lane & 3, mi = lane >> 3, lr = lane & 7;
  const int s0 = 16 * jb + 8 * hf;
  const int s = s0 + 2 * cq;
  const float b0s = v.bs[s], b1s = v.bs[s + 1];
#pragma unroll
  for (int jj = 0; jj < 3; ++jj) {
    if (jj != jb) continue;
    uint32_t xf[4][2];
    ldmatrix_x2_trans(xf[jj], v.sL + t64_off(16 * jj + (mi & 1) * 8 + lr, s0 >> 3));
#pragma unroll
    for (int i = jj + 1; i < 4; ++i) {
      float y[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int k = jj; k < i; ++k) {
        uint32_t a[4];
        ldmatrix_x4(a, v.sL + t64_off(16 * i + (mi & 1) * 8 + lr, 2 * k + (mi >> 1)));
        mma_f16_16816(y, a, xf[k]);
      }
      const uint32_t yb[2] = {movmatrix_trans(pack_f16(y[0], y[1])), movmatrix_trans(pack_f16(y[2], y[3]))};
      uint32_t a[4];
      ldmatrix_x4(a, v.sL + t64_off(16 * i + (mi & 1) * 8 + lr, 2 * i + (mi >> 1)));
      float x[4] = {0.f, 0.f, 0.f, 0.f};
      mma_f16_16816(x, a, yb);
      const int ta = 16 * i + g, tb2 = ta + 8;
      const float d0 = v.dec[ta], d1 = v.dec[tb2];
      *reinterpret_cast<uint32_t*>(v.B1 + t64_elem(ta, s)) = pack_f16(-d0 * x[0] * b0s, -d0 * x[1] * b1s);
      *reinterpret_cast<uint32_t*>(v.B1 + t64_elem(tb2, s)) = pack_f16(-d1 * x[2] * b0s, -d1 * x[3] * b1s);
      xf[i][0] = movmatrix_trans(pack_f16(-x[0], -x[1]));
      xf[i][1] = movmatrix_trans(pack_f16(-x[2], -x[3]));
    }
  }
}
__device__ __forceinline__ void prep_offdiag(const PrepView& v, int warp, int lane) {
  if (warp < 2) {
    prep_offdiag_task(v, 0, warp, lane);
  } else {
    prep_offdiag_task(v, 1, warp - 2, lane);
    prep_offdiag_task(v, 2, warp - 2, lane);
  }
}

struct Cp {
  static constexpr int THREADS = 128;
  static constexpr int K = 0;                      // K chunk tile, 16 KB; once K K^T is formed its
  static constexpr int B1 = K;                     //   space holds the B1 staging tile
  static constexpr int LD = K + SCH * SCH * 2;     //   and the diagonal blocks of L, fp32 (stride LDB)
  static constexpr int L = K + SCH * SD * 2;       // L below the diagonal blocks, Tm on them
  static constexpr int AB = L + SCH * SCH * 2;     // decay factors a[64], b[1..3][64]
  static constexpr int GAM = AB + 4 * SCH * 4;     // gam[64], decay[64]
  static constexpr int GB = GAM + 2 * SCH * 4;     // g[64], beta[64]
  static constexpr int BAR = GB + 2 * SCH * 4;
  static constexpr int BYTES = BAR + 16;
  static constexpr int ALLOC = BYTES + 1024;       // slack for 1024-byte alignment (TMA tile)
};

// grid (value head, chunk, sequence x layer in [l0, l0 + nl)): the value heads that share a key head
// are neighbours, so their K tile is read from L2.  4 warps; warp w owns the 16
// rows [16 w, 16 w + 16) of K K^T and L.
static_assert(Cp::LD + 4 * LDB * 4 <= Cp::L, "B1 and the diagonal blocks fit the K tile's space");
__global__ void __launch_bounds__(Cp::THREADS, 8)
    gdn_chunk_prep_kernel(const __grid_constant__ CUtensorMap mK, const GdnLaunch p, int l0, int nl) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint64_t* kbar = reinterpret_cast<uint64_t*>(sm + Cp::BAR);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x, c = blockIdx.y;
  const int slot = (blockIdx.z / nl) * p.n_gdn + l0 + blockIdx.z % nl;  // layers [l0, l0 + nl)
  const int T = p.T, n_v = p.n_v;
  const int kh = h / (n_v / p.n_k);
  const int n_chunks = (T + SCH - 1) / SCH;
  const int t0c = c * SCH;
  const int64_t head = static_cast<int64_t>(slot) * n_v + h;

  float* gam = reinterpret_cast<float*>(sm + Cp::GAM);
  float* dec = gam + SCH;
  float* Ld = reinterpret_cast<float*>(sm + Cp::LD);
  float* ab = reinterpret_cast<float*>(sm + Cp::AB);
  float* gs = reinterpret_cast<float*>(sm + Cp::GB);
  float* bs = gs + SCH;
  uint8_t* B1 = sm + Cp::B1;
  const uint32_t sL = smem_u32(sm + Cp::L);
  const uint32_t kb = smem_u32(sm + Cp::K);
  griddep_wait_and_release();  // K, g and beta come from the kernels before

  // K rows of the chunk, raw g and beta (zero past T: identity steps)
  if (tid == 0) {
    mbar_init(kbar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(kbar, SCH * SD * 2);
    tma_load_3d(sm + Cp::K, &mK, kbar, kh * SD, t0c, slot, l2_policy_evict_normal());
    tma_load_3d(sm + Cp::K + SCH * 64 * 2, &mK, kbar, kh * SD + 64, t0c, slot,
                l2_policy_evict_normal());
  }
  {
    const int t = t0c + (tid & (SCH - 1));
    const float* src =
        p.gbuf + (static_cast<int64_t>(slot) * 2 * n_v + (tid < SCH ? 0 : n_v) + h) * T;
    gs[tid] = t < T ? src[t] : 0.f;
  }
  __syncthreads();  // the barrier is initialised before anyone waits on it
  // every thread waits for the K tile (the load always completes: rows past T are
  // zero-filled); on a timeout the status is set and the block carries on
  if (!mbar_wait_limit(kbar, 0)) set_device_error(p.err, KVA_DEV_WAIT_TIMEOUT);

  const PrepView v{kb, sL, sm + Cp::L, B1, Ld, ab, gam, dec, gs, bs};
  float acc[8][4];
  prep_kkt(v, acc, warp, lane);
  if (warp == 0) prep_decays(v, p.scbuf + (head * n_chunks + c) * SC_FLOATS, lane);
  __syncthreads();  // K is read: its space takes B1 (from zero: the blocks above the diagonal
                    // stay zero) and the diagonal blocks of L
  for (int i = tid; i < B1_BYTES / 16; i += Cp::THREADS)
    reinterpret_cast<uint4*>(B1)[i] = make_uint4(0u, 0u, 0u, 0u);
  prep_l(v, acc, warp, lane);
  __syncthreads();
  if (tid < 64) prep_diag(v, tid);
  __syncthreads();
  prep_offdiag(v, warp, lane);
  __syncthreads();
  // (6) B1 to global memory, row-major [64][64] (16-byte pieces, coalesced)
  uint8_t* dst = static_cast<uint8_t*>(p.b1buf) + (head * n_chunks + c) * B1_BYTES;
  for (int i = tid; i < B1_BYTES / 16; i += Cp::THREADS) {
    const int r = i >> 3, c8 = i & 7;
    *reinterpret_cast<uint4*>(dst + r * 128 + c8 * 16) =
        *reinterpret_cast<const uint4*>(B1 + t64_off(r, c8));
  }
}

// ============================================================================
// state chain
// ============================================================================
constexpr int N_W = 8;                  // warps: two per TMEM lane quarter
constexpr int NTHREADS = N_W * 32;
constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t COL_S = 0;    // state, fp32 128 x 128
constexpr uint32_t COL_A = 128;  // 16-bit A operand (up to 128 x 128)
constexpr uint32_t COL_Y = 192;  // Y, then D: fp32 128 x 64
constexpr int kLoader = 32;      // the thread (warp 1) that issues the chunk loads

struct Sc {
  static constexpr int KT = SCH * SD * 2;     // K or V chunk: two [64][64] 128B-swizzled halves
  static constexpr int HALF = SCH * 64 * 2;
  static constexpr int K = 0;                 // 2 slots each: chunk c in slot c & 1
  static constexpr int V = K + 2 * KT;
  static constexpr int B1 = V + 2 * KT;
  static constexpr int SCL = B1 + 2 * B1_BYTES;
  static constexpr int BAR = SCL + 2 * SC_FLOATS * 4;
  static constexpr int N_BAR = 6;             // full[2], ybar, dbar, done, drain
  static constexpr int MISC = BAR + N_BAR * 8;  // TMEM base, abort flag
  static constexpr int BYTES = MISC + 16;
  static constexpr int ALLOC = BYTES + 1024;  // slack for 1024-byte alignment
  static constexpr uint32_t LOAD_BYTES = 2 * KT + B1_BYTES + SC_FLOATS * 4;
};

constexpr uint32_t ID_Y = idesc_f16kind_f32_major(128, 64, 0, false, false);   // TMEM A, K-major B
constexpr uint32_t ID_S = idesc_f16kind_f32_major(128, 128, 0, false, true);   // MN-major B

__global__ void __launch_bounds__(NTHREADS, 2)
    gdn_scan_tc_kernel(const __grid_constant__ CUtensorMap mK, const __grid_constant__ CUtensorMap mV,
                       const __grid_constant__ CUtensorMap mB, const GdnLaunch p, int l0) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Sc::BAR);
  uint64_t* full = bars;       // [2] K, V, B1 and scalars of a chunk landed
  uint64_t* ybar = bars + 2;
  uint64_t* dbar = bars + 3;
  uint64_t* done = bars + 4;   // the chunk's last MMA completed
  uint64_t* drain = bars + 5;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + Sc::MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + Sc::MISC + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qd = warp & 3, hc = warp >> 2;  // TMEM lane quarter, column half
  const int h = blockIdx.x, layer = l0 + blockIdx.y, seq = blockIdx.z;
  const int n_v = p.n_v;
  const int kh = h / (n_v / p.n_k);
  const int T = p.T;
  const int slot = seq * p.n_gdn + layer;
  const int head = slot * n_v + h;
  const int n_chunks = (T + SCH - 1) / SCH;

  if (tid == 0) {
    for (int i = 0; i < Sc::N_BAR; ++i) mbar_init(&bars[i], 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&mK);
    tma_prefetch_desc(&mV);
    tma_prefetch_desc(&mB);
  }
  if (warp == 0) {
    tmem_alloc(tslot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = *tslot;
  griddep_wait_and_release();  // state, K, V and B1 come from the kernels before
  const uint32_t lrow = static_cast<uint32_t>(32 * qd) << 16;
  const uint32_t tS = tb + lrow + COL_S + 64 * hc;  // this thread's 64 state columns
  const uint32_t tA = tb + lrow + COL_A;
  const uint32_t tY = tb + lrow + COL_Y + 32 * hc;  // this thread's 32 Y / D columns
  float* Sg = p.state + static_cast<int64_t>(head) * SD * SD + (32 * qd + lane) * SD + 64 * hc;

  const uint64_t pol_k = l2_policy_evict_normal(), pol_v = l2_policy_evict_first();
  int issued = 0;  // chunks whose operands were requested (the loader thread)
  auto load = [&](int c) {
    const int s = c & 1;
    uint64_t* bar = &full[s];
    mbar_arrive_expect_tx(bar, Sc::LOAD_BYTES);
    uint8_t* k = sm + Sc::K + s * Sc::KT;
    uint8_t* v = sm + Sc::V + s * Sc::KT;
    tma_load_3d(k, &mK, bar, kh * SD, c * SCH, slot, pol_k);
    tma_load_3d(k + Sc::HALF, &mK, bar, kh * SD + 64, c * SCH, slot, pol_k);
    tma_load_3d(v, &mV, bar, h * SD, c * SCH, slot, pol_v);
    tma_load_3d(v + Sc::HALF, &mV, bar, h * SD + 64, c * SCH, slot, pol_v);
    tma_load_3d(sm + Sc::B1 + s * B1_BYTES, &mB, bar, 0, c * SCH, head, pol_v);
    bulk_load(sm + Sc::SCL + s * SC_FLOATS * 4,
              p.scbuf + (static_cast<int64_t>(head) * n_chunks + c) * SC_FLOATS, SC_FLOATS * 4, bar);
    issued = c + 1;
  };
  // the first chunk's operands are requested before the state is read, so the two overlap
  if (tid == kLoader) load(0);
  __syncwarp();
#pragma unroll 1
  for (int q = 0; q < 2; ++q) {
    uint32_t r[32];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float4 v = reinterpret_cast<const float4*>(Sg + 32 * q)[j];
      r[4 * j] = __float_as_uint(v.x);
      r[4 * j + 1] = __float_as_uint(v.y);
      r[4 * j + 2] = __float_as_uint(v.z);
      r[4 * j + 3] = __float_as_uint(v.w);
    }
    tmem_st_32x32b_x32(tS + 32 * q, r);
  }
  tmem_st_wait();

  // warp 0's issuing lane, elected once: a commit tracks only its own lane's MMAs
  const uint32_t issuer = warp == 0 ? elect_one() : 0u;
  bool ok = true;
  for (int c = 0; c < n_chunks; ++c) {
    const int s = c & 1;
    const float* sc = reinterpret_cast<const float*>(sm + Sc::SCL + s * SC_FLOATS * 4);
    if (!*abort_flag) ok &= mbar_wait(&full[s], (c >> 1) & 1, abort_flag);
    if (c > 0 && !*abort_flag) ok &= mbar_wait(done, (c - 1) & 1, abort_flag);
    tc_fence_after();
    const uint32_t kb = smem_u32(sm + Sc::K + s * Sc::KT);
    const uint64_t dKk = sdesc_k_sw128(kb), dKm = sdesc_mn_sw128(kb, Sc::HALF);

    // pass 1: A <- fp16(S); the state values stay in registers for the rescale
    uint32_t r0[32], r1[32];
    tmem_ld_32x32b_x32(tS, r0);
    tmem_ld_32x32b_x32(tS + 32, r1);
    tmem_ld_wait();
    {
      uint32_t a[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) a[j] = pack_f16(u2f(r0[2 * j]), u2f(r0[2 * j + 1]));
      tmem_st_32x32b_x16(tA + 32 * hc, a);
#pragma unroll
      for (int j = 0; j < 16; ++j) a[j] = pack_f16(u2f(r1[2 * j]), u2f(r1[2 * j + 1]));
      tmem_st_32x32b_x16(tA + 32 * hc + 16, a);
    }
    tmem_st_wait();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
      tc_fence_after();
      if (issuer && !*abort_flag) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
          umma_f16_ts(tb + COL_Y, tb + COL_A + 8 * j, dKk + (((j >> 2) * Sc::HALF + (j & 3) * 32) >> 4),
                      ID_Y, j > 0);
        umma_commit(ybar);
      }
    } else if (tid == kLoader && !*abort_flag && c + 1 < n_chunks) {
      // the slot of chunk c - 1 is free (its MMAs completed before this chunk began, its
      // scalars and V rows were read before the barrier above): the next chunk's operands
      // go there while the tensor cores form Y (an L2 prefetch of the chunk after would put
      // five more TMA instructions, about 90 cycles each, on this thread)
      load(c + 1);
    }
    __syncwarp();
    // S <- e^gam_last S while the tensor cores form Y (those MMAs read only A and K)
    {
      const float egl = sc[SCH];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        r0[j] = __float_as_uint(u2f(r0[j]) * egl);
        r1[j] = __float_as_uint(u2f(r1[j]) * egl);
      }
      tmem_st_32x32b_x32(tS, r0);
      tmem_st_32x32b_x32(tS + 32, r1);
    }
    if (!*abort_flag) ok &= mbar_wait(ybar, c & 1, abort_flag);
    tc_fence_after();

    // pass 2: A <- fp16(V^T - Y diag(e^gam)), this thread's 32 columns (tokens); the
    // thread's value row of V comes from the swizzled tile while Y is read
    {
      uint32_t r[32], vp[16], a[16];
      tmem_ld_32x32b_x32(tY, r);
      const uint8_t* vt = sm + Sc::V + s * Sc::KT;
      const int vr = 32 * qd + lane;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int t = 32 * hc + 2 * j;
        const uint32_t lo = *reinterpret_cast<const uint16_t*>(vt + kv_off(t, vr >> 3) + (vr & 7) * 2);
        const uint32_t hi = *reinterpret_cast<const uint16_t*>(vt + kv_off(t + 1, vr >> 3) + (vr & 7) * 2);
        vp[j] = lo | (hi << 16);
      }
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float4 e = reinterpret_cast<const float4*>(sc + 32 * hc)[j];
        const float2 v0 = F16<__half>::unpack(vp[2 * j]), v1 = F16<__half>::unpack(vp[2 * j + 1]);
        a[2 * j] = pack_f16(v0.x - e.x * u2f(r[4 * j]), v0.y - e.y * u2f(r[4 * j + 1]));
        a[2 * j + 1] = pack_f16(v1.x - e.z * u2f(r[4 * j + 2]), v1.y - e.w * u2f(r[4 * j + 3]));
      }
      tmem_st_32x32b_x16(tA + 16 * hc, a);
    }
    tmem_st_wait();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
      tc_fence_after();
      if (issuer && !*abort_flag) {
        const uint64_t dB = sdesc_k_sw128(smem_u32(sm + Sc::B1 + s * B1_BYTES));
#pragma unroll
        for (int j = 0; j < 4; ++j)
          umma_f16_ts(tb + COL_Y, tb + COL_A + 8 * j, dB + ((j * 32) >> 4), ID_Y, j > 0);
        umma_commit(dbar);
      }
    }
    __syncwarp();
    if (!*abort_flag) ok &= mbar_wait(dbar, c & 1, abort_flag);
    tc_fence_after();

    // pass 3: A <- fp16(D)
    {
      uint32_t r[32], a[16];
      tmem_ld_32x32b_x32(tY, r);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 16; ++j) a[j] = pack_f16(u2f(r[2 * j]), u2f(r[2 * j + 1]));
      tmem_st_32x32b_x16(tA + 16 * hc, a);
    }
    tmem_st_wait();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
      tc_fence_after();
      if (issuer && !*abort_flag) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          umma_f16_ts(tb + COL_S, tb + COL_A + 8 * j, dKm + ((j * 2048) >> 4), ID_S, 1);
        umma_commit(done);
      }
    }
    __syncwarp();
  }
  if (!*abort_flag) ok &= mbar_wait(done, (n_chunks - 1) & 1, abort_flag);
  tc_fence_after();
  if (!ok) {
    *abort_flag = 1;
    set_device_error(p.err, KVA_DEV_WAIT_TIMEOUT);
  }
#pragma unroll 1
  for (int q = 0; q < 2; ++q) {
    uint32_t r[32];
    tmem_ld_32x32b_x32(tS + 32 * q, r);
    tmem_ld_wait();
#pragma unroll
    for (int j = 0; j < 8; ++j)
      reinterpret_cast<float4*>(Sg + 32 * q)[j] =
          make_float4(u2f(r[4 * j]), u2f(r[4 * j + 1]), u2f(r[4 * j + 2]), u2f(r[4 * j + 3]));
  }
  // every copy and MMA this block issued has landed before it exits
  if (tid == kLoader) {
    for (int s = 0; s < 2; ++s)
      if (issued > s) {
        const int cl = s + 2 * ((issued - 1 - s) / 2);
        if (!mbar_wait_limit(&full[s], (cl >> 1) & 1)) set_device_error(p.err, KVA_DEV_WAIT_TIMEOUT);
      }
  }
  if (warp == 0) {
    if (issuer) {
      umma_commit(drain);
      if (!mbar_wait_limit(drain, 0)) set_device_error(p.err, KVA_DEV_WAIT_TIMEOUT);
    }
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tb, TMEM_COLS);
}

}  // namespace

size_t gdn_chunk_bytes(int n_seq, int n_gdn, int n_v, int T) {
  const size_t units = static_cast<size_t>(n_seq) * n_gdn * n_v * ((T + SCH - 1) / SCH);
  return units * (B1_BYTES + SC_FLOATS * 4);
}

void gdn_chunk_split(void* base, int n_seq, int n_gdn, int n_v, int T, void** b1, float** sc) {
  const size_t units = static_cast<size_t>(n_seq) * n_gdn * n_v * ((T + SCH - 1) / SCH);
  *b1 = base;
  *sc = base ? reinterpret_cast<float*>(static_cast<uint8_t*>(base) + units * B1_BYTES) : nullptr;
}

static int check_scan_tc(const GdnLaunch& g) {
  if (g.d_k != SD || g.d_v != SD) return KVA_ERR_UNSUPPORTED;
  if (!g.b1buf || !g.scbuf) return KVA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(g.kbuf) | reinterpret_cast<uintptr_t>(g.vbuf) |
       reinterpret_cast<uintptr_t>(g.b1buf) | reinterpret_cast<uintptr_t>(g.scbuf)) & 15u)
    return KVA_ERR_ALIGNMENT;
  return KVA_OK;
}

int launch_gdn_chunk_prep(const GdnLaunch& g, int l0, int nl, cudaStream_t s) {
  if (g.T == 0 || nl <= 0 || g.n_seq == 0) return KVA_OK;
  int e = check_scan_tc(g);
  if (e) return e;
  if (l0 < 0 || l0 + nl > g.n_gdn) return KVA_ERR_INVALID_ARG;
  const int n_chunks = (g.T + SCH - 1) / SCH;
  const int64_t slots = static_cast<int64_t>(g.n_seq) * g.n_gdn;
  CUtensorMap mK;
  if (!make_map_3d_16bit(&mK, g.kbuf, true, static_cast<int64_t>(g.n_k) * SD, g.T, slots, 64, SCH))
    return KVA_ERR_CUDA;
  if (cudaFuncSetAttribute(gdn_chunk_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           Cp::ALLOC) != cudaSuccess)
    return KVA_ERR_CUDA;
  dim3 gp(g.n_v, n_chunks, static_cast<unsigned>(g.n_seq * nl));
  return launch_pdl(gdn_chunk_prep_kernel, gp, dim3(Cp::THREADS), Cp::ALLOC, s, mK, g, l0, nl) == cudaSuccess
             ? KVA_OK
             : KVA_ERR_CUDA;
}

int launch_gdn_chain(const GdnLaunch& g, int l0, int nl, cudaStream_t s) {
  if (g.T == 0 || nl <= 0 || g.n_seq == 0) return KVA_OK;
  int e = check_scan_tc(g);
  if (e) return e;
  if (l0 < 0 || l0 + nl > g.n_gdn || !g.state) return KVA_ERR_INVALID_ARG;
  const int n_chunks = (g.T + SCH - 1) / SCH;
  const int64_t slots = static_cast<int64_t>(g.n_seq) * g.n_gdn;
  CUtensorMap mK, mV, mB;
  if (!make_map_3d_16bit(&mK, g.kbuf, true, static_cast<int64_t>(g.n_k) * SD, g.T, slots, 64, SCH) ||
      !make_map_3d_16bit(&mV, g.vbuf, true, static_cast<int64_t>(g.n_v) * SD, g.T, slots, 64, SCH) ||
      !make_map_3d_16bit(&mB, g.b1buf, true, SCH, static_cast<int64_t>(n_chunks) * SCH,
                         slots * g.n_v, 64, SCH))
    return KVA_ERR_CUDA;
  if (cudaFuncSetAttribute(gdn_scan_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           Sc::ALLOC) != cudaSuccess)
    return KVA_ERR_CUDA;
  dim3 grid(g.n_v, nl, g.n_seq);
  return launch_pdl(gdn_scan_tc_kernel, grid, dim3(NTHREADS), Sc::ALLOC, s, mK, mV, mB, g, l0) == cudaSuccess
             ? KVA_OK
             : KVA_ERR_CUDA;
}

int launch_gdn_scan_tc(const GdnLaunch& g, cudaStream_t s) {
  int e = launch_gdn_chunk_prep(g, 0, g.n_gdn, s);
  if (e) return e;
  return launch_gdn_chain(g, 0, g.n_gdn, s);
}

}  // namespace kva
