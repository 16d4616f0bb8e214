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
// One CTA per (sequence, layer, v head), two CTAs per SM.  The state S (128 x 128
// fp32) lives in tensor memory for the whole ubatch: TMEM lane v holds state row v.
// Per chunk, four TMEM warps (thread v <-> lane v) and one issuing thread run
//     pass 1: A <- fp16(S), S <- e^gam_last S          (tcgen05.ld / st)
//     MMA   : Y  = A K^T                                (A from TMEM, K from smem)
//     pass 2: A <- fp16(-Y diag(e^gam))
//     MMA   : D  = V^T B1^T + A B1^T                    (V^T as an MN-major operand)
//     pass 3: A <- fp16(D)
//     MMA   : S += A K                                  (K as an MN-major operand)
// while eight prep warps build the next chunk's decays and B1 (K K^T and the
// 16 x 16 block products on mma.sync, the diagonal blocks of Tm by substitution
// in fp32).  K and V chunk tiles arrive by TMA (two and one chunks ahead), the
// gates by cp.async.  Every wait is bounded; on a timeout the block raises its
// abort flag, runs the remaining steps without waiting or issuing, drains its own
// copies and MMAs, and returns with the device status set.
#include "kva_common.cuh"

namespace kva {
namespace {

constexpr int SD = 128;             // d_k = d_v
constexpr int SCH = 64;             // chunk length
constexpr int N_TM = 4;             // TMEM warps
constexpr int N_PREP = 8;           // prep warps
constexpr int PREP_N = N_PREP * 32;
constexpr int NTHREADS = (N_TM + N_PREP) * 32;
constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t COL_S = 0;    // state, fp32 128 x 128
constexpr uint32_t COL_A = 128;  // 16-bit A operand (up to 128 x 128)
constexpr uint32_t COL_Y = 192;  // Y, then D: fp32 128 x 64

struct Sm {
  static constexpr int KT = SCH * SD * 2;    // K or V chunk: two [64][64] 128B-swizzled halves
  static constexpr int HALF = SCH * 64 * 2;
  static constexpr int BT = SCH * SCH * 2;   // [64][64] 16-bit tile
  static constexpr int K = 0;                // 3 slots
  static constexpr int V = K + 3 * KT;       // 2 slots
  static constexpr int B1 = V + 2 * KT;      // 2 buffers
  static constexpr int L = B1 + 2 * BT;      // L below the diagonal blocks, Tm on them
  static constexpr int LD = L + BT;          // diagonal blocks of L, fp32 [4][16][17]
  static constexpr int SC = LD + 4 * 16 * 17 * 4;  // 2 x {e^gam[64], e^gam_last}
  static constexpr int SC_BYTES = 80 * 4;
  static constexpr int GAM = SC + 2 * SC_BYTES;    // gam[64], decay[64]
  static constexpr int GB = GAM + 2 * SCH * 4;     // raw g, beta of 2 chunks
  static constexpr int BAR = GB + 2 * 2 * SCH * 4;
  static constexpr int N_BAR = 12;
  static constexpr int MISC = BAR + N_BAR * 8;     // TMEM base, abort flag
  static constexpr int BYTES = MISC + 16;
  static constexpr int ALLOC = BYTES + 1024;       // slack for 1024-byte alignment
};

// byte offset of (row, 16-byte chunk c16 in 0..15) in a K or V chunk tile
__device__ __forceinline__ uint32_t kv_off(int row, int c16) {
  return static_cast<uint32_t>((c16 >> 3) * Sm::HALF + row * 128 + (((c16 & 7) ^ (row & 7)) << 4));
}
// byte offset of (row, 16-byte chunk c8 in 0..7) in a [64][64] 16-bit tile
__device__ __forceinline__ uint32_t t64_off(int row, int c8) {
  return static_cast<uint32_t>(row * 128 + ((c8 ^ (row & 7)) << 4));
}
__device__ __forceinline__ uint32_t t64_elem(int row, int col) {
  return t64_off(row, col >> 3) + (col & 7) * 2;
}

__device__ __forceinline__ void tm_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
__device__ __forceinline__ void prep_sync() {
  asm volatile("bar.sync 2, %0;" ::"n"(PREP_N) : "memory");
}
__device__ __forceinline__ float u2f(uint32_t x) { return __uint_as_float(x); }

constexpr uint32_t ID_Y = idesc_f16kind_f32_major(128, 64, 0, false, false);   // TMEM A, K-major B
constexpr uint32_t ID_VB = idesc_f16kind_f32_major(128, 64, 0, true, false);   // MN-major A
constexpr uint32_t ID_S = idesc_f16kind_f32_major(128, 128, 0, false, true);   // MN-major B

__global__ void __launch_bounds__(NTHREADS, 2)
    gdn_scan_tc_kernel(const __grid_constant__ CUtensorMap mK, const __grid_constant__ CUtensorMap mV,
                       const GdnLaunch p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Sm::BAR);
  uint64_t* kfull = bars;        // [3] K chunk landed
  uint64_t* vfull = bars + 3;    // [2] V chunk landed
  uint64_t* ready = bars + 5;    // [2] prep -> chain: B1 and scalars of a chunk
  uint64_t* done = bars + 7;     // [2] the chunk's last MMA completed
  uint64_t* ybar = bars + 9;
  uint64_t* dbar = bars + 10;
  uint64_t* drain = bars + 11;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + Sm::MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + Sm::MISC + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x, layer = blockIdx.y, seq = blockIdx.z;
  const int n_v = p.n_v;
  const int kh = h / (n_v / p.n_k);
  const int T = p.T;
  const int slot = seq * p.n_gdn + layer;
  const int n_chunks = (T + SCH - 1) / SCH;

  if (tid == 0) {
    for (int i = 0; i < Sm::N_BAR; ++i) mbar_init(&bars[i], 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&mK);
    tma_prefetch_desc(&mV);
  }
  // both B1 buffers start at zero: the blocks above the diagonal are never written
  for (int i = tid; i < 2 * Sm::BT / 16; i += NTHREADS)
    reinterpret_cast<uint4*>(sm + Sm::B1)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  if (warp == 0) {
    tmem_alloc(tslot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = *tslot;

  if (warp < N_TM) {
    // ============================================================ TMEM warps
    const uint32_t lrow = static_cast<uint32_t>(32 * warp) << 16;
    const uint32_t tS = tb + lrow + COL_S, tA = tb + lrow + COL_A, tY = tb + lrow + COL_Y;
    float* Sg = p.state + (static_cast<int64_t>(slot) * n_v + h) * SD * SD + tid * SD;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
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

    const uint64_t pol_k = l2_policy_evict_normal(), pol_v = l2_policy_evict_first();
    int k_issued = 0, v_issued = 0;  // chunks whose K / V load was issued (thread 0)
    auto load_k = [&](int c) {
      uint8_t* dst = sm + Sm::K + (c % 3) * Sm::KT;
      uint64_t* bar = &kfull[c % 3];
      mbar_arrive_expect_tx(bar, Sm::KT);
      tma_load_3d(dst, &mK, bar, kh * SD, c * SCH, slot, pol_k);
      tma_load_3d(dst + Sm::HALF, &mK, bar, kh * SD + 64, c * SCH, slot, pol_k);
      k_issued = c + 1;
    };
    auto load_v = [&](int c) {
      uint8_t* dst = sm + Sm::V + (c & 1) * Sm::KT;
      uint64_t* bar = &vfull[c & 1];
      mbar_arrive_expect_tx(bar, Sm::KT);
      tma_load_3d(dst, &mV, bar, h * SD, c * SCH, slot, pol_v);
      tma_load_3d(dst + Sm::HALF, &mV, bar, h * SD + 64, c * SCH, slot, pol_v);
      v_issued = c + 1;
    };
    if (tid == 0) {
      load_k(0);
      if (n_chunks > 1) load_k(1);
      load_v(0);
    }
    __syncwarp();

    bool ok = true;
    for (int c = 0; c < n_chunks; ++c) {
      const int b = c & 1;
      const float* sc = reinterpret_cast<const float*>(sm + Sm::SC + b * Sm::SC_BYTES);
      if (!*abort_flag) ok &= mbar_wait(&ready[b], (c >> 1) & 1, abort_flag);
      if (c > 0 && !*abort_flag) ok &= mbar_wait(&done[(c - 1) & 1], ((c - 1) >> 1) & 1, abort_flag);
      tc_fence_after();
      // the slots of chunk c-1 are free: K two chunks ahead, V one chunk ahead
      if (tid == 0 && !*abort_flag) {
        if (c + 2 < n_chunks) load_k(c + 2);
        if (c + 1 < n_chunks) load_v(c + 1);
      }
      __syncwarp();

      // pass 1: A <- fp16(S), S <- e^gam_last S
      const float egl = sc[SCH];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t r[32], a[16];
        tmem_ld_32x32b_x32(tS + 32 * q, r);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) a[j] = pack_f16(u2f(r[2 * j]), u2f(r[2 * j + 1]));
        tmem_st_32x32b_x16(tA + 16 * q, a);
#pragma unroll
        for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(u2f(r[j]) * egl);
        tmem_st_32x32b_x32(tS + 32 * q, r);
      }
      tmem_st_wait();
      tc_fence_before();
      tm_sync();
      const uint32_t kb = smem_u32(sm + Sm::K + (c % 3) * Sm::KT);
      if (tid == 0) {
        tc_fence_after();
        if (!*abort_flag) ok &= mbar_wait(&kfull[c % 3], (c / 3) & 1, abort_flag);
        if (!*abort_flag) {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            umma_f16_ts(tb + COL_Y, tb + COL_A + 8 * j,
                        sdesc_k_sw128(kb + (j >> 2) * Sm::HALF + (j & 3) * 32), ID_Y, j > 0);
          umma_commit(ybar);
        }
      }
      __syncwarp();
      if (!*abort_flag) ok &= mbar_wait(ybar, c & 1, abort_flag);
      tc_fence_after();

      // pass 2: A <- fp16(-Y diag(e^gam))
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        uint32_t r[32], a[16];
        tmem_ld_32x32b_x32(tY + 32 * q, r);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float4 e = reinterpret_cast<const float4*>(sc + 32 * q)[j];
          a[2 * j] = pack_f16(-e.x * u2f(r[4 * j]), -e.y * u2f(r[4 * j + 1]));
          a[2 * j + 1] = pack_f16(-e.z * u2f(r[4 * j + 2]), -e.w * u2f(r[4 * j + 3]));
        }
        tmem_st_32x32b_x16(tA + 16 * q, a);
      }
      tmem_st_wait();
      tc_fence_before();
      tm_sync();
      if (tid == 0) {
        tc_fence_after();
        if (!*abort_flag) ok &= mbar_wait(&vfull[b], (c >> 1) & 1, abort_flag);
        if (!*abort_flag) {
          const uint32_t vb = smem_u32(sm + Sm::V + b * Sm::KT);
          const uint32_t bb = smem_u32(sm + Sm::B1 + b * Sm::BT);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            umma_f16_ss(tb + COL_Y, sdesc_mn_sw128(vb + j * 2048, Sm::HALF), sdesc_k_sw128(bb + j * 32),
                        ID_VB, j > 0);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            umma_f16_ts(tb + COL_Y, tb + COL_A + 8 * j, sdesc_k_sw128(bb + j * 32), ID_Y, 1);
          umma_commit(dbar);
        }
      }
      __syncwarp();
      if (!*abort_flag) ok &= mbar_wait(dbar, c & 1, abort_flag);
      tc_fence_after();

      // pass 3: A <- fp16(D)
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        uint32_t r[32], a[16];
        tmem_ld_32x32b_x32(tY + 32 * q, r);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) a[j] = pack_f16(u2f(r[2 * j]), u2f(r[2 * j + 1]));
        tmem_st_32x32b_x16(tA + 16 * q, a);
      }
      tmem_st_wait();
      tc_fence_before();
      tm_sync();
      if (tid == 0) {
        tc_fence_after();
        if (!*abort_flag) {
#pragma unroll
          for (int j = 0; j < 4; ++j)
            umma_f16_ts(tb + COL_S, tb + COL_A + 8 * j, sdesc_mn_sw128(kb + j * 2048, Sm::HALF), ID_S,
                        1);
          umma_commit(&done[b]);
        }
      }
      __syncwarp();
    }
    const int last = n_chunks - 1;
    if (!*abort_flag) ok &= mbar_wait(&done[last & 1], (last >> 1) & 1, abort_flag);
    tc_fence_after();
    if (!ok) {
      *abort_flag = 1;
      set_device_error(p.err, KVA_DEV_WAIT_TIMEOUT);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(tS + 32 * q, r);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 8; ++j)
        reinterpret_cast<float4*>(Sg + 32 * q)[j] =
            make_float4(u2f(r[4 * j]), u2f(r[4 * j + 1]), u2f(r[4 * j + 2]), u2f(r[4 * j + 3]));
    }
    if (tid == 0) {
      // every copy and MMA this block issued has landed before it exits
      for (int s = 0; s < 3; ++s)
        if (k_issued > s) {
          const int c = s + 3 * ((k_issued - 1 - s) / 3);
          if (!mbar_wait_limit(&kfull[s], (c / 3) & 1)) set_device_error(p.err, KVA_DEV_WAIT_TIMEOUT);
        }
      for (int s = 0; s < 2; ++s)
        if (v_issued > s) {
          const int c = s + 2 * ((v_issued - 1 - s) / 2);
          if (!mbar_wait_limit(&vfull[s], (c >> 1) & 1)) set_device_error(p.err, KVA_DEV_WAIT_TIMEOUT);
        }
      umma_commit(drain);
      if (!mbar_wait_limit(drain, 0)) set_device_error(p.err, KVA_DEV_WAIT_TIMEOUT);
    }
    __syncwarp();
  } else {
    // ============================================================ prep warps
    const int pt = tid - N_TM * 32;  // 0..255
    const int pw = warp - N_TM;      // 0..7
    const int g = lane >> 2, cq = lane & 3, mi = lane >> 3, lr = lane & 7;
    const float* gg = p.gbuf + static_cast<int64_t>(slot) * 2 * n_v * T + static_cast<int64_t>(h) * T;
    const float* bg = gg + static_cast<int64_t>(n_v) * T;
    float* gam = reinterpret_cast<float*>(sm + Sm::GAM);
    float* dec = gam + SCH;
    float* Ld = reinterpret_cast<float*>(sm + Sm::LD);
    const uint32_t sL = smem_u32(sm + Sm::L);

    // raw g and beta of chunk cj into its buffer (zero past T: identity steps)
    auto issue_gb = [&](int cj) {
      if (pt < 2 * SCH) {
        const int t = cj * SCH + (pt & (SCH - 1));
        const bool in = t < T;
        const float* src = (pt < SCH ? gg : bg) + (in ? t : 0);
        cp_async4(smem_u32(sm + Sm::GB + (cj & 1) * 2 * SCH * 4 + pt * 4), src, in ? 4u : 0u);
      }
      cp_async_commit();
    };

    bool ok = true;
    issue_gb(0);
    for (int c = 0; c < n_chunks; ++c) {
      const int b = c & 1;
      // B1[b] and the scalars of chunk c - 2 are no longer read
      if (c >= 2 && !*abort_flag) ok &= mbar_wait(&done[b], ((c >> 1) - 1) & 1, abort_flag);
      if (c + 1 < n_chunks) {
        issue_gb(c + 1);
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      if (!*abort_flag) ok &= mbar_wait(&kfull[c % 3], (c / 3) & 1, abort_flag);
      prep_sync();
      const float* gs = reinterpret_cast<const float*>(sm + Sm::GB + b * 2 * SCH * 4);
      const float* bs = gs + SCH;
      float* sc = reinterpret_cast<float*>(sm + Sm::SC + b * Sm::SC_BYTES);
      const uint32_t kb = smem_u32(sm + Sm::K + (c % 3) * Sm::KT);
      uint8_t* B1 = sm + Sm::B1 + b * Sm::BT;

      // (1) cumulative decays (warp 0)
      if (pw == 0) {
        const float v0 = gs[2 * lane], v1 = gs[2 * lane + 1];
        const float pair = v0 + v1;
        float sc_incl = pair;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const float y = __shfl_up_sync(0xffffffffu, sc_incl, o);
          if (lane >= o) sc_incl += y;
        }
        const float ex = sc_incl - pair;
        const float total = __shfl_sync(0xffffffffu, sc_incl, 31);
        const float ga = ex + v0, gb2 = ex + pair;
        gam[2 * lane] = ga;
        gam[2 * lane + 1] = gb2;
        sc[2 * lane] = expf(ga);
        sc[2 * lane + 1] = expf(gb2);
        dec[2 * lane] = expf(total - ga);
        dec[2 * lane + 1] = expf(total - gb2);
        if (lane == 0) sc[SCH] = expf(total);
      }
      // (2) K K^T: warp pw owns rows [16 (pw & 3), +16), columns [32 (pw >> 2), +32)
      const int mt = pw & 3, nh = pw >> 2;
      float acc[4][4];
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
      // (blocks entirely above the diagonal are not needed)
      if (nh * 32 < (mt + 1) * 16) {
#pragma unroll
      for (int ks = 0; ks < SD / 16; ++ks) {
        uint32_t a[4];
        ldmatrix_x4(a, kb + kv_off(mt * 16 + (mi & 1) * 8 + lr, ks * 2 + (mi >> 1)));
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          uint32_t bb[4];
          ldmatrix_x4(bb, kb + kv_off(nh * 32 + jj * 16 + (mi >> 1) * 8 + lr, ks * 2 + (mi & 1)));
          const uint32_t b0[2] = {bb[0], bb[1]}, b1[2] = {bb[2], bb[3]};
          mma_f16_16816(acc[2 * jj], a, b0);
          mma_f16_16816(acc[2 * jj + 1], a, b1);
        }
      }
      }
      prep_sync();  // gam ready
      // (3) L = beta_t e^(gam_t - gam_s) k_t.k_s below the diagonal: fp16 blocks below
      //     the diagonal blocks, fp32 copies of the diagonal blocks
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int s0 = nh * 32 + j * 8 + 2 * cq;
        if ((s0 >> 4) > mt) continue;
        float lv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int t = mt * 16 + g + (e >> 1) * 8;
          const int s = s0 + (e & 1);
          lv[e] = s < t ? bs[t] * expf(gam[t] - gam[s]) * acc[j][e] : 0.f;
        }
        if ((s0 >> 4) == mt) {
#pragma unroll
          for (int e = 0; e < 4; ++e)
            Ld[(mt * 16 + g + (e >> 1) * 8) * 17 + ((s0 + (e & 1)) & 15)] = lv[e];
        } else {
          const int t0 = mt * 16 + g;
          *reinterpret_cast<uint32_t*>(sm + Sm::L + t64_elem(t0, s0)) = pack_f16(lv[0], lv[1]);
          *reinterpret_cast<uint32_t*>(sm + Sm::L + t64_elem(t0 + 8, s0)) = pack_f16(lv[2], lv[3]);
        }
      }
      prep_sync();
      // (4) diagonal blocks of Tm = (I + L)^-1, one column per thread, in fp32
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
        const int s = blk * 16 + col;
        const float bsv = bs[s];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
          const int t = blk * 16 + r;
          *reinterpret_cast<__half*>(sm + Sm::L + t64_elem(t, s)) = __float2half_rn(x[r]);
          *reinterpret_cast<__half*>(B1 + t64_elem(t, s)) = __float2half_rn(dec[t] * x[r] * bsv);
        }
      }
      prep_sync();
      // (5) blocks below the diagonal, column block j (8 columns per warp):
      //     X_ij = -Tm_ii sum_{k=j}^{i-1} L_ik X_kj, B1_ij = diag(dec) X_ij diag(beta)
      if (pw < 6) {
        const int jb = pw >> 1, s0 = 16 * jb + 8 * (pw & 1);
        const int s = s0 + 2 * cq;
        const float b0s = bs[s], b1s = bs[s + 1];
#pragma unroll
        for (int jj = 0; jj < 3; ++jj) {
          if (jj != jb) continue;
          uint32_t xf[4][2];
          ldmatrix_x2_trans(xf[jj], sL + t64_off(16 * jj + (mi & 1) * 8 + lr, s0 >> 3));
#pragma unroll
          for (int i = jj + 1; i < 4; ++i) {
            float y[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int k = jj; k < i; ++k) {
              uint32_t a[4];
              ldmatrix_x4(a, sL + t64_off(16 * i + (mi & 1) * 8 + lr, 2 * k + (mi >> 1)));
              mma_f16_16816(y, a, xf[k]);
            }
            const uint32_t yb[2] = {movmatrix_trans(pack_f16(y[0], y[1])),
                                    movmatrix_trans(pack_f16(y[2], y[3]))};
            uint32_t a[4];
            ldmatrix_x4(a, sL + t64_off(16 * i + (mi & 1) * 8 + lr, 2 * i + (mi >> 1)));
            float x[4] = {0.f, 0.f, 0.f, 0.f};
            mma_f16_16816(x, a, yb);
            const int t0 = 16 * i + g, t1 = t0 + 8;
            const float d0 = dec[t0], d1 = dec[t1];
            *reinterpret_cast<uint32_t*>(B1 + t64_elem(t0, s)) = pack_f16(-d0 * x[0] * b0s, -d0 * x[1] * b1s);
            *reinterpret_cast<uint32_t*>(B1 + t64_elem(t1, s)) = pack_f16(-d1 * x[2] * b0s, -d1 * x[3] * b1s);
            xf[i][0] = movmatrix_trans(pack_f16(-x[0], -x[1]));
            xf[i][1] = movmatrix_trans(pack_f16(-x[2], -x[3]));
          }
        }
      }
      fence_proxy_async_smem();  // B1 is read by the tensor cores
      prep_sync();
      if (pt == 0) mbar_arrive(&ready[b]);
    }
    if (!ok) {
      *abort_flag = 1;
      set_device_error(p.err, KVA_DEV_WAIT_TIMEOUT);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tb, TMEM_COLS);
}

}  // namespace

int launch_gdn_scan_tc(const GdnLaunch& g, cudaStream_t s) {
  if (g.d_k != SD || g.d_v != SD) return KVA_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(g.kbuf) | reinterpret_cast<uintptr_t>(g.vbuf)) & 15u)
    return KVA_ERR_ALIGNMENT;
  const int64_t slots = static_cast<int64_t>(g.n_seq) * g.n_gdn;
  CUtensorMap mK, mV;
  if (!make_map_3d_16bit(&mK, g.kbuf, true, static_cast<int64_t>(g.n_k) * SD, g.T, slots, 64, SCH) ||
      !make_map_3d_16bit(&mV, g.vbuf, true, static_cast<int64_t>(g.n_v) * SD, g.T, slots, 64, SCH))
    return KVA_ERR_CUDA;
  if (cudaFuncSetAttribute(gdn_scan_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           Sm::ALLOC) != cudaSuccess)
    return KVA_ERR_CUDA;
  dim3 grid(g.n_v, g.n_gdn, g.n_seq);
  gdn_scan_tc_kernel<<<grid, NTHREADS, Sm::ALLOC, s>>>(mK, mV, g);
  return cudaPeekAtLastError() == cudaSuccess ? KVA_OK : KVA_ERR_CUDA;
}

}  // namespace kva
