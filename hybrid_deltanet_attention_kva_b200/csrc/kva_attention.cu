// Block-causal multi-head attention of the projector blocks ("Qwen3.8-27B-KVA"
// model card, architecture table, attention row: 128-dim heads; r3 cuts the causal
// mask into 1024-token blocks, r2 keeps it causal over the whole ubatch).
//
// Key j is visible to query i iff j <= i and floor(i/W) == floor(j/W), indices
// local to the ubatch (W = window, or the whole ubatch when window = 0).  qkv is
// [T, 3d] 16-bit (q | k | v, head h at columns h*128 of each part), the output [T, d]
// in the same format (bf16 or fp16).
//
// Flash attention on the tcgen05 tensor cores.  One CTA per (head, 128-query tile),
// the tiles with the most causal work first.
//   warp 8   TMA producer: Q once, then 128-key K and V tiles into two stages each
//            (128-byte swizzle; K and V have their own full / empty barriers, so the
//            next K tile is loaded as soon as its S product has read the stage)
//   warp 9   waits converged, one elected lane issues the MMAs: S_j = Q K_j^T (both operands K-major in
//            shared memory) into TMEM buffer j % 2, and O += P_j V_j with P_j read
//            from TMEM and V_j as an MN-major shared-memory operand
//   warps 0-7  two threads per query row (TMEM lane = row; warps w and w + 4 take
//            columns 0-63 and 64-127): read their half of the row of S_j, mask it,
//            trade half-row maxima through shared memory, keep a running reference
//            max (O and the row sum are rescaled only when the tile's max exceeds the
//            reference by more than 8 in log2 units, so P stays below 2^8), write
//            P_j = 2^(s - ref) in the operand format to TMEM buffer j % 2; at the end
//            divide O by the row sum and store it.
// TMEM columns: S0 [0,128), S1 [128,256), O [256,384), P0 [384,448), P1 [448,512).
// S_{j+1} is issued before P_j is ready, so the tensor cores compute the next scores
// while the softmax warps work.  Every barrier wait has a time limit.
#include <cmath>

#include "kva_common.cuh"

namespace kva {

constexpr int ATT_BQ = 128;
constexpr int ATT_BKV = 128;
constexpr int ATT_D = 128;
constexpr int ATT_THREADS = 320;
constexpr int ATT_HALF = 128 * 64 * 2;  // one 64-dim half of a 128-row tile (16 KB)
constexpr int ATT_TILE = 2 * ATT_HALF;  // a 128 x 128 16-bit tile
constexpr int ATT_OFF_K = ATT_TILE;     // K stages
constexpr int ATT_OFF_V = 3 * ATT_TILE; // V stages
constexpr int ATT_OFF_BAR = 5 * ATT_TILE;
// after the barriers: half-row maxima [parity 2][half 2][128] and row-sum halves [half 2][128]
constexpr int ATT_OFF_X = ATT_OFF_BAR + 256;
constexpr int ATT_X_BYTES = (2 * 2 * 128 + 2 * 128) * 4;
constexpr int ATT_SMEM = ATT_OFF_X + ATT_X_BYTES + 1024;  // + alignment slack

// the 256 softmax threads (named barrier 1), returning the AND of `v` over them
__device__ __forceinline__ bool att_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 256, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v))
      : "memory");
  return r != 0;
}
constexpr uint32_t ATT_COL_S = 0, ATT_COL_O = 256, ATT_COL_P = 384;
constexpr float ATT_RESCALE = 8.f;  // log2 of the largest P value allowed before a rescale

__device__ __forceinline__ float att_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <typename E>
__global__ void __launch_bounds__(ATT_THREADS, 1)
    attention_kernel(const __grid_constant__ CUtensorMap mQKV, E* __restrict__ out, int64_t ldo,
                     int T, int d_model, int n_heads, int window, float scale_log2, int* err) {
  extern __shared__ uint8_t att_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(att_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + ATT_OFF_BAR);
  uint64_t* bar_q = bars;        // Q landed
  uint64_t* fullK = bars + 1;    // [2] K tile landed
  uint64_t* emptyK = bars + 3;   // [2] S product done with the K stage
  uint64_t* fullV = bars + 5;    // [2] V tile landed
  uint64_t* emptyV = bars + 7;   // [2] P V product done with the V stage
  uint64_t* barS = bars + 9;     // [2] S_j in TMEM
  uint64_t* barP = bars + 11;    // [2] P_j in TMEM (256 softmax threads)
  uint64_t* barO = bars + 13;    // O += P_j V_j done
  uint64_t* bar_drain = bars + 14;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 15);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_qt = (T + ATT_BQ - 1) / ATT_BQ;
  const int qt = n_qt - 1 - static_cast<int>(blockIdx.x) / n_heads;  // most causal work first
  const int h = static_cast<int>(blockIdx.x) % n_heads;
  const int q0 = qt * ATT_BQ;
  const int W = window > 0 ? window : 0x3fffffff;
  const int q_last = min(T, q0 + ATT_BQ) - 1;
  const int t_lo = ((q0 / W) * W) / ATT_BKV;  // first key tile any row of the tile may see
  const int n_kv = q_last / ATT_BKV - t_lo + 1;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&fullK[i], 1);
      mbar_init(&emptyK[i], 1);
      mbar_init(&fullV[i], 1);
      mbar_init(&emptyV[i], 1);
      mbar_init(&barS[i], 1);
      mbar_init(&barP[i], 256);
    }
    mbar_init(barO, 1);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&mQKV);
  }
  if (warp == 9) {
    tmem_alloc(tslot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = *tslot;
  griddep_wait_and_release();  // q, k, v come from the GEMM before

  if (warp == 8) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      const uint64_t pol = l2_policy_evict_normal();
      const int cq = h * ATT_D, ck = d_model + h * ATT_D, cv = 2 * d_model + h * ATT_D;
      mbar_arrive_expect_tx(bar_q, ATT_TILE);
      tma_load_2d(sm, &mQKV, bar_q, cq, q0, pol);
      tma_load_2d(sm + ATT_HALF, &mQKV, bar_q, cq + 64, q0, pol);
      bool ok = true;
      int issued = 0;  // tiles whose K and V were both requested
      for (int j = 0; j < n_kv && ok; ++j) {
        const int s = j & 1;
        const uint32_t ph = ((j >> 1) & 1) ^ 1u;  // the release of tile j - 2
        const int k0 = (t_lo + j) * ATT_BKV;
        if (j >= 2 && !mbar_wait(&emptyK[s], ph, abort_flag)) {
          ok = false;
          break;
        }
        uint8_t* kd = sm + ATT_OFF_K + s * ATT_TILE;
        mbar_arrive_expect_tx(&fullK[s], ATT_TILE);
        tma_load_2d(kd, &mQKV, &fullK[s], ck, k0, pol);
        tma_load_2d(kd + ATT_HALF, &mQKV, &fullK[s], ck + 64, k0, pol);
        if (j >= 2 && !mbar_wait(&emptyV[s], ph, abort_flag)) {
          ok = false;
          mbar_wait_limit(&fullK[s], (j >> 1) & 1);  // this K tile lands before exit
          break;
        }
        uint8_t* vd = sm + ATT_OFF_V + s * ATT_TILE;
        mbar_arrive_expect_tx(&fullV[s], ATT_TILE);
        tma_load_2d(vd, &mQKV, &fullV[s], cv, k0, pol);
        tma_load_2d(vd + ATT_HALF, &mQKV, &fullV[s], cv + 64, k0, pol);
        issued = j + 1;
      }
      if (!ok) {
        *abort_flag = 1;
        set_device_error(err, KVA_DEV_WAIT_TIMEOUT);
      }
      // every copy requested has landed before the CTA exits
      mbar_wait_limit(bar_q, 0);
      for (int j = issued - 2 < 0 ? 0 : issued - 2; j < issued; ++j) {
        mbar_wait_limit(&fullK[j & 1], (j >> 1) & 1);
        mbar_wait_limit(&fullV[j & 1], (j >> 1) & 1);
      }
    }
  } else if (warp == 9) {
    {
      // ------------------------------------------------ MMA issuer
      // (the warp runs the loop converged and one elected lane issues)
      constexpr uint32_t idS = idesc_f16kind_f32(ATT_BQ, ATT_BKV, F16<E>::umma_fmt);
      constexpr uint32_t idO = idesc_f16kind_f32_major(ATT_BQ, ATT_D, F16<E>::umma_fmt, false, true);
      const uint32_t sQ = smem_u32(sm);
      const uint32_t issuer = elect_one();  // elected once: a commit tracks its own lane's MMAs
      bool ok = mbar_wait_warp(bar_q, 0, abort_flag);
      auto issue_s = [&](int j) -> bool {
        const int s = j & 1;
        if (!mbar_wait_warp(&fullK[s], (j >> 1) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t sK = smem_u32(sm + ATT_OFF_K + s * ATT_TILE);
        if (issuer) {
#pragma unroll
          for (int k = 0; k < ATT_D / 16; ++k) {  // 16 dims per MMA: half k / 4, 32 bytes each
            const uint32_t off = (k >> 2) * ATT_HALF + (k & 3) * 32;
            umma_f16_ss(tb + ATT_COL_S + s * 128, sdesc_k_sw128(sQ + off), sdesc_k_sw128(sK + off), idS,
                        k > 0 ? 1u : 0u);
          }
          umma_commit(&barS[s]);
          umma_commit(&emptyK[s]);
        }
        __syncwarp();
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 0; j < n_kv && ok; ++j) {
        const int s = j & 1;
        if (j + 1 < n_kv && !issue_s(j + 1)) {
          ok = false;
          break;
        }
        if (!mbar_wait_warp(&barP[s], (j >> 1) & 1, abort_flag) ||
            !mbar_wait_warp(&fullV[s], (j >> 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sV = smem_u32(sm + ATT_OFF_V + s * ATT_TILE);
        if (issuer) {
#pragma unroll
          for (int k = 0; k < ATT_BKV / 16; ++k)  // 16 keys per MMA: 8 columns of P, 16 rows of V
            umma_f16_ts(tb + ATT_COL_O, tb + ATT_COL_P + s * 64 + k * 8,
                        sdesc_mn_sw128(sV + k * 2048, ATT_HALF), idO, (j > 0 || k > 0) ? 1u : 0u);
          umma_commit(barO);
          umma_commit(&emptyV[s]);
        }
        __syncwarp();
      }
      if (!ok && lane == 0) {
        *abort_flag = 1;
        set_device_error(err, KVA_DEV_WAIT_TIMEOUT);
      }
      // every MMA issued completes before TMEM is released
      if (issuer) {
        umma_commit(bar_drain);
        mbar_wait_limit(bar_drain, 0);
      }
      __syncwarp();
    }
  } else {
    // ------------------------------------------------ softmax and output (warps 0-7)
    const int qd = warp & 3, hc = warp >> 2;  // TMEM lane quarter, column half
    const int r = qd * 32 + lane;
    const int i = q0 + r;                     // query row
    const int kb = (i / W) * W;               // its first visible key
    const uint32_t lrow = static_cast<uint32_t>(qd * 32) << 16;
    float* xch = reinterpret_cast<float*>(sm + ATT_OFF_X);  // [parity][half][row]
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;  // every wait so far succeeded; a failure stops all of them at the next vote
    for (int j = 0; j < n_kv; ++j) {
      const int s = j & 1;
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&barS[s], (j >> 1) & 1, abort_flag));
      float x[64];
      float mh = -INFINITY;
      if (ok) {
        tc_fence_after();
        uint32_t ra[32], rb[32];
        const uint32_t ts = tb + lrow + ATT_COL_S + s * 128 + hc * 64;
        tmem_ld_32x32b_x32(ts, ra);
        tmem_ld_32x32b_x32(ts + 32, rb);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          x[e] = __uint_as_float(ra[e]);
          x[32 + e] = __uint_as_float(rb[e]);
        }
        const int k0 = (t_lo + j) * ATT_BKV + hc * 64;
        if (k0 + 63 > i || k0 < kb) {
#pragma unroll
          for (int e = 0; e < 64; ++e)
            if (k0 + e > i || k0 + e < kb) x[e] = -INFINITY;
        }
        float mx[16];  // a tree of maxima instead of one 64-long dependent chain
#pragma unroll
        for (int e = 0; e < 16; ++e) mx[e] = fmaxf(fmaxf(x[e], x[16 + e]), fmaxf(x[32 + e], x[48 + e]));
#pragma unroll
        for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
          for (int e = 0; e < w; ++e) mx[e] = fmaxf(mx[e], mx[e + w]);
        mh = mx[0];
        xch[(s * 2 + hc) * 128 + r] = mh;
      }
      if (!att_all(ok)) {  // also: both halves' maxima are in shared memory
        ok = false;
        break;
      }
      // the tile max in log2 units (the scale is positive); a slot is rewritten two tiles
      // later, after the partner has passed the next vote
      const float mt = fmaxf(mh, xch[(s * 2 + (hc ^ 1)) * 128 + r]) * scale_log2;
      float factor = 1.f;
      bool resc = false;
      if (mt > m_ref + ATT_RESCALE) {  // also the first visible key (m_ref = -inf)
        factor = att_ex2(m_ref - mt);
        l *= factor;
        m_ref = mt;
        resc = j > 0;
      }
      const float ref = m_ref == -INFINITY ? 0.f : m_ref;  // nothing visible yet: P = 0
      uint32_t pk[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float p0 = att_ex2(fmaf(x[2 * e], scale_log2, -ref));
        const float p1 = att_ex2(fmaf(x[2 * e + 1], scale_log2, -ref));
        l += p0 + p1;
        pk[e] = F16<E>::pack(p0, p1);
      }
      tmem_st_32x32b_x32(tb + lrow + ATT_COL_P + s * 64 + hc * 32, pk);
      if (__any_sync(0xffffffffu, resc)) {
        // the reference moved: O (complete up to P_{j-1} V_{j-1}) scales with it
        ok = __all_sync(0xffffffffu, mbar_wait(barO, (j - 1) & 1, abort_flag));
        if (ok) {
          tc_fence_after();
          const float f = resc ? factor : 1.f;
#pragma unroll 1
          for (int c = 0; c < 2; ++c) {
            uint32_t o[32];
            const uint32_t to = tb + lrow + ATT_COL_O + hc * 64 + c * 32;
            tmem_ld_32x32b_x32(to, o);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
            tmem_st_32x32b_x32(to, o);
          }
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&barP[s]);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(barO, (n_kv - 1) & 1, abort_flag));
    float* lx = xch + 4 * 128;  // [half][row] row-sum halves
    lx[hc * 128 + r] = l;
    if (att_all(ok)) {
      tc_fence_after();
      const float lt = l + lx[(hc ^ 1) * 128 + r];
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      E* orow = out + static_cast<int64_t>(i) * ldo + h * ATT_D + hc * 64;
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        uint32_t o[32];
        tmem_ld_32x32b_x32(tb + lrow + ATT_COL_O + hc * 64 + c * 32, o);
        tmem_ld_wait();
        if (i < T) {
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint4 v;
            v.x = F16<E>::pack(__uint_as_float(o[8 * q4 + 0]) * inv, __uint_as_float(o[8 * q4 + 1]) * inv);
            v.y = F16<E>::pack(__uint_as_float(o[8 * q4 + 2]) * inv, __uint_as_float(o[8 * q4 + 3]) * inv);
            v.z = F16<E>::pack(__uint_as_float(o[8 * q4 + 4]) * inv, __uint_as_float(o[8 * q4 + 5]) * inv);
            v.w = F16<E>::pack(__uint_as_float(o[8 * q4 + 6]) * inv, __uint_as_float(o[8 * q4 + 7]) * inv);
            reinterpret_cast<uint4*>(orow + c * 32)[q4] = v;
          }
        }
      }
    } else {
      *abort_flag = 1;
      set_device_error(err, KVA_DEV_WAIT_TIMEOUT);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) tmem_dealloc(tb, 512);
}

// ------------------------------------------------------------------ host side
int launch_attention(const void* qkv, int64_t ldq, void* out, int64_t ldo, int T, int n_heads,
                     int window, cudaStream_t s, int dtype, int* err) {
  if (T == 0) return KVA_OK;
  if (!qkv || !out || T < 0 || n_heads <= 0 || window < 0) return KVA_ERR_INVALID_ARG;
  if (dtype != KVA_BF16 && dtype != KVA_F16) return KVA_ERR_INVALID_ARG;
  if ((ldq % 8) || (ldo % 8) ||
      ((reinterpret_cast<uintptr_t>(qkv) | reinterpret_cast<uintptr_t>(out)) & 15u))
    return KVA_ERR_ALIGNMENT;
  const int d_model = n_heads * ATT_D;
  if (ldq < 3 * d_model || ldo < d_model) return KVA_ERR_INVALID_ARG;
  const float scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(ATT_D));
  CUtensorMap m;
  if (!make_map_2d_16bit(&m, qkv, dtype == KVA_F16, 3 * static_cast<int64_t>(d_model), T, ldq, 64,
                         ATT_BQ))
    return KVA_ERR_CUDA;
  const int n_qt = (T + ATT_BQ - 1) / ATT_BQ;
  const dim3 grid(n_qt * n_heads);
  cudaError_t r;
  if (dtype == KVA_F16) {
    if (cudaFuncSetAttribute(attention_kernel<__half>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             ATT_SMEM) != cudaSuccess)
      return KVA_ERR_CUDA;
    r = launch_pdl(attention_kernel<__half>, grid, dim3(ATT_THREADS), ATT_SMEM, s, m,
                   static_cast<__half*>(out), ldo, T, d_model, n_heads, window, scale_log2, err);
  } else {
    if (cudaFuncSetAttribute(attention_kernel<__nv_bfloat16>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, ATT_SMEM) != cudaSuccess)
      return KVA_ERR_CUDA;
    r = launch_pdl(attention_kernel<__nv_bfloat16>, grid, dim3(ATT_THREADS), ATT_SMEM, s, m,
                   static_cast<__nv_bfloat16*>(out), ldo, T, d_model, n_heads, window, scale_log2, err);
  }
  return r == cudaSuccess ? KVA_OK : KVA_ERR_CUDA;
}

}  // namespace kva
