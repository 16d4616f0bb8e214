// Persistent 16-bit (fp16 or bf16 operands, fp32 accumulation) GEMM on the 5th-generation
// tensor cores (tcgen05 / TMEM),
// D = A * B^T with fused epilogues.  It serves every linear layer of the KVA
// projector ("Qwen3.8-27B-KVA" model card, architecture: Linear{5120 -> d},
// the q/k/v/o and SwiGLU projections of the 3 causal blocks, and the one wide
// GEMM over all per-layer heads concatenated).
//
// Two kernels share one design.  gemm_tc_kernel: one CTA per SM, 128 x BN tiles.
// gemm_pair_kernel (the path's default): a cluster of two CTAs on one 256 x 256
// tile through tcgen05.mma.cta_group::2.
//   warp 0      TMA producer: A tile [128 x 64] and this CTA's B tile per stage,
//               128-byte swizzle, into a STAGES-deep shared-memory ring (the
//               weights' first stages are requested before the PDL wait).
//   warp 1      TMEM allocator + MMA issuer (the warp waits converged, one elected
//               lane issues): 4 tcgen05.mma (K = 16) per stage into one of two TMEM
//               accumulators, tcgen05.commit frees the stage.
//   warps 2..   epilogue, while the MMA warp accumulates the next tile in the other
//               TMEM buffer: 16-bit stores and residual adds through per-warp
//               shared staging and TMA (bulk stores / reduce-adds), SwiGLU, or the
//               heads GEMM's state-update epilogue (eight warps, see below).
// Tiles are visited M-fastest so the M tiles of a 1024-token ubatch that share
// one weight tile run together and read it from HBM once.
#include <cuda.h>

#include <cstdio>
#include <mutex>
#include <type_traits>

#include "kva_common.cuh"

namespace kva {

template <int BN>
struct GemmCfg {
  static constexpr int BM = 128;
  static constexpr int BK = 64;  // 64 bf16 = one 128-byte swizzle row
  static constexpr int STAGES = BN == 256 ? 4 : 6;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TMEM_COLS = 2 * BN;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM = STAGES * STAGE_BYTES + 1024 + BAR_BYTES;
};

struct GemmParams {
  int M, N, K;
  int b_mode;
  int seg_rows;
  void* D;
  int64_t ldd;
  void* D1;
  int64_t ldd1;
  int64_t n_split;
  int splits;  // K ranges per tile (ADD_F32 only; each range's partial sum is added by a TMA reduce-add)
  int d_tma;   // CTA pairs: D written (ADD_F32: added) by TMA from staged chunks (tensor map mD)
  int b_const; // CTA pairs: the first stages' B tiles are loaded before griddepcontrol.wait
  int* err;
  int stall_item1;  // CTA pairs, test of the failure path: 1 + the work item whose MMA issuer
                    // first waits on a barrier that nothing arrives on (0: never)
};

template <typename T>
__device__ __forceinline__ void store16x32(T* dst, const float* v, int valid) {
  if (valid >= 32) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint4 pk;
      pk.x = F16<T>::pack(v[8 * q + 0], v[8 * q + 1]);
      pk.y = F16<T>::pack(v[8 * q + 2], v[8 * q + 3]);
      pk.z = F16<T>::pack(v[8 * q + 4], v[8 * q + 5]);
      pk.w = F16<T>::pack(v[8 * q + 6], v[8 * q + 7]);
      reinterpret_cast<uint4*>(dst)[q] = pk;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (i < valid) dst[i] = F16<T>::from(v[i]);
  }
}

// One accumulator tile (128 TMEM lanes x BN fp32 columns) to global memory with the
// fused epilogue.  Warp q of the epilogue group reads TMEM lanes [32q, 32q+32).
template <int BN, int EPI, typename T>
__device__ __forceinline__ void epilogue_tile(const GemmParams& p, uint32_t tmem_acc, int row0,
                                              int n_blk, int q, int lane) {
  const int row = row0 + q * 32 + lane;
  const bool row_ok = row < p.M;
  const uint32_t taddr = tmem_acc + (static_cast<uint32_t>(q * 32) << 16);
  if constexpr (EPI == EPI_SWIGLU_BF16) {
#pragma unroll 1
    for (int c = 0; c < BN / 2; c += 32) {
      uint32_t gr[32], ur[32];
      tmem_ld_32x32b_x32(taddr + c, gr);
      tmem_ld_32x32b_x32(taddr + BN / 2 + c, ur);
      tmem_ld_wait();
      const int col = n_blk * (BN / 2) + c;
      if (row_ok && col < p.N) {
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i)
          v[i] = silu_f(__uint_as_float(gr[i])) * __uint_as_float(ur[i]);
        T* dst = reinterpret_cast<T*>(p.D) + row * p.ldd + col;
        store16x32<T>(dst, v, p.N - col);
      }
    }
  } else {
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(taddr + c, r);
      tmem_ld_wait();
      int col = n_blk * BN + c;
      if (row_ok && col < p.N) {
        const int valid = min(32, p.N - col);
        void* base = p.D;
        int64_t ld = p.ldd;
        if (p.n_split > 0 && col >= p.n_split) {
          base = p.D1;
          ld = p.ldd1;
          col -= static_cast<int>(p.n_split);
        }
        if constexpr (EPI == EPI_STORE_BF16) {
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
          store16x32<T>(reinterpret_cast<T*>(base) + row * ld + col, v, valid);
        } else {
          float* dst = reinterpret_cast<float*>(base) + row * ld + col;
          if (EPI == EPI_ADD_F32 && p.splits > 1) {
            // partial sums of one K range: added atomically (16-byte vector adds)
            if (valid == 32) {
#pragma unroll
              for (int q4 = 0; q4 < 8; ++q4)
                atomicAdd(reinterpret_cast<float4*>(dst) + q4,
                          make_float4(__uint_as_float(r[4 * q4 + 0]), __uint_as_float(r[4 * q4 + 1]),
                                      __uint_as_float(r[4 * q4 + 2]), __uint_as_float(r[4 * q4 + 3])));
            } else {
              for (int i = 0; i < valid; ++i) atomicAdd(dst + i, __uint_as_float(r[i]));
            }
          } else if (valid == 32) {
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4) {
              float4 o;
              if constexpr (EPI == EPI_ADD_F32) o = reinterpret_cast<float4*>(dst)[q4];
              else o = make_float4(0.f, 0.f, 0.f, 0.f);
              o.x += __uint_as_float(r[4 * q4 + 0]);
              o.y += __uint_as_float(r[4 * q4 + 1]);
              o.z += __uint_as_float(r[4 * q4 + 2]);
              o.w += __uint_as_float(r[4 * q4 + 3]);
              reinterpret_cast<float4*>(dst)[q4] = o;
            }
          } else {
            for (int i = 0; i < valid; ++i) {
              if constexpr (EPI == EPI_ADD_F32) dst[i] += __uint_as_float(r[i]);
              else dst[i] = __uint_as_float(r[i]);
            }
          }
        }
      }
    }
  }
}

template <int BN, int EPI, typename T>
__global__ void __launch_bounds__(192, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap mA, const __grid_constant__ CUtensorMap mB0,
                   const __grid_constant__ CUtensorMap mB1, const __grid_constant__ CUtensorMap mB2,
                   const GemmParams p) {
  using Cfg = GemmCfg<BN>;
  constexpr int S = Cfg::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + S * Cfg::A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + S * Cfg::B_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  uint64_t* tfull = bars + 2 * S;
  uint64_t* tempty = bars + 2 * S + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 128);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&mA);
    tma_prefetch_desc(&mB0);
    if (p.b_mode != B_SINGLE) tma_prefetch_desc(&mB1);
    if (p.b_mode == B_SEGMENTS) tma_prefetch_desc(&mB2);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_wait_and_release();  // operands and outputs belong to earlier kernels

  const int num_m = (p.M + Cfg::BM - 1) / Cfg::BM;
  const int n_per_tile = (EPI == EPI_SWIGLU_BF16) ? BN / 2 : BN;
  const int num_n = (p.N + n_per_tile - 1) / n_per_tile;
  const int num_k = (p.K + Cfg::BK - 1) / Cfg::BK;
  const int splits = p.splits;
  const int tiles = num_m * num_n * splits;  // work items: (n tile, K range, m tile), m fastest

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      const uint64_t pol_a = l2_policy_evict_last();
      const uint64_t pol_b = l2_policy_evict_normal();
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0;  // stages with a load issued and not yet seen consumed
      bool ok = true;
      for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
        const int m_blk = tile % num_m;
        const int ns = tile / num_m;
        const int n_blk = ns / splits, sp = ns % splits;
        const int kb0 = sp * num_k / splits, kb1 = (sp + 1) * num_k / splits;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], Cfg::STAGE_BYTES);
          armed |= 1u << stage;
          const int kc = kb * Cfg::BK;
          tma_load_2d(sA + stage * Cfg::A_BYTES, &mA, &full[stage], kc, m_blk * Cfg::BM, pol_a);
          uint8_t* b = sB + stage * Cfg::B_BYTES;
          if (p.b_mode == B_PAIRED) {
            const int r = n_blk * (BN / 2);
            tma_load_2d(b, &mB0, &full[stage], kc, r, pol_b);
            tma_load_2d(b + (BN / 2) * 128, &mB1, &full[stage], kc, r, pol_b);
          } else if (p.b_mode == B_SEGMENTS) {
            const int n0 = n_blk * BN;
            const int seg = n0 / p.seg_rows;
            const int r = n0 - seg * p.seg_rows;
            const CUtensorMap* m = seg == 0 ? &mB0 : (seg == 1 ? &mB1 : &mB2);
            tma_load_2d(b, m, &full[stage], kc, r, pol_b);
          } else {
            tma_load_2d(b, &mB0, &full[stage], kc, n_blk * BN, pol_b);
          }
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        set_device_error(p.err, KVA_DEV_WAIT_TIMEOUT);
      }
      // Wait for the copies this thread issued to land before the CTA can exit.
      // The last phase armed on stage s has parity (phase of s at arm time);
      // waiting on it returns at once when it already completed.
      (void)armed;
      {
        int st = stage;
        uint32_t ph = phase;
        for (int i = 0; i < S; ++i) {
          // step back one stage
          if (st == 0) {
            st = S - 1;
            ph ^= 1u;
          } else {
            --st;
          }
          if (armed & (1u << st)) {
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&full[st], ph)) {
              if (globaltimer_ns() - t0 > kWaitLimitNs) break;
            }
          }
        }
      }
    }
  } else if (warp == 1) {
    {
      // ------------------------------------------------ MMA issuer
      // (the warp runs the loop converged and one elected lane issues, as in the pair kernel)
      constexpr uint32_t idesc = idesc_f16kind_f32(Cfg::BM, BN, F16<T>::umma_fmt);
      const uint32_t issuer = elect_one();
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
        if (!mbar_wait_warp(&tempty[acc], acc_phase ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        const int sp = (tile / num_m) % splits;
        const int kb0 = sp * num_k / splits, kb1 = (sp + 1) * num_k / splits;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait_warp(&full[stage], phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + stage * Cfg::A_BYTES);
          const uint32_t b_base = smem_u32(sB + stage * Cfg::B_BYTES);
          if (issuer) {
#pragma unroll
            for (int j = 0; j < Cfg::BK / 16; ++j) {
              umma_f16_ss(d_tmem, sdesc_k_sw128(a_base + 32 * j), sdesc_k_sw128(b_base + 32 * j),
                          idesc, (kb != kb0 || j != 0) ? 1u : 0u);
            }
            umma_commit(&empty[stage]);
          }
          __syncwarp();
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (issuer) umma_commit(&tfull[acc]);
        __syncwarp();
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (!ok && lane == 0) {
        *abort_flag = 1;
        set_device_error(p.err, KVA_DEV_WAIT_TIMEOUT);
      }
      // Drain: every MMA issued (by the issuing lane) completes before TMEM is freed.
      if (issuer) {
        umma_commit(&tfull[acc]);
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(&tfull[acc], acc_phase)) {
          if (globaltimer_ns() - t0 > kWaitLimitNs) break;
        }
      }
      __syncwarp();
    }
  } else {
    // ------------------------------------------------ epilogue warps 2..5
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
      const int m_blk = tile % num_m;
      const int n_blk = (tile / num_m) / splits;
      if (!mbar_wait(&tfull[acc], acc_phase, abort_flag)) {
        *abort_flag = 1;
        set_device_error(p.err, KVA_DEV_WAIT_TIMEOUT);
        break;
      }
      tc_fence_after();
      epilogue_tile<BN, EPI, T>(p, tmem_base + static_cast<uint32_t>(acc * BN), m_blk * Cfg::BM,
                                n_blk, q, lane);
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
}


// ------------------------------------------------------------------ state-update epilogue
// The heads GEMM's accumulator tile (128 tokens x 256 columns of one layer segment per
// CTA of the pair) goes straight to the state updates' inputs.  Every raw value is
// first rounded to the mixer's 16-bit format, so the results equal those of the plain
// path (mixer stored, then the conv / norm / gate / KV kernels).  Eight epilogue warps
// work in two groups of four: warp q of a group owns TMEM lanes (tokens) [32q, 32q+32),
// and the groups split the tile's columns in 16-column chunks (a DeltaNet key tile: one
// 128-channel head per group).  The groups meet only for the attention key's RMS over
// its 256 dims and for the per-tile abort vote.
constexpr int MIX_GROUPS = 2;
constexpr int MIX_EPI_WARPS = 4 * MIX_GROUPS;
constexpr int MIX_LD = 24;                          // 16-bit values per staged row (48-byte rows)
constexpr int MIX_BUF_BYTES = 128 * MIX_LD * 2;     // one group's buffer of 16 channels
constexpr int MIX_RMS_OFF = MIX_GROUPS * 2 * MIX_BUF_BYTES;         // [2][128] fp32 RMS partials
constexpr int MIX_W_OFF = MIX_RMS_OFF + MIX_GROUPS * 128 * 4;        // [2][128] float4 conv weights
constexpr int MIX_STAGE_BYTES = MIX_W_OFF + MIX_GROUPS * 128 * 16;

// tcgen05.wait::ld that also orders the loaded registers: later reads of `r` cannot be
// moved above the wait (used where the next chunk's load is in flight while the
// current one is processed)
__device__ __forceinline__ void tmem_wait_dep16(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                 "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                 "+r"(r[14]), "+r"(r[15])
               :
               : "memory");
}

// a group's 128 threads (named barriers 2 and 3)
__device__ __forceinline__ void mix_sync_group(int g) {
  asm volatile("bar.sync %0, 128;" ::"r"(2 + g) : "memory");
}
// all epilogue threads (named barrier 4), returning the AND of `v` over them
__device__ __forceinline__ bool mix_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 4, 256, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v))
      : "memory");
  return r != 0;
}

// 16 accumulator columns to the 16-bit grid: packed pairs and their float values
template <typename T>
__device__ __forceinline__ void mix_round16(const uint32_t (&r)[16], uint32_t (&pk)[8], float (&x)[16]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    pk[i] = F16<T>::pack(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
    const float2 f = F16<T>::unpack(pk[i]);
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
}

// the first `valid` of 16 packed 16-bit values to dst (16-byte aligned)
__device__ __forceinline__ void mix_put16(void* dst, const uint32_t (&pk)[8], int valid) {
  if (valid >= 16) {
    reinterpret_cast<uint4*>(dst)[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    reinterpret_cast<uint4*>(dst)[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
  } else {
    uint16_t* d = static_cast<uint16_t*>(dst);
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if (i < valid) d[i] = static_cast<uint16_t>((i & 1) ? (pk[i >> 1] >> 16) : (pk[i >> 1] & 0xffffu));
  }
}

// 16 floats packed in the 16-bit format C16
template <typename C16>
__device__ __forceinline__ void mix_pack16(const float (&x)[16], uint32_t (&pk)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) pk[i] = F16<C16>::pack(x[2 * i], x[2 * i + 1]);
}

// causal depthwise conv over tokens t-3..t of 16 channels (weights w4[i] = taps of channel
// i, staged in shared memory), then SiLU: this thread's row
// goes to the group's staging buffer (two buffers used in turn, so one barrier per chunk
// suffices: a buffer is rewritten only after every thread has passed the barrier of the
// chunk in between), rows r-1..r-3 come back from it.  Rows 0-2 of the block have no
// predecessors here; the block-edge fix-up computes their outputs.
template <typename T>
__device__ __forceinline__ void mix_conv16(const float4* w4, uint8_t* gstage, int& turn,
                                           int r, int g, const uint32_t (&pk)[8], const float (&x)[16],
                                           float (&z)[16]) {
  uint16_t* buf = reinterpret_cast<uint16_t*>(gstage + turn * MIX_BUF_BYTES);
  turn ^= 1;
  uint4* my = reinterpret_cast<uint4*>(buf + r * MIX_LD);
  my[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  my[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
  mix_sync_group(g);
  if (r < 3) {
#pragma unroll
    for (int i = 0; i < 16; ++i) z[i] = 0.f;
    return;
  }
  uint32_t p[3][8];
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    const uint4* src = reinterpret_cast<const uint4*>(buf + (r - 1 - k) * MIX_LD);
    const uint4 u0 = src[0], u1 = src[1];
    p[k][0] = u0.x; p[k][1] = u0.y; p[k][2] = u0.z; p[k][3] = u0.w;
    p[k][4] = u1.x; p[k][5] = u1.y; p[k][6] = u1.z; p[k][7] = u1.w;
  }
#pragma unroll
  for (int i = 0; i < 16; i += 2) {
    const float4 wa = w4[i], wb = w4[i + 1];
    const float2 x1 = F16<T>::unpack(p[0][i / 2]);
    const float2 x2 = F16<T>::unpack(p[1][i / 2]);
    const float2 x3 = F16<T>::unpack(p[2][i / 2]);
    z[i] = silu_tanh(wa.x * x3.x + wa.y * x2.x + wa.z * x1.x + wa.w * x[i]);
    z[i + 1] = silu_tanh(wb.x * x3.y + wb.y * x2.y + wb.z * x1.y + wb.w * x[i + 1]);
  }
}

// raw copies of gated-DeltaNet conv channels: the rows around 128-token block edges
// (key and value channels, for the edge fix-up) and the ubatch's last 3 rows (every
// channel: the new conv tail)
template <typename T>
__device__ __forceinline__ void mix_gdn_raw(const MixParams& mp, bool halo, int gdn, int t, int r,
                                            int ch0, const uint32_t (&pk)[8]) {
  if (t >= mp.T) return;
  if (halo && (r < 3 || r >= 125)) {
    const int slot = r < 3 ? r : r - 122;
    const int64_t row = (static_cast<int64_t>(gdn) * mp.nblk + (t >> 7)) * kMixHaloRows + slot;
    mix_put16(static_cast<T*>(mp.halo) + row * mp.C + ch0, pk, 16);
  }
  if (t >= mp.T - 3) {
    const int64_t row = static_cast<int64_t>(gdn) * 3 + (t - (mp.T - 3));
    mix_put16(static_cast<T*>(mp.tail_new) + row * mp.C + ch0, pk, 16);
  }
}

// row index of position `p` in a KV cache (sequence 0), or -1 when the page table is out of range
__device__ __forceinline__ int64_t mix_cache_row(const kva_kv_cache& cc, int head, int n_kv, int64_t p,
                                                 int* err) {
  if (cc.layout == KVA_KV_PAGED) {
    const int64_t pg_i = p / cc.page_size;
    if (pg_i < 0 || pg_i >= cc.pages_per_seq) {
      set_device_error(err, KVA_DEV_PAGE_OOB);
      return -1;
    }
    const int page = cc.page_table[pg_i];
    if (page < 0 || page >= cc.n_pages) {
      set_device_error(err, KVA_DEV_PAGE_OOB);
      return -1;
    }
    return (static_cast<int64_t>(page) * n_kv + head) * cc.page_size + p % cc.page_size;
  }
  return static_cast<int64_t>(head) * cc.max_pos + p;
}

// 16 values of one cache row (256 dims per head) from column c0, in the cache's format
__device__ __forceinline__ void mix_cache_put16(const kva_kv_cache& cc, void* base, int64_t row, int c0,
                                                const float (&v)[16]) {
  uint32_t pk[8];
  if (cc.dtype == KVA_F16) mix_pack16<__half>(v, pk);
  else mix_pack16<__nv_bfloat16>(v, pk);
  mix_put16(static_cast<uint16_t*>(base) + row * 256 + c0, pk, 16);
}

__device__ __forceinline__ void mix_sync_all() { asm volatile("bar.sync 4, 256;" ::: "memory"); }

template <typename T>
__device__ __forceinline__ void epilogue_mixer(const MixParams& mp, uint32_t tmem_acc, int row0,
                                               int n_blk, int q, int g, int lane, uint8_t* stage,
                                               int& turn) {
  const MixTile tl = mp.tiles[n_blk];
  const int r = q * 32 + lane;
  const int t = row0 + r;
  const bool row_ok = t < mp.T;
  const uint32_t taddr = tmem_acc + (static_cast<uint32_t>(q * 32) << 16);
  const int n16 = (tl.ncols + 15) / 16;
  uint8_t* gstage = stage + g * 2 * MIX_BUF_BYTES;
  float* rms_part = reinterpret_cast<float*>(stage + MIX_GROUPS * 2 * MIX_BUF_BYTES);

  // one 16-column chunk from TMEM in the 16-bit grid, with the raw mixer's debug copy
  auto load16 = [&](int c0, uint32_t(&pk)[8], float(&x)[16]) {
    uint32_t rr[16];
    tmem_ld_32x32b_x16(taddr + c0, rr);
    tmem_ld_wait();
    mix_round16<T>(rr, pk, x);
    if (mp.mixer_out && row_ok)
      mix_put16(static_cast<T*>(mp.mixer_out) + t * mp.ld_mix + tl.col0 + c0, pk, min(16, tl.ncols - c0));
  };

  if (tl.kind == MIX_GDN_K || tl.kind == MIX_GDN_V) {
    // conv tiles.  A key tile: one 128-channel head per group (chunks 8g..8g+7), whose
    // norm needs the whole head before any output, so the conv outputs wait as fp16
    // pairs (their sum of squares is taken in fp32).  A value tile: chunks g, g+2, ...
    // Each thread stages one channel's taps for its group; the next chunk's TMEM load
    // is in flight while the current one is processed.
    const bool is_k = tl.kind == MIX_GDN_K;
    auto chunk_col = [&](int k) { return is_k ? (g * 8 + k) * 16 : (g + 2 * k) * 16; };
    float4* wsm = reinterpret_cast<float4*>(stage + MIX_W_OFF) + g * 128;
    const float4 wv = __ldg(reinterpret_cast<const float4*>(mp.conv_w) +
                            static_cast<int64_t>(tl.layer) * mp.C + tl.sub + chunk_col(r >> 4) + (r & 15));
    const int nkdk = mp.n_k * 128, nvdv = mp.n_v * 128;
    uint32_t nx[16];
    tmem_ld_32x32b_x16(taddr + chunk_col(0), nx);
    uint32_t zk[64];
    float ss = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int c0 = chunk_col(k);
      tmem_wait_dep16(nx);
      uint32_t pk[8];
      float x[16], z[16];
      mix_round16<T>(nx, pk, x);
      if (k < 7) tmem_ld_32x32b_x16(taddr + chunk_col(k + 1), nx);
      if (k == 0) wsm[r] = wv;  // read after the first conv barrier
      if (mp.mixer_out && row_ok)
        mix_put16(static_cast<T*>(mp.mixer_out) + t * mp.ld_mix + tl.col0 + c0, pk, 16);
      mix_gdn_raw<T>(mp, true, tl.layer, t, r, tl.sub + c0, pk);
      mix_conv16<T>(wsm + k * 16, gstage, turn, r, g, pk, x, z);
      if (is_k) {
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
          ss += z[i] * z[i] + z[i + 1] * z[i + 1];
          zk[k * 8 + i / 2] = pack_f16(z[i], z[i + 1]);
        }
      } else if (r >= 3 && row_ok) {
        uint32_t o[8];
        mix_pack16<__half>(z, o);
        mix_put16(static_cast<__half*>(mp.vbuf) + (static_cast<int64_t>(tl.layer) * mp.T + t) * nvdv +
                      (tl.sub - 2 * nkdk) + c0,
                  o, 16);
      }
    }
    if (is_k && r >= 3 && row_ok) {
      const float sc = rsqrtf(ss + mp.eps);
      __half* dst = static_cast<__half*>(mp.kbuf) +
                    (static_cast<int64_t>(tl.layer) * mp.T + t) * nkdk + (tl.sub - nkdk) + g * 128;
#pragma unroll
      for (int q4 = 0; q4 < 16; ++q4) {
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = F16<__half>::unpack(zk[4 * q4 + e]);
          o[e] = pack_f16(f.x * sc, f.y * sc);
        }
        reinterpret_cast<uint4*>(dst)[q4] = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
  } else if (tl.kind == MIX_RAW) {
    // query channels feed only the new conv tail (and the debug copy): other warps skip them
    if (!mp.mixer_out && !__any_sync(0xffffffffu, row_ok && t >= mp.T - 3)) return;
#pragma unroll 1
    for (int ch = g; ch < n16; ch += MIX_GROUPS) {
      const int c0 = ch * 16;
      uint32_t pk[8];
      float x[16];
      load16(c0, pk, x);
      mix_gdn_raw<T>(mp, false, tl.layer, t, r, tl.sub + c0, pk);
    }
  } else if (tl.kind == MIX_GDN_AB) {
    // the gates of two layers, one per tile half (group g: columns [128 g, 128 g + 128)
    // from weight row g ? col1 : col0, layer g ? sub : layer; sub < 0: no second layer).
    // Columns [0, n_v) are a, [n_v, 2 n_v) are b: g = -exp(A_log) softplus(a + dt_bias),
    // beta = sigmoid(b), written [layer][2][n_v][T]
    const int lay = g ? tl.sub : tl.layer;
    if (lay < 0) return;  // no named barrier in this branch
    const int colbase = g ? tl.col1 : tl.col0;
    float* gb = mp.gbuf + static_cast<int64_t>(lay) * 2 * mp.n_v * mp.T;
#pragma unroll 1
    for (int ch = 0; ch < n16; ++ch) {
      const int c0 = ch * 16;
      uint32_t rr[16];
      tmem_ld_32x32b_x16(taddr + 128 * g + c0, rr);
      tmem_ld_wait();
      uint32_t pk[8];
      float x[16];
      mix_round16<T>(rr, pk, x);
      if (!row_ok) continue;
      if (mp.mixer_out)
        mix_put16(static_cast<T*>(mp.mixer_out) + t * mp.ld_mix + colbase + c0, pk, min(16, tl.ncols - c0));
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int j = c0 + i;
        if (j >= tl.ncols) continue;
        float o;
        if (j < mp.n_v) {
          const float xa = x[i] + mp.dt_bias[lay * mp.n_v + j];
          const float sp = xa > 20.f ? xa : log1pf(expf(xa));
          o = -expf(mp.A_log[lay * mp.n_v + j]) * sp;
        } else {
          o = 1.f / (1.f + expf(-x[i]));
        }
        gb[static_cast<int64_t>(j) * mp.T + t] = o;
      }
    }
  } else if ((tl.kind == MIX_ATT_K || tl.kind == MIX_ATT_V) && mp.att_raw) {
    // a q8_0 cache: the attention k / v stay raw (the KV writer rotates and quantizes them)
#pragma unroll 1
    for (int ch = g; ch < n16; ch += MIX_GROUPS) {
      uint32_t pk[8];
      float x[16];
      load16(ch * 16, pk, x);
      if (row_ok) mix_put16(static_cast<T*>(mp.att_raw) + t * mp.ld_att_raw + tl.col0 + ch * 16, pk, 16);
    }
  } else if (tl.kind == MIX_ATT_K) {
    // RMSNorm over the 256 dims x gain (each group sums its 128), then RoPE on dims
    // [0, 64): pairs (d, d + 32), angle (pos + t) theta^(-2d/64) (frequencies from the
    // host's fp64 table) formed and range-reduced in fp64
    const int cb = g * 128;
    float ss = 0.f;
#pragma unroll 1
    for (int ch = 0; ch < 8; ++ch) {
      uint32_t pk[8];
      float x[16];
      load16(cb + ch * 16, pk, x);
#pragma unroll
      for (int i = 0; i < 16; ++i) ss += x[i] * x[i];
    }
    rms_part[g * 128 + r] = ss;
    mix_sync_all();
    const float sc = rsqrtf((rms_part[r] + rms_part[128 + r]) / 256.f + mp.eps);
    const float* gain = mp.k_gain + tl.layer * 256;
    const int64_t p = mp.pos + t;
    const int64_t crow = row_ok ? mix_cache_row(mp.cache, tl.sub, mp.n_kv, p, mp.err) : -1;
    void* kbase = mp.cache.k[tl.layer];
    int ch0 = 0;
    if (g == 0) {
      const double two_pi = 6.283185307179586476925286766559;
      const double inv_two_pi = 0.15915494309189533576888376337251;
#pragma unroll 1
      for (int d0 = 0; d0 < 32; d0 += 16) {
        uint32_t ra[16], rb[16];
        tmem_ld_32x32b_x16(taddr + d0, ra);
        tmem_ld_32x32b_x16(taddr + 32 + d0, rb);
        tmem_ld_wait();
        uint32_t pa[8], pb[8];
        float a[16], b[16];
        mix_round16<T>(ra, pa, a);
        mix_round16<T>(rb, pb, b);
        if (crow < 0) continue;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int d = d0 + i;
          const float k0 = a[i] * sc * gain[d], k1 = b[i] * sc * gain[32 + d];
          const double ang = static_cast<double>(p) * mp.inv_freq[d];
          const double qq = rint(ang * inv_two_pi);
          const float red = static_cast<float>(fma(-qq, two_pi, ang));
          float sn, cs;
          sincosf(red, &sn, &cs);
          a[i] = k0 * cs - k1 * sn;
          b[i] = k1 * cs + k0 * sn;
        }
        mix_cache_put16(mp.cache, kbase, crow, d0, a);
        mix_cache_put16(mp.cache, kbase, crow, 32 + d0, b);
      }
      ch0 = 4;  // dims 64..127 follow
    }
#pragma unroll 1
    for (int ch = ch0; ch < 8; ++ch) {
      const int c0 = cb + ch * 16;
      uint32_t rr[16];
      tmem_ld_32x32b_x16(taddr + c0, rr);
      tmem_ld_wait();
      uint32_t pk[8];
      float x[16];
      mix_round16<T>(rr, pk, x);
      if (crow < 0) continue;
#pragma unroll
      for (int i = 0; i < 16; ++i) x[i] *= sc * gain[c0 + i];
      mix_cache_put16(mp.cache, kbase, crow, c0, x);
    }
  } else if (tl.kind == MIX_ATT_V) {
    // the value head as stored in the mixer, in the cache's format
    const int64_t crow = row_ok ? mix_cache_row(mp.cache, tl.sub, mp.n_kv, mp.pos + t, mp.err) : -1;
    void* vbase = mp.cache.v[tl.layer];
#pragma unroll 1
    for (int ch = g; ch < n16; ch += MIX_GROUPS) {
      uint32_t pk[8];
      float x[16];
      load16(ch * 16, pk, x);
      if (crow >= 0) mix_cache_put16(mp.cache, vbase, crow, ch * 16, x);
    }
  } else {  // MIX_DRAFT
#pragma unroll 1
    for (int ch = g; ch < n16; ch += MIX_GROUPS) {
      const int c0 = ch * 16;
      uint32_t rr[16];
      tmem_ld_32x32b_x16(taddr + c0, rr);
      tmem_ld_wait();
      uint32_t pk[8];
      float x[16];
      mix_round16<T>(rr, pk, x);
      if (row_ok && mp.draft)
        mix_put16(static_cast<T*>(mp.draft) + t * mp.ld_draft + tl.sub + c0, pk, min(16, tl.ncols - c0));
    }
  }
}

// ------------------------------------------------------------------ CTA-pair variant
// The same pipeline on a pair of CTAs (a cluster of 2) sharing one 256 x 256 tile
// through tcgen05.mma.cta_group::2: each CTA loads its 128 rows of A and its 128 rows
// of B (B rows 0-127 of the tile in the leader, 128-255 in the peer), the leader's
// elected issuing lane issues M = 256 MMAs that read both CTAs' operands, and each CTA's
// TMEM receives its own 128 rows of the accumulator.  Per CTA this halves the B
// bytes that the tensor core reads from shared memory per MMA, the limit of the
// one-CTA 128 x 256 tile.  TMA loads of both CTAs complete on the leader's barrier
// (no multicast loads); MMA completion is committed to both CTAs' barriers.
// ADD_F32 on CTA pairs: the fp32 accumulator tile goes to the residual stream by TMA
// reduce-add.  Each epilogue warp owns 32 rows; it stages every 32-column chunk of them
// (32 rows x 128 bytes, 128-byte swizzle: 16-byte piece j of row r at piece j ^ (r & 7),
// so the row-per-lane writes are conflict-free) in one of its two shared buffers, and
// its lane 0 adds the block to D with one bulk tensor reduction, coalesced and done at
// L2.  A buffer is refilled only after the reduction issued from it two chunks earlier
// has finished reading it.  No barrier is shared between warps.
constexpr int RED_BUF_BYTES = 32 * 128;

__device__ __forceinline__ void epilogue_add_tma(const CUtensorMap* mD, uint32_t tmem_acc, int row0,
                                                 int col0, int q, int lane, uint8_t* wstage, int& turn) {
  const uint32_t taddr = tmem_acc + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll 1
  for (int c = 0; c < 256; c += 32) {
    uint32_t v[32];
    tmem_ld_32x32b_x32(taddr + c, v);
    tmem_ld_wait();
    uint8_t* buf = wstage + turn * RED_BUF_BYTES;
    turn ^= 1;
    if (lane == 0) bulk_wait_read<1>();
    __syncwarp();  // the buffer is free
    uint8_t* row = buf + lane * 128;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      *reinterpret_cast<uint4*>(row + ((j ^ (lane & 7)) << 4)) =
          make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    fence_proxy_async_smem();
    __syncwarp();  // the block is staged
    if (lane == 0) {
      tma_reduce_add_2d(mD, buf, col0 + c, row0 + q * 32);
      bulk_commit();
    }
  }
}

// 16-bit outputs (STORE, SWIGLU) on CTA pairs: the same per-warp staging, chunks of 64
// output columns (32 rows x 128 bytes, 128-byte swizzle) written by TMA bulk stores.
template <int EPI, typename T>
__device__ __forceinline__ void epilogue_store_tma(const CUtensorMap* mD, uint32_t tmem_acc, int row0,
                                                   int col0, int ncols_tile, int q, int lane,
                                                   uint8_t* wstage, int& turn) {
  const uint32_t taddr = tmem_acc + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll 1
  for (int c = 0; c < ncols_tile; c += 64) {
    uint32_t pk[32];
    if constexpr (EPI == EPI_SWIGLU_BF16) {  // gate columns c.., up columns 128 + c..
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t gr[32], ur[32];
        tmem_ld_32x32b_x32(taddr + c + 32 * h, gr);
        tmem_ld_32x32b_x32(taddr + 128 + c + 32 * h, ur);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[16 * h + i] = F16<T>::pack(silu_f(__uint_as_float(gr[2 * i])) * __uint_as_float(ur[2 * i]),
                                        silu_f(__uint_as_float(gr[2 * i + 1])) * __uint_as_float(ur[2 * i + 1]));
      }
    } else {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(taddr + c + 32 * h, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[16 * h + i] = F16<T>::pack(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
      }
    }
    uint8_t* buf = wstage + turn * RED_BUF_BYTES;
    turn ^= 1;
    if (lane == 0) bulk_wait_read<1>();
    __syncwarp();  // the buffer is free
    uint8_t* row = buf + lane * 128;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      *reinterpret_cast<uint4*>(row + ((j ^ (lane & 7)) << 4)) =
          make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
    fence_proxy_async_smem();
    __syncwarp();  // the block is staged
    if (lane == 0) {
      tma_store_2d(mD, buf, col0 + c, row0 + q * 32);
      bulk_commit();
    }
  }
}

struct PairCfg {
  static constexpr int BM = 128;  // rows per CTA (256 per pair)
  static constexpr int BN = 256;  // tile columns (128 B rows held by each CTA)
  static constexpr int BK = 64;
  static constexpr int STAGES = 6;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = (BN / 2) * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TMEM_COLS = 2 * BN;
  static constexpr int SMEM = STAGES * STAGE_BYTES + 1024 + 256;
  static constexpr int SMEM_MIX = SMEM + MIX_STAGE_BYTES;  // + the conv staging buffers
  // ADD_F32 by TMA reduction: each epilogue warp's two staging buffers, 1024 bytes after
  // the barriers
  static constexpr int SMEM_RED = STAGES * STAGE_BYTES + 1024 + 1024 + 4 * 2 * RED_BUF_BYTES;
  // q8_0 weights: five stages, each with the raw codes (128 rows x 64 int8, 64-byte
  // swizzle) and scales ([2 blocks][128 rows] fp16) of this CTA's B half
  static constexpr int STAGES_Q8 = 5;
  static constexpr int RAW_CODES = 128 * 64;
  static constexpr int RAW_BYTES = RAW_CODES + 2 * 128 * 2;
  static constexpr int SMEM_Q8 = STAGES_Q8 * (STAGE_BYTES + RAW_BYTES) + 1024 + 256;
  // q4_0 weights: six stages, each with the packed codes (128 rows x 32 bytes, 32-byte
  // swizzle) and the same scales
  static constexpr int STAGES_Q4 = 6;
  static constexpr int RAW_CODES_Q4 = 128 * 32;
  static constexpr int RAW_BYTES_Q4 = RAW_CODES_Q4 + 2 * 128 * 2;
  static constexpr int SMEM_Q4 = STAGES_Q4 * (STAGE_BYTES + RAW_BYTES_Q4) + 1024 + 256;
  static constexpr int stages(int wq) { return wq == 1 ? STAGES_Q8 : (wq == 2 ? STAGES_Q4 : STAGES); }
  static constexpr int raw_bytes(int wq) { return wq == 1 ? RAW_BYTES : (wq == 2 ? RAW_BYTES_Q4 : 0); }
  static constexpr int raw_codes(int wq) { return wq == 1 ? RAW_CODES : RAW_CODES_Q4; }
  // producer warp, MMA warp, the epilogue warps (eight for the state-update epilogue), then
  // for quantized weights the converter warps: teams of four that take the stages in turn,
  // each warp one 32-row quarter of the B half.  Three teams where the registers allow (576
  // threads at up to 112 registers), two with the SwiGLU epilogue's larger register need.
  static constexpr int conv_teams(int epi) { return epi == EPI_SWIGLU_BF16 ? 2 : 3; }
  static constexpr int conv_warps(int epi) { return 4 * conv_teams(epi); }
  static constexpr int epi_warps(int epi) { return epi == EPI_MIXER ? MIX_EPI_WARPS : 4; }
  static constexpr int threads(int epi, int wq = 0) {
    return 64 + 32 * (epi_warps(epi) + (wq ? conv_warps(epi) : 0));
  }
};

// q8_0 weights: row r of this CTA's B half, values 32 h .. 32 h + 31 of one stage (one
// 32-value block): the codes (64-byte swizzle: 16-byte piece j at j ^ ((r >> 1) & 3)) times
// the block's scale, rounded once to the operand format, written in the 128-byte-swizzled
// K-major layout the MMA reads (16-byte piece c of 8 values at c ^ (r & 7)).  fp16: a code
// c sits in the mantissa of the half 1024 + 128 + c (one byte permute of c ^ 0x80 under the
// exponent byte 0x64), so subtracting 1152 gives c exactly and one half2 multiply by the
// scale rounds the exact product once, as an fp32 product rounded to fp16 would.
template <typename T>
__device__ __forceinline__ void q8_0_dequant_block(const uint8_t* raw, uint8_t* b_stage, int r, int h) {
  const uint8_t* crow = raw + r * 64;
  const __half sc = reinterpret_cast<const __half*>(raw + PairCfg::RAW_CODES)[h * 128 + r];
  uint8_t* brow = b_stage + r * 128;
#pragma unroll
  for (int jj = 0; jj < 2; ++jj) {  // 16 values per piece
    const int j = 2 * h + jj;
    const uint4 w = *reinterpret_cast<const uint4*>(crow + ((j ^ ((r >> 1) & 3)) << 4));
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
    uint32_t pk[8];
    if constexpr (std::is_same<T, __half>::value) {
      const __half2 s2 = __half2half2(sc);
      const __half2 bias = __float2half2_rn(1152.f);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t x = ws[q] ^ 0x80808080u;
        const uint32_t lo = __byte_perm(x, 0x64646464u, 0x4140), hi = __byte_perm(x, 0x64646464u, 0x4342);
        const __half2 a = __hmul2(__hsub2(*reinterpret_cast<const __half2*>(&lo), bias), s2);
        const __half2 b = __hmul2(__hsub2(*reinterpret_cast<const __half2*>(&hi), bias), s2);
        pk[2 * q] = *reinterpret_cast<const uint32_t*>(&a);
        pk[2 * q + 1] = *reinterpret_cast<const uint32_t*>(&b);
      }
    } else {
      const float d = __half2float(sc);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t v = ws[q];
        pk[2 * q] = F16<T>::pack(static_cast<float>(static_cast<int8_t>(v & 0xffu)) * d,
                                 static_cast<float>(static_cast<int8_t>((v >> 8) & 0xffu)) * d);
        pk[2 * q + 1] = F16<T>::pack(static_cast<float>(static_cast<int8_t>((v >> 16) & 0xffu)) * d,
                                     static_cast<float>(static_cast<int8_t>(v >> 24)) * d);
      }
    }
    *reinterpret_cast<uint4*>(brow + (((2 * j) ^ (r & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    *reinterpret_cast<uint4*>(brow + (((2 * j + 1) ^ (r & 7)) << 4)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
  }
}

// q4_0 weights: row r of this CTA's B half, values 32 h .. 32 h + 31 of one stage (one
// 32-value block): 16 bytes of codes (32-byte swizzle: 16-byte piece h at h ^ ((r >> 2) & 1)),
// byte j holding value j in its low nibble and value j + 16 in its high nibble; each value
// is fp16(d) (code - 8), rounded once to the operand format and written as in the q8_0
// case.  fp16: a code c under the exponent byte 0x64 is the half 1024 + c, so subtracting
// 1032 gives c - 8 exactly.
template <typename T>
__device__ __forceinline__ void q4_0_dequant_block(const uint8_t* raw, uint8_t* b_stage, int r, int h) {
  const __half sc = reinterpret_cast<const __half*>(raw + PairCfg::RAW_CODES_Q4)[h * 128 + r];
  const uint4 w = *reinterpret_cast<const uint4*>(raw + r * 32 + ((h ^ ((r >> 2) & 1)) << 4));
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
  uint8_t* brow = b_stage + r * 128;
#pragma unroll
  for (int c = 0; c < 4; ++c) {  // values 8 c .. 8 c + 7 of the block
    uint32_t pk[4];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const uint32_t word = ws[(c & 1) * 2 + t];
      const uint32_t nib = (c >> 1) ? (word >> 4) & 0x0F0F0F0Fu : word & 0x0F0F0F0Fu;
      if constexpr (std::is_same<T, __half>::value) {
        const __half2 s2 = __half2half2(sc);
        const __half2 bias = __float2half2_rn(1032.f);
        const uint32_t lo = __byte_perm(nib, 0x64646464u, 0x4140), hi = __byte_perm(nib, 0x64646464u, 0x4342);
        const __half2 a = __hmul2(__hsub2(*reinterpret_cast<const __half2*>(&lo), bias), s2);
        const __half2 b = __hmul2(__hsub2(*reinterpret_cast<const __half2*>(&hi), bias), s2);
        pk[2 * t] = *reinterpret_cast<const uint32_t*>(&a);
        pk[2 * t + 1] = *reinterpret_cast<const uint32_t*>(&b);
      } else {
        const float d = __half2float(sc);
        pk[2 * t] = F16<T>::pack(static_cast<float>(static_cast<int>(nib & 0xffu) - 8) * d,
                                 static_cast<float>(static_cast<int>((nib >> 8) & 0xffu) - 8) * d);
        pk[2 * t + 1] = F16<T>::pack(static_cast<float>(static_cast<int>((nib >> 16) & 0xffu) - 8) * d,
                                     static_cast<float>(static_cast<int>(nib >> 24) - 8) * d);
      }
    }
    *reinterpret_cast<uint4*>(brow + (((4 * h + c) ^ (r & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  }
}

// WQ = 1: B is q8_0, WQ = 2: B is q4_0 (mB* map the codes, mS* the fp16 scales); converter
// warps dequantize each stage into the 16-bit B buffer the MMA reads.
template <int EPI, typename T, int WQ = 0>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairCfg::threads(EPI, WQ), 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap mA, const __grid_constant__ CUtensorMap mB0,
                     const __grid_constant__ CUtensorMap mB1, const __grid_constant__ CUtensorMap mB2,
                     const __grid_constant__ CUtensorMap mS0, const __grid_constant__ CUtensorMap mS1,
                     const __grid_constant__ CUtensorMap mS2, const __grid_constant__ CUtensorMap mD,
                     const GemmParams p, const __grid_constant__ MixParams mp) {
  using Cfg = PairCfg;
  constexpr int S = Cfg::stages(WQ);
  constexpr int RAWB = Cfg::raw_bytes(WQ);
  constexpr int BN = Cfg::BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + S * Cfg::A_BYTES;
  uint8_t* sR = sB + S * Cfg::B_BYTES;  // raw stages of quantized weights (WQ)
  uint64_t* bars = reinterpret_cast<uint64_t*>(sR + S * RAWB);
  uint64_t* rawfull = bars + 20;        // WQ: this CTA's raw codes and scales of a stage landed
  static_assert(!WQ || (2 * S + 5 <= 20 && 20 + S <= 32), "barrier block");
  uint64_t* full = bars;            // leader: both CTAs' bytes of a stage
  uint64_t* empty = bars + S;       // both: the pair's MMAs on a stage completed
  uint64_t* tfull = bars + 2 * S;   // both: the pair's accumulator is ready
  uint64_t* tempty = bars + 2 * S + 2;  // leader: both CTAs' epilogues released it
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint8_t* mix_stage = reinterpret_cast<uint8_t*>(bars) + 256;
  (void)mix_stage;
  uint8_t* red_stage = reinterpret_cast<uint8_t*>(bars) + 1024;  // 1024-byte aligned
  (void)red_stage;
  uint64_t* stallbar = bars + 18;  // nothing arrives on it (p.stall_item1)
  static_assert(2 * S + 5 <= 18, "the stall barrier's slot is free");

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      // WQ: + one converter team's warps of both CTAs
      mbar_init(&full[i], WQ ? 1 + 2 * 4 : 1);
      mbar_init(&empty[i], 1);
      if (WQ) mbar_init(&rawfull[i], 1);
    }
    mbar_init(stallbar, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 2 * 32 * Cfg::epi_warps(EPI));  // every epilogue thread of both CTAs
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&mA);
    tma_prefetch_desc(&mB0);
    if (p.b_mode != B_SINGLE) tma_prefetch_desc(&mB1);
    if (p.b_mode == B_SEGMENTS) tma_prefetch_desc(&mB2);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer's barriers exist before anything arrives on them
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int num_m = (p.M + 2 * Cfg::BM - 1) / (2 * Cfg::BM);
  const int n_per_tile = (EPI == EPI_SWIGLU_BF16) ? BN / 2 : BN;
  const int num_n = (p.N + n_per_tile - 1) / n_per_tile;
  const int num_k = (p.K + Cfg::BK - 1) / Cfg::BK;
  const int splits = p.splits;
  const int items = num_m * num_n * splits;
  const int cid = blockIdx.x >> 1, ncl = gridDim.x >> 1;

  // producer state (warp 0, lane 0)
  const uint64_t pol_a = l2_policy_evict_last();
  const uint64_t pol_b = l2_policy_evict_normal();
  uint32_t armed = 0;
  // This CTA's half of the B tile of an item: tensor map and first row.  For EPI_MIXER
  // the row comes from the tile table; it is read once per item, so no global load sits
  // between the stages' TMA issues.
  struct BSrc {
    const CUtensorMap* m;  // the B matrix (WQ: its codes)
    const CUtensorMap* s;  // WQ: its scales
    int row;
  };
  auto b_src = [&](int it) -> BSrc {
    const int n_blk = (it / num_m) / splits;
    if constexpr (EPI == EPI_MIXER) {  // the table gives each half's first weight row
      return {&mB0, &mS0, rank ? mp.tiles[n_blk].col1 : mp.tiles[n_blk].col0};
    } else if (p.b_mode == B_PAIRED) {  // gate rows in the leader, up rows in the peer
      return {rank ? &mB1 : &mB0, rank ? &mS1 : &mS0, n_blk * (BN / 2)};
    } else if (p.b_mode == B_SEGMENTS) {
      const int n0 = n_blk * BN + static_cast<int>(rank) * (BN / 2);
      const int seg = n0 / p.seg_rows;
      return {seg == 0 ? &mB0 : (seg == 1 ? &mB1 : &mB2), seg == 0 ? &mS0 : (seg == 1 ? &mS1 : &mS2),
              n0 - seg * p.seg_rows};
    } else {
      return {&mB0, &mS0, n_blk * BN + static_cast<int>(rank) * (BN / 2)};
    }
  };
  auto k_range = [&](int it, int& kb0, int& kb1) {
    const int sp = (it / num_m) % splits;
    kb0 = sp * num_k / splits;
    kb1 = (sp + 1) * num_k / splits;
  };
  // Weights are never written by the kernels on the stream: the first item's first stages
  // of B are requested before waiting for the previous kernel (their stages are fresh, so
  // no empty-barrier wait is needed); only A waits.
  int npre = 0;
  if (!WQ && warp == 0 && lane == 0 && p.b_const && cid < items) {
    int kb0, kb1;
    k_range(cid, kb0, kb1);
    const BSrc bs = b_src(cid);
    npre = kb1 - kb0 < S ? kb1 - kb0 : S;
    for (int q = 0; q < npre; ++q) {
      if (leader) {
        mbar_arrive_expect_tx(&full[q], 2 * Cfg::STAGE_BYTES);
        armed |= 1u << q;
      }
      tma_load_2d_pair(sB + q * Cfg::B_BYTES, bs.m, mapa_shared(smem_u32(&full[q]), 0),
                       (kb0 + q) * Cfg::BK, bs.row, pol_b);
    }
  }
  griddep_wait_and_release();  // activations and outputs belong to earlier kernels

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer (both CTAs)
      int stage = 0;
      uint32_t phase = 0;
      int cnt = 0;  // k-blocks issued
      bool ok = true;
      int kb0, kb1;
      if (cid < items) k_range(cid, kb0, kb1);
      BSrc bs = cid < items ? b_src(cid) : BSrc{&mB0, &mS0, 0};
      uint32_t rarmed = 0;  // WQ: raw stages armed
      for (int it = cid; it < items && ok; it += ncl) {
        const int m_blk = it % num_m;
        const int nit = it + ncl;  // this CTA's next item
        int nkb0 = 0, nkb1 = 0;
        BSrc nbs = bs;
        if (nit < items) {
          k_range(nit, nkb0, nkb1);
          nbs = b_src(nit);
        }
        for (int kb = kb0; kb < kb1; ++kb, ++cnt) {
          const bool pre = cnt < npre;  // B already requested, stage armed
          if (!pre && !mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          if (leader && !pre) {  // WQ: the B bytes come from the converters' arrivals
            mbar_arrive_expect_tx(&full[stage], 2 * (WQ ? Cfg::A_BYTES : Cfg::STAGE_BYTES));
            armed |= 1u << stage;
          }
          const uint32_t fb = mapa_shared(smem_u32(&full[stage]), 0);
          const int kc = kb * Cfg::BK;
          tma_load_2d_pair(sA + stage * Cfg::A_BYTES, &mA, fb, kc,
                           m_blk * 2 * Cfg::BM + static_cast<int>(rank) * Cfg::BM, pol_a);
          if constexpr (WQ) {  // this CTA's codes (64 k x 128 rows) and scales (2 blocks x 128 rows)
            uint8_t* raw = sR + stage * RAWB;
            mbar_arrive_expect_tx(&rawfull[stage], RAWB);
            rarmed |= 1u << stage;
            tma_load_2d(raw, bs.m, &rawfull[stage], WQ == 2 ? kc / 2 : kc, bs.row, pol_b);
            tma_load_2d(raw + Cfg::raw_codes(WQ), bs.s, &rawfull[stage], bs.row, kc / 32, pol_b);
          } else if (!pre) {
            tma_load_2d_pair(sB + stage * Cfg::B_BYTES, bs.m, fb, kc, bs.row, pol_b);
          }
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        kb0 = nkb0;
        kb1 = nkb1;
        bs = nbs;
      }
      if (!ok) {
        *abort_flag = 1;
        set_device_error(p.err, KVA_DEV_WAIT_TIMEOUT);
      }
      if (leader) {  // every stage armed here has landed (both CTAs' bytes) before exit
        int st = stage;
        uint32_t ph = phase;
        for (int i = 0; i < S; ++i) {
          if (st == 0) {
            st = S - 1;
            ph ^= 1u;
          } else {
            --st;
          }
          if (armed & (1u << st)) {
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&full[st], ph)) {
              if (globaltimer_ns() - t0 > kWaitLimitNs) break;
            }
          }
        }
      }
      if (WQ) {  // and every raw stage this CTA requested
        int st = stage;
        uint32_t ph = phase;
        for (int i = 0; i < S; ++i) {
          if (st == 0) {
            st = S - 1;
            ph ^= 1u;
          } else {
            --st;
          }
          if (rarmed & (1u << st)) {
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&rawfull[st], ph)) {
              if (globaltimer_ns() - t0 > kWaitLimitNs) break;
            }
          }
        }
      }
    }
  } else if (warp == 1) {
    if (leader) {
      // ------------------------------------------------ MMA issuer (leader only)
      // The warp runs the loop converged and one elected lane issues: from a converged warp
      // the operands stay in uniform registers and an MMA issues in about half the time it
      // takes from a lone lane.  The lane is elected once: a commit only tracks the MMAs
      // of the lane that issues it.
      constexpr uint32_t idesc = idesc_f16kind_f32(2 * Cfg::BM, BN, F16<T>::umma_fmt);
      const uint32_t issuer = elect_one();
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int it = cid; it < items && ok; it += ncl) {
        if (p.stall_item1 == it + 1) {
          // test of the failure path: a wait that runs out (about a millisecond), then the
          // abort and drain below, as for any pipeline wait that gives up
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(stallbar, 0))
            if (globaltimer_ns() - t0 > 1000000ull) break;
          __syncwarp();
          ok = false;
          break;
        }
        if (!mbar_wait_warp(&tempty[acc], acc_phase ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        const int sp = (it / num_m) % splits;
        const int kb0 = sp * num_k / splits, kb1 = (sp + 1) * num_k / splits;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait_warp<WQ != 0>(&full[stage], phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + stage * Cfg::A_BYTES);
          const uint32_t b_base = smem_u32(sB + stage * Cfg::B_BYTES);
          if (issuer) {
#pragma unroll
            for (int j = 0; j < Cfg::BK / 16; ++j) {
              umma_f16_ss_pair(d_tmem, sdesc_k_sw128(a_base + 32 * j), sdesc_k_sw128(b_base + 32 * j),
                               idesc, (kb != kb0 || j != 0) ? 1u : 0u);
            }
            umma_commit_pair(&empty[stage], 0x3);
          }
          __syncwarp();
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (issuer) umma_commit_pair(&tfull[acc], 0x3);
        __syncwarp();
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (!ok && lane == 0) {
        *abort_flag = 1;
        set_device_error(p.err, KVA_DEV_WAIT_TIMEOUT);
      }
      // Drain: the pair's MMAs complete before either CTA releases TMEM or exits.
      if (issuer) {
        umma_commit_pair(&tfull[acc], 0x3);
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(&tfull[acc], acc_phase)) {
          if (globaltimer_ns() - t0 > kWaitLimitNs) break;
        }
      }
      __syncwarp();
    }
  } else if (WQ && warp >= 2 + Cfg::epi_warps(EPI)) {
    // ------------------------------------------------ q8_0 converters (both CTAs)
    // converter team t (warps 4 t .. 4 t + 3) takes the k-blocks whose running count is t
    // modulo the team count, so the teams' stages are converted at the same time; warp c
    // of a team owns rows 32 c .. 32 c + 31 of this CTA's B half.  Once a stage's raw codes
    // and scales have landed the warp writes its rows of the 16-bit B tile and arrives on
    // the leader's full barrier (its stores made visible to the tensor cores first)
    const int cw = warp - 2 - Cfg::epi_warps(EPI);
    const int team = cw / 4, r = (cw & 3) * 32 + lane;
    int stage = 0, cnt = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int it = cid; it < items && ok; it += ncl) {
      int kb0, kb1;
      k_range(it, kb0, kb1);
      for (int kb = kb0; kb < kb1; ++kb, ++cnt) {
        if (cnt % Cfg::conv_teams(EPI) == team) {
          ok = __all_sync(0xffffffffu, mbar_wait(&rawfull[stage], phase, abort_flag));
          if (!ok) break;
#pragma unroll
          for (int hb = 0; hb < 2; ++hb) {
            if constexpr (WQ == 2)
              q4_0_dequant_block<T>(sR + stage * RAWB, sB + stage * Cfg::B_BYTES, r, hb);
            else
              q8_0_dequant_block<T>(sR + stage * RAWB, sB + stage * Cfg::B_BYTES, r, hb);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (leader) mbar_arrive(&full[stage]);
            else mbar_arrive_remote(mapa_shared(smem_u32(&full[stage]), 0));
          }
        }
        if (++stage == S) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (!ok) {
      *abort_flag = 1;
      set_device_error(p.err, KVA_DEV_WAIT_TIMEOUT);
    }
  } else {
    // ------------------------------------------------ epilogue warps 2.. (both CTAs)
    const int q = warp & 3;                 // TMEM lane quarter this warp may access
    const int grp = (warp - 2) >> 2;        // column group (state-update epilogue)
    (void)grp;
    int turn = 0;                           // the next staging buffer (conv rows / reductions)
    (void)turn;

    const uint32_t tempty_lead[2] = {mapa_shared(smem_u32(&tempty[0]), 0),
                                     mapa_shared(smem_u32(&tempty[1]), 0)};
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int it = cid; it < items; it += ncl) {
      const int m_blk = it % num_m;
      const int n_blk = (it / num_m) / splits;
      const bool got = mbar_wait(&tfull[acc], acc_phase, abort_flag);
      if (!got) {
        *abort_flag = 1;
        set_device_error(p.err, KVA_DEV_WAIT_TIMEOUT);
      }
      if constexpr (EPI == EPI_MIXER) {
        // the epilogue warps meet at named barriers inside the epilogue, so they leave
        // together: a barrier-reduction vote over all of them
        if (!mix_all(got)) break;
      } else if (!got) {
        break;
      }
      tc_fence_after();
      if constexpr (EPI == EPI_MIXER)
        epilogue_mixer<T>(mp, tmem_base + static_cast<uint32_t>(acc * BN),
                          m_blk * 2 * Cfg::BM + static_cast<int>(rank) * Cfg::BM, n_blk, q, grp, lane,
                          mix_stage, turn);
      else if (EPI == EPI_ADD_F32 && p.d_tma)
        epilogue_add_tma(&mD, tmem_base + static_cast<uint32_t>(acc * BN),
                         m_blk * 2 * Cfg::BM + static_cast<int>(rank) * Cfg::BM, n_blk * BN, q, lane,
                         red_stage + q * 2 * RED_BUF_BYTES, turn);
      else if ((EPI == EPI_STORE_BF16 || EPI == EPI_SWIGLU_BF16) && p.d_tma)
        epilogue_store_tma<EPI, T>(&mD, tmem_base + static_cast<uint32_t>(acc * BN),
                                   m_blk * 2 * Cfg::BM + static_cast<int>(rank) * Cfg::BM,
                                   n_blk * n_per_tile, n_per_tile, q, lane,
                                   red_stage + q * 2 * RED_BUF_BYTES, turn);
      else
        epilogue_tile<BN, EPI, T>(p, tmem_base + static_cast<uint32_t>(acc * BN),
                                  m_blk * 2 * Cfg::BM + static_cast<int>(rank) * Cfg::BM, n_blk, q,
                                  lane);
      tc_fence_before();
      if (leader) mbar_arrive(&tempty[acc]);
      else mbar_arrive_remote(tempty_lead[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    // the reductions have read their buffers and written D before the CTA exits
    if (EPI != EPI_MIXER && p.d_tma && lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the leader's MMAs (reading the peer's shared memory) are done
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// 16-bit row-major [rows, inner] with row stride `ld` elements; box [box_rows, 64].
static bool make_map(CUtensorMap* m, const void* base, int64_t inner, int64_t rows, int64_t ld,
                     int box_rows, CUtensorMapDataType dt) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, dt, 2, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// fp32 row-major [rows, inner] (row stride ld elements) as a reduction target: box
// [32 rows, 32 columns] = 128 bytes per row, 128-byte swizzle.
static bool make_map_f32_red(CUtensorMap* m, const void* base, int64_t inner, int64_t rows, int64_t ld) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 4};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_map_2d_16bit(void* map, const void* base, bool fp16, int64_t inner, int64_t rows,
                       int64_t ld, int box_inner, int box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(static_cast<CUtensorMap*>(map),
                   fp16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// q8_0 weights: codes int8 [rows, K] (box 128 rows x 64 bytes, 64-byte swizzle) and scales
// fp16 [K / 32, rows] (box 2 blocks x 128 rows).
static bool make_map_q8_codes(CUtensorMap* m, const void* base, int64_t K, int64_t rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(K)};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// q4_0 weights: packed codes uint8 [rows, K / 2] (box 128 rows x 32 bytes, 32-byte swizzle)
static bool make_map_q4_codes(CUtensorMap* m, const void* base, int64_t K, int64_t rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 2)};
  cuuint32_t box[2] = {32, 128};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
static bool make_map_q8_scales(CUtensorMap* m, const void* base, int64_t K, int64_t rows, int64_t ld) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(K / 32)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  cuuint32_t box[2] = {128, 2};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_3d_16bit(void* map, const void* base, bool fp16, int64_t d0, int64_t d1,
                       int64_t d2, int box0, int box1) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d0), static_cast<cuuint64_t>(d1),
                        static_cast<cuuint64_t>(d2)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d0) * 2, static_cast<cuuint64_t>(d0 * d1) * 2};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(box0), static_cast<cuuint32_t>(box1), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(static_cast<CUtensorMap*>(map),
                   fp16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                   const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Split-K factor for the residual-add GEMMs (whose partial sums are added by TMA
// reduce-adds): the number of K ranges s in [1, 8] (each at least 4 K blocks) that
// minimises the waves of work items per unit of K work, ceil(tiles * s / slots) / s,
// with a small charge per extra split for its atomic traffic.
static int choose_splits(int tiles, int slots, int num_k) {
  int best = 1;
  double best_cost = 1e30;
  for (int sp = 1; sp <= 8; ++sp) {
    if (sp > 1 && num_k / sp < 4) break;
    const int waves = (tiles * sp + slots - 1) / slots;
    const double cost = static_cast<double>(waves) / sp + 0.02 * (sp - 1);
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best = sp;
    }
  }
  return best;
}

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
  return n;
}

template <int BN, int EPI, typename T>
static int launch_instance(const GemmArgs& a, cudaStream_t s) {
  const CUtensorMapDataType dt = std::is_same<T, __half>::value ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                                : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  using Cfg = GemmCfg<BN>;
  const bool paired = a.b_mode == B_PAIRED;
  const int box_b = paired ? BN / 2 : BN;
  CUtensorMap mA, mB[3];
  if (!make_map(&mA, a.A, a.K, a.M, a.lda, Cfg::BM, dt)) return KVA_ERR_CUDA;
  const int nb = a.b_mode == B_SINGLE ? 1 : (paired ? 2 : 3);
  const int64_t b_rows = a.b_mode == B_SEGMENTS ? a.seg_rows : a.N;
  for (int i = 0; i < 3; ++i) {
    const void* src = a.B[i < nb ? i : 0];
    if (!make_map(&mB[i], src, a.K, b_rows, a.ldb, box_b, dt)) return KVA_ERR_CUDA;
  }
  GemmParams p = {};
  p.M = a.M;
  p.N = a.N;
  p.K = a.K;
  p.b_mode = a.b_mode;
  p.seg_rows = static_cast<int>(a.seg_rows);
  p.D = a.D;
  p.ldd = a.ldd;
  p.D1 = a.D1;
  p.ldd1 = a.ldd1;
  p.n_split = a.n_split;
  p.err = a.err;
  const int n_per_tile = paired ? BN / 2 : BN;
  const int num_m = (a.M + Cfg::BM - 1) / Cfg::BM;
  const int num_k = (a.K + Cfg::BK - 1) / Cfg::BK;
  int splits = 1;
  if (EPI == EPI_ADD_F32) {
    const int t = num_m * ((a.N + n_per_tile - 1) / n_per_tile);
    splits = a.splits > 0 ? a.splits : choose_splits(t, num_sms(), num_k);
  }
  p.splits = splits;
  const int tiles = num_m * ((a.N + n_per_tile - 1) / n_per_tile) * splits;
  int grid = tiles < num_sms() ? tiles : num_sms();
  // whole groups of num_m CTAs: a CTA keeps its M tile, and the num_m CTAs that share
  // a weight tile run side by side
  if (tiles > grid && num_m > 1 && grid >= num_m && num_m <= 16) grid -= grid % num_m;
  auto kern = gemm_tc_kernel<BN, EPI, T>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM) !=
      cudaSuccess)
    return KVA_ERR_CUDA;
  if (launch_pdl(kern, dim3(grid), dim3(192), Cfg::SMEM, s, mA, mB[0], mB[1], mB[2], p) != cudaSuccess)
    return KVA_ERR_CUDA;
  return cudaPeekAtLastError() == cudaSuccess ? KVA_OK : KVA_ERR_CUDA;
}


static bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

template <int EPI, typename T>
static int launch_pair(const GemmArgs& a, cudaStream_t s) {
  using Cfg = PairCfg;
  const CUtensorMapDataType dt = std::is_same<T, __half>::value ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                                : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const bool paired = a.b_mode == B_PAIRED;
  CUtensorMap mA, mB[3];
  if (!make_map(&mA, a.A, a.K, a.M, a.lda, Cfg::BM, dt)) return KVA_ERR_CUDA;
  const int nb = a.b_mode == B_SINGLE ? 1 : (paired ? 2 : 3);
  const int64_t b_rows = a.b_mode == B_SEGMENTS ? a.seg_rows : a.N;
  for (int i = 0; i < 3; ++i) {
    const void* src = a.B[i < nb ? i : 0];
    if (!make_map(&mB[i], src, a.K, b_rows, a.ldb, Cfg::BN / 2, dt)) return KVA_ERR_CUDA;
  }
  GemmParams p = {};
  p.M = a.M;
  p.N = a.N;
  p.K = a.K;
  p.b_mode = a.b_mode;
  p.seg_rows = static_cast<int>(a.seg_rows);
  p.D = a.D;
  p.ldd = a.ldd;
  p.D1 = a.D1;
  p.ldd1 = a.ldd1;
  p.n_split = a.n_split;
  p.err = a.err;
  p.b_const = a.b_const ? 1 : 0;
  p.stall_item1 = a.stall_item1;
  // residual adds by TMA reduction when D is a plain fp32 matrix the tensor map can describe
  CUtensorMap mD = mA;
  p.d_tma = 0;
  if (EPI == EPI_ADD_F32 && a.n_split == 0 && (reinterpret_cast<uintptr_t>(a.D) & 15u) == 0 &&
      a.ldd % 4 == 0 && a.N % 4 == 0) {
    if (!make_map_f32_red(&mD, a.D, a.N, a.M, a.ldd)) return KVA_ERR_CUDA;
    p.d_tma = 1;
  }
  // 16-bit outputs by TMA stores (box 32 rows x 64 columns)
  if ((EPI == EPI_STORE_BF16 || EPI == EPI_SWIGLU_BF16) && a.n_split == 0 &&
      (reinterpret_cast<uintptr_t>(a.D) & 15u) == 0 && a.ldd % 8 == 0 && a.N % 8 == 0) {
    if (!make_map_2d_16bit(&mD, a.D, std::is_same<T, __half>::value, a.N, a.M, a.ldd, 64, 32))
      return KVA_ERR_CUDA;
    p.d_tma = 1;
  }
  const int smem = p.d_tma ? Cfg::SMEM_RED : Cfg::SMEM;
  const int n_per_tile = paired ? Cfg::BN / 2 : Cfg::BN;
  const int num_m = (a.M + 2 * Cfg::BM - 1) / (2 * Cfg::BM);
  const int num_k = (a.K + Cfg::BK - 1) / Cfg::BK;
  const int max_cl = num_sms() / 2;
  int splits = 1;
  if (EPI == EPI_ADD_F32) {
    const int t = num_m * ((a.N + n_per_tile - 1) / n_per_tile);
    splits = a.splits > 0 ? a.splits : choose_splits(t, max_cl, num_k);
  }
  p.splits = splits;
  const int items = num_m * ((a.N + n_per_tile - 1) / n_per_tile) * splits;
  int ncl = items < max_cl ? items : max_cl;
  if (items > ncl && num_m > 1 && ncl >= num_m && num_m <= 16) ncl -= ncl % num_m;
  auto kern = gemm_pair_kernel<EPI, T>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return KVA_ERR_CUDA;
  if (launch_pdl(kern, dim3(2 * ncl), dim3(Cfg::threads(EPI)), smem, s, mA, mB[0], mB[1], mB[2], mA, mA,
                 mA, mD, p, MixParams()) != cudaSuccess)
    return KVA_ERR_CUDA;
  return cudaPeekAtLastError() == cudaSuccess ? KVA_OK : KVA_ERR_CUDA;
}

// Quantized weights on CTA pairs (WQ 1: q8_0, 2: q4_0): B[i] are the codes, Bs[i] the fp16
// scales of matrix i.
template <int EPI, typename T, int WQ>
static int launch_pair_wq(const GemmArgs& a, cudaStream_t s) {
  using Cfg = PairCfg;
  const CUtensorMapDataType dt = std::is_same<T, __half>::value ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                                : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const bool paired = a.b_mode == B_PAIRED;
  CUtensorMap mA, mB[3], mS[3];
  if (!make_map(&mA, a.A, a.K, a.M, a.lda, Cfg::BM, dt)) return KVA_ERR_CUDA;
  const int nb = a.b_mode == B_SINGLE ? 1 : (paired ? 2 : 3);
  const int64_t b_rows = a.b_mode == B_SEGMENTS ? a.seg_rows : a.N;
  for (int i = 0; i < 3; ++i) {
    const int j = i < nb ? i : 0;
    const bool codes_ok = WQ == 2 ? make_map_q4_codes(&mB[i], a.B[j], a.K, b_rows)
                                  : make_map_q8_codes(&mB[i], a.B[j], a.K, b_rows);
    if (!codes_ok ||
        !make_map_q8_scales(&mS[i], a.Bs[j], a.K, b_rows, a.lds > 0 ? a.lds : b_rows))
      return KVA_ERR_CUDA;
  }
  GemmParams p = {};
  p.M = a.M;
  p.N = a.N;
  p.K = a.K;
  p.b_mode = a.b_mode;
  p.seg_rows = static_cast<int>(a.seg_rows);
  p.D = a.D;
  p.ldd = a.ldd;
  p.err = a.err;
  const int n_per_tile = paired ? Cfg::BN / 2 : Cfg::BN;
  const int num_m = (a.M + 2 * Cfg::BM - 1) / (2 * Cfg::BM);
  const int num_k = (a.K + Cfg::BK - 1) / Cfg::BK;
  const int max_cl = num_sms() / 2;
  int splits = 1;
  if (EPI == EPI_ADD_F32) {
    const int t = num_m * ((a.N + n_per_tile - 1) / n_per_tile);
    splits = a.splits > 0 ? a.splits : choose_splits(t, max_cl, num_k);
  }
  p.splits = splits;
  const int items = num_m * ((a.N + n_per_tile - 1) / n_per_tile) * splits;
  int ncl = items < max_cl ? items : max_cl;
  if (items > ncl && num_m > 1 && ncl >= num_m && num_m <= 16) ncl -= ncl % num_m;
  auto kern = gemm_pair_kernel<EPI, T, WQ>;
  constexpr int smem = WQ == 2 ? Cfg::SMEM_Q4 : Cfg::SMEM_Q8;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return KVA_ERR_CUDA;
  if (launch_pdl(kern, dim3(2 * ncl), dim3(Cfg::threads(EPI, WQ)), smem, s, mA, mB[0], mB[1], mB[2],
                 mS[0], mS[1], mS[2], mA, p, MixParams()) != cudaSuccess)
    return KVA_ERR_CUDA;
  return KVA_OK;
}

template <typename T>
static int launch_heads_fused_t(const void* A, int64_t lda, const void* W, int64_t n_rows_w, int M,
                                int K, int num_tiles, const MixParams& mp, cudaStream_t s) {
  using Cfg = PairCfg;
  const CUtensorMapDataType dt = std::is_same<T, __half>::value ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                                : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUtensorMap mA, mB;
  if (!make_map(&mA, A, K, M, lda, Cfg::BM, dt)) return KVA_ERR_CUDA;
  if (!make_map(&mB, W, K, n_rows_w, K, Cfg::BN / 2, dt)) return KVA_ERR_CUDA;
  GemmParams p = {};
  p.M = M;
  p.N = num_tiles * Cfg::BN;  // one tile per table entry
  p.K = K;
  p.b_mode = B_SINGLE;
  p.seg_rows = 0;
  p.D = nullptr;
  p.ldd = 0;
  p.D1 = nullptr;
  p.ldd1 = 0;
  p.n_split = 0;
  p.splits = 1;
  p.err = mp.err;
  p.b_const = 1;  // the heads matrix and the tile table are fixed
  const int num_m = (M + 2 * Cfg::BM - 1) / (2 * Cfg::BM);
  const int max_cl = num_sms() / 2;
  const int items = num_m * num_tiles;
  int ncl = items < max_cl ? items : max_cl;
  if (items > ncl && num_m > 1 && ncl >= num_m && num_m <= 16) ncl -= ncl % num_m;
  auto kern = gemm_pair_kernel<EPI_MIXER, T>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_MIX) !=
      cudaSuccess)
    return KVA_ERR_CUDA;
  if (launch_pdl(kern, dim3(2 * ncl), dim3(Cfg::threads(EPI_MIXER)), Cfg::SMEM_MIX, s, mA, mB, mB, mB, mA,
                 mA, mA, mA, p, mp) != cudaSuccess)
    return KVA_ERR_CUDA;
  return cudaPeekAtLastError() == cudaSuccess ? KVA_OK : KVA_ERR_CUDA;
}

int launch_heads_fused(int dtype, const void* A, int64_t lda, const void* W, int64_t n_rows_w,
                       int M, int K, int num_tiles, const MixParams& mp, cudaStream_t s) {
  if (M == 0 || num_tiles == 0) return KVA_OK;
  if (!A || !W || !mp.tiles || M < 0 || K <= 0) return KVA_ERR_INVALID_ARG;
  if (!aligned16(A) || !aligned16(W) || (lda % 8) || (K % 8)) return KVA_ERR_ALIGNMENT;
  if (dtype == KVA_F16) return launch_heads_fused_t<__half>(A, lda, W, n_rows_w, M, K, num_tiles, mp, s);
  if (dtype == KVA_BF16)
    return launch_heads_fused_t<__nv_bfloat16>(A, lda, W, n_rows_w, M, K, num_tiles, mp, s);
  return KVA_ERR_INVALID_ARG;
}


int launch_gemm(const GemmArgs& a, cudaStream_t s) {
  if (a.M <= 0 || a.N <= 0 || a.K <= 0) return a.M == 0 ? KVA_OK : KVA_ERR_INVALID_ARG;
  if (!a.A || !a.B[0] || !a.D) return KVA_ERR_INVALID_ARG;
  if (!aligned16(a.A) || !aligned16(a.B[0]) || !aligned16(a.D)) return KVA_ERR_ALIGNMENT;
  if ((a.lda % 8) || (a.ldb % 8) || (a.K % 8)) return KVA_ERR_ALIGNMENT;
  const bool f32out = a.epilogue == EPI_STORE_F32 || a.epilogue == EPI_ADD_F32;
  if (a.ldd % (f32out ? 4 : 8)) return KVA_ERR_ALIGNMENT;
  if (a.n_split > 0) {
    if (!a.D1 || !aligned16(a.D1) || (a.n_split % 32) || (a.ldd1 % (f32out ? 4 : 8)))
      return KVA_ERR_ALIGNMENT;
  }
  if (a.b_mode == B_PAIRED && (a.epilogue != EPI_SWIGLU_BF16 || !a.B[1] || !aligned16(a.B[1])))
    return KVA_ERR_INVALID_ARG;
  if (a.epilogue == EPI_SWIGLU_BF16 && a.b_mode != B_PAIRED) return KVA_ERR_INVALID_ARG;
  // block_n: 128 / 256 one-CTA tiles of that width, 512 a CTA pair on a 256 x 256 tile
  // (the default wherever the B layout allows it)
  int bn = a.block_n;
  if (bn == 0) bn = (a.b_mode != B_SEGMENTS || (a.seg_rows > 0 && a.seg_rows % 256 == 0)) ? 512 : 128;
  if (a.b_mode == B_SEGMENTS) {
    if (!a.B[1] || !a.B[2] || !aligned16(a.B[1]) || !aligned16(a.B[2])) return KVA_ERR_INVALID_ARG;
    const int seg_tile = bn == 512 ? 256 : bn;
    if (a.seg_rows <= 0 || a.seg_rows % seg_tile || a.N != 3 * a.seg_rows) return KVA_ERR_UNSUPPORTED;
  }
  if (bn != 128 && bn != 256 && bn != 512) return KVA_ERR_UNSUPPORTED;
  if (a.dtype != KVA_BF16 && a.dtype != KVA_F16) return KVA_ERR_INVALID_ARG;
  const bool h = a.dtype == KVA_F16;
  if (a.wq) {  // q8_0 / q4_0 weights: CTA pairs, plain epilogues (STORE, ADD_F32, SWIGLU)
    if (a.K % 64 || a.n_split || bn != 512) return KVA_ERR_UNSUPPORTED;
    const int64_t b_rows = a.b_mode == B_SEGMENTS ? a.seg_rows : a.N;
    if (b_rows % 8 || a.lds % 8) return KVA_ERR_ALIGNMENT;  // scale rows of 16-byte multiples
    for (int i = 0; i < (a.b_mode == B_SINGLE ? 1 : (a.b_mode == B_PAIRED ? 2 : 3)); ++i)
      if (!a.Bs[i] || !aligned16(a.Bs[i]) || !a.B[i] || !aligned16(a.B[i])) return KVA_ERR_INVALID_ARG;
    if (a.wq != 1 && a.wq != 2) return KVA_ERR_INVALID_ARG;
#define KVA_WQ_CASE(E)                                                                          \
  case E:                                                                                       \
    if (a.wq == 1) return h ? launch_pair_wq<E, __half, 1>(a, s) : launch_pair_wq<E, __nv_bfloat16, 1>(a, s); \
    return h ? launch_pair_wq<E, __half, 2>(a, s) : launch_pair_wq<E, __nv_bfloat16, 2>(a, s);
    switch (a.epilogue) {
      KVA_WQ_CASE(EPI_STORE_BF16)
      KVA_WQ_CASE(EPI_ADD_F32)
      KVA_WQ_CASE(EPI_SWIGLU_BF16)
      default:
        return KVA_ERR_UNSUPPORTED;
    }
#undef KVA_WQ_CASE
  }
#define KVA_GEMM_CASE(E)                                                                   \
  case E:                                                                                  \
    if (bn == 512) return h ? launch_pair<E, __half>(a, s) : launch_pair<E, __nv_bfloat16>(a, s); \
    if (h) return bn == 256 ? launch_instance<256, E, __half>(a, s)                        \
                            : launch_instance<128, E, __half>(a, s);                       \
    return bn == 256 ? launch_instance<256, E, __nv_bfloat16>(a, s)                        \
                     : launch_instance<128, E, __nv_bfloat16>(a, s);
  switch (a.epilogue) {
    KVA_GEMM_CASE(EPI_STORE_BF16)
    KVA_GEMM_CASE(EPI_STORE_F32)
    KVA_GEMM_CASE(EPI_ADD_F32)
    KVA_GEMM_CASE(EPI_SWIGLU_BF16)
    default:
      return KVA_ERR_INVALID_ARG;
  }
#undef KVA_GEMM_CASE
}

}  // namespace kva
