// Block-causal multi-head attention of the projector blocks ("Qwen3.8-27B-KVA"
// model card, architecture table row "attention": heads @ 128, causal within
// 1024-token blocks for r3, full causal within the ubatch for r2).
//
// Key j is visible to query i iff j <= i and floor(i/W) == floor(j/W), indices
// local to the ubatch (W = window, or the whole ubatch when window = 0).
// Flash-style: 64-query tiles, 4 warps x 16 query rows; a CTA takes the query tiles
// b and n-1-b of one head so every CTA does the same causal work (two CTAs per SM),
// 64-key tiles double-buffered in shared memory with cp.async, S = Q K^T and
// O += P V on mma.sync (16-bit in, fp32 accumulate), online softmax in fp32 with
// exp2.  qkv is [T, 3d] 16-bit (q | k | v, head h at columns h*128 of each
// part), output [T, d] in the same format (bf16 or fp16).
#include <cmath>

#include "kva_common.cuh"

namespace kva {

constexpr int ATT_BQ = 64;
constexpr int ATT_BKV = 64;
constexpr int ATT_D = 128;
constexpr int ATT_THREADS = 128;
constexpr int ATT_SMEM = (ATT_BQ + 4 * ATT_BKV) * ATT_D * 2;  // Q + 2 x (K, V)

// byte offset of (row, 16-byte chunk) in a [rows][128] 16-bit tile, XOR swizzled
__device__ __forceinline__ uint32_t att_off(int row, int chunk) {
  return static_cast<uint32_t>(row * 256 + ((chunk ^ (row & 7)) << 4));
}

template <typename E>
__device__ __forceinline__ void att_load_tile(uint32_t dst, const E* src, int64_t ld,
                                              int row0, int rows, int T, int tid) {
  // rows x 16 chunks of 16 bytes; rows at or beyond T are zero-filled
  for (int i = tid; i < rows * 16; i += ATT_THREADS) {
    const int r = i >> 4, c = i & 15;
    const int gr = row0 + r;
    const bool ok = gr < T;
    const E* g = src + static_cast<int64_t>(ok ? gr : 0) * ld + c * 8;
    cp_async16(dst + att_off(r, c), g, ok ? 16u : 0u);
  }
}

template <typename E>
__global__ void __launch_bounds__(ATT_THREADS)
    attention_kernel(const E* __restrict__ qkv, int64_t ldq, E* __restrict__ out, int64_t ldo,
                     int T, int d_model, int window, float scale_log2) {
  griddep_wait_and_release();
  extern __shared__ __align__(128) uint8_t att_smem[];
  const uint32_t sQ = smem_u32(att_smem);
  const uint32_t sK0 = sQ + ATT_BQ * 256;
  const uint32_t sV0 = sK0 + 2 * ATT_BKV * 256;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c = lane & 3;
  // causal balance: CTA b takes query tiles b and n_qt - 1 - b (equal total key tiles)
  const int n_qt = (T + ATT_BQ - 1) / ATT_BQ;
  const int h = blockIdx.y;
  for (int pass = 0; pass < 2; ++pass) {
    const int qt = pass == 0 ? static_cast<int>(blockIdx.x) : n_qt - 1 - static_cast<int>(blockIdx.x);
    if (pass == 1 && qt <= static_cast<int>(blockIdx.x)) break;
    const int q0 = qt * ATT_BQ;
    __syncthreads();  // the previous pass finished reading shared memory
    const int W = window > 0 ? window : 0x3fffffff;

    const E* Qg = qkv + h * ATT_D;
    const E* Kg = qkv + d_model + h * ATT_D;
    const E* Vg = qkv + 2 * d_model + h * ATT_D;

    const int q_last = min(T, q0 + ATT_BQ) - 1;
    const int kv_lo = (q0 / W) * W;             // first key any row of the tile may see
    const int kv_hi = q_last + 1;               // one past the last visible key
    const int t_lo = (kv_lo / ATT_BKV) * ATT_BKV;
    const int n_tiles = (kv_hi - t_lo + ATT_BKV - 1) / ATT_BKV;

    att_load_tile(sQ, Qg, ldq, q0, ATT_BQ, T, tid);
    att_load_tile(sK0, Kg, ldq, t_lo, ATT_BKV, T, tid);
    att_load_tile(sV0, Vg, ldq, t_lo, ATT_BKV, T, tid);
    cp_async_commit();

    // rows of this thread
    const int r0 = q0 + warp * 16 + g;
    const int r1 = r0 + 8;
    const int lo0 = (r0 / W) * W, lo1 = (r1 / W) * W;

    float o[16][4];
  #pragma unroll
    for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    uint32_t qf[8][4];

    for (int it = 0; it < n_tiles; ++it) {
      const int buf = it & 1;
      if (it + 1 < n_tiles) {
        const int nb = (it + 1) & 1;
        att_load_tile(sK0 + nb * ATT_BKV * 256, Kg, ldq, t_lo + (it + 1) * ATT_BKV, ATT_BKV, T, tid);
        att_load_tile(sV0 + nb * ATT_BKV * 256, Vg, ldq, t_lo + (it + 1) * ATT_BKV, ATT_BKV, T, tid);
        cp_async_commit();
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();
      if (it == 0) {
        // Q fragments for this warp's 16 rows, all 8 k-steps
  #pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const int mi = lane >> 3;
          const int row = warp * 16 + (mi & 1) * 8 + (lane & 7);
          const int ch = ks * 2 + (mi >> 1);
          ldmatrix_x4(qf[ks], sQ + att_off(row, ch));
        }
      }
      const uint32_t sK = sK0 + buf * ATT_BKV * 256;
      const uint32_t sV = sV0 + buf * ATT_BKV * 256;
      const int j0 = t_lo + it * ATT_BKV;

      float s[8][4];
  #pragma unroll
      for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
  #pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
  #pragma unroll
        for (int nt = 0; nt < 8; nt += 2) {
          uint32_t kb[4];
          const int mi = lane >> 3;
          const int row = nt * 8 + (mi >> 1) * 8 + (lane & 7);
          const int ch = ks * 2 + (mi & 1);
          ldmatrix_x4(kb, sK + att_off(row, ch));
          uint32_t b0[2] = {kb[0], kb[1]}, b1[2] = {kb[2], kb[3]};
          F16<E>::mma(s[nt], qf[ks], b0);
          F16<E>::mma(s[nt + 1], qf[ks], b1);
        }
      }
      // mask + row max
      float mx0 = -INFINITY, mx1 = -INFINITY;
  #pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
  #pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int j = j0 + nt * 8 + 2 * c + e;
          const bool v0 = j <= r0 && j >= lo0 && j < T;
          const bool v1 = j <= r1 && j >= lo1 && j < T;
          s[nt][e] = v0 ? s[nt][e] : -INFINITY;
          s[nt][2 + e] = v1 ? s[nt][2 + e] : -INFINITY;
          mx0 = fmaxf(mx0, s[nt][e]);
          mx1 = fmaxf(mx1, s[nt][2 + e]);
        }
      }
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
      const float ref0 = mn0 == -INFINITY ? 0.f : mn0 * scale_log2;
      const float ref1 = mn1 == -INFINITY ? 0.f : mn1 * scale_log2;
      const float al0 = exp2f(m0 == -INFINITY ? -INFINITY : m0 * scale_log2 - ref0);
      const float al1 = exp2f(m1 == -INFINITY ? -INFINITY : m1 * scale_log2 - ref1);
      m0 = mn0;
      m1 = mn1;
      float rs0 = 0.f, rs1 = 0.f;
  #pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
  #pragma unroll
        for (int e = 0; e < 2; ++e) {
          s[nt][e] = exp2f(s[nt][e] * scale_log2 - ref0);
          s[nt][2 + e] = exp2f(s[nt][2 + e] * scale_log2 - ref1);
          rs0 += s[nt][e];
          rs1 += s[nt][2 + e];
        }
      }
      rs0 += __shfl_xor_sync(0xffffffffu, rs0, 1);
      rs0 += __shfl_xor_sync(0xffffffffu, rs0, 2);
      rs1 += __shfl_xor_sync(0xffffffffu, rs1, 1);
      rs1 += __shfl_xor_sync(0xffffffffu, rs1, 2);
      l0 = l0 * al0 + rs0;
      l1 = l1 * al1 + rs1;
  #pragma unroll
      for (int i = 0; i < 16; ++i) {
        o[i][0] *= al0;
        o[i][1] *= al0;
        o[i][2] *= al1;
        o[i][3] *= al1;
      }
      // O += P V
  #pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        uint32_t a[4];
        a[0] = F16<E>::pack(s[2 * kk][0], s[2 * kk][1]);
        a[1] = F16<E>::pack(s[2 * kk][2], s[2 * kk][3]);
        a[2] = F16<E>::pack(s[2 * kk + 1][0], s[2 * kk + 1][1]);
        a[3] = F16<E>::pack(s[2 * kk + 1][2], s[2 * kk + 1][3]);
  #pragma unroll
        for (int dt = 0; dt < 16; dt += 2) {
          uint32_t vb[4];
          const int mi = lane >> 3;
          const int row = kk * 16 + (mi & 1) * 8 + (lane & 7);
          const int ch = dt + (mi >> 1);
          ldmatrix_x4_trans(vb, sV + att_off(row, ch));
          uint32_t b0[2] = {vb[0], vb[1]}, b1[2] = {vb[2], vb[3]};
          F16<E>::mma(o[dt], a, b0);
          F16<E>::mma(o[dt + 1], a, b1);
        }
      }
      __syncthreads();  // buffer `buf` is refilled two iterations later
    }

    const float inv0 = l0 > 0.f ? 1.f / l0 : 0.f;
    const float inv1 = l1 > 0.f ? 1.f / l1 : 0.f;
  #pragma unroll
    for (int dt = 0; dt < 16; ++dt) {
      const int col = h * ATT_D + dt * 8 + 2 * c;
      if (r0 < T)
        *reinterpret_cast<uint32_t*>(out + static_cast<int64_t>(r0) * ldo + col) =
            F16<E>::pack(o[dt][0] * inv0, o[dt][1] * inv0);
      if (r1 < T)
        *reinterpret_cast<uint32_t*>(out + static_cast<int64_t>(r1) * ldo + col) =
            F16<E>::pack(o[dt][2] * inv1, o[dt][3] * inv1);
    }
  }
}

int launch_attention(const void* qkv, int64_t ldq, void* out, int64_t ldo, int T, int n_heads,
                     int window, cudaStream_t s, int dtype) {
  if (T == 0) return KVA_OK;
  if (!qkv || !out || T < 0 || n_heads <= 0 || window < 0) return KVA_ERR_INVALID_ARG;
  if (dtype != KVA_BF16 && dtype != KVA_F16) return KVA_ERR_INVALID_ARG;
  if ((ldq % 8) || (ldo % 8) ||
      ((reinterpret_cast<uintptr_t>(qkv) | reinterpret_cast<uintptr_t>(out)) & 15u))
    return KVA_ERR_ALIGNMENT;
  const int d_model = n_heads * ATT_D;
  if (ldq < 3 * d_model || ldo < d_model) return KVA_ERR_INVALID_ARG;
  const float scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(ATT_D));
  const int n_qt = (T + ATT_BQ - 1) / ATT_BQ;
  dim3 grid((n_qt + 1) / 2, n_heads);
  if (dtype == KVA_F16) {
    if (cudaFuncSetAttribute(attention_kernel<__half>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             ATT_SMEM) != cudaSuccess)
      return KVA_ERR_CUDA;
    if (launch_pdl(attention_kernel<__half>, grid, dim3(ATT_THREADS), ATT_SMEM, s,
                   static_cast<const __half*>(qkv), ldq, static_cast<__half*>(out), ldo, T, d_model,
                   window, scale_log2) != cudaSuccess)
      return KVA_ERR_CUDA;
  } else {
    if (cudaFuncSetAttribute(attention_kernel<__nv_bfloat16>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, ATT_SMEM) != cudaSuccess)
      return KVA_ERR_CUDA;
    if (launch_pdl(attention_kernel<__nv_bfloat16>, grid, dim3(ATT_THREADS), ATT_SMEM, s,
                   static_cast<const __nv_bfloat16*>(qkv), ldq, static_cast<__nv_bfloat16*>(out), ldo,
                   T, d_model, window, scale_log2) != cudaSuccess)
      return KVA_ERR_CUDA;
  }
  return cudaPeekAtLastError() == cudaSuccess ? KVA_OK : KVA_ERR_CUDA;
}

}  // namespace kva
