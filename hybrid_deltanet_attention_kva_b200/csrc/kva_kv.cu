// Full-attention late layers: k RMSNorm per KV head, partial RoPE and the KV
// cache write ("Qwen3.8-27B-KVA" model card, late-layer table: the projector
// predicts the k and v projections, and the k norm and RoPE come after it;
// "Qwen3.8-27B-MLA" model card, "What this
// is": 4 KV heads of dim 256 with 64 rotary dims, whose lowest pairs turn
// 3.4 / 2.1 / 1.2 degrees across 131k tokens, i.e. theta = 1e7).
//
// One warp per (token, KV head): each lane holds d_h/32 consecutive dims as one
// 16- (or 8-) byte vector; the RMS is a warp reduction; RoPE pairs (i, i+r/2)
// meet through one xor shuffle; the angle (pos * theta^(-2i/r), the frequencies from a
// table the host fills in fp64) is formed and range-reduced in fp64 before sincosf, so
// it stays exact at 32k+ positions.
// K and V rows are written with one vector store per lane (coalesced rows of
// 512 bytes); V is copied bit for bit.  Paged caches go through the page table,
// an out-of-range entry skips the write and sets the device status word.
#include <type_traits>

#include "kva_common.cuh"

namespace kva {

template <int EPL>
struct VecT;
template <>
struct VecT<8> {
  using T = uint4;
};
template <>
struct VecT<4> {
  using T = uint2;
};

// The cache row of (sequence, head, position), or -1 for a page-table entry out of range
// (which sets the device status word).
__device__ __forceinline__ int64_t kv_row(const KvLaunch& p, int seq, int hh, int64_t pos, int lane) {
  const kva_kv_cache& cc = p.cache;
  if (cc.layout == KVA_KV_PAGED) {
    const int64_t pg_i = pos / cc.page_size;
    if (pg_i < 0 || pg_i >= cc.pages_per_seq) {
      if (lane == 0) set_device_error(p.err, KVA_DEV_PAGE_OOB);
      return -1;
    }
    const int page = cc.page_table[static_cast<int64_t>(seq) * cc.pages_per_seq + pg_i];
    if (page < 0 || page >= cc.n_pages) {
      if (lane == 0) set_device_error(p.err, KVA_DEV_PAGE_OOB);
      return -1;
    }
    return (static_cast<int64_t>(page) * p.n_kv + hh) * cc.page_size + pos % cc.page_size;
  }
  return (static_cast<int64_t>(seq) * p.n_kv + hh) * cc.max_pos + pos;
}

// This lane's EPL dims of the k row after RMSNorm x gain and RoPE, and the raw 16-bit
// v vector of the same dims.
template <int EPL, typename TM>
__device__ __forceinline__ void kv_k_rope(const KvLaunch& p, int t, int seq, int ai, int hh, int lane,
                                          float (&k)[EPL], typename VecT<EPL>::T& vv) {
  using V = typename VecT<EPL>::T;
  const int d_h = p.d_h;
  const TM* row = static_cast<const TM*>(p.mix) + seq * p.mix_seq_stride +
                  static_cast<int64_t>(t) * p.mix_ld + p.layer_col[ai];
  const int dim0 = lane * EPL;
  V kv = *reinterpret_cast<const V*>(row + hh * d_h + dim0);
  vv = *reinterpret_cast<const V*>(row + p.n_kv * d_h + hh * d_h + dim0);
  {
    const uint32_t* u = reinterpret_cast<const uint32_t*>(&kv);
#pragma unroll
    for (int i = 0; i < EPL / 2; ++i) {
      const float2 f = F16<TM>::unpack(u[i]);
      k[2 * i] = f.x;
      k[2 * i + 1] = f.y;
    }
  }
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < EPL; ++i) ss += k[i] * k[i];
  ss = warp_sum(ss);
  const float scale = rsqrtf(ss / static_cast<float>(d_h) + p.eps);
  const float* gain = p.k_gain + ai * d_h + dim0;
#pragma unroll
  for (int i = 0; i < EPL; ++i) k[i] *= scale * gain[i];

  const int64_t pos = p.pos[seq] + t;
  const int half = p.rope_dims / 2;
  const int off = half / EPL;  // lane distance between the two dims of a pair
  float partner[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) partner[i] = __shfl_xor_sync(0xffffffffu, k[i], off);
  if (dim0 < p.rope_dims) {
    const double two_pi = 6.283185307179586476925286766559;
    const double inv_two_pi = 0.15915494309189533576888376337251;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int d = dim0 + i;
      const int pi = d < half ? d : d - half;
      const double ang = static_cast<double>(pos) * p.inv_freq[pi];
      const double q = rint(ang * inv_two_pi);
      const float red = static_cast<float>(fma(-q, two_pi, ang));
      float sn, cs;
      sincosf(red, &sn, &cs);
      k[i] = d < half ? k[i] * cs - partner[i] * sn : k[i] * cs + partner[i] * sn;
    }
  }
}

template <int EPL, typename TM, typename TC>
__global__ void __launch_bounds__(256) kv_write_kernel(const KvLaunch p) {
  griddep_wait_and_release();
  using V = typename VecT<EPL>::T;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + warp;
  if (t >= p.T) return;
  const int seq = blockIdx.z;
  const int ai = blockIdx.y / p.n_kv, hh = blockIdx.y % p.n_kv;
  float k[EPL];
  V vv;
  kv_k_rope<EPL, TM>(p, t, seq, ai, hh, lane, k, vv);
  if constexpr (!std::is_same<TM, TC>::value) {
    // v is stored in the cache's format (a bit copy when the formats agree)
    uint32_t* u = reinterpret_cast<uint32_t*>(&vv);
#pragma unroll
    for (int i = 0; i < EPL / 2; ++i) {
      const float2 f = F16<TM>::unpack(u[i]);
      u[i] = F16<TC>::pack(f.x, f.y);
    }
  }
  V ko;
  {
    uint32_t* u = reinterpret_cast<uint32_t*>(&ko);
#pragma unroll
    for (int i = 0; i < EPL / 2; ++i) u[i] = F16<TC>::pack(k[2 * i], k[2 * i + 1]);
  }
  const int64_t rowidx = kv_row(p, seq, hh, p.pos[seq] + t, lane);
  if (rowidx < 0) return;
  const int dim0 = lane * EPL;
  TC* kd = static_cast<TC*>(p.cache.k[ai]) + rowidx * p.d_h + dim0;
  TC* vd = static_cast<TC*>(p.cache.v[ai]) + rowidx * p.d_h + dim0;
  *reinterpret_cast<V*>(kd) = ko;
  *reinterpret_cast<V*>(vd) = vv;
}

// ------------------------------------------------------------------ q8_0 cache rows
// Quantized KV cache ("Qwen3.8-27B-KVA" model card, other notes: with q8_0 caches the
// approximated K/V rows are rotated by the same Hadamard transform the exact layers use).
// Each d_h-dim row (k after RMSNorm and RoPE, v as predicted) is multiplied by the
// orthonormal Walsh-Hadamard matrix H / sqrt(d_h), Sylvester order, then stored as q8_0
// blocks of 32 values: fp16 scale d = max|x| / 127, int8 codes round(x / d), half away
// from zero.  A row is d_h / 32 blocks of 34 bytes (scale, then the 32 codes).

// x (this lane's EPL dims, dims lane*EPL + i) <- H x / sqrt(n), n = 32 * EPL: butterflies
// on dim bit b pair the values (a, b) into (a + b, a - b); the low bits of the dim sit
// inside a lane, the high bits across lanes (one xor shuffle per bit).
template <int EPL>
__device__ __forceinline__ void hadamard_warp(float (&x)[EPL], int lane) {
#pragma unroll
  for (int h = 1; h < EPL; h <<= 1)
#pragma unroll
    for (int i = 0; i < EPL; ++i)
      if ((i & h) == 0) {
        const float a = x[i], b = x[i + h];
        x[i] = a + b;
        x[i + h] = a - b;
      }
#pragma unroll
  for (int m = 1; m < 32; m <<= 1)
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const float o = __shfl_xor_sync(0xffffffffu, x[i], m);
      x[i] = (lane & m) ? o - x[i] : x[i] + o;
    }
  const float s = EPL == 8 ? 0.0625f : 0.08838834764831845f;  // 1 / sqrt(32 * EPL)
#pragma unroll
  for (int i = 0; i < EPL; ++i) x[i] *= s;
}

// one q8_0 row: the lanes of a 32-value block share its max through xor shuffles; the
// first lane of the block writes the scale, every lane its EPL codes (2-byte stores:
// the blocks are 34 bytes apart)
template <int EPL>
__device__ __forceinline__ void q8_0_store_row(uint8_t* row, const float (&x)[EPL], int lane) {
  constexpr int LPB = 32 / EPL;  // lanes per block
  float am = 0.f;
#pragma unroll
  for (int i = 0; i < EPL; ++i) am = fmaxf(am, fabsf(x[i]));
#pragma unroll
  for (int m = 1; m < LPB; m <<= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, m));
  const float d = am / 127.f;
  const float id = d > 0.f ? 1.f / d : 0.f;
  const int blk = lane / LPB, j = lane % LPB;
  uint8_t* b = row + blk * 34;
  if (j == 0) *reinterpret_cast<__half*>(b) = __float2half_rn(d);
  uint16_t* qd = reinterpret_cast<uint16_t*>(b + 2 + j * EPL);
#pragma unroll
  for (int i = 0; i < EPL; i += 2) {
    const int q0 = static_cast<int>(roundf(x[i] * id)), q1 = static_cast<int>(roundf(x[i + 1] * id));
    qd[i / 2] = static_cast<uint16_t>((q0 & 0xff) | ((q1 & 0xff) << 8));
  }
}

template <int EPL, typename TM>
__global__ void __launch_bounds__(256) kv_write_q8_kernel(const KvLaunch p) {
  griddep_wait_and_release();
  using V = typename VecT<EPL>::T;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + warp;
  if (t >= p.T) return;
  const int seq = blockIdx.z;
  const int ai = blockIdx.y / p.n_kv, hh = blockIdx.y % p.n_kv;
  float k[EPL], v[EPL];
  V vv;
  kv_k_rope<EPL, TM>(p, t, seq, ai, hh, lane, k, vv);
  {
    const uint32_t* u = reinterpret_cast<const uint32_t*>(&vv);
#pragma unroll
    for (int i = 0; i < EPL / 2; ++i) {
      const float2 f = F16<TM>::unpack(u[i]);
      v[2 * i] = f.x;
      v[2 * i + 1] = f.y;
    }
  }
  hadamard_warp<EPL>(k, lane);
  hadamard_warp<EPL>(v, lane);
  const int64_t rowidx = kv_row(p, seq, hh, p.pos[seq] + t, lane);
  if (rowidx < 0) return;
  const int64_t row_bytes = (p.d_h / 32) * 34;
  q8_0_store_row<EPL>(static_cast<uint8_t*>(p.cache.k[ai]) + rowidx * row_bytes, k, lane);
  q8_0_store_row<EPL>(static_cast<uint8_t*>(p.cache.v[ai]) + rowidx * row_bytes, v, lane);
}

int launch_kv_write(const KvLaunch& k, cudaStream_t s) {
  if (k.T == 0 || k.n_attn == 0 || k.n_seq == 0) return KVA_OK;
  if (!k.mix || !k.k_gain) return KVA_ERR_INVALID_ARG;
  if (k.d_h != 128 && k.d_h != 256) return KVA_ERR_UNSUPPORTED;
  const int epl = k.d_h / 32;
  const int half = k.rope_dims / 2;
  if (k.rope_dims < 0 || k.rope_dims % 2 || k.rope_dims > k.d_h) return KVA_ERR_UNSUPPORTED;
  if (k.rope_dims > 0) {
    if (half % epl) return KVA_ERR_UNSUPPORTED;
    const int off = half / epl;
    if (off & (off - 1)) return KVA_ERR_UNSUPPORTED;  // xor pairing needs a power of two
  }
  if ((k.mix_dtype != KVA_BF16 && k.mix_dtype != KVA_F16) ||
      (k.cache.dtype != KVA_BF16 && k.cache.dtype != KVA_F16 && k.cache.dtype != KVA_Q8_0))
    return KVA_ERR_INVALID_ARG;
  dim3 grid((k.T + 7) / 8, k.n_kv * k.n_attn, k.n_seq);
  if (k.cache.dtype == KVA_Q8_0) {
    const bool mh16 = k.mix_dtype == KVA_F16;
    cudaError_t r;
    if (epl == 8)
      r = mh16 ? launch_pdl(kv_write_q8_kernel<8, __half>, grid, dim3(256), 0, s, k)
               : launch_pdl(kv_write_q8_kernel<8, __nv_bfloat16>, grid, dim3(256), 0, s, k);
    else
      r = mh16 ? launch_pdl(kv_write_q8_kernel<4, __half>, grid, dim3(256), 0, s, k)
               : launch_pdl(kv_write_q8_kernel<4, __nv_bfloat16>, grid, dim3(256), 0, s, k);
    return r == cudaSuccess ? KVA_OK : KVA_ERR_CUDA;
  }
  const bool mh = k.mix_dtype == KVA_F16, ch = k.cache.dtype == KVA_F16;
  cudaError_t r;
#define KVA_KV_LAUNCH(EPL, TM, TC) r = launch_pdl(kv_write_kernel<EPL, TM, TC>, grid, dim3(256), 0, s, k)
  if (epl == 8) {
    if (mh && ch) KVA_KV_LAUNCH(8, __half, __half);
    else if (mh) KVA_KV_LAUNCH(8, __half, __nv_bfloat16);
    else if (ch) KVA_KV_LAUNCH(8, __nv_bfloat16, __half);
    else KVA_KV_LAUNCH(8, __nv_bfloat16, __nv_bfloat16);
  } else {
    if (mh && ch) KVA_KV_LAUNCH(4, __half, __half);
    else if (mh) KVA_KV_LAUNCH(4, __half, __nv_bfloat16);
    else if (ch) KVA_KV_LAUNCH(4, __nv_bfloat16, __half);
    else KVA_KV_LAUNCH(4, __nv_bfloat16, __nv_bfloat16);
  }
#undef KVA_KV_LAUNCH
  return r == cudaSuccess ? KVA_OK : KVA_ERR_CUDA;
}

}  // namespace kva
