// RMSNorm rows -> bf16 or fp16 ("Qwen3.8-27B-KVA" model card, architecture:
// RMSNorm before the input Linear, before each attention and FFN sub-block, and
// once before all heads).  out = x / sqrt(mean(x^2) + eps) * g, stats in fp32.
// Bandwidth-bound: one read of x (fp32 or 16-bit), one 16-bit write.
#include "kva_common.cuh"

namespace kva {

template <typename T>
__device__ __forceinline__ float4 load4(const T* p);
template <>
__device__ __forceinline__ float4 load4<float>(const float* p) {
  return *reinterpret_cast<const float4*>(p);
}
template <>
__device__ __forceinline__ float4 load4<__nv_bfloat16>(const __nv_bfloat16* p) {
  uint2 u = *reinterpret_cast<const uint2*>(p);
  float2 a = unpack_bf16(u.x), b = unpack_bf16(u.y);
  return make_float4(a.x, a.y, b.x, b.y);
}
template <>
__device__ __forceinline__ float4 load4<__half>(const __half* p) {
  uint2 u = *reinterpret_cast<const uint2*>(p);
  float2 a = F16<__half>::unpack(u.x), b = F16<__half>::unpack(u.y);
  return make_float4(a.x, a.y, b.x, b.y);
}

// One block of 256 threads per row (many rows' loads in flight across the GPU): each thread
// holds its up to NV groups of 4 values in registers from the one read of the row, the sum of
// squares is reduced through shared memory, and the output is written from the registers.
template <typename T, typename TO, int NV>
__global__ void __launch_bounds__(256) rmsnorm_kernel(const T* __restrict__ x, int64_t ldx,
                                                      const float* __restrict__ g,
                                                      TO* __restrict__ out, int64_t ldo, int n,
                                                      float eps, float* __restrict__ zero,
                                                      int64_t ldz, int nz) {
  griddep_wait_and_release();
  const int row = blockIdx.x;
  const T* xr = x + row * ldx;
  TO* orow = out + row * ldo;
  float4 v[NV];
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int i = (threadIdx.x + k * 256) * 4;
    v[k] = i < n ? load4<T>(xr + i) : make_float4(0.f, 0.f, 0.f, 0.f);
    ss += v[k].x * v[k].x + v[k].y * v[k].y + v[k].z * v[k].z + v[k].w * v[k].w;
  }
  if (zero) {  // clear this row of another buffer (the next GEMM accumulates into it)
    float* zr = zero + row * ldz;
    for (int i = threadIdx.x * 4; i < nz; i += blockDim.x * 4)
      *reinterpret_cast<float4*>(zr + i) = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  __shared__ float red[8];
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) tot += red[w];
  const float scale = rsqrtf(tot / static_cast<float>(n) + eps);
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int i = (threadIdx.x + k * 256) * 4;
    if (i < n) {
      const float4 gg = *reinterpret_cast<const float4*>(g + i);
      uint2 o;
      o.x = F16<TO>::pack(v[k].x * scale * gg.x, v[k].y * scale * gg.y);
      o.y = F16<TO>::pack(v[k].z * scale * gg.z, v[k].w * scale * gg.w);
      *reinterpret_cast<uint2*>(orow + i) = o;
    }
  }
}

template <typename T, typename TO>
static cudaError_t rms_launch(const T* x, int64_t ldx, const float* g, TO* o, int64_t ldo, int rows, int n,
                              float eps, cudaStream_t s, float* zero, int64_t ldz, int nz) {
  // groups of 4 values per thread: 1024 values a pass of the block
  const int nv = (n + 1023) / 1024;
  if (nv <= 2)
    return launch_pdl(rmsnorm_kernel<T, TO, 2>, dim3(rows), dim3(256), 0, s, x, ldx, g, o, ldo, n, eps, zero, ldz, nz);
  if (nv <= 4)
    return launch_pdl(rmsnorm_kernel<T, TO, 4>, dim3(rows), dim3(256), 0, s, x, ldx, g, o, ldo, n, eps, zero, ldz, nz);
  if (nv <= 8)
    return launch_pdl(rmsnorm_kernel<T, TO, 8>, dim3(rows), dim3(256), 0, s, x, ldx, g, o, ldo, n, eps, zero, ldz, nz);
  return launch_pdl(rmsnorm_kernel<T, TO, 16>, dim3(rows), dim3(256), 0, s, x, ldx, g, o, ldo, n, eps, zero, ldz, nz);
}

template <typename TO>
static cudaError_t rms_dispatch(const void* x, int x_dtype, int64_t ldx, const float* g, void* out,
                                int64_t ldo, int rows, int n, float eps, cudaStream_t s, float* zero,
                                int64_t ldz, int nz) {
  TO* o = static_cast<TO*>(out);
  if (x_dtype == KVA_F32)
    return rms_launch(static_cast<const float*>(x), ldx, g, o, ldo, rows, n, eps, s, zero, ldz, nz);
  if (x_dtype == KVA_BF16)
    return rms_launch(static_cast<const __nv_bfloat16*>(x), ldx, g, o, ldo, rows, n, eps, s, zero, ldz, nz);
  return rms_launch(static_cast<const __half*>(x), ldx, g, o, ldo, rows, n, eps, s, zero, ldz, nz);
}

int launch_rmsnorm(const void* x, int x_dtype, int64_t ldx, const float* g, void* out,
                   int64_t ldo, int rows, int n, float eps, cudaStream_t s, int out_dtype,
                   float* zero, int64_t ldz, int nz) {
  if (rows == 0) return KVA_OK;
  if (!x || !g || !out || rows < 0 || n <= 0) return KVA_ERR_INVALID_ARG;
  if (x_dtype != KVA_F32 && x_dtype != KVA_BF16 && x_dtype != KVA_F16) return KVA_ERR_INVALID_ARG;
  if (out_dtype != KVA_BF16 && out_dtype != KVA_F16) return KVA_ERR_INVALID_ARG;
  if (n > 16 * 1024) return KVA_ERR_UNSUPPORTED;
  if (n % 4 || ldx % 4 || ldo % 4 || nz % 4 || ldz % 4) return KVA_ERR_ALIGNMENT;
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(g) |
       reinterpret_cast<uintptr_t>(out) | reinterpret_cast<uintptr_t>(zero)) & 15u)
    return KVA_ERR_ALIGNMENT;
  const cudaError_t r =
      out_dtype == KVA_F16
          ? rms_dispatch<__half>(x, x_dtype, ldx, g, out, ldo, rows, n, eps, s, zero, ldz, nz)
          : rms_dispatch<__nv_bfloat16>(x, x_dtype, ldx, g, out, ldo, rows, n, eps, s, zero, ldz, nz);
  return r == cudaSuccess ? KVA_OK : KVA_ERR_CUDA;
}

}  // namespace kva
