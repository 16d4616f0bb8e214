// Allocation-free state update of one gated-DeltaNet layer.
//
// Some callers cannot hand this library a kva_handle, because creating one calls
// cudaMalloc for the workspace.  Examples: an inference engine that reserves
// (almost) all device memory for its own KV-cache pool at start-up and routes
// every later allocation through its own allocator, so a foreign cudaMalloc
// either fails or fragments that pool; or a plugin loaded into a host program
// that owns device memory and forbids its plugins to allocate.  For them this
// entry point keeps its scratch (the normalised keys, the values and the gates
// between the conv kernel and the scan) in a fixed-size array that lives in the
// library's own device image, so a call allocates nothing.
//
// This is an engineering addition of the library; the method it serves has no
// counterpart to it.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/kva.h"
#include "../../include/kva_ops.h"
#include "kva_internal.h"

namespace {

constexpr int kMaxT = KVA_NOALLOC_MAX_T;
constexpr size_t kKBytes = static_cast<size_t>(kMaxT) * KVA_NOALLOC_MAX_QK * 2;
constexpr size_t kVBytes = static_cast<size_t>(kMaxT) * KVA_NOALLOC_MAX_V * 2;
constexpr size_t kGBytes = static_cast<size_t>(2) * KVA_NOALLOC_MAX_NV * kMaxT * 4;
// per-chunk B1 tiles and scalars of the 128-dimensional scan
constexpr size_t kCBytes = static_cast<size_t>((kMaxT + 63) / 64) * KVA_NOALLOC_MAX_NV * (64 * 64 * 2 + 80 * 4);
constexpr size_t kScratchBytes = kKBytes + kVBytes + kGBytes + kCBytes;
static_assert(kKBytes % 256 == 0 && kVBytes % 256 == 0 && kGBytes % 256 == 0,
              "scratch parts stay 256-byte aligned");

// Every GPU that loads the library holds this array until the process exits.
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];
// Device status bits (KVA_DEV_*) of the calls: a pipeline wait inside the scan that gave
// up sets KVA_DEV_WAIT_TIMEOUT here.  Read and cleared by kva_gdn_layer_update_noalloc_status.
static __device__ int g_status;

// Device addresses of g_scratch and g_status per device.  In host code the symbols' names
// are only host-side stand-ins, so the addresses must come from the runtime.  They stay
// valid for the life of the device's primary context (a cudaDeviceReset invalidates them).
constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {nullptr};
int* g_status_ptr[kMaxDevices] = {nullptr};
std::mutex g_scratch_mu;

int symbols_for_current_device(void** scratch, int** status) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KVA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return KVA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    void* q = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p ||
        cudaGetSymbolAddress(&q, g_status) != cudaSuccess || !q) {
      cudaGetLastError();
      return KVA_ERR_CUDA;
    }
    g_status_ptr[dev] = static_cast<int*>(q);
    g_scratch_ptr[dev] = p;
  }
  *scratch = g_scratch_ptr[dev];
  *status = g_status_ptr[dev];
  return KVA_OK;
}

bool a16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int kva_gdn_layer_update_noalloc(const void* mixer_in, int64_t mixer_ld, int32_t T,
                                            int32_t n_k, int32_t n_v, int32_t d,
                                            const float* conv_w, const float* A_log,
                                            const float* dt_bias, float* state,
                                            void* conv_state, float eps, void* stream) {
  if (!mixer_in || !conv_w || !A_log || !dt_bias || !state || !conv_state) return KVA_ERR_INVALID_ARG;
  if (T < 0 || n_k <= 0 || n_v <= 0 || d <= 0 || !(eps >= 0.f)) return KVA_ERR_INVALID_ARG;
  if (n_v % n_k) return KVA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return KVA_ERR_UNSUPPORTED;
  if ((n_k * d) % 128) return KVA_ERR_UNSUPPORTED;
  // sizes beyond the fixed scratch are refused, never truncated
  if (T > kMaxT || n_k * d > KVA_NOALLOC_MAX_QK || n_v * d > KVA_NOALLOC_MAX_V ||
      n_v > KVA_NOALLOC_MAX_NV)
    return KVA_ERR_TOO_LARGE;
  const int C = 2 * n_k * d + n_v * d;
  if (mixer_ld < C + 2 * n_v) return KVA_ERR_INVALID_ARG;
  if (!a16(mixer_in) || !a16(state) || !a16(conv_state) || mixer_ld % 8) return KVA_ERR_ALIGNMENT;
  if (T == 0) return KVA_OK;

  void* base = nullptr;
  int* status = nullptr;
  int e = symbols_for_current_device(&base, &status);
  if (e) return e;
  unsigned char* b = static_cast<unsigned char*>(base);

  kva::GdnLaunch g;
  g.mix = mixer_in;
  g.mix_ld = mixer_ld;
  g.mix_seq_stride = static_cast<int64_t>(T) * mixer_ld;
  g.n_seq = 1;
  g.T = T;
  g.n_gdn = 1;
  g.layer_col[0] = 0;
  g.n_k = n_k;
  g.n_v = n_v;
  g.d_k = g.d_v = d;
  g.C = C;
  g.conv_w = conv_w;
  g.A_log = A_log;
  g.dt_bias = dt_bias;
  g.conv_state = conv_state;
  g.state = state;
  g.kbuf = b;                      // every row < T is written before the scan reads it,
  g.vbuf = b + kKBytes;            // so nothing in the scratch has to start at zero
  g.gbuf = reinterpret_cast<float*>(b + kKBytes + kVBytes);
  if (d == 128) {
    // every chunk's B1 and scalars are written before the scan reads them
    kva::gdn_chunk_split(b + kKBytes + kVBytes + kGBytes, 1, 1, n_v, T, &g.b1buf, &g.scbuf);
  }
  g.eps = eps;
  g.err = status;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((e = kva::launch_gdn_prepare(g, s))) return e;
  if ((e = kva::launch_gdn_tail(g, s))) return e;
  return kva::launch_gdn_scan(g, s);
}

extern "C" int kva_gdn_layer_update_noalloc_status(void* stream, int32_t* status) {
  if (!status) return KVA_ERR_INVALID_ARG;
  *status = 0;
  void* base = nullptr;
  int* word = nullptr;
  int e = symbols_for_current_device(&base, &word);
  if (e) return e;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int v = 0;
  const int zero = 0;
  if (cudaMemcpyAsync(&v, word, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaMemcpyAsync(word, &zero, sizeof(int), cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess) {
    cudaGetLastError();
    return KVA_ERR_CUDA;
  }
  *status = v;
  return v ? KVA_ERR_DEVICE : KVA_OK;
}
