// noalloc.cu -- sparse_route_topk_static: shared routing (score scan + top-k
// select) with its scratch in a fixed device array inside this library, for
// callers that cannot allocate device memory or hand the library a workspace.
//
// The scratch (status word, radix histogram, fp32 scores) is one file-scope
// __device__ array, so every GPU that loads the library holds it until the
// process exits.  Its device address is looked up once per device with
// cudaGetSymbolAddress on the first call made with that device current (and
// again by a later call if that lookup failed); that first call should
// therefore come before any stream capture.  The stream must belong to the
// current device.  Every call
// shares the array: the status word and the histogram rows a call uses are
// cleared at the start of the call (cudaMemsetAsync on the same stream), and
// two calls that overlap on the GPU (different streams, no ordering) race on
// it.  Nothing here calls cudaMalloc, cudaFree or an allocating routine.
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "sparse_decode.h"

namespace sd {
namespace {

constexpr size_t kStaticHeader = 4096;  // the workspace header's layout (status, scan counters)
constexpr int kStaticMaxHeads = 64;                 // B * Hkv
constexpr long long kStaticMaxScores = 1LL << 20;   // B * Hkv * N
constexpr size_t kStaticHistBytes = (size_t)kStaticMaxHeads * 2048 * sizeof(uint32_t);
constexpr size_t kStaticBytes =
    kStaticHeader + kStaticHistBytes + (size_t)kStaticMaxScores * sizeof(float);

static __device__ __align__(256) unsigned char g_route_scratch[kStaticBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch[kMaxDevices];  // set once the lookup for that device succeeded

// The array's device address on device dev (current), looked up on the first
// call that needs it and kept only when the lookup succeeds, so a failed
// lookup is retried by the next call.  A lookup is not attempted while `st`
// is being captured (it would call into the runtime inside the capture).
cudaError_t scratch_address(int dev, cudaStream_t st, char **out) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch[dev]) {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(st, &cap);
    if (e != cudaSuccess) return e;
    if (cap != cudaStreamCaptureStatusNone) return cudaErrorStreamCaptureUnsupported;
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_route_scratch);
    if (e != cudaSuccess || !p) {
      (void)cudaGetLastError();
      return e != cudaSuccess ? e : cudaErrorInvalidSymbol;
    }
    g_scratch[dev] = p;
  }
  *out = static_cast<char *>(g_scratch[dev]);
  return cudaSuccess;
}

}  // namespace
}  // namespace sd

extern "C" sparse_status_t sparse_route_topk_static(const sparse_shape_t *shape,
                                                    const void *q, const void *K,
                                                    int32_t k, int32_t *idx,
                                                    void *stream) {
  sd::Shape s;
  sparse_status_t r = sd::check_shape(shape, &s);
  if (r != SPARSE_OK) return r;
  if (!q || !K || !idx || k < 1 || k > s.N) return SPARSE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(q) & 15u) || (reinterpret_cast<uintptr_t>(K) & 15u) ||
      (reinterpret_cast<uintptr_t>(idx) & 3u))
    return SPARSE_ERR_INVALID_ARG;
  // the built-in scratch holds at most 64 heads and 2^20 scores
  if (s.BH() > sd::kStaticMaxHeads || (long long)s.BH() * s.N > sd::kStaticMaxScores)
    return SPARSE_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= sd::kMaxDevices)
    return SPARSE_ERR_CUDA;
  // the array is addressed on the current device: the stream must belong to it
  int sdev = dev;
  if (cudaStreamGetDevice(st, &sdev) != cudaSuccess) {
    (void)cudaGetLastError();
    return SPARSE_ERR_INVALID_ARG;
  }
  if (sdev != dev) return SPARSE_ERR_INVALID_ARG;
  char *base = nullptr;
  if (sd::scratch_address(dev, st, &base) != cudaSuccess) return SPARSE_ERR_CUDA;
  uint32_t *status = reinterpret_cast<uint32_t *>(base);
  uint32_t *hist = reinterpret_cast<uint32_t *>(base + sd::kStaticHeader);
  float *S = reinterpret_cast<float *>(base + sd::kStaticHeader + sd::kStaticHistBytes);
  // status word and this call's histogram rows must start at zero
  cudaError_t e = cudaMemsetAsync(
      base, 0, sd::kStaticHeader + (size_t)s.BH() * 2048 * sizeof(uint32_t), st);
  if (e == cudaSuccess) e = sd::launch_score(s, q, K, S, hist, status, st);
  if (e == cudaSuccess) e = sd::launch_select_split(s, S, k, idx, hist, status, st);
  return e == cudaSuccess ? SPARSE_OK : SPARSE_ERR_CUDA;
}
