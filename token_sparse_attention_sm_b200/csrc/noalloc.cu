// noalloc.cu -- sparse_route_topk_static: shared routing (score scan + top-k
// select) with its scratch in a fixed device array inside this library, for
// callers that cannot allocate device memory or hand the library a workspace.
//
// The scratch (status word, radix histogram, fp32 scores) is one file-scope
// __device__ array, so every GPU that loads the library holds it until the
// process exits.  Its device address is looked up once per device with
// cudaGetSymbolAddress on the first call made with that device current; that
// first call should therefore come before any stream capture.  Every call
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

constexpr size_t kStaticHeader = 256;
constexpr int kStaticMaxHeads = 64;                 // B * Hkv
constexpr long long kStaticMaxScores = 1LL << 20;   // B * Hkv * N
constexpr size_t kStaticHistBytes = (size_t)kStaticMaxHeads * 2048 * sizeof(uint32_t);
constexpr size_t kStaticBytes =
    kStaticHeader + kStaticHistBytes + (size_t)kStaticMaxScores * sizeof(float);

static __device__ __align__(256) unsigned char g_route_scratch[kStaticBytes];

constexpr int kMaxDevices = 64;
std::once_flag g_once[kMaxDevices];
void *g_scratch[kMaxDevices];
cudaError_t g_scratch_err[kMaxDevices];

}  // namespace
}  // namespace sd

extern "C" sparse_status_t sparse_route_topk_static(const sparse_shape_t *shape,
                                                    const void *q, const void *K,
                                                    int32_t k, int32_t *idx,
                                                    void *stream) {
  if (!shape) return SPARSE_ERR_INVALID_ARG;
  sd::Shape s{shape->B, shape->N, shape->Hq, shape->Hkv, shape->d, shape->dtype,
              shape->n_cap == 0 ? shape->N : shape->n_cap};
  if (s.Ncap < s.N) return SPARSE_ERR_INVALID_ARG;
  if (s.B < 1 || s.N < 1 || s.Hq < 1 || s.Hkv < 1 || s.Hq % s.Hkv != 0)
    return SPARSE_ERR_INVALID_ARG;
  if ((s.d != 64 && s.d != 128) || (s.dtype != 0 && s.dtype != 1) || s.G() > 16)
    return SPARSE_ERR_UNSUPPORTED;
  if (!q || !K || !idx || k < 1 || k > s.N) return SPARSE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(q) & 15u) || (reinterpret_cast<uintptr_t>(K) & 15u) ||
      (reinterpret_cast<uintptr_t>(idx) & 3u))
    return SPARSE_ERR_INVALID_ARG;
  // the built-in scratch holds at most 64 heads and 2^20 scores
  if (s.BH() > sd::kStaticMaxHeads || (long long)s.BH() * s.N > sd::kStaticMaxScores)
    return SPARSE_ERR_WORKSPACE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= sd::kMaxDevices)
    return SPARSE_ERR_CUDA;
  std::call_once(sd::g_once[dev], [dev]() {
    sd::g_scratch_err[dev] = cudaGetSymbolAddress(&sd::g_scratch[dev], sd::g_route_scratch);
  });
  if (sd::g_scratch_err[dev] != cudaSuccess || !sd::g_scratch[dev]) return SPARSE_ERR_CUDA;
  char *base = static_cast<char *>(sd::g_scratch[dev]);
  uint32_t *status = reinterpret_cast<uint32_t *>(base);
  uint32_t *hist = reinterpret_cast<uint32_t *>(base + sd::kStaticHeader);
  float *S = reinterpret_cast<float *>(base + sd::kStaticHeader + sd::kStaticHistBytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // status word and this call's histogram rows must start at zero
  cudaError_t e = cudaMemsetAsync(
      base, 0, sd::kStaticHeader + (size_t)s.BH() * 2048 * sizeof(uint32_t), st);
  if (e == cudaSuccess) e = sd::launch_score(s, q, K, S, hist, status, st);
  if (e == cudaSuccess)
    e = sd::launch_select(s, S, k, nullptr, 0, idx, nullptr, k, hist, status, st);
  return e == cudaSuccess ? SPARSE_OK : SPARSE_ERR_CUDA;
}
