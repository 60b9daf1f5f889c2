// kv_append.cu -- the self-decoder's per-step cache write: the new token's key
// and value rows become row N-1 of every (sequence, KV head), where N is the
// cache length including the new token (CLSA article, section CLSAの仕組み: the
// self-decoder writes the shared KV cache once; routing and every
// cross-decoder layer then read it, the new token included).
//
// One warp per (sequence, KV head) moves the two rows in 16-byte pieces (a
// row is d * element-size bytes, 256 B at d = 128 in bf16).
#include "common.cuh"
#include "internal.h"
#include "sparse_decode.h"

namespace sd {
namespace {

constexpr int kAppendHeadsPerBlock = 8;  // one warp each

__global__ void __launch_bounds__(32 * kAppendHeadsPerBlock)
    kv_append_kernel(uint4 *__restrict__ K, uint4 *__restrict__ V,
                     const uint4 *__restrict__ k_new, const uint4 *__restrict__ v_new,
                     int BH, int row, int rows_per_head, int chunks_per_row) {
  grid_dep_wait();  // earlier kernels may still read the rows being replaced
  grid_dep_launch();
  const int bh = blockIdx.x * kAppendHeadsPerBlock + (threadIdx.x >> 5);
  if (bh >= BH) return;
  const size_t dst = ((size_t)bh * rows_per_head + row) * chunks_per_row;
  const size_t src = (size_t)bh * chunks_per_row;
  for (int c = threadIdx.x & 31; c < chunks_per_row; c += 32) {
    K[dst + c] = k_new[src + c];
    V[dst + c] = v_new[src + c];
  }
}

}  // namespace
}  // namespace sd

extern "C" sparse_status_t sparse_kv_append(const sparse_shape_t *shape, void *K, void *V,
                                            const void *k_new, const void *v_new,
                                            void *stream) {
  if (!shape) return SPARSE_ERR_INVALID_ARG;
  const int B = shape->B, N = shape->N, Hkv = shape->Hkv, d = shape->d;
  const int n_cap = shape->n_cap == 0 ? N : shape->n_cap;
  if (B < 1 || N < 1 || Hkv < 1 || n_cap < N) return SPARSE_ERR_INVALID_ARG;
  if ((d != 64 && d != 128) || (shape->dtype != 0 && shape->dtype != 1))
    return SPARSE_ERR_UNSUPPORTED;
  if ((long long)B * Hkv > 65535) return SPARSE_ERR_UNSUPPORTED;
  if (!K || !V || !k_new || !v_new) return SPARSE_ERR_INVALID_ARG;
  for (const void *p : {static_cast<const void *>(K), static_cast<const void *>(V), k_new, v_new})
    if (reinterpret_cast<uintptr_t>(p) & 15u) return SPARSE_ERR_INVALID_ARG;
  const int BH = B * Hkv;
  const int chunks = d * (shape->dtype == 0 ? 4 : 2) / 16;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((BH + sd::kAppendHeadsPerBlock - 1) / sd::kAppendHeadsPerBlock),
                     1, 1);
  cfg.blockDim = dim3(32 * sd::kAppendHeadsPerBlock, 1, 1);
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attrs[1];
  cfg.attrs = attrs;
  cfg.numAttrs = 0;
  sd::add_pdl_attr(cfg, attrs);
  cudaError_t e = cudaLaunchKernelEx(&cfg, sd::kv_append_kernel, static_cast<uint4 *>(K),
                                     static_cast<uint4 *>(V), static_cast<const uint4 *>(k_new),
                                     static_cast<const uint4 *>(v_new), BH, N - 1, n_cap,
                                     chunks);
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? SPARSE_OK : SPARSE_ERR_CUDA;
}
