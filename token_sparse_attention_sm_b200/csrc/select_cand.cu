// select_cand.cu -- A2 after the routing scan, as its own kernel (the top-k
// routing call, and decode steps the fused attention kernel does not take):
// one CTA per (sequence, KV head) runs the exact select of topk_cand.cuh on
// the scan's histogram and candidate lists (or its score row) and writes the
// head's k indices in ascending order (CLSA article, section 研究の背景と課題:
// the k highest scores, ties to the lower key index).
//
// The select reads the histogram, the sample histogram and the sample count
// of its head and clears them for the next call.
#include "internal.h"
#include "topk_cand.cuh"

namespace sd {
namespace {

constexpr int kSelSmallBytes = 256;  // TkSmall, rounded up

__global__ void __launch_bounds__(kTkThreads, 1)
    select_cand_kernel(const float *__restrict__ S, int N, int k, int *__restrict__ idx,
                       uint32_t *__restrict__ hist, const __grid_constant__ CandArgs cand,
                       int use_lists, int bitmap_words, uint32_t *status) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  TkSmall *sm = reinterpret_cast<TkSmall *>(smem_raw);
  unsigned char *scratch = smem_raw + kSelSmallBytes;
  const int bh = blockIdx.x, tid = threadIdx.x;
  grid_dep_wait();
  grid_dep_launch();
  int *out = idx + (size_t)bh * k;
  auto emit = [&](uint32_t pos, uint32_t j) {
    if (pos < (uint32_t)k) out[pos] = (int)j;
  };
  TkNoSure no_hook;
  const uint32_t n = tk_select(S + (size_t)bh * N, N, (uint32_t)k,
                               hist ? hist + (size_t)bh * kHistBins : nullptr, cand,
                               use_lists != 0, bh, scratch, bitmap_words, sm, status, emit,
                               no_hook, 0u, (uint32_t)k);
  if (tid == 0 && n != (uint32_t)k) raise_flag(status, FLAG_INTERNAL);
  __syncthreads();  // every thread is done with the histogram
  if (hist)
    for (int i = tid; i < kHistBins; i += kTkThreads) hist[(size_t)bh * kHistBins + i] = 0u;
  if (use_lists) {
    for (int i = tid; i < kHistBins; i += kTkThreads)
      cand.smp_hist[(size_t)bh * kHistBins + i] = 0u;
    if (tid == 0) cand.smp_cnt[bh] = 0u;
  }
}

}  // namespace

cudaError_t launch_select_cand(const Shape &s, const float *S, int k, int *idx, uint32_t *hist,
                               const CandArgs *cand, uint32_t *status, cudaStream_t st) {
  DeviceInfo di;
  cudaError_t e = device_info(&di);
  if (e != cudaSuccess) return e;
  // the on-chip bitmap of the head when it fits, else none (the select then
  // takes its streaming path)
  int words = ((s.N + 31) / 32 + 1) & ~1;
  if ((size_t)kSelSmallBytes + tk_scratch_bytes(words) > (size_t)di.max_smem_optin) words = 0;
  const size_t smem = kSelSmallBytes + tk_scratch_bytes(words);
  auto kern = select_cand_kernel;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)s.BH(), 1, 1);
  cfg.blockDim = dim3(kTkThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  cfg.attrs = attr;
  cfg.numAttrs = 0;
  add_pdl_attr(cfg, attr);
  const bool use_lists = cand && cand->lists;
  const CandArgs none{};
  e = cudaLaunchKernelEx(&cfg, kern, S, s.N, k, idx, hist, use_lists ? *cand : none,
                         use_lists ? 1 : 0, words, status);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace sd
