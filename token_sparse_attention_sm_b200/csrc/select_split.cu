// select_split.cu -- A2 after the routing scan as its own kernel (the top-k
// routing call, and decode steps the fused attention kernel does not take):
// one thread-block cluster per (sequence, KV head) runs the split select of
// topk_split.cuh on the scan's histogram and score row, and every CTA writes
// the selected keys of its run of the row to the head's idx row, ascending
// (CLSA article, section 研究の背景と課題: the k highest scores, ties to the
// lower key index).  The head's histogram is cleared for the next call.
#include <atomic>

#include "internal.h"
#include "topk_split.cuh"

namespace sd {
namespace {

constexpr size_t kSelShowOff = ts_scratch_bytes();
constexpr size_t kSelBookOff = kSelShowOff + sizeof(TsShow);
constexpr size_t kSelSmallOff = kSelBookOff + sizeof(TsBook);
constexpr size_t kSelSmem = kSelSmallOff + sizeof(TkSmall);
constexpr int kSelMaxDevices = 64;

// Two CTAs per SM (64 registers a thread): with one, only 7 clusters of 16
// are resident at once, and an 8th head waits for a second wave.
__global__ void __launch_bounds__(kTkThreads, 2)
    select_split_kernel(const float *__restrict__ S, int N, int k, int *__restrict__ idx,
                        uint32_t *__restrict__ hist, uint32_t *status) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  TsShow *show = reinterpret_cast<TsShow *>(smem_raw + kSelShowOff);
  TsBook *book = reinterpret_cast<TsBook *>(smem_raw + kSelBookOff);
  TkSmall *sm = reinterpret_cast<TkSmall *>(smem_raw + kSelSmallOff);
  const int nsplit = (int)gridDim.x, rank = (int)blockIdx.x, bh = (int)blockIdx.y;
  grid_dep_wait();
  grid_dep_launch();
  int *out = idx + (size_t)bh * k;
  auto emit = [&](uint32_t, uint32_t pos, uint32_t j) {
    if (pos < (uint32_t)k) out[pos] = (int)j;
  };
  uint32_t *h = hist + (size_t)bh * kHistBins;
  ts_select(S + (size_t)bh * N, N, (uint32_t)k, h, rank, nsplit, (uint32_t)k, smem_raw, show,
            book, sm, status, emit);
  // no CTA leaves while a peer may still read its list, and the histogram
  // is cleared only after every CTA is done with it
  if (nsplit > 1)
    cluster_sync_all();
  else
    __syncthreads();
  if (rank == 0)
    for (int i = threadIdx.x; i < kHistBins; i += kTkThreads) h[i] = 0u;
}

// Cluster size for `heads` heads: enough CTAs to fill the device (up to
// kTsMaxSplits per head), at least enough for runs of at most kTsMaxWords
// words where that is possible, and a size the device can hold (asked of the
// occupancy calculator once per device and size).
int select_splits(const Shape &s, int sm_count) {
  static std::atomic<int> cache[kSelMaxDevices][kTsMaxSplits + 1];  // 0 unknown, 1 no, 2 yes
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kSelMaxDevices) {
    (void)cudaGetLastError();
    return 1;
  }
  const int nw = (s.N + 31) / 32;
  int want = (2 * sm_count) / s.BH();
  const int by_words = (nw + kTsMaxWords - 1) / kTsMaxWords;
  if (want < by_words) want = by_words;
  if (want > kTsMaxSplits) want = kTsMaxSplits;
  if (want > nw) want = nw;
  for (int n = want; n >= 2; --n) {
    int v = cache[dev][n].load(std::memory_order_relaxed);
    if (v == 0) {
      auto kern = select_split_kernel;
      int act = 0;
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)kSelSmem);
      if (e == cudaSuccess && n > 8)
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e == cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)n, 1, 1);
        cfg.blockDim = dim3(kTkThreads, 1, 1);
        cfg.dynamicSmemBytes = kSelSmem;
        cudaLaunchAttribute at;
        at.id = cudaLaunchAttributeClusterDimension;
        at.val.clusterDim.x = (unsigned)n;
        at.val.clusterDim.y = 1;
        at.val.clusterDim.z = 1;
        cfg.attrs = &at;
        cfg.numAttrs = 1;
        e = cudaOccupancyMaxActiveClusters(&act, kern, &cfg);
      }
      if (e != cudaSuccess) {
        (void)cudaGetLastError();
        act = 0;
      }
      v = act > 0 ? 2 : 1;
      cache[dev][n].store(v, std::memory_order_relaxed);
    }
    if (v == 2) return n;
  }
  return 1;
}

}  // namespace

cudaError_t launch_select_split(const Shape &s, const float *S, int k, int *idx, uint32_t *hist,
                                uint32_t *status, cudaStream_t st) {
  DeviceInfo di;
  cudaError_t e = device_info(&di);
  if (e != cudaSuccess) return e;
  const int nsplit = select_splits(s, di.sm_count);
  auto kern = select_split_kernel;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSelSmem);
  if (e == cudaSuccess && nsplit > 8)
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)nsplit, (unsigned)s.BH(), 1);
  cfg.blockDim = dim3(kTkThreads, 1, 1);
  cfg.dynamicSmemBytes = kSelSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  cfg.attrs = attr;
  cfg.numAttrs = 0;
  if (nsplit > 1) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)nsplit;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.numAttrs = 1;
  }
  add_pdl_attr(cfg, attr);
  e = cudaLaunchKernelEx(&cfg, kern, S, s.N, k, idx, hist, status);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace sd
