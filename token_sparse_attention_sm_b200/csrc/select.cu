// select.cu -- A2 (exact top-k) and A2' (threshold set) from the scores.
//
// Top-k keeps the k highest-scoring keys of each (sequence, KV head), ties to
// the lower key index (CLSA article, section 研究の背景と課題).  The threshold
// form keeps every key with score >= tau, with no false negatives (Louver
// summary, sections 問題定義 and 1. 半空間範囲検索への帰着).  Both return the set
// in ascending key order.
//
// Design: one thread-block cluster per (sequence, KV head).  The C CTAs of a
// cluster split the head's N scores into C contiguous slices and keep their
// slice in shared memory as order-preserving 32-bit keys (so every pass after
// the first reads on-chip memory, and no global workspace or counter is
// needed).
//  * Top-k is a radix select without any sort: an 11-bit histogram of the top
//    key bits, then (only if the boundary bin still holds more keys than
//    needed) 11 more bits, then the last 10 bits.  The result is either a key
//    threshold T (take every key >= T) or the exact k-th key value v plus the
//    number t of keys equal to v to take, which go to the lowest indices.
//  * Each level builds a shared-memory histogram per CTA, one cluster
//    barrier, and every CTA sums the C histograms through distributed shared
//    memory.  (Routing calls, where the score scan has already counted the
//    top 11 bits, select in select_split.cu or in the fused attention kernel
//    instead; this kernel serves selections from given scores and the Louver
//    index build.)
//  * Compaction is order preserving: each warp owns a contiguous run of its
//    CTA's slice and walks it 32 keys at a time; warp ballots and popcounts
//    give positions, one more cluster barrier exchanges the per-CTA totals,
//    and every selected index is written straight to its final position.
//    The output is therefore deterministic and ascending.
#include "internal.h"
#include "select_common.cuh"

namespace sd {
namespace {

// k >= 1: top-k (general path); k == 0: threshold (tau, cap, count).
// hist (top-k only, may be null): a head histogram to clear for the next call.
template <bool IN_SMEM>
__global__ void __launch_bounds__(kSelThreads)
    select_kernel(const float *__restrict__ S, int N, int k,
                  const float *__restrict__ tau, int cap, int *__restrict__ idx,
                  int *__restrict__ count, int stride,
                  uint32_t *__restrict__ hist, uint32_t *status) {
  cg::cluster_group cluster = cg::this_cluster();
  const int csize = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int bh = blockIdx.x / csize;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SelShared *sh = reinterpret_cast<SelShared *>(smem_raw);
  uint32_t *keys = reinterpret_cast<uint32_t *>(smem_raw + kSelFixedSmem);
  const int tid = threadIdx.x;

  const int lo = (int)((long long)N * rank / csize);
  const int hi = (int)((long long)N * (rank + 1) / csize);
  const int n = hi - lo;
  const float *Sh = S + (size_t)bh * N + lo;
  grid_dep_wait();
  grid_dep_launch();

  // Load the slice (8 independent loads in flight per thread) and keep it as
  // order-preserving keys.
  bool bad = false;
  for (int t0 = 0; t0 < n; t0 += kSelThreads * 8) {
    float f[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int t = t0 + u * kSelThreads + tid;
      f[u] = t < n ? Sh[t] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int t = t0 + u * kSelThreads + tid;
      if (t < n) {
        bad |= !isfinite(f[u]);
        if (IN_SMEM) keys[t] = order_key(f[u]);
      }
    }
  }
  if (__syncthreads_or(bad) && tid == 0) raise_flag(status, FLAG_NONFINITE);
  auto key_at = [&](int t) -> uint32_t {
    return IN_SMEM ? keys[t] : order_key(Sh[t]);
  };

  uint64_t t_ge = 0;
  uint32_t tie_val = 0, n_ties = 0;
  if (k > 0) {
    radix_general(cluster, sh, key_at, n, (uint32_t)k, csize, rank,
                  hist ? hist + (size_t)bh * kBins : nullptr, t_ge, tie_val, n_ties);
  } else {
    const float tv = tau[bh];
    if (!isfinite(tv) && tid == 0 && rank == 0) raise_flag(status, FLAG_NONFINITE);
    t_ge = order_key(tv);
  }
  const uint32_t limit = k > 0 ? (uint32_t)k : (uint32_t)cap;
  const uint32_t total_sel =
      compact_general(cluster, sh, key_at, n, lo, csize, rank, t_ge, tie_val, n_ties,
                      idx + (size_t)bh * stride, limit);
  if (rank == 0 && tid == 0) {
    if (k > 0) {
      if (total_sel != (uint32_t)k) raise_flag(status, FLAG_INTERNAL);
    } else {
      count[bh] = (int)total_sel;
      if (total_sel > (uint32_t)cap) raise_flag(status, FLAG_CAPACITY);
    }
  }
  cluster.sync();  // no CTA leaves while others may read its shared memory
}

}  // namespace

struct SelectPlan {
  int csize = 0;
  bool in_smem = false;
  size_t smem = 0;
};

static cudaError_t plan_select(const Shape &s, SelectPlan *plan) {
  DeviceInfo di;
  cudaError_t e = device_info(&di);
  if (e != cudaSuccess) return e;
  const int csize = di.select_cluster;
  const int per = (s.N + csize - 1) / csize;
  const size_t keys_bytes = (size_t)per * 4;
  plan->csize = csize;
  plan->in_smem = kSelFixedSmem + keys_bytes <= (size_t)di.max_smem_optin;
  plan->smem = kSelFixedSmem + (plan->in_smem ? keys_bytes : 0);
  return cudaSuccess;
}

cudaError_t select_cluster_size(int sm_count, int smem_optin, int *out);

cudaError_t launch_select(const Shape &s, const float *S, int k,
                          const float *tau, int cap, int *idx, int *count,
                          int stride, uint32_t *hist, uint32_t *status,
                          cudaStream_t st) {
  SelectPlan plan;
  cudaError_t e = plan_select(s, &plan);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(s.BH() * plan.csize), 1, 1);
  cfg.blockDim = dim3(kSelThreads, 1, 1);
  cfg.dynamicSmemBytes = plan.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)plan.csize;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  add_pdl_attr(cfg, attr);
  if (plan.in_smem) {
    auto kern = select_kernel<true>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)plan.smem);
    if (e == cudaSuccess && plan.csize > 8)
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    e = cudaLaunchKernelEx(&cfg, kern, S, s.N, k, tau, cap, idx, count, stride, hist, status);
  } else {
    auto kern = select_kernel<false>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)plan.smem);
    if (e == cudaSuccess && plan.csize > 8)
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    e = cudaLaunchKernelEx(&cfg, kern, S, s.N, k, tau, cap, idx, count, stride, hist, status);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Largest cluster size (16 or 8) for which the select kernel with a typical
// shared-memory footprint can keep at least 8 clusters resident at once.
cudaError_t select_cluster_size(int sm_count, int smem_optin, int *out) {
  (void)sm_count;
  (void)smem_optin;
  int best = 8;
  auto kern = select_kernel<true>;
  const int smem = kSelFixedSmem + 64 * 1024;
  cudaError_t e = cudaFuncSetAttribute(
      kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(16 * 8, 1, 1);
  cfg.blockDim = dim3(kSelThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 16;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int nclusters = 0;
  e = cudaOccupancyMaxActiveClusters(&nclusters, kern, &cfg);
  if (e == cudaSuccess && nclusters >= 8) best = 16;
  cudaGetLastError();  // a refused query is not an error for the caller
  *out = best;
  return cudaSuccess;
}

}  // namespace sd
