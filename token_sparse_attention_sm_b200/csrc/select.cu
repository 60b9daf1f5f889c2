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
//    needed) 11 more bits, then the last 10 bits.  Each level builds a
//    shared-memory histogram per CTA, one cluster barrier, and every CTA sums
//    the C histograms through distributed shared memory and finds the bin in
//    which the descending cumulative count reaches k (block-wide scan).  The
//    result is either a key threshold T (take every key >= T) or the exact
//    k-th key value v plus the number t of keys equal to v to take, which go
//    to the lowest indices.
//  * Compaction is order preserving: each thread owns a contiguous run of its
//    CTA's slice; block scans give per-thread offsets, one more cluster
//    barrier exchanges the per-CTA totals, and every selected index is
//    written straight to its final position.  The output is therefore
//    deterministic and ascending.
#include <cooperative_groups.h>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace sd {
namespace {

constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kBins = 2048;
constexpr int kBinsPerThread = kBins / kSelThreads;
constexpr int kSelFixedSmem = 2 * kBins * 4 + 256;

struct SelShared {
  uint32_t hist[2][kBins];
  uint32_t warp_buf[33];
  uint32_t pub[2];        // this CTA's (>= T count, == v count), read remotely
  uint32_t bnd[3];        // boundary bin, count above it, count in it
  uint32_t pad[24];
};
static_assert(sizeof(SelShared) <= kSelFixedSmem, "fixed select smem");

// Exclusive block-wide prefix sum of x over the 512 threads; *total gets the
// block sum.  Contains barriers: every thread must call it.
__device__ uint32_t block_excl_scan(uint32_t x, uint32_t *warp_buf,
                                    uint32_t *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t inc = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) warp_buf[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    const uint32_t w = lane < kSelWarps ? warp_buf[lane] : 0u;
    uint32_t wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    if (lane < kSelWarps) warp_buf[lane] = wi - w;
    if (lane == kSelWarps - 1) warp_buf[32] = wi;
  }
  __syncthreads();
  const uint32_t r = warp_buf[warp] + inc - x;
  *total = warp_buf[32];
  __syncthreads();
  return r;
}

// Sum the histogram `h` of every CTA of the cluster and find the bin where
// the count of keys, accumulated from the highest bin down, reaches `need`
// (1 <= need <= total).  Result in sh->bnd = {bin, keys above it, keys in it}.
__device__ void find_boundary(cg::cluster_group &cluster, uint32_t *h,
                              int csize, uint32_t need, SelShared *sh) {
  const int t = threadIdx.x;
  uint32_t c[kBinsPerThread];
  uint32_t sum = 0;
#pragma unroll
  for (int e = 0; e < kBinsPerThread; ++e) {
    const int b = kBins - 1 - (kBinsPerThread * t + e);
    uint32_t acc = 0;
    for (int r = 0; r < csize; ++r) acc += cluster.map_shared_rank(h, r)[b];
    c[e] = acc;
    sum += acc;
  }
  uint32_t tot;
  uint32_t above = block_excl_scan(sum, sh->warp_buf, &tot);
  if (above < need && above + sum >= need) {
#pragma unroll
    for (int e = 0; e < kBinsPerThread; ++e) {
      if (above + c[e] >= need) {
        sh->bnd[0] = (uint32_t)(kBins - 1 - (kBinsPerThread * t + e));
        sh->bnd[1] = above;
        sh->bnd[2] = c[e];
        break;
      }
      above += c[e];
    }
  }
  __syncthreads();
}

// k >= 1: top-k; k == 0: threshold (tau, cap, count).
template <bool IN_SMEM>
__global__ void __launch_bounds__(kSelThreads)
    select_kernel(const float *__restrict__ S, int N, int k,
                  const float *__restrict__ tau, int cap, int *__restrict__ idx,
                  int *__restrict__ count, int stride, uint32_t *status) {
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

  bool bad = false;
  if (IN_SMEM) {
    for (int t = tid; t < n; t += kSelThreads) {
      const float f = Sh[t];
      bad |= !isfinite(f);
      keys[t] = order_key(f);
    }
  } else {
    for (int t = tid; t < n; t += kSelThreads) bad |= !isfinite(Sh[t]);
  }
  if (__syncthreads_or(bad) && tid == 0) raise_flag(status, FLAG_NONFINITE);
  auto key_at = [&](int t) -> uint32_t {
    return IN_SMEM ? keys[t] : order_key(Sh[t]);
  };

  // Selection rule: key >= t_ge, or (key == tie_val and its rank among the
  // keys equal to tie_val, in index order, is < n_ties).
  uint64_t t_ge;
  uint32_t tie_val = 0, n_ties = 0;
  const uint32_t limit = k > 0 ? (uint32_t)k : (uint32_t)cap;
  if (k > 0) {
    for (int b = tid; b < kBins; b += kSelThreads) sh->hist[0][b] = 0;
    __syncthreads();
    for (int t = tid; t < n; t += kSelThreads)
      atomicAdd(&sh->hist[0][key_at(t) >> 21], 1u);
    cluster.sync();
    find_boundary(cluster, sh->hist[0], csize, (uint32_t)k, sh);
    const uint32_t b1 = sh->bnd[0];
    uint32_t need = (uint32_t)k - sh->bnd[1];
    if (sh->bnd[2] == need) {
      t_ge = (uint64_t)b1 << 21;
    } else {
      for (int b = tid; b < kBins; b += kSelThreads) sh->hist[1][b] = 0;
      __syncthreads();
      for (int t = tid; t < n; t += kSelThreads) {
        const uint32_t key = key_at(t);
        if ((key >> 21) == b1) atomicAdd(&sh->hist[1][(key >> 10) & 2047u], 1u);
      }
      cluster.sync();  // also: every CTA has finished reading hist[0]
      find_boundary(cluster, sh->hist[1], csize, need, sh);
      const uint32_t b2 = sh->bnd[0];
      need -= sh->bnd[1];
      const uint32_t p2 = (b1 << 11) | b2;
      if (sh->bnd[2] == need) {
        t_ge = (uint64_t)p2 << 10;
      } else {
        for (int b = tid; b < kBins; b += kSelThreads) sh->hist[0][b] = 0;
        __syncthreads();
        for (int t = tid; t < n; t += kSelThreads) {
          const uint32_t key = key_at(t);
          if ((key >> 10) == p2) atomicAdd(&sh->hist[0][key & 1023u], 1u);
        }
        cluster.sync();
        find_boundary(cluster, sh->hist[0], csize, need, sh);
        const uint32_t v = (p2 << 10) | sh->bnd[0];
        need -= sh->bnd[1];
        if (sh->bnd[2] == need) {
          t_ge = v;
        } else {
          t_ge = (uint64_t)v + 1;
          tie_val = v;
          n_ties = need;
        }
      }
    }
  } else {
    const float tv = tau[bh];
    if (!isfinite(tv) && tid == 0 && rank == 0) raise_flag(status, FLAG_NONFINITE);
    t_ge = order_key(tv);
  }

  // ---- order-preserving compaction -----------------------------------------
  const int per = (n + kSelThreads - 1) / kSelThreads;
  const int c0 = min(n, tid * per), c1 = min(n, c0 + per);
  uint32_t n_ge = 0, n_eq = 0;
  for (int t = c0; t < c1; ++t) {
    const uint32_t key = key_at(t);
    n_ge += (uint64_t)key >= t_ge;
    n_eq += (n_ties != 0u) & (key == tie_val);
  }
  uint32_t cta_ge, cta_eq;
  const uint32_t ex_ge = block_excl_scan(n_ge, sh->warp_buf, &cta_ge);
  const uint32_t ex_eq = block_excl_scan(n_eq, sh->warp_buf, &cta_eq);
  (void)ex_ge;
  if (tid == 0) {
    sh->pub[0] = cta_ge;
    sh->pub[1] = cta_eq;
  }
  cluster.sync();
  uint32_t base_sel = 0, base_eq = 0, total_sel = 0, eq_pre = 0;
  for (int r = 0; r < csize; ++r) {
    const uint32_t *p = cluster.map_shared_rank(sh->pub, r);
    const uint32_t ge_r = p[0], eq_r = p[1];
    const uint32_t ties_r = n_ties > eq_pre ? min(eq_r, n_ties - eq_pre) : 0u;
    if (r < rank) base_sel += ge_r + ties_r;
    if (r == rank) base_eq = eq_pre;
    total_sel += ge_r + ties_r;
    eq_pre += eq_r;
  }
  const uint32_t tie0 = base_eq + ex_eq;
  const uint32_t my_ties = n_ties > tie0 ? min(n_eq, n_ties - tie0) : 0u;
  uint32_t cta_sel;
  const uint32_t ex_sel = block_excl_scan(n_ge + my_ties, sh->warp_buf, &cta_sel);
  uint32_t pos = base_sel + ex_sel;
  uint32_t tie_rank = tie0;
  int *out = idx + (size_t)bh * stride;
  for (int t = c0; t < c1; ++t) {
    const uint32_t key = key_at(t);
    bool take = (uint64_t)key >= t_ge;
    if (!take && n_ties != 0u && key == tie_val) take = tie_rank++ < n_ties;
    if (take) {
      if (pos < limit) out[pos] = lo + t;
      ++pos;
    }
  }
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

struct SelectPlan {
  int csize = 0;
  bool in_smem = false;
  size_t smem = 0;
};

}  // namespace

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
                          int stride, uint32_t *status, cudaStream_t st) {
  SelectPlan plan;
  cudaError_t e = plan_select(s, &plan);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(s.BH() * plan.csize), 1, 1);
  cfg.blockDim = dim3(kSelThreads, 1, 1);
  cfg.dynamicSmemBytes = plan.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)plan.csize;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (plan.in_smem) {
    auto kern = select_kernel<true>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)plan.smem);
    if (e == cudaSuccess && plan.csize > 8)
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    e = cudaLaunchKernelEx(&cfg, kern, S, s.N, k, tau, cap, idx, count, stride, status);
  } else {
    auto kern = select_kernel<false>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)plan.smem);
    if (e == cudaSuccess && plan.csize > 8)
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    e = cudaLaunchKernelEx(&cfg, kern, S, s.N, k, tau, cap, idx, count, stride, status);
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
