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
//  * Fast path: the score scan has already counted the top 11 bits per head
//    (global histogram).  Every CTA reads it and finds the boundary bin; the
//    few keys inside that bin (about k/... of N, a couple of thousand) are
//    gathered from all CTAs of the cluster through distributed shared memory
//    after one cluster barrier, and each CTA finishes the remaining 21 bits
//    on that small candidate list locally, with no further cluster barrier.
//    Rank 0 then clears the head's histogram for the next call.
//  * General path (no histogram, a histogram that does not sum to N, or more
//    candidates than fit): each level builds a shared-memory histogram per
//    CTA, one cluster barrier, and every CTA sums the C histograms through
//    distributed shared memory.
//  * Compaction is order preserving: each warp owns a contiguous run of its
//    CTA's slice and walks it 32 keys at a time; warp ballots and popcounts
//    give positions, one more cluster barrier exchanges the per-CTA totals,
//    and every selected index is written straight to its final position.
//    The output is therefore deterministic and ascending.
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
constexpr int kCandLocal = 2048;  // boundary-bin keys one CTA may hold
constexpr int kCandAll = 8192;    // boundary-bin keys of a whole head
constexpr int kSelFixedSmem = 2 * kBins * 4 + (kCandLocal + kCandAll) * 4 + 384;

struct SelShared {
  uint32_t hist[2][kBins];
  uint32_t cand_local[kCandLocal];  // read remotely by the other CTAs
  uint32_t cand_all[kCandAll];
  uint32_t warp_buf[33];
  uint32_t pub[2];        // this CTA's (>= T count, == v count), read remotely
  uint32_t bnd[3];        // boundary bin, count above it, count in it
  uint32_t ncand;         // candidates in cand_local (may exceed kCandLocal)
  uint32_t cinfo[2];      // total candidates, overflow flag
  uint32_t wge[kSelWarps];  // per-warp counts of keys >= threshold
  uint32_t weq[kSelWarps];  // per-warp counts of keys == tie value
  uint32_t pad[2];
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
#pragma unroll 4
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

// As find_boundary, for a histogram held by this CTA alone.
__device__ void find_boundary_local(const uint32_t *h, uint32_t need,
                                    SelShared *sh) {
  const int t = threadIdx.x;
  uint32_t c[kBinsPerThread];
  uint32_t sum = 0;
#pragma unroll
  for (int e = 0; e < kBinsPerThread; ++e) {
    c[e] = h[kBins - 1 - (kBinsPerThread * t + e)];
    sum += c[e];
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

// k >= 1: top-k; k == 0: threshold (tau, cap, count).  hist (top-k only,
// may be null): per-head counts of the top 11 key bits from the score scan.
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

  // Selection rule: key >= t_ge, or (key == tie_val and its rank among the
  // keys equal to tie_val, in index order, is < n_ties).
  uint64_t t_ge = 0;
  uint32_t tie_val = 0, n_ties = 0;
  const uint32_t limit = k > 0 ? (uint32_t)k : (uint32_t)cap;
  bool fast = false;
  bool hist_cleared = hist == nullptr;
  if (k > 0 && hist) {
    // ---- fast path: level 1 from the scan's histogram ----------------------
    uint32_t *gh = hist + (size_t)bh * kBins;
    uint32_t c[kBinsPerThread], sum = 0;
#pragma unroll
    for (int e = 0; e < kBinsPerThread; ++e) {
      c[e] = gh[kBins - 1 - (kBinsPerThread * tid + e)];
      sum += c[e];
    }
    uint32_t tot;
    uint32_t above = block_excl_scan(sum, sh->warp_buf, &tot);
    if (tid == 0) sh->ncand = 0;
    if (tot == (uint32_t)N) {  // block-uniform: a clean, complete histogram
      if (above < (uint32_t)k && above + sum >= (uint32_t)k) {
#pragma unroll
        for (int e = 0; e < kBinsPerThread; ++e) {
          if (above + c[e] >= (uint32_t)k) {
            sh->bnd[0] = (uint32_t)(kBins - 1 - (kBinsPerThread * tid + e));
            sh->bnd[1] = above;
            sh->bnd[2] = c[e];
            break;
          }
          above += c[e];
        }
      }
      fast = true;
    }
    __syncthreads();
    uint32_t b1 = sh->bnd[0];
    if (fast) {
      const int lane = tid & 31;
      for (int t0 = 0; t0 < n; t0 += kSelThreads) {
        const int t = t0 + tid;
        const uint32_t key = t < n ? key_at(t) : 0u;
        const bool hit = t < n && (key >> 21) == b1;
        const uint32_t m = __ballot_sync(0xffffffffu, hit);
        if (m) {  // warp-aggregated slot reservation
          uint32_t base = 0;
          if (lane == 0) base = atomicAdd(&sh->ncand, (uint32_t)__popc(m));
          base = __shfl_sync(0xffffffffu, base, 0);
          const uint32_t slot = base + __popc(m & ((1u << lane) - 1u));
          if (hit && slot < (uint32_t)kCandLocal) sh->cand_local[slot] = key;
        }
      }
    }
    cluster.sync();  // candidates published; everyone has read the histogram
    if (rank == 0)
      for (int b = tid; b < kBins; b += kSelThreads) gh[b] = 0u;
    hist_cleared = true;
    if (fast) {
      if (tid == 0) {
        uint32_t total = 0, over = 0;
        for (int r = 0; r < csize; ++r) {
          const uint32_t nr = *cluster.map_shared_rank(&sh->ncand, r);
          over |= nr > (uint32_t)kCandLocal;
          total += nr;
        }
        sh->cinfo[0] = total;
        sh->cinfo[1] = over | (total > (uint32_t)kCandAll);
      }
      __syncthreads();
      if (sh->cinfo[1] == 0u) {
        uint32_t off = 0;
        for (int r = 0; r < csize; ++r) {
          const uint32_t nr = *cluster.map_shared_rank(&sh->ncand, r);
          const uint32_t *src = cluster.map_shared_rank(sh->cand_local, r);
          for (uint32_t i = tid; i < nr; i += kSelThreads) sh->cand_all[off + i] = src[i];
          off += nr;
        }
        const uint32_t ncand = sh->cinfo[0];
        uint32_t need = (uint32_t)k - sh->bnd[1];
        __syncthreads();
        // level 2 on the candidates only (bits 20..10)
        for (int b = tid; b < kBins; b += kSelThreads) sh->hist[1][b] = 0;
        __syncthreads();
        for (uint32_t i = tid; i < ncand; i += kSelThreads)
          atomicAdd(&sh->hist[1][(sh->cand_all[i] >> 10) & 2047u], 1u);
        __syncthreads();
        find_boundary_local(sh->hist[1], need, sh);
        const uint32_t b2 = sh->bnd[0];
        need -= sh->bnd[1];
        const uint32_t p2 = (b1 << 11) | b2;
        if (sh->bnd[2] == need) {
          t_ge = (uint64_t)p2 << 10;
        } else {
          for (int b = tid; b < kBins; b += kSelThreads) sh->hist[0][b] = 0;
          __syncthreads();
          for (uint32_t i = tid; i < ncand; i += kSelThreads) {
            const uint32_t key = sh->cand_all[i];
            if ((key >> 10) == p2) atomicAdd(&sh->hist[0][key & 1023u], 1u);
          }
          __syncthreads();
          find_boundary_local(sh->hist[0], need, sh);
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
      } else {
        fast = false;  // uniform: every CTA saw the same counts
      }
    }
  }
  if (k > 0 && !fast) {
    // ---- general path ------------------------------------------------------
    for (int b = tid; b < kBins; b += kSelThreads) sh->hist[0][b] = 0;
    __syncthreads();
    for (int t = tid; t < n; t += kSelThreads)
      atomicAdd(&sh->hist[0][key_at(t) >> 21], 1u);
    cluster.sync();
    if (!hist_cleared && rank == 0)
      for (int b = tid; b < kBins; b += kSelThreads) hist[(size_t)bh * kBins + b] = 0u;
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
  } else if (k == 0) {
    const float tv = tau[bh];
    if (!isfinite(tv) && tid == 0 && rank == 0) raise_flag(status, FLAG_NONFINITE);
    t_ge = order_key(tv);
  }

  // ---- order-preserving compaction -----------------------------------------
  // Warp w owns the contiguous segment [s0, s1) of this CTA's slice and walks
  // it 32 keys at a time (conflict-free reads); ballots keep index order.
  const int lane = tid & 31, wid = tid >> 5;
  const uint32_t lt_mask = (1u << lane) - 1u;
  const int s0 = (int)((long long)n * wid / kSelWarps);
  const int s1 = (int)((long long)n * (wid + 1) / kSelWarps);
  uint32_t w_ge = 0, w_eq = 0;
  for (int t0 = s0; t0 < s1; t0 += 32) {
    const int t = t0 + lane;
    const bool in = t < s1;
    const uint32_t key = in ? key_at(t) : 0u;
    w_ge += __popc(__ballot_sync(0xffffffffu, in && (uint64_t)key >= t_ge));
    if (n_ties) w_eq += __popc(__ballot_sync(0xffffffffu, in && key == tie_val));
  }
  if (lane == 0) {
    sh->wge[wid] = w_ge;
    sh->weq[wid] = w_eq;
  }
  __syncthreads();
  uint32_t cta_ge = 0, cta_eq = 0;
  for (int i = 0; i < kSelWarps; ++i) {
    cta_ge += sh->wge[i];
    cta_eq += sh->weq[i];
  }
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
  // keys taken by the warps before this one, and this warp's first tie rank
  uint32_t pos = base_sel, tie_rank = base_eq;
  for (int i = 0; i < wid; ++i) {
    const uint32_t ties_i = n_ties > tie_rank ? min(sh->weq[i], n_ties - tie_rank) : 0u;
    pos += sh->wge[i] + ties_i;
    tie_rank += sh->weq[i];
  }
  int *out = idx + (size_t)bh * stride;
  for (int t0 = s0; t0 < s1; t0 += 32) {
    const int t = t0 + lane;
    const bool in = t < s1;
    const uint32_t key = in ? key_at(t) : 0u;
    const uint32_t ge = __ballot_sync(0xffffffffu, in && (uint64_t)key >= t_ge);
    uint32_t take = ge;
    if (n_ties) {
      const uint32_t eq = __ballot_sync(0xffffffffu, in && key == tie_val);
      const bool mine = ((eq >> lane) & 1u) && tie_rank + __popc(eq & lt_mask) < n_ties;
      take |= __ballot_sync(0xffffffffu, mine);
      tie_rank += __popc(eq);
    }
    if ((take >> lane) & 1u) {
      const uint32_t p = pos + __popc(take & lt_mask);
      if (p < limit) out[p] = lo + t;
    }
    pos += __popc(take);
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
