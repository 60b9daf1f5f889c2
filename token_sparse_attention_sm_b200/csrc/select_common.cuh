// select_common.cuh -- the cluster radix select of select.cu (general top-k
// and threshold selection from given scores).
#pragma once
#include <cooperative_groups.h>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace sd {
namespace {

constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kBins = 2048;
constexpr int kBinsPerThread = kBins / kSelThreads;
constexpr int kMaxCluster = 16;
constexpr int kSelFixedSmem = 2 * kBins * 4 + 1024;

struct SelShared {
  uint32_t hist[2][kBins];
  uint32_t warp_buf[33];
  alignas(8) uint32_t pub[2];  // this CTA's (>= T, == v) counts, read remotely
  uint32_t bnd[3];             // boundary bin, count above it, count in it
  uint32_t wge[kSelWarps];     // per-warp counts of keys >= threshold
  uint32_t weq[kSelWarps];     // per-warp counts of keys == tie value
  uint32_t rge[kMaxCluster];   // per-CTA counts, copied from remote pub[]
  uint32_t req[kMaxCluster];
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


// General multi-level radix select over the cluster (keys via key_at).  Sets
// t_ge / tie_val / n_ties.  If hist_to_clear is not null, rank 0 zeroes that
// head histogram after the first cluster barrier (every CTA has read it).
template <typename KeyAt>
__device__ void radix_general(cg::cluster_group &cluster, SelShared *sh, KeyAt key_at,
                              int n, uint32_t k, int csize, int rank,
                              uint32_t *hist_to_clear, uint64_t &t_ge,
                              uint32_t &tie_val, uint32_t &n_ties) {
  const int tid = threadIdx.x;
  for (int b = tid; b < kBins; b += kSelThreads) sh->hist[0][b] = 0;
  __syncthreads();
  for (int t = tid; t < n; t += kSelThreads)
    atomicAdd(&sh->hist[0][key_at(t) >> 21], 1u);
  cluster.sync();
  if (hist_to_clear && rank == 0)
    for (int b = tid; b < kBins; b += kSelThreads) hist_to_clear[b] = 0u;
  find_boundary(cluster, sh->hist[0], csize, k, sh);
  const uint32_t b1 = sh->bnd[0];
  uint32_t need = k - sh->bnd[1];
  if (sh->bnd[2] == need) {
    t_ge = (uint64_t)b1 << 21;
    return;
  }
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
    return;
  }
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

// Order-preserving compaction of the CTA slice: every key >= t_ge, plus the
// first n_ties keys equal to tie_val in index order (across the cluster).
// Writes min(total, limit) indices; returns the cluster-wide total.  Warp w
// owns a contiguous segment and walks it 32 keys at a time; ballots keep the
// index order.
template <typename KeyAt>
__device__ uint32_t compact_general(cg::cluster_group &cluster, SelShared *sh,
                                    KeyAt key_at, int n, int lo, int csize, int rank,
                                    uint64_t t_ge, uint32_t tie_val, uint32_t n_ties,
                                    int *out, uint32_t limit) {
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
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
  if (tid < csize) {
    const uint2 p = *reinterpret_cast<const uint2 *>(cluster.map_shared_rank(sh->pub, tid));
    sh->rge[tid] = p.x;
    sh->req[tid] = p.y;
  }
  __syncthreads();
  uint32_t base_sel = 0, base_eq = 0, total_sel = 0, eq_pre = 0;
  for (int r = 0; r < csize; ++r) {
    const uint32_t ge_r = sh->rge[r], eq_r = sh->req[r];
    const uint32_t ties_r = n_ties > eq_pre ? min(eq_r, n_ties - eq_pre) : 0u;
    if (r < rank) base_sel += ge_r + ties_r;
    if (r == rank) base_eq = eq_pre;
    total_sel += ge_r + ties_r;
    eq_pre += eq_r;
  }
  uint32_t pos = base_sel, tie_rank = base_eq;
  for (int i = 0; i < wid; ++i) {
    const uint32_t ties_i = n_ties > tie_rank ? min(sh->weq[i], n_ties - tie_rank) : 0u;
    pos += sh->wge[i] + ties_i;
    tie_rank += sh->weq[i];
  }
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
  return total_sel;
}

}  // namespace
}  // namespace sd
