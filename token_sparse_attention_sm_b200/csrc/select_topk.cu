// select_topk.cu -- A2 fast path: exact top-k of each (sequence, KV head)
// when the score scan has already counted the top 11 key bits per head.
//
// Same contract as the general select kernel (select.cu): the k highest
// scores, ties to the lower key index (CLSA article, section 研究の背景と課題),
// written in ascending key order.
//
// One thread-block cluster per head; CTA r owns a contiguous slice of the
// head's scores and each warp owns a contiguous segment of that slice, which
// it walks one float4 (four keys) per lane at a time.
//  1. Every CTA reads the head's global histogram and finds the boundary bin
//     b1 where the descending count reaches k: keys above b1 are in, keys
//     below are out, and only the keys inside b1 (a couple of thousand at the
//     headline sizes) need the remaining 21 bits.
//  2. One pass loads the slice, keeps it on chip as order-preserving keys,
//     and appends every key at or above b1 (with its slice index) to its
//     warp's list, in index order (a warp scan per float4 column).
//  3. Each CTA pushes its candidate keys into every CTA's shared memory
//     (distributed shared-memory stores); after one cluster barrier every CTA
//     finishes the selection on that small list locally: one more 11-bit
//     histogram level, then the few keys left in its boundary bin are ranked
//     exactly by pairwise counts within one warp (a 10-bit histogram level
//     only if more than 64 remain).  Rank 0 clears the head's histogram for the
//     next call.
//  4. Each warp counts the entries of its list that pass; the per-CTA
//     totals are pushed the same way; one more cluster barrier gives every
//     warp its output offset, and the warp writes its passing entries in
//     list (= ascending index) order -- no second pass over the slice.
//     All exchanges are pushes, so no CTA reads another's shared memory
//     after the last barrier and no trailing barrier is needed.
// Falls back to the general multi-level cluster path when the histogram is
// not complete (the counts do not sum to N), the candidates overflow the
// on-chip lists, or the k-th score is shared by several keys (ties).
#include "internal.h"
#include "select_common.cuh"

namespace sd {
namespace {

__global__ void __launch_bounds__(kSelThreads, 1)
    select_topk_fast_kernel(const float *__restrict__ S, int N, int k,
                            int *__restrict__ idx, uint32_t *__restrict__ hist,
                            uint32_t *status) {
  cg::cluster_group cluster = cg::this_cluster();
  const int csize = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int bh = blockIdx.x / csize;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SelShared *sh = reinterpret_cast<SelShared *>(smem_raw);
  uint32_t *keys = reinterpret_cast<uint32_t *>(smem_raw + kSelFixedSmem);
  uint4 *keys4 = reinterpret_cast<uint4 *>(keys);
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const uint32_t lt_mask = (1u << lane) - 1u;
  const int per_rank = kCandAll / csize;  // receive slots per source CTA
  grid_dep_wait();
  grid_dep_launch();

  const int N4 = N >> 2;  // N % 4 == 0 on this path
  const int lo4 = (int)((long long)N4 * rank / csize);
  const int n4 = (int)((long long)N4 * (rank + 1) / csize) - lo4;
  const int lo = lo4 * 4, n = n4 * 4;
  const float4 *S4 = reinterpret_cast<const float4 *>(S + (size_t)bh * N) + lo4;
  uint32_t *gh = hist + (size_t)bh * kBins;

  // ---- 1. boundary bin from the scan's histogram ------------------------------
  uint32_t c[kBinsPerThread], sum = 0;
#pragma unroll
  for (int e = 0; e < kBinsPerThread; ++e) {
    c[e] = gh[kBins - 1 - (kBinsPerThread * tid + e)];
    sum += c[e];
  }
  uint32_t tot;
  uint32_t above = block_excl_scan(sum, sh->warp_buf, &tot);
  const bool fast = tot == (uint32_t)N;  // block-uniform: a complete histogram
  if (fast && above < (uint32_t)k && above + sum >= (uint32_t)k) {
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
  if (tid == 0) sh->ncand = 0;
  if (tid < kSelWarps) sh->wpass[tid] = 0;
  if (tid <= kSelWarps) sh->seg4[tid] = (int)((long long)n4 * tid / kSelWarps);
  __syncthreads();
  const uint32_t b1 = sh->bnd[0];
  const uint32_t above1 = sh->bnd[1];

  // ---- 2. load (a whole warp segment in flight), keep as keys, classify ------
  const int sg0 = (int)((long long)n4 * wid / kSelWarps);
  const int sg1 = (int)((long long)n4 * (wid + 1) / kSelWarps);
  constexpr int U = 8;  // float4 per lane per batch
  // Per-warp list, in index order, of the keys whose top 11 bits are >= b1
  // (every key that can be selected); a few dozen per warp in practice.
  uint32_t *wl_key = sh->wl_key[wid];
  uint32_t *wl_idx = sh->wl_idx[wid];
  uint32_t wn = 0, wcand = 0;  // list length, boundary-bin keys in it
  bool wover = false;
  bool bad = false;
  for (int b4 = sg0; b4 < sg1; b4 += U * 32) {
    float4 f[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i4 = b4 + u * 32 + lane;
      f[u] = i4 < sg1 ? S4[i4] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i4 = b4 + u * 32 + lane;
      const bool in = i4 < sg1;
      const uint4 kk = make_uint4(order_key(f[u].x), order_key(f[u].y),
                                  order_key(f[u].z), order_key(f[u].w));
      if (in) {
        keys4[i4] = kk;
        bad |= !isfinite(f[u].x) | !isfinite(f[u].y) | !isfinite(f[u].z) |
               !isfinite(f[u].w);
      }
      if (!fast) continue;
      const uint32_t kv[4] = {kk.x, kk.y, kk.z, kk.w};
      uint32_t qm = 0, cm = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t top = kv[e] >> 21;
        qm |= (in && top >= b1) ? (1u << e) : 0u;
        cm |= (in && top == b1) ? (1u << e) : 0u;
      }
      const uint32_t c = __popc(qm);
      if (!__any_sync(0xffffffffu, c != 0)) continue;
      uint32_t inc = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
      }
      uint32_t slot = wn + inc - c;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if ((qm >> e) & 1u) {
          if (slot < (uint32_t)kWarpList) {
            wl_key[slot] = kv[e];
            wl_idx[slot] = (uint32_t)(4 * i4 + e);
          }
          ++slot;
        }
      }
      wn += __shfl_sync(0xffffffffu, inc, 31);
      wcand += __popc(__ballot_sync(0xffffffffu, cm & 1u)) +
               __popc(__ballot_sync(0xffffffffu, cm & 2u)) +
               __popc(__ballot_sync(0xffffffffu, cm & 4u)) +
               __popc(__ballot_sync(0xffffffffu, cm & 8u));
    }
  }
  wover = wn > (uint32_t)kWarpList;
  if (lane == 0) {
    sh->wdef[wid] = wcand;          // this warp's boundary-bin keys
    sh->wpass[wid] = wover ? 1u : 0u;
  }
  if (__syncthreads_or(bad) && tid == 0) raise_flag(status, FLAG_NONFINITE);
  auto key_at = [&](int t) -> uint32_t { return keys[t]; };
  // candidates of this CTA = boundary-bin entries of every warp list, in
  // warp order; any list overflow turns the fast path off cluster-wide
  uint32_t cand_off = 0, my_cand = 0, my_over = 0;
#pragma unroll
  for (int i = 0; i < kSelWarps; ++i) {
    cand_off += i < wid ? sh->wdef[i] : 0u;
    my_cand += sh->wdef[i];
    my_over |= sh->wpass[i];
  }

  // push this CTA's candidate count (with the overflow flag in bit 31) and
  // keys into every CTA of the cluster (remote stores; the barrier below makes
  // them visible)
  if (fast) {
    if (tid < csize)
      cluster.map_shared_rank(sh->rcnt, tid)[rank] = my_cand | (my_over << 31);
    if (!wover) {
      uint32_t o = cand_off;
      for (uint32_t i0 = 0; i0 < wn; i0 += 32) {
        const uint32_t i = i0 + lane;
        const uint32_t key = i < wn ? wl_key[i] : 0u;
        const bool c = i < wn && (key >> 21) == b1;
        const uint32_t m = __ballot_sync(0xffffffffu, c);
        const uint32_t slot = o + __popc(m & lt_mask);
        if (c && slot < (uint32_t)per_rank)
          for (int r = 0; r < csize; ++r)
            cluster.map_shared_rank(sh->cand_all, r)[rank * per_rank + slot] = key;
        o += __popc(m);
      }
    }
  }
  cluster.sync();  // candidates delivered; every CTA has read the histogram
  if (rank == 0)
    for (int b = tid; b < kBins; b += kSelThreads) gh[b] = 0u;

  // ---- 3. refine the boundary bin on the candidate keys, locally ---------------
  uint64_t t_ge = 0;
  uint32_t tie_val = 0, n_ties = 0;
  bool fast_ok = fast;
  if (fast) {
    uint32_t over = 0;
    for (int r = 0; r < csize; ++r) {
      over |= sh->rcnt[r] >> 31;
      over |= (sh->rcnt[r] & 0x7FFFFFFFu) > (uint32_t)per_rank;
    }
    fast_ok = over == 0u;  // uniform: every CTA received the same counts
    if (fast_ok) {
      for (int b = tid; b < kBins; b += kSelThreads) sh->hist[1][b] = 0;
      __syncthreads();
      for (int r = 0; r < csize; ++r) {
        const uint32_t nr = sh->rcnt[r];
        for (uint32_t i = tid; i < nr; i += kSelThreads)
          atomicAdd(&sh->hist[1][(sh->cand_all[r * per_rank + i] >> 10) & 2047u], 1u);
      }
      __syncthreads();
      uint32_t need = (uint32_t)k - above1;
      find_boundary_local(sh->hist[1], need, sh);
      const uint32_t b2 = sh->bnd[0];
      need -= sh->bnd[1];
      const uint32_t p2 = (b1 << 11) | b2;
      const uint32_t cnt2 = sh->bnd[2];
      if (cnt2 == need) {
        t_ge = (uint64_t)p2 << 10;
      } else if (cnt2 <= (uint32_t)kFinMax) {
        // few keys left in the level-2 boundary bin: rank them exactly within
        // one warp (pairwise counts) instead of another histogram level
        if (tid == 0) sh->nfin = 0;
        __syncthreads();
        for (int r = 0; r < csize; ++r) {
          const uint32_t nr = sh->rcnt[r];
          for (uint32_t i = tid; i < nr; i += kSelThreads) {
            const uint32_t key = sh->cand_all[r * per_rank + i];
            if ((key >> 10) == p2) sh->fin[atomicAdd(&sh->nfin, 1u)] = key;
          }
        }
        __syncthreads();
        if (wid == 0) {
          const uint32_t nf = sh->nfin;  // == cnt2
          uint32_t best_v = 0, best_gt = 0, best_eq = 0;
          bool found = false;
          for (uint32_t a = lane; a < nf; a += 32) {
            const uint32_t v = sh->fin[a];
            uint32_t gt = 0, eq = 0;
            for (uint32_t c2 = 0; c2 < nf; ++c2) {
              const uint32_t u = sh->fin[c2];
              gt += u > v;
              eq += u == v;
            }
            if (gt < need && need <= gt + eq) {
              found = true;
              best_v = v;
              best_gt = gt;
              best_eq = eq;
            }
          }
          // every lane that found it holds the same value; take the lowest
          const uint32_t m = __ballot_sync(0xffffffffu, found);
          const int src = m ? __ffs(m) - 1 : 0;
          best_v = __shfl_sync(0xffffffffu, best_v, src);
          best_gt = __shfl_sync(0xffffffffu, best_gt, src);
          best_eq = __shfl_sync(0xffffffffu, best_eq, src);
          if (lane == 0) {
            sh->bnd[0] = best_v;
            sh->bnd[1] = best_gt;
            sh->bnd[2] = best_eq;
            if (!m) raise_flag(status, FLAG_INTERNAL);
          }
        }
        __syncthreads();
        const uint32_t v = sh->bnd[0];
        const uint32_t rest = need - sh->bnd[1];  // keys equal to v still needed
        if (sh->bnd[2] == rest) {
          t_ge = v;
        } else {
          t_ge = (uint64_t)v + 1;
          tie_val = v;
          n_ties = rest;
        }
      } else {
        for (int b = tid; b < kBins; b += kSelThreads) sh->hist[0][b] = 0;
        __syncthreads();
        for (int r = 0; r < csize; ++r) {
          const uint32_t nr = sh->rcnt[r];
          for (uint32_t i = tid; i < nr; i += kSelThreads) {
            const uint32_t key = sh->cand_all[r * per_rank + i];
            if ((key >> 10) == p2) atomicAdd(&sh->hist[0][key & 1023u], 1u);
          }
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
    }
  }

  int *out = idx + (size_t)bh * k;
  if (!fast_ok || n_ties) {
    // general path (pulls from remote shared memory, so it ends with a
    // cluster barrier that keeps every CTA's shared memory alive)
    if (!fast_ok)
      radix_general(cluster, sh, key_at, n, (uint32_t)k, csize, rank, nullptr, t_ge,
                    tie_val, n_ties);
    const uint32_t total_sel = compact_general(cluster, sh, key_at, n, lo, csize, rank,
                                               t_ge, tie_val, n_ties, out, (uint32_t)k);
    if (rank == 0 && tid == 0 && total_sel != (uint32_t)k) raise_flag(status, FLAG_INTERNAL);
    cluster.sync();
    return;
  }

  // ---- 4. per-warp counts from the lists, pushed offsets, ordered write ------
  // t_ge <= 2^32 here; keep the compares 32-bit
  const bool none = t_ge > 0xFFFFFFFFull;
  const uint32_t t32 = (uint32_t)t_ge;
  uint32_t wsel = 0;
  for (uint32_t i0 = 0; i0 < wn; i0 += 32) {
    const uint32_t i = i0 + lane;
    wsel += __popc(__ballot_sync(0xffffffffu, i < wn && !none && wl_key[i] >= t32));
  }
  __syncthreads();  // every warp has read wdef / wpass above
  if (lane == 0) sh->wge[wid] = wsel;
  __syncthreads();
  uint32_t before = 0, cta_sel = 0;
#pragma unroll
  for (int i = 0; i < kSelWarps; ++i) {
    const uint32_t sel = sh->wge[i];
    before += i < wid ? sel : 0u;
    cta_sel += sel;
  }
  if (tid < csize) cluster.map_shared_rank(sh->rge, tid)[rank] = cta_sel;
  cluster.sync();  // last barrier: no remote access after it
  uint32_t pos = before, total_sel = 0;
  for (int r = 0; r < csize; ++r) {
    pos += r < rank ? sh->rge[r] : 0u;
    total_sel += sh->rge[r];
  }
  for (uint32_t i0 = 0; i0 < wn; i0 += 32) {
    const uint32_t i = i0 + lane;
    const bool take = i < wn && !none && wl_key[i] >= t32;
    const uint32_t m = __ballot_sync(0xffffffffu, take);
    const uint32_t p = pos + __popc(m & lt_mask);
    if (take && p < (uint32_t)k) out[p] = lo + (int)wl_idx[i];
    pos += __popc(m);
  }
  if (rank == 0 && tid == 0 && total_sel != (uint32_t)k) raise_flag(status, FLAG_INTERNAL);
}

}  // namespace

// Launch the fast top-k kernel if its preconditions hold; returns
// cudaErrorNotSupported (nothing launched) otherwise.
cudaError_t launch_select_topk_fast(const Shape &s, const float *S, int k, int *idx,
                                    uint32_t *hist, uint32_t *status, cudaStream_t st) {
  DeviceInfo di;
  cudaError_t e = device_info(&di);
  if (e != cudaSuccess) return e;
  const int csize = di.select_cluster;
  if (!hist || (s.N & 3) != 0) return cudaErrorNotSupported;
  const size_t keys_bytes = (size_t)((s.N / 4 + csize - 1) / csize) * 16;
  const size_t smem = kSelFixedSmem + keys_bytes;
  if (smem > (size_t)di.max_smem_optin) return cudaErrorNotSupported;
  auto kern = select_topk_fast_kernel;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess && csize > 8)
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(s.BH() * csize), 1, 1);
  cfg.blockDim = dim3(kSelThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)csize;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  add_pdl_attr(cfg, attr);
  e = cudaLaunchKernelEx(&cfg, kern, S, s.N, k, idx, hist, status);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace sd
