// threshold.cu -- A2' after the marking scan: the per-head bitmaps of keys
// with score >= tau (threshold_mark_kernel in score.cu) become the ascending
// index sets (Louver summary, sections 問題定義 and 1. 半空間範囲検索への帰着:
// every key in the halfspace, none missed).
//
// One thread-block cluster of kTSlices CTAs per (sequence, KV head); CTA c
// owns the c-th contiguous slice of the head's words.  Each CTA counts its
// slice's set bits (thread t a contiguous run of words, block scan), the
// slice totals are exchanged through distributed shared memory after a
// cluster barrier, and each CTA writes its slice's indices from its base:
// staged in shared memory and copied out with coalesced stores (a direct
// store per index costs one memory sector each).  Only the first cap indices
// of a head are written; count holds the full size and CAPACITY is flagged
// when it exceeds cap.  The bitmaps are not cleared: the marking scan
// rewrites every word on each call.
#include <cooperative_groups.h>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace sd {
namespace {

constexpr int kTSlices = 8;
constexpr int kTThreads = 256;
constexpr int kTStage = 8192;  // indices staged per CTA (32 KB)

__device__ uint32_t t_block_scan(uint32_t x, uint32_t *wbuf, uint32_t *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t inc = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  __syncthreads();
  if (lane == 31) wbuf[warp] = inc;
  __syncthreads();
  uint32_t pre = 0, tot = 0;
  for (int w = 0; w < kTThreads / 32; ++w) {
    pre += w < warp ? wbuf[w] : 0u;
    tot += wbuf[w];
  }
  *total = tot;
  return pre + inc - x;
}

__global__ void __launch_bounds__(kTThreads)
    bitmap_compact_kernel(const uint32_t *__restrict__ bits, int N, int cap,
                          int *__restrict__ idx, int *__restrict__ count, uint32_t *status) {
  cg::cluster_group cluster = cg::this_cluster();
  __shared__ uint32_t wbuf[kTThreads / 32];
  __shared__ uint32_t slice_total;
  __shared__ int stage[kTStage];
  const int rank = (int)cluster.block_rank();
  const int bh = blockIdx.y, tid = threadIdx.x;
  const int nw = (N + 31) / 32;
  const int per_slice = (nw + kTSlices - 1) / kTSlices;
  const int s0 = min(nw, rank * per_slice), s1 = min(nw, s0 + per_slice);
  const int wpt = (s1 - s0 + kTThreads - 1) / kTThreads;
  const int r0 = min(s1, s0 + tid * wpt), r1 = min(s1, r0 + wpt);
  grid_dep_wait();
  grid_dep_launch();
  const uint32_t *bm = bits + (size_t)bh * nw;
  uint32_t cnt = 0;
  for (int wi = r0; wi < r1; ++wi) cnt += __popc(__ldcg(bm + wi));
  uint32_t total;
  const uint32_t off = t_block_scan(cnt, wbuf, &total);
  if (tid == 0) slice_total = total;
  cluster.sync();
  uint32_t base = 0, head_total = 0;
  for (int c = 0; c < kTSlices; ++c) {
    const uint32_t v = *cluster.map_shared_rank(&slice_total, c);
    base += c < rank ? v : 0u;
    head_total += v;
  }
  int *out = idx + (size_t)bh * cap;
  const uint32_t lim = (uint32_t)(cap < kTStage ? cap : kTStage);
  uint32_t pos = base + off;
  for (int wi = r0; wi < r1; ++wi) {
    uint32_t m = __ldcg(bm + wi);
    while (m) {
      const int bit = __ffs(m) - 1;
      m &= m - 1u;
      if (pos < (uint32_t)cap) {
        const uint32_t sp = pos - base;
        if (sp < lim) stage[sp] = wi * 32 + bit;
        else out[pos] = wi * 32 + bit;
      }
      ++pos;
    }
  }
  __syncthreads();
  const uint32_t hi = base + total < (uint32_t)cap ? base + total : (uint32_t)cap;
  const uint32_t nst = hi > base ? min(hi - base, lim) : 0u;
  for (uint32_t i = tid; i < nst; i += kTThreads) out[base + i] = stage[i];
  if (rank == kTSlices - 1 && tid == 0) {
    count[bh] = (int)head_total;
    if (head_total > (uint32_t)cap) raise_flag(status, FLAG_CAPACITY);
  }
  cluster.sync();  // no CTA leaves while another may read its shared memory
}

}  // namespace

cudaError_t launch_bitmap_compact(const Shape &s, const uint32_t *bits, int cap, int *idx,
                                  int *count, uint32_t *status, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)kTSlices, (unsigned)s.BH(), 1);
  cfg.blockDim = dim3(kTThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attrs[2];
  attrs[0].id = cudaLaunchAttributeClusterDimension;
  attrs[0].val.clusterDim.x = kTSlices;
  attrs[0].val.clusterDim.y = 1;
  attrs[0].val.clusterDim.z = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 1;
  add_pdl_attr(cfg, attrs);
  cudaError_t e = cudaLaunchKernelEx(&cfg, bitmap_compact_kernel, bits, s.N, cap, idx, count,
                                     status);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace sd
