// louver.cu -- the Louver index for threshold routing, one subspace (Louver
// summary, section 2. Louver インデックス): the keys of each (sequence, KV
// head) are grouped into clusters of r keys by a balanced PCA tree, each
// cluster is enclosed in a bounding ball, and a threshold query tests every
// ball against its halfspace {p : <qbar, p> >= tau} (section 1.
// 半空間範囲検索への帰着), prunes the clusters whose ball misses it and checks
// the keys of the surviving clusters exactly -- no false negatives.
//
// One subspace (S = 1): the page splits d into S subspaces and leaves the
// per-subspace threshold rule open; with S = 1 its two query algorithms
// coincide in the ball test.  N / r must be a power of two (balanced splits
// down to exactly r keys).
//
// Build (level by level, every node of a level at once; a node is a
// contiguous range of the permutation `perm` of the head's key ids):
//  1. node sums (means) of the key rows;
//  2. power iteration for the node's principal direction (kPowerIters
//     passes of v <- C v / |C v| with C the node's covariance, each pass one
//     read of the node's rows);
//  3. projections on that direction;
//  4. the n/2 largest projections by the library's exact radix select (ties
//     to the lower position), then a stable partition: the other half first,
//     the selected half second;
// down to leaves of 32 keys (a cluster of r keys is r/32 consecutive
// leaves); then the cluster-ordered copy of the keys, and one warp per
// cluster and per leaf computes the centre (mean) and the radius (largest
// distance, inflated by 1e-5 relative to cover fp32 rounding).  The fp32 atomic sums
// make the build's directions depend on summation order, so two builds can
// differ; every build is a valid index and query results do not depend on
// it.
//
// Query (one kernel, louver_query_kernel below): a ball test per cluster
// (bound <qbar, c> + |qbar| rho against tau - band - slack, band =
// 1e-4 |tau| + 1e-6 and slack = 1e-5 |qbar| (|c| + rho), which bounds the
// fp32 rounding of a member's score, so no rounding can prune a key that
// scores >= tau), an exact check of the survivors' keys with the scan's own
// per-key arithmetic (bit-identical to sparse_route_threshold's scores), a
// bitmap of the passing keys and the ordered set written from it.
#include "common.cuh"
#include "internal.h"
#include "scan.cuh"
#include "sparse_decode.h"

namespace sd {
namespace {

constexpr int kPowerIters = 8;
constexpr int kChunk = 256;       // keys per CTA in the per-node passes
constexpr int kPU = 4;            // keys whose loads a warp has in flight in those passes
constexpr int kLvThreads = 512;   // partition CTAs
constexpr size_t kLvHeader = 4096;

template <typename T, int EPL>
__device__ __forceinline__ void load_elems(const T *p, float (&x)[EPL]) {
#pragma unroll
  for (int e = 0; e < EPL; ++e) x[e] = DT<T>::to_f(p[e]);
}

// A key id read from the permutation, checked: an id outside [0, N) (only a
// corrupted permutation or workspace can produce one) raises INTERNAL and is
// replaced by 0, so no load or store leaves the head's rows.
__device__ __forceinline__ int checked_id(const int *perm, long long i, int N, uint32_t *status) {
  const int j = perm[i];
  if ((unsigned)j < (unsigned)N) return j;
  raise_flag(status, FLAG_INTERNAL);
  return 0;
}

// Exclusive prefix sum over a block of NT threads; *total = block sum.
template <int NT>
__device__ uint32_t lv_block_scan(uint32_t x, uint32_t *wbuf, uint32_t *total) {
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
  for (int w = 0; w < NT / 32; ++w) {
    pre += w < warp ? wbuf[w] : 0u;
    tot += wbuf[w];
  }
  *total = tot;
  return pre + inc - x;
}

__global__ void identity_perm_kernel(int *perm, int N, long long total) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < total) perm[i] = (int)(i % N);
}

// sums[seg][e] += sum of dimension e over the segment's keys.  Four warps
// per CTA of kChunk keys, a warp per key with D/32 dimensions per lane and
// kPU keys' loads in flight per warp.
template <typename T, int D>
__global__ void __launch_bounds__(128)
    seg_sum_kernel(const T *__restrict__ K, const int *__restrict__ perm, int n, int N,
                   int rows, float *__restrict__ sums, uint32_t *status) {
  constexpr int EPL = D / 32;
  __shared__ float red[4][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long base = (long long)blockIdx.x * n;
  const int bh = (int)(base / N);
  const int p0 = blockIdx.y * kChunk, p1 = min(n, p0 + kChunk);
  float acc[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
  for (int pb = p0 + warp; pb < p1; pb += 4 * kPU) {
    float x[kPU][EPL];
#pragma unroll
    for (int u = 0; u < kPU; ++u) {
      const int p = pb + 4 * u;
      if (p < p1) {
        const int j = checked_id(perm, base + p, N, status);
        load_elems<T, EPL>(K + ((size_t)bh * rows + j) * D + lane * EPL, x[u]);
      } else {
#pragma unroll
        for (int e = 0; e < EPL; ++e) x[u][e] = 0.f;
      }
    }
#pragma unroll
    for (int u = 0; u < kPU; ++u)
#pragma unroll
      for (int e = 0; e < EPL; ++e) acc[e] += x[u][e];
  }
#pragma unroll
  for (int e = 0; e < EPL; ++e) red[warp][lane * EPL + e] = acc[e];
  __syncthreads();
  for (int i = threadIdx.x; i < D; i += 128)
    atomicAdd(&sums[(size_t)blockIdx.x * D + i], red[0][i] + red[1][i] + red[2][i] + red[3][i]);
}

// One pass of the power iteration over the segment's keys: with v = v_in /
// |v_in| (the fixed start vector on the first pass) and mu = sums / n,
// acc_out += sum_keys ((x - mu) . v) (x - mu); or, when proj is given, the
// projection (x - mu) . v of each key is written to proj instead.  Four warps
// per CTA, a warp per key, D/32 dimensions per lane.
template <typename T, int D>
__global__ void __launch_bounds__(128)
    power_kernel(const T *__restrict__ K, const int *__restrict__ perm, int n, int N, int rows,
                 const float *__restrict__ sums, const float *__restrict__ v_in, int first,
                 float *__restrict__ acc_out, float *__restrict__ proj, uint32_t *status) {
  constexpr int EPL = D / 32;
  __shared__ float red[4][D];
  const int seg = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long base = (long long)seg * n;
  const int bh = (int)(base / N);
  float v[EPL], mu[EPL], nrm2 = 0.f;
#pragma unroll
  for (int e = 0; e < EPL; ++e) {
    const int i = lane * EPL + e;
    v[e] = first ? 1.f + (float)i / D : v_in[(size_t)seg * D + i];
    mu[e] = sums[(size_t)seg * D + i] / (float)n;
    nrm2 += v[e] * v[e];
  }
  nrm2 = warp_sum(nrm2);
  const float inv = nrm2 > 0.f ? rsqrtf(nrm2) : 0.f;
#pragma unroll
  for (int e = 0; e < EPL; ++e) v[e] *= inv;
  float acc[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
  const int p0 = blockIdx.y * kChunk, p1 = min(n, p0 + kChunk);
  for (int pb = p0 + warp; pb < p1; pb += 4 * kPU) {
    float x[kPU][EPL];
#pragma unroll
    for (int u = 0; u < kPU; ++u) {
      const int p = pb + 4 * u;
      if (p < p1) {
        const int j = checked_id(perm, base + p, N, status);
        load_elems<T, EPL>(K + ((size_t)bh * rows + j) * D + lane * EPL, x[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < kPU; ++u) {
      const int p = pb + 4 * u;
      if (p >= p1) break;
      float y = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        x[u][e] -= mu[e];
        y += x[u][e] * v[e];
      }
      y = warp_sum(y);
      if (proj) {
        if (lane == 0) proj[base + p] = y;
      } else {
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[e] += y * x[u][e];
      }
    }
  }
  if (proj) return;
#pragma unroll
  for (int e = 0; e < EPL; ++e) red[warp][lane * EPL + e] = acc[e];
  __syncthreads();
  for (int i = threadIdx.x; i < D; i += 128)
    atomicAdd(&acc_out[(size_t)seg * D + i], red[0][i] + red[1][i] + red[2][i] + red[3][i]);
}

// Stable partition of each segment: the positions not in sel (sel holds the
// n/2 selected positions of the segment, ascending) first, in order, then the
// selected ones.  One CTA per segment, a bitmap of n bits in shared memory.
__global__ void __launch_bounds__(kLvThreads)
    partition_kernel(const int *__restrict__ perm, const int *__restrict__ sel, int n,
                     int *__restrict__ perm_out, uint32_t *status) {
  extern __shared__ uint32_t bits[];
  __shared__ uint32_t wbuf[kLvThreads / 32];
  const int tid = threadIdx.x, half = n / 2, nw = n / 32;
  const long long base = (long long)blockIdx.x * n;
  const int *s = sel + (long long)blockIdx.x * half;
  for (int w = tid; w < nw; w += kLvThreads) bits[w] = 0u;
  __syncthreads();
  for (int i = tid; i < half; i += kLvThreads) {
    const int p = s[i];
    if ((unsigned)p >= (unsigned)n) {  // only if the select failed (flagged)
      raise_flag(status, FLAG_INTERNAL);
      continue;
    }
    atomicOr(&bits[p >> 5], 1u << (p & 31));
    perm_out[base + half + i] = perm[base + p];
  }
  __syncthreads();
  const int per = (nw + kLvThreads - 1) / kLvThreads;
  const int w0 = min(nw, tid * per), w1 = min(nw, w0 + per);
  uint32_t cnt = 0;
  for (int w = w0; w < w1; ++w) cnt += __popc(~bits[w]);
  uint32_t total;
  uint32_t pos = lv_block_scan<kLvThreads>(cnt, wbuf, &total);
  for (int w = w0; w < w1; ++w) {
    uint32_t m = ~bits[w];
    while (m) {
      const int b = __ffs(m) - 1;
      m &= m - 1u;
      perm_out[base + pos++] = perm[base + w * 32 + b];
    }
  }
}

// The index's cluster-ordered copy of the keys: row p of head bh is key
// perm[bh][p]; one thread per 16-byte piece.
template <typename T, int D>
__global__ void gather_keys_kernel(const T *__restrict__ K, const int *__restrict__ perm, int N,
                                   int rows, long long total_rows, T *__restrict__ keys,
                                   uint32_t *status) {
  constexpr int CPR = D * (int)sizeof(T) / 16;
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= total_rows * CPR) return;
  const long long row = i / CPR;
  const int part = (int)(i % CPR);
  const long long bh = row / N;
  const int j = checked_id(perm, row, N, status);
  const uint4 *src = reinterpret_cast<const uint4 *>(K + ((size_t)bh * rows + j) * D);
  reinterpret_cast<uint4 *>(keys + (size_t)row * D)[part] = src[part];
}

// Median split of a small node in one kernel (n a power of two, 64 <= n <=
// kSmallSplit; one CTA per node): the node's projections are sorted by
// (value descending, position ascending) in shared memory with a bitonic
// network, the first n/2 positions of that order are the upper half (the
// n/2 largest, ties to the lower position, exactly as the radix select takes
// them), and a stable partition writes the other half, then the upper half,
// each in position order -- what the select and partition kernels produce
// for large nodes, without a cluster per node.
constexpr int kSmallSplit = 2048;
constexpr int kSmallThreads = 256;

__global__ void __launch_bounds__(kSmallThreads)
    split_small_kernel(const float *__restrict__ proj, const int *__restrict__ perm, int n,
                       int *__restrict__ perm_out, uint32_t *status) {
  __shared__ unsigned long long kv[kSmallSplit];
  __shared__ unsigned char upper[kSmallSplit];
  __shared__ uint32_t wbuf[kSmallThreads / 32];
  const long long base = (long long)blockIdx.x * n;
  const int tid = threadIdx.x;
  bool bad = false;
  for (int i = tid; i < n; i += kSmallThreads) {
    const float f = proj[base + i];
    bad |= !isfinite(f);
    kv[i] = ((unsigned long long)(~order_key(f)) << 32) | (unsigned)i;
  }
  if (__syncthreads_or(bad) && tid == 0) raise_flag(status, FLAG_NONFINITE);
  for (int k = 2; k <= n; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < n; i += kSmallThreads) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const unsigned long long a = kv[i], b = kv[ixj];
          if ((a > b) == ((i & k) == 0)) {
            kv[i] = b;
            kv[ixj] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int i = tid; i < n; i += kSmallThreads)
    upper[(unsigned)(kv[i] & 0xffffffffull)] = i < n / 2 ? 1 : 0;
  __syncthreads();
  // thread tid owns positions [p0, p1)
  const int per = (n + kSmallThreads - 1) / kSmallThreads;
  const int p0 = min(n, tid * per), p1 = min(n, p0 + per);
  uint32_t nlow = 0;
  for (int p = p0; p < p1; ++p) nlow += upper[p] ? 0u : 1u;
  uint32_t total;
  uint32_t lo = lv_block_scan<kSmallThreads>(nlow, wbuf, &total);
  uint32_t hi = (uint32_t)(n / 2) + ((uint32_t)p0 - lo);
  for (int p = p0; p < p1; ++p) {
    const int key = perm[base + p];
    if (upper[p]) perm_out[base + hi++] = key;
    else perm_out[base + lo++] = key;
  }
}

// Centre (mean) and radius (largest distance from it, inflated) of each leaf
// cluster of r keys; one warp per cluster.
template <typename T, int D>
__global__ void __launch_bounds__(128)
    bounds_kernel(const T *__restrict__ K, const int *__restrict__ perm, int r, int N, int rows,
                  long long nclusters, float *__restrict__ centres, float *__restrict__ radii,
                  uint32_t *status) {
  constexpr int EPL = D / 32;
  const long long cl = (long long)blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (cl >= nclusters) return;
  const long long base = cl * r;
  const int bh = (int)(base / N);
  float c[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) c[e] = 0.f;
  for (int p = 0; p < r; ++p) {
    float x[EPL];
    load_elems<T, EPL>(K + ((size_t)bh * rows + checked_id(perm, base + p, N, status)) * D +
                           lane * EPL, x);
#pragma unroll
    for (int e = 0; e < EPL; ++e) c[e] += x[e];
  }
#pragma unroll
  for (int e = 0; e < EPL; ++e) c[e] /= (float)r;
  float dmax = 0.f;
  for (int p = 0; p < r; ++p) {
    float x[EPL];
    load_elems<T, EPL>(K + ((size_t)bh * rows + checked_id(perm, base + p, N, status)) * D +
                           lane * EPL, x);
    float d2 = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) d2 += (x[e] - c[e]) * (x[e] - c[e]);
    dmax = fmaxf(dmax, warp_sum(d2));
  }
#pragma unroll
  for (int e = 0; e < EPL; ++e) centres[cl * D + lane * EPL + e] = c[e];
  if (lane == 0) radii[cl] = sqrtf(dmax) * (1.f + 1e-5f) + 1e-6f;
}

// The query's first kernel: ball tests and exact checks, results as bits in
// the heads' bitmaps.  Grid (splits, heads), kQThreads threads, one CTA per
// SM; CTA x of head bh owns the head's clusters x, x + splits, ...
//  1. ball test of the owned clusters, eight lanes per cluster (64 clusters
//     per round with all their loads in flight; the first round's before
//     q's); survivors listed in shared memory;
//  1b. the 32-key leaves of the surviving clusters (the tree continues below
//     the clusters down to leaves of 32 keys, each with its own ball) get
//     the same ball test, and only the leaves that pass are checked;
//  2. exact check of the surviving leaves' keys (32 per item), each warp
//     taking every kQWarps-th item through its own ring of nb shared-memory
//     slots: an item's rows are contiguous in the index's cluster-ordered key
//     copy, so one bulk copy (TMA, completion on the slot's mbarrier) brings
//     them in, nb - 1 items ahead of the one being scored; the rows' key ids
//     are read one item ahead of their copy.  Scores come from the scan's
//     warp routine with qbar formed as the scan forms it; keys >= tau are
//     marked in the head's bitmap.
//  3. once every CTA of the head has marked its keys (a per-head arrival
//     counter, bounded wait), each CTA writes a slice of the ordered set
//     (compact_slice).  The bitmaps are double-buffered per head: a query
//     marks one and clears the other (the previous query's), and the last
//     CTA of the head to leave flips the head's parity and resets its
//     counters.
constexpr int kQWarps = 8;
constexpr int kQThreads = kQWarps * 32;
constexpr int kQGroupsPerRound = kQThreads / 8;   // clusters tested at once
constexpr int kQMaxSlots = 4;

// One CTA's share of turning a head's bitmap (nw words) into its ascending
// indices: the words [s0, s1).  The CTA counts the set bits before s0 (its
// base) and in its slice; thread t owns a contiguous run of the slice, so a
// block scan orders the threads.  The indices are staged in shared memory
// (stage_cap entries; a direct store per index would cost one memory sector
// each) and written out with coalesced stores; only the first cap are kept.
// Returns base + the slice's count (the head's total for the last slice).
__device__ uint32_t compact_slice(const uint32_t *__restrict__ bm, int s0, int s1, int cap,
                                  int *__restrict__ out, int *stage, int stage_cap,
                                  uint32_t *wbuf) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // base: set bits in words [0, s0), coalesced, 8 loads in flight per thread
  uint32_t pre = 0;
  for (int w0 = 0; w0 < s0; w0 += 8 * kQThreads) {
    uint32_t v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int wi = w0 + u * kQThreads + tid;
      v[u] = wi < s0 ? __ldcg(bm + wi) : 0u;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) pre += __popc(v[u]);
  }
  pre = __reduce_add_sync(0xffffffffu, pre);
  __syncthreads();
  if (lane == 0) wbuf[warp] = pre;
  __syncthreads();
  uint32_t base = 0;
  for (int w = 0; w < kQWarps; ++w) base += wbuf[w];
  // the slice: thread tid owns words [r0, r1)
  const int wpt = (s1 - s0 + kQThreads - 1) / kQThreads;
  const int r0 = min(s1, s0 + tid * wpt), r1 = min(s1, r0 + wpt);
  uint32_t cnt = 0;
  for (int wi = r0; wi < r1; ++wi) cnt += __popc(__ldcg(bm + wi));
  uint32_t total;
  uint32_t pos = base + lv_block_scan<kQThreads>(cnt, wbuf, &total);
  const uint32_t lim = (uint32_t)(cap < stage_cap ? cap : stage_cap);
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
  for (uint32_t i = tid; i < nst; i += kQThreads) out[base + i] = stage[i];
  return base + total;
}

template <typename T, int D>
__global__ void __launch_bounds__(kQThreads, 1)
    louver_query_kernel(const T *__restrict__ q, int Hq, int Hkv, int N, float scale,
                        const int *__restrict__ perm, const float *__restrict__ centres,
                        const float *__restrict__ radii, const float *__restrict__ sub_centres,
                        const float *__restrict__ sub_radii, const T *__restrict__ keys, int r,
                        int nc, const float *__restrict__ tau, int nb, int cap,
                        uint32_t *__restrict__ bitmap, uint32_t *__restrict__ parity,
                        int *__restrict__ nsurv, uint32_t *__restrict__ done,
                        int *__restrict__ idx, int *__restrict__ count,
                        int *__restrict__ survivors_out, uint32_t *status) {
  using C = ScoreCfg<T, D>;
  constexpr int EPG = D / 8;                  // centre elements per lane of a group
  constexpr int kItemBytes = 32 * C::kRowBytes;
  constexpr int kSlotBytes = kItemBytes + 32 * 4;  // rows + their key ids
  extern __shared__ __align__(128) unsigned char lv_smem[];
  __shared__ __align__(16) float qb[D];
  __shared__ __align__(8) uint64_t bars[kQWarps][kQMaxSlots];
  __shared__ float qn_s;
  __shared__ int nlist, nitem, ready;
  __shared__ uint32_t wbuf[kQWarps];
  const int bh = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int splits = gridDim.x;
  const int mc = (nc - (int)blockIdx.x + splits - 1) / splits;  // clusters owned
  int *list = reinterpret_cast<int *>(lv_smem + (size_t)kQWarps * nb * kSlotBytes);
  if (lane == 0)
    for (int i = 0; i < nb; ++i) mbar_init(&bars[warp][i], 1);
  fence_mbar_init();
  grid_dep_wait();
  grid_dep_launch();
  // this query marks bitmap `par` of the head and clears (its share of) the
  // other one, which the previous query used and the next one will mark
  const int nw = N / 32, BH = gridDim.y;
  const uint32_t par = __ldcg(parity + bh) & 1u;
  uint32_t *bm = bitmap + ((size_t)par * BH + bh) * nw;
  {
    uint32_t *old = bitmap + ((size_t)(par ^ 1u) * BH + bh) * nw;
    const int c0 = (int)((long long)nw * blockIdx.x / splits);
    const int c1 = (int)((long long)nw * (blockIdx.x + 1) / splits);
    for (int wi = c0 + tid; wi < c1; wi += kQThreads) old[wi] = 0u;
  }

  // ---- 1. ball test
  const int grp = tid >> 3, gl = tid & 7;
  float4 cv[2][EPG / 4];
  float rho[2];
  int ci[2];
  auto load_round = [&](int m0) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int m = m0 + u * kQGroupsPerRound + grp;
      ci[u] = m < mc ? (int)blockIdx.x + m * splits : -1;
      const float4 *c = reinterpret_cast<const float4 *>(
          centres + ((size_t)bh * nc + (ci[u] < 0 ? 0 : ci[u])) * D + gl * EPG);
#pragma unroll
      for (int v = 0; v < EPG / 4; ++v)
        cv[u][v] = ci[u] < 0 ? make_float4(0.f, 0.f, 0.f, 0.f) : __ldg(c + v);
      rho[u] = ci[u] < 0 ? 0.f : __ldg(radii + (size_t)bh * nc + ci[u]);
    }
  };
  load_round(0);
  if (tid < D) qb[tid] = qbar_elem<T, D>(q, bh, Hq, Hkv, tid, scale);
  if (tid == 0) nlist = 0;
  __syncthreads();
  if (tid < 32) {
    float s = 0.f;
    for (int i = tid; i < D; i += 32) s += qb[i] * qb[i];
    s = warp_sum(s);
    if (tid == 0) qn_s = sqrtf(s);
  }
  __syncthreads();
  const float qn = qn_s;
  const float t = tau[bh];
  if (!isfinite(t) && tid == 0 && blockIdx.x == 0) raise_flag(status, FLAG_NONFINITE);
  const float lim = t - (1e-4f * fabsf(t) + 1e-6f);
  {
    float qv[EPG];
#pragma unroll
    for (int e = 0; e < EPG; ++e) qv[e] = qb[gl * EPG + e];
    for (int m0 = 0; m0 < mc; m0 += 2 * kQGroupsPerRound) {
      if (m0 > 0) load_round(m0);
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        float dot = 0.f, cc = 0.f;
#pragma unroll
        for (int v = 0; v < EPG / 4; ++v) {
          const float4 c4 = cv[u][v];
          dot = fmaf(qv[4 * v + 0], c4.x, dot);
          dot = fmaf(qv[4 * v + 1], c4.y, dot);
          dot = fmaf(qv[4 * v + 2], c4.z, dot);
          dot = fmaf(qv[4 * v + 3], c4.w, dot);
          cc = fmaf(c4.x, c4.x, fmaf(c4.y, c4.y, fmaf(c4.z, c4.z, fmaf(c4.w, c4.w, cc))));
        }
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) {
          dot += __shfl_xor_sync(0xffffffffu, dot, o);
          cc += __shfl_xor_sync(0xffffffffu, cc, o);
        }
        const float ub = dot + qn * rho[u];
        const float slack = 1e-5f * qn * (sqrtf(cc) + rho[u]);
        if (gl == 0 && ci[u] >= 0 && (ub >= lim - slack || !(ub == ub)))
          list[atomicAdd(&nlist, 1)] = ci[u];
      }
    }
  }
  __syncthreads();
  const int ns = nlist;
  if (tid == 0 && ns) atomicAdd(&nsurv[2 * bh], ns);

  // ---- 1b. the 32-key leaves of the surviving clusters: their own balls,
  // the same test; the leaves that pass are the exact check's items (with
  // r = 32 the clusters are the leaves)
  const int ipc = r / 32;  // leaves per cluster
  int *items = list + mc;  // leaf ids within the head
  if (ipc == 1) {
    items = list;
  } else {
    if (tid == 0) nitem = 0;
    __syncthreads();
    const int ntest = ns * ipc;
    float qv[EPG];
#pragma unroll
    for (int e = 0; e < EPG; ++e) qv[e] = qb[gl * EPG + e];
    for (int m0 = 0; m0 < ntest; m0 += 2 * kQGroupsPerRound) {
      float4 sv[2][EPG / 4];
      float srho[2];
      int leaf[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int m = m0 + u * kQGroupsPerRound + grp;
        leaf[u] = m < ntest ? list[m / ipc] * ipc + m % ipc : -1;
        const size_t g = (size_t)bh * nc * ipc + (leaf[u] < 0 ? 0 : leaf[u]);
        const float4 *c = reinterpret_cast<const float4 *>(sub_centres + g * D + gl * EPG);
#pragma unroll
        for (int v = 0; v < EPG / 4; ++v)
          sv[u][v] = leaf[u] < 0 ? make_float4(0.f, 0.f, 0.f, 0.f) : __ldg(c + v);
        srho[u] = leaf[u] < 0 ? 0.f : __ldg(sub_radii + g);
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        float dot = 0.f, cc = 0.f;
#pragma unroll
        for (int v = 0; v < EPG / 4; ++v) {
          const float4 c4 = sv[u][v];
          dot = fmaf(qv[4 * v + 0], c4.x, dot);
          dot = fmaf(qv[4 * v + 1], c4.y, dot);
          dot = fmaf(qv[4 * v + 2], c4.z, dot);
          dot = fmaf(qv[4 * v + 3], c4.w, dot);
          cc = fmaf(c4.x, c4.x, fmaf(c4.y, c4.y, fmaf(c4.z, c4.z, fmaf(c4.w, c4.w, cc))));
        }
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) {
          dot += __shfl_xor_sync(0xffffffffu, dot, o);
          cc += __shfl_xor_sync(0xffffffffu, cc, o);
        }
        const float ub = dot + qn * srho[u];
        const float slack = 1e-5f * qn * (sqrtf(cc) + srho[u]);
        if (gl == 0 && leaf[u] >= 0 && (ub >= lim - slack || !(ub == ub)))
          items[atomicAdd(&nitem, 1)] = leaf[u];
      }
    }
    __syncthreads();
  }
  const int nitems = ipc == 1 ? ns : nitem;
  if (tid == 0 && nitems) atomicAdd(&nsurv[2 * bh + 1], nitems);

  // ---- 2. exact check, 32 keys per item, a private ring of slots per warp
  float qs[C::kEpl];
#pragma unroll
  for (int e = 0; e < C::kEpl; ++e) qs[e] = qb[(lane % C::kLpk) * C::kEpl + e];
  const uint32_t tkey = order_key(t);
  unsigned char *wb = lv_smem + (size_t)warp * nb * kSlotBytes;
  const size_t head0 = (size_t)bh * nc * r;  // the head's first cluster-ordered row
  // cluster-ordered row of row 0 of item it
  auto item_row = [&](int it) -> size_t { return head0 + (size_t)items[it] * 32; };
  // key id of row `lane` of item it (0 past the end)
  auto load_id = [&](int it) -> int { return it < nitems ? __ldg(perm + item_row(it) + lane) : 0; };
  // item it's rows into slot `slot` (its key ids j, one per lane)
  auto issue = [&](int it, int slot, int j) {
    if (it < nitems) {
      unsigned char *dst = wb + slot * kSlotBytes;
      reinterpret_cast<int *>(dst + kItemBytes)[lane] = j;
      if (lane == 0) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // slot reuse
        mbar_arrive_expect_tx(&bars[warp][slot], kItemBytes);
        bulk_g2s(dst, keys + item_row(it) * D, kItemBytes, &bars[warp][slot]);
      }
    }
  };
  __syncwarp();
  int jn = load_id(warp);
  for (int p = 0; p < nb - 1; ++p) {
    const int j = jn;
    jn = load_id(warp + (p + 1) * kQWarps);
    issue(warp + p * kQWarps, p, j);
  }
  int kfail = -1;
  for (int k = 0, it = warp; it < nitems; ++k, it += kQWarps) {
    const int itn = it + (nb - 1) * kQWarps;
    const int j = jn;
    jn = load_id(itn + kQWarps);
    issue(itn, (k + nb - 1) % nb, j);
    const int slot = k % nb;
    const bool ok = mbar_wait(&bars[warp][slot], (uint32_t)((k / nb) & 1), status);
    if (!__all_sync(0xffffffffu, ok)) {  // expired wait (flagged): stop
      kfail = k;
      break;
    }
    __syncwarp();
    const unsigned char *sp = wb + slot * kSlotBytes;
    const float score = warp_tile_scores<T, D>(sp, 0, qs, lane);
    const int row = (lane % C::kLpk) * C::kKpr + lane / C::kLpk;
    const int jk = reinterpret_cast<const int *>(sp + kItemBytes)[row];
    if ((unsigned)jk >= (unsigned)N) {  // only with a corrupted index (flagged)
      raise_flag(status, FLAG_INTERNAL);
    } else if (order_key(score) >= tkey) {
      atomicOr(&bm[jk >> 5], 1u << (jk & 31));
    }
    if (__any_sync(0xffffffffu, !isfinite(score)) && lane == 0)
      raise_flag(status, FLAG_NONFINITE);
    __syncwarp();  // the slot is read before it is refilled
  }
  // after an expired wait, the copies issued and not consumed (items kfail
  // .. kfail + nb - 1) are waited for, again with a limit, before going on
  if (kfail >= 0)
    for (int k2 = kfail; k2 < kfail + nb && warp + k2 * kQWarps < nitems; ++k2)
      mbar_wait(&bars[warp][k2 % nb], (uint32_t)((k2 / nb) & 1), status);

  // ---- 3. the head's CTAs turn the bitmap into the ordered set, a slice
  // each, once all of them have marked their keys: an arrival counter per
  // head (bounded wait; the grid is one wave, one CTA per SM).  The barrier
  // orders each CTA's bitmap updates before thread 0's release; thread 0's
  // acquire and the barrier after it order every CTA's updates before the
  // reads below.
  __syncthreads();
  if (tid == 0) {
    uint32_t *arrive = done + 2 * bh;
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(arrive) : "memory");
    ready = wait_counter_geq(arrive, (uint32_t)splits, kWaitLimitNs, status);
  }
  __syncthreads();
  if (!ready) return;
  const int s0 = (int)((long long)nw * blockIdx.x / splits);
  const int s1 = (int)((long long)nw * (blockIdx.x + 1) / splits);
  const uint32_t end = compact_slice(bm, s0, s1, cap, idx + (size_t)bh * cap,
                                     reinterpret_cast<int *>(lv_smem),
                                     (int)(((size_t)kQWarps * nb * kSlotBytes) / sizeof(int)),
                                     wbuf);
  if (tid == 0) {
    if (blockIdx.x == splits - 1) {  // the last slice ends at the head's total
      count[bh] = (int)end;
      if (end > (uint32_t)cap) raise_flag(status, FLAG_CAPACITY);
    }
    // the last CTA to leave resets the head's counters and flips its bitmaps
    if (atomicAdd(done + 2 * bh + 1, 1u) == (uint32_t)splits - 1) {
      if (survivors_out) {
        survivors_out[2 * bh] = __ldcg(nsurv + 2 * bh);
        survivors_out[2 * bh + 1] = __ldcg(nsurv + 2 * bh + 1);
      }
      nsurv[2 * bh] = 0;
      nsurv[2 * bh + 1] = 0;
      parity[bh] = par ^ 1u;
      done[2 * bh] = 0u;
      done[2 * bh + 1] = 0u;
    }
  }
}

// ---- host side ----------------------------------------------------------------

struct LvLayout {
  size_t perm, centres, radii, keys, sub_centres, sub_radii, index_total;  // index
  size_t sums, va, vb, proj, perm2, sel, bitmap, parity, nsurv, done, ws_total;  // workspace
};

size_t lv_align(size_t x) { return (x + 255) / 256 * 256; }

bool lv_shape_ok(const Shape &s, int r) {
  if (r < 32 || r > 256 || (r & (r - 1))) return false;
  if (s.N % r || s.N > (1 << 20)) return false;  // the partition's bitmap is on chip
  const int nc = s.N / r;
  return (nc & (nc - 1)) == 0;
}

LvLayout lv_layout(const Shape &s, int r) {
  LvLayout l;
  const size_t BH = (size_t)s.BH(), N = (size_t)s.N, nc = N / r, d = (size_t)s.d;
  l.perm = 0;
  l.centres = lv_align(BH * N * 4);
  l.radii = l.centres + lv_align(BH * nc * d * 4);
  l.keys = l.radii + lv_align(BH * nc * 4);
  l.sub_centres = l.keys + lv_align(BH * N * d * (size_t)s.esize());
  l.sub_radii = l.sub_centres + lv_align(BH * (N / 32) * d * 4);
  l.index_total = l.sub_radii + lv_align(BH * (N / 32) * 4);
  // the deepest split level has nodes of 64 keys (leaves of 32): the most
  // segments any level has
  const size_t nseg = BH * N / 64;
  l.sums = kLvHeader;
  l.va = l.sums + lv_align(nseg * d * 4);
  l.vb = l.va + lv_align(nseg * d * 4);
  l.proj = l.vb + lv_align(nseg * d * 4);
  l.perm2 = l.proj + lv_align(BH * N * 4);
  l.sel = l.perm2 + lv_align(BH * N * 4);
  l.bitmap = l.sel + lv_align(BH * N / 2 * 4 + 4);  // two per head (double-buffered)
  l.parity = l.bitmap + lv_align(2 * BH * N / 32 * 4);
  l.nsurv = l.parity + lv_align(BH * 4);
  l.done = l.nsurv + lv_align(2 * BH * 4);  // surviving clusters and leaves per head
  l.ws_total = l.done + lv_align(2 * BH * 4);
  return l;
}

template <typename T, int D>
cudaError_t lv_build_t(const Shape &s, const void *Kv, int r, char *index, char *ws,
                       cudaStream_t st) {
  const T *K = static_cast<const T *>(Kv);
  const LvLayout l = lv_layout(s, r);
  int *perm = reinterpret_cast<int *>(index + l.perm);
  int *perm2 = reinterpret_cast<int *>(ws + l.perm2);
  float *sums = reinterpret_cast<float *>(ws + l.sums);
  float *va = reinterpret_cast<float *>(ws + l.va);
  float *vb = reinterpret_cast<float *>(ws + l.vb);
  float *proj = reinterpret_cast<float *>(ws + l.proj);
  int *sel = reinterpret_cast<int *>(ws + l.sel);
  uint32_t *status = reinterpret_cast<uint32_t *>(ws);
  const long long total = (long long)s.BH() * s.N;
  identity_perm_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(perm, s.N, total);
  cudaError_t e = cudaGetLastError();
  int *cur = perm, *nxt = perm2;
  for (int n = s.N; n > 32 && e == cudaSuccess; n /= 2) {  // down to 32-key leaves
    const int nseg = (int)(total / n);
    const dim3 grid((unsigned)nseg, (unsigned)((n + kChunk - 1) / kChunk));
    e = cudaMemsetAsync(sums, 0, (size_t)nseg * D * 4, st);
    if (e != cudaSuccess) break;
    seg_sum_kernel<T, D><<<grid, 128, 0, st>>>(K, cur, n, s.N, s.Ncap, sums, status);
    float *vin = va, *vout = vb;
    for (int it = 0; it < kPowerIters && e == cudaSuccess; ++it) {
      e = cudaMemsetAsync(vout, 0, (size_t)nseg * D * 4, st);
      if (e != cudaSuccess) break;
      power_kernel<T, D><<<grid, 128, 0, st>>>(K, cur, n, s.N, s.Ncap, sums, vin, it == 0, vout,
                                                nullptr, status);
      float *t = vin;
      vin = vout;
      vout = t;
    }
    if (e != cudaSuccess) break;
    power_kernel<T, D><<<grid, 128, 0, st>>>(K, cur, n, s.N, s.Ncap, sums, vin, 0, nullptr, proj,
                                             status);
    e = cudaGetLastError();
    if (e != cudaSuccess) break;
    if (n <= kSmallSplit) {
      // small nodes: sort-based split, one CTA per node
      split_small_kernel<<<(unsigned)nseg, kSmallThreads, 0, st>>>(proj, cur, n, nxt, status);
      e = cudaGetLastError();
    } else {
      // the n/2 largest projections of every segment (ties to the lower position)
      Shape ss{1, n, nseg, nseg, 64, 0, n};
      e = launch_select(ss, proj, n / 2, nullptr, 0, sel, nullptr, n / 2, nullptr, status, st);
      if (e != cudaSuccess) break;
      const int psmem = (n / 32) * 4;
      if (psmem > 48 * 1024) {
        e = cudaFuncSetAttribute(partition_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 psmem);
        if (e != cudaSuccess) break;
      }
      partition_kernel<<<(unsigned)nseg, kLvThreads, (size_t)psmem, st>>>(cur, sel, n, nxt,
                                                                         status);
      e = cudaGetLastError();
    }
    int *t = cur;
    cur = nxt;
    nxt = t;
  }
  if (e == cudaSuccess && cur != perm)
    e = cudaMemcpyAsync(perm, cur, (size_t)total * 4, cudaMemcpyDeviceToDevice, st);
  if (e != cudaSuccess) return e;
  constexpr int CPR = D * (int)sizeof(T) / 16;
  gather_keys_kernel<T, D><<<(unsigned)((total * CPR + 255) / 256), 256, 0, st>>>(
      K, perm, s.N, s.Ncap, total, reinterpret_cast<T *>(index + l.keys), status);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const long long ncl = total / r;
  bounds_kernel<T, D><<<(unsigned)((ncl + 3) / 4), 128, 0, st>>>(
      K, perm, r, s.N, s.Ncap, ncl, reinterpret_cast<float *>(index + l.centres),
      reinterpret_cast<float *>(index + l.radii), status);
  const long long nleaf = total / 32;
  bounds_kernel<T, D><<<(unsigned)((nleaf + 3) / 4), 128, 0, st>>>(
      K, perm, 32, s.N, s.Ncap, nleaf, reinterpret_cast<float *>(index + l.sub_centres),
      reinterpret_cast<float *>(index + l.sub_radii), status);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t lv_query_t(const Shape &s, const void *qv, int r, const char *index, const float *tau,
                       int cap, int *idx, int *count, int *survivors, char *ws,
                       uint32_t *status, cudaStream_t st) {
  using C = ScoreCfg<T, D>;
  const LvLayout l = lv_layout(s, r);
  const int nc = s.N / r;
  const float scale = (float)(1.0 / __builtin_sqrt((double)D));
  DeviceInfo di;
  cudaError_t e = device_info(&di);
  if (e != cudaSuccess) return e;
  // one CTA per SM over all heads (one wave); clusters dealt round-robin to
  // a head's CTAs
  int splits = di.sm_count / s.BH();
  splits = splits < 1 ? 1 : (splits > nc ? nc : splits);
  const int mc = (nc + splits - 1) / splits;
  const size_t slot = 32 * (size_t)C::kRowBytes + 32 * 4;
  const size_t list_bytes = (size_t)mc * (1 + r / 32) * sizeof(int);  // clusters, leaves
  // as many slots per warp as fit next to the static shared memory, up to 4
  const size_t static_smem = 2048;
  int nb = (int)(((size_t)di.max_smem_optin - static_smem - list_bytes) / (kQWarps * slot));
  nb = nb > kQMaxSlots ? kQMaxSlots : nb;
  if (nb < 1) return cudaErrorNotSupported;
  const size_t smem = kQWarps * nb * slot + list_bytes;
  auto kern = louver_query_kernel<T, D>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attrs[2];
  attrs[0].id = cudaLaunchAttributeCooperative;
  attrs[0].val.cooperative = 1;
  cfg.attrs = attrs;
  cfg.stream = st;
  cfg.gridDim = dim3((unsigned)splits, (unsigned)s.BH(), 1);
  cfg.blockDim = dim3(kQThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  // the CTAs of a head meet at a counter barrier: a cooperative launch makes
  // the driver guarantee that they are all resident (at the price of not
  // overlapping with the previous kernel); a single CTA per head needs neither
  cfg.numAttrs = splits > 1 ? 1 : 0;
  if (splits == 1) add_pdl_attr(cfg, attrs);
  e = cudaLaunchKernelEx(&cfg, kern, static_cast<const T *>(qv), s.Hq, s.Hkv, s.N, scale,
                         reinterpret_cast<const int *>(index + l.perm),
                         reinterpret_cast<const float *>(index + l.centres),
                         reinterpret_cast<const float *>(index + l.radii),
                         reinterpret_cast<const float *>(index + l.sub_centres),
                         reinterpret_cast<const float *>(index + l.sub_radii),
                         reinterpret_cast<const T *>(index + l.keys), r, nc, tau, nb, cap,
                         reinterpret_cast<uint32_t *>(ws + l.bitmap),
                         reinterpret_cast<uint32_t *>(ws + l.parity),
                         reinterpret_cast<int *>(ws + l.nsurv),
                         reinterpret_cast<uint32_t *>(ws + l.done), idx, count, survivors,
                         status);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

bool louver_shape_ok(const Shape &s, int r) { return lv_shape_ok(s, r); }

void louver_sizes(const Shape &s, int r, size_t *index_bytes, size_t *ws_bytes) {
  const LvLayout l = lv_layout(s, r);
  *index_bytes = l.index_total;
  *ws_bytes = l.ws_total;
}

cudaError_t louver_build(const Shape &s, const void *K, int r, void *index, void *ws,
                         cudaStream_t st) {
  char *ix = static_cast<char *>(index);
  char *w = static_cast<char *>(ws);
  if (s.dtype == 1)
    return s.d == 128 ? lv_build_t<__nv_bfloat16, 128>(s, K, r, ix, w, st)
                      : lv_build_t<__nv_bfloat16, 64>(s, K, r, ix, w, st);
  return s.d == 128 ? lv_build_t<float, 128>(s, K, r, ix, w, st)
                    : lv_build_t<float, 64>(s, K, r, ix, w, st);
}

cudaError_t louver_query(const Shape &s, const void *q, int r, const void *index,
                         const float *tau, int cap, int *idx, int *count, int *survivors,
                         void *ws, uint32_t *status, cudaStream_t st) {
  const char *ix = static_cast<const char *>(index);
  char *w = static_cast<char *>(ws);
  if (!status) status = reinterpret_cast<uint32_t *>(ws);
  if (s.dtype == 1)
    return s.d == 128 ? lv_query_t<__nv_bfloat16, 128>(s, q, r, ix, tau, cap, idx, count,
                                                       survivors, w, status, st)
                      : lv_query_t<__nv_bfloat16, 64>(s, q, r, ix, tau, cap, idx, count,
                                                      survivors, w, status, st);
  return s.d == 128
             ? lv_query_t<float, 128>(s, q, r, ix, tau, cap, idx, count, survivors, w, status, st)
             : lv_query_t<float, 64>(s, q, r, ix, tau, cap, idx, count, survivors, w, status, st);
}

}  // namespace sd
