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
// and at the leaves one warp per cluster computes the centre (mean) and the
// radius (largest distance, inflated by 1e-5 relative to cover fp32
// rounding).  The fp32 atomic sums make the build's directions depend on
// summation order, so two builds can differ; every build is a valid index
// and query results do not depend on it.
//
// Query: a ball test per cluster (bound <qbar, c> + |qbar| rho against
// tau - band - slack, band = 1e-4 |tau| + 1e-6 and slack = 1e-5 |qbar|
// (|c| + rho), which bounds the fp32 rounding of a member's score, so no
// rounding can prune a key that scores >= tau), an exact check of the survivors' keys with the scan's own
// per-key arithmetic (bit-identical to sparse_route_threshold's scores), a
// bitmap of the passing keys and an ordered compaction into ascending
// indices.
#include "common.cuh"
#include "internal.h"
#include "scan.cuh"
#include "sparse_decode.h"

namespace sd {
namespace {

constexpr int kPowerIters = 8;
constexpr int kChunk = 256;       // keys per CTA in the per-node passes
constexpr int kLvThreads = 512;   // partition / compaction / filter CTAs
constexpr size_t kLvHeader = 4096;

__device__ __forceinline__ void cp_async16(uint32_t saddr, const void *gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(saddr), "l"(gmem) : "memory");
}

template <typename T, int EPL>
__device__ __forceinline__ void load_elems(const T *p, float (&x)[EPL]) {
#pragma unroll
  for (int e = 0; e < EPL; ++e) x[e] = DT<T>::to_f(p[e]);
}

// Exclusive prefix sum over a kLvThreads block; *total = block sum.
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
  for (int w = 0; w < kLvThreads / 32; ++w) {
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

// sums[seg][e] += sum of dimension e over the segment's keys (one CTA of D
// threads per (segment, chunk)).
template <typename T, int D>
__global__ void __launch_bounds__(D)
    seg_sum_kernel(const T *__restrict__ K, const int *__restrict__ perm, int n, int N,
                   int rows, float *__restrict__ sums) {
  const long long base = (long long)blockIdx.x * n;
  const int bh = (int)(base / N);
  const int p0 = blockIdx.y * kChunk, p1 = min(n, p0 + kChunk);
  float acc = 0.f;
  for (int p = p0; p < p1; ++p) {
    const int j = perm[base + p];
    acc += DT<T>::to_f(K[((size_t)bh * rows + j) * D + threadIdx.x]);
  }
  atomicAdd(&sums[(size_t)blockIdx.x * D + threadIdx.x], acc);
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
                 float *__restrict__ acc_out, float *__restrict__ proj) {
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
  for (int p = p0 + warp; p < p1; p += 4) {
    const int j = perm[base + p];
    float x[EPL];
    load_elems<T, EPL>(K + ((size_t)bh * rows + j) * D + lane * EPL, x);
    float y = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      x[e] -= mu[e];
      y += x[e] * v[e];
    }
    y = warp_sum(y);
    if (proj) {
      if (lane == 0) proj[base + p] = y;
    } else {
#pragma unroll
      for (int e = 0; e < EPL; ++e) acc[e] += y * x[e];
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
  uint32_t pos = lv_block_scan(cnt, wbuf, &total);
  for (int w = w0; w < w1; ++w) {
    uint32_t m = ~bits[w];
    while (m) {
      const int b = __ffs(m) - 1;
      m &= m - 1u;
      perm_out[base + pos++] = perm[base + w * 32 + b];
    }
  }
}

// Centre (mean) and radius (largest distance from it, inflated) of each leaf
// cluster of r keys; one warp per cluster.
template <typename T, int D>
__global__ void __launch_bounds__(128)
    bounds_kernel(const T *__restrict__ K, const int *__restrict__ perm, int r, int N, int rows,
                  long long nclusters, float *__restrict__ centres, float *__restrict__ radii) {
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
    load_elems<T, EPL>(K + ((size_t)bh * rows + perm[base + p]) * D + lane * EPL, x);
#pragma unroll
    for (int e = 0; e < EPL; ++e) c[e] += x[e];
  }
#pragma unroll
  for (int e = 0; e < EPL; ++e) c[e] /= (float)r;
  float dmax = 0.f;
  for (int p = 0; p < r; ++p) {
    float x[EPL];
    load_elems<T, EPL>(K + ((size_t)bh * rows + perm[base + p]) * D + lane * EPL, x);
    float d2 = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) d2 += (x[e] - c[e]) * (x[e] - c[e]);
    dmax = fmaxf(dmax, warp_sum(d2));
  }
#pragma unroll
  for (int e = 0; e < EPL; ++e) centres[cl * D + lane * EPL + e] = c[e];
  if (lane == 0) radii[cl] = sqrtf(dmax) * (1.f + 1e-5f) + 1e-6f;
}

// Ball test of every cluster of a head against its halfspace; the survivors'
// cluster ids are appended to surv[bh][..] (any order), their number counted
// in nsurv[bh] (zero on entry; the compaction kernel resets it).  Grid
// (splits, heads), a warp per cluster.
template <typename T, int D>
__global__ void __launch_bounds__(kLvThreads)
    louver_filter_kernel(const T *__restrict__ q, int Hq, int Hkv, float scale,
                         const float *__restrict__ centres, const float *__restrict__ radii,
                         int nc, const float *__restrict__ tau, int *__restrict__ surv,
                         int *__restrict__ nsurv, uint32_t *status) {
  constexpr int EPL = D / 32;
  __shared__ float qb[D];
  __shared__ float qn;
  const int bh = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = bh / Hkv, h = bh % Hkv, G = Hq / Hkv;
  grid_dep_wait();
  grid_dep_launch();
  if (tid < D) {
    float s = 0.f;
    for (int g = 0; g < G; ++g) s += DT<T>::to_f(q[((size_t)b * Hq + (size_t)h * G + g) * D + tid]);
    qb[tid] = s * scale;
  }
  __syncthreads();
  if (tid < 32) {
    float s = 0.f;
    for (int i = tid; i < D; i += 32) s += qb[i] * qb[i];
    s = warp_sum(s);
    if (tid == 0) qn = sqrtf(s);
  }
  __syncthreads();
  const float t = tau[bh];
  if (!isfinite(t) && tid == 0 && blockIdx.x == 0) raise_flag(status, FLAG_NONFINITE);
  const float lim = t - (1e-4f * fabsf(t) + 1e-6f);
  float qv[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) qv[e] = qb[lane * EPL + e];
  const int nwarps = gridDim.x * (kLvThreads / 32);
  for (int i = blockIdx.x * (kLvThreads / 32) + warp; i < nc; i += nwarps) {
    const float *c = centres + ((size_t)bh * nc + i) * D + lane * EPL;
    float dot = 0.f, cc = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      dot = fmaf(qv[e], c[e], dot);
      cc = fmaf(c[e], c[e], cc);
    }
    dot = warp_sum(dot);
    cc = warp_sum(cc);
    const float rho = radii[(size_t)bh * nc + i];
    const float ub = dot + qn * rho;
    const float slack = 1e-5f * qn * (sqrtf(cc) + rho);
    if (lane == 0 && (ub >= lim - slack || !(ub == ub))) {
      const int slot = atomicAdd(&nsurv[bh], 1);
      if (slot < nc)
        surv[(size_t)bh * nc + slot] = i;
      else  // the count did not start at zero (workspace not initialised)
        raise_flag(status, FLAG_INTERNAL);
    }
  }
}

// Exact check of the surviving clusters: their rows are gathered into shared
// memory as one scan tile and scored by the scan's warp routine (the same
// per-key arithmetic, so the same bits); keys at or above tau are marked in
// the head's bitmap.  Grid (splits, heads); four warps per CTA.
template <typename T, int D>
__global__ void __launch_bounds__(128)
    louver_exact_kernel(const T *__restrict__ q, const T *__restrict__ K, int Hq, int Hkv,
                        int N, int rows, float scale, const int *__restrict__ perm, int r,
                        const int *__restrict__ surv, const int *__restrict__ nsurv, int nc,
                        const float *__restrict__ tau, uint32_t *__restrict__ bitmap,
                        uint32_t *status) {
  using C = ScoreCfg<T, D>;
  constexpr int CPR = C::kRowBytes / 16;  // 16-byte pieces per row
  extern __shared__ __align__(128) unsigned char tile[];
  const int bh = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int sub = lane % C::kLpk;
  grid_dep_wait();
  grid_dep_launch();
  float qs[C::kEpl];
  load_qbar<T, D>(q, bh, Hq, Hkv, sub, scale, qs);
  const uint32_t tkey = order_key(tau[bh]);
  const int ns = min(nsurv[bh], nc);
  const int *pbase = perm + (size_t)bh * N;
  uint32_t *bm = bitmap + (size_t)bh * (N / 32);
  const uint32_t tile_s = smem_u32(tile);
  for (int i = blockIdx.x; i < ns; i += gridDim.x) {
    const int cl = surv[(size_t)bh * nc + i];
    if ((unsigned)cl >= (unsigned)nc) {  // uniform across the CTA
      if (tid == 0) raise_flag(status, FLAG_INTERNAL);
      continue;
    }
    const int *cp = pbase + (size_t)cl * r;
    for (int c = tid; c < r * CPR; c += 128) {
      const int row = c / CPR, part = c % CPR;
      cp_async16(tile_s + row * C::kRowBytes + part * 16,
                 reinterpret_cast<const unsigned char *>(K + ((size_t)bh * rows + cp[row]) * D) +
                     part * 16);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();
    for (int wt = warp; wt < r / 32; wt += 4) {
      const float score = warp_tile_scores<T, D>(tile, wt * 32, qs, lane);
      const int kk = wt * 32 + sub * C::kKpr + lane / C::kLpk;
      const int j = cp[kk];
      if (order_key(score) >= tkey) atomicOr(&bm[j >> 5], 1u << (j & 31));
      if (__any_sync(0xffffffffu, !isfinite(score)) && lane == 0)
        raise_flag(status, FLAG_NONFINITE);
    }
    __syncthreads();  // the tile is read before the next gather
  }
}

// Bitmap -> ascending indices (the first cap), count; clears the bitmap and
// the survivor count for the next query.
__global__ void __launch_bounds__(kLvThreads)
    louver_compact_kernel(uint32_t *__restrict__ bitmap, int N, int cap, int *__restrict__ idx,
                          int *__restrict__ count, int *__restrict__ nsurv,
                          int *__restrict__ survivors_out, uint32_t *status) {
  __shared__ uint32_t wbuf[kLvThreads / 32];
  const int bh = blockIdx.x, tid = threadIdx.x, nw = N / 32;
  grid_dep_wait();
  grid_dep_launch();
  uint32_t *bm = bitmap + (size_t)bh * nw;
  const int per = (nw + kLvThreads - 1) / kLvThreads;
  const int w0 = min(nw, tid * per), w1 = min(nw, w0 + per);
  uint32_t cnt = 0;
  for (int w = w0; w < w1; ++w) cnt += __popc(bm[w]);
  uint32_t total;
  uint32_t pos = lv_block_scan(cnt, wbuf, &total);
  int *out = idx + (size_t)bh * cap;
  for (int w = w0; w < w1; ++w) {
    uint32_t m = bm[w];
    bm[w] = 0u;
    while (m) {
      const int b = __ffs(m) - 1;
      m &= m - 1u;
      if (pos < (uint32_t)cap) out[pos] = w * 32 + b;
      ++pos;
    }
  }
  if (tid == 0) {
    count[bh] = (int)total;
    if (total > (uint32_t)cap) raise_flag(status, FLAG_CAPACITY);
    if (survivors_out) survivors_out[bh] = nsurv[bh];
    nsurv[bh] = 0;
  }
}

// ---- host side ----------------------------------------------------------------

struct LvLayout {
  size_t perm, centres, radii, index_total;                            // index
  size_t sums, va, vb, proj, perm2, sel, bitmap, surv, nsurv, ws_total;  // workspace
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
  l.index_total = l.radii + lv_align(BH * nc * 4);
  const size_t nseg = BH * N / r;  // bound on the segments of any level
  l.sums = kLvHeader;
  l.va = l.sums + lv_align(nseg * d * 4);
  l.vb = l.va + lv_align(nseg * d * 4);
  l.proj = l.vb + lv_align(nseg * d * 4);
  l.perm2 = l.proj + lv_align(BH * N * 4);
  l.sel = l.perm2 + lv_align(BH * N * 4);
  l.bitmap = l.sel + lv_align(BH * N / 2 * 4 + 4);
  l.surv = l.bitmap + lv_align(BH * N / 32 * 4);
  l.nsurv = l.surv + lv_align(BH * nc * 4);
  l.ws_total = l.nsurv + lv_align(BH * 4);
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
  for (int n = s.N; n > r && e == cudaSuccess; n /= 2) {
    const int nseg = (int)(total / n);
    const dim3 grid((unsigned)nseg, (unsigned)((n + kChunk - 1) / kChunk));
    e = cudaMemsetAsync(sums, 0, (size_t)nseg * D * 4, st);
    if (e != cudaSuccess) break;
    seg_sum_kernel<T, D><<<grid, D, 0, st>>>(K, cur, n, s.N, s.Ncap, sums);
    float *vin = va, *vout = vb;
    for (int it = 0; it < kPowerIters && e == cudaSuccess; ++it) {
      e = cudaMemsetAsync(vout, 0, (size_t)nseg * D * 4, st);
      if (e != cudaSuccess) break;
      power_kernel<T, D><<<grid, 128, 0, st>>>(K, cur, n, s.N, s.Ncap, sums, vin, it == 0, vout,
                                                nullptr);
      float *t = vin;
      vin = vout;
      vout = t;
    }
    if (e != cudaSuccess) break;
    power_kernel<T, D><<<grid, 128, 0, st>>>(K, cur, n, s.N, s.Ncap, sums, vin, 0, nullptr, proj);
    e = cudaGetLastError();
    if (e != cudaSuccess) break;
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
    int *t = cur;
    cur = nxt;
    nxt = t;
  }
  if (e == cudaSuccess && cur != perm)
    e = cudaMemcpyAsync(perm, cur, (size_t)total * 4, cudaMemcpyDeviceToDevice, st);
  if (e != cudaSuccess) return e;
  const long long ncl = total / r;
  bounds_kernel<T, D><<<(unsigned)((ncl + 3) / 4), 128, 0, st>>>(
      K, perm, r, s.N, s.Ncap, ncl, reinterpret_cast<float *>(index + l.centres),
      reinterpret_cast<float *>(index + l.radii));
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t lv_query_t(const Shape &s, const void *qv, const void *Kv, int r, const char *index,
                       const float *tau, int cap, int *idx, int *count, int *survivors,
                       char *ws, cudaStream_t st) {
  using C = ScoreCfg<T, D>;
  const T *q = static_cast<const T *>(qv);
  const T *K = static_cast<const T *>(Kv);
  const LvLayout l = lv_layout(s, r);
  const int nc = s.N / r;
  const float scale = (float)(1.0 / __builtin_sqrt((double)D));
  uint32_t *status = reinterpret_cast<uint32_t *>(ws);
  int *surv = reinterpret_cast<int *>(ws + l.surv);
  int *nsurv = reinterpret_cast<int *>(ws + l.nsurv);
  uint32_t *bitmap = reinterpret_cast<uint32_t *>(ws + l.bitmap);
  const int *perm = reinterpret_cast<const int *>(index + l.perm);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attrs[1];
  cfg.attrs = attrs;
  cfg.stream = st;
  DeviceInfo di;
  cudaError_t e = device_info(&di);
  if (e != cudaSuccess) return e;
  // ball test
  int fsplit = (di.sm_count + s.BH() - 1) / s.BH();
  const int fmax = (nc + kLvThreads / 32 - 1) / (kLvThreads / 32);
  fsplit = fsplit < 1 ? 1 : (fsplit > fmax ? fmax : fsplit);
  cfg.gridDim = dim3((unsigned)fsplit, (unsigned)s.BH(), 1);
  cfg.blockDim = dim3(kLvThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.numAttrs = 0;
  add_pdl_attr(cfg, attrs);
  e = cudaLaunchKernelEx(&cfg, louver_filter_kernel<T, D>, q, s.Hq, s.Hkv, scale,
                         reinterpret_cast<const float *>(index + l.centres),
                         reinterpret_cast<const float *>(index + l.radii), nc, tau, surv, nsurv,
                         status);
  if (e != cudaSuccess) return e;
  // exact check of the survivors
  const int smem = r * C::kRowBytes;
  auto kx = louver_exact_kernel<T, D>;
  e = cudaFuncSetAttribute(kx, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int splits = (4 * di.sm_count + s.BH() - 1) / s.BH();
  splits = splits < 1 ? 1 : (splits > nc ? nc : splits);
  cfg.gridDim = dim3((unsigned)splits, (unsigned)s.BH(), 1);
  cfg.blockDim = dim3(128, 1, 1);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.numAttrs = 0;
  add_pdl_attr(cfg, attrs);
  e = cudaLaunchKernelEx(&cfg, kx, q, K, s.Hq, s.Hkv, s.N, s.Ncap, scale, perm, r,
                         static_cast<const int *>(surv), static_cast<const int *>(nsurv), nc,
                         tau, bitmap, status);
  if (e != cudaSuccess) return e;
  // ordered compaction
  cfg.gridDim = dim3((unsigned)s.BH(), 1, 1);
  cfg.blockDim = dim3(kLvThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.numAttrs = 0;
  add_pdl_attr(cfg, attrs);
  e = cudaLaunchKernelEx(&cfg, louver_compact_kernel, bitmap, s.N, cap, idx, count, nsurv,
                         survivors, status);
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

cudaError_t louver_query(const Shape &s, const void *q, const void *K, int r, const void *index,
                         const float *tau, int cap, int *idx, int *count, int *survivors,
                         void *ws, cudaStream_t st) {
  const char *ix = static_cast<const char *>(index);
  char *w = static_cast<char *>(ws);
  if (s.dtype == 1)
    return s.d == 128 ? lv_query_t<__nv_bfloat16, 128>(s, q, K, r, ix, tau, cap, idx, count,
                                                       survivors, w, st)
                      : lv_query_t<__nv_bfloat16, 64>(s, q, K, r, ix, tau, cap, idx, count,
                                                      survivors, w, st);
  return s.d == 128 ? lv_query_t<float, 128>(s, q, K, r, ix, tau, cap, idx, count, survivors, w, st)
                    : lv_query_t<float, 64>(s, q, K, r, ix, tau, cap, idx, count, survivors, w,
                                            st);
}

}  // namespace sd
