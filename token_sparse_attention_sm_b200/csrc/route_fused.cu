// route_fused.cu -- A1 + A2 in one persistent kernel: the routing score scan
// and the exact top-k of every (sequence, KV head), without a second pass
// over the scores.
//
// Contract (same as sparse_route_topk): the k highest group scores of each
// head, ties to the lower key index (CLSA article, section 研究の背景と課題),
// written in ascending key order; S is also written (fp32, [B,Hkv,N]).
//
// The scan (scan.cuh) runs as in the score kernel, and every CTA also keeps
// the order-preserving 32-bit keys of its scores in shared memory (at most
// 8192 keys: the kernel is used when a CTA's share fits) and counts their top
// 11 bits.  Every CTA scans a contiguous share of one head's tiles (the
// grid is a whole number of CTAs per head, 18 at 128K keys and 8 heads on
// 148 SMs).  Then the CTAs of a head cooperate through global memory with two
// counting barriers:
//  A. every CTA has added its counts to the head's histogram.  Each CTA reads
//     the histogram, finds the boundary bin b1 (where the descending count
//     reaches k) and walks its own keys on chip: keys above b1 are in, keys
//     below are out.  Each lane counts the keys at or above b1 in its own
//     run of keys, then (after a warp scan) lists them in key order, so each
//     warp holds an ordered list of a few dozen.  Each CTA publishes its
//     boundary-bin keys (about a hundred) and its count of keys above b1.
//  B. every CTA has published.  Each CTA loads the head's published keys
//     (about 2K, in one round trip: a group of threads per publishing CTA),
//     finishes the selection on them locally -- an 11-bit
//     histogram level, then a pairwise rank of the few keys left (or a last
//     10-bit level) -- and derives every CTA's number of selected keys, hence
//     its own output offset, from the published data alone; its warps then
//     write their listed keys that pass, in order.  Keys equal to the k-th
//     score are all boundary-bin keys, so ties to the lower index are
//     resolved from the published keys too.
// The last CTA to leave a head resets its barrier counter, and the head's
// first CTA clears its histogram row, so the workspace is ready for the next
// call.  When the published keys do not fit (a boundary bin holding
// thousands of keys: many equal scores) or the histogram is not consistent
// (counts not summing to N: a dirty workspace), the head's first CTA selects
// alone from the fp32 scores in global memory (three radix levels and an
// ordered compaction); slow, but exact.
//
// The barriers need every CTA of the grid resident at once: the grid is at
// most one CTA per SM and the kernel occupies a whole SM.  Every wait is
// bounded (TIMEOUT flag on expiry).
#include <stdlib.h>

#include "common.cuh"
#include "internal.h"
#include "scan.cuh"

namespace sd {
namespace {

constexpr int kFThreads = 512;  // warps 0-4 run the scan, all 16 the select
constexpr int kFWarps = kFThreads / 32;
constexpr int kFMaxKeys = 8192;           // keys a CTA keeps on chip
constexpr int kFWarpList = 512;           // list entries per warp and head slot
constexpr int kFCandMax = 12288;          // published keys of one head, on chip
constexpr int kFFinMax = 64;              // keys ranked pairwise
constexpr uint32_t kNone = 0xFFFFFFFFu;

struct FMisc {
  uint32_t wbuf[kFWarps];
  uint32_t bnd[4];          // boundary bin, count above it, count in it, total
  uint32_t wq[kFWarps];     // per warp: keys at or above the boundary bin
  uint32_t wc[kFWarps];     // per warp: keys in the boundary bin
  uint32_t wge[kFWarps];    // per warp: keys at or above the threshold
  uint32_t weq[kFWarps];    // per warp: keys equal to the tie value
  uint32_t res[4];          // output offset, ties allowed, total selected, bad flag
  uint32_t nfin;
  uint32_t fin[kFFinMax];
  int ok;
};

// shared memory: the scan ring, reused after the scan for the select
constexpr int kFRingBytes = kScanStages * kScanStageBytes;
constexpr int kFShistOff = kFRingBytes;
constexpr int kFKeysOff = kFShistOff + kScanBins * 4;
constexpr int kFBarOff = kFKeysOff + kFMaxKeys * 4;
constexpr int kFMiscOff = kFBarOff + 2 * kScanStages * 8;
constexpr int kFSmem = kFMiscOff + (int)sizeof(FMisc);
constexpr int kFListOff = 0;  // [kFWarps][kFWarpList] (key, j)
constexpr int kFCandOff = kFListOff + kFWarps * kFWarpList * 8;
constexpr int kFRhistOff = kFCandOff + kFCandMax * 4;
constexpr int kFSegOff = kFRhistOff + kScanBins * 4;
constexpr int kFSegFields = 5;  // off, cnt, def, ge, eq per publishing CTA
constexpr int kFSegBytes = kFSegFields * (kFusedMaxCtas + 1) * 4;
static_assert(kFSegOff + kFSegBytes <= kFRingBytes, "select scratch fits in the ring");
static_assert(kFSmem <= 227 * 1024, "fits the shared-memory opt-in limit");

__device__ __forceinline__ void arrive(uint32_t *ctr) {
  __threadfence();
  asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(ctr) : "memory");
}

// thread 0 only: wait until *ctr >= target (bounded)
__device__ bool wait_count(const uint32_t *ctr, uint32_t target, uint32_t *status) {
  return wait_counter_geq(ctr, target, kWaitLimitNs, status);
}

// Bins taken from the top down: bnd[0] = the bin at which the running count
// reaches `need` (kNone if the counts sum to less), bnd[1] = count in higher
// bins, bnd[2] = count in the bin, bnd[3] = total.  h may be shared or
// global memory.  Every thread of the block calls it.
template <int NBINS>
__device__ void desc_boundary(const uint32_t *h, uint32_t need, FMisc *m) {
  constexpr int PER = (NBINS + kFThreads - 1) / kFThreads;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  __syncthreads();  // earlier results have been read
  if (tid == 0) m->bnd[0] = kNone;
  uint32_t c[PER], sum = 0;
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    const int d = tid * PER + e;
    c[e] = d < NBINS ? h[NBINS - 1 - d] : 0u;
    sum += c[e];
  }
  uint32_t inc = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) m->wbuf[warp] = inc;
  __syncthreads();
  uint32_t pre = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kFWarps; ++w) {
    pre += w < warp ? m->wbuf[w] : 0u;
    tot += m->wbuf[w];
  }
  uint32_t above = pre + inc - sum;
  if (above < need && above + sum >= need) {
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      if (above + c[e] >= need) {
        m->bnd[0] = (uint32_t)(NBINS - 1 - (tid * PER + e));
        m->bnd[1] = above;
        m->bnd[2] = c[e];
        break;
      }
      above += c[e];
    }
  }
  if (tid == 0) m->bnd[3] = tot;
  __syncthreads();
}

__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += y;
  }
  return v;
}

// One warp writes, in key order, the keys of its run of 4-key columns
// [c0, c1) (key j = jbase + 4*col + e) that are >= t_ge, or equal to tie_val
// and among the first `allow` such keys of the run, from output slot pos on.
// load(col, in) returns the column's four order-preserving keys.
template <typename Load>
__device__ __forceinline__ void warp_ordered_write(Load load, int c0, int c1, int jbase,
                                                   uint64_t t_ge, uint32_t tie_val, bool ties,
                                                   uint32_t allow, uint32_t pos,
                                                   int *__restrict__ out, int k) {
  const int lane = threadIdx.x & 31;
  uint32_t tseen = 0;
  for (int b = c0; b < c1; b += 32) {
    const int i = b + lane;
    const bool in = i < c1;
    const uint4 kk = load(i, in);
    const uint32_t kv[4] = {kk.x, kk.y, kk.z, kk.w};
    uint32_t gm = 0, tm = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      gm |= (in && (uint64_t)kv[e] >= t_ge) ? (1u << e) : 0u;
      tm |= (in && ties && kv[e] == tie_val) ? (1u << e) : 0u;
    }
    if (!__any_sync(0xffffffffu, (gm | tm) != 0)) continue;
    const uint32_t tc = __popc(tm);
    const uint32_t tinc = warp_incl_scan(tc);
    uint32_t tr = tseen + tinc - tc;  // tie rank of this lane's first tie key
    uint32_t take = gm;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if ((tm >> e) & 1u) {
        if (tr < allow) take |= 1u << e;
        ++tr;
      }
    }
    const uint32_t cc = __popc(take);
    const uint32_t cinc = warp_incl_scan(cc);
    uint32_t p = pos + cinc - cc;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if ((take >> e) & 1u) {
        if (p < (uint32_t)k) out[p] = jbase + 4 * i + e;
        ++p;
      }
    }
    pos += __shfl_sync(0xffffffffu, cinc, 31);
    tseen += __shfl_sync(0xffffffffu, tinc, 31);
  }
}

// The whole selection of one head by one CTA, from the fp32 scores in global
// memory: three radix levels (11, 11, 10 bits) on the order-preserving key,
// then an ordered compaction (each warp owns a contiguous run of keys).
__device__ void cta_select_full(const float *__restrict__ Srow, int N, int k,
                                int *__restrict__ out, uint32_t *rhist, FMisc *m,
                                uint32_t *status) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float4 *S4 = reinterpret_cast<const float4 *>(Srow);
  const int N4 = N >> 2;
  uint32_t prefix = 0, need = (uint32_t)k;
  uint64_t t_ge = 0;
  uint32_t tie_val = 0, n_ties = 0;
  bool exact = false;
  for (int level = 0; level < 3 && !exact; ++level) {
    const int shift = level == 0 ? 21 : (level == 1 ? 10 : 0);
    const int bits = level == 2 ? 10 : 11;
    const uint32_t nb = 1u << bits;
    __syncthreads();
    for (uint32_t i = tid; i < nb; i += kFThreads) rhist[i] = 0u;
    __syncthreads();
    for (int b = tid; b < N4; b += 4 * kFThreads) {
      float4 f[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = b + u * kFThreads;
        f[u] = i < N4 ? S4[i] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (b + u * kFThreads >= N4) continue;
        const uint32_t kv[4] = {order_key(f[u].x), order_key(f[u].y), order_key(f[u].z),
                                order_key(f[u].w)};
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (level == 0 || (kv[e] >> (shift + bits)) == prefix)
            atomicAdd(&rhist[(kv[e] >> shift) & (nb - 1u)], 1u);
      }
    }
    if (bits == 11) desc_boundary<2048>(rhist, need, m);
    else desc_boundary<1024>(rhist, need, m);
    const uint32_t bin = m->bnd[0];
    if (bin == kNone) {  // cannot happen for 1 <= k <= N
      if (tid == 0) raise_flag(status, FLAG_INTERNAL);
      return;
    }
    prefix = (prefix << bits) | bin;
    need -= m->bnd[1];
    if (m->bnd[2] == need) {
      t_ge = (uint64_t)prefix << shift;
      exact = true;
    }
  }
  if (!exact) {  // prefix is the k-th key itself, held by more keys than needed
    tie_val = prefix;
    t_ge = (uint64_t)prefix + 1;
    n_ties = need;
  }
  // ordered compaction: counts per warp, then the writes
  const int s0 = (int)((long long)N4 * warp / kFWarps);
  const int s1 = (int)((long long)N4 * (warp + 1) / kFWarps);
  uint32_t ge = 0, eq = 0;
  for (int b = s0; b < s1; b += 32) {
    const int i = b + lane;
    if (i < s1) {
      const float4 f = S4[i];
      const uint32_t kv[4] = {order_key(f.x), order_key(f.y), order_key(f.z), order_key(f.w)};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        ge += (uint64_t)kv[e] >= t_ge;
        eq += n_ties && kv[e] == tie_val;
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    ge += __shfl_xor_sync(0xffffffffu, ge, o);
    eq += __shfl_xor_sync(0xffffffffu, eq, o);
  }
  __syncthreads();
  if (lane == 0) {
    m->wge[warp] = ge;
    m->weq[warp] = eq;
  }
  __syncthreads();
  uint32_t pos = 0, tb = 0, total = 0, my_taken = 0;
  for (int w = 0; w < kFWarps; ++w) {
    const uint32_t taken = n_ties > tb ? min(n_ties - tb, m->weq[w]) : 0u;
    if (w < warp) pos += m->wge[w] + taken;
    if (w == warp) my_taken = taken;
    total += m->wge[w] + taken;
    tb += m->weq[w];
  }
  warp_ordered_write(
      [&](int i, bool in) -> uint4 {
        const float4 f = in ? S4[i] : make_float4(0.f, 0.f, 0.f, 0.f);
        return make_uint4(order_key(f.x), order_key(f.y), order_key(f.z), order_key(f.w));
      },
      s0, s1, 0, t_ge, tie_val, n_ties != 0, my_taken, pos, out, k);
  if (tid == 0 && total != (uint32_t)k) raise_flag(status, FLAG_INTERNAL);
}

template <typename T, int D>
__global__ void __launch_bounds__(kFThreads, 1)
    route_topk_fused_kernel(const T *__restrict__ q, const T *__restrict__ K,
                            float *__restrict__ S, int N, int kv_rows, int Hq, int Hkv,
                            int tph, int cpp,
                            float scale, int k, uint32_t *__restrict__ hist,
                            uint32_t *__restrict__ ctr, uint2 *__restrict__ meta,
                            uint32_t *__restrict__ gcand, int *__restrict__ idx,
                            uint32_t *status) {
  using C = ScoreCfg<T, D>;
  extern __shared__ __align__(128) unsigned char smem[];
  uint32_t *shist = reinterpret_cast<uint32_t *>(smem + kFShistOff);
  uint32_t *keys = reinterpret_cast<uint32_t *>(smem + kFKeysOff);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kFBarOff);
  uint64_t *empty = full + kScanStages;
  FMisc *m = reinterpret_cast<FMisc *>(smem + kFMiscOff);
  uint2 *lists = reinterpret_cast<uint2 *>(smem + kFListOff);
  uint32_t *cand = reinterpret_cast<uint32_t *>(smem + kFCandOff);
  uint32_t *rhist = reinterpret_cast<uint32_t *>(smem + kFRhistOff);
  uint32_t *seg = reinterpret_cast<uint32_t *>(smem + kFSegOff);
  uint32_t *seg_off = seg, *seg_cnt = seg + (kFusedMaxCtas + 1),
           *seg_def = seg + 2 * (kFusedMaxCtas + 1), *seg_ge = seg + 3 * (kFusedMaxCtas + 1),
           *seg_eq = seg + 4 * (kFusedMaxCtas + 1);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t lt = (1u << lane) - 1u;
  // CTA c scans share r of head bh: tiles [tl, th) of the head
  const int c = (int)blockIdx.x, bh = c / cpp, r = c % cpp, c0 = bh * cpp;
  const int tl = (int)((long long)r * tph / cpp), th = (int)((long long)(r + 1) * tph / cpp);
  const int jlo = tl * C::kStageKeys, jhi = min(N, th * C::kStageKeys);
  const int nkeys = jhi - jlo;  // a multiple of 4 (N % 4 == 0)
  uint32_t *gh = hist + (size_t)bh * kScanBins;
  uint32_t *hc = ctr + bh;

  for (int i = tid; i < kScanBins; i += kFThreads) shist[i] = 0u;
  if (tid == 0) {
    for (int s = 0; s < kScanStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kScanConsumerWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();
  grid_dep_wait();
  grid_dep_launch();

  // ---- scan: scores to S, keys and top-11-bit counts on chip -------------------
  {
    ScanOut o;
    o.S = S;
    o.hist = hist;
    o.shist = shist;
    o.keys = keys;
    o.key_off = -jlo;
    o.bits = nullptr;
    o.tau = nullptr;
    scan_tiles<T, D, 1>(q, K, N, kv_rows, Hq, Hkv, tph, (long long)bh * tph + tl, th - tl, bh,
                        scale,
                        smem, full, empty, o, status);
  }
  __syncthreads();  // the ring is free and every count is in shared memory
  for (int i = tid; i < kScanBins; i += kFThreads) {
    const uint32_t v = shist[i];
    if (v) atomicAdd(&gh[i], v);
  }
  __syncthreads();
  if (tid == 0) arrive(hc);

  // ---- A: boundary bin; ordered lists; publish the boundary-bin keys ---------
  if (tid == 0) m->ok = wait_count(hc, (uint32_t)cpp, status);
  __syncthreads();
  const bool okA = m->ok != 0;
  desc_boundary<kScanBins>(okA ? gh : shist /* unused when failed */, (uint32_t)k, m);
  const uint32_t b1 = m->bnd[0], above1 = m->bnd[1], cnt1 = m->bnd[2];
  const bool fast = okA && m->bnd[3] == (uint32_t)N && b1 != kNone;

  // warp w owns 4-key columns [sg0, sg1); lane l the contiguous run [l0, l1)
  const int n4 = nkeys >> 2;
  const int sg0 = (int)((long long)n4 * warp / kFWarps);
  const int sg1 = (int)((long long)n4 * (warp + 1) / kFWarps);
  const int l0 = sg0 + (sg1 - sg0) * lane / 32, l1 = sg0 + (sg1 - sg0) * (lane + 1) / 32;
  const uint4 *k4 = reinterpret_cast<const uint4 *>(keys);
  uint32_t nq = 0, nc = 0;  // this lane: keys >= b1, keys in b1
  if (fast) {
    for (int i = l0; i < l1; ++i) {
      const uint4 kk = k4[i];
      const uint32_t kv[4] = {kk.x, kk.y, kk.z, kk.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        nq += (kv[e] >> 21) >= b1;
        nc += (kv[e] >> 21) == b1;
      }
    }
  }
  const uint32_t qinc = warp_incl_scan(nq), cinc = warp_incl_scan(nc);
  const uint32_t wq = __shfl_sync(0xffffffffu, qinc, 31);
  const uint32_t wcn = __shfl_sync(0xffffffffu, cinc, 31);
  if (lane == 0) {
    m->wq[warp] = wq;
    m->wc[warp] = wcn;
  }
  __syncthreads();
  uint32_t coff = 0, ctot = 0, qtot = 0;
#pragma unroll
  for (int w = 0; w < kFWarps; ++w) {
    coff += w < warp ? m->wc[w] : 0u;
    ctot += m->wc[w];
    qtot += m->wq[w];
  }
  const bool over = ctot > (uint32_t)kFusedSegCap;
  const bool list_ok = wq <= (uint32_t)kFWarpList;
  uint2 *wl = lists + warp * kFWarpList;
  if (fast && (list_ok || !over)) {
    uint32_t pq = qinc - nq, pc = coff + cinc - nc;
    uint32_t *mycand = gcand + (size_t)c * kFusedSegCap;
    for (int i = l0; i < l1; ++i) {
      const uint4 kk = k4[i];
      const uint32_t kv[4] = {kk.x, kk.y, kk.z, kk.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t top = kv[e] >> 21;
        if (top >= b1) {
          if (list_ok) wl[pq] = make_uint2(kv[e], (uint32_t)(jlo + 4 * i + e));
          ++pq;
          if (top == b1) {
            if (!over) mycand[pc] = kv[e];
            ++pc;
          }
        }
      }
    }
  }
  if (tid == 0) meta[c] = make_uint2(ctot | (over ? 0x80000000u : 0u), qtot - ctot);
  __syncthreads();
  if (tid == 0) arrive(hc);

  // ---- B: refine on the published keys, ordered write -------------------------
  if (tid == 0) m->ok = okA ? wait_count(hc, 2u * cpp, status) : 0;
  __syncthreads();
  const bool okB = m->ok != 0;
  bool go = okB && fast;
  int *out = idx + (size_t)bh * k;
  if (go) {
    for (int i = tid; i < cpp; i += kFThreads) {
      const uint2 mt = meta[c0 + i];
      seg_cnt[i] = mt.x;
      seg_def[i] = mt.y;
      seg_ge[i] = 0u;
      seg_eq[i] = 0u;
    }
    __syncthreads();
    if (warp == 0) {
      uint32_t run = 0, bad = 0;
      for (int i0 = 0; i0 < cpp; i0 += 32) {
        const int i = i0 + lane;
        const uint32_t v = i < cpp ? seg_cnt[i] : 0u;
        bad |= v >> 31;
        const uint32_t cnt = v & 0x7FFFFFFFu;
        const uint32_t inc = warp_incl_scan(cnt);
        if (i < cpp) {
          seg_off[i] = run + inc - cnt;
          seg_cnt[i] = cnt;
        }
        run += __shfl_sync(0xffffffffu, inc, 31);
      }
      bad = __any_sync(0xffffffffu, bad != 0) ? 1u : 0u;
      if (lane == 0) {
        seg_off[cpp] = run;
        m->res[3] = bad || run > (uint32_t)kFCandMax;
      }
    }
    __syncthreads();
    go = m->res[3] == 0u;
  }
  // a group of tps threads per publishing CTA (tps a power of two)
  int tps = 1;
  while (tps * 2 * cpp <= kFThreads) tps *= 2;
  const int gseg = tid / tps, gsub = tid % tps;
  if (go) {
    const uint32_t M = seg_off[cpp];
    if (gseg < cpp) {
      const uint32_t cnt = seg_cnt[gseg], off = seg_off[gseg];
      const uint32_t *src = gcand + (size_t)(c0 + gseg) * kFusedSegCap;
      for (uint32_t j0 = gsub; j0 < cnt; j0 += 16u * tps) {
        uint32_t v[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const uint32_t j = j0 + u * tps;
          v[u] = j < cnt ? src[j] : 0u;
        }
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const uint32_t j = j0 + u * tps;
          if (j < cnt) cand[off + j] = v[u];
        }
      }
    }
    __syncthreads();
    // ---- threshold ------------------------------------------------------------
    uint64_t t_ge;
    uint32_t tie_val = 0, n_ties = 0;
    uint32_t need = (uint32_t)k - above1;
    if (cnt1 == need) {
      t_ge = (uint64_t)b1 << 21;
    } else {
      for (int i = tid; i < kScanBins; i += kFThreads) rhist[i] = 0u;
      __syncthreads();
      for (uint32_t i = tid; i < M; i += kFThreads)
        atomicAdd(&rhist[(cand[i] >> 10) & 2047u], 1u);
      desc_boundary<kScanBins>(rhist, need, m);
      const uint32_t b2 = m->bnd[0];
      need -= m->bnd[1];
      const uint32_t cnt2 = m->bnd[2];
      const uint32_t p2 = (b1 << 11) | b2;
      if (b2 == kNone) {
        if (tid == 0) raise_flag(status, FLAG_INTERNAL);
        t_ge = 0;
      } else if (cnt2 == need) {
        t_ge = (uint64_t)p2 << 10;
      } else if (cnt2 <= (uint32_t)kFFinMax) {
        // rank the few keys left exactly, within one warp, from registers
        if (tid == 0) m->nfin = 0;
        __syncthreads();
        for (uint32_t i = tid; i < M; i += kFThreads) {
          const uint32_t key = cand[i];
          if ((key >> 10) == p2) {
            const uint32_t f = atomicAdd(&m->nfin, 1u);
            if (f < (uint32_t)kFFinMax) m->fin[f] = key;
          }
        }
        __syncthreads();
        if (warp == 0) {
          const uint32_t nf = min(m->nfin, (uint32_t)kFFinMax);
          const uint32_t a0 = (uint32_t)lane < nf ? m->fin[lane] : 0u;
          const uint32_t a1 = (uint32_t)lane + 32u < nf ? m->fin[lane + 32] : 0u;
          uint32_t gt0 = 0, eq0 = 0, gt1 = 0, eq1 = 0;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int c2 = 0; c2 < 32; ++c2) {
              const uint32_t u = __shfl_sync(0xffffffffu, h ? a1 : a0, c2);
              const bool vu = (uint32_t)(h * 32 + c2) < nf;
              gt0 += vu && u > a0;
              eq0 += vu && u == a0;
              gt1 += vu && u > a1;
              eq1 += vu && u == a1;
            }
          }
          const bool f0 = (uint32_t)lane < nf && gt0 < need && need <= gt0 + eq0;
          const bool f1 = (uint32_t)lane + 32u < nf && gt1 < need && need <= gt1 + eq1;
          const uint32_t m0 = __ballot_sync(0xffffffffu, f0), m1 = __ballot_sync(0xffffffffu, f1);
          // every lane that found it holds the same value; take the first
          const bool use0 = m0 != 0u;
          const int src = use0 ? __ffs(m0) - 1 : (m1 ? __ffs(m1) - 1 : 0);
          const uint32_t bv = __shfl_sync(0xffffffffu, use0 ? a0 : a1, src);
          const uint32_t bg = __shfl_sync(0xffffffffu, use0 ? gt0 : gt1, src);
          const uint32_t be = __shfl_sync(0xffffffffu, use0 ? eq0 : eq1, src);
          if (lane == 0) {
            m->bnd[0] = bv;
            m->bnd[1] = bg;
            m->bnd[2] = be;
            if (!(m0 | m1)) raise_flag(status, FLAG_INTERNAL);
          }
        }
        __syncthreads();
        const uint32_t v = m->bnd[0];
        const uint32_t rest = need - m->bnd[1];
        if (m->bnd[2] == rest) {
          t_ge = v;
        } else {
          t_ge = (uint64_t)v + 1;
          tie_val = v;
          n_ties = rest;
        }
      } else {
        for (int i = tid; i < 1024; i += kFThreads) rhist[i] = 0u;
        __syncthreads();
        for (uint32_t i = tid; i < M; i += kFThreads) {
          const uint32_t key = cand[i];
          if ((key >> 10) == p2) atomicAdd(&rhist[key & 1023u], 1u);
        }
        desc_boundary<1024>(rhist, need, m);
        const uint32_t v = (p2 << 10) | m->bnd[0];
        need -= m->bnd[1];
        if (m->bnd[0] == kNone) {
          if (tid == 0) raise_flag(status, FLAG_INTERNAL);
          t_ge = 0;
        } else if (m->bnd[2] == need) {
          t_ge = v;
        } else {
          t_ge = (uint64_t)v + 1;
          tie_val = v;
          n_ties = need;
        }
      }
    }
    // ---- every publishing CTA's selected count, hence this CTA's offset -------
    {
      uint32_t ge = 0, eq = 0;
      if (gseg < cpp) {
        const uint32_t cnt = seg_cnt[gseg], off = seg_off[gseg];
        for (uint32_t j = gsub; j < cnt; j += tps) {
          const uint32_t key = cand[off + j];
          ge += (uint64_t)key >= t_ge;
          eq += n_ties && key == tie_val;
        }
      }
      const int g = tps < 32 ? tps : 32;
      for (int o = 1; o < g; o <<= 1) {
        ge += __shfl_xor_sync(0xffffffffu, ge, o);
        eq += __shfl_xor_sync(0xffffffffu, eq, o);
      }
      if (gseg < cpp && (lane & (g - 1)) == 0) {
        atomicAdd(&seg_ge[gseg], ge);
        atomicAdd(&seg_eq[gseg], eq);
      }
    }
    __syncthreads();
    if (warp == 0) {
      uint32_t sel_run = 0, tie_run = 0, pos = 0, allow = 0;
      for (int i0 = 0; i0 < cpp; i0 += 32) {
        const int i = i0 + lane;
        const uint32_t eq = i < cpp ? seg_eq[i] : 0u;
        const uint32_t inc = warp_incl_scan(eq);
        const uint32_t tb = tie_run + inc - eq;  // ties in earlier CTAs
        const uint32_t taken = n_ties > tb ? min(n_ties - tb, eq) : 0u;
        const uint32_t sel = i < cpp ? seg_def[i] + seg_ge[i] + taken : 0u;
        const uint32_t sinc = warp_incl_scan(sel);
        if (i == r) {
          pos = sel_run + sinc - sel;
          allow = taken;
        }
        sel_run += __shfl_sync(0xffffffffu, sinc, 31);
        tie_run += __shfl_sync(0xffffffffu, inc, 31);
      }
      pos = __reduce_add_sync(0xffffffffu, pos);
      allow = __reduce_add_sync(0xffffffffu, allow);
      if (lane == 0) {
        m->res[0] = pos;
        m->res[1] = allow;
        m->res[2] = sel_run;
        if (r == 0 && sel_run != (uint32_t)k) raise_flag(status, FLAG_INTERNAL);
      }
    }
    // ---- this CTA's keys: per-warp counts, then the ordered writes ------------
    uint32_t ge = 0, eq = 0;
    if (list_ok) {
      for (uint32_t i = lane; i < wq; i += 32) {
        const uint32_t key = wl[i].x;
        ge += (uint64_t)key >= t_ge;
        eq += n_ties && key == tie_val;
      }
    } else {
      for (int i = sg0 + lane; i < sg1; i += 32) {
        const uint4 kk = k4[i];
        const uint32_t kv[4] = {kk.x, kk.y, kk.z, kk.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          ge += (uint64_t)kv[e] >= t_ge;
          eq += n_ties && kv[e] == tie_val;
        }
      }
    }
    ge = __reduce_add_sync(0xffffffffu, ge);
    eq = __reduce_add_sync(0xffffffffu, eq);
    if (lane == 0) {
      m->wge[warp] = ge;
      m->weq[warp] = eq;
    }
    __syncthreads();
    uint32_t pos = m->res[0];
    const uint32_t allow = m->res[1];
    uint32_t tb = 0;
    for (int w = 0; w < warp; ++w) {
      const uint32_t tk = allow > tb ? min(allow - tb, m->weq[w]) : 0u;
      pos += m->wge[w] + tk;
      tb += m->weq[w];
    }
    const uint32_t my_allow = allow > tb ? min(allow - tb, eq) : 0u;
    if (list_ok) {
      uint32_t tseen = 0;
      for (uint32_t i0 = 0; i0 < wq; i0 += 32) {
        const uint32_t i = i0 + lane;
        const uint2 ent = i < wq ? wl[i] : make_uint2(0u, 0u);
        const bool g = i < wq && (uint64_t)ent.x >= t_ge;
        const bool t = i < wq && n_ties && ent.x == tie_val;
        const uint32_t tm = __ballot_sync(0xffffffffu, t);
        const bool take = g || (t && tseen + __popc(tm & lt) < my_allow);
        const uint32_t mm = __ballot_sync(0xffffffffu, take);
        if (take) {
          const uint32_t p = pos + __popc(mm & lt);
          if (p < (uint32_t)k) out[p] = (int)ent.y;
        }
        pos += __popc(mm);
        tseen += __popc(tm);
      }
    } else {  // the list overflowed: walk the keys again
      warp_ordered_write(
          [&](int i, bool in) -> uint4 { return in ? k4[i] : make_uint4(0u, 0u, 0u, 0u); },
          sg0, sg1, jlo, t_ge, tie_val, n_ties != 0, my_allow, pos, out, k);
    }
  } else if (okB && r == 0) {
    // the head's first CTA selects alone from the scores in global memory
    cta_select_full(S + (size_t)bh * N, N, k, out, rhist, m, status);
  }
  // ---- leave: the first CTA clears the histogram row; count departures --------
  if (r == 0 && okB)
    for (int i = tid; i < kScanBins; i += kFThreads) gh[i] = 0u;
  __syncthreads();
  if (tid == 0) {
    const uint32_t old = atomicAdd(hc, 1u);
    if (old == 3u * cpp - 1u) {
      __threadfence();
      atomicExch(hc, 0u);
    }
  }
}

template <typename T, int D>
cudaError_t launch_fused_t(const Shape &s, const void *q, const void *K, int k, float *S,
                           uint32_t *hist, uint32_t *ctr, void *seg_area, int *idx,
                           uint32_t *status, cudaStream_t st) {
  using C = ScoreCfg<T, D>;
  DeviceInfo di;
  cudaError_t e = device_info(&di);
  if (e != cudaSuccess) return e;
  // a whole number of CTAs per head, at most one CTA per SM
  const int tph = (s.N + C::kStageKeys - 1) / C::kStageKeys;
  if (s.BH() > di.sm_count || s.BH() > kFusedMaxHeads) return cudaErrorNotSupported;
  int cpp = di.sm_count / s.BH();
  cpp = cpp < tph ? cpp : tph;
  const long long grid = (long long)s.BH() * cpp;
  if (grid > kFusedMaxCtas) return cudaErrorNotSupported;
  const long long per = (tph + cpp - 1) / cpp;  // most tiles a CTA scans
  if (per * C::kStageKeys > kFMaxKeys) return cudaErrorNotSupported;
  if (kFSmem > di.max_smem_optin) return cudaErrorNotSupported;
  auto kern = route_topk_fused_kernel<T, D>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kFSmem);
  if (e != cudaSuccess) return e;
  const float scale = (float)(1.0 / __builtin_sqrt((double)D));
  uint2 *meta = static_cast<uint2 *>(seg_area);
  uint32_t *gcand = reinterpret_cast<uint32_t *>(static_cast<char *>(seg_area) +
                                                 kFusedMetaBytes);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3(kFThreads, 1, 1);
  cfg.dynamicSmemBytes = kFSmem;
  cfg.stream = st;
  cudaLaunchAttribute attrs[2];
  cfg.attrs = attrs;
  cfg.numAttrs = 0;
  if (cooperative_forced()) {
    attrs[0].id = cudaLaunchAttributeCooperative;
    attrs[0].val.cooperative = 1;
    cfg.numAttrs = 1;
  }
  add_pdl_attr(cfg, attrs);
  e = cudaLaunchKernelEx(&cfg, kern, static_cast<const T *>(q), static_cast<const T *>(K), S,
                         s.N, s.Ncap, s.Hq, s.Hkv, tph, cpp, scale, k, hist, ctr, meta, gcand,
                         idx,
                         status);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

bool fused_route_enabled() {
  const char *v = getenv("SPARSE_DECODE_FUSED_ROUTE");
  return v && v[0] == '1';
}

cudaError_t launch_route_topk_fused(const Shape &s, const void *q, const void *K, int k,
                                    float *S, uint32_t *hist, uint32_t *ctr, void *seg_area,
                                    int *idx, uint32_t *status, cudaStream_t st) {
  if (!fused_route_enabled() || !hist || !ctr || !seg_area || (s.N & 3) != 0 || k < 1 ||
      k > s.N)
    return cudaErrorNotSupported;
  if (s.dtype == 1) {
    if (s.d == 128)
      return launch_fused_t<__nv_bfloat16, 128>(s, q, K, k, S, hist, ctr, seg_area, idx,
                                                status, st);
    return launch_fused_t<__nv_bfloat16, 64>(s, q, K, k, S, hist, ctr, seg_area, idx, status,
                                             st);
  }
  if (s.d == 128)
    return launch_fused_t<float, 128>(s, q, K, k, S, hist, ctr, seg_area, idx, status, st);
  return launch_fused_t<float, 64>(s, q, K, k, S, hist, ctr, seg_area, idx, status, st);
}

}  // namespace sd
