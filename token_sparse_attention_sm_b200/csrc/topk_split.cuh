// topk_split.cuh -- exact top-k of one (sequence, KV head) from what the
// routing scan leaves (the fp32 score row and the histogram of the top 11
// bits of every score), split over the CTAs of a thread-block cluster.
//
// The set is the k highest scores, ties to the lower key index (CLSA
// article, section 研究の背景と課題).  Its positions follow key order.  CTA r
// of a head's cluster of C owns one contiguous run of the row's 32-key words,
// [r nw / C, (r + 1) nw / C), and ends up holding the selected keys of its
// run, in ascending order, together with their positions in the whole set:
// the keys of CTAs 0..r-1 come first.
//
//  1. The histogram gives the boundary bin b1 where the descending count
//     reaches k: every key above b1 is in, every key below it out.  Every
//     CTA reads it.
//  2. Each CTA reads its run once (16-byte loads, four keys per lane): the
//     keys above b1 go into an on-chip bitmap of the run, the keys in b1 onto
//     an on-chip list whose order keys the peers may read.
//  3. One cluster barrier.  Every CTA reads the peers' counts and copies all
//     of their lists through distributed shared memory: the whole boundary
//     bin, a few thousand keys, lands in every CTA.
//  4. Every CTA pins the k-th value inside the bin with the next 11 bits and,
//     if needed, the last 10 (histograms on chip), then counts per peer the
//     listed keys above it and equal to it.  Keys equal to the k-th value go
//     to the lowest indices, which live in the lowest-ranked CTAs first, so
//     every CTA can tell how many each CTA takes -- hence its own count and
//     the position of its first key -- without a second exchange.
//  5. Each CTA marks its own boundary keys in the run's bitmap, and a block
//     scan over the run's words hands out the positions.
// The cluster agrees on the path without talking: the fast path needs a
// complete histogram, runs of at most kTsMaxWords words, lists within
// capacity, list totals equal to the histogram's counts and at most
// `max_own` keys in every run -- all read from the same data by every CTA.
// Otherwise every CTA runs the exact streaming select over the whole row
// (three radix levels, each a pass over S, then one ordered pass) and takes
// an equal share of the positions; that raises the informational
// FLAG_SLOW_SELECT.
#pragma once

#include "common.cuh"

namespace sd {
namespace {

constexpr int kTkThreads = 512;
constexpr int kTkWarps = kTkThreads / 32;
constexpr int kTsMaxSplits = 16;    // CTAs in a head's cluster
constexpr int kTsMaxWords = 4096;   // 32-key words of one CTA's run (131072 keys)
constexpr int kTsOwnCap = 2048;     // boundary-bin keys one CTA lists
constexpr int kTsGatherCap = 8192;  // boundary-bin keys of the head gathered on chip

// Shared-memory scratch of ts_select, free again when it returns: the run's
// bitmap | the own list's key indices | the gathered keys | level-2 and
// level-3 histograms.
__host__ __device__ constexpr size_t ts_scratch_bytes() {
  return (size_t)(kTsMaxWords + kTsOwnCap + kTsGatherCap + 2048 + 1024) * 4;
}

// Block-level bookkeeping, in shared memory.
struct TkSmall {
  uint32_t warp_buf[33];
  uint32_t bnd[3];  // boundary bin, keys above it, keys in it
};

// What a CTA shows its peers: it must stay in place until the caller's last
// cluster barrier (peers read it after the select's barrier).
struct TsShow {
  uint32_t n_above;  // keys of the run above the boundary bin
  uint32_t n_list;   // keys of the run in the boundary bin (listed up to kTsOwnCap)
  uint32_t pad[2];
  uint32_t lkey[kTsOwnCap];  // their order keys
};

// Per-CTA bookkeeping of ts_select, in shared memory.
struct TsBook {
  uint32_t cnt[kTsMaxSplits], seg[kTsMaxSplits], above[kTsMaxSplits];
  uint32_t gt[kTsMaxSplits], eq[kTsMaxSplits];
  uint32_t part_lo[kTsMaxSplits + 1];  // fast path: CTA s holds positions [part_lo[s], part_lo[s+1])
  uint32_t nab, nlist, ok, own_take, verdict;
};

// Exclusive prefix sum of x over the 512 threads; *total = the block sum.
// Every thread must call it (it contains barriers).
__device__ __forceinline__ uint32_t tk_scan(uint32_t x, TkSmall *sm, uint32_t *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t inc = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) sm->warp_buf[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    const uint32_t w = lane < kTkWarps ? sm->warp_buf[lane] : 0u;
    uint32_t wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    if (lane < kTkWarps) sm->warp_buf[lane] = wi - w;
    if (lane == kTkWarps - 1) sm->warp_buf[32] = wi;
  }
  __syncthreads();
  const uint32_t r = sm->warp_buf[warp] + inc - x;
  *total = sm->warp_buf[32];
  __syncthreads();
  return r;
}

// The bin of a histogram of NB bins, read highest first, where the
// descending count reaches need: sm->bnd = {bin, keys above it, keys in it},
// or bnd[0] = ~0 when the histogram holds fewer than need keys; *total = its
// sum.  This thread's bins come already loaded: c[e] = bin NB - 1 -
// (NB / 512 * t + e) (so the loads can be issued ahead of other work).
template <int NB>
__device__ __forceinline__ void tk_boundary_of(const uint32_t (&c)[NB / kTkThreads], uint32_t need,
                                               TkSmall *sm, uint32_t *total) {
  constexpr int BPT = NB / kTkThreads;
  const int t = threadIdx.x;
  uint32_t sum = 0;
#pragma unroll
  for (int e = 0; e < BPT; ++e) sum += c[e];
  if (t == 0) sm->bnd[0] = ~0u;
  uint32_t above = tk_scan(sum, sm, total);  // its barriers order the write above
  if (above < need && above + sum >= need) {
#pragma unroll
    for (int e = 0; e < BPT; ++e) {
      if (above + c[e] >= need) {
        sm->bnd[0] = (uint32_t)(NB - 1 - (BPT * t + e));
        sm->bnd[1] = above;
        sm->bnd[2] = c[e];
        break;
      }
      above += c[e];
    }
  }
  __syncthreads();
}

// The same, reading histogram h.
template <int NB>
__device__ __forceinline__ void tk_boundary(const uint32_t *h, uint32_t need, TkSmall *sm, uint32_t *total) {
  constexpr int BPT = NB / kTkThreads;
  uint32_t c[BPT];
#pragma unroll
  for (int e = 0; e < BPT; ++e) c[e] = h[NB - 1 - (BPT * threadIdx.x + e)];
  tk_boundary_of<NB>(c, need, sm, total);
}

// Where the k-th key lies: every key with key >= t_ge is selected, plus the
// n_ties lowest-index keys equal to tie_val.
struct TkCut {
  uint64_t t_ge;
  uint32_t tie_val, n_ties;
};

// Exact streaming selection over the score row (any N): levels 2 and 3 of
// the radix select as passes over S, level 1 from the histogram when it is
// complete (hist_ok) or from one more pass.  h: 2048 words of scratch.
__device__ __forceinline__ TkCut tk_stream_cut(const float *__restrict__ S, int N, uint32_t k,
                               const uint32_t *__restrict__ hist, bool hist_ok, uint32_t *h,
                               TkSmall *sm) {
  const int tid = threadIdx.x;
  uint32_t tot;
  TkCut cut{0, 0, 0};
  if (!hist_ok) {
    for (int b = tid; b < 2048; b += kTkThreads) h[b] = 0u;
    __syncthreads();
    for (int j = tid; j < N; j += kTkThreads) sh_red_add(&h[order_key(S[j]) >> 21], 1u);
    __syncthreads();
    tk_boundary<2048>(h, k, sm, &tot);
  } else {
    tk_boundary<2048>(hist, k, sm, &tot);
  }
  const uint32_t b1 = sm->bnd[0];
  uint32_t need = k - sm->bnd[1];
  if (sm->bnd[2] == need) {
    cut.t_ge = (uint64_t)b1 << 21;
    return cut;
  }
  __syncthreads();  // every thread has read bnd
  for (int b = tid; b < 2048; b += kTkThreads) h[b] = 0u;
  __syncthreads();
  for (int j = tid; j < N; j += kTkThreads) {
    const uint32_t key = order_key(S[j]);
    if ((key >> 21) == b1) sh_red_add(&h[(key >> 10) & 2047u], 1u);
  }
  __syncthreads();
  tk_boundary<2048>(h, need, sm, &tot);
  const uint32_t p2 = (b1 << 11) | sm->bnd[0];
  need -= sm->bnd[1];
  if (sm->bnd[2] == need) {
    cut.t_ge = (uint64_t)p2 << 10;
    return cut;
  }
  __syncthreads();
  for (int b = tid; b < 1024; b += kTkThreads) h[b] = 0u;
  __syncthreads();
  for (int j = tid; j < N; j += kTkThreads) {
    const uint32_t key = order_key(S[j]);
    if ((key >> 10) == p2) sh_red_add(&h[key & 1023u], 1u);
  }
  __syncthreads();
  tk_boundary<1024>(h, need, sm, &tot);
  const uint32_t v = (p2 << 10) | sm->bnd[0];
  need -= sm->bnd[1];
  if (sm->bnd[2] == need) {
    cut.t_ge = v;
  } else {
    cut.t_ge = (uint64_t)v + 1;
    cut.tie_val = v;
    cut.n_ties = need;
  }
  return cut;
}

// Ordered pass over the score row: emits every key >= t_ge and the first
// n_ties keys equal to tie_val, in index order.  Returns the number emitted.
template <typename Emit>
__device__ __forceinline__ uint32_t tk_stream_emit(const float *__restrict__ S, int N, TkCut cut, TkSmall *sm,
                                   Emit &emit) {
  const int tid = threadIdx.x;
  uint32_t pos_base = 0, tie_base = 0;
  for (int c0 = 0; c0 < N; c0 += 4 * kTkThreads) {
    uint32_t key[4];
    bool ge[4], eq[4];
    uint32_t neq = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = c0 + 4 * tid + e;
      const bool in = j < N;
      key[e] = in ? order_key(S[j]) : 0u;
      ge[e] = in && (uint64_t)key[e] >= cut.t_ge;
      eq[e] = in && cut.n_ties && key[e] == cut.tie_val;
      neq += eq[e];
    }
    uint32_t tie_tot, take_tot;
    uint32_t tie_rank = tie_base + tk_scan(neq, sm, &tie_tot);
    bool take[4];
    uint32_t ntake = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      take[e] = ge[e] || (eq[e] && tie_rank < cut.n_ties);
      tie_rank += eq[e];
      ntake += take[e];
    }
    uint32_t pos = pos_base + tk_scan(ntake, sm, &take_tot);
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (take[e]) emit(pos++, (uint32_t)(c0 + 4 * tid + e));
    pos_base += take_tot;
    tie_base += tie_tot;
  }
  return pos_base;
}

// Ordered emission of the set bits of a bitmap of nwords words (on chip or
// in global memory): thread t owns a contiguous run of words.  emit(pos, j)
// is called for the positions in [lo, hi) (a thread whose run lies outside
// does not walk its words).  Returns the number of set bits.
template <typename Emit>
__device__ __forceinline__ uint32_t tk_bitmap_emit(const uint32_t *bits, int nwords, TkSmall *sm,
                                                   Emit &emit, uint32_t lo, uint32_t hi) {
  const int tid = threadIdx.x;
  const int per = (nwords + kTkThreads - 1) / kTkThreads;
  const int w0 = min(nwords, tid * per), w1 = min(nwords, w0 + per);
  uint32_t n = 0;
  for (int w = w0; w < w1; ++w) n += __popc(bits[w]);
  uint32_t total;
  uint32_t pos = tk_scan(n, sm, &total);
  if (pos < hi && pos + n > lo) {
    for (int w = w0; w < w1; ++w) {
      uint32_t m = bits[w];
      while (m) {
        const int b = __ffs(m) - 1;
        m &= m - 1;
        if (pos >= lo && pos < hi) emit(pos, (uint32_t)(32 * w + b));
        ++pos;
      }
    }
  }
  return total;
}

// This CTA's part of the set: positions [lo, lo + n).
struct TsOut {
  uint32_t lo, n;
  bool split;  // fast path: the parts follow the runs (bk->part_lo has them all);
               // else equal shares of ceil(k / nsplit) positions
};

// The exact top-k of one head (see the file comment), as CTA `rank` of
// `nsplit` (nsplit == 1: no cluster).  S: the head's score row; hist: its
// histogram (complete when it sums to N); scratch: ts_scratch_bytes() of
// shared memory; show, bk, sm: this CTA's shared structures.  max_own: the
// most keys the caller can take in one CTA on the fast path (the fallback's
// equal share, ceil(k / nsplit), must not exceed it).  Calls emit(i, pos, j)
// for the CTA's i-th key j at position pos of the set (i = pos - lo).  On the
// fast path (split) the CTA's part is its run's keys and bk->part_lo holds
// every CTA's first position (and k after the last).  Every
// thread of every CTA of the cluster must call it; it contains one cluster
// barrier (on the fast path, which the whole cluster takes or leaves).
template <typename Emit>
__device__ __forceinline__ TsOut ts_select(const float *__restrict__ S, int N, uint32_t k,
                                           const uint32_t *__restrict__ hist, int rank,
                                           int nsplit, uint32_t max_own, unsigned char *scratch,
                                           TsShow *show, TsBook *bk, TkSmall *sm,
                                           uint32_t *status, Emit &emit) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t *bits = reinterpret_cast<uint32_t *>(scratch);  // the run's words
  uint32_t *lidx = bits + kTsMaxWords;                     // own list: key indices
  uint32_t *gk = lidx + kTsOwnCap;                         // gathered order keys
  uint32_t *h2 = gk + kTsGatherCap;
  uint32_t *h3 = h2 + 2048;
  const int nw = (N + 31) / 32;
  const int w_lo = (int)((long long)rank * nw / nsplit);
  const int w_hi = (int)((long long)(rank + 1) * nw / nsplit);
  const int ow = w_hi - w_lo;

  // The run is read in blocks of 128 keys, lane l of a warp taking keys
  // 4l .. 4l+3 of a block (one 16-byte load when the row is 16-byte aligned,
  // which N % 4 == 0 makes true of every row).  The first blocks are loaded
  // before the histogram is read (the two latencies overlap).
  const int j_lo = 32 * w_lo, j_end = min(N, 32 * w_hi);
  const int nblk = (ow + 3) / 4;
  const bool vec = (N & 3) == 0;
  constexpr int U = 4;  // blocks a warp has in flight
  float sc[U][4];
  auto load_blocks = [&](int b0) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int j0 = j_lo + 128 * (b0 + u * kTkWarps) + 4 * lane;
      if (vec) {
        float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
        if (j0 < j_end) f = *reinterpret_cast<const float4 *>(S + j0);
        sc[u][0] = f.x;
        sc[u][1] = f.y;
        sc[u][2] = f.z;
        sc[u][3] = f.w;
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) sc[u][e] = j0 + e < j_end ? S[j0 + e] : 0.f;
      }
    }
  };
  // the histogram's bins first (the boundary needs them first), then the
  // run's first blocks
  uint32_t hb[2048 / kTkThreads];
#pragma unroll
  for (int e = 0; e < 2048 / kTkThreads; ++e) hb[e] = hist[2047 - (2048 / kTkThreads * tid + e)];
  load_blocks(warp);

  // ---- 1. the boundary bin ------------------------------------------------------
  uint32_t tot;
  tk_boundary_of<2048>(hb, k, sm, &tot);
  const uint32_t b1 = sm->bnd[0], above1 = sm->bnd[1], cb1 = sm->bnd[2];
  bool hist_ok = tot == (uint32_t)N && b1 != ~0u;
  bool fast = hist_ok && (nw + nsplit - 1) / nsplit <= kTsMaxWords;
  for (int i = tid; i < 2048 + 1024; i += kTkThreads) h2[i] = 0u;  // h3 follows h2
  if (tid == 0) {
    bk->nab = 0u;
    bk->nlist = 0u;
  }
  __syncthreads();

  if (fast) {
    // ---- 2. classify the run ----------------------------------------------------
    uint32_t nab = 0;
    for (int b0 = warp; b0 < nblk; b0 += U * kTkWarps) {
      if (b0 != warp) load_blocks(b0);
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int blk = b0 + u * kTkWarps;
        if (blk >= nblk) break;  // warp-uniform
        const int j0 = j_lo + 128 * blk + 4 * lane;
        uint32_t key[4], un = 0, inn = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          key[e] = order_key(sc[u][e]);
          const bool valid = j0 + e < j_end;
          const uint32_t bin = key[e] >> 21;
          un |= (valid && bin > b1) ? 1u << e : 0u;
          inn |= (valid && bin == b1) ? 1u << e : 0u;
        }
        // the run's bitmap word of keys 32 g .. 32 g + 31 of the block is the
        // nibbles of lanes 8 g .. 8 g + 7: one reduction per group of 8 lanes,
        // one plain store
        const uint32_t grp8 = 0xffu << (lane & 24);
        const uint32_t word = __reduce_or_sync(grp8, un << (j0 & 31));
        if ((lane & 7) == 0 && j0 < j_end) bits[(j0 - j_lo) >> 5] = word;
        nab += (uint32_t)__popc(un);
        // boundary-bin keys join the list, ordered by nibble bit then lane:
        // four ballots give every entry its slot, one shared counter update
        // per warp gives the warp's base
        uint32_t m[4], tot4 = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          m[e] = __ballot_sync(0xffffffffu, (inn >> e) & 1u);
          tot4 += (uint32_t)__popc(m[e]);
        }
        if (tot4) {
          uint32_t base = 0;
          if (lane == 0) base = sh_atom_add(&bk->nlist, tot4);
          base = __shfl_sync(0xffffffffu, base, 0);
          const uint32_t lt = (1u << lane) - 1u;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            if ((m[e] >> lane) & 1u) {
              const uint32_t slot = base + (uint32_t)__popc(m[e] & lt);
              if (slot < (uint32_t)kTsOwnCap) {
                show->lkey[slot] = key[e];
                lidx[slot] = (uint32_t)(j0 + e);
              }
            }
            base += (uint32_t)__popc(m[e]);
          }
        }
      }
    }
    nab = __reduce_add_sync(0xffffffffu, nab);
    if (lane == 0 && nab) sh_red_add(&bk->nab, nab);
    __syncthreads();
    if (tid == 0) {
      show->n_above = bk->nab;
      show->n_list = bk->nlist;
    }

    // ---- 3. the peers' counts and lists -------------------------------------------
    if (nsplit > 1)
      cluster_sync_all();
    else
      __syncthreads();
    if (warp == 0) {
      uint32_t na = 0, nl = 0;
      if (lane < nsplit) {
        if (lane == rank) {
          na = show->n_above;
          nl = show->n_list;
        } else {
          na = cl_ld_u32(cl_addr(&show->n_above, lane));
          nl = cl_ld_u32(cl_addr(&show->n_list, lane));
        }
      }
      const bool over = __any_sync(0xffffffffu, nl > (uint32_t)kTsOwnCap);
      uint32_t inc = nl;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
      }
      const uint32_t total = __shfl_sync(0xffffffffu, inc, 31);
      const uint32_t sum_above = __reduce_add_sync(0xffffffffu, na);
      if (lane < kTsMaxSplits) {
        bk->cnt[lane] = nl;
        bk->seg[lane] = inc - nl;
        bk->above[lane] = na;
      }
      // ok: 1 fast path, 2 the lists disagree with the histogram, 0 over capacity
      if (lane == 0)
        bk->ok = (total != cb1 || sum_above != above1)
                     ? 2u
                     : ((over || total > (uint32_t)kTsGatherCap) ? 0u : 1u);
    }
    __syncthreads();
    fast = bk->ok == 1u;
    if (bk->ok == 2u) hist_ok = false;
  }

  if (fast) {
    // ---- 4a. gather the bin's keys (a warp per peer), level-2 histogram ------------
    for (int s2 = warp; s2 < nsplit; s2 += kTkWarps) {
      const uint32_t off = bk->seg[s2], n = bk->cnt[s2];
      const uint32_t src = cl_addr(show->lkey, s2);
      for (uint32_t i0 = 0; i0 < n; i0 += 4 * 32) {
        uint32_t key[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t i = i0 + (uint32_t)(u * 32 + lane);
          key[u] = i < n ? (s2 == rank ? show->lkey[i] : cl_ld_u32(src + 4u * i)) : 0u;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t i = i0 + (uint32_t)(u * 32 + lane);
          if (i < n) {
            gk[off + i] = key[u];
            sh_red_add(&h2[(key[u] >> 10) & 2047u], 1u);
          }
        }
      }
    }
    __syncthreads();

    // ---- 4b. the k-th value -------------------------------------------------------
    const uint32_t need = k - above1;  // keys still to take from bin b1 (>= 1)
    tk_boundary<2048>(h2, need, sm, &tot);
    const uint32_t p2 = (b1 << 11) | sm->bnd[0];
    const uint32_t need2 = need - sm->bnd[1];
    TkCut cut{0, 0, 0};
    if (sm->bnd[2] == need2) {
      cut.t_ge = (uint64_t)p2 << 10;
    } else {
      for (uint32_t p = tid; p < cb1; p += kTkThreads) {
        const uint32_t key = gk[p];
        if ((key >> 10) == p2) sh_red_add(&h3[key & 1023u], 1u);
      }
      __syncthreads();
      tk_boundary<1024>(h3, need2, sm, &tot);
      const uint32_t v = (p2 << 10) | sm->bnd[0];
      const uint32_t need3 = need2 - sm->bnd[1];
      if (sm->bnd[2] == need3) {
        cut.t_ge = v;
      } else {
        cut.t_ge = (uint64_t)v + 1;
        cut.tie_val = v;
        cut.n_ties = need3;
      }
    }

    // ---- 4c. per peer: listed keys above the cut and equal to the tie value ------------
    for (int s = warp; s < nsplit; s += kTkWarps) {
      const uint32_t off = bk->seg[s], n = bk->cnt[s];
      uint32_t g = 0, e = 0;
      for (uint32_t i = lane; i < n; i += 32) {
        const uint32_t key = gk[off + i];
        g += (uint64_t)key >= cut.t_ge ? 1u : 0u;
        e += (cut.n_ties && key == cut.tie_val) ? 1u : 0u;
      }
      g = __reduce_add_sync(0xffffffffu, g);
      e = __reduce_add_sync(0xffffffffu, e);
      if (lane == 0) {
        bk->gt[s] = g;
        bk->eq[s] = e;
      }
    }
    __syncthreads();
    // every CTA's part: lane s of warp 0 takes CTA s (ties go to the lowest
    // indices, i.e. to the lowest-ranked CTAs first)
    if (warp == 0) {
      const uint32_t e = lane < nsplit ? bk->eq[lane] : 0u;
      uint32_t ie = e;  // inclusive scan of the tie counts
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, ie, o);
        if (lane >= o) ie += y;
      }
      const uint32_t before = ie - e;
      const uint32_t t = cut.n_ties > before ? min(cut.n_ties - before, e) : 0u;
      const uint32_t ns = lane < nsplit ? bk->above[lane] + bk->gt[lane] + t : 0u;
      uint32_t in = ns;  // inclusive scan of the part sizes
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, in, o);
        if (lane >= o) in += y;
      }
      if (lane <= nsplit) bk->part_lo[lane] = in - ns;  // lane nsplit: the total
      if (lane == rank) bk->own_take = t;
      const uint32_t most = __reduce_max_sync(0xffffffffu, ns);
      const uint32_t sum = __shfl_sync(0xffffffffu, in, 31);
      if (lane == 0) {
        if (sum != k) raise_flag(status, FLAG_INTERNAL);
        bk->verdict = (sum == k && most <= max_own) ? 1u : 0u;
      }
    }
    __syncthreads();
    const uint32_t pre = bk->part_lo[rank], mine = bk->part_lo[rank + 1] - pre;
    const uint32_t own_take = bk->own_take;
    fast = bk->verdict != 0;

    if (fast) {
      // ---- 5. own boundary keys into the run's bitmap, then positions -------------------
      const uint32_t nl = show->n_list;  // <= kTsOwnCap on this path
      const uint32_t own_eq = bk->eq[rank];
      const bool all_ties = own_take == own_eq;
      for (uint32_t i = tid; i < nl; i += kTkThreads) {
        const uint32_t key = show->lkey[i], j = lidx[i];
        if ((uint64_t)key >= cut.t_ge || (all_ties && cut.n_ties && key == cut.tie_val))
          sh_red_or(&bits[(j >> 5) - w_lo], 1u << (j & 31));
      }
      if (!all_ties) {
        // only the own_take lowest-index keys of the run equal to the tie
        // value: their bitmap (over the gathered keys, read for the last
        // time above), ranked by a block scan in index order
        uint32_t *tb = gk;
        for (int w = tid; w < ow; w += kTkThreads) tb[w] = 0u;
        __syncthreads();
        for (uint32_t i = tid; i < nl; i += kTkThreads) {
          const uint32_t j = lidx[i];
          if (show->lkey[i] == cut.tie_val) sh_red_or(&tb[(j >> 5) - w_lo], 1u << (j & 31));
        }
        __syncthreads();
        const int per = (ow + kTkThreads - 1) / kTkThreads;
        const int a0 = min(ow, tid * per), a1 = min(ow, a0 + per);
        uint32_t n = 0;
        for (int w = a0; w < a1; ++w) n += __popc(tb[w]);
        uint32_t tt;
        uint32_t r = tk_scan(n, sm, &tt);
        for (int w = a0; w < a1 && r < own_take; ++w) {
          uint32_t m = tb[w];
          while (m && r < own_take) {
            const int b = __ffs(m) - 1;
            m &= m - 1;
            sh_red_or(&bits[w], 1u << b);
            ++r;
          }
        }
      }
      __syncthreads();
      auto em = [&](uint32_t i, uint32_t jl) { emit(i, pre + i, 32u * (uint32_t)w_lo + jl); };
      const uint32_t n = tk_bitmap_emit(bits, ow, sm, em, 0u, 0xffffffffu);
      if (tid == 0 && n != mine) raise_flag(status, FLAG_INTERNAL);
      return {pre, mine, true};
    }
  }

  // ---- fallback: exact streaming select, an equal share of the positions ------------
  if (tid == 0) raise_flag(status, FLAG_SLOW_SELECT);
  __syncthreads();
  const TkCut cut = tk_stream_cut(S, N, k, hist, hist_ok, h2, sm);
  __syncthreads();
  const uint32_t per = (k + (uint32_t)nsplit - 1) / (uint32_t)nsplit;
  const uint32_t lo = min(k, (uint32_t)rank * per), hi = min(k, lo + per);
  auto em = [&](uint32_t pos, uint32_t j) {
    if (pos >= lo && pos < hi) emit(pos - lo, pos, j);
  };
  tk_stream_emit(S, N, cut, sm, em);
  return {lo, hi - lo, false};
}

}  // namespace
}  // namespace sd
