// topk_cand.cuh -- exact top-k of one (sequence, KV head) by one CTA of 512
// threads, from what the routing scan leaves: the head's histogram of the
// top 11 score bits, the fp32 score row, and (top-k routing) the candidate
// lists of route_cand.cuh.
//
// The set is the k highest scores, ties to the lower key index (CLSA
// article, section 研究の背景と課題), handed out in ascending key order through
// a callback emit(pos, j): key j is the pos-th smallest index of the set.
//
// Fast path (every step of the usual case works on a few thousand keys):
//  1. The histogram gives the boundary bin b1 where the descending count
//     reaches k: every key above b1 is in, every key below it out.
//  2. One pass over the candidates (the lists, or the whole score row when
//     there are none) sets the bits of the keys above b1 in an on-chip
//     bitmap of the head, keeps the keys inside b1 in an on-chip list, and
//     counts their next 11 bits.  The candidates must hold exactly the
//     histogram's number of keys at or above b1; if not (the sample's bound
//     was too high, a list overflowed), the exact streaming path below runs.
//  3. The next 11 bits, and if needed the last 10, pin the k-th key value;
//     keys of b1 above it join the bitmap, and keys equal to it are ranked by
//     index (the lower ones win).
//  4. A block scan over the bitmap's word counts gives every selected key
//     its position.
// Streaming path (any N, any data): the same three radix levels, each a
// pass over the score row, then one ordered pass that writes every key
// above the k-th value and the first keys equal to it.
#pragma once

#include "common.cuh"
#include "route_cand.cuh"

namespace sd {
namespace {

constexpr int kTkThreads = 512;
constexpr int kTkWarps = kTkThreads / 32;
constexpr int kTkBcap = 6144;      // keys of the boundary bin kept on chip
constexpr int kTkTieCap = 1024;    // keys equal to the k-th value ranked on chip
constexpr int kTkFin = 64;         // level-2 boundary-bin keys one warp ranks directly
// On-chip scratch: bitmap | boundary list | level-2 and level-3 histograms | ties.
__host__ __device__ constexpr size_t tk_scratch_bytes(int bitmap_words) {
  return (size_t)bitmap_words * 4 + (size_t)kTkBcap * 8 + 2048 * 4 + 1024 * 4 +
         (size_t)kTkTieCap * 4;
}

// Block-level bookkeeping, in shared memory.
struct TkSmall {
  uint32_t warp_buf[33];
  uint32_t bnd[3];  // boundary bin, keys above it, keys in it
  uint32_t nb;      // boundary-bin keys seen
  uint32_t nt;      // keys equal to the k-th value seen
  uint32_t nge;     // candidates at or above the boundary bin
  uint32_t bad;     // a candidate list was missing or overflowed
  uint32_t nfin;    // keys of the level-2 boundary bin collected
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

// The bin of histogram h (NB bins, read highest first) where the descending
// count reaches need: sm->bnd = {bin, keys above it, keys in it}, or bnd[0] =
// ~0 when the histogram holds fewer than need keys.  *total = its sum.
template <int NB>
__device__ __forceinline__ void tk_boundary(const uint32_t *h, uint32_t need, TkSmall *sm, uint32_t *total) {
  constexpr int BPT = NB / kTkThreads;
  const int t = threadIdx.x;
  uint32_t c[BPT], sum = 0;
#pragma unroll
  for (int e = 0; e < BPT; ++e) {
    c[e] = h[NB - 1 - (BPT * t + e)];
    sum += c[e];
  }
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

// A no-op for tk_select's `sure` hook.
struct TkNoSure {
  __device__ void operator()(uint32_t) const {}
};

// The exact top-k of head bh (see the file comment).  S: the head's score
// row; hist: its histogram (complete when it sums to N; nullable); cand /
// use_lists: the scan's candidate lists; scratch: tk_scratch_bytes(
// bitmap_words) bytes of shared memory (bitmap_words * 32 >= N for the fast
// path).  emit(pos, j) is called for the positions in [lo, hi) only; sure(j)
// for every key known to be selected as soon as that is known (the fast
// path's keys above the boundary bin), e.g. to prefetch its rows.  Returns
// the number of keys selected (k).  Sets the informational FLAG_SLOW_SELECT
// in *status when the streaming path ran.
template <typename Emit, typename Sure>
__device__ __forceinline__ uint32_t tk_select(const float *__restrict__ S, int N, uint32_t k,
                                              const uint32_t *__restrict__ hist,
                                              const CandArgs &cand, bool use_lists, int bh,
                                              unsigned char *scratch, int bitmap_words,
                                              TkSmall *sm, uint32_t *status, Emit &emit,
                                              Sure &sure, uint32_t lo, uint32_t hi) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t *bits = reinterpret_cast<uint32_t *>(scratch);
  uint2 *blist = reinterpret_cast<uint2 *>(scratch + (size_t)bitmap_words * 4);
  uint32_t *h2 = reinterpret_cast<uint32_t *>(scratch + (size_t)bitmap_words * 4 + kTkBcap * 8);
  uint32_t *h3 = h2 + 2048;
  uint32_t *ties = h3 + 1024;
  uint2 *fin = reinterpret_cast<uint2 *>(h3);  // <= kTkFin (key, index) pairs, step 3
  const int nwords = (N + 31) / 32;

  // ---- 1. loads: the head's lists (their first `spec` entries, their lengths,
  // the head's span) and its histogram, all issued before any is used --------
  const int nl = use_lists ? cand.head_ctas : 0;  // lists: the CTAs a head can span
  const uint32_t *cnt_g = use_lists ? cand.counts + (size_t)bh * nl : nullptr;
  const uint64_t *lst = use_lists ? cand.lists + (size_t)bh * nl * kCandListCap : nullptr;
  const int spec = use_lists ? cand.spec : 0;
  const int spec_shift = __ffs(spec > 0 ? spec : 1) - 1;
  constexpr int kSpecLoads = 8;  // 16-byte loads per thread
  uint4 ev[kSpecLoads];
  uint32_t c0 = 0, c1 = 0, nsp = 0;
  if (use_lists) {
    nsp = cand.nspan[bh];
    if (tid < nl) c0 = cnt_g[tid];
    if (tid + kTkThreads < nl) c1 = cnt_g[tid + kTkThreads];
    const int npairs = (nl * spec) >> 1;
#pragma unroll
    for (int i = 0; i < kSpecLoads; ++i) {
      const int p = tid + i * kTkThreads;
      ev[i] = make_uint4(0u, 0u, 0u, 0u);
      if (p < npairs) {
        const int e = 2 * p;
        ev[i] = *reinterpret_cast<const uint4 *>(lst + (size_t)(e >> spec_shift) * kCandListCap +
                                                 (e & (spec - 1)));
      }
    }
  }
  uint32_t tot = 0;
  bool fast = hist != nullptr;
  if (fast) {
    tk_boundary<2048>(hist, k, sm, &tot);
    fast = tot == (uint32_t)N && sm->bnd[0] != ~0u;
  }
  const bool hist_ok = fast;
  fast = fast && nwords <= bitmap_words && sm->bnd[2] <= (uint32_t)kTkBcap;
  const uint32_t b1 = sm->bnd[0], above1 = sm->bnd[1], cb1 = sm->bnd[2];
  if (fast) {
    uint32_t *cnt_s = ties;  // the list lengths, on chip until step 3
    if (use_lists) {
      if (tid < nl) cnt_s[tid] = c0;
      if (tid + kTkThreads < nl) cnt_s[tid + kTkThreads] = c1;
    }
    for (int w = tid; w < nwords; w += kTkThreads) bits[w] = 0u;
    for (int b = tid; b < 2048; b += kTkThreads) h2[b] = 0u;
    if (tid == 0) {
      sm->nb = 0;
      sm->nt = 0;
      sm->nge = 0;
      sm->bad = 0;
      sm->nfin = 0;
    }
    __syncthreads();

    // ---- 2. one pass over the candidates -----------------------------------------
    // A batch of NE entries per thread: keys above the boundary bin set their
    // bit (and are announced to `sure`), boundary-bin keys count their next
    // 11 bits and join the on-chip list through one shared counter update
    // per warp and batch.
    uint32_t my_nge = 0;
    bool bad = false;
    auto classify = [&](auto &ent, uint32_t valid) {
      constexpr int NE = sizeof(ent) / sizeof(ent[0]);
      uint32_t inb1 = 0;
#pragma unroll
      for (int e = 0; e < NE; ++e) {
        const uint32_t key = (uint32_t)(ent[e] >> 32), j = (uint32_t)ent[e];
        if (!((valid >> e) & 1u)) continue;
        if (j >= (uint32_t)N) {  // never from a list this call wrote; refuse, do not trust
          bad = true;
          continue;
        }
        const uint32_t bin = key >> 21;
        if (bin > b1) {
          sh_red_or(&bits[j >> 5], 1u << (j & 31));
          ++my_nge;
          sure(j);
        } else if (bin == b1) {
          ++my_nge;
          sh_red_add(&h2[(key >> 10) & 2047u], 1u);
          inb1 |= 1u << e;
        }
      }
      const uint32_t n = __popc(inb1);
      uint32_t inc = n;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
      }
      const uint32_t wtot = __shfl_sync(0xffffffffu, inc, 31);
      if (wtot) {
        uint32_t base = 0;
        if (lane == 0) base = sh_atom_add(&sm->nb, wtot);
        base = __shfl_sync(0xffffffffu, base, 0) + inc - n;
#pragma unroll
        for (int e = 0; e < NE; ++e) {
          if ((inb1 >> e) & 1u) {
            if (base < (uint32_t)kTkBcap)
              blist[base] = make_uint2((uint32_t)(ent[e] >> 32), (uint32_t)ent[e]);
            ++base;
          }
        }
      }
    };
    if (use_lists) {
      // list l (of the l-th CTA covering the head) is live when l < nspan;
      // its first min(length, spec) entries are in registers already
      const int npairs = (nl * spec) >> 1;
      uint64_t ent[2 * kSpecLoads];
      uint32_t valid = 0;
#pragma unroll
      for (int i = 0; i < kSpecLoads; ++i) {
        const int p = tid + i * kTkThreads;
        const int e = 2 * p;
        const int l = e >> spec_shift, off = e & (spec - 1);
        uint32_t n = 0;
        if (p < npairs && l < (int)nsp) n = min(cnt_s[l], (uint32_t)kCandListCap);
        ent[2 * i] = (uint64_t)ev[i].y << 32 | ev[i].x;
        ent[2 * i + 1] = (uint64_t)ev[i].w << 32 | ev[i].z;
        valid |= (off < (int)n ? 1u : 0u) << (2 * i);
        valid |= (off + 1 < (int)n ? 1u : 0u) << (2 * i + 1);
      }
      classify(ent, valid);
      // the rest of the lists longer than spec, a warp per list, four loads
      // in flight per lane
      bool over = nsp == 0 || (int)nsp > nl;
      for (int l = warp; l < nl; l += kTkWarps) {
        if (l >= (int)nsp) continue;
        const uint32_t cnt = cnt_s[l];
        over |= cnt > (uint32_t)kCandListCap;
        const int n = (int)min(cnt, (uint32_t)kCandListCap);
        for (int i0 = spec; i0 < n; i0 += 128) {
          uint64_t e4[4];
          uint32_t v4 = 0;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int i = i0 + u * 32 + lane;
            e4[u] = i < n ? lst[(size_t)l * kCandListCap + i] : 0ull;
            v4 |= (i < n ? 1u : 0u) << u;
          }
          classify(e4, v4);
        }
      }
      if (over) bad = true;
    } else {
      for (int j0 = 0; j0 < N; j0 += 4 * kTkThreads) {
        uint64_t e4[4];
        uint32_t v4 = 0;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int j = j0 + u * kTkThreads + tid;
          const float f = j < N ? S[j] : 0.f;
          e4[u] = (uint64_t)order_key(f) << 32 | (uint32_t)j;
          v4 |= (j < N ? 1u : 0u) << u;
        }
        classify(e4, v4);
      }
    }
    if (bad) sm->bad = 1u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) my_nge += __shfl_xor_sync(0xffffffffu, my_nge, o);
    if (lane == 0 && my_nge) sh_red_add(&sm->nge, my_nge);
    __syncthreads();
    fast = !sm->bad && sm->nge == above1 + cb1 && sm->nb == cb1;
  }

  if (fast) {
    // ---- 3. the k-th value inside the boundary bin --------------------------------
    const uint32_t nb = cb1;
    uint32_t need = k - above1;
    tk_boundary<2048>(h2, need, sm, &tot);
    const uint32_t p2 = (b1 << 11) | sm->bnd[0];
    need -= sm->bnd[1];
    const uint32_t cb2 = sm->bnd[2];
    if (cb2 == need || cb2 <= (uint32_t)kTkFin) {
      // one pass: keys above the level-2 bin are in; when the whole bin is
      // taken its keys are too, else they are collected and one warp ranks
      // them exactly (key descending, then index ascending: ties to the
      // lower index) and marks the `need` first
      const bool all2 = cb2 == need;
      for (uint32_t i = tid; i < nb; i += kTkThreads) {
        const uint2 e = blist[i];
        const uint32_t top = e.x >> 10;
        if (top > p2 || (all2 && top == p2)) {
          sh_red_or(&bits[e.y >> 5], 1u << (e.y & 31));
        } else if (top == p2) {
          const uint32_t slot = sh_atom_add(&sm->nfin, 1u);
          if (slot < (uint32_t)kTkFin) fin[slot] = e;
        }
      }
      __syncthreads();
      if (!all2 && warp == 0) {
        const uint32_t nf = sm->nfin;  // == cb2
#pragma unroll
        for (int h = 0; h < kTkFin / 32; ++h) {
          const uint32_t a = lane + 32u * h;
          if (a < nf) {
            const uint2 x = fin[a];
            uint32_t rank = 0;
            for (uint32_t c = 0; c < nf; ++c) {
              const uint2 y = fin[c];
              rank += (y.x > x.x) || (y.x == x.x && y.y < x.y);
            }
            if (rank < need) sh_red_or(&bits[x.y >> 5], 1u << (x.y & 31));
          }
        }
      }
      __syncthreads();
    } else {
      // many keys share the level-2 bin: a third histogram level on the last
      // 10 bits, then the keys equal to the k-th value ranked by index
      for (int b = tid; b < 1024; b += kTkThreads) h3[b] = 0u;  // it held list lengths
      __syncthreads();
      for (uint32_t i = tid; i < nb; i += kTkThreads) {
        const uint32_t key = blist[i].x;
        if ((key >> 10) == p2) sh_red_add(&h3[key & 1023u], 1u);
      }
      __syncthreads();
      tk_boundary<1024>(h3, need, sm, &tot);
      const uint32_t v = (p2 << 10) | sm->bnd[0];
      need -= sm->bnd[1];
      TkCut cut{0, 0, 0};
      if (sm->bnd[2] == need) {
        cut.t_ge = v;
      } else {
        cut.t_ge = (uint64_t)v + 1;
        cut.tie_val = v;
        cut.n_ties = need;
      }
      for (uint32_t i = tid; i < nb; i += kTkThreads) {
        const uint2 e = blist[i];
        if ((uint64_t)e.x >= cut.t_ge) {
          sh_red_or(&bits[e.y >> 5], 1u << (e.y & 31));
        } else if (cut.n_ties && e.x == cut.tie_val) {
          const uint32_t slot = sh_atom_add(&sm->nt, 1u);
          if (slot < (uint32_t)kTkTieCap) ties[slot] = e.y;
        }
      }
      __syncthreads();
      if (cut.n_ties) {
        const uint32_t nt = sm->nt;
        if (nt > (uint32_t)kTkTieCap) {
          fast = false;  // too many equal keys to rank on chip
        } else {
          for (uint32_t i = tid; i < nt; i += kTkThreads) {
            const uint32_t j = ties[i];
            uint32_t r = 0;
            for (uint32_t i2 = 0; i2 < nt; ++i2) r += ties[i2] < j;
            if (r < cut.n_ties) sh_red_or(&bits[j >> 5], 1u << (j & 31));
          }
          __syncthreads();
        }
      }
    }
    // ---- 4. ordered positions ----------------------------------------------------
    if (fast) return tk_bitmap_emit(bits, nwords, sm, emit, lo, hi);
  }

  // ---- streaming path ----------------------------------------------------------
  if (tid == 0) raise_flag(status, FLAG_SLOW_SELECT);
  __syncthreads();
  const TkCut cut = tk_stream_cut(S, N, k, hist, hist_ok, h2, sm);
  __syncthreads();
  return tk_stream_emit(S, N, cut, sm, emit);
}

}  // namespace
}  // namespace sd
