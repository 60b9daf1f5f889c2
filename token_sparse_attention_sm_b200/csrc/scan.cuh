// scan.cuh -- the streaming q.K scan of the routing score kernels (score.cu)
// and the scoring routine the Louver query shares with it (louver.cu).
//
// S[b,h,j] = (sum over the G query heads of KV head h: <q_g, K[b,h,j]>)/sqrt(d)
// (CLSA article, section CLSAの仕組み).  A CTA owns a contiguous run of 32 KB
// key tiles (tiles never straddle heads).  One producer thread streams them
// into a shared-memory ring with 1-D bulk copies (cp.async.bulk + mbarrier
// transaction counts, L2 evict-first: K is read once); two groups of four
// consumer warps take alternate stages and read them back with
// conflict-free 128-bit shared loads.  A warp handles 32
// keys at a time: each lane loads 16 bytes of a row per round (rows are split
// over LPK lanes), keeps one partial dot per round, and a transposing shuffle
// reduction leaves one finished score per lane, stored as one coalesced
// 128-byte write.  The G query rows are summed once into qbar (fp32) and
// pre-scaled by 1/sqrt(d); by linearity this is the group sum, only the fp32
// rounding order differs.
#pragma once

#include "common.cuh"

namespace sd {
namespace {

// Two groups of four consumer warps; stage s of the ring is always consumed
// by group s % 2 (so a warp never waits on a stage two phases ahead of its
// barrier), which gives each warp two tile times per tile of work.
constexpr int kScanGroupWarps = 4;
constexpr int kScanGroups = 2;
constexpr int kScanConsumerWarps = kScanGroupWarps * kScanGroups;
constexpr int kScanStages = 6;
static_assert(kScanStages % kScanGroups == 0, "a stage belongs to one consumer group");
constexpr int kScanStageBytes = 32768;
constexpr int kScanThreads = (kScanConsumerWarps + 1) * 32;  // + the copy-issuing warp
constexpr int kScanBins = 2048;  // top 11 bits of the order-preserving key

// The scan's tiles are dealt to its CTAs in contiguous runs: CTA c's run
// starts at scan_tile_begin(c) (q = total / grid tiles each, the first
// total % grid runs one more).
__host__ __device__ inline long long scan_tile_begin(int c, long long total, int grid) {
  const long long q = total / grid, r = total % grid;
  return (long long)c * q + (c < r ? c : r);
}

// Dynamic claiming of the runs' tiles.  Some SMs stream K measurably slower
// than others (the same ones from call to call), so a static split leaves
// the whole scan waiting for its slowest CTAs.  Each run has a claim counter
// (the next tile of the run is run_begin + atomicAdd(counter, 1)); a CTA
// claims from its own run first, then from other runs: each probe round
// reads the counters of kScanStealSpan runs spread evenly over the grid
// (the slow CTAs come in blocks of neighbouring indices, so nearby runs are
// the wrong place to look) and claims from the one with the most tiles
// left.  The last CTA to finish zeroes the counters for the next call.
constexpr int kScanMaxCtas = 511;     // counters: [kScanMaxCtas + 1] words
constexpr int kScanStealSpan = 16;    // runs probed per round
constexpr int kScanStealRounds = 4;   // probe rounds before a CTA gives up

template <typename T, int D>
struct ScoreCfg {
  static constexpr int kRowBytes = D * (int)sizeof(T);
  static constexpr int kEpl = 16 / (int)sizeof(T);  // elements per 16 B
  static constexpr int kLpk = D / kEpl;              // lanes per key row
  static constexpr int kKpr = 32 / kLpk;             // keys per round
  static constexpr int kStageKeys = kScanStageBytes / kRowBytes;
  static constexpr int kWarpTiles = kStageKeys / 32;
  static_assert(kKpr * kRowBytes == 512, "a round covers 512 contiguous bytes");
  static_assert(kWarpTiles >= 1, "stage holds at least one warp tile");
};

// Transposing reduction: on entry v[0..R) are per-lane partial sums of R
// different keys; partners `O` lanes apart exchange halves.  On exit v[0]
// holds the finished sum of key (lane % (2*O_top)).
template <int R, int O>
struct TReduce {
  static __device__ __forceinline__ void run(float *v, int lane) {
    const bool upper = (lane & O) != 0;
#pragma unroll
    for (int i = 0; i < R / 2; ++i) {
      const float send = upper ? v[i] : v[i + R / 2];
      const float keep = upper ? v[i + R / 2] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, O);
    }
    TReduce<R / 2, O / 2>::run(v, lane);
  }
};
template <int R>
struct TReduce<R, 0> {
  static __device__ __forceinline__ void run(float *, int) {}
};

// Element i of qbar for head bh: the group's query rows summed in fp32 in
// head order, then scaled.  Every kernel whose scores must agree bit for bit
// with the scan forms qbar this way.
template <typename T, int D>
__device__ __forceinline__ float qbar_elem(const T *__restrict__ q, int bh, int Hq, int Hkv,
                                           int i, float scale) {
  const int b = bh / Hkv, h = bh % Hkv, G = Hq / Hkv;
  float s = 0.f;
  for (int g = 0; g < G; ++g) s += DT<T>::to_f(q[((size_t)b * Hq + (size_t)h * G + g) * D + i]);
  return s * scale;
}

// This lane's slice of qbar: lane `sub` of a row holds elements
// sub*kEpl .. sub*kEpl+kEpl-1 (the same arithmetic as qbar_elem).
template <typename T, int D>
__device__ __forceinline__ void load_qbar(const T *__restrict__ q, int bh, int Hq, int Hkv,
                                          int sub, float scale,
                                          float (&qs)[ScoreCfg<T, D>::kEpl]) {
  using C = ScoreCfg<T, D>;
  const int b = bh / Hkv, h = bh % Hkv, G = Hq / Hkv;
#pragma unroll
  for (int e = 0; e < C::kEpl; ++e) qs[e] = 0.f;
  for (int g = 0; g < G; ++g) {
    const T *qp = q + ((size_t)b * Hq + (size_t)h * G + g) * D + sub * C::kEpl;
#pragma unroll
    for (int e = 0; e < C::kEpl; ++e) qs[e] += DT<T>::to_f(qp[e]);
  }
#pragma unroll
  for (int e = 0; e < C::kEpl; ++e) qs[e] *= scale;
}

// Scores of the 32 keys of one warp tile: rows key0 .. key0+31 of a block of
// contiguous rows in shared memory (kRowBytes each).  Returns, in every lane,
// the score of key key0 + (lane % kLpk) * kKpr + lane / kLpk.  The one place
// that fixes the scan's fp32 arithmetic (used by every kernel whose scores
// must agree bit for bit).
template <typename T, int D>
__device__ __forceinline__ float warp_tile_scores(const unsigned char *rows, int key0,
                                                  const float (&qs)[ScoreCfg<T, D>::kEpl],
                                                  int lane) {
  using C = ScoreCfg<T, D>;
  const unsigned char *base = rows + (size_t)key0 * C::kRowBytes + lane * 16;
  float v[C::kLpk];
#pragma unroll
  for (int r = 0; r < C::kLpk; ++r) {
    float f[C::kEpl];
    unpack16<T>(lds128(base + r * 512), f);
    float acc = 0.f;
#pragma unroll
    for (int e = 0; e < C::kEpl; ++e) acc = fmaf(qs[e], f[e], acc);
    v[r] = acc;
  }
  TReduce<C::kLpk, C::kLpk / 2>::run(v, lane);
  return v[0];
}

// Where the scan puts its by-products.  shist: kSlots per-head shared-memory
// histograms (heads bh_first .. bh_first + kSlots - 1; later heads go to the
// global histogram directly); hist == nullptr disables counting.
struct ScanOut {
  float *S;
  uint32_t *hist;
  uint32_t *shist;
  // threshold marking (scan_tiles<..., true>): bits [heads][ceil(N/32)] gets,
  // for each 32-key word, bit t set iff key 32*word + t scores >= tau[head]
  // (order-preserving keys compared, as the threshold select compares);
  // nothing else is written.
  uint32_t *bits;
  const float *tau;
};

// One CTA's share of the scan: its run of tiles [t_begin, t_end), then tiles
// claimed from other runs (see kScanStealSpan).  K holds kv_rows rows
// per (sequence, KV head), the first N of them scanned.  Warps 0..7 consume
// (warp w in group w / 4, which takes the tiles in stages of its parity),
// warp 8 produces: its lane 0 claims the tiles, tells the consumers which
// tile each stage holds (sinfo: head, tile of the head; head -1 ends a
// group's loop) and issues the copies; its other lanes (and any further
// warps) return at once.  ctr: the claim counters of the grid's runs, zero
// on entry and left zero.  Barriers full/empty must be initialised (count 1
// / kScanGroupWarps).
template <typename T, int D, int kSlots, bool kMark = false>
__device__ __forceinline__ void scan_tiles(const T *__restrict__ q, const T *__restrict__ K,
                                           int N, int kv_rows, int Hq, int Hkv,
                                           int tiles_per_head, long long total_tiles,
                                           long long t_begin, long long t_end, int bh_first,
                                           float scale, unsigned char *ring, uint64_t *full,
                                           uint64_t *empty, int2 *sinfo, uint32_t *ctr,
                                           ScanOut o, uint32_t *status) {
  const int nw = (N + 31) / 32;
  using C = ScoreCfg<T, D>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp > kScanConsumerWarps) return;  // extra warps of a larger CTA idle here
  if (warp == kScanConsumerWarps) {
    // ---- producer: one thread claims tiles and issues the bulk copies -------
    if (lane == 0) {
      const uint64_t pol = l2_evict_first_policy();
      const int grid = (int)gridDim.x, me = (int)blockIdx.x;
      const long long rq = total_tiles / grid, rr = total_tiles % grid;
      int victim = me;
      long long vb = t_begin, vlen = t_end - t_begin;
      uint32_t pend = atomicAdd(&ctr[victim], 1u);
      int issued = 0, rounds = 0;
      bool ok = true;
      while (true) {
        long long t = -1;
        while (true) {
          if ((long long)pend < vlen) {
            t = vb + pend;
            break;
          }
          // this run is exhausted: kScanStealSpan runs spread over the grid
          // (shifted each round), their counters read all at once; claim
          // from the one with the most tiles left
          if (++rounds > kScanStealRounds) break;
          uint32_t seen[kScanStealSpan];
          int pv[kScanStealSpan];
#pragma unroll
          for (int j = 0; j < kScanStealSpan; ++j) {
            pv[j] = (me + rounds + j * grid / kScanStealSpan) % grid;
            asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(seen[j]) : "l"(ctr + pv[j])
                         : "memory");
          }
          long long best_left = 0;
          int best = -1;
#pragma unroll
          for (int j = 0; j < kScanStealSpan; ++j) {
            const int v = pv[j];
            if (v == me) continue;
            const long long len = rq + (v < rr ? 1 : 0);
            const long long left = len - (long long)seen[j];
            if (left > best_left) {
              best_left = left;
              best = v;
            }
          }
          if (best < 0) break;
          victim = best;
          vb = (long long)victim * rq + (victim < rr ? victim : rr);
          vlen = rq + (victim < rr ? 1 : 0);
          pend = atomicAdd(&ctr[victim], 1u);
        }
        if (t < 0) break;
        pend = atomicAdd(&ctr[victim], 1u);  // the next claim, in flight while this tile is issued
        const int s = issued % kScanStages;
        if (issued >= kScanStages &&
            !mbar_wait(&empty[s], ((issued / kScanStages) - 1) & 1, status)) {
          ok = false;
          break;
        }
        const int bh = (int)((unsigned long long)t / (unsigned)tiles_per_head);
        const int u = (int)(t - (long long)bh * tiles_per_head);
        const int j0 = u * C::kStageKeys;
        const int nk = min(C::kStageKeys, N - j0);
        const uint32_t bytes = (uint32_t)nk * C::kRowBytes;
        sinfo[s] = make_int2(bh, u);
        mbar_arrive_expect_tx(&full[s], bytes);
        bulk_g2s(ring + (size_t)s * kScanStageBytes, K + ((size_t)bh * kv_rows + j0) * D,
                 bytes, &full[s], pol);
        ++issued;
      }
      // Do not leave while copies may still be landing in shared memory.
      for (int i = max(0, issued - kScanStages); i < issued; ++i)
        mbar_wait(&full[i % kScanStages], (i / kScanStages) & 1, status);
      // one end marker per consumer group
      for (int e = 0, i = issued; e < kScanGroups && ok; ++e, ++i) {
        const int s = i % kScanStages;
        if (i >= kScanStages && !mbar_wait(&empty[s], ((i / kScanStages) - 1) & 1, status))
          break;
        sinfo[s] = make_int2(-1, 0);
        mbar_arrive(&full[s]);
      }
      // every claim of this CTA has returned; the last CTA out resets the counters
      if (atomicAdd(&ctr[grid], 1u) == (uint32_t)grid - 1u)
        for (int v = 0; v <= grid; ++v) ctr[v] = 0u;
    }
    return;
  }

  // ---- consumers ------------------------------------------------------------
  const int grp = warp / kScanGroupWarps, wq = warp % kScanGroupWarps;
  const int sub = lane % C::kLpk;  // which 16-byte slice of the row
  int cur_bh = -1;
  uint32_t tkey = 0;  // threshold marking: order key of the head's tau
  float qs[C::kEpl];
  for (int i = 0;; ++i) {
    const int s = i % kScanStages;
    if (s % kScanGroups != grp) continue;  // the other group's stage
    if (!mbar_wait(&full[s], (i / kScanStages) & 1, status)) break;
    const int2 tile = sinfo[s];
    if (tile.x < 0) break;  // the producer's end marker
    const int bh = tile.x;
    const int j0 = tile.y * C::kStageKeys;
    const int nk = min(C::kStageKeys, N - j0);
    if (bh != cur_bh) {
      cur_bh = bh;
      load_qbar<T, D>(q, bh, Hq, Hkv, sub, scale, qs);
      if constexpr (kMark) {
        const float tv = o.tau[bh];
        tkey = order_key(tv);
        if (!isfinite(tv) && lane == 0 && warp == 0) raise_flag(status, FLAG_NONFINITE);
      }
    }
    const unsigned char *stage = ring + (size_t)s * kScanStageBytes;
    float *Srow = kMark ? nullptr : o.S + (size_t)bh * N + j0;
    const int slot = bh - bh_first;
    for (int wt = wq; wt < C::kWarpTiles; wt += kScanGroupWarps) {
      const int key0 = wt * 32;
      if (key0 >= nk) break;
      const float score = warp_tile_scores<T, D>(stage, key0, qs, lane);
      const int kk = key0 + sub * C::kKpr + lane / C::kLpk;
      const bool valid = kk < nk;
      if constexpr (kMark) {
        // one word per 32 keys, written whole by this warp (no atomics)
        const bool pass = valid && order_key(score) >= tkey;
        const uint32_t word = __reduce_or_sync(0xffffffffu, pass ? 1u << (kk - key0) : 0u);
        if (lane == 0) o.bits[(size_t)bh * nw + (j0 + key0) / 32] = word;
      } else {
        const uint32_t key = order_key(score);
        if (valid) {
          Srow[kk] = score;
          if (o.hist) {
            const uint32_t bin = key >> 21;
            if ((unsigned)slot < (unsigned)kSlots)
              atomicAdd(&o.shist[slot * kScanBins + bin], 1u);
            else
              atomicAdd(&o.hist[(size_t)bh * kScanBins + bin], 1u);
          }
        }
      }
      if (__any_sync(0xffffffffu, valid && !isfinite(score)) && lane == 0)
        raise_flag(status, FLAG_NONFINITE);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
}

}  // namespace
}  // namespace sd
