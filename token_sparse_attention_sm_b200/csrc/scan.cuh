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

// First tile of scan CTA c (tiles are dealt in contiguous runs).
__host__ __device__ inline long long scan_tile_begin(int c, long long total, int grid) {
  return (long long)c * total / grid;
}

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

// A CTA's walk over its tiles [t_begin, t_end) in ascending order, kept as
// (head, tile of the head) and stepped without any division: the walk runs
// once per tile in the copy-issuing thread, where a 64-bit division per tile
// is enough to slow the stream down.
struct TileWalk {
  int bh, u, tph;
  __device__ void init(long long b, int tiles_per_head) {
    tph = tiles_per_head;
    bh = (int)(b / tph);
    u = (int)(b - (long long)bh * tph);
  }
  __device__ void next() {
    if (++u == tph) {
      u = 0;
      ++bh;
    }
  }
};

// One CTA's share of the scan: tiles [t_begin, t_end).  K holds kv_rows rows
// per (sequence, KV head), the first N of them scanned.  Warps 0..7 consume
// (warp w in group w / 4, which takes the tiles in stages of its parity),
// warp 8 produces: its lane 0 issues the copies and waits for the last ones
// to land, its other lanes (and any further warps) return at once.  Barriers
// full/empty must be initialised (count 1 / kScanGroupWarps).
template <typename T, int D, int kSlots, bool kMark = false>
__device__ __forceinline__ void scan_tiles(const T *__restrict__ q, const T *__restrict__ K,
                                           int N, int kv_rows, int Hq, int Hkv,
                                           int tiles_per_head, long long t_begin, long long t_end,
                                           int bh_first, float scale, unsigned char *ring,
                                           uint64_t *full, uint64_t *empty, ScanOut o,
                                           uint32_t *status) {
  const int nw = (N + 31) / 32;
  using C = ScoreCfg<T, D>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = (int)(t_end - t_begin);
  if (warp > kScanConsumerWarps) return;  // extra warps of a larger CTA idle here
  if (warp == kScanConsumerWarps) {
    // ---- producer: one thread issues the bulk copies -------------------------
    if (lane == 0) {
      const uint64_t pol = l2_evict_first_policy();
      TileWalk seq;
      seq.init(t_begin, tiles_per_head);
      int issued = 0;
      for (int i = 0; i < ntiles; ++i, seq.next()) {
        const int s = i % kScanStages;
        if (i >= kScanStages &&
            !mbar_wait(&empty[s], ((i / kScanStages) - 1) & 1, status))
          break;
        const int bh = seq.bh;
        const int j0 = seq.u * C::kStageKeys;
        const int nk = min(C::kStageKeys, N - j0);
        const uint32_t bytes = (uint32_t)nk * C::kRowBytes;
        mbar_arrive_expect_tx(&full[s], bytes);
        bulk_g2s(ring + (size_t)s * kScanStageBytes, K + ((size_t)bh * kv_rows + j0) * D,
                 bytes, &full[s], pol);
        ++issued;
      }
      // Do not leave while copies may still be landing in shared memory.
      for (int i = max(0, issued - kScanStages); i < issued; ++i)
        mbar_wait(&full[i % kScanStages], (i / kScanStages) & 1, status);
    }
    return;
  }

  // ---- consumers ------------------------------------------------------------
  const int grp = warp / kScanGroupWarps, wq = warp % kScanGroupWarps;
  const int sub = lane % C::kLpk;  // which 16-byte slice of the row
  int cur_bh = -1;
  uint32_t tkey = 0;  // threshold marking: order key of the head's tau
  float qs[C::kEpl];
  TileWalk seq;
  seq.init(t_begin, tiles_per_head);
  for (int i = 0; i < ntiles; ++i, seq.next()) {
    const int s = i % kScanStages;
    if (s % kScanGroups != grp) continue;  // the other group's stage
    const int bh = seq.bh;
    const int j0 = seq.u * C::kStageKeys;
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
    if (!mbar_wait(&full[s], (i / kScanStages) & 1, status)) break;
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
            if (slot < kSlots)
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
