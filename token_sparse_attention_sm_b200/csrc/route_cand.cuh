// route_cand.cuh -- the hand-off between the routing scan and the top-k
// select: the scan's partition of key tiles over its CTAs, the sample it
// draws to estimate each head's candidate bound, and the candidate lists it
// leaves behind.
//
// The exact top-k of a head (CLSA article, section 研究の背景と課題: the k
// highest-scoring tokens) only ever takes keys at or above the k-th score.
// While the scan streams K it therefore keeps, per head, every key whose top
// 11 score bits reach a bound estimated from a sample of the head's tiles
// (scanned first).  The bound is an estimate, not a guarantee: the select
// checks that the lists hold every key of the boundary bin and above (the
// scan's histogram says how many there are) and otherwise selects from the
// full score row instead.  So a poor estimate costs time, never correctness.
#pragma once

#include <stdint.h>

namespace sd {

constexpr int kScanMaxGrid = 160;    // routing-scan CTAs at most
constexpr int kCandSlots = 2;        // heads per scan CTA that keep candidate lists
constexpr int kCandListCap = 4096;   // entries per (scan CTA, head) list
constexpr int kSampleTiles = 32;     // sample tiles per head (about)
constexpr int kCandMaxLists = 1024;  // lists (scan CTAs) of one head the select can take
constexpr int kHistBins = 2048;      // top 11 bits of the order-preserving key

// Lists of head bh: list j holds the candidates of the j-th scan CTA covering
// the head (every warp of that CTA appends to it), at
//   lists + (bh * head_ctas + j) * kCandListCap,
// its length at counts[bh * head_ctas + j], and nspan[bh] = the number of
// scan CTAs covering the head (lists of j >= nspan[bh] are stale).
// head_ctas bounds the CTAs a head can span.
struct CandArgs {
  uint64_t *lists;     // (key << 32) | j entries, as above
  uint32_t *counts;    // entries appended (may exceed the cap)
  uint32_t *nspan;     // [B*Hkv]
  uint32_t *smp_hist;  // [B*Hkv][kHistBins]: histogram of the sample keys (zero between calls)
  uint32_t *smp_cnt;   // [B*Hkv]: sample keys counted so far (zero between calls)
  int grid;            // scan CTAs
  int tiles_per_head;  // scan tiles per head
  long long total_tiles;
  int head_ctas;       // scan CTAs a head can span (list slots per head)
  int spec;            // entries per list the select reads before it knows the lengths (2^n)
  int smp_stride;      // tile u of a head is a sample tile iff u % smp_stride == 0
  uint32_t smp_keys;   // keys in the sample tiles of one head
  uint32_t smp_min;    // sample keys counted before a bound is drawn (a part of smp_keys)
  float k_over_n;      // k / N: the share of the keys the select takes
};

// The scan CTAs a head of tph tiles can span when the runs are at least
// total / grid tiles long.
__host__ __device__ inline int cand_head_ctas(long long tph, long long total, int grid) {
  const long long run = total / grid;
  return (int)((tph + run - 1) / run + 1);
}

// First tile of scan CTA c (tiles are dealt in contiguous runs).
__host__ __device__ inline long long scan_tile_begin(int c, long long total, int grid) {
  return (long long)c * total / grid;
}

// The scan CTA whose run holds tile t.
__host__ __device__ inline int scan_cta_of_tile(long long t, long long total, int grid) {
  int c = (int)(((t + 1) * grid - 1) / total);
  while (c > 0 && scan_tile_begin(c, total, grid) > t) --c;
  while (c + 1 < grid && scan_tile_begin(c + 1, total, grid) <= t) ++c;
  return c;
}

// The list of the j-th scan CTA covering head bh, and its length.
__host__ __device__ inline uint64_t *cand_list(const CandArgs &a, int bh, int j) {
  return a.lists + ((size_t)bh * a.head_ctas + j) * kCandListCap;
}
__host__ __device__ inline uint32_t *cand_count(const CandArgs &a, int bh, int j) {
  return a.counts + (size_t)bh * a.head_ctas + j;
}

}  // namespace sd
