// score.cu -- A1, the routing score scan.
//
// S[b,h,j] = (sum over the G query heads of KV head h: <q_g, K[b,h,j]>)/sqrt(d)
// for every cached key: one streaming pass over the whole shared KV cache
// (CLSA article, section CLSAの仕組み: the routing set is computed once over
// the shared cache; section 研究の背景と課題: at 128K this scan alone costs
// about as much as dense attention, because decode is bound by reading the
// KV cache).
//
// Design (HBM-bound; 4 flop per byte of K):
//  * The G query rows of a KV head are summed once into qbar (fp32) and
//    pre-scaled by 1/sqrt(d), so each key costs one d-long dot product:
//    S_j = <qbar, K_j>.  By linearity this is the group sum; only the fp32
//    rounding order differs from summing per-head dot products.
//  * Persistent grid, one CTA per SM.  Each CTA owns a contiguous run of
//    32 KB key tiles (tiles never straddle heads).  One producer thread
//    streams tiles into a 5-stage shared-memory ring with 1-D bulk copies
//    (cp.async.bulk + mbarrier transaction counts, L2 evict-first: K is read
//    once).  Four consumer warps read the tiles back with conflict-free
//    128-bit shared loads.
//  * A warp handles 32 keys at a time: each lane loads 16 bytes of a row per
//    round (rows are split over LPK lanes), keeps one partial dot per round,
//    and a transposing shuffle reduction (LPK-1 shuffles for 32 keys) leaves
//    one finished score per lane, stored as one coalesced 128-byte write.
//  * Optionally (hist != nullptr) the scan also counts, per (sequence, KV
//    head), the scores by the top 11 bits of their order-preserving key --
//    the first level of the radix top-k -- in shared memory, and adds the
//    non-zero bins to the global histogram at the end.  This costs nothing
//    in a memory-bound scan and saves the select kernel a pass.
#include "common.cuh"
#include "internal.h"
#include "scan.cuh"

namespace sd {
namespace {

constexpr int kHistSlots = 2;  // heads a CTA can count in shared memory (later ones: global)
constexpr int kScoreSmem = kScanStages * kScanStageBytes + kHistSlots * kScanBins * 4 +
                           2 * kScanStages * 8 + (int)sizeof(CandShared);
constexpr int kSampleWarp = kScanConsumerWarps + 1;  // the warp after the producer

// The sample warp of a candidate scan (top-k routing).  For each head this
// CTA covers (at most kCandSlots): wait until a share (smp_min) of the head's
// sample keys has been counted -- the sample tiles are every CTA's first
// tiles, so this takes a few tile times, and it never waits past the end of
// this CTA's own consumers, so no CTA ever depends on another being
// resident -- then draw the head's bound from the sample histogram as it
// stands: m sample keys, of which mu = m * k / N are expected among the top
// k; the bound is the highest bin whose descending count reaches mu plus four
// standard deviations plus four, so it lies below the k-th score unless the
// sample is unrepresentative (the select then finds out and reads the full
// score rows).  It publishes the bound to the consumer warps, checks this
// CTA's own sample tiles against it from S (the consumers scanned them before
// the bound existed), and finally writes its list counts and meets the
// consumers at named barrier 2.
template <typename T, int D>
__device__ void sample_warp(const float *__restrict__ S, int N, long long t_begin,
                            long long t_end, int bh_first, int bh_last, const CandArgs &cand,
                            CandShared *cs) {
  using C = ScoreCfg<T, D>;
  const int lane = threadIdx.x & 31;
  const int tph = cand.tiles_per_head;
#pragma unroll
  for (int s = 0; s < kCandSlots; ++s) {
    const int bh = bh_first + s;
    if (bh > bh_last) continue;
    // one lane polls (a relaxed load, then a pause: every CTA polls, so the
    // rate matters to the L2); once enough keys are counted every lane takes
    // the count with acquire order before reading the histogram
    bool ready = false;
    if (lane == 0) {
      bool last = false;
      while (true) {
        uint32_t v;
        asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(cand.smp_cnt + bh)
                     : "memory");
        ready = v >= cand.smp_min;
        if (ready || last) break;
        // once the consumers are done, one last look, then give up
        if (cs->consumers_done >= (uint32_t)kScanConsumerWarps)
          last = true;
        else
          __nanosleep(256);
      }
    }
    ready = __shfl_sync(0xffffffffu, ready, 0);
    if (!ready) continue;
    {
      uint32_t v;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(cand.smp_cnt + bh)
                   : "memory");
      (void)v;
    }
    // lane l sums bins [2048 - 64 (l + 1), 2048 - 64 l) of the histogram as
    // it stands (later sample keys may still be arriving: m counts what was read)
    const uint32_t *h = cand.smp_hist + (size_t)bh * kScanBins;
    const uint4 *h4 = reinterpret_cast<const uint4 *>(h + kScanBins - 64 * (lane + 1));
    uint32_t hv[64];
    uint32_t sum = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint4 v = h4[i];
      hv[4 * i] = v.x;
      hv[4 * i + 1] = v.y;
      hv[4 * i + 2] = v.z;
      hv[4 * i + 3] = v.w;
      sum += v.x + v.y + v.z + v.w;
    }
    uint32_t inc = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    const uint32_t m_keys = __shfl_sync(0xffffffffu, inc, 31);
    const float mu = cand.k_over_n * (float)m_keys;
    const uint32_t c_star = (uint32_t)(mu + 4.f * sqrtf(mu) + 4.f) + 1u;
    const uint32_t m = __ballot_sync(0xffffffffu, inc >= c_star);
    uint32_t bound = 0;  // the sample holds fewer than c_star keys: every bin
    if (m) {
      const int L = __ffs(m) - 1;
      if (lane == L) {
        // the bins of this lane, highest first (hv[63] is the highest)
        uint32_t cum = inc - sum;
        int i = 63;
        for (; i > 0; --i) {
          cum += hv[i];
          if (cum >= c_star) break;
        }
        bound = (uint32_t)(kScanBins - 64 * (L + 1) + i);
      }
      bound = __shfl_sync(0xffffffffu, bound, L);
    }
    if (lane == 0) cs->bound[s] = bound + 1;
    // this CTA's sample tiles of head bh, checked from S
    uint64_t *list = cand_list(cand, bh, cs->jpos[s]);
    const long long h0 = (long long)bh * tph;
    long long u = t_begin > h0 ? t_begin - h0 : 0;
    u = (u + cand.smp_stride - 1) / cand.smp_stride * cand.smp_stride;
    for (; u < tph && h0 + u < t_end; u += cand.smp_stride) {
      const int j0 = (int)u * C::kStageKeys;
      const int nk = min(C::kStageKeys, N - j0);
      for (int kk0 = 0; kk0 < nk; kk0 += 32) {
        const int kk = kk0 + lane;
        const bool valid = kk < nk;
        const uint32_t key = valid ? order_key(S[(size_t)bh * N + j0 + kk]) : 0u;
        cand_append(list, &cs->lcount[s], valid && (key >> 21) >= bound, key,
                    (uint32_t)(j0 + kk), lane);
      }
    }
  }
  asm volatile("bar.sync 2, %0;" ::"r"((kScanConsumerWarps + 1) * 32) : "memory");
}

// kCand: top-k routing with candidate lists (one more warp draws the sample
// bound, see sample_warp; cand describes the lists).
template <typename T, int D, bool kCand>
__global__ void __launch_bounds__(kScanThreads + (kCand ? 32 : 0), 1)
    score_kernel(const T *__restrict__ q, const T *__restrict__ K,
                 float *__restrict__ S, int N, int kv_rows, int Hq, int Hkv,
                 int tiles_per_head, long long total_tiles, float scale,
                 uint32_t *__restrict__ hist, const __grid_constant__ CandArgs cand,
                 uint32_t *status) {
  extern __shared__ __align__(128) unsigned char smem[];
  uint32_t *shist = reinterpret_cast<uint32_t *>(smem + kScanStages * kScanStageBytes);
  uint64_t *full = reinterpret_cast<uint64_t *>(
      smem + kScanStages * kScanStageBytes + kHistSlots * kScanBins * 4);
  uint64_t *empty = full + kScanStages;
  CandShared *cs = reinterpret_cast<CandShared *>(empty + kScanStages);

  const long long t_begin = scan_tile_begin(blockIdx.x, total_tiles, gridDim.x);
  const long long t_end = scan_tile_begin(blockIdx.x + 1, total_tiles, gridDim.x);
  const int ntiles = (int)(t_end - t_begin);
  const int bh_first = (int)(t_begin / tiles_per_head);
  const int bh_last = ntiles > 0 ? (int)((t_end - 1) / tiles_per_head) : bh_first - 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (hist) {
    for (int i = threadIdx.x; i < kHistSlots * kScanBins; i += blockDim.x) shist[i] = 0u;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kScanStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kScanGroupWarps);
    }
    for (int s = 0; s < kCandSlots; ++s) {
      cs->bound[s] = 0u;
      cs->lcount[s] = 0u;
      // this CTA's place among the CTAs covering the head of slot s
      const long long h0 = (long long)(bh_first + s) * tiles_per_head;
      cs->jpos[s] = kCand ? (int)blockIdx.x - scan_cta_of_tile(h0, total_tiles, gridDim.x) : 0;
    }
    cs->consumers_done = 0u;
    fence_mbar_init();
  }
  __syncthreads();
  grid_dep_wait();
  grid_dep_launch();
  if (kCand && threadIdx.x == 0) {
    // the CTA holding a head's last tile tells the select how many CTAs
    // (and so lists) the head has
    for (int s = 0; s < kCandSlots; ++s) {
      const int bh = bh_first + s;
      if (bh <= bh_last && (long long)(bh + 1) * tiles_per_head <= t_end)
        cand.nspan[bh] = (uint32_t)(cs->jpos[s] + 1);
    }
  }

  if constexpr (kCand) {
    if (warp == kSampleWarp) {
      sample_warp<T, D>(S, N, t_begin, t_end, bh_first, bh_last, cand, cs);
      return;
    }
  }
  ScanOut o;
  o.S = S;
  o.hist = hist;
  o.shist = shist;
  o.bits = nullptr;
  o.tau = nullptr;
  int ndef = 0;
  scan_tiles<T, D, kHistSlots, false, kCand>(q, K, N, kv_rows, Hq, Hkv, tiles_per_head, t_begin,
                                             t_end, bh_first, scale, smem, full, empty, o, cand,
                                             cs, ndef, status);
  if (threadIdx.x >= kScanConsumerWarps * 32) return;  // producer warp
  if constexpr (kCand) {
    // consumers: wait for the sample warp, re-check deferred tiles, publish
    // the list lengths
    __syncwarp();
    if (lane == 0) atomicAdd(const_cast<uint32_t *>(&cs->consumers_done), 1u);
    asm volatile("bar.sync 2, %0;" ::"r"((kScanConsumerWarps + 1) * 32) : "memory");
    cand_deferred<T, D>(S, N, tiles_per_head, bh_first, cand, cs, ndef);
    // every append of this CTA is done: publish the list lengths
    asm volatile("bar.sync 1, %0;" ::"r"(kScanConsumerWarps * 32) : "memory");
    if (threadIdx.x == 0) {
      for (int s = 0; s < kCandSlots; ++s)
        if (bh_first + s <= bh_last) *cand_count(cand, bh_first + s, cs->jpos[s]) = cs->lcount[s];
    }
  }
  if (hist) {
    // consumer warps only (named barrier 1): every count is in shared memory
    asm volatile("bar.sync 1, %0;" ::"r"(kScanConsumerWarps * 32) : "memory");
    const int nslots = min(kHistSlots, bh_last - bh_first + 1);
    for (int i = threadIdx.x; i < nslots * kScanBins; i += kScanConsumerWarps * 32) {
      const uint32_t c = shist[i];
      if (c) atomicAdd(&hist[(size_t)(bh_first + i / kScanBins) * kScanBins + (i % kScanBins)], c);
    }
  }
}

// A1 + A2' for the full-scan threshold routing: the same scan, but instead of
// the scores it writes, per 32 keys, the word of bits "score >= tau" (one
// plain store per warp tile: the words are owned by one warp each, every word
// of a head is rewritten on every call, so nothing needs clearing).
template <typename T, int D>
__global__ void __launch_bounds__(kScanThreads, 1)
    threshold_mark_kernel(const T *__restrict__ q, const T *__restrict__ K,
                          const float *__restrict__ tau, uint32_t *__restrict__ bits, int N,
                          int kv_rows, int Hq, int Hkv, int tiles_per_head, long long total_tiles,
                          float scale, uint32_t *status) {
  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kScanStages * kScanStageBytes);
  uint64_t *empty = full + kScanStages;
  const long long t_begin = scan_tile_begin(blockIdx.x, total_tiles, gridDim.x);
  const long long t_end = scan_tile_begin(blockIdx.x + 1, total_tiles, gridDim.x);
  if (threadIdx.x == 0) {
    for (int s = 0; s < kScanStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kScanGroupWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();
  grid_dep_wait();
  grid_dep_launch();
  ScanOut o;
  o.S = nullptr;
  o.hist = nullptr;
  o.shist = nullptr;
  o.bits = bits;
  o.tau = tau;
  const CandArgs none{};
  int ndef = 0;
  scan_tiles<T, D, kHistSlots, true>(q, K, N, kv_rows, Hq, Hkv, tiles_per_head, t_begin, t_end,
                                     (int)(t_begin / tiles_per_head), scale, smem, full, empty, o,
                                     none, nullptr, ndef, status);
}

template <typename T, int D>
cudaError_t launch_mark_t(const Shape &s, const void *q, const void *K, const float *tau,
                          uint32_t *bits, uint32_t *status, cudaStream_t st) {
  using C = ScoreCfg<T, D>;
  DeviceInfo di;
  cudaError_t e = device_info(&di);
  if (e != cudaSuccess) return e;
  constexpr int kSmem = kScanStages * kScanStageBytes + 2 * kScanStages * 8;
  auto kern = threshold_mark_kernel<T, D>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  const int tiles_per_head = (s.N + C::kStageKeys - 1) / C::kStageKeys;
  const long long total = (long long)s.BH() * tiles_per_head;
  const int grid = (int)(total < di.sm_count ? total : di.sm_count);
  const float scale = (float)(1.0 / __builtin_sqrt((double)D));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3(kScanThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = st;
  cudaLaunchAttribute attrs[1];
  cfg.attrs = attrs;
  cfg.numAttrs = 0;
  add_pdl_attr(cfg, attrs);
  e = cudaLaunchKernelEx(&cfg, kern, static_cast<const T *>(q), static_cast<const T *>(K), tau,
                         bits, s.N, s.Ncap, s.Hq, s.Hkv, tiles_per_head, total, scale, status);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_score_t(const Shape &s, const void *q, const void *K, float *S,
                           uint32_t *hist, const CandArgs *cand, uint32_t *status,
                           cudaStream_t st) {
  using C = ScoreCfg<T, D>;
  DeviceInfo di;
  cudaError_t e = device_info(&di);
  if (e != cudaSuccess) return e;
  const bool use_cand = cand && cand->lists;
  auto kern = use_cand ? score_kernel<T, D, true> : score_kernel<T, D, false>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kScoreSmem);
  if (e != cudaSuccess) return e;
  const int tiles_per_head = (s.N + C::kStageKeys - 1) / C::kStageKeys;
  const long long total = (long long)s.BH() * tiles_per_head;
  const int grid = scan_grid(s, di.sm_count);
  if (use_cand && (cand->grid != grid || cand->tiles_per_head != tiles_per_head ||
                   cand->total_tiles != total))
    return cudaErrorInvalidValue;  // the plan was made for another partition
  const float scale = (float)(1.0 / __builtin_sqrt((double)D));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3(kScanThreads + (use_cand ? 32 : 0), 1, 1);
  cfg.dynamicSmemBytes = kScoreSmem;
  cfg.stream = st;
  cudaLaunchAttribute attrs[1];
  cfg.attrs = attrs;
  cfg.numAttrs = 0;
  add_pdl_attr(cfg, attrs);
  const CandArgs none{};
  e = cudaLaunchKernelEx(&cfg, kern, static_cast<const T *>(q), static_cast<const T *>(K), S,
                         s.N, s.Ncap, s.Hq, s.Hkv, tiles_per_head, total, scale, hist,
                         use_cand ? *cand : none, status);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_threshold_mark(const Shape &s, const void *q, const void *K,
                                  const float *tau, uint32_t *bits, uint32_t *status,
                                  cudaStream_t st) {
  if (s.dtype == 1) {
    if (s.d == 128) return launch_mark_t<__nv_bfloat16, 128>(s, q, K, tau, bits, status, st);
    return launch_mark_t<__nv_bfloat16, 64>(s, q, K, tau, bits, status, st);
  }
  if (s.d == 128) return launch_mark_t<float, 128>(s, q, K, tau, bits, status, st);
  return launch_mark_t<float, 64>(s, q, K, tau, bits, status, st);
}

cudaError_t launch_score(const Shape &s, const void *q, const void *K, float *S, uint32_t *hist,
                         const CandArgs *cand, uint32_t *status, cudaStream_t st) {
  if (s.dtype == 1) {
    if (s.d == 128)
      return launch_score_t<__nv_bfloat16, 128>(s, q, K, S, hist, cand, status, st);
    return launch_score_t<__nv_bfloat16, 64>(s, q, K, S, hist, cand, status, st);
  }
  if (s.d == 128) return launch_score_t<float, 128>(s, q, K, S, hist, cand, status, st);
  return launch_score_t<float, 64>(s, q, K, S, hist, cand, status, st);
}

int scan_stage_keys(const Shape &s) { return kScanStageBytes / (s.d * s.esize()); }

int scan_grid(const Shape &s, int sm_count) {
  const int stage_keys = scan_stage_keys(s);
  const long long tph = (s.N + stage_keys - 1) / stage_keys;
  const long long total = (long long)s.BH() * tph;
  return (int)(total < sm_count ? total : sm_count);
}

// Candidate lists apply when every scan CTA covers at most kCandSlots heads,
// a head spreads over few enough CTAs for the select to take all its lists,
// the lists fit their workspace area (cand_list_bytes), a head has enough
// tiles to sample, and the sample bound keeps a small share of the keys: the
// sample warp draws it from the first smp_min sample keys counted (a quarter
// of the sample, at least 512) with c* = mu + 4 sqrt(mu) + 4, mu = k * m / N
// the sample keys expected in the top k; the plan asks c* <= smp_min / 4.
bool plan_cand(const Shape &s, int k, int sm_count, CandArgs *cand) {
  const int stage_keys = scan_stage_keys(s);
  const int tph = (s.N + stage_keys - 1) / stage_keys;
  const long long total = (long long)s.BH() * tph;
  const int grid = scan_grid(s, sm_count);
  if (grid > kScanMaxGrid || tph < 8 || k < 1) return false;
  const int hctas = cand_head_ctas_of(s);
  if (hctas <= 0 || cand_head_ctas(tph, total, grid) > hctas) return false;
  const int stride = tph / kSampleTiles > 1 ? tph / kSampleTiles : 1;
  const int ns = (tph + stride - 1) / stride;
  const long long u_last = (long long)(ns - 1) * stride;
  const long long nk_last = s.N - u_last * stage_keys < stage_keys ? s.N - u_last * stage_keys
                                                                   : stage_keys;
  const long long smp_keys = (long long)(ns - 1) * stage_keys + nk_last;
  const long long smp_min = smp_keys / 4 > 512 ? smp_keys / 4 : (smp_keys < 512 ? smp_keys : 512);
  const double mu = (double)k * (double)smp_min / (double)s.N;
  const long long c_star = (long long)(mu + 4.0 * __builtin_sqrt(mu) + 4.0) + 1;
  if (c_star > smp_min / 4) return false;
  for (int cta = 0; cta < grid; ++cta) {
    const long long b = scan_tile_begin(cta, total, grid);
    const long long e = scan_tile_begin(cta + 1, total, grid);
    if ((e - 1) / tph - b / tph + 1 > kCandSlots) return false;
  }
  // entries per list read before the lengths are known: a power of two with
  // every list's share in 8 loads of 16 bytes per select thread
  const int nl = hctas;
  int spec = 2;
  while (spec * 2 <= kCandListCap && (long long)nl * spec * 2 <= 8 * 1024) spec *= 2;
  cand->grid = grid;
  cand->tiles_per_head = tph;
  cand->total_tiles = total;
  cand->head_ctas = hctas;
  cand->spec = spec;
  cand->smp_stride = stride;
  cand->smp_keys = (uint32_t)smp_keys;
  cand->smp_min = (uint32_t)smp_min;
  cand->k_over_n = (float)((double)k / (double)s.N);
  return true;
}

// The CTAs a head can span (worst case over grids up to kScanMaxGrid), or 0
// when candidate lists do not apply to the shape (too short a head, too
// many lists per head, or a list area above kCandMaxListBytes).
int cand_head_ctas_of(const Shape &s) {
  const int stage_keys = scan_stage_keys(s);
  const long long tph = (s.N + stage_keys - 1) / stage_keys;
  const long long total = (long long)s.BH() * tph;
  if (tph < 8) return 0;
  const int g = total < kScanMaxGrid ? (int)total : kScanMaxGrid;
  const int hc = cand_head_ctas(tph, total, g);
  if (hc > kCandMaxLists) return 0;
  if ((size_t)s.BH() * hc * kCandListCap * 8 > kCandMaxListBytes) return 0;
  return hc;
}

size_t cand_list_bytes(const Shape &s) {
  return (size_t)s.BH() * cand_head_ctas_of(s) * kCandListCap * 8;
}

size_t cand_count_bytes(const Shape &s) {
  return (size_t)s.BH() * cand_head_ctas_of(s) * 4;
}

}  // namespace sd
