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
//    streams tiles into a 6-stage shared-memory ring with 1-D bulk copies
//    (cp.async.bulk + mbarrier transaction counts, L2 evict-first: K is read
//    once).  Two groups of four consumer warps take alternate stages and read
//    them back with conflict-free 128-bit shared loads.
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
                           2 * kScanStages * 8 + kScanStages * 8;

template <typename T, int D>
__global__ void __launch_bounds__(kScanThreads, 1)
    score_kernel(const T *__restrict__ q, const T *__restrict__ K,
                 float *__restrict__ S, int N, int kv_rows, int Hq, int Hkv,
                 int tiles_per_head, long long total_tiles, float scale,
                 uint32_t *__restrict__ hist, uint32_t *ctr, uint32_t *status) {
  extern __shared__ __align__(128) unsigned char smem[];
  uint32_t *shist = reinterpret_cast<uint32_t *>(smem + kScanStages * kScanStageBytes);
  uint64_t *full = reinterpret_cast<uint64_t *>(
      smem + kScanStages * kScanStageBytes + kHistSlots * kScanBins * 4);
  uint64_t *empty = full + kScanStages;
  int2 *sinfo = reinterpret_cast<int2 *>(empty + kScanStages);

  const long long t_begin = scan_tile_begin(blockIdx.x, total_tiles, gridDim.x);
  const long long t_end = scan_tile_begin(blockIdx.x + 1, total_tiles, gridDim.x);
  const int bh_first = (int)(t_begin / tiles_per_head);

  if (hist) {
    for (int i = threadIdx.x; i < kHistSlots * kScanBins; i += blockDim.x) shist[i] = 0u;
  }
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
  o.S = S;
  o.hist = hist;
  o.shist = shist;
  o.bits = nullptr;
  o.tau = nullptr;
  scan_tiles<T, D, kHistSlots, false>(q, K, N, kv_rows, Hq, Hkv, tiles_per_head, total_tiles,
                                      t_begin, t_end, bh_first, scale, smem, full, empty, sinfo,
                                      ctr, o, status);
  if (threadIdx.x >= kScanConsumerWarps * 32) return;  // producer warp
  if (hist) {
    // consumer warps only (named barrier 1): every count is in shared memory
    asm volatile("bar.sync 1, %0;" ::"r"(kScanConsumerWarps * 32) : "memory");
    // every slot that names a head may hold counts: tiles of the head after
    // this CTA's own run can be claimed from a neighbour's run
    const int nheads = (int)(total_tiles / tiles_per_head);
    const int nslots = min(kHistSlots, nheads - bh_first);
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
                          float scale, uint32_t *ctr, uint32_t *status) {
  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kScanStages * kScanStageBytes);
  uint64_t *empty = full + kScanStages;
  int2 *sinfo = reinterpret_cast<int2 *>(empty + kScanStages);
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
  scan_tiles<T, D, kHistSlots, true>(q, K, N, kv_rows, Hq, Hkv, tiles_per_head, total_tiles,
                                     t_begin, t_end, (int)(t_begin / tiles_per_head), scale, smem,
                                     full, empty, sinfo, ctr, o, status);
}

template <typename T, int D>
cudaError_t launch_mark_t(const Shape &s, const void *q, const void *K, const float *tau,
                          uint32_t *bits, uint32_t *status, cudaStream_t st) {
  using C = ScoreCfg<T, D>;
  DeviceInfo di;
  cudaError_t e = device_info(&di);
  if (e != cudaSuccess) return e;
  constexpr int kSmem = kScanStages * kScanStageBytes + 2 * kScanStages * 8 + kScanStages * 8;
  auto kern = threshold_mark_kernel<T, D>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  const int tiles_per_head = (s.N + C::kStageKeys - 1) / C::kStageKeys;
  const long long total = (long long)s.BH() * tiles_per_head;
  const int grid = scan_grid(s, di.sm_count);
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
                         bits, s.N, s.Ncap, s.Hq, s.Hkv, tiles_per_head, total, scale,
                         scan_counters(status), status);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_score_t(const Shape &s, const void *q, const void *K, float *S,
                           uint32_t *hist, uint32_t *status, cudaStream_t st) {
  using C = ScoreCfg<T, D>;
  DeviceInfo di;
  cudaError_t e = device_info(&di);
  if (e != cudaSuccess) return e;
  auto kern = score_kernel<T, D>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kScoreSmem);
  if (e != cudaSuccess) return e;
  const int tiles_per_head = (s.N + C::kStageKeys - 1) / C::kStageKeys;
  const long long total = (long long)s.BH() * tiles_per_head;
  const int grid = scan_grid(s, di.sm_count);
  const float scale = (float)(1.0 / __builtin_sqrt((double)D));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3(kScanThreads, 1, 1);
  cfg.dynamicSmemBytes = kScoreSmem;
  cfg.stream = st;
  cudaLaunchAttribute attrs[1];
  cfg.attrs = attrs;
  cfg.numAttrs = 0;
  add_pdl_attr(cfg, attrs);
  e = cudaLaunchKernelEx(&cfg, kern, static_cast<const T *>(q), static_cast<const T *>(K), S,
                         s.N, s.Ncap, s.Hq, s.Hkv, tiles_per_head, total, scale, hist,
                         scan_counters(status), status);
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
                         uint32_t *status, cudaStream_t st) {
  if (s.dtype == 1) {
    if (s.d == 128) return launch_score_t<__nv_bfloat16, 128>(s, q, K, S, hist, status, st);
    return launch_score_t<__nv_bfloat16, 64>(s, q, K, S, hist, status, st);
  }
  if (s.d == 128) return launch_score_t<float, 128>(s, q, K, S, hist, status, st);
  return launch_score_t<float, 64>(s, q, K, S, hist, status, st);
}

int scan_stage_keys(const Shape &s) { return kScanStageBytes / (s.d * s.esize()); }

int scan_grid(const Shape &s, int sm_count) {
  const int stage_keys = scan_stage_keys(s);
  const long long tph = (s.N + stage_keys - 1) / stage_keys;
  const long long total = (long long)s.BH() * tph;
  const int cap = sm_count < kScanMaxCtas ? sm_count : kScanMaxCtas;
  return (int)(total < cap ? total : cap);
}

}  // namespace sd
