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

namespace sd {
namespace {

constexpr int kConsumerWarps = 4;
constexpr int kStages = 5;
constexpr int kStageBytes = 32768;
constexpr int kScoreThreads = (kConsumerWarps + 1) * 32;
constexpr int kHistBins = 2048;
constexpr int kHistSlots = 4;  // heads a CTA can count in shared memory
constexpr int kScoreSmem =
    kStages * kStageBytes + kHistSlots * kHistBins * 4 + 2 * kStages * 8;

template <typename T, int D>
struct ScoreCfg {
  static constexpr int kRowBytes = D * (int)sizeof(T);
  static constexpr int kEpl = 16 / (int)sizeof(T);  // elements per 16 B
  static constexpr int kLpk = D / kEpl;              // lanes per key row
  static constexpr int kKpr = 32 / kLpk;             // keys per round
  static constexpr int kStageKeys = kStageBytes / kRowBytes;
  static constexpr int kWarpTiles = kStageKeys / 32;
  static_assert(kKpr * kRowBytes == 512, "a round covers 512 contiguous bytes");
  static_assert(kWarpTiles >= 1, "stage holds at least one warp tile");
};

// Transposing reduction: on entry v[0..R) are per-lane partial sums of R
// different keys; partners `O` lanes apart exchange halves.  On exit v[0]
// holds the sum over 2*O... lanes of key index (lane % (2*O_top)).
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

template <typename T, int D>
__global__ void __launch_bounds__(kScoreThreads, 1)
    score_kernel(const T *__restrict__ q, const T *__restrict__ K,
                 float *__restrict__ S, int N, int Hq, int Hkv,
                 int tiles_per_head, long long total_tiles, float scale,
                 uint32_t *__restrict__ hist, uint32_t *status) {
  using C = ScoreCfg<T, D>;
  extern __shared__ __align__(128) unsigned char smem[];
  uint32_t *shist = reinterpret_cast<uint32_t *>(smem + kStages * kStageBytes);
  uint64_t *full = reinterpret_cast<uint64_t *>(
      smem + kStages * kStageBytes + kHistSlots * kHistBins * 4);
  uint64_t *empty = full + kStages;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long t_begin = (long long)blockIdx.x * total_tiles / gridDim.x;
  const long long t_end = (long long)(blockIdx.x + 1) * total_tiles / gridDim.x;
  const int ntiles = (int)(t_end - t_begin);
  const int bh_first = (int)(t_begin / tiles_per_head);

  if (hist) {
    for (int i = threadIdx.x; i < kHistSlots * kHistBins; i += kScoreThreads)
      shist[i] = 0u;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();
  grid_dep_wait();
  grid_dep_launch();

  if (warp == kConsumerWarps) {
    // ---- producer: one thread issues the bulk copies -----------------------
    if (lane == 0) {
      const uint64_t pol = l2_evict_first_policy();
      int issued = 0;
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % kStages;
        if (i >= kStages &&
            !mbar_wait(&empty[s], ((i / kStages) - 1) & 1, status))
          break;
        const long long t = t_begin + i;
        const int bh = (int)(t / tiles_per_head);
        const int j0 = (int)(t % tiles_per_head) * C::kStageKeys;
        const int nk = min(C::kStageKeys, N - j0);
        const uint32_t bytes = (uint32_t)nk * C::kRowBytes;
        mbar_arrive_expect_tx(&full[s], bytes);
        bulk_g2s(smem + (size_t)s * kStageBytes, K + ((size_t)bh * N + j0) * D,
                 bytes, &full[s], pol);
        ++issued;
      }
      // Do not leave while copies may still be landing in shared memory.
      for (int i = max(0, issued - kStages); i < issued; ++i)
        mbar_wait(&full[i % kStages], (i / kStages) & 1, status);
    }
    return;
  }

  // ---- consumers ------------------------------------------------------------
  const int sub = lane % C::kLpk;  // which 16-byte slice of the row
  int cur_bh = -1;
  float qs[C::kEpl];
  for (int i = 0; i < ntiles; ++i) {
    const int s = i % kStages;
    const long long t = t_begin + i;
    const int bh = (int)(t / tiles_per_head);
    const int j0 = (int)(t % tiles_per_head) * C::kStageKeys;
    const int nk = min(C::kStageKeys, N - j0);
    if (bh != cur_bh) {
      cur_bh = bh;
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
    if (!mbar_wait(&full[s], (i / kStages) & 1, status)) break;
    const unsigned char *stage = smem + (size_t)s * kStageBytes;
    float *Srow = S + (size_t)bh * N + j0;
    for (int wt = warp; wt < C::kWarpTiles; wt += kConsumerWarps) {
      const int key0 = wt * 32;
      if (key0 >= nk) break;
      const unsigned char *base = stage + (size_t)key0 * C::kRowBytes + lane * 16;
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
      const int kk = key0 + sub * C::kKpr + lane / C::kLpk;
      const bool valid = kk < nk;
      if (valid) {
        Srow[kk] = v[0];
        if (hist) {
          const uint32_t bin = order_key(v[0]) >> 21;
          const int slot = bh - bh_first;
          if (slot < kHistSlots)
            atomicAdd(&shist[slot * kHistBins + bin], 1u);
          else
            atomicAdd(&hist[(size_t)bh * kHistBins + bin], 1u);
        }
      }
      if (__any_sync(0xffffffffu, valid && !isfinite(v[0])) && lane == 0)
        raise_flag(status, FLAG_NONFINITE);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
  if (hist) {
    // consumer warps only (named barrier 1): every count is in shared memory
    asm volatile("bar.sync 1, %0;" ::"r"(kConsumerWarps * 32) : "memory");
    const int bh_last = ntiles > 0 ? (int)((t_end - 1) / tiles_per_head) : bh_first - 1;
    const int nslots = min(kHistSlots, bh_last - bh_first + 1);
    for (int i = threadIdx.x; i < nslots * kHistBins; i += kConsumerWarps * 32) {
      const uint32_t c = shist[i];
      if (c) atomicAdd(&hist[(size_t)(bh_first + i / kHistBins) * kHistBins + (i % kHistBins)], c);
    }
  }
}

template <typename T, int D>
cudaError_t launch_score_t(const Shape &s, const void *q, const void *K,
                           float *S, uint32_t *hist, uint32_t *status,
                           cudaStream_t st) {
  using C = ScoreCfg<T, D>;
  DeviceInfo di;
  cudaError_t e = device_info(&di);
  if (e != cudaSuccess) return e;
  auto kern = score_kernel<T, D>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kScoreSmem);
  if (e != cudaSuccess) return e;
  const int tiles_per_head = (s.N + C::kStageKeys - 1) / C::kStageKeys;
  const long long total = (long long)s.BH() * tiles_per_head;
  const int grid = (int)(total < di.sm_count ? total : di.sm_count);
  const float scale = (float)(1.0 / __builtin_sqrt((double)D));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3(kScoreThreads, 1, 1);
  cfg.dynamicSmemBytes = kScoreSmem;
  cfg.stream = st;
  cudaLaunchAttribute attrs[1];
  cfg.attrs = attrs;
  cfg.numAttrs = 0;
  add_pdl_attr(cfg, attrs);
  e = cudaLaunchKernelEx(&cfg, kern, static_cast<const T *>(q), static_cast<const T *>(K), S,
                         s.N, s.Hq, s.Hkv, tiles_per_head, total, scale, hist, status);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_score(const Shape &s, const void *q, const void *K,
                         float *S, uint32_t *hist, uint32_t *status,
                         cudaStream_t st) {
  if (s.dtype == 1) {
    if (s.d == 128)
      return launch_score_t<__nv_bfloat16, 128>(s, q, K, S, hist, status, st);
    return launch_score_t<__nv_bfloat16, 64>(s, q, K, S, hist, status, st);
  }
  if (s.d == 128) return launch_score_t<float, 128>(s, q, K, S, hist, status, st);
  return launch_score_t<float, 64>(s, q, K, S, hist, status, st);
}

}  // namespace sd
