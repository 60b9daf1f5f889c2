// attn_fused.cu -- A3 + A4 (and, fused in front of them, the tail of A2 /
// A2') for bf16 on the 5th-generation tensor cores: gather attention over
// one shared index set with the accumulators in tensor memory.
//
// Every cross-decoder layer attends over the one shared index set (CLSA
// article, section CLSAの仕組み), so for one (sequence, KV head) the M = L*G
// query vectors of all layers and query heads form one dense block against
// the same gathered keys: S = Q K^T and O = P V are real dense contractions.
//
// Grid (key splits, query blocks, sequence x KV head); the splits of a head
// form one thread-block cluster.  Each CTA first learns its share of the
// head's index set (its split is a contiguous run of the set in ascending
// key order), in one of three ways:
//  * given sets (sparse_attn_gather): from the caller's idx rows, a chunk at
//    a time;
//  * top-k routing (sparse_decode_step): the head's CTAs run the split
//    select of topk_split.cuh on the routing scan's histogram and score row
//    -- each classifies its own run of the row, the boundary bin's keys are
//    exchanged through distributed shared memory -- and each keeps the
//    selected keys of its own run on chip (their positions in the set come
//    with them) and writes them to the caller's idx row; after one more
//    cluster barrier each CTA takes an equal share of the set's positions,
//    reading the indices from their owners' lists, so the CTAs run equal
//    numbers of chunks and split the set exactly as the gather call does;
//  * threshold routing: every CTA counts the marking scan's bitmap of keys
//    with score >= tau (Louver summary, 1. 半空間範囲検索への帰着) and keeps
//    an equal share of the ascending set; rank 0 writes the count.
// Either way the set never makes a round trip through global memory before
// the attention, and no kernel boundary separates the select from it.
//
// Then, per chunk of up to 128 keys:
//  1. 16-byte async copies gather the chunk's K and V rows straight into
//     128-byte-swizzled shared-memory tiles (the canonical K-major layout for
//     K, the MN-major layout for V -- the same bytes, read two ways).
//  2. One thread issues tcgen05.mma (kind::f16, bf16 in, fp32 accumulate,
//     M = 128, N = 64 keys per tile) for S into tensor memory.
//  3. Query row i lives in tensor-memory lane i; the four warps sharing a
//     lane quadrant split each 64-key tile in quarters, take the exact row
//     maximum of the chunk (joined through shared memory), and write P =
//     exp2(S*scale*log2e - max) as two bf16 parts (P = P_hi + P_lo, about 16
//     significant bits) into swizzled shared memory over the dead K tiles.
//  4. One thread issues O += P_hi V + P_lo V into tensor memory.
// A running maximum rescales O between chunks.  With one split the CTA
// normalises O and writes the output; with several, each CTA writes its
// partial (O, max, sum) to the workspace, and after a cluster barrier each
// merges a share of the rows by log-sum-exp, reading every split's partial
// from L2.  Only hardware cluster barriers join the CTAs, so no CTA ever
// waits for one that is not resident.
//
// Query blocks of at most 64 rows (L*G <= 64, the usual decode shape) keep
// only the 64 real rows of Q and P on chip: the MMA still reads 128 rows, and
// rows 64..127 land on other live buffers -- harmless, since a row of the
// MMA's A operand only feeds the same row of its result, and rows 64..127 of
// S and O are never read.  That halves Q and P, so two CTAs fit on an SM.
//
// Every mbarrier wait is bounded; on expiry the kernel raises the TIMEOUT
// flag, stops issuing work, still meets its cluster barriers, frees its
// tensor memory and returns.
#include <atomic>

#include "common.cuh"
#include "internal.h"
#include "topk_split.cuh"

namespace sd {
namespace {

constexpr int kFuThreads = kTkThreads;  // 512: 16 warps, 4 per TMEM lane quadrant
constexpr int kGroups = 4;              // warps sharing a tensor-memory lane quadrant
constexpr int kTileN = 64;              // keys per S tile (MMA N of QK^T, K of PV)
constexpr int KPT = kTileN / kGroups;   // keys per thread of each tile
constexpr int kChunkTiles = 2;
constexpr int kChunkKeys = kTileN * kChunkTiles;
constexpr int kTmemCols = 256;          // S (128 columns) + O (d <= 128 columns)
constexpr int kMaxSplits = 16;
constexpr int kMaxPer = 2048;           // keys of one split held on chip (routing modes)
constexpr int kFuSlotBound = 512;       // CTA slots the split count may spread a head block over
static_assert(kMaxSplits == kTsMaxSplits, "a head's cluster is the select's cluster");
constexpr int kMaxDevices = 64;

constexpr int cmax_i(int a, int b) { return a > b ? a : b; }

template <int D, bool kHalf>
struct FuCfg {
  static constexpr int kRows = kHalf ? 64 : 128;       // query rows kept on chip
  static constexpr int kQCb = kRows * 128;             // one 64-column block of Q
  static constexpr int kQBytes = (D / 64) * kQCb;
  static constexpr int kKTile = kTileN * D * 2;        // one 64-key tile of K or V
  static constexpr int kPTile = 2 * kRows * 128;       // P_hi and P_lo of one tile
  static constexpr int kKPBytes = cmax_i(kChunkTiles * kKTile, kChunkTiles * kPTile);
  static constexpr int kVBytes = kChunkTiles * kKTile;
  static constexpr int kQOff = 0;
  static constexpr int kKPOff = kQBytes;
  static constexpr int kVOff = kKPOff + kKPBytes;
  static constexpr int kAttnBytes = kVOff + kVBytes;
  // the select's scratch sits after Q (whose copy starts before the select)
  static constexpr int kSelOff = kQBytes;
  static constexpr int kSelBytes = (int)ts_scratch_bytes();
  static constexpr int kBigBytes = cmax_i(kAttnBytes, kSelOff + kSelBytes);
  // small area: barriers, TMEM slot, select bookkeeping, row reductions,
  // validity flags, chunk indices, the split's indices, and what the select
  // shows its peers
  static constexpr int kSmallOff = (kBigBytes + 1023) / 1024 * 1024;
  static constexpr int kBarsOff = 0, kTmemSlotOff = 64, kTkOff = 128, kXredOff = 512;
  static constexpr int kKvalOff = kXredOff + kGroups * 128 * 4;
  static constexpr int kCidxOff = kKvalOff + kChunkKeys;
  static constexpr int kSidxOff = kCidxOff + kChunkKeys * 4;
  static constexpr int kShowOff = kSidxOff + kMaxPer * 4;
  static constexpr int kBookOff = kShowOff + (int)sizeof(TsShow);
  static constexpr int kSmallBytes = kBookOff + (int)sizeof(TsBook);
  // merge scratch in the (then free) tile buffers: [kFuThreads] float4 + [kFuThreads] float
  static_assert(kFuThreads * 20 <= kBigBytes, "merge scratch fits");
  static constexpr int kSmem = kSmallOff + kSmallBytes + 1024;  // + alignment slack
  static_assert(sizeof(TkSmall) <= kXredOff - kTkOff, "select bookkeeping fits");
};

// ---- tcgen05 helpers --------------------------------------------------------
// ---- tcgen05 helpers --------------------------------------------------------
// Shared-memory matrix descriptor: 128-byte swizzle, version 1 (sm_100).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo,
                                               uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;  // descriptor version for sm_100
  d |= (uint64_t)2 << 61;  // SWIZZLE_128B
  return d;
}

// Instruction descriptor for kind::f16 with bf16 A/B and fp32 D.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a, uint64_t b,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
      ::"r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t *r) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
               : "r"(taddr));
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t *r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
               :: "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
               : "memory");
}

__device__ __forceinline__ void cp_async16(uint32_t saddr, const void *gmem, bool pred) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(saddr),
               "l"(gmem), "r"(pred ? 16u : 0u)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// 2^x with the hardware approximation (ex2.approx.ftz: relative error about
// 2^-22, results below 2^-126 flush to zero -- harmless for softmax weights).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

// Byte offset of 16-byte chunk c (0..7) of row r inside a 128B-swizzled
// block of 128-byte rows.
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4));
}


// Everything the fused kernel needs (one struct, passed as a grid constant).
struct FuArgs {
  const __nv_bfloat16 *q, *K, *V;
  int *idx;        // given sets (read) or the routed sets (written), rows of `stride`
  int stride;
  int *count;      // given set sizes (nullable: all `stride`) / threshold counts (written)
  int N, kv_rows, B, Hq, Hkv, L;
  float scale_log2;
  __nv_bfloat16 *out;
  float *lse;
  uint32_t *status;
  const float *S;        // top-k: score rows
  uint32_t *hist;        // top-k: the scan's histograms (cleared here)
  const uint32_t *bits;  // threshold: the marking scan's bitmaps
  int k_or_cap;
  float *part;           // several splits: their partials, fu_workspace_bytes()
};

enum : int { kModeIdx = 0, kModeTopk = 1, kModeThresh = 2 };

template <int D, bool kHalf, int kMode>
__global__ void __launch_bounds__(kFuThreads, kHalf ? 2 : 1)
    attn_fused_kernel(const __grid_constant__ FuArgs a) {
  using C = FuCfg<D, kHalf>;
  constexpr int KSTEPS = D / 16;  // MMA k-steps of S = Q K^T
  constexpr int CPR = D / 8;      // 16-byte chunks per K/V/Q row
  const int nsplit = (int)gridDim.x, rank = (int)blockIdx.x;
  const int qb = blockIdx.y, bh = blockIdx.z;
  const int N = a.N, Hq = a.Hq, Hkv = a.Hkv, B = a.B;
  const int b = bh / Hkv, h = bh % Hkv, G = Hq / Hkv;
  const int M = a.L * G;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quad = warp & 3, grp = warp >> 2;
  const int row = quad * 32 + lane;
  // warps whose tensor-memory lanes hold rows kept on chip (warp-uniform)
  const bool live = row - lane < C::kRows;

  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t base_s = (raw_s + 1023u) & ~1023u;  // swizzle atoms need 1 KB alignment
  unsigned char *base = smem_raw + (base_s - raw_s);
  const uint32_t q_s = base_s + C::kQOff;
  const uint32_t kp_s = base_s + C::kKPOff;
  const uint32_t v_s = base_s + C::kVOff;
  unsigned char *small = base + C::kSmallOff;
  uint64_t *bars = reinterpret_cast<uint64_t *>(small + C::kBarsOff);  // S done, chunk done
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(small + C::kTmemSlotOff);
  TkSmall *tks = reinterpret_cast<TkSmall *>(small + C::kTkOff);
  float *xred = reinterpret_cast<float *>(small + C::kXredOff);  // [kGroups][128]
  unsigned char *kval = small + C::kKvalOff;                      // [128] valid flags
  int *cidx = reinterpret_cast<int *>(small + C::kCidxOff);       // [128] chunk indices
  int *sidx = reinterpret_cast<int *>(small + C::kSidxOff);       // [kMaxPer] this split's keys
  TsShow *show = reinterpret_cast<TsShow *>(small + C::kShowOff);
  TsBook *book = reinterpret_cast<TsBook *>(small + C::kBookOff);

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(tmem_slot)), "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
    for (int i = 0; i < 2; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // The query block (rows beyond M zero) into its swizzled tile.  In the
  // routing modes the kernel before this one on the stream is the routing
  // scan, which never writes the queries and released this launch only once
  // every kernel before it had finished: the copy starts before the wait for
  // the scan, in a copy group of its own.
  auto issue_q = [&]() {
    for (int p = tid; p < C::kRows * CPR; p += kFuThreads) {
      const int r = p / CPR, c = p % CPR;
      const int m = qb * 128 + r;
      const __nv_bfloat16 *qr = nullptr;
      if (m < M) qr = a.q + (((size_t)(m / G) * B + b) * Hq + (size_t)h * G + m % G) * D;
      const uint32_t dst = q_s + (c >> 3) * C::kQCb + swz(r, c & 7);
      cp_async16(dst, qr ? qr + c * 8 : a.q, qr != nullptr);
    }
  };
  if constexpr (kMode != kModeIdx) {
    issue_q();
    cp_async_commit();
  }
  grid_dep_wait();  // sets, scores, bitmaps and queries come from earlier kernels
  grid_dep_launch();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_S = tmem;               // columns [0, 128)
  const uint32_t t_O = tmem + kChunkKeys;  // columns [128, 128 + D)
  const uint32_t lane_off = (uint32_t)(quad * 32) << 16;

  // ---- this split's part [lo, lo + nmine) of the head's set ---------------------
  int lo = 0, nmine = 0;
  bool from_peers = false;  // the split's keys are read from their owners' lists
  int *orow = a.idx + (size_t)bh * a.stride;
  if constexpr (kMode == kModeTopk) {
    auto emit = [&](uint32_t i, uint32_t pos, uint32_t j) {
      sidx[i] = (int)j;
      if (qb == 0) orow[pos] = (int)j;
    };
    const TsOut part = ts_select(a.S + (size_t)bh * N, N, (uint32_t)a.k_or_cap,
                                 a.hist + (size_t)bh * kHistBins, rank, nsplit, kMaxPer,
                                 base + C::kSelOff, show, book, tks, a.status, emit);
    __syncthreads();  // the split's indices are on chip; the select's scratch is free
    if (part.split && nsplit > 1) {
      // the runs hold unequal parts of the set: every CTA attends over an
      // equal share instead (so each runs the same number of chunks), its
      // indices read from their owners' lists chunk by chunk once every
      // list is complete; the owners keep their lists until the merge's
      // first cluster barrier
      cluster_sync_all();
      const int per = (a.k_or_cap + nsplit - 1) / nsplit;
      lo = min(a.k_or_cap, rank * per);
      nmine = min(a.k_or_cap, lo + per) - lo;
      from_peers = true;
    } else {
      lo = (int)part.lo;
      nmine = (int)part.n;
    }
    // with one split this CTA was the head's only reader: clear the scan's
    // histogram for the next call now (with several, after the merge's first
    // cluster barrier)
    if (nsplit == 1)
      for (int i = tid; i < kHistBins; i += kFuThreads) a.hist[(size_t)bh * kHistBins + i] = 0u;
  } else {
    int cnt = 0;
    if constexpr (kMode == kModeIdx) {
      cnt = a.count ? min(max(a.count[bh], 0), a.stride) : a.stride;
    } else {
      // threshold: the set is the marking scan's bitmap of the head
      const int nw = (N + 31) / 32;
      const uint32_t *words = a.bits + (size_t)bh * nw;
      uint32_t n = 0;
      for (int w = tid; w < nw; w += kFuThreads) n += __popc(words[w]);
      uint32_t total;
      tk_scan(n, tks, &total);
      cnt = (int)min(total, (uint32_t)a.k_or_cap);
      if (rank == 0 && qb == 0 && tid == 0) {
        a.count[bh] = (int)total;
        if (total > (uint32_t)a.k_or_cap) raise_flag(a.status, FLAG_CAPACITY);
      }
    }
    const int per = (cnt + nsplit - 1) / nsplit;
    lo = min(cnt, rank * per);
    const int hi = min(cnt, lo + per);
    nmine = hi - lo;
    if constexpr (kMode == kModeThresh) {
      auto emit = [&](uint32_t pos, uint32_t j) {
        if (pos >= (uint32_t)lo && pos < (uint32_t)hi) {
          sidx[pos - lo] = (int)j;
          if (qb == 0) orow[pos] = (int)j;
        }
      };
      const int nw = (N + 31) / 32;
      tk_bitmap_emit(a.bits + (size_t)bh * nw, nw, tks, emit, (uint32_t)lo, (uint32_t)hi);
      __syncthreads();  // the split's indices are on chip
    }
  }
  const size_t head_off = (size_t)bh * a.kv_rows * D;

  bool failed = false;
  float mrun = -INFINITY, lsum = 0.f;
  uint32_t phase_s = 0, phase_done = 0;
  bool first_pv = true;
  const uint32_t idS = idesc_bf16(128, kTileN, false);
  const uint32_t idPV = idesc_bf16(128, D, true);

  for (int c0 = 0; c0 < nmine && !failed; c0 += kChunkKeys) {
    const int nk = min(kChunkKeys, nmine - c0);
    const int ntile = (nk + kTileN - 1) / kTileN;
    const int *cix = sidx + c0;
    if constexpr (kMode == kModeIdx) {
      if (tid < kChunkKeys) cidx[tid] = tid < nk ? orow[lo + c0 + tid] : -1;
      __syncthreads();
      cix = cidx;
    } else if constexpr (kMode == kModeTopk) {
      if (from_peers) {
        if (tid < kChunkKeys) {
          int j = -1;
          if (tid < nk) {
            const uint32_t pos = (uint32_t)(lo + c0 + tid);
            int o = 0, hi2 = nsplit - 1;  // the last CTA whose part starts at or before pos
            while (o < hi2) {
              const int mid = (o + hi2 + 1) >> 1;
              if (book->part_lo[mid] <= pos) o = mid;
              else hi2 = mid - 1;
            }
            const uint32_t i = pos - book->part_lo[o];
            j = o == rank ? sidx[i] : (int)cl_ld_u32(cl_addr(sidx + i, o));
          }
          cidx[tid] = j;
        }
        __syncthreads();
        cix = cidx;
      }
    }
    if (c0 == 0 && kMode == kModeIdx) issue_q();  // in the same copy group as K
    // gather the chunk's K rows, then its V rows (two async-copy groups)
    for (int p = tid; p < ntile * kTileN * CPR; p += kFuThreads) {
      const int r = p / CPR, c = p % CPR;
      const int j = r < nk ? cix[r] : -1;
      const bool ok = r < nk && j >= 0 && j < N;
      if (r < nk && !ok && c == 0) raise_flag(a.status, FLAG_INDEX);
      if (c == 0) kval[r] = ok;
      const uint32_t dst = kp_s + (r >> 6) * C::kKTile + (c >> 3) * (kTileN * 128) +
                           swz(r & 63, c & 7);
      cp_async16(dst, a.K + head_off + (size_t)(ok ? j : 0) * D + c * 8, ok);
    }
    cp_async_commit();
    for (int p = tid; p < ntile * kTileN * CPR; p += kFuThreads) {
      const int r = p / CPR, c = p % CPR;
      const int j = r < nk ? cix[r] : -1;
      const bool ok = r < nk && j >= 0 && j < N;
      const uint32_t dst = v_s + (r >> 6) * C::kKTile + (c >> 3) * (kTileN * 128) +
                           swz(r & 63, c & 7);
      cp_async16(dst, a.V + head_off + (size_t)(ok ? j : 0) * D + c * 8, ok);
    }
    cp_async_commit();
    cp_async_wait<1>();  // Q and K have landed (this thread's copies)
    fence_async_smem();  // make them visible to the tensor-core proxy
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- S = Q K^T for every tile of the chunk, one issuing thread -----------
    if (tid == 0) {
      for (int t = 0; t < ntile; ++t) {
#pragma unroll
        for (int s = 0; s < KSTEPS; ++s) {
          const uint64_t qa = sw128_desc(q_s + (s >> 2) * C::kQCb + (s & 3) * 32, 16, 1024);
          const uint64_t kb = sw128_desc(
              kp_s + t * C::kKTile + (s >> 2) * (kTileN * 128) + (s & 3) * 32, 16, 1024);
          mma_f16(t_S + t * kTileN, qa, kb, idS, s > 0 ? 1u : 0u);
        }
      }
      mma_commit(&bars[0]);
    }
    // validity of this thread's KPT keys of each tile, as bit masks
    uint32_t vmask[kChunkTiles];
#pragma unroll
    for (int t = 0; t < kChunkTiles; ++t) {
      constexpr int PER32 = 32 / KPT;  // groups covered by one 32-key ballot
      const int key = t * kTileN + (grp / PER32) * 32 + lane;
      const uint32_t bm = __ballot_sync(0xffffffffu, key < nk && kval[key] != 0);
      vmask[t] = (bm >> ((grp % PER32) * KPT)) & ((1u << KPT) - 1u);
    }
    if (!mbar_wait(&bars[0], phase_s & 1u, a.status)) failed = true;
    ++phase_s;
    tc_fence_after();
    if (__syncthreads_or(failed)) {
      failed = true;
      break;
    }

    // ---- row maximum over the chunk (four warps per row, joined in smem) ------
    float cmax = -INFINITY;
    if (live) {
#pragma unroll
      for (int t = 0; t < kChunkTiles; ++t) {
        if (t < ntile) {
          uint32_t r[KPT];
          tmem_ld16(t_S + lane_off + t * kTileN + grp * KPT, r);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < KPT; ++i)
            if ((vmask[t] >> i) & 1u) cmax = fmaxf(cmax, __uint_as_float(r[i]));
        }
      }
      xred[grp * 128 + row] = cmax;
    }
    __syncthreads();
    float muse = 0.f;
    if (live) {
#pragma unroll
      for (int g = 0; g < kGroups; ++g) cmax = fmaxf(cmax, xred[g * 128 + row]);
      cmax *= a.scale_log2;  // scale > 0
      const float mnew = fmaxf(mrun, cmax);
      muse = mnew == -INFINITY ? 0.f : mnew;
      const bool rescale = !first_pv && mnew != mrun;
      if (__any_sync(0xffffffffu, rescale)) {
        // a later chunk raised some row's max: rescale O (this warp's share of
        // the columns); tcgen05.ld/st are warp-collective, so the whole warp
        // takes this path
        const float corr = rescale ? exp2f(mrun - muse) : 1.f;
        lsum *= corr;
#pragma unroll
        for (int cb = 0; cb < D / kGroups / 16; ++cb) {
          uint32_t r[16];
          const uint32_t col = t_O + lane_off + grp * (D / kGroups) + cb * 16;
          tmem_ld16(col, r);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * corr);
          tmem_st16(col, r);
        }
        tmem_wait_st();
      }
      mrun = mnew;
    }

    // ---- P tiles (over the dead K tiles) and O += P V -------------------------
    for (int t = 0; t < ntile; ++t) {
      const uint32_t ph = kp_s + t * C::kPTile;  // hi, then lo
      const uint32_t pl = ph + C::kRows * 128;
      if (live) {
        const uint32_t vm = t == 0 ? vmask[0] : vmask[kChunkTiles - 1];
        uint32_t r[KPT];
        tmem_ld16(t_S + lane_off + t * kTileN + grp * KPT, r);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < KPT / 8; ++c) {  // 16-byte chunks of 8 keys
          uint32_t hi4[4], lo4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = c * 8 + e * 2;
            const float p0 = ((vm >> i) & 1u)
                                 ? fast_exp2(fmaf(__uint_as_float(r[i]), a.scale_log2, -muse))
                                 : 0.f;
            const float p1 =
                ((vm >> (i + 1)) & 1u)
                    ? fast_exp2(fmaf(__uint_as_float(r[i + 1]), a.scale_log2, -muse))
                    : 0.f;
            lsum += p0 + p1;
            hi4[e] = pack_bf16x2(p0, p1);
            const __nv_bfloat162 hb = *reinterpret_cast<const __nv_bfloat162 *>(&hi4[e]);
            lo4[e] = pack_bf16x2(p0 - __low2float(hb), p1 - __high2float(hb));
          }
          const uint32_t off = swz(row, grp * (KPT / 8) + c);
          asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(ph + off), "r"(hi4[0]),
                       "r"(hi4[1]), "r"(hi4[2]), "r"(hi4[3])
                       : "memory");
          asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(pl + off), "r"(lo4[0]),
                       "r"(lo4[1]), "r"(lo4[2]), "r"(lo4[3])
                       : "memory");
        }
      }
      if (t == 0) cp_async_wait<0>();  // V tiles have landed (this thread's copies)
      fence_async_smem();
      tc_fence_before();
      __syncthreads();
      tc_fence_after();
      if (tid == 0) {
#pragma unroll
        for (int kk = 0; kk < kTileN / 16; ++kk) {
          const uint64_t bv = sw128_desc(v_s + t * C::kKTile + kk * 2048, kTileN * 128, 1024);
          mma_f16(t_O, sw128_desc(ph + kk * 32, 16, 1024), bv, idPV,
                  (first_pv && kk == 0) ? 0u : 1u);
          mma_f16(t_O, sw128_desc(pl + kk * 32, 16, 1024), bv, idPV, 1u);
        }
      }
      first_pv = false;
    }
    // every MMA of this chunk done before its shared memory is reused (and
    // before O is read)
    if (tid == 0) mma_commit(&bars[1]);
    if (!mbar_wait(&bars[1], phase_done & 1u, a.status)) failed = true;
    ++phase_done;
    tc_fence_after();
    if (__syncthreads_or(failed)) failed = true;
  }
  cp_async_wait<0>();

  // ---- this CTA's result --------------------------------------------------------
  const int mrows = min(C::kRows, M - qb * 128);  // real query rows of the block
  const bool have = !first_pv && !failed;
  __syncthreads();
  float *xsum = xred;  // [kGroups][128]: the warps' parts of each row's sum
  if (live) xsum[grp * 128 + row] = have ? lsum : 0.f;
  if (nsplit == 1) {
    // one split: normalise straight from tensor memory
    __syncthreads();
    if (live) {
      float ls = 0.f;
#pragma unroll
      for (int g = 0; g < kGroups; ++g) ls += xsum[g * 128 + row];
      const float inv = (have && ls > 0.f) ? 1.f / ls : 0.f;
      const int m = qb * 128 + row;
      const size_t orw = m < M ? ((size_t)(m / G) * B + b) * Hq + (size_t)h * G + m % G : 0;
#pragma unroll
      for (int cb = 0; cb < D / kGroups / 16; ++cb) {
        uint32_t r[16];
        if (have) {
          tmem_ld16(t_O + lane_off + grp * (D / kGroups) + cb * 16, r);
          tmem_wait_ld();
        }
        if (row < mrows) {
#pragma unroll
          for (int i = 0; i < 16; i += 8) {
            uint4 pk;
            pk.x = pack_bf16x2(have ? __uint_as_float(r[i]) * inv : 0.f,
                               have ? __uint_as_float(r[i + 1]) * inv : 0.f);
            pk.y = pack_bf16x2(have ? __uint_as_float(r[i + 2]) * inv : 0.f,
                               have ? __uint_as_float(r[i + 3]) * inv : 0.f);
            pk.z = pack_bf16x2(have ? __uint_as_float(r[i + 4]) * inv : 0.f,
                               have ? __uint_as_float(r[i + 5]) * inv : 0.f);
            pk.w = pack_bf16x2(have ? __uint_as_float(r[i + 6]) * inv : 0.f,
                               have ? __uint_as_float(r[i + 7]) * inv : 0.f);
            *reinterpret_cast<uint4 *>(a.out + orw * D + grp * (D / kGroups) + cb * 16 + i) = pk;
          }
        }
      }
      if (a.lse && grp == 0 && row < mrows)
        a.lse[orw] = (have && ls > 0.f) ? (mrun + log2f(ls)) * 0.69314718055994531f : -INFINITY;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                   "r"(kTmemCols)
                   : "memory");
    return;
  }

  // Several splits: each writes its partial (O, max, sum) of the real rows
  // to the workspace -- [split][row][D] fp32, then [split][row] (max, sum)
  // -- one cluster barrier (release / acquire at cluster scope) makes them
  // visible to the head's CTAs, and each CTA merges a share of the rows by
  // log-sum-exp, reading the partials from L2.  No CTA reads another's
  // shared memory after the barrier, so none waits for another to finish.
  float *pbase = a.part + (size_t)(bh * gridDim.y + qb) * nsplit * C::kRows * (D + 2);
  const float2 *pml = reinterpret_cast<const float2 *>(pbase + (size_t)nsplit * C::kRows * D);
  if (live) {
    // tcgen05.ld is warp-collective: every lane of a live warp loads (have
    // and live are warp-uniform); only the stores depend on the lane's row
    float *dst = pbase + ((size_t)rank * C::kRows + row) * D + grp * (D / kGroups);
#pragma unroll
    for (int cb = 0; cb < D / kGroups / 16; ++cb) {
      uint32_t r[16];
      if (have) {
        tmem_ld16(t_O + lane_off + grp * (D / kGroups) + cb * 16, r);
        tmem_wait_ld();
      }
      if (row < mrows) {
#pragma unroll
        for (int i = 0; i < 16; i += 4)
          *reinterpret_cast<float4 *>(dst + cb * 16 + i) =
              have ? make_float4(__uint_as_float(r[i]), __uint_as_float(r[i + 1]),
                                 __uint_as_float(r[i + 2]), __uint_as_float(r[i + 3]))
                   : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  }
  __syncthreads();
  if (live && grp == 0 && row < mrows) {
    float ls = 0.f;
#pragma unroll
    for (int g = 0; g < kGroups; ++g) ls += xsum[g * 128 + row];
    reinterpret_cast<float2 *>(pbase + (size_t)nsplit * C::kRows * D)[rank * C::kRows + row] =
        make_float2(have ? mrun : -INFINITY, ls);
  }
  // tensor memory is no longer needed
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  cluster_sync_all();  // every split's partial is in the workspace
  if constexpr (kMode == kModeTopk) {
    if (rank == 0)
      for (int i = tid; i < kHistBins; i += kFuThreads) a.hist[(size_t)bh * kHistBins + i] = 0u;
  }
  // merge rows lr = rank, rank + nsplit, ...: thread = (peer group q, row
  // slot, float4 chunk); every (max, sum) pair and the thread's peers'
  // partial O are loaded at once (L2 only: they were written by other SMs
  // during this kernel), and with several peer groups the group partials
  // are added in shared memory (the tile buffers are free now).
  {
    constexpr int CH = D / 4;
    const int nrows = (mrows - rank + nsplit - 1) / nsplit;
    int qg = 1;  // peer groups: as many as one pass of the rows leaves threads for
    while (qg < 4 && qg * 2 <= nsplit && nrows * CH * qg * 2 <= kFuThreads) qg *= 2;
    const int rpq = kFuThreads / (CH * qg);  // row slots per pass
    const int ch = tid % CH, slot = (tid / CH) % rpq, q = tid / (CH * rpq);
    float4 *red = reinterpret_cast<float4 *>(base);
    float *red_ls = reinterpret_cast<float *>(base + kFuThreads * 16);
    for (int i0 = 0; i0 < nrows; i0 += rpq) {
      const int i = i0 + slot;
      const int lr = rank + i * nsplit;
      const bool mine = i < nrows;
      float mx = -INFINITY, ls = 0.f;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      // the CH lanes of a row slot (CH >= kMaxSplits) each load one split's
      // (max, sum) pair and share them by shuffles
      float2 mlv = make_float2(-INFINITY, 0.f);
      if (mine && ch < nsplit) mlv = __ldcg(pml + ch * C::kRows + lr);
      float4 v[4];  // this thread's first peers' partial O, in flight with the pairs
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int r = q + u * qg;
        if (mine && r < nsplit)
          v[u] = __ldcg(reinterpret_cast<const float4 *>(
              pbase + ((size_t)r * C::kRows + lr) * D + ch * 4));
      }
      mx = mlv.x;
#pragma unroll
      for (int o = CH / 2; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o, CH));
      // this thread's peers q, q + qg, ..., four loads in flight at a time
      for (int r0 = q; r0 < nsplit; r0 += 4 * qg) {
        if (r0 != q) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int r = r0 + u * qg;
            if (mine && r < nsplit)
              v[u] = __ldcg(reinterpret_cast<const float4 *>(
                  pbase + ((size_t)r * C::kRows + lr) * D + ch * 4));
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int r = r0 + u * qg;
          // every lane of the row slot takes part in the shuffles
          const float mr = __shfl_sync(0xffffffffu, mlv.x, r & (CH - 1), CH);
          const float lr_sum = __shfl_sync(0xffffffffu, mlv.y, r & (CH - 1), CH);
          if (mine && r < nsplit && mx != -INFINITY) {
            const float w = mr == -INFINITY ? 0.f : fast_exp2(mr - mx);
            ls += lr_sum * w;
            acc.x += w * v[u].x;
            acc.y += w * v[u].y;
            acc.z += w * v[u].z;
            acc.w += w * v[u].w;
          }
        }
      }
      if (qg > 1) {
        red[tid] = acc;
        if (ch == 0) red_ls[tid / CH] = ls;
        __syncthreads();
        if (q == 0) {
          for (int g = 1; g < qg; ++g) {
            const float4 o = red[tid + g * CH * rpq];
            acc.x += o.x;
            acc.y += o.y;
            acc.z += o.z;
            acc.w += o.w;
            ls += red_ls[(tid + g * CH * rpq) / CH];
          }
        }
        __syncthreads();
      }
      if (mine && q == 0) {
        const float inv = ls > 0.f ? 1.f / ls : 0.f;
        const int m = qb * 128 + lr;
        const size_t orw = ((size_t)(m / G) * B + b) * Hq + (size_t)h * G + m % G;
        uint2 pk;
        pk.x = pack_bf16x2(acc.x * inv, acc.y * inv);
        pk.y = pack_bf16x2(acc.z * inv, acc.w * inv);
        *reinterpret_cast<uint2 *>(a.out + orw * D + ch * 4) = pk;
        if (a.lse && ch == 0)
          a.lse[orw] = ls > 0.f ? (mx + log2f(ls)) * 0.69314718055994531f : -INFINITY;
      }
    }
  }
}

// The kernel's dynamic shared memory, with the whole unified L1/shared
// storage given to shared memory (so two 64-row CTAs fit on an SM).
template <typename Kern>
cudaError_t fu_set_attrs(Kern kern, int smem) {
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
  return e;
}

// A kernel with the fused kernel's threads, registers bound and shared
// memory but no tensor-memory allocation: the occupancy calculator counts a
// kernel that allocates tensor memory as one CTA per SM, while two 64-row
// CTAs (256 columns each of an SM's 512) do share an SM, so cluster
// capacity is asked of this twin.
template <int D, bool kHalf>
__global__ void __launch_bounds__(kFuThreads, kHalf ? 2 : 1) attn_fused_occupancy_twin(int *p) {
  extern __shared__ unsigned char smem_raw[];
  if (p) p[threadIdx.x] = smem_raw[threadIdx.x];
}

// Clusters of nsplit CTAs the device can hold at once (the variant's
// occupancy does not depend on the mode), cached per (device, variant,
// split count).
template <int D, bool kHalf>
int fu_active_clusters(int nsplit) {
  using C = FuCfg<D, kHalf>;
  static std::atomic<int> cache[kMaxDevices][kMaxSplits + 1];  // 0 unknown, else 1 + count
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    (void)cudaGetLastError();
    return 0;
  }
  int v = cache[dev][nsplit].load(std::memory_order_relaxed);
  if (v == 0) {
    auto kern = attn_fused_occupancy_twin<D, kHalf>;
    int n = 0;
    cudaError_t e = fu_set_attrs(kern, C::kSmem);
    if (e == cudaSuccess && nsplit > 8)
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e == cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)nsplit, 1, 1);
      cfg.blockDim = dim3(kFuThreads, 1, 1);
      cfg.dynamicSmemBytes = C::kSmem;
      cudaLaunchAttribute at;
      at.id = cudaLaunchAttributeClusterDimension;
      at.val.clusterDim.x = (unsigned)nsplit;
      at.val.clusterDim.y = 1;
      at.val.clusterDim.z = 1;
      cfg.attrs = &at;
      cfg.numAttrs = 1;
      e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
    }
    if (e != cudaSuccess) {
      (void)cudaGetLastError();
      n = 0;
    }
    v = 1 + n;
    cache[dev][nsplit].store(v, std::memory_order_relaxed);
  }
  return v - 1;
}

// Key splits per head, the same for every mode of a shape (so a decode step
// and a gather over its sets split alike): enough CTAs to fill the device
// (two per SM for 64-row blocks), at least 64 keys per split, at most
// kMaxPer keys per split where that is possible with kMaxSplits splits (a
// routed split must fit on chip; routed = true refuses shapes where it does
// not), and a cluster size the device can hold -- preferably one with every
// head's cluster resident at once, or at least half the device busy.
template <int D, bool kHalf>
int fu_splits(long long blocks, int max_keys, bool routed, int sm_count) {
  const int slots = sm_count * (kHalf ? 2 : 1);
  long long want = slots / blocks;
  if (want > (kFuSlotBound + blocks - 1) / blocks) want = (kFuSlotBound + blocks - 1) / blocks;
  const int by_keys = (max_keys + kTileN - 1) / kTileN;
  if (want > by_keys) want = by_keys;
  if (want > kMaxSplits) want = kMaxSplits;
  int need = (max_keys + kMaxPer - 1) / kMaxPer;
  if (need > kMaxSplits) {
    if (routed) return 0;
    need = 1;
  }
  if (want < need) want = need;
  if (want <= 1) return 1;
  int fallback = 0;
  for (int n = (int)want; n >= need && n >= 2; --n) {
    const int act = fu_active_clusters<D, kHalf>(n);
    if (act >= blocks || 2LL * act * n >= slots) return n;
    if (act > 0 && !fallback) fallback = n;
  }
  if (fallback) return fallback;
  return need <= 1 ? 1 : 0;
}

template <int D, bool kHalf, int kMode>
cudaError_t launch_fu_t(const FuArgs &a, int BH, int qblocks, int max_keys, cudaStream_t st) {
  using C = FuCfg<D, kHalf>;
  DeviceInfo di;
  cudaError_t e = device_info(&di);
  if (e != cudaSuccess) return e;
  const int nsplit =
      fu_splits<D, kHalf>((long long)BH * qblocks, max_keys, kMode != kModeIdx, di.sm_count);
  if (nsplit < 1) return cudaErrorNotSupported;
  auto kern = attn_fused_kernel<D, kHalf, kMode>;
  e = fu_set_attrs(kern, C::kSmem);
  if (e == cudaSuccess && nsplit > 8)
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)nsplit, (unsigned)qblocks, (unsigned)BH);
  cfg.blockDim = dim3(kFuThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  cfg.attrs = attr;
  cfg.numAttrs = 0;
  if (nsplit > 1) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)nsplit;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.numAttrs = 1;
  }
  add_pdl_attr(cfg, attr);
  e = cudaLaunchKernelEx(&cfg, kern, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int D, int kMode>
cudaError_t launch_fu_d(const FuArgs &a, const Shape &s, int max_keys, cudaStream_t st) {
  const int M = a.L * s.G();
  if (M <= 64) return launch_fu_t<D, true, kMode>(a, s.BH(), 1, max_keys, st);
  return launch_fu_t<D, false, kMode>(a, s.BH(), (M + 127) / 128, max_keys, st);
}

template <int kMode>
cudaError_t launch_fu(const FuArgs &a, const Shape &s, int max_keys, cudaStream_t st) {
  if (s.d == 128) return launch_fu_d<128, kMode>(a, s, max_keys, st);
  return launch_fu_d<64, kMode>(a, s, max_keys, st);
}

FuArgs fu_base(const Shape &s, int L, const void *q, const void *K, const void *V, int *idx,
               int stride, int *count, void *out, float *lse, uint32_t *status, void *part) {
  FuArgs a{};
  a.q = static_cast<const __nv_bfloat16 *>(q);
  a.K = static_cast<const __nv_bfloat16 *>(K);
  a.V = static_cast<const __nv_bfloat16 *>(V);
  a.idx = idx;
  a.stride = stride;
  a.count = count;
  a.N = s.N;
  a.kv_rows = s.Ncap;
  a.B = s.B;
  a.Hq = s.Hq;
  a.Hkv = s.Hkv;
  a.L = L;
  a.scale_log2 = (float)(1.4426950408889634 / __builtin_sqrt((double)s.d));
  a.out = static_cast<__nv_bfloat16 *>(out);
  a.lse = lse;
  a.status = status;
  a.part = static_cast<float *>(part);
  return a;
}

}  // namespace

size_t attn_fused_workspace_bytes(const Shape &s, int L, int stride) {
  // the split count is at most kMaxSplits, one split per kTileN keys and,
  // beyond what the on-chip capacity forces, kFuSlotBound slots over the
  // head blocks (fu_splits keeps to the same bound)
  const int M = L * s.G();
  const int qblocks = M <= 64 ? 1 : (M + 127) / 128;
  const int rows = M <= 64 ? 64 : 128;
  const long long blocks = (long long)s.BH() * qblocks;
  long long ns = (kFuSlotBound + blocks - 1) / blocks;
  const long long by_keys = (stride + kTileN - 1) / kTileN;
  if (ns > by_keys) ns = by_keys;
  const long long need = (stride + kMaxPer - 1) / kMaxPer;
  if (ns < need) ns = need;
  if (ns > kMaxSplits) ns = kMaxSplits;
  if (ns < 2) return 0;  // one split: no partials
  return (size_t)blocks * ns * rows * (s.d + 2) * sizeof(float);
}

cudaError_t launch_attn_fused(const Shape &s, int L, const void *q, const void *K, const void *V,
                              const int *idx, int stride, const int *count, void *out, float *lse,
                              void *part, uint32_t *status, cudaStream_t st) {
  FuArgs a = fu_base(s, L, q, K, V, const_cast<int *>(idx), stride, const_cast<int *>(count), out,
                     lse, status, part);
  return launch_fu<kModeIdx>(a, s, stride, st);
}

bool fused_route_ok(const Shape &s, int L, int k_or_cap) {
  return s.dtype == 1 && L * s.G() <= 128 && s.N <= kTsMaxWords * 32 &&
         (k_or_cap + kMaxPer - 1) / kMaxPer <= kMaxSplits;
}

cudaError_t launch_route_attn_topk(const Shape &s, int L, const void *q_layers, const void *K,
                                   const void *V, int k, const float *S, uint32_t *hist,
                                   int *idx, void *out, float *lse, void *part,
                                   uint32_t *status, cudaStream_t st) {
  FuArgs a = fu_base(s, L, q_layers, K, V, idx, k, nullptr, out, lse, status, part);
  a.S = S;
  a.hist = hist;
  a.k_or_cap = k;
  return launch_fu<kModeTopk>(a, s, k, st);
}

cudaError_t launch_route_attn_threshold(const Shape &s, int L, const void *q_layers,
                                        const void *K, const void *V, const uint32_t *bits,
                                        int cap, int *idx, int *count, void *out, float *lse,
                                        void *part, uint32_t *status, cudaStream_t st) {
  FuArgs a = fu_base(s, L, q_layers, K, V, idx, cap, count, out, lse, status, part);
  a.bits = bits;
  a.k_or_cap = cap;
  return launch_fu<kModeThresh>(a, s, cap, st);
}

}  // namespace sd
