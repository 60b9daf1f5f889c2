// attn_tc.cu -- A3 + A4 for bf16 on the 5th-generation tensor cores
// (tcgen05): gather attention with the accumulators in tensor memory.
//
// Every cross-decoder layer attends over the one shared index set (CLSA
// article, section CLSAの仕組み), so for one (sequence, KV head) the M = L*G
// query vectors of all layers and query heads form a dense block against the
// same gathered keys: S = Q K^T and O = P V are real dense contractions.
//
// Grid: (key splits, blocks of 128 query vectors, sequence x KV head), one CTA
// per SM (tile buffers and 512 tensor-memory columns).  CTA r owns a
// contiguous share of the head's selected keys and works through it in
// chunks of up to 256 keys:
//  1. 16-byte async copies gather the chunk's K and V rows straight into
//     128-byte-swizzled shared-memory tiles (the canonical K-major layout
//     for K, the MN-major layout for V -- the same bytes, read two ways).
//  2. One thread issues tcgen05.mma (kind::f16, bf16 in, fp32 accumulate,
//     M=128 query rows, N=64 keys per tile) for S into tensor memory.
//  3. Query row i lives in tensor-memory lane i; the four warps that share
//     a lane quadrant split every 64-key tile in quarters.  They read S with
//     tcgen05.ld, take the exact row maximum of the chunk (joined through
//     shared memory), and write P = exp2(S*scale*log2e - max) as two bf16
//     parts (P = P_hi + P_lo, ~16 significant bits) into swizzled shared
//     memory that reuses the K tiles.
//  4. One thread issues O += P_hi V + P_lo V (M=128, N=d, K=64 per tile)
//     into tensor memory, double-buffered against step 3.
// A running max carried between chunks rescales O in tensor memory (only
// when a CTA holds more than 256 keys).  With one split the CTA normalises O
// and writes out directly.  With several, each writes its partial (O, max,
// sum) for the real query rows to the workspace, arrives on a per-head
// counter and waits (bounded) for the other splits -- the grid is at most
// one CTA per SM, so all of them are resident -- then merges its share of the
// rows by log-sum-exp rescaling; the last split to leave resets the counters.
// When the splits of a head can run as one thread-block cluster (up to 16
// CTAs, all clusters resident at once), the partials stay in shared memory
// instead: one cluster barrier, then each CTA merges its rows reading every
// split's partial through distributed shared memory, and a second barrier
// keeps each partial in place until its readers are done.
//
// Every wait is bounded; on expiry the kernel raises the TIMEOUT flag, stops
// issuing work, frees its tensor memory and returns.
#include <cooperative_groups.h>

#include <atomic>

#include "common.cuh"
#include "internal.h"

namespace sd {
namespace {

namespace cg = cooperative_groups;

constexpr int kGroups = 4;          // warps sharing a tensor-memory lane quadrant
constexpr int kTcThreads = 128 * kGroups;
constexpr int KPT = 64 / kGroups;    // keys per thread of each 64-key tile
constexpr int kTcRows = 128;        // MMA M
constexpr int kTileN = 64;          // keys per S tile (MMA N of QK^T, K of PV)
constexpr int kChunkTiles = 4;      // tiles per chunk (S uses 256 TMEM columns)
constexpr int kChunkKeys = kTileN * kChunkTiles;
constexpr int kTmemCols = 512;
constexpr int kTcMaxSplits = 16;
constexpr int kTcMaxDevices = 64;

template <int D>
struct TcCfg {
  static constexpr int kQBytes = kTcRows * D * 2;               // 32 KB at d=128
  static constexpr int kKTile = kTileN * D * 2;                 // 16 KB
  static constexpr int kPBuf = kTcRows * kTileN * 2;            // 16 KB (hi or lo)
  static constexpr int kKPBytes =
      (kChunkTiles * kKTile > 4 * kPBuf) ? kChunkTiles * kKTile : 4 * kPBuf;
  static constexpr int kVBytes = kChunkTiles * kKTile;
  static constexpr int kQOff = 0;
  static constexpr int kKPOff = kQOff + kQBytes;
  static constexpr int kVOff = kKPOff + kKPBytes;
  static constexpr int kSmallOff = kVOff + kVBytes;
  static constexpr int kSmallBytes = 4096;
  static constexpr int kSmem = kSmallOff + kSmallBytes + 1024;  // + alignment slack
  static_assert(kTcRows * (D + 4) * 4 <= kKPBytes + kVBytes, "staging area fits");
};

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

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t *r) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
               : "r"(taddr));
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

template <int D, bool kCluster>
__global__ void __launch_bounds__(kTcThreads, 1)
    attn_tc_kernel(const __nv_bfloat16 *__restrict__ q,
                   const __nv_bfloat16 *__restrict__ K,
                   const __nv_bfloat16 *__restrict__ V,
                   const int *__restrict__ idx, int stride,
                   const int *__restrict__ count, int N, int kv_rows, int B, int Hq, int Hkv,
                   int L, float scale_log2, __nv_bfloat16 *__restrict__ out,
                   float *__restrict__ lse, float *__restrict__ part,
                   uint32_t *__restrict__ counters, uint32_t *status) {
  using C = TcCfg<D>;
  constexpr int KSTEPS = D / 16;  // MMA k-steps of S = Q K^T
  constexpr int CPR = D / 8;      // 16-byte chunks per K/V row
  const int csize = (int)gridDim.x;   // key splits of this head
  const int rank = (int)blockIdx.x;
  const int qb = blockIdx.y, bh = blockIdx.z;
  const int b = bh / Hkv, h = bh % Hkv, G = Hq / Hkv;
  const int M = L * G;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // Warps w, w+4, ... share tensor-memory lane quadrant w%4 (query rows
  // 32*(w%4) .. +31); they split every 64-key tile into kGroups parts.
  const int quad = warp & 3, grp = warp >> 2;
  const int row = quad * 32 + lane;

  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t base_s = (raw_s + 1023u) & ~1023u;  // swizzle atoms need 1 KB alignment
  unsigned char *base = smem_raw + (base_s - raw_s);
  const uint32_t q_s = base_s + C::kQOff;
  const uint32_t kp_s = base_s + C::kKPOff;
  const uint32_t v_s = base_s + C::kVOff;
  unsigned char *small = base + C::kSmallOff;
  uint64_t *bars = reinterpret_cast<uint64_t *>(small);        // s, pv0, pv1, done
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(small + 64);
  int *sidx = reinterpret_cast<int *>(small + 128);            // [256] chunk indices
  unsigned char *kval = small + 128 + 4 * kChunkKeys;          // [256] valid flags
  float *xred = reinterpret_cast<float *>(small + 128 + 5 * kChunkKeys);  // [kGroups][128]

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(tmem_slot)), "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
    for (int i = 0; i < 4; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  grid_dep_wait();  // the index set and queries may come from earlier kernels
  grid_dep_launch();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_S = tmem;                          // columns [0, 256)
  const uint32_t t_O = tmem + kChunkKeys;             // columns [256, 256 + D)
  const uint32_t lane_off = (uint32_t)(quad * 32) << 16;

  int cnt = stride;
  if (count) cnt = min(max(count[bh], 0), stride);
  const int per = (cnt + csize - 1) / csize;
  const int k0 = min(cnt, rank * per), k1 = min(cnt, k0 + per);
  const int *rowidx = idx + (size_t)bh * stride;
  const size_t head_off = (size_t)bh * kv_rows * D;

  // ---- Q block (rows beyond M are zero): thread = (row, part of the row) ----
  {
    const int r = tid & (kTcRows - 1), part = tid >> 7;
    const int m = qb * kTcRows + r;
    const __nv_bfloat16 *qr = nullptr;
    if (m < M) qr = q + (((size_t)(m / G) * B + b) * Hq + (size_t)h * G + m % G) * D;
#pragma unroll
    for (int cc = 0; cc < CPR / kGroups; ++cc) {
      const int c = part * (CPR / kGroups) + cc;
      const uint32_t dst = q_s + (c >> 3) * (kTcRows * 128) + swz(r, c & 7);
      cp_async16(dst, qr ? qr + c * 8 : q, qr != nullptr);
    }
    cp_async_commit();
  }

  bool failed = false;
  float mrun = -INFINITY, lsum = 0.f;
  uint32_t phase_s = 0, phase_done = 0, pv_uses[2] = {0u, 0u};
  bool first_pv = true;
  const uint32_t idS = idesc_bf16(kTcRows, kTileN, false);
  const uint32_t idPV = idesc_bf16(kTcRows, D, true);

  for (int c0 = k0; c0 < k1 && !failed; c0 += kChunkKeys) {
    const int nk = min(kChunkKeys, k1 - c0);
    const int ntile = (nk + kTileN - 1) / kTileN;
    // indices of the chunk
    if (tid < kChunkKeys) sidx[tid] = tid < nk ? rowidx[c0 + tid] : -1;
    __syncthreads();
    // gather the chunk's K rows, then its V rows (two async-copy groups)
    for (int p = tid; p < ntile * kTileN * CPR; p += kTcThreads) {
      const int r = p / CPR, c = p % CPR;
      const int j = sidx[r];
      const bool ok = r < nk && j >= 0 && j < N;
      if (r < nk && !ok && c == 0) raise_flag(status, FLAG_INDEX);
      if (c == 0) kval[r] = ok;
      const uint32_t dst = kp_s + (r >> 6) * C::kKTile + (c >> 3) * (kTileN * 128) +
                           swz(r & 63, c & 7);
      cp_async16(dst, K + head_off + (size_t)(ok ? j : 0) * D + c * 8, ok);
    }
    cp_async_commit();
    for (int p = tid; p < ntile * kTileN * CPR; p += kTcThreads) {
      const int r = p / CPR, c = p % CPR;
      const int j = sidx[r];
      const bool ok = r < nk && j >= 0 && j < N;
      const uint32_t dst = v_s + (r >> 6) * C::kKTile + (c >> 3) * (kTileN * 128) +
                           swz(r & 63, c & 7);
      cp_async16(dst, V + head_off + (size_t)(ok ? j : 0) * D + c * 8, ok);
    }
    cp_async_commit();
    cp_async_wait<1>();      // Q and K have landed (this thread's copies)
    fence_async_smem();      // make them visible to the tensor-core proxy
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- S = Q K^T for every tile of the chunk, one issuing thread ----------
    if (tid == 0) {
      for (int t = 0; t < ntile; ++t) {
#pragma unroll
        for (int s = 0; s < KSTEPS; ++s) {
          const uint64_t a = sw128_desc(q_s + (s >> 2) * (kTcRows * 128) + (s & 3) * 32, 16, 1024);
          const uint64_t bk = sw128_desc(kp_s + t * C::kKTile + (s >> 2) * (kTileN * 128) + (s & 3) * 32,
                                         16, 1024);
          mma_f16(t_S + t * kTileN, a, bk, idS, s > 0 ? 1u : 0u);
        }
      }
      mma_commit(&bars[0]);
    }
    // validity of this warp's 32 keys of each tile, as bit masks (ballots over
    // the flags written by the gather; identical in every warp)
    uint32_t vmask[kChunkTiles];  // this thread's KPT keys of each tile
#pragma unroll
    for (int t = 0; t < kChunkTiles; ++t) {
      constexpr int PER32 = 32 / KPT;  // groups covered by one 32-key ballot
      const int key = t * kTileN + (grp / PER32) * 32 + lane;
      const uint32_t b = __ballot_sync(0xffffffffu, key < nk && kval[key] != 0);
      vmask[t] = KPT == 32 ? b : (b >> ((grp % PER32) * KPT)) & ((1u << KPT) - 1u);
    }
    if (!mbar_wait(&bars[0], phase_s & 1u, status)) failed = true;
    ++phase_s;
    tc_fence_after();
    if (__syncthreads_or(failed)) {
      failed = true;
      break;
    }

    // ---- row maximum over the chunk (two warps per row, joined in smem) -------
    float cmax = -INFINITY;
#pragma unroll
    for (int t = 0; t < kChunkTiles; ++t) {
      if (t < ntile) {
        uint32_t r[KPT];
        if (KPT == 32) tmem_ld32(t_S + lane_off + t * kTileN + grp * KPT, r);
        else tmem_ld16(t_S + lane_off + t * kTileN + grp * KPT, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < KPT; ++i)
          if ((vmask[t] >> i) & 1u) cmax = fmaxf(cmax, __uint_as_float(r[i]));
      }
    }
    xred[grp * kTcRows + row] = cmax;
    __syncthreads();
#pragma unroll
    for (int g = 0; g < kGroups; ++g) cmax = fmaxf(cmax, xred[g * kTcRows + row]);
    cmax *= scale_log2;  // scale > 0
    const float mnew = fmaxf(mrun, cmax);
    const float muse = mnew == -INFINITY ? 0.f : mnew;
    const bool rescale = !first_pv && mnew != mrun;
    if (__any_sync(0xffffffffu, rescale)) {
      // a later chunk raised some row's max: rescale O (this warp's half of
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

    // ---- P tiles and O += P V ---------------------------------------------------
    for (int t = 0; t < ntile; ++t) {
      const int buf = t & 1;
      if (pv_uses[buf] > 0) {  // PV of tile t-2 must be done with this buffer
        if (!mbar_wait(&bars[1 + buf], (pv_uses[buf] - 1) & 1u, status)) failed = true;
        tc_fence_after();
      }
      const uint32_t ph = kp_s + buf * 2 * C::kPBuf;  // hi, then lo
      const uint32_t pl = ph + C::kPBuf;
      uint32_t vm = 0;
#pragma unroll
      for (int u = 0; u < kChunkTiles; ++u)
        if (u == t) vm = vmask[u];
      uint32_t r[KPT];
      if (KPT == 32) tmem_ld32(t_S + lane_off + t * kTileN + grp * KPT, r);
      else tmem_ld16(t_S + lane_off + t * kTileN + grp * KPT, r);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < KPT / 8; ++c) {  // 16-byte chunks of 8 keys
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = c * 8 + e * 2;
          const float p0 = ((vm >> i) & 1u) ? fast_exp2(fmaf(__uint_as_float(r[i]), scale_log2, -muse)) : 0.f;
          const float p1 = ((vm >> (i + 1)) & 1u) ? fast_exp2(fmaf(__uint_as_float(r[i + 1]), scale_log2, -muse)) : 0.f;
          lsum += p0 + p1;
          hi[e] = pack_bf16x2(p0, p1);
          const __nv_bfloat162 hb = *reinterpret_cast<const __nv_bfloat162 *>(&hi[e]);
          lo[e] = pack_bf16x2(p0 - __low2float(hb), p1 - __high2float(hb));
        }
        const uint32_t off = swz(row, grp * (KPT / 8) + c);
        asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(ph + off), "r"(hi[0]),
                     "r"(hi[1]), "r"(hi[2]), "r"(hi[3])
                     : "memory");
        asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(pl + off), "r"(lo[0]),
                     "r"(lo[1]), "r"(lo[2]), "r"(lo[3])
                     : "memory");
      }
      if (t == 0) cp_async_wait<0>();  // V tiles have landed (this thread's copies)
      fence_async_smem();
      tc_fence_before();
      if (__syncthreads_or(failed)) {
        failed = true;
        break;
      }
      tc_fence_after();
      if (tid == 0) {
#pragma unroll
        for (int kk = 0; kk < kTileN / 16; ++kk) {
          const uint64_t bv = sw128_desc(v_s + t * C::kKTile + kk * 2048, kTileN * 128, 1024);
          mma_f16(t_O, sw128_desc(ph + kk * 32, 16, 1024), bv, idPV,
                  (first_pv && kk == 0) ? 0u : 1u);
          mma_f16(t_O, sw128_desc(pl + kk * 32, 16, 1024), bv, idPV, 1u);
        }
        mma_commit(&bars[1 + buf]);
      }
      first_pv = false;
      ++pv_uses[buf];
    }
    // every MMA of this chunk done before its shared memory is reused
    if (!failed) {
      if (tid == 0) mma_commit(&bars[3]);
      if (!mbar_wait(&bars[3], phase_done & 1u, status)) failed = true;
      ++phase_done;
      tc_fence_after();
    }
    if (__syncthreads_or(failed)) failed = true;
  }
  cp_async_wait<0>();

  // ---- this CTA's partial -------------------------------------------------------
  const int mrows = min(kTcRows, M - qb * kTcRows);  // real query rows of the block
  const bool have = !first_pv && !failed;
  __syncthreads();
  float *xsum = xred;  // [kGroups][128]: the warps' parts of each row's sum
  xsum[grp * kTcRows + row] = have ? lsum : 0.f;
  if (csize == 1) {
    // one split: normalise straight from tensor memory
    __syncthreads();
    float ls = 0.f;
#pragma unroll
    for (int g = 0; g < kGroups; ++g) ls += xsum[g * kTcRows + row];
    const float inv = (have && ls > 0.f) ? 1.f / ls : 0.f;
    const int m = qb * kTcRows + row;
    const size_t orow = m < M ? ((size_t)(m / G) * B + b) * Hq + (size_t)h * G + m % G : 0;
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
          pk.x = pack_bf16x2(have ? __uint_as_float(r[i]) * inv : 0.f, have ? __uint_as_float(r[i + 1]) * inv : 0.f);
          pk.y = pack_bf16x2(have ? __uint_as_float(r[i + 2]) * inv : 0.f, have ? __uint_as_float(r[i + 3]) * inv : 0.f);
          pk.z = pack_bf16x2(have ? __uint_as_float(r[i + 4]) * inv : 0.f, have ? __uint_as_float(r[i + 5]) * inv : 0.f);
          pk.w = pack_bf16x2(have ? __uint_as_float(r[i + 6]) * inv : 0.f, have ? __uint_as_float(r[i + 7]) * inv : 0.f);
          *reinterpret_cast<uint4 *>(out + orow * D + grp * (D / kGroups) + cb * 16 + i) = pk;
        }
      }
    }
    if (lse && grp == 0 && row < mrows)
      lse[orow] = (have && ls > 0.f) ? (mrun + log2f(ls)) * 0.69314718055994531f : -INFINITY;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                   "r"(kTmemCols)
                   : "memory");
    return;
  }

  // Several splits: write (O, max, sum) of the real rows to the partials,
  // [head][qblock][split][row][D + 4] fp32 (O, max, sum, pad), staged through
  // shared memory (the tile buffers are free now) so the global stores are
  // coalesced.
  constexpr int PR = D + 4;  // partial row stride in floats (16-byte aligned)
  float *stage = reinterpret_cast<float *>(base + C::kKPOff);  // [128][PR]
  float *mypart = part + (((size_t)bh * gridDim.y + qb) * csize + rank) * kTcRows * PR;
#pragma unroll
  for (int cb = 0; cb < D / kGroups / 16; ++cb) {
    uint32_t r[16];
    if (have) {
      tmem_ld16(t_O + lane_off + grp * (D / kGroups) + cb * 16, r);
      tmem_wait_ld();
    }
    if (row < mrows) {
      float *dst = stage + row * PR + grp * (D / kGroups) + cb * 16;
#pragma unroll
      for (int i = 0; i < 16; i += 4)
        *reinterpret_cast<float4 *>(dst + i) =
            have ? make_float4(__uint_as_float(r[i]), __uint_as_float(r[i + 1]),
                               __uint_as_float(r[i + 2]), __uint_as_float(r[i + 3]))
                 : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  __syncthreads();
  if (grp == 0 && row < mrows) {
    float ls = 0.f;
#pragma unroll
    for (int g = 0; g < kGroups; ++g) ls += xsum[g * kTcRows + row];
    *reinterpret_cast<float4 *>(stage + row * PR + D) =
        make_float4(have ? mrun : -INFINITY, ls, 0.f, 0.f);
  }
  __syncthreads();
  if constexpr (!kCluster) {
    const int n4 = mrows * PR / 4;
    const float4 *src = reinterpret_cast<const float4 *>(stage);
    float4 *dst = reinterpret_cast<float4 *>(mypart);
    for (int i = tid; i < n4; i += kTcThreads) dst[i] = src[i];
  }
  // tensor memory is no longer needed
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  // merge rows lr = rank, rank + csize, ...: thread = (row slot, float4
  // chunk); every split's values are loaded before any is used.  prow(r, lr)
  // is split r's partial row lr.
  auto merge = [&](auto prow) {
    constexpr int CH = D / 4;
    constexpr int RPP = kTcThreads / CH;  // rows per pass
    const int nmine = (mrows - rank + csize - 1) / csize;
    for (int i = tid / CH; i < nmine; i += RPP) {
      const int lr = rank + i * csize;
      const int ch = tid % CH;
      float2 ml[kTcMaxSplits];
      float4 v[kTcMaxSplits];
#pragma unroll
      for (int r = 0; r < kTcMaxSplits; ++r) {
        if (r < csize) {
          const float *pr = prow(r, lr);
          ml[r] = *reinterpret_cast<const float2 *>(pr + D);
          v[r] = *reinterpret_cast<const float4 *>(pr + ch * 4);
        } else {
          ml[r] = make_float2(-INFINITY, 0.f);
          v[r] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
      float mx = -INFINITY;
#pragma unroll
      for (int r = 0; r < kTcMaxSplits; ++r) mx = fmaxf(mx, ml[r].x);
      float ls = 0.f;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      if (mx != -INFINITY) {
#pragma unroll
        for (int r = 0; r < kTcMaxSplits; ++r) {
          const float w = ml[r].x == -INFINITY ? 0.f : exp2f(ml[r].x - mx);
          ls += ml[r].y * w;
          acc.x += w * v[r].x;
          acc.y += w * v[r].y;
          acc.z += w * v[r].z;
          acc.w += w * v[r].w;
        }
      }
      const float inv = ls > 0.f ? 1.f / ls : 0.f;
      const int m = qb * kTcRows + lr;
      const size_t orow = ((size_t)(m / G) * B + b) * Hq + (size_t)h * G + m % G;
      uint2 pk;
      pk.x = pack_bf16x2(acc.x * inv, acc.y * inv);
      pk.y = pack_bf16x2(acc.z * inv, acc.w * inv);
      *reinterpret_cast<uint2 *>(out + orow * D + ch * 4) = pk;
      if (lse && ch == 0)
        lse[orow] = ls > 0.f ? (mx + log2f(ls)) * 0.69314718055994531f : -INFINITY;
    }
  };
  if constexpr (kCluster) {
    // the head's splits are this cluster (cluster rank = blockIdx.x); the
    // barriers are hardware cluster barriers that every CTA reaches (nothing
    // above returns early)
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();  // every split's partial is staged in its shared memory
    merge([&](int r, int lr) -> const float * {
      return cluster.map_shared_rank(stage, r) + (size_t)lr * PR;
    });
    cluster.sync();  // no CTA leaves while another reads its partial
    return;
  } else {
    // arrive, then wait (bounded) until every split of this head block
    // arrived; the grid (at most one CTA per SM) is resident as a whole
    uint32_t *arrive = counters + 2 * ((size_t)bh * gridDim.y + qb);
    __shared__ int ready;
    if (tid == 0) {
      __threadfence();
      asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(arrive) : "memory");
      ready = wait_counter_geq(arrive, (uint32_t)csize, kWaitLimitNs, status);
    }
    __syncthreads();
    const float *hp = part + ((size_t)bh * gridDim.y + qb) * csize * kTcRows * PR;
    if (ready)
      merge([&](int r, int lr) -> const float * {
        return hp + ((size_t)r * kTcRows + lr) * PR;
      });
  }
  // the last split to leave resets both counters for the next call
  __syncthreads();
  if (tid == 0) {
    uint32_t *arrive = counters + 2 * ((size_t)bh * gridDim.y + qb);
    uint32_t *depart = arrive + 1;
    const uint32_t old = atomicAdd(depart, 1u);
    if (old == (uint32_t)csize - 1) {
      *arrive = 0u;
      *depart = 0u;
      __threadfence();
    }
  }
}

template <int D>
size_t tc_part_bytes(const Shape &s, int L) {
  const int M = L * s.G();
  const int qblocks = (M + kTcRows - 1) / kTcRows;
  return (size_t)s.BH() * qblocks * kTcMaxSplits * kTcRows * (D + 4) * sizeof(float);
}

// Whether `blocks` clusters of `nsplit` attention CTAs can all be resident
// at once (cudaOccupancyMaxActiveClusters), cached per device and split
// count; sizes above the portable 8 need the non-portable opt-in.
template <int D>
bool tc_clusters_fit(int nsplit, long long blocks) {
  using C = TcCfg<D>;
  static std::atomic<int> cache[kTcMaxDevices][kTcMaxSplits + 1];  // 0 unknown, 1 + max
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kTcMaxDevices ||
      nsplit > kTcMaxSplits) {
    (void)cudaGetLastError();
    return false;
  }
  int v = cache[dev][nsplit].load(std::memory_order_relaxed);
  if (v == 0) {
    auto kern = attn_tc_kernel<D, true>;
    int n = 0;
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (e == cudaSuccess && nsplit > 8)
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e == cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)nsplit, 1, 1);
      cfg.blockDim = dim3(kTcThreads, 1, 1);
      cfg.dynamicSmemBytes = C::kSmem;
      cudaLaunchAttribute a;
      a.id = cudaLaunchAttributeClusterDimension;
      a.val.clusterDim.x = (unsigned)nsplit;
      a.val.clusterDim.y = 1;
      a.val.clusterDim.z = 1;
      cfg.attrs = &a;
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
  return (long long)(v - 1) >= blocks;
}

template <int D>
cudaError_t launch_tc_t(const Shape &s, int L, const void *q, const void *K,
                        const void *V, const int *idx, int stride, const int *count,
                        void *out, float *lse, void *ws, uint32_t *counters,
                        uint32_t *status, cudaStream_t st) {
  using C = TcCfg<D>;
  DeviceInfo di;
  cudaError_t e = device_info(&di);
  if (e != cudaSuccess) return e;
  const int M = L * s.G();
  const int qblocks = (M + kTcRows - 1) / kTcRows;
  // key splits per head block: enough CTAs to cover the SMs (one CTA per SM:
  // the tile buffers and 512 tensor-memory columns), every split at least one
  // 64-key tile, all CTAs resident at once when there is more than one split
  const long long blocks = (long long)s.BH() * qblocks;
  int nsplit = (int)(di.sm_count / blocks);
  const int by_keys = (stride + kTileN - 1) / kTileN;
  nsplit = nsplit > by_keys ? by_keys : nsplit;
  nsplit = nsplit > kTcMaxSplits ? kTcMaxSplits : nsplit;
  nsplit = nsplit < 1 ? 1 : nsplit;
  if (blocks > kAttnMaxCounterBlocks) nsplit = 1;  // counters live in a fixed area
  float *part = static_cast<float *>(ws);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)nsplit, (unsigned)qblocks, (unsigned)s.BH());
  cfg.blockDim = dim3(kTcThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  // merge through distributed shared memory when each head block's splits
  // can form one cluster and all those clusters fit on the device at once
  bool cluster = nsplit > 1 && !cooperative_forced() && attn_cluster_merge_enabled() &&
                 tc_clusters_fit<D>(nsplit, blocks);
  auto kern = cluster ? attn_tc_kernel<D, true> : attn_tc_kernel<D, false>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  if (cluster && nsplit > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  if (cluster) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)nsplit;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.numAttrs = 1;
  } else {
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.numAttrs = (nsplit > 1 && cooperative_forced()) ? 1 : 0;
  }
  cfg.attrs = attr;
  add_pdl_attr(cfg, attr);
  const float scale_log2 = (float)(1.4426950408889634 / __builtin_sqrt((double)D));
  e = cudaLaunchKernelEx(&cfg, kern, static_cast<const __nv_bfloat16 *>(q),
                         static_cast<const __nv_bfloat16 *>(K),
                         static_cast<const __nv_bfloat16 *>(V), idx, stride, count, s.N, s.Ncap,
                         s.B, s.Hq, s.Hkv, L, scale_log2, static_cast<__nv_bfloat16 *>(out),
                         lse, part, counters, status);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

size_t attn_tc_workspace_bytes(const Shape &s, int L) {
  return s.d == 128 ? tc_part_bytes<128>(s, L) : tc_part_bytes<64>(s, L);
}

cudaError_t launch_attn_tc(const Shape &s, int L, const void *q, const void *K,
                           const void *V, const int *idx, int stride,
                           const int *count, void *out, float *lse, void *ws,
                           uint32_t *counters, uint32_t *status, cudaStream_t st) {
  if (s.d == 128)
    return launch_tc_t<128>(s, L, q, K, V, idx, stride, count, out, lse, ws, counters,
                            status, st);
  return launch_tc_t<64>(s, L, q, K, V, idx, stride, count, out, lse, ws, counters, status,
                         st);
}

}  // namespace sd
