// attn_mma.cu -- A3 + A4 for bf16: gather attention on the tensor cores with
// the split-k merge done through distributed shared memory.
//
// All L layers attend over one shared index set (CLSA article, section
// CLSAの仕組み), so for one (sequence, KV head) the L*G query vectors of all
// layers and all query heads of the group form a dense [M = L*G, d] block
// against the same gathered [k, d] key and value tiles.  That is a real
// dense contraction: S = Q K^T and O = P V run as bf16 mma.sync tiles
// (m16n8k16, fp32 accumulate), with the fp32 online softmax in registers.
//
// Work decomposition: a thread-block cluster of C CTAs per (sequence, KV head,
// block of 64 query vectors); CTA r of the cluster owns a contiguous share of
// the selected keys.  Each CTA gathers its keys' K and V rows (16-byte async
// copies into XOR-swizzled shared memory, double buffered in tiles of 64
// keys), runs four warps of 16 query rows each, and leaves its partial
// (running max, running sum, unnormalised output) in shared memory.  After a
// cluster barrier every CTA merges a slice of the rows by log-sum-exp
// rescaling, reading the other CTAs' partials through distributed shared
// memory, and writes out and lse.  Nothing goes through global scratch.
//
// Precision: K, V and Q are bf16 operands (exact products, fp32 sums).  The
// softmax weights P are split as P = P_hi + P_lo with both parts bf16, and
// the PV product runs twice (hi and lo), so P carries ~16 significant bits
// instead of bf16's 8.
#include <cooperative_groups.h>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace sd {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kRowsPerCta = kWarps * 16;  // query vectors per CTA
constexpr int kTileKeys = 64;
constexpr int kMaxCluster = 16;

template <int D>
struct MmaCfg {
  static constexpr int kChunks = D / 8;                  // 16-byte chunks per row
  static constexpr int kTileBytes = kTileKeys * D * 2;   // one K or V tile
  static constexpr int kMergeBytes = kRowsPerCta * D * 4 + kRowsPerCta * 8;
  static constexpr int kLoopBytes = 4 * kTileBytes + 2 * kTileKeys * 4;
  static constexpr int kSmem = kLoopBytes > kMergeBytes ? kLoopBytes : kMergeBytes;
};

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem, bool pred) {
  const uint32_t bytes = pred ? 16u : 0u;  // 0 -> zero fill
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem)),
               "l"(gmem), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                        uint32_t &r3, const void *p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                          uint32_t &r3, const void *p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_u32(p)));
}

__device__ __forceinline__ void mma_bf16(float *c, const uint32_t *a, uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

// Address of 16-byte chunk `c` of row `r` in a swizzled [64][D] bf16 tile.
template <int D>
__device__ __forceinline__ __nv_bfloat16 *tile_at(__nv_bfloat16 *tile, int r, int c) {
  return tile + r * D + ((c ^ (r & 7)) << 3);
}

template <int D>
__global__ void __launch_bounds__(kThreads)
    attn_mma_kernel(const __nv_bfloat16 *__restrict__ q,
                    const __nv_bfloat16 *__restrict__ K,
                    const __nv_bfloat16 *__restrict__ V,
                    const int *__restrict__ idx, int stride,
                    const int *__restrict__ count, int N, int kv_rows, int B, int Hq,
                    int Hkv, int L, float scale_log2,
                    __nv_bfloat16 *__restrict__ out, float *__restrict__ lse,
                    uint32_t *status) {
  using C = MmaCfg<D>;
  constexpr int KS = D / 16;  // k-steps over d for S = Q K^T
  constexpr int NT = D / 8;   // n-tiles over d for O = P V
  cg::cluster_group cluster = cg::this_cluster();
  const int csize = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int qb = blockIdx.y, bh = blockIdx.z;
  const int b = bh / Hkv, h = bh % Hkv, G = Hq / Hkv;
  const int M = L * G;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t4 = lane & 3;

  grid_dep_wait();
  grid_dep_launch();
  extern __shared__ __align__(128) unsigned char smem[];
  __nv_bfloat16 *Ks = reinterpret_cast<__nv_bfloat16 *>(smem);
  __nv_bfloat16 *Vs = Ks + 2 * kTileKeys * D;
  int *kval = reinterpret_cast<int *>(smem + 4 * C::kTileBytes);  // [2][64]

  int cnt = stride;
  if (count) cnt = min(max(count[bh], 0), stride);
  const int per = (cnt + csize - 1) / csize;
  const int k0 = min(cnt, rank * per), k1 = min(cnt, k0 + per);
  const int *row = idx + (size_t)bh * stride;
  const size_t head_off = (size_t)bh * kv_rows * D;

  auto load_tile = [&](int buf, int t0) {
    __nv_bfloat16 *kt = Ks + buf * kTileKeys * D;
    __nv_bfloat16 *vt = Vs + buf * kTileKeys * D;
    constexpr int ITER = kTileKeys * C::kChunks / kThreads;
    int jj[ITER];
#pragma unroll
    for (int u = 0; u < ITER; ++u) {  // all index loads in flight at once
      const int key = t0 + (threadIdx.x + u * kThreads) / C::kChunks;
      jj[u] = key < k1 ? row[key] : -1;
    }
#pragma unroll
    for (int u = 0; u < ITER; ++u) {
      const int p = threadIdx.x + u * kThreads;
      const int r = p / C::kChunks, c = p % C::kChunks;
      const int key = t0 + r;
      const int j = jj[u];
      const bool ok = j >= 0 && j < N;
      if (key < k1 && !ok && c == 0) raise_flag(status, FLAG_INDEX);
      const size_t off = head_off + (size_t)(ok ? j : 0) * D + c * 8;
      cp_async16(tile_at<D>(kt, r, c), K + off, ok);
      cp_async16(tile_at<D>(vt, r, c), V + off, ok);
      if (c == 0) kval[buf * kTileKeys + r] = ok;
    }
    cp_async_commit();
  };

  // Q fragments (A operand, row-major 16 x 16 per k-step), pre-loaded.
  uint32_t qa[KS][4];
  {
    const int m0 = qb * kRowsPerCta + warp * 16 + g;
    const int m1 = m0 + 8;
    const __nv_bfloat16 *q0 = nullptr, *q1 = nullptr;
    if (m0 < M) q0 = q + (((size_t)(m0 / G) * B + b) * Hq + (size_t)h * G + m0 % G) * D;
    if (m1 < M) q1 = q + (((size_t)(m1 / G) * B + b) * Hq + (size_t)h * G + m1 % G) * D;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      const int c0 = ks * 16 + 2 * t4;
      qa[ks][0] = q0 ? *reinterpret_cast<const uint32_t *>(q0 + c0) : 0u;
      qa[ks][1] = q1 ? *reinterpret_cast<const uint32_t *>(q1 + c0) : 0u;
      qa[ks][2] = q0 ? *reinterpret_cast<const uint32_t *>(q0 + c0 + 8) : 0u;
      qa[ks][3] = q1 ? *reinterpret_cast<const uint32_t *>(q1 + c0 + 8) : 0u;
    }
  }

  float o[NT][4];
#pragma unroll
  for (int i = 0; i < NT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float mrow[2] = {-INFINITY, -INFINITY};  // running max (log2-scaled logits)
  float lrow[2] = {0.f, 0.f};              // this thread's share of the sum

  const int ntiles = (k1 - k0 + kTileKeys - 1) / kTileKeys;
  if (ntiles > 0) load_tile(0, k0);
  for (int it = 0; it < ntiles; ++it) {
    const int buf = it & 1;
    if (it + 1 < ntiles) {
      load_tile(buf ^ 1, k0 + (it + 1) * kTileKeys);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const __nv_bfloat16 *kt = Ks + buf * kTileKeys * D;
    const __nv_bfloat16 *vt = Vs + buf * kTileKeys * D;
    const int *kv = kval + buf * kTileKeys;

    // ---- S = Q K^T (16 x 64 per warp) --------------------------------------
    float s[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        const int mi = lane >> 3;
        const int key = np * 16 + ((mi & 2) ? 8 : 0) + (lane & 7);
        const int ch = ks * 2 + (mi & 1);
        uint32_t r0, r1, r2, r3;
        ldsm_x4(r0, r1, r2, r3, tile_at<D>(const_cast<__nv_bfloat16 *>(kt), key, ch));
        mma_bf16(s[2 * np], qa[ks], r0, r1);
        mma_bf16(s[2 * np + 1], qa[ks], r2, r3);
      }
    }
    // ---- online softmax (rows g and g+8) ------------------------------------
    float tmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = nt * 8 + 2 * t4 + (e & 1);
        const bool ok = (k0 + it * kTileKeys + key < k1) && kv[key];
        const float v = ok ? s[nt][e] * scale_log2 : -INFINITY;
        s[nt][e] = v;
        tmax[e >> 1] = fmaxf(tmax[e >> 1], v);
      }
    }
    float corr[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      tmax[r] = fmaxf(tmax[r], __shfl_xor_sync(0xffffffffu, tmax[r], 1));
      tmax[r] = fmaxf(tmax[r], __shfl_xor_sync(0xffffffffu, tmax[r], 2));
      const float mnew = fmaxf(mrow[r], tmax[r]);
      const float muse = mnew == -INFINITY ? 0.f : mnew;
      corr[r] = exp2f(mrow[r] - muse);
      mrow[r] = mnew;
      tmax[r] = muse;
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) lrow[r] *= corr[r];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      o[nt][0] *= corr[0];
      o[nt][1] *= corr[0];
      o[nt][2] *= corr[1];
      o[nt][3] *= corr[1];
    }
    uint32_t pa_hi[4][4], pa_lo[4][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      float p[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        p[e] = exp2f(s[nt][e] - tmax[e >> 1]);
        lrow[e >> 1] += p[e];
      }
      const uint32_t hi01 = pack_bf16(p[0], p[1]);
      const uint32_t hi23 = pack_bf16(p[2], p[3]);
      const __nv_bfloat162 h01 = *reinterpret_cast<const __nv_bfloat162 *>(&hi01);
      const __nv_bfloat162 h23 = *reinterpret_cast<const __nv_bfloat162 *>(&hi23);
      const uint32_t lo01 = pack_bf16(p[0] - __low2float(h01), p[1] - __high2float(h01));
      const uint32_t lo23 = pack_bf16(p[2] - __low2float(h23), p[3] - __high2float(h23));
      // the C layout of n-tiles 2kk and 2kk+1 is the A layout of k-step kk
      const int kk = nt >> 1, half = nt & 1;
      pa_hi[kk][half * 2 + 0] = hi01;
      pa_hi[kk][half * 2 + 1] = hi23;
      pa_lo[kk][half * 2 + 0] = lo01;
      pa_lo[kk][half * 2 + 1] = lo23;
    }
    // ---- O += P V ------------------------------------------------------------
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
      for (int dp = 0; dp < D / 16; ++dp) {
        const int mi = lane >> 3;
        const int key = kk * 16 + ((mi & 1) ? 8 : 0) + (lane & 7);
        const int ch = dp * 2 + (mi >> 1);
        uint32_t r0, r1, r2, r3;
        ldsm_x4_t(r0, r1, r2, r3, tile_at<D>(const_cast<__nv_bfloat16 *>(vt), key, ch));
        mma_bf16(o[2 * dp], pa_hi[kk], r0, r1);
        mma_bf16(o[2 * dp], pa_lo[kk], r0, r1);
        mma_bf16(o[2 * dp + 1], pa_hi[kk], r2, r3);
        mma_bf16(o[2 * dp + 1], pa_lo[kk], r2, r3);
      }
    }
    __syncthreads();  // the other buffer is refilled at the top of the loop
  }

  // ---- split merge through distributed shared memory ------------------------
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 1);
    lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 2);
  }
  __syncthreads();
  float *Op = reinterpret_cast<float *>(smem);   // [64][D] partial outputs
  float *ML = Op + kRowsPerCta * D;              // [64][2] (max, sum)
  {
    const int lr0 = warp * 16 + g, lr1 = lr0 + 8;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int c = nt * 8 + 2 * t4;
      *reinterpret_cast<float2 *>(&Op[lr0 * D + c]) = make_float2(o[nt][0], o[nt][1]);
      *reinterpret_cast<float2 *>(&Op[lr1 * D + c]) = make_float2(o[nt][2], o[nt][3]);
    }
    if (t4 == 0) {
      ML[lr0 * 2] = mrow[0];
      ML[lr0 * 2 + 1] = lrow[0];
      ML[lr1 * 2] = mrow[1];
      ML[lr1 * 2 + 1] = lrow[1];
    }
  }
  cluster.sync();
  constexpr int CH = D / 4;                // float4 chunks per row
  constexpr int RPP = kThreads / CH;       // rows merged per pass
  const int nmine = (kRowsPerCta - rank + csize - 1) / csize;
  for (int i = threadIdx.x / CH; i < nmine; i += RPP) {
    const int lr = rank + i * csize;
    const int m = qb * kRowsPerCta + lr;
    if (m >= M) continue;
    const int ch = threadIdx.x % CH;
    // all remote loads issued before any is used (distributed shared memory
    // latency is paid once, not once per rank)
    float mr[kMaxCluster], lr_[kMaxCluster];
    float4 vr[kMaxCluster];
#pragma unroll
    for (int r = 0; r < kMaxCluster; ++r) {
      if (r < csize) {
        const float2 ml = *reinterpret_cast<const float2 *>(cluster.map_shared_rank(ML, r) + lr * 2);
        mr[r] = ml.x;
        lr_[r] = ml.y;
        vr[r] = *reinterpret_cast<const float4 *>(cluster.map_shared_rank(Op, r) + lr * D + ch * 4);
      } else {
        mr[r] = -INFINITY;
        lr_[r] = 0.f;
        vr[r] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    float mx = -INFINITY;
#pragma unroll
    for (int r = 0; r < kMaxCluster; ++r) mx = fmaxf(mx, mr[r]);
    float lsum = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (mx != -INFINITY) {
#pragma unroll
      for (int r = 0; r < kMaxCluster; ++r) {
        const float w = mr[r] == -INFINITY ? 0.f : exp2f(mr[r] - mx);
        lsum += lr_[r] * w;
        acc.x += w * vr[r].x;
        acc.y += w * vr[r].y;
        acc.z += w * vr[r].z;
        acc.w += w * vr[r].w;
      }
    }
    const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
    const int l = m / G, gq = m % G;
    const size_t orow = ((size_t)l * B + b) * Hq + (size_t)h * G + gq;
    uint2 pk;
    pk.x = pack_bf16(acc.x * inv, acc.y * inv);
    pk.y = pack_bf16(acc.z * inv, acc.w * inv);
    *reinterpret_cast<uint2 *>(out + orow * D + ch * 4) = pk;
    if (lse && ch == 0)
      lse[orow] = lsum > 0.f ? (mx + log2f(lsum)) * 0.69314718055994531f : -INFINITY;
  }
  cluster.sync();  // keep this CTA's partials alive until every CTA merged
}

template <int D>
cudaError_t launch_mma_t(const Shape &s, int L, const void *q, const void *K,
                         const void *V, const int *idx, int stride,
                         const int *count, void *out, float *lse,
                         uint32_t *status, cudaStream_t st) {
  using C = MmaCfg<D>;
  DeviceInfo di;
  cudaError_t e = device_info(&di);
  if (e != cudaSuccess) return e;
  const int M = L * s.G();
  const int qblocks = (M + kRowsPerCta - 1) / kRowsPerCta;
  int csize = (stride + kTileKeys - 1) / kTileKeys;  // at least one tile each
  csize = csize < 1 ? 1 : csize;
  csize = csize > di.select_cluster ? di.select_cluster : csize;
  csize = csize > kMaxCluster ? kMaxCluster : csize;
  auto kern = attn_mma_kernel<D>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e == cudaSuccess && csize > 8)
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)csize, (unsigned)qblocks, (unsigned)s.BH());
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)csize;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const float scale_log2 = (float)(1.4426950408889634 / __builtin_sqrt((double)D));
  e = cudaLaunchKernelEx(&cfg, kern, static_cast<const __nv_bfloat16 *>(q),
                         static_cast<const __nv_bfloat16 *>(K),
                         static_cast<const __nv_bfloat16 *>(V), idx, stride, count,
                         s.N, s.Ncap, s.B, s.Hq, s.Hkv, L, scale_log2,
                         static_cast<__nv_bfloat16 *>(out), lse, status);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_mma(const Shape &s, int L, const void *q, const void *K,
                            const void *V, const int *idx, int stride,
                            const int *count, void *out, float *lse,
                            uint32_t *status, cudaStream_t st) {
  if (s.d == 128)
    return launch_mma_t<128>(s, L, q, K, V, idx, stride, count, out, lse, status, st);
  return launch_mma_t<64>(s, L, q, K, V, idx, stride, count, out, lse, status, st);
}

}  // namespace sd
