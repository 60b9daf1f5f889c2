// attn.cu -- A3 + A4 for fp32 inputs (bf16 inputs take attn_fused.cu).
//
// Every query vector of every layer attends over the same selected rows of
// its KV head (CLSA article, section CLSAの仕組み: the routing set is reused
// unchanged by every cross-decoder layer; section 研究の背景と課題: attention
// over the selected tokens only).
//
// Split-k design: the index row of a (sequence, KV head) is cut into splits;
// one CTA gathers the K and V rows of its split into shared memory once and
// uses them for all L*G query vectors of that head (so the selected rows are
// read from memory once per call, whatever L is).  Each CTA runs an fp32
// online softmax (running max, rescaled sum) per query and writes a partial
// (max, sum, unnormalised output).  A merge kernel combines the partials of
// the splits by log-sum-exp rescaling and writes out and lse.
#include <stdlib.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"

namespace sd {
namespace {

constexpr int kAttnThreads = 256;
constexpr int kAttnWarps = kAttnThreads / 32;
constexpr int kQPerWarp = 8;
constexpr int kQPerCta = kAttnWarps * kQPerWarp;  // 64 query vectors
constexpr int kChunk = 32;                         // keys per smem chunk
constexpr int kTargetCtas = 512;
constexpr int kMaxSplits = 64;

inline int num_splits(int BH, int qblocks, int stride) {
  int want = (kTargetCtas + BH * qblocks - 1) / (BH * qblocks);
  const int most = (stride + kChunk - 1) / kChunk;
  if (want > most) want = most;
  if (want > kMaxSplits) want = kMaxSplits;
  return want < 1 ? 1 : want;
}

// Transposing reduction over the 32 lanes (see score.cu for the pattern).
template <int R, int O>
struct TR32 {
  static __device__ __forceinline__ void run(float *v, int lane) {
    const bool upper = (lane & O) != 0;
#pragma unroll
    for (int i = 0; i < R / 2; ++i) {
      const float send = upper ? v[i] : v[i + R / 2];
      const float keep = upper ? v[i + R / 2] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, O);
    }
    TR32<R / 2, O / 2>::run(v, lane);
  }
};
template <int R>
struct TR32<R, 0> {
  static __device__ __forceinline__ void run(float *, int) {}
};

// partials layout: [BH][nsplit][Mtot][D + 2] fp32 = (acc[D], m, l)
template <typename T, int D>
__global__ void __launch_bounds__(kAttnThreads)
    attn_partial_kernel(const T *__restrict__ q, const T *__restrict__ K,
                        const T *__restrict__ V, const int *__restrict__ idx,
                        int stride, const int *__restrict__ count,
                        int count_cap, int N, int kv_rows, int B, int Hq, int Hkv, int L,
                        int nsplit, float scale, float *__restrict__ part,
                        uint32_t *status) {
  constexpr int EPL = D / 32;  // fp32 elements per lane
  grid_dep_wait();
  grid_dep_launch();
  __shared__ __align__(16) float Ks[kChunk][D];
  __shared__ __align__(16) float Vs[kChunk][D];
  __shared__ int valid[kChunk];

  const int split = blockIdx.x, bh = blockIdx.y, qb = blockIdx.z;
  const int b = bh / Hkv, h = bh % Hkv, G = Hq / Hkv;
  const int Mtot = L * G;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  int cnt = stride;
  if (count) cnt = min(max(count[bh], 0), min(stride, count_cap));
  const int per = (stride + nsplit - 1) / nsplit;
  const int k0 = split * per, k1 = min(cnt, k0 + per);
  const int *row = idx + (size_t)bh * stride;

  // queries of this warp
  float qr[kQPerWarp][EPL];
  float acc[kQPerWarp][EPL];
  float mrun[kQPerWarp], lrun[kQPerWarp];
#pragma unroll
  for (int i = 0; i < kQPerWarp; ++i) {
    const int m = qb * kQPerCta + warp * kQPerWarp + i;
    const bool ok = m < Mtot;
    const int l = ok ? m / G : 0, g = ok ? m % G : 0;
    const T *qp = q + (((size_t)l * B + b) * Hq + (size_t)h * G + g) * D + lane * EPL;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      qr[i][e] = ok ? DT<T>::to_f(qp[e]) * scale : 0.f;
      acc[i][e] = 0.f;
    }
    mrun[i] = -INFINITY;
    lrun[i] = 0.f;
  }

  for (int c0 = k0; c0 < k1; c0 += kChunk) {
    const int nc = min(kChunk, k1 - c0);
    __syncthreads();
    // gather rows: each thread moves 16-byte pieces of K and V
    constexpr int EV = 16 / (int)sizeof(T);
    constexpr int PIECES = kChunk * D / EV;
    for (int p = threadIdx.x; p < PIECES; p += kAttnThreads) {
      const int r = p / (D / EV), c = (p % (D / EV)) * EV;
      int j = r < nc ? row[c0 + r] : -1;
      const bool ok = j >= 0 && j < N;
      if (r < nc && !ok && c == 0) raise_flag(status, FLAG_INDEX);
      float fk[EV], fv[EV];
      if (ok) {
        const size_t off = ((size_t)bh * kv_rows + j) * D + c;
        unpack16<T>(*reinterpret_cast<const uint4 *>(K + off), fk);
        unpack16<T>(*reinterpret_cast<const uint4 *>(V + off), fv);
      } else {
#pragma unroll
        for (int e = 0; e < EV; ++e) fk[e] = fv[e] = 0.f;
      }
#pragma unroll
      for (int e = 0; e < EV; ++e) {
        Ks[r][c + e] = fk[e];
        Vs[r][c + e] = fv[e];
      }
      if (c == 0) valid[r] = ok;
    }
    __syncthreads();
    const bool kvalid = valid[lane] != 0;
#pragma unroll
    for (int i = 0; i < kQPerWarp; ++i) {
      float v[32];
#pragma unroll
      for (int r = 0; r < 32; ++r) {
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) a = fmaf(qr[i][e], Ks[r][lane * EPL + e], a);
        v[r] = a;
      }
      TR32<32, 16>::run(v, lane);
      // lane now holds the logit of key `lane`
      const float z = kvalid ? v[0] : -INFINITY;
      const float mx = warp_max(z);
      const float mnew = fmaxf(mrun[i], mx);
      if (mnew == -INFINITY) continue;
      const float p = expf(z - mnew);
      const float corr = expf(mrun[i] - mnew);
      lrun[i] = lrun[i] * corr + warp_sum(p);
#pragma unroll
      for (int e = 0; e < EPL; ++e) acc[i][e] *= corr;
      for (int r = 0; r < nc; ++r) {
        const float pr = __shfl_sync(0xffffffffu, p, r);
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[i][e] = fmaf(pr, Vs[r][lane * EPL + e], acc[i][e]);
      }
      mrun[i] = mnew;
    }
  }

#pragma unroll
  for (int i = 0; i < kQPerWarp; ++i) {
    const int m = qb * kQPerCta + warp * kQPerWarp + i;
    if (m >= Mtot) continue;
    float *pp = part + (((size_t)bh * nsplit + split) * Mtot + m) * (D + 2);
#pragma unroll
    for (int e = 0; e < EPL; ++e) pp[lane * EPL + e] = acc[i][e];
    if (lane == 0) {
      pp[D] = mrun[i];
      pp[D + 1] = lrun[i];
    }
  }
}

// One warp per (bh, query m): combine the splits.
template <typename T, int D>
__global__ void __launch_bounds__(256)
    attn_merge_kernel(const float *__restrict__ part, int BHM, int nsplit,
                      int Mtot, int B, int Hq, int Hkv, T *__restrict__ out,
                      float *__restrict__ lse) {
  constexpr int EPL = D / 32;
  grid_dep_wait();
  grid_dep_launch();
  const int wid = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= BHM) return;
  const int bh = wid / Mtot, m = wid % Mtot;
  const int b = bh / Hkv, h = bh % Hkv, G = Hq / Hkv;
  const int l = m / G, g = m % G;
  float M = -INFINITY;
  for (int s = 0; s < nsplit; ++s)
    M = fmaxf(M, part[(((size_t)bh * nsplit + s) * Mtot + m) * (D + 2) + D]);
  float o[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) o[e] = 0.f;
  float Lsum = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < nsplit; ++s) {
      const float *pp = part + (((size_t)bh * nsplit + s) * Mtot + m) * (D + 2);
      const float ms = pp[D];
      if (ms == -INFINITY) continue;
      const float w = expf(ms - M);
      Lsum += pp[D + 1] * w;
#pragma unroll
      for (int e = 0; e < EPL; ++e) o[e] = fmaf(pp[lane * EPL + e], w, o[e]);
    }
  }
  const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
  T *op = out + (((size_t)l * B + b) * Hq + (size_t)h * G + g) * D + lane * EPL;
#pragma unroll
  for (int e = 0; e < EPL; ++e) op[e] = DT<T>::from_f(o[e] * inv);
  if (lse && lane == 0)
    lse[((size_t)l * B + b) * Hq + (size_t)h * G + g] =
        Lsum > 0.f ? M + logf(Lsum) : -INFINITY;
}

template <typename T, int D>
cudaError_t launch_attn_t(const Shape &s, int L, const void *q, const void *K,
                          const void *V, const int *idx, int stride,
                          const int *count, int count_cap, void *out,
                          float *lse, void *ws, uint32_t *status,
                          cudaStream_t st) {
  const int Mtot = L * s.G();
  const int qblocks = (Mtot + kQPerCta - 1) / kQPerCta;
  const int nsplit = num_splits(s.BH(), qblocks, stride);
  float *part = static_cast<float *>(ws);
  const float scale = (float)(1.0 / __builtin_sqrt((double)D));
  dim3 grid(nsplit, s.BH(), qblocks);
  attn_partial_kernel<T, D><<<grid, kAttnThreads, 0, st>>>(
      static_cast<const T *>(q), static_cast<const T *>(K),
      static_cast<const T *>(V), idx, stride, count, count_cap, s.N, s.Ncap, s.B,
      s.Hq, s.Hkv, L, nsplit, scale, part, status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int BHM = s.BH() * Mtot;
  attn_merge_kernel<T, D><<<(BHM + 7) / 8, 256, 0, st>>>(
      part, BHM, nsplit, Mtot, s.B, s.Hq, s.Hkv, static_cast<T *>(out), lse);
  return cudaGetLastError();
}

}  // namespace

size_t attn_workspace_bytes(const Shape &s, int L, int stride) {
  if (s.dtype == 1) return attn_fused_workspace_bytes(s, L, stride);
  const int Mtot = L * s.G();
  const int qblocks = (Mtot + kQPerCta - 1) / kQPerCta;
  const int nsplit = num_splits(s.BH(), qblocks, stride);
  return (size_t)s.BH() * nsplit * Mtot * (s.d + 2) * sizeof(float);
}

cudaError_t launch_attn(const Shape &s, int L, const void *q, const void *K,
                        const void *V, const int *idx, int stride,
                        const int *count, int count_cap, void *out, float *lse,
                        void *ws, uint32_t *status, cudaStream_t st) {
  if (s.dtype == 1)
    return launch_attn_fused(s, L, q, K, V, idx, stride, count, out, lse, ws, status, st);
  if (s.d == 128)
    return launch_attn_t<float, 128>(s, L, q, K, V, idx, stride, count, count_cap,
                                     out, lse, ws, status, st);
  return launch_attn_t<float, 64>(s, L, q, K, V, idx, stride, count, count_cap,
                                  out, lse, ws, status, st);
}

}  // namespace sd
