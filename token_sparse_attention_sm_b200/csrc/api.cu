// api.cu -- the C ABI of libsparse_decode (declared in sparse_decode.h).
//
// Every entry point validates its arguments on the host and returns an error
// before anything is enqueued; then it enqueues the kernels on the caller's
// stream and returns.  The library allocates nothing: scratch lives in the
// caller's workspace, whose layout is
//   [0, 4096)      header: device status word (uint32) at offset 0; offset
//                  64: a word no kernel writes (the bounded-wait self-test
//                  waits on it); [1024, 3072): the routing scan's tile claim
//                  counters (zero between calls; the scan leaves them zero)
//   hist           radix histogram [max(B*Hkv, 256)][2048] uint32 (scan ->
//                  select; cleared after use) -- it must be zero between
//                  calls and sits at a fixed offset for up to 256 heads, so
//                  calls of different shapes sharing one workspace never put
//                  other data there
//   scores         fp32 S [B,Hkv,N]; threshold routing keeps its per-head
//                  bitmaps [B*Hkv][ceil(N/32)] here
//   attn           fp32 attention split partials (fp32 inputs only)
#include <stdlib.h>
#include <string.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "sparse_decode.h"

namespace sd {

cudaError_t select_cluster_size(int sm_count, int smem_optin, int *out);

namespace {
constexpr int kMaxDevices = 64;
std::once_flag g_once[kMaxDevices];
DeviceInfo g_info[kMaxDevices];
cudaError_t g_info_err[kMaxDevices];

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
constexpr size_t kHeader = 4096;
constexpr size_t kSelftestOff = 64;  // a header word no kernel writes
constexpr int kHistMinRows = 256;

struct Layout {
  size_t hist_off, scores_off, attn_off, total;
};

Layout layout(const Shape &s, int stride, int L) {
  const size_t rows = (size_t)(s.BH() > kHistMinRows ? s.BH() : kHistMinRows);
  Layout l;
  l.hist_off = kHeader;
  l.scores_off = l.hist_off + rows * kHistBins * sizeof(uint32_t);
  l.attn_off = l.scores_off + align_up((size_t)s.BH() * s.N * sizeof(float), 256);
  l.total = l.attn_off + align_up(attn_workspace_bytes(s, L, stride), 256);
  return l;
}

bool aligned(const void *p, size_t a) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

}  // namespace

sparse_status_t check_shape(const sparse_shape_t *shape, Shape *s) {
  if (!shape) return SPARSE_ERR_INVALID_ARG;
  s->B = shape->B;
  s->N = shape->N;
  s->Hq = shape->Hq;
  s->Hkv = shape->Hkv;
  s->d = shape->d;
  s->dtype = shape->dtype;
  s->Ncap = shape->n_cap == 0 ? shape->N : shape->n_cap;
  if (s->B < 1 || s->N < 1 || s->Hq < 1 || s->Hkv < 1 || s->d < 1)
    return SPARSE_ERR_INVALID_ARG;
  if (s->Ncap < s->N) return SPARSE_ERR_INVALID_ARG;
  if (s->Hq % s->Hkv != 0) return SPARSE_ERR_INVALID_ARG;
  if (s->d != 64 && s->d != 128) return SPARSE_ERR_UNSUPPORTED;
  if (s->dtype != SPARSE_DTYPE_F32 && s->dtype != SPARSE_DTYPE_BF16)
    return SPARSE_ERR_UNSUPPORTED;
  if (s->G() > 16) return SPARSE_ERR_UNSUPPORTED;
  if ((long long)s->B * s->Hkv > 65535) return SPARSE_ERR_UNSUPPORTED;
  return SPARSE_OK;
}

namespace {

sparse_status_t check_ws(const Shape &s, int stride, int L, void *ws,
                         size_t ws_bytes) {
  if (!ws || !aligned(ws, 256)) return SPARSE_ERR_INVALID_ARG;
  if (ws_bytes < layout(s, stride, L).total) return SPARSE_ERR_WORKSPACE;
  return SPARSE_OK;
}

sparse_status_t from_cuda(cudaError_t e) {
  return e == cudaSuccess ? SPARSE_OK : SPARSE_ERR_CUDA;
}

uint32_t *status_word(void *ws) { return static_cast<uint32_t *>(ws); }

template <typename T>
T *at(void *ws, size_t off) {
  return reinterpret_cast<T *>(static_cast<char *>(ws) + off);
}
uint32_t *hist_ptr(void *ws, const Layout &l) { return at<uint32_t>(ws, l.hist_off); }
float *scores_ptr(void *ws, const Layout &l) { return at<float>(ws, l.scores_off); }
void *attn_ptr(void *ws, const Layout &l) { return at<char>(ws, l.attn_off); }

// A1 + A2 (top-k): the scan (scores and histogram), then the split select.
cudaError_t route_topk_any(const Shape &s, const void *q, const void *K, int k, int *idx,
                           void *ws, const Layout &l, cudaStream_t st) {
  float *S = scores_ptr(ws, l);
  uint32_t *hist = hist_ptr(ws, l);
  cudaError_t e = launch_score(s, q, K, S, hist, status_word(ws), st);
  if (e == cudaSuccess) e = launch_select_split(s, S, k, idx, hist, status_word(ws), st);
  return e;
}

// A1 + A2' (threshold): the scan marks the keys >= tau in per-head bitmaps
// (in the scores area, which threshold routing does not need), then one
// cluster per head writes the ordered sets.
cudaError_t route_threshold_any(const Shape &s, const void *q, const void *K, const float *tau,
                                int cap, int *idx, int *count, void *ws, const Layout &l,
                                cudaStream_t st) {
  uint32_t *bits = reinterpret_cast<uint32_t *>(scores_ptr(ws, l));
  cudaError_t e = launch_threshold_mark(s, q, K, tau, bits, status_word(ws), st);
  if (e == cudaSuccess) e = launch_bitmap_compact(s, bits, cap, idx, count, status_word(ws), st);
  return e;
}

}  // namespace

bool pdl_enabled() {
  static const bool on = [] {
    const char *v = getenv("SPARSE_DECODE_PDL");
    return !(v && v[0] == '0');
  }();
  return on;
}

cudaError_t device_info(DeviceInfo *out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::call_once(g_once[dev], [dev]() {
    DeviceInfo di;
    cudaError_t err =
        cudaDeviceGetAttribute(&di.sm_count, cudaDevAttrMultiProcessorCount, dev);
    if (err == cudaSuccess)
      err = cudaDeviceGetAttribute(&di.max_smem_optin,
                                   cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (err == cudaSuccess)
      err = select_cluster_size(di.sm_count, di.max_smem_optin,
                                &di.select_cluster);
    g_info[dev] = di;
    g_info_err[dev] = err;
  });
  *out = g_info[dev];
  return g_info_err[dev];
}

// Checks shared by the decode-step entry points (L layers per routing set).
sparse_status_t check_decode_args(const Shape &s, int32_t L, const void *q_route,
                                  const void *q_layers, const void *K, const void *V,
                                  int32_t k, const float *tau, int32_t cap, int32_t *idx,
                                  int32_t *count, void *out, float *lse) {
  if (L < 1 || !q_route || !q_layers || !K || !V || !idx || !out)
    return SPARSE_ERR_INVALID_ARG;
  if ((long long)L * s.G() > 1024) return SPARSE_ERR_UNSUPPORTED;
  if (k > 0) {
    if (k > s.N || tau) return SPARSE_ERR_INVALID_ARG;
  } else {
    if (k < 0 || !tau || !count || cap < 1) return SPARSE_ERR_INVALID_ARG;
  }
  if (!aligned(q_route, 16) || !aligned(q_layers, 16) || !aligned(K, 16) ||
      !aligned(V, 16) || !aligned(out, 16) || !aligned(idx, 4) ||
      (count && !aligned(count, 4)) || (tau && !aligned(tau, 4)) ||
      (lse && !aligned(lse, 4)))
    return SPARSE_ERR_INVALID_ARG;
  return SPARSE_OK;
}

// Route once with q_route, then attend L layers over that set (arguments
// checked by the caller; the workspace layout l fits L layers).  bf16 steps
// whose shape allows it finish the routing inside the attention kernel (the
// scan, then one kernel); the others run the select (or the threshold
// compaction) as a kernel of its own before the attention.
// layers_ready (may be null): an event the attention waits on after the
// routing is enqueued, so the layers' queries may still be in flight while
// the routing runs.
cudaError_t decode_step_enqueue(const Shape &s, int L, const void *q_route,
                                const void *q_layers, const void *K, const void *V, int k,
                                const float *tau, int cap, int *idx, int *count, void *out,
                                float *lse, void *ws, const Layout &l, cudaStream_t st,
                                cudaEvent_t layers_ready) {
  const bool topk = k > 0;
  const int stride = topk ? k : cap;
  uint32_t *status = status_word(ws);
  const bool fused = fused_route_ok(s, L, stride);
  auto join = [&]() {
    return layers_ready ? cudaStreamWaitEvent(st, layers_ready, 0) : cudaSuccess;
  };
  cudaError_t e;
  if (topk && fused) {
    float *S = scores_ptr(ws, l);
    uint32_t *hist = hist_ptr(ws, l);
    e = launch_score(s, q_route, K, S, hist, status, st);
    if (e == cudaSuccess) e = join();
    if (e == cudaSuccess)
      e = launch_route_attn_topk(s, L, q_layers, K, V, k, S, hist, idx, out, lse, attn_ptr(ws, l),
                                 status, st);
    return e;
  }
  if (!topk && fused) {
    uint32_t *bits = reinterpret_cast<uint32_t *>(scores_ptr(ws, l));
    e = launch_threshold_mark(s, q_route, K, tau, bits, status, st);
    if (e == cudaSuccess) e = join();
    if (e == cudaSuccess)
      e = launch_route_attn_threshold(s, L, q_layers, K, V, bits, cap, idx, count, out, lse,
                                      attn_ptr(ws, l), status, st);
    return e;
  }
  if (topk) {
    e = route_topk_any(s, q_route, K, k, idx, ws, l, st);
  } else {
    e = route_threshold_any(s, q_route, K, tau, cap, idx, count, ws, l, st);
  }
  if (e == cudaSuccess) e = join();
  if (e == cudaSuccess)
    e = launch_attn(s, L, q_layers, K, V, idx, stride, topk ? nullptr : count, stride, out,
                    lse, attn_ptr(ws, l), status, st);
  return e;
}

}  // namespace sd

using sd::Shape;

extern "C" {

const char *sparse_status_string(sparse_status_t status) {
  switch (status) {
    case SPARSE_OK: return "SPARSE_OK";
    case SPARSE_ERR_INVALID_ARG: return "SPARSE_ERR_INVALID_ARG: invalid argument";
    case SPARSE_ERR_UNSUPPORTED: return "SPARSE_ERR_UNSUPPORTED: unsupported shape or dtype";
    case SPARSE_ERR_WORKSPACE: return "SPARSE_ERR_WORKSPACE: workspace too small";
    case SPARSE_ERR_CAPACITY: return "SPARSE_ERR_CAPACITY: threshold set larger than cap";
    case SPARSE_ERR_NONFINITE: return "SPARSE_ERR_NONFINITE: non-finite score or tau";
    case SPARSE_ERR_CUDA: return "SPARSE_ERR_CUDA: CUDA runtime error";
    case SPARSE_ERR_TIMEOUT: return "SPARSE_ERR_TIMEOUT: bounded device wait expired";
    case SPARSE_ERR_INDEX: return "SPARSE_ERR_INDEX: index outside [0, N)";
    case SPARSE_ERR_INTERNAL: return "SPARSE_ERR_INTERNAL: internal consistency check failed";
  }
  return "SPARSE_ERR_UNKNOWN";
}

int32_t sparse_version(void) { return 100; }

sparse_status_t sparse_workspace_size(const sparse_shape_t *shape,
                                      int32_t k_or_cap, int32_t L,
                                      size_t *bytes) {
  Shape s;
  sparse_status_t r = sd::check_shape(shape, &s);
  if (r != SPARSE_OK) return r;
  if (!bytes || k_or_cap < 1 || L < 1) return SPARSE_ERR_INVALID_ARG;
  if ((long long)L * s.G() > 1024) return SPARSE_ERR_UNSUPPORTED;
  *bytes = sd::layout(s, k_or_cap, L).total;
  return SPARSE_OK;
}

sparse_status_t sparse_workspace_init(void *ws, size_t ws_bytes, void *stream) {
  if (!ws || ws_bytes < 256) return SPARSE_ERR_INVALID_ARG;
  return sd::from_cuda(
      cudaMemsetAsync(ws, 0, ws_bytes, static_cast<cudaStream_t>(stream)));
}

sparse_status_t sparse_score(const sparse_shape_t *shape, const void *q,
                             const void *K, float *S, void *ws,
                             size_t ws_bytes, void *stream) {
  Shape s;
  sparse_status_t r = sd::check_shape(shape, &s);
  if (r != SPARSE_OK) return r;
  if (!q || !K || !S) return SPARSE_ERR_INVALID_ARG;
  if (!sd::aligned(q, 16) || !sd::aligned(K, 16) || !sd::aligned(S, 16))
    return SPARSE_ERR_INVALID_ARG;
  if ((r = sd::check_ws(s, 1, 1, ws, ws_bytes)) != SPARSE_OK) return r;
  return sd::from_cuda(
      sd::launch_score(s, q, K, S, nullptr, sd::status_word(ws), static_cast<cudaStream_t>(stream)));
}

sparse_status_t sparse_select_topk(const sparse_shape_t *shape,
                                   const float *S, int32_t k, int32_t *idx,
                                   void *ws, size_t ws_bytes, void *stream) {
  Shape s;
  sparse_status_t r = sd::check_shape(shape, &s);
  if (r != SPARSE_OK) return r;
  if (!S || !idx || k < 1 || k > s.N) return SPARSE_ERR_INVALID_ARG;
  if (!sd::aligned(S, 16) || !sd::aligned(idx, 4)) return SPARSE_ERR_INVALID_ARG;
  if ((r = sd::check_ws(s, k, 1, ws, ws_bytes)) != SPARSE_OK) return r;
  return sd::from_cuda(sd::launch_select(s, S, k, nullptr, 0, idx, nullptr, k,
                                         nullptr, sd::status_word(ws),
                                         static_cast<cudaStream_t>(stream)));
}

sparse_status_t sparse_select_threshold(const sparse_shape_t *shape,
                                        const float *S, const float *tau,
                                        int32_t cap, int32_t *idx,
                                        int32_t *count, void *ws,
                                        size_t ws_bytes, void *stream) {
  Shape s;
  sparse_status_t r = sd::check_shape(shape, &s);
  if (r != SPARSE_OK) return r;
  if (!S || !tau || !idx || !count || cap < 1) return SPARSE_ERR_INVALID_ARG;
  if (!sd::aligned(S, 16) || !sd::aligned(tau, 4) || !sd::aligned(idx, 4) ||
      !sd::aligned(count, 4))
    return SPARSE_ERR_INVALID_ARG;
  if ((r = sd::check_ws(s, cap, 1, ws, ws_bytes)) != SPARSE_OK) return r;
  return sd::from_cuda(sd::launch_select(s, S, 0, tau, cap, idx, count, cap,
                                         nullptr, sd::status_word(ws),
                                         static_cast<cudaStream_t>(stream)));
}

sparse_status_t sparse_route_topk(const sparse_shape_t *shape, const void *q,
                                  const void *K, int32_t k, int32_t *idx,
                                  void *ws, size_t ws_bytes, void *stream) {
  Shape s;
  sparse_status_t r = sd::check_shape(shape, &s);
  if (r != SPARSE_OK) return r;
  if (!q || !K || !idx || k < 1 || k > s.N) return SPARSE_ERR_INVALID_ARG;
  if (!sd::aligned(q, 16) || !sd::aligned(K, 16) || !sd::aligned(idx, 4))
    return SPARSE_ERR_INVALID_ARG;
  if ((r = sd::check_ws(s, k, 1, ws, ws_bytes)) != SPARSE_OK) return r;
  const sd::Layout l = sd::layout(s, k, 1);
  cudaError_t e =
      sd::route_topk_any(s, q, K, k, idx, ws, l, static_cast<cudaStream_t>(stream));
  return sd::from_cuda(e);
}

sparse_status_t sparse_route_threshold(const sparse_shape_t *shape,
                                       const void *q, const void *K,
                                       const float *tau, int32_t cap,
                                       int32_t *idx, int32_t *count, void *ws,
                                       size_t ws_bytes, void *stream) {
  Shape s;
  sparse_status_t r = sd::check_shape(shape, &s);
  if (r != SPARSE_OK) return r;
  if (!q || !K || !tau || !idx || !count || cap < 1) return SPARSE_ERR_INVALID_ARG;
  if (!sd::aligned(q, 16) || !sd::aligned(K, 16) || !sd::aligned(tau, 4) ||
      !sd::aligned(idx, 4) || !sd::aligned(count, 4))
    return SPARSE_ERR_INVALID_ARG;
  if ((r = sd::check_ws(s, cap, 1, ws, ws_bytes)) != SPARSE_OK) return r;
  const sd::Layout l = sd::layout(s, cap, 1);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return sd::from_cuda(sd::route_threshold_any(s, q, K, tau, cap, idx, count, ws, l, st));
}

sparse_status_t sparse_attn_gather(const sparse_shape_t *shape, int32_t L,
                                   const void *q, const void *K,
                                   const void *V, const int32_t *idx,
                                   int32_t stride, const int32_t *count,
                                   void *out, float *lse, void *ws,
                                   size_t ws_bytes, void *stream) {
  Shape s;
  sparse_status_t r = sd::check_shape(shape, &s);
  if (r != SPARSE_OK) return r;
  if (L < 1 || !q || !K || !V || !idx || stride < 1 || !out)
    return SPARSE_ERR_INVALID_ARG;
  if ((long long)L * s.G() > 1024) return SPARSE_ERR_UNSUPPORTED;
  if (!sd::aligned(q, 16) || !sd::aligned(K, 16) || !sd::aligned(V, 16) ||
      !sd::aligned(out, 16) || !sd::aligned(idx, 4) ||
      (count && !sd::aligned(count, 4)) || (lse && !sd::aligned(lse, 4)))
    return SPARSE_ERR_INVALID_ARG;
  if ((r = sd::check_ws(s, stride, L, ws, ws_bytes)) != SPARSE_OK) return r;
  const sd::Layout l = sd::layout(s, stride, L);
  return sd::from_cuda(sd::launch_attn(s, L, q, K, V, idx, stride, count, stride, out, lse,
                                       sd::attn_ptr(ws, l), sd::status_word(ws),
                                       static_cast<cudaStream_t>(stream)));
}

sparse_status_t sparse_decode_step(const sparse_shape_t *shape, int32_t L,
                                   const void *q_route, const void *q_layers,
                                   const void *K, const void *V, int32_t k,
                                   const float *tau, int32_t cap,
                                   int32_t *idx, int32_t *count, void *out,
                                   float *lse, void *ws, size_t ws_bytes,
                                   void *stream) {
  return sparse_decode_step_join(shape, L, q_route, q_layers, K, V, k, tau, cap, idx, count, out,
                                 lse, ws, ws_bytes, stream, nullptr);
}

sparse_status_t sparse_decode_step_join(const sparse_shape_t *shape, int32_t L,
                                        const void *q_route, const void *q_layers,
                                        const void *K, const void *V, int32_t k,
                                        const float *tau, int32_t cap, int32_t *idx,
                                        int32_t *count, void *out, float *lse, void *ws,
                                        size_t ws_bytes, void *stream, void *layers_ready) {
  Shape s;
  sparse_status_t r = sd::check_shape(shape, &s);
  if (r != SPARSE_OK) return r;
  if ((r = sd::check_decode_args(s, L, q_route, q_layers, K, V, k, tau, cap, idx, count, out,
                                 lse)) != SPARSE_OK)
    return r;
  const int stride = k > 0 ? k : cap;
  if ((r = sd::check_ws(s, stride, L, ws, ws_bytes)) != SPARSE_OK) return r;
  return sd::from_cuda(sd::decode_step_enqueue(s, L, q_route, q_layers, K, V, k, tau, cap, idx,
                                               count, out, lse, ws, sd::layout(s, stride, L),
                                               static_cast<cudaStream_t>(stream),
                                               static_cast<cudaEvent_t>(layers_ready)));
}

sparse_status_t sparse_decode_step_fused(const sparse_shape_t *shape, int32_t L, int32_t k,
                                         int32_t cap, int32_t *fused) {
  Shape s;
  sparse_status_t r = sd::check_shape(shape, &s);
  if (r != SPARSE_OK) return r;
  if (!fused || L < 1 || k < 0 || (k == 0 && cap < 1) || (k > 0 && k > s.N))
    return SPARSE_ERR_INVALID_ARG;
  *fused = sd::fused_route_ok(s, L, k > 0 ? k : cap) ? 1 : 0;
  return SPARSE_OK;
}

sparse_status_t sparse_decode_step_grouped(const sparse_shape_t *shape, int32_t L, int32_t R,
                                           const void *q_routes, const void *q_layers,
                                           const void *K, const void *V, int32_t k,
                                           const float *tau, int32_t cap, int32_t *idx,
                                           int32_t *count, void *out, float *lse, void *ws,
                                           size_t ws_bytes, void *stream) {
  Shape s;
  sparse_status_t r = sd::check_shape(shape, &s);
  if (r != SPARSE_OK) return r;
  if (R < 1) return SPARSE_ERR_INVALID_ARG;
  const int Lg = R < L ? R : L;  // layers per routing group
  if ((r = sd::check_decode_args(s, Lg, q_routes, q_layers, K, V, k, tau, cap, idx, count, out,
                                 lse)) != SPARSE_OK)
    return r;
  if (L < 1) return SPARSE_ERR_INVALID_ARG;
  const int stride = k > 0 ? k : cap;
  if ((r = sd::check_ws(s, stride, Lg, ws, ws_bytes)) != SPARSE_OK) return r;
  const sd::Layout l = sd::layout(s, stride, Lg);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t qsz = (size_t)s.B * s.Hq * s.d * s.esize();  // one [B,Hq,d] query set
  const int ngroups = (L + R - 1) / R;
  cudaError_t e = cudaSuccess;
  for (int g = 0; g < ngroups && e == cudaSuccess; ++g) {
    const int l0 = g * R, lg = L - l0 < R ? L - l0 : R;
    e = sd::decode_step_enqueue(
        s, lg, static_cast<const char *>(q_routes) + g * qsz,
        static_cast<const char *>(q_layers) + (size_t)l0 * qsz, K, V, k,
        tau ? tau + (size_t)g * s.BH() : nullptr, cap, idx + (size_t)g * s.BH() * stride,
        count ? count + (size_t)g * s.BH() : nullptr, static_cast<char *>(out) + (size_t)l0 * qsz,
        lse ? lse + (size_t)l0 * s.B * s.Hq : nullptr, ws, l, st, nullptr);
  }
  return sd::from_cuda(e);
}

sparse_status_t sparse_louver_sizes(const sparse_shape_t *shape, int32_t r,
                                    size_t *index_bytes, size_t *ws_bytes) {
  Shape s;
  sparse_status_t rc = sd::check_shape(shape, &s);
  if (rc != SPARSE_OK) return rc;
  if (!index_bytes || !ws_bytes) return SPARSE_ERR_INVALID_ARG;
  if (!sd::louver_shape_ok(s, r)) return SPARSE_ERR_UNSUPPORTED;
  sd::louver_sizes(s, r, index_bytes, ws_bytes);
  return SPARSE_OK;
}

sparse_status_t sparse_louver_build(const sparse_shape_t *shape, const void *K, int32_t r,
                                    void *index, size_t index_bytes, void *ws,
                                    size_t ws_bytes, void *stream) {
  Shape s;
  sparse_status_t rc = sd::check_shape(shape, &s);
  if (rc != SPARSE_OK) return rc;
  if (!K || !index || !ws) return SPARSE_ERR_INVALID_ARG;
  if (!sd::aligned(K, 16) || !sd::aligned(index, 256) || !sd::aligned(ws, 256))
    return SPARSE_ERR_INVALID_ARG;
  if (!sd::louver_shape_ok(s, r)) return SPARSE_ERR_UNSUPPORTED;
  size_t ib = 0, wb = 0;
  sd::louver_sizes(s, r, &ib, &wb);
  if (index_bytes < ib || ws_bytes < wb) return SPARSE_ERR_WORKSPACE;
  return sd::from_cuda(sd::louver_build(s, K, r, index, ws, static_cast<cudaStream_t>(stream)));
}

sparse_status_t sparse_louver_route_threshold(const sparse_shape_t *shape, const void *q,
                                              const void *index, size_t index_bytes, int32_t r,
                                              const float *tau, int32_t cap, int32_t *idx,
                                              int32_t *count, int32_t *survivors, void *ws,
                                              size_t ws_bytes, void *stream) {
  Shape s;
  sparse_status_t rc = sd::check_shape(shape, &s);
  if (rc != SPARSE_OK) return rc;
  if (!q || !index || !tau || !idx || !count || !ws || cap < 1) return SPARSE_ERR_INVALID_ARG;
  if (!sd::aligned(q, 16) || !sd::aligned(index, 256) ||
      !sd::aligned(tau, 4) || !sd::aligned(idx, 4) || !sd::aligned(count, 4) ||
      !sd::aligned(survivors, 4) || !sd::aligned(ws, 256))
    return SPARSE_ERR_INVALID_ARG;
  if (!sd::louver_shape_ok(s, r)) return SPARSE_ERR_UNSUPPORTED;
  size_t ib = 0, wb = 0;
  sd::louver_sizes(s, r, &ib, &wb);
  if (index_bytes < ib || ws_bytes < wb) return SPARSE_ERR_WORKSPACE;
  return sd::from_cuda(sd::louver_query(s, q, r, index, tau, cap, idx, count, survivors, ws,
                                        nullptr, static_cast<cudaStream_t>(stream)));
}

sparse_status_t sparse_louver_decode_step(const sparse_shape_t *shape, int32_t L,
                                          const void *q_route, const void *q_layers,
                                          const void *K, const void *V, const void *index,
                                          size_t index_bytes, int32_t r, const float *tau,
                                          int32_t cap, int32_t *idx, int32_t *count, void *out,
                                          float *lse, void *louver_ws, size_t louver_ws_bytes,
                                          void *ws, size_t ws_bytes, void *stream) {
  Shape s;
  sparse_status_t rc = sd::check_shape(shape, &s);
  if (rc != SPARSE_OK) return rc;
  if ((rc = sd::check_decode_args(s, L, q_route, q_layers, K, V, 0, tau, cap, idx, count, out,
                                  lse)) != SPARSE_OK)
    return rc;
  if (!index || !louver_ws || !sd::aligned(index, 256) || !sd::aligned(louver_ws, 256))
    return SPARSE_ERR_INVALID_ARG;
  if (!sd::louver_shape_ok(s, r)) return SPARSE_ERR_UNSUPPORTED;
  size_t ib = 0, wb = 0;
  sd::louver_sizes(s, r, &ib, &wb);
  if (index_bytes < ib || louver_ws_bytes < wb) return SPARSE_ERR_WORKSPACE;
  if ((rc = sd::check_ws(s, cap, L, ws, ws_bytes)) != SPARSE_OK) return rc;
  const sd::Layout l = sd::layout(s, cap, L);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // one status word for the step: the attention workspace's
  cudaError_t e = sd::louver_query(s, q_route, r, index, tau, cap, idx, count, nullptr,
                                   louver_ws, sd::status_word(ws), st);
  if (e == cudaSuccess)
    e = sd::launch_attn(s, L, q_layers, K, V, idx, cap, count, cap, out, lse, sd::attn_ptr(ws, l),
                        sd::status_word(ws), st);
  return sd::from_cuda(e);
}

sparse_status_t sparse_selftest_bounded_wait(void *ws, size_t ws_bytes, uint64_t limit_ns,
                                             void *stream) {
  if (!ws || !sd::aligned(ws, 256) || ws_bytes < sd::kHeader) return SPARSE_ERR_INVALID_ARG;
  // a header word that no kernel writes: the wait cannot be satisfied
  uint32_t *ctr = reinterpret_cast<uint32_t *>(static_cast<char *>(ws) + sd::kSelftestOff);
  return sd::from_cuda(sd::launch_selftest_wait(ctr, limit_ns, sd::status_word(ws),
                                                static_cast<cudaStream_t>(stream)));
}

sparse_status_t sparse_read_device_status(void *ws, void *stream,
                                          uint32_t *flags) {
  if (!ws) return SPARSE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t f = 0;
  cudaError_t e = cudaStreamSynchronize(st);
  if (e == cudaSuccess) e = cudaMemcpy(&f, ws, sizeof(f), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemsetAsync(ws, 0, sizeof(f), st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return SPARSE_ERR_CUDA;
  if (flags) *flags = f;
  if (f & sd::FLAG_TIMEOUT) return SPARSE_ERR_TIMEOUT;
  if (f & sd::FLAG_INTERNAL) return SPARSE_ERR_INTERNAL;
  if (f & sd::FLAG_INDEX) return SPARSE_ERR_INDEX;
  if (f & sd::FLAG_NONFINITE) return SPARSE_ERR_NONFINITE;
  if (f & sd::FLAG_CAPACITY) return SPARSE_ERR_CAPACITY;
  return SPARSE_OK;
}

sparse_status_t sparse_graph_launch(void *graph_exec, void *stream) {
  if (!graph_exec) return SPARSE_ERR_INVALID_ARG;
  return sd::from_cuda(cudaGraphLaunch(static_cast<cudaGraphExec_t>(graph_exec),
                                       static_cast<cudaStream_t>(stream)));
}

sparse_status_t sparse_graph_upload(void *graph_exec, void *stream) {
  if (!graph_exec) return SPARSE_ERR_INVALID_ARG;
  return sd::from_cuda(cudaGraphUpload(static_cast<cudaGraphExec_t>(graph_exec),
                                       static_cast<cudaStream_t>(stream)));
}

sparse_status_t sparse_pointer_device_usable(const void *p, int32_t *usable) {
  if (!p || !usable) return SPARSE_ERR_INVALID_ARG;
  *usable = 0;
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    (void)cudaGetLastError();  // an unknown pointer is an answer, not a failure
    return SPARSE_OK;
  }
  switch (a.type) {
    case cudaMemoryTypeDevice:
    case cudaMemoryTypeHost:
      *usable = a.devicePointer == p ? 1 : 0;
      break;
    case cudaMemoryTypeManaged:
      *usable = 1;
      break;
    default:
      break;
  }
  return SPARSE_OK;
}

}  // extern "C"
