// internal.h -- launchers shared between the translation units of
// libsparse_decode.  Host-side only; no torch types anywhere.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "sparse_decode.h"

namespace sd {

// Routing histogram rows: counts of the top 11 bits of the order-preserving
// score key, per (sequence, KV head).
constexpr int kHistBins = 2048;

struct Shape {
  int B, N, Hq, Hkv, d, dtype;  // dtype: 0 = fp32, 1 = bf16
  int Ncap;                     // rows allocated per (sequence, KV head) in K, V (>= N)
  int G() const { return Hq / Hkv; }
  int BH() const { return B * Hkv; }
  int esize() const { return dtype == 0 ? 4 : 2; }
};

// Reads and checks a caller's shape (the checks every entry point shares).
sparse_status_t check_shape(const sparse_shape_t *shape, Shape *s);

// Device properties cached per device (SM count, cluster support).
struct DeviceInfo {
  int sm_count = 0;
  int max_smem_optin = 0;
  int select_cluster = 0;  // largest cluster size the library launches
};
cudaError_t device_info(DeviceInfo *out);

// Programmatic dependent launch: a kernel may be scheduled while the previous
// kernel on the stream drains; it waits (griddepcontrol.wait) before using
// that kernel's results.  On unless SPARSE_DECODE_PDL=0.
bool pdl_enabled();
inline void add_pdl_attr(cudaLaunchConfig_t &cfg, cudaLaunchAttribute *attrs) {
  if (!pdl_enabled()) return;
  attrs[cfg.numAttrs].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[cfg.numAttrs].val.programmaticStreamSerializationAllowed = 1;
  ++cfg.numAttrs;
}

// The routing scan's tile claim counters live in the workspace header, at a
// fixed word offset from the status word (which is the header's first word):
// kScanCtrWord .. kScanCtrWord + 512, zero between calls.
constexpr int kScanCtrWord = 256;  // byte offset 1024
inline uint32_t *scan_counters(uint32_t *status) { return status + kScanCtrWord; }

// A1: S[b,h,j] for every key; one streaming pass over K.  hist (nullable):
// [B*Hkv][kHistBins] counts of the top 11 key bits, accumulated (must start
// zero).
cudaError_t launch_score(const Shape &s, const void *q, const void *K, float *S, uint32_t *hist,
                         uint32_t *status, cudaStream_t st);
// Keys per scan tile, and the scan's grid (one CTA per SM, at most one per tile).
int scan_stage_keys(const Shape &s);
int scan_grid(const Shape &s, int sm_count);
// A2 after the scan: one cluster per head selects the exact top-k from the
// scan's score rows S and histogram hist (complete), writes idx
// [B*Hkv][k] and clears hist.
cudaError_t launch_select_split(const Shape &s, const float *S, int k, int *idx, uint32_t *hist,
                                uint32_t *status, cudaStream_t st);

// A2 / A2': selection from S.  k >= 1: top-k (tau ignored); k == 0:
// threshold with tau and cap, count written.  idx rows have `stride`
// entries.
// hist (top-k, nullable): the scan's histogram; consumed and cleared.
cudaError_t launch_select(const Shape &s, const float *S, int k,
                          const float *tau, int cap, int *idx, int *count,
                          int stride, uint32_t *hist, uint32_t *status,
                          cudaStream_t st);

// A3 + A4: L query sets over the same index rows.  bf16 runs on the tcgen05
// tensor cores (attn_fused.cu), fp32 on the CUDA cores (attn.cu); both keep
// their split partials in the workspace (attn_workspace_bytes).
size_t attn_workspace_bytes(const Shape &s, int L, int stride);
size_t attn_fused_workspace_bytes(const Shape &s, int L, int stride);
cudaError_t launch_attn(const Shape &s, int L, const void *q, const void *K,
                        const void *V, const int *idx, int stride,
                        const int *count, int count_cap, void *out, float *lse,
                        void *ws, uint32_t *status, cudaStream_t st);
cudaError_t launch_attn_fused(const Shape &s, int L, const void *q, const void *K, const void *V,
                              const int *idx, int stride, const int *count, void *out, float *lse,
                              void *part, uint32_t *status, cudaStream_t st);
// The tail of routing fused into the attention kernel (bf16, L*G <= 128,
// N <= 131072, every split's keys on chip): top-k from the scan's score rows
// and histogram (writes idx [B*Hkv][k], clears hist), or the threshold sets
// from the marking scan's bitmaps (writes idx rows of `cap` and count).
bool fused_route_ok(const Shape &s, int L, int k_or_cap);
// part: the workspace's attention area (attn_workspace_bytes).
cudaError_t launch_route_attn_topk(const Shape &s, int L, const void *q_layers, const void *K,
                                   const void *V, int k, const float *S, uint32_t *hist,
                                   int *idx, void *out, float *lse, void *part, uint32_t *status,
                                   cudaStream_t st);
cudaError_t launch_route_attn_threshold(const Shape &s, int L, const void *q_layers,
                                        const void *K, const void *V, const uint32_t *bits,
                                        int cap, int *idx, int *count, void *out, float *lse,
                                        void *part, uint32_t *status, cudaStream_t st);

// Louver index (louver.cu).  louver_shape_ok: r and N fit the balanced tree.
bool louver_shape_ok(const Shape &s, int r);
void louver_sizes(const Shape &s, int r, size_t *index_bytes, size_t *ws_bytes);
cudaError_t louver_build(const Shape &s, const void *K, int r, void *index, void *ws,
                         cudaStream_t st);
// status: the status word to raise flags in (nullptr: the Louver workspace's).
cudaError_t louver_query(const Shape &s, const void *q, int r, const void *index,
                         const float *tau, int cap, int *idx, int *count, int *survivors,
                         void *ws, uint32_t *status, cudaStream_t st);

// Self-test of the bounded wait (selftest.cu): one thread waits on *ctr >= 1
// for limit_ns (at most the library's limit); nothing increments ctr.
cudaError_t launch_selftest_wait(uint32_t *ctr, uint64_t limit_ns, uint32_t *status,
                                 cudaStream_t st);

// A2' by marking: the scan writes, per 32 keys, the word of bits "score >=
// tau[head]" into bits [B*Hkv][ceil(N/32)] (score.cu); the compaction turns
// the words into ascending idx rows (stride cap) and counts (threshold.cu).
cudaError_t launch_threshold_mark(const Shape &s, const void *q, const void *K,
                                  const float *tau, uint32_t *bits, uint32_t *status,
                                  cudaStream_t st);
cudaError_t launch_bitmap_compact(const Shape &s, const uint32_t *bits, int cap, int *idx,
                                  int *count, uint32_t *status, cudaStream_t st);

}  // namespace sd
