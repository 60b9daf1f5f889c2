// internal.h -- launchers shared between the translation units of
// libsparse_decode.  Host-side only; no torch types anywhere.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace sd {

struct Shape {
  int B, N, Hq, Hkv, d, dtype;  // dtype: 0 = fp32, 1 = bf16
  int Ncap;                     // rows allocated per (sequence, KV head) in K, V (>= N)
  int G() const { return Hq / Hkv; }
  int BH() const { return B * Hkv; }
  int esize() const { return dtype == 0 ? 4 : 2; }
};

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

// A1: S[b,h,j] for every key; one streaming pass over K.  hist (nullable):
// [B*Hkv][2048] counts of the top 11 key bits, accumulated (must start zero).
cudaError_t launch_score(const Shape &s, const void *q, const void *K,
                         float *S, uint32_t *hist, uint32_t *status,
                         cudaStream_t st);

// A1 + A2 fused (route_fused.cu): the scan and the exact top-k in one
// persistent kernel whose CTAs synchronise per head through counters in
// global memory.  ctr: one uint32 per head, zero between calls (the kernel
// resets them); seg_area: kFusedSegAreaBytes of scratch.  Returns
// cudaErrorNotSupported, launching nothing, when the shape does not fit (a
// CTA's keys must fit on chip) or unless SPARSE_DECODE_FUSED_ROUTE=1 (the
// scan followed by the select kernel is the default: at the 128K decode
// shapes the two are on par and the two-kernel path leaves SMs free for the
// attention kernel to start early).
constexpr int kFusedMaxCtas = 256;
constexpr int kFusedMaxHeads = 768;
constexpr int kFusedSegCap = 1024;  // boundary-bin keys a CTA publishes per head
constexpr size_t kFusedMetaBytes = (size_t)kFusedMaxCtas * 2 * 8;
constexpr size_t kFusedSegAreaBytes =
    kFusedMetaBytes + (size_t)kFusedMaxCtas * 2 * kFusedSegCap * sizeof(uint32_t);
bool fused_route_enabled();
cudaError_t launch_route_topk_fused(const Shape &s, const void *q, const void *K, int k,
                                    float *S, uint32_t *hist, uint32_t *ctr, void *seg_area,
                                    int *idx, uint32_t *status, cudaStream_t st);

// Kernels whose CTAs wait for one another (the fused routing kernel, the
// split merge of the tcgen05 attention) rely on the whole grid being resident
// at once -- at most one CTA per SM.  They are launched as ordinary kernels so
// that programmatic dependent launch can overlap them with their predecessor;
// SPARSE_DECODE_COOPERATIVE=1 launches them cooperatively instead (the driver
// then guarantees co-residency even next to other work on the device).
bool cooperative_forced();
// The split attention merges its partials inside a thread-block cluster
// (distributed shared memory) when the clusters fit; SPARSE_DECODE_ATTN_MERGE=global
// selects the merge through global memory and a counter barrier instead.
bool attn_cluster_merge_enabled();

// A2 / A2': selection from S.  k >= 1: top-k (tau ignored); k == 0:
// threshold with tau and cap, count written.  idx rows have `stride`
// entries.
// hist (top-k, nullable): the scan's histogram; consumed and cleared.
cudaError_t launch_select(const Shape &s, const float *S, int k,
                          const float *tau, int cap, int *idx, int *count,
                          int stride, uint32_t *hist, uint32_t *status,
                          cudaStream_t st);

// A3 + A4: L query sets over the same index rows.  bf16 runs on the tcgen05
// tensor cores (split partials in the workspace) or, on request, the mma.sync
// kernel (split merge in distributed shared memory); fp32 runs on the CUDA
// cores with split partials in the workspace.
size_t attn_workspace_bytes(const Shape &s, int L, int stride);
cudaError_t launch_attn_mma(const Shape &s, int L, const void *q, const void *K,
                            const void *V, const int *idx, int stride,
                            const int *count, void *out, float *lse,
                            uint32_t *status, cudaStream_t st);
size_t attn_tc_workspace_bytes(const Shape &s, int L);
// Split-merge counters of the tcgen05 attention: two per (head, query block)
// in a fixed, shape-independent area of the workspace header (zero between
// calls: the kernel resets them).  More blocks than this run unsplit.
constexpr int kAttnMaxCounterBlocks = 96;
cudaError_t launch_attn_tc(const Shape &s, int L, const void *q, const void *K,
                           const void *V, const int *idx, int stride,
                           const int *count, void *out, float *lse, void *ws,
                           uint32_t *counters, uint32_t *status, cudaStream_t st);
cudaError_t launch_attn(const Shape &s, int L, const void *q, const void *K,
                        const void *V, const int *idx, int stride,
                        const int *count, int count_cap, void *out, float *lse,
                        void *ws, uint32_t *counters, uint32_t *status,
                        cudaStream_t st);

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
