/*
 * sparse_decode.h -- C ABI of the shared-routing token-sparse decode
 * attention library for NVIDIA B200 (sm_100a).
 *
 * What the library computes (page title, section):
 *  - CLSA article "CLSAとは？ルーティング共有で128Kコンテキスト推論を17倍高速化する
 *    スパースアテンション", section 研究の背景と課題: token-level sparse
 *    attention attends only to the k highest-scoring cached tokens;
 *  - same page, section CLSAの仕組み: the top-k routing set is computed once
 *    per query token over the one shared (YOCO) KV cache, and every
 *    cross-decoder layer reuses that set unchanged;
 *  - same page, section 計算コストの削減効果: routing costs one pass over the
 *    context per step instead of one per layer;
 *  - Louver summary "技術サマリー：スパースアテンションを範囲検索問題として捉える",
 *    sections 問題定義 and 1. 半空間範囲検索への帰着: the threshold variant keeps
 *    every key whose score is >= tau (the halfspace {p : <q,p> >= tau}),
 *    with no false negatives and a set size that varies per query.
 *
 * Definitions used by every entry point:
 *  - G = Hq / Hkv query heads share one KV head; query head hq reads KV head
 *    hq / G (contiguous groups).
 *  - Routing score of key j for KV head h of sequence b:
 *        S[b,h,j] = (sum over the G query heads g of h: <q[b,g,:], K[b,h,j,:]>)
 *                   / sqrt(d), accumulated in fp32.
 *  - Top-k set: the k keys with the largest S; at equal S the lower key
 *    index wins; -0.0 and +0.0 are equal.  Threshold set: every j with
 *    S[b,h,j] >= tau[b,h] (inclusive, tau in the units of S).  Sets are
 *    returned in ascending key order.
 *  - Attention of query vector x over a set I of keys of head h:
 *        z_j = <x, K[b,h,j,:]> / sqrt(d),  o = sum_j softmax(z)_j V[b,h,j,:],
 *        lse = log sum_j exp(z_j); fp32 softmax and accumulation; o is
 *    written in the input dtype (round to nearest even).  An empty set gives
 *    o = 0 and lse = -inf.
 *
 * Layouts: every tensor is dense and row-major in the order shown.
 *    q, q_route [B,Hq,d]      q_layers [L,B,Hq,d]      K, V [B,Hkv,N,d]
 *    S [B,Hkv,N] fp32         tau [B,Hkv] fp32         count [B,Hkv] int32
 *    idx [B,Hkv,stride] int32 out [L,B,Hq,d]           lse [L,B,Hq] fp32
 * q/K/V/out share one dtype (fp32 or bf16).  All pointers are device
 * pointers owned by the caller; the library allocates nothing and keeps no
 * per-call state.  q, K, V, S and out must be 16-byte aligned.  out may also
 * be pinned host memory that kernels reach at its own address (checked with
 * sparse_pointer_device_usable): the attention then writes the results
 * straight to the host, and they are there once the stream has passed the
 * call.
 *
 * Supported: d in {64, 128}; dtype fp32 or bf16; 1 <= G <= 16; N >= 1;
 * B*Hkv <= 65535; L*G <= 1024.
 *
 * Errors: argument problems are returned synchronously, before anything is
 * enqueued.  Conditions only the device can see (a non-finite score, a
 * threshold set larger than its capacity, an index outside [0,N), a bounded
 * wait that expired) are OR-ed into a status word kept in the workspace and
 * read back with sparse_read_device_status().  Kernels never trap.
 *
 * Workspace: every compute entry point takes (ws, ws_bytes); ws_bytes must
 * be at least sparse_workspace_size() for the same arguments.  The
 * workspace must be zero-filled once before its first use (for example with
 * sparse_workspace_init); the library leaves it reusable afterwards.  Calls
 * that share a workspace must be ordered (same stream, or synchronised).
 *
 * Asynchrony: every compute entry point enqueues its kernels on `stream`
 * and returns without synchronising.
 *
 * Co-residency: no kernel of the library waits for a CTA that is not
 * already running.  The top-k select and the bf16 attention split each head
 * over up to 16 CTAs that form one thread-block cluster (the hardware
 * schedules a cluster's CTAs together) and meet only at cluster barriers.
 * The routing scan's CTAs never wait for one another: they claim tiles
 * through counters (a CTA whose claims fail simply stops).  The Louver
 * query, whose CTAs of a head meet at a counter barrier in global memory, is
 * launched cooperatively (the driver then guarantees that the whole grid is
 * resident) whenever a head spans several CTAs.  So another kernel or
 * process sharing the device can slow a call down but cannot stall it.
 *
 * Environment variables read by the library:
 *   SPARSE_DECODE_PDL=0           no programmatic dependent launch between
 *                                 the library's kernels
 */
#ifndef SPARSE_DECODE_H_
#define SPARSE_DECODE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SPARSE_OK = 0,
  SPARSE_ERR_INVALID_ARG = 1, /* null pointer, bad size, misalignment */
  SPARSE_ERR_UNSUPPORTED = 2, /* d, dtype or G outside the supported set */
  SPARSE_ERR_WORKSPACE = 3,   /* ws_bytes smaller than required */
  SPARSE_ERR_CAPACITY = 4,    /* device: a threshold set exceeded cap */
  SPARSE_ERR_NONFINITE = 5,   /* device: a score (or tau) was NaN/Inf */
  SPARSE_ERR_CUDA = 6,        /* a CUDA runtime call or launch failed */
  SPARSE_ERR_TIMEOUT = 7,     /* device: a bounded wait expired */
  SPARSE_ERR_INDEX = 8,       /* device: an idx entry was outside [0,N) */
  SPARSE_ERR_INTERNAL = 9     /* device: an internal consistency check failed */
} sparse_status_t;

typedef enum { SPARSE_DTYPE_F32 = 0, SPARSE_DTYPE_BF16 = 1 } sparse_dtype_t;

typedef struct {
  int32_t B;     /* sequences */
  int32_t N;     /* cached tokens per sequence (the current length) */
  int32_t Hq;    /* query heads */
  int32_t Hkv;   /* KV heads; Hq % Hkv == 0 */
  int32_t d;     /* head dimension */
  int32_t dtype; /* sparse_dtype_t of q, K, V and out */
  int32_t n_cap; /* rows allocated per (sequence, KV head) in K and V: K and V
                    are [B,Hkv,n_cap,d] and rows 0..N-1 are the cache; 0 means
                    n_cap = N (a dense cache); otherwise n_cap >= N */
} sparse_shape_t;

/* Human-readable name of a status code (static string, never NULL). */
const char *sparse_status_string(sparse_status_t status);

/* Library version as major*10000 + minor*100 + patch. */
int32_t sparse_version(void);

/* Bytes of workspace needed by every entry point for this shape, where
 * k_or_cap is the top-k size or threshold capacity (the idx stride) and L
 * the number of query sets (layers) attended per call.  Synchronous. */
sparse_status_t sparse_workspace_size(const sparse_shape_t *shape,
                                      int32_t k_or_cap, int32_t L,
                                      size_t *bytes);

/* Zero-fill the workspace (enqueued on stream). */
sparse_status_t sparse_workspace_init(void *ws, size_t ws_bytes,
                                      void *stream);

/* Routing scores only: S[b,h,j] as defined above, for every cached key
 * (CLSA article, section 研究の背景と課題: the score that decides which
 * tokens matter).  One streaming pass over K. */
sparse_status_t sparse_score(const sparse_shape_t *shape, const void *q,
                             const void *K, float *S, void *ws,
                             size_t ws_bytes, void *stream);

/* Top-k selection from given scores S [B,Hkv,N] (shape->Hq, d and dtype are
 * ignored): idx [B,Hkv,k] ascending, ties to the lower index (CLSA
 * article, section 研究の背景と課題).  1 <= k <= N. */
sparse_status_t sparse_select_topk(const sparse_shape_t *shape,
                                   const float *S, int32_t k, int32_t *idx,
                                   void *ws, size_t ws_bytes, void *stream);

/* Threshold selection from given scores: every j with S >= tau[b,h]
 * (Louver summary, section 1. 半空間範囲検索への帰着).  count[b,h] receives
 * the true set size; the lowest min(count, cap) indices are written to
 * idx [B,Hkv,cap] in ascending order.  A set larger than cap raises
 * SPARSE_ERR_CAPACITY in the device status. */
sparse_status_t sparse_select_threshold(const sparse_shape_t *shape,
                                        const float *S, const float *tau,
                                        int32_t cap, int32_t *idx,
                                        int32_t *count, void *ws,
                                        size_t ws_bytes, void *stream);

/* Shared routing, top-k form: scores of q [B,Hq,d] against every key of K,
 * then the top-k set per (b, KV head) into idx [B,Hkv,k] (CLSA article,
 * section CLSAの仕組み: computed once, reused by all layers). */
sparse_status_t sparse_route_topk(const sparse_shape_t *shape, const void *q,
                                  const void *K, int32_t k, int32_t *idx,
                                  void *ws, size_t ws_bytes, void *stream);

/* Shared routing, threshold form (Louver summary, sections 問題定義 and
 * 1. 半空間範囲検索への帰着): the set sparse_select_threshold returns on the
 * scores of q (the same fp32 scores, the same comparison), computed without
 * storing them: the scan marks the keys >= tau[b,h] in per-head bitmaps in
 * the workspace and one cluster per head writes the ascending idx rows and
 * count (SPARSE_ERR_CAPACITY through the status word when count > cap). */
sparse_status_t sparse_route_threshold(const sparse_shape_t *shape,
                                       const void *q, const void *K,
                                       const float *tau, int32_t cap,
                                       int32_t *idx, int32_t *count, void *ws,
                                       size_t ws_bytes, void *stream);

/* Sparse attention over a given index set (CLSA article, section
 * 研究の背景と課題: attention restricted to the selected tokens).
 * q holds L query sets [L,B,Hq,d] (L = 1 for one layer); every set attends
 * over the same idx rows [B,Hkv,stride]; count [B,Hkv] gives the valid
 * prefix of each row (NULL: all stride entries; counts above stride are
 * clamped to stride).  Writes out [L,B,Hq,d] (dtype) and, if lse is not
 * NULL, lse [L,B,Hq]. */
sparse_status_t sparse_attn_gather(const sparse_shape_t *shape, int32_t L,
                                   const void *q, const void *K,
                                   const void *V, const int32_t *idx,
                                   int32_t stride, const int32_t *count,
                                   void *out, float *lse, void *ws,
                                   size_t ws_bytes, void *stream);

/* One fused decode step (CLSA article, sections CLSAの仕組み and
 * 計算コストの削減効果): route once with q_route [B,Hq,d], then run the
 * attention of all L layers' queries q_layers [L,B,Hq,d] over that one set.
 *   top-k mode:     k >= 1, tau == NULL, count may be NULL; idx [B,Hkv,k].
 *   threshold mode: k == 0, tau [B,Hkv] and count [B,Hkv] given, cap >= 1;
 *                   idx [B,Hkv,cap]; each layer uses min(count, cap) keys.
 * out [L,B,Hq,d]; lse [L,B,Hq] or NULL. */
sparse_status_t sparse_decode_step(const sparse_shape_t *shape, int32_t L,
                                   const void *q_route, const void *q_layers,
                                   const void *K, const void *V, int32_t k,
                                   const float *tau, int32_t cap,
                                   int32_t *idx, int32_t *count, void *out,
                                   float *lse, void *ws, size_t ws_bytes,
                                   void *stream);

/* sparse_decode_step with the layers' queries arriving late: the routing
 * (which reads only q_route) is enqueued first, then the stream waits on
 * layers_ready (a cudaEvent_t recorded after q_layers was written, e.g. by a
 * copy on another stream; NULL: no wait), then the attention is enqueued.
 * The same arguments, checks and results as sparse_decode_step otherwise.
 * When the step runs on the fused kernels (sparse_decode_step_fused), idx,
 * count and out are only written, never read back, so they may point into
 * mapped pinned host memory (sparse_pointer_device_usable); on the other
 * path the attention reads idx and count, which then belong in device
 * memory. */
sparse_status_t sparse_decode_step_join(const sparse_shape_t *shape, int32_t L,
                                        const void *q_route, const void *q_layers,
                                        const void *K, const void *V, int32_t k,
                                        const float *tau, int32_t cap, int32_t *idx,
                                        int32_t *count, void *out, float *lse, void *ws,
                                        size_t ws_bytes, void *stream, void *layers_ready);

/* Whether sparse_decode_step on this shape (k >= 1: top-k; k == 0: threshold
 * with cap >= 1) takes the fused kernels -- the routing scan, then one
 * kernel that selects and attends -- (*fused = 1) or routes and attends in
 * separate kernels (*fused = 0).  Fused: bf16, L * Hq / Hkv <= 128, N <=
 * 131072 and k (or cap) <= 32768.  Pure shape logic: no device call.
 * Returns SPARSE_ERR_INVALID_ARG for a null fused or invalid L, k, cap. */
sparse_status_t sparse_decode_step_fused(const sparse_shape_t *shape, int32_t L, int32_t k,
                                         int32_t cap, int32_t *fused);

/* Decode step that re-routes every R layers (CLSA article, section
 * 計算コストの削減効果: token-sparse attention with per-layer routing (DSA)
 * scores the context once per layer, CLSA once per step; section
 * 推論速度の改善結果: IndexCache shares an index set across only some layers).
 * The L layers form ngroups = ceil(L/R) groups of R consecutive layers (the
 * last one shorter when R does not divide L); group g routes with its own
 * query q_routes[g] and its layers attend over that group's set.  R >= L is
 * sparse_decode_step (one shared set); R = 1 is per-layer routing.
 *   q_routes [ngroups,B,Hq,d]; q_layers [L,B,Hq,d]; out [L,B,Hq,d];
 *   lse [L,B,Hq] or NULL;
 *   top-k mode:     k >= 1, tau == NULL; idx [ngroups,B,Hkv,k];
 *   threshold mode: k == 0, tau [ngroups,B,Hkv], count [ngroups,B,Hkv],
 *                   cap >= 1; idx [ngroups,B,Hkv,cap].
 * The workspace is sized for the layers of one group: ws_bytes >=
 * sparse_workspace_size(shape, k or cap, min(R, L)).  The groups run one after
 * another on `stream`, reusing the workspace. */
sparse_status_t sparse_decode_step_grouped(const sparse_shape_t *shape, int32_t L,
                                           int32_t R, const void *q_routes,
                                           const void *q_layers, const void *K,
                                           const void *V, int32_t k, const float *tau,
                                           int32_t cap, int32_t *idx, int32_t *count,
                                           void *out, float *lse, void *ws,
                                           size_t ws_bytes, void *stream);

/* The self-decoder's cache write for one decode step (CLSA article, section
 * CLSAの仕組み: the self-decoder generates the shared KV cache once; routing
 * and every cross-decoder layer read it, the new token included): copies
 * k_new[b,h,:] and v_new[b,h,:] ([B,Hkv,d], dtype of the cache, 16-byte
 * aligned) into row N-1 of K and V ([B,Hkv,n_cap,d]) for every (b, h), where
 * N = shape->N is the cache length counting the new token (N <= n_cap).  A
 * model's step is then this call followed by sparse_decode_step with the same
 * shape.  Hq is not used.  Asynchronous on `stream`; no workspace. */
sparse_status_t sparse_kv_append(const sparse_shape_t *shape, void *K, void *V,
                                 const void *k_new, const void *v_new, void *stream);

/* ---- Louver index (threshold routing with cluster pruning) ----------------
 * Louver summary, section 2. Louver インデックス: the keys of every (sequence,
 * KV head) are grouped into clusters of r keys by a balanced PCA tree and each
 * cluster is enclosed in a bounding ball; a threshold query (section 1.
 * 半空間範囲検索への帰着: keep every key in the halfspace {p : <qbar,p> >= tau},
 * no false negatives) skips the clusters whose ball misses the halfspace and
 * checks the keys of the others exactly.  One subspace (the page's S = 1).
 * Requirements: r a power of two in [32, 256], N a multiple of r, N / r a
 * power of two and N <= 1048576; the usual shape limits.
 *
 * Index buffer (device, caller-owned, index_bytes, 256-byte aligned), each
 * part at the next 256-byte boundary after the one before:
 *   perm [B*Hkv][N] int32: key ids in cluster order (cluster c of head bh is
 *        perm[bh][c*r .. c*r+r));
 *   centres [B*Hkv][N/r][d] fp32;  radii [B*Hkv][N/r] fp32;
 *   keys [B*Hkv][N][d] of the cache's dtype: row p of head bh is key
 *        perm[bh][p], so that each cluster's keys are contiguous;
 *   leaf centres [B*Hkv][N/32][d] fp32;  leaf radii [B*Hkv][N/32] fp32: the
 *        tree continues below the clusters to leaves of 32 keys (cluster c
 *        is leaves c*r/32 .. (c+1)*r/32 - 1); a query tests the leaves of
 *        the clusters that pass, with the same rule, before checking keys.
 * The index describes K's first N rows and holds a copy of them; it must be
 * rebuilt when those rows change.
 * Workspace: ws_bytes from sparse_louver_sizes, zero-filled once before first
 * use like the other workspaces.  Build and query calls may share one
 * (ordered), but it must not be shared with the other entry points: their
 * scratch areas overlap and each side keeps parts of its own zero between
 * calls. */

/* Sizes of the index buffer and of the workspace for this shape and r. */
sparse_status_t sparse_louver_sizes(const sparse_shape_t *shape, int32_t r,
                                    size_t *index_bytes, size_t *ws_bytes);

/* Builds the index of K [B,Hkv,n_cap,d] (first N rows) into `index`.
 * Each tree level splits every node at the median of its keys' projections
 * on the node's principal direction (8 power-iteration passes); leaves get
 * their mean as centre and the largest distance to it (inflated by 1e-5
 * relative) as radius.  fp32 atomic sums make the directions depend on
 * summation order: two builds may differ, every build is a valid index and
 * query results do not depend on it.  Asynchronous on `stream`. */
sparse_status_t sparse_louver_build(const sparse_shape_t *shape, const void *K, int32_t r,
                                    void *index, size_t index_bytes, void *ws,
                                    size_t ws_bytes, void *stream);

/* Threshold routing through the index (which holds the keys; K is not
 * read): the same set as sparse_route_threshold on the indexed keys
 * (identical scores, keys with S >= tau[b,h]) in
 * ascending order in idx [B,Hkv,cap], its size in count [B,Hkv]
 * (SPARSE_ERR_CAPACITY is reported through the status word when a count
 * exceeds cap, as there).  A cluster is skipped only when its ball bound
 * <qbar,c> + |qbar| rho is below tau - (1e-4 |tau| + 1e-6) - 1e-5 |qbar|
 * (|c| + rho), a margin above the fp32 rounding of any member's score, so
 * rounding cannot drop a key.  survivors (nullable) [B,Hkv,2] int32: the
 * clusters that passed the ball test and, of their 32-key leaves, those
 * that passed theirs (the keys checked exactly are 32 per such leaf).  q [B,Hq,d] of the shape's dtype; the shape is the
 * one the index was built for (Hq may differ; n_cap is not used).  One
 * kernel: its CTAs of a head meet at a bounded wait before writing the set
 * (see Co-residency); a wait that expires reports SPARSE_ERR_TIMEOUT and
 * leaves the workspace to be zero-filled again before the next query. */
sparse_status_t sparse_louver_route_threshold(const sparse_shape_t *shape, const void *q,
                                              const void *index, size_t index_bytes, int32_t r,
                                              const float *tau, int32_t cap, int32_t *idx,
                                              int32_t *count, int32_t *survivors, void *ws,
                                              size_t ws_bytes, void *stream);

/* One decode step with threshold routing through the Louver index: the set
 * of sparse_louver_route_threshold (q_route, tau [B,Hkv], cap), then every
 * layer's attention over it, as sparse_decode_step does in threshold mode
 * (the same outputs as that call on the indexed keys).  Two workspaces:
 * louver_ws (the index's, sizes from sparse_louver_sizes) and ws
 * (sparse_workspace_size(shape, cap, L)); device conditions of both parts
 * are reported in ws's status word.  K, V [B,Hkv,n_cap,d] are the cache the
 * index was built from (its first N rows); idx [B,Hkv,cap], count [B,Hkv],
 * out [L,B,Hq,d], lse [L,B,Hq] or NULL. */
sparse_status_t sparse_louver_decode_step(const sparse_shape_t *shape, int32_t L,
                                          const void *q_route, const void *q_layers,
                                          const void *K, const void *V, const void *index,
                                          size_t index_bytes, int32_t r, const float *tau,
                                          int32_t cap, int32_t *idx, int32_t *count, void *out,
                                          float *lse, void *louver_ws, size_t louver_ws_bytes,
                                          void *ws, size_t ws_bytes, void *stream);

/* Self-test of failure detection, with no fault: one device thread waits,
 * through the bounded wait that every counter barrier of the library uses
 * (the Louver query's per-head barrier), on a workspace word that nothing
 * ever increments.
 * After limit_ns of the GPU's global timer (capped at the library's own 2 s
 * limit) the wait gives up and raises the TIMEOUT flag in the status word,
 * so sparse_read_device_status then returns SPARSE_ERR_TIMEOUT and the
 * context stays usable.  ws: any library workspace (>= 4096 bytes, 256-byte
 * aligned); the word waited on is not used by any other call. */
sparse_status_t sparse_selftest_bounded_wait(void *ws, size_t ws_bytes, uint64_t limit_ns,
                                             void *stream);

/* Shared routing, top-k form (as sparse_route_topk) for callers that cannot
 * allocate device memory: a plugin inside a host framework that owns every
 * device allocation, or code that must not call cudaMalloc once it is
 * running (an allocation can synchronise the device and is not allowed while
 * a stream is being captured).  It takes no workspace: its scratch (status
 * word, radix histogram, fp32 scores) is a fixed array of about 4.5 MB built
 * into the library, so every GPU that loads the library holds it until the
 * process exits.  No page counterpart: this is a packaging variant, not part
 * of the method the pages describe.
 *   - Limit: B*Hkv <= 64 and B*Hkv*N <= 1048576 (the 128K-token, 8-head
 *     headline fits exactly); larger shapes return SPARSE_ERR_WORKSPACE.
 *   - The first call made with a given device current looks up the array's
 *     device address (cudaGetSymbolAddress); make that first call before any
 *     stream capture.
 *   - Every call shares the one array; the call clears the parts that must
 *     start at zero (status word, its histogram rows) on `stream` before
 *     using them.  Calls that overlap on the GPU (different streams without
 *     ordering) race on the array.
 *   - Device-detected conditions are not reported (the status word lives in
 *     the shared array); use sparse_route_topk with a workspace to read them.
 *   - Calls no cudaMalloc, cudaFree or allocating library routine. */
sparse_status_t sparse_route_topk_static(const sparse_shape_t *shape,
                                         const void *q, const void *K,
                                         int32_t k, int32_t *idx,
                                         void *stream);

/* Synchronise `stream`, read the device status word of ws, reset it to
 * zero, and return the most severe condition recorded since the last read
 * (TIMEOUT > INTERNAL > INDEX > NONFINITE > CAPACITY > OK).  *flags (if not NULL)
 * receives the raw bit set. */
sparse_status_t sparse_read_device_status(void *ws, void *stream,
                                          uint32_t *flags);

/* Enqueue an instantiated CUDA graph (a cudaGraphExec_t, e.g. a captured
 * decode step with its host transfers) on `stream`: one C call per replayed
 * step.  Returns SPARSE_ERR_INVALID_ARG for a NULL graph, SPARSE_ERR_CUDA if
 * the launch fails, else SPARSE_OK.  Does not synchronise. */
sparse_status_t sparse_graph_launch(void *graph_exec, void *stream);

/* Upload an instantiated CUDA graph's work to the device ahead of its first
 * launch (cudaGraphUpload on `stream`), so that launch does not pay for it.
 * Returns SPARSE_ERR_INVALID_ARG for a NULL graph, SPARSE_ERR_CUDA if the
 * upload fails, else SPARSE_OK.  Runs nothing of the graph. */
sparse_status_t sparse_graph_upload(void *graph_exec, void *stream);

/* *usable = 1 when kernels can read and write p at its own address: device
 * memory, managed memory, or pinned host memory mapped into the device's
 * address space (cudaHostAlloc memory under unified addressing); 0 for
 * anything else, including pageable host memory and pointers the CUDA
 * runtime does not know.  Returns SPARSE_ERR_INVALID_ARG for NULL arguments,
 * else SPARSE_OK.  Enqueues nothing. */
sparse_status_t sparse_pointer_device_usable(const void *p, int32_t *usable);

#ifdef __cplusplus
}
#endif

#endif /* SPARSE_DECODE_H_ */
