/*
 * zha.h - C ABI of the ZHA decode library (libzha.so), sm_100a (NVIDIA B200).
 *
 * Zyphra Hierarchical Attention (ZHA) answers a decode query by searching a
 * tree of summaries of the KV cache instead of scoring every cached key:
 *   - build:  contiguous blocks of `block` raw keys are summarised by tangent
 *             planes of their log attention mass at `n_refs` reference
 *             queries; summaries are merged exactly, `block` children per
 *             parent, up to `levels` levels ("Zyphra Hierarchical Attention",
 *             Zyphra blog, section "Building the tree"; tanhow.com summary
 *             "Zyphra发布ZHA稀疏注意力方法，可改造冻结大模型", section "How does ZHA's
 *             tree indexer work?");
 *   - route:  each query head descends the tree with top-p selection at every
 *             step (blog, section "Routing in the tree"; summary, section
 *             "How does top-p routing choose tokens?");
 *   - attend: ordinary softmax attention over the kept raw keys, the first
 *             token (attention sink) and the tail tokens that are not yet in a
 *             complete block (same sections).
 *
 * Conventions for every entry point:
 *   - All device memory is owned by the caller.  The library allocates only
 *     the small host handle of zha_tree_create.  Sizes come from
 *     zha_tree_bytes / zha_dense_scratch_bytes.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Every call only enqueues work on it and returns; results are
 *     ready once the stream has been synchronised.
 *   - Work runs on the CUDA device that is current when the call is made;
 *     all pointers must be on that device.
 *   - Return value: ZHA_OK (0) or a negative ZHA_ERR_* code.  Nothing throws
 *     across the ABI; zha_last_error() gives a thread-local message for the
 *     last failing call on the calling thread.  Device-side faults that the
 *     kernels detect (a capacity bound that would be exceeded, a bounded wait
 *     that ran out) set a status word that zha_tree_status() returns.
 *   - Element types: ZHA_F32 stores K, V, Q, refs and the node slopes (mu) as
 *     fp32; ZHA_BF16 stores them as bf16 (round-to-nearest-even).  Node values
 *     f and intercepts b are always fp32, all arithmetic accumulates in fp32,
 *     and the decode output O is fp32.
 */
#ifndef ZHA_H_
#define ZHA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ZHA_API __attribute__((visibility("default")))
#else
#define ZHA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

enum {
  ZHA_OK = 0,
  ZHA_ERR_INVALID = -1,     /* bad argument: null pointer, negative size, p outside (0, 1] */
  ZHA_ERR_CAPACITY = -2,    /* more tokens / batch than the tree was created for */
  ZHA_ERR_UNSUPPORTED = -3, /* head dim not 64/128, block < 2, levels < 1, n_refs > 32 ... */
  ZHA_ERR_CUDA = -4,        /* a CUDA runtime call or kernel launch failed */
  ZHA_ERR_TIMEOUT = -5      /* a bounded device-side wait gave up (reported through the status word) */
};

enum { ZHA_F32 = 0, ZHA_BF16 = 1 };

/* Router planes: the slopes the routing steps read.  ZHA_PLANES_KEY reads the
 * stored nodes (mu in the element type).  ZHA_PLANES_FP4 keeps, beside them,
 * a copy of every node's slopes in 4-bit e2m1 with one e4m3 scale per 16
 * dimensions (an FP4 router: the tanhow.com summary "Zyphra发布ZHA稀疏注意力方法,
 * 可改造冻结大模型", TL;DR, reports that one was tested, without details),
 * which the routing steps read instead: a record is
 * R*(d/2 + d/16 + 4) bytes (1216 at R = 16, d = 128) instead of
 * R*(d*es + 4).  Quantisation of a group of 16 stored slopes v (converted
 * exactly to fp32): amax = max |v|; scale = e4m3(amax / 6) (the division in
 * fp32, then round to nearest, ties to even, at most 448; 0 when amax is 0);
 * code of v = e2m1(v / scale) (fp32 division, nearest value of
 * {0, 0.5, 1, 1.5, 2, 3, 4, 6} with the sign, ties to the even mantissa,
 * at most 6; 0 when the scale is 0).  The slope the router uses is
 * code * scale (exact in fp16).  Intercepts stay fp32 and unchanged.
 * bf16 configurations only (ZHA_ERR_UNSUPPORTED otherwise). */
enum { ZHA_PLANES_KEY = 0, ZHA_PLANES_FP4 = 1 };

/* Geometry and limits of one layer's tree.  Passed by pointer, read only. */
typedef struct {
  int32_t d;           /* head dimension: 64 or 128 */
  int32_t n_q_heads;   /* query heads Hq; a multiple of n_kv_heads */
  int32_t n_kv_heads;  /* KV heads Hkv; one tree per KV head */
  int32_t block;       /* b >= 2: raw keys per leaf block and children per parent */
  int32_t levels;      /* L >= 1: depth of the tree (level 1 = leaf blocks) */
  int32_t n_refs;      /* R in [1, 32]: reference queries per tree */
  float p;             /* top-p threshold in (0, 1]; 1 keeps every node (dense) */
  int32_t dtype;       /* ZHA_F32 or ZHA_BF16 */
  int64_t capacity;    /* maximum number of cached tokens per KV head */
  int32_t max_batch;   /* maximum decode batch B per zha_decode call */
  int32_t planes;      /* ZHA_PLANES_KEY (0) or ZHA_PLANES_FP4 */
} zha_config;

typedef struct zha_tree zha_tree; /* opaque host handle */

/* Per-call counters written by zha_decode when `stats` is non-NULL.  Device
 * memory, int64 entries, laid out [B][Hq][ZHA_STAT_COUNT]. */
enum {
  ZHA_STAT_NODES_SCORED = 0, /* tree nodes whose planes the query head scored */
  ZHA_STAT_LEAVES_KEPT = 1,  /* level-1 blocks the query head keeps */
  ZHA_STAT_KEYS = 2,         /* keys attended: kept blocks + sink (if not kept) + tail */
  ZHA_STAT_STEPS = 3,        /* routing steps taken */
  ZHA_STAT_COUNT = 4
};

/*
 * zha_tree_bytes: device bytes the caller must provide for a tree.
 *   node_bytes    - node storage (all levels, all KV heads), any alignment >= 256 B.
 *   scratch_bytes - decode/append workspace, alignment >= 256 B.
 * Returns ZHA_ERR_INVALID / ZHA_ERR_UNSUPPORTED for a bad config.  Host only.
 */
ZHA_API int zha_tree_bytes(const zha_config* cfg, size_t* node_bytes, size_t* scratch_bytes);

/*
 * zha_tree_layout: where level `level` (1..L) lives inside node_buf, so that
 * callers (tests, exporters) can read the stored planes.
 *   rec_offset   - byte offset of the records [Hkv][cap_nodes] of rec_bytes each:
 *                  mu[R][d] in the element type, then bias[R] fp32 (zero padded
 *                  to a multiple of 16 bytes);
 *   f_offset     - byte offset of f[Hkv][cap_nodes][R] fp32;
 *   cap_nodes    - node slots per KV head at this level (floor(capacity / b^level));
 *   rec_bytes    - bytes per record.
 * Host only.
 */
ZHA_API int zha_tree_layout(const zha_config* cfg, int32_t level, size_t* rec_offset, size_t* f_offset,
                    int64_t* cap_nodes, size_t* rec_bytes);

/*
 * zha_tree_layout_fp4: where the FP4 router records of level `level` live
 * inside node_buf (configurations with planes = ZHA_PLANES_FP4; else
 * ZHA_ERR_INVALID).  Records [Hkv][cap_nodes] of rec_bytes each: codes
 * [R][d/2] bytes (dimension 2i in the low nibble, 2i+1 in the high one; e2m1
 * bits s|e1 e0|m), then scales [R][d/16] e4m3 bytes, then bias[R] fp32, zero
 * padded to a multiple of 16 bytes.  Host only.
 */
ZHA_API int zha_tree_layout_fp4(const zha_config* cfg, int32_t level, size_t* rec_offset, size_t* rec_bytes);

/*
 * zha_tree_create: bind caller-owned buffers into a tree handle (host only).
 *   K, V     - [Hkv][capacity][d] element type; the KV cache.  Tokens [0, n) must be
 *              written before zha_tree_build(n); zha_tree_append writes new tokens.
 *   refs     - [Hkv][R][d] element type; reference queries of each KV head's tree.
 *   node_buf - node_bytes from zha_tree_bytes.
 *   scratch  - scratch_bytes from zha_tree_bytes; zeroed by zha_tree_build.
 * The buffers must stay alive until zha_tree_destroy.  *out receives the handle.
 */
ZHA_API int zha_tree_create(const zha_config* cfg, void* K, void* V, const void* refs, void* node_buf,
                    void* scratch, zha_tree** out);

/*
 * zha_tree_build: (re)build every complete node over tokens [0, n) of K.
 * Any earlier tree state is discarded.  n in [0, capacity].
 */
ZHA_API int zha_tree_build(zha_tree* tree, int64_t n, void* stream);

/*
 * zha_tree_append: copy m new tokens (K_new, V_new: [Hkv][m][d], device memory,
 * element type) to positions [n, n+m) of the cache and build every node that
 * they complete.  The result is bit-identical to zha_tree_build(n+m).
 * Returns ZHA_ERR_CAPACITY if n + m > capacity.
 */
ZHA_API int zha_tree_append(zha_tree* tree, const void* K_new, const void* V_new, int64_t m, void* stream);

/* Tokens currently in the tree (host-side bookkeeping; no sync). */
ZHA_API int64_t zha_tree_size(const zha_tree* tree);

/*
 * zha_decode: route and attend B decode queries against the tree.
 *   Q        - [B][Hq][d] element type, device.
 *   O        - [B][Hq][d] fp32, device; softmax attention over each head's
 *              attended set (kept blocks, token 0, tail tokens).
 *   kept     - optional [B][Hq][cap_leaves] int32 (cap_leaves = capacity / block):
 *              the kept level-1 block indices of each head, ascending;
 *              kept_cnt [B][Hq] int32 receives their number.  Both NULL or
 *              both non-NULL.
 *   stats    - optional [B][Hq][ZHA_STAT_COUNT] int64 counters.
 *   scored   - optional [B][Hq][scored_cap] int32: the codes (level << 27 | index)
 *              of every node the head scored, step by step (in no particular
 *              order within a step); ZHA_STAT_NODES_SCORED
 *              gives how many (entries past scored_cap are dropped).  Used to
 *              count the bytes a decode must read; leave NULL on the hot path.
 * Requires 1 <= B <= max_batch and at least one cached token.  The call
 * launches a fixed sequence of kernels on `stream` (per routing step a scoring
 * and a select kernel, then one attention kernel) and
 * returns without synchronizing; calls on one tree share its scratch and must
 * be issued in order on one stream.  A wait of a scoring warp on a record copy
 * is bounded: when it runs out the status word reports ZHA_ERR_TIMEOUT.
 */
ZHA_API int zha_decode(const zha_tree* tree, const void* Q, float* O, int32_t B, int32_t* kept,
               int32_t* kept_cnt, int64_t* stats, int32_t* scored, int64_t scored_cap, void* stream);

/*
 * zha_route_multi: route and attend m queries of the same context at once,
 * e.g. the queries of a prefill chunk against the cached context before it.
 * Each query head is routed exactly as in zha_decode (the top-down top-p
 * descent of "Zyphra Hierarchical Attention", Zyphra blog, section "Routing
 * in the tree"; tanhow.com summary, section "How does top-p routing choose
 * tokens?"), and attends to its kept blocks, the sink and the tail; the
 * pages model the speed of decode only (summary, section "ZHA 有多快？"),
 * and a query's attention to the other queries of its own chunk is not part
 * of this call.  Every query starts from the same candidates, the forest
 * roots, so the first routing step of all queries is one contraction of the
 * roots' slope rows with the queries on the tensor cores (bf16
 * configurations; fp32 ones score it per query); the later steps run as in
 * zha_decode, max_batch queries at a time.
 *   Q        - [m][Hq][d] element type, device;  O - [m][Hq][d] fp32, device.
 *   kept     - optional [m][Hq][cap_leaves] int32 with kept_cnt [m][Hq] int32
 *              (as in zha_decode); both NULL or both non-NULL.
 *   m >= 1 (any size; the queries are processed in groups of max_batch).
 * Asynchronous on `stream`; shares the tree's scratch with zha_decode (calls
 * on one tree must be issued in order on one stream).  Errors as zha_decode.
 */
ZHA_API int zha_route_multi(zha_tree* tree, const void* Q, float* O, int32_t m, int32_t* kept, int32_t* kept_cnt,
                    void* stream);

/*
 * zha_decode_step_host: one decode step from host memory - copies the new
 * token's K/V (host [Hkv][d] each) and the queries (host [B][Hq][d]) to the
 * device, appends the token, decodes, and copies O back to host o_host
 * ([B][Hq][d] fp32).  Host buffers should be pinned for asynchronous copies.
 * k_host/v_host may be NULL to decode without appending.
 */
ZHA_API int zha_decode_step_host(zha_tree* tree, const void* k_host, const void* v_host, const void* q_host,
                         float* o_host, int32_t B, void* stream);

/*
 * zha_dense_scratch_bytes / zha_dense_decode: dense softmax attention of B
 * queries over tokens [0, n) of K, V (the in-run comparator; no tree).
 *   K, V   - [Hkv][ld][d] element type (ld = row stride in tokens >= n).
 *   Q      - [B][Hq][d]; O - [B][Hq][d] fp32.
 *   scratch - at least zha_dense_scratch_bytes(cfg, B, n) bytes (0 for an invalid
 *            request): the split partials of every call with B' <= B sequences
 *            and n' <= n tokens fit in it, so one scratch serves all such calls.
 *            Its contents need no initialisation; each call writes the partials
 *            it reads.  B <= cfg->max_batch.  A smaller scratch is not detected
 *            (the call takes no size): the caller must size it with this
 *            function.
 */
ZHA_API size_t zha_dense_scratch_bytes(const zha_config* cfg, int32_t B, int64_t n);
ZHA_API int zha_dense_decode(const zha_config* cfg, const void* K, const void* V, int64_t ld, int64_t n,
                     const void* Q, float* O, int32_t B, void* scratch, void* stream);

/*
 * zha_dense_decode_noalloc: zha_dense_decode for callers that cannot allocate
 * device memory - a serving loop whose device memory is fixed and
 * pre-partitioned at start-up (an allocation there can fail or fragment the
 * pool at the worst moment), or a host framework that owns the whole device
 * arena and gives plug-ins no allocator.  The pages describe nothing like it;
 * it is a deployment convenience of this library.
 *   Same arguments and result as zha_dense_decode, without `scratch`: the
 *   split partials go to a fixed array of 2^20 floats (4 MiB) that the library
 *   holds on every device that loads it, until the process exits.
 *   Requires B * n_q_heads * splits * (d + 2) <= 2^20 (splits as planned for
 *   zha_dense_scratch_bytes, at most 4 * 148 / (B * n_kv_heads) rounded up);
 *   larger requests return ZHA_ERR_CAPACITY without launching anything.
 *   The first call on a device looks up the array's device address (with
 *   that device current); make that first call before any stream capture.
 *   No cudaMalloc, cudaFree or other allocation happens in any call.  Every
 *   call on a device shares the array and overwrites it: calls whose work
 *   overlaps on the GPU (other streams, other threads) race and must be
 *   serialised by the caller.  Nothing in the array needs to start at zero.
 */
ZHA_API int zha_dense_decode_noalloc(const zha_config* cfg, const void* K, const void* V, int64_t ld, int64_t n,
                             const void* Q, float* O, int32_t B, void* stream);

/*
 * zha_tree_set_step_p: top-p thresholds per routing step, for routing whose
 * threshold changes with the depth in the tree and with the context length
 * ("Zyphra Hierarchical Attention", closing section on matching the degree of
 * compression to the predictive information in the data: a fixed top-p at
 * every level is not enough, the threshold has to evolve with tree depth and
 * context length; the "ZHA 階層注意力研究" review, section on thresholds that
 * follow depth and content).  The pages give no schedule, so the caller
 * chooses one.
 *   p - host array of n thresholds, p[s] for routing step s (s = 0 scores the
 *       roots, step s the children of step s-1's kept nodes); steps past n-1
 *       use p[n-1].  Each value in (0, 1]; 1 keeps every candidate of the step.
 *   n - 0 .. 20; n = 0 returns to the configuration's single p.
 * Applies to the decode calls issued after it; copied (the array may be
 * freed).  ZHA_ERR_INVALID for a NULL tree, n out of range, a NULL p with
 * n > 0, or a value outside (0, 1].
 */
ZHA_API int zha_tree_set_step_p(zha_tree* tree, const float* p, int32_t n);

/* Synchronise `stream` and return the tree's device status word (ZHA_OK or a
 * ZHA_ERR_* code raised inside a kernel); clears it. */
ZHA_API int zha_tree_status(zha_tree* tree, void* stream);

ZHA_API void zha_tree_destroy(zha_tree* tree);

/* Number of kernels this library has launched in this process (all threads,
 * all devices) - lets a caller verify which work ran on the GPU. */
ZHA_API uint64_t zha_launch_count(void);

/* Message for the last failing call on this thread ("" if none). */
ZHA_API const char* zha_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* ZHA_H_ */
