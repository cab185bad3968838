/*
 * park.h - C ABI of the PARK block-retrieval + block-sparse attention library
 * (libpark.so, CUDA, sm_100a).
 *
 * The operation is the one described in "PARK: Accurate Block Retrieval for
 * Sparse Attention in Video Diffusion Transformers" (abstract; Figure 2
 * caption; Table 1 caption): for one attention layer, cluster the queries with
 * Euclidean K-means, cluster the keys with K-means under a metric computed from
 * this layer's queries (QRKC), give every original query its own Softmax over
 * the key centroids and take the mean of those within each query cluster
 * (PAMA), keep key clusters per query cluster up to cumulative importance p
 * (top-p), and compute attention only on the kept (query-cluster,
 * key-cluster) pairs.
 *
 * Definitions fixed by this library where the pages are silent:
 *   metric       M = (1/N) sum_i q_i q_i^T (float64); key distance
 *                (k - c)^T M (k - c) = mean_i (q_i.k - q_i.c)^2.
 *   K-means      init c_k = x_floor(k N / K); `iters` x (assign, update), no
 *                early stop; assign ties go to the lowest index; update
 *                c_k = round_dtype(fl64(exact sum of members) / n_k), empty
 *                clusters keep their centroid.  Key centroids live in raw key
 *                space.
 *   PAMA         P_im = softmax over NON-EMPTY key clusters m of (q_i.c_m)/sqrt(D);
 *                I_rm = mean over members i of query cluster r of P_im.
 *   top-p        per non-empty query cluster: key clusters sorted by I_rm
 *                descending (ties: lower m first); keep the shortest prefix
 *                whose running sum is >= p (crossing block kept); p >= 1 keeps
 *                every non-empty key cluster.
 *   attention    o_i = sum_{j in J_r} softmax_j(q_i.k_j/sqrt(D)) v_j with J_r the
 *                keys of the kept key clusters of i's query cluster r.
 *
 * Conventions
 *   - Every pointer argument named Q, K, V, O, ws and every pointer inside
 *     park_retrieval is a DEVICE pointer; shape structs and `bytes` are host.
 *   - Ownership: the caller allocates and frees everything.  The library never
 *     allocates, frees or synchronises; all work is enqueued on `stream` (a
 *     cudaStream_t passed as void*, NULL = legacy default stream).
 *   - Layout: Q, K, V, O are [B, H, N, D] contiguous, N = T*Hg*W + n_text
 *     (video tokens in (t, y, w) order, text tokens last).  Both dtypes
 *     require D % 32 == 0 and D <= 128; PARK_BF16 with D == 128 runs the
 *     tensor-core kernels, every other shape the float64 / SIMT kernels (the
 *     same results, certified the same way, slower).
 *   - Range precondition: every input element is 0 or has 2^-40 <= |x| < 2^40
 *     (and is finite).  Inside it the centroid sums are exact (128-bit fixed
 *     point at 2^-64), whatever the order of the terms.
 *   - Sizes: N <= 2^20, B*H*N < 2^31, 1 <= NQ, NK <= N, NK <= 4096,
 *     NQ <= 65536, p > 0, iters >= 1.
 *   - Errors: argument errors are returned synchronously (nothing is enqueued).
 *     Conditions only the device can see (an input outside the range
 *     precondition, a bounded wait that ran out) are written to *status; the
 *     outputs are valid only if *status == PARK_OK after the stream has
 *     reached the end of the call.  A launch failure returns PARK_ERR_CUDA.
 */
#ifndef PARK_H
#define PARK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------ */
#define PARK_OK 0
#define PARK_ERR_INVALID_ARG 1 /* null pointer, bad shape or parameter       */
#define PARK_ERR_UNSUPPORTED 2 /* valid but not implemented (e.g. bf16, D!=128) */
#define PARK_ERR_WORKSPACE 3   /* ws_bytes smaller than park_workspace_size   */
#define PARK_ERR_CUDA 4        /* a kernel launch or memset failed            */
#define PARK_ERR_RANGE 5       /* device: input outside the range precondition */
#define PARK_ERR_TIMEOUT 6     /* device: a bounded wait ran out              */

/* ---- element types ----------------------------------------------------- */
#define PARK_BF16 0
#define PARK_F32 1

/* ---- park_retrieval.flags (inputs) ------------------------------------- */
/* Start query / key K-means from the centroids already in q_centroids /
 * k_centroids instead of the strided initialisation (mask and cluster reuse
 * across denoising steps, PARK Appendix Table 9). */
#define PARK_FLAG_WARM_START_Q 0x1u
#define PARK_FLAG_WARM_START_K 0x2u
/* Selection variants (PARK Table 3 ablations, Table 10 top-k, and a size prior
 * that the pages do not have); any combination may be set:
 *   NO_QRKC          "w/o QRKC": key K-means is Euclidean (M = I); out->metric,
 *                    when non-NULL, is still written.
 *   CENTROID_QUERY   "w/o PAMA": I_rm = softmax_m(s c_r . c_m) with the query
 *                    centroid c_r in place of every member query; computed in
 *                    float64 (importance_bound rows are 0).
 *   TOPK             keep the ceil(p * L_r) most important key clusters of each
 *                    non-empty query cluster (L_r = non-empty key clusters; ties:
 *                    lower m; at least one), p read as the retrieval ratio in
 *                    (0, 1] (the float32 value passed).
 *   SIZE_PRIOR       PAMA logits gain log |B_m|: P_im proportional to
 *                    |B_m| exp(s q_i . c_m).
 *   SIP              sampling with inclusion-probability weighting ("AB-Attention
 *                    Brings More Accurate Sparse Attention to Video Diffusion",
 *                    SIP paragraph), p read as a ratio in (0, 1]: per non-empty
 *                    query cluster, pi_m = min(1, c I_rm) with sum_m pi_m =
 *                    ceil(p L_r) (the largest blocks become certain first); block
 *                    m is kept when sip_uniform[r][m] < pi_m, with weight 1 / pi_m
 *                    in both Softmax sums of the attention; if none is drawn the
 *                    most important block is kept.  Needs sip_uniform and
 *                    block_weight; not combinable with TOPK. */
#define PARK_FLAG_NO_QRKC 0x4u
#define PARK_FLAG_CENTROID_QUERY 0x8u
#define PARK_FLAG_TOPK 0x10u
#define PARK_FLAG_SIZE_PRIOR 0x20u
#define PARK_FLAG_SIP 0x40u
/* HyperVAttention's clustering parts ("HyperVAttention: Efficient Sparse
 * Attention with Spatio-Temporal Clustering for Video Diffusion", abstract):
 *   MERGE_Q          after the selection, query clusters merge in parallel
 *                    agglomerative rounds: each non-empty cluster g picks the
 *                    partner h with the largest gain cost(g) + cost(h) -
 *                    cost(g u h) > 0 (ties: lowest h), with cost(n, L) =
 *                    ceil(n/128) ceil(L/128) the attention's (query tile, key
 *                    tile) pairs for n query rows whose kept key clusters fill L
 *                    key rows (each cluster rounded up to 8 rows), the merged
 *                    cluster keeping the union of the kept sets; mutual pairs
 *                    merge into the lower index; rounds repeat until one merges
 *                    nothing, at most merge_rounds (0 = 8, at most 64).  The
 *                    outputs then describe the merged clustering (labels, perm,
 *                    offsets, centroids recomputed as exact means, mask and CSR
 *                    rows of merged-away clusters empty) except importance and
 *                    importance_bound, which keep the values the selection used.
 *                    Not combinable with SIP; NQ <= 2048 (else
 *                    PARK_ERR_UNSUPPORTED).
 *   LOCAL_WINDOW     both K-means run on 3D local windows: the video grid is tiled
 *                    by boxes of window_t x window_h x window_w tokens (the last
 *                    box of an axis may be shorter; nW boxes, numbered with the
 *                    column box fastest); box w owns centroids floor(w K / nW) ..
 *                    floor((w+1) K / nW) - 1, initialised at its members
 *                    floor(j n_w / K_w) in token order (without WARM_START), and
 *                    a video token is assigned among its box's centroids only;
 *                    text tokens among all.  Needs 1 <= window extents <= grid
 *                    extents and nW <= min(NQ, NK) (else PARK_ERR_INVALID_ARG),
 *                    at most 256 centroids per box (else PARK_ERR_UNSUPPORTED). */
#define PARK_FLAG_MERGE_Q 0x80u
#define PARK_FLAG_LOCAL_WINDOW 0x100u
/* Implementation switch, no change to the result (up to float32 summation
 * order): on the tensor-core path (bf16, D == 128) park_sparse_attn packs the
 * last 128-row tile of a query cluster with several tiles into the single
 * tile of a cluster with enough free rows when that needs fewer key tiles
 * (every row still attends only to its own cluster's kept key clusters; done
 * only for NQ <= 2048); this flag turns it off. */
#define PARK_FLAG_NO_TILE_PACKING 0x200u

/* ---- park_retrieval.counters indices (outputs, int64) ------------------ */
#define PARK_CNT_Q_RECHECK 0    /* query rows whose bf16 score margin was not
                                   certified and were rescored in float64    */
#define PARK_CNT_K_RECHECK 1    /* same for key rows                          */
#define PARK_CNT_FULL_RESCORE 2 /* rows rescored against every centroid       */
#define PARK_CNT_PAMA_RECHECK 3 /* query clusters whose top-p cut was not
                                   certified and were recomputed in float64  */
#define PARK_CNT_KEPT_BLOCKS 4  /* kept (query cluster, key cluster) pairs    */
#define PARK_CNT_KEPT_PAIRS 5   /* sum_r |Q_r| * |J_r|: attended query-key pairs */
#define PARK_CNT_WORK_ITEMS 6   /* query tiles scheduled for attention        */
#define PARK_CNT_KEY_TILES 7   /* (query tile, key tile) pairs computed by attention */
#define PARK_NUM_COUNTERS 8

/* Problem shape.  N = T*Hg*W + n_text. */
typedef struct {
    int B, H;          /* batch, heads                                       */
    int T, Hg, W;      /* video token grid (frames, height, width)           */
    int n_text;        /* text tokens appended after the video tokens        */
    int D;             /* head dimension                                     */
    int dtype;         /* PARK_BF16 or PARK_F32 (Q, K, V, O and centroids)   */
} park_shape;

/* Retrieval result.  All arrays are caller-allocated DEVICE memory, [B, H, ...]
 * contiguous; "bh" below is b*H + h.  Written by park_retrieve, read by
 * park_sparse_attn. */
typedef struct {
    uint32_t flags;        /* in: PARK_FLAG_* bits                                */
    int32_t *q_labels;     /* [B,H,N]      query cluster of each token            */
    int32_t *k_labels;     /* [B,H,N]      key cluster of each token              */
    int32_t *q_perm;       /* [B,H,N]      sorted position -> token (stable by cluster) */
    int32_t *k_perm;       /* [B,H,N]                                             */
    int32_t *q_offsets;    /* [B,H,NQ+1]   first sorted position of each cluster  */
    int32_t *k_offsets;    /* [B,H,NK+1]                                          */
    void *q_centroids;     /* [B,H,NQ,D]   input dtype                            */
    void *k_centroids;     /* [B,H,NK,D]   input dtype, raw key space             */
    float *importance;     /* [B,H,NQ,NK]  PAMA block importance I               */
    uint8_t *mask;         /* [B,H,NQ,NK]  1 = kept                               */
    int32_t *kept_ptr;     /* [B,H,NQ+1]   CSR row pointers, per (b,h) from 0     */
    int32_t *kept_idx;     /* [B,H,NQ*NK]  kept m per row, ascending; row r of
                              head bh starts at bh*NQ*NK + kept_ptr[bh*(NQ+1)+r]   */
    double *metric;        /* [B,H,D,D]    optional (may be NULL): the metric M   */
    float *importance_bound; /* [B,H,NQ]   optional (may be NULL): relative error
                              bound of row r of importance; 0 where the row was
                              computed in float64                              */
    int64_t *counters;     /* [PARK_NUM_COUNTERS], zeroed by park_retrieve        */
    int32_t *status;       /* [1] device status word, zeroed by park_retrieve     */
    const float *sip_uniform; /* [B,H,NQ,NK] in, with PARK_FLAG_SIP: uniforms on [0,1) */
    float *block_weight;   /* [B,H,NQ,NK] out, with PARK_FLAG_SIP: 1/pi_m for kept
                              blocks, 0 elsewhere; read by park_sparse_attn     */
    int32_t window_t, window_h, window_w; /* in, with PARK_FLAG_LOCAL_WINDOW: box
                              extent in frames, rows and columns of the grid    */
    int32_t merge_rounds;  /* in, with PARK_FLAG_MERGE_Q: most merging rounds (0 = 8) */
} park_retrieval;

/* Bytes of device workspace that park_retrieve, park_sparse_attn and
 * park_layer need for this shape (one buffer serves all three).  Host only;
 * returns PARK_ERR_INVALID_ARG / PARK_ERR_UNSUPPORTED for bad shapes. */
int park_workspace_size(const park_shape *shape, int NQ, int NK, size_t *bytes);

/* Block retrieval (PARK Figure 2): metric, query K-means, QRKC key K-means,
 * PAMA, top-p, CSR of kept blocks.  Q, K: device [B,H,N,D].  Fills every array
 * of *out except that out->metric is written only when non-NULL. */
int park_retrieve(const void *Q, const void *K, const park_shape *shape, int NQ, int NK, float p,
                  int iters, park_retrieval *out, void *ws, size_t ws_bytes, void *stream);

/* Block-sparse attention over the kept blocks of a retrieval result (PARK
 * abstract: attention is computed inside the retrieved blocks alone).  Reads
 * labels, perms, offsets and the CSR of *r; writes O [B,H,N,D] in the input
 * dtype, original token order.  Also sets r->counters[PARK_CNT_WORK_ITEMS] and
 * may set *r->status. */
int park_sparse_attn(const void *Q, const void *K, const void *V, const park_shape *shape, int NQ,
                     int NK, const park_retrieval *r, void *O, void *ws, size_t ws_bytes,
                     void *stream);

/* park_retrieve followed by park_sparse_attn on the same stream. */
int park_layer(const void *Q, const void *K, const void *V, const park_shape *shape, int NQ, int NK,
               float p, int iters, void *O, park_retrieval *out, void *ws, size_t ws_bytes,
               void *stream);

/* Static description of a status code (never NULL). */
const char *park_status_string(int code);

/* Number of CUDA kernels this library has launched in this process. */
uint64_t park_launch_count(void);

/* Library version, major*10000 + minor*100 + patch. */
int park_version(void);

/* Limit, in nanoseconds of device time, of every bounded wait inside this
 * library's kernels (a wait for a tensor-memory-access copy or a tensor-core
 * result; default 2 s; ns = 0 restores the default).  Host state, read at each
 * launch.  A wait that runs out sets *status to PARK_ERR_TIMEOUT; the kernel
 * then lets its copies and MMAs in flight finish, frees its tensor memory and
 * returns, so the context stays usable and later calls are unaffected.  A tiny
 * limit (1 ns) makes the waits run out on purpose: that is how the timeout path
 * is tested.  Never needed in normal use. */
int park_set_wait_limit_ns(uint64_t ns);

/* ---- per-kernel timing for measurement tools --------------------------- */
typedef struct {
    char name[48];     /* kernel name                                        */
    double total_ms;   /* summed device time between its begin/end events    */
    int64_t launches;  /* number of launches recorded                        */
} park_kernel_time;

/* on != 0: every later kernel launch of this library records a CUDA event
 * before and after it on its stream (host state, all threads).  Off by
 * default; costs two event records per launch. */
int park_profile_enable(int on);

/* Aggregate the recorded launches by kernel name into out[0..cap) and clear
 * the record; *n = entries written.  Call only after every recorded stream has
 * been synchronised.  Returns PARK_ERR_CUDA if an event could not be read. */
int park_profile_collect(park_kernel_time *out, int cap, int *n);

/* ---- metric without caller workspace ----------------------------------- */
/* The paper has no counterpart of this entry point: it exists for callers
 * that cannot allocate device memory where they need the QRKC metric (for
 * example while a CUDA graph is being captured, where cudaMalloc is not
 * allowed, or inside a host framework that passes only input and output
 * buffers).  It computes the same M = (1/N) sum_i q_i q_i^T per (b, h) as
 * park_retrieve writes to out->metric.
 *   Q: device [B,H,N,D] (same dtypes and D as park_retrieve); M: device float64
 *   [B,H,D,D], written; stream: cudaStream_t or NULL.
 * Scratch comes from a 16 MiB array compiled into the library (held by every
 * GPU that loads it until exit), so B*H may be at most 16 MiB / (8*D*D)
 * (128 at D = 128); larger shapes return PARK_ERR_UNSUPPORTED with nothing
 * enqueued.  No allocation of any kind.  The first call on each device looks
 * up the array's device address (with that device current): make it before
 * any stream capture.  All calls share the array, so calls that overlap on the
 * GPU race; serialise them (one stream, or events). */
int park_qrkc_metric_static(const void *Q, const park_shape *shape, double *M, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* PARK_H */
