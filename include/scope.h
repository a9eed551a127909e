/*
 * scope.h -- C ABI of the SCOPE per-layer sparse-attention hot path on B200 (sm_100a).
 *
 * SCOPE ("Subspace Clustering with Online Per-Head Top-K Estimation for Sparse Video
 * Attention", arXiv 2608.12780) runs, per attention layer of a video diffusion
 * transformer and per (batch, head):
 *   1. clustering: post-RoPE queries into Cq clusters; post-RoPE keys split into the
 *      temporal / height / width channel ranges of 3D RoPE and each range clustered
 *      independently into Cm centroids (abstract; review page "major_comments": Eq. 3);
 *   2. selection: per query cluster c, lookup tables of centroid dot products summed
 *      into a proxy logit per key (Eq. 6), hybrid Top-p / fixed Top-k base counts
 *      (Eqs. 7-8), the online per-head Top-k k_head (Eq. 9) and the top-up of clusters
 *      below it (Eq. 10) (review page "key_machinery");
 *   3. exact softmax attention of each query over its cluster's selected ORIGINAL
 *      keys and values (abstract; review page "forward_implications").
 *
 * Conventions for every entry point
 *  - Tensors are dense, row-major, on the device of the current CUDA context:
 *    Q, K, V, O are [B, H, N, d] with N = T*Hg*Wg and token n = t*Hg*Wg + h*Wg + w;
 *    channels [0, d_t) / [d_t, d_t+d_h) / [d_t+d_h, d) are the temporal / height /
 *    width subspaces.  Element type of Q, K, V, O is params->dtype.
 *  - The caller owns every buffer, including the workspace `ws` of at least
 *    scope_workspace_bytes(params) bytes (256-byte aligned).  The workspace is
 *    dominated by the attention gather lists, 4 * B*H*Cq*N bytes (3.4 GB for 24 heads
 *    of 118800 tokens and Cq = 300).  The library allocates
 *    no device memory, keeps no state between calls and never synchronises the
 *    stream, except scope_get_device_status.  Calls on one workspace must not overlap.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Work is enqueued;
 *    results are valid once the stream has completed and the status is SCOPE_OK.
 *  - Arguments are validated on the host before anything is enqueued; a failure
 *    returns SCOPE_ERR_INVALID_ARGUMENT / SCOPE_ERR_UNSUPPORTED /
 *    SCOPE_ERR_WORKSPACE_TOO_SMALL and enqueues nothing.  A failed launch returns
 *    SCOPE_ERR_CUDA.  Conditions only the device can see (an init index out of range,
 *    an unresolvable selection tie) set bits in a status word inside the workspace,
 *    read by scope_get_device_status; each entry point clears that word first.
 *  - Limits: d in {64, 128}; d_t, d_h, d_w >= 1 with d_t + d_h + d_w = d;
 *    1 <= Cq, Cm <= min(N, 2048); 1 <= iters <= 64; 0 < rho <= 1; 0 <= alpha <= 1;
 *    N <= 2^22; B*H <= 16383; B*H*N < 2^31.  Device pointers must be 16-byte aligned.
 */
#ifndef SCOPE_H
#define SCOPE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SCOPE_OK = 0,
    SCOPE_ERR_INVALID_ARGUMENT = 1,
    SCOPE_ERR_UNSUPPORTED = 2,
    SCOPE_ERR_WORKSPACE_TOO_SMALL = 3,
    SCOPE_ERR_CUDA = 4,
    SCOPE_ERR_DEVICE_CHECK = 5,
    SCOPE_ERR_TIMEOUT = 6
} scope_status;

typedef enum { SCOPE_F32 = 0, SCOPE_BF16 = 1 } scope_dtype;

/* Device status bits (scope_get_device_status). */
#define SCOPE_DEV_BAD_INIT_INDEX 0x1   /* an init index was outside [0, N); row 0 was used */
#define SCOPE_DEV_SELECT_TIE     0x2   /* a selection boundary could not be resolved exactly */
#define SCOPE_DEV_BAD_ASSIGN     0x4   /* a cluster index >= C or a code >= Cm was supplied (clamped) */
#define SCOPE_DEV_TIMEOUT        0x8   /* an on-chip pipeline wait gave up (~4 s); outputs invalid */
#define SCOPE_DEV_BAD_COUNTS     0x10  /* a selection mask row holds fewer keys than its r_c; the
                                          missing keys were taken as key 0 */
#define SCOPE_DEV_DEBUG_CHECK    0x20  /* debug builds (-DSCOPE_DEBUG) only: an internal index was
                                          out of range; the access used element 0 instead */

/* k_head handling (scope_params.khead_mode).  ONLINE: Eqs. 9-10, every cluster is
 * topped up to the head's k_head (the method).  OFF: the ablation the review page
 * proposes (significance; forward_implications: the online k_head switched off): k_head is
 * still computed and reported, but r_c = b_c (hybrid Top-p / fixed Top-k only). */
typedef enum { SCOPE_KHEAD_ONLINE = 0, SCOPE_KHEAD_OFF = 1 } scope_khead_mode;

/* Key clustering (scope_params.key_clustering).  SUBSPACES: the method, three k-means over
 * the temporal / height / width channel ranges.  FULL: the ablation the review page asks
 * for (significance; falsifier: scoring with clusters over all channels): one k-means of the
 * keys over all d channels into Cm centroids, so that the proxy of Eq. 6 becomes the
 * cluster-level s~_cj = q_c . mu_{z_j} / sqrt d.  k_codes row 0 then holds z_j and rows 1
 * and 2 are zero; selection reads it as a one-subspace product code with split (d, 0, 0),
 * where the two empty subspaces contribute exact zeros. */
typedef enum { SCOPE_KEYS_SUBSPACES = 0, SCOPE_KEYS_FULL = 1 } scope_key_clustering;

/* Shape and hyperparameters of one layer.  rho: Top-p threshold of Eq. 7 (the paper
 * does not report it; 0.9 is the usual choice).  alpha: fixed Top-k minimum as a
 * fraction of N, k_fix = ceil(alpha * N) (the paper gives alpha = 0.1).  iters: Lloyd
 * iterations of every k-means.  khead_mode: a scope_khead_mode, key_clustering: a
 * scope_key_clustering (a zero-initialised struct gets the method in both). */
typedef struct {
    int B, H;
    int T, Hg, Wg;
    int d, d_t, d_h, d_w;
    int Cq, Cm;
    int iters;
    double rho, alpha;
    scope_dtype dtype;
    int khead_mode;
    int key_clustering;
} scope_params;

/* Optional intermediate outputs of scope_forward (device pointers; NULL = keep the
 * value in the workspace only).  Layouts as in the stage functions below. */
typedef struct {
    double *q_centroids;   /* [B, H, Cq, d] */
    uint16_t *q_assign;    /* [B, H, N] */
    int32_t *q_sizes;      /* [B, H, Cq] */
    double *k_centroids;   /* [B, H, Cm, d] */
    uint16_t *k_codes;     /* [B, H, 3, N] */
    int32_t *topp_counts;  /* [B, H, Cq]  p_c */
    int32_t *base_counts;  /* [B, H, Cq]  b_c */
    int32_t *k_head;       /* [B, H] */
    int32_t *final_counts; /* [B, H, Cq]  r_c */
    uint32_t *sel_mask;    /* [B, H, Cq, ceil(N/32)] */
    /* Optional cudaEvent_t handles (NULL = skip) recorded on the stream at the stage
     * boundaries: [0] start, [1] after clustering, [2] after selection, [3] after the
     * attention work list is built, [4] after the attention kernel. */
    void *stage_events[5];
} scope_intermediates;

/* Bytes of workspace every entry point below needs for `p` (0 if p is invalid). */
size_t scope_workspace_bytes(const scope_params *p);

/*
 * Query clustering (abstract: the queries are grouped into clusters; review page, major_comments[0]: the
 * cluster centroid q_c; major_comments[1]: Cq = 300).  Lloyd k-means on all d
 * channels, params->iters iterations.  One iteration assigns every token to its
 * nearest centroid in squared Euclidean distance (lowest index on a tie), then moves
 * every non-empty centroid to the mean of its members; empty centroids stay.
 *   Q            [B,H,N,d] dtype
 *   init_idx     [B,H,Cq] int32 token indices of the initial centroids, or NULL
 *   init_cent    [B,H,Cq,d] double initial centroids (used when init_idx is NULL)
 *   q_centroids  out [B,H,Cq,d] double: means of the final members
 *   q_assign     out [B,H,N] uint16: final assignments
 *   q_sizes      out [B,H,Cq] int32: final member counts n_c
 * Assignments are exact: distances are certified against binary64 sums over the
 * channels in order, so they equal a binary64 evaluation of the definition.
 */
scope_status scope_cluster_queries(const scope_params *p, const void *Q, const int32_t *init_idx,
                                   const double *init_cent, double *q_centroids,
                                   uint16_t *q_assign, int32_t *q_sizes, void *ws,
                                   size_t ws_bytes, void *stream);

/*
 * Key subspace clustering (abstract: keys partitioned into temporal, height and width
 * subspaces and clustered independently; review page, load_bearing_attack: Eq. 3,
 * k-means minimising Euclidean reconstruction error per subspace; Cm = 333).  Three
 * independent Lloyd k-means, one per channel range, same rules as the queries.
 *   K            [B,H,N,d] dtype
 *   init_idx     [B,H,3,Cm] int32 (subspace-major), or NULL
 *   init_cent    [B,H,Cm,d] double (used when init_idx is NULL)
 *   k_centroids  out [B,H,Cm,d] double: centroid z of subspace m in m's channel range
 *   k_codes      out [B,H,3,N] uint16: z^T_j, z^H_j, z^W_j
 */
scope_status scope_cluster_keys(const scope_params *p, const void *K, const int32_t *init_idx,
                                const double *init_cent, double *k_centroids, uint16_t *k_codes,
                                void *ws, size_t ws_bytes, void *stream);

/*
 * Lookup tables, proxy logits and selection (review page, key_machinery: Eq. 6
 * s_cj = (1/sqrt d) sum_m P^m[c, z^m_j] and Eq. 9 k_head = ceil(sum n_c b_c / sum n_c);
 * major_comments[1]: hybrid Top-p / fixed Top-k (Eq. 7), base counts b_c (Eq. 8),
 * top-up (Eq. 10)).  Per (b, h, c):
 *   P^m[c,z] = sum_{i in m} q_c[i] * mu^m_z[i];  s_cj = (1/sqrt d)((P^T + P^H) + P^W);
 *   keys ranked by s_cj descending, key index ascending on equal logits;
 *   p_c = least r whose first r keys hold softmax mass >= rho (rho = 1: p_c = N);
 *   b_c = max(p_c, ceil(alpha N)); k_head = ceil(sum_c n_c b_c / N);
 *   r_c = max(b_c, k_head); S_c = first r_c keys of the ranking.
 *   q_centroids [B,H,Cq,d] double, q_sizes [B,H,Cq] int32,
 *   k_centroids [B,H,Cm,d] double, k_codes [B,H,3,N] uint16  (as produced above)
 *   topp_counts  out [B,H,Cq] int32 p_c (may be NULL)
 *   base_counts  out [B,H,Cq] int32 b_c
 *   k_head       out [B,H] int32
 *   final_counts out [B,H,Cq] int32 r_c
 *   sel_mask     out [B,H,Cq,ceil(N/32)] uint32: bit (j%32) of word j/32 set iff j in S_c
 * Logits and ranks are binary64 and exact; the softmax mass is summed in binary64, so
 * p_c can differ from another binary64 evaluation only where the mass of a prefix is
 * within ~1e-12 (relative) of rho.
 */
scope_status scope_build_lut_and_select(const scope_params *p, const double *q_centroids,
                                        const int32_t *q_sizes, const double *k_centroids,
                                        const uint16_t *k_codes, int32_t *topp_counts,
                                        int32_t *base_counts, int32_t *k_head,
                                        int32_t *final_counts, uint32_t *sel_mask, void *ws,
                                        size_t ws_bytes, void *stream);

/*
 * Sparse attention over the selected original keys and values (abstract: "sparse
 * attention is then computed over the selected original keys and values"):
 *   O_i = sum_{j in S_c} softmax_j(q_i . k_j / sqrt d) v_j  for every token i, c = q_assign[i].
 * Queries are grouped by cluster on the device; bf16 runs on the tensor cores
 * (tcgen05, fp32 accumulation and softmax), fp32 on the CUDA cores.
 *   Q, K, V      [B,H,N,d] dtype;  O out [B,H,N,d] dtype
 *   q_assign     [B,H,N] uint16;  sel_mask [B,H,Cq,ceil(N/32)] uint32
 *   final_counts [B,H,Cq] int32 r_c (popcount of each mask row; used for scheduling)
 * A query whose cluster selects no key gets O_i = 0.
 */
scope_status scope_sparse_attention(const scope_params *p, const void *Q, const void *K,
                                    const void *V, const uint16_t *q_assign,
                                    const uint32_t *sel_mask, const int32_t *final_counts,
                                    void *O, void *ws, size_t ws_bytes, void *stream);

/*
 * The whole layer: query and key clustering (initial centroids from q_init_idx
 * [B,H,Cq] and k_init_idx [B,H,3,Cm]), selection and sparse attention, enqueued with
 * no host synchronisation.  `inter` may be NULL or name buffers that receive the
 * intermediates.
 */
scope_status scope_forward(const scope_params *p, const void *Q, const void *K, const void *V,
                           const int32_t *q_init_idx, const int32_t *k_init_idx, void *O,
                           const scope_intermediates *inter, void *ws, size_t ws_bytes,
                           void *stream);

/*
 * Selection without a workspace.  The SCOPE paper has no counterpart: this is an
 * integration variant of scope_build_lut_and_select (same arguments minus the workspace,
 * same kernels, same outputs) for callers that cannot call cudaMalloc, such as a host
 * application that owns every device allocation through its own pool and does not let
 * libraries allocate, or a latency-critical loop in which cudaMalloc / cudaFree (which
 * may synchronise the device) are not allowed.  Its scratch -- a status word and 64
 * bytes per (b, h, query cluster) unit -- lives in a fixed device array of the library
 * (256 B + 1 MiB, held by every GPU that loads the library until the process exits).
 *  - B*H*Cq must not exceed SCOPE_NOALLOC_MAX_UNITS; larger layers are rejected with
 *    SCOPE_ERR_UNSUPPORTED before anything is enqueued.
 *  - Every call looks up the array's device address on the current device
 *    (cudaGetSymbolAddress: no allocation, no stream operation), so the address stays right
 *    after a device reset; the first call on a device also loads the library's device code
 *    there, so make that first call before any stream capture.
 *  - Every call shares the array and it keeps the last call's contents; each call clears
 *    the status word it needs.  Calls whose work overlaps on the GPU (other streams, or
 *    other host threads on the same device) race on the array: serialise them.
 *  - The device status word of this variant is not readable through
 *    scope_get_device_status (use the workspace entry point when the status is needed).
 * Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 */
#define SCOPE_NOALLOC_MAX_UNITS 16384
scope_status scope_build_lut_and_select_noalloc(const scope_params *p, const double *q_centroids,
                                                const int32_t *q_sizes, const double *k_centroids,
                                                const uint16_t *k_codes, int32_t *topp_counts,
                                                int32_t *base_counts, int32_t *k_head,
                                                int32_t *final_counts, uint32_t *sel_mask,
                                                void *stream);

/*
 * Proxy-ranking fidelity (review page, falsifier and skeptic's concrete test: how many of
 * a query's dominant keys the centroid-product proxy of Eq. 6 and the selected set keep).
 * For every sampled query g = (b*H + h)*N + i of a layer that went through the stages
 * above: T = its ceil(frac*N) keys of largest exact logit q_i.k_j (binary64, channels in
 * order; ties to the lower key index); recall_sel[s] = |T n S_c| / |T|, S_c the selection
 * of its cluster c = q_assign[g]; recall_proxy[s] = |T n P| / |T|, P the ceil(frac*N) keys
 * of largest proxy logit of cluster c (Eq. 6, binary64; ties to the lower index).
 * Inputs (device): Q, K [B,H,N,d] in params->dtype; q_assign [B,H,N]; q_centroids
 * [B,H,Cq,d]; k_centroids [B,H,Cm,d]; k_codes [B,H,3,N]; sel_mask [B,H,Cq,ceil(N/32)];
 * samples: n_samples int64 query indices.  Outputs (device): recall_sel, recall_proxy,
 * n_samples doubles each (NaN for an index outside the layer).  scratch: caller-owned
 * device memory, 16*N bytes per sample processed at once (at least 16*N; up to one sample
 * per SM).  Requires 0 < frac <= 1 and Cm <= 1024; invalid arguments return an error
 * before any launch.  Allocates nothing; enqueues on `stream`.
 */
scope_status scope_selection_recall(const scope_params *p, const void *Q, const void *K,
                                    const uint16_t *q_assign, const double *q_centroids,
                                    const double *k_centroids, const uint16_t *k_codes,
                                    const uint32_t *sel_mask, const int64_t *samples, int n_samples,
                                    double frac, double *recall_sel, double *recall_proxy,
                                    void *scratch, size_t scratch_bytes, void *stream);

/*
 * Rank correlation of the proxy with the true logits (review page: the test the skeptic asks
 * for, how well the Eq. 6 proxy ranking of the keys follows the true one).  For every
 * sampled query g = (b*H + h)*N + i: spearman[s] = Spearman's rho over the N keys of head
 * (b, h) between x_j = q_i . k_j (exact, binary64, channels in order) and y_j = s~_{c,j}, the
 * Eq. 6 proxy logits of its cluster c = q_assign[g]: the Pearson correlation of the two
 * vectors of average ranks (tied values share the mean of their 1-based ranks).  NaN for an
 * index outside the layer.  Inputs as for scope_selection_recall; scratch: caller-owned
 * device memory of at least scope_rank_correlation_scratch_bytes(p, n_samples) bytes (about
 * 64 * N bytes per sample plus the sort's temporary storage); requires Cm <= 1024 and
 * 2 * n_samples * N < 2^31.  Allocates nothing; enqueues on `stream`.
 */
size_t scope_rank_correlation_scratch_bytes(const scope_params *p, int n_samples);
scope_status scope_rank_correlation(const scope_params *p, const void *Q, const void *K, const uint16_t *q_assign,
                                    const double *q_centroids, const double *k_centroids, const uint16_t *k_codes,
                                    const int64_t *samples, int n_samples, double *spearman, void *scratch,
                                    size_t scratch_bytes, void *stream);

/*
 * Channel permutation for the review page's ablation that partitions the channels at random
 * (significance): Y[b,h,n,e] = X[b,h,n,perm[e]] for e < d.  One permutation applied to
 * both Q and K leaves every logit q.k unchanged, so the layer run on the permuted Q and K
 * (and the original V) is SCOPE with the key subspaces T, H, W made of the channel subsets
 * perm[0 .. d_t), perm[d_t .. d_t+d_h), perm[d_t+d_h .. d) instead of the 3D-RoPE ranges.
 * X, Y: [B,H,N,d] in params->dtype (device, distinct buffers); perm: d int32 (device), a
 * permutation of 0 .. d-1 (entries outside [0, d) are clamped).  Enqueues on `stream`.
 */
scope_status scope_permute_channels(const scope_params *p, const void *X, const int32_t *perm, void *Y,
                                    void *stream);

/*
 * Dense attention, O_i = sum_j softmax_j(q_i . k_j / sqrt d) v_j over all N keys, on the
 * same kernels as scope_sparse_attention (one query cluster that selects every key).  It is
 * the dense branch of the dense-prefix schedule (review page, major_comments: "§4,
 * Implementation details": the first attention layer runs dense at every denoising step,
 * and every layer runs dense during the first 20 % (Wan2.1/2.2) or 10 % (HunyuanVideo) of
 * the steps).
 *   Q, K, V [B,H,N,d] dtype;  O out [B,H,N,d] dtype
 *   ws      workspace of at least scope_workspace_bytes(p) bytes (p->Cq, p->Cm, p->iters,
 *           p->rho, p->alpha and p->khead_mode are validated but not used)
 */
scope_status scope_dense_attention(const scope_params *p, const void *Q, const void *K, const void *V, void *O,
                                   void *ws, size_t ws_bytes, void *stream);

/*
 * 3D rotary position embedding (RoPE) of pre-RoPE queries and keys, the step before the
 * path: SCOPE clusters post-RoPE q and k, whose channels split into the temporal, height and
 * width ranges of 3D RoPE (SCOPE abstract; the rotation is RoFormer's, the page's reference
 * [31]).  For token n = t*Hg*Wg + h*Wg + w and channel range a in {T, H, W} (start c_a, width
 * d_a, position p_a = t, h, w), pair i = channels (c_a + 2i, c_a + 2i + 1) turns by
 * phi = p_a * base^(-2i / d_a):
 *   y[c_a+2i] = x[c_a+2i] cos phi - x[c_a+2i+1] sin phi
 *   y[c_a+2i+1] = x[c_a+2i] sin phi + x[c_a+2i+1] cos phi
 *   Q  [B,H,N,d] dtype, Qr out [B,H,N,d] dtype (Qr may be Q: in place)
 *   K, Kr  the same for the keys, or both NULL to rotate Q only
 *   base   > 0 (10000 for the usual RoPE)
 * Result: angle, cos and sin in binary64, the two products and their sum each rounded
 * to binary64 (no fused multiply-add), then one rounding to dtype (for bf16 a binary32
 * evaluation is kept only where an error bound proves it rounds the same).  Requires even
 * d_t, d_h, d_w (else SCOPE_ERR_INVALID_ARGUMENT) and 24 * (T*d_t + Hg*d_h + Wg*d_w) / 2 <= 196608
 * (the cos/sin table lives in shared memory; else SCOPE_ERR_UNSUPPORTED).  Input and output
 * must be the same buffer or not overlap at all.  No workspace; allocates nothing.
 */
scope_status scope_rope3d(const scope_params *p, double base, const void *Q, const void *K, void *Qr, void *Kr,
                          void *stream);

/* Where a layer sits in the sampling loop, and the dense-prefix schedule (review page,
 * major_comments: "§4, Implementation details"): a layer runs dense attention when
 * layer < dense_layers (the paper: the first layer, dense_layers = 1) or step < dense_steps
 * (the paper: the first 20 % of the denoising steps on Wan2.1/2.2, 10 % on HunyuanVideo;
 * e.g. 10 or 5 of 50 steps), and SCOPE otherwise.  rope != 0: Q and K are pre-RoPE and get
 * scope_rope3d with rope_base first. */
typedef struct {
    int layer;        /* attention layer index in the model, from 0 */
    int step;         /* denoising step index, from 0 */
    int dense_layers;
    int dense_steps;
    int rope;
    double rope_base;
} scope_layer_schedule;

/* 1 when the schedule makes this layer dense, 0 when it runs SCOPE, -1 for a NULL
 * schedule or a negative field.  Host only; touches no device. */
int scope_layer_is_dense(const scope_layer_schedule *sched);

/*
 * One attention layer under the dense-prefix schedule: [3D RoPE of Q and K into Qr, Kr]
 * then scope_dense_attention or scope_forward.
 *   q_init_idx, k_init_idx  as for scope_forward (may be NULL on a dense layer)
 *   Qr, Kr  [B,H,N,d] dtype outputs of the rotation when sched->rope (may be Q and K: in
 *           place); ignored otherwise
 *   ws      at least scope_workspace_bytes(p) bytes
 * All arguments of both stages are validated before anything is enqueued.
 */
scope_status scope_attention_layer(const scope_params *p, const scope_layer_schedule *sched, const void *Q,
                                   const void *K, const void *V, const int32_t *q_init_idx,
                                   const int32_t *k_init_idx, void *O, void *Qr, void *Kr, void *ws,
                                   size_t ws_bytes, void *stream);

/*
 * Check of the device-side wait limit (failure detection; the paper has no counterpart).
 * Every pipeline wait of the tensor-core kernels gives up after a limit, sets
 * SCOPE_DEV_TIMEOUT in the status word and lets the kernel drain and return, so that a lost
 * signal ends in an error status instead of a hung GPU.  This entry point makes such a wait
 * run out on purpose: it launches the bf16 attention kernel with its work-item scheduler
 * held back (no item is ever published), so the first wait of every warp gives up after
 * wait_limit_ns, before any copy or tensor-core product is issued.  Afterwards
 * scope_get_device_status(ws) returns SCOPE_ERR_TIMEOUT with SCOPE_DEV_TIMEOUT set, and the
 * context stays usable for the next call.
 *   p              a valid bf16 layer (else SCOPE_ERR_UNSUPPORTED); its tensors are not read
 *   wait_limit_ns  1 .. 10^10 (else SCOPE_ERR_INVALID_ARGUMENT)
 *   ws             workspace of at least scope_workspace_bytes(p) bytes (its status word
 *                  and scheduler counters are written)
 * Allocates nothing; enqueues one kernel on `stream`.
 */
scope_status scope_check_wait_timeout(const scope_params *p, uint64_t wait_limit_ns, void *ws, size_t ws_bytes,
                                      void *stream);

/*
 * Accumulation check of the tensor-core products (a diagnostic; the paper has no
 * counterpart).  The certified k-means assignment bounds the fp32 error of its
 * tcgen05.mma scores with an allowance per 16-channel step for the sum the tensor core
 * forms of its exact bf16 products and the accumulator, which NVIDIA does not document.
 * This runs that instruction form (kind::f16, M = 128, bf16 operands in 128-byte swizzled
 * K-major shared memory, fp32 accumulator in TMEM) as one chain of K/16 steps:
 *   D[i][j] = sum_k A[i][k] B[j][k]   (the tensor core's own fp32 result)
 *   A  [128, K] bf16, B [N, K] bf16, D out [128, N] float (device, 16-byte aligned)
 *   64 <= K <= 512 with K % 64 == 0; 16 <= N <= 256 with N % 16 == 0; the operands must fit
 *   in shared memory: (K/64) * (128 + N) * 128 bytes <= 231 KB (else SCOPE_ERR_UNSUPPORTED).
 * One CTA; allocates nothing; enqueues on `stream`.
 */
scope_status scope_tc_accumulation_probe(const void *A, const void *B, int K, int N, float *D, void *stream);

/* Human-readable name of a status code (static storage). */
const char *scope_status_string(scope_status s);

/* Synchronises `stream` and returns the device status word of the last call that used
 * `ws` in *out (0 = clean; SCOPE_DEV_* bits otherwise).  Returns SCOPE_OK for a clean word,
 * SCOPE_ERR_TIMEOUT when SCOPE_DEV_TIMEOUT is set (a pipeline wait gave up; the outputs of
 * that call are invalid, the context stays usable), SCOPE_ERR_DEVICE_CHECK for any other
 * bit, SCOPE_ERR_CUDA if the copy or the synchronisation failed. */
scope_status scope_get_device_status(const void *ws, void *stream, int32_t *out);

/* Top-p decision statistics of the last selection that used `ws` (scope_forward or
 * scope_build_lut_and_select with parameters `p`): synchronises `stream` and writes
 * out[0] = Top-p decisions made (one per unit (b, h, c) when rho < 1), out[1] = those whose
 * margin is below 1e-6, out[2] = below 3e-7, out[3] = 0.  The margin of a decision is
 * min(|M_{p-1} - rho Z|, |M_p - rho Z|) / Z, with M_r the softmax mass of the first r keys of
 * the ranking and Z the total (Eq. 7; the same quantity the binary64 reference logs as a near
 * tie below 1e-6), computed from the fixed-point masses of the selection (relative error below
 * 3e-7, so only a decision with a margin below 3e-7 can differ from the binary64 one).  The
 * margin is at most half the mass of the crossing key, so at large N a sizeable share of the
 * decisions falls below 1e-6.  SCOPE_ERR_INVALID_ARGUMENT for a NULL pointer or invalid `p`, SCOPE_ERR_CUDA if the
 * copy or the synchronisation failed. */
scope_status scope_get_selection_stats(const scope_params *p, const void *ws, void *stream, int32_t *out);

#ifdef __cplusplus
}
#endif

#endif /* SCOPE_H */
