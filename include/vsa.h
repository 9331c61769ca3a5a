/*
 * vsa.h -- C ABI of libvsa, block-sparse self-attention over long video-DiT
 * token sequences on NVIDIA B200 (sm_100a).
 *
 * The path, one call per step:
 *   vsa_pool_qk          block means of Q and K                     (pooling)
 *   vsa_select_blocks    per-head block mask from the pooled scores (selection)
 *   vsa_block_sparse_fwd attention over the kept tiles -> O, LSE    (Macro / Micro pass)
 *   vsa_select_micro     Micro tiles inside omitted blocks          (Micro selection)
 *   vsa_block_sparse_fwd again on the Micro lists, merged by LSE    (Micro pass + merge)
 *   (vsa_block_sparse_fwd_heads: either pass on a subset of the heads)
 * and, for the cluster-permuted layout, vsa_cluster_tokens + vsa_permute_rows;
 * for cluster-aligned blocks, vsa_select_clusters, vsa_merge_clusters,
 * vsa_cluster_plan, vsa_gather_rows and vsa_cluster_group_fwd; for pooled
 * rectification of omitted blocks, vsa_pool_kv_bf16 + vsa_rectify_fwd.
 * plus vsa_mask_to_lists (an explicit block mask instead of selection) and
 * vsa_lse_merge (the stand-alone exact merge).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Layout.   Q, K, V, O are contiguous row-major [B, H, n_pad, d]: token rows of
 *           one (batch, head) are consecutive, d is innermost.  Tokens are in
 *           the video's frame-first (t, y, x) order; blocks are consecutive
 *           token ranges of that order.  Rows n_valid <= row < n_pad are
 *           padding: their Q/K/V content is never read into a result, their
 *           O is written as 0 and their LSE as -inf.
 * Pointers. Every tensor pointer is a DEVICE pointer (cudaMalloc'd or
 *           equivalent) unless stated otherwise; the caller allocates and
 *           owns every buffer, including workspaces.  The library allocates
 *           no device memory and never synchronises the stream, except
 *           vsa_read_device_status.  ``stream`` is a cudaStream_t (NULL =
 *           legacy default stream).  All work is enqueued asynchronously.
 * Errors.   Argument errors are detected on the host before anything is
 *           enqueued and returned synchronously (VSA_ERR_INVALID_ARG /
 *           VSA_ERR_UNSUPPORTED); a failed launch returns VSA_ERR_CUDA.
 *           Conditions found on the device (a list longer than its capacity,
 *           an out-of-range index in a caller-given list, a pipeline wait that
 *           ran out of its time limit) are latched into a device status word
 *           that vsa_read_device_status returns and clears: the caller's word
 *           bound to the call's stream (vsa_bind_status_word), else a
 *           process-wide word per device.
 * Numerics. Pooling, pooled scores and selection are fp32 (FFMA; no TF32).
 *           Attention multiplies bf16 operands on the tensor cores with fp32
 *           accumulation; P is rounded to bf16 before the P.V product; LSE is
 *           fp32, natural log, softmax scale included.
 *
 * Sources (pages by title, section / equation):
 *   [HVA]   HyperVAttention: Efficient Sparse Attention with Spatio-Temporal
 *           Clustering for Video Diffusion (arXiv 2607.03012v1)
 *   [HyMoR] HyMoR-Attn: Granularity-Matched Repair of Omitted Attention
 *           Support for Video Diffusion (abstract)
 *   [RSA]   Rectified SpaAttn: Revisiting Attention Sparsity for Efficient
 *           Video Generation (abstract)
 *   [LVSA]  Long Video Sparse Attention (abstract on the "FreqFormer" page)
 *   [MOD]   MOD-DiT (arXiv 2601.11641), "Block-wise Attention Computation"
 */
#ifndef VSA_H_
#define VSA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define VSA_API __attribute__((visibility("default")))
#else
#define VSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  VSA_OK = 0,
  VSA_ERR_INVALID_ARG = 1,   /* null pointer, bad size or inconsistent shape      */
  VSA_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. d not in {64,128}) */
  VSA_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed                   */
  VSA_ERR_CAPACITY = 4,      /* device: a list exceeded its caller-given capacity   */
  VSA_ERR_BAD_INDEX = 5,     /* device: a caller-given list holds an invalid index  */
  VSA_ERR_TIMEOUT = 6,       /* device: a pipeline wait exceeded its time limit     */
  VSA_ERR_SCRATCH_LIMIT = 7  /* the problem needs more scratch than the fixed
                                scratch of vsa_select_micro_noalloc holds         */
} vsa_status;

/* Problem shape.  d in {64, 128}; n_valid <= n_pad; n_pad a multiple of 128. */
typedef struct {
  int B, H;
  int n_valid;   /* real tokens per (batch, head)                     */
  int n_pad;     /* padded row count of every [B, H, n_pad, *] tensor */
  int d;         /* head dimension                                    */
} vsa_shape;

/* Block selection knobs ([HVA] section 2 Eq. (3), App. A.1 "Min-kc"; [LVSA]).
 *   fixed_k > 0 : keep exactly min(fixed_k, n_k) blocks per row, cum_mass ignored.
 *   otherwise   : keep max(k_min, m_p) blocks, m_p = the smallest m whose top-m
 *                 size-weighted pooled probabilities sum to at least cum_mass
 *                 (cum_mass <= 0 disables Top-p, leaving the k_min floor).
 *   n_anchor    : add the key-block columns (anchor_rot + t*floor(n_k/n_anchor))
 *                 mod n_k, t = 0..n_anchor-1, to every non-empty row.        */
typedef struct {
  int k_min;
  float cum_mass;
  int fixed_k;
  int n_anchor;
  int anchor_rot;
} vsa_select_params;

/* Micro selection knobs ([HyMoR] abstract: a fine residual over tiles inside
 * omitted blocks, chosen online).  Micro rows are 64 query rows, Micro tiles
 * 16 keys; a tile is a candidate for a Micro row iff it lies in a key block the
 * row's Macro query block omitted and holds at least one valid key.  Score =
 * mean(Q rows of the Micro row) . mean(K rows of the tile) * scale.
 *   mode 1 : per Micro row, the min(topk, #candidates) highest scores
 *            (ties to the lower tile index); 1 <= topk <= 32.
 *   mode 2 : per enabled head, every candidate whose score is strictly above
 *            tau = the ceil(percentile * M)-th smallest of the head's M
 *            candidate scores (ceil evaluated in IEEE double).
 *   head_enable : HOST array of H flags (NULL = every head); disabled heads
 *            select nothing.
 *   row_capacity : entries per Micro row in m_idx (>= 1).                   */
typedef struct {
  int mode;
  int topk;
  double percentile;
  const uint8_t *head_enable;
  int row_capacity;
} vsa_micro_params;

/* Human-readable name of a status code (static storage). */
VSA_API const char *vsa_status_string(vsa_status s);

/* Library version as major*10000 + minor*100 + patch. */
VSA_API int vsa_version(void);

/* Synchronise ``stream``, then return and clear the status word of that
 * stream (the first device-side error latched since the last read; VSA_OK if
 * none): the caller's word bound to ``stream`` by vsa_bind_status_word, or
 * else the library's process-wide word of the current device. */
VSA_API vsa_status vsa_read_device_status(void *stream);

/* Per-stream status words in caller memory (no counterpart on the pages).
 * After binding, every call enqueued on ``stream`` (on the current device)
 * latches its device-side conditions -- capacity, bad index, timeout -- into
 * ``word`` instead of the process-wide word, so callers on different streams
 * can tell whose work failed, and a bounded wait that runs out of time aborts
 * only the waits reporting into the same word.
 *   word : DEVICE memory of VSA_STATUS_WORD_BYTES bytes, 4-byte aligned,
 *          owned by the caller and kept alive while bound; the call clears
 *          it on ``stream``.  NULL removes the stream's binding.
 * At most 256 bindings at once (VSA_ERR_CAPACITY beyond).  Rebinding a stream
 * replaces its word.  A binding is looked up when a call is enqueued: bind
 * before enqueueing the calls it should cover. */
#define VSA_STATUS_WORD_BYTES 8
VSA_API vsa_status vsa_bind_status_word(void *stream, int32_t *word);

/* Self-test of the bounded pipeline waits (no counterpart on the pages): one
 * thread waits on a shared-memory barrier that nothing completes, for at most
 * limit_ns nanoseconds (1e3 <= limit_ns <= 5e9), then returns.  The status
 * word then reads VSA_ERR_TIMEOUT and the device stays usable; the kernel
 * neither faults nor traps.  Like every timeout it also makes other waits
 * still running give up, until vsa_read_device_status clears it. */
VSA_API vsa_status vsa_selftest_wait_timeout(unsigned long long limit_ns, void *stream);

/* Self-test of the exponential the attention softmax evaluates on the FMA
 * pipe for part of its logits (no counterpart on the pages; the softmax of
 * HyperVAttention Eq. (4) needs 2^x per kept logit): y[i] = 2^x[i] by range
 * reduction to x = n + f, |f| <= 1/2, a degree-3 polynomial for 2^f (relative
 * error at most 7.5e-5) and an exponent add.  Inputs below -125 (and -inf)
 * give 2^-125.  x, y: device fp32 [n], n >= 0.
 * Asynchronous on ``stream``; argument errors return synchronously. */
VSA_API vsa_status vsa_selftest_exp2(const float *x, float *y, int n, void *stream);

/* ---------------------------------------------------------------------------
 * a1 Pooling  ([RSA]: pooled query-key interactions; [HVA] section 4.1: a
 * centroid is the mean of its tokens; [MOD]: fixed non-overlapping blocks.)
 *
 * q, k      : bf16 [B, H, n_pad, d].
 * bq, bk    : Macro query / key block rows, each in {64, 128}.
 * q_pool    : fp32 [B, H, n_pad/bq, d]  mean of the valid Q rows of each block.
 * k_pool    : fp32 [B, H, n_pad/bk, d]  mean of the valid K rows of each block.
 * q_pool64  : fp32 [B, H, n_pad/64, d]  Micro-row means (NULL to skip).
 * k_pool16  : fp32 [B, H, n_pad/16, d]  Micro-tile means (NULL to skip).
 * A block without a valid row has mean 0.  One pass reads Q and K once.
 * ------------------------------------------------------------------------- */
VSA_API vsa_status vsa_pool_qk(const void *q, const void *k, const vsa_shape *shape, int bq, int bk,
                       float *q_pool, float *k_pool, float *q_pool64, float *k_pool16, void *stream);

/* ---------------------------------------------------------------------------
 * a2 + a3 Scoring and selection ([HVA] section 2 Eq. (2) and Eq. (3);
 * App. A.1 "Min-kc"; [LVSA] rotating anchors.)
 *
 * Per (b, h, query block i): S_ij = q_pool_i . k_pool_j * scale;
 * P'_ij = s_j exp(S_ij) / sum_o s_o exp(S_io) with s_j the number of valid keys
 * of block j; blocks ranked by descending S_ij + ln s_j (ties to the lower j);
 * kept = the rule of vsa_select_params.  A query block without a valid row
 * keeps nothing.
 *
 * n_k = n_pad/bk must be <= 1024.
 * counts : int32 [B, H, n_pad/bq]           kept blocks per row.
 * idx    : int32 [B, H, n_pad/bq, n_k]      kept key-block indices, ascending,
 *          in the first counts[row] slots of the row (the rest is untouched).
 * mask   : uint8 [B, H, n_pad/bq, n_k] dense 0/1 block mask, or NULL.
 * ------------------------------------------------------------------------- */
VSA_API vsa_status vsa_select_blocks(const float *q_pool, const float *k_pool, const vsa_shape *shape, int bq,
                             int bk, float scale, const vsa_select_params *params, int32_t *counts,
                             int32_t *idx, uint8_t *mask, void *stream);

/* ---------------------------------------------------------------------------
 * Cluster-level selection ([HVA] section 2 Eq. (2) and Eq. (3) with query and
 * key clusters as the units: the logits are centroid products, s_j is the
 * size of key cluster j).
 *
 * Per (batch-head, query cluster i): S_ij = mu_q_i . mu_k_j * scale; the same
 * ranking (descending S_ij + ln s_j, ties to the lower j, s_j = 0 ranks last)
 * and the same Top-p / Min-kc / fixed-k rule as vsa_select_blocks; anchors are
 * not used (params->n_anchor must be 0).  A query cluster of size 0 keeps
 * nothing.
 *
 * mu_q    : fp32 [batch_heads, n_q, d]  query centroids (16-byte aligned).
 * mu_k    : fp32 [batch_heads, n_k, d]  key centroids.
 * sizes_q : int32 [batch_heads, n_q]    tokens per query cluster.
 * sizes_k : int32 [batch_heads, n_k]    tokens per key cluster.
 * d in {64, 128}; n_k <= 1024 (VSA_ERR_UNSUPPORTED above).
 * counts  : int32 [batch_heads, n_q]       kept key clusters per query cluster.
 * idx     : int32 [batch_heads, n_q, n_k]  kept key-cluster indices, ascending,
 *           in the first counts[row] slots of the row.
 * ------------------------------------------------------------------------- */
VSA_API vsa_status vsa_select_clusters(const float *mu_q, const float *mu_k, const int32_t *sizes_q,
                                       const int32_t *sizes_k, int batch_heads, int n_q, int n_k, int d,
                                       float scale, const vsa_select_params *params, int32_t *counts,
                                       int32_t *idx, void *stream);

/* ---------------------------------------------------------------------------
 * Explicit block mask -> lists (the mask-passed-in path of the same
 * attention, [HVA] section 2: m_ij = 1 iff key block j is attended by row i).
 *
 * mask   : uint8 [B, H, n_pad/bq, n_pad/bk], nonzero = keep.  n_pad/bk <= 1024.
 * counts, idx : as vsa_select_blocks (idx row stride n_pad/bk).
 * ------------------------------------------------------------------------- */
VSA_API vsa_status vsa_mask_to_lists(const uint8_t *mask, const vsa_shape *shape, int bq, int bk, int32_t *counts,
                             int32_t *idx, void *stream);

/* ---------------------------------------------------------------------------
 * a5 Micro selection ([HyMoR] abstract: online selection of the omitted tail
 * at fine granularity; readings in vsa_micro_params.)
 *
 * q_pool64, k_pool16 : from vsa_pool_qk.
 * counts, idx        : the Macro lists (row = Macro query block of bq rows,
 *                      idx row stride n_pad/bk).
 * m_counts : int32 [B, H, n_pad/64]                   tiles per Micro row.
 * m_idx    : int32 [B, H, n_pad/64, row_capacity]     16-key tile indices,
 *            ascending.  A row with more selected tiles than row_capacity
 *            keeps the lowest row_capacity of them and latches
 *            VSA_ERR_CAPACITY.
 * workspace: device scratch of vsa_select_micro_workspace_bytes() bytes,
 *            16-byte aligned; its content on entry is irrelevant.
 * H <= 1024 and n_pad/bk <= 1024 (VSA_ERR_UNSUPPORTED above).  The head
 * flags are read on the host during the call and handed to the device by
 * value: no host-to-device copy, so the call never waits on the host.
 * ------------------------------------------------------------------------- */
VSA_API size_t vsa_select_micro_workspace_bytes(const vsa_shape *shape, const vsa_micro_params *params);

VSA_API vsa_status vsa_select_micro(const float *q_pool64, const float *k_pool16, const int32_t *counts,
                            const int32_t *idx, const vsa_shape *shape, int bq, int bk, float scale,
                            const vsa_micro_params *params, int32_t *m_counts, int32_t *m_idx,
                            void *workspace, size_t workspace_bytes, void *stream);

/* ---------------------------------------------------------------------------
 * Allocation-free Micro selection.  The pages have no counterpart of this
 * entry point: it exists for callers that cannot allocate device memory of
 * their own -- for example a plugin whose host engine owns every byte of
 * device memory and hands out no extra workspace, or a service running under
 * a fixed device-memory budget that another allocator controls (cudaMalloc
 * can also block the whole device while it runs, which such callers avoid).
 *
 * Same arguments, meaning and results as vsa_select_micro, minus the
 * workspace: its scratch lives in one fixed array of
 * VSA_MICRO_NOALLOC_MAX_BYTES bytes of device memory that this library
 * reserves statically in every GPU that loads it, until the process exits.
 * No call allocates or frees anything (no cudaMalloc, cudaFree or allocating
 * library routine).
 *   - A problem whose scratch (vsa_select_micro_workspace_bytes for the same
 *     shape and params) exceeds VSA_MICRO_NOALLOC_MAX_BYTES is rejected with
 *     VSA_ERR_SCRATCH_LIMIT before anything is enqueued.  B*H <= 1024.
 *   - Every call looks up the device address of the fixed array on the
 *     current device (a host-side query that allocates nothing; the first
 *     one on a device may load the library's device code, so make it before
 *     any stream capture).
 *   - Every call on a device shares the one array.  Calls whose GPU work
 *     overlaps in time (different streams, or other threads without
 *     ordering between them) race on it and give undefined lists; order them
 *     on one stream or synchronise between them.  The state that must start
 *     at zero is cleared on the call's stream by every call.
 * ------------------------------------------------------------------------- */
#define VSA_MICRO_NOALLOC_MAX_BYTES ((size_t)16 << 20)

VSA_API vsa_status vsa_select_micro_noalloc(const float *q_pool64, const float *k_pool16, const int32_t *counts,
                                            const int32_t *idx, const vsa_shape *shape, int bq, int bk, float scale,
                                            const vsa_micro_params *params, int32_t *m_counts, int32_t *m_idx,
                                            void *stream);

/* ---------------------------------------------------------------------------
 * a4 / a6 Block-sparse attention forward ([HVA] section 2 Eq. (4): attention of
 * each query block restricted to its selected key blocks; section 4.3: the
 * selected key blocks of a row are walked as one packed sequence.  [HyMoR]
 * abstract: Micro pass merged with the Macro output by exact LSE merging.)
 *
 * For every list row r (list_rows consecutive query rows) and every entry e of
 * its list, the keys [idx[r][e]*seg_keys, idx[r][e]*seg_keys + seg_keys) are
 * attended: O = softmax(Q K^T * scale) V over the union of the row's
 * segments, keys >= n_valid excluded; LSE = ln sum exp(Q K^T * scale).
 *   Macro pass : list_rows = bq, seg_keys = bk, lists from vsa_select_blocks.
 *   Micro pass : list_rows = 64, seg_keys = 16, lists from vsa_select_micro.
 * list_rows in {64, 128}; seg_keys in {16, 32, 64, 128}; entries of a row
 * strictly ascending and < n_pad/seg_keys (violations latch
 * VSA_ERR_BAD_INDEX and the row's output is undefined).
 *
 * counts    : int32 [B, H, n_pad/list_rows];  idx : int32 [.., idx_stride].
 * o         : [B, H, n_pad, d], bf16 (o_fp32 = 0) or fp32 (o_fp32 = 1).
 * lse       : fp32 [B, H, n_pad].
 * merge_o, merge_lse : NULL, or an fp32 [B, H, n_pad, d] output and its fp32
 *             LSE over a key support disjoint from this pass's; then o/lse
 *             receive the exact merge L = ln(e^{L_1} + e^{L_2}),
 *             O = e^{L_1-L} O_1 + e^{L_2-L} O_2 (a row with an empty list
 *             passes merge_o through).  o may not alias merge_o.
 * A row with an empty list and no merge input gets O = 0, LSE = -inf.
 * ------------------------------------------------------------------------- */
VSA_API vsa_status vsa_block_sparse_fwd(const void *q, const void *k, const void *v, const vsa_shape *shape,
                                int list_rows, int seg_keys, const int32_t *counts, const int32_t *idx,
                                int idx_stride, float scale, void *o, int o_fp32, float *lse,
                                const float *merge_o, const float *merge_lse, void *stream);

/* ---------------------------------------------------------------------------
 * The same forward on a subset of the (batch, head) pairs.  Every (batch,
 * head) is an independent problem ([HVA] section 2 Eq. (4) is per head), so a
 * caller may run one pass on some heads and another pass on the rest: the
 * Micro repair of [HyMoR] (abstract) is applied to some heads only, and those
 * heads keep their Macro output in fp32 for the merge while the other heads'
 * Macro output is already final.
 *
 * heads   : NULL (then n_heads must be B*H and the call equals
 *           vsa_block_sparse_fwd), or a DEVICE int32 array of n_heads flattened
 *           indices b*H + h, each in [0, B*H), no index twice.
 * n_heads : 0 <= n_heads <= min(B*H, 65535); 0 enqueues nothing.
 * Only the listed heads are read (their lists, Q/K/V, merge inputs) and
 * written (their rows of o and lse); every other row of o and lse keeps its
 * contents.  An out-of-range entry latches VSA_ERR_BAD_INDEX and writes
 * nothing for that entry; a repeated entry makes two CTAs write the same rows
 * (undefined result).  All other arguments as for vsa_block_sparse_fwd.
 * ------------------------------------------------------------------------- */
VSA_API vsa_status vsa_block_sparse_fwd_heads(const void *q, const void *k, const void *v, const vsa_shape *shape,
                                              int list_rows, int seg_keys, const int32_t *counts, const int32_t *idx,
                                              int idx_stride, float scale, void *o, int o_fp32, float *lse,
                                              const float *merge_o, const float *merge_lse, const int32_t *heads,
                                              int n_heads, void *stream);

/* ---------------------------------------------------------------------------
 * Stand-alone exact LSE merge of two attention results over disjoint key
 * supports ([HyMoR] abstract).  o_a, o_b fp32 [B, H, n_pad, d]; lse_* fp32
 * [B, H, n_pad]; o_out bf16 or fp32 (o_out_fp32); lse_out fp32.  Rows with
 * both LSE = -inf give O = 0, LSE = -inf.  Outputs may alias inputs of the
 * same type.
 * ------------------------------------------------------------------------- */
VSA_API vsa_status vsa_lse_merge(const float *o_a, const float *lse_a, const float *o_b, const float *lse_b,
                         const vsa_shape *shape, void *o_out, int o_out_fp32, float *lse_out, void *stream);

/* ---------------------------------------------------------------------------
 * The whole path in one call ([HVA] section 2 Eq. (2)-(4): pooled scores,
 * selection, attention over the kept blocks; [HyMoR] abstract: Micro repair
 * merged by exact LSE): vsa_pool_qk -> vsa_select_blocks -> Macro pass ->
 * vsa_select_micro -> Micro pass with the fused merge, exactly as a caller
 * would chain the entry points above, on buffers carved from one workspace.
 * Heads without the Micro repair take their final O from the Macro pass;
 * heads with it keep an fp32 Macro output that the Micro pass merges into.
 *
 *   bq, bk           : Macro block rows, each 64 or 128 (n_pad/bk <= 1024).
 *   scale            : softmax scale; 0 = 1/sqrt(d).
 *   select           : the vsa_select_blocks rule.
 *   micro_mode       : 0 = no Micro repair; 1, 2 as vsa_micro_params.mode.
 *   micro_topk, micro_percentile : as vsa_micro_params.
 *   micro_heads      : HOST array of H flags (NULL = every head); H <= 1024.
 *   micro_capacity   : entries per Micro row; 0 = n_pad/16 (no row can overflow).
 *   o_fp32           : 1 = O written in fp32, 0 = bf16.
 * ------------------------------------------------------------------------- */
typedef struct {
  int bq, bk;
  float scale;
  vsa_select_params select;
  int micro_mode;
  int micro_topk;
  double micro_percentile;
  const uint8_t *micro_heads;
  int micro_capacity;
  int o_fp32;
} vsa_path_params;

/* Device workspace of vsa_path_fwd for this shape and params (0 if invalid). */
VSA_API size_t vsa_path_workspace_bytes(const vsa_shape *shape, const vsa_path_params *params);

/* q, k, v: bf16 [B, H, n_pad, d] DEVICE; o: [B, H, n_pad, d] (bf16 or fp32);
 * lse: fp32 [B, H, n_pad].  workspace: DEVICE, 256-byte aligned, at least
 * vsa_path_workspace_bytes(); its content on entry is irrelevant; after the
 * call it holds the pooled means, the kept lists and the Micro lists.
 * Asynchronous on stream. */
VSA_API vsa_status vsa_path_fwd(const void *q, const void *k, const void *v, const vsa_shape *shape,
                                const vsa_path_params *params, void *o, float *lse, void *workspace,
                                size_t workspace_bytes, void *stream);

/* The same path on HOST buffers: q_host, k_host, v_host bf16 [B, H, n_pad, d]
 * in, o_host ([B, H, n_pad, d], bf16 or fp32) and lse_host (fp32 [B, H,
 * n_pad]) out.  Every (batch, head) is an independent problem, so the
 * flattened heads are cut into chunks of at most chunk_heads (the first and
 * the last of half that size, so that the copy-in before the first compute
 * and the work after the last copy-in are short) and pipelined over three
 * workspace slots: the host-to-device copies of chunk i+1 and the
 * device-to-host copies of chunk i-1 overlap the path on chunk i (two
 * library-owned copy streams per device,
 * created on first use and kept until exit; one cudaMemcpyAsync per tensor
 * and chunk).  The results equal vsa_path_fwd's on all heads at once, bit for
 * bit.  Host buffers should be page-locked (cudaHostAlloc) for the copies to
 * overlap; pageable buffers work but serialise.
 *   workspace : DEVICE, 256-byte aligned, at least
 *               vsa_path_host_workspace_bytes(shape, params, chunk_heads).
 * The call returns once everything is enqueued; the work is complete when
 * ``stream`` is (synchronise it before reading o_host / lse_host).  Calls
 * from several host threads are enqueued one at a time. */
VSA_API size_t vsa_path_host_workspace_bytes(const vsa_shape *shape, const vsa_path_params *params,
                                             int chunk_heads);

VSA_API vsa_status vsa_path_fwd_host(const void *q_host, const void *k_host, const void *v_host,
                                     const vsa_shape *shape, const vsa_path_params *params, int chunk_heads,
                                     void *o_host, float *lse_host, void *workspace, size_t workspace_bytes,
                                     void *stream);

/* ---------------------------------------------------------------------------
 * Cluster-permuted layout ([HVA] §4.1 Eq. (5) 3D local-window clustering;
 * §2 Eq. (1) the permutation that makes each cluster's tokens contiguous;
 * Eq. (4) the output put back in token order).
 *
 * The n_valid = lattice_t * lattice_h * lattice_w valid tokens of every
 * (batch, head) form a T x H x W lattice in frame-first order.  The lattice is
 * cut into cells of (cell_t, cell_h, cell_w) tokens (ceil per axis; an edge
 * cell holds the rest), one centroid per cell initialised from the cell's
 * centre token (offset (e-1)/2 along an axis of extent e).  Each of `iters`
 * rounds assigns every token to the nearest centroid (squared Euclidean,
 * fp32, ties to the lower cell) among the cells of a (win_t, win_h, win_w)
 * window around its own cell (offsets -((w-1)/2) .. w/2, clipped), then sets
 * every centroid to the mean of its tokens (an empty cluster keeps its
 * centroid).  The permutation lists the tokens cluster by cluster (cells in
 * flat t-major order), in token order inside a cluster; padding rows
 * n_valid .. n_pad-1 stay in place.  Everything is deterministic.
 * ------------------------------------------------------------------------- */
typedef struct {
  int lattice_t, lattice_h, lattice_w; /* lattice_t*lattice_h*lattice_w == n_valid */
  int cell_t, cell_h, cell_w;          /* >= 1; cell_t*cell_h*cell_w <= 128 */
  int win_t, win_h, win_w;             /* >= 1; win_t*win_h*win_w <= 128 */
  int iters;                           /* 1 .. 64 */
} vsa_cluster_params;

/* Number of cells (clusters) of the parameters, 0 if they are invalid.  Host only. */
VSA_API int vsa_cluster_count(const vsa_cluster_params *params);

/* x: bf16 [B, H, n_pad, d] (Q or K).  Outputs, caller-allocated DEVICE memory:
 *   assign    int32 [B, H, n_valid]   cluster (flat cell index) of each token
 *   centroids fp32  [B, H, n_cells, d]
 *   sizes     int32 [B, H, n_cells]   tokens per cluster
 *   perm      int32 [B, H, n_pad]     row i of the permuted sequence is token perm[i]
 * Invalid parameters or a lattice that does not match n_valid return
 * VSA_ERR_INVALID_ARG; d must be 64 or 128. */
VSA_API vsa_status vsa_cluster_tokens(const void *x, const vsa_shape *shape, const vsa_cluster_params *params,
                                      int32_t *assign, float *centroids, int32_t *sizes, int32_t *perm,
                                      void *stream);

/* Hybrid clustering across denoising steps ([HVA] section 4.2, Eq. (6); App.
 * A.1: full clustering at anchor steps, a cached subset of the most ambiguous
 * tokens updated at the steps in between).
 *
 * vsa_cluster_anchor: vsa_cluster_tokens (params->iters >= 1 rounds) whose
 * last assignment round also writes Lowe's ratio rho = d1 / d2 of every token
 * (Euclidean distances to the nearest and second-nearest centroid of its
 * window, the centroids that round compared; 0 for a window of one centroid,
 * 1 when both distances are 0), then the n_sub tokens of largest rho (ties to
 * the lower token index), ascending:
 *   ratio  fp32  [B, H, n_valid];  subset int32 [B, H, n_sub], 1 <= n_sub <= n_valid.
 *
 * vsa_cluster_refine: an intermediate step on the current embeddings x.  Each
 * token of subset is reassigned to the nearest centroid of the whole set
 * (squared Euclidean distance, ties to the lower cluster); tokens outside the
 * subset keep their cluster.  Every cluster that gained or lost a token gets
 * the mean of its members' current embeddings (an emptied one keeps its
 * centroid); the others are unchanged.  sizes and perm are rebuilt from the
 * new assignment (clusters in order, tokens in token order, padding rows in
 * place).  assign and centroids are read and updated in place.
 *   workspace: device scratch of vsa_cluster_refine_workspace_bytes() bytes,
 *   256-byte aligned.  At most 4096 clusters.
 * An assignment or subset entry out of range latches VSA_ERR_BAD_INDEX. */
VSA_API vsa_status vsa_cluster_anchor(const void *x, const vsa_shape *shape, const vsa_cluster_params *params,
                                      int n_sub, int32_t *assign, float *centroids, int32_t *sizes, int32_t *perm,
                                      float *ratio, int32_t *subset, void *stream);

VSA_API size_t vsa_cluster_refine_workspace_bytes(const vsa_shape *shape, const vsa_cluster_params *params);

VSA_API vsa_status vsa_cluster_refine(const void *x, const vsa_shape *shape, const vsa_cluster_params *params,
                                      const int32_t *subset, int n_sub, int32_t *assign, float *centroids,
                                      int32_t *sizes, int32_t *perm, void *workspace, size_t workspace_bytes,
                                      void *stream);

/* Row permutation along the token axis of [B*H, n_pad, row] data (rows of
 * row_bytes, a multiple of 4, 16-byte aligned when a multiple of 16):
 *   inverse = 0: dst[bh][i] = src[bh][perm[bh][i]]   (Eq. (1): X' = Pi X)
 *   inverse = 1: dst[bh][perm[bh][i]] = src[bh][i]   (Eq. (4): O = Pi^-1 O')
 * perm is int32 [B*H, n_pad], each row a permutation of 0 .. n_pad-1; an entry
 * out of range latches VSA_ERR_BAD_INDEX and that row is not copied.
 * src and dst must not overlap. */
VSA_API vsa_status vsa_permute_rows(const void *src, const int32_t *perm, int batch_heads, int n_pad, int row_bytes,
                                    int inverse, void *dst, void *stream);

/* ---------------------------------------------------------------------------
 * Hardware-aware cluster merging ([HVA] section 4.3, Eq. (7)-(10), Algorithm 1
 * "Parallel Agglomerative Merging").
 *
 * Query clusters are merged into groups S; a group's cost is
 * C(S) = tau_q ceil(s_q(S) / tau_q) * tau_k ceil(w_k(S) / tau_k), s_q(S) its
 * query tokens and w_k(S) the summed sizes of chi(S), the union of the key
 * clusters its members kept (Eq. (8)).  Starting from singletons, each of
 * `rounds` rounds splits the current groups by sides[r][leader] (0 = side A,
 * else B; the leader of a group is its lowest member), lets every A group
 * pick the B group of smallest dC = C(A u B) - C(A) - C(B) (ties to the lower
 * leader), keeps for every B the picking A of smallest dC (ties to the lower
 * leader), and merges the kept pairs with dC < 0.  The random bipartition is
 * an input so that runs are reproducible.  A query cluster of size 0 never
 * merges.  All arithmetic is integer: the result is exact.
 *
 * sizes_q : int32 [batch_heads, n_q]        tokens per query cluster (>= 0).
 * sizes_k : int32 [batch_heads, n_k]        tokens per key cluster (>= 0).
 * counts, idx : the kept lists (vsa_select_clusters layout; idx row stride n_k).
 * sides   : uint8 [batch_heads, rounds, n_q] bipartition bits; may be NULL when
 *           rounds == 0.
 * n_q, n_k <= 1024 (VSA_ERR_UNSUPPORTED above); 0 <= rounds <= 64;
 * 1 <= tau_q, tau_k <= 2^20.
 * workspace : device scratch of vsa_merge_clusters_workspace_bytes() bytes,
 *           256-byte aligned; its content on entry is irrelevant.
 * Outputs:
 *   group_of : int32 [batch_heads, n_q]       leader of each cluster's group.
 *   g_counts : int32 [batch_heads, n_q]       at a leader: |chi(S)|; else 0.
 *   g_idx    : int32 [batch_heads, n_q, n_k]  at a leader: chi(S) ascending in
 *              the first g_counts slots (other rows untouched).
 * An invalid kept list (not strictly ascending, out of range) or a negative
 * size latches VSA_ERR_BAD_INDEX; that list counts as empty.
 * ------------------------------------------------------------------------- */
VSA_API size_t vsa_merge_clusters_workspace_bytes(int batch_heads, int n_q);

VSA_API vsa_status vsa_merge_clusters(const int32_t *sizes_q, const int32_t *sizes_k, const int32_t *counts,
                                      const int32_t *idx, const uint8_t *sides, int batch_heads, int n_q,
                                      int n_k, int rounds, int tau_q, int tau_k, void *workspace,
                                      size_t workspace_bytes, int32_t *group_of, int32_t *g_counts,
                                      int32_t *g_idx, void *stream);

/* ---------------------------------------------------------------------------
 * Cluster-aligned blocks: layout and attention ([HVA] section 2 Eq. (1), (4):
 * attention runs on the cluster-permuted tokens and the output is put back in
 * token order; section 4.3: each group of query clusters is one block row,
 * executed in whole CTA tiles, its selected key clusters packed one after the
 * other).
 *
 * Query rows: groups in ascending leader order; a group's rows are its member
 * clusters in ascending order, each cluster's tokens in the order of the query
 * permutation (vsa_cluster_tokens), padded with rows of zeros to a multiple of
 * 128.  Key rows: the key permutation itself (clusters one after the other).
 *
 * vsa_cluster_rows_capacity: rows per head that the query layout can need,
 * 128 * ceil((n_valid + 127 * n_q) / 128) (0 on invalid input).  Host only.
 *
 * vsa_cluster_plan (n_q, n_k <= 1024):
 *   group_of : int32 [BH, n_q]  (vsa_merge_clusters; group_of[i] = i for no merging)
 *   sizes_q  : int32 [BH, n_q];  perm_q : int32 [BH, n_pad]  (vsa_cluster_tokens of Q)
 *   sizes_k  : int32 [BH, n_k]
 *   n_rows   : rows per head of the query layout, a multiple of 128 (the capacity).
 * Outputs:
 *   qmap      int32 [BH, n_rows]      token of each layout row; -1 = padding row of
 *             a group, -2 = row of an unused tile past the last group.
 *   qinv      int32 [BH, n_pad]       layout row of each token; -1 at or past n_valid.
 *   tile_list int32 [BH, n_rows/128]  group (leader) of each 128-row tile, -1 unused.
 *   kc_off    int32 [BH, n_k]         first row of key cluster j in the key
 *             permutation (the exclusive prefix sum of sizes_k).
 * More rows needed than n_rows latches VSA_ERR_CAPACITY; a group_of entry that
 * is not a leader, or a perm_q entry outside [0, n_valid), VSA_ERR_BAD_INDEX.
 *
 * vsa_gather_rows: dst[bh][i] = src[bh][map[bh][i]] for rows of row_bytes (a
 * multiple of 4; 16-byte aligned buffers when a multiple of 16); map -1 writes
 * the 32-bit word `fill` over the row, map -2 leaves the row untouched; any
 * other entry outside [0, n_src) latches VSA_ERR_BAD_INDEX.  src [BH, n_src],
 * dst [BH, n_dst]; the buffers must not overlap.  Used for Q -> query layout
 * (qmap, fill 0) and for the output back to token order (qinv; fill 0 for O,
 * 0xff800000 = -inf for LSE).
 *
 * vsa_cluster_group_fwd: attention of every query layout tile to the keys of
 * its group's key clusters.
 *   q_rows : bf16 [B, H, n_rows, d]  the query layout.
 *   k, v   : bf16 [B, H, n_pad, d]   keys / values in the key permutation.
 *   tile_list, kc_off : from vsa_cluster_plan;  kc_size : sizes_k.
 *   counts, idx : int32 [BH, n_lists], [BH, n_lists, n_kc]: the key clusters of
 *            each group at its leader's row, ascending (vsa_merge_clusters'
 *            g_counts / g_idx, or vsa_select_clusters' lists without merging).
 *   n_kc <= 2048.
 *   o      : [B, H, n_rows, d] bf16 (o_fp32 = 0) or fp32;  lse : fp32 [B, H, n_rows].
 * A key cluster is walked as 16-key segments, the last one partial; keys are
 * rows [kc_off[j], kc_off[j] + kc_size[j]) of K and V.  Rows of unused tiles
 * are not written; padding rows of a group are computed like any other row
 * (zero queries) and are dropped by the gather back to token order.
 * ------------------------------------------------------------------------- */
VSA_API int vsa_cluster_rows_capacity(int n_valid, int n_q);

VSA_API vsa_status vsa_cluster_plan(const int32_t *group_of, const int32_t *sizes_q, const int32_t *perm_q,
                                    const int32_t *sizes_k, int batch_heads, int n_q, int n_k, int n_valid,
                                    int n_pad, int n_rows, int32_t *qmap, int32_t *qinv, int32_t *tile_list,
                                    int32_t *kc_off, void *stream);

VSA_API vsa_status vsa_gather_rows(const void *src, const int32_t *map, int batch_heads, int n_src, int n_dst,
                                   int row_bytes, uint32_t fill, void *dst, void *stream);

VSA_API vsa_status vsa_cluster_group_fwd(const void *q_rows, const void *k, const void *v, const vsa_shape *shape,
                                         int n_rows, const int32_t *tile_list, const int32_t *kc_off,
                                         const int32_t *kc_size, int n_kc, const int32_t *counts,
                                         const int32_t *idx, int n_lists, float scale, void *o, int o_fp32,
                                         float *lse, void *stream);

/* ---------------------------------------------------------------------------
 * Pooled rectification of omitted blocks ([RSA] abstract: sparse attention
 * amplifies the kept keys' weights and drops the omitted keys' weight; both
 * are rectified from pooled query-key interactions).  Readings (the page has
 * no formulas): an omitted key block j of query block i stands for s_j copies
 * of its mean key and mean value, s_j its valid key count; every query row of
 * block i gets s_j exp(scale q.kbar_j) vbar_j in the numerator and
 * s_j exp(scale q.kbar_j) in the denominator of its softmax, which the kept
 * keys share, so their weights are no longer amplified.  Every omitted block
 * with a valid key is rectified.  Used instead of the Micro repair.
 *
 * vsa_pool_kv_bf16: k_bar, v_bar bf16 [B, H, n_rows, d] = the means of the
 * valid rows of each bk-row key block of K and V (fp32 sums, one rounding to
 * bf16); rows past the last key block are zeros.  n_rows is a multiple of 128
 * and at least n_pad / bk.
 *
 * vsa_rectify_fwd: the pooled pass of the query tiles of the given heads:
 *   q       : bf16 [B, H, n_pad, d];  k_bar, v_bar : from vsa_pool_kv_bf16.
 *   counts, idx : the kept lists (vsa_select_blocks layout: bq-row lists,
 *             idx row stride idx_stride); the pass attends to the other blocks.
 *   merge_o, merge_lse : fp32 [B, H, n_pad, d] / [B, H, n_pad] output of the
 *             kept blocks (vsa_block_sparse_fwd with o_fp32 = 1), merged exactly
 *             by LSE into the result (NULL: the pooled terms alone).
 *   o, lse  : the rectified output (bf16 or fp32) and its LSE.
 *   heads, n_heads : as vsa_block_sparse_fwd_heads.
 *   n_pad / bk <= 1024.
 * ------------------------------------------------------------------------- */
VSA_API vsa_status vsa_pool_kv_bf16(const void *k, const void *v, const vsa_shape *shape, int bk, int n_rows,
                                    void *k_bar, void *v_bar, void *stream);

VSA_API vsa_status vsa_rectify_fwd(const void *q, const void *k_bar, const void *v_bar, const vsa_shape *shape,
                                   int bq, int bk, int n_rows, const int32_t *counts, const int32_t *idx,
                                   int idx_stride, float scale, const float *merge_o, const float *merge_lse,
                                   void *o, int o_fp32, float *lse, const int32_t *heads, int n_heads,
                                   void *stream);

#ifdef __cplusplus
}
#endif

#endif /* VSA_H_ */
