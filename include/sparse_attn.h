/*
 * sparse_attn.h -- C ABI of the B200 (sm_100a) selector-driven block-sparse
 * attention library (libsparse_attn.so).
 *
 * The method: every query tile (prefill) or decode query scores each earlier
 * KV block through a landmark (the mean of the block's keys), keeps the top-K
 * blocks plus the sink block 0 and its own (local) block, and attends only to
 * the kept blocks.  Pages followed, cited by title and section:
 *   [SAS]  "Учёные научили трансформеры отбирать контекст напрямую, а не через
 *          имитацию полного внимания" -- opening section and "Ключевые
 *          факты": a light selector scores context units (tokens or blocks),
 *          hard top-K keeps the best; the current block is always kept; the
 *          selector's continuous score enters the attention logits inside the
 *          softmax in log form, normalised against the current block; the
 *          kernel runs FlashAttention-style, blockwise, without the square
 *          matrix.
 *   [HiLS] "HiLS-Attention: иерархическое разреженное внимание для
 *          сверхдлинного контекста в языковых моделях" -- opening section:
 *          each query reads every selected chunk on its own and the per-chunk
 *          results are combined with weights given by the retrieval scores.
 *   [LSA]  Latent Sparse Attention post (rit.work), section "Индекс перестаёт
 *          перебирать весь контекст": adjacent keys are pooled before
 *          scoring; the start of the context and a recent window are always
 *          added; the flat clustered index (sparse_attn_lsa_*) follows its
 *          cluster-centre scan.
 *
 * Groups of entry points: the path (landmarks, selection, prefill, decode),
 * ragged decode batches and landmark refresh, the backward of the gated
 * prefill (sparse_attn_prefill_backward, sparse_attn_select_backward), the
 * flat clustered index (sparse_attn_lsa_*), a decode that allocates nothing
 * (sparse_attn_decode_static), and helpers (workspace sizes, status word,
 * error strings, counters).
 *
 * Conventions for every call
 *   - All tensor pointers are DEVICE pointers, 16-byte aligned, dense
 *     row-major with the layouts given below; the caller owns every buffer.
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL = the legacy default stream).  Host-side argument errors return
 *     before anything is launched.
 *   - Return value: SA_OK (0) or a negative SA_ERR_* code.  No exception and
 *     no allocation crosses the ABI; the library keeps no global state
 *     besides CUDA's own per-device kernel images, a launch counter and the
 *     static scratch array of sparse_attn_decode_static.
 *   - Device-side problems (an index list entry out of range, a NaN score, a
 *     bounded wait that expired, and in the address-checking build a gather
 *     outside its slab) never trap: the kernel skips the bad item and records
 *     a code in the workspace's status word, which sparse_attn_check_status()
 *     returns and clears.
 *   - Layouts.  Q, O: [B, Hq, N, d]; K, V: [B, Hkv, N, d]; landmarks L:
 *     [B, Hkv, nb, d] with nb = ceil(N / block); decode query q and output o:
 *     [B, Hq, d]; LSE: [B, Hq, N] (prefill) or [B, Hq] (decode), fp32.
 *     Query tile j = rows [j*block, (j+1)*block) and aligns with KV block j.
 *     q-head h reads kv-head h / (Hq / Hkv).
 *   - Selection lists, one per unit.  A unit is (batch, kv-head, query tile)
 *     for prefill and (batch, kv-head) for decode -- with
 *     SA_SELECT_PER_QHEAD, (batch, q-head, ...) instead.  Per unit:
 *       idx   int32 [top_k + 2]  kept blocks, ascending, padded with -1
 *       score fp32  [top_k + 2]  retrieval score s_b of each kept block,
 *                                s_b = scale * <pooled query, L_b>, padded 0
 *       count int32              number of kept blocks
 *     so idx/score are [B, Hsel, ntiles, top_k + 2] (prefill) or
 *     [B, Hsel, top_k + 2] (decode), count [B, Hsel, ntiles] or [B, Hsel],
 *     where Hsel = Hkv (Hq with SA_SELECT_PER_QHEAD) and ntiles = nb.
 */
#ifndef SPARSE_ATTN_H
#define SPARSE_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* flags */
enum {
    SA_SINK = 1,              /* block 0 always kept [LSA]                         */
    SA_LOCAL = 2,             /* the unit's own block always kept [SAS]            */
    SA_GATE = 4,              /* log_sigmoid(s_b - s_local) added to the logits of
                                 every selected (not forced) block [SAS]; needs
                                 SA_LOCAL, excludes SA_HIER                        */
    SA_HIER = 8,              /* hierarchical mode [HiLS]: per-block softmax,
                                 outputs combined by softmax_b(s_b); lse returned
                                 = logsumexp_b(s_b)                                */
    SA_CAUSAL = 16,           /* inside the local block key t is visible from
                                 query i only when t <= i                          */
    SA_SELECT_PER_QHEAD = 32  /* one list per q-head instead of per kv-head        */
};

/* dtypes of Q/K/V/L/O */
enum { SA_BF16 = 0, SA_FP32 = 1 };

/* operations, for sparse_attn_workspace_size */
enum {
    SA_OP_LANDMARKS = 0,
    SA_OP_SELECT = 1,         /* prefill selection                                 */
    SA_OP_SELECT_DECODE = 2,
    SA_OP_PREFILL = 3,
    SA_OP_DECODE = 4,
    SA_OP_PREFILL_BACKWARD = 5,
    SA_OP_SELECT_BACKWARD = 6
};

/* return codes */
enum {
    SA_OK = 0,
    SA_ERR_ARG = -1,          /* null pointer, bad shape, misaligned pointer       */
    SA_ERR_UNSUPPORTED = -2,  /* valid but unsupported combination                 */
    SA_ERR_WORKSPACE = -3,    /* workspace missing or smaller than required        */
    SA_ERR_LAUNCH = -4,       /* a CUDA launch failed                              */
    SA_ERR_DEVICE = -5        /* the status word reports a device-side problem     */
};

typedef struct {
    int B;        /* batch (independent sequences)                                 */
    int Hq;       /* query heads                                                   */
    int Hkv;      /* key/value heads; Hq % Hkv == 0                                */
    int d;        /* head dim: 64 or 128 (bf16 prefill fast path: 128)             */
    int N;        /* prefill: sequence length; decode: context length including
                     the query's own key (the query sits at position N - 1)        */
    int block;    /* block size in keys = query tile size: 16..128, multiple of 16 */
    int top_k;    /* budget of selected blocks, 0..256                             */
    int flags;    /* SA_* flags above                                              */
    int dtype;    /* SA_BF16 or SA_FP32                                            */
    float scale;  /* logit scale; 0 selects 1/sqrt(d)                              */
} sa_params;

/* Bytes of workspace `op` needs (at least 256: the first 16 bytes hold the
 * status word).  The workspace must be zero-filled once when allocated; the
 * library leaves the status word zero unless a device-side problem occurs,
 * and returns every completion counter it keeps there to zero by the end of
 * each call.  Calls that share a workspace must not overlap on the GPU.
 * Layout: the status word, then one counter region per operation that keeps
 * counters (prefill selection, decode selection, decode records and merge
 * CTAs, backward key tiles), the per-list publication words of
 * sparse_attn_decode_step (a number per call, never reset), then scratch
 * shared by all operations.  After a call that reported a device-side
 * timeout, zero-fill the workspace again.  The regions are sized from the
 * parameters, so a workspace serves the operations of the parameter set it
 * was sized for (any op, the largest size over the ops used); one sized for
 * another set must not be reused unless it is at least as large for every op
 * with the same geometry (same B, Hq, Hkv, N, block).  */
size_t sparse_attn_workspace_size(const sa_params *p, int op);

/* Landmarks (first step of the path; [HiLS] landmark, [LSA] keys pooled
 * before scoring): L[b,g,k,:] = mean of K[b,g,t,:] over the keys t of block k that
 * exist (t < N), summed in fp32, stored in the KV dtype rounded to nearest
 * even.  K [B,Hkv,N,d] -> L [B,Hkv,nb,d]. */
int sparse_attn_landmarks(const sa_params *p, const void *K, void *L, void *stream);

/* Landmarks of the blocks that changed: for every kv-head of sequence b,
 * recompute blocks first_block[b] .. ceil(seq_len[b] / block) - 1 and leave
 * the others untouched.  After an append that grew sequence b from n0 to n1
 * keys, first_block[b] = n0 / block refreshes exactly the partial block and
 * the new ones (the Latent Sparse Attention post, "Индекс перестаёт
 * перебирать весь контекст": a block's composition is fixed once complete).
 * seq_len (device, [B], may be NULL = N for all) gives each sequence's
 * length; a length outside [1, N] is clamped to it.  first_block (device,
 * [B], may be NULL = 0) gives the first block to refresh.  K and L as in
 * sparse_attn_landmarks (N = the cache capacity). */
int sparse_attn_landmarks_update(const sa_params *p, const void *K, void *L, const int32_t *seq_len,
                                 const int32_t *first_block, void *stream);

/* Prefill selection ([SAS] hard top-K over block scores; [LSA] start of
 * context always added; [SAS] current block always kept).  For tile j of a
 * unit: pooled query = mean of Q over the unit's query heads and the tile's
 * rows; s_b = scale * <pooled, L_b> for b <= j; candidates = blocks before j
 * (block 0 excluded with SA_SINK); the top_k candidates by (s desc, index
 * asc, decided on fp32 scores) are kept together with block 0 (SA_SINK) and
 * block j (SA_LOCAL).  Q [B,Hq,N,d], L [B,Hkv,nb,d] -> idx, score, count.
 * A NaN score is ranked lowest and flagged in the status word. */
int sparse_attn_select(const sa_params *p, const void *Q, const void *L, int32_t *idx, float *score,
                       int32_t *count, void *ws, size_t ws_bytes, void *stream);

/* Decode selection: as sparse_attn_select for the one query per sequence at
 * position N-1; its local block is (N-1)/block.  q [B,Hq,d] -> idx, score,
 * count of shape [B,Hsel,top_k+2] / [B,Hsel]. */
int sparse_attn_select_decode(const sa_params *p, const void *q, const void *L, int32_t *idx, float *score,
                              int32_t *count, void *ws, size_t ws_bytes, void *stream);

/* Decode selection for a ragged batch: sequence b holds seq_len[b] keys
 * (device, [B], clamped to [1, N]; N = the cache capacity of K/V/L) and its
 * query sits at position seq_len[b] - 1, so its local block is
 * (seq_len[b] - 1) / block.  L must hold each sequence's landmarks over its
 * own length (sparse_attn_landmarks_update with the same seq_len).
 * Otherwise as sparse_attn_select_decode; seq_len NULL returns SA_ERR_ARG. */
int sparse_attn_select_decode_varlen(const sa_params *p, const void *q, const void *L, const int32_t *seq_len,
                                     int32_t *idx, float *score, int32_t *count, void *ws, size_t ws_bytes,
                                     void *stream);

/* Block-sparse prefill over the kept lists ([SAS] FlashAttention-style,
 * blockwise, online softmax).  Gated mode: z_t = scale * <q_i, k_t> + gate_b
 * for keys t of kept blocks (t <= i inside the local block when causal),
 * gate_b = log_sigmoid(s_b - s_local) on selected blocks (SA_GATE), 0 on the
 * sink and local blocks; O_i = softmax(z) V, LSE_i = log sum exp z.
 * Hierarchical mode (SA_HIER): per-block softmax outputs combined with
 * weights softmax_b(s_b).  An empty list gives O = 0, LSE = -inf.
 * Q,K,V + idx/score/count (as written by sparse_attn_select) -> O, LSE. */
int sparse_attn_prefill(const sa_params *p, const void *Q, const void *K, const void *V, const int32_t *idx,
                        const float *score, const int32_t *count, void *O, float *lse, void *ws,
                        size_t ws_bytes, void *stream);

/* Which kernel sparse_attn_prefill runs for these parameters:
 *   2 = the persistent tensor-core kernel (tcgen05/TMEM/TMA, one CTA per SM,
 *       256 query rows per work unit; bf16, d = 128, block 64 or 128, query
 *       heads per kv-head a multiple of 256/block; gated, plain or
 *       hierarchical),
 *   1 = the two-CTA-per-SM tensor-core kernel (same types, query heads per
 *       kv-head a multiple of 128/block; also hierarchical mode at block 64),
 *   0 = the CUDA-core kernel (every other supported shape, fp32, per-q-head
 *       lists),
 *   negative = invalid parameters.
 * The environment variable SPARSE_ATTN_PREFILL_PATH=tc1 rules out 2, and
 * SPARSE_ATTN_PREFILL_PATH=simt forces 0. */
int sparse_attn_prefill_kernel(const sa_params *p);

/* Block-sparse decode: the same attention for one query per sequence at
 * position N-1 over the cache K, V [B,Hkv,N,d] (it already holds the query's
 * own key/value); split over the kept blocks, partials merged by
 * log-sum-exp.  q [B,Hq,d] + decode lists -> o [B,Hq,d], lse [B,Hq].
 * bf16, d = 128, block 64 runs the tensor-core (mma.sync) gather kernel;
 * every other shape the CUDA-core kernel.  The environment variable
 * SPARSE_ATTN_DECODE_PATH=simt forces the CUDA-core kernel (a cross-check
 * hook: both kernels compute the same result). */
int sparse_attn_decode(const sa_params *p, const void *q, const void *K, const void *V, const int32_t *idx,
                       const float *score, const int32_t *count, void *o, float *lse, void *ws,
                       size_t ws_bytes, void *stream);

/* Decode without a caller workspace, for callers that cannot allocate device
 * memory (custom-allocator callbacks, servers whose memory pool owns every
 * device byte, plugins handed only the tensors of one call).  The pages
 * describe no counterpart: this is a deployment convenience.  Same arguments
 * and results as sparse_attn_decode minus `ws`/`ws_bytes`; the scratch is an
 * 2 MiB array inside the library (held on every GPU that loads it until
 * exit).  The first call on each device looks up that array's address -- make
 * it before any stream capture.  All calls on a device share the array, so
 * calls that overlap on the GPU race: keep them on one stream.  Problems
 * whose split partials exceed the array return SA_ERR_WORKSPACE before any
 * launch.  Never calls cudaMalloc or cudaFree.  Device-side list problems are
 * skipped as in sparse_attn_decode but not reported. */
int sparse_attn_decode_static(const sa_params *p, const void *q, const void *K, const void *V,
                              const int32_t *idx, const float *score, const int32_t *count, void *o, float *lse,
                              void *stream);

/* Block-sparse decode for a ragged batch: as sparse_attn_decode with
 * sequence b reading only its first seq_len[b] cached keys (clamped to
 * [1, N]), its query at position seq_len[b] - 1; lists from
 * sparse_attn_select_decode_varlen.  Uses the workspace size of
 * SA_OP_DECODE; seq_len NULL returns SA_ERR_ARG. */
int sparse_attn_decode_varlen(const sa_params *p, const void *q, const void *K, const void *V, const int32_t *seq_len,
                              const int32_t *idx, const float *score, const int32_t *count, void *o, float *lse,
                              void *ws, size_t ws_bytes, void *stream);

/* One decode step: sparse_attn_select_decode (or its _varlen form when
 * seq_len is not NULL) followed by sparse_attn_decode on the lists it
 * writes into idx/score/count, with the same results as those two calls.
 * When both run their tensor-core / bulk-copy kernels (bf16, d = 128, block
 * 64, no SPARSE_ATTN_*_PATH override) the two launches overlap: the
 * selection publishes each (batch, selection head)'s list as soon as it is
 * final (a per-call number stored into the workspace), and the decode's
 * work for that list starts then instead of after the whole selection, so
 * the cache gather of early lists overlaps the end of the selection.  Uses
 * a workspace at least as large as both SA_OP_SELECT_DECODE and
 * SA_OP_DECODE need. */
int sparse_attn_decode_step(const sa_params *p, const void *q, const void *L, const void *K, const void *V,
                            const int32_t *seq_len, int32_t *idx, float *score, int32_t *count, void *o,
                            float *lse, void *ws, size_t ws_bytes, void *stream);

/* Backward of the gated (or plain) block-sparse prefill -- [SAS] "Как это
 * применить": the selector's score enters the softmax as the gate
 * g_c = log_sigmoid(s_c - s_local), which is how the loss reaches the
 * selector; the top-K choice itself is hard ("Ключевые факты") and the kept
 * lists of the forward pass are reused as they are.
 * Inputs: Q [B,Hq,N,d], K, V [B,Hkv,N,d] (dtype of p), the forward's O
 * [B,Hq,N,d] and LSE [B,Hq,N] (fp32, natural log), the upstream gradient dO
 * [B,Hq,N,d] (dtype of p) and the lists idx/score/count of
 * sparse_attn_select.  Outputs, all fp32 and overwritten:
 *   dQ [B,Hq,N,d]  = scale dZ K over the kept keys of each row,
 *   dK, dV [B,Hkv,N,d] = scale dZ^T Q and P^T dO summed over every row that
 *                  keeps the key (accumulated with atomics, so the last bits
 *                  may vary between runs),
 *   dscore [B,Hkv,nb,cap]: gradient with respect to each list entry's score:
 *                  dg_c sigmoid(-(s_c - s_local)) for gated entries, minus
 *                  their sum for the local block's entry, 0 otherwise,
 * with P = exp(z - LSE), dZ = P (dO V^T - rowsum(dO O)) and dg_c the sum of
 * dZ over entry c's keys.  Workspace: SA_OP_PREFILL_BACKWARD.  Gated or plain
 * mode with per-kv-head lists, d = 64 or 128; SA_HIER or
 * SA_SELECT_PER_QHEAD give SA_ERR_UNSUPPORTED.  CUDA cores, fp32. */
int sparse_attn_prefill_backward(const sa_params *p, const void *Q, const void *K, const void *V, const void *O,
                                 const float *lse, const void *dO, const int32_t *idx, const float *score,
                                 const int32_t *count, float *dQ, float *dK, float *dV, float *dscore, void *ws,
                                 size_t ws_bytes, void *stream);

/* The selector's part of the backward: the scores s_c = scale <qbar, L_c>
 * ([SAS] "Ключевые факты": a light selector scores the blocks) carry dscore
 * back to the pooled query qbar (mean of the unit's G heads x block rows of
 * Q) and to the landmarks L (means of the blocks' keys, landmark rounding
 * taken as the identity):  dQ[rows of the unit] += scale sum_c dscore_c L_c / R
 * and dK[keys of block b] += scale sum over entries c with block b of
 * dscore_c qbar / n_b.  Adds into the dQ and dK of
 * sparse_attn_prefill_backward (fp32).  Q, L as given to sparse_attn_select.
 * Workspace: SA_OP_SELECT_BACKWARD.  Same support as above. */
int sparse_attn_select_backward(const sa_params *p, const void *Q, const void *L, const int32_t *idx,
                                const float *dscore, const int32_t *count, float *dQ, float *dK, void *ws,
                                size_t ws_bytes, void *stream);

/* ---- Flat clustered index (the Latent Sparse Attention post, section
 * "Индекс перестаёт перебирать весь контекст") -----------------------------
 * Keys are pooled into items (means of `pool` adjacent keys); every complete
 * segment of `seg` items (all seg * pool keys present) is clustered by Ward's
 * method into `clusters` clusters, frozen from then on; the index keeps each
 * cluster's centre and its items.  A decode query (the mean of its kv-group's
 * query heads) is scored against every centre, scale * <q, centre>; the best
 * `top_clusters`, by (score desc, cluster id asc), are expanded back to their
 * key positions; the first `sink` and the last `window` positions are always
 * added; each query head attends (plain softmax) to that set.  The clustering
 * runs in the raw key space: the post's learned projections are not modelled.
 * Clusters of a segment are numbered by their first item; cluster c of
 * segment g has global id g * clusters + c. */
typedef struct {
    int B, Hq, Hkv;     /* batch, query heads, key/value heads (Hq % Hkv == 0)       */
    int d;              /* head dim: 64 or 128                                         */
    int N;              /* context length (the query sits at N - 1), 1 .. 2^20         */
    int pool;           /* keys per item, >= 1                                         */
    int seg;            /* items per segment, 2 .. 64                                  */
    int clusters;       /* clusters per segment, 1 .. seg                              */
    int top_clusters;   /* clusters a query expands, 0 .. 4096                         */
    int sink, window;   /* always-kept first / last positions, >= 0                    */
    int dtype;          /* SA_BF16 or SA_FP32 for q, K, V and o                        */
    float scale;        /* score and logit scale; 0 -> 1/sqrt(d)                       */
} sa_lsa_params;

/* Clusters per (batch, kv-head): (N / (pool * seg)) * clusters, or a negative
 * SA_ERR_* code for invalid / unsupported parameters. */
int sparse_attn_lsa_clusters(const sa_lsa_params *p);

/* Workspace bytes for sparse_attn_lsa_decode, 0 when the parameters are
 * invalid or unsupported.  Holds the status word, the chunks' candidate
 * clusters, the list of kept key positions, the split attention partials and
 * two completion counters; zero-fill it once when allocated (the counters are
 * returned to zero by every call).  Calls sharing a workspace must not
 * overlap on the GPU. */
size_t sparse_attn_lsa_workspace_size(const sa_lsa_params *p);

/* Builds the index of every (batch, kv-head) from K [B,Hkv,N,d]:
 * centres [B,Hkv,C,d] (fp64: the clustering's own precision), members
 * [B,Hkv,C,seg] (item ids of each cluster, ascending, -1 padded), sizes
 * [B,Hkv,C]; C = sparse_attn_lsa_clusters(p).  Caller-owned buffers. */
int sparse_attn_lsa_build(const sa_lsa_params *p, const void *K, double *centres, int32_t *members, int32_t *sizes,
                          void *stream);

/* Decode through the index: q [B,Hq,d], K, V [B,Hkv,N,d] and the index of
 * sparse_attn_lsa_build -> o [B,Hq,d] (dtype of p), lse [B,Hq] (fp32, natural
 * log; -inf when nothing is kept), and, when `kept` is not NULL, the number
 * of key positions each (batch, kv-head) attended to (int32 [B,Hkv]).
 * Two kernels: centre scores (fp64) in chunks over many CTAs with an exact
 * top_clusters merge (a block-wide radix select), expanded to the list of
 * kept key positions; then the kept keys split over many CTAs with a
 * log-sum-exp merge.  The merge of the chunks' candidates
 * runs in one CTA: parameters with top_clusters x ceil(C / 8192) > 12288
 * (C = clusters per (batch, kv-head)) return SA_ERR_UNSUPPORTED.  A member
 * entry outside the complete segments sets status bit 1 and is skipped; a
 * NaN centre score sets bit 2 and ranks below every number. */
int sparse_attn_lsa_decode(const sa_lsa_params *p, const void *q, const void *K, const void *V,
                           const double *centres, const int32_t *members, const int32_t *sizes, void *o, float *lse,
                           int32_t *kept, void *ws, size_t ws_bytes, void *stream);

/* ---- Tree over the flat index's clusters (same section of the post: the
 * clusters are grouped into a hierarchy that a query walks with a beam
 * search, keeping a few good branches per level, so that it is compared
 * against far fewer centres than in a flat scan) -------------------------
 * Construction (the post gives none; this is the reading the library takes):
 * the flat clusters are the leaves (level 0); every level above is a Ward
 * clustering of the level below into ceil(n / fanout) nodes, each node
 * weighted by the key positions it holds, numbered by their first child;
 * a node's centre is the mass-weighted mean of its children's centres;
 * levels are added while a level holds more than `fanout` nodes.  Search:
 * the pooled query is scored against every node of the top level, the
 * `beam` best of a level by (score desc, id asc) are expanded into their
 * children, and at the leaves the `top_clusters` best are kept; they are
 * expanded to key positions, with the sink and window, as in the flat
 * decode.  Supports 2 <= fanout <= 64 and 1 .. 4096 clusters per (batch,
 * kv-head); anything else returns SA_ERR_UNSUPPORTED (fanout < 2:
 * SA_ERR_ARG). */

/* Bytes of the caller-owned tree buffer (0 when invalid or unsupported);
 * *levels (may be NULL) receives the number of levels, leaves included.
 * Layout, per level l >= 1 and (batch, kv-head): centres [n_l][d] fp64,
 * masses [n_l] fp64, first-child offsets [n_l + 1] int32, children
 * [n_(l-1)] int32 (ascending within each parent); level 0: masses only. */
size_t sparse_attn_lsa_tree_size(const sa_lsa_params *p, int fanout, int *levels);

/* Workspace bytes for sparse_attn_lsa_tree_build and _tree_decode (one
 * buffer serves both; zero-fill it once when allocated). */
size_t sparse_attn_lsa_tree_workspace_size(const sa_lsa_params *p, int fanout);

/* Builds the tree of every (batch, kv-head) from the flat index's centres
 * and sizes (sparse_attn_lsa_build) into `tree`.  One CTA per (batch,
 * kv-head) runs Ward's merges level by level in fp64. */
int sparse_attn_lsa_tree_build(const sa_lsa_params *p, int fanout, const double *centres, const int32_t *sizes,
                               void *tree, void *ws, size_t ws_bytes, void *stream);

/* Decode through the tree: beam search (beam >= 1) down to the leaves, the
 * `top_clusters` best leaves expanded to key positions with the sink and
 * window, then attention as in sparse_attn_lsa_decode.  Outputs o, lse and,
 * when not NULL, kept [B,Hkv] (key positions attended) and compared [B,Hkv]
 * (centres scored on the way down). */
int sparse_attn_lsa_tree_decode(const sa_lsa_params *p, int fanout, int beam, const void *q, const void *K,
                                const void *V, const double *centres, const int32_t *members, const int32_t *sizes,
                                const void *tree, void *o, float *lse, int32_t *kept, int32_t *compared, void *ws,
                                size_t ws_bytes, void *stream);

/* Synchronises `stream`, returns SA_OK or SA_ERR_DEVICE from the status
 * word in `ws`, and clears it.  *detail (may be NULL) receives the raw bits:
 * 1 index list entry out of range, 2 NaN score, 4 bounded wait expired, 8 a
 * gather whose first row lies outside the slab it means to read (only in the
 * address-checking build, libsparse_attn_bounds.so, compiled with
 * -DSA_DEBUG_BOUNDS; the release build makes no such check). */
int sparse_attn_check_status(void *ws, void *stream, int *detail);

/* Static string for a return code. */
const char *sparse_attn_status_string(int code);

/* Library version: major * 10000 + minor * 100 + patch. */
int sparse_attn_version(void);

/* The cudaError_t behind the last SA_ERR_LAUNCH returned on the calling host
 * thread (0 if none), and CUDA's text for such a code. */
int sparse_attn_last_cuda_error(void);
const char *sparse_attn_cuda_error_string(int err);

/* Number of CUDA kernels this library has launched in this process so far
 * (a reporting counter; the only process-wide state the library keeps). */
unsigned long long sparse_attn_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* SPARSE_ATTN_H */
