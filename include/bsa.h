/*
 * bsa.h — C ABI of libbsa: input-adaptive 3D block-sparse self-attention for
 * video diffusion transformers on NVIDIA B200 (sm_100a).
 *
 * The operation is the head-wise sparse attention executor of
 *   SPADE: An Input-Adaptive Sparse Attention Engine for Fast Video Diffusion
 *   Models Inference (arXiv 2608.03335), §3.3 "Head-wise Sparse Attention":
 *   Q, K, V are rearranged into a blocked layout by a 3D blocking scheme, one
 *   mean summary (centroid) is formed per Q/K block, an inter-block importance
 *   matrix is computed from the summaries and filtered by Top-K or Top-P, a
 *   flash block-sparse attention kernel computes softmax(QK^T/sqrt(d) + M)V
 *   (§2.2, Eq. (2)) over the selected block pairs, and the output blocks are
 *   restored to the original token order.
 * Block shapes follow the DecoupAttn Plans README ("Contents" table: block
 * shape = frames x rows x cols of one key block). Density follows the blog
 * "Does sparse attention actually speed up video generation?" ("How this was
 * measured": the fraction of key blocks each query block keeps).
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Every tensor pointer is DEVICE memory owned by the caller, contiguous,
 *    16-byte aligned, on the current CUDA device.  `stream` is a cudaStream_t
 *    (NULL = legacy default stream).  Calls are asynchronous on that stream:
 *    host-side validation happens first, and a call that returns anything but
 *    BSA_OK has launched nothing and written nothing.
 *  - Element type of Q/K/V/O and of the blocked tensors is the plan's dtype
 *    (BSA_F32: float, BSA_BF16: __nv_bfloat16).  Centroids and scores are
 *    float.  Index lists are int32.
 *  - Token layout ("original order") of Q/K/V/O: [B, Ntot, Hd, D] with
 *    Ntot = T*H*W + n_text.  Video token (t, y, x) sits at n = (t*H + y)*W + x
 *    (frame-major raster, the DiT flattening of SPADE §2.1); text token u sits
 *    at n = T*H*W + u.
 *  - Blocked layout: [B, Hd, Npad_tot, D], Npad_tot = (nb + nb_text) * bs.
 *    The grid is padded at the high end of each axis to Tp = ceil(T/bf)*bf
 *    (likewise Hp, Wp).  Video block (tb, yb, xb) has id
 *    (tb*nby + yb)*nbx + xb; inside a block, slot (dt, dy, dx) is
 *    (dt*br + dy)*bc + dx.  Text tokens fill nb_text = ceil(n_text/bs)
 *    trailing blocks (ids nb .. nb+nb_text-1) in order.  Pad slots hold 0,
 *    are never attended as keys, and produce output 0 as queries.
 *  - Text key blocks are attended by every query; text query blocks attend
 *    every key block (dense rows).  Text blocks take no part in scoring.
 *  - Errors: every call returns a bsa_status; bsa_last_error_string() gives a
 *    thread-local message for the last failure.
 *  - bsa_forward makes no synchronous CUDA call and allocates nothing (the
 *    caller passes the workspace), so it can be captured in a CUDA graph;
 *    its per-head parameters are read on the host at the call (at capture)
 *    and travel in the kernel arguments.  bsa_check_status synchronises.
 */
#ifndef BSA_H_
#define BSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define BSA_VERSION 100

typedef enum {
  BSA_OK = 0,
  BSA_ERR_INVALID_ARG = 1, /* bad shape, pointer, parameter or list width   */
  BSA_ERR_UNSUPPORTED = 2, /* valid request the library does not serve      */
  BSA_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed              */
  BSA_ERR_TIMEOUT = 4,     /* a bounded in-kernel wait ran out (dev_status)  */
  BSA_ERR_WORKSPACE = 5,   /* workspace missing or smaller than required     */
  BSA_ERR_BAD_INDEX = 6    /* an index list entry was out of range (skipped) */
} bsa_status;

typedef enum { BSA_F32 = 0, BSA_BF16 = 1 } bsa_dtype;

/* Selection rule of the inter-block estimator (SPADE §3.1 "Top-K/Top-P
 * mode", §3.3 "Scores are filtered by Top-K or Top-P").
 *  BSA_TOPK: per head h, keep k_h = ceil(rho_h * nb - 1e-9) (clamped to
 *            [1, nb]) video key blocks with the largest centroid scores;
 *            param = rho_h, the density in (0, 1].
 *  BSA_TOPP: per head h, keep the shortest prefix, in descending score
 *            order, whose softmax mass reaches tau_h; param = tau_h in (0, 1].
 * Equal scores are ordered by ascending key-block index. */
typedef enum { BSA_TOPK = 0, BSA_TOPP = 1 } bsa_select_mode;

typedef struct bsa_plan_s* bsa_plan_t;

/* Derived sizes of a plan (all counts per batch element and head). */
typedef struct {
  int batch, T, H, W, bf, br, bc, heads, head_dim, n_text;
  int dtype;            /* bsa_dtype                                        */
  int Tp, Hp, Wp;       /* padded grid                                      */
  int nbt, nby, nbx;    /* blocks per axis                                  */
  int nb;               /* video blocks = nbt*nby*nbx                       */
  int nb_text;          /* text blocks = ceil(n_text / bs)                  */
  int bs;               /* tokens per block = bf*br*bc                      */
  long long n_video;    /* T*H*W                                            */
  long long n_tot;      /* n_video + n_text (rows of the original layout)   */
  long long npad_tot;   /* (nb + nb_text) * bs (rows of the blocked layout) */
  int attn_path;        /* 1 = tcgen05 tensor-core path, 0 = fp32 SIMT path */
} bsa_plan_info_t;

/* bsa_plan_create — describe one attention problem (SPADE §3 "Let the head
 * dimension be d_head ... BS the block size and NB the number of blocks";
 * §3.1 blocking schemes, Fig. 3).
 *   batch >= 1; T, H, W >= 1 (latent frames, rows, cols); bf, br, bc >= 1
 *   (block extent per axis, at most the padded grid); heads >= 1;
 *   head_dim in {64, 128}; n_text >= 0 trailing text tokens; dtype.
 *   Block size bs = bf*br*bc must be in [1, 256].  The tensor-core path
 *   serves dtype BSA_BF16 with bs == 128; every other valid plan runs the
 *   fp32 SIMT path (exact fp32 arithmetic, slower).
 * Ownership: the plan is library-owned and immutable; it holds a few bytes of
 * device memory on the device current at creation (status word).  Destroy it
 * with bsa_plan_destroy on the same device. */
bsa_status bsa_plan_create(bsa_plan_t* out, int batch, int T, int H, int W,
                           int bf, int br, int bc, int heads, int head_dim,
                           int n_text, bsa_dtype dtype);
bsa_status bsa_plan_destroy(bsa_plan_t plan);
bsa_status bsa_plan_get_info(bsa_plan_t plan, bsa_plan_info_t* info);

/* bsa_kmax_for — the index-list width that every selection under `mode` and
 * the host array param_per_head[heads] fits in: max_h k_h + nb_text for
 * BSA_TOPK, nb + nb_text for BSA_TOPP.  Validates the parameters. */
bsa_status bsa_kmax_for(bsa_plan_t plan, bsa_select_mode mode,
                        const double* param_per_head, int* kmax);

/* bsa_workspace_size — bytes of device workspace that bsa_select and
 * bsa_forward need for list width kmax. */
bsa_status bsa_workspace_size(bsa_plan_t plan, int kmax, size_t* select_ws,
                              size_t* forward_ws);

/* bsa_permute — layout transform into the blocked layout (SPADE §3.3,
 * "rearranged into a blocked layout by the Selected Blocking Scheme"),
 * optionally fused with the mean summarizer (§3.3 "Operator fusion";
 * MEAN-SPADE, §3.1 (q_mean, k_mean)).
 *   x         [B, Ntot, Hd, D]      input in original order (read only)
 *   x_blk     [B, Hd, Npad_tot, D]  output, pad slots written as 0
 *   centroids [B, Hd, nb, D] float  optional (NULL = skip): per video block,
 *             the mean over its valid tokens, summed in fp32.
 * bsa_permute_qkv does Q, K and V in one launch (centroids for Q and K). */
bsa_status bsa_permute(bsa_plan_t plan, const void* x, void* x_blk,
                       float* centroids, void* stream);
bsa_status bsa_permute_qkv(bsa_plan_t plan, const void* q, const void* k,
                           const void* v, void* q_blk, void* k_blk,
                           void* v_blk, float* q_cent, float* k_cent,
                           void* stream);

/* bsa_centroids — the mean summarizer straight from the original layout
 * (SPADE §3.1 MEAN-SPADE (q_mean, k_mean); §3.3 summaries Q', K'), without
 * materialising the blocked tensors: the same values bsa_permute writes.
 *   q, k            [B, Ntot, Hd, D] original order (read only)
 *   q_cent, k_cent  [B, Hd, nb, D] float out (either may be NULL). */
bsa_status bsa_centroids(bsa_plan_t plan, const void* q, const void* k,
                         float* q_cent, float* k_cent, void* stream);

/* bsa_sics — the intra-block estimator of SPADE §3.2, Eq. (4): for every
 * video block of the plan's blocking scheme, the sum over all ordered pairs
 * (a, b) of the block's valid rows (diagonal included) of the cosine
 * similarity x_a . x_b / (|x_a| |x_b|).  It equals |sum_a x_a/|x_a| |^2 and
 * lies in [0, n^2] for a block of n valid rows; a zero row has no direction
 * and contributes nothing.  Computed in fp32 (rows widened exactly from the
 * plan dtype).  Text tokens belong to no 3D block and take no part.
 *   x     [B, Ntot, Hd, D] original order (read only)
 *   sics  [B, Hd, nb] float out */
bsa_status bsa_sics(bsa_plan_t plan, const void* x, float* sics, void* stream);

/* bsa_aggregation_scores — aggregation evaluation and blocking-scheme choice
 * (SPADE §3.2): for each candidate plan c (a blocking scheme), the SICS of
 * every video block, the Aggregation Score AS(x | c) = sum of SICS over the
 * video blocks (Eq. (3)), and per (b, h) the candidate with the largest AS
 * (the Selected Blocking Scheme; the lowest c among equal scores).
 *   plans   host array of n_plans (1..8) plans on the current device that
 *           agree in batch, T, H, W, heads, head_dim, n_text and dtype
 *   x       [B, Ntot, Hd, D] original order (read only)
 *   sics    host array of n_plans device pointers, sics[c] = [B, Hd, nb_c]
 *           float out (required: it also carries AS's terms)
 *   as      [n_plans, B, Hd] double out, optional (NULL = skip); the fp32
 *           SICS values summed in double in a fixed order
 *   choice  [B, Hd] int32 out, optional (NULL = skip)
 * One launch evaluates all candidates, with the candidates of a head
 * scheduled together so that the head's rows are read from HBM once. */
bsa_status bsa_aggregation_scores(const bsa_plan_t* plans, int n_plans,
                                  const void* x, float* const* sics,
                                  double* as, int32_t* choice, void* stream);

/* bsa_unpermute — restore blocked output to the original token order (SPADE
 * §3.3, "output blocks are restored to the original layout"); pad slots are
 * dropped.   o_blk [B, Hd, Npad_tot, D] -> o [B, Ntot, Hd, D]. */
bsa_status bsa_unpermute(bsa_plan_t plan, const void* o_blk, void* o,
                         void* stream);

/* bsa_select — index search (SPADE §3.3: summaries Q', K' of shape
 * (N_blocks, d_head); inter-block importance N_Qb x N_Kb; Top-K / Top-P).
 *   q_blk, k_blk  blocked Q and K (plan dtype)
 *   mode, param_per_head  host array [Hd] of densities or thresholds
 *   kmax          list width (>= bsa_kmax_for result)
 *   idx  [B, Hd, nb, kmax] int32 out: per video query block, the selected
 *        video key blocks in ascending id, then the nb_text text key blocks;
 *        entries past cnt are left untouched
 *   cnt  [B, Hd, nb] int32 out: list length (selected video blocks + nb_text)
 *   scores [B, Hd, nb, nb] float out, optional (NULL = skip): the row-softmax
 *        p_ij = softmax_j(qbar_i . kbar_j / sqrt(D)) computed in fp32
 *   ws, ws_bytes  device workspace of at least select_ws bytes (centroids)
 * Text query blocks have no list: they attend densely. */
bsa_status bsa_select(bsa_plan_t plan, const void* q_blk, const void* k_blk,
                      bsa_select_mode mode, const double* param_per_head,
                      int kmax, int32_t* idx, int32_t* cnt, float* scores,
                      void* ws, size_t ws_bytes, void* stream);

/* bsa_select_centroids — bsa_select from precomputed fp32 centroids
 * [B, Hd, nb, D] (as written by bsa_permute); needs no workspace. */
bsa_status bsa_select_centroids(bsa_plan_t plan, const float* q_cent,
                                const float* k_cent, bsa_select_mode mode,
                                const double* param_per_head, int kmax,
                                int32_t* idx, int32_t* cnt, float* scores,
                                void* stream);

/* bsa_select_static — bsa_select for callers that cannot allocate device
 * memory.  The paper has no counterpart to this call; it exists for engines
 * and plugin hosts that plan all device memory before serving and forbid
 * allocation afterwards, and for hot loops that must not pay cudaMalloc's
 * implicit synchronisation.  It takes no workspace and calls no allocator:
 * the Q and K centroids live in a fixed 16 MiB device array inside libbsa,
 * which every GPU that loads the library holds until the process exits.
 *   Arguments, outputs and results are those of bsa_select.
 *   Limit: 2 * batch * heads * nb * head_dim * 4 bytes (each half rounded up
 *   to 256 bytes) must fit in 16 MiB, else BSA_ERR_UNSUPPORTED and nothing is
 *   launched.
 *   The first call on a device looks up that device's copy of the array
 *   (cudaGetSymbolAddress, with the device current) and caches it with the
 *   id of the current context (a call in another context, e.g. after a
 *   device reset, looks it up again); make that first call before any stream
 *   capture begins.
 *   All calls on a device share the array and it keeps the last call's
 *   contents (each call rewrites every centroid it reads, so nothing needs
 *   clearing); calls whose kernels overlap on the GPU race on it. */
bsa_status bsa_select_static(bsa_plan_t plan, const void* q_blk, const void* k_blk,
                             bsa_select_mode mode, const double* param_per_head,
                             int kmax, int32_t* idx, int32_t* cnt, float* scores,
                             void* stream);

/* bsa_attention — flash block-sparse attention (SPADE §2.2 Eq. (2) with M = 0
 * on selected block pairs and valid keys, -inf elsewhere; §3.3 (3): online
 * softmax, no dense score matrix).
 *   q_blk, k_blk, v_blk  blocked inputs;  o_blk  blocked output (pad rows 0)
 *   idx, cnt, kmax       lists as written by bsa_select (any ascending list
 *                        of distinct ids in [0, nb+nb_text) is accepted)
 *   dev_status           optional int32 device word (NULL = plan-owned):
 *                        0 on success, BSA_ERR_TIMEOUT if a bounded wait ran
 *                        out, BSA_ERR_BAD_INDEX if a list entry was out of
 *                        range (that entry is skipped).  The caller reads it
 *                        after synchronising; bsa_check_status does that for
 *                        the plan-owned word.
 * Output rows are softmax-weighted sums accumulated in fp32 and rounded to
 * the plan dtype (round to nearest even). */
bsa_status bsa_attention(bsa_plan_t plan, const void* q_blk, const void* k_blk,
                         const void* v_blk, const int32_t* idx,
                         const int32_t* cnt, int kmax, void* o_blk,
                         int32_t* dev_status, void* stream);

/* bsa_attention_orig — bsa_attention on the ORIGINAL layout: the layout
 * transform is fused into the tile loads (a 5D TMA box (d, head, x, y, t) per
 * block, out-of-grid elements read as 0; a 3D box for text blocks) and its
 * inverse into the epilogue (each real slot's row is written to its token).
 * SPADE §3.3 "(1) Operator fusion ... (2) fuse Q/K gather-scatter with the
 * layout transform".
 *   q, k, v   [B, Ntot, Hd, D] original order;  o  [B, Ntot, Hd, D] out
 *   idx, cnt, kmax, dev_status  as for bsa_attention
 * Tensor-core plans only (bf16, 128-token blocks): other plans get
 * BSA_ERR_UNSUPPORTED. */
bsa_status bsa_attention_orig(bsa_plan_t plan, const void* q, const void* k,
                              const void* v, const int32_t* idx,
                              const int32_t* cnt, int kmax, void* o,
                              int32_t* dev_status, void* stream);

/* bsa_forward — the whole executor on one stream (SPADE §3.3, Fig. 2(c)).
 * Tensor-core plans: bsa_centroids -> selection -> bsa_attention_orig (the
 * layout transform and its inverse are fused into the attention's loads and
 * stores).  Other plans: permute (+centroids) -> selection -> attention ->
 * unpermute through blocked workspace tensors.
 *   q, k, v, o        original-order tensors [B, Ntot, Hd, D]
 *   idx_out, cnt_out  optional copies of the lists (NULL = keep internal)
 *   kmax              list width (>= bsa_kmax_for result)
 *   ws, ws_bytes      device workspace of at least forward_ws bytes */
bsa_status bsa_forward(bsa_plan_t plan, const void* q, const void* k,
                       const void* v, bsa_select_mode mode,
                       const double* param_per_head, int kmax, void* o,
                       int32_t* idx_out, int32_t* cnt_out, void* ws,
                       size_t ws_bytes, int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------
 * Mask union (SPADE §3.3: "intra scores are broadcast and OR-combined with
 * inter scores.  The result is united with local-window and attention-sink
 * masks to form a binary attention mask"; §3.2: each head's sparsity-ratio
 * scheme has a local-window length, an intra-top value and an inter-top
 * value; §3.1: attention-sink length).  Every entry is a whole video key
 * block added to the lists of a head, so the attention kernels are unchanged.
 * For video query block i of head h the list is the ascending union of
 *   inter   the Top-K / Top-P selection of bsa_select;
 *   window  key blocks j with i - window_left <= j <= i + window_right, a
 *           sliding window over the block sequence in block units, like the
 *           (left, right) window_size of LongLive's attention ("How to
 *           Configure Local Attention Size for Long Video Generation in
 *           LongLive"); a negative side is unbounded, and window_left < 0
 *           together with window_right < 0 adds nothing;
 *   sink    the key blocks that hold any of the first sink_tokens tokens of
 *           the original order (0 = none);
 *   intra   when intra_param is not NULL and intra_param[h] > 0: the key
 *           blocks the intra_mode rule selects from one intra score per key
 *           block, broadcast to every query block of the head.  Top-K keeps
 *           ceil(intra_param[h] * nb - 1e-9) blocks with the largest scores;
 *           Top-P keeps the shortest descending prefix whose score sum
 *           reaches intra_param[h] * (sum of the head's scores).  Equal
 *           scores are ordered by ascending block id;
 * followed by the nb_text text key blocks.  Text query blocks stay dense. */
typedef struct {
  int window_left;               /* blocks before i; < 0 = unbounded         */
  int window_right;              /* blocks after i;  < 0 = unbounded         */
  long long sink_tokens;         /* >= 0                                      */
  bsa_select_mode intra_mode;    /* rule applied to the intra scores          */
  const double* intra_param;     /* host [Hd] in [0, 1], or NULL (no intra)   */
} bsa_mask_union_t;

/* bsa_kmax_for_union — list width that suffices under `u` (NULL = plain
 * selection): the inter bound plus what the window, sink and intra parts can
 * add, at most nb, plus nb_text. */
bsa_status bsa_kmax_for_union(bsa_plan_t plan, bsa_select_mode mode,
                              const double* param_per_head,
                              const bsa_mask_union_t* u, int* kmax);

/* bsa_union_workspace_size — device workspace (256-byte aligned) of
 * bsa_select_union (select_ws: the intra bit sets, 0 without intra) and of
 * bsa_forward_union (forward_ws: bsa_forward's plus, with intra, the SICS of
 * the K blocks and the bit sets). */
bsa_status bsa_union_workspace_size(bsa_plan_t plan, int kmax,
                                    const bsa_mask_union_t* u,
                                    size_t* select_ws, size_t* forward_ws);

/* bsa_select_union — bsa_select_centroids with the mask union.
 *   intra_scores  [B, Hd, nb] float device, one score per key block
 *                 (required when u->intra_param is set; e.g. bsa_sics of K)
 *   ws, ws_bytes  at least select_ws bytes (may be NULL / 0 without intra)
 * Other arguments as bsa_select_centroids; kmax >= bsa_kmax_for_union. */
bsa_status bsa_select_union(bsa_plan_t plan, const float* q_cent,
                            const float* k_cent, bsa_select_mode mode,
                            const double* param_per_head,
                            const bsa_mask_union_t* u,
                            const float* intra_scores, int kmax,
                            int32_t* idx, int32_t* cnt, float* scores,
                            void* ws, size_t ws_bytes, void* stream);

/* bsa_forward_union — bsa_forward with the mask union; the intra scores are
 * the SICS of the K blocks (SPADE §3.2 Eq. (4)), computed in the centroid
 * pass that reads K anyway (SPADE §3.3 (1): layout transform, summarization
 * and intra-estimation fused).  ws_bytes >= forward_ws of
 * bsa_union_workspace_size; kmax >= bsa_kmax_for_union.  u = NULL is
 * bsa_forward. */
bsa_status bsa_forward_union(bsa_plan_t plan, const void* q, const void* k,
                             const void* v, bsa_select_mode mode,
                             const double* param_per_head,
                             const bsa_mask_union_t* u, int kmax, void* o,
                             int32_t* idx_out, int32_t* cnt_out, void* ws,
                             size_t ws_bytes, int32_t* dev_status,
                             void* stream);

/* ---------------------------------------------------------------------------
 * Inter-estimators (SPADE §3.1: DSA-SPADE estimates with
 * (k_max, k_min, (q_max + q_min)/2), DSA2-SPADE with (k_max, k_min, q_max,
 * q_min), MEAN-SPADE with (q_mean, k_mean); the estimator equations sit in
 * the paper's Fig. 4, which its text does not reproduce).  Reading taken
 * here: the box estimators bound the largest dot product a block pair can
 * reach given the per-dimension (max, min) summaries of its blocks:
 *   DSA   est_ij = sum_d max(c_d kmax_d, c_d kmin_d),  c = (qmax + qmin) / 2
 *         (the largest c . k over the key block's box);
 *   DSA2  est_ij = sum_d max(qmax_d kmax_d, qmax_d kmin_d, qmin_d kmax_d,
 *         qmin_d kmin_d)  (the largest q . k over both boxes);
 * s_ij = est_ij / sqrt(D), selected by Top-K / Top-P on softmax_j(s_i) as
 * for MEAN.  The (max, min) are taken over the block's valid tokens. */
typedef enum { BSA_EST_MEAN = 0, BSA_EST_DSA = 1, BSA_EST_DSA2 = 2 } bsa_estimator;

/* bsa_box_summaries — per video block and dimension the (max, min) of the
 * valid tokens, straight from the original layout.
 *   q, k          [B, Ntot, Hd, D] original order (read only)
 *   q_box, k_box  [B, Hd, nb, D, 2] float out, (max, min) pairs (either may
 *                 be NULL) */
bsa_status bsa_box_summaries(bsa_plan_t plan, const void* q, const void* k,
                             float* q_box, float* k_box, void* stream);

/* bsa_select_box — bsa_select_union with the DSA or DSA2 estimator on box
 * summaries (as written by bsa_box_summaries).  est must be BSA_EST_DSA or
 * BSA_EST_DSA2; u may be NULL; other arguments as bsa_select_union. */
bsa_status bsa_select_box(bsa_plan_t plan, bsa_estimator est,
                          const float* q_box, const float* k_box,
                          bsa_select_mode mode, const double* param_per_head,
                          const bsa_mask_union_t* u, const float* intra_scores,
                          int kmax, int32_t* idx, int32_t* cnt, float* scores,
                          void* ws, size_t ws_bytes, void* stream);

/* bsa_estimator_workspace_size — workspace of bsa_forward_estimator. */
bsa_status bsa_estimator_workspace_size(bsa_plan_t plan, bsa_estimator est,
                                        int kmax, const bsa_mask_union_t* u,
                                        size_t* forward_ws);

/* bsa_forward_estimator — bsa_forward_union with the chosen inter-estimator:
 * the summarizer pass writes centroids (MEAN) or boxes (DSA, DSA2), plus the
 * K-block SICS when u has an intra part.  est = BSA_EST_MEAN is
 * bsa_forward_union.  ws_bytes >= bsa_estimator_workspace_size. */
bsa_status bsa_forward_estimator(bsa_plan_t plan, const void* q, const void* k,
                                 const void* v, bsa_estimator est,
                                 bsa_select_mode mode,
                                 const double* param_per_head,
                                 const bsa_mask_union_t* u, int kmax, void* o,
                                 int32_t* idx_out, int32_t* cnt_out, void* ws,
                                 size_t ws_bytes, int32_t* dev_status,
                                 void* stream);

/* ---------------------------------------------------------------------------
 * Head grouping with per-head blocking schemes (SPADE §3.3 (2): "groups heads
 * sharing a blocking scheme to increase per-launch work"; §3.2: each head
 * takes its Selected Blocking Scheme).  The candidate plans describe one
 * problem with different block shapes (as for bsa_aggregation_scores); each
 * (b, h) is served by the plan head_plan[b * Hd + h] names — for instance the
 * choice bsa_aggregation_scores returns, copied to the host.  The heads of
 * one plan are one group: one centroid launch, one selection launch and one
 * attention launch per batch element cover exactly those heads; the output
 * rows of every head are written once. */

/* bsa_grouped_workspace_size — workspace of bsa_forward_grouped: per plan its
 * centroids, lists (kmax_per_plan[c] wide) and, with an intra part in u, its
 * K-block SICS and bit sets. */
bsa_status bsa_grouped_workspace_size(const bsa_plan_t* plans, int n_plans,
                                      const int* kmax_per_plan,
                                      const bsa_mask_union_t* u,
                                      size_t* forward_ws);

/* bsa_forward_grouped — bsa_forward_union with a blocking scheme per (b, h).
 *   plans, n_plans  1..8 tensor-core plans (bf16, 128-token blocks) on the
 *                   current device that agree in everything but the block
 *                   shape; batch * heads <= 256
 *   head_plan       host [B * Hd] int32: plan index of each (b, h)
 *   q, k, v, o      [B, Ntot, Hd, D] original order
 *   mode, param_per_head, u   selection and mask union, as bsa_forward_union
 *                   (per-head parameters apply whatever the head's plan)
 *   kmax_per_plan   host [n_plans]: list width per plan (>= the plan's
 *                   bsa_kmax_for_union)
 *   idx_out, cnt_out  host arrays of n_plans device pointers to
 *                   [B, Hd, nb_c, kmax_c] / [B, Hd, nb_c] lists, or NULL
 *                   (either array or entry); only the (b, h) of plan c are
 *                   written in plan c's lists
 *   ws, ws_bytes    >= bsa_grouped_workspace_size
 * BSA_ERR_UNSUPPORTED for plans off the tensor-core path. */
bsa_status bsa_forward_grouped(const bsa_plan_t* plans, int n_plans,
                               const int32_t* head_plan, const void* q,
                               const void* k, const void* v,
                               bsa_select_mode mode,
                               const double* param_per_head,
                               const bsa_mask_union_t* u,
                               const int* kmax_per_plan, void* o,
                               int32_t* const* idx_out, int32_t* const* cnt_out,
                               void* ws, size_t ws_bytes, int32_t* dev_status,
                               void* stream);

/* ---------------------------------------------------------------------------
 * Tile pairing (no counterpart on the pages: a scheduling step of this
 * implementation).  The tensor-core attention runs two query tiles per CTA.
 * bsa_pair_tiles matches the video query blocks of every (b, h) in pairs
 * whose lists overlap most and writes, into its workspace, a schedule whose
 * two lists per pair start with the shared blocks; bsa_attention_paired then
 * fetches each shared K and V tile once for both tiles.  bsa_forward does
 * both on tensor-core plans.  Lists must be as bsa_select writes them
 * (ascending video blocks, then every text block).  The result equals
 * bsa_attention_orig up to the rounding of the reordered sums.  The text
 * query tiles (dense rows) run as key chunks about one list long, each in
 * its head's group of CTAs; their partial rows (unnormalised output, running
 * maximum, row sum) are kept in the tail of the pairing workspace and merged
 * by a second launch (SPADE §3.3 (3)'s online softmax finished across
 * chunks). */

/* bsa_pair_workspace_size — bytes of the pairing workspace (0 off the
 * tensor-core path). */
bsa_status bsa_pair_workspace_size(bsa_plan_t plan, int kmax, size_t* bytes);

/* bsa_pair_tiles — pairs the query tiles of idx / cnt ([B, Hd, nb, kmax],
 * [B, Hd, nb]) into `ws` (256-byte aligned, >= bsa_pair_workspace_size).
 * Serves plans with at most 1536 video blocks (BSA_ERR_UNSUPPORTED beyond;
 * bsa_forward then runs the attention unpaired). */
bsa_status bsa_pair_tiles(bsa_plan_t plan, const int32_t* idx,
                          const int32_t* cnt, int kmax, void* ws,
                          size_t ws_bytes, void* stream);

/* bsa_attention_paired — bsa_attention_orig on the schedule bsa_pair_tiles
 * wrote into ws from the same idx / cnt (same plan limits as
 * bsa_pair_tiles).  It writes the text rows' partials into the workspace's
 * tail (the schedule itself is only read). */
bsa_status bsa_attention_paired(bsa_plan_t plan, const void* q, const void* k,
                                const void* v, const int32_t* idx,
                                const int32_t* cnt, int kmax, void* ws,
                                size_t ws_bytes, void* o, int32_t* dev_status,
                                void* stream);

/* bsa_check_status — synchronise `stream`, read and clear the plan-owned
 * status word; returns BSA_OK or the recorded error. */
bsa_status bsa_check_status(bsa_plan_t plan, void* stream);

/* Device times of the phases of one bsa_forward call, in milliseconds (CUDA
 * events recorded on the call's stream at each phase boundary).  SPADE Fig. 5
 * splits one layer's sparse attention into "Pattern Search" and "Attention
 * Computation"; here pattern search = summaries_ms + select_ms + pairing_ms. */
typedef struct {
  float summaries_ms;  /* tensor-core plans: the centroid pass over Q and K;
                          other plans: the permute of Q, K, V with its centroids */
  float select_ms;     /* scores, softmax and the Top-K / Top-P lists          */
  float pairing_ms;    /* tile pairing (tensor-core plans; 0 when not run)     */
  float attention_ms;  /* block-sparse attention (on tensor-core plans with the
                          layout transform fused into its loads and stores)   */
  float unpermute_ms;  /* inverse permute (other plans only)                   */
  float total_ms;      /* first to last boundary                               */
} bsa_timings_t;

/* bsa_forward_timed — bsa_forward with per-phase device times.  Same
 * arguments, outputs and errors as bsa_forward, plus `timings` (host
 * pointer, must not be NULL; zeroed first).  Unlike bsa_forward it creates
 * six CUDA events and synchronises on the last one before returning, so it
 * is not for use inside a stream capture and costs a host round trip; the
 * results are those of a plain bsa_forward call. */
bsa_status bsa_forward_timed(bsa_plan_t plan, const void* q, const void* k,
                             const void* v, bsa_select_mode mode,
                             const double* param_per_head, int kmax, void* o,
                             int32_t* idx_out, int32_t* cnt_out, void* ws,
                             size_t ws_bytes, int32_t* dev_status, void* stream,
                             bsa_timings_t* timings);

/* bsa_plan_set_watchdog — bound of the tensor-core attention kernel's
 * in-kernel waits (failure detection; no counterpart on the pages, which
 * describe no failure handling).
 *   wait_limit_cycles  every mbarrier wait of the kernel (a K/V copy landing,
 *                      S or P ready, a ring slot freed) gives up after this
 *                      many SM clock cycles; 0 = the default of 2^31 (about
 *                      a second).  When a wait runs out the kernel raises a
 *                      CTA-wide abort, waits (with the same bound) for the
 *                      copies and MMAs it has already issued, frees its TMEM,
 *                      writes zeros for its rows and records BSA_ERR_TIMEOUT
 *                      in the status word; the context stays usable.
 *   withhold_copy      test hook of that path: n > 0 makes CTA 0 of every
 *                      tensor-core attention launch skip its n-th K/V copy
 *                      (so its consumer's wait runs out); 0 = off.  Never set
 *                      it outside tests.
 * Takes effect for launches issued after the call; do not change it while a
 * call on this plan is being issued on another thread.  Negative values are
 * BSA_ERR_INVALID_ARG. */
bsa_status bsa_plan_set_watchdog(bsa_plan_t plan, long long wait_limit_cycles,
                                 int withhold_copy);

/* Thread-local message describing the last non-OK return of this thread. */
const char* bsa_last_error_string(void);
int bsa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BSA_H_ */
