/*
 * tsa.h: C ABI of libtsa, the Token Sparse Attention layer for NVIDIA B200 (sm_100a).
 *
 * The method is from "Token Sparse Attention: Efficient Long-Context Inference with
 * Interleaved Token Selection".  Page citations below:
 *   [notes] the papernotes.org notes on that paper (方法详解 › 整体框架; 关键设计 1
 *           Compress-then-Decompress; 关键设计 2 Dynamic Token Coverage; 关键设计 3
 *           Inter-Layer Representation Drift; 消融实验 ablations);
 *   [blog]  the bxzpzcl.cn post (§1.1 核心算法实现细节; §2 稀疏层选择 by drift;
 *           §2.1 重要性评估机制);
 *   [gist]  the gist.science summary (§2 Methodology: Core Architecture; Dynamic
 *           Token Coverage).
 *
 * Conventions shared by every call
 *   Memory   The caller owns every buffer.  All pointers are device pointers on the
 *            current CUDA device, 16-byte aligned and densely packed in the layout
 *            stated.  The library allocates, frees and synchronises nothing
 *            (tsa_get_device_status is the one call that synchronises).
 *   Streams  Every call only enqueues work on `stream` (a cudaStream_t passed as
 *            void*, NULL = legacy default stream) and returns.  L' stays on the
 *            device, so no call reads results back to the host.
 *   Layouts  Q  [B, L, H, d];  K, V [B, L, Hkv, d];  X, Y [B, L, H*d]  (row-major);
 *            s_h [B, H, L] fp32;  s_l [B, L] fp32;  Lkeep [B] int32;
 *            idx [B, H, L] int32;  Qh, Kh, Vh, Oh [B, H, L, d] (compressed, head-major).
 *            Query head h reads KV head h / (H / Hkv).
 *   Types    dtype TSA_BF16: Q, K, V, X, Y, Qh, Kh, Vh, Oh are bfloat16, with fp32
 *            accumulation everywhere.  dtype TSA_F32: the same tensors are fp32.
 *            d must be 64 or 128.  G * min(q, L) <= 256 where G = H / Hkv.
 *   Errors   Each call returns a status and never aborts.  Argument errors are found
 *            on the host before anything is enqueued.  A failed launch returns
 *            TSA_ERR_CUDA.  tsa_last_error() gives a message for the calling thread.
 *            Errors found on the device (a bounded wait that ran out, a score that is
 *            not a finite value in [0, 1]) are recorded in the workspace's error word
 *            and returned by tsa_get_device_status.  The word keeps the first error
 *            until it is read; after a device error, the results of later calls that
 *            use the same workspace are undefined until tsa_get_device_status has
 *            returned it (reading it also resets the workspace's grid-barrier words).
 *   Workspace `ws` is caller-owned device scratch of at least tsa_workspace_size()
 *            bytes (tsa_layer_workspace_size() for tsa_layer), 256-byte aligned,
 *            zero-filled once before its first use.  Calls that share a workspace
 *            must be ordered on one stream.
 */
#ifndef TSA_H_
#define TSA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TSA_API __attribute__((visibility("default")))
#else
#define TSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    TSA_OK = 0,
    TSA_ERR_INVALID_ARG = 1,    /* a null pointer, a bad size, tau or scale      */
    TSA_ERR_ALIGNMENT = 2,      /* a pointer that is not 16-byte aligned          */
    TSA_ERR_UNSUPPORTED = 3,    /* a shape or dtype the library does not implement */
    TSA_ERR_WORKSPACE = 4,      /* workspace too small or misaligned              */
    TSA_ERR_CUDA = 5,           /* a CUDA runtime or launch error                 */
    TSA_ERR_DEVICE_TIMEOUT = 6, /* a bounded device-side wait ran out             */
    TSA_ERR_NONFINITE = 7       /* s_l outside [0, 1], s_h < 0, or a NaN / inf score */
} tsa_status;

typedef enum { TSA_F32 = 0, TSA_BF16 = 1 } tsa_dtype;

typedef struct {
    int32_t B;     /* batch                                   */
    int32_t L;     /* tokens per sequence, 1 <= L <= 2^21      */
    int32_t H;     /* query heads                              */
    int32_t Hkv;   /* key/value heads, H % Hkv == 0            */
    int32_t d;     /* head dimension, 64 or 128                */
    int32_t dtype; /* tsa_dtype                                */
} tsa_dims;

/* Bytes of workspace needed by tsa_score, tsa_budget, tsa_select and tsa_attn for
 * these dims and q (0 on invalid arguments). */
TSA_API size_t tsa_workspace_size(const tsa_dims *dims, int32_t q);

/* Bytes of workspace needed by tsa_layer: the above plus room for every
 * intermediate (s_h, s_l, Lkeep, idx, Qh, Kh, Vh, Oh). */
TSA_API size_t tsa_layer_workspace_size(const tsa_dims *dims, int32_t q);

/* Dynamic Token Coverage scoring ([notes] 关键设计 2; [blog] §2.1; [gist] §2).
 * For each batch b, query head h and each of the last q_eff = min(q, L) positions
 * p = L - q_eff + i, the softmax over keys t <= p of scale * <Q[b,p,h], K[b,t,kv(h)]>
 * gives A[i, t]; s_h[b,h,t] = sum_i A[i,t].  Then u[t] = sum_h s_h[b,h,t] and
 * s_l[b,t] = u[t] / sum_t u[t].  Causal scoring and the shared scale are readings of
 * the pages.  Deterministic: every sum runs in a fixed order.
 * Q [B,L,H,d], K [B,L,Hkv,d]; s_h [B,H,L] and s_l [B,L] fp32 outputs.  scale > 0
 * (normally 1/sqrt(d)). */
TSA_API tsa_status tsa_score(const tsa_dims *dims, const void *Q, const void *K, int32_t q,
                     float scale, float *s_h, float *s_l, void *ws, size_t ws_bytes,
                     void *stream);

/* ---- One layer sharded by KV group across GPUs -------------------------------------- */
/* [blog] §2.1 层级预算分配 and [notes] 关键设计 2: s_l is the normalised sum over all
 * heads of s_h, so u[t] = sum_h s_h[h, t] is the only quantity that couples the heads.
 * A GPU that holds a contiguous range of KV groups (its query heads, their K and V, and
 * their columns of X and Y) runs:
 *   tsa_score_partial        s_h of its heads and their unnormalised partial u;
 *   an all-gather of every GPU's partial u (the caller's collective, e.g. NCCL);
 *   tsa_layer_score_combine  the fixed-order sum of the gathered partials and s_l;
 * then tsa_budget, tsa_select, tsa_gather_qkv, tsa_attn and tsa_scatter_residual on
 * its own heads.  Every GPU combines the same partials in the same order, so s_l and
 * L' are bit-identical on every GPU. */

/* Scoring of this shard's heads: as tsa_score (dims, Q [B,L,H,d] and K [B,L,Hkv,d] are
 * the shard's own: H and Hkv count its heads), writing s_h [B,H,L] and, in place of
 * s_l, the partial layer score u_part[b,t] = sum over the shard's heads, in head order,
 * of s_h[b,h,t] ([B,L] fp32, not normalised).  ws: tsa_workspace_size(dims, q) bytes. */
TSA_API tsa_status tsa_score_partial(const tsa_dims *dims, const void *Q, const void *K,
                                     int32_t q, float scale, float *s_h, float *u_part,
                                     void *ws, size_t ws_bytes, void *stream);

/* Layer score from the partials of nparts shards: u_parts [nparts, B, L] fp32 (shard r's
 * u_part at u_parts + r*B*L; order them by rank), u[b,t] = sum over r = 0 .. nparts-1 in
 * that order of u_parts[r,b,t], s_l[b,t] = u[b,t] / sum_t u[b,t] (the total in a fixed
 * order).  Deterministic: the same partials give the same s_l bit for bit on every GPU.
 * Only dims->B and dims->L are used (the other fields must be valid).  1 <= nparts <=
 * 1024; s_l must not overlap u_parts.  ws: tsa_workspace_size(dims, 1) bytes. */
TSA_API tsa_status tsa_layer_score_combine(const tsa_dims *dims, int32_t nparts,
                                           const float *u_parts, float *s_l, void *ws,
                                           size_t ws_bytes, void *stream);

/* Coverage budget ([notes] 关键设计 2; [blog] §2.1 层级预算分配; [gist] §2 Budget
 * Allocation).  Sort s_l[b,:] ascending and find the smallest k whose cumulative mass
 * reaches tau; Lkeep[b] = L - k (k = L, so Lkeep = 0, if it is never reached).  The
 * cumulative mass is exact: each s_l is taken as floor(s_l * 2^62) in uint64 and
 * compared with ceil(tau * 2^62).  s_l values must lie in [0, 1] and sum to at most 4
 * (tsa_score's sum to 1).  0 <= tau < 1.  Lkeep [B] int32 device output. */
TSA_API tsa_status tsa_budget(const tsa_dims *dims, const float *s_l, double tau, int32_t *Lkeep,
                      void *ws, size_t ws_bytes, void *stream);

/* Per-head top-L' selection ([notes] 关键设计 2; [gist] §2 Head-Wise Selection).
 * For each (b, h): the Lkeep[b] tokens with the largest s_h[b,h,:], ties to the lower
 * token index, written to idx[b,h,0:Lkeep[b]] in ascending token order; the other
 * L - Lkeep[b] tokens follow in idx[b,h,Lkeep[b]:L], also ascending, so each row of
 * idx is a permutation of 0..L-1.  Lkeep is read on the device. */
TSA_API tsa_status tsa_select(const tsa_dims *dims, const float *s_h, const int32_t *Lkeep,
                      int32_t *idx, void *ws, size_t ws_bytes, void *stream);

/* Compress ([notes] 整体框架, 关键设计 1; [blog] §1.1 压缩阶段; [gist] §2 Compression).
 * For i < Lkeep[b]: Qh[b,h,i] = Q[b,idx[b,h,i],h], Kh[b,h,i] = K[b,idx[b,h,i],kv(h)],
 * Vh likewise.  Rows i in [Lkeep[b], min(L, ceil128(Lkeep[b]))) of Qh, Kh, Vh are
 * zero-filled (the attention kernel reads whole 128-row tiles); later rows are not
 * written.  An index outside [0, L) is skipped and reported as TSA_ERR_INVALID_ARG in the
 * workspace's error word (ws supplies only the error word).  Lkeep[b] outside [0, L] is
 * clamped to that range. */
TSA_API tsa_status tsa_gather_qkv(const tsa_dims *dims, const void *Q, const void *K,
                          const void *V, const int32_t *idx, const int32_t *Lkeep,
                          void *Qh, void *Kh, void *Vh, void *ws, size_t ws_bytes,
                          void *stream);

/* Attention ([notes] 整体框架; [blog] §1.1 softmax(Q̂K̂ᵀ/√d)V̂).
 * dense == 0 (compressed): for each (b, h) and i < Lkeep[b],
 *   Oh[b,h,i] = sum_{j<=i} softmax_j(scale * <Qh[b,h,i], Kh[b,h,j]>) Vh[b,h,j];
 *   inputs and output are [B,H,L,d].  Because idx lists kept tokens in ascending
 *   order, j <= i is the causal mask on original positions.  Rows of Kh/Vh in
 *   [Lkeep[b], ceil128(Lkeep[b])) must hold finite values (tsa_gather_qkv zeroes
 *   them).  Rows i >= Lkeep[b] of Oh are not written.
 * dense == 1: dense causal GQA attention of the full sequence (the pages' dense
 *   branch for layers outside the sparse set): Qh = Q [B,L,H,d], Kh = K and
 *   Vh = V [B,L,Hkv,d], Oh = O [B,L,H,d]; Lkeep is ignored and may be NULL.
 * scale > 0 (normally 1/sqrt(d)).  ws supplies the error word.  A compressed-mode
 * Lkeep[b] outside [0, L] is clamped to that range (no row at or past L is read or
 * written) and reported as TSA_ERR_INVALID_ARG in the error word. */
TSA_API tsa_status tsa_attn(const tsa_dims *dims, const void *Qh, const void *Kh, const void *Vh,
                    const int32_t *Lkeep, int32_t dense, float scale, void *Oh,
                    void *ws, size_t ws_bytes, void *stream);

/* Decompress and residual ([notes] 关键设计 1: X_{l+1} = X_l + Decompress(Ô), unselected
 * rows of the decompressed tensor are zero; [blog] §1.1 解压缩阶段; [gist] §2
 * Decompression).
 *   idx != NULL: Y[b, idx[b,h,i], h*d:(h+1)*d] = X[...] + Oh[b,h,i] for i < Lkeep[b].
 *     If Y != X, every other segment gets Y = X; this reads the complement that
 *     tsa_select stores in idx[b,h,Lkeep[b]:L].  If Y == X the update is in place
 *     and only the kept segments are touched.
 *   idx == NULL: dense layer, Oh is O [B,L,H,d] and Y = X + O (Lkeep ignored).
 * The sum is formed in fp32 and rounded once to the output type.  Y may equal X;
 * no other aliasing is allowed.  Preconditions, enforced on the device without an error
 * report (this call has no workspace): Lkeep[b] outside [0, L] is clamped to that range,
 * and an index outside [0, L) is skipped, so no segment outside Y is written. */
TSA_API tsa_status tsa_scatter_residual(const tsa_dims *dims, const void *Oh, const int32_t *idx,
                                const int32_t *Lkeep, const void *X, void *Y, void *stream);

/* The whole layer ([notes] 整体框架): is_sparse != 0 runs tsa_score, tsa_budget,
 * tsa_select, tsa_gather_qkv, tsa_attn and tsa_scatter_residual in order with no host
 * synchronisation; is_sparse == 0 runs dense causal attention and the residual (the
 * dense branch for layers outside the sparse set; which layers are sparse is the
 * caller's input).  s_h_out, s_l_out, Lkeep_out, idx_out are optional (NULL: kept in
 * ws); when given they receive those intermediates.  stage_events, if not NULL,
 * points to 7 cudaEvent_t (as void*) recorded before scoring and after each of the
 * six stages (for a dense layer the first five are recorded at the start; for L <= 8192
 * budget and selection run in one launch, and the events after them are recorded
 * together).  Without stage events the kernels after the scoring are launched as a
 * programmatic-dependent chain (each may start launching while the one before it
 * finishes; the results are the same bit for bit); with them, each kernel waits for the
 * event before it.  Y may equal X. */
TSA_API tsa_status tsa_layer(const tsa_dims *dims, const void *Q, const void *K, const void *V,
                     const void *X, void *Y, int32_t is_sparse, int32_t q, double tau,
                     float scale, float *s_h_out, float *s_l_out, int32_t *Lkeep_out,
                     int32_t *idx_out, void *ws, size_t ws_bytes, void *stream,
                     void *const *stage_events);

/* Compress, attention and decompress in one pass ([notes] 关键设计 1: the compressed
 * Q̂K̂V̂ are the rows S_h of Q, K, V; Decompress writes Ô back into those rows): the same
 * result as tsa_gather_qkv + tsa_attn + tsa_scatter_residual, bit for bit, without the
 * compressed copies.  The attention kernel reads the rows idx[b,h,0:Lkeep[b]] of Q
 * [B,L,H,d] and of K, V [B,L,Hkv,d] (KV head h / (H / Hkv)) directly, and its epilogue
 * writes Y[b,t,h*d:(h+1)*d] = X + bf16(Ô) (fp32 add, one rounding) for every kept token
 * t; the other segments of Y are copied from X (nothing to do when Y == X).  idx as
 * tsa_select writes it (kept tokens ascending, then the rest); an index outside [0, L)
 * is reported in the workspace's error word.  bf16 only (TSA_ERR_UNSUPPORTED for fp32).
 * ws supplies the error word (>= 256 bytes). */
TSA_API tsa_status tsa_attn_gather(const tsa_dims *dims, const void *Q, const void *K,
                                   const void *V, const int32_t *idx, const int32_t *Lkeep,
                                   float scale, const void *X, void *Y, void *ws,
                                   size_t ws_bytes, void *stream);

/* ---- Block-sparse attention inside the compressed space ---------------------------- */
/* [notes] 关键发现 (token sparsity stacked on block-level sparsity is the most valuable
 * pairing) and [blog] §3.2 ("token selection first, then block-sparse computation").
 * The block choice is this library's own definition (the pages give none).  In head h's
 * compressed order: query pair p = rows [256p, 256p + 256), key block j = rows
 * [128j, 128j + 128), NP = ceil(L / 256) pairs, NB = ceil(L / 128) blocks of capacity.
 *   logits[b,h,p,j] = scale * < mean of the pair's Qh rows, mean of block j's Kh rows >
 *                     for j < 2p (NaN otherwise);
 *   mask[b,h,p] (NW = ceil(NB / 32) uint32 words, bit j of word j / 32): block 0, the
 *                     diagonal blocks 2p and 2p + 1 (if it exists), and every j < 2p with
 *                     logits >= max_j logits - theta (one fp32 subtraction, fp32 compare).
 * Means are fp32 sums in row order, dot products fp32 in a fixed order: deterministic.
 * theta in [0, 3e38] (3e38 keeps every block).  logits [B,H,NP,NB] fp32 is optional
 * (NULL: not written).  Qh, Kh as tsa_gather_qkv writes them.  ws:
 * tsa_block_workspace_size() bytes. */
TSA_API size_t tsa_block_workspace_size(const tsa_dims *dims);
TSA_API tsa_status tsa_block_select(const tsa_dims *dims, const void *Qh, const void *Kh,
                                    const int32_t *Lkeep, float scale, double theta,
                                    float *logits, uint32_t *mask, void *ws, size_t ws_bytes,
                                    void *stream);

/* Compressed attention restricted to the kept blocks of `mask` (as tsa_block_select
 * writes it): row i attends to the keys i' <= i whose block is kept for the pair of i.
 * Otherwise as tsa_attn with dense == 0.  bf16 only. */
TSA_API tsa_status tsa_attn_block(const tsa_dims *dims, const void *Qh, const void *Kh,
                                  const void *Vh, const int32_t *Lkeep, const uint32_t *mask,
                                  float scale, void *Oh, void *ws, size_t ws_bytes, void *stream);

/* ---- Budget and score variants ([notes] 消融实验 and 关键设计 2) ------------------- */

typedef enum { TSA_POOL_NONE = 0, TSA_POOL_MAX = 1, TSA_POOL_MEAN = 2 } tsa_pool_kind;
typedef enum { TSA_BUDGET_COVERAGE = 0, TSA_BUDGET_FIXED = 1 } tsa_budget_kind;

/* Fixed-ratio budget, the ablation the notes compare the coverage budget with
 * (消融实验, "Fixed s = 0.3 / 0.5"): `sparsity` is the fraction of tokens pruned, so
 * Lkeep[b] = L - floor(sparsity * L) for every b (the product taken in double).
 * sparsity in [0, 1], else TSA_ERR_INVALID_ARG.  Lkeep is [B] int32 on the device. */
TSA_API tsa_status tsa_budget_fixed(const tsa_dims *dims, double sparsity, int32_t *Lkeep,
                                    void *stream);

/* Pooling of the head scores along the token axis ([notes] 关键设计 2: the column sums
 * are pooled into s_h before the layer score; the pages name neither kind nor window):
 *   s_h_out[b,h,t] = max or mean of s_h[b,h,u] over u in [t - r, t + r] clipped to
 *   [0, L), width = 2r + 1; the mean divides by the number of tokens in range (fp32
 *   sum in token order, one division).
 * Then s_l_out[b,t] = u[t] / sum_t u with u[t] = sum_h s_h_out[b,h,t], as in tsa_score.
 * kind TSA_POOL_MAX or TSA_POOL_MEAN; width odd, 1 <= width <= 255 (else
 * TSA_ERR_INVALID_ARG / TSA_ERR_UNSUPPORTED).  s_h_out must not overlap s_h.  ws as for
 * tsa_score with q = 1 (tsa_workspace_size(dims, 1) bytes). */
TSA_API tsa_status tsa_pool_scores(const tsa_dims *dims, const float *s_h, int32_t kind,
                                   int32_t width, float *s_h_out, float *s_l_out, void *ws,
                                   size_t ws_bytes, void *stream);

/* Options of tsa_layer_ex.  budget TSA_BUDGET_COVERAGE uses tau (as tsa_layer);
 * TSA_BUDGET_FIXED uses sparsity (as tsa_budget_fixed).  pool TSA_POOL_NONE uses the
 * scores as they are (as tsa_layer); otherwise selection and budget use the pooled head
 * scores (as tsa_pool_scores with pool_width). */
typedef struct {
    int32_t budget;     /* tsa_budget_kind                      */
    double tau;         /* coverage threshold, [0, 1)           */
    double sparsity;    /* fixed fraction pruned, [0, 1]        */
    int32_t pool;          /* tsa_pool_kind                        */
    int32_t pool_width;    /* odd, 1..255 (ignored for POOL_NONE)  */
    int32_t direct_gather; /* 1: tsa_attn_gather instead of gather, attention, scatter
                              (bf16 only; same Y bit for bit)      */
    double block_theta;    /* >= 0: block-sparse attention inside the compressed space with
                              this theta (tsa_block_select, tsa_attn_block; bf16, staged
                              path); negative or NaN: every block  */
} tsa_layer_opts;

/* tsa_layer with the budget and score variants of tsa_layer_opts (opts NULL: coverage
 * budget with tau = 0.005, no pooling).  When pooling, s_h_out and s_l_out receive the
 * pooled head scores and their layer score (the ones budget and selection used); the
 * raw scores stay in ws.  Workspace: tsa_layer_workspace_size() bytes.  Everything else
 * as tsa_layer. */
TSA_API tsa_status tsa_layer_ex(const tsa_dims *dims, const void *Q, const void *K,
                                const void *V, const void *X, void *Y, int32_t is_sparse,
                                int32_t q, const tsa_layer_opts *opts, float scale,
                                float *s_h_out, float *s_l_out, int32_t *Lkeep_out,
                                int32_t *idx_out, void *ws, size_t ws_bytes, void *stream,
                                void *const *stage_events);

/* ---- Choice of the sparse layers ([notes] 关键设计 3) ------------------------------ */

/* Bytes of workspace tsa_drift needs (0 on invalid arguments). */
TSA_API size_t tsa_drift_workspace_size(int32_t n_layers, int64_t tokens);

/* Inter-layer representation drift on calibration hidden states and the sparse-layer
 * mask ([notes] 关键设计 3; [blog] §2):
 *   R[l] = mean over t of ||h[l+1,t] - h[l,t]||_2 / (||h[l,t]||_2 + eps),
 *   mask[l] = 1 iff rank_l / n_layers <= delta, rank_l the 1-based position of R[l] in
 *   ascending order (ties: lower layer first); delta = 0.5 makes the half of the layers
 *   with the smallest drift sparse.
 * h: [n_layers + 1, tokens, d_model] contiguous, dtype TSA_BF16 or TSA_F32 (h[0] the
 * input of layer 0, h[l+1] the output of layer l), 16-byte aligned.  Norms are summed in
 * fp32 per token, the token mean in fp64, in a fixed order (deterministic).  R [n_layers]
 * fp64 and mask [n_layers] int32 are device outputs.  1 <= n_layers <= 512;
 * d_model * element size a multiple of 16 bytes; eps >= 0; delta in [0, 1].
 * ws: tsa_drift_workspace_size() bytes, 256-byte aligned. */
TSA_API tsa_status tsa_drift(int32_t n_layers, int64_t tokens, int32_t d_model, int32_t dtype,
                             const void *h, double eps, double delta, double *R, int32_t *mask,
                             void *ws, size_t ws_bytes, void *stream);

/* Scoring for callers that cannot allocate device memory when they call in, such as an
 * engine whose device memory is fully planned up front by its own allocator, or a host
 * thread that must not enter the CUDA allocator.  Those callers cannot create the `ws`
 * tsa_score needs.  The pages have no counterpart: this is tsa_score (same arguments
 * minus the workspace, same kernels, same results) with its scratch taken from a fixed
 * 2 MiB array in the library's device image, held on every GPU that loads the library
 * until the process exits.  The caller still passes Q, K, s_h and s_l.
 *   Limit   dims and q whose scoring workspace (tsa_workspace_size) exceeds 2 MiB are
 *           rejected with TSA_ERR_WORKSPACE before any device work; for example
 *           B = 1, L = 131072, 32/8 heads, q = 16 needs about 540 KB.
 *   Set-up  the first call on each device looks up the array's device address (with
 *           that device current) and caches it; make that first call before any stream
 *           capture.
 *   Sharing every call on a device uses the same array, which keeps the last call's
 *           contents; the scoring writes every scratch byte it reads before reading it.
 *           Calls whose work overlaps on the GPU (other streams, or other host threads)
 *           race on it and must be serialised by the caller.
 *   Errors  device-side errors (a bounded wait that ran out) go to an error word in
 *           the array, which keeps the first one until
 *           tsa_score_fixed_scratch_status reads and clears it; until then the results
 *           of later calls on that device are undefined.
 *   Reset   the cached address belongs to the device's primary context; after
 *           cudaDeviceReset (or another teardown of that context) call
 *           tsa_score_fixed_scratch_forget() before calling again on that device.
 * It allocates and frees nothing. */
TSA_API tsa_status tsa_score_fixed_scratch(const tsa_dims *dims, const void *Q, const void *K,
                                           int32_t q, float scale, float *s_h, float *s_l,
                                           void *stream);

/* Device errors of tsa_score_fixed_scratch on the current device: synchronises
 * `stream`, returns the error word of the fixed array (TSA_OK if none) and clears it
 * (with the array's grid-barrier words, which a failed launch can leave part-way).
 * Allocates nothing. */
TSA_API tsa_status tsa_score_fixed_scratch_status(void *stream);

/* Drops the cached device addresses of the fixed array on every device, so that the
 * next tsa_score_fixed_scratch or tsa_score_fixed_scratch_status call on a device looks
 * its address up again (needed after cudaDeviceReset).  Never fails. */
TSA_API void tsa_score_fixed_scratch_forget(void);

/* Synchronises `stream`, returns the device error word recorded in `ws` (TSA_OK if
 * none) and, if it is set, clears the 256-byte control block at the start of `ws` (the
 * error word and the grid-barrier words). */
TSA_API tsa_status tsa_get_device_status(void *ws, void *stream);

/* Upper bound, in microseconds, of every device-side wait (on an mbarrier) in later
 * launches from any thread; default 2 000 000 (2 s).  A wait that runs out makes its
 * kernel record TSA_ERR_DEVICE_TIMEOUT, finish the copies and MMAs it started, free its
 * tensor memory and exit; tests lower the limit to check that path. */
TSA_API void tsa_set_wait_limit(uint32_t microseconds);

/* Test hook for the failure path, off by default.  When `on` is non-zero, later launches
 * of the tensor-core kernels (scoring of bf16 inputs, attention of bf16 inputs) first
 * make their MMA-issuing thread wait on a barrier that nothing completes.  The wait
 * runs out after the wait limit; the kernel then records TSA_ERR_DEVICE_TIMEOUT, winds
 * down as described above, and exits.  Nothing faults, traps or hangs. */
TSA_API void tsa_set_test_stall(int32_t on);

/* Scoring schedule of bf16 inputs, for tests and measurements; default (0, 0).  Two
 * kernels compute the same exact two-pass scores, within fp32 rounding (they differ in
 * summation order only):
 *   the single-wave kernel: every KV group at once; pass 1 with the recent-query rows on
 *     the TMEM lanes, pass 2 with the tokens on the lanes; K read from HBM twice;
 *   the wave-scheduled kernel: shapes whose recent-query count min(q, L) is 16, with at
 *     most 4 query heads per KV head and d = 64 or 128; tokens on the TMEM lanes in both
 *     passes; the KV groups in waves (one wave, or a few groups per wave so that pass 2
 *     rereads K from L2).
 * wave = 0 (automatic, the default): the wave-scheduled kernel with every KV group in one
 *   wave for the shapes it covers whose K tensor holds at least 192 MiB (B*L*Hkv*d*2
 *   bytes, 1.5 x the L2 size) with B * Hkv no more than the SMs, else the single-wave
 *   kernel (measured on one B200: the one-wave schedule is 4-6% faster with 268 MB of K,
 *   3% slower with 134 MB, which L2 nearly holds).
 * wave = 1: the wave-scheduled kernel for every shape it covers, about 40 MB of K per
 *   wave; max_groups_per_wave > 0 caps the groups of one wave (more waves on small
 *   inputs), 0 lets the library choose.
 * wave = 2: the single-wave kernel for every shape.
 * Other values act as 0.  Applies to later launches from any thread. */
TSA_API void tsa_set_score_schedule(int32_t wave, int32_t max_groups_per_wave);

/* Number of CUDA kernels this library has launched in this process, on every device and
 * thread (a host-side counter; memset and copy operations are not counted).  Callers take
 * the difference around a region to count its launches.  Never fails. */
TSA_API uint64_t tsa_kernel_launches(void);

TSA_API const char *tsa_status_string(tsa_status s);
TSA_API const char *tsa_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* TSA_H_ */
