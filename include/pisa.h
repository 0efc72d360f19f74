/*
 * pisa.h -- C ABI of the B200 (sm_100a) PISA block-sparse attention library.
 *
 * PISA ("Block Sparse Attention with Log-Linear Complexity") selects, for every
 * query, K leaf blocks of C keys by walking a mean-pooled key pyramid from the
 * root down, keeping the Top-K nodes at each level, and then runs causal softmax
 * attention over the keys of the selected leaves. Citations below name the page
 * "论文精读 · Block Sparse Attention with Log-Linear Complexity (PISA)"
 * (qqtang-code.github.io) as "close reading", by section and equation.
 *
 * Conventions shared by every call
 * --------------------------------
 * Layout.   Q, O: [B, Hq, N, d]; K, V: [B, Hkv, N, d]; all contiguous, row-major,
 *           element type cfg->dtype (fp32 or bf16). pyr: fp32 [B, Hkv, R, d] with
 *           R = pisa_pyramid_rows(cfg), levels 1..L concatenated (leaves first).
 *           idx: int32 [B, Hkv, N, K]: per query position and KV head, the selected
 *           leaf indices sorted ascending, padded with -1 when fewer than K leaves
 *           are eligible. Leaf i covers tokens [i*C, min((i+1)*C, N)).
 * Indices.  0-based. Node i of level l covers tokens [i*C*g^(l-1), ...).
 * Heads.    G = Hq / Hkv query heads share one KV head; selection runs per
 *           (token, KV head) with node scores summed over the G heads (close
 *           reading §04 4.4, Eq.(11)); MHA is G = 1.
 * Causal.   When cfg->causal, query t sees key j iff j <= t; nodes whose first
 *           token is > t are not candidates; nodes containing t are always kept
 *           and never ranked (close reading §5.3).
 * Forced.   cfg->forced_mask bit0 = first leaf, bit1 = previous leaf, bit2 =
 *           current leaf (implied when causal); their ancestor paths are kept
 *           unranked and they count against K (close reading §5.3, Eq.(6)).
 * Ties.     Equal scores rank the lower node index first.
 * Memory.   The caller owns every buffer (device memory unless stated). The
 *           library allocates nothing and keeps no state between calls.
 * Streams.  `stream` is a cudaStream_t passed as void*; NULL is the legacy
 *           default stream. Every call only enqueues work; it returns before
 *           the GPU finishes, and the caller synchronises.
 * Errors.   Calls return PISA_OK (0) or a negative PISA_E_* code. Arguments are
 *           validated on the host before anything is enqueued; a call that
 *           fails validation writes nothing. PISA_E_CUDA reports a launch error
 *           (cudaGetLastError after the launch). No device-side assert or trap
 *           is ever used.
 * Limits.   GPU path: g = 2, d in {64, 128}, 1 <= K <= 16, 1 <= C <= 1024,
 *           G in {1, 2, 4, 8, 16}, at most 32 pyramid levels, N < 2^31,
 *           16-byte aligned tensor pointers.
 */
#ifndef PISA_H
#define PISA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum pisa_dtype { PISA_DTYPE_F32 = 0, PISA_DTYPE_BF16 = 1 };

/* Node score used for ranking (close reading §04 4.3). From the children's
 * logits z_r = q . kbar_r / sqrt(d) (raw keys at the leaves), summed over a
 * GQA group (Eq.11):
 *   PISA_SCORE_LSE      Eq.(7): log sum_r exp(z_r) (the method; default);
 *   PISA_SCORE_MEAN     PISA-1, Eq.(8) truncated: the mean of the z_r;
 *   PISA_SCORE_MEAN_VAR PISA-2, Eq.(9): the mean plus half the population
 *                       variance of the z_r.
 * Only the ranking changes: attention always uses the exact softmax. */
enum pisa_score { PISA_SCORE_LSE = 0, PISA_SCORE_MEAN = 1, PISA_SCORE_MEAN_VAR = 2 };

enum pisa_status {
    PISA_OK = 0,
    PISA_E_INVALID = -1,      /* null pointer, bad size, inconsistent config */
    PISA_E_UNSUPPORTED = -2,  /* valid for the method, outside the GPU limits */
    PISA_E_CUDA = -3,         /* a CUDA launch or runtime call failed */
    PISA_E_ALIGNMENT = -4,    /* a tensor pointer is not 16-byte aligned (pyramid of the *_ws calls: 32) */
    PISA_E_TIMEOUT = -5,      /* a kernel gave up a bounded wait (see pisa_workspace_status) */
    PISA_E_SCRATCH_LIMIT = -6 /* problem too large for pisa_select_noalloc's fixed scratch */
};

/* Problem statement (close reading §02-§04: N, d, C, K, g, causal). */
typedef struct pisa_cfg {
    int32_t B;            /* batch (sequences) */
    int32_t Hq;           /* query heads */
    int32_t Hkv;          /* key/value heads; Hq % Hkv == 0 */
    int32_t N;            /* tokens per sequence (decode calls: cache capacity) */
    int32_t d;            /* head dimension */
    int32_t C;            /* leaf block size g_0 (Eq.(3)) */
    int32_t K;            /* blocks kept per level (Eq.(6)) */
    int32_t g;            /* branching factor above the leaves (Eq.(3)); must be 2 */
    int32_t causal;       /* 1: causal mask and causal eligibility; 0: none */
    int32_t forced_mask;  /* bit0 first, bit1 previous, bit2 current leaf */
    int32_t dtype;        /* enum pisa_dtype of Q, K, V, O and the decode caches */
    int32_t score_variant; /* enum pisa_score: how a node is ranked from its children */
} pisa_cfg;

/* ---- geometry (close reading §04 4.1, Eq.(3)) -------------------------------
 * M_1 = ceil(N / C), M_{l+1} = ceil(M_l / g), L = first level with one node. */

/* Number of pyramid levels L (0 when N == 0; negative status on a bad cfg). */
int pisa_num_levels(const pisa_cfg *cfg);
/* M_l, nodes of level l (1 <= l <= L); negative status on error. */
int64_t pisa_level_nodes(const pisa_cfg *cfg, int level);
/* Row offset of level l inside one (b, kv-head) pyramid; negative on error. */
int64_t pisa_level_offset(const pisa_cfg *cfg, int level);
/* R = sum_l M_l: fp32 rows of d elements per (b, kv-head) pyramid. The whole
 * pyramid buffer holds B * Hkv * R * d floats. Negative status on error. */
int64_t pisa_pyramid_rows(const pisa_cfg *cfg);

/* ---- prefill path ------------------------------------------------------------ */

/* Key pyramid (close reading §04 4.1, Eq.(3)-(4)): leaf summaries are the mean
 * of the C raw keys of each leaf, every higher node the mean of its existing
 * children summaries; all levels are written.
 * K: [B, Hkv, N, d] (dtype); pyr: fp32 [B, Hkv, R, d] (written). */
int pisa_build_pyramid(const pisa_cfg *cfg, const void *K, float *pyr, void *stream);

/* Pyramid Top-K selection (close reading §04 4.2-4.4, Eq.(5)-(7), (11); §5.3).
 * For every (b, kv-head, t): start from the root; at each level the candidates
 * are the eligible children of the nodes kept one level up; when there are at
 * most K of them all are kept, otherwise the forced ones plus the best-scoring
 * others up to K, where a node's score is the LSE over its child summaries of
 * q . kbar / sqrt(d) (raw keys at the leaves) summed over the G query heads.
 * Q: [B, Hq, N, d]; K: [B, Hkv, N, d]; pyr from pisa_build_pyramid;
 * idx: int32 [B, Hkv, N, K] (written). */
int pisa_select(const pisa_cfg *cfg, const void *Q, const void *K, const float *pyr,
                int32_t *idx, void *stream);

/* Attention over the selected blocks (close reading §02, Eq.(2)): for query
 * head h at position t, softmax(q . k_j / sqrt(d)) over the keys j of the leaves
 * in idx[b, h / G, t, :] (j <= t when causal), applied to V. The score matrix
 * is never stored. Q: [B, Hq, N, d]; K, V: [B, Hkv, N, d]; idx as written by
 * pisa_select (entries < 0 are skipped); O: [B, Hq, N, d] (written, dtype). */
int pisa_sparse_attn(const pisa_cfg *cfg, const void *Q, const void *K, const void *V,
                     const int32_t *idx, void *O, void *stream);

/* Backward of pisa_sparse_attn with the selection idx held fixed (close
 * reading §5.3: the gradient flows only through the selected attention
 * entries). Given Q, K, V, idx as in the forward and dO (the gradient of the
 * loss with respect to O; [B, Hq, N, d], dtype of Q), writes
 *   dQ: fp32 [B, Hq, N, d];  dK, dV: fp32 [B, Hkv, N, d] (summed over the
 *   query heads of each KV head; both are zeroed by the call first).
 * The softmax statistics are recomputed from Q, K, V and idx. Same limits and
 * errors as pisa_sparse_attn. */
int pisa_sparse_attn_backward(const pisa_cfg *cfg, const void *Q, const void *K, const void *V,
                              const int32_t *idx, const void *dO, float *dQ, float *dK, float *dV,
                              void *stream);

/* The whole prefill path, in order on one stream: pisa_build_pyramid, then
 * pisa_select, then pisa_sparse_attn. pyr and idx are caller-owned outputs. */
int pisa_forward(const pisa_cfg *cfg, const void *Q, const void *K, const void *V,
                 float *pyr, int32_t *idx, void *O, void *stream);

/* Flat block selection, the quadratic comparison (close reading §02, Eq.(1)):
 * every eligible leaf is scored by q . kbar_i / sqrt(d) against its mean
 * summary (summed over the G heads), with the same forced/causal rules and
 * ranking key as pisa_select. Reads only level 1 of pyr.
 * Q: [B, Hq, N, d]; idx: int32 [B, Hkv, N, K] (written). */
int pisa_bsa_select(const pisa_cfg *cfg, const void *Q, const float *pyr, int32_t *idx,
                    void *stream);
/* Flat BSA selection (close reading §02, Eq.(1)) on the tensor cores: the
 * same selection as pisa_bsa_select (forced leaves first, the best eligible
 * leaves by the mean-summary dot summed over the group, ties to the lower
 * leaf; idx sorted ascending, -1 padded), computed as S = Q x leaves^T per tile
 * of 128 (position, head) rows with a streaming Top-K. Rows whose K-th and
 * (K+1)-th scores differ by less than about 1e-5 may differ from the CUDA-core
 * call (the summaries enter as bf16 high and low parts). Limits and workspace
 * as pisa_select_ws (bf16, d = 128, C = 64; pisa_workspace_bytes bytes,
 * 256-byte aligned; it uses the workspace's pyramid-split region);
 * pisa_workspace_status reports a tile that gave up a bounded wait. */
int pisa_bsa_select_ws(const pisa_cfg *cfg, const void *Q, const float *pyr, int32_t *idx, void *workspace,
                       size_t workspace_bytes, void *stream);

/* ---- block-major tensor-core prefill (close reading §05 Algorithm 1, §5.1) ------
 * The pages' two-stage form: Stage 1 walks the internal levels (here the
 * coarse ones for tiles of consecutive positions on the tensor cores, the fine
 * ones per query); Stage 2 groups the (query, candidate leaf) pairs by leaf so that each leaf's
 * 64 keys are loaded once per tile of up to 128 query rows and scored with one
 * tcgen05 MMA (exact leaf LSE in the epilogue, Eq.(7)); a final Top-K per
 * query follows. Attention runs the same way: per (leaf, tile of queries that
 * kept it) S = Q K^T and O += softmax-weighted V on the tensor cores, using the
 * per-query normaliser taken from the leaf LSEs. Results equal pisa_select /
 * pisa_sparse_attn up to fp32 rounding (a row whose keep decision has a
 * margin below about 1e-5 may differ: the tile walk takes the fp32 summaries
 * as bf16 high and low parts).
 * Limits: dtype bf16, d = 128, C = 64, K <= 16, G in {1,2,4,8,16}, N < 2^27,
 * B * Hkv * N * 32 < 2^31, B * Hkv <= 65535. Other shapes return
 * PISA_E_UNSUPPORTED. The pyramid pointer must be 32-byte aligned (its rows are
 * read with 256-bit loads), else PISA_E_ALIGNMENT.
 * Workspace: caller-owned device memory of pisa_workspace_bytes(cfg) bytes,
 * 256-byte aligned; its contents are scratch (overwritten by every call, nothing
 * persists between calls except what pisa_forward_ws passes from its selection
 * to its attention). Calls sharing one workspace must not overlap on the GPU. */

/* Bytes of workspace the *_ws calls need for cfg (negative status on error). */
int64_t pisa_workspace_bytes(const pisa_cfg *cfg);

/* Waits for `stream`, then reads the error word the *_ws kernels leave in the
 * workspace: PISA_OK, or PISA_E_TIMEOUT if a tensor-core tile gave up waiting
 * for its MMA (each wait is bounded to about one second; the tile's output is
 * then left unwritten). Synchronous; for tests and diagnostics. */
int pisa_workspace_status(const pisa_cfg *cfg, const void *workspace, void *stream);

/* Same contract and outputs as pisa_select, block-major on the tensor cores. */
int pisa_select_ws(const pisa_cfg *cfg, const void *Q, const void *K, const float *pyr, int32_t *idx,
                   void *workspace, size_t workspace_bytes, void *stream);

/* Same contract and output as pisa_sparse_attn, block-major on the tensor cores
 * (first scores the listed leaves for the per-query softmax normaliser). */
int pisa_sparse_attn_ws(const pisa_cfg *cfg, const void *Q, const void *K, const void *V, const int32_t *idx,
                        void *O, void *workspace, size_t workspace_bytes, void *stream);

/* pisa_build_pyramid, pisa_select_ws, then the attention of pisa_sparse_attn_ws
 * reusing the selection's leaf LSEs for the normaliser. */
int pisa_forward_ws(const pisa_cfg *cfg, const void *Q, const void *K, const void *V, float *pyr, int32_t *idx,
                    void *O, void *workspace, size_t workspace_bytes, void *stream);

/* pisa_forward_ws from and to HOST memory: copies Q_host, K_host, V_host
 * (layouts as above) into the caller's device buffers Q, K, V, runs
 * pisa_forward_ws, and copies idx and O back into idx_host and O_host, all
 * enqueued on `stream` (one cudaMemcpyAsync per tensor). The host buffers
 * should be page-locked (cudaHostAlloc / pinned) for the copies to be
 * asynchronous; the call returns before they complete. Callers that keep two
 * sets of device buffers on two streams overlap one step's copies with the
 * other step's kernels. Same limits and errors as pisa_forward_ws; null host
 * pointers give PISA_E_INVALID. */
int pisa_forward_host(const pisa_cfg *cfg, const void *Q_host, const void *K_host, const void *V_host,
                      int32_t *idx_host, void *O_host, void *Q, void *K, void *V, float *pyr, int32_t *idx,
                      void *O, void *workspace, size_t workspace_bytes, void *stream);

/* pisa_forward_ws that also records caller-created CUDA events (cudaEvent_t
 * passed as void*, NULL entries skipped) on `stream` at its phase boundaries,
 * for per-phase timing with cudaEventElapsedTime. Index i marks the start of
 * phase i: 0 pyramid, 1 stage 1 (internal levels), 2 grouping of candidates,
 * 3 leaf scoring tiles, 4 final Top-K, 5 grouping of kept leaves, 6 forced
 * leaves (dense tiles), 7 attention tiles, 8 output conversion; index 9 marks
 * the end. n_events <= 10 are used. Records only: no synchronisation, no
 * allocation. */
#define PISA_NUM_PHASES 9
int pisa_forward_ws_events(const pisa_cfg *cfg, const void *Q, const void *K, const void *V, float *pyr,
                           int32_t *idx, void *O, void *workspace, size_t workspace_bytes, void *const *events,
                           int n_events, void *stream);

/* Backward of the attention with the selection idx held fixed, block-major on
 * the tensor cores: same contract, inputs and outputs as
 * pisa_sparse_attn_backward (dQ fp32 [B, Hq, N, d]; dK, dV fp32 [B, Hkv, N, d];
 * all three are zeroed by the call first). Steps, all on `stream`: the
 * (query, leaf) pairs of idx are grouped by leaf (each leaf's forced positions
 * first); a statistics pass over those tiles computes S = Q K^T and dP = dO V^T
 * and, per pair, the leaf's log-sum-exp and P-weighted dP, combined per
 * (query, head) into the normaliser L and D = sum_j p_j dp_j (= dO . o); then
 * per tile: P = softmax weights, dS = P (dP - D) in bf16, dV += P^T dO and
 * dK += dS^T Q accumulated on chip across the leaf's tiles, dQ += dS K added to
 * its rows. P and dS enter the tensor cores
 * as bf16 (as the forward's P does), so results equal the CUDA-core call to
 * within bf16 rounding of those operands, not bit for bit.
 * Limits and alignment as the other *_ws calls (bf16, d = 128, C = 64, ...).
 * Workspace: pisa_backward_workspace_bytes(cfg) bytes, 256-byte aligned;
 * pisa_workspace_status reads its error word as for the other *_ws calls. */
int64_t pisa_backward_workspace_bytes(const pisa_cfg *cfg);
int pisa_sparse_attn_backward_ws(const pisa_cfg *cfg, const void *Q, const void *K, const void *V,
                                 const int32_t *idx, const void *dO, float *dQ, float *dK, float *dV,
                                 void *workspace, size_t workspace_bytes, void *stream);
/* pisa_sparse_attn_backward_ws without the statistics pass, for training
 * steps that keep the forward's workspace: the workspace must hold what
 * pisa_forward_ws or pisa_sparse_attn_ws left in it for the same cfg, Q, K, V
 * and idx, with nothing else run on it since (it must be at least
 * pisa_backward_workspace_bytes(cfg) bytes for both calls). Those calls leave
 * the normaliser, the fp32 output (D = dO . O is taken from it) and the
 * grouping of the selected leaves there, so the statistics pass is skipped.
 * Results and limits as pisa_sparse_attn_backward_ws; the contents are not
 * checked. */
int pisa_sparse_attn_backward_saved_ws(const pisa_cfg *cfg, const void *Q, const void *K, const void *V,
                                       const int32_t *idx, const void *dO, float *dQ, float *dK, float *dV,
                                       void *workspace, size_t workspace_bytes, void *stream);
/* pisa_sparse_attn_backward_ws recording caller events (as
 * pisa_forward_ws_events) at its phase boundaries: 0 statistics (grouping,
 * tile list, statistics pass, combine), 1 zeroing of the gradients,
 * 2 backward tiles; index 3 marks the end. */
#define PISA_NUM_BWD_PHASES 3
int pisa_sparse_attn_backward_ws_events(const pisa_cfg *cfg, const void *Q, const void *K, const void *V,
                                        const int32_t *idx, const void *dO, float *dQ, float *dK, float *dV,
                                        void *workspace, size_t workspace_bytes, void *const *events,
                                        int n_events, void *stream);

/* Allocation-free selection. The pages have no counterpart to this call: it
 * exists for callers that cannot allocate device memory (a host application
 * that owns the GPU memory pool and gives plugins no allocator, serving loops
 * that forbid allocations after start-up, plain C callers without an
 * allocator). Same contract and outputs as pisa_select_ws, but its scratch is
 * a fixed array of PISA_NOALLOC_SCRATCH_BYTES compiled into the library (held
 * on every GPU that loads the library until the process exits) instead of a
 * caller workspace; it calls no allocating routine.
 * - Problems whose selection scratch exceeds that size return
 *   PISA_E_SCRATCH_LIMIT (about 73 K query units B*Hkv*N for G = 1).
 * - The first call in a CUDA context (a device's primary context, or one the
 *   caller made current through the driver API) looks up the array's device
 *   address there, with that context current; make it before any stream
 *   capture. A failed lookup is retried on the next call.
 * - All calls in a context share the array and it keeps the previous call's
 *   contents; each call clears what must start at zero. Calls that overlap on
 *   the GPU (other streams, other threads) race on the array: serialise them. */
#define PISA_NOALLOC_SCRATCH_BYTES (32u << 20)
int pisa_select_noalloc(const pisa_cfg *cfg, const void *Q, const void *K, const float *pyr, int32_t *idx,
                        void *stream);
/* Error word of the last pisa_select_noalloc on this device (no counterpart on
 * the pages, like the call itself): synchronises `stream` and returns PISA_OK,
 * or PISA_E_TIMEOUT when a tensor-core tile gave up a bounded wait or a
 * self-check of the selection failed (its idx is then not to be used).
 * `cfg` must be the configuration of that call; the same size limits apply. */
int pisa_select_noalloc_status(const pisa_cfg *cfg, void *stream);

/* ---- decode path (close reading §5.1 last paragraph; §5.3 "decode cache") ----
 * For decode calls cfg->N is the cache CAPACITY: Kc, Vc: [B, Hkv, N, d] and the
 * pyramid is laid out for length N (pisa_pyramid_rows(cfg) rows per head).
 * pos: int32 [B] device array, the position n of each sequence's new token
 * (its cache length before the append). Rows with pos[b] outside [0, N) are
 * left untouched by the append and produce idx = -1 and o = 0 in the step. */

/* Pyramid of the first len[b] keys of each cached sequence (len: int32 [B]
 * device array, values clamped to [0, N]), laid out for capacity N. */
int pisa_build_pyramid_prefix(const pisa_cfg *cfg, const void *Kc, const int32_t *len,
                              float *pyr, void *stream);

/* Grow a decode pyramid cache (close reading §5.3: the cache's capacity grows
 * by a fixed ratio as tokens arrive; the caller picks the new capacity, e.g.
 * twice the old one). pyr_old is laid out for cfg_old->N, pyr_new (a separate
 * caller buffer of pisa_pyramid_rows(cfg_new) rows per (b, kv-head)) for
 * cfg_new->N >= cfg_old->N; every other cfg field must match. Every summary of
 * the old pyramid, for any lengths up to the old capacity, lands where the
 * new layout keeps it (the levels added above the old root repeat the old
 * root); rows past the old capacity are zeroed. The caller copies its K/V
 * cache rows into caches of the new capacity itself. Mismatched configs, a
 * smaller new capacity or pyr_new == pyr_old give PISA_E_INVALID. */
int pisa_pyramid_grow(const pisa_cfg *cfg_old, const float *pyr_old, const pisa_cfg *cfg_new, float *pyr_new,
                      void *stream);

/* Geometric capacity policy of a growing decode cache (close reading §5.3:
 * capacity grows by a fixed ratio, so the upkeep stays amortised O(1) copies
 * per token): the smallest C * 2^k (k >= 0) that holds n keys. Host only, no
 * GPU; PISA_E_INVALID for n < 0 or C <= 0, PISA_E_UNSUPPORTED past 2^41. */
int64_t pisa_cache_capacity(int64_t n, int C);

/* Grow a whole decode cache: K and V caches ([B, Hkv, cfg_old->N, d] of the
 * cfg dtype) are copied into caches of capacity cfg_new->N (rows from the old
 * capacity on are zeroed) and the pyramid is re-laid out as pisa_pyramid_grow
 * does; all on `stream`, in the library's kernels. The caller allocates the
 * new buffers (pisa_cache_capacity gives the size to grow to) and keeps its
 * per-sequence positions. Config rules as pisa_pyramid_grow; null, aliased
 * (new == old, or K and V sharing a buffer) pointers give PISA_E_INVALID,
 * pointers not 16-byte aligned PISA_E_ALIGNMENT. From an empty cache
 * (cfg_old->N == 0) there is nothing to move: the call returns PISA_OK and
 * leaves the new buffers as they are (the caller zeroes them). */
int pisa_cache_grow(const pisa_cfg *cfg_old, const void *Kc_old, const void *Vc_old, const float *pyr_old,
                    const pisa_cfg *cfg_new, void *Kc_new, void *Vc_new, float *pyr_new, void *stream);

/* Append one token per sequence: k_new, v_new [B, Hkv, d] are written to cache
 * row pos[b]; the leaf holding pos[b] and each of its ancestors is recomputed
 * as the mean of what exists at length pos[b] + 1 (O(C + L) work per head). */
int pisa_pyramid_append(const pisa_cfg *cfg, void *Kc, void *Vc, float *pyr,
                        const void *k_new, const void *v_new, const int32_t *pos,
                        void *stream);

/* One fused decode step (close reading §5.1: a single-stage kernel per query
 * that walks the levels, scores the leaves and attends): for each sequence b
 * and KV head, select K leaves for the query q_new[b] at t = pos[b] against
 * the first pos[b] + 1 cached keys, then attend over them.
 * q_new: [B, Hq, d]; idx: int32 [B, Hkv, K] (written); o: [B, Hq, d] (written). */
int pisa_decode(const pisa_cfg *cfg, const void *q_new, const void *Kc, const void *Vc,
                const float *pyr, const int32_t *pos, int32_t *idx, void *o, void *stream);

/* pisa_pyramid_append followed by pisa_decode, as one kernel launch: the whole
 * decode step of the close reading's §5.3 (append the token, update the leaf
 * and its ancestors, then select and attend for the new query). Same
 * arguments, layouts and results as the two calls in sequence (up to fp32
 * summation order in the updated summaries). The append reuses the step's
 * shared memory and overlaps its first walk levels, which never read the
 * rows it rewrites (the new token's leaf and its ancestors are forced nodes). */
int pisa_decode_step(const pisa_cfg *cfg, const void *q_new, const void *k_new, const void *v_new,
                     void *Kc, void *Vc, float *pyr, const int32_t *pos, int32_t *idx, void *o,
                     void *stream);

/* ---- misc --------------------------------------------------------------------- */

/* Static English text for a status code (never NULL). */
/* ---- measurement ----
 * CUDA-core fp32 FMA throughput probe (no counterpart on the pages): `blocks`
 * blocks of 256 threads, each thread running 8 independent chains of
 * 4 * `iters` FMAs, scalar (`packed` = 0) or packed fp32x2 (`packed` = 1);
 * FLOP per launch = blocks * 256 * iters * 64 (x2 when packed). `out` receives
 * blocks * 256 floats (device memory, caller-owned). Returns PISA_E_INVALID on
 * a null `out` or non-positive sizes. Used to measure the peak that the walk
 * kernels' arithmetic is compared against. */
int pisa_fma_probe(float *out, int blocks, int iters, int packed, void *stream);

const char *pisa_status_string(int status);
/* Library version string, e.g. "pisa-b200 0.1.0 sm_100a". */
const char *pisa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PISA_H */
