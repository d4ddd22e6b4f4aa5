/*
 * spava.h -- C ABI of libspava: B200 (sm_100a) kernels for the per-host
 * approximate attention of APB-V / Spava long-video prefill, with every ZigZag
 * virtual host on one GPU.
 *
 * Method source: "Riepilogo Tecnico: APB-V" (gist.science/it/paper/2601.21444),
 * section "Metodologia: APB-V" -- 1. "Design del Framework" (context split into
 * anchor block, query block and context blocks; ZigZag pairing of virtual hosts
 * h and 2H-1-h; passing blocks of the most essential KV found by query-to-context
 * attention scores; attention over anchor, local context, aggregated passing
 * blocks and query) and 2. "Ottimizzazioni a Livello di Sistema" ("Forward Fuso
 * di Contesto e Query": query partial results merged through log-sum-exp;
 * "Bilanciamento del Carico dell'Attenzione Approssimata").  Also "Spava:
 * Accelerating Long-Video Understanding via Sequence-Parallelism-aware
 * Approximate Attention", abstract.
 *
 * Conventions shared by every entry point
 *   - Tensors are DEVICE pointers unless the name says host, contiguous,
 *     token-major: Q [N, Hq, d], K and V [N, Hkv, d], O [N, Hq, d], all bf16
 *     (passed as void*), and 16-byte aligned.  lse is float32 [Hq, N], natural
 *     log.  scores are float32 [Hkv, C], C = N - a - q, context token t at
 *     column t - a.  idx is int32 [2H-1, Hkv, l]: absolute token positions,
 *     ascending, padded with -1.  Packed passing K/V are bf16 [Hkv, L, d] with
 *     L = a + sum_u min(l, n_u): the anchor rows first, then P_0, P_1, ...
 *   - The caller owns every buffer.  The library allocates no device or host
 *     memory, frees nothing and never synchronises the stream (except
 *     spava_device_status, which says so).
 *   - Calls are asynchronous and ordered on `stream` (a cudaStream_t; NULL is
 *     the legacy default stream).
 *   - Arguments are checked before any launch; on error nothing is launched
 *     and the status says why.  SPAVA_ERR_CUDA means a CUDA runtime call
 *     failed; spava_last_cuda_error() returns its code (per thread).
 *   - Kernels never trap.  A wait inside a kernel that exceeds its bound sets a
 *     flag in the workspace status word and the kernel returns early; read it
 *     with spava_device_status().
 *   - Thread-safe: no mutable global state besides per-thread error codes and
 *     the once-per-process kernel attribute set-up.
 */
#ifndef SPAVA_H_
#define SPAVA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SPAVA_OK = 0,
    SPAVA_ERR_INVALID_ARG = 1, /* a size, offset or pointer is invalid */
    SPAVA_ERR_UNSUPPORTED = 2, /* valid, but outside what the library supports (d, H, ...) */
    SPAVA_ERR_MISALIGNED = 3,  /* a device pointer is not 16-byte aligned */
    SPAVA_ERR_WORKSPACE = 4,   /* workspace missing or smaller than required */
    SPAVA_ERR_CUDA = 5,        /* a CUDA runtime call failed */
    SPAVA_ERR_TIMEOUT = 6      /* a kernel-side bounded wait gave up */
} spava_status;

/* One prefill attention layer.  Sequence split of "Suddivisione del Contesto e
 * Disposizione ZigZag": [anchor a | 2H context chunks | query block q]. */
typedef struct {
    int32_t H;            /* physical hosts = virtual-host pairs; 2H chunks; 1..32 */
    int32_t n_q_heads;    /* Hq */
    int32_t n_kv_heads;   /* Hkv; Hq % Hkv == 0, q-head h uses KV head h / (Hq/Hkv) */
    int32_t head_dim;     /* d: 64 or 128 */
    int64_t n_tokens;     /* N < 2^31 */
    int64_t anchor_len;   /* a >= 0 */
    int64_t query_len;    /* q >= 1 */
    const int64_t *chunk_offsets; /* HOST array [2H+1]: off[0]=a, off[2H]=N-q,
                                     strictly increasing; chunk v = [off[v], off[v+1]) */
    int32_t top_l;        /* l >= 0: passing-block size per KV head per chunk */
    float scale;          /* softmax scale; <= 0 selects 1/sqrt(d) */
    int32_t local_pair_full; /* 1: the later virtual host of a ZigZag pair sees its
                                partner chunk in full and takes no passing block from
                                it; 0: every virtual host takes the passing blocks of
                                all earlier chunks and no full partner chunk */
    /* Selection variants (ablations of the score reading; the pages fix
     * neither): */
    int32_t score_norm;   /* 0 (default): each query row's softmax over the chunk
                             being scored; 1: the row's own attention weights,
                             normalised over every key it attends, [0, t] */
    int32_t score_pool;   /* 0 or 1 (default): rank the scores themselves; odd w
                             in 3..255: rank each key by the sum of the scores of
                             the w keys centred on it inside its chunk (the w-key
                             window mean with zero padding, up to the factor 1/w);
                             spava_score still returns the unpooled scores */
} spava_config;

/* Workspace bytes that any entry point below needs for this config (the
 * largest of them: spava_prefill_attention).  Pass the same buffer to every
 * call; it must be 256-byte aligned.  Its first 256 bytes are the status block:
 * the status word at byte 0 (must start at zero; see spava_device_status) and
 * the work-item counter of the attention kernel's persistent grid at byte 128
 * (zeroed by every spava_attn before its launch).  Calls that share a
 * workspace must be ordered on one stream. */
spava_status spava_workspace_size(const spava_config *cfg, size_t *bytes);

/* L = a + sum_u min(l, n_u): rows of the packed passing K/V per KV head. */
spava_status spava_packed_len(const spava_config *cfg, int64_t *rows);

/* Query-to-context scores ("Blocchi di Passaggio"): for every chunk u < 2H-1,
 * KV head g and key j of chunk u,
 *   scores[g, j-a] = sum_{h in group g} sum_{i in query block}
 *                    softmax_{j' in chunk u}(scale * q_{h,i} . k_{g,j'}) at j'=j.
 * The softmax runs over chunk u only (score_norm 0); no causal mask.  With
 * score_norm 1 each row's weights are instead normalised over every key the
 * row attends, [0, t].  The last chunk has no successor and its columns are
 * left untouched.  Two passes over K: row statistics, then probability column
 * sums.  Reads q, k; writes scores. */
spava_status spava_score(const spava_config *cfg, const void *q, const void *k, float *scores,
                         void *ws, size_t ws_bytes, void *stream);

/* Passing-block selection ("Blocchi di Passaggio": the most essential KV): for
 * every chunk u < 2H-1 and KV head g, the min(l, n_u) largest scores of chunk u
 * (with score_pool w >= 3: the largest sums of the w scores centred on each key
 * inside the chunk, added in ascending order in fp32; ties: the lower token
 * index wins), written as ascending absolute positions into idx[u, g, :], the
 * remaining slots set to -1.  Exact: no approximation in the selection. */
spava_status spava_topk_select(const spava_config *cfg, const float *scores, int32_t *idx,
                               void *stream);

/* Passing-block aggregation ("aggregate in blocchi di passaggio"): pk[g, r] =
 * k[r, g] for r < a (anchor), then for each chunk u the rows k[idx[u,g,s], g],
 * s < min(l, n_u), in that order; pv likewise from v.  On one GPU this gather
 * replaces the cross-host transfer of the passing blocks. */
spava_status spava_pack_passing(const spava_config *cfg, const void *k, const void *v,
                                const int32_t *idx, void *pk, void *pv, void *stream);

/* Approximate attention ("Computazione") with online softmax:
 *   anchor row t < a:        keys [0, t]
 *   context row t, chunk v:  anchor + passing blocks of the earlier chunks
 *                            (local_pair_full=1: those on another physical host)
 *                            + partner chunk 2H-1-v in full (v >= H,
 *                            local_pair_full=1) + own chunk up to t
 *   query row t >= N-q:      keys [0, t], computed as one partial per segment
 *                            (anchor, each chunk, query block) merged by
 *                            log-sum-exp ("Forward Fuso di Contesto e Query").
 * Writes o [N, Hq, d] bf16 and, if lse != NULL, lse [Hq, N] float32. */
spava_status spava_attn(const spava_config *cfg, const void *q, const void *k, const void *v,
                        const void *pk, const void *pv, void *o, float *lse, void *ws,
                        size_t ws_bytes, void *stream);

/* The whole layer, in the order of the fused forward ("Forward Fuso di
 * Contesto e Query"): first the anchor rows and the query rows' per-segment
 * partials, whose per-chunk log-sum-exps are the scoring's normaliser; then
 * scoring, selection and gather of every passing block in one launch; then the
 * context rows and the query-row merge.  Scores, idx and the packed K/V stay in
 * the workspace.  The outputs equal, byte for byte, those of spava_score ->
 * spava_topk_select -> spava_pack_passing -> spava_attn.  If idx_out != NULL
 * the passing-block indices are also written there. */
spava_status spava_prefill_attention(const spava_config *cfg, const void *q, const void *k,
                                     const void *v, void *o, float *lse, int32_t *idx_out,
                                     void *ws, size_t ws_bytes, void *stream);

/* spava_prefill_attention from HOST buffers: copies q_host, k_host, v_host
 * into the caller's device buffers q, k, v, runs the layer, and copies o (and
 * lse if both lse and lse_host are non-NULL) back to o_host / lse_host.
 * Host buffers should be page-locked for the copies to be asynchronous; the
 * call does not wait for them.
 * copy_stream NULL (or equal to stream): everything is ordered on `stream`.
 * Otherwise the copies run on copy_stream, overlapped with the kernels,
 * chunk by chunk in token order: the query block's Q rows and the anchor go up
 * first, then each chunk's Q, K and V rows; once a chunk (and the rows its last
 * 128-row tile reaches into) has arrived, its passing block is scored, selected
 * and gathered and its rows are computed, and its O (and lse) rows go down
 * while later chunks compute; the query block's rows come last.  The kernels
 * of this mode run on three streams the call creates and destroys: scoring at
 * the device's highest stream priority, and the attention launches alternating
 * between two others, each launch waiting only for its rows and the passing
 * blocks before them, so that one launch's CTAs take the SMs its
 * predecessor's last work items leave idle.
 * (With score_norm 1 -- whose statistics need every segment first -- K and the
 * query block's Q rows go up first, then V, and the attention runs in up to 8
 * groups of whole regions as their Q rows arrive.)  The outputs equal
 * spava_prefill_attention's byte for byte.  The copies begin only after
 * all work already enqueued on `stream` (an earlier call may still be reading
 * the device buffers), and `stream` is made to wait for the last copy, so the
 * call's work is complete when `stream` is and back-to-back calls on the same
 * buffers stay ordered.  The call creates and destroys its own CUDA events
 * and streams (no memory).  Neither stream may be capturing a graph.  On an error return, work
 * already enqueued may still run. */
spava_status spava_prefill_attention_host(const spava_config *cfg, const void *q_host,
                                          const void *k_host, const void *v_host, void *o_host,
                                          float *lse_host, void *q, void *k, void *v, void *o,
                                          float *lse, void *ws, size_t ws_bytes, void *stream,
                                          void *copy_stream);

/* Synchronises `stream`, reads the workspace status word (bit 0: a bounded wait
 * in a kernel gave up), writes it to *flags and clears it.  Returns
 * SPAVA_ERR_TIMEOUT if bit 0 was set, SPAVA_OK otherwise. */
spava_status spava_device_status(void *ws, size_t ws_bytes, void *stream, int32_t *flags);

/* Self-test of the failure path (the pages have no counterpart): launches one
 * thread that waits on a barrier nothing arrives on.  Its bounded wait gives up
 * after about two seconds, sets bit 0 of the workspace status word and the
 * kernel returns, leaving the context usable; spava_device_status() then
 * reports SPAVA_ERR_TIMEOUT and clears the bit.  Needs the first 256 bytes of a
 * workspace (256-byte aligned). */
spava_status spava_selftest_wait_timeout(void *ws, size_t ws_bytes, void *stream);

/* Exact number of (row, key) pairs per query head that spava_attn attends,
 * by row class: pairs[0] anchor rows, pairs[1] context rows, pairs[2] query
 * rows.  Algorithmic FLOPs of spava_attn = 4 * d * Hq * (sum of the three).
 * per_host (may be NULL) receives H entries: the context pairs of each
 * physical host, i.e. of its two virtual hosts p and 2H-1-p (ZigZag balance,
 * "Bilanciamento del Carico dell'Attenzione Approssimata").  Host only. */
spava_status spava_attended_pairs(const spava_config *cfg, int64_t pairs[3], int64_t *per_host);

/* Chunk offsets from a frame list ("Riepilogo Tecnico: APB-V", Metodologia,
 * "Bilanciamento del Carico Visivo": the frames are spread evenly over the
 * virtual hosts).  frame_tokens: HOST array of the n_frames frames' token
 * counts, in order (each >= 1); the 2H chunks take consecutive whole frames,
 * chunk v taking floor(n_frames / 2H) frames plus one more for
 * v < n_frames mod 2H.  Writes chunk_offsets[0..2H] (HOST, int64):
 * off[0] = anchor_len, off[v+1] = off[v] + the tokens of chunk v's frames, so a
 * layer built from them has N = off[2H] + query_len.  SPAVA_ERR_INVALID_ARG if
 * H is outside 1..32, n_frames < 2H (a chunk would be empty), a frame has no
 * token, anchor_len < 0, a pointer is NULL or the sum passes 2^31.  Host only. */
spava_status spava_plan_chunks(int32_t H, const int64_t *frame_tokens, int64_t n_frames,
                               int64_t anchor_len, int64_t *chunk_offsets);

/* ---------------------------------------------------------------------------
 * Multi-GPU ZigZag sequence parallelism ("Riepilogo Tecnico: APB-V",
 * Metodologia, "Suddivisione del Contesto e Disposizione ZigZag": physical host
 * p holds virtual hosts p and 2H-1-p; Ottimizzazioni a Livello di Sistema,
 * "Comunicazione Sovrapposta": the passing blocks travel between hosts while
 * the hosts compute, and "Forward Fuso di Contesto e Query": the query rows'
 * partial results of every host are merged through their log-sum-exp).
 *
 * `world` GPUs, one process each; H % world == 0.  Rank r holds the physical
 * hosts p in [r*m, (r+1)*m), m = H/world -- the chunks v with
 * pair(v) / m == r, pair(v) = v < H ? v : 2H-1-v -- plus the anchor and the
 * query block, which every rank holds.  Its token-major buffers (q, k, v, o:
 * [n_local, heads, d]; lse: [Hq, n_local]) are LOCAL: [anchor | its chunks in
 * increasing v | query block].  A rank computes its chunks' context rows, and
 * (like every rank) the anchor rows and the query rows.
 *
 * One layer on each rank, in this order (all on `stream`, asynchronous):
 *   spava_shard_front        scores, top-l and gather of its chunks' passing
 *                            blocks; writes its pass message
 *   all-gather #1            the caller gathers every rank's pass message,
 *                            rank-major, into pass_all (e.g. NCCL
 *                            all-gather into this GPU's own memory)
 *   spava_shard_local_attn   anchor rows and the query rows' partials over
 *                            the anchor, its chunks and the query block: needs
 *                            nothing from other ranks, so it runs while
 *                            all-gather #1 is in flight; writes its part message
 *   all-gather #2            every rank's part message into part_all
 *   spava_shard_context_attn unpacks pass_all, then the context rows of its
 *                            chunks (runs while all-gather #2 is in flight)
 *   spava_shard_merge        unpacks part_all, merges the query rows
 * The messages have the same size on every rank (spava_shard_sizes).  The
 * outputs equal spava_prefill_attention's rows bit for bit.  score_norm 1 is
 * not offered (SPAVA_ERR_UNSUPPORTED): it needs every chunk's statistics of the
 * query rows before scoring.  The same workspace serves all four calls of a
 * rank; the caller keeps pass_send / part_send unchanged until its gathers
 * have read them.
 * ------------------------------------------------------------------------- */

/* Host only.  local_first (HOST [2H+2], may be NULL): first local row of the
 * anchor (index 0), chunk v (1+v), the query block (2H+1), -1 where the rank
 * does not hold the region; *n_local: rows of its local buffers; slot_chunk
 * (HOST [2H/world], may be NULL): the chunk in each slot of its messages.
 * SPAVA_ERR_INVALID_ARG for rank outside [0, world) or world < 1,
 * SPAVA_ERR_UNSUPPORTED if world does not divide H or score_norm is 1. */
spava_status spava_shard_layout(const spava_config *cfg, int32_t rank, int32_t world,
                                int64_t *local_first, int64_t *n_local, int32_t *slot_chunk);

/* Host only: workspace bytes of a rank (256-byte aligned buffer, first 256
 * bytes the status block as for spava_workspace_size), and the bytes of one
 * rank's pass and part messages (pass_all / part_all hold world of each). */
spava_status spava_shard_sizes(const spava_config *cfg, int32_t world, size_t *ws_bytes,
                               size_t *pass_msg_bytes, size_t *part_msg_bytes);

/* Reads local q, k, v; writes pass_send (device, 16-byte aligned,
 * pass_msg_bytes): per slot the indices and the K and V rows of that chunk's
 * passing block. */
spava_status spava_shard_front(const spava_config *cfg, int32_t rank, int32_t world, const void *q,
                               const void *k, const void *v, void *pass_send, void *ws,
                               size_t ws_bytes, void *stream);

/* Writes the anchor rows of o / lse and part_send (device, part_msg_bytes):
 * the query rows' partials over this rank's chunks. */
spava_status spava_shard_local_attn(const spava_config *cfg, int32_t rank, int32_t world,
                                    const void *q, const void *k, const void *v, void *o, float *lse,
                                    void *part_send, void *ws, size_t ws_bytes, void *stream);

/* Reads pass_all (device, world * pass_msg_bytes, rank-major); writes the
 * context rows of this rank's chunks into o / lse, and, if idx_out != NULL,
 * every chunk's passing-block indices [2H-1, Hkv, l]. */
spava_status spava_shard_context_attn(const spava_config *cfg, int32_t rank, int32_t world,
                                      const void *q, const void *k, const void *v,
                                      const void *pass_all, void *o, float *lse, int32_t *idx_out,
                                      void *ws, size_t ws_bytes, void *stream);

/* Reads part_all (device, world * part_msg_bytes, rank-major); writes the
 * query rows of o / lse. */
spava_status spava_shard_merge(const spava_config *cfg, int32_t rank, int32_t world,
                               const void *part_all, void *o, float *lse, void *ws, size_t ws_bytes,
                               void *stream);

/* spava_score for callers that cannot allocate device memory: same inputs,
 * same scores output, no workspace argument.  (The pages have no counterpart:
 * this is an interface choice of the library, not part of the method.)
 * Who needs it: code that is handed only its input and output buffers, such
 * as a plug-in inside an engine that owns all device memory, or code that must
 * not allocate after start-up (real-time or certified deployments, or a
 * latency-critical path where cudaMalloc would synchronise the device).
 * The scratch for the per-chunk softmax statistics is a fixed 4 MiB array
 * compiled into the library (each GPU that loads the library holds it until
 * the process exits).  Limit: 256 + 4*(2H-1)*Hq*q bytes must fit in 4 MiB
 * (e.g. H=16, Hq=32, q=512 needs 2 MiB); larger layers get
 * SPAVA_ERR_WORKSPACE and nothing is launched.  No allocation of any kind
 * (no cudaMalloc, cudaFree or allocating library routine).
 * Each call looks up the array's device address with the calling thread's
 * current device (cudaGetSymbolAddress; the first lookup on a device loads the
 * library's module there): make the first call on a device before any stream
 * capture.
 * All calls share the one array: calls that overlap on the GPU (other streams,
 * other host threads) race and must be serialised by the caller.  A kernel
 * wait that gives up is recorded in the array's status word, which each call
 * clears at its start; read it with spava_score_noalloc_status. */
spava_status spava_score_noalloc(const spava_config *cfg, const void *q, const void *k,
                                 float *scores, void *stream);

/* Status of the last spava_score_noalloc call on the current device (the
 * pages have no counterpart): synchronises `stream`, reads the status word of
 * the library's fixed scratch array (bit 0: a bounded wait in a kernel gave
 * up, the scores are incomplete), writes it to *flags and clears it.  Returns
 * SPAVA_ERR_TIMEOUT if bit 0 was set, SPAVA_OK otherwise.  Allocates nothing. */
spava_status spava_score_noalloc_status(void *stream, int32_t *flags);

const char *spava_status_string(spava_status s);

/* The CUDA error code of this thread's last SPAVA_ERR_CUDA (0 if none). */
int32_t spava_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* SPAVA_H_ */
