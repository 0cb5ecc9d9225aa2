/*
 * spark.h — C ABI of the B200 (sm_100a) block-sparse video attention forward.
 *
 * The method: "Spark-H3: speeding up MiniMax-H3 in ComfyUI with block-sparse
 * attention" (comfyui-wiki news, 2026-10-11), section "What Spark-Attn changes":
 * an exact branch over the top-ranked key/value blocks and a compressed branch that
 * covers the rest (Spark-Reweight), optionally over a data-dependent block layout
 * (Spark-Reblock). Block selection follows "ComfyUI adds a core sparse-attention node
 * and the Comfy Compiler" (comfyui-wiki news, 2026-09-08), section "Block-sparse
 * attention: one node, three backends" (top-k keep ratio; Sol-Attn per-head tau;
 * sink_conditioning), and the dense-row policy of the "H3 Optimizations" README,
 * section "Nodes".
 *
 * Conventions shared by every call
 * --------------------------------
 * - Q, K, V are contiguous [B, H, N, d] bf16 (passed as uint16_t bit patterns),
 *   16-byte aligned. Per (b, h) the first nb*64 rows are video rows, nb =
 *   floor((N - n_sink) / 64); all remaining rows (a ragged video tail shorter than
 *   one block, then the n_sink sink/text rows) are dense rows: their queries attend
 *   to every key and their keys are attended by every query. Dense rows are never
 *   pooled, scored, compressed or reblocked.
 * - block must be 64; d must be 64 or 128; scale <= 0 means 1/sqrt(d).
 * - Every pointer is a device pointer owned by the caller (spark_forward_host also takes
 *   host buffers); the library allocates no memory, keeps no state beyond one device-side
 *   error word (and the fixed scratch array of spark_score_select_noalloc), and never
 *   synchronises except in spark_device_error. Calls are asynchronous on `stream`
 *   (a cudaStream_t, NULL = legacy default stream) and re-entrant.
 * - Return value: SPARK_OK, or a negative status for arguments rejected on the host
 *   (nothing is launched then). Faults found by a kernel (an out-of-range block index
 *   supplied by the caller, a capacity overflow, a bounded wait that gave up) do not
 *   abort the launch: the kernel skips the offending work and records the first such
 *   status in the device error word, which spark_device_error reads and clears.
 */
#ifndef SPARK_H_
#define SPARK_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SPARK_OK 0
#define SPARK_EINVAL (-1)        /* bad shape, null pointer, alignment, ratio/tau, kcap */
#define SPARK_EUNSUPPORTED (-2)  /* d or block not supported, sizes beyond the limits */
#define SPARK_ECUDA (-3)         /* a CUDA launch failed */
#define SPARK_ETIMEOUT (-4)      /* device: a bounded wait gave up */
#define SPARK_EDEVICE_INDEX (-5) /* device: a selected block index was out of range */
#define SPARK_ECAPACITY (-6)     /* device: tau kept more blocks than kcap; list truncated */
#define SPARK_ESCRATCH (-7)      /* B*H beyond the static scratch of spark_score_select_noalloc */

#define SPARK_SELECT_TOPK_RATIO 0
#define SPARK_SELECT_TAU 1

#define SPARK_POOL_REWEIGHT 0 /* Spark-Reweight: softmax-weighted value summary + log-mass bias */
#define SPARK_POOL_MEAN 1     /* plain mean pooling: mean value, bias log(64) */

#define SPARK_CALL_POOL 0
#define SPARK_CALL_SELECT 1
#define SPARK_CALL_ATTN 2
#define SPARK_CALL_REBLOCK 3

typedef struct spark_shape {
  int32_t B, H, N, d; /* Q/K/V are [B, H, N, d] */
  int32_t n_sink;     /* sink/text rows at the end of each (b, h) */
  int32_t block;      /* video block size; must be 64 */
  float scale;        /* softmax scale; <= 0 selects 1/sqrt(d) */
  int32_t q_tile;     /* query tile of the route: 64 (0 means 64) or 128 */
} spark_shape;

/* The query tile ("H3 Optimizations" README, section "Manual Sparse Sage recovery": the
 * sparse backends consume a 128-query x 64-key route). With q_tile = 128 a query tile is
 * two consecutive video blocks (the last one holds one block when nb is odd): q_pool has
 * one row per tile (the mean of the tile's queries), the score and selection rows are the
 * nt = ceil(nb / 2) tiles against the nb key blocks (k = spark_topk_count(ratio, nb); tau
 * moments over all nt x nb scores), idx / cnt are [B, H, nt, kcap] / [B, H, nt], and every
 * query of a tile attends to the tile's selection. Keys, the anchor, the compressed branch,
 * the dense rows and Reblock do not change. With q_tile = 64, nt = nb. */
int32_t spark_num_query_tiles(const spark_shape* s);

/* Number of full video blocks nb = floor((N - n_sink) / 64) (0 when N <= n_sink). */
int32_t spark_num_blocks(const spark_shape* s);

/* Bytes of the caller-owned buffer that call `call_id` needs:
 *   SPARK_CALL_POOL    the pooled pack written by spark_pool_kv and read by
 *                      spark_attn_fwd: bf16 copies of k_pool and v_summ ([B*H*nb, d]
 *                      each) followed by beta * log2(e) in fp32 with each (b, h) row
 *                      padded to nbp = 64 * ceil(nb / 64) entries (-inf past nb):
 *                      2*B*H*nb*d*2 + B*H*nbp*4 bytes;
 *   SPARK_CALL_SELECT  scratch of spark_score_select: fp64 tau moments (2*B*H doubles,
 *                      padded to 256 bytes) and the score keys of every head
 *                      (B*H*nt*nbp uint32, nbp = nb rounded up to 4);
 *   SPARK_CALL_ATTN    scratch of spark_attn_fwd: 256 bytes (the launch's counter of
 *                      work items handed out to the CTAs; zeroed by the call);
 *   SPARK_CALL_REBLOCK scratch of spark_reblock.
 * Returns 0 for an invalid shape or call id. */
size_t spark_workspace_bytes(const spark_shape* s, int call_id);

/* Block-count rule of the top-k mode: k = min(nb, max(1, ceil(ratio*nb - 1e-9))),
 * evaluated in double precision. Returns -1 for ratio outside (0, 1]. */
int32_t spark_topk_count(double ratio, int32_t nb);

/* Pooling, anchor and compressed-branch summaries ("What Spark-Attn changes",
 * Spark-Reweight bullet and the figure caption after it).
 * Per (b, h):  q_pool[i]  = mean of the queries of query tile i           fp32 [B,H,nt,d]
 *              anchor     = mean of all video queries (the row-weighted mean of q_pool)
 *                                                                          fp32 [B,H,d]
 *              s_j        = anchor . k_j * scale for every video key j
 *              k_pool[i]  = mean of the 64 keys of block i                  fp32 [B,H,nb,d]
 *              v_summ[i]  = sum_j softmax_i(s)_j v_j (REWEIGHT) | mean v     fp32 [B,H,nb,d]
 *              beta[i]    = logsumexp_i(s) - anchor . k_pool[i] * scale      fp32 [B,H,nb]
 *                           (REWEIGHT) | log(64) (MEAN)
 * pool_pack (spark_workspace_bytes(s, SPARK_CALL_POOL) bytes, 16-byte aligned) receives
 * bf16 copies of k_pool and v_summ and a padded log2-scaled copy of beta, the operands
 * of the compressed branch in spark_attn_fwd.
 * Any of q_pool/k_pool/v_summ/anchor may not be NULL; all are written. */
int spark_pool_kv(const spark_shape* s, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                  int pool_mode, float* q_pool, float* k_pool, float* v_summ, float* beta,
                  float* anchor, void* pool_pack, size_t pool_pack_bytes, void* stream);

/* Block scores and selection ("Block-sparse attention: one node, three backends").
 * S[i, j] = q_pool[i] . k_pool[j] * scale for query tile i (a block unless q_tile = 128)
 * and video key block j, computed in fp32.
 *   mode SPARK_SELECT_TOPK_RATIO, param = ratio in (0, 1]: keeps the k =
 *       spark_topk_count(ratio, nb) largest scores of each row, ties to the lower j;
 *       requires kcap >= k.
 *   mode SPARK_SELECT_TAU, param = tau (finite): keeps S[i, j] > mu + tau * sigma,
 *       mu and sigma (population) over all nt*nb scores of the head, obtained in fp64
 *       from the d x d second moments of q_pool and k_pool. No per-row floor: a row
 *       may keep nothing. More than kcap kept blocks truncates the row to its first
 *       kcap indices in the row's order (below) and records SPARK_ECAPACITY (kcap = nb
 *       never overflows).
 * Outputs: idx int32 [B, H, nt, kcap], cnt int32 [B, H, nt]. Row i holds its cnt kept
 * block indices in the first cnt slots (later slots unspecified) in sweep order: ascending
 * from the first one at or above p_i = floor((i mod W) * nb / W) rounded down to a
 * multiple of 32, then the ones below p_i, ascending, with W the number of query tiles
 * spark_attn_fwd runs at once on the current device (2 per SM for q_tile = 64, 1 per SM
 * for q_tile = 128). spark_attn_fwd visits a row's blocks in the order given (any order is
 * valid input); in this one the tiles at work at any moment read K/V near one position of
 * the head. The order changes no kept set: top-k ties still go to the lower indices.
 * The scores are computed by a tiled fp32 kernel into ws and each row is selected from
 * there (per score: even and odd d terms in two fp32 chains, then scaled).
 * ws: spark_workspace_bytes(s, SPARK_CALL_SELECT) bytes, 16-byte aligned (both modes). */
int spark_score_select(const spark_shape* s, const float* q_pool, const float* k_pool, int mode,
                       double param, int32_t kcap, int32_t* idx, int32_t* cnt, void* ws,
                       size_t ws_bytes, void* stream);

/* Attention forward ("What Spark-Attn changes": exact + compressed branches merged in
 * one softmax; sink_conditioning: sink keys attended exactly; "Nodes": dense rows).
 * A video query of tile i attends to the 64 keys of each selected block idx[i, :cnt[i]]
 * and to every dense key; when pool_pack is not NULL it also attends to one pooled
 * entry per unselected video block b, with logit q . k_pool[b] * scale + beta[b] and
 * value v_summ[b] (bf16 k_pool / v_summ and fp32 beta, all read from pool_pack; the
 * `beta` argument is not read and may be NULL). Dense query rows attend
 * to every key and never to pooled entries. A row with nothing to attend to gets
 * O = 0 and LSE = -inf.
 * perm (nullable) int32 [B, H, nb*64]: the inputs are in a reblocked order and output
 * row p of a video query is written to original row perm[p] (dense rows unchanged).
 * Outputs: O bf16 [B, H, N, d]; lse fp32 [B, H, N] natural-log (nullable).
 * Block indices outside [0, nb) are skipped and recorded as SPARK_EDEVICE_INDEX.
 * q_tile = 64 runs 64-query tiles on M = 64 tensor-core MMAs, q_tile = 128 runs 128-query
 * tiles (dense rows too) on M = 128 MMAs; the 128-query kernel hands the tiles out to the
 * CTAs at run time, head by head (each head's dense-row tiles, the longest, lead its tiles).
 * extra_pack / extra_tokens: with extra_tokens > 0 the extra pack written by
 * spark_extra_tokens (same shape, same extra_tokens, 16-byte aligned, not NULL): every
 * video query also attends exactly to the head's extra tokens that lie outside its selected
 * blocks (those inside are attended as part of the block); dense query rows already attend
 * to every key and are unchanged. extra_tokens = 0: extra_pack is not read (may be NULL).
 * ws: spark_workspace_bytes(s, SPARK_CALL_ATTN) bytes, 16-byte aligned, not shared with a
 * launch in flight on another stream. */
int spark_attn_fwd(const spark_shape* s, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                   const int32_t* idx, const int32_t* cnt, int32_t kcap, const void* pool_pack,
                   const float* beta, const int32_t* perm, const void* extra_pack, int32_t extra_tokens,
                   uint16_t* O, float* lse, void* ws, size_t ws_bytes, void* stream);

/* Extra tokens ("ComfyUI adds a core sparse-attention node and the Comfy Compiler",
 * section "Block-sparse attention: one node, three backends": extra_tokens adds the
 * highest-scoring tokens beyond the selected blocks, to stay close to dense attention).
 * The pages give neither the score nor the count's unit; this library reads it as a
 * per-head budget E = min(extra_tokens, nb*64) of video keys ranked by the anchor score
 * s_j = anchor . k_j * scale (the per-token score of the compressed branch), ties to the
 * lower token index. Runs after spark_pool_kv on the same (reblocked) K, V and its anchor:
 *   - writes the extra pack: the tokens' row indices (ascending, int32 [B*H, ep], -1 past
 *     E; ep = 64 * ceil(E / 64)), the anchor scores of every video key (fp32 [B*H, nb*64])
 *     and the tokens' K and V rows (bf16 [B*H*ep, d] each, zero past E);
 *   - when pool_pack is not NULL, rewrites the compressed entry of every block that lost
 *     tokens so that it stands for the block's remaining tokens R_b only: bf16 key mean of
 *     R_b and value summary over R_b in pool_pack, log-mass bias lse(s over R_b) -
 *     anchor . mean_k(R_b) * scale (pool_mode SPARK_POOL_MEAN: mean value of R_b and
 *     log |R_b|) in pool_pack and in v_summ / beta when those are not NULL; a block whose
 *     64 tokens are all extra gets beta = -inf (no entry). k_pool (the block scores) is
 *     not changed.
 * extra_pack: spark_extra_pack_bytes(s, extra_tokens) bytes, 16-byte aligned, caller-owned.
 * extra_tokens = 0 (or no video block) does nothing. */
size_t spark_extra_pack_bytes(const spark_shape* s, int32_t extra_tokens);
int spark_extra_tokens(const spark_shape* s, const uint16_t* K, const uint16_t* V, const float* anchor,
                       int32_t extra_tokens, int pool_mode, float* v_summ, float* beta, void* pool_pack,
                       size_t pool_pack_bytes, void* extra_pack, size_t extra_pack_bytes, void* stream);

/* Spark-Reblock ("What Spark-Attn changes", Spark-Reblock bullet; "Workflows":
 * reblock_layout=q_reuse_k). Per (b, h): M = mean over video keys of k k^T;
 * x_i = L^T q_i / |L^T q_i| with M = L L^T (Mahalanobis cosine geometry); recursive
 * bisection of the video tokens: a node of m blocks takes the leading eigenvector v of
 * the centred covariance of its x (signed so the projections' third central moment is
 * >= 0), orders its tokens by (x . v, token index) and gives the first floor(m/2)*64 to
 * the left child, until every leaf holds 64 tokens. perm int32 [B, H, nb*64] lists the
 * leaves by their smallest token index, tokens ascending inside a leaf. Qp/Kp/Vp
 * (bf16 [B,H,N,d], may not alias the inputs) receive the permuted rows (keys reuse the
 * query partition), dense rows copied unchanged. tree (nullable) int32
 * [B, H, L+1, nb*64], L = ceil(log2 nb): node label of every token at every level
 * (a node c splits into 2c (left) and 2c+1; a leaf moves to 2c).
 * ws: spark_workspace_bytes(s, SPARK_CALL_REBLOCK) bytes. */
int spark_reblock(const spark_shape* s, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                  int32_t* perm, uint16_t* Qp, uint16_t* Kp, uint16_t* Vp, int32_t* tree, void* ws,
                  size_t ws_bytes, void* stream);

/* Spark-Reblock with a partition of its own for the keys (the alternative to
 * reblock_layout=q_reuse_k named in "Workflows"; the Spark-Reblock bullet whitens each side
 * by the opposite side's second moment). perm_q is exactly what spark_reblock writes into
 * perm; perm_k int32 [B, H, nb*64] partitions the video keys the same way with the roles of
 * Q and K swapped (x_j = L^T k_j / |L^T k_j| with L L^T = mean over video queries of
 * q q^T). Qp receives Q in the perm_q order, Kp and Vp receive K and V in the perm_k order
 * (dense rows unchanged). Pass perm_q to spark_attn_fwd to get O back in the original
 * query order. Same workspace as spark_reblock; about twice its time. No tree output. */
int spark_reblock_kv(const spark_shape* s, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                     int32_t* perm_q, int32_t* perm_k, uint16_t* Qp, uint16_t* Kp, uint16_t* Vp,
                     void* ws, size_t ws_bytes, void* stream);

/* The whole forward from host memory, pipelined over groups of heads (the pages have no
 * counterpart; a library convenience for callers whose Q/K/V start in host memory). Every
 * step of the method is per (b, h), so the flattened B*H heads are cut into groups of
 * heads_per_group (the last group may be smaller) and each group runs as a forward of its
 * own shape [1, G, N, d]: its Q/K/V are copied host-to-device on one internal stream, the
 * group is computed on `stream` (optional Reblock, spark_pool_kv, spark_score_select,
 * spark_attn_fwd), and its O (and lse) are copied device-to-host on a second internal
 * stream, so that the copies of neighbouring groups overlap the compute. Two staging slots
 * alternate between groups.
 * - hQ, hK, hV: host bf16 [B, H, N, d]; hO: host bf16 [B, H, N, d]; hlse: host fp32
 *   [B, H, N] or NULL. Page-locked (pinned) host memory is needed for the copies to
 *   overlap; pageable memory works but the copies then serialise with the compute.
 *   Outputs are those of the device calls with the same configuration.
 * - cfg: select_mode / param / kcap as in spark_score_select (kcap <= 0 picks k for top-k
 *   and nb for tau); pool_mode as in spark_pool_kv; compressed != 0 turns the compressed
 *   branch on; reblock 0 = none, 1 = spark_reblock (keys reuse the query partition),
 *   2 = spark_reblock_kv; heads_per_group <= 0 picks the fewest heads whose Q/K/V reach
 *   32 MiB (ceil(2^25 / (6*N*d)), at most B*H): one head at a time for video-sized heads.
 * - ws: device buffer of spark_forward_host_workspace_bytes(s, cfg) bytes, 256-byte
 *   aligned, holding both staging slots and every intermediate of one group. The current
 *   device must be the one that holds ws and `stream` (the internal streams are created
 *   there).
 * - Asynchronous: returns once everything is enqueued; `stream` waits for the last copy
 *   back, so synchronising `stream` means hO / hlse are complete. The host buffers must
 *   stay valid and unchanged until then. Unlike the other calls this one creates two
 *   streams and seven events per call (released by the driver once their work completes).
 * - Returns SPARK_EINVAL / SPARK_EUNSUPPORTED for rejected arguments (nothing enqueued),
 *   SPARK_ECUDA if a copy or launch fails to enqueue, or the first error status of a
 *   per-group call (groups before it are enqueued). */
typedef struct spark_fwd_config {
  double param;            /* top-k ratio in (0, 1] or tau */
  int32_t select_mode;     /* SPARK_SELECT_TOPK_RATIO or SPARK_SELECT_TAU */
  int32_t kcap;            /* selection slots per row; <= 0: k (top-k) or nb (tau) */
  int32_t pool_mode;       /* SPARK_POOL_REWEIGHT or SPARK_POOL_MEAN */
  int32_t compressed;      /* compressed branch on (!= 0) or off */
  int32_t reblock;         /* 0 none, 1 spark_reblock, 2 spark_reblock_kv */
  int32_t heads_per_group; /* heads per pipeline group; <= 0: automatic (see above) */
  int32_t extra_tokens;    /* extra tokens per head (spark_extra_tokens); 0: none */
} spark_fwd_config;

/* Device workspace bytes of spark_forward_host; 0 for an invalid shape or config. */
size_t spark_forward_host_workspace_bytes(const spark_shape* s, const spark_fwd_config* cfg);

int spark_forward_host(const spark_shape* s, const spark_fwd_config* cfg, const uint16_t* hQ,
                       const uint16_t* hK, const uint16_t* hV, uint16_t* hO, float* hlse,
                       void* ws, size_t ws_bytes, void* stream);

/* spark_score_select without a scratch argument, for callers that cannot allocate device
 * memory of their own (the paper has no counterpart; this is a library convenience).
 * Some hosts own every byte of device memory up front - an engine that hands out one
 * arena at start-up, a plugin running inside another framework's allocator, a real-time
 * loop that must never reach the driver's allocator - and so cannot provide the scratch
 * that spark_score_select asks for. This entry point uses a file-scope device array of
 * SPARK_NOALLOC_MAX_HEADS * 2 doubles (64 KiB, held by every GPU that loads the library
 * until the process exits) for the tau moments instead, and keeps each CTA's score rows
 * in shared memory rather than writing the score matrix out (a slower kernel with the
 * same per-score arithmetic), with the same arguments and outputs.
 * - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 * - B*H above SPARK_NOALLOC_MAX_HEADS returns SPARK_ESCRATCH before any launch.
 * - The first call on a device looks the array's device address up (cudaGetSymbolAddress,
 *   with that device current) and caches it with the unique ID of the device's current
 *   context; make that first call before any stream capture on the device. After a
 *   device reset (cudaDeviceReset, or the primary context released and created again)
 *   the context ID changes and the next call looks the address up again, so that call
 *   too should come before any capture. A call from a host thread on which the runtime
 *   has not yet made the context current also repeats the lookup.
 * - Every call shares the one array: calls whose work overlaps on the GPU (different
 *   streams, or different host threads without ordering) race on it. The part that must
 *   start at zero is cleared by each call. */
#define SPARK_NOALLOC_MAX_HEADS 4096
int spark_score_select_noalloc(const spark_shape* s, const float* q_pool, const float* k_pool,
                               int mode, double param, int32_t kcap, int32_t* idx, int32_t* cnt,
                               void* stream);

/* Reads the device error word into *host_word (may be NULL) and clears it; synchronises
 * `stream`. Returns SPARK_OK or SPARK_ECUDA when the copy itself failed. */
int spark_device_error(int32_t* host_word, void* stream);

/* Human-readable text of a status code. */
const char* spark_strerror(int status);

/* Number of kernels this process has launched through the library so far (all devices
 * and threads), counted on the host as each launch is issued. No counterpart in the
 * method: it lets a caller account for the device work of a region of calls. */
uint64_t spark_kernel_launches(void);

/* Limit, in SM clocks, of every pipeline wait of the attention kernels launched after this
 * call (all devices and threads of the process); clocks <= 0 restores the default of
 * 2^31 clocks (about a second). No counterpart in the method: it exists so that the
 * failure path can be exercised without faulting a GPU. A wait that runs out records
 * SPARK_ETIMEOUT in the device error word, every role of the CTA stops, the copies and
 * MMAs still in flight are drained (those drains keep the default limit) and tensor
 * memory is released; the call's outputs are then undefined, and the device stays usable.
 * A limit of a few hundred clocks makes the first waits of a launch give up. */
int spark_set_wait_limit(int64_t clocks);

#ifdef __cplusplus
}
#endif

#endif /* SPARK_H_ */
