/*
 * cp_attn.h -- C ABI of libcpattn: zigzag context-parallel causal attention on
 * one B200 (sm_100a), with every context-parallel rank run as a virtual rank
 * (a shard loop in HBM) on the same GPU.
 *
 * The problem, as the pages state it:
 *   - Q, K and V are sharded along the sequence; rank i keeps its query shard
 *     Q_i, attends it to its own K_i,V_i and then to every other rank's
 *     K_j,V_j, and the partial attentions are combined
 *     (Accelerate "Context Parallel" concept guide, "So how does it work?").
 *     Each shard has the layout [batch, num_heads, seq_len/cp, head_dim].
 *   - The K/V shards are visited in all-gather order (gather once, compute in
 *     rank order) or ring order ("all-to-all": take the neighbour's shard
 *     cp-1 times) (concept guide, "all-to-all vs all-gather";
 *     "Configurable options": cp_size and cp_comm_strategy).
 *   - seq_len must be divisible by 2*cp (NeMo "Hierarchical Context Parallel
 *     Skill", "Required constraints"); the 2*cp chunks are paired head/tail
 *     so every rank gets the same causal work.
 *   - An invalid strategy or size is an error, not a silent fallback
 *     (Accelerate FullyShardedDataParallelPlugin.__post_init__ checks).
 *
 * Conventions shared by every call:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     never allocates, frees or retains memory.  Pointers must be 16-byte
 *     aligned.
 *   - Attention tensors are contiguous bf16 [batch][heads][seq][head_dim]
 *     (BHSD) in SHARD order: position p = r*2C + t is local token t of virtual
 *     rank r, C = seq_len/(2*cp).  LSE tensors are fp32 [batch][heads][seq],
 *     natural log of the sum of exp(scaled scores).  cu_seqlens is in ORIGINAL
 *     order.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream).  Argument checks run on the host before any launch and
 *     return an error without touching the GPU.  Errors found on the device
 *     (a bounded wait that timed out) are recorded in a device status word that
 *     cp_get_device_status() reads and clears.
 *   - Workspace: calls that take (ws, ws_bytes) report the bytes they need in
 *     *ws_bytes and launch nothing when ws == NULL.  Otherwise *ws_bytes must
 *     be at least that size (else CP_ERR_WORKSPACE); ws must be 256-byte
 *     aligned.  The workspace is scratch: its contents need not be preserved.
 *   - No call is thread-safe with respect to another call on the same buffers.
 */
#ifndef CP_ATTN_H
#define CP_ATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define CP_API __attribute__((visibility("default")))
#else
#define CP_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    CP_OK = 0,
    CP_ERR_INVALID_ARG = 1, /* bad size, null pointer, bad enum, bad cu_seqlens */
    CP_ERR_UNSUPPORTED = 2, /* valid problem outside what the kernels cover   */
    CP_ERR_CUDA = 3,        /* a CUDA runtime call failed (launch, no device)  */
    CP_ERR_TIMEOUT = 4,     /* a bounded device wait gave up                  */
    CP_ERR_WORKSPACE = 5    /* workspace smaller than required                */
} cp_status_t;

typedef enum { CP_ROTATE_ALLGATHER = 0, CP_ROTATE_RING = 1 } cp_rotate_t;
/* Masks.  CP_MASK_CAUSAL: the query at original position q sees keys k <= q.
 * CP_MASK_DOC_CAUSAL: additionally only keys of its own document (cu_seqlens).
 * CP_MASK_FULL: no mask, every query sees every key (bidirectional attention);
 * it takes no documents (cu_seqlens NULL, num_docs 0) and no window. */
typedef enum { CP_MASK_CAUSAL = 0, CP_MASK_DOC_CAUSAL = 1, CP_MASK_FULL = 2 } cp_mask_t;

/* How the sequence is cut into shards.
 *   CP_SHARD_SEQUENCE: the sequence in 2*cp chunks, rank r holding chunks r and
 *     2cp-1-r (the zigzag of the pages).
 *   CP_SHARD_PER_DOC: every packed document in 2*cp chunks, rank r holding,
 *     document after document, its chunk r then its chunk 2cp-1-r, so every rank
 *     gets an equal share of every document's causal work (FlashCP abstract:
 *     "Per-Doc" sharding).  Needs CP_MASK_DOC_CAUSAL; every document's length a
 *     multiple of 256*cp_size (chunks of whole 128-row tiles), else
 *     cp_plan_shards records CP_ERR_UNSUPPORTED in the device status word. */
typedef enum { CP_SHARD_SEQUENCE = 0, CP_SHARD_PER_DOC = 1 } cp_shard_t;

/* How cp_attn_fwd combines the per-step partial attentions.
 *   CP_MERGE_SEPARATE: each (rank, step) unit writes its partial (O, LSE) in
 *     fp32 to the workspace, then the cp_lse_merge kernel folds the cp
 *     partials in visit order (the literal shard loop + combine).
 *   CP_MERGE_FUSED: the forward kernel folds each step into the running
 *     (O, LSE) in registers / tensor memory as it goes, in the same visit
 *     order, and writes only the final result. */
typedef enum { CP_MERGE_SEPARATE = 0, CP_MERGE_FUSED = 1 } cp_merge_t;

/* The problem.  Field meaning:
 *   batch         >= 1; batch * num_heads * seq_len must stay below 2^31
 *                 (CP_ERR_UNSUPPORTED otherwise: flat row indices are int32)
 *   seq_len       S, tokens per sequence; S % (2*cp_size) == 0
 *   cp_size       number of virtual ranks, 1..1024 (CP_ERR_UNSUPPORTED above)
 *   num_heads     query heads Hq; num_kv_heads Hkv divides Hq (GQA: query head
 *                 h reads KV head h / (Hq/Hkv))
 *   head_dim      D
 *   rotate        cp_rotate_t
 *   mask          cp_mask_t; CP_MASK_DOC_CAUSAL needs cu_seqlens
 *   merge         cp_merge_t (forward only)
 *   softmax_scale 0 => 1/sqrt(head_dim)
 *   num_docs      documents in cu_seqlens (doc mask only)
 *   window        0: no window.  W > 0: sliding window on top of the mask --
 *                 the query at original position q sees only keys k with
 *                 q - W < k <= q (and, with documents, k in q's document).
 *                 Negative values are CP_ERR_INVALID_ARG; W > 0 with
 *                 CP_MASK_FULL is CP_ERR_UNSUPPORTED.
 *   shard         cp_shard_t (CP_SHARD_PER_DOC needs the document mask)
 *   bwd_one_pass  backward only.  0 (default): two passes, a dK/dV pass and a
 *                 dQ pass that recomputes S and dP (three at head_dim 256: dV,
 *                 dK and dQ); bit-for-bit reproducible, and the faster form on
 *                 B200 (128k: 438 vs 475 ms).
 *                 1: one pass, dK, dV and dQ from one recomputation of S and dP,
 *                 dQ summed in an fp32 accumulator by atomic reductions (its
 *                 last bits depend on their order); bound by those reductions.
 *                 head_dim 64 and 128 only (256: CP_ERR_UNSUPPORTED).
 *   cu_seqlens    DEVICE int32 [num_docs+1], 0 = cu[0] < cu[1] < ... <
 *                 cu[num_docs] = S, original order; the same documents apply to
 *                 every batch entry.  NULL for the plain causal mask.
 *                 cp_plan_shards checks it on the device: a list that is not
 *                 strictly increasing from 0 to S records CP_ERR_INVALID_ARG in
 *                 the device status word (the host cannot see device memory
 *                 without synchronising).  The backward calls (cp_attn_bwd,
 *                 cp_attn_bwd_noalloc, cp_attn_bwd_rank, cp_attn_bwd_step) read
 *                 it again on the device, for the document end of each key
 *                 tile, without checking it: the list must stay allocated and
 *                 unchanged from cp_plan_shards until the backward has run.
 *                 The forward calls read only the plan. */
typedef struct {
    int32_t batch;
    int32_t seq_len;
    int32_t cp_size;
    int32_t num_heads;
    int32_t num_kv_heads;
    int32_t head_dim;
    int32_t rotate;
    int32_t mask;
    int32_t merge;
    float softmax_scale;
    int32_t num_docs;
    int32_t window;
    int32_t bwd_one_pass;
    int32_t shard;
    const int32_t* cu_seqlens;
} cp_problem_t;

/* The shard plan, written by cp_plan_shards into caller-owned DEVICE buffers:
 *   perm        int32 [S]          original index of shard position p
 *   inv_perm    int32 [S]          shard position of original index o
 *   src         int32 [cp*cp]      K/V shard visited by rank r at step s:
 *                                  s (all-gather) or (r - s) mod cp (ring)
 *   doc_start   int32 [S]          original start of the document of token
 *                                  perm[p] (0 everywhere for CP_MASK_CAUSAL)
 *   rank_cu_off int32 [cp+1]       rank r's entries are rank_cu[off[r]..off[r+1])
 *   rank_cu     int32 [3*cp + num_docs] (CP_SHARD_SEQUENCE) or
 *               int32 [cp*(2*num_docs + 1)] (CP_SHARD_PER_DOC)
 *                                  per rank, local offsets where a segment
 *                                  starts, then 2C: sequence sharding, 0, the
 *                                  chunk boundary C and every document start
 *                                  inside the rank's chunks; per-document
 *                                  sharding, the start of each of the rank's
 *                                  two chunks of every document
 *   tile_orig   int32 [ceil(S/128)] original start of the 128-row tile at shard
 *                                  position 128*i
 *   tile_shard  int32 [ceil(S/128)] shard tile index of the tile starting at
 *                                  original position 128*i (inverse of tile_orig);
 *                                  both defined when the chunks are whole tiles
 *                                  (what the attention calls need) and read by
 *                                  them for per-document plans only
 *   pairs       int64 [cp]         unmasked (q, k) pairs whose query lives on
 *                                  rank r (equal across ranks for the plain
 *                                  causal mask without a window; 2C * S each
 *                                  for CP_MASK_FULL) */
typedef struct {
    int32_t* perm;
    int32_t* inv_perm;
    int32_t* src;
    int32_t* doc_start;
    int32_t* rank_cu_off;
    int32_t* rank_cu;
    int64_t* pairs;
    int32_t* tile_orig;
    int32_t* tile_shard;
} cp_plan_t;

/*
 * cp_plan_shards -- build the zigzag plan on the GPU and gather n_bufs tensors
 * from ORIGINAL into SHARD order (rank r's chunk r then chunk 2cp-1-r), the
 * counterpart of sharding the context buffers along their sequence dimension
 * (concept guide, "Accelerate's interface": buffers / buffer_seq_dims).
 *   bufs_in[i], bufs_out[i]  device tensors [outer_i][S][row_bytes_i]; in and
 *                            out must not overlap
 *   buf_outer[i]             outer extent (batch*heads) of buffer i
 *   buf_row_bytes[i]         bytes per token row (head_dim*2 for bf16), a
 *                            multiple of 16
 *   n_bufs                   0..16; with 0 only the plan is built
 * Reads problem->cu_seqlens for the doc mask.  Plan arrays and gathered
 * tensors are complete when the stream reaches this point.
 * Errors: CP_ERR_INVALID_ARG for the checks listed in cp_problem_t, a NULL
 * plan array, bad buffer sizes; CP_ERR_CUDA on a launch failure.
 */
CP_API cp_status_t cp_plan_shards(const cp_problem_t* problem, const cp_plan_t* plan, int32_t n_bufs,
                           const void* const* bufs_in, void* const* bufs_out,
                           const int64_t* buf_outer, const int64_t* buf_row_bytes, void* ws,
                           size_t* ws_bytes, void* stream);

/*
 * cp_unshard -- scatter n_bufs tensors from SHARD back to ORIGINAL order with
 * the plan's perm (the "restore" of the sharded buffers).  Same buffer
 * conventions as cp_plan_shards.
 */
CP_API cp_status_t cp_unshard(const cp_problem_t* problem, const cp_plan_t* plan, int32_t n_bufs,
                       const void* const* bufs_in, void* const* bufs_out,
                       const int64_t* buf_outer, const int64_t* buf_row_bytes, void* stream);

/*
 * cp_attn_fwd -- causal (optionally packed-document, optionally sliding-window)
 * or unmasked (CP_MASK_FULL) attention of every virtual rank's query shard
 * against the K/V shards in the plan's visit order,
 * combined into the exact unsharded result (concept guide, "So how does it
 * work?": local attention, then every other shard, then combine).
 *   q     bf16 [B][Hq][S][D]  shard order
 *   k, v  bf16 [B][Hkv][S][D] shard order
 *   o     bf16 [B][Hq][S][D]  output, shard order
 *   lse   fp32 [B][Hq][S]     output, natural-log LSE of the scaled scores
 * Supported: head_dim 64, 128 or 256; C = S/(2cp) a multiple of 128;
 * S <= 2^29.
 * Workspace: CP_MERGE_SEPARATE needs cp fp32 partial (O, LSE) sets (each
 * region rounded up to 256 bytes; the O partials in an internal 128-row
 * tile-interleaved layout, not the row layout cp_lse_merge takes);
 * CP_MERGE_FUSED needs none (0 bytes).
 * Errors: CP_ERR_INVALID_ARG, CP_ERR_UNSUPPORTED, CP_ERR_WORKSPACE, CP_ERR_CUDA.
 */
CP_API cp_status_t cp_attn_fwd(const cp_problem_t* problem, const cp_plan_t* plan, const void* q,
                        const void* k, const void* v, void* o, float* lse, void* ws,
                        size_t* ws_bytes, void* stream);

/*
 * cp_attn_bwd -- gradients of the attention output with respect to Q, K, V
 * given the upstream gradient dO, from the saved final LSE (backward through
 * the context-parallel attention; FLOPs counted as twice the forward, as the
 * Accelerate example's model-FLOPs helper does).  dK_j and dV_j collect the
 * contributions of every virtual rank that visits shard j.
 *   q, k, v, o, dout  bf16, shard order (o and lse from cp_attn_fwd)
 *   dq                bf16 [B][Hq][S][D]  output
 *   dk, dv            bf16 [B][Hkv][S][D] output
 * Workspace: two fp32 values per query row, dot(dO, O) and -LSE * log2(e)
 * (each array rounded up to 256 bytes), and for the one-pass backward
 * (problem->bwd_one_pass == 1) an fp32 dQ accumulator of head_dim values per
 * query row (rounded up to 256 bytes).
 * Errors: as cp_attn_fwd.
 */
CP_API cp_status_t cp_attn_bwd(const cp_problem_t* problem, const cp_plan_t* plan, const void* q,
                        const void* k, const void* v, const void* o, const float* lse,
                        const void* dout, void* dq, void* dk, void* dv, void* ws,
                        size_t* ws_bytes, void* stream);

/*
 * cp_lse_merge -- combine n_parts partial attentions row by row, folding them
 * in the given order: for running (O_a, L_a) and next (O_b, L_b),
 * m = max(L_a, L_b); if m = -inf the row stays (0, -inf); else
 * w = exp(L - m), L = m + ln(w_a + w_b), O = (w_a O_a + w_b O_b)/(w_a + w_b)
 * (the concept guide's "combine(attn)", read as the exact log-sum-exp merge).
 *   o_parts    fp32 [n_parts][rows][head_dim]
 *   lse_parts  fp32 [n_parts][rows]; -inf marks a row with no key in that part
 *              (its O part is not read)
 *   o_out      bf16 [rows][head_dim] (round to nearest even)
 *   lse_out    fp32 [rows]
 * head_dim must be a positive multiple of 4 no larger than 256; 1 <= n_parts
 * <= 64; rows >= 0.
 * Errors: CP_ERR_INVALID_ARG, CP_ERR_CUDA.
 */
CP_API cp_status_t cp_lse_merge(int64_t rows, int32_t head_dim, int32_t n_parts, const float* o_parts,
                         const float* lse_parts, void* o_out, float* lse_out, void* stream);

/*
 * cp_attn_bwd_noalloc -- cp_attn_bwd for callers that cannot hand the library a
 * workspace.  Some callers cannot allocate device memory at the point where they
 * run the backward: code that runs while a CUDA graph is being captured (device
 * allocation is not allowed there), or a host program whose device memory is
 * entirely pre-planned by a framework allocator that has no way to hand out
 * scratch.  This entry point takes the same arguments as cp_attn_bwd minus the
 * workspace and uses a fixed scratch array that the library holds in device
 * memory instead (there is no counterpart of this entry point on the pages; it
 * is a convenience of this library).
 *   - Limit: batch * num_heads * seq_len <= CP_NOALLOC_MAX_ROWS (4,194,304
 *     rows, e.g. 131072 tokens x 32 heads); larger problems get
 *     CP_ERR_WORKSPACE and nothing is launched.
 *   - Cost: every GPU that loads the library holds the 32 MiB array until the
 *     process exits.
 *   - A call made outside stream capture looks up the array's device address
 *     (a runtime query) and remembers it for its device; a call made while
 *     `stream` is being captured uses the remembered address, so the first
 *     call on each device must come before any stream capture (a first call
 *     inside a capture returns CP_ERR_CUDA).  Looking the address up again on
 *     each uncaptured call keeps it right after cudaDeviceReset.
 *   - Every call on a device shares the one array, and the array keeps the last
 *     call's contents (nothing in it needs to start at zero: each call writes
 *     every scratch value it reads).  Calls that can overlap on the GPU (two
 *     streams, or two host threads) race on the array: serialise them.
 *   - The library allocates and frees nothing in this call.
 * Errors: as cp_attn_bwd, plus CP_ERR_WORKSPACE beyond the limit and
 * CP_ERR_CUDA if the array's address cannot be obtained.
 */
#define CP_NOALLOC_MAX_ROWS 4194304
CP_API cp_status_t cp_attn_bwd_noalloc(const cp_problem_t* problem, const cp_plan_t* plan,
                                       const void* q, const void* k, const void* v,
                                       const void* o, const float* lse, const void* dout,
                                       void* dq, void* dk, void* dv, void* stream);

/*
 * Per-rank calls: context parallelism across GPUs, one process per GPU.  Rank r
 * of cp_size holds its own query shard -- Q_r, O_r, LSE_r, dO_r, dQ_r, each
 * [B][heads][2C][...] with 2C = seq_len / cp_size rows per head, local row t being
 * shard position r*2C + t -- and gets the K/V shards of the other ranks over the
 * interconnect, as the concept guide describes ("So how does it work?": Q_i stays,
 * K_j/V_j travel; "all-to-all vs all-gather": gather them all at once, or take the
 * neighbour's shard cp-1 times).  The plan is the same on every rank (built by
 * cp_plan_shards from the same problem).  The library moves no data between
 * GPUs: the caller runs the collectives (NCCL all-gather, send/recv,
 * reduce-scatter) between these calls.
 */

/*
 * cp_attn_fwd_rank -- rank r's attention against K/V of every shard, already
 * gathered in shard order (all-gather):
 *   q        bf16 [B][Hq][2C][D]   rank r's query shard
 *   k, v     bf16 [B][Hkv][S][D]   every shard, shard order
 *   o        bf16 [B][Hq][2C][D]   output, lse fp32 [B][Hq][2C]
 * The cp steps are visited in the plan's order and combined as problem->merge
 * says (fused in the kernel, or per-step fp32 partials in the workspace merged by
 * the LSE-merge kernel).  Supported sizes as cp_attn_fwd.
 * Errors: as cp_attn_fwd; CP_ERR_INVALID_ARG for rank outside [0, cp_size).
 */
CP_API cp_status_t cp_attn_fwd_rank(const cp_problem_t* problem, const cp_plan_t* plan,
                                    int32_t rank, const void* q, const void* k, const void* v,
                                    void* o, float* lse, void* ws, size_t* ws_bytes, void* stream);

/*
 * cp_attn_fwd_step -- one step of the ring: rank r's queries against the single
 * K/V shard j = src[r][step] that it holds at that step:
 *   q                 bf16 [B][Hq][2C][D]   rank r's query shard
 *   k, v              bf16 [B][Hkv][2C][D]  shard j
 *   o_part, lse_part  fp32 [B][Hq][2C][D] and [B][Hq][2C]: the step's partial
 *                     attention, O normalised over the step's keys, LSE = -inf for
 *                     rows with no visible key in shard j (their O is not written)
 * After all cp steps, cp_lse_merge over the cp partials (in step order) gives
 * rank r's O and LSE: the ring form of the shard loop and combine.
 * Errors: as cp_attn_fwd; CP_ERR_INVALID_ARG for rank or step outside [0, cp_size).
 */
CP_API cp_status_t cp_attn_fwd_step(const cp_problem_t* problem, const cp_plan_t* plan,
                                    int32_t rank, int32_t step, const void* q, const void* k,
                                    const void* v, float* o_part, float* lse_part, void* stream);

/*
 * cp_attn_bwd_rank -- rank r's backward: dQ of its query shard, and the
 * contribution of its queries to dK and dV of every key.
 *   q, o, dout      bf16 [B][Hq][2C][D], lse fp32 [B][Hq][2C]   rank r's shard
 *   k, v            bf16 [B][Hkv][S][D]                          every shard, gathered
 *   dq              bf16 [B][Hq][2C][D]   output
 *   dk_part, dv_part  fp32 [B][Hkv][S][D] output: rank r's share of dK / dV for
 *                   every key (zero where none of its queries sees the key).
 * The caller sums dk_part / dv_part over the ranks (a reduce-scatter hands rank
 * j the sum for its own shard j) and casts with cp_f32_to_bf16.
 * Workspace: two fp32 values per local query row (as cp_attn_bwd).
 * Errors: as cp_attn_bwd; CP_ERR_INVALID_ARG for rank outside [0, cp_size).
 */
CP_API cp_status_t cp_attn_bwd_rank(const cp_problem_t* problem, const cp_plan_t* plan,
                                    int32_t rank, const void* q, const void* k, const void* v,
                                    const void* o, const float* lse, const void* dout, void* dq,
                                    float* dk_part, float* dv_part, void* ws, size_t* ws_bytes,
                                    void* stream);

/*
 * cp_attn_bwd_step -- one step of the ring form of the backward: rank r's
 * queries against the single K/V shard j = src[r][step] it holds at that step
 * (the ring rotation of the concept guide's "all-to-all vs all-gather", run
 * for the gradients of the attention it computes), their gradients added into
 * fp32 sums:
 *   q, o, dout      bf16 [B][Hq][2C][D], lse fp32 [B][Hq][2C]   rank r's shard
 *   k, v            bf16 [B][Hkv][2C][D]                         shard j
 *   dq_sum          fp32 [B][Hq][2C][D]   rank r's dQ, this step's share added
 *   dk_sum, dv_sum  fp32 [B][Hkv][2C][D]  shard j's dK / dV, rank r's share added
 * The sums are read and written (the caller zeroes them first), without
 * atomics: two calls that add into the same sums must not run concurrently
 * (issue them on one stream, or order them with events).  In a ring the
 * dK / dV sums travel with the K/V shard: after the cp steps (and one more hop)
 * every shard's sums have been added to by every rank and are back with their
 * owner; cp_f32_to_bf16 casts them (and dq_sum).  Two passes (a dK/dV pass over
 * shard j's keys, a dQ pass over that step) whatever problem->bwd_one_pass says.
 * Workspace: two fp32 values per local query row (as cp_attn_bwd_rank).
 * Errors: as cp_attn_bwd; CP_ERR_INVALID_ARG for rank or step outside
 * [0, cp_size).
 */
CP_API cp_status_t cp_attn_bwd_step(const cp_problem_t* problem, const cp_plan_t* plan,
                                    int32_t rank, int32_t step, const void* q, const void* k,
                                    const void* v, const void* o, const float* lse,
                                    const void* dout, float* dq_sum, float* dk_sum, float* dv_sum,
                                    void* ws, size_t* ws_bytes, void* stream);

/* out[i] = bf16(in[i]) (round to nearest even) for n floats; n a multiple of 4, in
 * 16-byte and out 8-byte aligned. */
CP_API cp_status_t cp_f32_to_bf16(const float* in, void* out, int64_t n, void* stream);

/* Read and clear the device status word on `stream` (synchronises the stream).
 * *status receives CP_OK or the first device-side error since the last read. */
CP_API cp_status_t cp_get_device_status(int32_t* status, void* stream);

/* Set the limit, in nanoseconds, after which a bounded device wait gives up
 * (default 2 s).  Synchronous. */
CP_API cp_status_t cp_set_wait_limit_ns(uint64_t limit_ns);

/* Self-test of the bounded-wait machinery: one CTA waits on an mbarrier that
 * nothing will ever complete, gives up after limit_ns and records
 * CP_ERR_TIMEOUT in the device status word.  The GPU context stays usable. */
CP_API cp_status_t cp_selftest_wait_timeout(uint64_t limit_ns, void* stream);

/* Test hook of the bounded-wait teardown inside the attention kernels.  Runs
 * cp_attn_fwd (kernel = CP_K_FWD) or cp_attn_bwd (kernel = CP_K_BWD_DKDV or
 * CP_K_BWD_DQ: the two-pass backward; CP_K_BWD_FUSED: the one-pass backward,
 * whatever problem->bwd_one_pass says) with the same arguments and checks as
 * those calls (o and lse are
 * the forward's outputs or the backward's inputs; dout, dq, dk, dv are unused by
 * CP_K_FWD and may be NULL there), except that in the named kernel the producer
 * warp of CTA 0 skips its first K/V tile load.  The MMA warp of that CTA then
 * waits on a barrier nothing completes: once the wait limit (cp_set_wait_limit_ns)
 * passes it records CP_ERR_TIMEOUT in the device status word, the CTA's other
 * warps give up their waits, the copies and tensor-core work already issued
 * drain, the CTA frees its tensor memory and exits; every other CTA runs its
 * work normally.  The outputs of CTA 0's work items are left unwritten.  After
 * the call (and cp_get_device_status) the context is usable and later calls are
 * unaffected.  Errors: as the call it runs; CP_ERR_INVALID_ARG for another
 * kernel id. */
CP_API cp_status_t cp_selftest_stall(int32_t kernel, const cp_problem_t* problem,
                                     const cp_plan_t* plan, const void* q, const void* k,
                                     const void* v, void* o, float* lse, const void* dout,
                                     void* dq, void* dk, void* dv, void* ws, size_t* ws_bytes,
                                     void* stream);

/* Kernels of the library, as reported by the launch trace. */
typedef enum {
    CP_K_PLAN_META = 1,  /* plan: cu_seqlens check, src table, segment lists */
    CP_K_PLAN_INDEX = 2, /* plan: perm, inv_perm, doc_start, pair counts     */
    CP_K_GATHER = 3,     /* shard / unshard row gather                      */
    CP_K_FWD = 4,        /* forward attention                               */
    CP_K_MERGE = 5,      /* LSE merge                                       */
    CP_K_BWD_PREP = 6,   /* backward: dot(dO, O), -LSE * log2(e)            */
    CP_K_BWD_DKDV = 7,   /* backward: dK, dV                                */
    CP_K_BWD_DQ = 8,     /* backward: dQ                                    */
    CP_K_SELFTEST = 9,
    CP_K_SELFTEST_EXP2 = 10,
    CP_K_CAST = 11,      /* fp32 -> bf16 cast of summed dK / dV partials    */
    CP_K_BWD_FUSED = 12, /* one-pass backward: dK, dV, dQ partials          */
    CP_K_DQ_CONVERT = 13 /* one-pass backward: dQ accumulator -> bf16       */
} cp_kernel_t;

/* Number of kernels this library has launched in this process. */
CP_API int64_t cp_launch_count(void);

/* Launch trace.  cp_trace_begin hands the library `capacity` pairs of CUDA
 * events (cudaEvent_t, created by the caller with timing enabled; 2*capacity
 * handles).  Each later kernel launch k (k < capacity) records events[2k] on
 * its stream just before the launch and events[2k+1] just after it, and notes
 * its cp_kernel_t.  cp_trace_end stops recording and returns the number of
 * launches seen (which may exceed capacity; only the first `capacity` carry
 * events) and their kernel ids in kernel_ids[capacity].  Not thread-safe; the
 * events stay owned by the caller. */
CP_API cp_status_t cp_trace_begin(void* const* events, int32_t capacity);
CP_API cp_status_t cp_trace_end(int32_t* n_launches, int32_t* kernel_ids);

/* Self-test of the forward kernel's software exp2 (range reduction plus a
 * polynomial on the FMA pipe): y_soft[i] = software 2^x[i], y_hw[i] = the
 * hardware ex2.approx result, for n device floats (finite, <= 127). */
CP_API cp_status_t cp_selftest_exp2(const float* x, float* y_soft, float* y_hw, int64_t n,
                                    void* stream);

/* Library version, major*10000 + minor*100 + patch. */
CP_API int32_t cp_version(void);

#ifdef __cplusplus
}
#endif

#endif /* CP_ATTN_H */
