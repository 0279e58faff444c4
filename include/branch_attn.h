/*
 * branch_attn.h -- C ABI of the B200 (sm_100a) branch-attention library.
 *
 * What it computes ("Online Draft Co-Training", arXiv 2609.07108; paper
 * summary pages, technical-contribution and method-detail sections): the
 * attention layer of a speculative-decoding draft trained online next to its
 * target.  Tokens are packed without padding.  Main tokens form sequences
 * given by cu_seqlens; a main query attends causally to its own sequence.
 * Each branch (an EAGLE-3 TTT chain, a DFlash block or a DSpark block) hangs
 * off one main position, its anchor, and owns `depth` branch tokens with their
 * own Q/K/V.  A branch query attends to
 *   (1) the main keys of the anchor's sequence at positions <= anchor, and
 *   (2) the keys of its own branch: depth <= own depth (TTT-causal,
 *       block-causal) or the whole block (block-bidirectional),
 * and the two partial results (O_m, l_m), (O_b, l_b) are merged by the
 * online-softmax rule  l = log(e^{l_m} + e^{l_b}),
 *                      O = e^{l_m - l} O_m + e^{l_b - l} O_b.
 * The zigzag layout of the core-innovation section (each sequence cut into
 * 2C chunks, shard i holding chunks i and 2C-1-i, branches staying with their
 * anchor's shard) is available as a virtual shard order on one GPU: partial
 * results of every ring step are merged by the same rule.
 *
 * Conventions for every call below
 *   - Tensors are contiguous, row-major, bf16 unless stated:
 *       Q, O, dO, dQ  [tokens, Hq,  d]
 *       K, V, dK, dV  [tokens, Hkv, d]
 *       LSE           [Hq, tokens] fp32, natural log, softmax scale included.
 *     "_m" tensors cover the n_main main tokens, "_b" tensors the
 *     n_branch_tokens branch tokens, stored anchor-major, depth-minor.
 *   - q head h reads kv head h / (Hq / Hkv) (grouped-query attention).
 *   - All pointers except the ba_problem struct itself are DEVICE pointers
 *     owned by the caller; the library never allocates device memory and
 *     keeps no pointer after a call returns.  Tensor pointers must be 16-byte
 *     aligned (else BA_ERR_MISALIGNED), index arrays 4-byte aligned.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream).  Host-side argument checks run before any launch; a
 *     call that returns an error has launched nothing.
 *   - Content checks of the index arrays (sorted anchors, depth range, ...)
 *     run on the device inside ba_plan; they set a status word inside the
 *     plan workspace, every later kernel that reads that plan returns without
 *     touching its outputs when the word is non-zero, and ba_plan_status()
 *     reads it back (synchronising the stream).
 *   - Errors return a negative ba_status; ba_last_error() gives a message for
 *     the calling thread's last failing call.
 */
#ifndef BRANCH_ATTN_H
#define BRANCH_ATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define BA_API __attribute__((visibility("default")))
#else
#define BA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st *ba_stream_t;

/* Branch-local mask kinds (research-background section: EAGLE-3 test-time
 * training chains, DFlash block diffusion, DSpark Markov heads). */
typedef enum {
  BA_MASK_TTT_CAUSAL = 0,   /* depth j sees own-branch depths 0..j        */
  BA_MASK_BLOCK_BIDIR = 1,  /* every block token sees the whole block     */
  BA_MASK_BLOCK_CAUSAL = 2  /* block token j sees block tokens 0..j       */
} ba_mask_kind;

typedef enum {
  BA_OK = 0,
  BA_ERR_INVALID_ARG = -1,         /* bad size, enum, NULL pointer          */
  BA_ERR_UNSUPPORTED = -2,         /* valid but not built (head_dim, GPU)  */
  BA_ERR_MISALIGNED = -3,          /* pointer alignment violated           */
  BA_ERR_WORKSPACE_TOO_SMALL = -4, /* caller's workspace below the query   */
  BA_ERR_CUDA = -5,                /* a CUDA runtime call failed           */
  BA_ERR_DEVICE_TIMEOUT = -6,      /* a bounded device-side wait gave up   */
  BA_ERR_BAD_METADATA = -7         /* the plan's device-side checks failed */
} ba_status;

/* Device-side content-check bits reported by ba_plan_status(). */
#define BA_META_CU_START 0x01       /* cu_seqlens[0] != 0                  */
#define BA_META_CU_ORDER 0x02       /* cu_seqlens not strictly increasing  */
#define BA_META_CU_TOTAL 0x04       /* cu_seqlens[n_seqs] != n_main        */
#define BA_META_ANCHOR_RANGE 0x08   /* anchor outside [0, n_main)          */
#define BA_META_ANCHOR_ORDER 0x10   /* anchors decrease                    */
#define BA_META_DEPTH_RANGE 0x20    /* depth outside [1, 64]               */
#define BA_META_DEPTH_TOTAL 0x40    /* sum(depth) != n_branch_tokens       */

/* One packed batch.  The index arrays are device pointers, int32:
 *   cu_seqlens    [n_seqs + 1], cu_seqlens[0] = 0, strictly increasing,
 *                 cu_seqlens[n_seqs] = n_main
 *   branch_anchor [n_branches], packed main index, non-decreasing
 *   branch_depth  [n_branches], 1..64; sum = n_branch_tokens
 * scale: softmax scale (> 0), usually 1/sqrt(head_dim).
 * zigzag_C: 1 = monolithic; C > 1 = forward computed as C virtual zigzag
 *   shards (2C chunks per sequence) whose ring-step partials are merged by
 *   the LSE rule; the result equals the monolithic one up to rounding. */
typedef struct {
  int32_t n_seqs;
  int32_t n_main;
  int32_t n_branches;
  int32_t n_branch_tokens;
  int32_t hq;
  int32_t hkv;
  int32_t head_dim;      /* 64 or 128 */
  float scale;
  int32_t mask;          /* ba_mask_kind */
  int32_t zigzag_C;      /* 1..64 */
  const int32_t *cu_seqlens;
  const int32_t *branch_anchor;
  const int32_t *branch_depth;
} ba_problem;

/* Byte offsets of the metadata arrays inside a plan workspace (all int32).
 * Query tiles are BA_TILE_M rows (main tiles first, then branch tiles), key
 * tiles BA_TILE_N rows.
 *   status      [4]           word 0 = OR of BA_META_* bits; word 1 = sites of
 *               bounded device waits that gave up; word 2 = the backward's
 *               whole walk, the sum over key tiles of the query tiles visiting
 *               them (the backward's work in chunks; reported, not read back)
 *   cu_branch   [n_branches+1]  exclusive scan of branch_depth
 *   branch_seq  [n_branches]    sequence holding each anchor
 *   row_iv      [(n_main + n_branch_tokens) * 4]  per query row: first and
 *               last visible main key, first and last visible branch-local
 *               key row (empty = 0, -1); main rows first
 *   qtile       [n_qtiles * 6]  kv_begin, full_begin, full_end, kv_end
 *               (main key tiles; [full_begin, full_end) need no mask),
 *               bl_begin, bl_end (branch-local key rows)
 *   kv_main     [n_kv_main * 4]  main / branch query-tile ranges that visit
 *               each main key tile (backward work list)
 *   kv_branch   [n_kv_branch * 2]  branch query-tile range per branch key tile
 *   fwd_order   [n_qtiles]       query tiles by decreasing cost
 *   bwd_order   [n_kv_main + n_kv_branch]  key tiles by decreasing cost
 *   fwd_cost, bwd_cost           the costs used for the two orders
 *   zz_tiles    [zigzag_C * n_qtiles * 4]  (zigzag_C > 1 only) per ring step
 *               and query tile, two key-tile ranges [b0, e0), [b1, e1)
 *   key_iv      [(n_main + n_branch_tokens) * 4]  per key row (main keys
 *               first): the main query rows that see it [x, y) and the branch
 *               query rows that see it [z, w) (branch rows counted from 0);
 *               empty = (0, 0).  Contiguous because row bounds are
 *               non-decreasing; used by the backward's key-stationary walk.
 *   bwd_prefix  [n_kv_main + n_kv_branch]  walk ahead of each position of
 *               bwd_order: the sum of bwd_cost over the key tiles ranked
 *               before it (the dK/dV launch order reads it). */
#define BA_TILE_M 128
#define BA_TILE_N 128
typedef struct {
  size_t total_bytes;
  size_t off_status, off_cu_branch, off_branch_seq, off_row_iv, off_qtile;
  size_t off_kv_main, off_kv_branch, off_fwd_order, off_bwd_order;
  size_t off_fwd_cost, off_bwd_cost, off_zz_tiles, off_key_iv, off_bwd_prefix;
  int32_t n_qtiles_main, n_qtiles_branch, n_kv_main, n_kv_branch;
} ba_plan_layout;

/* Workspace sizes for one problem (host-only; no device access).
 * plan_bytes: the plan (metadata) workspace, written by ba_plan and read by
 *   branch_attn_fwd / branch_attn_bwd.
 * fwd_bytes:  scratch of branch_attn_fwd (0 when zigzag_C == 1; otherwise
 *   fp32 accumulators of O and LSE for every query row and head).
 * bwd_bytes:  scratch of branch_attn_bwd: D = rowsum(dO * O) fp32
 *   [Hq, rows], per-query records {LSE log2 e, D} (8 bytes per row and head,
 *   rows padded to 128 per token kind) and the fp32 dQ accumulator
 *   [rows, Hq, d] of the fused backward. */
BA_API ba_status ba_workspace_size(const ba_problem *p, size_t *plan_bytes,
                            size_t *fwd_bytes, size_t *bwd_bytes);

/* Layout of the plan workspace (host-only). */
BA_API ba_status ba_plan_layout_query(const ba_problem *p, ba_plan_layout *out);

/* Builds the tile metadata on the device (method-detail section: which main
 * keys and which branch keys each query sees).  Async on `stream`. */
BA_API ba_status ba_plan(const ba_problem *p, void *plan_ws, size_t plan_bytes,
                  ba_stream_t stream);

/* Synchronises `stream` and returns the plan's content-check word
 * (0 = valid) in *status_out; BA_ERR_BAD_METADATA when it is non-zero.  The
 * workspace also carries a second word that kernels reading this plan set
 * when one of their bounded waits on the device gave up (the kernel then
 * returns early and its outputs are not valid); that case returns
 * BA_ERR_DEVICE_TIMEOUT.  ba_plan clears both words. */
BA_API ba_status ba_plan_status(const void *plan_ws, ba_stream_t stream,
                         int32_t *status_out);

/* Forward.  Main rows: causal attention over their own sequence.  Branch
 * rows: main prefix up to the anchor plus own branch, merged by the LSE rule
 * (the branch-local partial is merged into the main partial in the kernel's
 * epilogue).  Writes o_m, o_b (bf16) and lse_m [Hq, n_main],
 * lse_b [Hq, n_branch_tokens] (fp32).  fwd_ws may be NULL when fwd_bytes is
 * 0.  Requires a plan built by ba_plan for the same problem. */
BA_API ba_status branch_attn_fwd(const ba_problem *p, const void *plan_ws,
                          void *fwd_ws, size_t fwd_bytes,
                          const void *q_m, const void *k_m, const void *v_m,
                          const void *q_b, const void *k_b, const void *v_b,
                          void *o_m, void *o_b, float *lse_m, float *lse_b,
                          ba_stream_t stream);

/* Backward of sum(O * dO): dQ, dK, dV for main and branch tokens.  P is
 * recomputed from the merged LSE written by branch_attn_fwd (lse_m, lse_b),
 * D = rowsum(dO * O) from the forward outputs.  dK/dV are summed over the q
 * heads of each kv group.  All six gradient tensors are fully overwritten. */
BA_API ba_status branch_attn_bwd(const ba_problem *p, const void *plan_ws,
                          void *bwd_ws, size_t bwd_bytes,
                          const void *q_m, const void *k_m, const void *v_m,
                          const void *q_b, const void *k_b, const void *v_b,
                          const void *o_m, const void *o_b,
                          const float *lse_m, const float *lse_b,
                          const void *do_m, const void *do_b,
                          void *dq_m, void *dk_m, void *dv_m,
                          void *dq_b, void *dk_b, void *dv_b,
                          ba_stream_t stream);

/* branch_attn_bwd for callers that cannot allocate device memory (no
 * counterpart in the paper; an interface addition of this library).
 * Some host programs manage all device memory themselves (a process that
 * reserves its whole HBM budget in its own pool at start-up, or a plugin whose
 * host forbids allocation at run time) and cannot cudaMalloc the backward
 * workspace.  This call takes the same arguments as branch_attn_bwd minus the
 * workspace and keeps its scratch (D, the per-query backward records and the
 * fp32 dQ accumulator) in a 32 MiB array compiled into the library,
 * which every GPU that loads the library holds until exit.  It allocates
 * nothing.
 *   - Problems whose backward scratch (see ba_workspace_size) exceeds 32 MiB
 *     are rejected with BA_ERR_WORKSPACE_TOO_SMALL before any launch.
 *   - The first call on a device looks up the array's device address (with
 *     that device current); make that first call before any stream capture.
 *     The address is looked up again when the device's context changes (after
 *     cudaDeviceReset, for example): an address from a context that no longer
 *     exists is never reused.
 *   - All calls on a device share the array; each call re-initialises what it
 *     needs, but calls whose kernels overlap on the GPU race on it. */
BA_API ba_status branch_attn_bwd_static_scratch(
    const ba_problem *p, const void *plan_ws, const void *q_m, const void *k_m,
    const void *v_m, const void *q_b, const void *k_b, const void *v_b, const void *o_m,
    const void *o_b, const float *lse_m, const float *lse_b, const void *do_m,
    const void *do_b, void *dq_m, void *dk_m, void *dv_m, void *dq_b, void *dk_b, void *dv_b,
    ba_stream_t stream);

/* One training step on host buffers (no counterpart in the paper; an
 * interface addition for callers whose tensors live in host memory).
 * Copies the metadata and the eight inputs into `staging` (device memory of
 * at least ba_step_host_workspace_size bytes, owned by the caller), builds
 * the plan, runs branch_attn_fwd and branch_attn_bwd, and copies O, LSE and
 * the six gradients back, all enqueued on `stream`; the call returns without
 * waiting.  Here the metadata pointers of *p (cu_seqlens, branch_anchor,
 * branch_depth) are HOST pointers, like every tensor argument.  Layouts are
 * those of branch_attn_fwd / branch_attn_bwd.
 *   - Copies run on two streams the library keeps per device (one upload,
 *     one download): dO is uploaded while the forward runs and O / LSE are
 *     downloaded while the backward runs, and the upload of a step issued on
 *     another stream (with its own staging) overlaps this step's download.
 *   - Host buffers should be page-locked; pageable memory works but the
 *     copies then do not overlap.
 *   - The host outputs are complete once `stream` reaches the point after
 *     this call.  Inputs must stay unchanged until then.  A call that returns
 *     an error has waited for every copy it had already queued, so its host
 *     buffers are free again when it returns.
 *   - Plan content errors are not checked here; ba_plan_status on the plan
 *     inside the staging area (at offset 0) reports them after the step. */
BA_API ba_status ba_step_host_workspace_size(const ba_problem *p, size_t *bytes);
BA_API ba_status branch_attn_step_host(
    const ba_problem *p, void *staging, size_t staging_bytes, const void *q_m,
    const void *k_m, const void *v_m, const void *q_b, const void *k_b, const void *v_b,
    const void *do_m, const void *do_b, void *o_m, void *o_b, float *lse_m, float *lse_b,
    void *dq_m, void *dk_m, void *dv_m, void *dq_b, void *dk_b, void *dv_b, ba_stream_t stream);

/* Standalone online-softmax merge (technical-contribution section):
 *   l = log(e^{l_a} + e^{l_b}),  O = e^{l_a - l} O_a + e^{l_b - l} O_b.
 * O_* are [rows, heads, head_dim] (fp32 when o_is_fp32, else bf16), l_*
 * [heads, rows] fp32.  An empty partial (l = -inf) contributes nothing; two
 * empty partials give O = 0, l = -inf.  o_out may alias o_a and lse_out may
 * alias lse_a (in-place accumulation); other overlaps are undefined. */
BA_API ba_status lse_merge(int64_t rows, int32_t heads, int32_t head_dim,
                    int32_t o_is_fp32, const void *o_a, const float *lse_a,
                    const void *o_b, const float *lse_b, void *o_out,
                    float *lse_out, ba_stream_t stream);

/* ---- Zigzag context parallelism across ranks --------------------------------
 * The core-innovation and method-detail sections shard a packed batch over C
 * context-parallel ranks in zigzag order and send the main-sequence K/V round
 * a ring: every sequence of length L is cut into 2C chunks, chunk k covering
 * positions [floor(kL/2C), floor((k+1)L/2C)); shard q holds chunks q and
 * 2C-1-q of every sequence and the branches anchored in them (branch K/V never
 * leave their rank).  At ring step t the rank holding shard q attends its
 * queries to the main keys of shard (q - t) mod C and merges the step's
 * partial (O, l) into an fp32 accumulator by the LSE rule; the rank-local
 * branch keys are merged last.  A shard is kept as its own packed problem
 * (the "local" problem): per sequence, its two chunks in position order.
 * Every sequence must hold at least 2C tokens. */

/* Host-only: the local problem of one shard.  cu_seqlens [n_seqs + 1],
 * branch_anchor and branch_depth [n_branches] are HOST arrays of the whole
 * batch (anchors non-decreasing).  Writes the shard's sizes to the three
 * count pointers and, for every output pointer that is not NULL (host arrays
 * sized by those counts): cu_local [n_seqs + 1] (local cu_seqlens: every
 * sequence keeps its index), anchor_local / depth_local [n_branches_local]
 * (anchors as local main rows), main_rows [n_main_local] (the batch's main
 * row of each local main row) and branch_rows [n_branch_tokens_local] (the
 * batch's branch row of each local branch row).  BA_ERR_UNSUPPORTED if a
 * sequence is shorter than 2C, BA_ERR_INVALID_ARG for other bad input. */
BA_API ba_status ba_zigzag_shard(const int32_t *cu_seqlens, int32_t n_seqs,
                                 const int32_t *branch_anchor, const int32_t *branch_depth,
                                 int32_t n_branches, int32_t C, int32_t shard,
                                 int32_t *n_main_local, int32_t *n_branches_local,
                                 int32_t *n_branch_tokens_local, int32_t *cu_local,
                                 int32_t *anchor_local, int32_t *depth_local,
                                 int32_t *main_rows, int32_t *branch_rows);

/* Workspace sizes of a ring rank (host-only): one plan workspace per step
 * (plan_bytes, the layout of ba_plan for the local problem) and the fp32
 * accumulator of O and LSE for every local query row and head (acc_bytes). */
BA_API ba_status ba_ring_workspace_size(const ba_problem *local, int32_t C, size_t *plan_bytes,
                                        size_t *acc_bytes);

/* Plan of ring step `step` (0 <= step < C) for the rank holding `shard`,
 * against shard (shard - step) mod C.  `local` is the rank's local problem
 * (device index arrays, zigzag_C = 1).  Step 0 is the local causal plan (the
 * plan of ba_plan; it also carries the branch-local intervals that
 * branch_attn_ring_finish reads).  For step > 0, cu_global [n_seqs + 1] is
 * the whole batch's cu_seqlens and cu_visit [n_seqs + 1] the visiting shard's
 * local cu_seqlens, both device arrays.  Async on `stream`. */
BA_API ba_status ba_ring_plan(const ba_problem *local, int32_t C, int32_t shard, int32_t step,
                              const int32_t *cu_global, const int32_t *cu_visit, void *plan_ws,
                              size_t plan_bytes, ba_stream_t stream);

/* One ring step: the rank's queries (q_m [n_main, Hq, d], q_b [n_branch_tokens,
 * Hq, d] of the local problem) against the visiting shard's main K/V
 * (k_m_visit, v_m_visit [n_main_visit, Hkv, d], in that shard's local order),
 * with the plan of ba_plan for the same step.  Step 0 initialises the
 * accumulator acc_ws (ba_ring_workspace_size bytes), later steps merge into it
 * by the LSE rule.  Steps of one rank must run in order 0 .. C-1 on one
 * stream (or be ordered by the caller).  Async on `stream`. */
BA_API ba_status branch_attn_ring_step(const ba_problem *local, int32_t C, int32_t step,
                                       const void *plan_ws, void *acc_ws, size_t acc_bytes,
                                       int32_t n_main_visit, const void *q_m,
                                       const void *k_m_visit, const void *v_m_visit,
                                       const void *q_b, ba_stream_t stream);

/* Last step: the branch-local partial of every branch query (own branch K/V,
 * k_b / v_b of the local problem), merged into the accumulator, which then
 * gives the outputs o_m, o_b (bf16) and lse_m, lse_b (fp32) of the local rows,
 * in the layouts of branch_attn_fwd.  plan_ws is the step-0 plan.  The result
 * equals branch_attn_fwd of the whole batch on the shard's rows, up to
 * rounding. */
BA_API ba_status branch_attn_ring_finish(const ba_problem *local, int32_t C, const void *plan_ws,
                                         void *acc_ws, size_t acc_bytes, const void *q_m,
                                         const void *q_b, const void *k_b, const void *v_b,
                                         void *o_m, void *o_b, float *lse_m, float *lse_b,
                                         ba_stream_t stream);

/* ---- TapChannel: target features across pipeline stages ---------------------
 * The method-detail section's pipeline transport (and the technical
 * contribution's mailboxes, sequence stamps and pre-allocated slots): stages
 * that compute target features write them straight into slots the draft's
 * stage allocated beforehand, outside the pipeline's schedule, and the
 * consumer reads a slot once its sequence stamp shows the message it expects.
 * Within a node the mailbox is shared through CUDA IPC (the producer's copy
 * engine writes over NVLink when the consumer is another GPU).
 *
 * The consumer owns one device region, the mailbox (ba_tap_mailbox_size
 * bytes: stamps and acks [n_producers][n_slots] int64, then the slots).
 * Message `seq` of producer p travels through slot seq mod n_slots:
 *   - ba_tap_send (producer) waits on the host until that slot's previous
 *     message (seq - n_slots) has been released, copies the payload into the
 *     slot on `stream` and then writes the stamp, in stream order;
 *   - ba_tap_wait (consumer) polls the stamp on the host until it equals seq
 *     and returns the slot's device address;
 *   - ba_tap_release (consumer) marks the slot free on `stream`, after the
 *     work that reads it.
 * No kernel ever waits for another process; every wait is a host poll bounded
 * by timeout_ns (BA_ERR_DEVICE_TIMEOUT when it runs out).  Producers and the
 * consumer may run on different GPUs of a node or on the same one. */
typedef struct ba_tap ba_tap;

/* Bytes of a mailbox: n_producers in [1, 256], n_slots in [1, 1024],
 * slot_bytes a positive multiple of 16.  Host-only. */
BA_API ba_status ba_tap_mailbox_size(int32_t n_producers, int32_t n_slots, int64_t slot_bytes,
                                     size_t *bytes);

/* Consumer side: turns caller-owned device memory (`mailbox`, 256-byte
 * aligned, at least ba_tap_mailbox_size bytes, on the current device) into a
 * channel, clears its stamps and acks (synchronising the device) and writes
 * into handle_out (at least 128 bytes) the blob producers attach with; the
 * caller hands it to them (any byte transport).  *out must be released with
 * ba_tap_close; the mailbox memory stays the caller's. */
BA_API ba_status ba_tap_create(void *mailbox, size_t mailbox_bytes, int32_t n_producers,
                               int32_t n_slots, int64_t slot_bytes, void *handle_out,
                               size_t handle_bytes, ba_tap **out);

/* Producer side: maps the consumer's mailbox (CUDA IPC, in another process)
 * as producer `producer`, on the current device. */
BA_API ba_status ba_tap_attach(const void *handle, size_t handle_bytes, int32_t producer,
                               ba_tap **out);

/* Producer: message seq (>= 0, consecutive per producer) of `bytes` (at most
 * the slot size) from device memory `src`; returns once the copy and the
 * stamp are enqueued on `stream` (src must stay unchanged until then). */
BA_API ba_status ba_tap_send(ba_tap *t, int64_t seq, const void *src, int64_t bytes,
                             int64_t timeout_ns, ba_stream_t stream);

/* Consumer: waits for message seq of `producer`; *slot receives its device
 * address (valid until ba_tap_release). */
BA_API ba_status ba_tap_wait(ba_tap *t, int32_t producer, int64_t seq, int64_t timeout_ns,
                             void **slot);

/* Consumer: frees the slot of message seq of `producer` once `stream` reaches
 * this point. */
BA_API ba_status ba_tap_release(ba_tap *t, int32_t producer, int64_t seq, ba_stream_t stream);

/* Either side: unmaps (producer) and frees the channel object. */
BA_API ba_status ba_tap_close(ba_tap *t);

/* Device self-check of the exponentials available to the softmax (no
 * counterpart in the paper): the hardware ex2 unit the kernels use, and a
 * range-reduced cubic on the FMA pipe (max relative error 7.5e-5) kept as an
 * alternative for offloading the ex2 unit.  Writes both for n inputs x
 * (device pointers, fp32): y_fma[i] = polynomial 2^x[i],
 * y_hw[i] = ex2.approx(x[i]).  Inputs below -125 (and -inf) give y_fma = 0. */
BA_API ba_status ba_exp2_check(const float *x, float *y_fma, float *y_hw, int64_t n,
                               ba_stream_t stream);

/* Device self-check of failure detection (no counterpart in the paper).  One
 * thread waits, with the bounded mbarrier wait every tcgen05 kernel uses
 * (limit 2 s), on an mbarrier in shared memory.  arrive = 1: the thread
 * arrives on it first and the wait completes at once.  arrive = 0: nothing
 * arrives, the wait gives up after its limit and sets bit 15 of the plan
 * workspace's device-timeout word, as a kernel whose wait gave up does, so
 * ba_plan_status then returns BA_ERR_DEVICE_TIMEOUT (ba_plan clears it).
 * Nothing traps or faults; the context stays usable.  plan_ws: a workspace
 * written by ba_plan (device pointer, 16-byte aligned); async on `stream`.
 * Returns BA_ERR_INVALID_ARG for a NULL workspace or another arrive value,
 * BA_ERR_MISALIGNED for a misaligned one. */
BA_API ba_status ba_wait_check(void *plan_ws, int32_t arrive, ba_stream_t stream);

/* Backward kernel family (the forward is the same for both):
 *   0 = default: split backward, a key-stationary dK/dV kernel and a
 *       query-stationary dQ kernel (S and dP computed in both, seven tile
 *       products), every gradient written once in bf16; bit-reproducible
 *       from run to run;
 *   1 = fused backward: one tcgen05 kernel per (key tile, kv head) computing
 *       S, dP, dV, dK and dQ (the method's five tile products); dQ partials
 *       are summed in fp32 in the workspace and converted to bf16 by a final
 *       pass, so dQ may differ in the last bits from run to run (the order of
 *       the fp32 sums is not fixed).  It moves 64 KB of fp32 partials into L2
 *       per (key tile, query tile, head), which on B200 makes it slower than
 *       family 0 at head_dim 128.
 * Returns BA_ERR_INVALID_ARG for other values.  Process-wide. */
BA_API ba_status ba_set_kernel_family(int32_t family);
BA_API int32_t ba_get_kernel_family(void);

/* Benchmark instrumentation.  After ba_set_kernel_events(which, start, stop)
 * every later call records the caller-owned CUDA event `start` (a cudaEvent_t)
 * on the call's stream right before its attention kernels and `stop` right
 * after them (which = 0: branch_attn_fwd, all ring-step launches of the
 * zigzag forward included; 1: branch_attn_bwd's attention kernels and the dQ
 * conversion, without the preprocess; 2: branch_attn_bwd's preprocess
 * kernel D = rowsum(dO * O) alone).  NULL events switch it off.
 * Process-wide; not for concurrent use from several threads. */
BA_API ba_status ba_set_kernel_events(int32_t which, void *start_event, void *stop_event);

/* Number of kernel launches the library has issued in this process. */
BA_API int64_t ba_launch_count(void);

/* Message for the calling thread's last failing call ("" if none). */
BA_API const char *ba_last_error(void);

/* Library version string. */
BA_API const char *ba_version(void);

#ifdef __cplusplus
}
#endif
#endif /* BRANCH_ATTN_H */
