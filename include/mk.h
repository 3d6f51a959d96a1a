/*
 * mk.h -- C ABI of the persistent decode megakernel for B200 (sm_100a).
 *
 * One autoregressive decode step of a Llama-style decoder (dense, or with a
 * routed mixture of experts) runs as ONE persistent kernel: exactly one CTA
 * per SM stays resident for the whole step, CTAs pull per-tile tasks from a
 * task list that the host builds once, and event counters in global memory
 * take the place of kernel boundaries.
 *
 * Sources for the operation (titles of the pages this follows):
 *  - "Cohere megakerneles kiszolgálót mutatott be a North Mini Code
 *    modellhez", section "Egyetlen tartós kernelre épül a kiszolgálás": one
 *    threadblock per SM resident for the whole decode step; blocks work from a
 *    host-prepared task list; global-memory counters signal dependencies; the
 *    scheduling unit is one tile of one operation.
 *  - same page, section "Honnan jön a gyorsulás?": no per-operation wave
 *    quantization; O-projection of a KV group may start when that group's
 *    attention is done; expert down-projection depends only on its own up-
 *    projection; weight tiles are prefetched before the activation dependency.
 *  - same page, section "Folyamatos batchkezelés, paged attention ...":
 *    continuous batching, paged attention, ragged sequences.
 *  - "LLM को MegaKernel में compile करके low-latency inference हासिल करना"
 *    (MPK digest), sections "Part 1. Compiler" (operator graph -> fine-grained
 *    task graph; events as synchronisation points) and "Part 2. Runtime"
 *    ("Event-आधारित execution तरीका": a finished task increments its event
 *    counter; the event fires when the counter reaches its threshold).
 *
 * Conventions for every entry point:
 *  - Return MK_OK or an error code; mk_last_error_string() describes the last
 *    error of the calling thread.  No entry point aborts the process.
 *  - "device pointer" = memory of the current CUDA device; "host pointer" =
 *    ordinary host memory.  The library never frees memory it did not
 *    allocate.
 *  - Kernels run asynchronously on the given stream.  Errors that the host
 *    can see (null pointers, sizes out of range) are returned before any
 *    launch.  Errors found on the device (a wait that timed out, a position,
 *    token id or page index out of range) set a device status word that the
 *    next mk_sync() or mk_decode_step() on the same state returns.
 *  - A state is not thread-safe: one host thread and one stream per state.
 */
#ifndef MK_H
#define MK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MK_OK = 0,
    MK_ERR_INVALID_ARG = 1,   /* bad argument (host check) or bad index (device check) */
    MK_ERR_CUDA = 2,          /* a CUDA runtime call failed */
    MK_ERR_OOM = 3,           /* device allocation failed */
    MK_ERR_UNSUPPORTED = 4,   /* shape or option this build does not support */
    MK_ERR_TIMEOUT = 5,       /* a device-side wait exceeded its time limit */
    MK_ERR_DEVICE_FAULT = 6   /* the device reported an inconsistent state */
} mk_status;

typedef struct mk_model mk_model;   /* weights (borrowed) + shape */
typedef struct mk_graph mk_graph;   /* host-built task list + event table */
typedef struct mk_state mk_state;   /* per-stream device state of one graph */

/* Any cudaStream_t may be passed where an mk_stream is expected (0 = legacy default). */
typedef struct CUstream_st* mk_stream;

#define MK_DTYPE_BF16 0

/* Flags of mk_model_desc.flags */
#define MK_FLAG_TRACE 0x1u   /* record per-task timestamps (mk_state_read_trace) */

/* Model shape.  n_experts == 0 selects the dense SiLU-gated FFN of width ffn;
 * n_experts > 0 selects a routed MoE with top_k experts of width expert_ffn
 * (router softmax over all experts; top-k ties to the lower expert index;
 * selected weights renormalised to sum 1 when moe_renorm != 0). */
typedef struct {
    int n_layers, hidden, n_q_heads, n_kv_heads, head_dim, ffn, vocab;
    float rms_eps, rope_theta;
    int n_experts, top_k, expert_ffn, moe_renorm;
    int dtype;        /* MK_DTYPE_BF16 only */
    unsigned flags;   /* MK_FLAG_* */
} mk_model_desc;

/* Paged KV cache, owned by the caller, device memory.
 *   k_pages, v_pages: bf16 [n_layers][n_pages][n_kv_heads][page_size][head_dim]
 *     (within a page, each KV head's page_size x head_dim block is contiguous)
 *   page_table: int32 [batch][max_pages_per_seq]; entry j of row b is the
 *     physical page holding positions 16j..16j+15 of sequence b.
 * The library never allocates pages: the caller guarantees that every page
 * the step touches (positions 0..positions[b]) is mapped. */
typedef struct {
    void* k_pages;
    void* v_pages;
    const int32_t* page_table;
    int n_pages;
    int page_size;          /* must be 16 */
    int max_pages_per_seq;
} mk_paged_kv;

/* ---------------------------------------------------------------- model */

/* Passage: Cohere page ("Cohere megakerneles kiszolgálót mutatott be a
 * North Mini Code modellhez"), section "A szűk keresztmetszet a memória-
 * sávszélesség": the step streams the model's bf16 weights from HBM once per
 * token; this call registers those weights.
 * Records the shape and the weight pointers (device, bf16, row-major
 * [out][in]).  Order of weight_ptrs: tok_emb [vocab][hidden]; then per layer
 * attn_norm [hidden], wq [n_q*d][hidden], wk [n_kv*d][hidden], wv
 * [n_kv*d][hidden], wo [hidden][n_q*d], ffn_norm [hidden], then dense:
 * w_gate [ffn][hidden], w_up [ffn][hidden], w_down [hidden][ffn]; or MoE:
 * w_router [E][hidden], w_gate [E][Fe][hidden], w_up [E][Fe][hidden],
 * w_down [E][hidden][Fe]; then final_norm [hidden], lm_head [vocab][hidden].
 * n_ptrs must equal 1 + n_layers*(9 dense | 10 MoE) + 2.  Weights are
 * borrowed: the caller keeps them alive and unchanged until
 * mk_model_destroy.  Every pointer must be 16-byte aligned.
 * Supported: head_dim in {64, 128}, n_q_heads a multiple of n_kv_heads,
 * hidden, ffn, expert_ffn and n_q*d multiples of 8, top_k <= 16. */
mk_status mk_load_model(const mk_model_desc* desc, const void* const* weight_ptrs, int n_ptrs,
                        mk_model** out);
/* Passage: none of its own.  Releases the model record (never the weights). */
void mk_model_destroy(mk_model* model);

/* ---------------------------------------------------------------- task graph */

/* Passage: MPK digest ("LLM को MegaKernel में compile करके low-latency
 * inference हासिल करना"), section "Part 1. Compiler": the operator graph is
 * turned into a fine-grained task graph with events as the
 * synchronisation points; Cohere page, section "Egyetlen tartós kernelre épül a
 * kiszolgálás": the blocks work from a task list prepared on the host.
 * Builds the task list for batches up to max_batch and contexts up to max_ctx
 * tokens (positions 0..max_ctx-1) on the current device (its SM count sets
 * the tile sizes and the grid) and uploads it.  max_batch 1 streams every
 * weight row through CUDA-core GEMV tiles; max_batch 2..64 (dense models
 * only) uses tcgen05 tensor-core tiles for the projections, with the batch as
 * the MMA's N dimension (padded to 16, 32 or 64).  Operator graph -> per-tile
 * tasks; a task depends on the tasks whose output rows overlap its input
 * rows (MPK digest, "Part 1. Compiler"; HN thread answer on task granularity
 * and dependency analysis). */
mk_status mk_build_taskgraph(mk_model* model, int max_batch, int max_ctx, mk_graph** out);

/* Passage: none of its own (a measurement aid for the per-tile-type evidence).
 * Profiling aid: the graph's tasks of one dense operator kind only (op in
 * MK_OP_QKV..MK_OP_LMHEAD, every layer), with no dependencies, so one tile type
 * can be timed and profiled alone.  Its outputs are not a decode step. */
mk_status mk_build_taskgraph_solo(mk_model* model, int max_batch, int max_ctx, int op, mk_graph** out);

/* Passage: MPK digest, "Part 1. Compiler" (as mk_build_taskgraph).
 * The same plan on the host only (no device memory, no CUDA call), for an
 * SM count given by the caller: for inspecting and checking the graph. */
mk_status mk_plan_taskgraph(const mk_model_desc* desc, int max_batch, int max_ctx, int n_sm,
                            mk_graph** out);
/* Passage: none of its own.  Releases a graph (host and device copies). */
void mk_graph_destroy(mk_graph* graph);

typedef struct {
    int n_tasks, n_events, n_sm, max_batch, max_ctx;
    int attn_splits;       /* split-K factor of decode attention per (sequence, kv head) */
    int n_ops;             /* operator kinds used (see mk_task_info.op) */
    int64_t weight_bytes_per_step;   /* bf16 weight bytes streamed by one B=1 step (dense: all
                                        but the embedding table; MoE: router + top_k experts) */
} mk_graph_info;
/* Passage: MPK digest, "Part 1. Compiler" (the task graph's size).  Copies the
 * graph's summary to *info (host memory). */
mk_status mk_graph_get_info(const mk_graph* graph, mk_graph_info* info);

/* Operator kinds of a task. */
enum {
    MK_OP_QKV = 1,        /* rows of [Wq;Wk;Wv] . rmsnorm(x)           */
    MK_OP_ATTN = 2,       /* decode attention split (b, kv head, split) */
    MK_OP_OPROJ = 3,      /* rows of Wo . o, plus the residual          */
    MK_OP_GATEUP = 4,     /* rows of silu(Wg h) * (Wu h)                */
    MK_OP_DOWN = 5,       /* rows of Wd . a, plus the residual          */
    MK_OP_LMHEAD = 6,     /* rows of Wlm . rmsnorm(x)                   */
    MK_OP_ROUTER = 7,     /* rows of Wr . rmsnorm(x); last tile: top-k  */
    MK_OP_EXP_GATEUP = 8, /* expert slot k: rows of silu(Wg_e h)*(Wu_e h) */
    MK_OP_EXP_DOWN = 9,   /* expert slot k: rows of Wd_e . a_e          */
    /* Batched graphs (max_batch > 1, dense models) replace the GEMV tiles with
     * tensor-core tiles: 128 weight rows times all batch rows, over one K-split.
     * The last split of a tile to finish reduces the splits' partial sums in
     * split order and applies the operator's epilogue. */
    MK_OP_NORM = 10,      /* rmsnorm of batch rows [r0, r1) into the bf16 hi/lo operand
                             of the next projection (aux: 0 attention, 1 FFN, 2 final) */
    MK_OP_MM_QKV = 11,    /* rows [r0, r1) of [Wq;Wk;Wv] . h for every batch row */
    MK_OP_MM_OPROJ = 12,  /* rows of Wo . o plus the residual */
    MK_OP_MM_GATEUP = 13, /* FFN rows [r0, r1) (<= 64): silu(Wg h) * (Wu h) */
    MK_OP_MM_DOWN = 14,   /* rows of Wd . a plus the residual */
    MK_OP_MM_LMHEAD = 15, /* rows of Wlm . rmsnorm(x) */
    MK_OP_KVAPPEND = 16,  /* batched graphs: K (rotated) and V of batch rows [r0, r1) into
                             their pages; the attention tasks of the layer wait for them */
    MK_OP_ATTN_MERGE = 17,/* long-context batch-1 graphs: q heads [r0, r1) of sequence b, the
                             splits' softmax partials merged (their attention tasks cover every
                             KV head of a page, exported with aux = -1) */
    MK_OP_TP_REDUCE = 18  /* tensor-parallel graphs: rows [r0, r1) of the residual stream after
                             attention (aux 0) or the FFN (aux 1): waits until every rank has
                             pushed its partial sums of those rows, adds them in rank order */
};

#define MK_NO_EVENT 0xFFFFFFFFu

/* One task as the device sees it.  Rows [r0, r1) of the operator's output;
 * for MK_OP_ATTN r0 is the split index and r1 the split count; b is the batch
 * row (MK_OP_ATTN / expert ops) and aux the kv head or expert slot.  The task
 * waits until counter[wait[i]] >= threshold[wait[i]] * epoch, then signals
 * counter[signal] += 1 (attention splits: only the last split of a
 * (b, kv head) signals, after merging the partial results; router tiles: only
 * the last tile of a layer, after selecting the experts).  Expert tasks also
 * wait on pointer_wait (the router's event) before the weight address of the
 * routed expert is read; MK_NO_EVENT elsewhere.  Tensor-core tiles
 * (MK_OP_MM_*) export b = their split index and aux = the tile's split count;
 * all splits of a tile name its event, and only the last to finish signals it. */
typedef struct {
    int op, layer, b, aux;
    uint32_t r0, r1;
    uint32_t wait[2];
    uint32_t signal;
    uint32_t pointer_wait;
} mk_task_info;

/* Passage: MPK digest, "Part 1. Compiler" (tasks, events and the edges between
 * them).  Copies min(cap, n_tasks) tasks in list order to out (host memory);
 * returns the count written via *n. */
mk_status mk_graph_export_tasks(const mk_graph* graph, mk_task_info* out, int cap, int* n);
/* Passage: MPK digest, "Part 2. Runtime", "Event-आधारित execution तरीका" (an
 * event fires when its counter reaches the threshold).  thresholds[e] for
 * e < n_events (per step), to host memory. */
mk_status mk_graph_export_thresholds(const mk_graph* graph, uint32_t* out, int cap, int* n);

/* Wave-quantisation arithmetic used by the tile sizer: n_tiles equal tiles on
 * n_sm SMs take ceil(n_tiles / n_sm) waves and leave idle SMs in the last
 * wave (Cohere page, "Honnan jön a gyorsulás?": 200 tiles on 132 SMs -> 2
 * waves, 64 SMs idle). */
mk_status mk_wave_stats(int n_tiles, int n_sm, int* waves, int* idle_sms_last_wave);

/* ---------------------------------------------------------------- state and steps */

/* Passage: Cohere page, section "Egyetlen tartós kernelre épül a
 * kiszolgálás": data dependencies are signalled by counters in global memory;
 * MPK digest, "Part 2. Runtime" (event counters and thresholds).
 * Allocates the device state of a graph (event counters, work-queue head,
 * activation buffers, attention partials): library-owned until
 * mk_state_destroy. */
mk_status mk_state_create(mk_graph* graph, mk_state** out);
/* Passage: none of its own.  Frees the state's device memory (after the work
 * queued on its stream has finished: the caller synchronises first). */
void mk_state_destroy(mk_state* state);

/* Passage: none of its own (every device-side wait is bounded).
 * Device-side wait limit in nanoseconds (default 2e9).  A wait that exceeds
 * it sets MK_ERR_TIMEOUT; the kernel then drains and returns. */
mk_status mk_state_set_timeout(mk_state* state, int64_t timeout_ns);

/* Passage: Cohere page, "Honnan jön a gyorsulás?", last paragraph: weight
 * tiles are fetched before their activation dependency is met.  The ring
 * already does that into shared memory; this optional hint also asks L2.
 * L2 prefetch distance, in tasks ahead of each CTA's latest claim (default 0
 * = off; every distance measured slower than none on B200).  A hint only:
 * results do not depend on it. */
mk_status mk_state_set_prefetch(mk_state* state, int tasks_ahead);

/* Passage: none of its own.
 * Test hook for failure detection: adds `offset` to the target of every
 * device-side event wait of later steps (0 = normal).  With offset 1 no wait
 * can be satisfied, so the step ends with MK_ERR_TIMEOUT after the state's
 * timeout, without faulting or hanging the device. */
mk_status mk_state_debug_wait_offset(mk_state* state, uint32_t offset);

/* Passage: Cohere page, section "Egyetlen tartós kernelre épül a
 * kiszolgálás": one persistent kernel runs a whole forward pass, exactly one
 * threadblock per SM resident for the decode step; section "Folyamatos
 * batchkezelés, paged attention ...": continuous batching over a paged KV
 * cache with ragged sequences.
 * One decode step for `batch` sequences (1 <= batch <= max_batch).
 *   token_ids  device int32 [batch]: the token fed to each sequence
 *   positions  device int32 [batch]: its position = tokens already cached
 *              (0 <= positions[b] < max_ctx); the step writes K/V at that
 *              position and attends to positions 0..positions[b]
 *   kv         paged cache (see mk_paged_kv); page_table rows 0..batch-1
 *   logits_out device fp32 [batch][vocab]
 * One kernel launch on `stream`.  Returns a device error recorded by an
 * earlier step of this state, if any (the state is then reset). */
mk_status mk_decode_step(mk_state* state, const int32_t* token_ids, const int32_t* positions,
                         int batch, const mk_paged_kv* kv, float* logits_out, mk_stream stream);

/* Passage: MPK digest, the benefits list (the launch and host overhead is
 * paid once, not per operator); Cohere page, "Honnan jön a gyorsulás?", first
 * reason (launch and synchronisation overhead paid once per step).
 * Greedy generation without a host round trip per token: n_steps decode steps
 * for `batch` sequences, enqueued at once on `stream`.  Step k feeds each
 * sequence the token chosen at step k - 1 (step 0: first_tokens, device int32
 * [batch]) at position positions[b] + k (positions: device int32 [batch]).
 * Inside the same launch the step's last LM-head tile writes the argmax of each
 * logits row (ties to the lowest index) to tokens_out[k][b] (device int32
 * [n_steps][batch]), so generation is one launch per token.
 * logits_out (device fp32 [batch][vocab]) holds each step's logits in turn.
 * Not for tensor-parallel states (each rank holds a vocabulary shard). */
mk_status mk_generate(mk_state* state, const int32_t* first_tokens, const int32_t* positions, int batch,
                      int n_steps, const mk_paged_kv* kv, int32_t* tokens_out, float* logits_out,
                      mk_stream stream);

/* Passage: Cohere page, "Honnan jön a gyorsulás?", first reason: between two
 * kernels every SM must finish before the next grid starts; HN thread
 * "Compiling LLMs into a MegaKernel", post #51 (CUDA graphs cannot overlap
 * across layers).
 * The same step as a kernel-per-operator baseline (the pages' comparison point:
 * kernels with boundaries between operators, MPK digest "Part 1"): one launch per
 * maximal run of tasks of one (operator, layer) in the task list, in order on
 * `stream`, each running the same tiles without the events that let the
 * megakernel overlap them.  Counters are zeroed first, so the whole call can be
 * captured into a CUDA graph and replayed.  Results equal mk_decode_step's.
 * n_launches (optional) receives the number of launches. */
mk_status mk_decode_step_per_op(mk_state* state, const int32_t* token_ids, const int32_t* positions,
                                int batch, const mk_paged_kv* kv, float* logits_out, mk_stream stream,
                                int* n_launches);

/* Passage: as mk_decode_step (the end-to-end form of the same step).
 * Same step with HOST inputs and outputs: copies token_ids and positions
 * (host int32 [batch]) to the device, runs the step, copies the logits back
 * to logits_host (host fp32 [batch][vocab]) and waits for the stream. */
mk_status mk_decode_step_host(mk_state* state, const int32_t* token_ids, const int32_t* positions,
                              int batch, const mk_paged_kv* kv, float* logits_host,
                              mk_stream stream);

/* Passage: MPK digest, "MPK का मुख्य मूल्य" (the measured workload: a
 * 39-token prompt, then generation); the prompt is one batched operator of the
 * task graph ("Part 1. Compiler": operators become tile tasks).
 * Runs the prompt of ONE sequence, the one whose page-table row is
 * kv->page_table[seq_slot] (0 <= seq_slot < max_batch; 0 for batch-1 graphs),
 * at positions 0 .. n_tokens-1: tokens is device int32 [n_tokens]; the logits
 * of the last prompt token go to last_logits (device fp32 [vocab]).
 *  - batch-1 graph: one token per step; the LM head is skipped for all but the
 *    last token;
 *  - batched graph (max_batch > 1): up to max_batch prompt tokens per step, as
 *    the batch rows of the tensor-core tiles (row i at position i), with causal
 *    attention over the cache: each row's K/V is appended before any row
 *    attends.
 * Errors: MK_ERR_INVALID_ARG for a null pointer, n_tokens < 1, n_tokens >
 * max_ctx or seq_slot out of range (returned before any launch). */
mk_status mk_prefill(mk_state* state, const int32_t* tokens, int n_tokens, int seq_slot,
                     const mk_paged_kv* kv, float* last_logits, mk_stream stream);

/* Passage: as mk_prefill.  mk_prefill continuing a sequence: the prompt goes
 * to positions pos0 .. pos0+n_tokens-1 of the sequence whose page-table row is
 * kv->page_table[seq_slot] (its positions 0..pos0-1 must already be cached). */
mk_status mk_prefill_seq(mk_state* state, const int32_t* tokens, int n_tokens, int pos0, int seq_slot,
                         const mk_paged_kv* kv, float* last_logits, mk_stream stream);

/* ---------------------------------------------------------------- tensor parallelism
 *
 * Passage: MPK digest, section "Part 1. Compiler": an all-reduce after a
 * matrix multiplication is a task of the graph like any other, and it can start
 * on the parts of the product that are done instead of after the whole
 * operator; the runtime of the same digest (one kernel per GPU computing and
 * communicating).  Russian MPK overview, the task-graph pseudocode (an
 * all-reduce task waiting on the matmul's event).
 *
 * A dense model split over tp ranks (one GPU each): rank r holds q heads
 * [r*nq/tp, (r+1)*nq/tp) with their KV heads, FFN rows [r*F/tp, (r+1)*F/tp)
 * and vocabulary rows [r*V/tp, (r+1)*V/tp) of the LM head.  Each O-projection
 * and down-projection tile stores its partial sums of its residual rows into
 * every rank's receive buffer (plain stores into peer memory) and raises that
 * tile's arrival flag on every rank (system-scope release); a reduce task per
 * tile on each rank waits for tp arrivals and adds the ranks' parts in rank
 * order, then the residual.  Only plain stores and reductions cross GPUs. */

#define MK_TP_IPC_HANDLE_BYTES 64

/* Registers rank tp_rank's shard of the model described by desc (the WHOLE
 * model's shape).  weight_ptrs follows mk_load_model's order with the shard's
 * shapes: tok_emb [vocab][hidden] whole; wq [nq/tp*d][hidden], wk and wv
 * [nkv/tp*d][hidden], wo [hidden][nq/tp*d] (the rank's columns), w_gate and
 * w_up [ffn/tp][hidden], w_down [hidden][ffn/tp], norms whole, lm_head
 * [vocab/tp][hidden].  Needs a dense model, 2 <= tp_size <= 8, n_kv_heads,
 * ffn (in multiples of 8 per rank) and vocab divisible by tp_size.
 * Errors: MK_ERR_UNSUPPORTED when the model does not divide; as mk_load_model
 * otherwise.  Graphs built from the model are batch-1 tensor-parallel graphs;
 * a state's KV cache holds the rank's nkv/tp heads and its logits the rank's
 * vocab/tp rows. */
mk_status mk_load_model_tp(const mk_model_desc* desc, int tp_size, int tp_rank, const void* const* weight_ptrs,
                           int n_ptrs, mk_model** out);

/* Host-only plan of rank tp_rank's batch-1 task graph (for inspection and
 * tests; no device needed), with the shard shapes mk_load_model_tp derives from
 * the whole model's desc.  The O- and down-projection tiles of each layer are
 * followed by one MK_OP_TP_REDUCE task per tile (same rows; aux 0 after
 * attention, 1 after the FFN), whose signal the next operator waits on; the
 * reduce tasks themselves wait on arrival flags, not events. */
mk_status mk_plan_taskgraph_tp(const mk_model_desc* desc, int tp_size, int tp_rank, int max_ctx, int n_sm,
                               mk_graph** out);

/* The state's own receive buffer and arrival flags (one device allocation of
 * *bytes bytes at *base, owned by the state).  Errors: MK_ERR_INVALID_ARG for a
 * state that is not tensor-parallel. */
mk_status mk_state_tp_buffer(mk_state* state, void** base, size_t* bytes);

/* Rank `rank`'s buffer (its mk_state_tp_buffer base) as addressable from this
 * state's device: a peer pointer after cudaDeviceEnablePeerAccess, or the same
 * device's pointer when the ranks are emulated on one GPU.  Borrowed.  Every
 * other rank must be set before a step. */
mk_status mk_state_tp_set_peer(mk_state* state, int rank, void* peer_base);

/* For ranks in separate processes: the IPC handle (MK_TP_IPC_HANDLE_BYTES
 * bytes to handle_out, host memory) of this state's buffer, and the opening of
 * a peer's handle (kept open until mk_state_destroy). */
mk_status mk_state_tp_ipc_handle(mk_state* state, void* handle_out);
mk_status mk_state_tp_open_peer(mk_state* state, int rank, const void* handle);

/* A tensor-parallel decode step on every rank: each rank launches
 * mk_decode_step on its own GPU with the same token and position (the ranks'
 * kernels meet through the flags).  For n ranks on ONE GPU this call runs the
 * n ranks' steps in a single cooperative launch, each rank on n_sm/n of the
 * SMs (states[r] is rank r of n, 2 <= n <= 4, head_dim 128; kvs[r] and
 * logits_out[r] are the rank's cache and logits shard).  token_ids and
 * positions: device int32 [1]. */
mk_status mk_decode_step_tp_emulated(mk_state* const* states, int n, const int32_t* token_ids,
                                     const int32_t* positions, const mk_paged_kv* const* kvs,
                                     float* const* logits_out, mk_stream stream);

/* The decode step of mk_decode_step for callers that cannot allocate device
 * memory: code running where cudaMalloc is not allowed (inside a host callback,
 * a signal or real-time path, or a runtime that owns a fixed memory budget and
 * forbids later allocations).  The pages describe no such entry point; it is a
 * convenience of this library.
 *   It allocates no device memory and needs no mk_model / mk_graph / mk_state:
 * the task list, RoPE table, per-layer pointer table, event counters,
 * activations and attention partials live in one fixed 32 MiB device array
 * (file scope, per GPU, held until the process exits).  Arguments are those of
 * mk_load_model + mk_decode_step for one sequence (batch must be 1) with
 * contexts up to max_ctx tokens; the caller passes the weights, the paged KV
 * cache, token and position (device int32 [1]) and logits_out (device fp32
 * [vocab]).  A model/context whose scratch would exceed 32 MiB is rejected with
 * MK_ERR_UNSUPPORTED (mk_last_error_string() gives the size needed).
 *   The first call on a device (and the first after the model, its weight
 * pointers or max_ctx change) looks up the array's device address, plans the
 * task list on the host and copies it into the array; later calls only clear
 * the counters and launch.  Every call shares the array: calls that overlap on
 * the GPU (other streams, other host threads' work in flight) race.  The call
 * waits for its step and returns the step's device status. */
mk_status mk_decode_step_noalloc(const mk_model_desc* desc, const void* const* weight_ptrs, int n_ptrs,
                                 int max_ctx, const int32_t* token_ids, const int32_t* positions,
                                 int batch, const mk_paged_kv* kv, float* logits_out, mk_stream stream);

/* Passage: none of its own (error reporting of the persistent kernel's bounded
 * waits: Cohere page, "Egyetlen tartós kernelre épül a kiszolgálás", counters
 * in global memory).
 * Waits for the stream and returns the device status word of the last step
 * (MK_OK, MK_ERR_TIMEOUT, MK_ERR_INVALID_ARG, ...). */
mk_status mk_sync(mk_state* state, mk_stream stream);

/* ---------------------------------------------------------------- inspection */

typedef struct {
    uint32_t epoch;            /* steps completed since creation or reset */
    uint32_t done;             /* tasks completed, total (= n_tasks * epoch) */
    uint64_t queue_head;       /* work-queue head (= (n_tasks + n_sm) * epoch) */
    int32_t error;             /* device status word */
    int32_t error_info[4];     /* where: task, event, value, detail */
} mk_state_counters;

/* Passage: MPK digest, "Part 2. Runtime", "Event-आधारित execution तरीका": each
 * finished task increments its event counter up to the threshold.
 * Synchronises the stream, then copies the counters; events (host uint32
 * [n_events]) may be NULL. */
mk_status mk_state_read_counters(mk_state* state, mk_stream stream, mk_state_counters* c,
                                 uint32_t* events, int cap);

/* Passage: none of its own (inspection of the step's intermediate results).
 * Copies an activation buffer of the last step to host fp32 memory.
 *   which 0: residual stream after attention [batch][hidden] of `layer`
 *         1: residual stream after the FFN   [batch][hidden] of `layer`
 *            (dense models; an MoE layer keeps its FFN output per expert slot)
 *         3: MoE selected experts of `layer`, as fp32 [batch][top_k]
 *         4: MoE combine weights of `layer`           [batch][top_k]
 * n = number of floats to copy. */
mk_status mk_state_read_buffer(mk_state* state, int which, int layer, float* host, size_t n,
                               mk_stream stream);

/* Passage: none of its own; it measures what the Cohere page's "Honnan jön a
 * gyorsulás?" describes (idle SMs between dependent tiles).
 * Per-task trace of the last step (needs MK_FLAG_TRACE): host uint64
 * [n_tasks][4] = {wait start ns, compute start ns, end ns, sm id}. */
mk_status mk_state_read_trace(mk_state* state, uint64_t* host, int cap_tasks, mk_stream stream);

/* Passage: none of its own (as mk_state_read_trace).
 * Per-CTA cycle counters accumulated since the last read (needs
 * MK_FLAG_TRACE), then cleared: host uint64 [n_sm][8] = {producer waits for a
 * free ring slot, consumer waits for streamed data, dependency waits, kernel
 * cycles, -, signal-slot waits, -, -}. */
mk_status mk_state_read_stats(mk_state* state, uint64_t* host, int cap, mk_stream stream);

/* Passage: none of its own.  Text of the last error of the calling thread
 * ("" if none); the pointer stays valid until that thread's next call. */
const char* mk_last_error_string(void);

/* Passage: none of its own.  Library version string (static storage). */
const char* mk_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MK_H */
