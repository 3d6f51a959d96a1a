// Internal layout shared by the host task-graph compiler and the megakernel.
// Plain C++ (no CUDA types) so the host compiler can include it.
#pragma once

#include <stdint.h>

#include "../../include/mk.h"

namespace mk {

// Kernel geometry.  One CTA per SM: 8 consumer warps compute, 1 producer warp
// streams weights and KV pages into a shared-memory ring with bulk async copies,
// 1 epilogue warp finishes tasks (reduction, stores) and publishes completions.
constexpr int kConsumerWarps = 8;
constexpr int kConsumerThreads = kConsumerWarps * 32;
constexpr int kProducerWarp = kConsumerWarps;        // warp 8
constexpr int kEpilogueWarp = kConsumerWarps + 1;    // warp 9: task epilogues and event signals
constexpr int kPrefetchWarp = kConsumerWarps + 2;    // warp 10 (warp 11 idles)
constexpr int kThreads = 384;                        // 3 warpgroups: 2 consumer + 1 support
// Register split between the warpgroups (setmaxnreg): the support warpgroup gives
// registers to the consumers.  256*216 + 128*72 = 64512 must not exceed the
// launch's 384 * (registers per thread at launch); the build checks the launch
// count is at least kMinLaunchRegs.
constexpr int kConsumerRegs = 216;
constexpr int kSupportRegs = 72;
constexpr int kMinLaunchRegs = (256 * kConsumerRegs + 128 * kSupportRegs + 383) / 384;   // 168
constexpr int kStageBytes = 16 * 1024;
constexpr int kStages = 11;
constexpr int kMaxTaskRows = 64;        // rows (all weight blocks) of one GEMV task
constexpr int kMaxVecPerThread = 8;     // 16-byte vectors of x per consumer thread (K <= 16384)
constexpr int kMaxHeadsPerGroup = 8;
constexpr int kMaxTopK = 16;
constexpr int kPageSize = 16;

// GEMV fast-path variants (rows whose 16-byte vectors split evenly over the 256
// consumer threads): vectors per thread, rows per 16 KB stage, rows per task.
enum FastPath : uint8_t {
    kFastNone = 0,
    kFastV2R2N16 = 1,   // K = 4096, 2 rows per stage, 16 rows
    kFastV2R2N8 = 2,    // K = 4096, 2 rows per stage, 8 rows
    kFastV1R4N16 = 3,   // K = 2048, 4 rows per stage, 16 rows
    kFastV1R4N8 = 4,    // K = 2048, 4 rows per stage, 8 rows
    kFastV7S4N4 = 5,    // K = 14336, rows in 2 segments (4 + 3 vectors per thread), 4 rows
    kFastV7S4N2 = 6,    // K = 14336, 2 rows
    kFastV2R2N4 = 7,    // K = 4096, 4 rows (tail tiles)
    kFastV1R4N4 = 8,    // K = 2048, 4 rows (tail tiles)
    kFastV7S4N1 = 9,    // K = 14336, 1 row (tail tiles)
    kFastW2 = 10,       // K = 512: one row per warp per stage (8 rows per stage)
    kFastW3 = 11,       // K = 768
    kFastW4 = 12,       // K = 1024
};

// Short rows are given one warp each: a stage holds 8 rows, one per consumer warp.
#ifdef __CUDACC__
__host__ __device__
#endif
inline bool is_warp_row(uint8_t f) { return f >= kFastW2 && f <= kFastW4; }
constexpr int kWarpRows = 8;

// The variant for a GEMV tile of `rows` rows per weight block, `nblk` blocks, K columns.
inline uint8_t fast_path_for(int K, int rows, int nblk) {
    const int nvec = K / 8;
    if (nblk == 1 && rows <= kMaxTaskRows) {
        if (K == 512) return kFastW2;
        if (K == 768) return kFastW3;
        if (K == 1024) return kFastW4;
    }
    if (K % 8 != 0 || nvec % kConsumerThreads != 0) return kFastNone;
    const int vpt = nvec / kConsumerThreads, total = rows * nblk;
    const long long rb = 2LL * K;
    if (rb <= kStageBytes) {
        const int rps = (int)(kStageBytes / rb);
        if (rows % rps != 0) return kFastNone;
        if (vpt == 2 && rps == 2 && total == 16) return kFastV2R2N16;
        if (vpt == 2 && rps == 2 && total == 8) return kFastV2R2N8;
        if (vpt == 1 && rps == 4 && total == 16) return kFastV1R4N16;
        if (vpt == 1 && rps == 4 && total == 8) return kFastV1R4N8;
        if (vpt == 2 && rps == 2 && total == 4) return kFastV2R2N4;
        if (vpt == 1 && rps == 4 && total == 4) return kFastV1R4N4;
        return kFastNone;
    }
    if (vpt == 7 && total == 4) return kFastV7S4N4;
    if (vpt == 7 && total == 2) return kFastV7S4N2;
    if (vpt == 7 && total == 1) return kFastV7S4N1;
    return kFastNone;
}

// Batched projection tiles (tcgen05): 128 weight rows (the MMA's M) by the
// padded batch (its N: 16, 32 or 64) per tile, streamed in K-blocks of 64
// columns.  Each K-block's weight box (128 rows x 128 bytes, 128-byte swizzle,
// 16 KB) takes a ring stage; the activation boxes (the N hi rows then the N lo
// rows of the bf16 split of the fp32 input, 128-byte swizzle) of up to 4
// consecutive K-blocks share one more stage.
constexpr int kMmRows = 128;
constexpr int kMmK = 64;
constexpr int kMaxMmBatch = 64;
constexpr int kNormRowsPerTask = 1;     // a norm task: one batch row, all consumer threads
// Tensor maps: the five activation operands first, then the weights.
enum MmOperand { kOpXq = 0, kOpXf = 1, kOpAo = 2, kOpAct = 3, kOpXl = 4, kNumOperands = 5 };
constexpr int kMapsPerLayer = 7;        // wq, wk, wv, wo, w_gate, w_up, w_down
inline int weight_map_index(int layer, int which) { return kNumOperands + layer * kMapsPerLayer + which; }
inline int lm_map_index(int n_layers) { return kNumOperands + n_layers * kMapsPerLayer; }
#ifdef __CUDACC__
__host__ __device__
#endif
inline bool is_mm_op(int op) { return op >= MK_OP_MM_QKV && op <= MK_OP_MM_LMHEAD; }

// Decode attention over every KV head of a page at once ("wide" tasks, batch-1
// graphs from kWideAttnCtx positions of context): per split, the pages' keys and
// values of all heads stream as contiguous blocks (a page holds each head's 16 x d
// block back to back), and separate merge tasks combine the splits per q head.
constexpr int kWideAttnCtx = 32768;
constexpr uint8_t kAttnWide = 1;       // Task::flags of a wide attention task

// Tensor parallelism (dense batch-1 graphs): up to kMaxTp ranks; a launch that
// emulates the ranks on one GPU runs up to kMaxTpEmulated of them side by side.
constexpr int kMaxTp = 8;
constexpr int kMaxTpEmulated = 4;
constexpr uint32_t kTpFlagBit = 0x80000000u;   // epilogue: "raise tensor-parallel flag i" marker

// Device task record (32 bytes).
struct Task {
    uint8_t op;
    uint8_t flags;   // GEMV: fast-path variant chosen by the planner (kFast*), 0 = generic
    uint16_t layer;
    uint16_t b;      // batch row (attention / expert tasks)
    uint16_t aux;    // kv head (attention) or expert slot (expert tasks)
    uint32_t r0, r1; // output rows; attention: split index, split count
    uint32_t wait0, wait1;
    uint32_t sig;
    uint32_t pad;        // expert tasks: router event to wait on before reading the expert id
    // Streaming plan of a dense GEMV tile, filled when the graph is built for a
    // loaded model (zero otherwise): the weight rows of each block start at src[i];
    // chunks are chunk_rows whole rows, or (chunk_rows == 0) rows in stage-sized
    // segments.
    //
    // Tensor-core tiles (MK_OP_MM_*) use the same fields differently:
    //   src[i]     weight box i: tensor-map index (low 32 bits), first row (high 32)
    //   row_bytes  first K-block of this split; pad2: one past its last K-block
    //   chunk_rows split index s; nblk: the tile's split count
    //   nchunks    stages: one per K-block's weight box, plus one per group of
    //              16 KB / (2 * bp * 128 B) K-blocks' activation boxes
    //   pad        the tile's arrival counter; aux: partial-sum slot of split 0
    uint64_t src[2];
    uint32_t row_bytes;
    uint16_t chunk_rows;
    uint16_t nblk;
    uint32_t nchunks;
    uint32_t pad2;
};
static_assert(sizeof(Task) == 64, "task record is 64 bytes");

// (value, index) of a partial maximum (the in-step argmax), 8 bytes.
struct alignas(8) ArgVal {
    float v;
    int i;
};

// Per-layer weight pointers (bf16 bits).
struct LayerW {
    const uint16_t* attn_norm;
    const uint16_t* wq;
    const uint16_t* wk;
    const uint16_t* wv;
    const uint16_t* wo;
    const uint16_t* ffn_norm;
    const uint16_t* w_router;
    const uint16_t* w_gate;
    const uint16_t* w_up;
    const uint16_t* w_down;
};

struct Params {
    // task list and synchronisation
    const Task* tasks;
    uint32_t n_tasks;
    uint32_t epoch;              // 1-based step counter; thresholds are thr * epoch
    const uint32_t* thr;         // per-event threshold per step
    uint32_t* events;
    unsigned long long* queue;   // global work-queue head
    unsigned long long queue_base;
    uint32_t pf_dist;            // L2 prefetch at most this many tasks ahead of the CTA's claims (0: off)
    uint32_t* done;              // completed-task counter
    int* err;                    // [0] status, [1..4] info
    uint32_t* router_cnt;        // [L] router tile arrivals
    uint32_t* attn_cnt;          // [L][B][nkv] attention split arrivals (the last one merges)
    long long timeout_ns;
    uint32_t wait_offset;        // added to every wait target (0; tests set 1 to force a timeout)
    unsigned long long* trace;   // [n_tasks][4] or null
    unsigned long long* stats;   // [grid][8] per-CTA cycle counters (with trace) or null

    // model
    const LayerW* layers;
    const uint16_t* tok_emb;
    const uint16_t* final_norm;
    const uint16_t* lm_head;
    int L, H, nq, nkv, hd, F, V, E, topk, Fe, renorm;
    float eps;
    int max_ctx, max_batch, S, n_router_tiles;
    const float* rope;           // [max_ctx][hd/2][2] = cos, sin (fp32)

    // activations (fp32), per layer
    float* x_mid;    // [L][B][H]   residual after attention
    float* x_out;    // [L][B][H]   residual after the dense FFN
    float* qkv;      // [L][B][(nq+2nkv)*hd]
    float* act;      // dense: [L][B][F]; MoE: [L][B][topk][Fe]
    float* part;     // attention split partials: o [L][B][nkv][S][hpg][hd], then (m, l) pairs
    float* attn_o;   // [L][B][nq*hd] attention output, the splits merged and normalised
    float* rlogits;  // [L][B][E]
    float* moe_w;    // [L][B][topk]
    int* moe_sel;    // [L][B][topk]
    float* ypart;    // [L][B][topk][H]

    // per step
    const int* tokens;
    const int* positions;        // may be null (then position = pos_offset)
    int pos_offset;
    int pos_stride;              // position of row b = positions[b] + pos_offset + b * pos_stride
    int seq_row;                 // >= 0: every batch row uses this page-table row (batched prefill)
    int batch;
    int skip_lm;                 // 1: LM-head tasks do nothing
    uint16_t* k_pages;
    uint16_t* v_pages;
    const int* page_table;
    int n_pages, max_pages;
    float* logits;

    int wide;                    // 1: the graph's attention tasks cover every KV head
    int cta0, ncta;              // this step's CTAs: blockIdx.x - cta0 in [0, ncta) (several ranks
                                 // share a launch when tensor parallelism is emulated)
    // tensor parallelism: rank tp_rank of tp; the O- and down-projection tiles push
    // their partial sums into every rank's receive buffer and raise the tile's flag
    // there; reduce tasks wait on their own rank's flags and add the ranks in order
    int tp, tp_rank, tp_tiles;
    float* tp_recv[kMaxTp];      // rank q's receive buffer [tp][L][2][H]
    uint32_t* tp_flag[kMaxTp];   // rank q's flags [L][2][tp_tiles]
    // batched projection tiles (max_batch > 1)
    int mm;                      // 1: the graph uses tensor-core tiles
    int bp;                      // padded batch: the MMA's N (16, 32 or 64)
    const void* tmaps;           // CUtensorMap array (operands, then weights), 64-byte aligned
    uint16_t* opnd[kNumOperands];   // bf16 [rows][K]: per layer 2 * bp rows (hi, then lo)
    float* mm_part;              // split partial sums: [slot][bp][128]
    uint32_t* mm_cnt;            // per-tile split arrivals

    // greedy argmax inside the step (mk_generate): each LM-head tile leaves the
    // (value, index) of its rows' maximum per batch row, groups of kArgGroup tiles
    // are reduced by their last tile, and the last group writes the token
    int* argmax_out;             // device int32 [batch], or null: no argmax this step
    uint32_t arg_epoch;          // 1-based count of argmax steps since the counters were cleared
    int n_lm_tiles;              // LM-head tiles (their aux is the tile's ordinal)
    ArgVal* lm_arg;              // [n_lm_tiles * kArgParts][max_batch]
    ArgVal* lm_garg;             // [groups][max_batch]
    uint32_t* lm_cnt;            // [groups + 1] arrivals: per group, then of the groups
};
// The launch parameters of emulated tensor parallelism: the ranks' parameter
// blocks; the grid's CTAs are shared out among them.
struct TpLaunch {
    Params r[kMaxTpEmulated];
    int n;
};
// Parts per LM-head tile (a batched tile reduces its 128 rows in 4 warps) and tiles
// per reduction group of the in-step argmax.
constexpr int kArgParts = 4;
constexpr int kArgGroup = 32;

// Sets the text returned by mk_last_error_string() for the calling thread.
void set_last_error(const char* msg);

// Error status values written by the device (match mk_status).
constexpr int kErrInvalid = MK_ERR_INVALID_ARG;
constexpr int kErrTimeout = MK_ERR_TIMEOUT;
constexpr int kErrFault = MK_ERR_DEVICE_FAULT;

}  // namespace mk
