// Host task-graph compiler interface.
#pragma once

#include <stdint.h>

#include <string>
#include <vector>

#include "mk_internal.h"

namespace mk {

struct GraphPlan {
    mk_model_desc desc{};
    int max_batch = 0, max_ctx = 0, n_sm = 0;
    int S = 1;                   // attention splits per (sequence, kv head)
    bool wide_attn = false;      // attention tasks cover every KV head (long contexts, batch 1)
    int n_router_tiles = 0;
    int n_events = 0;
    int64_t weight_bytes = 0;    // bf16 bytes streamed per B=1 step
    std::vector<int> tile_rows;  // qkv, o, gate/up, down, lm, router, expert gate/up, expert down
    std::vector<Task> tasks;     // topological order
    std::vector<uint32_t> thr;   // per-event threshold per step
    // batched graphs (max_batch > 1): tensor-core projection tiles
    int bp = 0;                  // padded batch (the MMA's N); 0 for batch-1 graphs
    int mm_slots = 0;            // split partial-sum slots per layer (each bp x 128 floats)
    int mm_counters = 0;         // per-tile split arrival counters
    int n_lm_tiles = 0;          // LM-head tiles (numbered by their aux)
    int tp = 1;                  // tensor-parallel ranks (desc holds this rank's shard shapes)
    int tp_tiles = 0;            // row tiles of the residual stream per reduce phase
};

int64_t ceil_div(int64_t a, int64_t b);
void wave_stats(int n_tiles, int n_sm, int* waves, int* idle);
int choose_tile_rows(int64_t rows, int64_t row_bytes, int n_blocks, int n_sm, int64_t target,
                     int divide);
bool validate_desc(const mk_model_desc& d, std::string& err);
bool plan_graph(const mk_model_desc& d, int max_batch, int max_ctx, int n_sm, GraphPlan& g,
                std::string& err, int tp = 1);
// The shapes of rank `rank`'s shard under tensor parallelism of `tp` ranks: q and
// KV heads, FFN rows and LM-head (vocabulary) rows divided evenly; false (with the
// reason) when the model does not divide.
bool tp_shard_desc(const mk_model_desc& full, int tp, int rank, mk_model_desc& out, std::string& err);
// Keeps only the tasks of operator `op` (all layers), without dependencies:
// a list for timing and profiling one tile type alone.
void make_solo(GraphPlan& g, int op);
// Fills each dense GEMV task's streaming plan (weight addresses, chunking) from
// the model's weight pointers (order of the C ABI's weight list).
void attach_weights(GraphPlan& g, const void* const* w);

}  // namespace mk
