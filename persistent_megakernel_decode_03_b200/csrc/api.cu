// C ABI of the decode megakernel (declared in include/mk.h): model
// registration, task-graph build and upload, per-stream state, decode steps.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "graph.h"
#include "megakernel.h"
#include "mk_internal.h"

using mk::GraphPlan;

struct mk_model {
    mk_model_desc desc{};        // this rank's shapes (tensor parallelism: the shard's)
    int device = 0;
    int tp = 1, tp_rank = 0;     // tensor-parallel size and rank
    int vocab_full = 0;          // rows of the token embedding (the whole vocabulary)
    std::vector<const void*> w;
    std::vector<mk::LayerW> h_layers;
    mk::LayerW* d_layers = nullptr;
};

struct mk_graph {
    GraphPlan plan;
    mk_model* model = nullptr;   // null for a host-only plan
    int device = -1;
    mk::Task* d_tasks = nullptr;
    uint32_t* d_thr = nullptr;
    float* d_rope = nullptr;
    std::vector<CUtensorMap> wmaps;   // batched graphs: operand slots (filled per state), then weights
    std::vector<std::pair<int, int>> phases;   // (first task, task count) of each (operator, layer) run
};

struct mk_state {
    mk_graph* g = nullptr;
    uint32_t epoch = 0;
    bool needs_reset = false;
    long long timeout_ns = 2000000000LL;
    uint32_t wait_offset = 0;
    // device memory
    uint32_t* events = nullptr;
    unsigned long long* queue = nullptr;   // [0] work queue ([1] unused)
    uint32_t pf_dist = 0;
    uint32_t* done = nullptr;
    int* err = nullptr;
    uint32_t* router_cnt = nullptr;
    uint32_t* attn_cnt = nullptr;
    float *x_mid = nullptr, *x_out = nullptr, *qkv = nullptr, *act = nullptr;
    float *part = nullptr, *attn_o = nullptr, *rlogits = nullptr, *moe_w = nullptr, *ypart = nullptr;
    int* moe_sel = nullptr;
    uint16_t* opnd[mk::kNumOperands] = {};   // batched graphs: bf16 hi/lo operands
    float* mm_part = nullptr;
    uint32_t* mm_cnt = nullptr;
    void* tmaps = nullptr;         // device copy of the tensor maps (operands, then weights)
    mk::ArgVal* lm_arg = nullptr;  // greedy generation: LM-head tiles' (max, index) parts
    mk::ArgVal* lm_garg = nullptr; // ... and the groups' results
    uint32_t* lm_cnt = nullptr;    // arrivals per group, then of the groups
    int32_t* tokpos = nullptr;     // host-input variant: [2][max_batch]
    float* logits = nullptr;       // host-output variant: [max_batch][vocab]
    unsigned long long* trace = nullptr;
    unsigned long long* stats = nullptr;
    int ncta = 0;                  // CTAs of the last step (the queue head advances by tasks + CTAs)
    // tensor parallelism: this rank's receive buffer [tp][L][2][H] floats followed by
    // its arrival flags [L][2][tiles] (one allocation, so one IPC handle covers it),
    // and every rank's copy as mapped here (own included)
    void* tp_buf = nullptr;
    size_t tp_recv_bytes = 0, tp_bytes = 0;
    void* tp_peer[mk::kMaxTp] = {};
    bool tp_ipc[mk::kMaxTp] = {};  // opened through an IPC handle (closed on destroy)
    std::vector<void*> allocs;
};

namespace {

thread_local std::string g_err;

mk_status fail(mk_status s, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_err = buf;
    return s;
}

mk_status cuda_fail(cudaError_t e, const char* what) {
    return fail(e == cudaErrorMemoryAllocation ? MK_ERR_OOM : MK_ERR_CUDA, "%s: %s", what,
                cudaGetErrorString(e));
}

int slots_per_layer(const mk_model_desc& d) { return d.n_experts > 0 ? 10 : 9; }

// cuTensorMapEncodeTiled, reached through the runtime's driver entry point (no
// link against the driver library).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    }
    return fn;
}

// A 2-D bf16 matrix [rows][cols] (row pitch cols * 2 bytes) loaded in boxes of
// box_rows x 64 columns (128 bytes) with the 128-byte swizzle; rows or columns
// past the matrix read as zeros.
bool encode_bf16_2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    EncodeTiledFn fn = encode_tiled_fn();
    if (!fn || ((uintptr_t)base & 15) || (cols * 2) % 16 != 0) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {(cuuint32_t)mk::kMmK, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename T>
mk_status dev_alloc(mk_state* s, T** p, size_t count) {
    if (count == 0) count = 1;
    void* v = nullptr;
    cudaError_t e = cudaMalloc(&v, count * sizeof(T));
    if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc");
    e = cudaMemset(v, 0, count * sizeof(T));
    if (e != cudaSuccess) {
        cudaFree(v);
        return cuda_fail(e, "cudaMemset");
    }
    s->allocs.push_back(v);
    *p = static_cast<T*>(v);
    return MK_OK;
}

void free_state_memory(mk_state* s) {
    for (int q = 0; q < mk::kMaxTp; ++q)
        if (s->tp_ipc[q] && s->tp_peer[q]) cudaIpcCloseMemHandle(s->tp_peer[q]);
    for (void* v : s->allocs) cudaFree(v);
    s->allocs.clear();
}

bool tp_ready(const mk_state* s) {
    const int tp = s->g->model ? s->g->model->tp : 1;
    for (int q = 0; q < tp; ++q)
        if (!s->tp_peer[q]) return false;
    return true;
}

mk_status reset_counters(mk_state* s, cudaStream_t st) {
    const GraphPlan& P = s->g->plan;
    const mk_model_desc& d = P.desc;
    cudaError_t e = cudaMemsetAsync(s->events, 0, sizeof(uint32_t) * std::max(1, P.n_events), st);
    if (e == cudaSuccess) e = cudaMemsetAsync(s->queue, 0, 2 * sizeof(unsigned long long), st);
    if (e == cudaSuccess) e = cudaMemsetAsync(s->done, 0, sizeof(uint32_t), st);
    if (e == cudaSuccess) e = cudaMemsetAsync(s->err, 0, sizeof(int) * 8, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(s->router_cnt, 0, sizeof(uint32_t) * d.n_layers, st);
    if (e == cudaSuccess)
        e = cudaMemsetAsync(s->attn_cnt, 0,
                            sizeof(uint32_t) * d.n_layers * s->g->plan.max_batch * d.n_kv_heads, st);
    if (e == cudaSuccess && s->mm_cnt)
        e = cudaMemsetAsync(s->mm_cnt, 0, sizeof(uint32_t) * std::max(1, s->g->plan.mm_counters), st);
    // the arrival flags count from zero again (every rank resets together: the flags
    // are raised by all ranks against the same step count)
    if (e == cudaSuccess && s->tp_buf)
        e = cudaMemsetAsync(static_cast<char*>(s->tp_buf) + s->tp_recv_bytes, 0, s->tp_bytes - s->tp_recv_bytes, st);
    if (e != cudaSuccess) return cuda_fail(e, "reset");
    s->epoch = 0;
    s->needs_reset = false;
    return MK_OK;
}

mk_status check_kv(const mk_state* s, const mk_paged_kv* kv) {
    if (!kv || !kv->k_pages || !kv->v_pages || !kv->page_table)
        return fail(MK_ERR_INVALID_ARG, "paged KV: null pointer");
    if (kv->page_size != mk::kPageSize) return fail(MK_ERR_INVALID_ARG, "paged KV: page_size must be 16");
    if (kv->n_pages < 1 || kv->max_pages_per_seq < 1)
        return fail(MK_ERR_INVALID_ARG, "paged KV: n_pages and max_pages_per_seq must be >= 1");
    if (((uintptr_t)kv->k_pages | (uintptr_t)kv->v_pages) & 15)
        return fail(MK_ERR_INVALID_ARG, "paged KV: pools must be 16-byte aligned");
    (void)s;
    return MK_OK;
}

mk::Params base_params(mk_state* s) {
    const GraphPlan& P = s->g->plan;
    const mk_model_desc& d = P.desc;
    const mk_model* m = s->g->model;
    mk::Params p;
    std::memset(&p, 0, sizeof(p));
    p.tasks = s->g->d_tasks;
    p.n_tasks = (uint32_t)P.tasks.size();
    p.thr = s->g->d_thr;
    p.events = s->events;
    p.queue = s->queue;
    p.pf_dist = s->pf_dist;
    p.done = s->done;
    p.err = s->err;
    p.router_cnt = s->router_cnt;
    p.attn_cnt = s->attn_cnt;
    p.timeout_ns = s->timeout_ns;
    p.wait_offset = s->wait_offset;
    p.trace = s->trace;
    p.stats = s->stats;
    p.layers = m->d_layers;
    const int L = d.n_layers;
    p.tok_emb = static_cast<const uint16_t*>(m->w[0]);
    p.final_norm = static_cast<const uint16_t*>(m->w[1 + L * slots_per_layer(d)]);
    p.lm_head = static_cast<const uint16_t*>(m->w[2 + L * slots_per_layer(d)]);
    p.L = L;
    p.H = d.hidden;
    p.nq = d.n_q_heads;
    p.nkv = d.n_kv_heads;
    p.hd = d.head_dim;
    p.F = d.ffn;
    p.V = m->vocab_full;             // embedding rows (the LM head's rows are the graph's)
    p.E = d.n_experts;
    p.topk = d.top_k;
    p.Fe = d.expert_ffn;
    p.renorm = d.moe_renorm;
    p.eps = d.rms_eps;
    p.max_ctx = P.max_ctx;
    p.max_batch = P.max_batch;
    p.S = P.S;
    p.n_router_tiles = P.n_router_tiles;
    p.rope = s->g->d_rope;
    p.x_mid = s->x_mid;
    p.x_out = s->x_out;
    p.qkv = s->qkv;
    p.act = s->act;
    p.part = s->part;
    p.attn_o = s->attn_o;
    p.rlogits = s->rlogits;
    p.moe_w = s->moe_w;
    p.moe_sel = s->moe_sel;
    p.ypart = s->ypart;
    p.seq_row = -1;
    p.pos_stride = 0;
    p.mm = P.bp > 0 ? 1 : 0;
    p.wide = P.wide_attn ? 1 : 0;
    p.bp = P.bp;
    p.tmaps = s->tmaps;
    for (int i = 0; i < mk::kNumOperands; ++i) p.opnd[i] = s->opnd[i];
    p.mm_part = s->mm_part;
    p.mm_cnt = s->mm_cnt;
    p.argmax_out = nullptr;
    p.n_lm_tiles = P.n_lm_tiles;
    p.lm_arg = s->lm_arg;
    p.lm_garg = s->lm_garg;
    p.lm_cnt = s->lm_cnt;
    p.tp = m->tp;
    p.tp_rank = m->tp_rank;
    p.tp_tiles = P.tp_tiles;
    for (int q = 0; q < m->tp && q < mk::kMaxTp; ++q) {
        char* b = static_cast<char*>(s->tp_peer[q]);
        p.tp_recv[q] = reinterpret_cast<float*>(b);
        p.tp_flag[q] = b ? reinterpret_cast<uint32_t*>(b + s->tp_recv_bytes) : nullptr;
    }
    return p;
}

// Starts a step of `ncta` CTAs: the epoch and the queue base (the queue head moved
// by tasks + CTAs in every earlier step since the last reset).
mk_status begin_step(mk_state* s, mk::Params& p, int ncta, cudaStream_t st) {
    if (s->ncta != ncta && s->epoch > 0) s->needs_reset = true;
    if (s->needs_reset) {
        mk_status r = reset_counters(s, st);
        if (r != MK_OK) return r;
    }
    s->ncta = ncta;
    s->epoch += 1;
    p.epoch = s->epoch;
    p.queue_base = (unsigned long long)(s->epoch - 1) * (s->g->plan.tasks.size() + (size_t)ncta);
    p.cta0 = 0;
    p.ncta = ncta;
    return MK_OK;
}

mk_status launch_step(mk_state* s, mk::Params& p, cudaStream_t st) {
    const GraphPlan& P = s->g->plan;
    if (P.tp > 1 && !tp_ready(s))
        return fail(MK_ERR_INVALID_ARG, "tensor-parallel step: the peers' receive buffers are not all set");
    mk_status r = begin_step(s, p, P.n_sm, st);
    if (r != MK_OK) return r;
    cudaError_t e = mk::megakernel_launch(p, P.n_sm, st);
    if (e != cudaSuccess) {
        s->needs_reset = true;
        return cuda_fail(e, "megakernel launch");
    }
    return MK_OK;
}

}  // namespace

namespace mk {
void set_last_error(const char* msg) { g_err = msg; }
}  // namespace mk

extern "C" {

const char* mk_last_error_string(void) { return g_err.c_str(); }
const char* mk_version(void) { return "mk 0.1 (sm_100a persistent decode megakernel)"; }

mk_status mk_wave_stats(int n_tiles, int n_sm, int* waves, int* idle) {
    if (n_tiles < 0 || n_sm < 1 || !waves || !idle) return fail(MK_ERR_INVALID_ARG, "wave_stats: bad argument");
    mk::wave_stats(n_tiles, n_sm, waves, idle);
    return MK_OK;
}

// ---------------------------------------------------------------- model

static mk_status load_model(const mk_model_desc* desc, const void* const* wp, int n_ptrs, int tp, int tp_rank,
                            int vocab_full, mk_model** out) {
    const mk_model_desc& d = *desc;
    std::string err;
    if (!mk::validate_desc(d, err)) return fail(MK_ERR_UNSUPPORTED, "mk_load_model: %s", err.c_str());
    if (!mk::megakernel_supports(d.n_q_heads / d.n_kv_heads, d.head_dim))
        return fail(MK_ERR_UNSUPPORTED, "mk_load_model: heads per group must be 1, 2, 4 or 8");
    const int need = 1 + d.n_layers * slots_per_layer(d) + 2;
    if (n_ptrs != need) return fail(MK_ERR_INVALID_ARG, "mk_load_model: expected %d weight pointers, got %d", need, n_ptrs);
    for (int i = 0; i < n_ptrs; ++i) {
        if (!wp[i]) return fail(MK_ERR_INVALID_ARG, "mk_load_model: weight pointer %d is null", i);
        if ((uintptr_t)wp[i] & 15) return fail(MK_ERR_INVALID_ARG, "mk_load_model: weight pointer %d is not 16-byte aligned", i);
    }
    mk_model* m = new (std::nothrow) mk_model;
    if (!m) return fail(MK_ERR_OOM, "mk_load_model: host allocation");
    m->desc = d;
    m->tp = tp;
    m->tp_rank = tp_rank;
    m->vocab_full = vocab_full;
    cudaGetDevice(&m->device);
    m->w.assign(wp, wp + n_ptrs);
    const int S = slots_per_layer(d);
    for (int l = 0; l < d.n_layers; ++l) {
        const void* const* q = wp + 1 + l * S;
        mk::LayerW lw;
        std::memset(&lw, 0, sizeof(lw));
        lw.attn_norm = (const uint16_t*)q[0];
        lw.wq = (const uint16_t*)q[1];
        lw.wk = (const uint16_t*)q[2];
        lw.wv = (const uint16_t*)q[3];
        lw.wo = (const uint16_t*)q[4];
        lw.ffn_norm = (const uint16_t*)q[5];
        if (d.n_experts > 0) {
            lw.w_router = (const uint16_t*)q[6];
            lw.w_gate = (const uint16_t*)q[7];
            lw.w_up = (const uint16_t*)q[8];
            lw.w_down = (const uint16_t*)q[9];
        } else {
            lw.w_gate = (const uint16_t*)q[6];
            lw.w_up = (const uint16_t*)q[7];
            lw.w_down = (const uint16_t*)q[8];
        }
        m->h_layers.push_back(lw);
    }
    cudaError_t e = cudaMalloc(&m->d_layers, sizeof(mk::LayerW) * d.n_layers);
    if (e == cudaSuccess)
        e = cudaMemcpy(m->d_layers, m->h_layers.data(), sizeof(mk::LayerW) * d.n_layers, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) {
        if (m->d_layers) cudaFree(m->d_layers);
        delete m;
        return cuda_fail(e, "mk_load_model");
    }
    *out = m;
    return MK_OK;
}

mk_status mk_load_model(const mk_model_desc* desc, const void* const* wp, int n_ptrs, mk_model** out) {
    if (!desc || !wp || !out) return fail(MK_ERR_INVALID_ARG, "mk_load_model: null argument");
    *out = nullptr;
    return load_model(desc, wp, n_ptrs, 1, 0, desc->vocab, out);
}

mk_status mk_load_model_tp(const mk_model_desc* desc, int tp_size, int tp_rank, const void* const* wp, int n_ptrs,
                           mk_model** out) {
    if (!desc || !wp || !out) return fail(MK_ERR_INVALID_ARG, "mk_load_model_tp: null argument");
    *out = nullptr;
    mk_model_desc d;
    std::string err;
    if (!mk::tp_shard_desc(*desc, tp_size, tp_rank, d, err))
        return fail(MK_ERR_UNSUPPORTED, "mk_load_model_tp: %s", err.c_str());
    return load_model(&d, wp, n_ptrs, tp_size, tp_rank, desc->vocab, out);
}

void mk_model_destroy(mk_model* m) {
    if (!m) return;
    if (m->d_layers) cudaFree(m->d_layers);
    delete m;
}

// ---------------------------------------------------------------- graph

mk_status mk_plan_taskgraph(const mk_model_desc* desc, int max_batch, int max_ctx, int n_sm, mk_graph** out) {
    if (!desc || !out) return fail(MK_ERR_INVALID_ARG, "mk_plan_taskgraph: null argument");
    *out = nullptr;
    mk_graph* g = new (std::nothrow) mk_graph;
    if (!g) return fail(MK_ERR_OOM, "mk_plan_taskgraph: host allocation");
    std::string err;
    if (!mk::plan_graph(*desc, max_batch, max_ctx, n_sm, g->plan, err)) {
        delete g;
        return fail(MK_ERR_UNSUPPORTED, "mk_plan_taskgraph: %s", err.c_str());
    }
    *out = g;
    return MK_OK;
}

mk_status mk_plan_taskgraph_tp(const mk_model_desc* desc, int tp_size, int tp_rank, int max_ctx, int n_sm,
                               mk_graph** out) {
    if (!desc || !out) return fail(MK_ERR_INVALID_ARG, "mk_plan_taskgraph_tp: null argument");
    *out = nullptr;
    mk_model_desc d;
    std::string err;
    if (!mk::tp_shard_desc(*desc, tp_size, tp_rank, d, err))
        return fail(MK_ERR_UNSUPPORTED, "mk_plan_taskgraph_tp: %s", err.c_str());
    mk_graph* g = new (std::nothrow) mk_graph;
    if (!g) return fail(MK_ERR_OOM, "mk_plan_taskgraph_tp: host allocation");
    if (!mk::plan_graph(d, 1, max_ctx, n_sm, g->plan, err, tp_size)) {
        delete g;
        return fail(MK_ERR_UNSUPPORTED, "mk_plan_taskgraph_tp: %s", err.c_str());
    }
    *out = g;
    return MK_OK;
}

static mk_status build_graph(mk_model* model, int max_batch, int max_ctx, int solo_op, mk_graph** out);

mk_status mk_build_taskgraph(mk_model* model, int max_batch, int max_ctx, mk_graph** out) {
    return build_graph(model, max_batch, max_ctx, 0, out);
}

mk_status mk_build_taskgraph_solo(mk_model* model, int max_batch, int max_ctx, int op, mk_graph** out) {
    if (op < MK_OP_QKV || op > MK_OP_EXP_DOWN || op == MK_OP_ROUTER || op == MK_OP_EXP_GATEUP ||
        op == MK_OP_EXP_DOWN)
        return fail(MK_ERR_INVALID_ARG, "mk_build_taskgraph_solo: op must be a dense operator (1..6)");
    return build_graph(model, max_batch, max_ctx, op, out);
}

static mk_status build_graph(mk_model* model, int max_batch, int max_ctx, int solo_op, mk_graph** out) {
    if (!model || !out) return fail(MK_ERR_INVALID_ARG, "mk_build_taskgraph: null argument");
    *out = nullptr;
    int dev = 0, n_sm = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "mk_build_taskgraph: device query");
    int coop = 0;
    cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev);
    if (!coop) return fail(MK_ERR_UNSUPPORTED, "mk_build_taskgraph: device lacks cooperative launch");
    const mk_model_desc& d = model->desc;
    int per_sm = 0;
    e = mk::megakernel_occupancy(d.n_q_heads / d.n_kv_heads, d.head_dim, &per_sm);
    if (e != cudaSuccess) return cuda_fail(e, "mk_build_taskgraph: occupancy query");
    if (per_sm < 1) return fail(MK_ERR_UNSUPPORTED, "mk_build_taskgraph: megakernel does not fit on one SM");
    mk_graph* g = nullptr;
    g = new (std::nothrow) mk_graph;
    if (!g) return fail(MK_ERR_OOM, "mk_build_taskgraph: host allocation");
    std::string perr;
    if (!mk::plan_graph(d, max_batch, max_ctx, n_sm, g->plan, perr, model->tp)) {
        delete g;
        return fail(MK_ERR_UNSUPPORTED, "mk_build_taskgraph: %s", perr.c_str());
    }
    g->model = model;
    g->device = dev;
    if (solo_op && g->plan.bp > 0) {
        mk_graph_destroy(g);
        return fail(MK_ERR_UNSUPPORTED, "mk_build_taskgraph_solo: batch-1 graphs only");
    }
    if (solo_op) mk::make_solo(g->plan, solo_op);
    mk::attach_weights(g->plan, model->w.data());
    const GraphPlan& P = g->plan;
    if (P.bp > 0) {
        // tensor maps of the weights for the tensor-core tiles (the operand slots in
        // front are filled by each state, which owns the operand buffers)
        const int L = d.n_layers, H = d.hidden, S = slots_per_layer(d);
        const uint64_t qr = (uint64_t)d.n_q_heads * d.head_dim, kr = (uint64_t)d.n_kv_heads * d.head_dim;
        g->wmaps.assign((size_t)mk::lm_map_index(L) + 1, CUtensorMap{});
        bool ok = true;
        for (int l = 0; l < L && ok; ++l) {
            const void* const* q = model->w.data() + 1 + l * S;
            ok = encode_bf16_2d(&g->wmaps[mk::weight_map_index(l, 0)], q[1], qr, H, mk::kMmRows) &&
                 encode_bf16_2d(&g->wmaps[mk::weight_map_index(l, 1)], q[2], kr, H, mk::kMmRows) &&
                 encode_bf16_2d(&g->wmaps[mk::weight_map_index(l, 2)], q[3], kr, H, mk::kMmRows) &&
                 encode_bf16_2d(&g->wmaps[mk::weight_map_index(l, 3)], q[4], H, qr, mk::kMmRows) &&
                 encode_bf16_2d(&g->wmaps[mk::weight_map_index(l, 4)], q[6], d.ffn, H, mk::kMmRows / 2) &&
                 encode_bf16_2d(&g->wmaps[mk::weight_map_index(l, 5)], q[7], d.ffn, H, mk::kMmRows / 2) &&
                 encode_bf16_2d(&g->wmaps[mk::weight_map_index(l, 6)], q[8], H, d.ffn, mk::kMmRows);
        }
        if (ok) ok = encode_bf16_2d(&g->wmaps[mk::lm_map_index(L)], model->w[2 + L * S], d.vocab, H, mk::kMmRows);
        if (!ok) {
            mk_graph_destroy(g);
            return fail(MK_ERR_CUDA, "mk_build_taskgraph: tensor map encoding failed");
        }
    }
    // RoPE table: cos/sin of pos * theta^(-2i/d), computed in double, stored fp32
    const int half = d.head_dim / 2;
    std::vector<float> rope((size_t)max_ctx * half * 2);
    for (int pos = 0; pos < max_ctx; ++pos)
        for (int i = 0; i < half; ++i) {
            double inv = std::pow((double)d.rope_theta, -2.0 * i / (double)d.head_dim);
            double a = (double)pos * inv;
            rope[((size_t)pos * half + i) * 2 + 0] = (float)std::cos(a);
            rope[((size_t)pos * half + i) * 2 + 1] = (float)std::sin(a);
        }
    // the kernel-per-op baseline launches each maximal run of one (operator, layer,
    // and for norm tasks their kind)
    for (size_t i = 0; i < P.tasks.size();) {
        size_t j = i + 1;
        while (j < P.tasks.size() && P.tasks[j].op == P.tasks[i].op && P.tasks[j].layer == P.tasks[i].layer &&
               (P.tasks[i].op != MK_OP_NORM || P.tasks[j].aux == P.tasks[i].aux))
            ++j;
        g->phases.emplace_back((int)i, (int)(j - i));
        i = j;
    }
    e = cudaMalloc(&g->d_tasks, sizeof(mk::Task) * P.tasks.size());
    if (e == cudaSuccess) e = cudaMalloc(&g->d_thr, sizeof(uint32_t) * std::max<size_t>(1, P.thr.size()));
    if (e == cudaSuccess) e = cudaMalloc(&g->d_rope, sizeof(float) * rope.size());
    if (e == cudaSuccess)
        e = cudaMemcpy(g->d_tasks, P.tasks.data(), sizeof(mk::Task) * P.tasks.size(), cudaMemcpyHostToDevice);
    if (e == cudaSuccess && !P.thr.empty())
        e = cudaMemcpy(g->d_thr, P.thr.data(), sizeof(uint32_t) * P.thr.size(), cudaMemcpyHostToDevice);
    if (e == cudaSuccess)
        e = cudaMemcpy(g->d_rope, rope.data(), sizeof(float) * rope.size(), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) {
        mk_graph_destroy(g);
        return cuda_fail(e, "mk_build_taskgraph: upload");
    }
    *out = g;
    return MK_OK;
}

void mk_graph_destroy(mk_graph* g) {
    if (!g) return;
    if (g->d_tasks) cudaFree(g->d_tasks);
    if (g->d_thr) cudaFree(g->d_thr);
    if (g->d_rope) cudaFree(g->d_rope);
    delete g;
}

mk_status mk_graph_get_info(const mk_graph* g, mk_graph_info* info) {
    if (!g || !info) return fail(MK_ERR_INVALID_ARG, "mk_graph_get_info: null argument");
    const GraphPlan& P = g->plan;
    info->n_tasks = (int)P.tasks.size();
    info->n_events = P.n_events;
    info->n_sm = P.n_sm;
    info->max_batch = P.max_batch;
    info->max_ctx = P.max_ctx;
    info->attn_splits = P.S;
    info->n_ops = P.bp > 0 ? 8 : (P.desc.n_experts > 0 ? 7 : 6);   // batched: norm, append, attention, 5 tiles
    info->weight_bytes_per_step = P.weight_bytes;
    return MK_OK;
}

mk_status mk_graph_export_tasks(const mk_graph* g, mk_task_info* out, int cap, int* n) {
    if (!g || !n || (cap > 0 && !out)) return fail(MK_ERR_INVALID_ARG, "mk_graph_export_tasks: bad argument");
    const auto& T = g->plan.tasks;
    int k = std::min<int>(cap, (int)T.size());
    for (int i = 0; i < k; ++i) {
        out[i].op = T[i].op;
        out[i].layer = T[i].layer;
        out[i].b = T[i].b;
        out[i].aux = T[i].aux;
        out[i].r0 = T[i].r0;
        out[i].r1 = T[i].r1;
        out[i].wait[0] = T[i].wait0;
        out[i].wait[1] = T[i].wait1;
        out[i].signal = T[i].sig;
        out[i].pointer_wait = T[i].pad;
        if (T[i].op == MK_OP_ATTN && (T[i].flags & mk::kAttnWide)) out[i].aux = -1;   // every KV head
        // tensor parallelism: pad is a projection tile's ordinal (its arrival flag)
        if (g->plan.tp > 1 && (T[i].op == MK_OP_OPROJ || T[i].op == MK_OP_DOWN || T[i].op == MK_OP_TP_REDUCE))
            out[i].pointer_wait = MK_NO_EVENT;
        if (mk::is_mm_op(T[i].op)) {          // split s of a tile with nblk splits
            out[i].b = T[i].chunk_rows;
            out[i].aux = T[i].nblk;
            out[i].pointer_wait = MK_NO_EVENT;
        }
    }
    *n = k;
    return MK_OK;
}

mk_status mk_graph_export_thresholds(const mk_graph* g, uint32_t* out, int cap, int* n) {
    if (!g || !n || (cap > 0 && !out)) return fail(MK_ERR_INVALID_ARG, "mk_graph_export_thresholds: bad argument");
    int k = std::min<int>(cap, (int)g->plan.thr.size());
    for (int i = 0; i < k; ++i) out[i] = g->plan.thr[i];
    *n = k;
    return MK_OK;
}

// ---------------------------------------------------------------- state

mk_status mk_state_create(mk_graph* g, mk_state** out) {
    if (!g || !out) return fail(MK_ERR_INVALID_ARG, "mk_state_create: null argument");
    if (!g->model || !g->d_tasks) return fail(MK_ERR_INVALID_ARG, "mk_state_create: graph was planned on the host only");
    *out = nullptr;
    mk_state* s = new (std::nothrow) mk_state;
    if (!s) return fail(MK_ERR_OOM, "mk_state_create: host allocation");
    s->g = g;
    const GraphPlan& P = g->plan;
    const mk_model_desc& d = P.desc;
    const size_t L = d.n_layers, B = P.max_batch, H = d.hidden;
    const size_t qkvw = (size_t)(d.n_q_heads + 2 * d.n_kv_heads) * d.head_dim;
    const size_t hpg = d.n_q_heads / d.n_kv_heads;
    mk_status st = MK_OK;
#define ALLOC(ptr, n) if (st == MK_OK) st = dev_alloc(s, &s->ptr, (n))
    ALLOC(events, (size_t)std::max(1, P.n_events));
    ALLOC(queue, 2);
    ALLOC(done, 1);
    ALLOC(err, 8);
    ALLOC(router_cnt, L);
    ALLOC(attn_cnt, L * B * d.n_kv_heads);
    ALLOC(x_mid, L * B * H);
    ALLOC(x_out, L * B * H);
    ALLOC(qkv, L * B * qkvw);
    if (d.n_experts > 0) {
        ALLOC(act, L * B * d.top_k * d.expert_ffn);
        ALLOC(rlogits, L * B * d.n_experts);
        ALLOC(moe_w, L * B * d.top_k);
        ALLOC(moe_sel, L * B * d.top_k);
        ALLOC(ypart, L * B * d.top_k * H);
    } else {
        ALLOC(act, L * B * d.ffn);
    }
    ALLOC(part, L * B * d.n_kv_heads * P.S * hpg * (d.head_dim + 2));
    ALLOC(attn_o, L * B * d.n_q_heads * d.head_dim);
    if (P.bp > 0) {
        const size_t BP = P.bp, qr = (size_t)d.n_q_heads * d.head_dim;
        ALLOC(opnd[mk::kOpXq], L * 2 * BP * H);
        ALLOC(opnd[mk::kOpXf], L * 2 * BP * H);
        ALLOC(opnd[mk::kOpAo], L * 2 * BP * qr);
        ALLOC(opnd[mk::kOpAct], L * 2 * BP * d.ffn);
        ALLOC(opnd[mk::kOpXl], 2 * BP * H);
        ALLOC(mm_part, (size_t)std::max(1, P.mm_slots) * BP * mk::kMmRows);
        ALLOC(mm_cnt, (size_t)std::max(1, P.mm_counters));
        if (st == MK_OK) {
            std::vector<CUtensorMap> maps = g->wmaps;
            const uint64_t rows = (uint64_t)L * 2 * BP;
            const uint32_t box = (uint32_t)(2 * BP);
            bool ok = encode_bf16_2d(&maps[mk::kOpXq], s->opnd[mk::kOpXq], rows, H, box) &&
                      encode_bf16_2d(&maps[mk::kOpXf], s->opnd[mk::kOpXf], rows, H, box) &&
                      encode_bf16_2d(&maps[mk::kOpAo], s->opnd[mk::kOpAo], rows, qr, box) &&
                      encode_bf16_2d(&maps[mk::kOpAct], s->opnd[mk::kOpAct], rows, d.ffn, box) &&
                      encode_bf16_2d(&maps[mk::kOpXl], s->opnd[mk::kOpXl], 2 * BP, H, box);
            if (!ok) st = fail(MK_ERR_CUDA, "mk_state_create: tensor map encoding failed");
            unsigned char* dm = nullptr;
            if (st == MK_OK) st = dev_alloc(s, &dm, maps.size() * sizeof(CUtensorMap));
            if (st == MK_OK) {
                cudaError_t e = cudaMemcpy(dm, maps.data(), maps.size() * sizeof(CUtensorMap), cudaMemcpyHostToDevice);
                if (e != cudaSuccess) st = cuda_fail(e, "mk_state_create: tensor maps");
                s->tmaps = dm;
            }
        }
    }
    {
        const size_t groups = (size_t)(P.n_lm_tiles + mk::kArgGroup - 1) / mk::kArgGroup;
        ALLOC(lm_arg, (size_t)P.n_lm_tiles * mk::kArgParts * B);
        ALLOC(lm_garg, groups * B);
        ALLOC(lm_cnt, groups + 1);
    }
    ALLOC(tokpos, 2 * B);
    ALLOC(logits, B * (size_t)d.vocab);
    if (d.flags & MK_FLAG_TRACE) ALLOC(trace, P.tasks.size() * 4);
    if (d.flags & MK_FLAG_TRACE) ALLOC(stats, (size_t)P.n_sm * 8);
    if (P.tp > 1 && st == MK_OK) {
        // receive buffer (every rank's partial sums of both phases of every layer) and
        // the arrival flags; the flags start at zero
        s->tp_recv_bytes = sizeof(float) * (size_t)P.tp * L * 2 * H;
        s->tp_bytes = s->tp_recv_bytes + sizeof(uint32_t) * L * 2 * (size_t)std::max(1, P.tp_tiles);
        unsigned char* b = nullptr;
        st = dev_alloc(s, &b, s->tp_bytes);
        s->tp_buf = b;
        s->tp_peer[g->model->tp_rank] = b;
    }
#undef ALLOC
    if (st != MK_OK) {
        free_state_memory(s);
        delete s;
        return st;
    }
    *out = s;
    return MK_OK;
}

void mk_state_destroy(mk_state* s) {
    if (!s) return;
    free_state_memory(s);
    delete s;
}

mk_status mk_state_set_timeout(mk_state* s, int64_t ns) {
    if (!s || ns < 1000) return fail(MK_ERR_INVALID_ARG, "mk_state_set_timeout: bad argument");
    s->timeout_ns = ns;
    return MK_OK;
}

mk_status mk_state_set_prefetch(mk_state* s, int tasks_ahead) {
    if (!s || tasks_ahead < 0) return fail(MK_ERR_INVALID_ARG, "mk_state_set_prefetch: bad argument");
    s->pf_dist = (uint32_t)tasks_ahead;
    return MK_OK;
}

mk_status mk_state_debug_wait_offset(mk_state* s, uint32_t offset) {
    if (!s) return fail(MK_ERR_INVALID_ARG, "mk_state_debug_wait_offset: null state");
    s->wait_offset = offset;
    return MK_OK;
}

mk_status mk_decode_step(mk_state* s, const int32_t* token_ids, const int32_t* positions, int batch,
                         const mk_paged_kv* kv, float* logits_out, mk_stream stream) {
    if (!s || !token_ids || !positions || !logits_out) return fail(MK_ERR_INVALID_ARG, "mk_decode_step: null argument");
    if (batch < 1 || batch > s->g->plan.max_batch)
        return fail(MK_ERR_INVALID_ARG, "mk_decode_step: batch %d outside 1..%d", batch, s->g->plan.max_batch);
    mk_status r = check_kv(s, kv);
    if (r != MK_OK) return r;
    mk::Params p = base_params(s);
    p.tokens = token_ids;
    p.positions = positions;
    p.pos_offset = 0;
    p.batch = batch;
    p.skip_lm = 0;
    p.k_pages = static_cast<uint16_t*>(kv->k_pages);
    p.v_pages = static_cast<uint16_t*>(kv->v_pages);
    p.page_table = kv->page_table;
    p.n_pages = kv->n_pages;
    p.max_pages = kv->max_pages_per_seq;
    p.logits = logits_out;
    return launch_step(s, p, (cudaStream_t)stream);
}

mk_status mk_decode_step_per_op(mk_state* s, const int32_t* token_ids, const int32_t* positions, int batch,
                                const mk_paged_kv* kv, float* logits_out, mk_stream stream, int* n_launches) {
    if (!s || !token_ids || !positions || !logits_out)
        return fail(MK_ERR_INVALID_ARG, "mk_decode_step_per_op: null argument");
    if (batch < 1 || batch > s->g->plan.max_batch)
        return fail(MK_ERR_INVALID_ARG, "mk_decode_step_per_op: batch %d outside 1..%d", batch, s->g->plan.max_batch);
    mk_status r = check_kv(s, kv);
    if (r != MK_OK) return r;
    if (s->g->plan.tp > 1)
        return fail(MK_ERR_UNSUPPORTED, "mk_decode_step_per_op: tensor-parallel graphs run as one launch per step");
    cudaStream_t st = (cudaStream_t)stream;
    // counters from zero, epoch 1 in every launch: each launch's waits are met by the
    // launches before it on the stream, and the next megakernel step starts afresh
    r = reset_counters(s, st);
    if (r != MK_OK) return r;
    const GraphPlan& P = s->g->plan;
    unsigned long long base = 0;
    for (const auto& ph : s->g->phases) {
        mk::Params p = base_params(s);
        p.tasks = s->g->d_tasks + ph.first;
        p.n_tasks = (uint32_t)ph.second;
        p.trace = nullptr;
        p.stats = nullptr;
        p.pf_dist = 0;
        p.tokens = token_ids;
        p.positions = positions;
        p.pos_offset = 0;
        p.batch = batch;
        p.skip_lm = 0;
        p.k_pages = static_cast<uint16_t*>(kv->k_pages);
        p.v_pages = static_cast<uint16_t*>(kv->v_pages);
        p.page_table = kv->page_table;
        p.n_pages = kv->n_pages;
        p.max_pages = kv->max_pages_per_seq;
        p.logits = logits_out;
        p.epoch = 1;
        p.queue_base = base;                       // each launch claims its tasks + one per CTA
        base += (unsigned long long)ph.second + (unsigned long long)P.n_sm;
        cudaError_t e = mk::megakernel_launch(p, P.n_sm, st, /*cooperative=*/false);
        if (e != cudaSuccess) {
            s->needs_reset = true;
            return cuda_fail(e, "per-op launch");
        }
    }
    s->epoch = 1;
    s->needs_reset = true;    // the queue head is not (n_tasks + grid) x epoch: reset before a megakernel step
    if (n_launches) *n_launches = (int)s->g->phases.size();
    return MK_OK;
}

mk_status mk_generate(mk_state* s, const int32_t* first_tokens, const int32_t* positions, int batch, int n_steps,
                      const mk_paged_kv* kv, int32_t* tokens_out, float* logits_out, mk_stream stream) {
    if (!s || !first_tokens || !positions || !tokens_out || !logits_out)
        return fail(MK_ERR_INVALID_ARG, "mk_generate: null argument");
    if (batch < 1 || batch > s->g->plan.max_batch || n_steps < 1)
        return fail(MK_ERR_INVALID_ARG, "mk_generate: batch %d or steps %d out of range", batch, n_steps);
    if (s->g->plan.tp > 1)
        return fail(MK_ERR_UNSUPPORTED, "mk_generate: a tensor-parallel rank holds only its vocabulary shard");
    mk_status r = check_kv(s, kv);
    if (r != MK_OK) return r;
    cudaStream_t st = (cudaStream_t)stream;
    // the argmax arrivals count from zero for this call
    const size_t groups = (size_t)(s->g->plan.n_lm_tiles + mk::kArgGroup - 1) / mk::kArgGroup;
    cudaError_t e = cudaMemsetAsync(s->lm_cnt, 0, sizeof(uint32_t) * (groups + 1), st);
    if (e != cudaSuccess) return cuda_fail(e, "mk_generate: clearing the argmax counters");
    for (int k = 0; k < n_steps; ++k) {
        // one launch per token: the step's last LM-head tile writes the argmax to
        // tokens_out[k], which the next launch reads as its tokens
        mk::Params p = base_params(s);
        p.tokens = (k == 0) ? first_tokens : tokens_out + (size_t)(k - 1) * batch;   // the previous choice
        p.positions = positions;
        p.pos_offset = k;
        p.batch = batch;
        p.skip_lm = 0;
        p.k_pages = static_cast<uint16_t*>(kv->k_pages);
        p.v_pages = static_cast<uint16_t*>(kv->v_pages);
        p.page_table = kv->page_table;
        p.n_pages = kv->n_pages;
        p.max_pages = kv->max_pages_per_seq;
        p.logits = logits_out;
        p.argmax_out = tokens_out + (size_t)k * batch;
        p.arg_epoch = (uint32_t)(k + 1);
        r = launch_step(s, p, st);
        if (r != MK_OK) return r;
    }
    return MK_OK;
}

mk_status mk_decode_step_host(mk_state* s, const int32_t* token_ids, const int32_t* positions, int batch,
                              const mk_paged_kv* kv, float* logits_host, mk_stream stream) {
    if (!s || !token_ids || !positions || !logits_host) return fail(MK_ERR_INVALID_ARG, "mk_decode_step_host: null argument");
    if (batch < 1 || batch > s->g->plan.max_batch)
        return fail(MK_ERR_INVALID_ARG, "mk_decode_step_host: batch %d outside 1..%d", batch, s->g->plan.max_batch);
    cudaStream_t st = (cudaStream_t)stream;
    const int B = s->g->plan.max_batch;
    cudaError_t e = cudaMemcpyAsync(s->tokpos, token_ids, sizeof(int32_t) * batch, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(s->tokpos + B, positions, sizeof(int32_t) * batch, cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess) return cuda_fail(e, "mk_decode_step_host: H2D");
    mk_status r = mk_decode_step(s, s->tokpos, s->tokpos + B, batch, kv, s->logits, stream);
    if (r != MK_OK) return r;
    e = cudaMemcpyAsync(logits_host, s->logits, sizeof(float) * (size_t)batch * s->g->plan.desc.vocab,
                        cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "mk_decode_step_host: D2H");
    return MK_OK;
}

mk_status mk_prefill_seq(mk_state* s, const int32_t* tokens, int n_tokens, int pos0, int seq_slot,
                         const mk_paged_kv* kv, float* last_logits, mk_stream stream) {
    if (!s || !tokens || !last_logits) return fail(MK_ERR_INVALID_ARG, "mk_prefill: null argument");
    const GraphPlan& P = s->g->plan;
    if (n_tokens < 1 || pos0 < 0 || pos0 + n_tokens > P.max_ctx)
        return fail(MK_ERR_INVALID_ARG, "mk_prefill: positions %d..%d outside the graph's context", pos0, pos0 + n_tokens - 1);
    if (seq_slot < 0 || seq_slot >= P.max_batch)
        return fail(MK_ERR_INVALID_ARG, "mk_prefill: sequence slot %d outside 0..%d", seq_slot, P.max_batch - 1);
    mk_status r = check_kv(s, kv);
    if (r != MK_OK) return r;
    auto common = [&](mk::Params& p) {
        p.positions = nullptr;
        p.seq_row = seq_slot;
        p.k_pages = static_cast<uint16_t*>(kv->k_pages);
        p.v_pages = static_cast<uint16_t*>(kv->v_pages);
        p.page_table = kv->page_table;
        p.n_pages = kv->n_pages;
        p.max_pages = kv->max_pages_per_seq;
    };
    if (P.bp > 0) {
        // batched graph: up to max_batch prompt tokens per launch, as the batch rows
        // (row i at position pos0 + start + i of the one sequence)
        const int B = P.max_batch;
        for (int start = 0; start < n_tokens; start += B) {
            const int chunk = std::min(B, n_tokens - start);
            mk::Params p = base_params(s);
            common(p);
            p.tokens = tokens + start;
            p.pos_offset = pos0 + start;
            p.pos_stride = 1;
            p.batch = chunk;
            p.skip_lm = 0;
            p.logits = s->logits;
            r = launch_step(s, p, (cudaStream_t)stream);
            if (r != MK_OK) return r;
            if (start + chunk == n_tokens) {
                cudaError_t e = cudaMemcpyAsync(last_logits, s->logits + (size_t)(chunk - 1) * P.desc.vocab,
                                                sizeof(float) * P.desc.vocab, cudaMemcpyDeviceToDevice,
                                                (cudaStream_t)stream);
                if (e != cudaSuccess) return cuda_fail(e, "mk_prefill: logits");
            }
        }
        return MK_OK;
    }
    for (int i = 0; i < n_tokens; ++i) {
        mk::Params p = base_params(s);
        common(p);
        p.tokens = tokens + i;
        p.pos_offset = pos0 + i;
        p.batch = 1;
        p.skip_lm = (i + 1 < n_tokens) ? 1 : 0;
        p.logits = last_logits;
        r = launch_step(s, p, (cudaStream_t)stream);
        if (r != MK_OK) return r;
    }
    return MK_OK;
}

mk_status mk_prefill(mk_state* s, const int32_t* tokens, int n_tokens, int seq_slot, const mk_paged_kv* kv,
                     float* last_logits, mk_stream stream) {
    return mk_prefill_seq(s, tokens, n_tokens, 0, seq_slot, kv, last_logits, stream);
}

// ---------------------------------------------------------------- tensor parallelism

mk_status mk_state_tp_buffer(mk_state* s, void** base, size_t* bytes) {
    if (!s || !base || !bytes) return fail(MK_ERR_INVALID_ARG, "mk_state_tp_buffer: null argument");
    if (!s->tp_buf) return fail(MK_ERR_INVALID_ARG, "mk_state_tp_buffer: not a tensor-parallel state");
    *base = s->tp_buf;
    *bytes = s->tp_bytes;
    return MK_OK;
}

mk_status mk_state_tp_set_peer(mk_state* s, int rank, void* peer_base) {
    if (!s || !s->tp_buf) return fail(MK_ERR_INVALID_ARG, "mk_state_tp_set_peer: not a tensor-parallel state");
    const mk_model* m = s->g->model;
    if (rank < 0 || rank >= m->tp || rank == m->tp_rank || !peer_base || ((uintptr_t)peer_base & 15))
        return fail(MK_ERR_INVALID_ARG, "mk_state_tp_set_peer: bad rank or pointer");
    if (s->tp_ipc[rank] && s->tp_peer[rank]) cudaIpcCloseMemHandle(s->tp_peer[rank]);
    s->tp_ipc[rank] = false;
    s->tp_peer[rank] = peer_base;
    return MK_OK;
}

mk_status mk_state_tp_ipc_handle(mk_state* s, void* handle_out) {
    if (!s || !s->tp_buf || !handle_out) return fail(MK_ERR_INVALID_ARG, "mk_state_tp_ipc_handle: bad argument");
    cudaIpcMemHandle_t h;
    cudaError_t e = cudaIpcGetMemHandle(&h, s->tp_buf);
    if (e != cudaSuccess) return cuda_fail(e, "mk_state_tp_ipc_handle");
    static_assert(sizeof(h) == MK_TP_IPC_HANDLE_BYTES, "IPC handle size");
    std::memcpy(handle_out, &h, sizeof(h));
    return MK_OK;
}

mk_status mk_state_tp_open_peer(mk_state* s, int rank, const void* handle) {
    if (!s || !s->tp_buf || !handle) return fail(MK_ERR_INVALID_ARG, "mk_state_tp_open_peer: bad argument");
    const mk_model* m = s->g->model;
    if (rank < 0 || rank >= m->tp || rank == m->tp_rank)
        return fail(MK_ERR_INVALID_ARG, "mk_state_tp_open_peer: bad rank");
    cudaIpcMemHandle_t h;
    std::memcpy(&h, handle, sizeof(h));
    void* ptr = nullptr;
    cudaError_t e = cudaIpcOpenMemHandle(&ptr, h, cudaIpcMemLazyEnablePeerAccess);
    if (e != cudaSuccess) return cuda_fail(e, "mk_state_tp_open_peer");
    if (s->tp_ipc[rank] && s->tp_peer[rank]) cudaIpcCloseMemHandle(s->tp_peer[rank]);
    s->tp_peer[rank] = ptr;
    s->tp_ipc[rank] = true;
    return MK_OK;
}

mk_status mk_decode_step_tp_emulated(mk_state* const* states, int n, const int32_t* token_ids,
                                     const int32_t* positions, const mk_paged_kv* const* kvs,
                                     float* const* logits_out, mk_stream stream) {
    if (!states || !token_ids || !positions || !kvs || !logits_out)
        return fail(MK_ERR_INVALID_ARG, "mk_decode_step_tp_emulated: null argument");
    if (n < 2 || n > mk::kMaxTpEmulated)
        return fail(MK_ERR_INVALID_ARG, "mk_decode_step_tp_emulated: %d ranks (2..4 in one launch)", n);
    int dev = 0, n_sm = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    const int per = n_sm / n;
    bool reset = false;
    for (int r = 0; r < n; ++r) {
        const mk_state* s = states[r];
        if (!s || !s->tp_buf || !logits_out[r])
            return fail(MK_ERR_INVALID_ARG, "mk_decode_step_tp_emulated: rank %d: not a tensor-parallel state", r);
        const mk_model* m = s->g->model;
        if (m->tp != n || m->tp_rank != r || s->g->device != dev)
            return fail(MK_ERR_INVALID_ARG, "mk_decode_step_tp_emulated: state %d is not rank %d of %d on this device",
                        r, r, n);
        if (!tp_ready(s)) return fail(MK_ERR_INVALID_ARG, "mk_decode_step_tp_emulated: rank %d: peers not set", r);
        mk_status st = check_kv(s, kvs[r]);
        if (st != MK_OK) return st;
        if (s->needs_reset || s->epoch != states[0]->epoch || (s->ncta != per && s->epoch > 0)) reset = true;
    }
    cudaStream_t st = (cudaStream_t)stream;
    mk::TpLaunch L;
    std::memset(&L, 0, sizeof(L));
    L.n = n;
    for (int r = 0; r < n; ++r) {
        mk_state* s = states[r];
        if (reset) s->needs_reset = true;      // the ranks count their steps together
        mk::Params p = base_params(s);
        p.tokens = token_ids;
        p.positions = positions;
        p.pos_offset = 0;
        p.batch = 1;
        p.skip_lm = 0;
        p.k_pages = static_cast<uint16_t*>(kvs[r]->k_pages);
        p.v_pages = static_cast<uint16_t*>(kvs[r]->v_pages);
        p.page_table = kvs[r]->page_table;
        p.n_pages = kvs[r]->n_pages;
        p.max_pages = kvs[r]->max_pages_per_seq;
        p.logits = logits_out[r];
        mk_status rs = begin_step(s, p, per, st);
        if (rs != MK_OK) return rs;
        p.cta0 = r * per;
        L.r[r] = p;
    }
    cudaError_t e = mk::megakernel_launch_tp_emulated(L, per * n, st);
    if (e != cudaSuccess) {
        for (int r = 0; r < n; ++r) states[r]->needs_reset = true;
        return cuda_fail(e, "mk_decode_step_tp_emulated: launch");
    }
    return MK_OK;
}

mk_status mk_sync(mk_state* s, mk_stream stream) {
    if (!s) return fail(MK_ERR_INVALID_ARG, "mk_sync: null state");
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "mk_sync");
    int err[8];
    e = cudaMemcpy(err, s->err, sizeof(err), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "mk_sync: status read");
    if (err[0] != 0) {
        s->needs_reset = true;
        return fail((mk_status)err[0], "device status %d (task %d, event/where %d, value %d, detail %d)", err[0],
                    err[1], err[2], err[3], err[4]);
    }
    return MK_OK;
}

// ---------------------------------------------------------------- inspection

mk_status mk_state_read_counters(mk_state* s, mk_stream stream, mk_state_counters* c, uint32_t* events, int cap) {
    if (!s || !c) return fail(MK_ERR_INVALID_ARG, "mk_state_read_counters: null argument");
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    int err[8];
    unsigned long long q = 0;
    uint32_t done = 0;
    if (e == cudaSuccess) e = cudaMemcpy(err, s->err, sizeof(err), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess) e = cudaMemcpy(&q, s->queue, sizeof(q), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess) e = cudaMemcpy(&done, s->done, sizeof(done), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess && events && cap > 0)
        e = cudaMemcpy(events, s->events, sizeof(uint32_t) * std::min(cap, s->g->plan.n_events), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "mk_state_read_counters");
    c->epoch = s->epoch;
    c->done = done;
    c->queue_head = q;
    c->error = err[0];
    for (int i = 0; i < 4; ++i) c->error_info[i] = err[1 + i];
    return MK_OK;
}

mk_status mk_state_read_buffer(mk_state* s, int which, int layer, float* host, size_t n, mk_stream stream) {
    if (!s || !host) return fail(MK_ERR_INVALID_ARG, "mk_state_read_buffer: null argument");
    const GraphPlan& P = s->g->plan;
    const mk_model_desc& d = P.desc;
    if (layer < 0 || layer >= d.n_layers) return fail(MK_ERR_INVALID_ARG, "mk_state_read_buffer: bad layer");
    const size_t B = P.max_batch;
    const void* src = nullptr;
    size_t avail = 0;
    std::vector<int> tmp;
    switch (which) {
        case 0: src = s->x_mid + layer * B * d.hidden; avail = B * d.hidden; break;
        case 1: src = s->x_out + layer * B * d.hidden; avail = B * d.hidden; break;
        case 3:
        case 4:
            if (d.n_experts == 0) return fail(MK_ERR_INVALID_ARG, "mk_state_read_buffer: not an MoE model");
            avail = B * d.top_k;
            src = (which == 3) ? (const void*)(s->moe_sel + layer * avail) : (const void*)(s->moe_w + layer * avail);
            break;
        default: return fail(MK_ERR_INVALID_ARG, "mk_state_read_buffer: bad buffer id");
    }
    if (n > avail) return fail(MK_ERR_INVALID_ARG, "mk_state_read_buffer: %zu floats requested, %zu available", n, avail);
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e == cudaSuccess) {
        if (which == 3) {
            tmp.resize(n);
            e = cudaMemcpy(tmp.data(), src, sizeof(int) * n, cudaMemcpyDeviceToHost);
            for (size_t i = 0; i < n; ++i) host[i] = (float)tmp[i];
        } else {
            e = cudaMemcpy(host, src, sizeof(float) * n, cudaMemcpyDeviceToHost);
        }
    }
    if (e != cudaSuccess) return cuda_fail(e, "mk_state_read_buffer");
    return MK_OK;
}

mk_status mk_state_read_stats(mk_state* s, uint64_t* host, int cap, mk_stream stream) {
    if (!s || !host) return fail(MK_ERR_INVALID_ARG, "mk_state_read_stats: null argument");
    if (!s->stats) return fail(MK_ERR_INVALID_ARG, "mk_state_read_stats: model was loaded without MK_FLAG_TRACE");
    int n = std::min<int>(cap, s->g->plan.n_sm * 8);
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e == cudaSuccess) e = cudaMemcpy(host, s->stats, sizeof(uint64_t) * n, cudaMemcpyDeviceToHost);
    if (e == cudaSuccess) e = cudaMemset(s->stats, 0, sizeof(uint64_t) * s->g->plan.n_sm * 8);
    if (e != cudaSuccess) return cuda_fail(e, "mk_state_read_stats");
    return MK_OK;
}

mk_status mk_state_read_trace(mk_state* s, uint64_t* host, int cap_tasks, mk_stream stream) {
    if (!s || !host) return fail(MK_ERR_INVALID_ARG, "mk_state_read_trace: null argument");
    if (!s->trace) return fail(MK_ERR_INVALID_ARG, "mk_state_read_trace: model was loaded without MK_FLAG_TRACE");
    int n = std::min<int>(cap_tasks, (int)s->g->plan.tasks.size());
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e == cudaSuccess) e = cudaMemcpy(host, s->trace, sizeof(uint64_t) * 4 * n, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "mk_state_read_trace");
    return MK_OK;
}

}  // extern "C"
