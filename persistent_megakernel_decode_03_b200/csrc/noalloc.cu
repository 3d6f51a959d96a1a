// mk_decode_step_noalloc: the decode step of mk_decode_step for callers that
// cannot allocate device memory (for example code that runs where cudaMalloc is
// forbidden or would disturb a fixed memory budget).  Everything the step needs
// besides its inputs and outputs lives in one file-scope device array of fixed
// size, which every GPU that loads this library keeps until the process exits.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "graph.h"
#include "megakernel.h"
#include "mk_internal.h"

namespace {

constexpr size_t kScratchBytes = 32ull << 20;   // 32 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

struct Layout {
    size_t tasks, thr, rope, layers, events, queue, done, err, router_cnt, attn_cnt;
    size_t x_mid, x_out, qkv, act, part, attn_o, rlogits, moe_w, moe_sel, ypart, end;
    size_t counters_begin, counters_end;   // [events .. attn_cnt] is cleared every call
};

struct DeviceCache {
    bool have_base = false;
    unsigned long long ctx_id = 0;         // CUDA context the address below belongs to
    unsigned char* base = nullptr;         // device address of g_scratch on this device
    bool have_plan = false;
    std::vector<unsigned char> key;        // desc + weight pointers + max_ctx + n_sm
    mk::GraphPlan plan;
    Layout lay{};
};

std::mutex g_mutex;
DeviceCache g_cache[kMaxDevices];

// Unique id of the calling thread's current CUDA context (driver calls reached
// through the runtime's entry-point query: no link against the driver library).
// A device reset or a new primary context loads the module afresh, and its array
// then holds nothing of earlier calls: the cache is keyed on this id.
bool current_ctx_id(unsigned long long* id) {
    using GetCur = CUresult (*)(CUcontext*);
    using GetId = CUresult (*)(CUcontext, unsigned long long*);
    static GetCur get_cur = nullptr;
    static GetId get_id = nullptr;
    if (!get_cur || !get_id) {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return false;
        get_cur = reinterpret_cast<GetCur>(f);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return false;
        get_id = reinterpret_cast<GetId>(f);
    }
    CUcontext ctx = nullptr;
    if (get_cur(&ctx) != CUDA_SUCCESS || !ctx) return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

Layout make_layout(const mk::GraphPlan& P) {
    const mk_model_desc& d = P.desc;
    const size_t L = d.n_layers, B = P.max_batch, H = d.hidden;
    const size_t hpg = d.n_q_heads / d.n_kv_heads;
    const size_t qkvw = (size_t)(d.n_q_heads + 2 * d.n_kv_heads) * d.head_dim;
    Layout o{};
    size_t at = 0;
    auto take = [&](size_t bytes) { const size_t r = at; at = align256(at + (bytes ? bytes : 1)); return r; };
    o.tasks = take(sizeof(mk::Task) * P.tasks.size());
    o.thr = take(sizeof(uint32_t) * P.thr.size());
    o.rope = take(sizeof(float) * (size_t)P.max_ctx * d.head_dim);
    o.layers = take(sizeof(mk::LayerW) * L);
    o.counters_begin = at;
    o.events = take(sizeof(uint32_t) * P.thr.size());
    o.queue = take(2 * sizeof(unsigned long long));
    o.done = take(sizeof(uint32_t));
    o.err = take(8 * sizeof(int));
    o.router_cnt = take(sizeof(uint32_t) * L);
    o.attn_cnt = take(sizeof(uint32_t) * L * B * d.n_kv_heads);
    o.counters_end = at;
    o.x_mid = take(sizeof(float) * L * B * H);
    o.x_out = take(sizeof(float) * L * B * H);
    o.qkv = take(sizeof(float) * L * B * qkvw);
    if (d.n_experts > 0) {
        o.act = take(sizeof(float) * L * B * d.top_k * d.expert_ffn);
        o.rlogits = take(sizeof(float) * L * B * d.n_experts);
        o.moe_w = take(sizeof(float) * L * B * d.top_k);
        o.moe_sel = take(sizeof(int) * L * B * d.top_k);
        o.ypart = take(sizeof(float) * L * B * d.top_k * H);
    } else {
        o.act = take(sizeof(float) * L * B * d.ffn);
        o.rlogits = o.moe_w = o.moe_sel = o.ypart = 0;
    }
    o.part = take(sizeof(float) * L * B * d.n_kv_heads * P.S * hpg * (d.head_dim + 2));
    o.attn_o = take(sizeof(float) * L * B * d.n_q_heads * d.head_dim);
    o.end = at;
    return o;
}

mk_status nfail(mk_status s, const char* msg) {
    mk::set_last_error(msg);   // read back with mk_last_error_string()
    return s;
}

}  // namespace

extern "C" mk_status mk_decode_step_noalloc(const mk_model_desc* desc, const void* const* weight_ptrs,
                                            int n_ptrs, int max_ctx, const int32_t* token_ids,
                                            const int32_t* positions, int batch,
                                            const mk_paged_kv* kv, float* logits_out, mk_stream stream) {
    if (!desc || !weight_ptrs || !token_ids || !positions || !logits_out || !kv)
        return nfail(MK_ERR_INVALID_ARG, "mk_decode_step_noalloc: null argument");
    if (batch != 1) return nfail(MK_ERR_INVALID_ARG, "mk_decode_step_noalloc: batch must be 1");
    if (!kv->k_pages || !kv->v_pages || !kv->page_table || kv->page_size != mk::kPageSize ||
        kv->n_pages < 1 || kv->max_pages_per_seq < 1 || (((uintptr_t)kv->k_pages | (uintptr_t)kv->v_pages) & 15))
        return nfail(MK_ERR_INVALID_ARG, "mk_decode_step_noalloc: bad paged KV description");
    const mk_model_desc& d = *desc;
    const int per_layer = d.n_experts > 0 ? 10 : 9;
    if (n_ptrs != 1 + d.n_layers * per_layer + 2)
        return nfail(MK_ERR_INVALID_ARG, "mk_decode_step_noalloc: wrong number of weight pointers");
    for (int i = 0; i < n_ptrs; ++i)
        if (!weight_ptrs[i] || ((uintptr_t)weight_ptrs[i] & 15))
            return nfail(MK_ERR_INVALID_ARG, "mk_decode_step_noalloc: null or unaligned weight pointer");
    if (!mk::megakernel_supports(d.n_q_heads > 0 && d.n_kv_heads > 0 ? d.n_q_heads / d.n_kv_heads : 0, d.head_dim))
        return nfail(MK_ERR_UNSUPPORTED, "mk_decode_step_noalloc: unsupported head layout");

    int dev = 0, n_sm = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return nfail(MK_ERR_CUDA, "mk_decode_step_noalloc: device query failed");
    if (dev < 0 || dev >= kMaxDevices) return nfail(MK_ERR_UNSUPPORTED, "mk_decode_step_noalloc: device index too large");
    cudaStream_t st = (cudaStream_t)stream;

    // the runtime makes the device's primary context current on first use; do that
    // before asking which context this is (cudaFree(nullptr) allocates nothing)
    e = cudaFree(nullptr);
    if (e != cudaSuccess) return nfail(MK_ERR_CUDA, "mk_decode_step_noalloc: no CUDA context");
    unsigned long long ctx_id = 0;
    if (!current_ctx_id(&ctx_id)) return nfail(MK_ERR_CUDA, "mk_decode_step_noalloc: context query failed");

    std::lock_guard<std::mutex> guard(g_mutex);
    DeviceCache& c = g_cache[dev];
    if (c.have_base && c.ctx_id != ctx_id) {
        // another context (after a device reset, or a new primary context): the array
        // was loaded afresh, so its address is looked up and the plan uploaded again
        c.have_base = false;
        c.have_plan = false;
    }
    if (!c.have_base) {
        // once per device and context, with that device current: the array's address
        void* base = nullptr;
        e = cudaGetSymbolAddress(&base, g_scratch);
        if (e != cudaSuccess || !base) return nfail(MK_ERR_CUDA, "mk_decode_step_noalloc: cudaGetSymbolAddress failed");
        c.base = static_cast<unsigned char*>(base);
        c.ctx_id = ctx_id;
        c.have_base = true;
    }
    // (re)plan when the model, its weights, the context or the device changed
    std::vector<unsigned char> key(sizeof(mk_model_desc) + sizeof(void*) * n_ptrs + 2 * sizeof(int));
    std::memcpy(key.data(), &d, sizeof(mk_model_desc));
    std::memcpy(key.data() + sizeof(mk_model_desc), weight_ptrs, sizeof(void*) * n_ptrs);
    std::memcpy(key.data() + sizeof(mk_model_desc) + sizeof(void*) * n_ptrs, &max_ctx, sizeof(int));
    std::memcpy(key.data() + sizeof(mk_model_desc) + sizeof(void*) * n_ptrs + sizeof(int), &n_sm, sizeof(int));
    if (!c.have_plan || c.key != key) {
        c.have_plan = false;
        mk::GraphPlan plan;
        std::string err;
        if (!mk::plan_graph(d, 1, max_ctx, n_sm, plan, err))
            return nfail(MK_ERR_UNSUPPORTED, ("mk_decode_step_noalloc: " + err).c_str());
        mk::attach_weights(plan, weight_ptrs);
        const Layout lay = make_layout(plan);
        if (lay.end > kScratchBytes) {
            char buf[256];
            snprintf(buf, sizeof(buf), "mk_decode_step_noalloc: this model and context need %zu bytes of "
                     "scratch, more than the %zu available", lay.end, kScratchBytes);
            return nfail(MK_ERR_UNSUPPORTED, buf);
        }
        std::vector<mk::LayerW> lw(d.n_layers);
        for (int l = 0; l < d.n_layers; ++l) {
            const void* const* q = weight_ptrs + 1 + l * per_layer;
            std::memset(&lw[l], 0, sizeof(mk::LayerW));
            lw[l].attn_norm = (const uint16_t*)q[0];
            lw[l].wq = (const uint16_t*)q[1];
            lw[l].wk = (const uint16_t*)q[2];
            lw[l].wv = (const uint16_t*)q[3];
            lw[l].wo = (const uint16_t*)q[4];
            lw[l].ffn_norm = (const uint16_t*)q[5];
            if (d.n_experts > 0) {
                lw[l].w_router = (const uint16_t*)q[6];
                lw[l].w_gate = (const uint16_t*)q[7];
                lw[l].w_up = (const uint16_t*)q[8];
                lw[l].w_down = (const uint16_t*)q[9];
            } else {
                lw[l].w_gate = (const uint16_t*)q[6];
                lw[l].w_up = (const uint16_t*)q[7];
                lw[l].w_down = (const uint16_t*)q[8];
            }
        }
        const int half = d.head_dim / 2;
        std::vector<float> rope((size_t)max_ctx * half * 2);
        for (int pos = 0; pos < max_ctx; ++pos)
            for (int i = 0; i < half; ++i) {
                const double a = (double)pos * std::pow((double)d.rope_theta, -2.0 * i / (double)d.head_dim);
                rope[((size_t)pos * half + i) * 2 + 0] = (float)std::cos(a);
                rope[((size_t)pos * half + i) * 2 + 1] = (float)std::sin(a);
            }
        // plain copies into the array (pageable host memory: staged before return)
        e = cudaMemcpyAsync(c.base + lay.tasks, plan.tasks.data(), sizeof(mk::Task) * plan.tasks.size(),
                            cudaMemcpyHostToDevice, st);
        if (e == cudaSuccess && !plan.thr.empty())
            e = cudaMemcpyAsync(c.base + lay.thr, plan.thr.data(), sizeof(uint32_t) * plan.thr.size(),
                                cudaMemcpyHostToDevice, st);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(c.base + lay.rope, rope.data(), sizeof(float) * rope.size(), cudaMemcpyHostToDevice, st);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(c.base + lay.layers, lw.data(), sizeof(mk::LayerW) * lw.size(),
                                cudaMemcpyHostToDevice, st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
        if (e != cudaSuccess) return nfail(MK_ERR_CUDA, "mk_decode_step_noalloc: upload of the task list failed");
        c.plan = std::move(plan);
        c.lay = lay;
        c.key = std::move(key);
        c.have_plan = true;
    }
    const mk::GraphPlan& P = c.plan;
    const Layout& lay = c.lay;
    // every call starts from zeroed counters (epoch 1): earlier calls leave nothing behind
    e = cudaMemsetAsync(c.base + lay.counters_begin, 0, lay.counters_end - lay.counters_begin, st);
    if (e != cudaSuccess) return nfail(MK_ERR_CUDA, "mk_decode_step_noalloc: clearing the counters failed");

    unsigned char* b = c.base;
    mk::Params p;
    std::memset(&p, 0, sizeof(p));
    p.tasks = reinterpret_cast<const mk::Task*>(b + lay.tasks);
    p.n_tasks = (uint32_t)P.tasks.size();
    p.epoch = 1;
    p.thr = reinterpret_cast<const uint32_t*>(b + lay.thr);
    p.events = reinterpret_cast<uint32_t*>(b + lay.events);
    p.queue = reinterpret_cast<unsigned long long*>(b + lay.queue);
    p.pf_dist = 0;
    p.queue_base = 0;
    p.done = reinterpret_cast<uint32_t*>(b + lay.done);
    p.err = reinterpret_cast<int*>(b + lay.err);
    p.router_cnt = reinterpret_cast<uint32_t*>(b + lay.router_cnt);
    p.attn_cnt = reinterpret_cast<uint32_t*>(b + lay.attn_cnt);
    p.timeout_ns = 2000000000LL;
    p.layers = reinterpret_cast<const mk::LayerW*>(b + lay.layers);
    p.tok_emb = static_cast<const uint16_t*>(weight_ptrs[0]);
    p.final_norm = static_cast<const uint16_t*>(weight_ptrs[1 + d.n_layers * per_layer]);
    p.lm_head = static_cast<const uint16_t*>(weight_ptrs[2 + d.n_layers * per_layer]);
    p.L = d.n_layers; p.H = d.hidden; p.nq = d.n_q_heads; p.nkv = d.n_kv_heads; p.hd = d.head_dim;
    p.F = d.ffn; p.V = d.vocab; p.E = d.n_experts; p.topk = d.top_k; p.Fe = d.expert_ffn;
    p.renorm = d.moe_renorm; p.eps = d.rms_eps;
    p.max_ctx = P.max_ctx; p.max_batch = P.max_batch; p.S = P.S; p.n_router_tiles = P.n_router_tiles;
    p.rope = reinterpret_cast<const float*>(b + lay.rope);
    p.x_mid = reinterpret_cast<float*>(b + lay.x_mid);
    p.x_out = reinterpret_cast<float*>(b + lay.x_out);
    p.qkv = reinterpret_cast<float*>(b + lay.qkv);
    p.act = reinterpret_cast<float*>(b + lay.act);
    p.part = reinterpret_cast<float*>(b + lay.part);
    p.attn_o = reinterpret_cast<float*>(b + lay.attn_o);
    p.wide = P.wide_attn ? 1 : 0;
    if (d.n_experts > 0) {
        p.rlogits = reinterpret_cast<float*>(b + lay.rlogits);
        p.moe_w = reinterpret_cast<float*>(b + lay.moe_w);
        p.moe_sel = reinterpret_cast<int*>(b + lay.moe_sel);
        p.ypart = reinterpret_cast<float*>(b + lay.ypart);
    }
    p.tokens = token_ids;
    p.positions = positions;
    p.seq_row = -1;
    p.pos_stride = 0;
    p.batch = 1;
    p.k_pages = static_cast<uint16_t*>(kv->k_pages);
    p.v_pages = static_cast<uint16_t*>(kv->v_pages);
    p.page_table = kv->page_table;
    p.n_pages = kv->n_pages;
    p.max_pages = kv->max_pages_per_seq;
    p.logits = logits_out;
    e = mk::megakernel_launch(p, P.n_sm, st);
    if (e != cudaSuccess) return nfail(MK_ERR_CUDA, "mk_decode_step_noalloc: launch failed");
    // wait and report the step's device status
    int errw[8];
    e = cudaMemcpyAsync(errw, b + lay.err, sizeof(errw), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return nfail(MK_ERR_CUDA, "mk_decode_step_noalloc: reading the status failed");
    if (errw[0] != 0) return nfail((mk_status)errw[0], "mk_decode_step_noalloc: the device reported an error");
    return MK_OK;
}
