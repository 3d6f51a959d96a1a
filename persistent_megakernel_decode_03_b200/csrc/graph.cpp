// Host task-graph compiler: operator graph of one decode step -> per-tile
// tasks in a topological list + event counters with per-step thresholds.
//
// Follows the MPK digest ("LLM को MegaKernel में compile करके low-latency
// inference हासिल करना", section "Part 1. Compiler"): each operator is split
// into tasks of about one threadblock's work, events are the synchronisation
// points between tasks, and (HN thread "Compiling LLMs into a MegaKernel",
// answer #58) task B depends on task A when A's output elements overlap B's
// inputs.  Tile sizes avoid per-operator wave quantisation on the device's SM
// count (Cohere page, section "Honnan jön a gyorsulás?"), and dependencies
// stay at producer granularity: attention of one KV head waits only for the
// QKV tiles of that head's rows, an expert's down-projection only for its own
// gate/up tiles.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <map>
#include <numeric>
#include <string>
#include <vector>

#include "graph.h"

namespace mk {

namespace {

// Tensor kinds for the region-overlap analysis.
enum TensorKind { T_XIN = 1, T_QKV, T_O, T_XMID, T_ACT, T_ACTE, T_SEL, T_LOGITS,
                  T_PART,                     // wide attention: the splits' softmax partials
                  T_XQOP, T_XFOP, T_XLOP,     // bf16 hi/lo operands of batched tiles
                  T_KV,                       // batched graphs: this step's K/V rows in the cache
                  T_TPP };                    // tensor parallelism: a rank's partial sums (pushed to peers)

struct Region {
    int tensor;         // encoded (kind, layer, slot)
    int b_lo, b_hi;     // batch rows [b_lo, b_hi)
    int64_t lo, hi;     // element rows [lo, hi)
};

struct Entity {         // a producer: one task, or a merge / router-final reached by the last of several tasks
    std::vector<int> tasks;  // tasks that may signal on its behalf
    std::vector<Region> outs;
};

int tensor_key(int kind, int layer, int slot) { return (kind * 4096 + layer) * 64 + slot; }

bool overlaps(const Region& a, const Region& b) {
    return a.tensor == b.tensor && a.b_lo < b.b_hi && b.b_lo < a.b_hi && a.lo < b.hi && b.lo < a.hi;
}

struct UnionFind {
    std::vector<int> p;
    int add() { p.push_back((int)p.size()); return (int)p.size() - 1; }
    int find(int x) { while (p[x] != x) { p[x] = p[p[x]]; x = p[x]; } return x; }
    void unite(int a, int b) { a = find(a); b = find(b); if (a != b) p[std::max(a, b)] = std::min(a, b); }
};

int largest_divisor_at_most(int n, int cap) {
    for (int r = std::min(n, cap); r >= 1; --r)
        if (n % r == 0) return r;
    return 1;
}

}  // namespace

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

void wave_stats(int n_tiles, int n_sm, int* waves, int* idle) {
    int w = (int)ceil_div(n_tiles, n_sm);
    *waves = w;
    *idle = (n_tiles == 0) ? 0 : w * n_sm - n_tiles;
}

// Rows per GEMV tile.  Aims at `target` bytes per task; shrinks the tile while
// the operator would leave SMs without a tile; when `divide` > 0 the row count
// divides it (QKV tiles never straddle two heads, so each feeds one KV head).
int choose_tile_rows(int64_t rows, int64_t row_bytes, int n_blocks, int n_sm, int64_t target,
                     int divide) {
    // <= 16 rows per task where the fast GEMV path keeps row sums in registers; short
    // rows (<= 2 KB, no fast path) take up to 64 rows so a task still moves ~100 KB
    int cap = (row_bytes <= 2048) ? kMaxTaskRows / n_blocks : 16 / n_blocks;
    int R = (int)std::max<int64_t>(1, std::min<int64_t>(cap, target / (row_bytes * n_blocks)));
    if (divide > 0) R = largest_divisor_at_most(divide, R);
    const int64_t min_bytes = 16 * 1024;
    while (R > 1 && ceil_div(rows, R) < n_sm) {
        int next = (divide > 0) ? largest_divisor_at_most(divide, R - 1) : R - 1;
        if ((int64_t)next * row_bytes * n_blocks < min_bytes) break;
        R = next;
    }
    return R;
}

bool validate_desc(const mk_model_desc& d, std::string& err) {
    auto fail = [&](const std::string& m) { err = m; return false; };
    const int L = d.n_layers, H = d.hidden, nq = d.n_q_heads, nkv = d.n_kv_heads, hd = d.head_dim;
    const bool moe = d.n_experts > 0;
    if (moe && d.n_experts > 1024) return fail("at most 1024 experts");
    if (L <= 0 || H <= 0 || nq <= 0 || nkv <= 0 || hd <= 0 || d.vocab <= 0)
        return fail("model shape has a non-positive dimension");
    if (hd != 64 && hd != 128) return fail("head_dim must be 64 or 128");
    if (nq % nkv != 0) return fail("n_q_heads must be a multiple of n_kv_heads");
    if (nq / nkv > kMaxHeadsPerGroup) return fail("more than 8 q heads per kv head");
    if (H % 8 || (nq * hd) % 8) return fail("hidden and n_q*head_dim must be multiples of 8");
    if (H > 16384) return fail("hidden must be <= 16384");
    if (nq * hd > 8192) return fail("n_q*head_dim must be <= 8192");
    if (moe) {
        if (d.top_k <= 0 || d.top_k > kMaxTopK || d.top_k > d.n_experts)
            return fail("top_k must be in 1..min(16, n_experts)");
        if (d.expert_ffn <= 0 || d.expert_ffn % 8 || d.expert_ffn > 16384)
            return fail("expert_ffn must be a positive multiple of 8, <= 16384");
    } else {
        if (d.ffn <= 0 || d.ffn % 8 || d.ffn > 16384)
            return fail("ffn must be a positive multiple of 8, <= 16384");
    }
    if (d.dtype != MK_DTYPE_BF16) return fail("only bf16 weights are supported");

    return true;
}

bool plan_graph(const mk_model_desc& d, int max_batch, int max_ctx, int n_sm, GraphPlan& g,
                std::string& err, int tp) {
    auto fail = [&](const std::string& m) { err = m; return false; };
    if (!validate_desc(d, err)) return false;
    const int L = d.n_layers, H = d.hidden, nq = d.n_q_heads, nkv = d.n_kv_heads, hd = d.head_dim;
    const bool moe = d.n_experts > 0;
    if (max_batch < 1) return fail("max_batch must be >= 1");
    if (max_batch > kMaxMmBatch) return fail("max_batch must be <= 64");
    if (max_batch > 1 && moe) return fail("max_batch > 1 needs a dense model (MoE decode is batch 1)");
    if (max_ctx < 1 || max_ctx > (1 << 22)) return fail("max_ctx must be in 1..4194304");
    if (n_sm < 1) return fail("n_sm must be >= 1");
    if (tp < 1 || tp > kMaxTp) return fail("tensor-parallel size must be in 1..8");
    if (tp > 1 && (max_batch != 1 || moe)) return fail("tensor parallelism needs a dense model at batch 1");

    g = GraphPlan();
    g.desc = d;
    g.max_batch = max_batch;
    g.max_ctx = max_ctx;
    g.n_sm = n_sm;
    g.tp = tp;
    const int B = max_batch;
    const int hpg = nq / nkv;
    const int64_t qkv_rows = (int64_t)(nq + 2 * nkv) * hd;
    const int64_t target = 128 * 1024;

    // attention split-K: as many (sequence, kv head, split) tasks as fit in one wave
    // over the SMs (one more would make every layer's attention phase take two
    // task durations), but at most one split per 64 positions of context.
    // Batched graphs aim at about four tasks per SM instead (ragged context lengths
    // make the splits unequal; the dynamic queue evens them out), with splits of at
    // least ~512 positions of a half-full context (shorter ones cost more in fixed
    // per-task work than they gain in balance).
    // Long contexts at batch 1: one task per split covers every KV head (its pages'
    // blocks of all heads are contiguous: large copies), one wave of splits over the
    // SMs, and merge tasks per q head combine the splits.
    g.wide_attn = (B == 1) && tp == 1 && max_ctx >= kWideAttnCtx && kConsumerWarps % nkv == 0;   // warps per head
    int S = (B == 1) ? n_sm / (g.wide_attn ? 1 : nkv)
                     : (int)std::min<int64_t>(std::lround(4.0 * n_sm / (double)(B * nkv)), ceil_div(max_ctx, 1024));
    S = std::max(1, std::min<int>(S, (int)ceil_div(max_ctx, 64)));
    g.S = S;

    const int R_qkv = choose_tile_rows(qkv_rows, 2LL * H, 1, n_sm, target, hd);
    const int R_o = choose_tile_rows(H, 2LL * nq * hd, 1, n_sm, target, 0);
    const int R_lm = choose_tile_rows(d.vocab, 2LL * H, 1, n_sm, target, 0);
    int R_gu = 0, R_dn = 0, R_rt = 0, R_egu = 0, R_edn = 0;
    if (!moe) {
        R_gu = choose_tile_rows(d.ffn, 2LL * H, 2, n_sm, target, 0);
        R_dn = choose_tile_rows(H, 2LL * d.ffn, 1, n_sm, target, 0);
    } else {
        R_rt = choose_tile_rows(d.n_experts, 2LL * H, 1, n_sm, 64 * 1024, 0);
        // expert tiles: all top_k slots share the SMs
        R_egu = choose_tile_rows(d.expert_ffn, 2LL * H, 2, std::max(1, n_sm / d.top_k), target, 0);
        R_edn = choose_tile_rows(H, 2LL * d.expert_ffn, 1, std::max(1, n_sm / d.top_k), target, 0);
    }
    g.n_router_tiles = moe ? (int)ceil_div(d.n_experts, R_rt) : 0;
    g.tile_rows = {R_qkv, R_o, R_gu, R_dn, R_lm, R_rt, R_egu, R_edn};

    std::vector<Task>& T = g.tasks;
    std::vector<Entity> ent;                     // producer entities
    std::vector<int> task_entity;                // entity a task belongs to
    std::vector<std::vector<Region>> task_in;    // primary input regions per task
    std::vector<int> router_ent(L, -1);          // router-final entity per layer (MoE)

    auto new_task = [&](int op, int layer, int b, int aux, uint32_t r0, uint32_t r1) {
        Task t;
        std::memset(&t, 0, sizeof(t));
        t.op = (uint8_t)op;
        t.layer = (uint16_t)layer;
        t.b = (uint16_t)b;
        t.aux = (uint16_t)aux;
        t.r0 = r0;
        t.r1 = r1;
        t.wait0 = t.wait1 = MK_NO_EVENT;
        t.sig = MK_NO_EVENT;
        t.pad = MK_NO_EVENT;
        T.push_back(t);
        task_entity.push_back(-1);
        task_in.emplace_back();
        return (int)T.size() - 1;
    };
    auto own_entity = [&](int task, std::vector<Region> outs) {
        Entity e;
        e.tasks = {task};
        e.outs = std::move(outs);
        ent.push_back(std::move(e));
        task_entity[task] = (int)ent.size() - 1;
    };
    auto all_rows = [&](int kind, int layer, int slot, int64_t n) {
        return Region{tensor_key(kind, layer, slot), 0, B, 0, n};
    };
    auto gemv_op = [&](int op, int layer, int64_t rows, int R, int out_kind, int out_layer,
                       std::vector<Region> in) {
        for (int64_t r0 = 0; r0 < rows;) {
            int64_t r1 = std::min<int64_t>(rows, r0 + R);
            int t = new_task(op, layer, 0, 0, (uint32_t)r0, (uint32_t)r1);
            task_in[t] = in;
            own_entity(t, {Region{tensor_key(out_kind, out_layer, 0), 0, B, r0, r1}});
            r0 = r1;
        }
    };

    // QKV rows of one KV group: its q heads, then its k and v rows
    auto qkv_group = [&](int l, int kh) {
        const std::vector<Region> in = {all_rows(T_XIN, l, 0, H)};
        const int64_t spans[3][2] = {{(int64_t)kh * hpg * hd, (int64_t)(kh + 1) * hpg * hd},
                                     {(int64_t)nq * hd + kh * hd, (int64_t)nq * hd + (kh + 1) * hd},
                                     {(int64_t)(nq + nkv) * hd + kh * hd, (int64_t)(nq + nkv) * hd + (kh + 1) * hd}};
        for (const auto& sp : spans)
            for (int64_t r0 = sp[0]; r0 < sp[1];) {
                int64_t r1 = std::min<int64_t>(sp[1], r0 + R_qkv);
                int t = new_task(MK_OP_QKV, l, 0, 0, (uint32_t)r0, (uint32_t)r1);
                task_in[t] = in;
                own_entity(t, {Region{tensor_key(T_QKV, l, 0), 0, B, r0, r1}});
                r0 = r1;
            }
    };
    // wide attention of a layer: per split, every KV head; then per q head a merge task
    auto attn_wide = [&](int l) {
        const int64_t qkv_rows = (int64_t)(nq + 2 * nkv) * hd;
        for (int s = 0; s < S; ++s) {
            int t = new_task(MK_OP_ATTN, l, 0, 0, (uint32_t)s, (uint32_t)S);
            T[t].flags = kAttnWide;
            task_in[t] = {Region{tensor_key(T_QKV, l, 0), 0, B, 0, qkv_rows}};
            own_entity(t, {Region{tensor_key(T_PART, l, 0), 0, B, s, s + 1}});
        }
        for (int qh = 0; qh < nq; ++qh) {
            int t = new_task(MK_OP_ATTN_MERGE, l, 0, 0, (uint32_t)qh, (uint32_t)(qh + 1));
            task_in[t] = {Region{tensor_key(T_PART, l, 0), 0, B, 0, S}};
            own_entity(t, {Region{tensor_key(T_O, l, 0), 0, B, (int64_t)qh * hd, (int64_t)(qh + 1) * hd}});
        }
    };
    // attention of one KV group: per (sequence, split); each split writes its softmax
    // partial, and the O-projection's input stage merges the splits
    auto attn_group = [&](int l, int kh) {
        for (int b = 0; b < B; ++b)
            for (int s = 0; s < S; ++s) {
                int t = new_task(MK_OP_ATTN, l, b, kh, (uint32_t)s, (uint32_t)S);
                int key = tensor_key(T_QKV, l, 0);
                task_in[t] = {Region{key, 0, B, (int64_t)kh * hpg * hd, (int64_t)(kh + 1) * hpg * hd},
                              Region{key, 0, B, (int64_t)nq * hd + kh * hd, (int64_t)nq * hd + (kh + 1) * hd},
                              Region{key, 0, B, (int64_t)(nq + nkv) * hd + kh * hd,
                                     (int64_t)(nq + nkv) * hd + (kh + 1) * hd}};
                // batched graphs: the appended K/V of every row (whose tasks wait on all of
                // QKV) is the one input, so the event is theirs alone
                if (B > 1) task_in[t] = {Region{tensor_key(T_KV, l, 0), 0, B, 0, 1}};
                own_entity(t, {Region{tensor_key(T_O, l, 0), b, b + 1, (int64_t)kh * hpg * hd,
                                      (int64_t)(kh + 1) * hpg * hd}});
            }
    };

    // tensor parallelism: the projection tiles since task `first` wrote this rank's
    // partial sums of their rows (pushed to every rank); one reduce task per tile adds
    // the ranks' parts and the residual into the residual stream.  The tile's ordinal
    // (pad) names its arrival flag; the reduce task waits on that flag, not on an event.
    auto tp_reduce = [&](int l, int phase, int first, int out_kind, int out_layer) {
        const int last = (int)T.size();
        int ord = 0;
        for (int i = first; i < last; ++i, ++ord) {
            T[i].pad = (uint32_t)ord;
            int t = new_task(MK_OP_TP_REDUCE, l, 0, phase, T[i].r0, T[i].r1);
            T[t].pad = (uint32_t)ord;
            own_entity(t, {Region{tensor_key(out_kind, out_layer, 0), 0, B, (int64_t)T[i].r0, (int64_t)T[i].r1}});
        }
        g.tp_tiles = std::max(g.tp_tiles, ord);
    };

    if (B > 1) {
        // ---- batched step: tensor-core tiles of 128 weight rows x all batch rows.
        // A tile's K range is cut into splits so that (tiles x splits) fills the SMs;
        // every split of a tile belongs to one producer entity, and the last split to
        // arrive reduces the partial sums and signals.
        g.bp = (B <= 16) ? 16 : (B <= 32) ? 32 : 64;
        auto choose_splits = [&](int64_t tiles, int64_t kblocks) {
            int best = 1;
            double best_eff = 0.0;
            const int cap = (int)std::max<int64_t>(1, std::min<int64_t>(16, kblocks / 2));
            for (int sp = 1; sp <= cap; ++sp) {
                const int64_t n = tiles * sp, w = ceil_div(n, n_sm);
                const double eff = (double)n / (double)(w * n_sm);
                if (eff >= 0.9) return sp;
                if (eff > best_eff + 1e-9) { best_eff = eff; best = sp; }
            }
            return best;
        };
        int slot = 0;   // partial-sum slots, numbered per layer (layers reuse them in turn)
        // one operator: blocks of (rows, weight map(s)); tiles of `tile_rows` output rows
        struct WBlock { int64_t out0, n; int map0, map1; };
        auto mm_op = [&](int op, int l, const std::vector<WBlock>& blocks, int tile_rows, int64_t K,
                         std::vector<Region> in, int out_kind, int out_layer) {
            int64_t tiles = 0;
            for (const WBlock& wb : blocks) tiles += ceil_div(wb.n, tile_rows);
            const int64_t kblocks = ceil_div(K, kMmK);
            const int Sk = choose_splits(tiles, kblocks);
            for (const WBlock& wb : blocks)
                for (int64_t y = 0; y < wb.n; y += tile_rows) {
                    const int64_t r0 = wb.out0 + y, r1 = wb.out0 + std::min<int64_t>(wb.n, y + tile_rows);
                    Entity e;
                    e.outs = {Region{tensor_key(out_kind, out_layer, 0), 0, B, r0, r1}};
                    const int eid = (int)ent.size();
                    ent.push_back(e);
                    const int counter = g.mm_counters++;
                    for (int sp = 0; sp < Sk; ++sp) {
                        const int64_t kb0 = kblocks * sp / Sk, kb1 = kblocks * (sp + 1) / Sk;
                        int t = new_task(op, l, 0, slot, (uint32_t)r0, (uint32_t)r1);
                        Task& tk = T[t];
                        tk.src[0] = (uint64_t)(uint32_t)wb.map0 | ((uint64_t)y << 32);
                        tk.src[1] = (wb.map1 >= 0) ? ((uint64_t)(uint32_t)wb.map1 | ((uint64_t)y << 32)) : 0;
                        tk.row_bytes = (uint32_t)kb0;
                        tk.pad2 = (uint32_t)kb1;
                        tk.chunk_rows = (uint16_t)sp;
                        tk.nblk = (uint16_t)Sk;
                        // a stage per weight box, plus one per group of kx activation boxes
                        const int64_t kx = std::max(1, kStageBytes / (2 * g.bp * 128));
                        tk.nchunks = (uint32_t)((kb1 - kb0) + ceil_div(kb1 - kb0, kx));
                        tk.pad = (uint32_t)counter;
                        task_in[t] = in;
                        task_entity[t] = eid;
                        ent[eid].tasks.push_back(t);
                    }
                    slot += Sk;
                }
        };
        // rmsnorm of the batch rows into an operand, kNormRowsPerTask rows per task
        auto norm_op = [&](int l, int kind, int in_kind, int in_layer, int out_kind) {
            for (int b0 = 0; b0 < B; b0 += kNormRowsPerTask) {
                const int b1 = std::min(B, b0 + kNormRowsPerTask);
                int t = new_task(MK_OP_NORM, l, 0, kind, (uint32_t)b0, (uint32_t)b1);
                task_in[t] = {Region{tensor_key(in_kind, in_layer, 0), b0, b1, 0, H}};
                own_entity(t, {Region{tensor_key(out_kind, l, 0), b0, b1, 0, H}});
            }
        };
        const int64_t qr = (int64_t)nq * hd, kr = (int64_t)nkv * hd;
        for (int l = 0; l < L; ++l) {
            slot = 0;
            norm_op(l, 0, T_XIN, l, T_XQOP);
            mm_op(MK_OP_MM_QKV, l,
                  {{0, qr, weight_map_index(l, 0), -1}, {qr, kr, weight_map_index(l, 1), -1},
                   {qr + kr, kr, weight_map_index(l, 2), -1}},
                  kMmRows, H, {all_rows(T_XQOP, l, 0, H)}, T_QKV, l);
            // each sequence's new K/V into its pages; every attention task of the layer
            // waits for all of them (under batched prefill, the rows are one sequence)
            for (int b = 0; b < B; ++b) {
                int t = new_task(MK_OP_KVAPPEND, l, 0, 0, (uint32_t)b, (uint32_t)(b + 1));
                task_in[t] = {all_rows(T_QKV, l, 0, qr + 2 * kr)};
                own_entity(t, {Region{tensor_key(T_KV, l, 0), b, b + 1, 0, 1}});
            }
            for (int kh = 0; kh < nkv; ++kh) attn_group(l, kh);
            mm_op(MK_OP_MM_OPROJ, l, {{0, H, weight_map_index(l, 3), -1}}, kMmRows, qr,
                  {all_rows(T_O, l, 0, qr)}, T_XMID, l);
            norm_op(l, 1, T_XMID, l, T_XFOP);
            mm_op(MK_OP_MM_GATEUP, l, {{0, d.ffn, weight_map_index(l, 4), weight_map_index(l, 5)}},
                  kMmRows / 2, H, {all_rows(T_XFOP, l, 0, H)}, T_ACT, l);
            mm_op(MK_OP_MM_DOWN, l, {{0, H, weight_map_index(l, 6), -1}}, kMmRows, d.ffn,
                  {all_rows(T_ACT, l, 0, d.ffn)}, T_XIN, l + 1);
            g.mm_slots = std::max(g.mm_slots, slot);
        }
        slot = 0;
        norm_op(L, 2, T_XIN, L, T_XLOP);
        mm_op(MK_OP_MM_LMHEAD, L, {{0, d.vocab, lm_map_index(L), -1}}, kMmRows, H,
              {all_rows(T_XLOP, L, 0, H)}, T_LOGITS, 0);
        g.mm_slots = std::max(g.mm_slots, slot);
        if (g.mm_slots > 65535) return fail("too many tensor-core tiles per layer");
    }
    for (int l = 0; l < L && B == 1; ++l) {
        // QKV (input: the residual stream entering the layer), one KV group at a time,
        // so that the first groups' attention can start while the last QKV tiles
        // stream.  Attention follows all QKV tiles: a CTA that claimed a task still
        // waiting on its inputs streams nothing meanwhile.
        for (int kh = 0; kh < nkv; ++kh) qkv_group(l, kh);
        if (g.wide_attn) attn_wide(l);
        else
            for (int kh = 0; kh < nkv; ++kh) attn_group(l, kh);
        if (tp > 1) {
            int first = (int)T.size();
            gemv_op(MK_OP_OPROJ, l, H, R_o, T_TPP, l, {all_rows(T_O, l, 0, (int64_t)nq * hd)});
            tp_reduce(l, 0, first, T_XMID, l);
            gemv_op(MK_OP_GATEUP, l, d.ffn, R_gu, T_ACT, l, {all_rows(T_XMID, l, 0, H)});
            first = (int)T.size();
            gemv_op(MK_OP_DOWN, l, H, R_dn, T_TPP, l, {all_rows(T_ACT, l, 0, d.ffn)});
            tp_reduce(l, 1, first, T_XIN, l + 1);
            continue;
        }
        gemv_op(MK_OP_OPROJ, l, H, R_o, T_XMID, l, {all_rows(T_O, l, 0, (int64_t)nq * hd)});
        if (!moe) {
            gemv_op(MK_OP_GATEUP, l, d.ffn, R_gu, T_ACT, l, {all_rows(T_XMID, l, 0, H)});
            gemv_op(MK_OP_DOWN, l, H, R_dn, T_XIN, l + 1, {all_rows(T_ACT, l, 0, d.ffn)});
        } else {
            Entity rf;
            rf.outs = {all_rows(T_SEL, l, 0, d.top_k)};
            int rid = (int)ent.size();
            ent.push_back(rf);
            router_ent[l] = rid;
            for (int r0 = 0; r0 < d.n_experts; r0 += R_rt) {
                int t = new_task(MK_OP_ROUTER, l, 0, 0, (uint32_t)r0,
                                 (uint32_t)std::min(d.n_experts, r0 + R_rt));
                task_in[t] = {all_rows(T_XMID, l, 0, H)};
                task_entity[t] = rid;
                ent[rid].tasks.push_back(t);
            }
            for (int b = 0; b < B; ++b)
                for (int k = 0; k < d.top_k; ++k)
                    for (int r0 = 0; r0 < d.expert_ffn; r0 += R_egu) {
                        int r1 = std::min(d.expert_ffn, r0 + R_egu);
                        int t = new_task(MK_OP_EXP_GATEUP, l, b, k, (uint32_t)r0, (uint32_t)r1);
                        task_in[t] = {all_rows(T_SEL, l, 0, d.top_k)};
                        own_entity(t, {Region{tensor_key(T_ACTE, l, k), b, b + 1, r0, r1}});
                    }
            for (int b = 0; b < B; ++b)
                for (int k = 0; k < d.top_k; ++k)
                    for (int r0 = 0; r0 < H; r0 += R_edn) {
                        int r1 = std::min(H, r0 + R_edn);
                        int t = new_task(MK_OP_EXP_DOWN, l, b, k, (uint32_t)r0, (uint32_t)r1);
                        task_in[t] = {Region{tensor_key(T_ACTE, l, k), b, b + 1, 0, d.expert_ffn}};
                        own_entity(t, {Region{tensor_key(T_XIN, l + 1, 0), b, b + 1, r0, r1}});
                    }
        }
    }
    if (B == 1) gemv_op(MK_OP_LMHEAD, L, d.vocab, R_lm, T_LOGITS, 0, {all_rows(T_XIN, L, 0, H)});

    // ---- dependency analysis: producers overlapping each task's primary input
    std::map<int, std::vector<int>> by_tensor;   // tensor -> entities writing it
    for (int e = 0; e < (int)ent.size(); ++e)
        for (const Region& r : ent[e].outs) by_tensor[r.tensor].push_back(e);
    UnionFind uf;
    for (size_t e = 0; e < ent.size(); ++e) uf.add();
    std::vector<int> first_dep(T.size(), -1);
    for (size_t t = 0; t < T.size(); ++t) {
        int first = -1;
        for (const Region& in : task_in[t]) {
            auto it = by_tensor.find(in.tensor);
            if (it == by_tensor.end()) continue;       // e.g. the embedding: no producer task
            for (int e : it->second)
                for (const Region& o : ent[e].outs)
                    if (overlaps(in, o)) {
                        if (first < 0) first = e;
                        else uf.unite(first, e);
                    }
        }
        first_dep[t] = first;
    }
    // events = connected components of producer entities that some task waits on
    std::map<int, int> comp_event;
    std::vector<uint32_t>& thr = g.thr;
    auto event_of = [&](int e) -> int {
        int c = uf.find(e);
        auto it = comp_event.find(c);
        if (it != comp_event.end()) return it->second;
        int id = (int)thr.size();
        comp_event[c] = id;
        thr.push_back(0);
        return id;
    };
    for (size_t t = 0; t < T.size(); ++t)
        if (first_dep[t] >= 0) T[t].wait0 = (uint32_t)event_of(first_dep[t]);
    // producers signal their component's event; thresholds count entities
    for (int e = 0; e < (int)ent.size(); ++e) {
        int c = uf.find(e);
        auto it = comp_event.find(c);
        if (it == comp_event.end()) continue;          // nobody waits on it (e.g. LM head)
        thr[it->second] += 1;
        for (int t : ent[e].tasks) T[t].sig = (uint32_t)it->second;
    }
    // expert tasks: the producer warp waits on the router event before it reads the expert id
    for (size_t t = 0; t < T.size(); ++t)
        if (T[t].op == MK_OP_EXP_GATEUP || T[t].op == MK_OP_EXP_DOWN) {
            int c = uf.find(router_ent[T[t].layer]);
            T[t].pad = (uint32_t)comp_event.at(c);
        }
    // ---- checks: every wait is satisfied only by tasks earlier in the list
    std::vector<int> last_signaler(thr.size(), -1);
    for (int t = 0; t < (int)T.size(); ++t)
        if (T[t].sig != MK_NO_EVENT) last_signaler[T[t].sig] = t;
    for (int t = 0; t < (int)T.size(); ++t) {
        uint32_t w = T[t].wait0;
        if (w != MK_NO_EVENT && last_signaler[w] >= t) {
            const Task& a = T[t];
            const Task& z = T[last_signaler[w]];
            return fail("internal: task list is not topologically ordered (task " + std::to_string(t) + " op " +
                        std::to_string(a.op) + " layer " + std::to_string(a.layer) + " waits on event " +
                        std::to_string(w) + ", signalled by task " + std::to_string(last_signaler[w]) +
                        " op " + std::to_string(z.op) + " layer " + std::to_string(z.layer) + ")");
        }
    }
    g.n_events = (int)thr.size();
    // LM-head tiles are numbered for the in-step argmax's partial results: a GEMV
    // tile in aux, every split of a tensor-core tile in b
    {
        int n = 0;
        for (Task& t : T) {
            if (t.op == MK_OP_LMHEAD) t.aux = (uint16_t)n++;
        }
        // batched LM-head tiles: every split of a tile carries the tile's ordinal in b
        int nt = 0;
        uint32_t last_r0 = 0xFFFFFFFFu;
        for (Task& t : T) {
            if (t.op != MK_OP_MM_LMHEAD) continue;
            if (t.r0 != last_r0) { last_r0 = t.r0; ++nt; }
            t.b = (uint16_t)(nt - 1);
        }
        g.n_lm_tiles = std::max(n, nt);
        if (g.n_lm_tiles > 65535) return fail("too many LM-head tiles");
    }

    // ---- GEMV fast-path variant per task (the device dispatches on it without any
    //      geometry arithmetic)
    for (Task& t : T) {
        int K = 0, nblk = 1;
        switch (t.op) {
            case MK_OP_QKV: case MK_OP_LMHEAD: case MK_OP_ROUTER: K = H; break;
            case MK_OP_GATEUP: case MK_OP_EXP_GATEUP: K = H; nblk = 2; break;
            case MK_OP_OPROJ: K = nq * hd; break;
            case MK_OP_DOWN: K = d.ffn; break;
            case MK_OP_EXP_DOWN: K = d.expert_ffn; break;
            default: break;
        }
        if (K) t.flags = fast_path_for(K, (int)(t.r1 - t.r0), nblk);   // (attention keeps its own flags)
    }

    // ---- bytes streamed per B=1 step
    int64_t wb = 2LL * H;                               // one embedding row
    for (int l = 0; l < L; ++l) {
        wb += 2LL * H * 2;                              // norm gains
        wb += 2LL * qkv_rows * H + 2LL * H * nq * hd;
        if (!moe) wb += 2LL * 3 * d.ffn * H;
        else wb += 2LL * d.n_experts * H + 2LL * 3 * d.top_k * d.expert_ffn * H;
    }
    wb += 2LL * H + 2LL * d.vocab * H;
    g.weight_bytes = wb;
    return true;
}

bool tp_shard_desc(const mk_model_desc& full, int tp, int rank, mk_model_desc& out, std::string& err) {
    auto fail = [&](const std::string& m) { err = m; return false; };
    if (!validate_desc(full, err)) return false;
    if (tp < 2 || tp > kMaxTp) return fail("tensor-parallel size must be in 2..8");
    if (rank < 0 || rank >= tp) return fail("tensor-parallel rank outside 0..tp-1");
    if (full.n_experts > 0) return fail("tensor parallelism covers dense models");
    if (full.n_kv_heads % tp) return fail("KV heads must divide evenly over the ranks");
    if (full.ffn % tp || (full.ffn / tp) % 8) return fail("FFN rows per rank must be a multiple of 8");
    if (full.vocab % tp) return fail("vocabulary rows must divide evenly over the ranks");
    out = full;
    out.n_q_heads = full.n_q_heads / tp;
    out.n_kv_heads = full.n_kv_heads / tp;
    out.ffn = full.ffn / tp;
    out.vocab = full.vocab / tp;
    return validate_desc(out, err);
}

void attach_weights(GraphPlan& g, const void* const* w) {
    const mk_model_desc& d = g.desc;
    const bool moe = d.n_experts > 0;
    const int S = moe ? 10 : 9, L = d.n_layers, H = d.hidden, hd = d.head_dim;
    const int qr = d.n_q_heads * hd, kr = d.n_kv_heads * hd;
    auto ptr = [&](int layer, int slot) { return reinterpret_cast<uint64_t>(w[1 + layer * S + slot]); };
    for (Task& t : g.tasks) {
        int K = 0, nblk = 1;
        uint64_t a = 0, b = 0;
        const int l = t.layer;
        switch (t.op) {
            case MK_OP_QKV: {
                K = H;
                const int r = (int)t.r0;
                if (r < qr) a = ptr(l, 1) + 2ull * r * H;
                else if (r < qr + kr) a = ptr(l, 2) + 2ull * (r - qr) * H;
                else a = ptr(l, 3) + 2ull * (r - qr - kr) * H;
                break;
            }
            case MK_OP_OPROJ: K = qr; a = ptr(l, 4) + 2ull * t.r0 * K; break;
            case MK_OP_GATEUP:
                K = H; nblk = 2; a = ptr(l, 6) + 2ull * t.r0 * H; b = ptr(l, 7) + 2ull * t.r0 * H; break;
            case MK_OP_DOWN: K = d.ffn; a = ptr(l, 8) + 2ull * t.r0 * K; break;
            case MK_OP_ROUTER: K = H; a = ptr(l, 6) + 2ull * t.r0 * H; break;
            case MK_OP_LMHEAD:
                K = H; a = reinterpret_cast<uint64_t>(w[2 + L * S]) + 2ull * t.r0 * H; break;
            default: continue;   // attention pages and routed experts are resolved on the device
        }
        const uint32_t rows = t.r1 - t.r0, rb = 2u * (uint32_t)K;
        t.src[0] = a;
        t.src[1] = b;
        t.row_bytes = rb;
        t.nblk = (uint16_t)nblk;
        if (rb <= (uint32_t)kStageBytes) {
            t.chunk_rows = (uint16_t)(is_warp_row(t.flags) ? kWarpRows : kStageBytes / rb);
            t.nchunks = (uint32_t)nblk * ((rows + t.chunk_rows - 1) / t.chunk_rows);
        } else {
            t.chunk_rows = 0;
            t.nchunks = (uint32_t)nblk * rows * ((rb + kStageBytes - 1) / kStageBytes);
        }
    }
}

void make_solo(GraphPlan& g, int op) {
    std::vector<Task> kept;
    for (const Task& t : g.tasks)
        if (t.op == op) {
            Task u = t;
            u.wait0 = u.wait1 = MK_NO_EVENT;
            u.sig = MK_NO_EVENT;
            u.pad = MK_NO_EVENT;
            kept.push_back(u);
        }
    g.tasks.swap(kept);
    g.thr.clear();
    g.n_events = 0;
}

}  // namespace mk
