// The persistent decode megakernel for sm_100a.
//
// One CTA per SM stays resident for the whole decode step and pulls tasks from
// the host-built list through one global atomic work-queue head (Cohere page
// "Cohere megakerneles kiszolgálót mutatott be a North Mini Code modellhez",
// section "Egyetlen tartós kernelre épül a kiszolgálás").  A task waits on an
// event counter in global memory until it reaches threshold * epoch, computes
// one tile, and increments its own event (MPK digest "LLM को MegaKernel में
// compile करके low-latency inference हासिल करना", section "Part 2. Runtime":
// worker loop fetch -> execute -> notify; event fires at its threshold).
//
// Warp roles inside a CTA:
//   warps 0-7  consumers: dependency wait, input stage (embedding, RMSNorm,
//              split merge), attention, dot products out of shared memory and
//              warp reductions; each warp leaves its partial row sums in a
//              rotating buffer and moves straight on to the next task
//   warp 8     producer: dequeues the next tasks and streams their weight rows
//              and KV pages into an 11-stage shared-memory ring with bulk
//              asynchronous copies (cp.async.bulk, mbarrier completion).
//              Weights never depend on activations, so the producer runs ahead
//              of the consumers across task and layer boundaries: the next
//              layer's weights are in flight while this layer's tail finishes
//              (Cohere page, "Honnan jön a gyorsulás?": weight tiles are
//              prefetched before the activation dependency is met).
//   warp 9     epilogue: reduces the consumers' partials in a fixed order,
//              applies each operator's tail (residual add, SiLU gate, expert
//              selection), stores, and publishes the completion (fence +
//              release add), so no consumer stalls on a task's tail or on the
//              gpu-scope fence.
//
// Deadlock freedom: tasks are dequeued in list order, the list is topological
// and each CTA runs its tasks in dequeue order, so the lowest unfinished task
// always has its producers finished and its CTA free to run it.
// Every wait (event counter, ring slot, buffer set) gives up after
// Params::timeout_ns, records MK_ERR_TIMEOUT and the kernel drains its own
// copies in flight and returns.
#include <cuda_runtime.h>
#include <limits.h>
#include <stddef.h>
#include <stdint.h>

#include "megakernel.h"
#include "mk_internal.h"

namespace mk {

// ----------------------------------------------------------------------------- PTX helpers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// Non-blocking test of an mbarrier phase.
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ void mbar_arrive_cnt(uint64_t* bar, uint32_t n) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(n) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t tx) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(tx)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
// Bulk async copy global -> this CTA's shared memory; completion counted on `bar`.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                         uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}
// Tiled TMA load of one 2-D box (tensor map in global memory) into shared memory;
// x is the inner (column) coordinate, a multiple of 64 bf16 elements here.
__device__ __forceinline__ void tma_load_2d(void* dst, const void* tmap, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(tmap), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void tma_load_2d_hint(void* dst, const void* tmap, int x, int y, uint64_t* bar,
                                                 uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
        "l"(tmap), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// ---- tcgen05: tensor memory and the fifth-generation MMA (one CTA, no cluster)
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {      // whole warp
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {                               // whole warp
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {    // whole warp
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// Arrives (once) on `bar` when every tcgen05 operation this thread issued so far has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}
// D[tmem] (+)= A[smem] . B[smem]^T, bf16 inputs, fp32 accumulator; accumulate = 0 overwrites D.
__device__ __forceinline__ void tc_mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// 32 TMEM lanes (one per thread of the warp) x 16 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// Shared-memory matrix descriptor: K-major operand in the 128-byte swizzle layout
// that a TMA box of 128-byte rows writes (8-row atoms of 1 KB; the leading
// offset is unused in this layout, the stride offset steps from one 8-row atom
// to the next).  Fields: start address >> 4, leading offset >> 4 at bit 16,
// stride offset >> 4 at bit 32, descriptor version 1 at bit 46, swizzle mode 2
// (128 B) at bit 61.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// Instruction descriptor of kind::f16: fp32 accumulator (bit 4), bf16 A (bit 7)
// and B (bit 10), both K-major, N >> 3 at bit 17, M >> 4 at bit 24.
__host__ __device__ constexpr uint32_t mm_idesc(int n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kMmRows >> 4) << 24);
}

// Hint: bring [src, src+bytes) into L2 (16-byte aligned, multiple of 16 bytes).
__device__ __forceinline__ void prefetch_l2(const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ int ld_relaxed_int(const int* p) {
    int v;
    asm volatile("ld.relaxed.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void red_release_add(uint32_t* p, uint32_t v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// Tensor-parallel arrival flags live in the receiving rank's memory and are raised
// by every rank's GPU: system scope on both sides.
__device__ __forceinline__ void red_release_add_sys(uint32_t* p, uint32_t v) {
    asm volatile("red.release.sys.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t ld_acquire_sys(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
// Arrival count with acquire-release semantics at GPU scope: publishes every write
// that precedes it in causality order (cumulative release) and makes the other
// arrivals' writes visible to what follows (acquire).  Returns the old value.
__device__ __forceinline__ uint32_t atom_add_acq_rel(uint32_t* p, uint32_t v) {
    uint32_t old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}


// (value, index) of a running maximum: a larger value wins, equal values go to the
// lower index (the greedy rule: ties to the lowest token id).
__device__ __forceinline__ void arg_better(float& v, int& i, float v2, int i2) {
    if (v2 > v || (v2 == v && i2 < i)) { v = v2; i = i2; }
}
__device__ __forceinline__ void warp_argmax(float& v, int& i) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float v2 = __shfl_xor_sync(0xFFFFFFFFu, v, o);
        const int i2 = __shfl_xor_sync(0xFFFFFFFFu, i, o);
        arg_better(v, i, v2, i2);
    }
}

__device__ __forceinline__ float bf_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }
__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }
// fp32 -> bf16 round-to-nearest-even (finite values)
__device__ __forceinline__ uint16_t f32_to_bf16_rne(float f) {
    uint32_t u = __float_as_uint(f);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
}
__device__ __forceinline__ float silu_f(float z) { return z / (1.0f + expf(-z)); }

__device__ __forceinline__ void set_error(const Params& p, int code, int a, int b, int c, int d) {
    if (atomicCAS(p.err, 0, code) == 0) {
        p.err[1] = a;
        p.err[2] = b;
        p.err[3] = c;
        p.err[4] = d;
    }
}

// ----------------------------------------------------------------------------- shared memory

struct StageInfo {
    int task;      // task index, -1 = end of work
    int chunk;     // chunk index within the task
    int nchunks;   // chunks of the task (0 for a task without streamed data)
    int aux;       // attention: first logical page of this chunk
    Task rec;      // the task record (read once, by the producer)
};

constexpr int kAttnScratch = kConsumerWarps * kMaxHeadsPerGroup * (128 + 2);   // >= n_q * head_dim floats too
// Rotating buffer sets (row sums, task record, residual rows) between the consumer
// warps and the epilogue warp: consumers may run kRedBufs - 1 tasks ahead of it.
constexpr int kRedBufs = 4;
// Page ids the producer reads ahead for an attention split: batches of 8, loaded
// when fewer than 8 ids beyond the current stage remain; the ring keeps up to 15
// ids ahead plus the current stage's (<= 4), so 32 entries never overwrite an id
// still in use.
constexpr int kPidBatch = 8;
constexpr int kPidRing = 4 * kPidBatch;

struct __align__(128) Smem {
    uint8_t ring[kStages][kStageBytes];
    float red[kRedBufs][kMaxTaskRows][kConsumerWarps];   // per-warp row sums, rotating per task
    union {
        float attn[kAttnScratch];             // per-warp (m, l, o) partials; O-proj merge scratch
        float rlog[1024];                     // router logits of one sequence
    };
    float qs[kMaxHeadsPerGroup * 128];        // rotated, pre-scaled q of one kv group
    float kn[128], vn[128];                   // the new token's k, v (bf16-rounded)
    float bcast[kConsumerWarps + 8];
    uint64_t full[kStages], empty[kStages];
    uint64_t csync;                          // all-consumer-warp sync (arrival count 8)
    uint64_t red_full[kRedBufs];             // 8 consumer-warp arrivals: the task's partials are in red[buf]
    uint64_t red_free[kRedBufs];             // the epilogue warp has finished with buffer set buf
    StageInfo info[kStages];
    Task ep_task[kRedBufs];                  // task record for the epilogue warp
    int ep_ti[kRedBufs];                     // its index (-1: end of work)
    float ep_resid[kRedBufs][kMaxTaskRows];  // residual rows (O-proj, down), loaded early by warp 0
    int attn_last;                           // this CTA's attention split arrived last
    uint64_t mm_acc[2];                      // tensor-core tiles: accumulator buffer a is complete
    uint64_t mm_free[2];                     // ... and has been read (4 arrivals: warps 4-7)
    uint64_t mm_drain;                       // tensor-core work drained before TMEM is freed
    uint64_t mm_sync;                        // consumer warps 4-7 (arrival count 4)
    uint32_t tmem_base;                      // TMEM address of the accumulator (batched graphs)
    int mm_last;                             // this CTA's split of a tile arrived last
    int pid[kPidRing];                       // producer: physical page ids read ahead
    int pf_claimed;                          // producer's latest claimed task (-1: finished), for the prefetcher
    int pf_wait;                             // 1 while consumer warp 0 waits on a dependency (the prefetcher runs)
    int started;                             // latest task the consumers have started (past its event wait)
    int attn_hold;                           // this step's attention splits hold the next claim (-1: not yet known)
    int flag[4];
};

// ----------------------------------------------------------------------------- geometry

__device__ __forceinline__ int hpg_of(const Params& p) { return p.nq / p.nkv; }

// Token position of batch row b this step (validated by the caller).
__device__ __forceinline__ int position_of(const Params& p, int b) {
    return (p.positions ? p.positions[b] : 0) + p.pos_offset + b * p.pos_stride;
}
// Page-table row of batch row b: its own, or (batched prefill) the one sequence's.
__device__ __forceinline__ const int* page_row(const Params& p, int b) {
    return p.page_table + (size_t)(p.seq_row >= 0 ? p.seq_row : b) * p.max_pages;
}

struct GemvGeom {
    int K;            // columns
    int rows;         // rows per weight block
    int nblk;         // 1 or 2 weight blocks (gate/up)
    const uint16_t* w[2];
};

// Weight blocks of a GEMV task.  Expert ops read the routed expert id (producer
// side only; the consumer needs just K and rows).
__device__ __forceinline__ void gemv_geom(const Params& p, const Task& t, GemvGeom& g, bool want_ptr) {
    const int H = p.H;
    g.rows = (int)(t.r1 - t.r0);
    g.nblk = 1;
    g.w[0] = g.w[1] = nullptr;
    const LayerW* lw = (t.op == MK_OP_LMHEAD) ? nullptr : &p.layers[t.layer];
    switch (t.op) {
        case MK_OP_QKV: {
            g.K = H;
            if (want_ptr) {
                int qr = p.nq * p.hd, kr = p.nkv * p.hd;
                int r = (int)t.r0;
                const uint16_t* base;
                if (r < qr) base = lw->wq + (size_t)r * H;
                else if (r < qr + kr) base = lw->wk + (size_t)(r - qr) * H;
                else base = lw->wv + (size_t)(r - qr - kr) * H;
                g.w[0] = base;
            }
            break;
        }
        case MK_OP_OPROJ:
            g.K = p.nq * p.hd;
            if (want_ptr) g.w[0] = lw->wo + (size_t)t.r0 * g.K;
            break;
        case MK_OP_GATEUP:
            g.K = H;
            g.nblk = 2;
            if (want_ptr) {
                g.w[0] = lw->w_gate + (size_t)t.r0 * H;
                g.w[1] = lw->w_up + (size_t)t.r0 * H;
            }
            break;
        case MK_OP_DOWN:
            g.K = p.F;
            if (want_ptr) g.w[0] = lw->w_down + (size_t)t.r0 * p.F;
            break;
        case MK_OP_LMHEAD:
            g.K = H;
            if (want_ptr) g.w[0] = p.lm_head + (size_t)t.r0 * H;
            break;
        case MK_OP_ROUTER:
            g.K = H;
            if (want_ptr) g.w[0] = lw->w_router + (size_t)t.r0 * H;
            break;
        case MK_OP_EXP_GATEUP: {
            g.K = H;
            g.nblk = 2;
            if (want_ptr) {
                int e = __ldcg(p.moe_sel + ((size_t)t.layer * p.max_batch + t.b) * p.topk + t.aux);
                if (e < 0 || e >= p.E) { set_error(p, kErrFault, -1, -7, e, t.layer); e = 0; }
                size_t off = ((size_t)e * p.Fe + t.r0) * H;
                g.w[0] = lw->w_gate + off;
                g.w[1] = lw->w_up + off;
            }
            break;
        }
        case MK_OP_EXP_DOWN: {
            g.K = p.Fe;
            if (want_ptr) {
                int e = __ldcg(p.moe_sel + ((size_t)t.layer * p.max_batch + t.b) * p.topk + t.aux);
                if (e < 0 || e >= p.E) { set_error(p, kErrFault, -1, -7, e, t.layer); e = 0; }
                g.w[0] = lw->w_down + ((size_t)e * H + t.r0) * p.Fe;
            }
            break;
        }
        default:
            g.K = 8;
            g.rows = 0;
            break;
    }
}

__device__ __forceinline__ bool is_gemv(int op) { return op != MK_OP_ATTN && op <= MK_OP_EXP_DOWN; }

// Chunks of a GEMV task: per weight block, groups of whole rows that fit one
// stage, or (rows longer than a stage) each row in stage-sized segments.
__device__ __forceinline__ int gemv_chunks(const GemvGeom& g, uint8_t flags) {
    const int64_t RB = (int64_t)g.K * 2;
    int per_blk;
    if (RB <= kStageBytes) {
        const int rps = is_warp_row(flags) ? kWarpRows : (int)(kStageBytes / RB);
        per_blk = (g.rows + rps - 1) / rps;
    } else {
        per_blk = g.rows * (int)((RB + kStageBytes - 1) / kStageBytes);
    }
    return per_blk * g.nblk;
}

// Splits of one (sequence, kv head) actually used this step, at most the graph's
// split count S (one wave of tasks over the SMs):
//  - up to kAttnLongCtx positions, one split per kAttnShortSplit positions: a
//    context of up to 512 is one split that writes the normalised output itself,
//    with no merge step (8B, position 300: 3.54 ms per step against 3.73 ms with
//    64-position splits and their merge);
//  - longer contexts, one split per kAttnSplitTokens positions, so that every SM
//    gets a split (30B MoE at 8192 tokens: 5.59 -> 5.42 ms per step against
//    512-position splits).
constexpr int kAttnShortSplit = 512;
constexpr int kAttnLongCtx = 2048;
constexpr int kAttnSplitTokens = 64;
__device__ __forceinline__ int attn_active_splits(int n_ctx, int S) {
    const int per = n_ctx < kAttnLongCtx ? kAttnShortSplit : kAttnSplitTokens;
    const int a = (n_ctx + per - 1) / per;
    return a < 1 ? 1 : (a > S ? S : a);
}

// Attention split range [j0, j1) of positions (inclusive of the new token).
__device__ __forceinline__ void attn_range(int n_ctx, int S, int s, int& j0, int& j1) {
    int per = (n_ctx + S - 1) / S;
    per = (per + kPageSize - 1) / kPageSize * kPageSize;
    j0 = s * per;
    j1 = min(n_ctx, j0 + per);
    if (j0 > n_ctx) j0 = n_ctx;
}

__device__ __forceinline__ int pages_per_stage(const Params& p) {
    return kStageBytes / (2 * kPageSize * p.hd * 2);
}

// ----------------------------------------------------------------------------- waits

struct Waiter {
    uint64_t t0;
    int spins;
};

// true when the deadline has passed or another CTA has recorded an error
// (polled every 256 spins: each poll is an L2 round trip)
__device__ __forceinline__ bool wait_should_stop(const Params& p, Waiter& w) {
    if (++w.spins & 255) return false;
    if (ld_relaxed_int(p.err) != 0) return true;
    if (w.t0 == 0) w.t0 = globaltimer();
    else if ((long long)(globaltimer() - w.t0) > p.timeout_ns) return true;
    return false;
}

// Per-CTA cycle counters (tracing builds of the state only): [0] producer waits for a
// free ring slot, [1] consumer thread 0 waits for data, [2] dependency waits,
// [3] kernel cycles, [4] tasks run, [5] signal-slot waits.
__device__ __forceinline__ void stat_add(const Params& p, int i, unsigned long long v) {
    if (p.stats) atomicAdd(&p.stats[(size_t)(blockIdx.x - p.cta0) * 8 + i], v);   // reduction, no return value
}

__device__ __forceinline__ void wait_stat(const Params& p, int where, long long c0) {
    if (!p.stats) return;
    const unsigned long long d = (unsigned long long)(clock64() - c0);
    if (where == 1) stat_add(p, 0, d);                                   // producer: ring full
    else if ((where == 3 || where == 4 || where == 5) && threadIdx.x == 0) stat_add(p, 1, d);
}

__device__ bool mbar_wait_slow(const Params& p, uint64_t* bar, uint32_t parity, int where) {
    Waiter w{0, 0};
    const long long c0 = p.stats ? clock64() : 0;
    while (!mbar_try_wait(bar, parity)) {
        if (wait_should_stop(p, w)) {
            if (ld_relaxed_int(p.err) == 0) set_error(p, kErrTimeout, -1, -1, where, (int)(blockIdx.x - p.cta0));
            wait_stat(p, where, c0);
            return false;
        }
    }
    wait_stat(p, where, c0);
    return true;
}

// Bounded wait on an mbarrier phase; the common case (phase complete) stays inline.
__device__ __forceinline__ bool mbar_wait_bounded(const Params& p, uint64_t* bar, uint32_t parity, int where) {
    if (mbar_try_wait(bar, parity)) return true;
    return mbar_wait_slow(p, bar, parity, where);
}

// Sync of the 8 consumer warps through an mbarrier (one arrival per warp, after
// __syncwarp).  Every wait is bounded: on a timeout the CTA's abort flag is
// raised instead of hanging, so no path can stall a consumer forever.  Each
// consumer thread keeps its own copy of the phase parity.
__device__ __forceinline__ void csync(const Params& p, Smem& sm, uint32_t& phase) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(&sm.csync);
    if (!mbar_wait_bounded(p, &sm.csync, phase, 8)) sm.flag[3] = 1;
    phase ^= 1;
}
// The same among consumer warps 4-7 (the warps that read the accumulators: warp
// w owns TMEM lane quarter w - 4); false when the wait gave up (the CTA is aborting).
__device__ __forceinline__ bool msync4(const Params& p, Smem& sm, uint32_t& phase) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(&sm.mm_sync);
    const bool ok = mbar_wait_bounded(p, &sm.mm_sync, phase, 13);
    if (!ok) sm.flag[3] = 1;
    phase ^= 1;
    return ok;
}


// Wait on a phase that another thread of this CTA has already seen complete
// (so it returns at once); bounded anyway: on failure it records a fault and
// raises the CTA's abort flag, which every consumer reads after its next barrier.
__device__ __forceinline__ void seen_complete_wait(const Params& p, uint64_t* bar, uint32_t parity, int* abort_flag) {
    for (int i = 0; i < (1 << 22); ++i)
        if (mbar_try_wait(bar, parity)) return;
    set_error(p, kErrFault, -1, -6, (int)parity, (int)(blockIdx.x - p.cta0));
    *abort_flag = 1;
}

// Spin (acquire) until events[e] >= target.  Single thread.
__device__ bool event_wait(const Params& p, uint32_t e, uint32_t target, int task) {
    Waiter w{0, 0};
    const long long c0 = p.stats ? clock64() : 0;
    bool ok = true;
    while (true) {
        uint32_t v = ld_acquire(&p.events[e]);
        if ((int32_t)(v - target) >= 0) break;
        if (wait_should_stop(p, w)) {
            if (ld_relaxed_int(p.err) == 0) set_error(p, kErrTimeout, task, (int)e, (int)v, (int)target);
            ok = false;
            break;
        }
        __nanosleep(32);
    }
    if (p.stats && threadIdx.x == 0) stat_add(p, 2, (unsigned long long)(clock64() - c0));
    return ok;
}

// Spin (acquire, system scope) until a tensor-parallel arrival flag reaches target.
// Single thread; bounded like every other wait.
__device__ bool tp_flag_wait(const Params& p, const uint32_t* f, uint32_t target, int task) {
    Waiter w{0, 0};
    while (true) {
        const uint32_t v = ld_acquire_sys(f);
        if ((int32_t)(v - target) >= 0) return true;
        if (wait_should_stop(p, w)) {
            if (ld_relaxed_int(p.err) == 0) set_error(p, kErrTimeout, task, -11, (int)v, (int)target);
            return false;
        }
        __nanosleep(32);
    }
}

// ----------------------------------------------------------------------------- producer

// Producer ring position: fill number n goes to stage n % kStages on lap
// n / kStages; a slot of lap k > 0 is free once the consumers released lap k-1.
struct PRing {
    int stage;
    uint32_t lap;
};
__device__ __forceinline__ bool pr_acquire(const Params& p, Smem& sm, const PRing& r) {
    if (r.lap == 0) return true;                       // first lap: slots start empty
    return mbar_wait_bounded(p, &sm.empty[r.stage], (r.lap - 1) & 1, 1);
}
__device__ __forceinline__ void pr_advance(PRing& r) {
    if (++r.stage == kStages) { r.stage = 0; ++r.lap; }
}

// The pages of a wide attention task: per page, stages of hps KV heads each (2 at
// d = 128), a stage holding the heads' key blocks then their value blocks (the page
// holds the heads' 16 x d blocks back to back, so each half is one contiguous copy):
// a warp finds both halves of its head in one stage.  The stage's info.aux is the
// logical page.  Page ids are read 8 at a time, a batch ahead, into the shared ring
// of ids; an id out of range is reported and its stages go out empty.
__device__ __noinline__ bool produce_wide_pages(const Params& p, Smem& sm, const Task& t, int ti, PRing& ring,
                                                uint64_t pol) {
    // the split's cached positions (the new token is attended from registers)
    int npages = 0, lp0 = 0;
    if (t.b < p.batch) {
        const int pos = position_of(p, t.b);
        if (pos >= 0 && pos < p.max_ctx && pos / kPageSize < p.max_pages) {
            int j0 = 0, j1 = 0;
            const int sa = attn_active_splits(pos + 1, (int)t.r1);
            if ((int)t.r0 < sa) attn_range(pos + 1, sa, (int)t.r0, j0, j1);
            const int jc = min(j1, pos);
            if (jc > j0) {
                lp0 = j0 / kPageSize;
                npages = (jc - 1) / kPageSize - lp0 + 1;
            }
        }
    }
    const int nkv = p.nkv, n_pages = p.n_pages;
    const uint32_t blk = (uint32_t)(kPageSize * p.hd * 2);
    const size_t blk_elems = (size_t)kPageSize * p.hd;
    const int hps = kStageBytes / (2 * (int)blk);           // KV heads per stage (keys and values)
    const int spp = (nkv + hps - 1) / hps;                  // stages per page
    const int nch = npages * spp;
    if (nch == 0) {
        if (!pr_acquire(p, sm, ring)) return false;
        sm.info[ring.stage] = StageInfo{ti, 0, 0, 0, t};
        mbar_arrive(&sm.full[ring.stage]);
        pr_advance(ring);
        return true;
    }
    const int* prow = page_row(p, t.b);
    int pid_have = 0;
    for (int c = 0; c < nch; ++c) {
        const int pg = c / spp, q = c % spp;
        if (q == 0) {
            while (pid_have < min(npages, pg + 1 + kPidBatch)) {
                int v[kPidBatch];
#pragma unroll
                for (int i = 0; i < kPidBatch; ++i) {
                    const int k = pid_have + i;
                    v[i] = (k < npages) ? __ldg(prow + lp0 + k) : 0;
                }
#pragma unroll
                for (int i = 0; i < kPidBatch; ++i) sm.pid[(pid_have + i) % kPidRing] = v[i];
                pid_have += kPidBatch;
            }
        }
        if (!pr_acquire(p, sm, ring)) return false;
        StageInfo& inf = sm.info[ring.stage];
        inf.task = ti;
        inf.chunk = c;
        inf.nchunks = nch;
        inf.aux = lp0 + pg;
        if (c == 0) inf.rec = t;
        const int ph = sm.pid[pg % kPidRing];
        if (ph < 0 || ph >= n_pages) {                       // validated before any copy of the page
            set_error(p, kErrInvalid, ti, -2, lp0 + pg, t.b);
            mbar_arrive(&sm.full[ring.stage]);
            pr_advance(ring);
            continue;
        }
        const int h0 = q * hps, nh = min(hps, nkv - h0);
        mbar_arrive_expect_tx(&sm.full[ring.stage], 2u * (uint32_t)nh * blk);
        const size_t off = (((size_t)t.layer * n_pages + ph) * nkv + h0) * blk_elems;
        bulk_g2s(sm.ring[ring.stage], p.k_pages + off, (uint32_t)nh * blk, &sm.full[ring.stage], pol);
        bulk_g2s(sm.ring[ring.stage] + (size_t)nh * blk, p.v_pages + off, (uint32_t)nh * blk, &sm.full[ring.stage], pol);
        pr_advance(ring);
    }
    return true;
}

// Attention splits of at least this many ring stages hold the producer's next claim
// until the consumers start them.
constexpr int kHoldStages = 6;

// Tasks whose streamed data is only known on the device: attention (KV pages of
// this step's positions) and routed experts (weights of the expert the router
// picked).  Out of line: it keeps the producer's hot loop small.
// MM: the instantiation for batched graphs (their KV appends run in tasks of their own).
template <bool MM>
__device__ __noinline__ bool produce_special(const Params& p, Smem& sm, const Task& t, int ti, PRing& ring,
                                             uint32_t& last_router_evt, uint64_t pol) {
    int& stage = ring.stage;
    bool ok = true;
    auto acquire_slot = [&]() -> bool { return pr_acquire(p, sm, ring); };
    auto advance = [&]() { pr_advance(ring); };
    do {
        if (t.op == MK_OP_ATTN) {
            const int b = t.b;
            int npages = 0, lp0 = 0;
            if (b < p.batch) {
                int pos = position_of(p, b);
                if (pos >= 0 && pos < p.max_ctx && pos / kPageSize < p.max_pages) {
                    int j0 = 0, j1 = 0;
                    const int sa = attn_active_splits(pos + 1, (int)t.r1);
                    if ((int)t.r0 < sa) attn_range(pos + 1, sa, (int)t.r0, j0, j1);
                    // batch-1 graphs: cached positions only (the new token is fresh);
                    // batched graphs: the new positions are in the cache too
                    int jc = MM ? j1 : min(j1, pos);
                    if (jc > j0) {
                        lp0 = j0 / kPageSize;
                        npages = (jc - 1) / kPageSize - lp0 + 1;
                    }
                }
            }
            // (this function is out of line: the parameters the loop needs are read once
            // into registers rather than through the parameter block's address per stage)
            const int nkv = p.nkv, n_pages = p.n_pages;
            const uint16_t* const kpool = p.k_pages;
            const uint16_t* const vpool = p.v_pages;
            const size_t blk_elems = (size_t)kPageSize * p.hd;
            const int pps = pages_per_stage(p);
            const int nch = (npages + pps - 1) / pps;
            const uint32_t blk = (uint32_t)(kPageSize * p.hd * 2);
            if (nch == 0) {
                if (!acquire_slot()) { ok = false; break; }
                sm.info[stage] = StageInfo{ti, 0, 0, 0, t};
                mbar_arrive(&sm.full[stage]);
                advance();
            }
            // physical page ids, read kPidBatch at a time (independent loads, one round
            // trip per batch) into a small ring in shared memory, a batch ahead of use
            const int* prow = page_row(p, b);
            int pid_have = 0;                              // ids [0, pid_have) of the split loaded
            // batched graphs append this step's K/V in tasks of their own: pages holding a
            // new position are loaded only after the attention task's event (which
            // counts those appends); older pages stream at once
            const int first_new = MM ? (p.seq_row >= 0 ? position_of(p, 0) : position_of(p, b)) : INT_MAX;
            bool appended = !MM || t.wait0 == MK_NO_EVENT;
            auto pid_ensure = [&](int upto) {
                while (pid_have < upto) {
                    int v[kPidBatch];
#pragma unroll
                    for (int i = 0; i < kPidBatch; ++i) {
                        const int k = pid_have + i;
                        v[i] = (k < npages) ? __ldg(prow + lp0 + k) : 0;
                    }
#pragma unroll
                    for (int i = 0; i < kPidBatch; ++i) sm.pid[(pid_have + i) % kPidRing] = v[i];
                    pid_have += kPidBatch;
                }
            };
            for (int c = 0; c < nch && ok; ++c) {
                int first = lp0 + c * pps;
                int n = min(pps, lp0 + npages - first);
                pid_ensure(min(npages, c * pps + n + kPidBatch));
                if (MM && !appended && (first + n) * kPageSize > first_new) {
                    if (!event_wait(p, t.wait0, p.thr[t.wait0] * p.epoch + p.wait_offset, ti)) { ok = false; break; }
                    asm volatile("fence.proxy.async.global;" ::: "memory");   // generic-proxy writes first
                    appended = true;
                }
                if (!acquire_slot()) { ok = false; break; }
                sm.info[stage].task = ti; sm.info[stage].chunk = c; sm.info[stage].nchunks = nch;
                sm.info[stage].aux = first;
                if (c == 0) sm.info[stage].rec = t;
                // validate page indices before issuing any copy
                bool bad = false;
                for (int i = 0; i < n; ++i) {
                    int ph = sm.pid[(c * pps + i) % kPidRing];
                    if (ph < 0 || ph >= n_pages) bad = true;
                }
                if (bad) {
                    set_error(p, kErrInvalid, ti, -2, first, b);
                    mbar_arrive(&sm.full[stage]);
                    advance();
                    continue;
                }
                mbar_arrive_expect_tx(&sm.full[stage], (uint32_t)n * 2u * blk);
                for (int i = 0; i < n; ++i) {
                    int ph = sm.pid[(c * pps + i) % kPidRing];
                    size_t off = (((size_t)t.layer * n_pages + ph) * nkv + t.aux) * blk_elems;
                    uint8_t* dst = sm.ring[stage] + (size_t)i * 2 * blk;
                    bulk_g2s(dst, kpool + off, blk, &sm.full[stage], pol);
                    bulk_g2s(dst + blk, vpool + off, blk, &sm.full[stage], pol);
                }
                advance();
            }
            break;
        }
        // GEMV-type task
        bool skip = (t.op == MK_OP_LMHEAD && p.skip_lm);
        if ((t.op == MK_OP_EXP_GATEUP || t.op == MK_OP_EXP_DOWN) && t.pad != MK_NO_EVENT &&
            t.pad != last_router_evt) {
            // the expert id comes from the router: wait for it before computing addresses
            if (!event_wait(p, t.pad, p.thr[t.pad] * p.epoch + p.wait_offset, ti)) { ok = false; break; }
            last_router_evt = t.pad;
        }
        GemvGeom g;
        gemv_geom(p, t, g, !skip);
        const int nch = skip ? 0 : gemv_chunks(g, t.flags);
        if (nch == 0) {
            if (!acquire_slot()) { ok = false; break; }
            sm.info[stage] = StageInfo{ti, 0, 0, 0, t};
            mbar_arrive(&sm.full[stage]);
            advance();
            continue;
        }
        // chunk sequence (the consumer walks the same one): per weight block, either
        // groups of whole rows that fit one stage, or one row in stage-sized segments
        const int64_t RB = (int64_t)g.K * 2;
        int c = 0;
        auto issue = [&](const uint8_t* src, uint32_t bytes) -> bool {
            if (!acquire_slot()) return false;
            sm.info[stage].task = ti; sm.info[stage].chunk = c; sm.info[stage].nchunks = nch;
            if (c == 0) sm.info[stage].rec = t;
            mbar_arrive_expect_tx(&sm.full[stage], bytes);
            bulk_g2s(sm.ring[stage], src, bytes, &sm.full[stage], pol);
            advance();
            ++c;
            return true;
        };
        for (int bi = 0; bi < g.nblk && ok; ++bi) {
            const uint8_t* base = reinterpret_cast<const uint8_t*>(g.w[bi]);
            if (RB <= kStageBytes) {
                const int rps = is_warp_row(t.flags) ? kWarpRows : (int)(kStageBytes / RB);
                for (int r0 = 0; r0 < g.rows && ok; r0 += rps) {
                    const int n = min(rps, g.rows - r0);
                    ok = issue(base + (int64_t)r0 * RB, (uint32_t)(n * RB));
                }
            } else {
                for (int r = 0; r < g.rows && ok; ++r)
                    for (int64_t off = 0; off < RB && ok; off += kStageBytes) {
                        const int64_t left = RB - off;
                        ok = issue(base + (int64_t)r * RB + off,
                                   (uint32_t)(left < kStageBytes ? left : (int64_t)kStageBytes));
                    }
            }
        }
    } while (false);
    return ok;
}

// Tensor-core tile: per K-block one weight box (128 rows, or the matching 64 gate
// and 64 up rows) in its own stage; the activation boxes (hi rows then lo rows)
// of up to mm_kblocks_per_xstage consecutive K-blocks share one stage ahead of
// their weight boxes, so most of the ring holds weights in flight.  The
// activations are written by earlier tasks: the loads wait for their event.
__device__ __forceinline__ int mm_kblocks_per_xstage(int bp) {
    const int k = kStageBytes / (2 * bp * 128);
    return k < 1 ? 1 : k;
}
__device__ __forceinline__ const void* tmap_at(const Params& p, uint32_t idx) {
    return reinterpret_cast<const uint8_t*>(p.tmaps) + (size_t)idx * 128;
}
__device__ __noinline__ bool produce_mm(const Params& p, Smem& sm, const Task& t, int ti, PRing& ring,
                                        uint64_t pol) {
    const bool two = (t.op == MK_OP_MM_GATEUP);
    const void* w0 = tmap_at(p, (uint32_t)t.src[0]);
    const void* w1 = two ? tmap_at(p, (uint32_t)t.src[1]) : nullptr;
    const int wy = (int)(t.src[0] >> 32);
    int xop = kOpXq;
    switch (t.op) {
        case MK_OP_MM_OPROJ: xop = kOpAo; break;
        case MK_OP_MM_GATEUP: xop = kOpXf; break;
        case MK_OP_MM_DOWN: xop = kOpAct; break;
        case MK_OP_MM_LMHEAD: xop = kOpXl; break;
        default: break;
    }
    const void* xm = tmap_at(p, (uint32_t)xop);
    const int xy = (t.op == MK_OP_MM_LMHEAD) ? 0 : (int)t.layer * 2 * p.bp;
    const uint32_t xbytes = 2u * (uint32_t)p.bp * 128u;
    const int kb0 = (int)t.row_bytes, kb1 = (int)t.pad2, nch = (int)t.nchunks;
    const int kx = mm_kblocks_per_xstage(p.bp);
    int c = 0;
    auto open_stage = [&](uint32_t bytes) -> bool {
        if (!pr_acquire(p, sm, ring)) return false;
        StageInfo& inf = sm.info[ring.stage];
        inf.task = ti;
        inf.chunk = c;
        inf.nchunks = nch;
        if (c == 0) inf.rec = t;
        mbar_arrive_expect_tx(&sm.full[ring.stage], bytes);
        return true;
    };
    if (t.wait0 != MK_NO_EVENT) {
        if (!event_wait(p, t.wait0, p.thr[t.wait0] * p.epoch + p.wait_offset, ti)) return false;
        // the operand was written through the generic proxy by other CTAs; order those
        // writes before this CTA's tensor loads
        asm volatile("fence.proxy.async.global;" ::: "memory");
    }
    for (int g0 = kb0; g0 < kb1; g0 += kx) {
        const int g1 = min(kb1, g0 + kx);
        // the activation boxes of the group's K-blocks, side by side in one stage, ahead
        // of the weight boxes: each weight box is multiplied as soon as it lands
        if (!open_stage(xbytes * (uint32_t)(g1 - g0))) return false;
        for (int kb = g0; kb < g1; ++kb)
            tma_load_2d(sm.ring[ring.stage] + (size_t)(kb - g0) * xbytes, xm, kb * kMmK, xy, &sm.full[ring.stage]);
        pr_advance(ring);
        ++c;
        for (int kb = g0; kb < g1; ++kb) {
            if (!open_stage((uint32_t)kStageBytes)) return false;
            uint8_t* dst = sm.ring[ring.stage];
            if (two) {
                tma_load_2d_hint(dst, w0, kb * kMmK, wy, &sm.full[ring.stage], pol);
                tma_load_2d_hint(dst + kStageBytes / 2, w1, kb * kMmK, wy, &sm.full[ring.stage], pol);
            } else {
                tma_load_2d_hint(dst, w0, kb * kMmK, wy, &sm.full[ring.stage], pol);
            }
            pr_advance(ring);
            ++c;
        }
    }
    return true;
}

// Whether this step's attention splits hold the producer's next claim (see
// producer_loop): batched graphs' splits (ragged, long contexts) always; a batch-1
// step's splits when its first split streams kHoldStages stages or more (all its
// splits are equal to within a page).  Decided once per step, so that no attention
// task's claim waits on a load of the position.  (Wide steps always hold.)
template <bool MM>
__device__ __forceinline__ bool attn_hold_this_step(const Params& p) {
    if (MM) return true;
    const int pos = position_of(p, 0);
    if (pos < 0 || pos >= p.max_ctx) return false;
    const int sa = attn_active_splits(pos + 1, p.S);
    int j0, j1;
    attn_range(pos + 1, sa, 0, j0, j1);
    const int jc = min(j1, pos);
    if (jc <= j0) return false;
    const int npages = (jc - 1) / kPageSize - j0 / kPageSize + 1;
    const int pps = pages_per_stage(p);
    return (npages + pps - 1) / pps >= kHoldStages;
}

// Producer: waits (bounded) until the consumers have started task ti.
__device__ bool wait_started(const Params& p, Smem& sm, int ti) {
    const volatile int* st = &sm.started;
    Waiter w{0, 0};
    while (*st < ti) {
        if (*reinterpret_cast<volatile int*>(&sm.flag[3])) return false;
        if (wait_should_stop(p, w)) {
            if (ld_relaxed_int(p.err) == 0) set_error(p, kErrTimeout, ti, -12, 0, (int)(blockIdx.x - p.cta0));
            return false;
        }
        __nanosleep(32);
    }
    return true;
}

// An attention task of a step whose splits hold: its pages, then a wait until the
// consumers have started it (the caller claims the next task after that).
template <bool MM, bool WIDE>
__device__ __forceinline__ bool produce_attention_held(const Params& p, Smem& sm, const Task& t, int ti, PRing& ring,
                                                    uint64_t pol) {
    bool ok;
    if (WIDE && (t.flags & kAttnWide)) {
        ok = produce_wide_pages(p, sm, t, ti, ring, pol);
    } else {
        uint32_t no_router = MK_NO_EVENT;
        ok = produce_special<MM>(p, sm, t, ti, ring, no_router, pol);
    }
    return ok && wait_started(p, sm, ti);
}

template <bool MM, bool WIDE>
__device__ void producer_loop(const Params& p, Smem& sm) {
    const uint64_t pol = l2_evict_first_policy();
    PRing ring{0, 0};
    bool ok = true;
    uint32_t last_router_evt = MK_NO_EVENT;
    // The next task is claimed while the current one's copies are issued, so the
    // atomic's round trip overlaps useful work.  Still exactly one failing claim
    // per CTA, which keeps the queue head at (n_tasks + grid) per step.
    // In the batched and long-attention kernels, attention tasks are the exception
    // when this step's splits are long (kHoldStages ring stages or more, every wide
    // split; attn_hold_this_step): after issuing one, the producer claims the next
    // task only once the consumers have started it.  Otherwise a CTA that reaches a
    // layer's attention early claims two or three of its tasks (their pages fit the
    // ring) and runs them one after another while other CTAs, whose next claims are
    // the O-projection tiles waiting for all attention, stay idle (30B MoE at an
    // 8192-token context: 6.37 -> 5.7 ms per step; 8B at 131072 tokens: 13.74 ->
    // 10.8 ms).
    if constexpr (MM || WIDE) sm.attn_hold = -1;     // decided at the step's first attention task
    unsigned long long q_next = atomicAdd(p.queue, 1ull) - p.queue_base;
    uint32_t n_claimed = 0;
    while (ok) {
        // abort checks: the CTA's own flag every task, the grid's status word (an L2
        // round trip) every 32 tasks; waits below poll it too
        if (sm.flag[3] != 0 || ((++n_claimed & 31) == 0 && ld_relaxed_int(p.err) != 0)) { ok = false; break; }
        const unsigned long long q = q_next;
        if (q >= p.n_tasks) break;
        const int ti = (int)q;
        *reinterpret_cast<volatile int*>(&sm.pf_claimed) = ti;
        const Task t = p.tasks[ti];
        if constexpr (MM || WIDE) {
            // a step whose attention splits hold: the claim after an attention task
            // waits until the consumers have started it
            if (sm.attn_hold > 0 && t.op == MK_OP_ATTN) {
                ok = produce_attention_held<MM, WIDE>(p, sm, t, ti, ring, pol);
                if (ok) q_next = atomicAdd(p.queue, 1ull) - p.queue_base;
                continue;
            }
        }
        q_next = atomicAdd(p.queue, 1ull) - p.queue_base;
        if constexpr (MM) {
            if (is_mm_op(t.op)) {
                ok = produce_mm(p, sm, t, ti, ring, pol);
                continue;
            }
        }
        if constexpr (WIDE) {
            if (t.op == MK_OP_ATTN && (t.flags & kAttnWide)) {
                sm.attn_hold = 1;                            // every wide step holds
                ok = produce_wide_pages(p, sm, t, ti, ring, pol);
                continue;
            }
        }
        const bool skip = (t.op == MK_OP_LMHEAD && p.skip_lm) || t.op == MK_OP_NORM || t.op == MK_OP_KVAPPEND ||
                          t.op == MK_OP_ATTN_MERGE || t.op == MK_OP_TP_REDUCE;
        if (skip) {                                      // nothing to stream: a marker stage
            if (!pr_acquire(p, sm, ring)) { ok = false; break; }
            sm.info[ring.stage] = StageInfo{ti, 0, 0, 0, t};
            mbar_arrive(&sm.full[ring.stage]);
            pr_advance(ring);
            continue;
        }
        if (t.nchunks == 0 || t.op == MK_OP_ATTN) {
            if constexpr (MM || WIDE) {
                // (the step's first attention task decides whether its splits hold)
                if (t.op == MK_OP_ATTN && sm.attn_hold < 0) sm.attn_hold = attn_hold_this_step<MM>(p) ? 1 : 0;
            }
            ok = produce_special<MM>(p, sm, t, ti, ring, last_router_evt, pol);
            continue;
        }
        // dense GEMV tile: the plan the host computed (the consumer walks the same
        // chunk sequence): per block, chunk_rows whole rows per stage, or each row in
        // stage-sized segments
        const uint32_t rb = t.row_bytes, rows = t.r1 - t.r0, nch = t.nchunks;
        uint32_t c = 0;
        for (int bi = 0; bi < t.nblk && ok; ++bi) {
            const uint8_t* base = reinterpret_cast<const uint8_t*>(t.src[bi]);
            const uint32_t step = t.chunk_rows ? t.chunk_rows * rb : (uint32_t)kStageBytes;
            const uint32_t total = rows * rb;
            for (uint32_t off = 0; off < total && ok; ) {
                uint32_t bytes;
                if (t.chunk_rows) {
                    bytes = (total - off < step) ? total - off : step;
                } else {
                    const uint32_t in_row = off % rb;          // segments restart at each row
                    bytes = (rb - in_row < step) ? rb - in_row : step;
                }
                if (!pr_acquire(p, sm, ring)) { ok = false; break; }
                StageInfo& inf = sm.info[ring.stage];
                inf.task = ti;
                inf.chunk = (int)c;
                inf.nchunks = (int)nch;
                if (c == 0) inf.rec = t;
                mbar_arrive_expect_tx(&sm.full[ring.stage], bytes);
                bulk_g2s(sm.ring[ring.stage], base + off, bytes, &sm.full[ring.stage], pol);
                pr_advance(ring);
                ++c;
                off += bytes;
            }
        }
    }
    *reinterpret_cast<volatile int*>(&sm.pf_claimed) = -1;   // the prefetcher stops
    int& stage = ring.stage;
    uint32_t& lap = ring.lap;
    auto acquire_slot = [&]() -> bool { return pr_acquire(p, sm, ring); };
    auto advance = [&]() { pr_advance(ring); };
    // end-of-work marker (best effort when aborting)
    if (acquire_slot()) {
        sm.info[stage].task = -1;
        mbar_arrive(&sm.full[stage]);
        advance();
    }
    // drain: every issued fill must have landed before the CTA's shared memory goes away
    // (stage s has had lap + (s < stage) fills; the last one has parity fills - 1)
    for (int s = 0; s < kStages; ++s) {
        const uint32_t fills = lap + (s < stage ? 1u : 0u);
        if (fills == 0) continue;
        Waiter w{0, 0};
        while (!mbar_try_wait(&sm.full[s], (fills - 1) & 1)) {
            if (++w.spins > (1 << 26)) break;   // copies of valid memory always land; hard cap only
        }
    }
}

// ----------------------------------------------------------------------------- L2 prefetcher

// Asks L2 to fetch the weight rows (and KV pages) of tasks a bounded distance
// ahead of the work queue, so that HBM keeps streaming while this CTA's consumers
// wait on a dependency (at an operator boundary the ring holds the next tile, and
// HBM would otherwise idle until the event fires).  It issues prefetches ONLY while
// consumer warp 0 is waiting: at any other time the stream is HBM-bound already and
// a prefetch would only compete with the tiles the next event waits for.  The task
// list is dealt to the CTAs statically (CTA c covers tasks c, c + grid, ...; the
// union over the CTAs covers every task of the window whoever claims it), tasks
// already claimed are skipped, and the window ends pf_dist tasks past this CTA's
// latest claim (shared memory): no atomics and no polling of global memory.
// Routed-expert weights are unknown until the router runs and are skipped.
__device__ void prefetch_loop(const Params& p, Smem& sm) {
    if (p.pf_dist == 0) return;
    const volatile int* claimed = &sm.pf_claimed;
    const volatile int* waiting = &sm.pf_wait;
    for (uint32_t i = blockIdx.x - p.cta0; i < p.n_tasks; i += p.ncta) {
        Waiter w{0, 0};
        bool skip = false;
        while (true) {
            const int c = *claimed;
            if (c < 0 || *reinterpret_cast<volatile int*>(&sm.flag[3])) return;   // producer done or aborting
            if (i <= (uint32_t)c) { skip = true; break; }                         // claimed: streaming already
            if ((uint32_t)c + p.pf_dist >= i && *waiting) break;
            if (wait_should_stop(p, w)) return;          // an error elsewhere; a slow step is not one
            __nanosleep(64);
        }
        if (skip) continue;
        const Task t = p.tasks[i];
        if (t.op == MK_OP_ATTN) {
            const int b = t.b;
            if (b >= p.batch) continue;
            const int pos = position_of(p, b);
            if (pos < 0 || pos >= p.max_ctx || pos / kPageSize >= p.max_pages) continue;
            const int sa = attn_active_splits(pos + 1, (int)t.r1);
            if ((int)t.r0 >= sa) continue;
            int j0, j1;
            attn_range(pos + 1, sa, (int)t.r0, j0, j1);
            const int jc = min(j1, pos);
            if (jc <= j0) continue;
            const int* prow = page_row(p, b);
            const uint32_t blk = (uint32_t)(kPageSize * p.hd * 2);
            for (int lp = j0 / kPageSize; lp <= (jc - 1) / kPageSize; ++lp) {
                const int ph = prow[lp];
                if (ph < 0 || ph >= p.n_pages) break;
                const size_t off = (((size_t)t.layer * p.n_pages + ph) * p.nkv + t.aux) * (size_t)kPageSize * p.hd;
                prefetch_l2(p.k_pages + off, blk);
                prefetch_l2(p.v_pages + off, blk);
            }
            continue;
        }
        if (t.op == MK_OP_EXP_GATEUP || t.op == MK_OP_EXP_DOWN || t.op >= MK_OP_NORM) continue;
        if (t.op == MK_OP_LMHEAD && p.skip_lm) continue;
        GemvGeom g;
        gemv_geom(p, t, g, true);
        const int64_t bytes = (int64_t)g.rows * g.K * 2;
        for (int bi = 0; bi < g.nblk; ++bi)
            for (int64_t off = 0; off < bytes; off += 32768) {
                const int64_t n = bytes - off < 32768 ? bytes - off : 32768;
                prefetch_l2(reinterpret_cast<const uint8_t*>(g.w[bi]) + off, (uint32_t)n);
            }
    }
}

// ----------------------------------------------------------------------------- consumer helpers

// bf16 split of an fp32 value: hi = bf16(v), lo = bf16(v - hi); hi + lo carries
// about 16 significant bits, so a bf16 x bf16 product of the weight and the pair
// keeps the activation's fp32 precision to within ~2^-17 relative.
__device__ __forceinline__ void split_hilo(float v, uint16_t& hi, uint16_t& lo) {
    hi = f32_to_bf16_rne(v);
    lo = f32_to_bf16_rne(v - bf16_to_f32(hi));
}
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Operand rows of batch row b: hi at row (base + b), lo at row (base + bp + b).
__device__ __forceinline__ void put_operand4(const Params& p, int op, int layer, int b, int K, int col,
                                             float4 v) {
    const size_t base = (size_t)layer * 2 * p.bp;
    uint16_t h[4], l[4];
    split_hilo(v.x, h[0], l[0]);
    split_hilo(v.y, h[1], l[1]);
    split_hilo(v.z, h[2], l[2]);
    split_hilo(v.w, h[3], l[3]);
    uint16_t* hi = p.opnd[op] + (base + b) * K + col;
    uint16_t* lo = p.opnd[op] + (base + p.bp + b) * K + col;
    *reinterpret_cast<uint2*>(hi) = make_uint2(h[0] | ((uint32_t)h[1] << 16), h[2] | ((uint32_t)h[3] << 16));
    *reinterpret_cast<uint2*>(lo) = make_uint2(l[0] | ((uint32_t)l[1] << 16), l[2] | ((uint32_t)l[3] << 16));
}


// Residual stream entering layer l (l == L: after the last layer), element i of batch row b.
__device__ __forceinline__ float x_in(const Params& p, int l, int b, int i) {
    if (l == 0) {
        int tok = p.tokens[b];
        if (tok < 0 || tok >= p.V) tok = 0;   // recorded as an error by the prologue
        return bf16_to_f32(p.tok_emb[(size_t)tok * p.H + i]);
    }
    if (p.E == 0) return __ldcg(p.x_out + ((size_t)(l - 1) * p.max_batch + b) * p.H + i);
    const size_t lb = (size_t)(l - 1) * p.max_batch + b;
    float v = __ldcg(p.x_mid + lb * p.H + i);
    for (int k = 0; k < p.topk; ++k)
        v = fmaf(__ldcg(p.moe_w + lb * p.topk + k), __ldcg(p.ypart + (lb * p.topk + k) * p.H + i), v);
    return v;
}

__device__ __forceinline__ float x_mid_at(const Params& p, int l, int b, int i) {
    return __ldcg(p.x_mid + ((size_t)l * p.max_batch + b) * p.H + i);
}

__device__ __forceinline__ const uint16_t* gemv_norm_gain(const Params& p, const Task& t) {
    switch (t.op) {
        case MK_OP_QKV: return p.layers[t.layer].attn_norm;
        case MK_OP_GATEUP:
        case MK_OP_ROUTER:
        case MK_OP_EXP_GATEUP: return p.layers[t.layer].ffn_norm;
        case MK_OP_LMHEAD: return p.final_norm;
        default: return nullptr;
    }
}

// Sum over all consumer threads, same order in every CTA.
__device__ __forceinline__ float block_sum(const Params& p, Smem& sm, uint32_t& cph, float v) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    v = warp_sum(v);
    if (lane == 0) sm.bcast[warp] = v;
    csync(p, sm, cph);
    float s = 0.0f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) s += sm.bcast[w];
    csync(p, sm, cph);   // bcast is free again
    return s;
}

struct ThreadMap {
    int nvec, wpg, G, grp, lig, gstride, vpt;
    bool active;
};

__device__ __forceinline__ ThreadMap thread_map(int K) {
    ThreadMap m;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    m.nvec = K / 8;
    int wneed = (m.nvec + 31) / 32;
    m.wpg = min(kConsumerWarps, wneed);
    m.G = kConsumerWarps / m.wpg;
    m.grp = warp / m.wpg;
    m.lig = (warp % m.wpg) * 32 + lane;
    m.gstride = m.wpg * 32;
    m.vpt = (m.nvec + m.gstride - 1) / m.gstride;
    m.active = m.grp < m.G;
    return m;
}

// Loads this thread's slice of the (normalised) input into registers.
// Split partials: o[L][B][nkv][S][HPG][hd] (not yet divided by l; 16-byte aligned
// rows) followed by ml[L][B][nkv][S][HPG][2] = (m in the log2 domain, l).
__device__ __forceinline__ size_t attn_part_index(const Params& p, int l, int b, int g, int s, int h) {
    return ((((size_t)l * p.max_batch + b) * p.nkv + g) * p.S + s) * hpg_of(p) + h;
}
__device__ __forceinline__ float* attn_part_o(const Params& p, size_t idx) { return p.part + idx * p.hd; }
__device__ __forceinline__ float* attn_part_ml(const Params& p, size_t idx) {
    return p.part + (size_t)p.L * p.max_batch * p.nkv * p.S * hpg_of(p) * p.hd + 2 * idx;
}

// The attention output of one (sequence, kv group): the active splits' partials
// merged in split order (m* = max m_s; o = sum 2^(m_s - m*) o_s / sum 2^(m_s - m*) l_s,
// the split-K merge of flash-decoding), normalised, for the group's q heads.  Run
// once, by all consumer threads of the CTA whose split arrived last: the (m, l)
// pairs go through shared memory in one parallel pass, then every thread merges
// four consecutive columns of one head with all of its loads in flight.
__device__ void attn_merge_group(const Params& p, Smem& sm, uint32_t& cph, int l, int b, int g) {
    const int hd = p.hd, hpg = hpg_of(p), tid = threadIdx.x;
    int pos = position_of(p, b);
    if (pos < 0 || pos >= p.max_ctx) pos = 0;
    const int sa = attn_active_splits(pos + 1, p.S);      // (2 S + 1) * hpg floats fit the scratch
    float* f = sm.attn;                                     // [sa][hpg] weights, then [hpg] 1/L, then [sa][hpg] l
    float* fl = f + (sa + 1) * hpg;
    const size_t i0 = attn_part_index(p, l, b, g, 0, 0);   // split s, head h at i0 + s*hpg + h
    // every split's (m, l) in one parallel pass: the loop below reads only shared memory
    for (int k = tid; k < sa * hpg; k += kConsumerThreads) {
        const float2 ml = __ldcg(reinterpret_cast<const float2*>(attn_part_ml(p, i0 + k)));
        f[k] = ml.x;
        fl[k] = ml.y;
    }
    csync(p, sm, cph);
    if (tid < hpg) {
        float M = -INFINITY;
        for (int sp = 0; sp < sa; ++sp) M = fmaxf(M, f[sp * hpg + tid]);
        float L = 0.0f;
        for (int sp = 0; sp < sa; ++sp) {
            const float mm = f[sp * hpg + tid];
            const float w = (mm == -INFINITY) ? 0.0f : exp2f(mm - M);
            L = fmaf(fl[sp * hpg + tid], w, L);
            f[sp * hpg + tid] = w;
        }
        f[sa * hpg + tid] = (L > 0.0f) ? 1.0f / L : 0.0f;
    }
    csync(p, sm, cph);
    float* out = p.attn_o + ((size_t)l * p.max_batch + b) * p.nq * hd + (size_t)g * hpg * hd;
    for (int q = tid; q < hpg * hd / 4; q += kConsumerThreads) {
        const int h = (q * 4) / hd, i = (q * 4) % hd;
        float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
        for (int sp = 0; sp < sa; ++sp) {
            const float w = f[sp * hpg + h];
            const float4 v = __ldcg(reinterpret_cast<const float4*>(attn_part_o(p, i0 + (size_t)sp * hpg + h) + i));
            o.x = fmaf(v.x, w, o.x); o.y = fmaf(v.y, w, o.y); o.z = fmaf(v.z, w, o.z); o.w = fmaf(v.w, w, o.w);
        }
        const float inv = f[sa * hpg + h];
        const float4 r = make_float4(o.x * inv, o.y * inv, o.z * inv, o.w * inv);
        *reinterpret_cast<float4*>(out + (size_t)h * hd + i) = r;
        if (p.mm) put_operand4(p, kOpAo, l, b, p.nq * hd, g * hpg * hd + h * hd + i, r);
    }
    if (p.mm) fence_proxy_async_global();
}

// Where a GEMV task's input vector lives: an fp32 row, a bf16 embedding row, and
// for an MoE residual the routed experts' outputs with their combine weights.
struct InSrc {
    const float* base;
    const uint16_t* emb;
    const float* parts;   // [nparts][pstride]
    const float* pw;      // [nparts]
    int nparts, pstride;
};

__device__ __forceinline__ InSrc xin_src(const Params& p, int l, int b) {
    InSrc s{nullptr, nullptr, nullptr, nullptr, 0, 0};
    if (l == 0) {
        int tok = p.tokens[b];
        if (tok < 0 || tok >= p.V) tok = 0;   // recorded as an error by the QKV task
        s.emb = p.tok_emb + (size_t)tok * p.H;
    } else if (p.E == 0) {
        s.base = p.x_out + ((size_t)(l - 1) * p.max_batch + b) * p.H;
    } else {
        const size_t lb = (size_t)(l - 1) * p.max_batch + b;
        s.base = p.x_mid + lb * p.H;
        s.parts = p.ypart + lb * p.topk * p.H;
        s.pw = p.moe_w + lb * p.topk;
        s.nparts = p.topk;
        s.pstride = p.H;
    }
    return s;
}

__device__ __forceinline__ InSrc gemv_src(const Params& p, const Task& t) {
    const int l = t.layer, b = t.b;
    InSrc s{nullptr, nullptr, nullptr, nullptr, 0, 0};
    switch (t.op) {
        case MK_OP_QKV: return xin_src(p, l, 0);
        case MK_OP_LMHEAD: return xin_src(p, p.L, 0);
        case MK_OP_OPROJ: s.base = p.attn_o + ((size_t)l * p.max_batch) * p.nq * p.hd; break;
        case MK_OP_GATEUP:
        case MK_OP_ROUTER: s.base = p.x_mid + ((size_t)l * p.max_batch) * p.H; break;
        case MK_OP_EXP_GATEUP: s.base = p.x_mid + ((size_t)l * p.max_batch + b) * p.H; break;
        case MK_OP_DOWN: s.base = p.act + ((size_t)l * p.max_batch) * p.F; break;
        case MK_OP_EXP_DOWN:
            s.base = p.act + (((size_t)l * p.max_batch + b) * p.topk + t.aux) * p.Fe;
            break;
        default: break;
    }
    return s;
}

// Eight consecutive input elements starting at col (a multiple of 8), as four
// pairs; every load is independent so a thread's whole slice is in flight at once.
template <bool PARTS>
__device__ __forceinline__ void load8(const InSrc& s, int col, float2 (&x)[4]) {
    if (s.emb) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(s.emb + col));
        x[0] = make_float2(bf_lo(u.x), bf_hi(u.x));
        x[1] = make_float2(bf_lo(u.y), bf_hi(u.y));
        x[2] = make_float2(bf_lo(u.z), bf_hi(u.z));
        x[3] = make_float2(bf_lo(u.w), bf_hi(u.w));
        return;
    }
    const float4 a = __ldcg(reinterpret_cast<const float4*>(s.base + col));
    const float4 c = __ldcg(reinterpret_cast<const float4*>(s.base + col + 4));
    x[0] = make_float2(a.x, a.y);
    x[1] = make_float2(a.z, a.w);
    x[2] = make_float2(c.x, c.y);
    x[3] = make_float2(c.z, c.w);
    if constexpr (PARTS) {
    for (int k = 0; k < s.nparts; ++k) {
        const float w = __ldcg(s.pw + k);
        const float4 pa = __ldcg(reinterpret_cast<const float4*>(s.parts + (size_t)k * s.pstride + col));
        const float4 pc = __ldcg(reinterpret_cast<const float4*>(s.parts + (size_t)k * s.pstride + col + 4));
        x[0] = make_float2(fmaf(w, pa.x, x[0].x), fmaf(w, pa.y, x[0].y));
        x[1] = make_float2(fmaf(w, pa.z, x[1].x), fmaf(w, pa.w, x[1].y));
        x[2] = make_float2(fmaf(w, pc.x, x[2].x), fmaf(w, pc.y, x[2].y));
        x[3] = make_float2(fmaf(w, pc.z, x[3].x), fmaf(w, pc.w, x[3].y));
    }
    }
}

// Loads this thread's slice of the (RMS-normalised) input into registers in one
// pass: the sum of squares comes from the slices of group 0, which together
// cover every column exactly once, so every CTA reduces in the same order.
template <bool PARTS>
__device__ void gemv_prologue_t(const Params& p, Smem& sm, uint32_t& cph, const Task& t, const ThreadMap& m,
                                int K, const InSrc& src, float2 (&xr)[kMaxVecPerThread][4]) {
    const uint16_t* gain = gemv_norm_gain(p, t);
    float ss = 0.0f;
    // the norm gains of this thread's columns are loaded together with the input, so
    // their latency overlaps the input loads and the block-wide sum
    uint4 gv[kMaxVecPerThread];
#pragma unroll
    for (int j = 0; j < kMaxVecPerThread; ++j) {
        const int v = m.lig + j * m.gstride;
        const bool mine = j < m.vpt && v < m.nvec && m.active;
        gv[j] = (gain && mine) ? __ldg(reinterpret_cast<const uint4*>(gain + v * 8)) : make_uint4(0u, 0u, 0u, 0u);
        if (mine) {
            load8<PARTS>(src, v * 8, xr[j]);
        } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) xr[j][e] = make_float2(0.0f, 0.0f);
        }
    }
#pragma unroll
    for (int j = 0; j < kMaxVecPerThread; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) ss = fmaf(xr[j][e].y, xr[j][e].y, fmaf(xr[j][e].x, xr[j][e].x, ss));
    if (gain) {
        const float tot = block_sum(p, sm, cph, (m.grp == 0 && m.active) ? ss : 0.0f);
        const float rstd = 1.0f / sqrtf(tot / (float)K + p.eps);
#pragma unroll
        for (int j = 0; j < kMaxVecPerThread; ++j) {
            const int v = m.lig + j * m.gstride;
            if (j < m.vpt && v < m.nvec && m.active) {
                const uint4 u = gv[j];
                const float g[8] = {bf_lo(u.x), bf_hi(u.x), bf_lo(u.y), bf_hi(u.y),
                                    bf_lo(u.z), bf_hi(u.z), bf_lo(u.w), bf_hi(u.w)};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    xr[j][e] = make_float2((xr[j][e].x * rstd) * g[2 * e], (xr[j][e].y * rstd) * g[2 * e + 1]);
            }
        }
    }
}

__device__ __forceinline__ void gemv_prologue(const Params& p, Smem& sm, uint32_t& cph, const Task& t,
                                              const ThreadMap& m, int K,
                                              float2 (&xr)[kMaxVecPerThread][4]) {
    const InSrc src = gemv_src(p, t);
    if (src.nparts > 0) gemv_prologue_t<true>(p, sm, cph, t, m, K, src, xr);
    else gemv_prologue_t<false>(p, sm, cph, t, m, K, src, xr);
}

// Packed fp32x2 fused multiply-add (sm_100): d = a * b + c, lane-wise on two floats.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n .reg .b64 ra, rb, rc, rd;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n"
        " mov.b64 rc, {%6, %7};\n fma.rn.f32x2 rd, ra, rb, rc;\n mov.b64 {%0, %1}, rd;\n}\n"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

// acc.x accumulates the even elements of 8 bf16 weights times x, acc.y the odd ones.
__device__ __forceinline__ void dot8(const uint4 q, const float2 (&x)[4], float2& acc) {
    acc = ffma2(make_float2(bf_lo(q.x), bf_hi(q.x)), x[0], acc);
    acc = ffma2(make_float2(bf_lo(q.y), bf_hi(q.y)), x[1], acc);
    acc = ffma2(make_float2(bf_lo(q.z), bf_hi(q.z)), x[2], acc);
    acc = ffma2(make_float2(bf_lo(q.w), bf_hi(q.w)), x[3], acc);
}
__device__ __forceinline__ void dot8(const uint4 q, const float2 (&x)[4], float& a0, float& a1) {
    float2 acc = make_float2(a0, a1);
    dot8(q, x, acc);
    a0 = acc.x;
    a1 = acc.y;
}

// Sums N per-lane values over the warp at once (reduce-scatter: N/2 + N/4 + ... + 1
// shuffles, then log2(32/N) more).  Lane l returns the total of value l / (32/N).
template <int N>
__device__ __forceinline__ float warp_reduce_rows(float (&v)[N]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int cnt = N, o = 16; cnt > 1; cnt >>= 1, o >>= 1) {
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < cnt / 2; ++i) {
            const float send = up ? v[i] : v[i + cnt / 2];
            const float keep = up ? v[i + cnt / 2] : v[i];
            v[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, o);
        }
    }
    float r = v[0];
#pragma unroll
    for (int o = 16 / N; o >= 1; o >>= 1) r += __shfl_xor_sync(0xFFFFFFFFu, r, o);
    return r;
}

// Whole rows [r0, r0+n) of block `blk` sit in `sv` back to back (nvec vectors each).
template <int VPT>
__device__ __forceinline__ void gemv_rows(Smem& sm, int buf, const uint4* sv, const ThreadMap& m,
                                          int rows, int blk, int r0, int n,
                                          const float2 (&xr)[kMaxVecPerThread][4]) {
    const int lane = threadIdx.x & 31, wig = (threadIdx.x >> 5) % m.wpg;
    const int nvec = m.nvec;
    float* red = &sm.red[buf][blk * rows + r0][0];
    if (m.G == 1) {
        int rr = 0;
        for (; rr + 1 < n; rr += 2) {
            const uint4* p0 = sv + rr * nvec;
            const uint4* p1 = p0 + nvec;
            float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
#pragma unroll
            for (int j = 0; j < VPT; ++j) {
                const int v = m.lig + j * m.gstride;
                if (v < nvec) {
                    const uint4 q0 = p0[v], q1 = p1[v];
                    dot8(q0, xr[j], a0, a1);
                    dot8(q1, xr[j], b0, b1);
                }
            }
            float a = a0 + a1, b = b0 + b1;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                a += __shfl_xor_sync(0xFFFFFFFFu, a, o);
                b += __shfl_xor_sync(0xFFFFFFFFu, b, o);
            }
            if (lane == 0) {
                red[rr * kConsumerWarps + wig] = a;
                red[(rr + 1) * kConsumerWarps + wig] = b;
            }
        }
        if (rr < n) {
            const uint4* p0 = sv + rr * nvec;
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int j = 0; j < VPT; ++j) {
                const int v = m.lig + j * m.gstride;
                if (v < nvec) dot8(p0[v], xr[j], a0, a1);
            }
            float a = warp_sum(a0 + a1);
            if (lane == 0) red[rr * kConsumerWarps + wig] = a;
        }
    } else {
        if (!m.active) return;
        int rr = ((m.grp - r0 % m.G) % m.G + m.G) % m.G;
        for (; rr < n; rr += m.G) {
            const uint4* p0 = sv + rr * nvec;
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int j = 0; j < VPT; ++j) {
                const int v = m.lig + j * m.gstride;
                if (v < nvec) dot8(p0[v], xr[j], a0, a1);
            }
            float a = warp_sum(a0 + a1);
            if (lane == 0) red[rr * kConsumerWarps + wig] = a;
        }
    }
}

// Streams one GEMV task's chunks out of the ring (same sequence as the producer)
// and leaves the warps' partial row sums in red[buf].  Returns false on abort.
template <int VPT>
__device__ bool gemv_task_body(const Params& p, Smem& sm, int ti, const GemvGeom& g,
                               const ThreadMap& m, const float2 (&xr)[kMaxVecPerThread][4], int buf,
                               int& stage, uint32_t& lap, bool skip) {
    const int lane = threadIdx.x & 31, wig = (threadIdx.x >> 5) % m.wpg;
    bool first = true;
    auto next_stage = [&]() -> bool {
        if (!first && !mbar_wait_bounded(p, &sm.full[stage], lap & 1, 5)) {
            sm.flag[3] = 1;
            return false;
        }
        first = false;
        if (sm.info[stage].task != ti) {
            set_error(p, kErrFault, ti, -4, sm.info[stage].task, 1);
            sm.flag[3] = 1;
            return false;
        }
        return true;
    };
    auto release = [&]() {
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty[stage]);
        if (++stage == kStages) { stage = 0; ++lap; }
    };
    if (skip) {
        if (!next_stage()) return false;
        release();
        return true;
    }
    const int64_t RB = (int64_t)g.K * 2;
    for (int blk = 0; blk < g.nblk; ++blk) {
        if (RB <= kStageBytes) {
            const int rps = (int)(kStageBytes / RB);
            for (int r0 = 0; r0 < g.rows; r0 += rps) {
                if (!next_stage()) return false;
                gemv_rows<VPT>(sm, buf, reinterpret_cast<const uint4*>(sm.ring[stage]), m, g.rows, blk,
                               r0, min(rps, g.rows - r0), xr);
                release();
            }
        } else {
            constexpr int kSegVec = kStageBytes / 16;
            for (int r = 0; r < g.rows; ++r) {
                float a0 = 0.f, a1 = 0.f;
                for (int vs = 0; vs < m.nvec; vs += kSegVec) {
                    if (!next_stage()) return false;
                    const int ve = min(m.nvec, vs + kSegVec);
                    const uint4* sv = reinterpret_cast<const uint4*>(sm.ring[stage]) - vs;
#pragma unroll
                    for (int j = 0; j < VPT; ++j) {
                        const int v = m.lig + j * m.gstride;
                        if (v >= vs && v < ve) dot8(sv[v], xr[j], a0, a1);
                    }
                    release();
                }
                const float a = warp_sum(a0 + a1);
                if (lane == 0) sm.red[buf][blk * g.rows + r][wig] = a;
            }
        }
    }
    return true;
}

// Fast paths for rows whose 16-byte vectors split evenly over the 256 consumer
// threads (hidden sizes that are multiples of 2048): every thread owns VPT
// vectors of every row, the NROWS row sums stay in registers across the task's
// stages, and the warp reduces them once at the end.

// Rows that fit a stage: RPS rows per stage, NROWS / RPS stages.
template <int VPT, int RPS, int NROWS>
__device__ bool gemv_fast_rows(const Params& p, Smem& sm, int ti, const float2 (&xr)[kMaxVecPerThread][4],
                               int buf, int& stage, uint32_t& lap) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // The stage loop stays rolled (small code: the SM's instruction cache is shared
    // with the producer and signal loops).  Each stage's RPS row sums enter at the
    // end of `acc` while the older ones shift down, so after NROWS / RPS stages
    // acc[r] holds row r.
    float acc[NROWS];
#pragma unroll
    for (int r = 0; r < NROWS; ++r) acc[r] = 0.f;
#pragma unroll 1
    for (int st = 0; st < NROWS / RPS; ++st) {
        if (st > 0 && !mbar_wait_bounded(p, &sm.full[stage], lap & 1, 5)) { sm.flag[3] = 1; return false; }
        if (sm.info[stage].task != ti) { set_error(p, kErrFault, ti, -4, sm.info[stage].task, 2); sm.flag[3] = 1; return false; }
        const uint4* sv = reinterpret_cast<const uint4*>(sm.ring[stage]) + threadIdx.x;
        uint4 q[RPS][VPT];
#pragma unroll
        for (int rr = 0; rr < RPS; ++rr)
#pragma unroll
            for (int j = 0; j < VPT; ++j) q[rr][j] = sv[(rr * VPT + j) * kConsumerThreads];
#pragma unroll
        for (int r = 0; r < NROWS - RPS; ++r) acc[r] = acc[r + RPS];
#pragma unroll
        for (int rr = 0; rr < RPS; ++rr) {
            float2 a = make_float2(0.f, 0.f);
#pragma unroll
            for (int j = 0; j < VPT; ++j) dot8(q[rr][j], xr[j], a);
            acc[NROWS - RPS + rr] = a.x + a.y;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty[stage]);
        if (++stage == kStages) { stage = 0; ++lap; }
    }
    const float tot = warp_reduce_rows<NROWS>(acc);
    if ((lane & (32 / NROWS - 1)) == 0) sm.red[buf][lane / (32 / NROWS)][warp] = tot;
    return true;
}

// Rows longer than a stage: each row arrives as segments of SEGJ*256 vectors
// (the last segment holds the rest); NROWS rows, one rolled iteration per row.
template <int VPT, int SEGJ, int NROWS>
__device__ bool gemv_fast_segs(const Params& p, Smem& sm, int ti, const float2 (&xr)[kMaxVecPerThread][4],
                               int buf, int& stage, uint32_t& lap, bool first_seen) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int NSEG = (VPT + SEGJ - 1) / SEGJ;
    float acc[NROWS];
#pragma unroll
    for (int r = 0; r < NROWS; ++r) acc[r] = 0.f;
#pragma unroll 1
    for (int r = 0; r < NROWS; ++r) {
        float2 a = make_float2(0.f, 0.f);
#pragma unroll
        for (int sg = 0; sg < NSEG; ++sg) {
            if ((r > 0 || sg > 0 || !first_seen) && !mbar_wait_bounded(p, &sm.full[stage], lap & 1, 5)) {
                sm.flag[3] = 1;
                return false;
            }
            if (sm.info[stage].task != ti) { set_error(p, kErrFault, ti, -4, sm.info[stage].task, 3); sm.flag[3] = 1; return false; }
            const uint4* sv = reinterpret_cast<const uint4*>(sm.ring[stage]) + threadIdx.x;
            uint4 q[SEGJ];
#pragma unroll
            for (int j = 0; j < SEGJ; ++j)
                if (sg * SEGJ + j < VPT) q[j] = sv[j * kConsumerThreads];
#pragma unroll
            for (int j = 0; j < SEGJ; ++j)
                if (sg * SEGJ + j < VPT) dot8(q[j], xr[sg * SEGJ + j], a);
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.empty[stage]);
            if (++stage == kStages) { stage = 0; ++lap; }
        }
#pragma unroll
        for (int i = 0; i < NROWS - 1; ++i) acc[i] = acc[i + 1];
        acc[NROWS - 1] = a.x + a.y;
    }
    const float tot = warp_reduce_rows<NROWS>(acc);
    if ((lane & (32 / NROWS - 1)) == 0) sm.red[buf][lane / (32 / NROWS)][warp] = tot;
    return true;
}

// Short rows (VPL 16-byte vectors per lane): each stage holds kWarpRows rows, warp w
// takes row w, sums it with a warp reduction and leaves the total in red[buf][row][0].
template <int VPL>
__device__ bool gemv_fast_warprow(const Params& p, Smem& sm, int ti, int rows,
                                  const float2 (&xr)[kMaxVecPerThread][4], int buf, int& stage, uint32_t& lap) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int rb = VPL * 32 * 16;                        // bytes per row
#pragma unroll 1
    for (int r0 = 0; r0 < rows; r0 += kWarpRows) {
        if (r0 > 0 && !mbar_wait_bounded(p, &sm.full[stage], lap & 1, 5)) { sm.flag[3] = 1; return false; }
        if (sm.info[stage].task != ti) { set_error(p, kErrFault, ti, -4, sm.info[stage].task, 4); sm.flag[3] = 1; return false; }
        if (r0 + warp < rows) {
            const uint4* sv = reinterpret_cast<const uint4*>(sm.ring[stage] + warp * rb) + lane;
            float2 a = make_float2(0.f, 0.f);
#pragma unroll
            for (int j = 0; j < VPL; ++j) dot8(sv[32 * j], xr[j], a);
            const float tot = warp_sum(a.x + a.y);
            if (lane == 0) sm.red[buf][r0 + warp][0] = tot;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty[stage]);
        if (++stage == kStages) { stage = 0; ++lap; }
    }
    return true;
}

// Runs the task's fast path (variant chosen by the planner); false on abort.
__device__ __forceinline__ bool gemv_fast_dispatch(const Params& p, Smem& sm, int ti, int variant, int rows,
                                                   const float2 (&xr)[kMaxVecPerThread][4], int buf,
                                                   int& stage, uint32_t& lap) {
    switch (variant) {
        case kFastW2: return gemv_fast_warprow<2>(p, sm, ti, rows, xr, buf, stage, lap);
        case kFastW3: return gemv_fast_warprow<3>(p, sm, ti, rows, xr, buf, stage, lap);
        case kFastW4: return gemv_fast_warprow<4>(p, sm, ti, rows, xr, buf, stage, lap);
        case kFastV2R2N16: return gemv_fast_rows<2, 2, 16>(p, sm, ti, xr, buf, stage, lap);
        case kFastV2R2N8: return gemv_fast_rows<2, 2, 8>(p, sm, ti, xr, buf, stage, lap);
        case kFastV1R4N16: return gemv_fast_rows<1, 4, 16>(p, sm, ti, xr, buf, stage, lap);
        case kFastV1R4N8: return gemv_fast_rows<1, 4, 8>(p, sm, ti, xr, buf, stage, lap);
        case kFastV2R2N4: return gemv_fast_rows<2, 2, 4>(p, sm, ti, xr, buf, stage, lap);
        case kFastV1R4N4: return gemv_fast_rows<1, 4, 4>(p, sm, ti, xr, buf, stage, lap);
        case kFastV7S4N4: return gemv_fast_segs<7, 4, 4>(p, sm, ti, xr, buf, stage, lap, true);
        case kFastV7S4N1: return gemv_fast_segs<7, 4, 1>(p, sm, ti, xr, buf, stage, lap, true);
        default: return gemv_fast_segs<7, 4, 2>(p, sm, ti, xr, buf, stage, lap, true);
    }
}

__device__ __forceinline__ bool gemv_task_dispatch(const Params& p, Smem& sm, int ti, const GemvGeom& g,
                                                   const ThreadMap& m,
                                                   const float2 (&xr)[kMaxVecPerThread][4], int buf,
                                                   int& stage, uint32_t& lap, bool skip) {
    switch (m.vpt) {
        case 1: return gemv_task_body<1>(p, sm, ti, g, m, xr, buf, stage, lap, skip);
        case 2: return gemv_task_body<2>(p, sm, ti, g, m, xr, buf, stage, lap, skip);
        case 3: return gemv_task_body<3>(p, sm, ti, g, m, xr, buf, stage, lap, skip);
        case 4: return gemv_task_body<4>(p, sm, ti, g, m, xr, buf, stage, lap, skip);
        case 5: return gemv_task_body<5>(p, sm, ti, g, m, xr, buf, stage, lap, skip);
        case 6: return gemv_task_body<6>(p, sm, ti, g, m, xr, buf, stage, lap, skip);
        case 7: return gemv_task_body<7>(p, sm, ti, g, m, xr, buf, stage, lap, skip);
        default: return gemv_task_body<8>(p, sm, ti, g, m, xr, buf, stage, lap, skip);
    }
}

// ----------------------------------------------------------------------------- consumer: attention


// ---- attention on the tensor cores (mma.sync m16n8k16, bf16 inputs, fp32 accumulators)
//
// Scores S = Q K^T and the output O = P V of one kv group, 16 tokens (one page) at a
// time.  The A operand has 16 rows: rows 0..7 carry the bf16 value of q (or of the
// probabilities p) of head h = row, rows 8..15 the bf16 rounding residual of the
// same values, so one MMA yields hi and lo products whose sum is the fp32
// product to about 2^-16 relative; each result row h is then the sum of rows h
// and h + 8.  Rows of heads >= HPG are zero.  Keys and values are bf16 already.
// A page is first copied by its warp into a per-warp staging buffer with its
// 16-byte chunks XOR-swizzled by row, so that the ldmatrix loads that gather MMA
// operands across 8 tokens hit 8 different bank groups.

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    return (uint32_t)f32_to_bf16_rne(lo) | ((uint32_t)f32_to_bf16_rne(hi) << 16);
}
// hi and lo parts of a pair of fp32 values as two bf16x2 words
__device__ __forceinline__ void split_bf16x2(float a, float b, uint32_t& hi, uint32_t& lo) {
    const uint16_t ha = f32_to_bf16_rne(a), hb = f32_to_bf16_rne(b);
    hi = (uint32_t)ha | ((uint32_t)hb << 16);
    lo = pack_bf16x2(a - bf16_to_f32(ha), b - bf16_to_f32(hb));
}
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr) : "memory");
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr) : "memory");
}

template <int HPG, int DPL>
struct AttnMma {
    static constexpr int HD = DPL * 32, KS = HD / 16, NT = HD / 8;
    uint32_t qa[KS][4];   // A fragments of q (rows 0..7 hi, 8..15 lo)
    float o[NT][4];       // accumulator fragments of P V
    float m, l;           // running max (log2 domain) and partial sum of this thread's row
};

// Byte offset of 16-byte chunk c of token row r in a swizzled staging page.
template <int HD>
__device__ __forceinline__ uint32_t stg_off(int r, int c) {
    return (uint32_t)(r * HD * 2 + 16 * (c ^ (r & 7)));
}

// Copies one 16 x HD bf16 page block from the ring into the warp's staging buffer,
// swizzled; with `zero_out` the rows outside [k_lo, k_hi) become zeros (values of
// masked tokens must not reach P V, whatever the cache holds there).
__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a)
                 : "memory");
    return v;
}
__device__ __forceinline__ void sts128(uint32_t a, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// (shared-memory addresses throughout: the ring and the staging page are both in
// this CTA's shared memory)
template <int HD>
__device__ __forceinline__ void stage_page(const uint16_t* src, uint8_t* stg, int k_lo, int k_hi, bool zero_out) {
    constexpr int CPR = HD / 8;                         // 16-byte chunks per row
    const int lane = threadIdx.x & 31;
    const uint32_t s0 = smem_u32(src), d0 = smem_u32(stg);
    uint4 v[kPageSize * CPR / 32];
#pragma unroll
    for (int i = 0; i < kPageSize * CPR / 32; ++i) v[i] = lds128(s0 + 16u * (lane + 32 * i));
#pragma unroll
    for (int i = 0; i < kPageSize * CPR / 32; ++i) {
        const int q = lane + 32 * i, r = q / CPR, c = q % CPR;
        if (zero_out && (r < k_lo || r >= k_hi)) v[i] = make_uint4(0u, 0u, 0u, 0u);
        sts128(d0 + stg_off<HD>(r, c), v[i]);
    }
}

// S (two n-tiles of 8 tokens) = Q K^T for the staged page.
template <int HPG, int DPL>
__device__ __forceinline__ void attn_qk(const AttnMma<HPG, DPL>& st, const uint8_t* stg, float (&s0)[4],
                                        float (&s1)[4]) {
    constexpr int HD = DPL * 32, KS = HD / 16;
    const int lane = threadIdx.x & 31, mi = lane >> 3, rr = lane & 7;
    const int tok = rr + ((mi & 2) ? 8 : 0);
    const uint32_t base = smem_u32(stg);
#pragma unroll
    for (int e = 0; e < 4; ++e) s0[e] = s1[e] = 0.0f;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
        uint32_t b[4];
        ldsm_x4(b, base + stg_off<HD>(tok, 2 * ks + (mi & 1)));
        mma_16816(s0, st.qa[ks], b[0], b[1]);
        mma_16816(s1, st.qa[ks], b[2], b[3]);
    }
}

// Online softmax over the page's 16 scores of this thread's row, then the
// hi/lo A fragments of the probabilities.
template <int HPG, int DPL>
__device__ __forceinline__ void attn_softmax(AttnMma<HPG, DPL>& st, const float (&s0)[4], const float (&s1)[4],
                                             int k_lo, int k_hi, uint32_t (&pa)[4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    float sc[4] = {s0[0] + s0[2], s0[1] + s0[3], s1[0] + s1[2], s1[1] + s1[3]};
    const int tk[4] = {2 * t, 2 * t + 1, 8 + 2 * t, 9 + 2 * t};
#pragma unroll
    for (int i = 0; i < 4; ++i)
        if (g >= HPG || tk[i] < k_lo || tk[i] >= k_hi) sc[i] = -INFINITY;
    float mb = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
    mb = fmaxf(mb, __shfl_xor_sync(0xFFFFFFFFu, mb, 1));
    mb = fmaxf(mb, __shfl_xor_sync(0xFFFFFFFFu, mb, 2));
    const float m_new = fmaxf(st.m, mb);
    float pr[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    if (m_new != -INFINITY) {
        const float corr = exp2f(st.m - m_new);         // 0 while m was -inf
#pragma unroll
        for (int i = 0; i < 4; ++i) pr[i] = exp2f(sc[i] - m_new);
        st.l = fmaf(st.l, corr, (pr[0] + pr[1]) + (pr[2] + pr[3]));
#pragma unroll
        for (int j = 0; j < AttnMma<HPG, DPL>::NT; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) st.o[j][e] *= corr;
        st.m = m_new;
    }
    split_bf16x2(pr[0], pr[1], pa[0], pa[1]);
    split_bf16x2(pr[2], pr[3], pa[2], pa[3]);
}

// O += P V for the staged page (values of masked tokens already zero).
template <int HPG, int DPL>
__device__ __forceinline__ void attn_pv(AttnMma<HPG, DPL>& st, const uint8_t* stg, const uint32_t (&pa)[4]) {
    constexpr int HD = DPL * 32, NT = HD / 8;
    const int lane = threadIdx.x & 31, mi = lane >> 3, rr = lane & 7;
    const int tok = rr + ((mi & 1) ? 8 : 0);
    const uint32_t base = smem_u32(stg);
#pragma unroll
    for (int jj = 0; jj < NT / 2; ++jj) {
        uint32_t b[4];
        ldsm_x4_trans(b, base + stg_off<HD>(tok, 2 * jj + ((mi & 2) ? 1 : 0)));
        mma_16816(st.o[2 * jj], pa, b[0], b[1]);
        mma_16816(st.o[2 * jj + 1], pa, b[2], b[3]);
    }
}

// One cached page of the split (tokens [k_lo, k_hi) of it valid).
template <int HPG, int DPL>
__device__ __forceinline__ void attn_page(AttnMma<HPG, DPL>& st, const uint16_t* kblk, const uint16_t* vblk,
                                          int k_lo, int k_hi, uint8_t* stg) {
    constexpr int HD = DPL * 32;
    stage_page<HD>(kblk, stg, k_lo, k_hi, false);
    __syncwarp();
    float s0[4], s1[4];
    attn_qk<HPG, DPL>(st, stg, s0, s1);
    uint32_t pa[4];
    attn_softmax<HPG, DPL>(st, s0, s1, k_lo, k_hi, pa);
    __syncwarp();                                        // every lane is done with the keys
    stage_page<HD>(vblk, stg, k_lo, k_hi, true);
    __syncwarp();
    attn_pv<HPG, DPL>(st, stg, pa);
    __syncwarp();                                        // staging is reused by the next page
}

// The new token (its k and v, bf16-rounded, in shared memory) as a one-token page.
template <int HPG, int DPL>
__device__ __forceinline__ void attn_new_token(AttnMma<HPG, DPL>& st, const float* kn, const float* vn,
                                               uint8_t* stg) {
    constexpr int HD = DPL * 32, CPR = HD / 8;
    const int lane = threadIdx.x & 31;
    auto stage_row0 = [&](const float* x) {             // row 0 = x, rows 1..15 = 0
        for (int q = lane; q < kPageSize * CPR; q += 32) {
            const int r = q / CPR, c = q % CPR;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (r == 0) {
                const float* e = x + 8 * c;
                v = make_uint4(pack_bf16x2(e[0], e[1]), pack_bf16x2(e[2], e[3]), pack_bf16x2(e[4], e[5]),
                               pack_bf16x2(e[6], e[7]));
            }
            sts128(smem_u32(stg) + stg_off<HD>(r, c), v);
        }
    };
    stage_row0(kn);
    __syncwarp();
    float s0[4], s1[4];
    attn_qk<HPG, DPL>(st, stg, s0, s1);
    uint32_t pa[4];
    attn_softmax<HPG, DPL>(st, s0, s1, 0, 1, pa);
    __syncwarp();
    stage_row0(vn);
    __syncwarp();
    attn_pv<HPG, DPL>(st, stg, pa);
    __syncwarp();
}

// One split of decode attention for (layer, sequence b, kv head g): RoPE on the
// group's q heads and the new k, KV-cache append (the split that owns the new
// position), softmax partial over the split's positions streamed from the paged
// cache.  Writes the partial and hands the completion to the signal warp; the
// O-projection's input stage merges the splits in a fixed order.
// MM: batched graphs, whose KV append runs in tasks of its own before attention;
// every position, the new one included, then comes from the cache.
template <int HPG, int DPL, bool MM>
__device__ void attention_task(const Params& p, Smem& sm, uint32_t& cph, const Task& t, int ti, int& stage,
                               uint32_t& lap, bool& abort_all) {
    constexpr int HD = DPL * 32;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = t.b, g = t.aux, s = (int)t.r0, S = (int)t.r1, l = t.layer;
    const bool active_row = b < p.batch;
    int pos = active_row ? position_of(p, b) : 0;
    bool valid = active_row && pos >= 0 && pos < p.max_ctx && pos / kPageSize < p.max_pages;
    if (active_row && !valid && tid == 0) set_error(p, kErrInvalid, ti, -3, pos, b);
    int j0 = 0, j1 = 0;
    if (valid) {
        const int sa = attn_active_splits(pos + 1, S);
        if (s < sa) attn_range(pos + 1, sa, s, j0, j1);
    }
    const bool has_new = !MM && valid && pos >= j0 && pos < j1;
    const float qscale = 1.4426950408889634f / sqrtf((float)HD);   // log2(e) / sqrt(d)

    AttnMma<HPG, DPL> st;
    st.m = -INFINITY;
    st.l = 0.0f;
#pragma unroll
    for (int j = 0; j < AttnMma<HPG, DPL>::NT; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) st.o[j][e] = 0.0f;
#pragma unroll
    for (int ks = 0; ks < AttnMma<HPG, DPL>::KS; ++ks)
#pragma unroll
        for (int e = 0; e < 4; ++e) st.qa[ks][e] = 0u;
    const bool work = valid && j1 > j0;
    csync(p, sm, cph);                                   // shared scratch of the previous task is free
    if (work) {
        // q of the group's heads and the new k (rotated at `pos`), the new v; all loads
        // of a thread are issued before any is used
        const float* qkv = p.qkv + ((size_t)l * p.max_batch + b) * ((p.nq + 2 * p.nkv) * HD);
        const float* rope = p.rope + (size_t)pos * HD;   // [HD/2][2] = cos, sin
        constexpr int NPAIR = (HPG + 1) * (HD / 2);
        constexpr int IT = (NPAIR + kConsumerThreads - 1) / kConsumerThreads;
        float x0[IT], x1[IT], cs[IT], sn[IT];
#pragma unroll
        for (int it = 0; it < IT; ++it) {
            const int idx = tid + it * kConsumerThreads;
            if (idx < NPAIR) {
                const int h = idx / (HD / 2), i = idx % (HD / 2);
                const float* src = (h < HPG) ? qkv + (size_t)(g * HPG + h) * HD : qkv + (size_t)(p.nq + g) * HD;
                x0[it] = __ldcg(src + i);
                x1[it] = __ldcg(src + i + HD / 2);
                const float2 r = __ldg(reinterpret_cast<const float2*>(rope) + i);
                cs[it] = r.x;
                sn[it] = r.y;
            }
        }
        float vv = 0.0f;
        if (tid < HD) vv = __ldcg(qkv + (size_t)(p.nq + p.nkv + g) * HD + tid);
#pragma unroll
        for (int it = 0; it < IT; ++it) {
            const int idx = tid + it * kConsumerThreads;
            if (idx < NPAIR) {
                const int h = idx / (HD / 2), i = idx % (HD / 2);
                const float r0 = x0[it] * cs[it] - x1[it] * sn[it], r1 = x1[it] * cs[it] + x0[it] * sn[it];
                if (h < HPG) {
                    sm.qs[h * HD + i] = r0 * qscale;
                    sm.qs[h * HD + i + HD / 2] = r1 * qscale;
                } else {
                    sm.kn[i] = bf16_to_f32(f32_to_bf16_rne(r0));
                    sm.kn[i + HD / 2] = bf16_to_f32(f32_to_bf16_rne(r1));
                }
            }
        }
        if (tid < HD) sm.vn[tid] = bf16_to_f32(f32_to_bf16_rne(vv));
        csync(p, sm, cph);
        // KV append: the split that owns the new position writes it
        if (has_new) {
            const int* prow = page_row(p, b);
            const int ph = prow[pos / kPageSize];
            if (ph >= 0 && ph < p.n_pages) {
                size_t off = ((((size_t)l * p.n_pages + ph) * p.nkv + g) * kPageSize + pos % kPageSize) * HD;
                if (tid < HD) {
                    p.k_pages[off + tid] = f32_to_bf16_rne(sm.kn[tid]);
                    p.v_pages[off + tid] = f32_to_bf16_rne(sm.vn[tid]);
                }
            } else if (tid == 0) {
                set_error(p, kErrInvalid, ti, -2, pos / kPageSize, b);
            }
        }
        // q as hi/lo bf16 A fragments: thread (g, t) holds head g's columns
        // 16ks + 2t, +1, +8, +9 (rows of heads >= HPG stay zero)
        const int g4 = lane >> 2, t4 = lane & 3;
        if (g4 < HPG) {
#pragma unroll
            for (int ks = 0; ks < AttnMma<HPG, DPL>::KS; ++ks) {
                const float* qh = sm.qs + g4 * HD + 16 * ks + 2 * t4;
                split_bf16x2(qh[0], qh[1], st.qa[ks][0], st.qa[ks][1]);
                split_bf16x2(qh[8], qh[9], st.qa[ks][2], st.qa[ks][3]);
            }
        }
    }

    // streamed chunks of cached pages (the first stage was seen complete by thread 0)
    const int jc = MM ? j1 : min(j1, pos);
    const int pps = pages_per_stage(p);
    const int blk_elems = kPageSize * HD;
    uint8_t* stg = reinterpret_cast<uint8_t*>(sm.attn) + warp * (kPageSize * HD * 2);   // staging page
    for (int c = 0;; ++c) {
        if (c == 0) {
            seen_complete_wait(p, &sm.full[stage], lap & 1, &sm.flag[3]);
        } else if (!mbar_wait_bounded(p, &sm.full[stage], lap & 1, 3)) {
            sm.flag[3] = 1;
            break;
        }
        const StageInfo inf = sm.info[stage];
        if (inf.task != ti) {
            set_error(p, kErrFault, ti, -4, inf.task, 0);
            sm.flag[3] = 1;
            break;
        }
        if (inf.nchunks > 0) {
            const uint16_t* base = reinterpret_cast<const uint16_t*>(sm.ring[stage]);
            const int first_page = inf.aux;
            const int tok_lo = max(j0, first_page * kPageSize);
            const int tok_hi = min(jc, (first_page + pps) * kPageSize);
            // pages are dealt to the warps round-robin over the whole stream
#pragma unroll 1
            for (int pi = 0; pi < pps; ++pi) {
                if (((inf.chunk * pps + pi) & (kConsumerWarps - 1)) != warp) continue;
                const int pf = (first_page + pi) * kPageSize;
                const int k_lo = max(tok_lo - pf, 0), k_hi = min(tok_hi - pf, kPageSize);
                if (k_hi <= k_lo) continue;
                const uint16_t* kb = base + (size_t)pi * 2 * blk_elems;
                attn_page<HPG, DPL>(st, kb, kb + blk_elems, k_lo, k_hi, stg);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty[stage]);
        const bool last = inf.nchunks == 0 || inf.chunk == inf.nchunks - 1;
        if (++stage == kStages) { stage = 0; ++lap; }
        if (last) break;
    }
    if (has_new && warp == 0) attn_new_token<HPG, DPL>(st, sm.kn, sm.vn, stg);
    // this thread's row sum over its quad (the four threads of head lane / 4)
    st.l += __shfl_xor_sync(0xFFFFFFFFu, st.l, 1);
    st.l += __shfl_xor_sync(0xFFFFFFFFu, st.l, 2);
    csync(p, sm, cph);                                   // every warp is done with its staging page
    // combine the warps' partials (fixed order) into this split's partial
    float* sc = sm.attn;
    {
        const int g4 = lane >> 2, t4 = lane & 3;
        if (g4 < HPG) {
            float* w = sc + ((size_t)warp * HPG + g4) * (HD + 2);
            if (t4 == 0) { w[0] = st.m; w[1] = st.l; }
#pragma unroll
            for (int j = 0; j < AttnMma<HPG, DPL>::NT; ++j) {
                w[2 + 8 * j + 2 * t4] = st.o[j][0] + st.o[j][2];
                w[2 + 8 * j + 2 * t4 + 1] = st.o[j][1] + st.o[j][3];
            }
        }
    }
    csync(p, sm, cph);
    if (sm.flag[3]) { abort_all = true; return; }
    if (valid && attn_active_splits(pos + 1, S) == 1) {
        // the whole context is in split 0: it writes the normalised output itself and
        // no merge follows (the other splits only count their arrival, which nobody
        // waits for; the task's event is signalled by the epilogue warp)
        if (s == 0) {
            float* out = p.attn_o + ((size_t)l * p.max_batch + b) * p.nq * HD + (size_t)g * HPG * HD;
            for (int q = tid; q < HPG * HD / 4; q += kConsumerThreads) {
                const int h = (q * 4) / HD, c = (q * 4) % HD;
                float M = -INFINITY;
#pragma unroll
                for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, sc[((size_t)w * HPG + h) * (HD + 2)]);
                float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
                float L = 0.0f;
                if (M != -INFINITY) {
#pragma unroll
                    for (int w = 0; w < kConsumerWarps; ++w) {
                        const float* ww = sc + ((size_t)w * HPG + h) * (HD + 2);
                        const float f = (ww[0] == -INFINITY) ? 0.0f : exp2f(ww[0] - M);
                        L = fmaf(ww[1], f, L);
                        o.x = fmaf(ww[2 + c], f, o.x);
                        o.y = fmaf(ww[3 + c], f, o.y);
                        o.z = fmaf(ww[4 + c], f, o.z);
                        o.w = fmaf(ww[5 + c], f, o.w);
                    }
                }
                const float inv = (L > 0.0f) ? 1.0f / L : 0.0f;
                const float4 r = make_float4(o.x * inv, o.y * inv, o.z * inv, o.w * inv);
                *reinterpret_cast<float4*>(out + (size_t)h * HD + c) = r;
                if (p.mm) put_operand4(p, kOpAo, l, b, p.nq * HD, g * HPG * HD + h * HD + c, r);
            }
            if (p.mm) fence_proxy_async_global();
        }
        if (tid == 0) atomicAdd(p.attn_cnt + ((size_t)l * p.max_batch + b) * p.nkv + g, 1u);
        return;
    }
    if (valid) {
        for (int idx = tid; idx < HPG * (HD + 2); idx += kConsumerThreads) {
            const int h = idx / (HD + 2), c = idx % (HD + 2);
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, sc[((size_t)w * HPG + h) * (HD + 2)]);
            float val;
            if (c == 0) {
                val = M;
            } else {
                float acc = 0.0f;
                if (M != -INFINITY) {
#pragma unroll
                    for (int w = 0; w < kConsumerWarps; ++w) {
                        const float* ww = sc + ((size_t)w * HPG + h) * (HD + 2);
                        const float f = (ww[0] == -INFINITY) ? 0.0f : exp2f(ww[0] - M);
                        acc = fmaf(ww[c], f, acc);
                    }
                }
                val = acc;
            }
            const size_t pidx = attn_part_index(p, l, b, g, s, h);
            if (c < 2) attn_part_ml(p, pidx)[c] = val;
            else attn_part_o(p, pidx)[c - 2] = val;
        }
    }
    // arrival of this split (active or not); the split that arrives last for its
    // (sequence, kv group) merges the partials once, before its completion is
    // signalled.  The CTA barrier orders every thread's partial stores before thread
    // 0's acquire-release arrival (cumulative), and the second barrier orders its
    // acquire before the merge's loads.
    csync(p, sm, cph);
    if (tid == 0) {
        const uint32_t old = atom_add_acq_rel(p.attn_cnt + ((size_t)l * p.max_batch + b) * p.nkv + g, 1u);
        sm.attn_last = (old == (uint32_t)S * p.epoch - 1u) ? 1 : 0;
    }
    csync(p, sm, cph);
    if (sm.flag[3]) { abort_all = true; return; }
    if (sm.attn_last && active_row) attn_merge_group(p, sm, cph, l, b, g);
}

// ---- wide attention (long contexts, batch 1): one task per split covers every KV
// head.  Warp w serves KV head w / (8 / n_kv); with fewer than 8 KV heads the
// warps of a head take its pages in turn.  Each page arrives as stage-sized blocks
// of all heads' keys, then values (produce_wide_pages).  The split owning the new
// position appends and attends the new token's k and v.  The split writes its
// softmax partial per (KV head, q head); merge tasks combine the splits.

// Row 0 of the warp's staging page from one head's fp32 vector in global memory
// (k: rotated at the position's (cos, sin) pairs; v: as is), rounded to bf16; rows
// 1..15 zero.  With `append`, the bf16 row is also written to the cache slot.
template <int HD>
__device__ __forceinline__ void stage_new_row(const float* src, const float* rope, bool rotate, uint8_t* stg,
                                              uint16_t* append) {
    constexpr int CPR = HD / 8;
    const int lane = threadIdx.x & 31;
    for (int q = lane; q < kPageSize * CPR; q += 32) {
        const int r = q / CPR, c = q % CPR;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (r == 0) {
            float e[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int col = 8 * c + k;
                float x = __ldcg(src + col);
                if (rotate) {
                    const int i = col % (HD / 2);
                    const float2 cs = __ldg(reinterpret_cast<const float2*>(rope) + i);
                    const float other = __ldcg(src + (col < HD / 2 ? col + HD / 2 : col - HD / 2));
                    x = (col < HD / 2) ? x * cs.x - other * cs.y : x * cs.x + other * cs.y;
                }
                e[k] = bf16_to_f32(f32_to_bf16_rne(x));
            }
            v = make_uint4(pack_bf16x2(e[0], e[1]), pack_bf16x2(e[2], e[3]), pack_bf16x2(e[4], e[5]),
                           pack_bf16x2(e[6], e[7]));
            if (append) *reinterpret_cast<uint4*>(append + 8 * c) = v;
        }
        sts128(smem_u32(stg) + stg_off<HD>(r, c), v);
    }
}

template <int HPG, int DPL>
__device__ void attention_wide_task(const Params& p, Smem& sm, uint32_t& cph, const Task& t, int ti, int& stage,
                                    uint32_t& lap, bool& abort_all) {
    constexpr int HD = DPL * 32;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = t.b, s = (int)t.r0, S = (int)t.r1, l = t.layer;
    const int nkv = p.nkv, wph = kConsumerWarps / nkv;
    const int head = warp / wph, sub = warp % wph;
    int pos = position_of(p, b);
    const bool valid = b < p.batch && pos >= 0 && pos < p.max_ctx && pos / kPageSize < p.max_pages;
    if (b < p.batch && !valid && tid == 0) set_error(p, kErrInvalid, ti, -3, pos, b);
    if (!valid) pos = 0;
    int j0 = 0, j1 = 0;
    if (valid) {
        const int sa = attn_active_splits(pos + 1, S);
        if (s < sa) attn_range(pos + 1, sa, s, j0, j1);
    }
    const bool has_new = valid && pos >= j0 && pos < j1;
    const float qscale = 1.4426950408889634f / sqrtf((float)HD);   // log2(e) / sqrt(d)

    AttnMma<HPG, DPL> st;
    st.m = -INFINITY;
    st.l = 0.0f;
#pragma unroll
    for (int j = 0; j < AttnMma<HPG, DPL>::NT; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) st.o[j][e] = 0.0f;
#pragma unroll
    for (int ks = 0; ks < AttnMma<HPG, DPL>::KS; ++ks)
#pragma unroll
        for (int e = 0; e < 4; ++e) st.qa[ks][e] = 0u;
    uint8_t* stg = reinterpret_cast<uint8_t*>(sm.attn) + warp * (kPageSize * HD * 2);   // staging page
    csync(p, sm, cph);                                   // shared scratch of the previous task is free
    const float* qkv = p.qkv + ((size_t)l * p.max_batch + b) * ((p.nq + 2 * p.nkv) * HD);
    const float* rope = p.rope + (size_t)pos * HD;       // [HD/2][2] = cos, sin
    if (valid && j1 > j0) {
        // q of this warp's head group, rotated at pos and pre-scaled, through the
        // staging page (fp32 [HPG][HD]) into the hi/lo A fragments
        float* qf = reinterpret_cast<float*>(stg);
        for (int idx = lane; idx < HPG * (HD / 2); idx += 32) {
            const int h = idx / (HD / 2), i = idx % (HD / 2);
            const float* src = qkv + (size_t)(head * HPG + h) * HD;
            const float x0 = __ldcg(src + i), x1 = __ldcg(src + i + HD / 2);
            const float2 cs = __ldg(reinterpret_cast<const float2*>(rope) + i);
            qf[h * HD + i] = (x0 * cs.x - x1 * cs.y) * qscale;
            qf[h * HD + i + HD / 2] = (x1 * cs.x + x0 * cs.y) * qscale;
        }
        __syncwarp();
        const int g4 = lane >> 2, t4 = lane & 3;
        if (g4 < HPG) {
#pragma unroll
            for (int ks = 0; ks < AttnMma<HPG, DPL>::KS; ++ks) {
                const float* qh = qf + g4 * HD + 16 * ks + 2 * t4;
                split_bf16x2(qh[0], qh[1], st.qa[ks][0], st.qa[ks][1]);
                split_bf16x2(qh[8], qh[9], st.qa[ks][2], st.qa[ks][3]);
            }
        }
        __syncwarp();
        if (has_new && sub == 0) {
            // the new token of this head: k rotated, both rounded to bf16, appended to the
            // cache and attended as a one-token page
            uint16_t* kapp = nullptr;
            uint16_t* vapp = nullptr;
            const int* prow = page_row(p, b);
            const int ph = prow[pos / kPageSize];
            if (ph >= 0 && ph < p.n_pages) {
                const size_t off = ((((size_t)l * p.n_pages + ph) * nkv + head) * kPageSize + pos % kPageSize) * HD;
                kapp = p.k_pages + off;
                vapp = p.v_pages + off;
            } else if (lane == 0) {
                set_error(p, kErrInvalid, ti, -2, pos / kPageSize, b);
            }
            stage_new_row<HD>(qkv + (size_t)(p.nq + head) * HD, rope, true, stg, kapp);
            __syncwarp();
            float s0[4], s1[4];
            attn_qk<HPG, DPL>(st, stg, s0, s1);
            uint32_t pa[4];
            attn_softmax<HPG, DPL>(st, s0, s1, 0, 1, pa);
            __syncwarp();
            stage_new_row<HD>(qkv + (size_t)(p.nq + nkv + head) * HD, rope, false, stg, vapp);
            __syncwarp();
            attn_pv<HPG, DPL>(st, stg, pa);
            __syncwarp();
        }
    }

    // the cached pages: per page spp stages of hps heads (their keys, then values)
    const int jc = min(j1, pos);
    const int blk_elems = kPageSize * HD;
    const int hps = kStageBytes / (blk_elems * 2 * 2), spp = (nkv + hps - 1) / hps;
    const int my_q = head / hps, my_slot = head % hps;
    for (int c = 0;; ++c) {
        if (c == 0) {
            seen_complete_wait(p, &sm.full[stage], lap & 1, &sm.flag[3]);
        } else if (!mbar_wait_bounded(p, &sm.full[stage], lap & 1, 3)) {
            sm.flag[3] = 1;
            break;
        }
        const StageInfo inf = sm.info[stage];
        if (inf.task != ti) {
            set_error(p, kErrFault, ti, -4, inf.task, 1);
            sm.flag[3] = 1;
            break;
        }
        if (inf.nchunks > 0) {
            const int q = inf.chunk % spp;
            const int lp = inf.aux;                          // logical page
            if (q == my_q && (lp % wph) == sub) {
                const int pf = lp * kPageSize;
                const int k_lo = max(j0 - pf, 0), k_hi = min(jc - pf, kPageSize);
                if (k_hi > k_lo) {
                    const int nh = min(hps, nkv - q * hps);
                    const uint16_t* kb = reinterpret_cast<const uint16_t*>(sm.ring[stage]) + (size_t)my_slot * blk_elems;
                    attn_page<HPG, DPL>(st, kb, kb + (size_t)nh * blk_elems, k_lo, k_hi, stg);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty[stage]);
        const bool last = inf.nchunks == 0 || inf.chunk == inf.nchunks - 1;
        if (++stage == kStages) { stage = 0; ++lap; }
        if (last) break;
    }
    st.l += __shfl_xor_sync(0xFFFFFFFFu, st.l, 1);
    st.l += __shfl_xor_sync(0xFFFFFFFFu, st.l, 2);
    csync(p, sm, cph);                                   // every warp is done with its staging page
    float* sc = sm.attn;                                 // [warp][HPG][m, l, o]
    {
        const int g4 = lane >> 2, t4 = lane & 3;
        if (g4 < HPG) {
            float* w = sc + ((size_t)warp * HPG + g4) * (HD + 2);
            if (t4 == 0) { w[0] = st.m; w[1] = st.l; }
#pragma unroll
            for (int j = 0; j < AttnMma<HPG, DPL>::NT; ++j) {
                w[2 + 8 * j + 2 * t4] = st.o[j][0] + st.o[j][2];
                w[2 + 8 * j + 2 * t4 + 1] = st.o[j][1] + st.o[j][3];
            }
        }
    }
    csync(p, sm, cph);
    if (sm.flag[3]) { abort_all = true; return; }
    if (!valid) return;
    // this split's partial per (KV head, q head): the head's warps combined in order
    for (int idx = tid; idx < nkv * HPG * (HD + 2); idx += kConsumerThreads) {
        const int g = idx / (HPG * (HD + 2)), r = idx % (HPG * (HD + 2)), h = r / (HD + 2), c = r % (HD + 2);
        float M = -INFINITY;
        for (int u = 0; u < wph; ++u) M = fmaxf(M, sc[((size_t)(g * wph + u) * HPG + h) * (HD + 2)]);
        float val;
        if (c == 0) {
            val = M;
        } else {
            float acc = 0.0f;
            if (M != -INFINITY)
                for (int u = 0; u < wph; ++u) {
                    const float* ww = sc + ((size_t)(g * wph + u) * HPG + h) * (HD + 2);
                    const float f = (ww[0] == -INFINITY) ? 0.0f : exp2f(ww[0] - M);
                    acc = fmaf(ww[c], f, acc);
                }
            val = acc;
        }
        const size_t pidx = attn_part_index(p, l, b, g, s, h);
        if (c < 2) attn_part_ml(p, pidx)[c] = val;
        else attn_part_o(p, pidx)[c - 2] = val;
    }
}

// Merge task of wide attention: q head t.r0 of sequence t.b, the active splits'
// partials combined (m* = max m_s; o = sum 2^(m_s - m*) o_s / sum 2^(m_s - m*) l_s),
// normalised and stored.  Warp 0 forms the weights; then thread (j, c4) sums splits
// j, j + 8, ... over four columns, and the eight partial sums are added in order.
__device__ void attn_merge_head(const Params& p, Smem& sm, uint32_t& cph, const Task& t, int ti) {
    const int tid = threadIdx.x, lane = tid & 31, hd = p.hd, hpg = hpg_of(p);
    const int b = t.b, l = t.layer, qh = (int)t.r0, g = qh / hpg, h = qh % hpg;
    int pos = (b < p.batch) ? position_of(p, b) : -1;
    if (pos < 0 || pos >= p.max_ctx) return;             // (the attention task reported it)
    const int sa = attn_active_splits(pos + 1, p.S);
    float* f = sm.attn;                                  // [sa] weights, [sa] l, then [8][hd] sums
    float* fl = f + sa;
    float* part = f + ((2 * sa + 3) & ~3);               // 16-byte aligned (float4 stores)
    csync(p, sm, cph);                                   // the scratch of the previous task is free
    for (int k = tid; k < sa; k += kConsumerThreads) {
        const float2 ml = __ldcg(reinterpret_cast<const float2*>(attn_part_ml(p, attn_part_index(p, l, b, g, k, h))));
        f[k] = ml.x;
        fl[k] = ml.y;
    }
    csync(p, sm, cph);
    if (tid < 32) {
        float M = -INFINITY;
        for (int k = lane; k < sa; k += 32) M = fmaxf(M, f[k]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xFFFFFFFFu, M, o));
        float L = 0.0f;
        for (int k = lane; k < sa; k += 32) {
            const float w = (f[k] == -INFINITY) ? 0.0f : exp2f(f[k] - M);
            f[k] = w;
            L = fmaf(fl[k], w, L);
        }
        L = warp_sum(L);
        if (lane == 0) fl[0] = (L > 0.0f) ? 1.0f / L : 0.0f;   // (fl is no longer needed)
    }
    csync(p, sm, cph);
    const int j = tid >> 5, c4 = lane;
    if (4 * c4 < hd) {
        float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
        for (int k = j; k < sa; k += kConsumerWarps) {
            const float w = f[k];
            const float4 v = __ldcg(reinterpret_cast<const float4*>(attn_part_o(p, attn_part_index(p, l, b, g, k, h)) + 4 * c4));
            o.x = fmaf(v.x, w, o.x); o.y = fmaf(v.y, w, o.y); o.z = fmaf(v.z, w, o.z); o.w = fmaf(v.w, w, o.w);
        }
        *reinterpret_cast<float4*>(part + (size_t)j * hd + 4 * c4) = o;
    }
    const float inv = fl[0];
    csync(p, sm, cph);
    if (tid < hd / 4) {
        float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int jj = 0; jj < kConsumerWarps; ++jj) {
            const float4 v = *reinterpret_cast<const float4*>(part + (size_t)jj * hd + 4 * tid);
            o.x += v.x; o.y += v.y; o.z += v.z; o.w += v.w;
        }
        float* out = p.attn_o + ((size_t)l * p.max_batch + b) * p.nq * hd + (size_t)qh * hd;
        *reinterpret_cast<float4*>(out + 4 * tid) = make_float4(o.x * inv, o.y * inv, o.z * inv, o.w * inv);
    }
    (void)ti;
}

// ----------------------------------------------------------------------------- consumer: router top-k

// Last router tile of a layer: softmax over the experts, top-k (ties to the
// lower index), optional renormalisation.  One warp (the caller) does the work.
__device__ void router_finalize(const Params& p, Smem& sm, int l) {
    const int lane = threadIdx.x & 31;
    for (int b = 0; b < p.max_batch; ++b) {
        const float* lg = p.rlogits + ((size_t)l * p.max_batch + b) * p.E;
        float mx = -INFINITY;
        for (int e = lane; e < p.E; e += 32) {
            float v = __ldcg(lg + e);
            sm.rlog[e] = v;
            mx = fmaxf(mx, v);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
        float sum = 0.0f;
        for (int e = lane; e < p.E; e += 32) {
            float v = expf(sm.rlog[e] - mx);
            sm.rlog[e] = v;
            sum += v;
        }
        sum = warp_sum(sum);
        __syncwarp();
        float selw[kMaxTopK];
        int sel[kMaxTopK];
        float wsum = 0.0f;
        for (int k = 0; k < p.topk; ++k) {
            float best = -1.0f;
            int bi = 0x7FFFFFFF;
            for (int e = lane; e < p.E; e += 32) {
                float v = sm.rlog[e];
                if (v > best || (v == best && e < bi)) { best = v; bi = e; }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                float ob = __shfl_xor_sync(0xFFFFFFFFu, best, o);
                int oi = __shfl_xor_sync(0xFFFFFFFFu, bi, o);
                if (ob > best || (ob == best && oi < bi)) { best = ob; bi = oi; }
            }
            sel[k] = bi;
            selw[k] = best / sum;
            wsum += selw[k];
            __syncwarp();
            if (lane == 0) sm.rlog[bi] = -2.0f;   // taken (probabilities are >= 0)
            __syncwarp();
        }
        if (lane == 0) {
            for (int k = 0; k < p.topk; ++k) {
                size_t o = ((size_t)l * p.max_batch + b) * p.topk + k;
                p.moe_sel[o] = sel[k];
                p.moe_w[o] = p.renorm ? selw[k] / wsum : selw[k];
            }
        }
        __syncwarp();
    }
}

// A batch-1 LM-head tile's part of the in-step argmax: the (max, index) of the
// logits rows it has just stored (this warp's own stores, read back).  One warp.
__device__ __forceinline__ void lmhead_arg_part(const Params& p, const Task& t, int lane) {
    __syncwarp();
    float v = -INFINITY;
    int i = 0x7FFFFFFF;
    for (int r = (int)t.r0 + lane; r < (int)t.r1; r += 32) arg_better(v, i, p.logits[r], r);
    warp_argmax(v, i);
    if (lane == 0) p.lm_arg[(size_t)t.aux * kArgParts * p.max_batch] = ArgVal{v, i};
}

// Greedy argmax inside the step (mk_generate).  An LM-head tile has stored the
// (value, index) of its rows' maximum for every batch row (nparts parts per
// tile); it arrives on its group of kArgGroup tiles, the group's last tile
// reduces the group, and the last group writes each batch row's token to
// argmax_out.  Ties go to the lower index at every level, so the result is the
// first index of the largest logit whatever the arrival order.  One warp.
__device__ __forceinline__ void argmax_arrive(const Params& p, int tile, int nparts, int lane) {
    const int ng = (p.n_lm_tiles + kArgGroup - 1) / kArgGroup;
    const int g = tile / kArgGroup, t0 = g * kArgGroup, t1 = min(p.n_lm_tiles, t0 + kArgGroup);
    __syncwarp();
    int last = 0;
    if (lane == 0) {
        const uint32_t old = atom_add_acq_rel(p.lm_cnt + g, 1u);
        last = (old == (uint32_t)(t1 - t0) * p.arg_epoch - 1u) ? 1 : 0;
    }
    last = __shfl_sync(0xFFFFFFFFu, last, 0);
    if (!last) return;
    __syncwarp();
    for (int b = 0; b < p.batch; ++b) {
        float v = -INFINITY;
        int i = 0x7FFFFFFF;
        for (int k = lane; k < (t1 - t0) * nparts; k += 32) {
            const float2 a = __ldcg(reinterpret_cast<const float2*>(
                p.lm_arg + ((size_t)(t0 + k / nparts) * kArgParts + k % nparts) * p.max_batch + b));
            arg_better(v, i, a.x, __float_as_int(a.y));
        }
        warp_argmax(v, i);
        if (lane == 0) p.lm_garg[(size_t)g * p.max_batch + b] = ArgVal{v, i};
    }
    __syncwarp();
    if (lane == 0) {
        const uint32_t old = atom_add_acq_rel(p.lm_cnt + ng, 1u);
        last = (old == (uint32_t)ng * p.arg_epoch - 1u) ? 1 : 0;
    }
    last = __shfl_sync(0xFFFFFFFFu, last, 0);
    if (!last) return;
    __syncwarp();
    for (int b = 0; b < p.batch; ++b) {
        float v = -INFINITY;
        int i = 0x7FFFFFFF;
        for (int k = lane; k < ng; k += 32) {
            const float2 a = __ldcg(reinterpret_cast<const float2*>(p.lm_garg + (size_t)k * p.max_batch + b));
            arg_better(v, i, a.x, __float_as_int(a.y));
        }
        warp_argmax(v, i);
        if (lane == 0) p.argmax_out[b] = (i == 0x7FFFFFFF) ? 0 : i;
    }
}

// ----------------------------------------------------------------------------- consumer loop

// ----------------------------------------------------------------------------- batched tiles

// K (rotated at the row's position with the RoPE table, as the attention tile
// rotates it) and V of batch rows [r0, r1) of layer l, rounded to bf16 (RNE),
// into their pages.  Batched graphs run this before the layer's attention, which
// then reads every position from the cache: under batched prefill, a prompt row
// attends to the rows before it.
__device__ __noinline__ void kvappend_task(const Params& p, const Task& t, int ti) {
    const int HD = p.hd, half = HD / 2, tid = threadIdx.x, l = t.layer;
    for (int b = (int)t.r0; b < (int)t.r1; ++b) {
        if (b >= p.batch) continue;
        const int pos = position_of(p, b);
        if (pos < 0 || pos >= p.max_ctx || pos / kPageSize >= p.max_pages) {
            if (tid == 0) set_error(p, kErrInvalid, ti, -3, pos, b);
            continue;
        }
        const int ph = page_row(p, b)[pos / kPageSize];
        if (ph < 0 || ph >= p.n_pages) {
            if (tid == 0) set_error(p, kErrInvalid, ti, -2, pos / kPageSize, b);
            continue;
        }
        const float* qkv = p.qkv + ((size_t)l * p.max_batch + b) * ((p.nq + 2 * p.nkv) * HD);
        const float2* rope = reinterpret_cast<const float2*>(p.rope + (size_t)pos * HD);   // [HD/2] (cos, sin)
        const size_t base = (((size_t)l * p.n_pages + ph) * p.nkv) * kPageSize;
        for (int idx = tid; idx < p.nkv * half; idx += kConsumerThreads) {
            const int g = idx / half, i = idx % half;
            const float* k = qkv + (size_t)(p.nq + g) * HD;
            const float x0 = __ldcg(k + i), x1 = __ldcg(k + i + half);
            const float2 r = __ldg(rope + i);
            const size_t off = ((base + (size_t)g * kPageSize) + pos % kPageSize) * HD;
            p.k_pages[off + i] = f32_to_bf16_rne(x0 * r.x - x1 * r.y);
            p.k_pages[off + i + half] = f32_to_bf16_rne(x1 * r.x + x0 * r.y);
        }
        for (int idx = tid; idx < p.nkv * HD; idx += kConsumerThreads) {
            const int g = idx / HD, i = idx % HD;
            const size_t off = ((base + (size_t)g * kPageSize) + pos % kPageSize) * HD;
            p.v_pages[off + i] = f32_to_bf16_rne(__ldcg(qkv + (size_t)(p.nq + p.nkv + g) * HD + i));
        }
    }
}

// Tensor-parallel reduction of rows [r0, r1) of the residual stream (aux 0: after
// attention, into x_mid; aux 1: after the FFN, into x_out): once every rank has
// pushed its partial sums of these rows (the tile's arrival flag in this rank's
// memory reaches tp per step), the parts are added in rank order and the residual
// last -- every rank computes the same sums in the same order, so the replicated
// residual stream stays bit-identical across ranks.  The reads go around L1: the
// receive buffer is written by other GPUs.
__device__ __noinline__ void tp_reduce_task(const Params& p, Smem& sm, uint32_t& cph, const Task& t, int ti) {
    const int tid = threadIdx.x, l = t.layer, ph = t.aux;
    if (tid == 0) {
        const uint32_t* f = p.tp_flag[p.tp_rank] + ((size_t)l * 2 + ph) * p.tp_tiles + t.pad;
        if (!tp_flag_wait(p, f, (uint32_t)p.tp * p.epoch + p.wait_offset, ti)) sm.flag[3] = 1;
    }
    // thread 0's acquire, then the consumers' barrier, before any thread reads the parts
    csync(p, sm, cph);
    if (sm.flag[3]) return;
    const float* recv = p.tp_recv[p.tp_rank];
    for (int r = (int)t.r0 + tid; r < (int)t.r1; r += kConsumerThreads) {
        float y = 0.0f;
        for (int q = 0; q < p.tp; ++q) y += __ldcg(recv + (((size_t)q * p.L + l) * 2 + ph) * p.H + r);
        if (ph == 0) p.x_mid[((size_t)l * p.max_batch) * p.H + r] = x_in(p, l, 0, r) + y;
        else p.x_out[((size_t)l * p.max_batch) * p.H + r] = x_mid_at(p, l, 0, r) + y;
    }
}

// RMSNorm of one batch row into the operand of the next projection, by all 256
// consumer threads: h = x / sqrt(mean(x^2) + eps) * g (kind 0: attention norm of
// the residual entering layer l, the token embedding at l = 0; kind 1: FFN norm
// of the residual after attention; kind 2: final norm).  Two passes over the row
// (sum of squares, then scale and store, re-reading x with the gains) around one
// block-wide sum.  Rows past the step's batch are written as zeros.
constexpr int kNormCols = 4 * kConsumerThreads;   // columns per pass chunk: 4 per thread
template <bool EMB>
__device__ __forceinline__ float4 norm_load4(const float* src, const uint16_t* emb, int i) {
    if constexpr (EMB) {
        const uint2 u = __ldg(reinterpret_cast<const uint2*>(emb + i));
        return make_float4(bf_lo(u.x), bf_hi(u.x), bf_lo(u.y), bf_hi(u.y));
    } else {
        return __ldcg(reinterpret_cast<const float4*>(src + i));
    }
}
// Each thread owns 4 consecutive columns of every 1024-column chunk; the sum of
// squares pass, a block-wide sum, then the scaling pass re-reads x with the gains.
template <bool EMB>
__device__ void norm_row(const Params& p, Smem& sm, uint32_t& cph, const float* src, const uint16_t* emb,
                         const uint16_t* gain, int op, int olayer, int b) {
    const int H = p.H, c0 = threadIdx.x * 4;
    float ss = 0.0f;
    for (int i = c0; i < H; i += kNormCols) {
        const float4 v = norm_load4<EMB>(src, emb, i);
        ss = fmaf(v.w, v.w, fmaf(v.z, v.z, fmaf(v.y, v.y, fmaf(v.x, v.x, ss))));
    }
    const float tot = block_sum(p, sm, cph, ss);
    const float rstd = 1.0f / sqrtf(tot / (float)H + p.eps);
    for (int i = c0; i < H; i += kNormCols) {
        const float4 v = norm_load4<EMB>(src, emb, i);
        const uint2 g = __ldg(reinterpret_cast<const uint2*>(gain + i));
        put_operand4(p, op, olayer, b, H, i,
                     make_float4((v.x * rstd) * bf_lo(g.x), (v.y * rstd) * bf_hi(g.x),
                                 (v.z * rstd) * bf_lo(g.y), (v.w * rstd) * bf_hi(g.y)));
    }
}
// (Out of line, like the tensor-core tile below: the batched tasks keep their
// registers out of the batch-1 consumer loop's allocation.)
__device__ __noinline__ void norm_task(const Params& p, Smem& sm, uint32_t& cph, const Task& t, int ti) {
    const int kind = t.aux, l = t.layer, H = p.H, tid = threadIdx.x;
    const int op = (kind == 0) ? kOpXq : (kind == 1) ? kOpXf : kOpXl;
    const int olayer = (kind == 2) ? 0 : l;
    const uint16_t* gain = (kind == 0) ? p.layers[l].attn_norm : (kind == 1) ? p.layers[l].ffn_norm : p.final_norm;
    for (int b = (int)t.r0; b < (int)t.r1; ++b) {
        if (b >= p.batch) {
            for (int i = tid * 4; i < H; i += kConsumerThreads * 4)
                put_operand4(p, op, olayer, b, H, i, make_float4(0.f, 0.f, 0.f, 0.f));
        } else if (kind == 0 && l == 0) {
            int tok = p.tokens[b];
            if (tok < 0 || tok >= p.V) {
                if (tid == 0) set_error(p, kErrInvalid, ti, -5, tok, b);
                tok = 0;
            }
            norm_row<true>(p, sm, cph, nullptr, p.tok_emb + (size_t)tok * H, gain, op, olayer, b);
        } else if (kind == 1) {
            norm_row<false>(p, sm, cph, p.x_mid + ((size_t)l * p.max_batch + b) * H, nullptr, gain, op, olayer, b);
        } else {   // kind 0 at l > 0, or kind 2 (l = L): the residual after layer l - 1
            norm_row<false>(p, sm, cph, p.x_out + ((size_t)(l - 1) * p.max_batch + b) * H, nullptr, gain, op,
                            olayer, b);
        }
    }
}

// The last split of a tile: the splits' partial sums added in split order (the
// same order on every run), then the operator's epilogue for every batch row of
// the step.  128 threads (consumer warps 4-7), each owning one tile row (gate/up:
// one FFN row and half of the batch rows).  The loads of 8 batch rows are issued
// before any of their stores, so a tile costs batch / 8 round trips to L2, not one
// per batch row.
constexpr int kEpiRows = 8;
__device__ __noinline__ void mm_epilogue(const Params& p, const Task& t, int tid) {
    const int Sk = t.nblk, l = t.layer, nrows = (int)(t.r1 - t.r0), batch = p.batch;
    const size_t sstride = (size_t)p.bp * kMmRows;
    const float* __restrict__ part0 = p.mm_part + (size_t)t.aux * sstride;
    if (t.op == MK_OP_MM_GATEUP) {            // rows 0..63 gate, 64..127 up, of FFN rows r0..r0+63
        const int i = tid & 63;
        if (i >= nrows) return;
        const int f = (int)t.r0 + i;
        const size_t base = (size_t)l * 2 * p.bp;
        for (int b0 = tid >> 6; b0 < batch; b0 += 2 * kEpiRows) {
            float g[kEpiRows], u[kEpiRows];
#pragma unroll
            for (int k = 0; k < kEpiRows; ++k) { g[k] = 0.0f; u[k] = 0.0f; }
            for (int sp = 0; sp < Sk; ++sp) {
                const float* ps = part0 + sp * sstride;
#pragma unroll
                for (int k = 0; k < kEpiRows; ++k) {
                    const int b = b0 + 2 * k;
                    if (b < batch) {
                        g[k] += __ldcg(ps + (size_t)b * kMmRows + i);
                        u[k] += __ldcg(ps + (size_t)b * kMmRows + 64 + i);
                    }
                }
            }
#pragma unroll
            for (int k = 0; k < kEpiRows; ++k) {
                const int b = b0 + 2 * k;
                if (b >= batch) continue;
                const float a = silu_f(g[k]) * u[k];
                p.act[((size_t)l * p.max_batch + b) * p.F + f] = a;
                uint16_t hi, lo;
                split_hilo(a, hi, lo);
                p.opnd[kOpAct][(base + b) * p.F + f] = hi;
                p.opnd[kOpAct][(base + p.bp + b) * p.F + f] = lo;
            }
        }
        return;
    }
    if (t.op == MK_OP_MM_LMHEAD) {
        // logits, and with the in-step argmax each warp's (max, index) per batch row
        // (every lane takes part in the shuffles: rows past the tile count as -inf)
        const int i = tid, w = tid >> 5, lane = tid & 31;
        const bool row_ok = i < nrows;
        const int r = (int)t.r0 + i;
        for (int b0 = 0; b0 < batch; b0 += kEpiRows) {
            float v[kEpiRows];
#pragma unroll
            for (int k = 0; k < kEpiRows; ++k) v[k] = 0.0f;
            if (row_ok)
                for (int sp = 0; sp < Sk; ++sp) {
                    const float* ps = part0 + sp * sstride;
#pragma unroll
                    for (int k = 0; k < kEpiRows; ++k)
                        if (b0 + k < batch) v[k] += __ldcg(ps + (size_t)(b0 + k) * kMmRows + i);
                }
#pragma unroll
            for (int k = 0; k < kEpiRows; ++k) {
                const int b = b0 + k;
                if (b >= batch) break;
                if (row_ok) p.logits[(size_t)b * p.V + r] = v[k];
                if (p.argmax_out) {
                    float bv = row_ok ? v[k] : -INFINITY;
                    int bi = row_ok ? r : 0x7FFFFFFF;
                    warp_argmax(bv, bi);
                    if (lane == 0)
                        p.lm_arg[((size_t)t.b * kArgParts + w) * p.max_batch + b] = ArgVal{bv, bi};
                }
            }
        }
        return;
    }
    const int i = tid;
    if (i >= nrows) return;
    const int r = (int)t.r0 + i;
    const size_t qkvw = (size_t)(p.nq + 2 * p.nkv) * p.hd;
    for (int b0 = 0; b0 < batch; b0 += kEpiRows) {
        float v[kEpiRows], res[kEpiRows];
#pragma unroll
        for (int k = 0; k < kEpiRows; ++k) { v[k] = 0.0f; res[k] = 0.0f; }
        for (int sp = 0; sp < Sk; ++sp) {
            const float* ps = part0 + sp * sstride;
#pragma unroll
            for (int k = 0; k < kEpiRows; ++k)
                if (b0 + k < batch) v[k] += __ldcg(ps + (size_t)(b0 + k) * kMmRows + i);
        }
        if (t.op == MK_OP_MM_OPROJ || t.op == MK_OP_MM_DOWN) {
#pragma unroll
            for (int k = 0; k < kEpiRows; ++k)
                if (b0 + k < batch)
                    res[k] = (t.op == MK_OP_MM_OPROJ) ? x_in(p, l, b0 + k, r) : x_mid_at(p, l, b0 + k, r);
        }
#pragma unroll
        for (int k = 0; k < kEpiRows; ++k) {
            const int b = b0 + k;
            if (b >= batch) continue;
            const size_t lb = (size_t)l * p.max_batch + b;
            switch (t.op) {
                case MK_OP_MM_QKV: p.qkv[lb * qkvw + r] = v[k]; break;
                case MK_OP_MM_OPROJ: p.x_mid[lb * p.H + r] = res[k] + v[k]; break;
                case MK_OP_MM_DOWN: p.x_out[lb * p.H + r] = res[k] + v[k]; break;
                case MK_OP_MM_LMHEAD: p.logits[(size_t)b * p.V + r] = v[k]; break;
                default: break;
            }
        }
    }
}

// Tensor-core tile (one K-split of 128 weight rows x bp batch columns).
//  * Every consumer warp waits for every stage of the tile and warps 1-7 release
//    it at once; one lane of warp 0 issues the MMAs of each weight box as it lands
//    (the group's activation stage came first) and adds the eighth arrival with a
//    tcgen05.commit, once the MMAs have read the stage.  (Every warp walks every
//    stage so that no warp can run a lap ahead of the producer on a stage's
//    barrier, where a parity wait could not tell two phases apart.)
//  * The accumulator is double-buffered in TMEM: tile k of this CTA uses buffer
//    k & 1, so warp 0 multiplies tile k + 1 while warps 4-7 (warp w owns TMEM lane
//    quarter w - 4, i.e. tile rows 32 (w - 4) ..) read tile k, store this split's
//    partial sums, and the last split of the tile to arrive reduces and finishes it.
__device__ __noinline__ bool mm_task(const Params& p, Smem& sm, const Task& t, int ti, int& stage, uint32_t& lap,
                        uint32_t& mm_seq, uint32_t& mph, int buf) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nch = (int)t.nchunks;
    const uint32_t abuf = mm_seq & 1u, use = mm_seq >> 1;   // accumulator buffer and its use count
    ++mm_seq;
    const uint32_t acc = sm.tmem_base + abuf * (uint32_t)(2 * p.bp);
    if (warp != 0) {
        for (int c = 0; c < nch; ++c) {
            if (c > 0 && !mbar_wait_bounded(p, &sm.full[stage], lap & 1, 10)) {
                sm.flag[3] = 1;
                return false;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.empty[stage]);
            if (++stage == kStages) { stage = 0; ++lap; }
        }
    } else {
        // one MMA per 16 columns of K multiplies the weight rows by the hi AND lo rows
        // of the activations (N = 2 bp: its cost does not depend on N); the two halves
        // of the accumulator are added when it is read
        const uint32_t idesc = mm_idesc(2 * p.bp);
        const uint32_t xbytes = 2u * (uint32_t)p.bp * 128u;
        const int kx = mm_kblocks_per_xstage(p.bp);
        int kb_left = (int)t.pad2 - (int)t.row_bytes;   // K-blocks not yet multiplied
        int gs = min(kx, kb_left), gk = -1;              // group size; -1: its activation stage is next
        int xst = stage;
        bool first_mma = true;
        for (int c = 0; c < nch; ++c) {
            if (c > 0 && !mbar_wait_bounded(p, &sm.full[stage], lap & 1, 10)) {
                sm.flag[3] = 1;
                return false;
            }
            if (sm.info[stage].task != ti) {
                set_error(p, kErrFault, ti, -4, sm.info[stage].task, 3);
                sm.flag[3] = 1;
                return false;
            }
            if (gk < 0) {
                xst = stage;
                gk = 0;
            } else {
                if (lane == 0) {
                    if (first_mma && use > 0 && !mbar_wait_bounded(p, &sm.mm_free[abuf], (use - 1) & 1, 14))
                        sm.flag[3] = 1;
                    tc_fence_after();
                    const uint32_t a = smem_u32(sm.ring[stage]);
                    const uint32_t x = smem_u32(sm.ring[xst]) + (uint32_t)gk * xbytes;
#pragma unroll
                    for (int kk = 0; kk < kMmK / 16; ++kk) {
                        tc_mma_bf16(acc, sw128_desc(a + kk * 32), sw128_desc(x + kk * 32), idesc,
                                    first_mma ? 0u : 1u);
                        first_mma = false;
                    }
                    tc_commit(&sm.empty[stage]);
                    if (gk == gs - 1) tc_commit(&sm.empty[xst]);
                    if (c == nch - 1) tc_commit(&sm.mm_acc[abuf]);
                }
                __syncwarp();
                if (sm.flag[3]) return false;
                if (++gk == gs) {
                    kb_left -= gs;
                    gs = min(kx, kb_left);
                    gk = -1;
                }
            }
            if (++stage == kStages) { stage = 0; ++lap; }
        }
    }
    if (warp < 4) return true;
    // ---- warps 4-7: read the accumulator, store this split's partial sums
    const int q = warp - 4, row = q * 32 + lane, etid = tid - 4 * 32;
    if (!mbar_wait_bounded(p, &sm.mm_acc[abuf], use & 1, 11)) {
        sm.flag[3] = 1;
        return false;
    }
    tc_fence_after();
    float* part = p.mm_part + ((size_t)t.aux + t.chunk_rows) * p.bp * kMmRows;
    const uint32_t lane_base = acc + ((uint32_t)(q * 32) << 16);
    for (int c0 = 0; c0 < p.bp; c0 += 16) {
        uint32_t h[16], lo[16];
        tmem_ld16(lane_base + (uint32_t)c0, h);                 // W . x_hi
        tmem_ld16(lane_base + (uint32_t)(p.bp + c0), lo);       // W . x_lo
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j)
            part[(size_t)(c0 + j) * kMmRows + row] = __uint_as_float(h[j]) + __uint_as_float(lo[j]);
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.mm_free[abuf]);        // the buffer may take the next tile
    __threadfence();
    if (!msync4(p, sm, mph)) return false;                // every partial of this split stored
    if (etid == 0) {
        const uint32_t old = atomicAdd(p.mm_cnt + t.pad, 1u);
        sm.mm_last = (old + 1u == (uint32_t)t.nblk * p.epoch) ? 1 : 0;
    }
    if (!msync4(p, sm, mph)) return false;
    const bool last = sm.mm_last != 0;
    if (last) {
        __threadfence();
        mm_epilogue(p, t, etid);
        fence_proxy_async_global();
        __threadfence();
        if (t.op == MK_OP_MM_LMHEAD && p.argmax_out) {
            if (!msync4(p, sm, mph)) return false;       // the four warps' parts are stored
            if (etid < 32) argmax_arrive(p, t.b, kArgParts, lane);
        }
    }
    if (etid == 0) sm.ep_task[buf].sig = last ? t.sig : MK_NO_EVENT;
    return true;
}

// MM: the instantiation for batched graphs (norm tasks, tensor-core tiles,
// attention); the batch-1 instantiation holds the GEMV tiles and none of that.
template <int HPG, int DPL, bool MM, bool WIDE>
__device__ __forceinline__ void consumer_loop(const Params& p, Smem& sm) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int stage = 0;
    uint32_t lap = 0;
    uint32_t seq = 0;                                   // tasks started by this CTA (same in every warp)
    uint32_t cph = 0;                                   // phase of sm.csync
    float2 xr[kMaxVecPerThread][4];
    int x_key_op = -1, x_key_layer = -1, x_key_b = -1, x_key_aux = -1;
    uint32_t ok_evt[4] = {MK_NO_EVENT, MK_NO_EVENT, MK_NO_EVENT, MK_NO_EVENT};   // per warp
    uint32_t mm_seq = 0;                                // tensor-core tiles started by this CTA
    uint32_t mph = 0;                                   // phase of sm.mm_sync (warps 4-7)
    const uint32_t tmem_cols = (uint32_t)(4 * p.bp);     // 64, 128 or 256: two buffers of hi and lo halves
    if constexpr (MM) {
        // the accumulators of the batched tiles: 128 lanes x 2 x 2 bp fp32 columns of TMEM
        if (warp == 0) {
            tmem_alloc(&sm.tmem_base, tmem_cols);
            tmem_relinquish();
        }
        tc_fence_before();
        csync(p, sm, cph);
        tc_fence_after();
    }

    // Each warp waits for its own data and dependencies, runs its share of the task,
    // leaves its partial row sums in red[buf] and arrives on red_full[buf]; the
    // epilogue warp reduces, stores and signals, so no consumer warp ever waits for
    // a task's tail.  Warps meet only inside prologues and attention tasks (bounded
    // mbarrier syncs).  A failure raises sm.flag[3]; every warp checks it before
    // its next task.
    while (true) {
        if (sm.flag[3]) break;
        bool ok = mbar_wait_bounded(p, &sm.full[stage], lap & 1, 4);
        const int ti = ok ? sm.info[stage].task : -2;
        if (ti == -1) {                                  // end of work (same stage for every warp)
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.empty[stage]);
            break;
        }
        if (!ok) { sm.flag[3] = 1; break; }
        const Task t = sm.info[stage].rec;
        if (p.trace && tid == 0) p.trace[(size_t)ti * 4 + 0] = globaltimer();
        const uint32_t e = t.wait0;
        if (e != MK_NO_EVENT && e != ok_evt[0] && e != ok_evt[1] && e != ok_evt[2] && e != ok_evt[3]) {
            int r = 1;
            if (lane == 0) {
                if (warp == 0) *reinterpret_cast<volatile int*>(&sm.pf_wait) = 1;   // the prefetcher may run
                r = event_wait(p, e, p.thr[e] * p.epoch + p.wait_offset, ti) ? 1 : 0;
                if (warp == 0) *reinterpret_cast<volatile int*>(&sm.pf_wait) = 0;
            }
            // lane 0's acquire, then the warp barrier (which orders memory among its
            // lanes), before any lane reads what the event's producers wrote
            r = __shfl_sync(0xFFFFFFFFu, r, 0);
            __syncwarp();
            if (!r) { sm.flag[3] = 1; break; }
            ok_evt[3] = ok_evt[2]; ok_evt[2] = ok_evt[1]; ok_evt[1] = ok_evt[0]; ok_evt[0] = e;
        }
        if (tid == 0) *reinterpret_cast<volatile int*>(&sm.started) = ti;   // the producer may claim on
        if (p.trace && tid == 0) {
            p.trace[(size_t)ti * 4 + 1] = globaltimer();
            p.trace[(size_t)ti * 4 + 3] = (uint64_t)(blockIdx.x - p.cta0);
        }
        const int buf = (int)(seq % kRedBufs);
        // buffer set `buf` is reused once the epilogue warp has finished the task that
        // used it kRedBufs tasks ago
        if (seq >= (uint32_t)kRedBufs &&
            !mbar_wait_bounded(p, &sm.red_free[buf], ((seq / kRedBufs) - 1) & 1, 9)) {
            sm.flag[3] = 1;
            break;
        }
        if (tid == 0) {
            sm.ep_task[buf] = t;
            sm.ep_ti[buf] = ti;
        }

        if constexpr (MM) {
        if (t.op == MK_OP_NORM || t.op == MK_OP_KVAPPEND) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.empty[stage]);     // the marker stage
            if (++stage == kStages) { stage = 0; ++lap; }
            if (t.op == MK_OP_NORM) norm_task(p, sm, cph, t, ti);
            else kvappend_task(p, t, ti);
            fence_proxy_async_global();
            __threadfence();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.red_full[buf]);
            ++seq;
            continue;
        }
        if (is_mm_op(t.op)) {
            if (!mm_task(p, sm, t, ti, stage, lap, mm_seq, mph, buf)) break;
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.red_full[buf]);
            ++seq;
            continue;
        }
        }
        if constexpr (WIDE) {
        if (t.op == MK_OP_ATTN_MERGE) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.empty[stage]);     // the marker stage
            if (++stage == kStages) { stage = 0; ++lap; }
            attn_merge_head(p, sm, cph, t, ti);
            if (sm.flag[3]) break;
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.red_full[buf]);
            ++seq;
            continue;
        }
        }
        if constexpr (!MM && !WIDE) {
        if (t.op == MK_OP_TP_REDUCE) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.empty[stage]);     // the marker stage
            if (++stage == kStages) { stage = 0; ++lap; }
            tp_reduce_task(p, sm, cph, t, ti);
            if (sm.flag[3]) break;
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.red_full[buf]);
            ++seq;
            continue;
        }
        }
        if (t.op == MK_OP_ATTN) {
            bool abort_all = false;
            if (WIDE && (t.flags & kAttnWide)) attention_wide_task<HPG, DPL>(p, sm, cph, t, ti, stage, lap, abort_all);
            else attention_task<HPG, DPL, MM>(p, sm, cph, t, ti, stage, lap, abort_all);
            if (abort_all) break;
            x_key_op = -1;
            // the input slice in registers is dead across an attention task (saves registers)
#pragma unroll
            for (int j = 0; j < kMaxVecPerThread; ++j)
#pragma unroll
                for (int q = 0; q < 4; ++q) xr[j][q] = make_float2(0.0f, 0.0f);
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.red_full[buf]);
            ++seq;
            continue;
        }

        if constexpr (MM) {
            // a batched graph holds no GEMV tiles
            set_error(p, kErrFault, ti, -10, t.op, 0);
            sm.flag[3] = 1;
            break;
        } else {
        // ---- GEMV task
        const bool skip = (t.op == MK_OP_LMHEAD && p.skip_lm);
        const bool fast = (t.flags != kFastNone) && !skip;
        GemvGeom g;
        gemv_geom(p, t, g, false);
        // fast-path tiles split every row over all 8 warps (wpg = 8, one group)
        ThreadMap m;
        if (fast && is_warp_row(t.flags)) {      // one row per warp: every warp holds the whole input
            m.nvec = g.K >> 3; m.wpg = 1; m.G = kConsumerWarps; m.grp = warp; m.lig = lane;
            m.gstride = 32; m.vpt = m.nvec / 32; m.active = true;
        } else if (fast) {
            m.nvec = g.K >> 3; m.wpg = kConsumerWarps; m.G = 1; m.grp = 0; m.lig = tid;
            m.gstride = kConsumerThreads; m.vpt = m.nvec / kConsumerThreads; m.active = true;
        } else {
            m = thread_map(g.K);
        }
        const int rows_total = g.rows * g.nblk;
        const bool resid = !skip && warp == 0 && (t.op == MK_OP_OPROJ || t.op == MK_OP_DOWN) && p.tp <= 1;
        float resid0 = 0.0f, resid1 = 0.0f;
        if (!skip) {
            if (t.op == MK_OP_QKV && t.layer == 0 && tid == 0) {
                const int tok = p.tokens[0];
                if (tok < 0 || tok >= p.V) set_error(p, kErrInvalid, ti, -5, tok, 0);
            }
            if (!(x_key_op == t.op && x_key_layer == t.layer && x_key_b == t.b &&
                  (x_key_aux == t.aux || t.op != MK_OP_EXP_DOWN))) {
                gemv_prologue(p, sm, cph, t, m, g.K, xr);
                x_key_op = t.op; x_key_layer = t.layer; x_key_b = t.b; x_key_aux = t.aux;
            }
            // residual rows for the epilogue warp, fetched by warp 0 now so the loads
            // overlap the streaming
            if (resid) {
                const int r0 = (int)t.r0;
                if (lane < rows_total)
                    resid0 = (t.op == MK_OP_OPROJ) ? x_in(p, t.layer, 0, r0 + lane) : x_mid_at(p, t.layer, 0, r0 + lane);
                if (lane + 32 < rows_total)
                    resid1 = (t.op == MK_OP_OPROJ) ? x_in(p, t.layer, 0, r0 + lane + 32)
                                                   : x_mid_at(p, t.layer, 0, r0 + lane + 32);
            }
        }
        const long long c_ch = (p.stats && tid == 0) ? clock64() : 0;
        if (fast) (void)gemv_fast_dispatch(p, sm, ti, t.flags, g.rows, xr, buf, stage, lap);
        else (void)gemv_task_dispatch(p, sm, ti, g, m, xr, buf, stage, lap, skip);
        if (p.stats && tid == 0) stat_add(p, 6, (unsigned long long)(clock64() - c_ch));
        if (sm.flag[3]) break;
        if (resid) {
            if (lane < rows_total) sm.ep_resid[buf][lane] = resid0;
            if (lane + 32 < rows_total) sm.ep_resid[buf][lane + 32] = resid1;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.red_full[buf]);
        ++seq;
        }
    }
    // end of work for the epilogue warp: a marker once every consumer warp has left
    // the loop (a full set of arrivals on the next buffer set)
    csync(p, sm, cph);
    if (tid == 0) {
        const int buf = (int)(seq % kRedBufs);
        if (seq < (uint32_t)kRedBufs || mbar_wait_bounded(p, &sm.red_free[buf], ((seq / kRedBufs) - 1) & 1, 7)) {
            sm.ep_ti[buf] = -1;
            mbar_arrive_cnt(&sm.red_full[buf], kConsumerWarps);
        }
    }
    if (MM && warp == 0) {
        // every MMA this CTA issued has completed (also after an abort) before the
        // tensor memory is released
        if (lane == 0) {
            tc_commit(&sm.mm_drain);
            (void)mbar_wait_bounded(p, &sm.mm_drain, 0, 12);
        }
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(sm.tmem_base, tmem_cols);
    }
}

// ----------------------------------------------------------------------------- epilogue warp

// The in-step argmax of a batch-1 LM-head tile, run by the epilogue warp after it
// stored the tile's logits (out of line: it keeps the epilogue loop's registers).
__device__ __noinline__ void lmhead_argmax(const Params& p, const Task& t, int lane) {
    lmhead_arg_part(p, t, lane);
    argmax_arrive(p, t.aux, 1, lane);
}

// Row r of a finished GEMV task: the consumer warps' partial sums added in a fixed
// order (bit-identical from run to run).
__device__ __forceinline__ float gemv_row_sum(const Smem& sm, int buf, int r, int wpg) {
    float y = 0.0f;
    if (wpg == kConsumerWarps) {
        const float4 a = *reinterpret_cast<const float4*>(&sm.red[buf][r][0]);
        const float4 c = *reinterpret_cast<const float4*>(&sm.red[buf][r][4]);
        y = a.x; y += a.y; y += a.z; y += a.w; y += c.x; y += c.y; y += c.z; y += c.w;
    } else {
        for (int w = 0; w < wpg; ++w) y += sm.red[buf][r][w];
    }
    return y;
}

// Tensor parallelism: a finished O- or down-projection tile's rows are this rank's
// partial sums of those residual rows; each goes into every rank's receive buffer
// at this rank's slot (plain stores; the peers' buffers are mapped into this GPU's
// address space).  Out of line: the epilogue warp's register budget is small.
__device__ __noinline__ void tp_store_tile(const Params& p, const Smem& sm, const Task& t, int rows, int wpg,
                                           int buf, int lane) {
    const int ph = (t.op == MK_OP_DOWN) ? 1 : 0;
    const size_t base = (((size_t)p.tp_rank * p.L + t.layer) * 2 + ph) * p.H + t.r0;
    for (int r = lane; r < rows; r += 32) {
        const float y = gemv_row_sum(sm, buf, r, wpg);
        for (int q = 0; q < p.tp; ++q) p.tp_recv[q][base + r] = y;
    }
}

// Output rows of a finished GEMV task: the consumer warps' partial sums reduced in
// a fixed order (bit-identical from run to run), then the operator's tail.
__device__ __forceinline__ void gemv_store(const Params& p, const Smem& sm, const Task& t, const GemvGeom& g,
                                           int wpg, int buf, int lane) {
    const int l = t.layer, b = t.b;
    const int rows_total = g.rows * g.nblk;
    const int nout = (g.nblk == 2) ? g.rows : rows_total;
    auto row_sum = [&](int r) -> float { return gemv_row_sum(sm, buf, r, wpg); };
    for (int r = lane; r < nout; r += 32) {
        const float y = row_sum(r);
        const int row = (int)t.r0 + r;
        switch (t.op) {
            case MK_OP_QKV:
                p.qkv[((size_t)l * p.max_batch) * ((p.nq + 2 * p.nkv) * p.hd) + row] = y;
                break;
            case MK_OP_OPROJ:
                p.x_mid[((size_t)l * p.max_batch) * p.H + row] = sm.ep_resid[buf][r] + y;
                break;
            case MK_OP_GATEUP:
                p.act[((size_t)l * p.max_batch) * p.F + row] = silu_f(y) * row_sum(g.rows + r);
                break;
            case MK_OP_DOWN:
                p.x_out[((size_t)l * p.max_batch) * p.H + row] = sm.ep_resid[buf][r] + y;
                break;
            case MK_OP_LMHEAD:
                p.logits[row] = y;
                break;
            case MK_OP_ROUTER:
                p.rlogits[((size_t)l * p.max_batch) * p.E + row] = y;
                break;
            case MK_OP_EXP_GATEUP:
                p.act[(((size_t)l * p.max_batch + b) * p.topk + t.aux) * p.Fe + row] =
                    silu_f(y) * row_sum(g.rows + r);
                break;
            case MK_OP_EXP_DOWN:
                p.ypart[(((size_t)l * p.max_batch + b) * p.topk + t.aux) * p.H + row] = y;
                break;
            default:
                break;
        }
    }
}

// One warp of the support warpgroup finishes every task of its CTA, in order: it
// stores the GEMV outputs, selects the experts after a layer's last router tile,
// makes the task's writes visible (fence) and adds to the task's event counter
// with release semantics (MPK digest, "Part 2. Runtime": a finished task
// increments its event).  Router finalisation uses the scratch that attention
// and O-projection input stages also use; no consumer can reach one of those
// before the router event it precedes is signalled, since every later attention
// and O-projection depends on it.
__device__ void epilogue_loop(const Params& p, Smem& sm) {
    const int lane = threadIdx.x & 31;
    uint32_t seq = 0;
    while (true) {
        if (!mbar_wait_bounded(p, &sm.red_full[seq % kRedBufs], (seq / kRedBufs) & 1, 2)) return;
        // finish every task whose partials are already in (up to all buffer sets), then
        // one fence for all of them, then their signals in task order
        uint32_t evts[kRedBufs];
        int tis[kRedBufs];
        int nb = 0;
        bool end = false;
        do {
            const int buf = (int)(seq % kRedBufs);
            const int ti = sm.ep_ti[buf];
            if (ti < 0) { end = true; break; }          // end of work
            const Task t = sm.ep_task[buf];
            uint32_t evt = t.sig;
            if (is_gemv(t.op) && !(t.op == MK_OP_LMHEAD && p.skip_lm)) {
                GemvGeom g;
                gemv_geom(p, t, g, false);
                const int wpg = is_warp_row(t.flags) ? 1
                                : (t.flags != kFastNone) ? kConsumerWarps : thread_map(g.K).wpg;
                if (p.tp > 1 && (t.op == MK_OP_OPROJ || t.op == MK_OP_DOWN))
                    tp_store_tile(p, sm, t, g.rows, wpg, buf, lane);
                else
                    gemv_store(p, sm, t, g, wpg, buf, lane);
                if (t.op == MK_OP_LMHEAD && p.argmax_out) lmhead_argmax(p, t, lane);
                if (t.op == MK_OP_ROUTER) {
                    // arrival of this router tile (acquire-release: the warp barrier orders
                    // the lanes' logit stores before it); the layer's last tile selects the
                    // experts and only it signals the router event
                    __syncwarp();
                    int last = 0;
                    if (lane == 0) {
                        const uint32_t old = atom_add_acq_rel(p.router_cnt + t.layer, 1u);
                        last = (old == (uint32_t)p.n_router_tiles * p.epoch - 1u) ? 1 : 0;
                    }
                    last = __shfl_sync(0xFFFFFFFFu, last, 0);
                    __syncwarp();
                    if (last) router_finalize(p, sm, t.layer);
                    else evt = MK_NO_EVENT;
                }
            }
            // tensor parallelism: a projection tile raises its arrival flag on every rank
            if (p.tp > 1 && (t.op == MK_OP_OPROJ || t.op == MK_OP_DOWN))
                evt = kTpFlagBit | (((uint32_t)t.layer * 2u + (t.op == MK_OP_DOWN ? 1u : 0u)) * (uint32_t)p.tp_tiles + t.pad);
            evts[nb] = evt;
            tis[nb] = ti;
            ++nb;
            ++seq;
        } while (nb < kRedBufs && mbar_test_wait(&sm.red_full[seq % kRedBufs], (seq / kRedBufs) & 1));
        // The events are released with red.release.gpu by lane 0.  Release is
        // cumulative: it publishes every write that precedes it in causality order --
        // the other lanes' stores (ordered by the warp barrier) and the consumer
        // warps' stores (ordered by their arrivals on red_full, which this warp
        // acquired).  A full fence here (fence.sc by every lane) cost 0.34 ms of an
        // 8B step's 3.88 ms and is not needed.
        __syncwarp();
        if (lane == 0) {
            for (int k = 0; k < nb; ++k) {
                if (evts[k] != MK_NO_EVENT) {
                    if (evts[k] & kTpFlagBit) {
                        // system-scope release: cumulative over the lanes' stores to the
                        // peers' buffers (ordered before it by the warp barrier)
                        for (int q = 0; q < p.tp; ++q) red_release_add_sys(p.tp_flag[q] + (evts[k] & ~kTpFlagBit), 1u);
                    } else {
                        red_release_add(&p.events[evts[k]], 1u);
                    }
                }
                atomicAdd(p.done, 1u);
                if (p.trace) p.trace[(size_t)tis[k] * 4 + 2] = globaltimer();
                mbar_arrive(&sm.red_free[(seq - nb + k) % kRedBufs]);
            }
        }
        if (end) return;
    }
}

// ----------------------------------------------------------------------------- kernel

// Instantiations that re-split their registers between the warpgroups: the batch-1
// kernels (GEMV tiles keep the input slice and row sums in registers) and the
// batched kernels with 128-wide heads (attention staging); the batched kernels with
// 64-wide heads need fewer than the launch allows, and ptxas launches them with less.
__host__ __device__ constexpr bool splits_registers(bool mm, int dpl) { return !mm || dpl == 4; }

// MM: batched graphs (tensor-core tiles); WIDE: batch-1 graphs with a long attention
// phase -- attention tasks that cover every KV head (long contexts) or MoE graphs --
// whose steps may hold the producer's claims after attention tasks.  Each graph
// kind has its own instantiation, so one kind's code never costs another registers
// (the dense batch-1 kernel keeps the plain claim loop: the hold logic in it cost
// the 8B step 2% even where no split held).
template <int HPG, int DPL, bool MM, bool WIDE>
__device__ __forceinline__ void megakernel_body(const Params& p) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], kConsumerWarps);
        }
        mbar_init(&sm.csync, kConsumerWarps);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.mm_acc[i], 1);
            mbar_init(&sm.mm_free[i], 4);
        }
        mbar_init(&sm.mm_drain, 1);
        mbar_init(&sm.mm_sync, 4);
        for (int i = 0; i < kRedBufs; ++i) {
            mbar_init(&sm.red_full[i], kConsumerWarps);
            mbar_init(&sm.red_free[i], 1);
        }
        for (int i = 0; i < 4; ++i) sm.flag[i] = 0;
        sm.pf_claimed = 0;
        sm.pf_wait = 0;
        sm.started = -1;
        // the 128-byte-swizzled tensor-core operands need 1 KB-aligned stages
        if (p.mm && (smem_u32(sm.ring) & 1023u) != 0) {
            set_error(p, kErrFault, -1, -9, (int)(smem_u32(sm.ring) & 1023u), 0);
            sm.flag[3] = 1;
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    // Hand registers from the support warpgroup to the two consumer warpgroups.
    // The two branches never meet again (each returns), so the register limit of
    // one never constrains the code of the other.  The split is only valid when the
    // kernel launches with at least kMinLaunchRegs registers per thread (the build
    // and the launch both check that); instantiations whose code needs fewer keep
    // the launch's even split (splits_registers).
    if (warp < kConsumerWarps) {
        if constexpr (splits_registers(MM, DPL)) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kConsumerRegs));
        const long long k0 = clock64();
        consumer_loop<HPG, DPL, MM, WIDE>(p, sm);
        if (threadIdx.x == 0) stat_add(p, 3, (unsigned long long)(clock64() - k0));
        return;
    }
    if constexpr (splits_registers(MM, DPL)) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kSupportRegs));
    if (warp == kProducerWarp) {
        if (lane == 0) producer_loop<MM, WIDE>(p, sm);
    } else if (warp == kEpilogueWarp) {
        epilogue_loop(p, sm);
    } else if (warp == kPrefetchWarp) {
        if (lane == 0) prefetch_loop(p, sm);
    }
}

template <int HPG, int DPL, bool MM, bool WIDE>
__global__ void __launch_bounds__(kThreads, 1) megakernel(const __grid_constant__ Params p) {
    megakernel_body<HPG, DPL, MM, WIDE>(p);
}

// Tensor parallelism emulated on one GPU: the ranks' steps in one launch, the grid's
// CTAs dealt out to the ranks in equal consecutive runs (rank r: CTAs
// [r * per, (r + 1) * per)).  All CTAs are co-resident (a cooperative launch), so
// a rank's reduce tasks waiting on another rank's tiles always make progress.
template <int HPG, int DPL>
__global__ void __launch_bounds__(kThreads, 1) megakernel_tp(const __grid_constant__ TpLaunch L) {
    const int per = (int)gridDim.x / L.n;
    const int r = min((int)blockIdx.x / per, L.n - 1);
    megakernel_body<HPG, DPL, false, false>(L.r[r]);
}

// ----------------------------------------------------------------------------- host launch

template <int HPG, int DPL>
static cudaError_t launch_t(const Params& p, int grid, cudaStream_t stream, bool cooperative) {
    const bool long_attn = p.wide || p.E > 0;
    const int kind = p.mm ? 1 : (long_attn ? 2 : 0);
    auto kern = p.mm ? megakernel<HPG, DPL, true, false>
                     : (long_attn ? megakernel<HPG, DPL, false, true> : megakernel<HPG, DPL, false, false>);
    // the shared-memory attribute, once per instantiation and device (so that a step
    // can be captured into a CUDA graph without host-side calls in between)
    // (devices 0..63 are remembered; a higher index sets the attribute every launch)
    static unsigned long long attr_set[3] = {0ull, 0ull, 0ull};
    int dev = 0;
    cudaGetDevice(&dev);
    const unsigned long long bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
    if (!bit || !(attr_set[kind] & bit)) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(Smem));
        if (e != cudaSuccess) return e;
        // a register split (setmaxnreg) needs the launch's registers: with fewer, the
        // consumers' increase would wait forever, so such a build is never launched
        cudaFuncAttributes fa{};
        e = cudaFuncGetAttributes(&fa, (const void*)kern);
        if (e != cudaSuccess) return e;
        if (splits_registers(p.mm != 0, DPL) && fa.numRegs < kMinLaunchRegs) return cudaErrorInvalidConfiguration;
        attr_set[kind] |= bit;
    }
    Params q = p;                 // this launch's CTAs: all of the grid
    q.cta0 = 0;
    q.ncta = grid;
    void* args[] = {&q};
    if (cooperative)
        return cudaLaunchCooperativeKernel((const void*)kern, dim3(grid), dim3(kThreads), args, sizeof(Smem), stream);
    return cudaLaunchKernel((const void*)kern, dim3(grid), dim3(kThreads), args, sizeof(Smem), stream);
}

size_t megakernel_smem_bytes() { return sizeof(Smem); }

cudaError_t megakernel_launch(const Params& p, int grid, cudaStream_t stream, bool cooperative) {
    const int hpg = p.nq / p.nkv;
    const int dpl = p.hd / 32;
    if (dpl == 4) {
        switch (hpg) {
            case 1: return launch_t<1, 4>(p, grid, stream, cooperative);
            case 2: return launch_t<2, 4>(p, grid, stream, cooperative);
            case 4: return launch_t<4, 4>(p, grid, stream, cooperative);
            case 8: return launch_t<8, 4>(p, grid, stream, cooperative);
        }
    } else if (dpl == 2) {
        switch (hpg) {
            case 1: return launch_t<1, 2>(p, grid, stream, cooperative);
            case 2: return launch_t<2, 2>(p, grid, stream, cooperative);
            case 4: return launch_t<4, 2>(p, grid, stream, cooperative);
            case 8: return launch_t<8, 2>(p, grid, stream, cooperative);
        }
    }
    return cudaErrorInvalidValue;
}

template <int HPG, int DPL>
static cudaError_t launch_tp_t(const TpLaunch& L, int grid, cudaStream_t stream) {
    auto kern = megakernel_tp<HPG, DPL>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(Smem));
    if (e != cudaSuccess) return e;
    cudaFuncAttributes fa{};
    e = cudaFuncGetAttributes(&fa, (const void*)kern);
    if (e != cudaSuccess) return e;
    if (fa.numRegs < kMinLaunchRegs) return cudaErrorInvalidConfiguration;
    void* args[] = {const_cast<TpLaunch*>(&L)};
    return cudaLaunchCooperativeKernel((const void*)kern, dim3(grid), dim3(kThreads), args, sizeof(Smem), stream);
}

cudaError_t megakernel_launch_tp_emulated(const TpLaunch& L, int grid, cudaStream_t stream) {
    if (L.n < 1 || L.n > kMaxTpEmulated || grid < L.n || grid % L.n) return cudaErrorInvalidValue;
    const Params& p = L.r[0];
    const int hpg = p.nq / p.nkv, dpl = p.hd / 32;
    if (dpl == 4) {
        switch (hpg) {
            case 1: return launch_tp_t<1, 4>(L, grid, stream);
            case 2: return launch_tp_t<2, 4>(L, grid, stream);
            case 4: return launch_tp_t<4, 4>(L, grid, stream);
            case 8: return launch_tp_t<8, 4>(L, grid, stream);
        }
    }
    return cudaErrorInvalidValue;
}

bool megakernel_supports(int hpg, int hd) {
    return (hd == 64 || hd == 128) && (hpg == 1 || hpg == 2 || hpg == 4 || hpg == 8);
}

cudaError_t megakernel_occupancy(int hpg, int hd, int* blocks_per_sm) {
    const int dpl = hd / 32;
    const void* f = nullptr;
    if (dpl == 4) {
        if (hpg == 1) f = (const void*)megakernel<1, 4, false, false>;
        if (hpg == 2) f = (const void*)megakernel<2, 4, false, false>;
        if (hpg == 4) f = (const void*)megakernel<4, 4, false, false>;
        if (hpg == 8) f = (const void*)megakernel<8, 4, false, false>;
    } else {
        if (hpg == 1) f = (const void*)megakernel<1, 2, false, false>;
        if (hpg == 2) f = (const void*)megakernel<2, 2, false, false>;
        if (hpg == 4) f = (const void*)megakernel<4, 2, false, false>;
        if (hpg == 8) f = (const void*)megakernel<8, 2, false, false>;
    }
    if (!f) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(Smem));
    if (e != cudaSuccess) return e;
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, f, kThreads, sizeof(Smem));
}

}  // namespace mk
