/*
 * Host fill routines of the synthetic input generator (definition in gen.h).
 * Built as libsynthetic_host.so; used by the tests and by the CPU side of the
 * benchmark to materialise weights, KV contents and token streams in host
 * memory.  Holds no arithmetic of the decode step.
 */
#include <stddef.h>
#include <stdint.h>

#include "gen.h"

/* out[k] = element (offset + k) of tensor (seed, tensor_id), k < n. */
void syn_fill_bf16(uint16_t* out, uint64_t n, uint64_t seed, uint64_t tensor_id,
                   uint64_t offset, float sigma, float mean) {
    const uint64_t key = syn_key(seed, tensor_id);
    const float scale = sigma * (1.0f / 131072.0f);
#pragma omp parallel for schedule(static)
    for (int64_t k = 0; k < (int64_t)n; ++k)
        out[k] = syn_bf16_value(key, offset + (uint64_t)k, scale, mean);
}

/* out[k] = uniform integer in [lo, lo + span) for element (offset + k). */
void syn_fill_int32(int32_t* out, uint64_t n, uint64_t seed, uint64_t tensor_id,
                    uint64_t offset, int64_t lo, uint64_t span) {
    const uint64_t key = syn_key(seed, tensor_id);
    for (uint64_t k = 0; k < n; ++k)
        out[k] = (int32_t)syn_uniform_int(key, offset + k, lo, span);
}

/* Raw 64-bit words (for host-side shuffles such as a page permutation). */
void syn_fill_words(uint64_t* out, uint64_t n, uint64_t seed, uint64_t tensor_id,
                    uint64_t offset) {
    const uint64_t key = syn_key(seed, tensor_id);
    for (uint64_t k = 0; k < n; ++k) out[k] = syn_word(key, offset + k, 0);
}

/*
 * KV cache contents for one (layer, K-or-V) tensor, one sequence, written to
 * a contiguous host array dst[pos - pos0][kv_head][dim] for pos in
 * [pos0, pos1).  The logical element index of (seq, pos, head, dim) is
 * ((seq * 2^20 + pos) * n_kv + head) * head_dim + dim, so the contents do not
 * depend on where a page lands in a paged pool.
 */
void syn_fill_kv_contig(uint16_t* dst, uint64_t seed, uint64_t tensor_id, int seq,
                        int pos0, int pos1, int n_kv, int head_dim, float sigma) {
    const uint64_t key = syn_key(seed, tensor_id);
    const float scale = sigma * (1.0f / 131072.0f);
    const int64_t row = (int64_t)n_kv * head_dim;
#pragma omp parallel for schedule(static)
    for (int p = pos0; p < pos1; ++p) {
        uint64_t base = (((uint64_t)seq << 20) + (uint64_t)p) * (uint64_t)row;
        uint16_t* d = dst + (int64_t)(p - pos0) * row;
        for (int64_t e = 0; e < row; ++e) d[e] = syn_bf16_value(key, base + (uint64_t)e, scale, 0.0f);
    }
}
