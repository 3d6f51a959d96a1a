/*
 * Device fill routines of the synthetic input generator (definition in gen.h).
 * Built as libsynthetic_dev.so.  They let the benchmark and the GPU tests
 * draw multi-GB weight sets and KV caches directly in HBM; the bits equal
 * those of the host fill in synthetic.c element for element.  Holds no
 * arithmetic of the decode step.
 */
#include <cuda_runtime.h>
#include <stdint.h>

#include "gen.h"

namespace {

__global__ void fill_bf16_kernel(uint16_t* out, uint64_t n, uint64_t key, uint64_t offset,
                                 float scale, float mean) {
    uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
    for (uint64_t k = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; k < n; k += stride)
        out[k] = syn_bf16_value(key, offset + k, scale, mean);
}

__global__ void fill_int32_kernel(int32_t* out, uint64_t n, uint64_t key, uint64_t offset,
                                  int64_t lo, uint64_t span) {
    uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
    for (uint64_t k = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; k < n; k += stride)
        out[k] = (int32_t)syn_uniform_int(key, offset + k, lo, span);
}

/* One layer's K (or V) pool, layout [n_pages][n_kv][page_size][head_dim]. */
__global__ void fill_kv_paged_kernel(uint16_t* pool, const int32_t* page_row, int seq, int pos0,
                                     int pos1, int n_kv, int page_size, int head_dim,
                                     uint64_t key, float scale) {
    const uint64_t row = (uint64_t)n_kv * head_dim;
    const uint64_t n = (uint64_t)(pos1 - pos0) * row;
    uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
    for (uint64_t k = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; k < n; k += stride) {
        int pos = pos0 + (int)(k / row);
        int rem = (int)(k % row);
        int g = rem / head_dim, i = rem % head_dim;
        int phys = page_row[pos / page_size];
        uint64_t logical = ((((uint64_t)seq << 20) + (uint64_t)pos) * row) + (uint64_t)rem;
        uint64_t dst = (((uint64_t)phys * n_kv + g) * page_size + (pos % page_size)) * head_dim + i;
        pool[dst] = syn_bf16_value(key, logical, scale, 0.0f);
    }
}

int grid_for(uint64_t n) {
    uint64_t b = (n + 255) / 256;
    if (b > 148ull * 64) b = 148ull * 64;
    if (b == 0) b = 1;
    return (int)b;
}

}  // namespace

extern "C" {

int syn_dev_fill_bf16(void* out, uint64_t n, uint64_t seed, uint64_t tensor_id, uint64_t offset,
                      float sigma, float mean, cudaStream_t stream) {
    if (n == 0) return 0;
    fill_bf16_kernel<<<grid_for(n), 256, 0, stream>>>((uint16_t*)out, n, syn_key(seed, tensor_id),
                                                      offset, sigma * (1.0f / 131072.0f), mean);
    return (int)cudaGetLastError();
}

int syn_dev_fill_int32(int32_t* out, uint64_t n, uint64_t seed, uint64_t tensor_id,
                       uint64_t offset, int64_t lo, uint64_t span, cudaStream_t stream) {
    if (n == 0) return 0;
    fill_int32_kernel<<<grid_for(n), 256, 0, stream>>>(out, n, syn_key(seed, tensor_id), offset,
                                                       lo, span);
    return (int)cudaGetLastError();
}

/* page_row: device pointer to this sequence's row of the page table. */
int syn_dev_fill_kv_paged(void* pool, const int32_t* page_row, int seq, int pos0, int pos1,
                          int n_kv, int page_size, int head_dim, uint64_t seed,
                          uint64_t tensor_id, float sigma, cudaStream_t stream) {
    if (pos1 <= pos0) return 0;
    uint64_t n = (uint64_t)(pos1 - pos0) * n_kv * head_dim;
    fill_kv_paged_kernel<<<grid_for(n), 256, 0, stream>>>(
        (uint16_t*)pool, page_row, seq, pos0, pos1, n_kv, page_size, head_dim,
        syn_key(seed, tensor_id), sigma * (1.0f / 131072.0f));
    return (int)cudaGetLastError();
}

}  // extern "C"
