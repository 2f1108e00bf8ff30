// KV append (pa_reshape_and_cache) and copy-on-write block copy
// (pa_copy_blocks).
//
// Append: paweldubiel.com "PagedAttention", "Mechanism and details" -- a new
// position goes into the free part of the last block (or a fresh block)
// without moving the prefix; its slot is phys * bs + off.  Copy:
// sanketn26 "PagedAttention", "Sharing needs ownership rules" -- a shared
// block is copied before one sharer changes it.
//
// Both are pure data movement: every thread moves 16-byte words with one
// 128-bit load and one 128-bit store; consecutive threads touch consecutive
// words of a row, so a warp moves 512 contiguous bytes.  The grids are sized
// in multiples of the SM count (grid-stride loops).
#include "common.cuh"
#include "launch.h"

namespace pa {

// One 16-byte word per iteration: word w of (token t, head h) row.
__global__ void __launch_bounds__(256) reshape_and_cache_kernel(
    const uint4 *__restrict__ k, const uint4 *__restrict__ v, uint4 *__restrict__ k_cache,
    uint4 *__restrict__ v_cache, const int64_t *__restrict__ slot_mapping, int num_tokens,
    int num_kv_heads, int words_per_row, int block_size, int64_t num_slots,
    unsigned int *err) {
    // a decode launched after this kernel may start its prologue now; it
    // waits for this grid's writes before reading the cache
    pdl_launch_dependents();
    const int64_t words_per_token = (int64_t)num_kv_heads * words_per_row;
    const int64_t total = (int64_t)num_tokens * words_per_token;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = i / words_per_token;
        const int64_t rem = i - t * words_per_token;
        const int64_t h = rem / words_per_row;
        const int64_t w = rem - h * words_per_row;
        const int64_t slot = __ldg(slot_mapping + t);
        if (slot < 0) continue;
        if (slot >= num_slots) {
            if (rem == 0) raise_device_error(err, PA_DEVERR_SLOT);
            continue;
        }
        const int64_t blk = slot / block_size;
        const int64_t off = slot - blk * block_size;
        const int64_t dst = ((blk * num_kv_heads + h) * block_size + off) * words_per_row + w;
        k_cache[dst] = __ldg(k + i);
        v_cache[dst] = __ldg(v + i);
    }
}

// Pair p copies words [0, words_per_block) of block src onto block dst, in
// both caches.  gridDim.y walks the pairs, gridDim.x the words of a block.
__global__ void __launch_bounds__(256) copy_blocks_kernel(
    uint4 *__restrict__ k_cache, uint4 *__restrict__ v_cache, const int64_t *__restrict__ pairs,
    int num_pairs, int64_t words_per_block, int num_blocks, unsigned int *err) {
    for (int p = blockIdx.y; p < num_pairs; p += gridDim.y) {
        const int64_t src = __ldg(pairs + 2 * p);
        const int64_t dst = __ldg(pairs + 2 * p + 1);
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
            if (blockIdx.x == 0 && threadIdx.x == 0) raise_device_error(err, PA_DEVERR_PAIR);
            continue;
        }
        const uint4 *ks = k_cache + src * words_per_block;
        const uint4 *vs = v_cache + src * words_per_block;
        uint4 *kd = k_cache + dst * words_per_block;
        uint4 *vd = v_cache + dst * words_per_block;
        for (int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; w < words_per_block;
             w += (int64_t)gridDim.x * blockDim.x) {
            const uint4 a = ks[w];
            const uint4 b = vs[w];
            kd[w] = a;
            vd[w] = b;
        }
    }
}

// Pair p copies block src of (src_k, src_v) onto block dst of (dst_k, dst_v);
// either side may be mapped host memory, so this is also the swap path.
__global__ void __launch_bounds__(256) swap_blocks_kernel(
    const uint4 *__restrict__ src_k, const uint4 *__restrict__ src_v, uint4 *__restrict__ dst_k,
    uint4 *__restrict__ dst_v, const int64_t *__restrict__ pairs, int num_pairs,
    int64_t words_per_block, int num_src_blocks, int num_dst_blocks, unsigned int *err) {
    for (int p = blockIdx.y; p < num_pairs; p += gridDim.y) {
        const int64_t src = pairs[2 * p];
        const int64_t dst = pairs[2 * p + 1];
        if (src < 0 || src >= num_src_blocks || dst < 0 || dst >= num_dst_blocks) {
            if (blockIdx.x == 0 && threadIdx.x == 0) raise_device_error(err, PA_DEVERR_PAIR);
            continue;
        }
        const uint4 *ks = src_k + src * words_per_block;
        const uint4 *vs = src_v + src * words_per_block;
        uint4 *kd = dst_k + dst * words_per_block;
        uint4 *vd = dst_v + dst * words_per_block;
        for (int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; w < words_per_block;
             w += (int64_t)gridDim.x * blockDim.x) {
            const uint4 a = ks[w];
            const uint4 b = vs[w];
            kd[w] = a;
            vd[w] = b;
        }
    }
}

cudaError_t launch_swap_blocks(void *dst_k, void *dst_v, const void *src_k, const void *src_v,
                               const int64_t *pairs, int num_pairs, size_t block_bytes,
                               int num_src_blocks, int num_dst_blocks, unsigned int *err,
                               cudaStream_t stream) {
    if (num_pairs == 0) return cudaSuccess;
    const int64_t words = (int64_t)(block_bytes / 16);
    const int threads = 256;
    int64_t bx = (words + threads - 1) / threads;
    if (bx > 64) bx = 64;
    int64_t by = num_pairs;
    const int64_t cap = (int64_t)num_sms() * 8;
    if (bx * by > cap) by = cap / bx > 0 ? cap / bx : 1;
    if (by > 65535) by = 65535;
    swap_blocks_kernel<<<dim3((unsigned)bx, (unsigned)by), threads, 0, stream>>>(
        static_cast<const uint4 *>(src_k), static_cast<const uint4 *>(src_v),
        static_cast<uint4 *>(dst_k), static_cast<uint4 *>(dst_v), pairs, num_pairs, words,
        num_src_blocks, num_dst_blocks, err);
    return cudaGetLastError();
}

cudaError_t launch_reshape_and_cache(const void *k, const void *v, void *k_cache, void *v_cache,
                                     const int64_t *slot_mapping, int num_tokens,
                                     int num_kv_heads, int row_bytes, int block_size,
                                     int num_blocks, unsigned int *err, cudaStream_t stream) {
    const int words_per_row = row_bytes / 16;
    const int64_t total = (int64_t)num_tokens * num_kv_heads * words_per_row;
    if (total == 0) return cudaSuccess;
    const int threads = 256;
    int64_t blocks = (total + threads - 1) / threads;
    const int64_t cap = (int64_t)num_sms() * 8;
    if (blocks > cap) blocks = cap;
    reshape_and_cache_kernel<<<(unsigned)blocks, threads, 0, stream>>>(
        static_cast<const uint4 *>(k), static_cast<const uint4 *>(v),
        static_cast<uint4 *>(k_cache), static_cast<uint4 *>(v_cache), slot_mapping, num_tokens,
        num_kv_heads, words_per_row, block_size, (int64_t)num_blocks * block_size, err);
    return cudaGetLastError();
}

cudaError_t launch_copy_blocks(void *k_cache, void *v_cache, const int64_t *pairs, int num_pairs,
                               size_t block_bytes, int num_blocks, unsigned int *err,
                               cudaStream_t stream) {
    if (num_pairs == 0) return cudaSuccess;
    const int64_t words = (int64_t)(block_bytes / 16);
    const int threads = 256;
    int64_t bx = (words + threads - 1) / threads;
    if (bx > 64) bx = 64;
    int64_t by = num_pairs;
    const int64_t cap = (int64_t)num_sms() * 8;
    if (bx * by > cap) by = cap / bx > 0 ? cap / bx : 1;
    if (by > 65535) by = 65535;
    copy_blocks_kernel<<<dim3((unsigned)bx, (unsigned)by), threads, 0, stream>>>(
        static_cast<uint4 *>(k_cache), static_cast<uint4 *>(v_cache), pairs, num_pairs, words,
        num_blocks, err);
    return cudaGetLastError();
}

}  // namespace pa
