// Host-side declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace pa {

// Most splits one decode call may have (max_seq_len / partition_size,
// rounded up): the wide split reduce keeps one weight per split in shared
// memory, and the entry points reject a call that would need more.
constexpr int kMaxSplits = 2048;

// Everything a decode kernel needs; passed by value.
struct DecodeParams {
    float *out;        // [B][Hq][D]
    float *part_o;     // [B][Hq][S][D]  unnormalised partial sums (S > 1 only)
    float *part_ml;    // [B][Hq][S][2]  (running max in log2 units, sum of weights)
    const void *q;     // [B][Hq][D]
    const void *k_cache, *v_cache;  // [NB][Hkv][bs][D]
    const int32_t *block_tables;    // [B][max_blocks_per_seq]
    const int32_t *seq_lens;        // [B]
    unsigned int *err;              // device error word
    int num_seqs, num_heads, num_kv_heads, head_dim, block_size;
    int max_blocks_per_seq, num_blocks, max_seq_len;
    int partition_size;  // tokens per split
    int max_splits;      // S = ceil(max_seq_len / partition_size), >= 1
    float scale_log2;    // softmax scale * log2(e)
    // In-kernel merge of the split partials (null: the reduce kernel merges):
    // one ticket per (sequence, KV head), high 32 bits the call's tag, low 32
    // bits the splits of that call done so far.
    unsigned long long *tickets;
    uint32_t tag;
    // Order in which the grid takes the sequences (grid row z works on
    // sequence seq_order[z]; null: z itself).  A runtime that knows the
    // lengths passes longest first, so that the last CTAs to start are short.
    const int32_t *seq_order;
    // Append fused into the decode (null: none): the new token of every
    // sequence, at position seq_lens[s] - 1, with its K/V rows in
    // k_new/v_new [B][Hkv][D] and its slot in slot_mapping[B]; the split CTA
    // holding that position writes its head's rows into the cache first.
    const void *k_new, *v_new;
    const int64_t *slot_mapping;
};

int num_sms();  // SMs of the current device (cached per device)

cudaError_t launch_reshape_and_cache(const void *k, const void *v, void *k_cache, void *v_cache,
                                     const int64_t *slot_mapping, int num_tokens,
                                     int num_kv_heads, int row_bytes, int block_size,
                                     int num_blocks, unsigned int *err, cudaStream_t stream);

cudaError_t launch_copy_blocks(void *k_cache, void *v_cache, const int64_t *pairs, int num_pairs,
                               size_t block_bytes, int num_blocks, unsigned int *err,
                               cudaStream_t stream);

cudaError_t launch_swap_blocks(void *dst_k, void *dst_v, const void *src_k, const void *src_v,
                               const int64_t *pairs, int num_pairs, size_t block_bytes,
                               int num_src_blocks, int num_dst_blocks, unsigned int *err,
                               cudaStream_t stream);

// CUDA-core decode (any dtype, any supported block size).  dtype: pa_dtype.
cudaError_t launch_decode_simt(const DecodeParams &p, int dtype, cudaStream_t stream);

// Tensor-core decode (bf16/f16, block_size >= 8): TMA-staged K/V, mma.sync.
// Returns cudaErrorNotSupported for shapes it does not cover.
cudaError_t launch_decode_tc(const DecodeParams &p, int dtype, cudaStream_t stream);
// Tensor-core decode with one KV head per consumer warp, heads_per_cta (1, 2
// or 4, dividing num_kv_heads, with heads_per_cta * max(16, block_size) <=
// 64) heads per CTA.  cudaErrorNotSupported for shapes it does not cover.
cudaError_t launch_decode_hw(const DecodeParams &p, int dtype, int heads_per_cta,
                             cudaStream_t stream);
// CTAs of that kernel with two KV heads per CTA resident per SM (block size 8
// or 16), or -1
int decode_hw2_resident_per_sm(int dtype, int head_dim, int block_size);
// CTAs of the tensor-core decode kernel for this shape resident per SM, or -1
int decode_tc_resident_per_sm(int dtype, int head_dim, int block_size);

// TMA map of a cache viewed as [rows][D] 16-bit elements: 128-byte boxes of
// box_rows rows, 128B swizzle.  False if the driver refuses it.
bool make_cache_tensor_map(CUtensorMap *m, const void *base, int dtype, int D, int64_t rows,
                           int box_rows);

// Causal multi-token attention over the paged cache (bf16/f16, bs >= 8).
struct PrefillParams {
    float *out;                     // [total][Hq][D]
    const void *q;                  // [total][Hq][D]
    const void *k_cache, *v_cache;  // [NB][Hkv][bs][D]
    const int32_t *block_tables;    // [B][max_blocks_per_seq]
    const int32_t *seq_lens;        // [B], context length including the chunk
    const int32_t *cu_q;            // [B + 1], chunk row offsets
    unsigned int *err;
    int num_seqs, num_heads, num_kv_heads, head_dim, block_size;
    int max_blocks_per_seq, num_blocks, max_seq_len, max_q_len;
    int tokens_per_cta;             // query tokens per CTA: 64 / G (mma.sync), 128 / G (tcgen05)
    float scale_log2;
};
// mma.sync kernel: 64 (token, head) rows per CTA, accumulators in registers.
cudaError_t launch_prefill_tc(const PrefillParams &p, int dtype, cudaStream_t stream);
// tcgen05 kernel: 128 rows per CTA, S and O accumulated in TMEM.  form 0:
// one tile per CTA; 1 (persistent): one CTA per SM walking a share of the
// token tiles, each tile's start overlapping the previous tile's end; 2: one
// tile per CTA with P entering the PV product as one fp16 per weight.
cudaError_t launch_prefill_umma(const PrefillParams &p, int dtype, int form,
                                cudaStream_t stream);

// One CTA waiting, bounded, on an mbarrier phase nothing completes (selftest.cu).
cudaError_t launch_wait_selftest(unsigned int *err, uint64_t limit_ns, uint64_t abort_after_ns,
                                 unsigned long long *elapsed_ns, cudaStream_t stream);

// Merge of split partials into out; a no-op when max_splits == 1.
cudaError_t launch_decode_reduce(const DecodeParams &p, cudaStream_t stream);

}  // namespace pa
