// Pieces of the decode kernels that the CUDA-core kernel, the tensor-core
// kernel and the split reduce must agree on.
#pragma once

#include "common.cuh"
#include "launch.h"

namespace pa {

// Length of sequence s, or 0 (with PA_DEVERR_SEQLEN raised once per
// sequence) when it is negative, above max_seq_len or longer than its table.
__device__ __forceinline__ int checked_seq_len(const DecodeParams &p, int s, bool report) {
    const int L = __ldg(p.seq_lens + s);
    const bool bad = L < 0 || L > p.max_seq_len ||
                     (int64_t)(L + p.block_size - 1) / p.block_size > p.max_blocks_per_seq;
    if (bad) {
        if (report) raise_device_error(p.err, PA_DEVERR_SEQLEN);
        return 0;
    }
    return L;
}

// Splits used by a sequence of L tokens: one for an empty sequence.
__device__ __forceinline__ int num_splits_for(int L, int partition_size) {
    return L <= 0 ? 1 : (L + partition_size - 1) / partition_size;
}

// Physical block of logical block j of sequence s, or -1 (PA_DEVERR_TABLE
// raised) when the entry is outside [0, num_blocks).
__device__ __forceinline__ int checked_block(const DecodeParams &p, int s, int j) {
    const int b = __ldg(p.block_tables + (int64_t)s * p.max_blocks_per_seq + j);
    if (b < 0 || b >= p.num_blocks) {
        raise_device_error(p.err, PA_DEVERR_TABLE);
        return -1;
    }
    return b;
}

// The same check on a raw table: entry j of row s, or -1 (PA_DEVERR_TABLE).
__device__ __forceinline__ int checked_block_row(const int32_t *tables, int max_blocks,
                                                 int num_blocks, unsigned int *err, int s, int j) {
    const int b = __ldg(tables + (int64_t)s * max_blocks + j);
    if (b < 0 || b >= num_blocks) {
        raise_device_error(err, PA_DEVERR_TABLE);
        return -1;
    }
    return b;
}

// Writes the result of one (sequence, head, split) unit: the normalised
// output when the sequence has a single split, else the partial triple.
// m is in log2 units; m == -inf with l == 0 means "no tokens".
__device__ __forceinline__ void store_unit(const DecodeParams &p, int s, int h, int split,
                                           int nsplit, int d, float m, float l, float o) {
    if (nsplit == 1) {
        p.out[((int64_t)s * p.num_heads + h) * p.head_dim + d] = l > 0.f ? o / l : 0.f;
    } else {
        const int64_t u = ((int64_t)s * p.num_heads + h) * p.max_splits + split;
        p.part_o[u * p.head_dim + d] = o;
        if (d == 0) {
            p.part_ml[2 * u] = m;
            p.part_ml[2 * u + 1] = l;
        }
    }
}

}  // namespace pa
