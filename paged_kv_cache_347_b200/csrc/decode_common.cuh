// Pieces of the decode kernels that the CUDA-core kernel, the tensor-core
// kernel and the split reduce must agree on.
#pragma once

#include "common.cuh"
#include "launch.h"

namespace pa {

// Sequence worked on by grid row z: seq_order[z] when the caller gave an
// order, else z; -1 (PA_DEVERR_SEQLEN raised once) for an entry outside
// [0, num_seqs).
__device__ __forceinline__ int seq_of(const DecodeParams &p, int z, bool report) {
    if (p.seq_order == nullptr) return z;
    const int s = __ldg(p.seq_order + z);
    if (s < 0 || s >= p.num_seqs) {
        if (report) raise_device_error(p.err, PA_DEVERR_SEQLEN);
        return -1;
    }
    return s;
}

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

// ---------------------------------------------------------------- fused append
// The append of mbrenndoerfer.com "Paged Attention > Summary", bullet 3 (a new
// token's K/V written into its sequence's last block) fused into the decode:
// the CTA whose split holds position L - 1 writes the new token's rows for
// KV heads g .. g + nh - 1 before it reads that block.  The slot must be the
// one the table gives position L - 1; another slot (a caller's mistake that
// could race with other CTAs' reads) is not written and sets PA_DEVERR_SLOT,
// and a negative slot means "no write", as for pa_reshape_and_cache.  The
// lanes of one warp copy 16-byte words; each fences its stores against the
// async proxy (the TMA loads that follow read the row), and the warp syncs.
__device__ __forceinline__ void fused_append_rows(const DecodeParams &p, int s, int g, int nh,
                                                  int L, int elem_bytes, int lane) {
    const int64_t slot = __ldg(p.slot_mapping + s);
    if (slot >= 0) {
        const int pos = L - 1;
        const int blk = checked_block(p, s, pos / p.block_size);
        const int64_t want = blk < 0 ? -1 : (int64_t)blk * p.block_size + pos % p.block_size;
        if (slot != want) {
            if (lane == 0 && blk >= 0) raise_device_error(p.err, PA_DEVERR_SLOT);
        } else {
            const int words = p.head_dim * elem_bytes / 16;  // per row
            const int64_t b = slot / p.block_size, off = slot % p.block_size;
            for (int c = lane; c < nh * words; c += 32) {
                const int h = g + c / words, w = c - (c / words) * words;
                const int64_t src = ((int64_t)s * p.num_kv_heads + h) * words + w;
                const int64_t dst = ((b * p.num_kv_heads + h) * p.block_size + off) * words + w;
                reinterpret_cast<uint4 *>(const_cast<void *>(p.k_cache))[dst] =
                    __ldg(reinterpret_cast<const uint4 *>(p.k_new) + src);
                reinterpret_cast<uint4 *>(const_cast<void *>(p.v_cache))[dst] =
                    __ldg(reinterpret_cast<const uint4 *>(p.v_new) + src);
            }
            asm volatile("fence.proxy.async.global;" ::: "memory");
        }
    }
    __syncwarp();
}

// ---------------------------------------------------------------- in-kernel merge
// The split-context partials of a (sequence, KV head) can be merged by the
// main kernel itself: the CTA of that pair to finish last merges them (the
// online-softmax rescale of mbrenndoerfer.com "Paged Attention > Summary",
// bullet 3, applied to whole splits).  Which CTA is last is decided by a
// ticket word in the workspace.  Its high half carries a tag that changes
// with every call, so the word never has to be cleared: a word left by an
// earlier call (or any old bytes) carries another tag and counts as zero.
// The last CTA leaves the count at zero under its own tag, so a CUDA graph
// that replays a call with the same tag counts from zero again.

// Counts this CTA's split as done; true for the CTA that completes the
// count.  One thread per CTA, after every thread's partial stores and a
// __threadfence() by each of them.
__device__ __forceinline__ bool ticket_arrive_last(unsigned long long *t, uint32_t tag,
                                                   int nsplit) {
    unsigned long long seen = *reinterpret_cast<volatile unsigned long long *>(t);
    uint32_t done = 0;
    for (;;) {
        done = (uint32_t)(seen >> 32) == tag ? (uint32_t)seen : 0u;
        const unsigned long long want = ((unsigned long long)tag << 32) | (done + 1u);
        const unsigned long long got = atomicCAS(t, seen, want);
        if (got == seen) break;
        seen = got;
    }
    if (done + 1u == (uint32_t)nsplit) {
        // every other split of this call has arrived: reset the count for a
        // replay of the same call
        atomicExch(t, (unsigned long long)tag << 32);
        __threadfence();
        return true;
    }
    return false;
}

// out[s][h0 .. h0+G-1][:] from the nsplit partials of those heads: threads
// tid = 0 .. nthreads-1 of the merging CTA each take float4 columns.  The
// partials were written by other CTAs of this grid: read through L2 (.cg).
__device__ __forceinline__ void merge_splits(const DecodeParams &p, int s, int h0, int G,
                                             int nsplit, int tid, int nthreads) {
    const int D4 = p.head_dim >> 2;
    for (int c = tid; c < G * D4; c += nthreads) {
        const int h = h0 + c / D4, d4 = c - (c / D4) * D4;
        const int64_t u0 = ((int64_t)s * p.num_heads + h) * p.max_splits;
        const float2 *ml = reinterpret_cast<const float2 *>(p.part_ml) + u0;
        const float4 *po = reinterpret_cast<const float4 *>(p.part_o + u0 * p.head_dim) + d4;
        float M = -INFINITY;
#pragma unroll 8
        for (int j = 0; j < nsplit; ++j) M = fmaxf(M, __ldcg(ml + j).x);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        float den = 0.f;
        if (M != -INFINITY) {
#pragma unroll 8
            for (int j = 0; j < nsplit; ++j) {
                const float2 v = __ldcg(ml + j);
                const float4 o = __ldcg(po + (int64_t)j * D4);
                const float w = exp2f(v.x - M);
                den = fmaf(w, v.y, den);
                acc.x = fmaf(w, o.x, acc.x);
                acc.y = fmaf(w, o.y, acc.y);
                acc.z = fmaf(w, o.z, acc.z);
                acc.w = fmaf(w, o.w, acc.w);
            }
        }
        const float inv = den > 0.f ? 1.f / den : 0.f;
        reinterpret_cast<float4 *>(p.out + ((int64_t)s * p.num_heads + h) * p.head_dim)[d4] =
            make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    }
}

}  // namespace pa
