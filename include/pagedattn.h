/*
 * pagedattn.h -- C ABI of the B200 paged-KV decode library (libpagedattn.so).
 *
 * The hot path of PagedAttention for single-query decode: a KV cache held in
 * fixed-size physical blocks, a per-sequence block table that maps logical
 * blocks to physical ones, the append of new tokens' K/V into their slots,
 * the copy-on-write block copy, and the host-side block allocator that hands
 * out slots, shares blocks and decides copies.
 *
 * Sources (the PagedAttention pages):
 *   [P1] paweldubiel.com "PagedAttention" -- blocks of a fixed number of
 *        positions; a block table gives the physical place of each logical
 *        block; appending never moves the prefix; paging does not change the
 *        attention result ("Text order is not a memory address").
 *   [P2] sanketn26 "PagedAttention -- grow the allocation with the sequence" --
 *        "Separate logical order from physical location", "Sharing needs
 *        ownership rules" (copy-on-write), "Exercise and checkpoint" (release
 *        on completion), "What this does not solve" (admission can fail).
 *   [P3] mbrenndoerfer.com "Paged Attention > Summary" -- bullet 2 (block
 *        table, one partial block per sequence), bullet 3 (K/V gathered
 *        through the table, block at a time, online softmax), bullet 4
 *        (copy-on-write sharing for beams).
 *
 * Conventions for every call:
 *   - Returns a pa_status (0 = PA_OK).  Nothing throws across the ABI.  On an
 *     error, pa_last_error() gives a message for the calling thread.
 *   - Device pointers are plain CUDA device addresses owned by the caller
 *     (e.g. allocated by PyTorch); the library allocates no device memory and
 *     keeps no pointer after a call returns (except a pa_runtime, which owns
 *     its buffers and keeps the caches it is given: see "Runtime").  Host pointers are plain host
 *     memory owned by the caller.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Device
 *     work is enqueued on it and the call returns without synchronising;
 *     argument checks that need no device data happen before anything is
 *     enqueued, so an error return means nothing was launched.
 *   - Faults found on the device (a block-table entry, slot or copy pair out
 *     of range, a pipeline wait that timed out) never trap: the kernel skips
 *     the access, sets a bit in the library's device error word and carries
 *     on.  pa_device_errors() reads that word.
 *   - All device buffers must be 16-byte aligned and contiguous in the
 *     layouts given below.
 *   - The library's own device variables (the error word, and the array of
 *     pa_decode_static) are located once per device, on the first call that
 *     needs them, and their addresses are kept.  Do not go on using the
 *     library in a process after cudaDeviceReset (or anything else that
 *     destroys the device's primary context): the kept addresses would
 *     then point into a context that no longer exists.
 *   - Supported: head_dim D in {64, 128}; block_size bs in {4, 8, 16, 32, 64};
 *     num_heads / num_kv_heads = G in 1..8; dtype f32, bf16, f16.  Anything
 *     else returns PA_ERR_UNSUPPORTED.
 */
#ifndef PAGEDATTN_H
#define PAGEDATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { PA_F32 = 0, PA_BF16 = 1, PA_F16 = 2 } pa_dtype;

typedef enum {
    PA_OK = 0,
    PA_ERR_INVALID_ARG = -1,   /* null/unaligned pointer, bad size, bad id     */
    PA_ERR_UNSUPPORTED = -2,   /* dtype, head_dim, block_size or G not built   */
    PA_ERR_OUT_OF_BLOCKS = -3, /* allocator: not enough free blocks            */
    PA_ERR_UNKNOWN_SEQ = -4,   /* allocator: no such sequence                  */
    PA_ERR_CUDA = -5,          /* a CUDA runtime call or launch failed         */
    PA_ERR_DEVICE_BOUNDS = -6, /* pa_device_errors(): the device word is set   */
    PA_ERR_SEQ_TOO_LONG = -7   /* allocator: table would exceed max_blocks     */
} pa_status;

/* Device error word bits (pa_device_errors). */
#define PA_DEVERR_TABLE 0x1u   /* block-table entry outside [0, num_blocks)   */
#define PA_DEVERR_SEQLEN 0x2u  /* seq_len < 0, > max_seq_len or > table width */
#define PA_DEVERR_SLOT 0x4u    /* slot >= num_blocks * block_size             */
#define PA_DEVERR_PAIR 0x8u    /* copy pair block outside [0, num_blocks)     */
#define PA_DEVERR_TIMEOUT 0x10u/* a pipeline wait gave up after ~2 s          */
#define PA_DEVERR_RANGE 0x20u  /* prefill variant 4, bf16 cache: a V value    */
                               /* beyond the fp16 range (non-finite rows)      */

/* Message of the last failed call on this thread ("" if none). */
const char *pa_last_error(void);

/* Library version, major*10000 + minor*100 + patch. */
int pa_version(void);

/*
 * Reads (and, if `clear`, zeroes) the device error word of the current device.
 * Synchronises the device.  Returns PA_OK when the word is 0,
 * PA_ERR_DEVICE_BOUNDS when any bit is set (bits in *flags_out if non-NULL),
 * PA_ERR_CUDA if the copy fails.
 */
int pa_device_errors(uint32_t *flags_out, int clear);

/*
 * KV append [P1 "Mechanism and details"; P2 "Separate logical order from
 * physical location"]: writes each new token's K and V rows into its slot.
 *   for t < num_tokens, h < num_kv_heads, with slot = slot_mapping[t] >= 0:
 *     k_cache[slot / bs][h][slot % bs][:] = k[t][h][:]   (same for v)
 * A negative slot skips the token.  Slots must be distinct (else which write
 * lands is unspecified).  The copy is bitwise.
 *   k, v          device, [num_tokens][num_kv_heads][head_dim], `dtype`
 *   k_cache,v_cache device, [num_blocks][num_kv_heads][block_size][head_dim]
 *   slot_mapping  device, int64 [num_tokens]
 * A slot >= num_blocks*block_size is skipped and sets PA_DEVERR_SLOT.
 */
int pa_reshape_and_cache(const void *k, const void *v, void *k_cache, void *v_cache,
                         const int64_t *slot_mapping, int num_tokens, int num_kv_heads,
                         int head_dim, int block_size, int num_blocks, int dtype, void *stream);

/*
 * Bytes of device workspace pa_decode needs for the split-context partials
 * and the tickets of their in-kernel merge: 0 when max_seq_len fits one
 * partition.  partition_size 0 means 512.  The workspace needs no clearing.
 */
size_t pa_decode_workspace_size(int num_seqs, int num_heads, int head_dim, int max_seq_len,
                                int partition_size);

/*
 * Paged decode attention [P1 "Text order is not a memory address"; P3 bullet
 * 3]: for sequence s and query head h (KV head g = h / G, G = num_heads /
 * num_kv_heads), over its tokens t < L_s = seq_lens[s]:
 *   pb = block_tables[s][t / bs], off = t % bs
 *   x_t = scale * <q[s][h], k_cache[pb][g][off]>
 *   out[s][h][:] = sum_t softmax(x)_t * v_cache[pb][g][off][:]
 * L_s == 0 gives zeros.  The context is cut into partitions of
 * `partition_size` tokens (512 by default) processed by separate CTAs; their
 * (max, sum, weighted sum) partials are merged by a second kernel (or, on
 * request, inside the main kernel: pa_decode_opt).
 *   out           device, float32 [num_seqs][num_heads][head_dim]
 *   q             device, [num_seqs][num_heads][head_dim], `dtype`
 *   k_cache,v_cache device, [num_blocks][num_kv_heads][block_size][head_dim]
 *   block_tables  device, int32 [num_seqs][max_blocks_per_seq]
 *   seq_lens      device, int32 [num_seqs]; each <= max_seq_len
 *   max_seq_len   host bound on seq_lens; sizes the grid and the workspace;
 *                 must be <= max_blocks_per_seq * block_size
 *   workspace     device, >= pa_decode_workspace_size(...) bytes (NULL if 0)
 * A seq_len above max_seq_len or the table width, or a table entry outside
 * [0, num_blocks), sets a PA_DEVERR_* bit; such a sequence's output is zero
 * (bad length) or computed with zero rows for the bad block (bad entry).
 */
int pa_decode(float *out, const void *q, const void *k_cache, const void *v_cache,
              const int32_t *block_tables, const int32_t *seq_lens, int num_seqs,
              int num_heads, int num_kv_heads, int head_dim, int block_size,
              int max_blocks_per_seq, int num_blocks, int max_seq_len, float scale, int dtype,
              void *workspace, size_t workspace_bytes, void *stream);

/*
 * pa_decode with two tuning knobs: partition_size (0 = 512; else a multiple
 * of 64 in [64, 1024]) and variant (0 = automatic; 1 = the CUDA-core kernel,
 * any dtype; 2 = the tensor-core kernel, bf16/f16 caches; 3 as for
 * pa_decode_opt).  The automatic choice (pa_decode's): fp32 caches, or a
 * cache past 2^31 rows, the CUDA-core kernel; 16-bit caches with block size
 * 8 or 16 and an even KV head count, variant 3 with two KV heads per CTA
 * when its grid (max_seq_len's splits x num_kv_heads / 2 x num_seqs) fills
 * at least one wave of the CTAs the device holds at once, else variant 2
 * (twice the CTAs for a thin batch).  Measured with 512-token splits and the
 * batch in its own order (back-to-back calls, us): Llama-8B-shaped 50.6
 * against 58.6 for variant 2, long context 167.8 against 172.5, the
 * continuous mix 187.1 against 189.8.
 */
int pa_decode_ex(float *out, const void *q, const void *k_cache, const void *v_cache,
                 const int32_t *block_tables, const int32_t *seq_lens, int num_seqs,
                 int num_heads, int num_kv_heads, int head_dim, int block_size,
                 int max_blocks_per_seq, int num_blocks, int max_seq_len, float scale,
                 int dtype, void *workspace, size_t workspace_bytes, int partition_size,
                 int variant, void *stream);

/*
 * pa_decode with every tuning choice in one struct (pa_decode_ex is this
 * call with merge 0).  Fields, 0 meaning the library's choice:
 *   partition_size  tokens per split, as for pa_decode_ex
 *   variant         0 automatic, 1 CUDA cores, 2 tensor cores (as pa_decode_ex),
 *                   3 tensor cores, one KV head per warp (below)
 *   merge           how a sequence's split partials are combined:
 *                   1 a separate reduce kernel (one CTA per (sequence, head));
 *                   2 inside the main kernel: the CTA of a (sequence, KV head)
 *                     to finish last merges that pair's partials, found with
 *                     a ticket word in the workspace (no further launch);
 *                   0 the library's choice: the first (the in-kernel merge
 *                     costs each split CTA a fence and a ticket round trip
 *                     before its slot frees, and measured no faster)
 *   heads_per_cta   variant 3 only: KV heads per CTA (1, 2 or 4; 0 = the
 *                   library's choice)
 *   seq_order       device int32 [num_seqs] or NULL: the order in which the
 *                   grid takes the sequences, a permutation of 0 .. num_seqs-1
 *                   (an entry outside that range skips its grid row and
 *                   sets PA_DEVERR_SEQLEN; a sequence no grid row names is
 *                   left unwritten, or with several splits merged from
 *                   stale partials).  The kernels' CTAs start roughly in grid
 *                   order, so longest first (what pa_step_plan writes and
 *                   pa_decode_order computes) puts short CTAs at the end of
 *                   the launch, where they fill the tail; out keeps the
 *                   batch's order whatever the order given.
 *   reserved        must be 0
 * Variant 3 is the tensor-core kernel with one KV head per consumer warp: a
 * CTA takes heads_per_cta adjacent KV heads of one (sequence, partition),
 * needs num_kv_heads divisible by it and heads_per_cta * max(16,
 * block_size) <= 64, and has no merge across its warps.
 * The tickets carry a tag that changes with every call, so the workspace
 * never needs clearing; a call that replays with the same tag (a CUDA graph)
 * finds its tickets reset by its own previous run.  Results agree with the
 * other merge within fp32 rounding.  Calls sharing one workspace must not
 * overlap on the GPU (as for the partials themselves).
 */
typedef struct {
    int partition_size;
    int variant;
    int merge;
    int heads_per_cta;
    const int32_t *seq_order;
    int reserved[4];
} pa_decode_opts;

/*
 * A decode step's append and attention in one launch [P1 "Mechanism and
 * details": a new token goes into its sequence's last block; P3 bullet 3]:
 * every sequence s appends one token, at position seq_lens[s] - 1, whose K
 * and V rows are k_new[s] and v_new[s] ([num_seqs][num_kv_heads][head_dim],
 * `dtype`, device) and whose slot is slot_mapping[s] (device int64); then
 * out is pa_decode_opt's result over seq_lens[s] tokens, the new one
 * included.  The CTA of each (sequence, KV head) whose partition holds the
 * new position writes that head's rows into the caches before it reads the
 * block (so the step needs no separate pa_reshape_and_cache launch).
 *   - A slot must be the one the table gives position seq_lens[s] - 1 (as
 *     the allocator's append returns it); another slot is not written and
 *     sets PA_DEVERR_SLOT.  A negative slot writes nothing.
 *   - A copy-on-write copy for the step (pa_copy_blocks) must come before
 *     this call on the stream; a sequence with seq_lens[s] == 0 appends
 *     nothing.
 * Same arguments otherwise, same results and errors as pa_decode_opt.
 */
int pa_append_decode(float *out, const void *q, const void *k_new, const void *v_new,
                     const int64_t *slot_mapping, void *k_cache, void *v_cache,
                     const int32_t *block_tables, const int32_t *seq_lens, int num_seqs,
                     int num_heads, int num_kv_heads, int head_dim, int block_size,
                     int max_blocks_per_seq, int num_blocks, int max_seq_len, float scale,
                     int dtype, void *workspace, size_t workspace_bytes,
                     const pa_decode_opts *opts, void *stream);

/*
 * The kernel, split length and heads per CTA for a decode batch, from the
 * lengths as the caller knows them on the host; fills opts->partition_size,
 * ->variant and ->heads_per_cta and leaves the other fields.  Measured on
 * B200 with the grid taking the sequences longest first:
 *   - fp32 caches: the CUDA-core kernel, pa_decode_partition_for's split;
 *   - 16-bit caches, block size 8 or 16, an even KV head count: variant 3
 *     with two KV heads per CTA (it matched or beat variant 2 on every batch
 *     measured, once its split fits the batch), and the split by the share
 *     of a wave it fills: the shortest of 256, 384, 512, 640, 768, 1024
 *     tokens whose CTAs ((num_kv_heads / 2) x the splits of each sequence)
 *     fill at most 0.85 of `slots`; if even 1024 fills more, 1024 when its
 *     CTAs fit in `slots`, else 512.  (Measured as first-to-last CTA spans:
 *     beam search, 16 sequences of ~2070 tokens: 256; Llama-8B-shaped, 32
 *     sequences of U[512, 4096]: 512, 48.8 us against 49.6 at 384 (0.95 of a
 *     wave) and 50.6 at 640; 64 such sequences: 1024, within 1.3% of the best
 *     split; long context and the continuous mix: 512.)
 *   - otherwise variant 2 with pa_decode_partition_for's split.
 * slots: CTAs resident at once; 0 asks the device (the chosen kernel's
 * occupancy times the SM count).  Host only.
 */
int pa_decode_choose(const int32_t *seq_lens_host, int num_seqs, int num_kv_heads,
                     int head_dim, int block_size, int dtype, int slots, pa_decode_opts *opts);

/*
 * Longest-first order of a decode batch for pa_decode_opts.seq_order, from
 * the lengths as the caller knows them on the host: order_out[i] is the
 * batch row of the i-th longest sequence, ties in batch order.  Host only.
 *   seq_lens_host  host int32 [num_seqs];  order_out  host int32 [num_seqs]
 */
int pa_decode_order(const int32_t *seq_lens_host, int num_seqs, int32_t *order_out);

int pa_decode_opt(float *out, const void *q, const void *k_cache, const void *v_cache,
                  const int32_t *block_tables, const int32_t *seq_lens, int num_seqs,
                  int num_heads, int num_kv_heads, int head_dim, int block_size,
                  int max_blocks_per_seq, int num_blocks, int max_seq_len, float scale,
                  int dtype, void *workspace, size_t workspace_bytes,
                  const pa_decode_opts *opts, void *stream);

/*
 * A partition_size for pa_decode_ex, from the sequence lengths as the caller
 * knows them on the host (a runtime does: it owns the block tables).  The
 * decode launches one CTA per (sequence, KV head, partition); when the 512-
 * token default gives between one and two waves of the CTAs the device holds
 * at once, the second wave runs part-empty and the kernel's tail grows.  In
 * that case the result is 1024 if its CTAs fit one wave.  It is 1024 too when
 * the longest sequence exceeds 512 tokens and twice the shortest: the rule
 * assumes the grid takes the sequences longest first (pa_decode_order),
 * whose short CTAs at the end fill the tail, so that fewer, longer splits
 * save start-ups and partials.  Otherwise it is 512.
 * (One alternative only: a runtime that keys CUDA graphs on the split length
 * then sees it change rarely as its sequences grow.)
 *   seq_lens_host   host, int32 [num_seqs], each >= 0 (a 0 counts as one CTA)
 *   slots           CTAs resident at once; 0 = ask the device for the
 *                   tensor-core kernel's occupancy of this shape times the
 *                   SM count (the CUDA-core kernel, fp32 or block_size 4,
 *                   always gets 512)
 * Returns the partition size (> 0), or a negative pa_status on bad arguments
 * or, with slots == 0, when the device cannot be queried.  Host only; it
 * launches nothing.
 */
int pa_decode_partition_for(const int32_t *seq_lens_host, int num_seqs, int num_kv_heads,
                            int head_dim, int block_size, int dtype, int slots);

/*
 * Multi-token (chunked prefill) attention over the paged cache [P1
 * "Mechanism and details": new positions are appended after the prefix,
 * whose blocks stay in place; P3 bullet 3: attention reads K/V through the
 * block table].  For sequence s the query rows are q[cu_q_lens[s] ..
 * cu_q_lens[s+1]): the last n_s = cu_q_lens[s+1] - cu_q_lens[s] positions of
 * the sequence, L_s - n_s .. L_s - 1 (their K/V already appended with
 * pa_reshape_and_cache).  Row r at position p attends causally to the
 * sequence's tokens 0..p:
 *   out[r][h][:] = sum_{t<=p} softmax_t(scale * <q[r][h], k_t>) v_t
 * (the decode is the case n_s = 1).
 *   out           device, float32 [total][num_heads][head_dim], total = cu_q_lens[B]
 *   q             device, [total][num_heads][head_dim], `dtype` (bf16/f16)
 *   cu_q_lens     device, int32 [num_seqs + 1], non-decreasing, cu_q_lens[0] = 0
 *   seq_lens      device, int32 [num_seqs]: L_s including the chunk
 *   max_q_len     host bound on n_s; max_seq_len host bound on L_s
 * block_size >= 8 and a 16-bit dtype; fp32 caches return PA_ERR_UNSUPPORTED.
 * n_s < 0, n_s > L_s or a bound exceeded leaves the sequence's rows
 * unwritten and sets PA_DEVERR_SEQLEN.
 */
int pa_prefill(float *out, const void *q, const void *k_cache, const void *v_cache,
               const int32_t *block_tables, const int32_t *seq_lens, const int32_t *cu_q_lens,
               int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
               int max_blocks_per_seq, int num_blocks, int max_q_len, int max_seq_len,
               float scale, int dtype, void *stream);

/*
 * pa_prefill with a choice of kernel:
 *   0  automatic: the tcgen05 kernel (pa_prefill uses it);
 *   1  the mma.sync kernel: 64 (token, head) rows per CTA, accumulators in
 *      registers;
 *   2  the tcgen05 kernel: 128 rows per CTA; Q, S = Q K^T, P and O = P V held
 *      in tensor memory, the MMAs issued by two threads;
 *   3  the same kernel persistent: one CTA per SM walks its share of the
 *      128-row tiles (in the order of kernel 2's grid), the
 *      next tile's Q going into a second TMEM buffer and its first products
 *      starting while the current tile's output is written;
 *   4  kernel 2 with the weights P entering the P V product as one fp16 per
 *      weight (kernels 1-3 carry a 16-bit high part and its remainder, two
 *      products): half the P V work.  A bf16 cache's V stages are converted
 *      to fp16 in shared memory by a fourth warpgroup (512 threads).  Each
 *      weight is then within 2^-11 of its value (2^-25 absolute below
 *      2^-14), against 2^-14 for kernels 2 and 3, so the output error bound
 *      grows to about 2^-11 * max|v|: within 3e-3 while |v| <= 6.  A bf16 V
 *      value of magnitude 65536 or more (beyond the fp16 range) makes its
 *      tile's rows non-finite and sets PA_DEVERR_RANGE; f16 caches have no
 *      such case.  Measured on 8 x (4096 + 1024) rows, 32/8 heads, D 128:
 *      0.733 ms vs 0.788 (bf16) and 0.683 vs 0.803 (f16) in 20-launch
 *      bursts, 11-18% faster in one-second loops at the power cap.
 * Same arguments, results (within the stated rounding) and errors as
 * pa_prefill; another variant returns PA_ERR_INVALID_ARG.  All kernels need
 * all of a sequence's table entries for positions < L_s to be valid blocks
 * (an entry outside [0, num_blocks) reads as zeros and sets
 * PA_DEVERR_TABLE).
 */
int pa_prefill_ex(float *out, const void *q, const void *k_cache, const void *v_cache,
                  const int32_t *block_tables, const int32_t *seq_lens, const int32_t *cu_q_lens,
                  int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
                  int max_blocks_per_seq, int num_blocks, int max_q_len, int max_seq_len,
                  float scale, int dtype, int variant, void *stream);

/*
 * pa_decode for callers that cannot allocate device memory.  The paper has no
 * counterpart: this is a deployment variant of pa_decode.
 *
 * Some callers can't call cudaMalloc or take a caller-sized workspace: code
 * inside a host runtime that owns every device allocation, plug-ins for which
 * an allocation (and the synchronisation it may imply) mid-step is not
 * allowed, or paths where an out-of-memory error cannot be handled.  This
 * call takes the same arguments as pa_decode minus the workspace and keeps
 * the split partials in a fixed 32 MiB array inside the library's device
 * image (a file-scope __device__ array, held by every GPU that loads the
 * library until the process exits).  It calls no cudaMalloc, cudaFree or
 * other allocating routine.
 *   - Limit: pa_decode_workspace_size(num_seqs, num_heads, head_dim,
 *     max_seq_len, 0) must be <= 32 MiB (e.g. 8 sequences x 64 heads x 32768
 *     tokens at head_dim 128 need 17 MB); larger requests return
 *     PA_ERR_INVALID_ARG before anything is launched.
 *   - The first call on a device looks up the array's device address (with
 *     that device current) and keeps it; make that first call before any
 *     stream capture, and do not use the call after cudaDeviceReset.
 *   - Every call shares the one array and it keeps the last call's contents;
 *     nothing in it needs to start at zero.  Calls that overlap on the GPU
 *     (e.g. on two streams at once) race on it: serialise them.
 * Output and device error behaviour are those of pa_decode.
 */
int pa_decode_static(float *out, const void *q, const void *k_cache, const void *v_cache,
                     const int32_t *block_tables, const int32_t *seq_lens, int num_seqs,
                     int num_heads, int num_kv_heads, int head_dim, int block_size,
                     int max_blocks_per_seq, int num_blocks, int max_seq_len, float scale,
                     int dtype, void *stream);

/*
 * Copy-on-write block copy [P2 "Sharing needs ownership rules"; P3 bullet 4]:
 * for each pair i, copies physical block src_dst_pairs[2i] onto block
 * src_dst_pairs[2i+1] in both caches, all heads and positions, bitwise.
 * Pairs act together: no destination may also be a source or repeat.
 *   src_dst_pairs device, int64 [num_pairs][2]
 *   block_bytes   num_kv_heads * block_size * head_dim * element size
 * A block id outside [0, num_blocks) skips the pair and sets PA_DEVERR_PAIR.
 */
int pa_copy_blocks(void *k_cache, void *v_cache, const int64_t *src_dst_pairs, int num_pairs,
                   size_t block_bytes, int num_blocks, void *stream);

/*
 * Block copy between two caches of the same block shape [P2 "What this does
 * not solve": preemption; the swap of a sequence's blocks]: for each pair i,
 * block src_dst_pairs[2i] of (src_k, src_v) is copied onto block
 * src_dst_pairs[2i+1] of (dst_k, dst_v), bitwise.  Each cache may be device
 * memory or page-locked host memory (pinned with cudaHostAlloc /
 * cudaHostRegister and mapped: the kernel reads or writes it over the bus);
 * src_dst_pairs likewise.  Any other host pointer returns PA_ERR_INVALID_ARG.
 * A block id outside [0, num_src_blocks) / [0, num_dst_blocks) skips the pair
 * and sets PA_DEVERR_PAIR.
 */
int pa_swap_blocks(void *dst_k, void *dst_v, const void *src_k, const void *src_v,
                   const int64_t *src_dst_pairs, int num_pairs, size_t block_bytes,
                   int num_src_blocks, int num_dst_blocks, void *stream);

/*
 * Measurement hook: when both events are non-NULL, the next pa_decode /
 * pa_decode_ex calls on this thread record ev_begin (a cudaEvent_t) before
 * their main kernel and ev_end after it, on the call's stream.  Pass NULLs
 * to stop.
 */
int pa_set_profile_events(void *ev_begin, void *ev_end);

/*
 * Self-test of the bounded pipeline wait that every TMA / tensor-core kernel
 * of this library uses (no counterpart on the pages: failure detection).
 * One CTA waits on an mbarrier phase that nothing completes.  The wait must
 * give up after limit_ns, or as soon as a second warp of the CTA sets the
 * abort flag (after abort_after_ns; 0 = never), then set PA_DEVERR_TIMEOUT in
 * the device error word and return; the CUDA context stays usable.
 *   limit_ns        (0, 10^10]
 *   elapsed_ns      device, one uint64: nanoseconds the wait took
 * Returns PA_ERR_INVALID_ARG for a limit out of range or a NULL elapsed_ns,
 * PA_ERR_CUDA if the launch fails.  Asynchronous on `stream`.
 */
int pa_selftest_wait(uint64_t limit_ns, uint64_t abort_after_ns, unsigned long long *elapsed_ns,
                     void *stream);

/* ------------------------------------------------------------------------
 * Host block allocator [P1 "Mechanism and details"; P2 "Separate logical
 * order from physical location", "Sharing needs ownership rules", "Exercise
 * and checkpoint", "What this does not solve"; P3 bullets 2 and 4].
 * Pure host code: no CUDA call, usable without a GPU.  Not thread-safe: one
 * handle per thread, or external locking.
 *
 * Policy (what the pages leave open is fixed here):
 *   - free list: FIFO queue initialised with free_order (NULL = 0..n-1);
 *     blocks are taken from the head and returned to the tail;
 *   - append: a block is taken when a token lands at position p with
 *     p % bs == 0; slot = table[p / bs] * bs + p % bs;
 *   - copy-on-write: at the first token of an append, if the last block is
 *     partially filled and shared (refcount > 1), the sequence takes a fresh
 *     block (before any other block of that append), the pair (old, new) is
 *     reported and the old block's refcount drops; the last owner writes in
 *     place;
 *   - fork: the child shares the parent's blocks (refcounts + 1);
 *   - free: blocks are released in ascending logical order; a block whose
 *     refcount reaches 0 goes to the free-list tail;
 *   - an append needing more free blocks than exist returns
 *     PA_ERR_OUT_OF_BLOCKS, one needing more than max_blocks_per_seq table
 *     entries returns PA_ERR_SEQ_TOO_LONG; neither changes any state.
 * ---------------------------------------------------------------------- */
typedef struct pa_alloc pa_alloc;

typedef struct {
    int64_t num_blocks;
    int64_t free_blocks;
    int64_t used_blocks;     /* refcount > 0              */
    int64_t shared_blocks;   /* refcount > 1              */
    int64_t num_seqs;
    int64_t table_entries;   /* sum of table lengths      */
    int64_t logical_tokens;  /* sum of sequence lengths   */
    int64_t reserved_slots;  /* used_blocks * block_size  */
    int64_t cached_blocks;        /* full blocks in the prefix index       */
    int64_t prefix_hit_blocks;    /* blocks reused by pa_seq_add_cached    */
    int64_t prefix_query_blocks;  /* full blocks looked up by it           */
    int64_t evicted_blocks;       /* indexed blocks handed out again       */
    int64_t host_blocks;          /* host pool size (pa_alloc_set_host_pool) */
    int64_t host_free_blocks;
    int64_t swapped_seqs;
} pa_alloc_stats_t;

/* max_blocks_per_seq 0 = unlimited.  free_order: host int32[num_blocks], a
 * permutation of 0..num_blocks-1, copied; NULL = identity. */
int pa_alloc_create(pa_alloc **out, int num_blocks, int block_size, int max_blocks_per_seq,
                    const int32_t *free_order);
void pa_alloc_destroy(pa_alloc *a);

/* New empty sequence; PA_ERR_INVALID_ARG if the id exists. */
int pa_seq_add(pa_alloc *a, int64_t seq_id);

/* Reserves slots for the next n_tokens positions.  slots_out: host
 * int64[n_tokens].  cow_pair_out: host int64[2] or NULL; *n_cow_out (if
 * non-NULL) receives 0 or 1.  n_tokens == 0 does nothing. */
int pa_seq_append(pa_alloc *a, int64_t seq_id, int n_tokens, int64_t *slots_out,
                  int64_t *cow_pair_out, int *n_cow_out);

/* Appends n_tokens[i] (all 1 if n_tokens is NULL) to seq_ids[i], in order.
 * slots_out: host int64[sum of tokens], in order; cow_pairs_out: host
 * int64[2*n_seqs] or NULL; *n_cow_out receives the pair count.  All or
 * nothing: on an error every earlier append of the batch is undone. */
int pa_batch_append(pa_alloc *a, const int64_t *seq_ids, int n_seqs, const int32_t *n_tokens,
                    int64_t *slots_out, int64_t *cow_pairs_out, int *n_cow_out);

int pa_seq_fork(pa_alloc *a, int64_t parent, int64_t child);
int pa_seq_free(pa_alloc *a, int64_t seq_id);

/* Copies up to `cap` table entries into out (host int32); *n_out = table
 * length, *len_out = sequence length (either may be NULL). */
int pa_seq_block_table(const pa_alloc *a, int64_t seq_id, int32_t *out, int cap, int *n_out,
                       int64_t *len_out);

/* Rows of a decode batch: tables_out host int32[n_seqs][width], entries past
 * a table's length set to 0; seq_lens_out host int32[n_seqs].  Returns
 * PA_ERR_SEQ_TOO_LONG if a table is longer than width. */
int pa_block_tables(const pa_alloc *a, const int64_t *seq_ids, int n_seqs, int32_t *tables_out,
                    int width, int32_t *seq_lens_out);

/* ------------------------------------------------------------------------
 * One decode step planned in one call.  The pages leave the runtime that
 * owns the block tables to hand the device what a step needs (sanketn26
 * "PagedAttention", "Use a runtime that owns the blocks": the runtime, not
 * the client, keeps the tables and the allocation).  pa_step_plan applies a
 * step's events to the allocator in order and writes everything the device
 * work of the step reads -- the slots of the appended tokens, the
 * copy-on-write pairs, and the decode batch's table rows and lengths -- into
 * one caller-given host buffer (page-locked, typically), so that the step
 * crosses to the device in one copy.
 *
 * Events: n_events triples {code, x, y} of int64, applied in order:
 *   {PA_EV_ADD, seq_id, 0}      pa_seq_add
 *   {PA_EV_FREE, seq_id, 0}     pa_seq_free
 *   {PA_EV_FORK, parent, child} pa_seq_fork
 *   {PA_EV_APPEND, seq_id, n}   n new tokens (pa_seq_append); a run of
 *                               consecutive appends is all or nothing, as in
 *                               pa_batch_append
 *   {PA_EV_DECODE, 0, 0}        at most one: the decode batch decode_ids
 *                               [num_seqs] is read here, after the events
 *                               before it and before those after it
 * Stage layout (byte offsets in *out, each 16-byte aligned; they depend only
 * on the events' kinds and token counts and on num_seqs and width, not on
 * what the allocator decides):
 *   off_slots   int64 [n_slots]          slots of every appended token, in
 *                                        event order (n_slots_pre of them
 *                                        before the decode event)
 *   off_pairs   int64 [n_pairs][2]       copy-on-write (src, dst) pairs, in
 *                                        event order (room for one per append
 *                                        event; n_pairs_pre before the decode)
 *   off_tables  int32 [num_seqs][width]  table rows as of the decode event;
 *                                        entries past a table's length are
 *                                        left as the buffer held them (no
 *                                        kernel reads them)
 *   off_lens    int32 [num_seqs]         lengths, as of the decode event
 *   off_order   int32 [num_seqs]         the batch rows longest first (ties
 *                                        in batch order), for
 *                                        pa_decode_opts.seq_order
 *   bytes       end of the last array
 * The device work of the step then follows the events' order: for each run
 * of consecutive appends its copies, then its rows; the decode at its place
 * -- so that blocks freed and reused after the decode are not written
 * before the decode reads them.
 * pairs_before (host int32 [n_events + 1], or NULL) receives, for each
 * event, the number of pairs the events before it produced, and the total
 * last: the pairs of events [i, j) are [pairs_before[i], pairs_before[j]).
 * A caller that keeps the order of the step's events on the device splits
 * the appends into runs at every other event, like the op-by-op calls would
 * (a fork or a free between two appends can make a later copy read, or a
 * later append reuse, a block written by an earlier one).
 * stage NULL: only the layout is computed (nothing is applied).  Errors: an
 * unknown code, more than one decode event, a bad count, or a stage smaller
 * than out->bytes return PA_ERR_INVALID_ARG before anything is applied; an
 * event that fails stops the call with its error, out->events_applied = the
 * index of the first event not applied (for a run of appends, the run's
 * first event), everything before it stays applied.
 */
#define PA_EV_ADD 1
#define PA_EV_FREE 2
#define PA_EV_FORK 3
#define PA_EV_APPEND 4
#define PA_EV_DECODE 5

typedef struct {
    int32_t n_slots;        /* appended tokens in the step */
    int32_t n_slots_pre;    /* of which before the decode event */
    int32_t n_pairs;        /* copy-on-write pairs */
    int32_t n_pairs_pre;    /* of which before the decode event */
    int32_t num_seqs;       /* decode batch rows */
    int32_t width;          /* table entries per row */
    int32_t max_seq_len;    /* longest length in the decode batch */
    int32_t events_applied; /* events applied (all of them on success) */
    int64_t off_slots, off_pairs, off_tables, off_lens, off_order, bytes;
} pa_step_layout;

int pa_step_plan(pa_alloc *a, const int64_t *events, int n_events, const int64_t *decode_ids,
                 int num_seqs, int width, void *stage, size_t stage_bytes,
                 int32_t *pairs_before, pa_step_layout *out);

/* ------------------------------------------------------------------------
 * A host-fed step's device work in one call: the executor a runtime uses
 * once a step's kernels are a CUDA graph (not from the pages; it is how the
 * runtime of sanketn26 "Use a runtime that owns the blocks" keeps its host
 * work per step small).  In order:
 *   stream_in:  waits for wait_before_in (if non-NULL: e.g. the last use of
 *               the staging buffer), runs the copies (one cudaMemcpyAsync
 *               host-to-device each; page-locked sources copy asynchronously),
 *               records event_in;
 *   stream_run: waits for event_in and wait_before_run (if non-NULL: e.g. the
 *               previous output copy of this graph), launches graph_run (a
 *               cudaGraphExec_t), records event_run;
 *   stream_out: if graph_out is non-NULL, waits for event_run, launches
 *               graph_out, records event_out.
 * Streams are cudaStream_t, events cudaEvent_t, graphs cudaGraphExec_t, all
 * the caller's.  Returns PA_ERR_CUDA if a call fails (work enqueued before it
 * stays enqueued), PA_ERR_INVALID_ARG on a NULL event or graph.
 * ---------------------------------------------------------------------- */
typedef struct {
    void *dst;       /* device */
    const void *src; /* host */
    size_t bytes;    /* 0 skips the entry */
} pa_host_copy;

int pa_step_launch(void *stream_in, void *stream_run, void *stream_out,
                   const pa_host_copy *copies, int n_copies, void *wait_before_in,
                   void *event_in, void *graph_run, void *wait_before_run, void *event_run,
                   void *graph_out, void *event_out);

/* ------------------------------------------------------------------------
 * Runtime: a decode runtime around the calls above, one call per host-fed
 * step (the pages leave tables and allocation to a runtime that owns them:
 * sanketn26 "PagedAttention", "Use a runtime that owns the blocks").
 *
 * pa_rt_create makes one for caller-owned caches k_cache, v_cache ([NB][Hkv]
 * [bs][D], `dtype`, device, left as they are) with its own allocator
 * (free_order as for pa_alloc_create).  Unlike the rest of the library it
 * owns device memory: two staging buffers (arrays + the largest step's new
 * K/V rows and queries), the split workspace, two output buffers, plus two
 * page-locked host buffers, three non-blocking streams and its CUDA graphs;
 * pa_rt_destroy waits for its streams and frees them.
 *
 * pa_rt_step takes a step's events as pa_step_plan does (decode_ids: the
 * decode batch), its new K/V rows k_new, v_new (host, [n new tokens][Hkv][D],
 * in event order), its queries q (host, [num_seqs][Hq][D]) and a host output
 * buffer out (float32 [num_seqs][Hq][D]); host buffers should be page-locked
 * (the copies are asynchronous).  It applies the events (pa_step_plan),
 * chooses the decode (pa_decode_choose, longest first; one-token appends of
 * exactly the decode batch go in with it, pa_append_decode), copies the
 * step's inputs in on one stream (the new rows and the queries first: they
 * need nothing from the plan, so the host link carries them while the host
 * plans; then the step's arrays), runs its kernels on another (from a CUDA
 * graph of the step's layout once that layout has run once; steps with
 * copy-on-write copies run directly) and copies the output out on a third.
 * It returns at once; *ready (if non-NULL) receives a cudaEvent_t that
 * completes once out holds the step's output and the inputs have been read.
 * Steps alternate between two staging slots: a step's host work (this call)
 * overlaps the previous step's kernels, and the call waits only for the copy
 * in of the step two back.  Keep the inputs unchanged and do not read out
 * until *ready completes.
 *   - Limits: num_seqs <= max_batch, new tokens <= max_new_tokens, table rows
 *     of table_width entries; beyond them PA_ERR_INVALID_ARG before anything
 *     is applied.  Errors of pa_step_plan are returned as it returns them; a
 *     call that fails after its input copies were enqueued waits for them
 *     before it returns, so the caller may reuse its buffers at once.
 *   - A CUDA error part-way leaves the runtime's allocator ahead of its
 *     device work: destroy the runtime.
 * pa_rt_wait synchronises the runtime's streams; pa_event_wait waits for an
 * event (e.g. *ready); pa_rt_allocator gives its allocator (for queries and
 * for ops the events do not cover); pa_rt_stats counts steps, graph replays
 * and captures.
 * ---------------------------------------------------------------------- */
typedef struct pa_runtime pa_runtime;

typedef struct {
    int num_blocks, block_size, num_heads, num_kv_heads, head_dim, dtype;
    int table_width;         /* table entries per decode row */
    int max_batch;           /* decode rows per step */
    int max_new_tokens;      /* appended tokens per step */
    int max_blocks_per_seq;  /* the allocator's bound, 0 = none */
    float scale;
} pa_runtime_config;

int pa_rt_create(pa_runtime **out, const pa_runtime_config *cfg, void *k_cache, void *v_cache,
                 const int32_t *free_order);
void pa_rt_destroy(pa_runtime *rt);
pa_alloc *pa_rt_allocator(pa_runtime *rt);
int pa_rt_step(pa_runtime *rt, const int64_t *events, int n_events, const int64_t *decode_ids,
               int num_seqs, const void *k_new, const void *v_new, const void *q, float *out,
               void **ready);
int pa_rt_wait(pa_runtime *rt);
int pa_event_wait(void *event);
int pa_rt_stats(const pa_runtime *rt, int64_t *steps, int64_t *replays, int64_t *captures);

int pa_alloc_stats(const pa_alloc *a, pa_alloc_stats_t *out);

/* Free list from head to tail into out (host int32, up to cap); *n_out =
 * its length. */
int pa_alloc_free_list(const pa_alloc *a, int32_t *out, int cap, int *n_out);

/* Refcount of one physical block (-1 if out of range). */
int pa_alloc_refcount(const pa_alloc *a, int block);

/* ------------------------------------------------------------------------
 * Prefix caching [P1 "Text order is not a memory address", last paragraph:
 * block sharing is useful for prefix caching; P2 "Use a runtime that owns the
 * blocks": prefix reuse inside a paged runtime].
 *
 * A full block whose token ids are known is indexed by (the physical block
 * holding the preceding tokens, or -1 for the first block; its bs token ids).
 * Matching is exact (no hash collisions).  A block enters the index when an
 * append by pa_seq_append_tokens fills it, unless an identical block is
 * indexed already.  Released blocks stay indexed while they wait in the free
 * list; taking a block from the free list for new use drops it from the
 * index ("evicted").  A prefix match on a block in the free list takes it
 * out of the free list (wherever it is) and gives it refcount 1.
 * ---------------------------------------------------------------------- */

/* New sequence whose first n_tokens token ids are token_ids: shares the
 * longest chain of indexed full blocks matching its leading tokens (at most
 * n_tokens / bs blocks) and starts with that many tokens in place;
 * *n_cached_out = matched blocks * bs.  The caller appends the rest with
 * pa_seq_append_tokens (and writes their K/V).  Never allocates, never fails
 * for lack of blocks. */
int pa_seq_add_cached(pa_alloc *a, int64_t seq_id, const int64_t *token_ids, int n_tokens,
                      int *n_cached_out);

/* pa_seq_append for a sequence made by pa_seq_add_cached (or forked from
 * one): same slots and copy-on-write rule, and every block the append fills
 * enters the prefix index.  PA_ERR_INVALID_ARG for other sequences.  (A plain
 * pa_seq_append on such a sequence ends its token history.) */
int pa_seq_append_tokens(pa_alloc *a, int64_t seq_id, const int64_t *token_ids, int n_tokens,
                         int64_t *slots_out, int64_t *cow_pair_out, int *n_cow_out);

/* ------------------------------------------------------------------------
 * Preemption by swap [P2 "What this does not solve": excess admission can
 * cause preemption; P3 bullet 5].  A pool of host blocks (same block shape)
 * with its own FIFO free list (identity order).  Swapping a sequence out
 * moves every block of its table to a host block, in logical order, and
 * releases the device blocks (a block shared with another sequence keeps its
 * other owners); swapping in takes fresh device blocks from the free list.
 * Swapped-out sequences can only be swapped in or freed.  The data moves with
 * pa_swap_blocks, using the returned pairs; run the swap-out copy before any
 * later write can reuse the released device blocks (same stream).
 * ---------------------------------------------------------------------- */

/* Sets the host pool size (host blocks 0..n-1, all free).  Fails while a
 * sequence is swapped out. */
int pa_alloc_set_host_pool(pa_alloc *a, int num_host_blocks);

/* pairs_out: host int64[cap][2] of (device block, host block), one per table
 * entry in logical order; PA_ERR_OUT_OF_BLOCKS (no change) when the host
 * pool is short. */
int pa_seq_swap_out(pa_alloc *a, int64_t seq_id, int64_t *pairs_out, int cap, int *n_pairs_out);

/* pairs_out: host int64[cap][2] of (host block, device block); PA_ERR_OUT_OF_
 * BLOCKS (no change) when the device free list is short. */
int pa_seq_swap_in(pa_alloc *a, int64_t seq_id, int64_t *pairs_out, int cap, int *n_pairs_out);

#ifdef __cplusplus
}
#endif
#endif /* PAGEDATTN_H */
