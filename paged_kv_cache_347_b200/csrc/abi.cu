// The C ABI of pagedattn.h for the device calls: argument checks, workspace
// layout, kernel choice and launch.  The allocator's half of the ABI is in
// allocator.cpp.
#include <cuda_runtime.h>

#include <atomic>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/pagedattn.h"
#include "launch.h"
#include "status.h"

namespace pa {

char *error_buffer() {
    static thread_local char buf[512];
    return buf;
}

// The device error word (one per device that loads the library).
__device__ unsigned int g_device_error = 0;

constexpr int kMaxDevices = 64;

static int current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    return dev;
}

static unsigned int *device_error_ptr() {
    static std::atomic<unsigned int *> ptrs[kMaxDevices];
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return nullptr;
    unsigned int *p = ptrs[dev].load(std::memory_order_acquire);
    if (!p) {
        void *a = nullptr;
        if (cudaGetSymbolAddress(&a, g_device_error) != cudaSuccess) return nullptr;
        p = static_cast<unsigned int *>(a);
        ptrs[dev].store(p, std::memory_order_release);
    }
    return p;
}

int num_sms() {
    static std::atomic<int> cache[kMaxDevices];
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return 148;
    int n = cache[dev].load(std::memory_order_relaxed);
    if (n <= 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cache[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

struct ProfileEvents {
    cudaEvent_t begin = nullptr, end = nullptr;
};
static thread_local ProfileEvents t_prof;

static int elem_bytes(int dtype) { return dtype == PA_F32 ? 4 : 2; }

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static int cuda_fail(cudaError_t e, const char *what) {
    return fail(PA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

static int check_shape(int num_kv_heads, int head_dim, int block_size, int dtype) {
    if (dtype != PA_F32 && dtype != PA_BF16 && dtype != PA_F16)
        return fail(PA_ERR_UNSUPPORTED, "dtype %d not supported", dtype);
    if (head_dim != 64 && head_dim != 128)
        return fail(PA_ERR_UNSUPPORTED, "head_dim %d not supported (64, 128)", head_dim);
    if (block_size != 4 && block_size != 8 && block_size != 16 && block_size != 32 &&
        block_size != 64)
        return fail(PA_ERR_UNSUPPORTED, "block_size %d not supported (4, 8, 16, 32, 64)",
                    block_size);
    if (num_kv_heads <= 0 || num_kv_heads > 65535)
        return fail(PA_ERR_INVALID_ARG, "num_kv_heads %d", num_kv_heads);
    return PA_OK;
}

constexpr int kDefaultPartition = 512;
// pa_prefill's kernel: 1 = mma.sync (registers), 2 = tcgen05 (TMEM).
constexpr int kPrefillDefault = 2;

static int partition_or_default(int partition_size) {
    return partition_size == 0 ? kDefaultPartition : partition_size;
}

// Splits of `partition` tokens covering max_seq_len (in 64-bit: max_seq_len
// may be close to INT_MAX).
static int splits_for(int max_seq_len, int partition) {
    return max_seq_len <= 0 ? 1 : (int)(((int64_t)max_seq_len + partition - 1) / partition);
}

// CTAs of the two-head variant-3 kernel resident at once on the current
// device (its occupancy, asked once per device and shape, times the SMs), or
// a negative status.
static int hw2_slots(int dtype, int head_dim, int block_size) {
    static std::atomic<int> cache[kMaxDevices][2][2][2];
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return fail(PA_ERR_CUDA, "no CUDA device");
    std::atomic<int> &c = cache[dev][dtype == PA_F16][head_dim == 128][block_size == 16];
    int per_sm = c.load(std::memory_order_relaxed);
    if (per_sm <= 0) {
        per_sm = decode_hw2_resident_per_sm(dtype, head_dim, block_size);
        if (per_sm <= 0) return fail(PA_ERR_CUDA, "occupancy query failed");
        c.store(per_sm, std::memory_order_relaxed);
    }
    return per_sm * num_sms();
}

static size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Workspace: part_o [B][Hq][S][D] float, part_ml [B][Hq][S][2] float, then
// the in-kernel merge's tickets, one 64-bit word per (sequence, KV head)
// (room for B * Hq of them: the KV head count is not an argument here).
static size_t workspace_part_ml_offset(int num_seqs, int num_heads, int head_dim, int splits) {
    return round256((size_t)num_seqs * num_heads * splits * head_dim * sizeof(float));
}
static size_t workspace_tickets_offset(int num_seqs, int num_heads, int head_dim, int splits) {
    return workspace_part_ml_offset(num_seqs, num_heads, head_dim, splits) +
           round256((size_t)num_seqs * num_heads * splits * 2 * sizeof(float));
}
static size_t workspace_bytes_for(int num_seqs, int num_heads, int head_dim, int splits) {
    if (splits <= 1) return 0;
    return workspace_tickets_offset(num_seqs, num_heads, head_dim, splits) +
           round256((size_t)num_seqs * num_heads * sizeof(unsigned long long));
}

// A tag per decode call for the in-kernel merge's tickets (never 0).
static uint32_t next_merge_tag() {
    static std::atomic<uint32_t> tag{0};
    uint32_t t = tag.fetch_add(1, std::memory_order_relaxed) + 1;
    if (t == 0) t = tag.fetch_add(1, std::memory_order_relaxed) + 1;
    return t;
}

}  // namespace pa

using namespace pa;

extern "C" {

const char *pa_last_error(void) { return error_buffer(); }

int pa_version(void) { return 10000; }

int pa_device_errors(uint32_t *flags_out, int clear) {
    clear_error();
    unsigned int v = 0;
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
    e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v));
    if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
    if (clear && v) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero));
        if (e != cudaSuccess) return cuda_fail(e, "clearing the device error word");
    }
    if (flags_out) *flags_out = v;
    if (v) return fail(PA_ERR_DEVICE_BOUNDS, "device error bits 0x%x", v);
    return PA_OK;
}

int pa_reshape_and_cache(const void *k, const void *v, void *k_cache, void *v_cache,
                         const int64_t *slot_mapping, int num_tokens, int num_kv_heads,
                         int head_dim, int block_size, int num_blocks, int dtype, void *stream) {
    clear_error();
    int rc = check_shape(num_kv_heads, head_dim, block_size, dtype);
    if (rc) return rc;
    if (num_tokens < 0 || num_blocks <= 0)
        return fail(PA_ERR_INVALID_ARG, "num_tokens %d, num_blocks %d", num_tokens, num_blocks);
    if (num_tokens == 0) return PA_OK;
    if (!k || !v || !k_cache || !v_cache || !slot_mapping)
        return fail(PA_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache) ||
        (reinterpret_cast<uintptr_t>(slot_mapping) & 7u))
        return fail(PA_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
    unsigned int *err = device_error_ptr();
    if (!err) return fail(PA_ERR_CUDA, "no CUDA device");
    cudaError_t e = launch_reshape_and_cache(k, v, k_cache, v_cache, slot_mapping, num_tokens,
                                             num_kv_heads, head_dim * elem_bytes(dtype),
                                             block_size, num_blocks, err,
                                             static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "reshape_and_cache launch");
    return PA_OK;
}

size_t pa_decode_workspace_size(int num_seqs, int num_heads, int head_dim, int max_seq_len,
                                int partition_size) {
    const int part = partition_or_default(partition_size);
    if (num_seqs <= 0 || num_heads <= 0 || head_dim <= 0 || part <= 0) return 0;
    return workspace_bytes_for(num_seqs, num_heads, head_dim, splits_for(max_seq_len, part));
}

int pa_decode_ex(float *out, const void *q, const void *k_cache, const void *v_cache,
                 const int32_t *block_tables, const int32_t *seq_lens, int num_seqs,
                 int num_heads, int num_kv_heads, int head_dim, int block_size,
                 int max_blocks_per_seq, int num_blocks, int max_seq_len, float scale,
                 int dtype, void *workspace, size_t workspace_bytes, int partition_size,
                 int variant, void *stream) {
    pa_decode_opts o;
    std::memset(&o, 0, sizeof(o));
    o.partition_size = partition_size;
    o.variant = variant;
    return pa_decode_opt(out, q, k_cache, v_cache, block_tables, seq_lens, num_seqs, num_heads,
                         num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks,
                         max_seq_len, scale, dtype, workspace, workspace_bytes, &o, stream);
}

}  // extern "C"

namespace pa {
// The new tokens of a fused append (pa_append_decode), or none.
struct AppendArgs {
    const void *k_new, *v_new;
    const int64_t *slot_mapping;
};
}  // namespace pa

static int decode_impl(float *out, const void *q, const void *k_cache, const void *v_cache,
                       const int32_t *block_tables, const int32_t *seq_lens, int num_seqs,
                       int num_heads, int num_kv_heads, int head_dim, int block_size,
                       int max_blocks_per_seq, int num_blocks, int max_seq_len, float scale,
                       int dtype, void *workspace, size_t workspace_bytes,
                       const pa_decode_opts *opts, const AppendArgs *app, void *stream);

extern "C" {

int pa_decode_opt(float *out, const void *q, const void *k_cache, const void *v_cache,
                  const int32_t *block_tables, const int32_t *seq_lens, int num_seqs,
                  int num_heads, int num_kv_heads, int head_dim, int block_size,
                  int max_blocks_per_seq, int num_blocks, int max_seq_len, float scale,
                  int dtype, void *workspace, size_t workspace_bytes,
                  const pa_decode_opts *opts, void *stream) {
    clear_error();
    return decode_impl(out, q, k_cache, v_cache, block_tables, seq_lens, num_seqs, num_heads,
                       num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks,
                       max_seq_len, scale, dtype, workspace, workspace_bytes, opts, nullptr,
                       stream);
}

int pa_append_decode(float *out, const void *q, const void *k_new, const void *v_new,
                     const int64_t *slot_mapping, void *k_cache, void *v_cache,
                     const int32_t *block_tables, const int32_t *seq_lens, int num_seqs,
                     int num_heads, int num_kv_heads, int head_dim, int block_size,
                     int max_blocks_per_seq, int num_blocks, int max_seq_len, float scale,
                     int dtype, void *workspace, size_t workspace_bytes,
                     const pa_decode_opts *opts, void *stream) {
    clear_error();
    if (num_seqs > 0 && (!k_new || !v_new || !slot_mapping))
        return fail(PA_ERR_INVALID_ARG, "NULL new-token pointer");
    if (num_seqs > 0 && (!aligned16(k_new) || !aligned16(v_new) ||
                         (reinterpret_cast<uintptr_t>(slot_mapping) & 7u)))
        return fail(PA_ERR_INVALID_ARG, "misaligned new-token pointer");
    const AppendArgs app = {k_new, v_new, slot_mapping};
    return decode_impl(out, q, k_cache, v_cache, block_tables, seq_lens, num_seqs, num_heads,
                       num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks,
                       max_seq_len, scale, dtype, workspace, workspace_bytes, opts, &app,
                       stream);
}

}  // extern "C"

static int decode_impl(float *out, const void *q, const void *k_cache, const void *v_cache,
                       const int32_t *block_tables, const int32_t *seq_lens, int num_seqs,
                       int num_heads, int num_kv_heads, int head_dim, int block_size,
                       int max_blocks_per_seq, int num_blocks, int max_seq_len, float scale,
                       int dtype, void *workspace, size_t workspace_bytes,
                       const pa_decode_opts *opts, const AppendArgs *app, void *stream) {
    pa_decode_opts o;
    std::memset(&o, 0, sizeof(o));
    if (opts) o = *opts;
    const int partition_size = o.partition_size;
    int variant = o.variant;
    if (o.merge < 0 || o.merge > 2) return fail(PA_ERR_INVALID_ARG, "merge %d", o.merge);
    int rc = check_shape(num_kv_heads, head_dim, block_size, dtype);
    if (rc) return rc;
    if (num_heads <= 0 || num_heads % num_kv_heads != 0)
        return fail(PA_ERR_INVALID_ARG, "num_heads %d not a multiple of num_kv_heads %d",
                    num_heads, num_kv_heads);
    const int G = num_heads / num_kv_heads;
    if (G > 8) return fail(PA_ERR_UNSUPPORTED, "GQA group %d > 8", G);
    if (num_seqs < 0 || num_seqs > 65535)
        return fail(PA_ERR_INVALID_ARG, "num_seqs %d outside [0, 65535]", num_seqs);
    if (num_blocks <= 0 || max_blocks_per_seq < 0 || max_seq_len < 0)
        return fail(PA_ERR_INVALID_ARG, "bad sizes");
    if ((int64_t)max_seq_len > (int64_t)max_blocks_per_seq * block_size)
        return fail(PA_ERR_INVALID_ARG, "max_seq_len %d > max_blocks_per_seq * block_size",
                    max_seq_len);
    if (!std::isfinite(scale)) return fail(PA_ERR_INVALID_ARG, "scale is not finite");
    const int part = partition_or_default(partition_size);
    if (part < 64 || part > 1024 || part % 64 != 0)
        return fail(PA_ERR_INVALID_ARG, "partition_size %d: a multiple of 64 in [64, 1024]",
                    partition_size);
    if (variant < 0 || variant > 3) return fail(PA_ERR_INVALID_ARG, "variant %d", variant);
    if (variant >= 2 && dtype == PA_F32)
        return fail(PA_ERR_UNSUPPORTED, "the tensor-core kernels take bf16/f16 caches");
    for (int r : o.reserved)
        if (r != 0) return fail(PA_ERR_INVALID_ARG, "reserved option fields must be 0");
    if (reinterpret_cast<uintptr_t>(o.seq_order) & 3u)
        return fail(PA_ERR_INVALID_ARG, "seq_order must be 4-byte aligned");
    int heads_per_cta = o.heads_per_cta;
    if (heads_per_cta != 0 && variant != 3)
        return fail(PA_ERR_INVALID_ARG, "heads_per_cta is an option of variant 3");
    if (variant == 3) {
        const int ts = block_size < 16 ? 16 : block_size;  // tokens per stage
        if (heads_per_cta == 0) heads_per_cta = num_kv_heads % 2 == 0 && 2 * ts <= 64 ? 2 : 1;
        if ((heads_per_cta != 1 && heads_per_cta != 2 && heads_per_cta != 4) ||
            num_kv_heads % heads_per_cta != 0 || heads_per_cta * ts > 64)
            return fail(PA_ERR_UNSUPPORTED,
                        "heads_per_cta %d: 1, 2 or 4, dividing num_kv_heads %d, with "
                        "heads_per_cta * max(16, block_size) <= 64",
                        heads_per_cta, num_kv_heads);
    }
    if (num_seqs == 0) return PA_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !seq_lens)
        return fail(PA_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) ||
        (reinterpret_cast<uintptr_t>(block_tables) & 3u) ||
        (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
        return fail(PA_ERR_INVALID_ARG, "misaligned pointer");
    const int splits = splits_for(max_seq_len, part);
    if (splits > kMaxSplits)
        return fail(PA_ERR_UNSUPPORTED, "max_seq_len %d needs %d splits of %d tokens (max %d)",
                    max_seq_len, splits, part, kMaxSplits);
    const size_t need = workspace_bytes_for(num_seqs, num_heads, head_dim, splits);
    if (need > 0 && (!workspace || workspace_bytes < need || !aligned16(workspace)))
        return fail(PA_ERR_INVALID_ARG, "workspace of %zu bytes needed, %zu given", need,
                    workspace ? workspace_bytes : (size_t)0);
    unsigned int *err = device_error_ptr();
    if (!err) return fail(PA_ERR_CUDA, "no CUDA device");

    DecodeParams p;
    std::memset(&p, 0, sizeof(p));
    p.out = out;
    // the library's choice is the reduce kernel: merging inside the main
    // kernel costs every split CTA a fence and a ticket round trip before it
    // frees its slot, which measured no faster on any workload of the bench
    const bool fused = need > 0 && o.merge == 2;
    if (need > 0) {
        char *ws = static_cast<char *>(workspace);
        p.part_o = reinterpret_cast<float *>(ws);
        p.part_ml = reinterpret_cast<float *>(
            ws + workspace_part_ml_offset(num_seqs, num_heads, head_dim, splits));
        if (fused) {
            p.tickets = reinterpret_cast<unsigned long long *>(
                ws + workspace_tickets_offset(num_seqs, num_heads, head_dim, splits));
            p.tag = next_merge_tag();
        }
    }
    p.q = q;
    p.k_cache = k_cache;
    p.v_cache = v_cache;
    p.block_tables = block_tables;
    p.seq_lens = seq_lens;
    p.err = err;
    p.num_seqs = num_seqs;
    p.num_heads = num_heads;
    p.num_kv_heads = num_kv_heads;
    p.head_dim = head_dim;
    p.block_size = block_size;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.num_blocks = num_blocks;
    p.max_seq_len = max_seq_len;
    p.partition_size = part;
    p.max_splits = splits;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.seq_order = o.seq_order;
    if (app) {
        p.k_new = app->k_new;
        p.v_new = app->v_new;
        p.slot_mapping = app->slot_mapping;
    }

    // 16-bit caches go to the tensor-core kernel (it needs the cache to fit
    // 2^31 TMA rows); fp32 caches to the CUDA-core kernel.
    const int64_t rows = (int64_t)num_blocks * num_kv_heads * block_size;
    const bool tc_ok = dtype != PA_F32 &&
                       rows + (int64_t)(num_kv_heads + 1) * block_size < (int64_t(1) << 31);
    if (variant >= 2 && !tc_ok)
        return fail(PA_ERR_UNSUPPORTED, "cache too large for the tensor-core kernels");
    // The automatic choice for 16-bit caches: two KV heads per CTA, one per
    // warp (variant 3), where the kernel exists for the block size and its
    // grid (every split of the longest length, empty ones included) fills at
    // least one wave of resident CTAs; else the tensor-core kernel with its
    // CTA per KV head, twice as many CTAs for a thin batch.
    if (variant == 0 && tc_ok && (block_size == 8 || block_size == 16) &&
        num_kv_heads % 2 == 0) {
        const int slots = hw2_slots(dtype, head_dim, block_size);
        if (slots < 0) return slots;
        if ((int64_t)p.max_splits * (num_kv_heads / 2) * num_seqs >= slots) {
            variant = 3;
            heads_per_cta = 2;
        }
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const ProfileEvents prof = t_prof;
    cudaError_t e;
    if (prof.begin && prof.end) {
        e = cudaEventRecord(prof.begin, st);
        if (e != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
    }
    if (variant == 3)
        e = launch_decode_hw(p, dtype, heads_per_cta, st);
    else if ((variant == 0 && tc_ok) || variant == 2)
        e = launch_decode_tc(p, dtype, st);
    else
        e = launch_decode_simt(p, dtype, st);
    if (e != cudaSuccess) return cuda_fail(e, "decode launch");
    if (prof.begin && prof.end) {
        e = cudaEventRecord(prof.end, st);
        if (e != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
    }
    if (!fused) {
        e = launch_decode_reduce(p, st);
        if (e != cudaSuccess) return cuda_fail(e, "reduce launch");
    }
    return PA_OK;
}

extern "C" {

int pa_decode_partition_for(const int32_t *seq_lens_host, int num_seqs, int num_kv_heads,
                            int head_dim, int block_size, int dtype, int slots) {
    clear_error();
    int rc = check_shape(num_kv_heads, head_dim, block_size, dtype);
    if (rc) return rc;
    if (num_seqs < 0 || num_seqs > 65535)
        return fail(PA_ERR_INVALID_ARG, "num_seqs %d outside [0, 65535]", num_seqs);
    if (num_seqs > 0 && !seq_lens_host) return fail(PA_ERR_INVALID_ARG, "NULL seq_lens_host");
    if (slots < 0) return fail(PA_ERR_INVALID_ARG, "slots %d", slots);
    for (int s = 0; s < num_seqs; ++s)
        if (seq_lens_host[s] < 0)
            return fail(PA_ERR_INVALID_ARG, "seq_lens_host[%d] = %d", s, seq_lens_host[s]);
    if (dtype == PA_F32) return kDefaultPartition;  // CUDA-core kernel
    if (slots == 0) {
        // per device and shape, asked once: [device][bf16|f16][D 64|128][bs 4..64]
        static std::atomic<int> cache[kMaxDevices][2][2][5];
        const int dev = current_device();
        if (dev < 0 || dev >= kMaxDevices) return fail(PA_ERR_CUDA, "no CUDA device");
        const int bsi = block_size == 4    ? 4
                        : block_size == 8  ? 0
                        : block_size == 16 ? 1
                        : block_size == 32 ? 2
                                           : 3;
        std::atomic<int> &c = cache[dev][dtype == PA_F16][head_dim == 128][bsi];
        int per_sm = c.load(std::memory_order_relaxed);
        if (per_sm <= 0) {
            per_sm = decode_tc_resident_per_sm(dtype, head_dim, block_size);
            if (per_sm <= 0) return fail(PA_ERR_CUDA, "occupancy query failed");
            c.store(per_sm, std::memory_order_relaxed);
        }
        slots = per_sm * num_sms();
    }
    // CTAs of a partition length: one per (sequence, KV head, partition)
    auto ctas = [&](int part) {
        int64_t n = 0;
        for (int s = 0; s < num_seqs; ++s)
            n += seq_lens_host[s] == 0 ? 1 : (seq_lens_host[s] + part - 1) / part;
        return n * num_kv_heads;
    };
    // one alternative only, so that a runtime replaying CUDA graphs keyed on
    // the split length sees it change rarely as its sequences grow
    const int64_t n0 = ctas(kDefaultPartition);
    if (n0 > slots && n0 <= 2 * (int64_t)slots && ctas(1024) <= slots) return 1024;
    // lengths that differ by more than 2x: with the grid taking the sequences
    // longest first (pa_decode_order), the short CTAs at the end fill the
    // tail, and fewer, longer splits save start-ups and partials
    int32_t lo = INT32_MAX, hi = 0;
    for (int s = 0; s < num_seqs; ++s) {
        lo = seq_lens_host[s] < lo ? seq_lens_host[s] : lo;
        hi = seq_lens_host[s] > hi ? seq_lens_host[s] : hi;
    }
    if (hi > kDefaultPartition && (int64_t)hi > 2 * (int64_t)lo) return 1024;
    return kDefaultPartition;
}

int pa_decode_choose(const int32_t *seq_lens_host, int num_seqs, int num_kv_heads,
                     int head_dim, int block_size, int dtype, int slots, pa_decode_opts *opts) {
    clear_error();
    if (!opts) return fail(PA_ERR_INVALID_ARG, "NULL opts");
    const int part = pa_decode_partition_for(seq_lens_host, num_seqs, num_kv_heads, head_dim,
                                             block_size, dtype, slots);
    if (part < 0) return part;
    opts->partition_size = part;
    opts->variant = dtype == PA_F32 ? 1 : 2;
    opts->heads_per_cta = 0;
    if (dtype == PA_F32 || num_kv_heads % 2 != 0 || (block_size != 8 && block_size != 16))
        return PA_OK;
    // Two KV heads per CTA, one per warp (variant 3), with the split chosen
    // by the share of a wave of resident CTAs it fills: the shortest split
    // whose CTAs fill at most 0.85 of the CTAs the device holds at once (as
    // many concurrent streams as fit in one wave with some slack, each CTA
    // short enough that the last ones do not bound the launch); if even
    // 1024-token splits fill more, 1024 when they still fit one wave, else
    // 512 (several waves, short CTAs to balance them).
    if (slots == 0) {
        slots = hw2_slots(dtype, head_dim, block_size);
        if (slots < 0) return slots;
    }
    auto ctas = [&](int p) {
        int64_t n = 0;
        for (int s = 0; s < num_seqs; ++s)
            n += seq_lens_host[s] <= p ? 1 : (seq_lens_host[s] + p - 1) / p;
        return n * (num_kv_heads / 2);
    };
    static const int kSplits[] = {256, 384, 512, 640, 768, 1024};  // fill falls as p grows
    int chosen = 0;
    for (int p : kSplits) {
        if (20 * ctas(p) <= 17 * (int64_t)slots) {
            chosen = p;
            break;
        }
    }
    if (chosen == 0) chosen = ctas(1024) <= slots ? 1024 : kDefaultPartition;
    opts->variant = 3;
    opts->heads_per_cta = 2;
    opts->partition_size = chosen;
    return PA_OK;
}

int pa_decode(float *out, const void *q, const void *k_cache, const void *v_cache,
              const int32_t *block_tables, const int32_t *seq_lens, int num_seqs,
              int num_heads, int num_kv_heads, int head_dim, int block_size,
              int max_blocks_per_seq, int num_blocks, int max_seq_len, float scale, int dtype,
              void *workspace, size_t workspace_bytes, void *stream) {
    return pa_decode_ex(out, q, k_cache, v_cache, block_tables, seq_lens, num_seqs, num_heads,
                        num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks,
                        max_seq_len, scale, dtype, workspace, workspace_bytes, 0, 0, stream);
}

int pa_prefill(float *out, const void *q, const void *k_cache, const void *v_cache,
               const int32_t *block_tables, const int32_t *seq_lens, const int32_t *cu_q_lens,
               int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
               int max_blocks_per_seq, int num_blocks, int max_q_len, int max_seq_len,
               float scale, int dtype, void *stream) {
    return pa_prefill_ex(out, q, k_cache, v_cache, block_tables, seq_lens, cu_q_lens, num_seqs,
                         num_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                         num_blocks, max_q_len, max_seq_len, scale, dtype, 0, stream);
}

int pa_prefill_ex(float *out, const void *q, const void *k_cache, const void *v_cache,
                  const int32_t *block_tables, const int32_t *seq_lens, const int32_t *cu_q_lens,
                  int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
                  int max_blocks_per_seq, int num_blocks, int max_q_len, int max_seq_len,
                  float scale, int dtype, int variant, void *stream) {
    clear_error();
    if (variant < 0 || variant > 4)
        return fail(PA_ERR_INVALID_ARG, "prefill variant %d not in {0, 1, 2, 3, 4}", variant);
    if (variant == 0) variant = kPrefillDefault;
    int rc = check_shape(num_kv_heads, head_dim, block_size, dtype);
    if (rc) return rc;
    if (dtype == PA_F32 || block_size < 8)
        return fail(PA_ERR_UNSUPPORTED, "pa_prefill takes bf16/f16 caches with block_size >= 8");
    if (num_heads <= 0 || num_heads % num_kv_heads != 0)
        return fail(PA_ERR_INVALID_ARG, "num_heads %d not a multiple of num_kv_heads %d",
                    num_heads, num_kv_heads);
    const int G = num_heads / num_kv_heads;
    if (G > 8) return fail(PA_ERR_UNSUPPORTED, "GQA group %d > 8", G);
    if (num_seqs < 0 || num_seqs > 65535)
        return fail(PA_ERR_INVALID_ARG, "num_seqs %d outside [0, 65535]", num_seqs);
    if (num_blocks <= 0 || max_blocks_per_seq < 0 || max_seq_len < 0 || max_q_len < 0 ||
        max_q_len > max_seq_len)
        return fail(PA_ERR_INVALID_ARG, "bad sizes");
    if ((int64_t)max_seq_len > (int64_t)max_blocks_per_seq * block_size)
        return fail(PA_ERR_INVALID_ARG, "max_seq_len %d > max_blocks_per_seq * block_size",
                    max_seq_len);
    if (!std::isfinite(scale)) return fail(PA_ERR_INVALID_ARG, "scale is not finite");
    if (num_seqs == 0 || max_q_len == 0) return PA_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !seq_lens || !cu_q_lens)
        return fail(PA_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) ||
        (reinterpret_cast<uintptr_t>(block_tables) & 3u) ||
        (reinterpret_cast<uintptr_t>(seq_lens) & 3u) ||
        (reinterpret_cast<uintptr_t>(cu_q_lens) & 3u))
        return fail(PA_ERR_INVALID_ARG, "misaligned pointer");
    const int64_t rows = (int64_t)num_blocks * num_kv_heads * block_size;
    if (rows + (int64_t)(num_kv_heads + 1) * block_size >= (int64_t(1) << 31))
        return fail(PA_ERR_UNSUPPORTED, "cache too large for 32-bit TMA row coordinates");
    unsigned int *err = device_error_ptr();
    if (!err) return fail(PA_ERR_CUDA, "no CUDA device");
    PrefillParams p;
    std::memset(&p, 0, sizeof(p));
    p.out = out;
    p.q = q;
    p.k_cache = k_cache;
    p.v_cache = v_cache;
    p.block_tables = block_tables;
    p.seq_lens = seq_lens;
    p.cu_q = cu_q_lens;
    p.err = err;
    p.num_seqs = num_seqs;
    p.num_heads = num_heads;
    p.num_kv_heads = num_kv_heads;
    p.head_dim = head_dim;
    p.block_size = block_size;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.num_blocks = num_blocks;
    p.max_seq_len = max_seq_len;
    p.max_q_len = max_q_len;
    p.tokens_per_cta = (variant >= 2 ? 128 : 64) / G;
    p.scale_log2 = scale * 1.4426950408889634f;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = variant >= 2 ? launch_prefill_umma(p, dtype, variant - 2, st)
                                 : launch_prefill_tc(p, dtype, st);
    if (e != cudaSuccess) return cuda_fail(e, "prefill launch");
    return PA_OK;
}

int pa_copy_blocks(void *k_cache, void *v_cache, const int64_t *src_dst_pairs, int num_pairs,
                   size_t block_bytes, int num_blocks, void *stream) {
    clear_error();
    if (num_pairs < 0 || num_blocks <= 0)
        return fail(PA_ERR_INVALID_ARG, "num_pairs %d, num_blocks %d", num_pairs, num_blocks);
    if (num_pairs == 0) return PA_OK;
    if (!k_cache || !v_cache || !src_dst_pairs) return fail(PA_ERR_INVALID_ARG, "NULL pointer");
    if (block_bytes == 0 || block_bytes % 16 != 0)
        return fail(PA_ERR_INVALID_ARG, "block_bytes %zu must be a positive multiple of 16",
                    block_bytes);
    if (!aligned16(k_cache) || !aligned16(v_cache) ||
        (reinterpret_cast<uintptr_t>(src_dst_pairs) & 7u))
        return fail(PA_ERR_INVALID_ARG, "misaligned pointer");
    unsigned int *err = device_error_ptr();
    if (!err) return fail(PA_ERR_CUDA, "no CUDA device");
    cudaError_t e = launch_copy_blocks(k_cache, v_cache, src_dst_pairs, num_pairs, block_bytes,
                                       num_blocks, err, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "copy_blocks launch");
    return PA_OK;
}

// Device-usable address of a device or page-locked (mapped) host pointer;
// nullptr for memory the GPU cannot reach.
static const void *device_view(const void *p) {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError();  // clear the sticky-free error of an unknown pointer
        return nullptr;
    }
    switch (at.type) {
    case cudaMemoryTypeDevice:
    case cudaMemoryTypeManaged: return p;
    case cudaMemoryTypeHost: return at.devicePointer;
    default: return nullptr;
    }
}

int pa_swap_blocks(void *dst_k, void *dst_v, const void *src_k, const void *src_v,
                   const int64_t *src_dst_pairs, int num_pairs, size_t block_bytes,
                   int num_src_blocks, int num_dst_blocks, void *stream) {
    clear_error();
    if (num_pairs < 0 || num_src_blocks <= 0 || num_dst_blocks <= 0)
        return fail(PA_ERR_INVALID_ARG, "num_pairs %d, blocks %d / %d", num_pairs,
                    num_src_blocks, num_dst_blocks);
    if (num_pairs == 0) return PA_OK;
    if (!dst_k || !dst_v || !src_k || !src_v || !src_dst_pairs)
        return fail(PA_ERR_INVALID_ARG, "NULL pointer");
    if (block_bytes == 0 || block_bytes % 16 != 0)
        return fail(PA_ERR_INVALID_ARG, "block_bytes %zu must be a positive multiple of 16",
                    block_bytes);
    const void *v[5] = {dst_k, dst_v, src_k, src_v, src_dst_pairs};
    const void *d[5];
    for (int i = 0; i < 5; ++i) {
        d[i] = device_view(v[i]);
        if (!d[i])
            return fail(PA_ERR_INVALID_ARG,
                        "pointer %d is neither device memory nor mapped page-locked host memory",
                        i);
    }
    if (!aligned16(d[0]) || !aligned16(d[1]) || !aligned16(d[2]) || !aligned16(d[3]) ||
        (reinterpret_cast<uintptr_t>(d[4]) & 7u))
        return fail(PA_ERR_INVALID_ARG, "misaligned pointer");
    unsigned int *err = device_error_ptr();
    if (!err) return fail(PA_ERR_CUDA, "no CUDA device");
    cudaError_t e = launch_swap_blocks(const_cast<void *>(d[0]), const_cast<void *>(d[1]), d[2],
                                       d[3], static_cast<const int64_t *>(d[4]), num_pairs,
                                       block_bytes, num_src_blocks, num_dst_blocks, err,
                                       static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "swap_blocks launch");
    return PA_OK;
}

// One host-fed step's device work in one call (the runtime's step executor):
// the step's copies in on one stream, its kernels' graph on a second, its
// output's copy graph on a third, ordered by events.
int pa_step_launch(void *stream_in, void *stream_run, void *stream_out,
                   const pa_host_copy *copies, int n_copies, void *wait_before_in,
                   void *event_in, void *graph_run, void *wait_before_run, void *event_run,
                   void *graph_out, void *event_out) {
    clear_error();
    if (n_copies < 0 || (n_copies > 0 && !copies))
        return fail(PA_ERR_INVALID_ARG, "bad copy list");
    if (!event_in || !graph_run || !event_run || (graph_out && !event_out))
        return fail(PA_ERR_INVALID_ARG, "NULL event or graph");
    cudaStream_t si = static_cast<cudaStream_t>(stream_in);
    cudaStream_t sr = static_cast<cudaStream_t>(stream_run);
    cudaStream_t so = static_cast<cudaStream_t>(stream_out);
    cudaError_t e = cudaSuccess;
    if (wait_before_in) e = cudaStreamWaitEvent(si, static_cast<cudaEvent_t>(wait_before_in), 0);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamWaitEvent");
    for (int i = 0; i < n_copies; ++i) {
        if (copies[i].bytes == 0) continue;
        if (!copies[i].dst || !copies[i].src) return fail(PA_ERR_INVALID_ARG, "NULL copy %d", i);
        e = cudaMemcpyAsync(copies[i].dst, copies[i].src, copies[i].bytes, cudaMemcpyHostToDevice,
                            si);
        if (e != cudaSuccess) return cuda_fail(e, "host-to-device copy");
    }
    if ((e = cudaEventRecord(static_cast<cudaEvent_t>(event_in), si)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(sr, static_cast<cudaEvent_t>(event_in), 0)) != cudaSuccess)
        return cuda_fail(e, "event after the copies");
    if (wait_before_run &&
        (e = cudaStreamWaitEvent(sr, static_cast<cudaEvent_t>(wait_before_run), 0)) != cudaSuccess)
        return cuda_fail(e, "cudaStreamWaitEvent");
    if ((e = cudaGraphLaunch(static_cast<cudaGraphExec_t>(graph_run), sr)) != cudaSuccess)
        return cuda_fail(e, "kernels' graph launch");
    if ((e = cudaEventRecord(static_cast<cudaEvent_t>(event_run), sr)) != cudaSuccess)
        return cuda_fail(e, "cudaEventRecord");
    if (graph_out) {
        if ((e = cudaStreamWaitEvent(so, static_cast<cudaEvent_t>(event_run), 0)) != cudaSuccess ||
            (e = cudaGraphLaunch(static_cast<cudaGraphExec_t>(graph_out), so)) != cudaSuccess ||
            (e = cudaEventRecord(static_cast<cudaEvent_t>(event_out), so)) != cudaSuccess)
            return cuda_fail(e, "output copy");
    }
    return PA_OK;
}

int pa_set_profile_events(void *ev_begin, void *ev_end) {
    clear_error();
    t_prof.begin = static_cast<cudaEvent_t>(ev_begin);
    t_prof.end = static_cast<cudaEvent_t>(ev_end);
    return PA_OK;
}

int pa_selftest_wait(uint64_t limit_ns, uint64_t abort_after_ns, unsigned long long *elapsed_ns,
                     void *stream) {
    clear_error();
    if (limit_ns == 0 || limit_ns > 10000000000ull || abort_after_ns > 10000000000ull)
        return fail(PA_ERR_INVALID_ARG, "limit_ns must be in (0, 1e10], abort_after_ns <= 1e10");
    if (!elapsed_ns) return fail(PA_ERR_INVALID_ARG, "NULL elapsed_ns");
    unsigned int *err = device_error_ptr();
    if (!err) return fail(PA_ERR_CUDA, "no CUDA device");
    cudaError_t e = launch_wait_selftest(err, limit_ns, abort_after_ns, elapsed_ns,
                                         static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "wait self-test launch");
    return PA_OK;
}

}  // extern "C"
