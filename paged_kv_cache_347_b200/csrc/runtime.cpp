// pa_runtime: a decode runtime around the library's calls, one C call per
// host-fed step (pagedattn.h, "Runtime").
//
// The pages leave the block tables and the allocation to a runtime that owns
// them (sanketn26 "PagedAttention", "Use a runtime that owns the blocks").
// This one owns the allocator, two staging slots (page-locked host memory
// and a device buffer each), the split workspace, two device output buffers,
// three streams and a cache of CUDA graphs.  A step:
//   1. on the copy-in stream: the new K/V rows and the queries go to fixed
//      places of the slot's device buffer (they need nothing from the plan,
//      so the host link carries them while the host plans);
//   2. pa_step_plan applies the step's events and writes slots, copy pairs,
//      table rows, lengths and the longest-first order into the slot's host
//      buffer;
//   3. pa_decode_choose picks the decode's kernel and split from the lengths;
//      a run of one-token appends of exactly the decode batch, right before
//      the decode, goes in with it (pa_append_decode); the arrays follow the
//      rows on the copy-in stream;
//   4. on the run stream: the step's kernels, replayed from a CUDA graph
//      captured for its layout (steps with copy-on-write copies, or a layout
//      seen for the first time, launch directly; a new layout is captured
//      after its first run);
//   5. on the copy-out stream: the output to the caller's host buffer.
// Steps alternate between the slots, so step i+1's host work and copies can
// go on while step i's kernels run.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <map>
#include <new>
#include <vector>

#include "../../include/pagedattn.h"
#include "status.h"

namespace {

size_t a256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// One device action of a step, in event order.
struct Act {
    int kind;          // 0 = write (a run of appends), 1 = decode
    int r0, r1;        // write: K/V rows
    int p0, p1;        // write: copy-on-write pairs
    bool fused;        // write: its rows go in with the decode
};

struct Graph {
    cudaGraphExec_t exec = nullptr;
};

}  // namespace

struct pa_runtime {
    pa_runtime_config cfg;
    pa_alloc *alloc = nullptr;
    void *k_cache = nullptr, *v_cache = nullptr;
    int dev = 0, elem = 2;
    size_t arrays_cap = 0, kv_cap = 0, q_cap = 0, slot_bytes = 0, out_bytes = 0;
    size_t off_k = 0, off_v = 0, off_q = 0;
    cudaStream_t s_in = nullptr, s_run = nullptr, s_out = nullptr;
    char *host[2] = {nullptr, nullptr};
    char *devb[2] = {nullptr, nullptr};
    float *out_dev[2] = {nullptr, nullptr};
    cudaEvent_t ev_in[2] = {nullptr, nullptr}, ev_run[2] = {nullptr, nullptr},
                ev_out[2] = {nullptr, nullptr};
    bool used[2] = {false, false};
    int next = 0;
    void *ws = nullptr;
    size_t ws_bytes = 0;
    std::map<std::vector<int64_t>, Graph> graphs;
    std::vector<int32_t> pairs_before;
    std::vector<Act> acts;
    int64_t steps = 0, replays = 0, captures = 0;
};

namespace {

int cuda_err(cudaError_t e, const char *what) {
    return pa::fail(PA_ERR_CUDA, "runtime: %s: %s", what, cudaGetErrorString(e));
}

void release(pa_runtime *rt) {
    if (!rt) return;
    for (auto &g : rt->graphs)
        if (g.second.exec) cudaGraphExecDestroy(g.second.exec);
    for (int i = 0; i < 2; ++i) {
        if (rt->host[i]) cudaFreeHost(rt->host[i]);
        if (rt->devb[i]) cudaFree(rt->devb[i]);
        if (rt->out_dev[i]) cudaFree(rt->out_dev[i]);
        for (cudaEvent_t e : {rt->ev_in[i], rt->ev_run[i], rt->ev_out[i]})
            if (e) cudaEventDestroy(e);
    }
    if (rt->ws) cudaFree(rt->ws);
    for (cudaStream_t s : {rt->s_in, rt->s_run, rt->s_out})
        if (s) cudaStreamDestroy(s);
    if (rt->alloc) pa_alloc_destroy(rt->alloc);
    delete rt;
}

// The step's device work on the run stream, in event order: each run of
// appends is its copies, then its rows (unless they go in with the decode);
// the decode in its place.
int launch_step(pa_runtime *rt, int slot, const pa_step_layout &lay, int num_seqs,
                const pa_decode_opts &opts, int max_len) {
    const pa_runtime_config &c = rt->cfg;
    char *d = rt->devb[slot];
    const int64_t *slots = reinterpret_cast<const int64_t *>(d + lay.off_slots);
    const int64_t *pairs = reinterpret_cast<const int64_t *>(d + lay.off_pairs);
    const char *k_new = d + rt->off_k, *v_new = d + rt->off_v;
    const size_t row = (size_t)c.num_kv_heads * c.head_dim * rt->elem;
    const size_t block_bytes = (size_t)c.num_kv_heads * c.block_size * c.head_dim * rt->elem;
    const int32_t *tables = reinterpret_cast<const int32_t *>(d + lay.off_tables);
    const int32_t *lens = reinterpret_cast<const int32_t *>(d + lay.off_lens);
    const int32_t *order = reinterpret_cast<const int32_t *>(d + lay.off_order);
    pa_decode_opts o = opts;
    o.seq_order = order;
    for (size_t i = 0; i < rt->acts.size(); ++i) {
        const Act &a = rt->acts[i];
        int rc = PA_OK;
        if (a.kind == 0) {
            if (a.p1 > a.p0)
                rc = pa_copy_blocks(rt->k_cache, rt->v_cache, pairs + 2 * a.p0, a.p1 - a.p0,
                                    block_bytes, c.num_blocks, rt->s_run);
            if (rc == PA_OK && a.r1 > a.r0 && !a.fused)
                rc = pa_reshape_and_cache(k_new + a.r0 * row, v_new + a.r0 * row, rt->k_cache,
                                          rt->v_cache, slots + a.r0, a.r1 - a.r0,
                                          c.num_kv_heads, c.head_dim, c.block_size,
                                          c.num_blocks, c.dtype, rt->s_run);
        } else {
            const Act *w = i > 0 && rt->acts[i - 1].fused ? &rt->acts[i - 1] : nullptr;
            if (w)
                rc = pa_append_decode(rt->out_dev[slot], d + rt->off_q, k_new + w->r0 * row,
                                      v_new + w->r0 * row, slots + w->r0, rt->k_cache,
                                      rt->v_cache, tables, lens, num_seqs, c.num_heads,
                                      c.num_kv_heads, c.head_dim, c.block_size, c.table_width,
                                      c.num_blocks, max_len, c.scale, c.dtype, rt->ws,
                                      rt->ws_bytes, &o, rt->s_run);
            else
                rc = pa_decode_opt(rt->out_dev[slot], d + rt->off_q, rt->k_cache, rt->v_cache,
                                   tables, lens, num_seqs, c.num_heads, c.num_kv_heads,
                                   c.head_dim, c.block_size, c.table_width, c.num_blocks,
                                   max_len, c.scale, c.dtype, rt->ws, rt->ws_bytes, &o,
                                   rt->s_run);
        }
        if (rc != PA_OK) return rc;
    }
    return PA_OK;
}

}  // namespace

extern "C" {

int pa_rt_create(pa_runtime **out, const pa_runtime_config *cfg, void *k_cache, void *v_cache,
                 const int32_t *free_order) {
    pa::clear_error();
    if (!out || !cfg) return pa::fail(PA_ERR_INVALID_ARG, "runtime: NULL argument");
    *out = nullptr;
    const pa_runtime_config &c = *cfg;
    if (c.dtype != PA_F32 && c.dtype != PA_BF16 && c.dtype != PA_F16)
        return pa::fail(PA_ERR_UNSUPPORTED, "runtime: dtype %d", c.dtype);
    if (c.num_blocks <= 0 || c.block_size <= 0 || c.num_heads <= 0 || c.num_kv_heads <= 0 ||
        c.head_dim <= 0 || c.table_width <= 0 || c.max_batch <= 0 || c.max_new_tokens <= 0 ||
        c.num_heads % c.num_kv_heads != 0)
        return pa::fail(PA_ERR_INVALID_ARG, "runtime: bad sizes");
    if (!k_cache || !v_cache) return pa::fail(PA_ERR_INVALID_ARG, "runtime: NULL cache");
    pa_runtime *rt = new (std::nothrow) pa_runtime();
    if (!rt) return pa::fail(PA_ERR_INVALID_ARG, "runtime: out of host memory");
    rt->cfg = c;
    rt->k_cache = k_cache;
    rt->v_cache = v_cache;
    rt->elem = c.dtype == PA_F32 ? 4 : 2;
    int rc = pa_alloc_create(&rt->alloc, c.num_blocks, c.block_size, c.max_blocks_per_seq,
                             free_order);
    if (rc != PA_OK) {
        release(rt);
        return rc;
    }
    // the arrays of the largest step: slots and pairs of max_new_tokens
    // appends, max_batch table rows, lengths and order
    rt->arrays_cap = a256(16 + 8 * (size_t)c.max_new_tokens) +
                     a256(16 * (size_t)c.max_new_tokens) +
                     a256(4 * (size_t)c.max_batch * c.table_width) +
                     2 * a256(4 * (size_t)c.max_batch) + 256;
    rt->kv_cap = a256((size_t)c.max_new_tokens * c.num_kv_heads * c.head_dim * rt->elem);
    rt->q_cap = a256((size_t)c.max_batch * c.num_heads * c.head_dim * rt->elem);
    rt->off_k = rt->arrays_cap;
    rt->off_v = rt->off_k + rt->kv_cap;
    rt->off_q = rt->off_v + rt->kv_cap;
    rt->slot_bytes = rt->off_q + rt->q_cap;
    rt->out_bytes = (size_t)c.max_batch * c.num_heads * c.head_dim * sizeof(float);
    // partials for the shortest split pa_decode_choose picks (256 tokens)
    rt->ws_bytes = pa_decode_workspace_size(c.max_batch, c.num_heads, c.head_dim,
                                            c.table_width * c.block_size, 256);
    cudaError_t e = cudaGetDevice(&rt->dev);
    for (int i = 0; i < 2 && e == cudaSuccess; ++i) {
        e = cudaHostAlloc(reinterpret_cast<void **>(&rt->host[i]), rt->arrays_cap,
                          cudaHostAllocDefault);
        if (e == cudaSuccess) e = cudaMalloc(reinterpret_cast<void **>(&rt->devb[i]), rt->slot_bytes);
        if (e == cudaSuccess) e = cudaMalloc(reinterpret_cast<void **>(&rt->out_dev[i]), rt->out_bytes);
        for (cudaEvent_t *ev : {&rt->ev_in[i], &rt->ev_run[i], &rt->ev_out[i]})
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
    }
    if (e == cudaSuccess && rt->ws_bytes) e = cudaMalloc(&rt->ws, rt->ws_bytes);
    for (cudaStream_t *s : {&rt->s_in, &rt->s_run, &rt->s_out})
        if (e == cudaSuccess) e = cudaStreamCreateWithFlags(s, cudaStreamNonBlocking);
    if (e != cudaSuccess) {
        rc = cuda_err(e, "creating buffers and streams");
        release(rt);
        return rc;
    }
    *out = rt;
    return PA_OK;
}

void pa_rt_destroy(pa_runtime *rt) {
    if (!rt) return;
    cudaStreamSynchronize(rt->s_in);
    cudaStreamSynchronize(rt->s_run);
    cudaStreamSynchronize(rt->s_out);
    release(rt);
}

pa_alloc *pa_rt_allocator(pa_runtime *rt) { return rt ? rt->alloc : nullptr; }

int pa_rt_stats(const pa_runtime *rt, int64_t *steps, int64_t *replays, int64_t *captures) {
    pa::clear_error();
    if (!rt) return pa::fail(PA_ERR_INVALID_ARG, "runtime: NULL");
    if (steps) *steps = rt->steps;
    if (replays) *replays = rt->replays;
    if (captures) *captures = rt->captures;
    return PA_OK;
}

int pa_event_wait(void *event) {
    pa::clear_error();
    if (!event) return pa::fail(PA_ERR_INVALID_ARG, "NULL event");
    const cudaError_t e = cudaEventSynchronize(static_cast<cudaEvent_t>(event));
    return e == cudaSuccess ? PA_OK : cuda_err(e, "cudaEventSynchronize");
}

int pa_rt_wait(pa_runtime *rt) {
    pa::clear_error();
    if (!rt) return pa::fail(PA_ERR_INVALID_ARG, "runtime: NULL");
    for (cudaStream_t s : {rt->s_in, rt->s_run, rt->s_out}) {
        const cudaError_t e = cudaStreamSynchronize(s);
        if (e != cudaSuccess) return cuda_err(e, "synchronize");
    }
    return PA_OK;
}

int pa_rt_step(pa_runtime *rt, const int64_t *events, int n_events, const int64_t *decode_ids,
               int num_seqs, const void *k_new, const void *v_new, const void *q, float *out,
               void **ready) {
    pa::clear_error();
    if (!rt) return pa::fail(PA_ERR_INVALID_ARG, "runtime: NULL");
    const pa_runtime_config &c = rt->cfg;
    if (num_seqs < 0 || num_seqs > c.max_batch)
        return pa::fail(PA_ERR_INVALID_ARG, "runtime: %d decode rows > max_batch %d", num_seqs,
                        c.max_batch);
    if (n_events < 0 || (n_events > 0 && !events))
        return pa::fail(PA_ERR_INVALID_ARG, "runtime: bad events");
    // sizes from the events, before anything is applied
    int64_t n_slots = 0;
    for (int i = 0; i < n_events; ++i)
        if (events[3 * i] == PA_EV_APPEND && events[3 * i + 2] > 0) n_slots += events[3 * i + 2];
    if (n_slots > c.max_new_tokens)
        return pa::fail(PA_ERR_INVALID_ARG, "runtime: %lld new tokens > max_new_tokens %d",
                        (long long)n_slots, c.max_new_tokens);
    if ((n_slots > 0 && (!k_new || !v_new)) || (num_seqs > 0 && (!q || !out)))
        return pa::fail(PA_ERR_INVALID_ARG, "runtime: NULL input or output");
    const int s = rt->next;
    rt->next ^= 1;
    cudaError_t e;
    // The new K/V rows and the queries go in first: they come from the
    // caller's buffers to fixed places of the slot's device buffer and need
    // nothing from the plan, so the host link starts on them while the host
    // plans.  The slot's device buffer is rewritten once its previous
    // kernels are done with it.
    const size_t row = (size_t)c.num_kv_heads * c.head_dim * rt->elem;
    const size_t qb = (size_t)num_seqs * c.num_heads * c.head_dim * rt->elem;
    if ((rt->used[s] && (e = cudaStreamWaitEvent(rt->s_in, rt->ev_run[s], 0)) != cudaSuccess) ||
        (n_slots > 0 &&
         ((e = cudaMemcpyAsync(rt->devb[s] + rt->off_k, k_new, n_slots * row,
                               cudaMemcpyHostToDevice, rt->s_in)) != cudaSuccess ||
          (e = cudaMemcpyAsync(rt->devb[s] + rt->off_v, v_new, n_slots * row,
                               cudaMemcpyHostToDevice, rt->s_in)) != cudaSuccess)) ||
        (qb > 0 && (e = cudaMemcpyAsync(rt->devb[s] + rt->off_q, q, qb, cudaMemcpyHostToDevice,
                                        rt->s_in)) != cudaSuccess))
        return cuda_err(e, "copy in");
    // (from here on, a failing call first lets those copies finish, so that
    // the caller may reuse its buffers once the call has returned)
    auto fail_after_copies = [&](int code) {
        cudaStreamSynchronize(rt->s_in);
        return code;
    };
    // the slot's host buffer is free once its previous copy in has run
    if (rt->used[s] && (e = cudaEventSynchronize(rt->ev_in[s])) != cudaSuccess)
        return fail_after_copies(cuda_err(e, "waiting for the staging buffer"));
    rt->pairs_before.resize((size_t)n_events + 1);
    pa_step_layout lay;
    int rc = pa_step_plan(rt->alloc, events, n_events, decode_ids, num_seqs, c.table_width,
                          rt->host[s], rt->arrays_cap, rt->pairs_before.data(), &lay);
    if (rc != PA_OK) return fail_after_copies(rc);
    // device actions in event order
    rt->acts.clear();
    int decode_at = -1;
    int64_t rows = 0;  // K/V rows of the appends before event i
    for (int i = 0; i < n_events;) {
        const int64_t code = events[3 * i];
        if (code == PA_EV_APPEND) {
            int j = i;
            const int64_t r0 = rows;
            while (j < n_events && events[3 * j] == PA_EV_APPEND) rows += events[3 * j++ + 2];
            rt->acts.push_back({0, (int)r0, (int)rows, rt->pairs_before[i],
                                rt->pairs_before[j], false});
            i = j;
            continue;
        }
        if (code == PA_EV_DECODE) {
            decode_at = (int)rt->acts.size();
            rt->acts.push_back({1, 0, 0, 0, 0, false});
            // one-token appends of exactly the decode batch, in its order
            if (decode_at > 0 && i > 0 && events[3 * (i - 1)] == PA_EV_APPEND) {
                Act &w = rt->acts[decode_at - 1];
                bool ok = w.r1 - w.r0 == num_seqs && i - num_seqs >= 0;
                for (int r = 0; ok && r < num_seqs; ++r) {
                    const int64_t *ev = events + 3 * (i - num_seqs + r);
                    ok = ev[0] == PA_EV_APPEND && ev[1] == decode_ids[r] && ev[2] == 1;
                }
                w.fused = ok && num_seqs > 0;
            }
        }
        ++i;
    }
    // the decode's kernel and split, from the lengths
    pa_decode_opts opts;
    std::memset(&opts, 0, sizeof(opts));
    int max_len = 0;
    if (decode_at >= 0 && num_seqs > 0) {
        const int32_t *lens = reinterpret_cast<const int32_t *>(rt->host[s] + lay.off_lens);
        rc = pa_decode_choose(lens, num_seqs, c.num_kv_heads, c.head_dim, c.block_size, c.dtype,
                              0, &opts);
        if (rc != PA_OK) return fail_after_copies(rc);
        // a power-of-two bound on the lengths (at least 512, at most the
        // table's capacity) keeps a graph's grid fixed while steps change little
        max_len = 512;
        while (max_len < lay.max_seq_len) max_len *= 2;
        max_len = std::min(max_len, c.table_width * c.block_size);
    }
    // the step's arrays (slots, pairs, table rows, lengths, order) follow
    // the rows on the copy-in stream; the kernels wait for all of it
    if ((e = cudaMemcpyAsync(rt->devb[s], rt->host[s], lay.bytes, cudaMemcpyHostToDevice,
                             rt->s_in)) != cudaSuccess ||
        (e = cudaEventRecord(rt->ev_in[s], rt->s_in)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(rt->s_run, rt->ev_in[s], 0)) != cudaSuccess)
        return fail_after_copies(cuda_err(e, "copy in"));
    // the slot's output buffer is rewritten once its previous copy out is done
    if (rt->used[s] && (e = cudaStreamWaitEvent(rt->s_run, rt->ev_out[s], 0)) != cudaSuccess)
        return cuda_err(e, "ordering the output");
    // the kernels: from a graph when the layout has one, else directly
    const bool graphable = lay.n_pairs == 0 && decode_at >= 0 && num_seqs > 0;
    std::vector<int64_t> key;
    if (graphable) {
        // everything the captured launches take: the array offsets (they
        // follow the events' counts), the decode's choice and bound, and the
        // actions' row ranges and fusion
        key = {s, lay.n_slots, num_seqs, lay.off_pairs, lay.off_tables, lay.off_lens,
               lay.off_order, opts.partition_size, opts.variant, opts.heads_per_cta, max_len,
               (int64_t)rt->acts.size()};
        for (const Act &a : rt->acts) {
            key.push_back(a.kind);
            key.push_back(a.r0);
            key.push_back(a.r1);
            key.push_back(a.fused);
        }
    }
    auto it = graphable ? rt->graphs.find(key) : rt->graphs.end();
    if (it != rt->graphs.end()) {
        if ((e = cudaGraphLaunch(it->second.exec, rt->s_run)) != cudaSuccess)
            return cuda_err(e, "graph launch");
        ++rt->replays;
    } else {
        rc = launch_step(rt, s, lay, num_seqs, opts, max_len);
        if (rc != PA_OK) return rc;
        if (graphable) {
            // capture the layout for the steps to come (capture runs nothing)
            cudaGraph_t g = nullptr;
            Graph gr;
            e = cudaStreamBeginCapture(rt->s_run, cudaStreamCaptureModeThreadLocal);
            if (e == cudaSuccess) {
                rc = launch_step(rt, s, lay, num_seqs, opts, max_len);
                e = cudaStreamEndCapture(rt->s_run, &g);
                if (rc == PA_OK && e == cudaSuccess)
                    e = cudaGraphInstantiateWithFlags(&gr.exec, g, 0);
                if (g) cudaGraphDestroy(g);
            }
            if (rc != PA_OK) return rc;
            if (e != cudaSuccess) return cuda_err(e, "graph capture");
            rt->graphs.emplace(key, gr);
            ++rt->captures;
        }
    }
    if ((e = cudaEventRecord(rt->ev_run[s], rt->s_run)) != cudaSuccess)
        return cuda_err(e, "cudaEventRecord");
    // copy out; the step's "ready" event follows its kernels in any case
    if ((e = cudaStreamWaitEvent(rt->s_out, rt->ev_run[s], 0)) != cudaSuccess)
        return cuda_err(e, "ordering the copy out");
    if (num_seqs > 0 && decode_at >= 0 &&
        (e = cudaMemcpyAsync(out, rt->out_dev[s],
                             (size_t)num_seqs * c.num_heads * c.head_dim * sizeof(float),
                             cudaMemcpyDeviceToHost, rt->s_out)) != cudaSuccess)
        return cuda_err(e, "copy out");
    if ((e = cudaEventRecord(rt->ev_out[s], rt->s_out)) != cudaSuccess)
        return cuda_err(e, "cudaEventRecord");
    rt->used[s] = true;
    ++rt->steps;
    if (ready) *ready = rt->ev_out[s];
    return PA_OK;
}

}  // extern "C"
