// Host block allocator behind the C ABI (pagedattn.h, "Host block allocator").
//
// PagedAttention's memory manager, as the pages describe it: fixed-size
// physical blocks handed out one at a time as a sequence grows (paweldubiel.com
// "PagedAttention", "Mechanism and details"), a per-sequence table from logical
// to physical block (sanketn26 "PagedAttention", "Separate logical order from
// physical location"), blocks shared between forks with copy-on-write before a
// shared block is changed ("Sharing needs ownership rules"; mbrenndoerfer.com
// "Paged Attention > Summary", bullet 4) and released when the last sequence
// using them finishes ("Exercise and checkpoint").  The free-list order, the
// copy-on-write decision point and the release order are fixed as stated in
// pagedattn.h so that slots and tables are reproducible bit for bit.
//
// Pure host code; no CUDA.
#include <cstdint>
#include <cstring>
#include <deque>
#include <new>
#include <string>
#include <unordered_map>
#include <vector>

#include "../../include/pagedattn.h"
#include "status.h"

namespace {

struct Seq {
    std::vector<int32_t> table;
    int64_t len = 0;
};

// What one append changed, enough to undo it exactly.
struct Undo {
    Seq *seq;
    int64_t prev_len;
    int32_t cow_old = -1, cow_new = -1;
    int n_new = 0;  // blocks pushed onto the table (after the copy, if any)
};

}  // namespace

struct pa_alloc {
    int32_t num_blocks = 0;
    int32_t bs = 0;
    int32_t max_blocks = 0;
    std::deque<int32_t> free_q;
    std::vector<int32_t> ref;
    std::unordered_map<int64_t, Seq> seqs;

    int append(Seq &s, int n, int64_t *slots, int64_t *pair, int *n_pair, Undo *u) {
        if (n_pair) *n_pair = 0;
        if (n == 0) {
            if (u) { u->seq = &s; u->prev_len = s.len; }
            return PA_OK;
        }
        const int64_t L = s.len;
        const int64_t before = (L + bs - 1) / bs;
        const int64_t after = (L + n + bs - 1) / bs;
        const bool cow = (L % bs) != 0 && ref[s.table.back()] > 1;
        const int64_t need = (after - before) + (cow ? 1 : 0);
        if (max_blocks > 0 && after > max_blocks)
            return pa::fail(PA_ERR_SEQ_TOO_LONG, "sequence would need %lld blocks > %d",
                            (long long)after, max_blocks);
        if (need > (int64_t)free_q.size())
            return pa::fail(PA_ERR_OUT_OF_BLOCKS, "need %lld blocks, %zu free", (long long)need,
                            free_q.size());
        if (u) { u->seq = &s; u->prev_len = L; }
        if (cow) {
            const int32_t old_b = s.table.back();
            const int32_t new_b = free_q.front();
            free_q.pop_front();
            ref[old_b] -= 1;
            ref[new_b] = 1;
            s.table.back() = new_b;
            if (pair) { pair[0] = old_b; pair[1] = new_b; }
            if (n_pair) *n_pair = 1;
            if (u) { u->cow_old = old_b; u->cow_new = new_b; }
        }
        for (int64_t p = L; p < L + n; ++p) {
            if (p % bs == 0) {
                const int32_t b = free_q.front();
                free_q.pop_front();
                ref[b] = 1;
                s.table.push_back(b);
                if (u) u->n_new += 1;
            }
            slots[p - L] = (int64_t)s.table[p / bs] * bs + p % bs;
        }
        s.len = L + n;
        return PA_OK;
    }

    // Reverses one append: blocks go back to the head of the free list in the
    // reverse of the order they were taken, which restores the queue exactly.
    void undo(const Undo &u) {
        Seq &s = *u.seq;
        for (int i = 0; i < u.n_new; ++i) {
            const int32_t b = s.table.back();
            s.table.pop_back();
            ref[b] = 0;
            free_q.push_front(b);
        }
        if (u.cow_new >= 0) {
            s.table.back() = u.cow_old;
            ref[u.cow_new] = 0;
            ref[u.cow_old] += 1;
            free_q.push_front(u.cow_new);
        }
        s.len = u.prev_len;
    }
};

extern "C" {

int pa_alloc_create(pa_alloc **out, int num_blocks, int block_size, int max_blocks_per_seq,
                    const int32_t *free_order) {
    pa::clear_error();
    if (!out) return pa::fail(PA_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    if (num_blocks <= 0 || block_size <= 0 || max_blocks_per_seq < 0)
        return pa::fail(PA_ERR_INVALID_ARG, "bad sizes: num_blocks=%d block_size=%d max=%d",
                        num_blocks, block_size, max_blocks_per_seq);
    pa_alloc *a = new (std::nothrow) pa_alloc();
    if (!a) return pa::fail(PA_ERR_INVALID_ARG, "out of host memory");
    a->num_blocks = num_blocks;
    a->bs = block_size;
    a->max_blocks = max_blocks_per_seq;
    a->ref.assign(num_blocks, 0);
    if (free_order) {
        std::vector<char> seen(num_blocks, 0);
        for (int i = 0; i < num_blocks; ++i) {
            const int32_t b = free_order[i];
            if (b < 0 || b >= num_blocks || seen[b]) {
                delete a;
                return pa::fail(PA_ERR_INVALID_ARG,
                                "free_order is not a permutation of 0..%d", num_blocks - 1);
            }
            seen[b] = 1;
            a->free_q.push_back(b);
        }
    } else {
        for (int i = 0; i < num_blocks; ++i) a->free_q.push_back(i);
    }
    *out = a;
    return PA_OK;
}

void pa_alloc_destroy(pa_alloc *a) { delete a; }

int pa_seq_add(pa_alloc *a, int64_t seq_id) {
    pa::clear_error();
    if (!a) return pa::fail(PA_ERR_INVALID_ARG, "allocator is NULL");
    if (a->seqs.count(seq_id))
        return pa::fail(PA_ERR_INVALID_ARG, "sequence %lld exists", (long long)seq_id);
    a->seqs.emplace(seq_id, Seq());
    return PA_OK;
}

int pa_seq_append(pa_alloc *a, int64_t seq_id, int n_tokens, int64_t *slots_out,
                  int64_t *cow_pair_out, int *n_cow_out) {
    pa::clear_error();
    if (!a) return pa::fail(PA_ERR_INVALID_ARG, "allocator is NULL");
    if (n_tokens < 0) return pa::fail(PA_ERR_INVALID_ARG, "negative token count");
    if (n_tokens > 0 && !slots_out) return pa::fail(PA_ERR_INVALID_ARG, "slots_out is NULL");
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end())
        return pa::fail(PA_ERR_UNKNOWN_SEQ, "unknown sequence %lld", (long long)seq_id);
    return a->append(it->second, n_tokens, slots_out, cow_pair_out, n_cow_out, nullptr);
}

int pa_batch_append(pa_alloc *a, const int64_t *seq_ids, int n_seqs, const int32_t *n_tokens,
                    int64_t *slots_out, int64_t *cow_pairs_out, int *n_cow_out) {
    pa::clear_error();
    if (!a) return pa::fail(PA_ERR_INVALID_ARG, "allocator is NULL");
    if (n_seqs < 0 || (n_seqs > 0 && (!seq_ids || !slots_out)))
        return pa::fail(PA_ERR_INVALID_ARG, "bad batch arguments");
    std::vector<Undo> done;
    done.reserve(n_seqs);
    int64_t off = 0;
    int npairs = 0;
    for (int i = 0; i < n_seqs; ++i) {
        const int n = n_tokens ? n_tokens[i] : 1;
        int rc = PA_OK;
        auto it = a->seqs.find(seq_ids[i]);
        if (n < 0) {
            rc = pa::fail(PA_ERR_INVALID_ARG, "negative token count at %d", i);
        } else if (it == a->seqs.end()) {
            rc = pa::fail(PA_ERR_UNKNOWN_SEQ, "unknown sequence %lld",
                          (long long)seq_ids[i]);
        } else {
            int got = 0;
            Undo u;
            rc = a->append(it->second, n, slots_out + off,
                           cow_pairs_out ? cow_pairs_out + 2 * npairs : nullptr, &got, &u);
            if (rc == PA_OK) {
                done.push_back(u);
                off += n;
                npairs += got;
            }
        }
        if (rc != PA_OK) {
            for (auto u = done.rbegin(); u != done.rend(); ++u) a->undo(*u);
            if (n_cow_out) *n_cow_out = 0;
            return rc;
        }
    }
    if (n_cow_out) *n_cow_out = npairs;
    return PA_OK;
}

int pa_seq_fork(pa_alloc *a, int64_t parent, int64_t child) {
    pa::clear_error();
    if (!a) return pa::fail(PA_ERR_INVALID_ARG, "allocator is NULL");
    auto it = a->seqs.find(parent);
    if (it == a->seqs.end())
        return pa::fail(PA_ERR_UNKNOWN_SEQ, "unknown sequence %lld", (long long)parent);
    if (a->seqs.count(child))
        return pa::fail(PA_ERR_INVALID_ARG, "sequence %lld exists", (long long)child);
    Seq c = it->second;  // copy before emplace may rehash
    for (int32_t b : c.table) a->ref[b] += 1;
    a->seqs.emplace(child, std::move(c));
    return PA_OK;
}

int pa_seq_free(pa_alloc *a, int64_t seq_id) {
    pa::clear_error();
    if (!a) return pa::fail(PA_ERR_INVALID_ARG, "allocator is NULL");
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end())
        return pa::fail(PA_ERR_UNKNOWN_SEQ, "unknown sequence %lld", (long long)seq_id);
    for (int32_t b : it->second.table) {
        a->ref[b] -= 1;
        if (a->ref[b] == 0) a->free_q.push_back(b);
    }
    a->seqs.erase(it);
    return PA_OK;
}

int pa_seq_block_table(const pa_alloc *a, int64_t seq_id, int32_t *out, int cap, int *n_out,
                       int64_t *len_out) {
    pa::clear_error();
    if (!a) return pa::fail(PA_ERR_INVALID_ARG, "allocator is NULL");
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end())
        return pa::fail(PA_ERR_UNKNOWN_SEQ, "unknown sequence %lld", (long long)seq_id);
    const auto &t = it->second.table;
    const int n = (int)t.size();
    if (out && cap > 0) std::memcpy(out, t.data(), sizeof(int32_t) * (size_t)(n < cap ? n : cap));
    if (n_out) *n_out = n;
    if (len_out) *len_out = it->second.len;
    return PA_OK;
}

int pa_block_tables(const pa_alloc *a, const int64_t *seq_ids, int n_seqs, int32_t *tables_out,
                    int width, int32_t *seq_lens_out) {
    pa::clear_error();
    if (!a) return pa::fail(PA_ERR_INVALID_ARG, "allocator is NULL");
    if (n_seqs < 0 || width < 0 || (n_seqs > 0 && (!seq_ids || (!tables_out && width > 0))))
        return pa::fail(PA_ERR_INVALID_ARG, "bad arguments");
    for (int i = 0; i < n_seqs; ++i) {
        auto it = a->seqs.find(seq_ids[i]);
        if (it == a->seqs.end())
            return pa::fail(PA_ERR_UNKNOWN_SEQ, "unknown sequence %lld", (long long)seq_ids[i]);
        const auto &t = it->second.table;
        if ((int64_t)t.size() > width)
            return pa::fail(PA_ERR_SEQ_TOO_LONG, "table of %lld has %zu entries > width %d",
                            (long long)seq_ids[i], t.size(), width);
        if (width > 0) {
            int32_t *row = tables_out + (size_t)i * width;
            if (!t.empty()) std::memcpy(row, t.data(), sizeof(int32_t) * t.size());
            std::memset(row + t.size(), 0, sizeof(int32_t) * (size_t)(width - (int)t.size()));
        }
        if (seq_lens_out) seq_lens_out[i] = (int32_t)it->second.len;
    }
    return PA_OK;
}

int pa_alloc_stats(const pa_alloc *a, pa_alloc_stats_t *out) {
    pa::clear_error();
    if (!a || !out) return pa::fail(PA_ERR_INVALID_ARG, "NULL argument");
    pa_alloc_stats_t s;
    std::memset(&s, 0, sizeof(s));
    s.num_blocks = a->num_blocks;
    s.free_blocks = (int64_t)a->free_q.size();
    for (int32_t r : a->ref) {
        s.used_blocks += r > 0;
        s.shared_blocks += r > 1;
    }
    s.num_seqs = (int64_t)a->seqs.size();
    for (const auto &kv : a->seqs) {
        s.table_entries += (int64_t)kv.second.table.size();
        s.logical_tokens += kv.second.len;
    }
    s.reserved_slots = s.used_blocks * a->bs;
    *out = s;
    return PA_OK;
}

int pa_alloc_free_list(const pa_alloc *a, int32_t *out, int cap, int *n_out) {
    pa::clear_error();
    if (!a) return pa::fail(PA_ERR_INVALID_ARG, "allocator is NULL");
    int i = 0;
    if (out)
        for (auto it = a->free_q.begin(); it != a->free_q.end() && i < cap; ++it) out[i++] = *it;
    if (n_out) *n_out = (int)a->free_q.size();
    return PA_OK;
}

int pa_alloc_refcount(const pa_alloc *a, int block) {
    if (!a || block < 0 || block >= a->num_blocks) return -1;
    return a->ref[block];
}

}  // extern "C"
