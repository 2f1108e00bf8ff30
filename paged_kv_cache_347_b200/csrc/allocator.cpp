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
// Two extensions sit on the same state:
//  * prefix caching (paweldubiel.com "PagedAttention": block sharing "is also
//    useful in Prefix Caching"; sanketn26 "Use a runtime that owns the
//    blocks": prefix reuse within a paged runtime): a full block whose tokens
//    are known is indexed by (parent block, its tokens); a new sequence whose
//    leading tokens match a chain of indexed blocks shares them instead of
//    recomputing them.  Indexed blocks stay indexed after release, while they
//    wait in the free list, and are dropped from the index when the free list
//    hands them out again;
//  * preemption by swap (sanketn26 "What this does not solve": excess
//    admission can cause "preemption"; mbrenndoerfer.com bullet 5): a
//    sequence's blocks move to a pool of host blocks and back.
//
// Pure host code; no CUDA.
#include <algorithm>
#include <cstdint>
#include <climits>
#include <cstring>
#include <deque>
#include <new>
#include <string>
#include <unordered_map>
#include <utility>
#include <vector>

#include "../../include/pagedattn.h"
#include "status.h"

namespace {

// FIFO of block ids that also lets any entry be taken out (a cached block
// reclaimed by a prefix match).  Removal is lazy: a generation counter per
// block marks queue entries that no longer count.
class FreeList {
  public:
    void init(int n) {
        q_.clear();
        gen_.assign(n, 0);
        in_.assign(n, 0);
        count_ = 0;
    }
    void push_back(int32_t b) {
        ++gen_[b];
        in_[b] = 1;
        q_.emplace_back(b, gen_[b]);
        ++count_;
    }
    void push_front(int32_t b) {
        ++gen_[b];
        in_[b] = 1;
        q_.emplace_front(b, gen_[b]);
        ++count_;
    }
    bool contains(int32_t b) const { return in_[b] != 0; }
    void remove(int32_t b) {
        if (!in_[b]) return;
        ++gen_[b];
        in_[b] = 0;
        --count_;
    }
    int32_t pop_front() {  // caller checks size() > 0
        while (!q_.empty()) {
            const auto e = q_.front();
            q_.pop_front();
            if (in_[e.first] && gen_[e.first] == e.second) {
                in_[e.first] = 0;
                --count_;
                return e.first;
            }
        }
        return -1;
    }
    int64_t size() const { return count_; }
    template <typename F> void for_each(F f) const {
        for (const auto &e : q_)
            if (in_[e.first] && gen_[e.first] == e.second) f(e.first);
    }

  private:
    std::deque<std::pair<int32_t, uint32_t>> q_;
    std::vector<uint32_t> gen_;
    std::vector<char> in_;
    int64_t count_ = 0;
};

// Identity of a full block for prefix caching: the physical block holding the
// preceding tokens (-1 for the first block) and this block's token ids.
struct BlockKey {
    int32_t parent = -1;
    std::vector<int64_t> tokens;
    bool operator==(const BlockKey &o) const { return parent == o.parent && tokens == o.tokens; }
};

struct BlockKeyHash {
    size_t operator()(const BlockKey &k) const {
        uint64_t h = 0x9e3779b97f4a7c15ull ^ (uint64_t)(uint32_t)k.parent;
        for (int64_t t : k.tokens) {
            h ^= (uint64_t)t + 0x9e3779b97f4a7c15ull + (h << 6) + (h >> 2);
            h *= 0xff51afd7ed558ccdull;
        }
        return (size_t)(h ^ (h >> 33));
    }
};

struct Seq {
    std::vector<int32_t> table;
    int64_t len = 0;
    bool tracked = false;          // token ids of every position known
    std::vector<int64_t> tokens;   // valid while tracked
    bool swapped = false;
    std::vector<int32_t> host_table;
};

// What one append changed, enough to undo it exactly.
struct Undo {
    Seq *seq = nullptr;
    int64_t prev_len = 0;
    bool prev_tracked = false;
    int32_t cow_old = -1, cow_new = -1;
    int n_new = 0;  // blocks pushed onto the table (after the copy, if any)
    std::vector<std::pair<int32_t, BlockKey>> evicted;
};

}  // namespace

struct pa_alloc {
    int32_t num_blocks = 0;
    int32_t bs = 0;
    int32_t max_blocks = 0;
    FreeList free_list;
    std::vector<int32_t> ref;
    std::unordered_map<int64_t, Seq> seqs;
    // prefix cache
    std::unordered_map<BlockKey, int32_t, BlockKeyHash> index;
    std::vector<char> indexed;
    std::vector<BlockKey> key_of;
    int64_t hit_blocks = 0, query_blocks = 0, evicted_blocks = 0;
    // host pool for swapped-out sequences
    int32_t num_host_blocks = 0;
    FreeList host_free;

    // Takes the head of the free list for new use; drops it from the prefix
    // index if it was cached there.
    int32_t take_block(Undo *u) {
        const int32_t b = free_list.pop_front();
        if (indexed[b]) {
            if (u) u->evicted.emplace_back(b, key_of[b]);
            index.erase(key_of[b]);
            indexed[b] = 0;
            ++evicted_blocks;
        }
        return b;
    }

    void release(int32_t b) {
        ref[b] -= 1;
        if (ref[b] == 0) free_list.push_back(b);
    }

    int append(Seq &s, int n, int64_t *slots, int64_t *pair, int *n_pair, Undo *u) {
        if (n_pair) *n_pair = 0;
        if (s.swapped) return pa::fail(PA_ERR_INVALID_ARG, "sequence is swapped out");
        if (u) {
            u->seq = &s;
            u->prev_len = s.len;
            u->prev_tracked = s.tracked;
        }
        if (n == 0) return PA_OK;
        const int64_t L = s.len;
        const int64_t before = (L + bs - 1) / bs;
        const int64_t after = (L + n + bs - 1) / bs;
        const bool cow = (L % bs) != 0 && ref[s.table.back()] > 1;
        const int64_t need = (after - before) + (cow ? 1 : 0);
        if (max_blocks > 0 && after > max_blocks)
            return pa::fail(PA_ERR_SEQ_TOO_LONG, "sequence would need %lld blocks > %d",
                            (long long)after, max_blocks);
        if (need > free_list.size())
            return pa::fail(PA_ERR_OUT_OF_BLOCKS, "need %lld blocks, %lld free", (long long)need,
                            (long long)free_list.size());
        if (cow) {
            const int32_t old_b = s.table.back();
            const int32_t new_b = take_block(u);
            ref[old_b] -= 1;
            ref[new_b] = 1;
            s.table.back() = new_b;
            if (pair) { pair[0] = old_b; pair[1] = new_b; }
            if (n_pair) *n_pair = 1;
            if (u) { u->cow_old = old_b; u->cow_new = new_b; }
        }
        for (int64_t p = L; p < L + n; ++p) {
            if (p % bs == 0) {
                const int32_t b = take_block(u);
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
    // reverse of the order they were taken, which restores the queue exactly,
    // and blocks dropped from the prefix index are indexed again.
    void undo(const Undo &u) {
        Seq &s = *u.seq;
        for (int i = 0; i < u.n_new; ++i) {
            const int32_t b = s.table.back();
            s.table.pop_back();
            ref[b] = 0;
            free_list.push_front(b);
        }
        if (u.cow_new >= 0) {
            s.table.back() = u.cow_old;
            ref[u.cow_new] = 0;
            ref[u.cow_old] += 1;
            free_list.push_front(u.cow_new);
        }
        for (auto e = u.evicted.rbegin(); e != u.evicted.rend(); ++e) {
            index.emplace(e->second, e->first);
            key_of[e->first] = e->second;
            indexed[e->first] = 1;
            --evicted_blocks;
        }
        s.len = u.prev_len;
        s.tracked = u.prev_tracked;
    }

    // Indexes block j of a tracked sequence (full, tokens known) unless an
    // identical block is already indexed.
    void index_block(const Seq &s, int64_t j) {
        BlockKey k;
        k.parent = j == 0 ? -1 : s.table[j - 1];
        k.tokens.assign(s.tokens.begin() + j * bs, s.tokens.begin() + (j + 1) * bs);
        const int32_t b = s.table[j];
        if (indexed[b] || index.count(k)) return;
        index.emplace(k, b);
        key_of[b] = std::move(k);
        indexed[b] = 1;
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
    a->indexed.assign(num_blocks, 0);
    a->key_of.resize(num_blocks);
    a->free_list.init(num_blocks);
    a->host_free.init(0);
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
            a->free_list.push_back(b);
        }
    } else {
        for (int i = 0; i < num_blocks; ++i) a->free_list.push_back(i);
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
    const int rc = a->append(it->second, n_tokens, slots_out, cow_pair_out, n_cow_out, nullptr);
    if (rc == PA_OK && n_tokens > 0) it->second.tracked = false;  // token ids now unknown
    return rc;
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
                if (n > 0) it->second.tracked = false;
                done.push_back(std::move(u));
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

int pa_seq_add_cached(pa_alloc *a, int64_t seq_id, const int64_t *token_ids, int n_tokens,
                      int *n_cached_out) {
    pa::clear_error();
    if (!a) return pa::fail(PA_ERR_INVALID_ARG, "allocator is NULL");
    if (n_tokens < 0 || (n_tokens > 0 && !token_ids))
        return pa::fail(PA_ERR_INVALID_ARG, "bad token arguments");
    if (a->seqs.count(seq_id))
        return pa::fail(PA_ERR_INVALID_ARG, "sequence %lld exists", (long long)seq_id);
    Seq s;
    s.tracked = true;
    const int bs = a->bs;
    int64_t full = n_tokens / bs;
    if (a->max_blocks > 0 && full > a->max_blocks) full = a->max_blocks;
    BlockKey k;
    int64_t matched = 0;
    for (; matched < full; ++matched) {
        k.parent = matched == 0 ? -1 : s.table.back();
        k.tokens.assign(token_ids + matched * bs, token_ids + (matched + 1) * bs);
        auto hit = a->index.find(k);
        if (hit == a->index.end()) break;
        const int32_t b = hit->second;
        if (a->ref[b] == 0) a->free_list.remove(b);
        a->ref[b] += 1;
        s.table.push_back(b);
    }
    a->hit_blocks += matched;
    a->query_blocks += full;
    s.len = matched * bs;
    s.tokens.assign(token_ids, token_ids + s.len);
    a->seqs.emplace(seq_id, std::move(s));
    if (n_cached_out) *n_cached_out = (int)(matched * bs);
    return PA_OK;
}

int pa_seq_append_tokens(pa_alloc *a, int64_t seq_id, const int64_t *token_ids, int n_tokens,
                         int64_t *slots_out, int64_t *cow_pair_out, int *n_cow_out) {
    pa::clear_error();
    if (!a) return pa::fail(PA_ERR_INVALID_ARG, "allocator is NULL");
    if (n_tokens < 0 || (n_tokens > 0 && (!token_ids || !slots_out)))
        return pa::fail(PA_ERR_INVALID_ARG, "bad token arguments");
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end())
        return pa::fail(PA_ERR_UNKNOWN_SEQ, "unknown sequence %lld", (long long)seq_id);
    Seq &s = it->second;
    if (!s.tracked)
        return pa::fail(PA_ERR_INVALID_ARG,
                        "sequence %lld has no token history (not made by pa_seq_add_cached)",
                        (long long)seq_id);
    const int64_t L = s.len;
    const int rc = a->append(s, n_tokens, slots_out, cow_pair_out, n_cow_out, nullptr);
    if (rc != PA_OK) return rc;
    s.tokens.insert(s.tokens.end(), token_ids, token_ids + n_tokens);
    for (int64_t j = L / a->bs; j < s.len / a->bs; ++j) a->index_block(s, j);
    return PA_OK;
}

int pa_seq_fork(pa_alloc *a, int64_t parent, int64_t child) {
    pa::clear_error();
    if (!a) return pa::fail(PA_ERR_INVALID_ARG, "allocator is NULL");
    auto it = a->seqs.find(parent);
    if (it == a->seqs.end())
        return pa::fail(PA_ERR_UNKNOWN_SEQ, "unknown sequence %lld", (long long)parent);
    if (it->second.swapped) return pa::fail(PA_ERR_INVALID_ARG, "sequence is swapped out");
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
    if (it->second.swapped) {
        for (int32_t h : it->second.host_table) a->host_free.push_back(h);
    } else {
        for (int32_t b : it->second.table) a->release(b);
    }
    a->seqs.erase(it);
    return PA_OK;
}

int pa_alloc_set_host_pool(pa_alloc *a, int num_host_blocks) {
    pa::clear_error();
    if (!a) return pa::fail(PA_ERR_INVALID_ARG, "allocator is NULL");
    if (num_host_blocks < 0) return pa::fail(PA_ERR_INVALID_ARG, "negative host pool");
    for (const auto &kv : a->seqs)
        if (kv.second.swapped)
            return pa::fail(PA_ERR_INVALID_ARG, "host pool in use by sequence %lld",
                            (long long)kv.first);
    a->num_host_blocks = num_host_blocks;
    a->host_free.init(num_host_blocks);
    for (int i = 0; i < num_host_blocks; ++i) a->host_free.push_back(i);
    return PA_OK;
}

int pa_seq_swap_out(pa_alloc *a, int64_t seq_id, int64_t *pairs_out, int cap, int *n_pairs_out) {
    pa::clear_error();
    if (!a) return pa::fail(PA_ERR_INVALID_ARG, "allocator is NULL");
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end())
        return pa::fail(PA_ERR_UNKNOWN_SEQ, "unknown sequence %lld", (long long)seq_id);
    Seq &s = it->second;
    if (s.swapped) return pa::fail(PA_ERR_INVALID_ARG, "sequence is already swapped out");
    const int n = (int)s.table.size();
    if (n > cap || (n > 0 && !pairs_out))
        return pa::fail(PA_ERR_INVALID_ARG, "pairs_out holds %d pairs, %d needed", cap, n);
    if (n > a->host_free.size())
        return pa::fail(PA_ERR_OUT_OF_BLOCKS, "need %d host blocks, %lld free", n,
                        (long long)a->host_free.size());
    s.host_table.clear();
    for (int j = 0; j < n; ++j) {
        const int32_t h = a->host_free.pop_front();
        pairs_out[2 * j] = s.table[j];
        pairs_out[2 * j + 1] = h;
        s.host_table.push_back(h);
        a->release(s.table[j]);
    }
    s.table.clear();
    s.swapped = true;
    if (n_pairs_out) *n_pairs_out = n;
    return PA_OK;
}

int pa_seq_swap_in(pa_alloc *a, int64_t seq_id, int64_t *pairs_out, int cap, int *n_pairs_out) {
    pa::clear_error();
    if (!a) return pa::fail(PA_ERR_INVALID_ARG, "allocator is NULL");
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end())
        return pa::fail(PA_ERR_UNKNOWN_SEQ, "unknown sequence %lld", (long long)seq_id);
    Seq &s = it->second;
    if (!s.swapped) return pa::fail(PA_ERR_INVALID_ARG, "sequence is not swapped out");
    const int n = (int)s.host_table.size();
    if (n > cap || (n > 0 && !pairs_out))
        return pa::fail(PA_ERR_INVALID_ARG, "pairs_out holds %d pairs, %d needed", cap, n);
    if (n > a->free_list.size())
        return pa::fail(PA_ERR_OUT_OF_BLOCKS, "need %d blocks, %lld free", n,
                        (long long)a->free_list.size());
    s.table.clear();
    for (int j = 0; j < n; ++j) {
        const int32_t b = a->take_block(nullptr);
        a->ref[b] = 1;
        s.table.push_back(b);
        pairs_out[2 * j] = s.host_table[j];
        pairs_out[2 * j + 1] = b;
        a->host_free.push_back(s.host_table[j]);
    }
    s.host_table.clear();
    s.swapped = false;
    if (n_pairs_out) *n_pairs_out = n;
    return PA_OK;
}

int pa_seq_block_table(const pa_alloc *a, int64_t seq_id, int32_t *out, int cap, int *n_out,
                       int64_t *len_out) {
    pa::clear_error();
    if (!a) return pa::fail(PA_ERR_INVALID_ARG, "allocator is NULL");
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end())
        return pa::fail(PA_ERR_UNKNOWN_SEQ, "unknown sequence %lld", (long long)seq_id);
    const auto &t = it->second.swapped ? it->second.host_table : it->second.table;
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
        if (it->second.swapped)
            return pa::fail(PA_ERR_INVALID_ARG, "sequence %lld is swapped out",
                            (long long)seq_ids[i]);
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

// One step's events in a single call, written straight into the caller's
// staging buffer (see pagedattn.h): a runtime then hands the device one
// contiguous copy per step, and the host does no per-sequence work outside
// this loop.
int pa_step_plan(pa_alloc *a, const int64_t *events, int n_events, const int64_t *decode_ids,
                 int num_seqs, int width, void *stage, size_t stage_bytes,
                 int32_t *pairs_before, pa_step_layout *out) {
    pa::clear_error();
    if (!a || !out) return pa::fail(PA_ERR_INVALID_ARG, "allocator or layout is NULL");
    std::memset(out, 0, sizeof(*out));
    if (n_events < 0 || (n_events > 0 && !events) || num_seqs < 0 || width < 0 ||
        (num_seqs > 0 && !decode_ids))
        return pa::fail(PA_ERR_INVALID_ARG, "bad step arguments");
    // sizes from the events alone, before anything is applied
    int64_t n_slots = 0, n_appends = 0;
    int n_decode = 0;
    for (int i = 0; i < n_events; ++i) {
        const int64_t code = events[3 * i], n = events[3 * i + 2];
        if (code == PA_EV_APPEND) {
            if (n < 0 || n > INT32_MAX)
                return pa::fail(PA_ERR_INVALID_ARG, "event %d: token count %lld", i,
                                (long long)n);
            n_slots += n;
            n_appends += 1;
        } else if (code == PA_EV_DECODE) {
            n_decode += 1;
        } else if (code != PA_EV_ADD && code != PA_EV_FREE && code != PA_EV_FORK) {
            return pa::fail(PA_ERR_INVALID_ARG, "event %d: unknown code %lld", i,
                            (long long)code);
        }
    }
    if (n_decode > 1) return pa::fail(PA_ERR_INVALID_ARG, "more than one decode event");
    if (n_decode == 0 && num_seqs > 0)
        return pa::fail(PA_ERR_INVALID_ARG, "decode rows given without a decode event");
    if (n_slots > INT32_MAX) return pa::fail(PA_ERR_INVALID_ARG, "too many appended tokens");
    auto a16 = [](int64_t x) { return (x + 15) & ~int64_t(15); };
    out->n_slots = (int32_t)n_slots;
    out->num_seqs = num_seqs;
    out->width = width;
    out->off_slots = 0;
    out->off_pairs = a16(8 * n_slots);
    out->off_tables = out->off_pairs + a16(16 * n_appends);
    out->off_lens = out->off_tables + a16(4 * (int64_t)num_seqs * width);
    out->off_order = out->off_lens + a16(4 * (int64_t)num_seqs);
    out->bytes = out->off_order + 4 * (int64_t)num_seqs;
    if (!stage) return PA_OK;  // size query: nothing applied
    if ((reinterpret_cast<uintptr_t>(stage) & 15u) != 0)
        return pa::fail(PA_ERR_INVALID_ARG, "stage must be 16-byte aligned");
    if ((int64_t)stage_bytes < out->bytes)
        return pa::fail(PA_ERR_INVALID_ARG, "stage of %zu bytes, %lld needed", stage_bytes,
                        (long long)out->bytes);
    char *base = static_cast<char *>(stage);
    int64_t *slots = reinterpret_cast<int64_t *>(base + out->off_slots);
    int64_t *pairs = reinterpret_cast<int64_t *>(base + out->off_pairs);
    int32_t *tables = reinterpret_cast<int32_t *>(base + out->off_tables);
    int32_t *lens = reinterpret_cast<int32_t *>(base + out->off_lens);
    int32_t *order = reinterpret_cast<int32_t *>(base + out->off_order);

    int64_t slot_off = 0;
    int npairs = 0;
    std::vector<Undo> run;
    int i = 0;
    while (i < n_events) {
        const int64_t code = events[3 * i], x = events[3 * i + 1], y = events[3 * i + 2];
        int rc = PA_OK;
        if (code == PA_EV_APPEND) {
            // a run of consecutive appends is applied all or nothing
            const int first = i;
            const int pairs0 = npairs;
            run.clear();
            for (; i < n_events && events[3 * i] == PA_EV_APPEND; ++i) {
                if (pairs_before) pairs_before[i] = npairs;
                const int64_t sid = events[3 * i + 1];
                const int n = (int)events[3 * i + 2];
                auto it = a->seqs.find(sid);
                if (it == a->seqs.end()) {
                    rc = pa::fail(PA_ERR_UNKNOWN_SEQ, "event %d: unknown sequence %lld", i,
                                  (long long)sid);
                    break;
                }
                int got = 0;
                Undo u;
                rc = a->append(it->second, n, slots + slot_off, pairs + 2 * npairs, &got, &u);
                if (rc != PA_OK) break;
                if (n > 0) it->second.tracked = false;
                run.push_back(std::move(u));
                slot_off += n;
                npairs += got;
            }
            if (rc != PA_OK) {
                for (auto u = run.rbegin(); u != run.rend(); ++u) a->undo(*u);
                out->events_applied = first;
                out->n_pairs = pairs0;
                return rc;
            }
            continue;
        }
        if (pairs_before) pairs_before[i] = npairs;
        if (code == PA_EV_ADD) {
            rc = pa_seq_add(a, x);
        } else if (code == PA_EV_FREE) {
            rc = pa_seq_free(a, x);
        } else if (code == PA_EV_FORK) {
            rc = pa_seq_fork(a, x, y);
        } else {  // PA_EV_DECODE: the batch's rows as they stand here
            out->n_slots_pre = (int32_t)slot_off;
            out->n_pairs_pre = npairs;
            // each row's live entries only: the kernels read no entry past a
            // sequence's last block, so the rest is left as the buffer held it
            int32_t mx = 0;
            for (int r = 0; r < num_seqs && rc == PA_OK; ++r) {
                auto it = a->seqs.find(decode_ids[r]);
                if (it == a->seqs.end()) {
                    rc = pa::fail(PA_ERR_UNKNOWN_SEQ, "decode row %d: unknown sequence %lld", r,
                                  (long long)decode_ids[r]);
                } else if (it->second.swapped) {
                    rc = pa::fail(PA_ERR_INVALID_ARG, "decode row %d: sequence %lld is swapped out",
                                  r, (long long)decode_ids[r]);
                } else if ((int64_t)it->second.table.size() > width) {
                    rc = pa::fail(PA_ERR_SEQ_TOO_LONG, "decode row %d: %zu blocks > width %d", r,
                                  it->second.table.size(), width);
                } else {
                    const auto &t = it->second.table;
                    if (!t.empty())
                        std::memcpy(tables + (size_t)r * width, t.data(), sizeof(int32_t) * t.size());
                    lens[r] = (int32_t)it->second.len;
                    mx = lens[r] > mx ? lens[r] : mx;
                }
            }
            if (rc == PA_OK) {
                out->max_seq_len = mx;
                rc = pa_decode_order(lens, num_seqs, order);
            }
        }
        if (rc != PA_OK) {
            out->events_applied = i;
            out->n_pairs = npairs;
            return rc;
        }
        ++i;
    }
    if (n_decode == 0) {
        out->n_slots_pre = (int32_t)slot_off;
        out->n_pairs_pre = npairs;
    }
    if (pairs_before) pairs_before[n_events] = npairs;
    out->n_pairs = npairs;
    out->events_applied = n_events;
    return PA_OK;
}

int pa_decode_order(const int32_t *seq_lens_host, int num_seqs, int32_t *order_out) {
    pa::clear_error();
    if (num_seqs < 0 || (num_seqs > 0 && (!seq_lens_host || !order_out)))
        return pa::fail(PA_ERR_INVALID_ARG, "bad arguments");
    for (int i = 0; i < num_seqs; ++i) order_out[i] = i;
    std::stable_sort(order_out, order_out + num_seqs, [&](int32_t x, int32_t y) {
        return seq_lens_host[x] > seq_lens_host[y];
    });
    return PA_OK;
}

int pa_alloc_stats(const pa_alloc *a, pa_alloc_stats_t *out) {
    pa::clear_error();
    if (!a || !out) return pa::fail(PA_ERR_INVALID_ARG, "NULL argument");
    pa_alloc_stats_t s;
    std::memset(&s, 0, sizeof(s));
    s.num_blocks = a->num_blocks;
    s.free_blocks = a->free_list.size();
    for (int32_t r : a->ref) {
        s.used_blocks += r > 0;
        s.shared_blocks += r > 1;
    }
    s.num_seqs = (int64_t)a->seqs.size();
    for (const auto &kv : a->seqs) {
        s.table_entries += (int64_t)kv.second.table.size();
        s.logical_tokens += kv.second.len;
        s.swapped_seqs += kv.second.swapped;
    }
    s.reserved_slots = s.used_blocks * a->bs;
    s.cached_blocks = (int64_t)a->index.size();
    s.prefix_hit_blocks = a->hit_blocks;
    s.prefix_query_blocks = a->query_blocks;
    s.evicted_blocks = a->evicted_blocks;
    s.host_blocks = a->num_host_blocks;
    s.host_free_blocks = a->host_free.size();
    *out = s;
    return PA_OK;
}

int pa_alloc_free_list(const pa_alloc *a, int32_t *out, int cap, int *n_out) {
    pa::clear_error();
    if (!a) return pa::fail(PA_ERR_INVALID_ARG, "allocator is NULL");
    int i = 0;
    if (out)
        a->free_list.for_each([&](int32_t b) {
            if (i < cap) out[i++] = b;
        });
    if (n_out) *n_out = (int)a->free_list.size();
    return PA_OK;
}

int pa_alloc_refcount(const pa_alloc *a, int block) {
    if (!a || block < 0 || block >= a->num_blocks) return -1;
    return a->ref[block];
}

}  // extern "C"
