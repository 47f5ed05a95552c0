// Host block allocator with reference-counted copy-on-write.
//
// Follows, by page and section:
//  "PagedAttention and vLLM Architecture" (initnode.dev): section 1, a fixed pool
//  of B-token physical blocks allocated at startup and a per-request block table
//  kept by the serving engine; "Why Internal Fragmentation is Bounded", a block is
//  taken only when a new token overflows the last one, so at most B-1 slots of a
//  sequence are unused; section 3, parallel-sampling streams share a prompt's
//  blocks with a reference count, and a write into a shared block takes a new block
//  from the free pool, copies the block, decrements the old count and repoints only
//  the writer's table.
//  "PagedAttention Paper Breakdown" (fullstackaihub.com): section 2, the slot of
//  token i is T[floor(i/B)]*B + (i mod B); section 3, the other streams keep the
//  shared blocks untouched.
//
// Where the pages are silent: the free pool is a FIFO queue (initial order given
// by the caller, freed blocks appended in table order); a fork copies the parent's
// table and token count; a copy happens only for a write into a shared, partially
// filled last block (full shared blocks are never written); every failing call
// leaves the state as it was.
#include <cstdint>
#include <cstring>
#include <deque>
#include <new>
#include <string>
#include <unordered_map>
#include <vector>

#include "pa.h"

namespace pa {
void set_error(const std::string& msg);
}

struct pa_allocator {
    struct Seq {
        std::vector<int32_t> table;
        int64_t tokens = 0;
    };
    int32_t num_blocks = 0;
    int32_t block_size = 0;
    std::deque<int32_t> free_q;
    std::vector<int32_t> ref;
    std::unordered_map<int64_t, Seq> seqs;
    int64_t cow_copies = 0;

    int64_t slot_of(const Seq& q, int64_t i) const
    {
        return (int64_t)q.table[(size_t)(i / block_size)] * block_size + i % block_size;
    }

    int32_t take()
    {
        const int32_t b = free_q.front();
        free_q.pop_front();
        ref[(size_t)b] = 1;
        return b;
    }

    void give_back_front(int32_t b)
    {
        ref[(size_t)b] = 0;
        free_q.push_front(b);
    }

    // Undo record of one append, so a failing batch can be rolled back exactly.
    struct Undo {
        int64_t seq;
        int32_t fresh;     // block appended to the table (or -1)
        int32_t cow_src;   // block replaced by copy-on-write (or -1)
        int32_t cow_dst;
    };

    pa_status append(int64_t seq_id, int64_t* slot, int32_t* src, int32_t* dst, Undo* undo)
    {
        auto it = seqs.find(seq_id);
        if (it == seqs.end()) {
            pa::set_error("pa_alloc_append_slot: unknown sequence " + std::to_string(seq_id));
            return PA_ERR_INVALID;
        }
        Seq& q = it->second;
        const int64_t i = q.tokens;
        Undo u{seq_id, -1, -1, -1};
        *src = -1;
        *dst = -1;
        if (i % block_size == 0) {
            if (free_q.empty()) {
                pa::set_error("pa_alloc_append_slot: out of blocks");
                return PA_ERR_OOM;
            }
            u.fresh = take();
            q.table.push_back(u.fresh);
        } else {
            const int32_t last = q.table.back();
            if (ref[(size_t)last] > 1) {
                if (free_q.empty()) {
                    pa::set_error("pa_alloc_append_slot: out of blocks (copy-on-write)");
                    return PA_ERR_OOM;
                }
                const int32_t d = take();
                ref[(size_t)last] -= 1;
                q.table.back() = d;
                u.cow_src = last;
                u.cow_dst = d;
                *src = last;
                *dst = d;
                cow_copies += 1;
            }
        }
        q.tokens = i + 1;
        *slot = slot_of(q, i);
        if (undo) *undo = u;
        return PA_OK;
    }

    void rollback(const Undo& u)
    {
        Seq& q = seqs[u.seq];
        q.tokens -= 1;
        if (u.fresh >= 0) {
            q.table.pop_back();
            give_back_front(u.fresh);
        } else if (u.cow_dst >= 0) {
            q.table.back() = u.cow_src;
            ref[(size_t)u.cow_src] += 1;
            give_back_front(u.cow_dst);
            cow_copies -= 1;
        }
    }
};

extern "C" {

pa_allocator* pa_alloc_create(int num_blocks, int block_size, const int32_t* free_order)
{
    if (num_blocks <= 0 || block_size <= 0) {
        pa::set_error("pa_alloc_create: num_blocks and block_size must be > 0");
        return nullptr;
    }
    pa_allocator* a = new (std::nothrow) pa_allocator();
    if (!a) {
        pa::set_error("pa_alloc_create: host allocation failed");
        return nullptr;
    }
    a->num_blocks = num_blocks;
    a->block_size = block_size;
    a->ref.assign((size_t)num_blocks, 0);
    if (free_order) {
        std::vector<char> seen((size_t)num_blocks, 0);
        for (int i = 0; i < num_blocks; ++i) {
            const int32_t b = free_order[i];
            if (b < 0 || b >= num_blocks || seen[(size_t)b]) {
                delete a;
                pa::set_error("pa_alloc_create: free_order is not a permutation of 0..num_blocks-1");
                return nullptr;
            }
            seen[(size_t)b] = 1;
            a->free_q.push_back(b);
        }
    } else {
        for (int i = 0; i < num_blocks; ++i) a->free_q.push_back(i);
    }
    return a;
}

void pa_alloc_destroy(pa_allocator* a) { delete a; }

pa_status pa_alloc_add_seq(pa_allocator* a, int64_t seq_id, int num_tokens, int64_t* slots_out)
{
    if (!a || num_tokens < 0) {
        pa::set_error("pa_alloc_add_seq: bad argument");
        return PA_ERR_INVALID;
    }
    if (a->seqs.count(seq_id)) {
        pa::set_error("pa_alloc_add_seq: sequence " + std::to_string(seq_id) + " exists");
        return PA_ERR_INVALID;
    }
    const int64_t need = ((int64_t)num_tokens + a->block_size - 1) / a->block_size;
    if (need > (int64_t)a->free_q.size()) {
        pa::set_error("pa_alloc_add_seq: out of blocks");
        return PA_ERR_OOM;
    }
    pa_allocator::Seq q;
    q.table.reserve((size_t)need);
    for (int64_t k = 0; k < need; ++k) q.table.push_back(a->take());
    q.tokens = num_tokens;
    if (slots_out)
        for (int64_t i = 0; i < num_tokens; ++i) slots_out[i] = a->slot_of(q, i);
    a->seqs.emplace(seq_id, std::move(q));
    return PA_OK;
}

pa_status pa_alloc_fork(pa_allocator* a, int64_t parent_id, int64_t child_id)
{
    if (!a) return PA_ERR_INVALID;
    auto it = a->seqs.find(parent_id);
    if (it == a->seqs.end() || a->seqs.count(child_id)) {
        pa::set_error("pa_alloc_fork: unknown parent or existing child");
        return PA_ERR_INVALID;
    }
    pa_allocator::Seq child = it->second;
    for (int32_t b : child.table) a->ref[(size_t)b] += 1;
    a->seqs.emplace(child_id, std::move(child));
    return PA_OK;
}

pa_status pa_alloc_append_slot(pa_allocator* a, int64_t seq_id, int64_t* slot_out, int32_t* cow_src_out,
                               int32_t* cow_dst_out)
{
    if (!a || !slot_out) {
        pa::set_error("pa_alloc_append_slot: bad argument");
        return PA_ERR_INVALID;
    }
    int32_t src, dst;
    const pa_status st = a->append(seq_id, slot_out, &src, &dst, nullptr);
    if (st != PA_OK) return st;
    if (cow_src_out) *cow_src_out = src;
    if (cow_dst_out) *cow_dst_out = dst;
    return PA_OK;
}

pa_status pa_alloc_append_slots(pa_allocator* a, const int64_t* seq_ids, int n, int64_t* slots_out,
                                int64_t* cow_pairs_out, int* num_cow_out)
{
    if (!a || n < 0 || (n > 0 && (!seq_ids || !slots_out || !cow_pairs_out)) || !num_cow_out) {
        pa::set_error("pa_alloc_append_slots: bad argument");
        return PA_ERR_INVALID;
    }
    std::vector<pa_allocator::Undo> log((size_t)n);
    int ncow = 0;
    for (int k = 0; k < n; ++k) {
        int32_t src, dst;
        const pa_status st = a->append(seq_ids[k], &slots_out[k], &src, &dst, &log[(size_t)k]);
        if (st != PA_OK) {
            for (int u = k - 1; u >= 0; --u) a->rollback(log[(size_t)u]);
            return st;
        }
        if (src >= 0) {
            cow_pairs_out[2 * ncow] = src;
            cow_pairs_out[2 * ncow + 1] = dst;
            ++ncow;
        }
    }
    *num_cow_out = ncow;
    return PA_OK;
}

pa_status pa_alloc_free_seq(pa_allocator* a, int64_t seq_id)
{
    if (!a) return PA_ERR_INVALID;
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end()) {
        pa::set_error("pa_alloc_free_seq: unknown sequence " + std::to_string(seq_id));
        return PA_ERR_INVALID;
    }
    for (int32_t b : it->second.table) {
        a->ref[(size_t)b] -= 1;
        if (a->ref[(size_t)b] == 0) a->free_q.push_back(b);
    }
    a->seqs.erase(it);
    return PA_OK;
}

pa_status pa_alloc_block_table(const pa_allocator* a, int64_t seq_id, int32_t* out, int capacity, int* n_out)
{
    if (!a || !n_out) return PA_ERR_INVALID;
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end()) {
        pa::set_error("pa_alloc_block_table: unknown sequence " + std::to_string(seq_id));
        return PA_ERR_INVALID;
    }
    const auto& t = it->second.table;
    if ((int64_t)t.size() > capacity || (!out && !t.empty())) {
        pa::set_error("pa_alloc_block_table: capacity too small");
        return PA_ERR_INVALID;
    }
    if (!t.empty()) std::memcpy(out, t.data(), t.size() * sizeof(int32_t));
    *n_out = (int)t.size();
    return PA_OK;
}

pa_status pa_alloc_block_tables(const pa_allocator* a, const int64_t* seq_ids, int n, int32_t* out,
                                int max_blocks, int32_t fill, int32_t* context_lens_out)
{
    if (!a || n < 0 || max_blocks < 0 || (n > 0 && (!seq_ids || !out))) {
        pa::set_error("pa_alloc_block_tables: bad argument");
        return PA_ERR_INVALID;
    }
    for (int k = 0; k < n; ++k) {
        auto it = a->seqs.find(seq_ids[k]);
        if (it == a->seqs.end()) {
            pa::set_error("pa_alloc_block_tables: unknown sequence " + std::to_string(seq_ids[k]));
            return PA_ERR_INVALID;
        }
        if ((int64_t)it->second.table.size() > max_blocks) {
            pa::set_error("pa_alloc_block_tables: max_blocks too small");
            return PA_ERR_INVALID;
        }
    }
    for (int k = 0; k < n; ++k) {
        const auto& q = a->seqs.find(seq_ids[k])->second;
        int32_t* row = out + (size_t)k * max_blocks;
        for (int j = 0; j < max_blocks; ++j) row[j] = j < (int)q.table.size() ? q.table[(size_t)j] : fill;
        if (context_lens_out) context_lens_out[k] = (int32_t)q.tokens;
    }
    return PA_OK;
}

int pa_alloc_ref_count(const pa_allocator* a, int32_t block)
{
    if (!a || block < 0 || block >= a->num_blocks) return -1;
    return a->ref[(size_t)block];
}

int pa_alloc_num_free(const pa_allocator* a) { return a ? (int)a->free_q.size() : -1; }

int pa_alloc_num_tokens(const pa_allocator* a, int64_t seq_id)
{
    if (!a) return -1;
    auto it = a->seqs.find(seq_id);
    return it == a->seqs.end() ? -1 : (int)it->second.tokens;
}

pa_status pa_alloc_stats(const pa_allocator* a, pa_alloc_stats_t* out)
{
    if (!a || !out) return PA_ERR_INVALID;
    pa_alloc_stats_t s{};
    s.num_blocks = a->num_blocks;
    s.num_free = (int64_t)a->free_q.size();
    s.num_seqs = (int64_t)a->seqs.size();
    for (int32_t r : a->ref) s.shared_blocks += r > 1 ? 1 : 0;
    s.cow_copies = a->cow_copies;
    for (const auto& kv : a->seqs) {
        s.tokens += kv.second.tokens;
        s.waste_tokens += (int64_t)kv.second.table.size() * a->block_size - kv.second.tokens;
    }
    *out = s;
    return PA_OK;
}

}  // extern "C"
