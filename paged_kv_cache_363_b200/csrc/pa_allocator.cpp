// Host block allocator with reference-counted copy-on-write and a prefix cache.
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
//  shared blocks untouched; "Paper Methods", shared prefix caching in a radix tree.
//
// Where the pages are silent: the free pool is a FIFO queue (initial order given
// by the caller, freed blocks appended in table order); a fork copies the parent's
// table and token count; a copy happens only for a write into a shared, partially
// filled last block (full shared blocks are never written); every failing call
// leaves the state as it was.
//
// Prefix cache (the pages name a radix tree and nothing more).  The tree is kept at
// block granularity: a node is a full physical block, its edge the B token ids it
// holds, its parent the block before it, so a node stands for the whole token
// prefix that ends with it.  A prompt added with its token ids walks the tree and
// reuses the blocks of its longest cached full-block prefix (their counts go up);
// its remaining full blocks are taken fresh and become new nodes; a partial last
// block stays private (it will be written).  A cached block whose count drops to
// zero is kept, unreferenced, for later prompts.  A block is taken from the free
// queue first; when that is empty, the unreferenced cached block released longest
// ago that has no cached children (a leaf) is evicted from the tree and reused.
#include <cstdint>
#include <cstring>
#include <deque>
#include <map>
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
        std::vector<int32_t> table;  // device blocks, or host blocks while swapped out
        int64_t tokens = 0;
        bool on_host = false;
        // scratch of the batch check: tokens and last block as if the batch's earlier
        // appends of this sequence had run (valid while epoch == the allocator's)
        uint64_t epoch = 0;
        int64_t pend_tokens = 0;
        int32_t pend_last = -1;
    };
    int32_t num_blocks = 0;
    int32_t block_size = 0;
    std::deque<int32_t> free_q;
    std::vector<int32_t> ref;
    std::unordered_map<int64_t, Seq> seqs;
    int64_t cow_copies = 0;

    // prefix tree: key = (parent block or -1, the block's B token ids) -> block, hashed
    // with 64-bit FNV-1a (Fowler, Noll and Vo) over the key's words
    struct KeyHash {
        size_t operator()(const std::vector<int32_t>& k) const noexcept
        {
            uint64_t h = 14695981039346656037ull;
            for (int32_t x : k) {
                h ^= (uint32_t)x;
                h *= 1099511628211ull;
            }
            return (size_t)h;
        }
    };
    std::unordered_map<std::vector<int32_t>, int32_t, KeyHash> tree;
    std::vector<std::vector<int32_t>> node_key;  // per block: its key (empty = not in the tree)
    std::vector<int32_t> nchild;                 // per block: cached children
    std::map<uint64_t, int32_t> lru;             // unreferenced cached blocks by release stamp
    std::map<uint64_t, int32_t> leaves;          // those of them with no cached child (the evictable ones)
    std::vector<uint64_t> stamp;                 // per block: its key in lru (and leaves)
    uint64_t clock = 0;

    // host tier for swapped-out sequences (0 blocks until pa_alloc_add_host_pool)
    int32_t num_host_blocks = 0;
    std::deque<int32_t> host_free;

    // scratch of the batch check, reused across calls (a handle serves one thread at a
    // time): per block, the batch that last changed its count and the change within it;
    // per batch entry, its sequence
    uint64_t epoch = 0;
    std::vector<uint64_t> blk_epoch;
    std::vector<int32_t> blk_dref;
    std::vector<Seq*> batch_seq;
    std::vector<int32_t> touched;          // beam step: blocks whose count it changes
    std::vector<const Seq*> beam_par;      // beam step: each new beam's parent

    // the sequence, if it exists and is resident on the device
    Seq* resident(int64_t seq_id)
    {
        auto it = seqs.find(seq_id);
        return it == seqs.end() || it->second.on_host ? nullptr : &it->second;
    }

    bool cached(int32_t b) const { return !node_key[(size_t)b].empty(); }
    int64_t available() const { return (int64_t)free_q.size() + (int64_t)lru.size(); }

    int64_t slot_of(const Seq& q, int64_t i) const
    {
        return (int64_t)q.table[(size_t)(i / block_size)] * block_size + i % block_size;
    }

    // Removes an unreferenced cached leaf from the tree.  Its parent may become a leaf;
    // an unreferenced one then joins the evictable set under its own release stamp.  (A
    // child is only ever hung under a referenced block, so an unreferenced block's child
    // count can only fall.)
    void evict(int32_t b)
    {
        const std::vector<int32_t>& k = node_key[(size_t)b];
        const int32_t p = k[0];
        tree.erase(k);
        node_key[(size_t)b].clear();
        lru.erase(stamp[(size_t)b]);
        leaves.erase(stamp[(size_t)b]);
        if (p >= 0 && --nchild[(size_t)p] == 0 && ref[(size_t)p] == 0) leaves.emplace(stamp[(size_t)p], p);
    }

    // A block with count 1: the free queue's head, else the oldest unreferenced cached
    // leaf.  Callers check available() first, so there always is one.
    int32_t take()
    {
        int32_t b;
        if (!free_q.empty()) {
            b = free_q.front();
            free_q.pop_front();
        } else {
            b = leaves.begin()->second;  // the earliest released unreferenced leaf
            evict(b);
        }
        ref[(size_t)b] = 1;
        return b;
    }

    void add_ref(int32_t b)
    {
        if (ref[(size_t)b]++ == 0) {
            lru.erase(stamp[(size_t)b]);
            leaves.erase(stamp[(size_t)b]);
        }
    }

    void drop_ref(int32_t b)
    {
        if (--ref[(size_t)b] > 0) return;
        if (cached(b)) {
            stamp[(size_t)b] = clock++;
            lru.emplace(stamp[(size_t)b], b);
            if (nchild[(size_t)b] == 0) leaves.emplace(stamp[(size_t)b], b);
        } else {
            free_q.push_back(b);
        }
    }

    // Blocks that appends of seq_ids[0..n) in order would take (fresh or copy-on-write),
    // without changing the allocation; -1 if a sequence is unknown or swapped out.  The
    // batch's sequences are left in batch_seq[0..n) for the appends that follow.  No
    // container is allocated per call: per-sequence and per-block scratch is tagged with
    // the call's epoch, and anything older counts as untouched.
    int64_t blocks_for_appends(const int64_t* seq_ids, int n)
    {
        ++epoch;
        batch_seq.resize((size_t)n);
        int64_t need = 0;
        for (int k = 0; k < n; ++k) {
            auto it = seqs.find(seq_ids[k]);
            if (it == seqs.end() || it->second.on_host) return -1;
            Seq& q = it->second;
            batch_seq[(size_t)k] = &q;
            if (q.epoch != epoch) {
                q.epoch = epoch;
                q.pend_tokens = q.tokens;
                q.pend_last = q.table.empty() ? -1 : q.table.back();
            }
            if (q.pend_tokens % block_size == 0) {
                need += 1;
                q.pend_last = -1;  // a private fresh block
            } else if (q.pend_last >= 0) {
                const size_t b = (size_t)q.pend_last;
                const int32_t d = blk_epoch[b] == epoch ? blk_dref[b] : 0;
                if (ref[b] + d > 1) {
                    need += 1;
                    blk_epoch[b] = epoch;
                    blk_dref[b] = d - 1;
                    q.pend_last = -1;  // a private copy
                }
            }
            q.pend_tokens += 1;
        }
        return need;
    }

    // One append; the caller has checked that the blocks it may take are available.
    int64_t append(int64_t seq_id, int32_t* src, int32_t* dst) { return append(seqs.find(seq_id)->second, src, dst); }

    int64_t append(Seq& q, int32_t* src, int32_t* dst)
    {
        const int64_t i = q.tokens;
        *src = -1;
        *dst = -1;
        if (i % block_size == 0) {
            q.table.push_back(take());
        } else {
            const int32_t last = q.table.back();
            if (ref[(size_t)last] > 1) {
                const int32_t d = take();
                drop_ref(last);
                q.table.back() = d;
                *src = last;
                *dst = d;
                cow_copies += 1;
            }
        }
        q.tokens = i + 1;
        return slot_of(q, i);
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
    a->node_key.assign((size_t)num_blocks, std::vector<int32_t>());
    a->nchild.assign((size_t)num_blocks, 0);
    a->stamp.assign((size_t)num_blocks, 0);
    a->blk_epoch.assign((size_t)num_blocks, 0);
    a->blk_dref.assign((size_t)num_blocks, 0);
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
    if (need > a->available()) {
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
    if (it == a->seqs.end() || it->second.on_host || a->seqs.count(child_id)) {
        pa::set_error("pa_alloc_fork: unknown or swapped-out parent, or existing child");
        return PA_ERR_INVALID;
    }
    pa_allocator::Seq child = it->second;
    for (int32_t b : child.table) a->add_ref(b);
    a->seqs.emplace(child_id, std::move(child));
    return PA_OK;
}

pa_status pa_alloc_add_seq_cached(pa_allocator* a, int64_t seq_id, const int32_t* token_ids, int num_tokens,
                                  int64_t* slots_out, int* num_cached_out)
{
    if (!a || num_tokens < 0 || (num_tokens > 0 && !token_ids) || !num_cached_out) {
        pa::set_error("pa_alloc_add_seq_cached: bad argument");
        return PA_ERR_INVALID;
    }
    if (a->seqs.count(seq_id)) {
        pa::set_error("pa_alloc_add_seq_cached: sequence " + std::to_string(seq_id) + " exists");
        return PA_ERR_INVALID;
    }
    const int B = a->block_size;
    const int nfull = num_tokens / B;
    // longest cached prefix of full blocks
    std::vector<int32_t> key((size_t)B + 1);
    std::vector<int32_t> hits;
    int32_t parent = -1;
    int64_t hits_unreferenced = 0;
    for (int j = 0; j < nfull; ++j) {
        key[0] = parent;
        std::memcpy(key.data() + 1, token_ids + (size_t)j * B, (size_t)B * sizeof(int32_t));
        auto it = a->tree.find(key);
        if (it == a->tree.end()) break;
        hits.push_back(it->second);
        hits_unreferenced += a->ref[(size_t)it->second] == 0 ? 1 : 0;
        parent = it->second;
    }
    const int64_t need = (int64_t)(nfull - (int)hits.size()) + (num_tokens % B ? 1 : 0);
    if (need > a->available() - hits_unreferenced) {
        pa::set_error("pa_alloc_add_seq_cached: out of blocks");
        return PA_ERR_OOM;
    }
    pa_allocator::Seq q;
    q.table.reserve((size_t)(hits.size() + need));
    for (int32_t b : hits) {
        a->add_ref(b);
        q.table.push_back(b);
    }
    for (int j = (int)hits.size(); j < nfull; ++j) {
        const int32_t b = a->take();
        key[0] = parent;
        std::memcpy(key.data() + 1, token_ids + (size_t)j * B, (size_t)B * sizeof(int32_t));
        a->tree.emplace(key, b);
        a->node_key[(size_t)b] = key;
        if (parent >= 0) a->nchild[(size_t)parent] += 1;
        q.table.push_back(b);
        parent = b;
    }
    if (num_tokens % B) q.table.push_back(a->take());
    q.tokens = num_tokens;
    if (slots_out)
        for (int64_t i = 0; i < num_tokens; ++i) slots_out[i] = a->slot_of(q, i);
    *num_cached_out = (int)hits.size() * B;
    a->seqs.emplace(seq_id, std::move(q));
    return PA_OK;
}

pa_status pa_alloc_append_slot(pa_allocator* a, int64_t seq_id, int64_t* slot_out, int32_t* cow_src_out,
                               int32_t* cow_dst_out)
{
    if (!a || !slot_out) {
        pa::set_error("pa_alloc_append_slot: bad argument");
        return PA_ERR_INVALID;
    }
    const int64_t need = a->blocks_for_appends(&seq_id, 1);
    if (need < 0) {
        pa::set_error("pa_alloc_append_slot: unknown or swapped-out sequence " + std::to_string(seq_id));
        return PA_ERR_INVALID;
    }
    if (need > a->available()) {
        pa::set_error("pa_alloc_append_slot: out of blocks");
        return PA_ERR_OOM;
    }
    int32_t src, dst;
    *slot_out = a->append(*a->batch_seq[0], &src, &dst);
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
    // all or nothing: count the blocks the whole batch takes before changing anything
    const int64_t need = a->blocks_for_appends(seq_ids, n);
    if (need < 0) {
        for (int k = 0; k < n; ++k)
            if (!a->resident(seq_ids[k])) {
                pa::set_error("pa_alloc_append_slots: unknown or swapped-out sequence " + std::to_string(seq_ids[k]));
                break;
            }
        return PA_ERR_INVALID;
    }
    if (need > a->available()) {
        pa::set_error("pa_alloc_append_slots: out of blocks");
        return PA_ERR_OOM;
    }
    int ncow = 0;
    for (int k = 0; k < n; ++k) {
        int32_t src, dst;
        slots_out[k] = a->append(*a->batch_seq[(size_t)k], &src, &dst);
        if (src >= 0) {
            cow_pairs_out[2 * ncow] = src;
            cow_pairs_out[2 * ncow + 1] = dst;
            ++ncow;
        }
    }
    *num_cow_out = ncow;
    return PA_OK;
}

pa_status pa_alloc_beam_step(pa_allocator* a, const int64_t* beam_ids, int num_beams, const int32_t* parents,
                             const int64_t* new_ids, int num_new, int64_t* slots_out, int64_t* cow_pairs_out,
                             int* num_cow_out)
{
    if (!a || num_beams < 0 || num_new < 0 || (num_beams > 0 && !beam_ids) ||
        (num_new > 0 && (!parents || !new_ids || !slots_out || !cow_pairs_out)) || !num_cow_out) {
        pa::set_error("pa_alloc_beam_step: bad argument");
        return PA_ERR_INVALID;
    }
    std::unordered_map<int64_t, int> old_index;
    for (int i = 0; i < num_beams; ++i) {
        if (!a->resident(beam_ids[i]) || !old_index.emplace(beam_ids[i], i).second) {
            pa::set_error("pa_alloc_beam_step: beam " + std::to_string(beam_ids[i]) +
                          " unknown, swapped out or listed twice");
            return PA_ERR_INVALID;
        }
    }
    std::unordered_map<int64_t, int> new_index;
    for (int j = 0; j < num_new; ++j) {
        if (parents[j] < 0 || parents[j] >= num_beams) {
            pa::set_error("pa_alloc_beam_step: parent index out of range");
            return PA_ERR_INVALID;
        }
        if (!new_index.emplace(new_ids[j], j).second || (a->seqs.count(new_ids[j]) && !old_index.count(new_ids[j]))) {
            pa::set_error("pa_alloc_beam_step: new beam id " + std::to_string(new_ids[j]) +
                          " repeated or held by a sequence outside the old beams");
            return PA_ERR_INVALID;
        }
    }
    // Count the blocks the appends take, on the reference counts the forks and frees leave.
    // The count changes live in the per-block scratch tagged with this call's epoch; the
    // blocks touched are listed once each.
    const uint64_t ep = ++a->epoch;
    std::vector<int32_t>& touched = a->touched;
    touched.clear();
    auto delta = [&](int32_t b) -> int32_t& {
        if (a->blk_epoch[(size_t)b] != ep) {
            a->blk_epoch[(size_t)b] = ep;
            a->blk_dref[(size_t)b] = 0;
            touched.push_back(b);
        }
        return a->blk_dref[(size_t)b];
    };
    std::vector<const pa_allocator::Seq*>& par = a->beam_par;
    par.resize((size_t)num_new);
    for (int j = 0; j < num_new; ++j) {
        par[(size_t)j] = &a->seqs.find(beam_ids[parents[j]])->second;
        for (int32_t b : par[(size_t)j]->table) delta(b) += 1;
    }
    for (int i = 0; i < num_beams; ++i)
        for (int32_t b : a->seqs.find(beam_ids[i])->second.table) delta(b) -= 1;
    int64_t released = 0;
    for (int32_t b : touched)
        if (a->ref[(size_t)b] > 0 && a->ref[(size_t)b] + a->blk_dref[(size_t)b] == 0) released += 1;
    int64_t need = 0;
    for (int j = 0; j < num_new; ++j) {
        const pa_allocator::Seq& p = *par[(size_t)j];
        if (p.tokens % a->block_size == 0) {
            need += 1;
        } else {
            const int32_t last = p.table.back();
            if (a->ref[(size_t)last] + delta(last) > 1) {
                need += 1;
                delta(last) -= 1;
            }
        }
    }
    if (need > a->available() + released) {
        pa::set_error("pa_alloc_beam_step: out of blocks");
        return PA_ERR_OOM;
    }
    // fork the chosen parents, free the old beams, install the new ones, append one slot each
    std::vector<pa_allocator::Seq> fresh((size_t)num_new);
    for (int j = 0; j < num_new; ++j) {
        fresh[(size_t)j] = *par[(size_t)j];
        for (int32_t b : fresh[(size_t)j].table) a->add_ref(b);
    }
    for (int i = 0; i < num_beams; ++i) {
        auto it = a->seqs.find(beam_ids[i]);
        for (int32_t b : it->second.table) a->drop_ref(b);
        a->seqs.erase(it);
    }
    for (int j = 0; j < num_new; ++j) a->seqs.emplace(new_ids[j], std::move(fresh[(size_t)j]));
    int ncow = 0;
    for (int j = 0; j < num_new; ++j) {
        int32_t src, dst;
        slots_out[j] = a->append(new_ids[j], &src, &dst);
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
    if (it->second.on_host) {
        for (int32_t h : it->second.table) a->host_free.push_back(h);
    } else {
        for (int32_t b : it->second.table) a->drop_ref(b);
    }
    a->seqs.erase(it);
    return PA_OK;
}

pa_status pa_alloc_add_host_pool(pa_allocator* a, int num_host_blocks)
{
    if (!a || num_host_blocks <= 0 || a->num_host_blocks > 0) {
        pa::set_error("pa_alloc_add_host_pool: bad argument or a host pool exists");
        return PA_ERR_INVALID;
    }
    a->num_host_blocks = num_host_blocks;
    for (int i = 0; i < num_host_blocks; ++i) a->host_free.push_back(i);
    return PA_OK;
}

pa_status pa_alloc_swap_out(pa_allocator* a, int64_t seq_id, int64_t* pairs_out, int* num_pairs_out)
{
    if (!a || !num_pairs_out) {
        pa::set_error("pa_alloc_swap_out: bad argument");
        return PA_ERR_INVALID;
    }
    pa_allocator::Seq* q = a->resident(seq_id);
    if (!q) {
        pa::set_error("pa_alloc_swap_out: unknown or swapped-out sequence " + std::to_string(seq_id));
        return PA_ERR_INVALID;
    }
    if (!q->table.empty() && !pairs_out) {
        pa::set_error("pa_alloc_swap_out: pairs_out is null");
        return PA_ERR_INVALID;
    }
    if (q->table.size() > a->host_free.size()) {
        pa::set_error("pa_alloc_swap_out: out of host blocks");
        return PA_ERR_OOM;
    }
    for (size_t i = 0; i < q->table.size(); ++i) {
        const int32_t h = a->host_free.front();
        a->host_free.pop_front();
        pairs_out[2 * i] = q->table[i];
        pairs_out[2 * i + 1] = h;
        a->drop_ref(q->table[i]);
        q->table[i] = h;
    }
    q->on_host = true;
    *num_pairs_out = (int)q->table.size();
    return PA_OK;
}

pa_status pa_alloc_swap_in(pa_allocator* a, int64_t seq_id, int64_t* pairs_out, int* num_pairs_out)
{
    if (!a || !num_pairs_out) {
        pa::set_error("pa_alloc_swap_in: bad argument");
        return PA_ERR_INVALID;
    }
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end() || !it->second.on_host) {
        pa::set_error("pa_alloc_swap_in: sequence " + std::to_string(seq_id) + " is not swapped out");
        return PA_ERR_INVALID;
    }
    pa_allocator::Seq& q = it->second;
    if (!q.table.empty() && !pairs_out) {
        pa::set_error("pa_alloc_swap_in: pairs_out is null");
        return PA_ERR_INVALID;
    }
    if ((int64_t)q.table.size() > a->available()) {
        pa::set_error("pa_alloc_swap_in: out of blocks");
        return PA_ERR_OOM;
    }
    for (size_t i = 0; i < q.table.size(); ++i) {
        const int32_t b = a->take();
        pairs_out[2 * i] = q.table[i];
        pairs_out[2 * i + 1] = b;
        a->host_free.push_back(q.table[i]);
        q.table[i] = b;
    }
    q.on_host = false;
    *num_pairs_out = (int)q.table.size();
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
        if (it == a->seqs.end() || it->second.on_host) {
            pa::set_error("pa_alloc_block_tables: unknown or swapped-out sequence " + std::to_string(seq_ids[k]));
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

int pa_alloc_num_cached_free(const pa_allocator* a) { return a ? (int)a->lru.size() : -1; }

int pa_alloc_num_host_free(const pa_allocator* a) { return a ? (int)a->host_free.size() : -1; }

int pa_alloc_is_swapped(const pa_allocator* a, int64_t seq_id)
{
    if (!a) return -1;
    auto it = a->seqs.find(seq_id);
    return it == a->seqs.end() ? -1 : (it->second.on_host ? 1 : 0);
}

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
    s.cached_blocks = (int64_t)a->tree.size();
    s.cached_free = (int64_t)a->lru.size();
    s.host_blocks = a->num_host_blocks;
    s.host_free = (int64_t)a->host_free.size();
    for (const auto& kv : a->seqs) s.swapped_seqs += kv.second.on_host ? 1 : 0;
    for (const auto& kv : a->seqs) {
        s.tokens += kv.second.tokens;
        s.waste_tokens += (int64_t)kv.second.table.size() * a->block_size - kv.second.tokens;
    }
    *out = s;
    return PA_OK;
}

}  // extern "C"
