// Host-side refcounted physical block pool and per-sequence block tables.
//
// "PagedAttention 机制" §5.3.4 (BlockAllocator: free list, reference counts,
// allocate / free / incr_ref, out-of-memory error when the list is empty);
// "01. PagedAttention 详解" self-check 3 (the free list is a FIFO queue:
// allocation takes the head, a block whose count reaches 0 goes to the tail);
// "PagedAttention 机制" §5.3.2 (a sequence of n tokens holds ceil(n / bs)
// blocks, mapped logical -> physical by its table); "01. PagedAttention 详解"
// §6 and summary (sharing by reference counts: common prefixes, beam search,
// parallel sampling); intelliparadigm PagedAttention article §3.3 (writing
// into a block with count > 1 first copies it: maybe_copy_block).
#include <cstdint>
#include <new>
#include <unordered_map>
#include <vector>

#include "pa_internal.h"

// FIFO of free blocks as an intrusive doubly linked list, so a cached block
// can leave the middle of the queue when a prefix-cache hit revives it.
struct FreeQueue {
    std::vector<int32_t> prev, next;
    std::vector<uint8_t> in;
    int32_t head = -1, tail = -1;
    int64_t count = 0;

    void init(int64_t nb) {
        prev.assign((size_t)nb, -1);
        next.assign((size_t)nb, -1);
        in.assign((size_t)nb, 0);
        head = tail = -1;
        count = 0;
        for (int64_t b = 0; b < nb; ++b) push_back((int32_t)b);
    }
    bool empty() const { return count == 0; }
    size_t size() const { return (size_t)count; }
    int32_t front() const { return head; }
    void push_back(int32_t b) {
        prev[b] = tail;
        next[b] = -1;
        if (tail >= 0) next[tail] = b; else head = b;
        tail = b;
        in[b] = 1;
        ++count;
    }
    void remove(int32_t b) {
        if (prev[b] >= 0) next[prev[b]] = next[b]; else head = next[b];
        if (next[b] >= 0) prev[next[b]] = prev[b]; else tail = prev[b];
        prev[b] = next[b] = -1;
        in[b] = 0;
        --count;
    }
    void pop_front() { remove(head); }
};

struct pa_pool {
    int64_t nb = 0;
    int bs = 0;
    FreeQueue free_q;
    std::vector<int32_t> ref;
    struct Seq {
        std::vector<int32_t> blocks;
        int64_t n = 0;
    };
    std::unordered_map<int64_t, Seq> seqs;
    int64_t next_seq = 0;
    int64_t cow = 0;
    // prefix cache: content hash of a full block -> the block holding it
    std::unordered_map<uint64_t, int32_t> by_hash;
    std::vector<uint64_t> hash_of;
    std::vector<uint8_t> hashed;
    int64_t hits = 0;

    bool in_range(int64_t b) const { return b >= 0 && b < nb; }
    Seq* find(int64_t s) {
        auto it = seqs.find(s);
        return it == seqs.end() ? nullptr : &it->second;
    }
    const Seq* find(int64_t s) const {
        auto it = seqs.find(s);
        return it == seqs.end() ? nullptr : &it->second;
    }
    void forget_hash(int32_t b) {
        if (!hashed[b]) return;
        auto it = by_hash.find(hash_of[b]);
        if (it != by_hash.end() && it->second == b) by_hash.erase(it);
        hashed[b] = 0;
    }
    int32_t take() {             // caller checked that the queue is not empty
        const int32_t b = free_q.front();
        free_q.pop_front();
        forget_hash(b);          // reusing the block evicts its cached content
        ref[b] = 1;
        return b;
    }
    void drop(int32_t b) {       // caller checked ref[b] > 0
        if (--ref[b] == 0) free_q.push_back(b);
    }
};

using pa::fail;

extern "C" pa_status pa_pool_create(int64_t NB, int bs, pa_pool** out) {
    pa::clear_error();
    if (!out) return fail(PA_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    if (NB <= 0 || NB > 0x7fffffffLL || bs <= 0)
        return fail(PA_ERR_INVALID_ARG, "NB must be in [1, 2^31), bs > 0");
    pa_pool* p = new (std::nothrow) pa_pool();
    if (!p) return fail(PA_ERR_INVALID_ARG, "out of host memory");
    p->nb = NB;
    p->bs = bs;
    p->ref.assign((size_t)NB, 0);
    p->hash_of.assign((size_t)NB, 0);
    p->hashed.assign((size_t)NB, 0);
    p->free_q.init(NB);
    *out = p;
    return PA_OK;
}

extern "C" void pa_pool_destroy(pa_pool* pool) { delete pool; }

extern "C" pa_status pa_pool_alloc(pa_pool* pool, int32_t* block) {
    pa::clear_error();
    if (!pool || !block) return fail(PA_ERR_INVALID_ARG, "NULL argument");
    if (pool->free_q.empty()) return fail(PA_ERR_OUT_OF_BLOCKS, "no free blocks");
    *block = pool->take();
    return PA_OK;
}

extern "C" pa_status pa_pool_free(pa_pool* pool, int32_t block) {
    pa::clear_error();
    if (!pool) return fail(PA_ERR_INVALID_ARG, "pool is NULL");
    if (!pool->in_range(block)) return fail(PA_ERR_BAD_INDEX, "block %d out of range", block);
    if (pool->ref[block] <= 0) return fail(PA_ERR_REFCOUNT, "block %d is already free", block);
    pool->drop(block);
    return PA_OK;
}

extern "C" pa_status pa_pool_incr_ref(pa_pool* pool, int32_t block) {
    pa::clear_error();
    if (!pool) return fail(PA_ERR_INVALID_ARG, "pool is NULL");
    if (!pool->in_range(block)) return fail(PA_ERR_BAD_INDEX, "block %d out of range", block);
    if (pool->ref[block] <= 0) return fail(PA_ERR_REFCOUNT, "block %d is free", block);
    ++pool->ref[block];
    return PA_OK;
}

extern "C" int pa_pool_ref(const pa_pool* pool, int32_t block) {
    if (!pool || !pool->in_range(block)) return -1;
    return pool->ref[block];
}

extern "C" pa_status pa_pool_seq_new(pa_pool* pool, int64_t* seq) {
    pa::clear_error();
    if (!pool || !seq) return fail(PA_ERR_INVALID_ARG, "NULL argument");
    const int64_t id = pool->next_seq++;
    pool->seqs.emplace(id, pa_pool::Seq{});
    *seq = id;
    return PA_OK;
}

extern "C" pa_status pa_pool_seq_fork(pa_pool* pool, int64_t parent, int64_t* child) {
    pa::clear_error();
    if (!pool || !child) return fail(PA_ERR_INVALID_ARG, "NULL argument");
    const pa_pool::Seq* par = pool->find(parent);
    if (!par) return fail(PA_ERR_BAD_INDEX, "unknown sequence %lld", (long long)parent);
    for (int32_t b : par->blocks)            // all or nothing
        if (pool->ref[b] <= 0) return fail(PA_ERR_REFCOUNT, "block %d is free", b);
    pa_pool::Seq copy = *par;
    for (int32_t b : copy.blocks) ++pool->ref[b];
    const int64_t id = pool->next_seq++;
    pool->seqs.emplace(id, std::move(copy));
    *child = id;
    return PA_OK;
}

extern "C" pa_status pa_pool_seq_share_prefix(pa_pool* pool, int64_t seq, const int32_t* blocks,
                                              int n, int64_t num_tokens) {
    pa::clear_error();
    if (!pool || (n > 0 && !blocks) || n < 0 || num_tokens < 0)
        return fail(PA_ERR_INVALID_ARG, "bad arguments");
    pa_pool::Seq* s = pool->find(seq);
    if (!s) return fail(PA_ERR_BAD_INDEX, "unknown sequence %lld", (long long)seq);
    if (s->n != 0 || !s->blocks.empty())
        return fail(PA_ERR_INVALID_ARG, "a prefix can only be shared into an empty sequence");
    if ((int64_t)n != (num_tokens + pool->bs - 1) / pool->bs)
        return fail(PA_ERR_INVALID_ARG, "%d blocks cannot hold exactly %lld tokens", n,
                    (long long)num_tokens);
    for (int i = 0; i < n; ++i) {
        if (!pool->in_range(blocks[i])) return fail(PA_ERR_BAD_INDEX, "block %d out of range", blocks[i]);
        if (pool->ref[blocks[i]] <= 0) return fail(PA_ERR_REFCOUNT, "block %d is free", blocks[i]);
    }
    for (int i = 0; i < n; ++i) ++pool->ref[blocks[i]];
    s->blocks.assign(blocks, blocks + n);
    s->n = num_tokens;
    return PA_OK;
}

extern "C" pa_status pa_pool_seq_append(pa_pool* pool, int64_t seq, int64_t* slot,
                                        int32_t* cow_src, int32_t* cow_dst) {
    pa::clear_error();
    if (!pool || !slot || !cow_src || !cow_dst) return fail(PA_ERR_INVALID_ARG, "NULL argument");
    pa_pool::Seq* s = pool->find(seq);
    if (!s) return fail(PA_ERR_BAD_INDEX, "unknown sequence %lld", (long long)seq);
    int32_t src = -1, dst = -1;
    const int64_t off = s->n % pool->bs;
    if (off == 0) {
        if (pool->free_q.empty()) return fail(PA_ERR_OUT_OF_BLOCKS, "no free blocks");
        s->blocks.push_back(pool->take());
    } else {
        const int32_t last = s->blocks.back();
        if (pool->ref[last] <= 1) pool->forget_hash(last);   // its content is about to change
        if (pool->ref[last] > 1) {
            if (pool->free_q.empty()) return fail(PA_ERR_OUT_OF_BLOCKS, "no free blocks");
            const int32_t fresh = pool->take();
            --pool->ref[last];               // other holders keep it (count stays >= 1)
            s->blocks.back() = fresh;
            src = last;
            dst = fresh;
            ++pool->cow;
        }
    }
    *slot = (int64_t)s->blocks.back() * pool->bs + off;
    *cow_src = src;
    *cow_dst = dst;
    ++s->n;
    return PA_OK;
}

extern "C" pa_status pa_pool_seq_append_batch(pa_pool* pool, const int64_t* seqs, int n,
                                              int64_t* slots, int32_t* cow_pairs, int* n_cow) {
    pa::clear_error();
    if (!pool || n < 0 || (n > 0 && (!seqs || !slots || !cow_pairs)) || !n_cow)
        return fail(PA_ERR_INVALID_ARG, "bad arguments");
    *n_cow = 0;
    // all or nothing: validate every sequence and count the blocks needed first
    std::unordered_map<int64_t, int> seen;
    seen.reserve(2 * (size_t)n);
    int64_t need = 0;
    for (int i = 0; i < n; ++i) {
        const pa_pool::Seq* s = pool->find(seqs[i]);
        if (!s) return fail(PA_ERR_BAD_INDEX, "unknown sequence %lld", (long long)seqs[i]);
        if (!seen.emplace(seqs[i], i).second)
            return fail(PA_ERR_INVALID_ARG, "sequence %lld appears twice", (long long)seqs[i]);
        if (s->n % pool->bs == 0 || pool->ref[s->blocks.back()] > 1) ++need;
    }
    if (need > (int64_t)pool->free_q.size())
        return fail(PA_ERR_OUT_OF_BLOCKS, "%lld blocks needed, %zu free", (long long)need,
                    pool->free_q.size());
    int nc = 0;
    for (int i = 0; i < n; ++i) {
        int32_t src = -1, dst = -1;
        pa_pool_seq_append(pool, seqs[i], &slots[i], &src, &dst);   // cannot fail now
        if (src >= 0) {
            cow_pairs[2 * nc] = src;
            cow_pairs[2 * nc + 1] = dst;
            ++nc;
        }
    }
    *n_cow = nc;
    return PA_OK;
}

extern "C" pa_status pa_pool_seq_free(pa_pool* pool, int64_t seq) {
    pa::clear_error();
    if (!pool) return fail(PA_ERR_INVALID_ARG, "pool is NULL");
    auto it = pool->seqs.find(seq);
    if (it == pool->seqs.end()) return fail(PA_ERR_BAD_INDEX, "unknown sequence %lld", (long long)seq);
    std::unordered_map<int32_t, int> held;   // all or nothing: check every reference first
    for (int32_t b : it->second.blocks) ++held[b];
    for (const auto& kv : held)
        if (pool->ref[kv.first] < kv.second)
            return fail(PA_ERR_REFCOUNT, "block %d has fewer references than the sequence holds",
                        kv.first);
    for (int32_t b : it->second.blocks) pool->drop(b);
    pool->seqs.erase(it);
    return PA_OK;
}

extern "C" int64_t pa_pool_seq_len(const pa_pool* pool, int64_t seq) {
    if (!pool) return -1;
    const pa_pool::Seq* s = pool->find(seq);
    return s ? s->n : -1;
}

extern "C" pa_status pa_pool_build_block_tables(const pa_pool* pool, const int64_t* seqs, int S,
                                                int MB, int32_t* tables_host,
                                                int32_t* ctx_lens_host) {
    pa::clear_error();
    if (!pool || S < 0 || MB < 0 || (S > 0 && (!seqs || !ctx_lens_host || (MB > 0 && !tables_host))))
        return fail(PA_ERR_INVALID_ARG, "bad arguments");
    for (int i = 0; i < S; ++i) {
        const pa_pool::Seq* s = pool->find(seqs[i]);
        if (!s) return fail(PA_ERR_BAD_INDEX, "unknown sequence %lld", (long long)seqs[i]);
        if ((int64_t)s->blocks.size() > MB)
            return fail(PA_ERR_INVALID_ARG, "sequence %lld holds %zu blocks > MB %d",
                        (long long)seqs[i], s->blocks.size(), MB);
        if (s->n > 0x7fffffffLL) return fail(PA_ERR_INVALID_ARG, "context length overflows int32");
    }
    for (int i = 0; i < S; ++i) {
        const pa_pool::Seq* s = pool->find(seqs[i]);
        int32_t* row = tables_host + (size_t)i * MB;
        const size_t nb = s->blocks.size();
        for (size_t j = 0; j < nb; ++j) row[j] = s->blocks[j];
        for (size_t j = nb; j < (size_t)MB; ++j) row[j] = -1;
        ctx_lens_host[i] = (int32_t)s->n;
    }
    return PA_OK;
}

extern "C" pa_status pa_pool_stats(const pa_pool* pool, pa_pool_stats_t* st) {
    pa::clear_error();
    if (!pool || !st) return fail(PA_ERR_INVALID_ARG, "NULL argument");
    st->num_blocks = pool->nb;
    st->free_blocks = (int64_t)pool->free_q.size();
    int64_t used = 0, shared = 0;
    for (int32_t r : pool->ref) {
        used += r > 0;
        shared += r > 1;
    }
    st->used_blocks = used;
    st->shared_blocks = shared;
    st->cow_copies = pool->cow;
    st->num_seqs = (int64_t)pool->seqs.size();
    st->cached_blocks = (int64_t)pool->by_hash.size();
    st->cache_hits = pool->hits;
    return PA_OK;
}

extern "C" pa_status pa_pool_seq_blocks(const pa_pool* pool, int64_t seq, int32_t* blocks, int cap,
                                        int* n) {
    pa::clear_error();
    if (!pool || !n || cap < 0 || (cap > 0 && !blocks)) return fail(PA_ERR_INVALID_ARG, "bad arguments");
    const pa_pool::Seq* s = pool->find(seq);
    if (!s) return fail(PA_ERR_BAD_INDEX, "unknown sequence %lld", (long long)seq);
    *n = (int)s->blocks.size();
    if ((int64_t)s->blocks.size() > cap) return fail(PA_ERR_INVALID_ARG, "cap %d < %zu blocks", cap,
                                                      s->blocks.size());
    for (size_t i = 0; i < s->blocks.size(); ++i) blocks[i] = s->blocks[i];
    return PA_OK;
}

extern "C" pa_status pa_pool_cache_block(pa_pool* pool, int32_t block, uint64_t hash, int* cached) {
    pa::clear_error();
    if (!pool || !cached) return fail(PA_ERR_INVALID_ARG, "NULL argument");
    if (!pool->in_range(block)) return fail(PA_ERR_BAD_INDEX, "block %d out of range", block);
    if (pool->ref[block] <= 0) return fail(PA_ERR_REFCOUNT, "block %d is free", block);
    *cached = 0;
    if (pool->hashed[block]) {
        if (pool->hash_of[block] != hash)
            return fail(PA_ERR_INVALID_ARG, "block %d already holds another hash", block);
        *cached = 1;
        return PA_OK;
    }
    auto it = pool->by_hash.find(hash);
    if (it != pool->by_hash.end()) return PA_OK;    // the content is cached in another block
    pool->by_hash.emplace(hash, block);
    pool->hash_of[block] = hash;
    pool->hashed[block] = 1;
    *cached = 1;
    return PA_OK;
}

// A hit takes a reference: a block still in use gains one more holder; a
// freed block that still holds the content leaves the free queue with
// count 1.
static int32_t cache_take(pa_pool* pool, uint64_t hash) {
    auto it = pool->by_hash.find(hash);
    if (it == pool->by_hash.end()) return -1;
    const int32_t b = it->second;
    if (pool->ref[b] == 0) {
        pool->free_q.remove(b);
        pool->ref[b] = 1;
    } else {
        ++pool->ref[b];
    }
    ++pool->hits;
    return b;
}

extern "C" pa_status pa_pool_cache_lookup(pa_pool* pool, uint64_t hash, int32_t* block) {
    pa::clear_error();
    if (!pool || !block) return fail(PA_ERR_INVALID_ARG, "NULL argument");
    *block = cache_take(pool, hash);
    return PA_OK;
}

extern "C" pa_status pa_pool_seq_match_prefix(pa_pool* pool, int64_t seq, const uint64_t* hashes,
                                              int n, int* matched) {
    pa::clear_error();
    if (!pool || !matched || n < 0 || (n > 0 && !hashes)) return fail(PA_ERR_INVALID_ARG, "bad arguments");
    pa_pool::Seq* s = pool->find(seq);
    if (!s) return fail(PA_ERR_BAD_INDEX, "unknown sequence %lld", (long long)seq);
    if (s->n != 0 || !s->blocks.empty())
        return fail(PA_ERR_INVALID_ARG, "a prefix can only be matched into an empty sequence");
    int m = 0;
    for (; m < n; ++m) {
        const int32_t b = cache_take(pool, hashes[m]);
        if (b < 0) break;
        s->blocks.push_back(b);
    }
    s->n = (int64_t)m * pool->bs;
    *matched = m;
    return PA_OK;
}

extern "C" pa_status pa_pool_step(pa_pool* pool, const int64_t* seqs, int n, int MB, int64_t* slots,
                                  int32_t* cow_pairs, int* n_cow, int32_t* tables_host,
                                  int32_t* ctx_lens_host) {
    PA_NVTX_RANGE("pa_pool_step");
    pa::clear_error();
    if (!pool || n < 0 || MB < 0 || !n_cow ||
        (n > 0 && (!seqs || !slots || !cow_pairs || !ctx_lens_host || (MB > 0 && !tables_host))))
        return fail(PA_ERR_INVALID_ARG, "bad arguments");
    *n_cow = 0;
    // all or nothing: every table must still fit MB entries after the append
    for (int i = 0; i < n; ++i) {
        const pa_pool::Seq* s = pool->find(seqs[i]);
        if (!s) return fail(PA_ERR_BAD_INDEX, "unknown sequence %lld", (long long)seqs[i]);
        const int64_t after = (int64_t)s->blocks.size() + (s->n % pool->bs == 0 ? 1 : 0);
        if (after > MB)
            return fail(PA_ERR_INVALID_ARG, "sequence %lld needs %lld blocks > MB %d",
                        (long long)seqs[i], (long long)after, MB);
        if (s->n + 1 > 0x7fffffffLL) return fail(PA_ERR_INVALID_ARG, "context length overflows int32");
    }
    pa_status st = pa_pool_seq_append_batch(pool, seqs, n, slots, cow_pairs, n_cow);
    if (st) return st;
    return pa_pool_build_block_tables(pool, seqs, n, MB, tables_host, ctx_lens_host);
}
