// block_allocator.cpp -- host-side block manager for the paged KV cache.
//
// "KV Cache Optimization and PagedAttention" (intro) and "PagedAttention:
// Optimizing KV Cache Utilization in Large Language Models" ("The Mechanics of
// PagedAttention"): the cache is split into fixed-size blocks; a request gets
// physical blocks on demand as its tokens arrive, and a per-request block table
// maps its logical blocks to them.  "KV Cache Management" ("The Solution:
// PagedAttention (vLLM)"): a request starts with one block and receives the
// next one when that fills; blocks need not be adjacent.  "The Bonus:
// Zero-Copy Sharing": requests with a common prefix point at the same physical
// blocks; here a block carries a reference count, and a request about to write
// into a shared, partially filled block first takes a private copy
// (copy-on-write) -- the allocator hands back the (src, dst) pair for
// pkv_copy_blocks.
//
// Free blocks are kept on a LIFO stack (the most recently freed block is reused
// first).  All state is host memory; nothing here touches the GPU.
#include <algorithm>
#include <cstdint>
#include <new>
#include <unordered_map>
#include <vector>

#include "pkv.h"

struct pkv_allocator {
    struct Seq {
        std::vector<int32_t> blocks;
        int64_t tokens = 0;
    };
    int32_t num_blocks = 0;
    int32_t block_size = 0;
    std::vector<int32_t> refcount;  // per physical block; 0 = free
    std::vector<int32_t> fill;      // valid slots written in the block
    std::vector<int32_t> free_stack;
    std::unordered_map<int64_t, Seq> seqs;
};

namespace {

bool is_pow2(int32_t x) { return x > 0 && (x & (x - 1)) == 0; }

int32_t pop_free(pkv_allocator* a) {
    const int32_t b = a->free_stack.back();
    a->free_stack.pop_back();
    a->refcount[b] = 1;
    a->fill[b] = 0;
    return b;
}

void release(pkv_allocator* a, int32_t b) {
    if (--a->refcount[b] == 0) {
        a->fill[b] = 0;
        a->free_stack.push_back(b);
    }
}

}  // namespace

extern "C" {

pkv_status pkv_allocator_create(int32_t num_blocks, int32_t block_size, pkv_allocator** out) {
    if (!out || num_blocks <= 0 || !is_pow2(block_size) || block_size > 256)
        return PKV_ERR_INVALID_ARG;
    pkv_allocator* a = new (std::nothrow) pkv_allocator();
    if (!a) return PKV_ERR_INVALID_ARG;
    a->num_blocks = num_blocks;
    a->block_size = block_size;
    a->refcount.assign(num_blocks, 0);
    a->fill.assign(num_blocks, 0);
    a->free_stack.reserve(num_blocks);
    // block 0 on top of the stack first
    for (int32_t b = num_blocks - 1; b >= 0; --b) a->free_stack.push_back(b);
    *out = a;
    return PKV_OK;
}

void pkv_allocator_destroy(pkv_allocator* a) { delete a; }

pkv_status pkv_allocator_add_seq(pkv_allocator* a, int64_t seq_id) {
    if (!a) return PKV_ERR_INVALID_ARG;
    if (a->seqs.count(seq_id)) return PKV_ERR_INVALID_ARG;
    a->seqs.emplace(seq_id, pkv_allocator::Seq{});
    return PKV_OK;
}

pkv_status pkv_allocator_fork(pkv_allocator* a, int64_t parent, int64_t child) {
    if (!a) return PKV_ERR_INVALID_ARG;
    auto it = a->seqs.find(parent);
    if (it == a->seqs.end() || a->seqs.count(child)) return PKV_ERR_INVALID_ARG;
    pkv_allocator::Seq s = it->second;  // copy of the table: the child shares every block
    for (int32_t b : s.blocks) ++a->refcount[b];
    a->seqs.emplace(child, std::move(s));
    return PKV_OK;
}

pkv_status pkv_allocator_append(pkv_allocator* a, int64_t seq_id, int32_t num_tokens,
                                int64_t* slots, int64_t* cow_pair, int32_t* num_cow) {
    if (!a || num_tokens < 0 || (num_tokens > 0 && !slots) || !cow_pair || !num_cow)
        return PKV_ERR_INVALID_ARG;
    *num_cow = 0;
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end()) return PKV_ERR_INVALID_ARG;
    pkv_allocator::Seq& s = it->second;
    if (num_tokens == 0) return PKV_OK;
    const int32_t bs = a->block_size;
    const int32_t in_last = (int32_t)(s.tokens % bs);  // tokens already in a partial last block
    const bool partial = in_last != 0;
    const bool cow = partial && a->refcount[s.blocks.back()] > 1;
    // blocks this append needs, checked before any state changes
    const int64_t room = partial ? bs - in_last : 0;
    const int64_t extra = num_tokens > room ? (num_tokens - room + bs - 1) / bs : 0;
    if ((int64_t)a->free_stack.size() < extra + (cow ? 1 : 0)) return PKV_ERR_OUT_OF_BLOCKS;
    if (cow) {
        const int32_t src = s.blocks.back();
        const int32_t dst = pop_free(a);
        a->fill[dst] = a->fill[src];
        release(a, src);
        s.blocks.back() = dst;
        cow_pair[0] = src;
        cow_pair[1] = dst;
        *num_cow = 1;
    }
    for (int32_t i = 0; i < num_tokens; ++i) {
        const int64_t t = s.tokens + i;
        if (t % bs == 0) s.blocks.push_back(pop_free(a));
        const int32_t b = s.blocks[t / bs];
        slots[i] = (int64_t)b * bs + t % bs;
        a->fill[b] = (int32_t)(t % bs) + 1;
    }
    s.tokens += num_tokens;
    return PKV_OK;
}

pkv_status pkv_allocator_free_seq(pkv_allocator* a, int64_t seq_id) {
    if (!a) return PKV_ERR_INVALID_ARG;
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end()) return PKV_ERR_INVALID_ARG;
    for (int32_t b : it->second.blocks) release(a, b);
    a->seqs.erase(it);
    return PKV_OK;
}

pkv_status pkv_allocator_block_table(const pkv_allocator* a, int64_t seq_id, int32_t* table,
                                     int32_t capacity, int32_t* num_blocks, int64_t* num_tokens) {
    if (!a || !num_blocks || !num_tokens || capacity < 0 || (capacity > 0 && !table))
        return PKV_ERR_INVALID_ARG;
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end()) return PKV_ERR_INVALID_ARG;
    const auto& s = it->second;
    *num_blocks = (int32_t)s.blocks.size();
    *num_tokens = s.tokens;
    if ((int32_t)s.blocks.size() > capacity) return PKV_ERR_INVALID_ARG;
    std::copy(s.blocks.begin(), s.blocks.end(), table);
    return PKV_OK;
}

pkv_status pkv_allocator_get_stats(const pkv_allocator* a, pkv_allocator_stats* out) {
    if (!a || !out) return PKV_ERR_INVALID_ARG;
    pkv_allocator_stats st{};
    st.num_blocks = a->num_blocks;
    st.free_blocks = (int32_t)a->free_stack.size();
    st.num_seqs = (int32_t)a->seqs.size();
    for (int32_t b = 0; b < a->num_blocks; ++b) {
        if (a->refcount[b] == 0) continue;
        st.used_blocks += 1;
        st.stored_tokens += a->fill[b];
        st.unused_slots += a->block_size - a->fill[b];
        if (a->refcount[b] > 1) st.shared_blocks += 1;
    }
    for (const auto& kv : a->seqs) st.logical_tokens += kv.second.tokens;
    *out = st;
    return PKV_OK;
}

int32_t pkv_allocator_refcount(const pkv_allocator* a, int32_t block) {
    if (!a || block < 0 || block >= a->num_blocks) return -1;
    return a->refcount[block];
}

// ---- admission / waste comparison ------------------------------------------------

pkv_status pkv_waste_compare(const int32_t* lengths, int32_t n, int32_t reserve_len,
                             int32_t block_size, int64_t pool_slots, pkv_waste_report* out) {
    if (!out || n < 0 || (n > 0 && !lengths) || reserve_len <= 0 || !is_pow2(block_size) ||
        pool_slots < 0)
        return PKV_ERR_INVALID_ARG;
    pkv_waste_report r{};
    for (int32_t i = 0; i < n; ++i) {
        const int64_t L = lengths[i];
        if (L < 0 || L > reserve_len) return PKV_ERR_INVALID_ARG;
        r.used_slots += L;
        r.contiguous_reserved += reserve_len;
        r.paged_reserved += (L + block_size - 1) / block_size * block_size;
    }
    // how many of the requests, admitted in order, fit in the pool at once
    int64_t c = 0, p = 0;
    for (int32_t i = 0; i < n; ++i) {
        if (c + reserve_len > pool_slots) break;
        c += reserve_len;
        ++r.contiguous_admitted;
    }
    for (int32_t i = 0; i < n; ++i) {
        const int64_t need = ((int64_t)lengths[i] + block_size - 1) / block_size * block_size;
        if (p + need > pool_slots) break;
        p += need;
        ++r.paged_admitted;
    }
    *out = r;
    return PKV_OK;
}

}  // extern "C"
