// Host block manager: free list, per-block reference counts, block tables,
// copy-on-write.  Plain C++17, no CUDA calls.
//
// Rules (pages cited by title and section):
//  * "大模型推理引擎高频优化：连续批处理、PagedAttention 与 KV Cache 实战拆解" 3.3:
//    blocks are taken from the end of the free list; allocate takes
//    ceil_div(num_tokens, block_size) blocks; append_token takes a new block
//    only when the last one is full, otherwise writes at the end of it.
//  * "vLLM推理加速框架：PagedAttention与连续批处理技术解析" 2.1-2.2: a per-block
//    ref_count; blocks shared by several sequences are copied before a write
//    (copy-on-write).
//  * "大模型推理显存优化实战：PagedAttention机制原理与vLLM连续批处理配置", section
//    "PagedAttention分页注意力机制原理": sequences share prefix blocks by
//    reference; finished requests return their blocks to the free pool.
//  Free pushes blocks whose count reaches zero in logical table order.
//
//  Prefix cache ("大模型推理显存优化实战：PagedAttention机制原理与vLLM连续批处理配置",
//  section "Prefix Caching前缀复用优化": a new request whose prefix matches
//  cached KV references those blocks and skips their prefill), when enabled:
//  a full block is keyed by (parent block, its token ids), which names the
//  whole prefix exactly (no hash collisions); allocate_prefix references the
//  longest cached run of full prompt blocks and allocates the rest; blocks
//  filled by allocate_prefix or append_token are registered; a registered
//  block whose count reaches zero stays cached on an LRU list and is evicted
//  (unregistered and reused) only when the free list is empty.  A partly
//  filled block is never shared through the cache.  A block is registered
//  only under a registered parent (or as a first block), and free_seq puts a
//  sequence's cached blocks on the LRU list last block first, so a child is
//  always evicted before its parent and no key can name a reused parent.
//
//  Swap ("大模型推理显存优化实战：PagedAttention机制原理与vLLM连续批处理配置", section
//  "生产部署注意事项": when GPU memory runs short, requests' KV cache moves out to
//  CPU memory and back when GPU memory is free): a host pool of equal blocks
//  on its own LIFO list.  swap_out moves the blocks a sequence holds alone, in
//  logical order, and frees their GPU blocks; shared blocks stay resident and
//  referenced.  swap_in takes fresh GPU blocks for them.  Both are all or
//  nothing and report the block copies the caller runs.

#include "block_manager.hpp"

#include <cstring>
#include <iterator>
#include <new>

namespace pa_host {

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

BlockManager::BlockManager(int num_blocks, int block_size, const int32_t* initial_free_order)
    : num_blocks_(num_blocks), block_size_(block_size), ref_(num_blocks, 0), lru_pos_(num_blocks),
      in_lru_(num_blocks, 0) {
    free_.reserve(num_blocks);
    for (int i = 0; i < num_blocks; ++i)
        free_.push_back(initial_free_order ? initial_free_order[i] : i);
}

bool BlockManager::valid_order(int num_blocks, const int32_t* order) {
    if (!order) return true;
    std::vector<char> seen(num_blocks, 0);
    for (int i = 0; i < num_blocks; ++i) {
        int32_t b = order[i];
        if (b < 0 || b >= num_blocks || seen[b]) return false;
        seen[b] = 1;
    }
    return true;
}

int32_t BlockManager::take_block() {
    if (!free_.empty()) {
        int32_t b = free_.back();
        free_.pop_back();
        return b;
    }
    if (!lru_.empty()) {                 // evict the least recently released cached block
        int32_t b = lru_.front();
        lru_.pop_front();
        in_lru_[b] = 0;
        auto it = key_of_.find(b);
        if (it != key_of_.end()) {
            block_of_.erase(it->second);
            key_of_.erase(it);
        }
        return b;
    }
    return -1;
}

void BlockManager::release_block(int32_t b) {
    if (key_of_.count(b)) {
        lru_.push_back(b);
        lru_pos_[b] = std::prev(lru_.end());
        in_lru_[b] = 1;
    } else {
        free_.push_back(b);
    }
}

void BlockManager::unlink_lru(int32_t b) {
    if (in_lru_[b]) {
        lru_.erase(lru_pos_[b]);
        in_lru_[b] = 0;
    }
}

// A cached block with count zero whose K/V is not to be trusted (the writes
// that filled it were abandoned): its key goes, and the block returns to the
// free list instead of waiting on the LRU list.
pa_status BlockManager::forget(int32_t b) {
    if (b < 0 || b >= num_blocks_ || ref_[b] != 0 || !key_of_.count(b)) return PA_ERR_INVALID_ARG;
    unlink_lru(b);
    auto it = key_of_.find(b);
    block_of_.erase(it->second);
    key_of_.erase(it);
    free_.push_back(b);
    return PA_OK;
}

bool BlockManager::cached_as(int64_t seq, const int32_t* tokens, int n) const {
    auto it = seqs_.find(seq);
    if (it == seqs_.end() || it->second.swapped || it->second.ctx != n || (n > 0 && !tokens)) return false;
    const std::vector<int32_t>& t = it->second.table;
    int32_t parent = -1;
    for (int j = 0; j < n / block_size_; ++j) {
        auto b = block_of_.find(make_key(parent, tokens + (int64_t)j * block_size_));
        if (b == block_of_.end() || b->second != t[j]) return false;
        parent = t[j];
    }
    return true;
}

std::string BlockManager::make_key(int32_t parent, const int32_t* tokens) const {
    std::string k(sizeof(int32_t) * (1 + block_size_), '\0');
    std::memcpy(&k[0], &parent, sizeof(int32_t));
    std::memcpy(&k[sizeof(int32_t)], tokens, sizeof(int32_t) * block_size_);
    return k;
}

void BlockManager::register_block(int32_t block, int32_t parent, const int32_t* tokens) {
    if (parent >= 0 && !key_of_.count(parent)) return;         // prefix not named by the cache
    std::string k = make_key(parent, tokens);
    if (block_of_.count(k) || key_of_.count(block)) return;   // identical content already cached
    block_of_.emplace(k, block);
    key_of_.emplace(block, std::move(k));
}

pa_status BlockManager::allocate(int64_t seq, int num_tokens) {
    if (num_tokens < 0 || seqs_.count(seq)) return PA_ERR_INVALID_ARG;
    int64_t need = ceil_div(num_tokens, block_size_);
    if (need > (int64_t)num_free()) return PA_ERR_NO_BLOCKS;
    Seq s;
    s.ctx = num_tokens;
    s.tail_known = num_tokens == 0;
    s.table.reserve(need);
    for (int64_t i = 0; i < need; ++i) {
        int32_t b = take_block();
        ref_[b] = 1;
        s.table.push_back(b);
    }
    seqs_.emplace(seq, std::move(s));
    return PA_OK;
}

pa_status BlockManager::allocate_prefix(int64_t seq, const int32_t* tokens, int num_tokens, int* cached_tokens) {
    if (num_tokens < 0 || seqs_.count(seq) || (num_tokens > 0 && !tokens)) return PA_ERR_INVALID_ARG;
    const int bs = block_size_;
    const int nfull = num_tokens / bs;
    // longest run of cached full blocks, probed before anything changes
    std::vector<int32_t> hit;
    int32_t parent = -1;
    int probed = 0;
    if (prefix_cache_) {
        for (int j = 0; j < nfull; ++j) {
            ++probed;
            auto it = block_of_.find(make_key(parent, tokens + (int64_t)j * bs));
            if (it == block_of_.end()) break;
            hit.push_back(it->second);
            parent = it->second;
        }
    }
    int64_t hits_in_lru = 0;
    for (int32_t b : hit) hits_in_lru += in_lru_[b];
    const int64_t need = ceil_div(num_tokens, bs) - (int64_t)hit.size();
    if (need > (int64_t)num_free() - hits_in_lru) return PA_ERR_NO_BLOCKS;
    lookups_ += probed;
    hits_ += (int64_t)hit.size();
    Seq s;
    s.ctx = num_tokens;
    for (int32_t b : hit) {
        if (in_lru_[b]) {
            lru_.erase(lru_pos_[b]);
            in_lru_[b] = 0;
        }
        ref_[b] += 1;
        s.table.push_back(b);
    }
    parent = hit.empty() ? -1 : hit.back();
    for (int64_t j = (int64_t)hit.size(); j < ceil_div(num_tokens, bs); ++j) {
        int32_t b = take_block();
        ref_[b] = 1;
        s.table.push_back(b);
        if (prefix_cache_ && j < nfull) {
            register_block(b, parent, tokens + j * bs);
            parent = b;
        }
    }
    s.tail.assign(tokens + (int64_t)nfull * bs, tokens + num_tokens);
    s.tail_known = true;
    seqs_.emplace(seq, std::move(s));
    if (cached_tokens) *cached_tokens = (int)hit.size() * bs;
    return PA_OK;
}

pa_status BlockManager::fork(int64_t parent, int64_t child) {
    auto it = seqs_.find(parent);
    if (it == seqs_.end() || seqs_.count(child) || it->second.swapped) return PA_ERR_INVALID_ARG;
    Seq c = it->second;
    for (int32_t b : c.table) ref_[b] += 1;
    seqs_.emplace(child, std::move(c));
    return PA_OK;
}

pa_status BlockManager::append_slot(int64_t seq, int64_t* slot, int32_t* cow_src, int32_t* cow_dst) {
    return append(seq, 0, false, slot, cow_src, cow_dst);
}

pa_status BlockManager::append_token(int64_t seq, int32_t token, int64_t* slot, int32_t* cow_src, int32_t* cow_dst) {
    return append(seq, token, true, slot, cow_src, cow_dst);
}

pa_status BlockManager::append(int64_t seq, int32_t token, bool known, int64_t* slot, int32_t* cow_src,
                               int32_t* cow_dst) {
    auto it = seqs_.find(seq);
    if (it == seqs_.end() || it->second.swapped) return PA_ERR_INVALID_ARG;
    Seq& s = it->second;
    const int64_t pos = s.ctx;
    int32_t src = -1, dst = -1;
    if (pos % block_size_ == 0) {
        // the last block is full (or there is none): open a fresh block
        if (num_free() == 0) return PA_ERR_NO_BLOCKS;
        int32_t b = take_block();
        ref_[b] = 1;
        s.table.push_back(b);
        s.tail.clear();
    } else {
        int32_t last = s.table.back();
        if (ref_[last] > 1) {
            // shared partly filled block: give this sequence a private copy
            if (num_free() == 0) return PA_ERR_NO_BLOCKS;
            int32_t b = take_block();
            ref_[b] = 1;
            ref_[last] -= 1;
            s.table.back() = b;
            src = last;
            dst = b;
        }
    }
    s.ctx = pos + 1;
    s.tail.push_back(token);
    s.tail_known = s.tail_known && known;
    if (prefix_cache_ && s.tail_known && (int)s.tail.size() == block_size_) {
        const size_t n = s.table.size();
        register_block(s.table[n - 1], n >= 2 ? s.table[n - 2] : -1, s.tail.data());
    }
    if (slot) *slot = (int64_t)s.table[pos / block_size_] * block_size_ + pos % block_size_;
    if (cow_src) *cow_src = src;
    if (cow_dst) *cow_dst = dst;
    return PA_OK;
}

pa_status BlockManager::free_seq(int64_t seq) {
    auto it = seqs_.find(seq);
    if (it == seqs_.end()) return PA_ERR_INVALID_ARG;
    std::vector<int32_t> cached;
    const Seq& sq = it->second;
    if (sq.swapped) {
        // host blocks go back to their list; shared GPU references are dropped (named
        // blocks reaching zero wait on the LRU list, last block first)
        for (size_t j = 0; j < sq.table.size(); ++j) {
            const int32_t b = sq.table[j];
            if (sq.on_cpu[j]) {
                cpu_free_.push_back(b);
            } else {
                if (ref_[b] <= 0) return PA_ERR_INVALID_ARG;
                if (--ref_[b] == 0) {
                    if (key_of_.count(b))
                        cached.push_back(b);
                    else
                        free_.push_back(b);
                }
            }
        }
        for (auto r = cached.rbegin(); r != cached.rend(); ++r) release_block(*r);
        --num_swapped_;
        seqs_.erase(it);
        return PA_OK;
    }
    for (int32_t b : it->second.table) {
        if (ref_[b] <= 0) return PA_ERR_INVALID_ARG;  // corrupted counts; never expected
        if (--ref_[b] == 0) {
            if (key_of_.count(b))
                cached.push_back(b);
            else
                free_.push_back(b);
        }
    }
    for (auto r = cached.rbegin(); r != cached.rend(); ++r) release_block(*r);   // last block first
    seqs_.erase(it);
    return PA_OK;
}

pa_status BlockManager::set_cpu_blocks(int n) {
    if (n < 0 || num_swapped_ > 0) return PA_ERR_INVALID_ARG;
    num_cpu_blocks_ = n;
    cpu_free_.clear();
    for (int i = 0; i < n; ++i) cpu_free_.push_back(i);
    return PA_OK;
}

bool BlockManager::swapped(int64_t seq) const {
    const Seq* s = find(seq);
    return s && s->swapped;
}

int BlockManager::swap_out_need(int64_t seq) const {
    const Seq* s = find(seq);
    if (!s || s->swapped) return -1;
    int n = 0;
    for (int32_t b : s->table) n += ref_[b] == 1;
    return n;
}

int BlockManager::swap_in_need(int64_t seq) const {
    const Seq* s = find(seq);
    if (!s || !s->swapped) return -1;
    int n = 0;
    for (char c : s->on_cpu) n += c != 0;
    return n;
}

pa_status BlockManager::swap_out(int64_t seq, std::vector<int32_t>& pairs) {
    const int need = swap_out_need(seq);
    if (need < 0) return PA_ERR_INVALID_ARG;
    if (need > (int)cpu_free_.size()) return PA_ERR_NO_BLOCKS;
    Seq& s = seqs_[seq];
    s.swapped = true;
    s.on_cpu.assign(s.table.size(), 0);
    s.left_block.assign(s.table.size(), -1);
    s.left_key.assign(s.table.size(), std::string());
    pairs.clear();
    std::vector<int32_t> named;
    for (size_t j = 0; j < s.table.size(); ++j) {
        const int32_t g = s.table[j];
        if (ref_[g] != 1) continue;              // shared: stays resident, still referenced
        const int32_t c = cpu_free_.back();
        cpu_free_.pop_back();
        pairs.push_back(g);
        pairs.push_back(c);
        ref_[g] = 0;
        auto k = key_of_.find(g);
        if (k != key_of_.end()) {                // stays named and reusable until evicted
            named.push_back(g);
            s.left_block[j] = g;
            s.left_key[j] = k->second;
        } else {
            free_.push_back(g);
        }
        s.table[j] = c;
        s.on_cpu[j] = 1;
    }
    for (auto r = named.rbegin(); r != named.rend(); ++r) release_block(*r);   // last block first
    ++num_swapped_;
    return PA_OK;
}

pa_status BlockManager::swap_in(int64_t seq, std::vector<int32_t>& pairs) {
    const int need = swap_in_need(seq);
    if (need < 0) return PA_ERR_INVALID_ARG;
    if (need > num_free()) return PA_ERR_NO_BLOCKS;
    Seq& s = seqs_[seq];
    pairs.clear();
    for (size_t j = 0; j < s.table.size(); ++j) {
        if (!s.on_cpu[j]) continue;
        const int32_t c = s.table[j];
        int32_t g = s.left_block.empty() ? -1 : s.left_block[j];
        if (g >= 0) {
            // taken back with no copy while the cache still names it by the same key
            auto b = block_of_.find(s.left_key[j]);
            if (b == block_of_.end() || b->second != g) g = -1;
        }
        if (g >= 0) {
            unlink_lru(g);
            ++ref_[g];
        } else {
            g = take_block();                     // may evict
            ref_[g] = 1;
            pairs.push_back(c);
            pairs.push_back(g);
        }
        cpu_free_.push_back(c);
        s.table[j] = g;
    }
    s.on_cpu.clear();
    s.left_block.clear();
    s.left_key.clear();
    s.swapped = false;
    --num_swapped_;
    return PA_OK;
}

void BlockManager::usage(int64_t* held_blocks, int64_t* filled_slots) const {
    // a shared block is counted once, filled up to the furthest of its holders
    std::vector<int32_t> fill(num_blocks_, 0);
    for (const auto& kv : seqs_) {
        const Seq& s = kv.second;
        for (size_t j = 0; j < s.table.size(); ++j) {
            if (s.swapped && s.on_cpu[j]) continue;              // a host block
            int64_t f = s.ctx - (int64_t)j * block_size_;
            int32_t n = (int32_t)(f < block_size_ ? f : block_size_);
            if (n > fill[s.table[j]]) fill[s.table[j]] = n;
        }
    }
    int64_t held = 0, filled = 0;
    for (int b = 0; b < num_blocks_; ++b) {
        if (ref_[b] > 0) {
            ++held;
            filled += fill[b];
        }
    }
    if (held_blocks) *held_blocks = held;
    if (filled_slots) *filled_slots = filled;
}

const BlockManager::Seq* BlockManager::find(int64_t seq) const {
    auto it = seqs_.find(seq);
    return it == seqs_.end() ? nullptr : &it->second;
}

pa_status BlockManager::slots(int64_t seq, int64_t start, int64_t count, int64_t* out) const {
    const Seq* s = find(seq);
    if (!s || s->swapped || start < 0 || count < 0) return PA_ERR_INVALID_ARG;
    if (start + count > (int64_t)s->table.size() * block_size_) return PA_ERR_INVALID_ARG;
    for (int64_t p = start; p < start + count; ++p)
        out[p - start] = (int64_t)s->table[p / block_size_] * block_size_ + p % block_size_;
    return PA_OK;
}

}  // namespace pa_host

using pa_host::BlockManager;

struct pa_bm {
    BlockManager impl;
    pa_bm(int nb, int bs, const int32_t* order) : impl(nb, bs, order) {}
};

extern "C" {

pa_status pa_bm_create(int num_blocks, int block_size, const int32_t* initial_free_order, pa_bm** out) {
    if (!out || num_blocks <= 0 || block_size <= 0) return PA_ERR_INVALID_ARG;
    if (!BlockManager::valid_order(num_blocks, initial_free_order)) return PA_ERR_INVALID_ARG;
    *out = new (std::nothrow) pa_bm(num_blocks, block_size, initial_free_order);
    return *out ? PA_OK : PA_ERR_INVALID_ARG;
}

void pa_bm_destroy(pa_bm* bm) { delete bm; }

pa_status pa_bm_allocate(pa_bm* bm, int64_t seq_id, int num_tokens) {
    return bm ? bm->impl.allocate(seq_id, num_tokens) : PA_ERR_INVALID_ARG;
}

pa_status pa_bm_fork(pa_bm* bm, int64_t parent, int64_t child) {
    return bm ? bm->impl.fork(parent, child) : PA_ERR_INVALID_ARG;
}

pa_status pa_bm_append_slot(pa_bm* bm, int64_t seq_id, int64_t* slot, int32_t* cow_src, int32_t* cow_dst) {
    return bm ? bm->impl.append_slot(seq_id, slot, cow_src, cow_dst) : PA_ERR_INVALID_ARG;
}

pa_status pa_bm_free(pa_bm* bm, int64_t seq_id) {
    return bm ? bm->impl.free_seq(seq_id) : PA_ERR_INVALID_ARG;
}

pa_status pa_bm_block_table(const pa_bm* bm, int64_t seq_id, int32_t* out, int cap, int* n) {
    if (!bm) return PA_ERR_INVALID_ARG;
    const BlockManager::Seq* s = bm->impl.find(seq_id);
    if (!s) return PA_ERR_INVALID_ARG;
    int len = (int)s->table.size();
    if (n) *n = len;
    if (len > cap || (len > 0 && !out)) return PA_ERR_INVALID_ARG;
    for (int i = 0; i < len; ++i) out[i] = s->table[i];
    return PA_OK;
}

pa_status pa_bm_slots(const pa_bm* bm, int64_t seq_id, int start, int count, int64_t* out) {
    if (!bm || (count > 0 && !out)) return PA_ERR_INVALID_ARG;
    return bm->impl.slots(seq_id, start, count, out);
}

pa_status pa_bm_stats(const pa_bm* bm, int64_t seq_id, int* num_free, int* num_used, int* context_len) {
    if (!bm) return PA_ERR_INVALID_ARG;
    if (num_free) *num_free = bm->impl.num_free();
    if (num_used) *num_used = bm->impl.num_blocks() - bm->impl.num_free();
    if (context_len) {
        const BlockManager::Seq* s = seq_id >= 0 ? bm->impl.find(seq_id) : nullptr;
        *context_len = s ? (int)s->ctx : -1;
    }
    return PA_OK;
}

pa_status pa_bm_ref_count(const pa_bm* bm, int32_t block, int* count) {
    if (!bm || !count || block < 0 || block >= bm->impl.num_blocks()) return PA_ERR_INVALID_ARG;
    *count = bm->impl.ref(block);
    return PA_OK;
}

pa_status pa_bm_free_list(const pa_bm* bm, int32_t* out, int cap, int* n) {
    if (!bm) return PA_ERR_INVALID_ARG;
    const auto& fl = bm->impl.free_list();
    int len = (int)fl.size();
    if (n) *n = len;
    if (len > cap || (len > 0 && !out)) return PA_ERR_INVALID_ARG;
    for (int i = 0; i < len; ++i) out[i] = fl[i];
    return PA_OK;
}

pa_status pa_bm_pack(const pa_bm* bm, const int64_t* seq_ids, int n, int width, int32_t* tables,
                     int32_t* context_lens) {
    if (!bm || n < 0 || width < 0 || (n > 0 && (!seq_ids || !tables || !context_lens)))
        return PA_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i) {
        const BlockManager::Seq* s = bm->impl.find(seq_ids[i]);
        if (!s || s->swapped || (int)s->table.size() > width) return PA_ERR_INVALID_ARG;
        int32_t* row = tables + (int64_t)i * width;
        int len = (int)s->table.size();
        for (int j = 0; j < width; ++j) row[j] = j < len ? s->table[j] : -1;
        context_lens[i] = (int32_t)s->ctx;
    }
    return PA_OK;
}

}  // extern "C"

pa_host::BlockManager* pa_bm_impl(pa_bm* bm) { return bm ? &bm->impl : nullptr; }

extern "C" {

pa_status pa_bm_enable_prefix_cache(pa_bm* bm, int enable) {
    if (!bm) return PA_ERR_INVALID_ARG;
    bm->impl.enable_prefix_cache(enable != 0);
    return PA_OK;
}

pa_status pa_bm_allocate_prefix(pa_bm* bm, int64_t seq_id, const int32_t* tokens, int num_tokens,
                                int* cached_tokens) {
    return bm ? bm->impl.allocate_prefix(seq_id, tokens, num_tokens, cached_tokens) : PA_ERR_INVALID_ARG;
}

pa_status pa_bm_append_token(pa_bm* bm, int64_t seq_id, int32_t token, int64_t* slot, int32_t* cow_src,
                             int32_t* cow_dst) {
    return bm ? bm->impl.append_token(seq_id, token, slot, cow_src, cow_dst) : PA_ERR_INVALID_ARG;
}

pa_status pa_bm_cache_stats(const pa_bm* bm, int* cached_blocks, int* evictable_blocks, int64_t* hits,
                            int64_t* lookups) {
    if (!bm) return PA_ERR_INVALID_ARG;
    if (cached_blocks) *cached_blocks = bm->impl.num_cached();
    if (evictable_blocks) *evictable_blocks = bm->impl.num_evictable();
    if (hits) *hits = bm->impl.hits();
    if (lookups) *lookups = bm->impl.lookups();
    return PA_OK;
}

pa_status pa_bm_usage(const pa_bm* bm, int64_t* held_blocks, int64_t* filled_slots) {
    if (!bm) return PA_ERR_INVALID_ARG;
    bm->impl.usage(held_blocks, filled_slots);
    return PA_OK;
}

pa_status pa_bm_set_cpu_blocks(pa_bm* bm, int num_cpu_blocks) {
    return bm ? bm->impl.set_cpu_blocks(num_cpu_blocks) : PA_ERR_INVALID_ARG;
}

static pa_status swap_common(pa_bm* bm, int64_t seq_id, int32_t* pairs, int cap, int* n, bool out) {
    if (!bm) return PA_ERR_INVALID_ARG;
    const int need = out ? bm->impl.swap_out_need(seq_id) : bm->impl.swap_in_need(seq_id);
    if (need < 0) return PA_ERR_INVALID_ARG;
    if (n) *n = need;
    if (need > cap || (need > 0 && !pairs)) return PA_ERR_INVALID_ARG;   // nothing changed
    std::vector<int32_t> p;
    pa_status st = out ? bm->impl.swap_out(seq_id, p) : bm->impl.swap_in(seq_id, p);
    if (st != PA_OK) return st;
    for (size_t i = 0; i < p.size(); ++i) pairs[i] = p[i];
    // the copies made: a swap-in takes blocks still cached back without one
    if (n) *n = (int)(p.size() / 2);
    return PA_OK;
}

pa_status pa_bm_swap_out(pa_bm* bm, int64_t seq_id, int32_t* pairs, int cap, int* n) {
    return swap_common(bm, seq_id, pairs, cap, n, true);
}

pa_status pa_bm_swap_in(pa_bm* bm, int64_t seq_id, int32_t* pairs, int cap, int* n) {
    return swap_common(bm, seq_id, pairs, cap, n, false);
}

pa_status pa_bm_swapped(const pa_bm* bm, int64_t seq_id, int* swapped) {
    if (!bm || !swapped || !bm->impl.find(seq_id)) return PA_ERR_INVALID_ARG;
    *swapped = bm->impl.swapped(seq_id) ? 1 : 0;
    return PA_OK;
}

pa_status pa_bm_cpu_free_list(const pa_bm* bm, int32_t* out, int cap, int* n) {
    if (!bm) return PA_ERR_INVALID_ARG;
    const auto& fl = bm->impl.cpu_free_list();
    int len = (int)fl.size();
    if (n) *n = len;
    if (len > cap || (len > 0 && !out)) return PA_ERR_INVALID_ARG;
    for (int i = 0; i < len; ++i) out[i] = fl[i];
    return PA_OK;
}

pa_status pa_bm_forget(pa_bm* bm, int32_t block) {
    return bm ? bm->impl.forget(block) : PA_ERR_INVALID_ARG;
}

pa_status pa_bm_evictable(const pa_bm* bm, int32_t* out, int cap, int* n) {
    if (!bm) return PA_ERR_INVALID_ARG;
    const auto& l = bm->impl.evictable();
    int len = (int)l.size();
    if (n) *n = len;
    if (len > cap || (len > 0 && !out)) return PA_ERR_INVALID_ARG;
    int i = 0;
    for (int32_t b : l) out[i++] = b;
    return PA_OK;
}

}  // extern "C"
