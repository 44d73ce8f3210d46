// Internal C++ interface of the host block manager (see block_manager.cpp).
#pragma once

#include <cstdint>
#include <list>
#include <string>
#include <unordered_map>
#include <vector>

#include "pa.h"

namespace pa_host {

int64_t ceil_div(int64_t a, int64_t b);

class BlockManager {
  public:
    struct Seq {
        std::vector<int32_t> table;   // physical ids, logical order
        int64_t ctx = 0;              // tokens held
        std::vector<int32_t> tail;    // token ids of the partly filled last block (prefix cache)
        bool tail_known = true;       // false once a token was appended without its id
        bool swapped = false;         // swapped out to the host pool
        std::vector<char> on_cpu;     // while swapped: per logical block, 1 = host block id
        // while swapped, prefix cache on: per logical block, the GPU block left named in
        // the cache (-1: none) and its key, to take it back without a copy
        std::vector<int32_t> left_block;
        std::vector<std::string> left_key;
    };

    BlockManager(int num_blocks, int block_size, const int32_t* initial_free_order);
    static bool valid_order(int num_blocks, const int32_t* order);

    pa_status allocate(int64_t seq, int num_tokens);
    pa_status fork(int64_t parent, int64_t child);
    pa_status append_slot(int64_t seq, int64_t* slot, int32_t* cow_src, int32_t* cow_dst);
    pa_status free_seq(int64_t seq);
    pa_status slots(int64_t seq, int64_t start, int64_t count, int64_t* out) const;

    // prefix cache
    void enable_prefix_cache(bool on) { prefix_cache_ = on; }
    bool prefix_cache() const { return prefix_cache_; }
    pa_status allocate_prefix(int64_t seq, const int32_t* tokens, int num_tokens, int* cached_tokens);
    pa_status append_token(int64_t seq, int32_t token, int64_t* slot, int32_t* cow_src, int32_t* cow_dst);
    int num_cached() const { return (int)key_of_.size(); }
    int num_evictable() const { return (int)lru_.size(); }
    int64_t hits() const { return hits_; }
    int64_t lookups() const { return lookups_; }
    const std::list<int32_t>& evictable() const { return lru_; }
    bool named(int32_t b) const { return key_of_.count(b) != 0; }
    pa_status forget(int32_t b);      // drop an unreferenced cached block's name, free it
    // true when seq holds exactly n tokens and each of its full blocks is the
    // block the cache names for those token ids
    bool cached_as(int64_t seq, const int32_t* tokens, int n) const;

    // host swap pool
    pa_status set_cpu_blocks(int n);
    pa_status swap_out(int64_t seq, std::vector<int32_t>& pairs);   // (gpu, cpu) pairs
    pa_status swap_in(int64_t seq, std::vector<int32_t>& pairs);    // (cpu, gpu) pairs
    int swap_out_need(int64_t seq) const;                           // host blocks swap_out takes, or -1
    int swap_in_need(int64_t seq) const;                            // GPU blocks swap_in takes, or -1
    bool swapped(int64_t seq) const;
    const std::vector<int32_t>& cpu_free_list() const { return cpu_free_; }

    // blocks held by live sequences, and their slots holding a token of some holder
    void usage(int64_t* held_blocks, int64_t* filled_slots) const;

    const Seq* find(int64_t seq) const;
    int num_free() const { return (int)(free_.size() + lru_.size()); }
    int num_blocks() const { return num_blocks_; }
    int block_size() const { return block_size_; }
    int ref(int32_t b) const { return ref_[b]; }
    const std::vector<int32_t>& free_list() const { return free_; }

  private:
    pa_status append(int64_t seq, int32_t token, bool known, int64_t* slot, int32_t* cow_src,
                     int32_t* cow_dst);
    int32_t take_block();                                   // free list first, then evict LRU
    std::string make_key(int32_t parent, const int32_t* tokens) const;
    void register_block(int32_t block, int32_t parent, const int32_t* tokens);
    void release_block(int32_t block);                      // ref reached zero
    void unlink_lru(int32_t block);                         // a cached block is referenced again

    int num_blocks_;
    int block_size_;
    std::vector<int32_t> free_;   // back() is taken next
    std::vector<int32_t> ref_;
    std::unordered_map<int64_t, Seq> seqs_;
    // prefix cache: (parent block, token ids) of a full block -> block, and back
    bool prefix_cache_ = false;
    std::unordered_map<std::string, int32_t> block_of_;
    std::unordered_map<int32_t, std::string> key_of_;
    std::list<int32_t> lru_;                                  // cached blocks with ref 0, oldest first
    std::vector<std::list<int32_t>::iterator> lru_pos_;
    std::vector<char> in_lru_;
    int64_t hits_ = 0, lookups_ = 0;
    // host swap pool: LIFO free list of host block ids
    std::vector<int32_t> cpu_free_;
    int num_cpu_blocks_ = 0;
    int num_swapped_ = 0;
};

}  // namespace pa_host

struct pa_bm;
pa_host::BlockManager* pa_bm_impl(pa_bm* bm);
