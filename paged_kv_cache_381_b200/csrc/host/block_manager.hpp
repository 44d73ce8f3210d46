// Internal C++ interface of the host block manager (see block_manager.cpp).
#pragma once

#include <cstdint>
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
    };

    BlockManager(int num_blocks, int block_size, const int32_t* initial_free_order);
    static bool valid_order(int num_blocks, const int32_t* order);

    pa_status allocate(int64_t seq, int num_tokens);
    pa_status fork(int64_t parent, int64_t child);
    pa_status append_slot(int64_t seq, int64_t* slot, int32_t* cow_src, int32_t* cow_dst);
    pa_status free_seq(int64_t seq);
    pa_status slots(int64_t seq, int64_t start, int64_t count, int64_t* out) const;

    const Seq* find(int64_t seq) const;
    int num_free() const { return (int)free_.size(); }
    int num_blocks() const { return num_blocks_; }
    int block_size() const { return block_size_; }
    int ref(int32_t b) const { return ref_[b]; }
    const std::vector<int32_t>& free_list() const { return free_; }

  private:
    int num_blocks_;
    int block_size_;
    std::vector<int32_t> free_;   // back() is taken next
    std::vector<int32_t> ref_;
    std::unordered_map<int64_t, Seq> seqs_;
};

}  // namespace pa_host

struct pa_bm;
pa_host::BlockManager* pa_bm_impl(pa_bm* bm);
