// Host scheduler: iteration-level (continuous) batching over the block
// manager.  Plain C++17, no CUDA calls.
//
// One step ("大模型推理引擎高频优化：连续批处理、PagedAttention 与 KV Cache 实战拆解" 2.2,
// Scheduler.schedule; "大模型推理显存优化实战：PagedAttention机制原理与vLLM连续批处理配置",
// section "连续批处理Continuous Batching配置"):
//  1. sequences that generated their output length leave and free their blocks;
//  2. admission, first-come first-served, against a free-block budget that each
//     admitted request charges with ceil(own_tokens / block_size) + 1 (+1 when it
//     forks a parallel-sampling child); the first request that does not fit
//     stops admission and stays at the head of the queue; the running count is
//     capped (max-num-seqs);
//  3. every running sequence reserves the slot of its next token; when the pool
//     is exhausted the most recently admitted running sequence is preempted
//     ("vLLM推理加速框架：PagedAttention与连续批处理技术解析" 3.2 names preemptive
//     scheduling; recompute-style preemption is the reading adopted): its blocks
//     are freed and it returns to the front of the queue with its progress, and
//     its whole history is written again when it is re-admitted.
// The step's record lists cache writes and copy-on-write copies in issue order.
// A preemption drops from it every op whose target block the preemption
// returned to the free list (dead work; the block may be taken again later in
// the same step), so within a step every slot is written at most once.
//
// Preemption by swap ("大模型推理显存优化实战：PagedAttention机制原理与vLLM连续批处理配置",
// section "生产部署注意事项": KV cache moved out to CPU memory when GPU memory
// runs short, back in later), when selected: a victim whose private blocks fit
// the host pool is swapped out instead (its "so" copies join the op list; its
// writes of the step stay, since the copies carry them out) and waits in a
// FIFO swapped queue; swapped sequences come back before any admission, each
// needing its host blocks + 1 from the budget ("si" copies), and new requests
// are admitted only once none is left.  Swap-out ops target host blocks and
// are never dead; a preemption happens only when no GPU block is free, so the
// blocks a swap-out freed earlier in the step are all taken again by then and
// only the recomputed victim's own ops die.  Ops run in issue order;
// consecutive writes form one launch with distinct slots.
//
// Admission through the prefix cache ("大模型推理显存优化实战：PagedAttention机制原理与
// vLLM连续批处理配置", section "Prefix Caching前缀复用优化": a request whose prompt
// starts with cached KV references those blocks and skips their prefill), when
// enabled: each sequence carries its token history; admission allocates through
// the cache with the whole history and lists writes only past the cached
// blocks; decode reservations record their token ids (from a caller-given
// function) so that filled blocks get cached.  A recompute preemption forgets
// every block that this step's ops target and that the preemption left cached
// with no holder, before dropping the dead ops, so no later lookup finds K/V
// whose writes were abandoned.

#include <deque>
#include <new>
#include <utility>
#include <vector>

#include "block_manager.hpp"

namespace {

struct SeqState {
    int64_t id = -1;
    int64_t output_len = 0;
    bool shares_prefix = false;
    int64_t history = 0;     // tokens held (shared prefix included)
    int64_t generated = 0;
    int64_t fork_child = -1;
    int64_t fork_output_len = 0;
    bool forked = false;
    std::vector<int32_t> tokens;   // token history (admission through the prefix cache)
};

}  // namespace

struct pa_sched {
    pa_host::BlockManager* bm = nullptr;
    int max_running = 0;
    int64_t prefix_seq = -1;
    int64_t prefix_len = 0;
    std::deque<SeqState> waiting;
    std::vector<SeqState> running;
    int preempt_mode = PA_PREEMPT_RECOMPUTE;
    std::deque<SeqState> swapped;
    std::vector<int64_t> swapped_out, swapped_in;
    // record of the last step
    std::vector<int64_t> finished, admitted, preempted;
    std::vector<int32_t> op_kind;
    std::vector<int64_t> op_a, op_b, op_c;
    std::vector<int64_t> run_ids;
    std::vector<int32_t> run_ctx;
    // admission through the prefix cache
    bool prefix_cache = false;
    std::vector<int32_t> prefix_tokens;
    pa_token_fn token_fn = nullptr;
    void* token_ctx = nullptr;

    void rec_write(int64_t seq, int64_t pos, int64_t slot) {
        op_kind.push_back(0); op_a.push_back(seq); op_b.push_back(pos); op_c.push_back(slot);
    }
    void rec_copy(int32_t src, int32_t dst) {
        op_kind.push_back(1); op_a.push_back(src); op_b.push_back(dst); op_c.push_back(-1);
    }
    void rec_swap(int kind, int32_t a, int32_t b) {
        op_kind.push_back(kind); op_a.push_back(a); op_b.push_back(b); op_c.push_back(-1);
    }
    // Remove ops (writes into, copies into, swap-ins into) whose target GPU block
    // is free again; swap-outs target host blocks and stay.
    void drop_dead_ops() {
        const int bs = bm->block_size();
        size_t w = 0;
        for (size_t i = 0; i < op_kind.size(); ++i) {
            if (op_kind[i] != 2) {
                const int64_t block = op_kind[i] == 0 ? op_c[i] / bs : op_b[i];
                if (bm->ref((int32_t)block) == 0) continue;
            }
            op_kind[w] = op_kind[i]; op_a[w] = op_a[i]; op_b[w] = op_b[i]; op_c[w] = op_c[i];
            ++w;
        }
        op_kind.resize(w); op_a.resize(w); op_b.resize(w); op_c.resize(w);
    }
    // Recompute preemption with the prefix cache: blocks targeted by this step's
    // ops, left cached with count zero by the victim's release, lose their keys.
    pa_status forget_abandoned() {
        const int bs = bm->block_size();
        std::vector<char> seen(bm->num_blocks(), 0);
        pa_status st;
        for (size_t i = 0; i < op_kind.size(); ++i) {
            if (op_kind[i] == 2) continue;
            const int32_t b = (int32_t)(op_kind[i] == 0 ? op_c[i] / bs : op_b[i]);
            if (seen[b]) continue;
            seen[b] = 1;
            if (bm->ref(b) == 0 && bm->named(b) && (st = bm->forget(b)) != PA_OK) return st;
        }
        return PA_OK;
    }
    int64_t own_tokens(const SeqState& s) const { return s.history - (s.shares_prefix ? prefix_len : 0); }
    int64_t required(const SeqState& s) const {
        int64_t need = pa_host::ceil_div(own_tokens(s), bm->block_size()) + 1;
        if (s.fork_child >= 0 && !s.forked) need += 1;
        return need;
    }
    pa_status admit(SeqState s);
    pa_status step();
};

pa_status pa_sched::admit(SeqState s) {
    pa_status st;
    if (prefix_cache) {
        int cached = 0;
        if ((st = bm->allocate_prefix(s.id, s.tokens.data(), (int)s.history, &cached)) != PA_OK) return st;
        const int64_t count = s.history - cached;
        std::vector<int64_t> slots(count);
        if (count > 0 && (st = bm->slots(s.id, cached, count, slots.data())) != PA_OK) return st;
        for (int64_t k = 0; k < count; ++k) rec_write(s.id, cached + k, slots[k]);
    } else if (s.shares_prefix) {
        if ((st = bm->fork(prefix_seq, s.id)) != PA_OK) return st;
        for (int64_t pos = prefix_len; pos < s.history; ++pos) {
            int64_t slot; int32_t src, dst;
            if ((st = bm->append_slot(s.id, &slot, &src, &dst)) != PA_OK) return st;
            if (src >= 0) rec_copy(src, dst);
            rec_write(s.id, pos, slot);
        }
    } else {
        if ((st = bm->allocate(s.id, (int)s.history)) != PA_OK) return st;
        std::vector<int64_t> slots(s.history);
        if (s.history > 0 && (st = bm->slots(s.id, 0, s.history, slots.data())) != PA_OK) return st;
        for (int64_t pos = 0; pos < s.history; ++pos) rec_write(s.id, pos, slots[pos]);
    }
    admitted.push_back(s.id);
    const bool spawn = s.fork_child >= 0 && !s.forked;
    if (spawn) s.forked = true;
    SeqState c;
    if (spawn) {
        if ((st = bm->fork(s.id, s.fork_child)) != PA_OK) return st;
        c.id = s.fork_child;
        c.output_len = s.fork_output_len;
        c.shares_prefix = s.shares_prefix;
        c.history = s.history;
        if (prefix_cache) c.tokens.assign(s.tokens.begin(), s.tokens.begin() + s.history);
    }
    running.push_back(std::move(s));
    if (spawn) {
        admitted.push_back(c.id);
        running.push_back(std::move(c));
    }
    return PA_OK;
}

pa_status pa_sched::step() {
    finished.clear(); admitted.clear(); preempted.clear();
    swapped_out.clear(); swapped_in.clear();
    op_kind.clear(); op_a.clear(); op_b.clear(); op_c.clear();
    run_ids.clear(); run_ctx.clear();
    pa_status st;
    // 1. finish
    std::vector<SeqState> keep;
    keep.reserve(running.size());
    for (SeqState& s : running) {
        if (s.generated >= s.output_len) {
            if ((st = bm->free_seq(s.id)) != PA_OK) return st;
            finished.push_back(s.id);
        } else {
            keep.push_back(std::move(s));
        }
    }
    running.swap(keep);
    // 2. swapped sequences come back first; then admit, FCFS against the free-block
    // budget, only once none is left swapped out
    int64_t budget = bm->num_free();
    std::vector<int32_t> pairs;
    while (!swapped.empty() && (int)running.size() < max_running) {
        const SeqState& head = swapped.front();
        const int64_t need = bm->swap_in_need(head.id) + 1;
        if (need > budget) break;
        if ((st = bm->swap_in(head.id, pairs)) != PA_OK) return st;
        for (size_t k = 0; k < pairs.size(); k += 2) rec_swap(3, pairs[k], pairs[k + 1]);
        budget -= need;
        swapped_in.push_back(head.id);
        running.push_back(std::move(swapped.front()));
        swapped.pop_front();
    }
    while (swapped.empty() && !waiting.empty() && budget > 0 && (int)running.size() < max_running) {
        const SeqState& head = waiting.front();
        int64_t need = required(head);
        if (need > budget) break;
        int extra = (head.fork_child >= 0 && !head.forked) ? 1 : 0;
        if ((int)running.size() + 1 + extra > max_running) break;
        SeqState s = std::move(waiting.front());
        waiting.pop_front();
        budget -= need;
        if ((st = admit(std::move(s))) != PA_OK) return st;
    }
    // 3. reserve every running sequence's next slot, preempting when exhausted
    size_t i = 0;
    while (i < running.size()) {
        SeqState& s = running[i];
        int64_t slot; int32_t src, dst;
        int32_t tok = 0;
        if (prefix_cache) {
            tok = token_fn(token_ctx, s.id, s.history);
            st = bm->append_token(s.id, tok, &slot, &src, &dst);
        } else {
            st = bm->append_slot(s.id, &slot, &src, &dst);
        }
        if (st == PA_ERR_NO_BLOCKS) {
            SeqState victim = std::move(running.back());
            running.pop_back();
            if (preempt_mode == PA_PREEMPT_SWAP) {
                const int need = bm->swap_out_need(victim.id);
                if (need >= 0 && need <= (int)bm->cpu_free_list().size()) {
                    if ((st = bm->swap_out(victim.id, pairs)) != PA_OK) return st;
                    for (size_t k = 0; k < pairs.size(); k += 2) rec_swap(2, pairs[k], pairs[k + 1]);
                    swapped_out.push_back(victim.id);
                    preempted.push_back(victim.id);
                    swapped.push_back(std::move(victim));
                    continue;
                }
            }
            if ((st = bm->free_seq(victim.id)) != PA_OK) return st;
            if (prefix_cache && (st = forget_abandoned()) != PA_OK) return st;
            drop_dead_ops();
            preempted.push_back(victim.id);
            waiting.push_front(std::move(victim));
            continue;   // retry the same index (or stop if the victim was this one)
        }
        if (st != PA_OK) return st;
        if (src >= 0) rec_copy(src, dst);
        rec_write(s.id, s.history, slot);
        if (prefix_cache) {
            s.tokens.resize(s.history);
            s.tokens.push_back(tok);
        }
        s.history += 1;
        s.generated += 1;
        ++i;
    }
    for (const SeqState& s : running) {
        run_ids.push_back(s.id);
        run_ctx.push_back((int32_t)s.history);
    }
    return PA_OK;
}

extern "C" {

pa_status pa_sched_create(pa_bm* bm, int max_running, int64_t prefix_seq, pa_sched** out) {
    pa_host::BlockManager* impl = pa_bm_impl(bm);
    if (!impl || !out || max_running <= 0) return PA_ERR_INVALID_ARG;
    int64_t plen = 0;
    if (prefix_seq >= 0) {
        const pa_host::BlockManager::Seq* p = impl->find(prefix_seq);
        if (!p) return PA_ERR_INVALID_ARG;
        plen = p->ctx;
    }
    pa_sched* s = new (std::nothrow) pa_sched();
    if (!s) return PA_ERR_INVALID_ARG;
    s->bm = impl;
    s->max_running = max_running;
    s->prefix_seq = prefix_seq;
    s->prefix_len = plen;
    *out = s;
    return PA_OK;
}

void pa_sched_destroy(pa_sched* s) { delete s; }

pa_status pa_sched_set_preemption(pa_sched* s, int mode) {
    if (!s || (mode != PA_PREEMPT_RECOMPUTE && mode != PA_PREEMPT_SWAP)) return PA_ERR_INVALID_ARG;
    if (mode == PA_PREEMPT_RECOMPUTE && !s->swapped.empty()) return PA_ERR_INVALID_ARG;
    s->preempt_mode = mode;
    return PA_OK;
}

pa_status pa_sched_swap_counts(const pa_sched* s, int* num_swapped_out, int* num_swapped_in, int* num_swapped) {
    if (!s) return PA_ERR_INVALID_ARG;
    if (num_swapped_out) *num_swapped_out = (int)s->swapped_out.size();
    if (num_swapped_in) *num_swapped_in = (int)s->swapped_in.size();
    if (num_swapped) *num_swapped = (int)s->swapped.size();
    return PA_OK;
}

pa_status pa_sched_swap_record(const pa_sched* s, int64_t* swapped_out, int64_t* swapped_in) {
    if (!s) return PA_ERR_INVALID_ARG;
    if (swapped_out) for (size_t i = 0; i < s->swapped_out.size(); ++i) swapped_out[i] = s->swapped_out[i];
    if (swapped_in) for (size_t i = 0; i < s->swapped_in.size(); ++i) swapped_in[i] = s->swapped_in[i];
    return PA_OK;
}

static pa_status queue_request(pa_sched* s, int64_t seq_id, const int32_t* tokens, int prompt_len,
                               int output_len, int shares_prefix, int64_t fork_child, int fork_output_len) {
    if (!s || prompt_len < 0 || output_len < 0 || fork_output_len < 0) return PA_ERR_INVALID_ARG;
    if (shares_prefix && s->prefix_seq < 0) return PA_ERR_INVALID_ARG;
    SeqState q;
    q.id = seq_id;
    q.output_len = output_len;
    q.shares_prefix = shares_prefix != 0;
    q.history = (q.shares_prefix ? s->prefix_len : 0) + prompt_len;
    q.fork_child = fork_child;
    q.fork_output_len = fork_output_len;
    if (s->prefix_cache) {
        if (q.shares_prefix) q.tokens = s->prefix_tokens;
        if (prompt_len > 0) q.tokens.insert(q.tokens.end(), tokens, tokens + prompt_len);
    }
    s->waiting.push_back(std::move(q));
    return PA_OK;
}

pa_status pa_sched_add_request(pa_sched* s, int64_t seq_id, int prompt_len, int output_len,
                               int shares_prefix, int64_t fork_child, int fork_output_len) {
    if (s && s->prefix_cache) return PA_ERR_INVALID_ARG;     // needs the prompt's token ids
    return queue_request(s, seq_id, nullptr, prompt_len, output_len, shares_prefix, fork_child, fork_output_len);
}

pa_status pa_sched_add_request_tokens(pa_sched* s, int64_t seq_id, const int32_t* tokens, int prompt_len,
                                      int output_len, int shares_prefix, int64_t fork_child,
                                      int fork_output_len) {
    if (!s || !s->prefix_cache || (prompt_len > 0 && !tokens)) return PA_ERR_INVALID_ARG;
    return queue_request(s, seq_id, tokens, prompt_len, output_len, shares_prefix, fork_child, fork_output_len);
}

pa_status pa_sched_enable_prefix_cache(pa_sched* s, const int32_t* prefix_tokens, int n, pa_token_fn token_fn,
                                       void* ctx) {
    if (!s || !token_fn || !s->bm->prefix_cache() || n < 0 || (n > 0 && !prefix_tokens)) return PA_ERR_INVALID_ARG;
    if (n != (s->prefix_seq >= 0 ? s->prefix_len : 0)) return PA_ERR_INVALID_ARG;
    // the holder's full blocks must be the cached blocks of these ids: then a
    // prefix-sharing admission finds them all and never takes more blocks than
    // the budget charges it
    if (s->prefix_seq >= 0 && !s->bm->cached_as(s->prefix_seq, prefix_tokens, n)) return PA_ERR_INVALID_ARG;
    if (!s->waiting.empty() || !s->running.empty() || !s->swapped.empty()) return PA_ERR_INVALID_ARG;
    s->prefix_cache = true;
    s->prefix_tokens.assign(prefix_tokens, prefix_tokens + n);
    s->token_fn = token_fn;
    s->token_ctx = ctx;
    return PA_OK;
}

pa_status pa_sched_step(pa_sched* s) { return s ? s->step() : PA_ERR_INVALID_ARG; }

pa_status pa_sched_counts_get(const pa_sched* s, pa_sched_counts* c) {
    if (!s || !c) return PA_ERR_INVALID_ARG;
    c->num_finished = (int)s->finished.size();
    c->num_admitted = (int)s->admitted.size();
    c->num_preempted = (int)s->preempted.size();
    c->num_ops = (int)s->op_kind.size();
    c->num_running = (int)s->run_ids.size();
    c->num_waiting = (int)s->waiting.size();
    return PA_OK;
}

pa_status pa_sched_record(const pa_sched* s, int64_t* finished, int64_t* admitted, int64_t* preempted,
                          int32_t* op_kind, int64_t* op_a, int64_t* op_b, int64_t* op_c,
                          int64_t* running, int32_t* context_lens) {
    if (!s) return PA_ERR_INVALID_ARG;
    auto put64 = [](int64_t* dst, const std::vector<int64_t>& src) {
        if (dst) for (size_t i = 0; i < src.size(); ++i) dst[i] = src[i];
    };
    put64(finished, s->finished);
    put64(admitted, s->admitted);
    put64(preempted, s->preempted);
    if (op_kind) for (size_t i = 0; i < s->op_kind.size(); ++i) op_kind[i] = s->op_kind[i];
    put64(op_a, s->op_a);
    put64(op_b, s->op_b);
    put64(op_c, s->op_c);
    put64(running, s->run_ids);
    if (context_lens) for (size_t i = 0; i < s->run_ctx.size(); ++i) context_lens[i] = s->run_ctx[i];
    return PA_OK;
}

}  // extern "C"
