// Iteration-level scheduling simulated on the block allocator.
//
// Follows "PagedAttention in vLLM: a throughput settings guide", section
// "Continuous Batching Keeps the GPU Busy" (the scheduler looks at the batch
// every decoding step, admits a waiting request or retires a finished one
// without waiting for the others; max_num_seqs caps concurrency; too many
// sequences for the KV budget cause preemption, where a request is evicted
// and later recomputed), and "Inside vLLM: How PagedAttention Changes Python
// LLM Inference at the Systems Level", section "Python LLM Inference
// Optimization with vLLM: Parameters That Actually Matter" (under memory
// pressure a sequence can be recomputed from scratch; recomputation is the
// default) and section "Tuning in Practice: Where to Start" (the two numbers
// to watch: KV cache usage and the preemption count).
// The interface is documented in include/pa_alloc.h.
#include <algorithm>
#include <cstdint>
#include <deque>
#include <vector>

#include "pa_alloc.h"
#include "pa_api.h"

extern "C" int pa_sim_continuous_batching(int32_t num_blocks, int32_t block_size,
                                          int32_t max_num_seqs, const int32_t *prompt_lens,
                                          const int32_t *output_lens, int32_t num_requests,
                                          int64_t max_steps, pa_sim_stats *out) {
    if (num_blocks <= 0 || block_size <= 0 || max_num_seqs <= 0 || num_requests < 0 ||
        (num_requests > 0 && (!prompt_lens || !output_lens)) || !out || max_steps <= 0)
        return PA_ERR_INVALID_ARG;
    for (int32_t r = 0; r < num_requests; ++r)
        if (prompt_lens[r] < 0 || output_lens[r] < 1) return PA_ERR_INVALID_ARG;
    pa_alloc *a = pa_alloc_create(num_blocks, block_size);
    if (!a) return PA_ERR_INVALID_ARG;

    pa_sim_stats st = {};
    std::vector<int32_t> generated(num_requests, 0);
    std::deque<int32_t> waiting;
    std::vector<int32_t> running;  // in admission order
    for (int32_t r = 0; r < num_requests; ++r) {
        // a request whose whole life cannot fit in the pool would cycle forever
        const int64_t need = ((int64_t)prompt_lens[r] + output_lens[r] + block_size - 1) / block_size;
        if (need > num_blocks)
            ++st.rejected;
        else
            waiting.push_back(r);
    }
    double usage_sum = 0.0, running_sum = 0.0;
    while ((!waiting.empty() || !running.empty()) && st.steps < max_steps) {
        // 1. admit: prefill prompt + tokens generated before any preemption
        while (!waiting.empty() && (int32_t)running.size() < max_num_seqs) {
            const int32_t r = waiting.front();
            if (pa_alloc_add_seq(a, r, prompt_lens[r] + generated[r]) != PA_OK) break;
            waiting.pop_front();
            running.push_back(r);
            ++st.admitted;
        }
        // 2. one decode step for every running sequence
        std::vector<int32_t> next;
        next.reserve(running.size());
        std::vector<char> evicted(num_requests, 0);
        for (size_t i = 0; i < running.size(); ++i) {
            const int32_t r = running[i];
            if (evicted[r]) continue;
            int64_t slot;
            int32_t src, dst;
            int rc = pa_alloc_append_slot(a, r, &slot, &src, &dst);
            while (rc == PA_ERR_NO_BLOCKS) {
                // evict the latest-admitted sequence still holding blocks
                int32_t victim = -1;
                for (size_t j = running.size(); j-- > 0;)
                    if (!evicted[running[j]]) {
                        victim = running[j];
                        break;
                    }
                pa_alloc_free_seq(a, victim);
                evicted[victim] = 1;
                ++st.preemptions;
                if (victim == r) break;
                rc = pa_alloc_append_slot(a, r, &slot, &src, &dst);
            }
            if (evicted[r]) continue;
            ++generated[r];
            ++st.tokens_generated;
            if (generated[r] == output_lens[r]) {
                pa_alloc_free_seq(a, r);
                ++st.finished;
            } else {
                next.push_back(r);
            }
        }
        // preempted sequences go back to the front of the queue, oldest first
        for (size_t j = running.size(); j-- > 0;)
            if (evicted[running[j]]) waiting.push_front(running[j]);
        running.swap(next);
        pa_alloc_stats as;
        pa_alloc_get_stats(a, &as);
        usage_sum += as.usage;
        running_sum += (double)running.size();
        if (as.usage > st.max_usage) st.max_usage = as.usage;
        ++st.steps;
    }
    st.mean_usage = st.steps ? usage_sum / (double)st.steps : 0.0;
    st.mean_running = st.steps ? running_sum / (double)st.steps : 0.0;
    pa_alloc_destroy(a);
    *out = st;
    return PA_OK;
}
