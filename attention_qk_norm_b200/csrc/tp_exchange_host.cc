// tp_exchange_host.cc -- the exchange protocol of tensor-parallel layerwise
// QK-Norm (tp_exchange.h) run on host threads, for tests with one process per
// rank on a host without a GPU.  The receive buffers are then shared host
// memory; a store is an atomic 64-bit relaxed store and a poll an atomic
// relaxed load, as the kernel's st/ld.relaxed.sys are.
//
// qkn_tp_host_rank_call plays one rank's kernel launch for one call: `blocks`
// threads take tokens b, b + blocks, ... in order; for each token a thread
// stores the rank's two sums into its slot of every rank's buffer, then polls
// its own buffer until every rank's words carry the call's tag (or the time
// limit passes, after which this call waits no more on this rank), and
// combines the world sums with the kernel's fixed rank tree.  It returns the
// number of waits that gave up.  This file is built only for the tests; the
// library proper does not contain it.
#include <stdint.h>

#include <atomic>
#include <chrono>
#include <thread>
#include <vector>

#include "tp_exchange.h"

namespace {

uint64_t load_relaxed(const uint64_t *p) { return __atomic_load_n(p, __ATOMIC_RELAXED); }
void store_relaxed(uint64_t *p, uint64_t v) { __atomic_store_n(p, v, __ATOMIC_RELAXED); }

}  // namespace

extern "C" int qkn_tp_host_rank_call(uint64_t *const *recv, int world, int rank,
                                     int64_t max_tokens, uint64_t call, int64_t T, int blocks,
                                     const float *sum_q, const float *sum_k, float *out_q,
                                     float *out_k, double timeout_s, int64_t skew_every,
                                     double skew_s)
{
    if (world < 1 || world > qkn_tp::kMaxWorld || rank < 0 || rank >= world || blocks < 1 ||
        T > max_tokens)
        return -1;
    const uint32_t parity = qkn_tp::call_parity((uint32_t)call), tag = qkn_tp::call_tag((uint32_t)call);
    std::atomic<bool> abort_call{false};
    std::atomic<int> gave_up_total{0};
    auto block = [&](int b) {
        bool gave_up = false;
        for (int64_t t = b; t < T; t += blocks) {
            if (skew_every > 0 && t % skew_every == 0)
                std::this_thread::sleep_for(std::chrono::duration<double>(skew_s));
            for (int r = 0; r < world; ++r) {
                uint64_t *dst = recv[r] + qkn_tp::slot_word(parity, t, rank, 0, max_tokens, world);
                store_relaxed(dst, qkn_tp::pack(sum_q[t], tag));
                store_relaxed(dst + 1, qkn_tp::pack(sum_k[t], tag));
            }
            float vq[qkn_tp::kMaxWorld], vk[qkn_tp::kMaxWorld];
            for (int src = 0; src < world; ++src) {
                const uint64_t *p =
                    recv[rank] + qkn_tp::slot_word(parity, t, src, 0, max_tokens, world);
                uint64_t wq = load_relaxed(p), wk = load_relaxed(p + 1);
                if (!gave_up && !(qkn_tp::arrived(wq, tag) && qkn_tp::arrived(wk, tag))) {
                    const auto t0 = std::chrono::steady_clock::now();
                    for (;;) {
                        wq = load_relaxed(p);
                        wk = load_relaxed(p + 1);
                        if (qkn_tp::arrived(wq, tag) && qkn_tp::arrived(wk, tag)) break;
                        const double waited = std::chrono::duration<double>(
                                                  std::chrono::steady_clock::now() - t0)
                                                  .count();
                        if (waited > timeout_s || abort_call.load(std::memory_order_relaxed)) {
                            gave_up = true;
                            gave_up_total.fetch_add(1);
                            abort_call.store(true, std::memory_order_relaxed);
                            break;
                        }
                        std::this_thread::yield();
                    }
                }
                vq[src] = qkn_tp::value_of(wq);
                vk[src] = qkn_tp::value_of(wk);
            }
            out_q[t] = qkn_tp::combine_ranks_host(vq, world);
            out_k[t] = qkn_tp::combine_ranks_host(vk, world);
        }
    };
    std::vector<std::thread> threads;
    for (int b = 0; b < blocks; ++b) threads.emplace_back(block, b);
    for (auto &th : threads) th.join();
    return gave_up_total.load();
}

extern "C" uint64_t qkn_tp_host_buffer_words(int64_t max_tokens, int world)
{
    return qkn_tp::buffer_words(max_tokens, world);
}
