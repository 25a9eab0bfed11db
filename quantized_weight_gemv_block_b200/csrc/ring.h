// ring.h - the schedule of the layer-streaming ring and the host's bounded wait, in
// plain C++ (no CUDA), so the order of operations can be checked on its own.
//
// The streamed layers ("Streaming SLEP" of the ntransformer news summary, "Funciones
// principales": host read, host-to-GPU copy and compute overlapped with double
// buffering) go through a ring of n_slots HBM slots.  Two queues run side by side:
// the copy queue fills slot i % n_slots with streamed layer i once the compute of
// layer i - n_slots (the slot's previous user) has been queued as finished; the
// compute queue runs layer i once its copy has landed.  Copies run n_slots layers
// ahead of compute.
#pragma once

#include <chrono>
#include <thread>

#include "ntx.h"

namespace ntx {
namespace ring {

// The operations the schedule queues; an implementation puts them on two streams
// (copy, compute) with events between them, or records them (tests).
struct Ops {
    virtual ~Ops() = default;
    virtual ntx_status copy_wait_slot(int slot) = 0;          // copy queue: wait until slot is released
    virtual ntx_status copy_layer(int layer, int slot) = 0;   // copy queue: the layer's matrices into slot
    virtual ntx_status copy_done(int slot) = 0;               // copy queue: mark the slot filled
    virtual ntx_status compute_wait_copy(int slot) = 0;       // compute queue: wait until slot is filled
    virtual ntx_status compute_layer(int layer, int slot) = 0;
    virtual ntx_status compute_done(int slot) = 0;            // compute queue: mark the slot released
    // compute queue, once, after the first copies are queued and before the first streamed
    // layer: the work that precedes the streamed layers (the resident layers)
    virtual ntx_status before_streamed() = 0;
};

// Queue streamed layers layers[0..n) in order through n_slots slots: the first n_slots
// copies, then before_streamed(), then per layer its compute and the copy n_slots
// ahead.  Stops at the first operation that fails and returns its status; nothing is
// queued after it (in particular no layer is computed whose copy was not queued).
inline ntx_status schedule(Ops& ops, const int* layers, int n, int n_slots)
{
    if (n_slots < 1 || n < 0) return NTX_EINVAL;
    ntx_status st = NTX_OK;
    auto copy = [&](int i) -> ntx_status {
        const int slot = i % n_slots;
        if ((st = ops.copy_wait_slot(slot)) != NTX_OK) return st;
        if ((st = ops.copy_layer(layers[i], slot)) != NTX_OK) return st;
        return ops.copy_done(slot);
    };
    for (int i = 0; i < n && i < n_slots; ++i)
        if ((st = copy(i)) != NTX_OK) return st;
    if ((st = ops.before_streamed()) != NTX_OK) return st;
    for (int i = 0; i < n; ++i) {
        const int slot = i % n_slots;
        if ((st = ops.compute_wait_copy(slot)) != NTX_OK) return st;
        if ((st = ops.compute_layer(layers[i], slot)) != NTX_OK) return st;
        if ((st = ops.compute_done(slot)) != NTX_OK) return st;
        if (i + n_slots < n)
            if ((st = copy(i + n_slots)) != NTX_OK) return st;
    }
    return NTX_OK;
}

// Poll `query` (NTX_OK: done, NTX_ETIMEOUT: not yet, anything else: an error, returned
// as it is) until it reports done or `timeout_ms` has passed (NTX_ETIMEOUT), sleeping
// `poll_us` between polls.
template <typename Query>
ntx_status wait_bounded(Query query, int64_t timeout_ms, int poll_us = 200)
{
    const auto deadline = std::chrono::steady_clock::now() + std::chrono::milliseconds(timeout_ms);
    for (;;) {
        const ntx_status q = query();
        if (q != NTX_ETIMEOUT) return q;
        if (std::chrono::steady_clock::now() > deadline) return NTX_ETIMEOUT;
        std::this_thread::sleep_for(std::chrono::microseconds(poll_us));
    }
}

}  // namespace ring
}  // namespace ntx
