// ring_mock.cpp - test harness (CPU only) for the layer-streaming ring schedule of
// libntx (csrc/ring.h): a mock transport records the operations the schedule queues and
// can fail the k-th copy; a mock query drives the bounded host wait.  Built by
// tests/test_ring_mock.py with g++; nothing here runs on a GPU.
#include <cstdint>
#include <vector>

#include "ring.h"

namespace {

// op codes in the log: (code, layer or -1, slot)
enum Op { COPY_WAIT = 1, COPY = 2, COPY_DONE = 3, COMP_WAIT = 4, COMP = 5, COMP_DONE = 6, BEFORE = 7 };

struct Mock final : ntx::ring::Ops {
    std::vector<int32_t> log;
    int copies = 0, fail_copy_at = -1, fail_compute_at = -1, computes = 0;
    void add(int op, int layer, int slot)
    {
        log.push_back(op);
        log.push_back(layer);
        log.push_back(slot);
    }
    ntx_status copy_wait_slot(int slot) override { add(COPY_WAIT, -1, slot); return NTX_OK; }
    ntx_status copy_layer(int layer, int slot) override
    {
        if (copies++ == fail_copy_at) return NTX_ECUDA;
        add(COPY, layer, slot);
        return NTX_OK;
    }
    ntx_status copy_done(int slot) override { add(COPY_DONE, -1, slot); return NTX_OK; }
    ntx_status compute_wait_copy(int slot) override { add(COMP_WAIT, -1, slot); return NTX_OK; }
    ntx_status compute_layer(int layer, int slot) override
    {
        if (computes++ == fail_compute_at) return NTX_ECUDA;
        add(COMP, layer, slot);
        return NTX_OK;
    }
    ntx_status compute_done(int slot) override { add(COMP_DONE, -1, slot); return NTX_OK; }
    ntx_status before_streamed() override { add(BEFORE, -1, -1); return NTX_OK; }
};

}  // namespace

extern "C" {

// Run the schedule over layers[0..n) with n_slots slots; fail the copy (compute) with
// index fail_copy_at (fail_compute_at), -1 for none.  The log (triples) goes to out,
// up to cap int32s; *n_out = its length.  Returns the schedule's status.
int ring_mock_run(const int32_t* layers, int n, int n_slots, int fail_copy_at, int fail_compute_at, int32_t* out,
                  int cap, int* n_out)
{
    Mock m;
    m.fail_copy_at = fail_copy_at;
    m.fail_compute_at = fail_compute_at;
    std::vector<int> ls(layers, layers + n);
    const ntx_status st = ntx::ring::schedule(m, ls.data(), n, n_slots);
    const int k = (int)m.log.size() < cap ? (int)m.log.size() : cap;
    for (int i = 0; i < k; ++i) out[i] = m.log[i];
    *n_out = (int)m.log.size();
    return st;
}

// The bounded wait over a query that reports "not yet" ready_after times, then done
// (or, with error_after >= 0, an error after that many polls).  *polls = polls made.
int ring_mock_wait(int ready_after, int error_after, int64_t timeout_ms, int* polls)
{
    int n = 0;
    const ntx_status st = ntx::ring::wait_bounded(
        [&]() -> ntx_status {
            ++n;
            if (error_after >= 0 && n > error_after) return NTX_ECUDA;
            return (ready_after >= 0 && n > ready_after) ? NTX_OK : NTX_ETIMEOUT;
        },
        timeout_ms, 100);
    *polls = n;
    return st;
}

}  // extern "C"
