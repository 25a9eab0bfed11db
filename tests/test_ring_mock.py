"""The layer-streaming ring's schedule and bounded host wait, on the CPU: the schedule
(quantized_weight_gemv_block_b200/csrc/ring.h, the same header ntx_stream_layers runs)
is driven through a mock transport that records every queued operation and can fail
the k-th copy or compute; a simulation of the two queues checks that no layer is
computed before its copy lands and no slot is refilled before its compute finished."""
import ctypes
import os
import subprocess

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(ROOT, "quantized_weight_gemv_block_b200", "csrc")
SRC = os.path.join(HERE, "native", "ring_mock.cpp")
LIB = os.path.join(HERE, "native", "_build", "libring_mock.so")

NTX_OK, NTX_EINVAL, NTX_ECUDA, NTX_ETIMEOUT = 0, 1, 4, 5
COPY_WAIT, COPY, COPY_DONE, COMP_WAIT, COMP, COMP_DONE, BEFORE = 1, 2, 3, 4, 5, 6, 7


@pytest.fixture(scope="module")
def mock():
    os.makedirs(os.path.dirname(LIB), exist_ok=True)
    deps = [SRC, os.path.join(CSRC, "ring.h")]
    if not os.path.exists(LIB) or os.path.getmtime(LIB) < max(os.path.getmtime(p) for p in deps):
        subprocess.check_call(["g++", "-std=c++17", "-O1", "-fPIC", "-shared", "-Wall", "-I", CSRC, "-I",
                               os.path.join(ROOT, "include"), "-o", LIB, SRC])
    L = ctypes.CDLL(LIB)
    L.ring_mock_run.argtypes = [ctypes.POINTER(ctypes.c_int32), ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                ctypes.c_int, ctypes.POINTER(ctypes.c_int32), ctypes.c_int, ctypes.POINTER(ctypes.c_int)]
    L.ring_mock_wait.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.POINTER(ctypes.c_int)]
    return L


def run(mock, layers, n_slots=2, fail_copy=-1, fail_compute=-1):
    arr = (ctypes.c_int32 * max(1, len(layers)))(*layers)
    cap = 3 * (8 * len(layers) + 8)
    out = (ctypes.c_int32 * cap)()
    n = ctypes.c_int(0)
    st = mock.ring_mock_run(arr, len(layers), n_slots, fail_copy, fail_compute, out, cap, ctypes.byref(n))
    log = np.array(out[:n.value], dtype=np.int64).reshape(-1, 3)
    return st, [tuple(int(v) for v in r) for r in log]


def simulate(log, n_slots):
    """Execute the logged operations as two in-order queues (copy, compute) joined by
    events, as CUDA runs them: a wait on a slot's fill (release) event waits for the
    fills (releases) of that slot recorded before the wait was queued.  Checks the data
    flow: every compute reads a slot that holds its own layer's copy, and no copy writes
    a slot whose previous layer has not been computed.  Returns the computed layers."""
    recorded = {COPY_DONE: {}, COMP_DONE: {}}
    ops = []
    for op, layer, slot in log:
        target = 0
        if op == COPY_WAIT:
            target = recorded[COMP_DONE].get(slot, 0)
        elif op == COMP_WAIT:
            target = recorded[COPY_DONE].get(slot, 0)
        elif op in (COPY_DONE, COMP_DONE):
            recorded[op][slot] = recorded[op].get(slot, 0) + 1
        ops.append((op, layer, slot, target))
    copy_q = [o for o in ops if o[0] in (COPY_WAIT, COPY, COPY_DONE)]
    comp_q = [o for o in ops if o[0] in (COMP_WAIT, COMP, COMP_DONE, BEFORE)]
    fills, releases, slot_layer, pending, computed = {}, {}, {}, {}, []
    ci = ki = 0
    while ci < len(copy_q) or ki < len(comp_q):
        progressed = False
        if ci < len(copy_q):
            op, layer, slot, target = copy_q[ci]
            if op != COPY_WAIT or releases.get(slot, 0) >= target:
                if op == COPY:
                    assert fills.get(slot, 0) == releases.get(slot, 0), ("slot refilled before release", slot)
                    pending[slot] = layer
                elif op == COPY_DONE:
                    slot_layer[slot] = pending.pop(slot)
                    fills[slot] = fills.get(slot, 0) + 1
                ci += 1
                progressed = True
        if ki < len(comp_q):
            op, layer, slot, target = comp_q[ki]
            if op != COMP_WAIT or fills.get(slot, 0) >= target:
                if op == COMP:
                    assert slot_layer.get(slot) == layer, ("compute reads another layer's copy", layer, slot)
                    computed.append(layer)
                elif op == COMP_DONE:
                    releases[slot] = releases.get(slot, 0) + 1
                ki += 1
                progressed = True
        assert progressed, "the two queues wait on each other"
    return computed


@pytest.mark.parametrize("layers", [[], [36], [36, 37], list(range(36, 80)), [3, 5, 6, 9, 12]])
@pytest.mark.parametrize("n_slots", [1, 2, 3])
def test_schedule_order_and_data_flow(mock, layers, n_slots):
    st, log = run(mock, layers, n_slots)
    assert st == NTX_OK
    assert [op[1] for op in log if op[0] == COPY] == layers          # each streamed layer copied once, in order
    assert simulate(log, n_slots) == layers                           # each computed once, in order, after its copy
    before = [i for i, op in enumerate(log) if op[0] == BEFORE]
    assert len(before) == 1
    first_copies = [i for i, op in enumerate(log) if op[0] == COPY][:n_slots]
    assert all(i < before[0] for i in first_copies)                   # the first copies overlap the resident layers
    # copies run at most n_slots layers ahead of compute
    n_copied = n_computed = 0
    for op in log:
        n_copied += op[0] == COPY
        n_computed += op[0] == COMP
        assert n_copied - n_computed <= n_slots


@pytest.mark.parametrize("k", [0, 1, 2, 5, 43])
def test_failed_copy_stops_the_schedule(mock, k):
    """A copy that fails (as a cudaMemcpyAsync would) ends the schedule with its status;
    nothing is queued after it and no layer is computed whose copy was not queued."""
    layers = list(range(36, 80))
    st, log = run(mock, layers, 2, fail_copy=k)
    assert st == NTX_ECUDA
    copied = [op[1] for op in log if op[0] == COPY]
    computed = [op[1] for op in log if op[0] == COMP]
    assert copied == layers[:k]
    assert set(computed) <= set(copied)
    # the failed copy is the last operation attempted: nothing after it
    assert log[-1][0] == COPY_WAIT and log[-1][2] == k % 2


def test_failed_compute_stops_the_schedule(mock):
    st, log = run(mock, list(range(10)), 2, fail_compute=3)
    assert st == NTX_ECUDA
    assert [op[1] for op in log if op[0] == COMP] == [0, 1, 2]
    assert log[-1][0] == COMP_WAIT


def test_bad_slot_count_is_rejected(mock):
    st, log = run(mock, [1, 2], 0)
    assert st == NTX_EINVAL and log == []


def test_bounded_wait(mock):
    polls = ctypes.c_int(0)
    # done after a few polls
    assert mock.ring_mock_wait(3, -1, 10000, ctypes.byref(polls)) == NTX_OK and polls.value == 4
    # a step that never finishes (a stalled copy): the wait gives up after its limit
    assert mock.ring_mock_wait(-1, -1, 20, ctypes.byref(polls)) == NTX_ETIMEOUT and polls.value > 1
    # an error reported while waiting is returned as it is
    assert mock.ring_mock_wait(-1, 2, 10000, ctypes.byref(polls)) == NTX_ECUDA and polls.value == 3
