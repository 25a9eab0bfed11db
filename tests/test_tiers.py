"""Automatic tier split (ntx_plan_resident) on the CPU: the planner reads only shapes and
formats, so a planning descriptor with null pointers is enough.  Its byte accounting is
checked against layer sizes computed here from the block layouts."""
import ctypes

import pytest


@pytest.fixture(scope="module")
def ntx():
    from quantized_weight_gemv_block_b200 import build
    build.build()
    import quantized_weight_gemv_block_b200 as ntx
    ntx.lib()
    return ntx


def desc_for(ntx, spec, n_layers=None, qts=None):
    n = spec.n_layers if n_layers is None else n_layers
    d = ntx.ModelDesc(n, spec.hidden, spec.n_q_heads, spec.n_kv_heads, spec.head_dim, spec.ffn, spec.vocab,
                      spec.max_ctx, spec.rms_eps, spec.rope_theta, spec.lib_code(spec.qtype), None, None, None,
                      None, n, None)
    if qts is not None:
        arr = (ctypes.c_int32 * len(qts))(*qts)
        d.tensor_qtypes = ctypes.cast(arr, ctypes.POINTER(ctypes.c_int32))
        d._keep = arr
    return d


def layer_parts(syn, spec, layer):
    """Bytes of the QKV, O, gate, up and down matrices of one layer, each rounded up to 256."""
    q = lambda k: spec.qtype_of(k, layer)
    h, f, qd = spec.hidden, spec.ffn, spec.q_dim
    parts = [spec.qkv_rows * syn.row_bytes(q("w_qkv"), h), h * syn.row_bytes(q("w_o"), qd),
             f * syn.row_bytes(q("w_gate"), h), f * syn.row_bytes(q("w_up"), h), h * syn.row_bytes(q("w_down"), f)]
    return [(p + 255) // 256 * 256 for p in parts]


def layer_bytes(syn, spec, layer):
    """The five packed matrices of one layer, from the row sizes of the block layouts."""
    q = lambda k: spec.qtype_of(k, layer)
    h, f, qd = spec.hidden, spec.ffn, spec.q_dim
    return (spec.qkv_rows * syn.row_bytes(q("w_qkv"), h) + h * syn.row_bytes(q("w_o"), qd)
            + 2 * f * syn.row_bytes(q("w_gate"), h) + h * syn.row_bytes(q("w_down"), f))


@pytest.mark.parametrize("mix", [None, "q4_k_m"])
def test_plan_resident_70b(ntx, syn, mix):
    spec = syn.ModelSpec(**dict(syn.LLAMA_70B_Q4_K, mix=mix), tiled=True)
    d = desc_for(ntx, spec, qts=spec.tensor_qtypes())
    L = spec.n_layers
    # HBM used with n resident layers, from budgets at the planner's own thresholds
    n_all, used_all = ntx.ntx_plan_resident(d, 1 << 62)
    assert n_all == L
    used = {}
    for n in (0, 1, 2, 35, 36, 37):
        # the smallest budget that admits n layers is found by bisection on the planner
        lo, hi = 0, used_all * 2
        while lo < hi:
            mid = (lo + hi) // 2
            try:
                got, _ = ntx.ntx_plan_resident(d, mid)
            except ntx.NtxError:
                got = -1
            if got >= n:
                hi = mid
            else:
                lo = mid + 1
        got, u = ntx.ntx_plan_resident(d, lo)
        assert got == n and u == lo, (n, got, u, lo)
        used[n] = u
    # each further resident layer costs exactly its matrices while the ring stays (the ring
    # holds the largest streamed matrices, which for these models does not change)
    for n in (0, 1, 35, 36):
        assert used[n + 1] - used[n] == layer_bytes(syn, spec, n), n
    # with every layer resident the ring (two slots of the largest streamed matrices)
    # disappears, so all 80 layers need less HBM than 79 plus the ring: the planner takes
    # all of them as soon as they fit
    ring = used[0] - (used_all - sum(layer_bytes(syn, spec, l) for l in range(L)))
    assert ring == 2 * sum(max(x) for x in zip(*[layer_parts(syn, spec, l) for l in range(L)]))
    assert ntx.ntx_plan_resident(d, used_all)[0] == L
    # too little HBM for even the fixed part
    with pytest.raises(ntx.NtxError) as e:
        ntx.ntx_plan_resident(d, used[0] - 1)
    assert e.value.status == ntx.NTX_ENOMEM


def test_plan_resident_matches_the_pages_split(ntx, syn):
    """The pages keep 36 of the 80 layers of the 70B Q4_K model in VRAM: with the HBM the
    planner reports for 36 layers, it chooses 36, and one byte less gives 35."""
    spec = syn.ModelSpec(**syn.LLAMA_70B_Q4_K, tiled=True)
    d = desc_for(ntx, spec)
    _, used80 = ntx.ntx_plan_resident(d, 1 << 62)
    # find the threshold of 36 by scanning the planner's answers on a coarse grid
    lo, hi = 0, used80
    while lo < hi:
        mid = (lo + hi) // 2
        try:
            n, _ = ntx.ntx_plan_resident(d, mid)
        except ntx.NtxError:
            n = -1
        if n >= 36:
            hi = mid
        else:
            lo = mid + 1
    assert ntx.ntx_plan_resident(d, lo)[0] == 36
    assert ntx.ntx_plan_resident(d, lo - 1)[0] == 35


def test_plan_rejects_bad_shapes(ntx, syn):
    spec = syn.ModelSpec(**syn.LLAMA_70B_Q4_K, tiled=True)
    d = desc_for(ntx, spec)
    d.head_dim = 64
    with pytest.raises(ntx.NtxError):
        ntx.ntx_plan_resident(d, 1 << 40)
