"""GPU parity of the whole decode step (ntx_decode_step / ntx_stream_layers
through the C ABI) with the CPU oracle on the same synthetic model."""
import numpy as np
import pytest
import torch

from gpu_util import TOL, elem_err, ntx_module, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ntx():
    return ntx_module()


NAMES_T = {0: "q8_0_t", 1: "q4_0_t", 2: "q4_k_t", 3: "q6_k_t", 4: "q5_k_t"}


def run_decode(ntx, model, token, pos, stream_layers=False):
    s = model.spec
    logits = torch.full((s.vocab,), float("nan"), dtype=torch.float32, device="cuda")
    if stream_layers:
        cs = torch.cuda.Stream()
        ks = torch.cuda.Stream()
        ntx.ntx_stream_layers(model.handle, token, pos, logits, cs.cuda_stream, ks.cuda_stream, 600000)
    else:
        ntx.ntx_decode_step(model.handle, token, pos, logits)
    torch.cuda.synchronize()
    assert ntx.ntx_device_error() == 0
    return logits.cpu().numpy()


def small_spec(syn, qtype, **kw):
    base = dict(n_layers=3, hidden=4096, n_q_heads=32, n_kv_heads=8, head_dim=128, ffn=14336, vocab=4000,
                max_ctx=300, n_prefill=257, qtype=qtype, seed=3)
    base.update(kw)
    return syn.ModelSpec(**base)


def kv_rows_at(model, layer, pos):
    """fp16 bit patterns [2, n_kv, head_dim] of the K and V rows a step wrote at pos."""
    s = model.spec
    t = model.layers[layer]
    rows = []
    for k in ("k_cache", "v_cache"):
        c = t[k].view(s.n_kv_heads, s.max_ctx, s.head_dim)[:, pos, :]
        rows.append(c.contiguous().view(torch.int16).cpu().numpy().astype(np.int32))
    return np.stack(rows)


def assert_kv_rows_match(got_bits, want_bits):
    """The K / V rows stored at pos are the oracle's fp16 rounding of k and v: most are the
    same bit pattern, and the rest differ only where fp32 summation order moved a value
    across an fp16 rounding boundary, i.e. by no more than the 2e-3 tolerance relative to
    the largest value of the head's row (a value near zero has fp16 steps far finer than
    its absolute error, so it may be several patterns away)."""
    got = np.asarray(got_bits, dtype=np.int16).view(np.float16).astype(np.float64)
    want = np.asarray(want_bits, dtype=np.int16).view(np.float16).astype(np.float64)
    scale = np.max(np.abs(want), axis=-1, keepdims=True)
    assert np.all(np.abs(got - want) <= TOL * scale)
    assert np.mean(got_bits == want_bits) > 0.95


@pytest.mark.parametrize("qtype", [0, 1, 2, 3], ids=["q8_0", "q4_0", "q4_k", "q6_k"])
def test_decode_step_small(ntx, syn, qtype):
    from oracle import model as om
    from synth.device_model import DeviceModel
    kw = dict(hidden=8192, ffn=8192 * 2, n_q_heads=64) if qtype == 3 else {}
    spec = small_spec(syn, qtype, **kw)
    m = DeviceModel(spec)
    token, pos = spec.token(), spec.n_prefill
    got = run_decode(ntx, m, token, pos)
    kv_got = [kv_rows_at(m, l, pos) for l in range(spec.n_layers)]
    kv_want = {}

    def hook(layer, t):
        kv_want[layer] = np.stack([t["k_cache"][:, pos, :].view(np.int16).astype(np.int32),
                                   t["v_cache"][:, pos, :].view(np.int16).astype(np.int32)])

    want, _ = om.decode(spec, layer_hook=hook)
    assert rel_err(got, want) <= TOL
    assert elem_err(got, want) <= TOL
    # the K / V rows written at pos match the oracle's fp16 rounding of k and v
    for l in range(spec.n_layers):
        assert_kv_rows_match(kv_got[l], kv_want[l])
    # a second step at the same position (its own row rewritten) gives the same logits
    again = run_decode(ntx, m, token, pos)
    assert np.array_equal(got, again)
    m.close()


@pytest.mark.parametrize("qtype", [0, 1, 2, 3], ids=["q8_0_t", "q4_0_t", "q4_k_t", "q6_k_t"])
def test_decode_step_tiled(ntx, syn, qtype):
    """Weights repacked to the tiled layout: same logits as the oracle on the GGUF-style bytes."""
    from oracle import model as om
    from synth.device_model import DeviceModel
    kw = dict(hidden=8192, ffn=8192 * 2, n_q_heads=64) if qtype == 3 else {}
    spec = small_spec(syn, qtype, n_layers=2, tiled=True, **kw)
    m = DeviceModel(spec)
    got = run_decode(ntx, m, spec.token(), spec.n_prefill)
    m.close()
    want, _ = om.decode(spec)
    assert rel_err(got, want) <= TOL
    assert elem_err(got, want) <= TOL


@pytest.mark.parametrize("qtype,mix", [(4, None), (5, None), (6, None), (2, "q4_k_m")],
                         ids=["q5_k_t", "f16", "f32", "q4_k_m_t"])
def test_decode_step_further_formats(ntx, syn, qtype, mix):
    """Whole decode steps of models in the further formats (Q5_K tiled, F16, F32) and of a
    model that mixes Q4_K and Q6_K tensors, against the oracle."""
    from oracle import model as om
    from synth.device_model import DeviceModel
    spec = small_spec(syn, qtype, n_layers=2, tiled=True, mix=mix)
    m = DeviceModel(spec)
    got = run_decode(ntx, m, spec.token(), spec.n_prefill)
    m.close()
    want, _ = om.decode(spec)
    assert rel_err(got, want) <= TOL
    assert elem_err(got, want) <= TOL


def test_decode_positions_and_tokens(ntx, syn):
    """pos 0 (one key), a middle position, and a different token."""
    from oracle import model as om
    from synth.device_model import DeviceModel
    spec = small_spec(syn, 0, n_layers=2)
    m = DeviceModel(spec)
    for token, pos in ((5, 0), (17, 100), (spec.vocab - 1, spec.max_ctx - 1)):
        m.reset_caches()
        got = run_decode(ntx, m, token, pos)
        want, _ = om.decode(spec, pos=pos, token=token)
        assert rel_err(got, want) <= TOL, (token, pos)
    m.close()


def test_graph_and_direct_launches_agree(ntx, syn, monkeypatch):
    from synth.device_model import DeviceModel
    spec = small_spec(syn, 2, n_layers=2)
    a = DeviceModel(spec)
    la = run_decode(ntx, a, 7, spec.n_prefill)
    a.close()
    monkeypatch.setenv("NTX_NO_GRAPH", "1")
    monkeypatch.setenv("NTX_NO_PDL", "1")
    b = DeviceModel(spec)
    lb = run_decode(ntx, b, 7, spec.n_prefill)
    b.close()
    assert np.array_equal(la, lb)


def test_kv_prefetch_changes_nothing(ntx, syn, monkeypatch):
    """The attention launch of each layer fetches the next layer's K / V rows into L2 (a
    hint); with it turned off the step's logits are the same bits, and with it on they
    match the oracle (tiled weights, 4 layers, so three layers prefetch for the next)."""
    from oracle import model as om
    from synth.device_model import DeviceModel
    spec = small_spec(syn, 3, n_layers=4, tiled=True)
    a = DeviceModel(spec)
    la = run_decode(ntx, a, spec.token(), spec.n_prefill)
    a.close()
    monkeypatch.setenv("NTX_L2_PF", "0")
    b = DeviceModel(spec)
    lb = run_decode(ntx, b, spec.token(), spec.n_prefill)
    b.close()
    assert np.array_equal(la, lb)
    want, _ = om.decode(spec)
    assert rel_err(la, want) <= TOL
    assert elem_err(la, want) <= TOL


def test_streamed_equals_resident(ntx, syn):
    """Same kernels, same bytes: streaming layers through the HBM ring is bit-identical."""
    from synth.device_model import DeviceModel
    spec = small_spec(syn, 2, n_layers=6, hidden=8192, n_q_heads=64, ffn=28672, vocab=2000, tiled=True)
    res = DeviceModel(spec)
    lr = run_decode(ntx, res, 11, spec.n_prefill)
    res.close()
    del res
    torch.cuda.empty_cache()
    st = DeviceModel(spec, n_resident=2)
    ls = run_decode(ntx, st, 11, spec.n_prefill, stream_layers=True)
    h2d, ms = ntx.ntx_stream_stats(st.handle)
    assert h2d == 4 * spec.layer_weight_bytes() and ms > 0
    st.reset_caches()
    ls2 = run_decode(ntx, st, 11, spec.n_prefill, stream_layers=True)     # second step reuses the ring
    st.close()
    assert np.array_equal(lr, ls) and np.array_equal(ls, ls2)


def compare_full(ntx, spec, label, **model_kw):
    """Decode one step of spec on the GPU and in the oracle; print and check both metrics."""
    from oracle import model as om
    from synth.device_model import DeviceModel
    m = DeviceModel(spec, **model_kw)
    streamed = m.n_resident < m.n_layers
    got = run_decode(ntx, m, spec.token(), spec.n_prefill, stream_layers=streamed)
    m.close()
    del m
    torch.cuda.empty_cache()
    want, _ = om.decode(spec)
    e, ee = rel_err(got, want), elem_err(got, want)
    print(f"{label}: logits normwise {e:.2e} per-element {ee:.2e} argmax gpu {int(np.argmax(got))} "
          f"oracle {int(np.argmax(want))}")
    assert e <= TOL, e
    assert ee <= TOL, ee
    return got, want


@pytest.mark.slow
@pytest.mark.parametrize("tiled", [False, True], ids=["gguf", "tiled"])
def test_decode_llama8b_q8_0_full(ntx, syn, tiled):
    """All 32 layers of the Llama-8B Q8_0 workload (4096 prefilled positions, token at 4096,
    vocabulary 128256) against the oracle's full decode, in both layouts (the tiled one is
    what the benchmark runs)."""
    spec = syn.ModelSpec(**syn.LLAMA_8B_Q8_0, tiled=tiled)
    compare_full(ntx, spec, f"llama8b q8_0 {'tiled' if tiled else 'gguf'} 32 layers")


@pytest.mark.parametrize("tiled", [False, True], ids=["gguf", "tiled"])
def test_decode_llama70b_q6_k_two_layers(ntx, syn, tiled):
    """Two layers at the full Llama-70B Q6_K width, FFN, vocabulary and context (8192
    prefilled positions), in both layouts."""
    spec = syn.ModelSpec(**dict(syn.LLAMA_70B_Q6_K, n_layers=2), tiled=tiled)
    compare_full(ntx, spec, f"llama70b q6_k {'tiled' if tiled else 'gguf'} 2 layers")


@pytest.mark.slow
def test_decode_llama70b_q6_k_tiled_eight_layers(ntx, syn):
    """Eight layers of the benchmarked configuration (tiled Q6_K, 70B width, full context and
    vocabulary): the residual stream after several layers still matches the oracle."""
    spec = syn.ModelSpec(**dict(syn.LLAMA_70B_Q6_K, n_layers=8), tiled=True)
    compare_full(ntx, spec, "llama70b q6_k tiled 8 layers")


def test_streamed_llama70b_q4_k_against_oracle(ntx, syn):
    """The streamed configuration at 70B width in Q4_K (tiled, full context and vocabulary):
    two resident layers and two layers streamed from pinned host memory through the HBM
    ring, against the oracle's decode of the same four layers."""
    spec = syn.ModelSpec(**dict(syn.LLAMA_70B_Q4_K, n_layers=4), tiled=True)
    compare_full(ntx, spec, "llama70b q4_k tiled, 2 of 4 layers streamed", n_resident=2)


def test_streamed_mixed_formats_against_oracle(ntx, syn):
    """A model mixing Q4_K and Q6_K matrices (the "q4_k_m" recipe) at 70B width, two layers
    resident and two streamed: the ring's slots hold each streamed layer's own sizes."""
    spec = syn.ModelSpec(**dict(syn.LLAMA_70B_Q4_K_M, n_layers=4, vocab=4000, max_ctx=600, n_prefill=512),
                         tiled=True)
    compare_full(ntx, spec, "llama70b q4_k_m tiled, 2 of 4 layers streamed", n_resident=2)


def test_layer_skip_by_similarity(ntx, syn):
    """The layer skip: per-layer cosine similarity of the hidden state before and after
    each layer matches the oracle's; a planted near-identity layer has the highest
    similarity; skipping it gives the oracle's logits with that layer left out, and
    clearing the mask gives the full model's again."""
    from oracle import model as om
    from synth.device_model import DeviceModel
    spec = small_spec(syn, 0, n_layers=4, tiled=True, extra={"quiet_layers": [2]})
    m = DeviceModel(spec)
    token, pos = spec.token(), spec.n_prefill
    cos = ntx.ntx_model_layer_similarity(m.handle, token, pos, spec.n_layers)
    want = om.layer_similarity(spec)
    print("layer similarity gpu", [round(c, 6) for c in cos], "oracle", [round(c, 6) for c in want])
    assert np.max(np.abs(np.array(cos) - np.array(want))) <= 1e-4
    assert int(np.argmax(cos)) == 2 and cos[2] > 0.999
    m.reset_caches()
    ntx.ntx_model_set_layer_skip(m.handle, [0, 0, 1, 0])
    got = run_decode(ntx, m, token, pos)
    ref, _ = om.decode(spec, skip={2})
    assert rel_err(got, ref) <= TOL and elem_err(got, ref) <= TOL
    m.reset_caches()
    ntx.ntx_model_set_layer_skip(m.handle, None)
    full = run_decode(ntx, m, token, pos)
    m.close()
    want_full, _ = om.decode(spec)
    assert rel_err(full, want_full) <= TOL


def test_layer_skip_streamed_layers_are_not_copied(ntx, syn):
    """A skipped streamed layer is neither copied nor computed: the step copies one layer
    fewer and still matches the oracle with that layer left out."""
    from oracle import model as om
    from synth.device_model import DeviceModel
    spec = small_spec(syn, 2, n_layers=4, tiled=True, extra={"quiet_layers": [3]})
    m = DeviceModel(spec, n_resident=2)
    token, pos = spec.token(), spec.n_prefill
    cs, ks = torch.cuda.Stream(), torch.cuda.Stream()
    cos = ntx.ntx_model_layer_similarity(m.handle, token, pos, spec.n_layers, cs.cuda_stream, ks.cuda_stream)
    assert int(np.argmax(cos)) == 3
    m.reset_caches()
    torch.cuda.synchronize()
    ntx.ntx_model_set_layer_skip(m.handle, [0, 0, 0, 1])
    got = run_decode(ntx, m, token, pos, stream_layers=True)
    h2d, _ = ntx.ntx_stream_stats(m.handle)
    m.close()
    assert h2d == spec.layer_weight_bytes(2)
    ref, _ = om.decode(spec, skip={3})
    assert rel_err(got, ref) <= TOL and elem_err(got, ref) <= TOL


@pytest.mark.parametrize("register", [True, False], ids=["registered", "pageable"])
def test_streamed_from_pageable_host_memory(ntx, syn, monkeypatch, register):
    """Streamed layers in ordinary (pageable) host memory: the library page-locks them in
    place (or, with NTX_NO_HOST_REGISTER, copies from pageable memory); either way the
    logits equal those of the same model streamed from page-locked memory."""
    from synth.device_model import DeviceModel
    spec = small_spec(syn, 2, n_layers=4, tiled=True)
    pinned = DeviceModel(spec, n_resident=2)
    assert ntx.ntx_model_host_path(pinned.handle) == ntx.NTX_HOST_PATH_PINNED
    want = run_decode(ntx, pinned, spec.token(), spec.n_prefill, stream_layers=True)
    pinned.close()
    if not register:
        monkeypatch.setenv("NTX_NO_HOST_REGISTER", "1")
    m = DeviceModel(spec, n_resident=2, host_pinned=False)
    path = ntx.ntx_model_host_path(m.handle)
    assert path == (ntx.NTX_HOST_PATH_REGISTERED if register else ntx.NTX_HOST_PATH_PAGEABLE), path
    got = run_decode(ntx, m, spec.token(), spec.n_prefill, stream_layers=True)
    m.close()
    assert np.array_equal(got, want)


def test_planned_split_runs(ntx, syn):
    """A split chosen by ntx_plan_resident builds and decodes: one byte below the HBM that
    all four layers need, the planner streams some of them (a streamed layer also needs its
    share of the two-slot ring), and the step matches the oracle."""
    from oracle import model as om
    from synth.device_model import DeviceModel
    spec = small_spec(syn, 2, n_layers=4, tiled=True)
    probe = DeviceModel(spec, n_resident=4)
    n_all, full = ntx.ntx_plan_resident(probe.desc, 1 << 62)
    n, used = ntx.ntx_plan_resident(probe.desc, full - 1)
    probe.close()
    assert n_all == 4 and 0 <= n < 4 and used <= full - 1
    m = DeviceModel(spec, n_resident=n)
    got = run_decode(ntx, m, spec.token(), spec.n_prefill, stream_layers=True)
    m.close()
    want, _ = om.decode(spec)
    assert rel_err(got, want) <= TOL


@pytest.mark.parametrize("n_resident", [3, 1], ids=["resident", "streamed"])
def test_verify_tokens_against_oracle(ntx, syn, n_resident):
    """One multi-token pass over four tokens (each attending to the rows the earlier ones
    wrote) against the oracle decoding them one after another; a streamed model copies each
    streamed layer once for the whole pass."""
    from oracle import model as om
    from synth.device_model import DeviceModel
    spec = small_spec(syn, 2, n_layers=3, tiled=True, vocab=1008)
    m = DeviceModel(spec, n_resident=n_resident)
    tokens, pos0 = [17, 5, 1007, 0], spec.n_prefill
    logits = torch.full((len(tokens), spec.vocab), float("nan"), dtype=torch.float32, device="cuda")
    cs, ks = torch.cuda.Stream(), torch.cuda.Stream()
    ntx.ntx_verify_tokens(m.handle, tokens, pos0, logits, cs.cuda_stream, ks.cuda_stream)
    torch.cuda.synchronize()
    assert ntx.ntx_device_error() == 0
    if n_resident < spec.n_layers:
        h2d, _ = ntx.ntx_stream_stats(m.handle)
        assert h2d == sum(spec.layer_weight_bytes(l) for l in range(n_resident, spec.n_layers))
    m.close()
    want = om.decode_sequence(spec, tokens, pos0)
    got = logits.cpu().numpy()
    for i in range(len(tokens)):
        assert rel_err(got[i], want[i]) <= TOL, i
        assert elem_err(got[i], want[i]) <= TOL, i


VERIFY_BATCH = [(0, 4, "dp4a"), (1, 4, "dp4a"), (2, 4, "dp4a"), (3, 4, "dp4a"), (4, 4, "dp4a"), (0, 6, "dp4a"),
                (3, 3, "dp4a"), (0, 2, "dp4a"), (0, 4, "tc"), (1, 4, "tc"), (2, 4, "tc"), (3, 4, "tc"), (4, 4, "tc"),
                (3, 6, "tc")]


@pytest.mark.parametrize("qtype,k,core", VERIFY_BATCH,
                         ids=[f"{NAMES_T[q]}-{k}tokens-{c}" for q, k, c in VERIFY_BATCH])
def test_verify_pass_batches_tokens(ntx, syn, monkeypatch, qtype, k, core):
    """The verification pass runs each fused GEMV kind once for up to four tokens (every
    weight streamed once for all of them: 4 + 2 launches for six tokens; three for the
    14336-column down projection, whose four x vectors do not fit in shared memory, then
    one), on the CUDA cores (dp4a) or the integer tensor cores (tc).  Per vector the
    arithmetic is the one-token kernel's on the same cores, so with whole rows per CTA
    (every shape here is below 16384 columns) the logits equal those of one launch per
    token bit for bit, and they match the oracle."""
    from oracle import model as om
    from synth.device_model import DeviceModel
    monkeypatch.setenv("NTX_VERIFY_CORE", core)
    monkeypatch.setenv("NTX_GEMV_CORE", core)
    spec = small_spec(syn, qtype, n_layers=2, tiled=True, vocab=1008)
    tokens = [17, 5, 1007, 0, 333, 64][:k]
    pos0 = spec.n_prefill
    cs, ks = torch.cuda.Stream(), torch.cuda.Stream()

    def verify():
        # a model of its own: a resident pass is recorded as a CUDA graph on first use
        m = DeviceModel(spec)
        out = torch.full((k, spec.vocab), float("nan"), dtype=torch.float32, device="cuda")
        ntx.ntx_verify_tokens(m.handle, tokens, pos0, out, cs.cuda_stream, ks.cuda_stream)
        torch.cuda.synchronize()
        assert ntx.ntx_device_error() == 0
        again = torch.full_like(out, float("nan"))
        ntx.ntx_verify_tokens(m.handle, tokens, pos0, again, cs.cuda_stream, ks.cuda_stream)   # replayed
        torch.cuda.synchronize()
        m.close()
        assert torch.equal(out, again)
        return out.cpu().numpy()

    batched = verify()
    monkeypatch.setenv("NTX_VERIFY_PER_TOKEN", "1")
    per_token = verify()
    assert np.array_equal(batched, per_token)
    want = om.decode_sequence(spec, tokens, pos0)
    for i in range(k):
        assert rel_err(batched[i], want[i]) <= TOL, i
        assert elem_err(batched[i], want[i]) <= TOL, i


def test_verify_pass_graph_equals_direct_launches(ntx, syn, monkeypatch):
    """A resident verification pass replayed from its CUDA graph (tokens and positions read
    from the lanes' step words) gives the bits of the same pass launched directly, at a
    second set of tokens and positions too (the graph recorded once is replayed)."""
    from synth.device_model import DeviceModel
    spec = small_spec(syn, 0, n_layers=2, tiled=True, vocab=1008)
    cs, ks = torch.cuda.Stream(), torch.cuda.Stream()

    def passes(m):
        outs = []
        for tokens, pos0 in (([17, 5, 1007], spec.n_prefill), ([2, 900, 44], spec.n_prefill - 20)):
            out = torch.full((3, spec.vocab), float("nan"), dtype=torch.float32, device="cuda")
            ntx.ntx_verify_tokens(m.handle, tokens, pos0, out, cs.cuda_stream, ks.cuda_stream)
            torch.cuda.synchronize()
            outs.append(out.cpu().numpy())
        return outs

    g = DeviceModel(spec)
    graphed = passes(g)
    g.close()
    monkeypatch.setenv("NTX_NO_GRAPH", "1")
    dm = DeviceModel(spec)
    direct = passes(dm)
    dm.close()
    for a, b in zip(graphed, direct):
        assert np.array_equal(a, b)
    assert not np.array_equal(graphed[0], graphed[1])


def greedy(ntx, m, token, pos, n, streamed):
    """n tokens of plain greedy decoding from (token, pos), one step each."""
    out = []
    for i in range(n):
        logits = run_decode(ntx, m, token, pos + i, stream_layers=streamed)
        token = int(np.argmax(logits))
        out.append(token)
    return out


@pytest.mark.parametrize("case", ["same-model", "quiet-layer-skipped", "streamed"])
def test_speculative_decoding_equals_greedy(ntx, syn, case):
    """Self-speculative decoding gives exactly the tokens of greedy decoding of the full
    model: with a draft identical to the model every drafted token is accepted; with a draft
    that leaves out a near-identity layer, or the streamed layers, some may be rejected, and
    the output is still the greedy sequence."""
    from synth.device_model import DeviceModel
    extra = {"quiet_layers": [1]} if case == "quiet-layer-skipped" else {}
    spec = small_spec(syn, 2, n_layers=3, tiled=True, vocab=1008, max_ctx=320, extra=extra)
    streamed = case == "streamed"
    m = DeviceModel(spec, n_resident=1 if streamed else None)
    token, pos, n_want, k = spec.token(), spec.n_prefill, 9, 4
    want = greedy(ntx, m, token, pos, n_want, streamed)
    m.reset_caches()
    torch.cuda.synchronize()
    cs, ks = torch.cuda.Stream(), torch.cuda.Stream()
    draft_skip = [0, 1, 0] if case == "quiet-layer-skipped" else None
    got, counts, t, p = [], [], token, pos
    while len(got) < n_want:
        out = ntx.ntx_speculative_step(m.handle, t, p, k, draft_skip, cs.cuda_stream, ks.cuda_stream)
        assert 1 <= len(out) <= k
        counts.append(len(out))
        got += out
        t, p = out[-1], p + len(out)
    m.close()
    print(f"speculative {case}: tokens per pass {counts}")
    assert got[:n_want] == want
    if case == "same-model":
        assert all(c == k for c in counts)
