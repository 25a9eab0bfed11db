"""GPU parity of the whole decode step (ntx_decode_step / ntx_stream_layers
through the C ABI) with the CPU oracle on the same synthetic model."""
import numpy as np
import pytest
import torch

from gpu_util import TOL, ntx_module, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ntx():
    return ntx_module()


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


@pytest.mark.parametrize("qtype", [0, 1, 2, 3], ids=["q8_0", "q4_0", "q4_k", "q6_k"])
def test_decode_step_small(ntx, syn, qtype):
    from oracle import model as om
    from synth.device_model import DeviceModel
    kw = dict(hidden=8192, ffn=8192 * 2, n_q_heads=64) if qtype == 3 else {}
    spec = small_spec(syn, qtype, **kw)
    m = DeviceModel(spec)
    token = spec.token()
    got = run_decode(ntx, m, token, spec.n_prefill)
    want, _ = om.decode(spec)
    assert rel_err(got, want) <= TOL
    # the KV rows written at pos match the oracle's fp16 rounding of k and v
    again = run_decode(ntx, m, token, spec.n_prefill)
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


@pytest.mark.slow
def test_decode_llama8b_q8_0_full(ntx, syn):
    """All 32 layers of the Llama-8B Q8_0 workload (4096 prefilled positions, token at 4096)
    against the oracle's full decode."""
    from oracle import model as om
    from synth.device_model import DeviceModel
    spec = syn.ModelSpec(**syn.LLAMA_8B_Q8_0)
    m = DeviceModel(spec)
    got = run_decode(ntx, m, spec.token(), spec.n_prefill)
    m.close()
    want, _ = om.decode(spec)
    e = rel_err(got, want)
    assert e <= TOL, e


def test_decode_llama70b_q6_k_two_layers(ntx, syn):
    """Two layers at the full Llama-70B Q6_K width and context (8192 prefilled positions)."""
    from oracle import model as om
    from synth.device_model import DeviceModel
    spec = syn.ModelSpec(**dict(syn.LLAMA_70B_Q6_K, n_layers=2))
    m = DeviceModel(spec)
    got = run_decode(ntx, m, spec.token(), spec.n_prefill)
    m.close()
    want, _ = om.decode(spec)
    assert rel_err(got, want) <= TOL
