"""Failure paths on the GPU, made to happen without faulting or hanging anything:
a bounded device-side wait that runs out (the GEMV's producer stops issuing copies,
so the consumers' wait for the next stage can never complete) and a host-side wait
of the streamed step that runs out (NTX_ETIMEOUT with the work left queued)."""
import time

import numpy as np
import pytest
import torch

from gpu_util import GEMV_TIGHT, ntx_module, rel_err

pytestmark = pytest.mark.gpu

DEVERR_FULL_WAIT = 1


@pytest.fixture(scope="module")
def ntx():
    return ntx_module()


def tiled_q8_0(ntx, syn, rows, cols, seed=3):
    qp = syn.sweep_qparams(syn.Q8_0)
    host = syn.blocks_host(syn.Q8_0, seed, 11, rows, cols, qp)
    dev = torch.from_numpy(host.reshape(-1)).cuda()
    t = torch.empty_like(dev)
    ntx.ntx_repack_q(syn.Q8_0, dev, t, rows, cols)
    torch.cuda.synchronize()
    return host, t


@pytest.mark.parametrize("stage", [0, 1])
def test_gemv_bounded_wait_runs_out_and_the_context_stays_usable(ntx, orc, syn, monkeypatch, stage):
    """With the producer stopped before stage `stage` (each CTA streams one 16-row group in
    two 4096-column stages here, so stage 1 stops it half way), every consumer warp's wait
    for that stage gives up after its poll limit: the kernel still finishes, records the
    consumer wait bit for ntx_device_error(), and the next launch on the same context is
    correct."""
    rows, cols = 32, 8192
    host, W = tiled_q8_0(ntx, syn, rows, cols)
    x = torch.from_numpy(syn.normal_f32_host(3, 12, cols)).cuda()
    y = torch.empty(rows, dtype=torch.float32, device="cuda")
    assert ntx.ntx_device_error() == 0
    monkeypatch.setenv("NTX_TEST_STALL_STAGE", str(stage))
    t0 = time.time()
    ntx.ntx_gemv_q(syn.Q8_0 | 16, W, rows, cols, x, y)
    torch.cuda.synchronize()
    elapsed = time.time() - t0
    code = ntx.ntx_device_error()
    assert code & DEVERR_FULL_WAIT, code
    assert elapsed < 60, elapsed
    monkeypatch.delenv("NTX_TEST_STALL_STAGE")
    ntx.ntx_gemv_q(syn.Q8_0 | 16, W, rows, cols, x, y)
    torch.cuda.synchronize()
    assert ntx.ntx_device_error() == 0
    assert rel_err(y.cpu().numpy(), orc.gemv(syn.Q8_0, host, rows, cols, x.cpu().numpy())) <= GEMV_TIGHT


def test_batched_gemv_bounded_wait_runs_out_and_the_pass_recovers(ntx, syn, monkeypatch):
    """The same for the batched GEMV of a verification pass (two tokens, every fused GEMV
    batched): with its producer stopped, the pass still completes and records the consumer
    wait bit; the next pass on the same context matches one launch per token bit for bit."""
    from synth.device_model import DeviceModel
    # one layer: each of its four batched GEMVs and the head waits out its poll limit once;
    # direct launches (no recorded pass), so each pass reads the test switches anew
    spec = syn.ModelSpec(n_layers=1, hidden=1024, n_q_heads=16, n_kv_heads=4, head_dim=128, ffn=2816, vocab=512,
                         max_ctx=80, n_prefill=64, qtype=syn.Q8_0, seed=2, tiled=True)
    monkeypatch.setenv("NTX_NO_GRAPH", "1")
    m = DeviceModel(spec)
    tokens = [3, 400]
    s = torch.cuda.current_stream().cuda_stream

    def verify():
        out = torch.full((2, spec.vocab), float("nan"), dtype=torch.float32, device="cuda")
        ntx.ntx_verify_tokens(m.handle, tokens, spec.n_prefill, out, s, s)
        torch.cuda.synchronize()
        return out.cpu().numpy()

    assert ntx.ntx_device_error() == 0
    monkeypatch.setenv("NTX_TEST_STALL_STAGE", "1")
    t0 = time.time()
    verify()
    assert time.time() - t0 < 120
    code = ntx.ntx_device_error()
    assert code & DEVERR_FULL_WAIT, code
    monkeypatch.delenv("NTX_TEST_STALL_STAGE")
    batched = verify()
    assert ntx.ntx_device_error() == 0
    monkeypatch.setenv("NTX_VERIFY_PER_TOKEN", "1")
    per_token = verify()
    m.close()
    assert np.array_equal(batched, per_token)


def test_stream_layers_host_wait_times_out_and_work_stays_queued(ntx, syn):
    """A 1 ms limit on a step that streams two ~480 MB layers over the host link runs out:
    NTX_ETIMEOUT, nothing lost; once the stream is synchronised the logits equal those of
    the same step run without a limit."""
    from synth.device_model import DeviceModel
    spec = syn.ModelSpec(**dict(syn.LLAMA_70B_Q4_K, n_layers=4, vocab=2000, max_ctx=600, n_prefill=512),
                         tiled=True)
    m = DeviceModel(spec, n_resident=2)
    cs, ks = torch.cuda.Stream(), torch.cuda.Stream()
    token, pos = spec.token(), spec.n_prefill
    ref = torch.empty(spec.vocab, dtype=torch.float32, device="cuda")
    ntx.ntx_stream_layers(m.handle, token, pos, ref, cs.cuda_stream, ks.cuda_stream, 0)
    torch.cuda.synchronize()
    m.reset_caches()
    torch.cuda.synchronize()
    got = torch.full((spec.vocab,), float("nan"), dtype=torch.float32, device="cuda")
    with pytest.raises(ntx.NtxError) as e:
        ntx.ntx_stream_layers(m.handle, token, pos, got, cs.cuda_stream, ks.cuda_stream, 1)
    assert e.value.status == ntx.NTX_ETIMEOUT
    torch.cuda.synchronize()
    assert ntx.ntx_device_error() == 0
    assert np.array_equal(got.cpu().numpy(), ref.cpu().numpy())
    m.close()
