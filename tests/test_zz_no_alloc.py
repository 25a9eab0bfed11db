"""The allocation-free attention entry point (ntx_attn_decode_noalloc), for
callers that have no device memory to hand over as a workspace.

Checked through the C ABI against the allocating entry point on the same
inputs, for two calls in a row with different inputs and context lengths (the
shared scratch keeps the previous call's partials, and the second call must not
be affected by them: every split's partial is rewritten before the merge reads
it), and for the size limit of the fixed scratch.  Collected last on purpose: it
must pass in a fresh process and after every other test."""
import numpy as np
import pytest
import torch

from gpu_util import ntx_module, rel_err

pytestmark = pytest.mark.gpu

ATTN_TOL = 1e-4     # the tolerance the attention parity tests use


@pytest.fixture(scope="module")
def ntx():
    return ntx_module()


def _inputs(syn, seed, nq, nkv, max_ctx):
    hd = 128
    q = torch.from_numpy(syn.normal_f32_host(seed, 1, nq * hd)).cuda()
    kc = torch.from_numpy(syn.normal_f16_host(seed, 2, nkv * max_ctx * hd).view(np.float16)).cuda()
    vc = torch.from_numpy(syn.normal_f16_host(seed, 3, nkv * max_ctx * hd).view(np.float16)).cuda()
    return q, kc, vc


@pytest.mark.parametrize("nq,nkv,n_ctx,max_ctx", [(32, 8, 4097, 4097), (8, 8, 700, 1000)])
def test_noalloc_matches_workspace_entry_point_twice(ntx, syn, nq, nkv, n_ctx, max_ctx):
    hd = 128
    for call, seed in enumerate((21, 22)):
        q, kc, vc = _inputs(syn, seed, nq, nkv, max_ctx)
        ctx = n_ctx - call                      # a different context length on the second call
        want = torch.empty(nq * hd, dtype=torch.float32, device="cuda")
        wsb = ntx.ntx_attn_workspace_bytes(nq, nkv, hd, max_ctx)
        ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
        ntx.ntx_attn_decode(q, kc, vc, want, nq, nkv, hd, ctx, max_ctx, ws, wsb)
        got = torch.full((nq * hd,), float("nan"), dtype=torch.float32, device="cuda")
        ntx.ntx_attn_decode_noalloc(q, kc, vc, got, nq, nkv, hd, ctx, max_ctx)
        torch.cuda.synchronize()
        assert rel_err(got.cpu().numpy(), want.cpu().numpy()) <= ATTN_TOL, call
        assert ntx.ntx_device_error() == 0


def test_noalloc_rejects_shapes_beyond_its_scratch(ntx):
    # 64 q heads over 8 kv heads needs more scratch than the fixed 512 KiB
    assert ntx.ntx_attn_workspace_bytes(64, 8, 128, 8193) > 512 * 1024
    p = torch.empty(1 << 20, dtype=torch.float32, device="cuda")
    with pytest.raises(ntx.NtxError) as e:
        ntx.ntx_attn_decode_noalloc(p, p, p, p, 64, 8, 128, 10, 8193)
    assert e.value.status == ntx.NTX_EUNSUPPORTED and "512 KiB" in str(e.value)
