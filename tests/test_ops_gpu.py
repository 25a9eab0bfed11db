"""GPU parity of the decode ops (through the C ABI) with the CPU oracle."""
import numpy as np
import pytest
import torch

from gpu_util import TOL, ntx_module, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ntx():
    return ntx_module()


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


@pytest.mark.parametrize("n", [1, 1000, 4096, 8192, 128256])
def test_rmsnorm(ntx, orc, syn, n):
    x = syn.normal_f32_host(1, 1, n) * np.float32(3.0)
    w = syn.uniform_f32_host(1, 2, n, *syn.NORM_W)
    y = torch.empty(n, dtype=torch.float32, device="cuda")
    ntx.ntx_rmsnorm(dev(x), dev(w), y, n, 1e-5)
    torch.cuda.synchronize()
    assert rel_err(y.cpu().numpy(), orc.rmsnorm(x, w, 1e-5)) <= 1e-5


@pytest.mark.parametrize("pos", [0, 1, 4096, 8192])
def test_rope(ntx, orc, syn, pos):
    nq, nkv, hd = 32, 8, 128
    q = syn.normal_f32_host(2, 1, nq * hd)
    k = syn.normal_f32_host(2, 2, nkv * hd)
    qd, kd = dev(q), dev(k)
    ntx.ntx_rope(qd, kd, nq, nkv, hd, pos, 5e5)
    torch.cuda.synchronize()
    qo, ko = orc.rope(q, k, nq, nkv, hd, pos, 5e5)
    assert rel_err(qd.cpu().numpy(), qo) <= 1e-5 and rel_err(kd.cpu().numpy(), ko) <= 1e-5


def test_rope_without_k(ntx, orc, syn):
    q = syn.normal_f32_host(2, 3, 4 * 128)
    qd = dev(q)
    ntx.ntx_rope(qd, None, 4, 0, 128, 77, 1e4)
    torch.cuda.synchronize()
    qo, _ = orc.rope(q, np.zeros(128, dtype=np.float32), 4, 0, 128, 77, 1e4)
    assert rel_err(qd.cpu().numpy(), qo) <= 1e-5


@pytest.mark.parametrize("n", [1, 14336, 28672])
def test_swiglu(ntx, orc, syn, n):
    g = syn.normal_f32_host(3, 1, n) * np.float32(2)
    u = syn.normal_f32_host(3, 2, n)
    out = torch.empty(n, dtype=torch.float32, device="cuda")
    ntx.ntx_swiglu(dev(g), dev(u), out, n)
    torch.cuda.synchronize()
    assert rel_err(out.cpu().numpy(), orc.swiglu(g, u)) <= 1e-5


@pytest.mark.parametrize("n", [1, 7, 128256])
def test_softmax_and_argmax(ntx, orc, syn, n):
    x = syn.normal_f32_host(4, 1, n) * np.float32(4)
    y = torch.empty(n, dtype=torch.float32, device="cuda")
    xd = dev(x)
    ntx.ntx_softmax(xd, y, n)
    idx = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    ntx.ntx_argmax(xd, n, idx)
    torch.cuda.synchronize()
    yo = orc.softmax(x)
    assert rel_err(y.cpu().numpy(), yo) <= 1e-5
    assert abs(float(y.double().sum()) - 1.0) < 1e-4
    assert int(idx.item()) == int(np.argmax(x))


def test_argmax_ties_take_lowest_index(ntx):
    x = np.zeros(5000, dtype=np.float32)
    x[[123, 4000, 77]] = 2.0
    idx = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    ntx.ntx_argmax(dev(x), x.size, idx)
    assert int(idx.item()) == 77


@pytest.mark.parametrize("qtype", [0, 1, 2, 3])
def test_embedding_row(ntx, orc, syn, qtype):
    vocab, hidden = 1000, 4096
    qp = syn.decode_qparams(qtype, 1)
    E = torch.empty(vocab * syn.row_bytes(qtype, hidden), dtype=torch.uint8, device="cuda")
    syn.blocks_dev(E, qtype, 5, 1, vocab, hidden, qp)
    for token in (0, 513, vocab - 1):
        t = torch.tensor([token], dtype=torch.int32, device="cuda")
        h = torch.empty(hidden, dtype=torch.float32, device="cuda")
        ntx.ntx_embed(qtype, E, vocab, hidden, t, h)
        torch.cuda.synchronize()
        row = syn.blocks_host(qtype, 5, 1, 1, hidden, qp, row0=token)
        assert np.array_equal(h.cpu().numpy(), orc.embed(qtype, row, hidden, 0))


ATTN = [(32, 8, 1, 4097), (32, 8, 5, 4097), (32, 8, 300, 4097), (32, 8, 4097, 4097), (64, 8, 8193, 8193),
        (64, 8, 1000, 8193), (8, 8, 33, 64), (16, 8, 257, 300), (4, 1, 4096, 20000)]


@pytest.mark.parametrize("nq,nkv,n_ctx,max_ctx", ATTN, ids=[f"{a}q{b}kv-{c}of{d}" for a, b, c, d in ATTN])
def test_attention(ntx, orc, syn, nq, nkv, n_ctx, max_ctx):
    hd = 128
    q = syn.normal_f32_host(6, 1, nq * hd)
    kc = syn.normal_f16_host(6, 2, nkv * max_ctx * hd)
    vc = syn.normal_f16_host(6, 3, nkv * max_ctx * hd)
    out = torch.full((nq * hd,), float("nan"), dtype=torch.float32, device="cuda")
    wsb = ntx.ntx_attn_workspace_bytes(nq, nkv, hd, max_ctx)
    ws = torch.full((wsb,), 0xFF, dtype=torch.uint8, device="cuda")     # NaN bytes: it needs no initialisation
    kd, vd = dev(kc.view(np.float16)), dev(vc.view(np.float16))
    o = orc.attn_decode(q, kc.reshape(nkv, max_ctx, hd), vc.reshape(nkv, max_ctx, hd), nq, nkv, hd, n_ctx, max_ctx)
    first = None
    for _ in range(2):       # a second call on the used workspace gives the same bits
        ntx.ntx_attn_decode(dev(q), kd, vd, out, nq, nkv, hd, n_ctx, max_ctx, ws, wsb)
        torch.cuda.synchronize()
        got = out.cpu().numpy().copy()
        assert rel_err(got, o) <= 1e-4
        if first is None:
            first = got
        else:
            assert np.array_equal(first, got)
