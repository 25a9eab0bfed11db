"""GPU parity of the further weight formats (Q5_K in both layouts, F16, F32) through the
C ABI with the CPU oracle: dequantization bit-exact, GEMV within the tolerances, the
tiled Q5_K bytes equal to the documented layout, and the fused decode-step GEMVs."""
import numpy as np
import pytest
import torch

from gpu_util import GEMV_TIGHT, TOL, elem_err, ntx_module, rel_err

pytestmark = pytest.mark.gpu

Q5_K, F16, F32 = 4, 5, 6
T = 16
NAMES = {Q5_K: "q5_k", F16: "f16", F32: "f32"}


@pytest.fixture(scope="module")
def ntx():
    return ntx_module()


def make(syn, qtype, rows, cols, seed=1, decode=False):
    qp = syn.decode_qparams(qtype, cols) if decode else syn.sweep_qparams(qtype)
    host = syn.blocks_host(qtype, seed, 11, rows, cols, qp)
    dev = torch.empty(host.size, dtype=torch.uint8, device="cuda")
    syn.blocks_dev(dev, qtype, seed, 11, rows, cols, qp)
    torch.cuda.synchronize()
    assert np.array_equal(dev.cpu().numpy().reshape(host.shape), host), "device generator differs from host"
    return host, dev


def tiled(ntx, qtype, dev, rows, cols):
    t = torch.empty_like(dev)
    ntx.ntx_repack_q(qtype, dev, t, rows, cols)
    torch.cuda.synchronize()
    return t


def gpu_gemv(ntx, qtype, W, rows, cols, x):
    xd = torch.from_numpy(x).cuda()
    y = torch.full((rows,), float("nan"), dtype=torch.float32, device="cuda")
    ntx.ntx_gemv_q(qtype, W, rows, cols, xd, y)
    torch.cuda.synchronize()
    return y.cpu().numpy()


DQ = [(Q5_K, 37, 4096 + 256), (Q5_K, 3, 768), (F16, 37, 4104), (F16, 5, 3), (F32, 37, 4100), (F32, 2, 7)]


@pytest.mark.parametrize("qtype,rows,cols", DQ, ids=[f"{NAMES[q]}-{r}x{c}" for q, r, c in DQ])
def test_dequant_bit_exact(ntx, orc, syn, qtype, rows, cols):
    host, dev = make(syn, qtype, rows, cols)
    out = torch.empty((rows, cols), dtype=torch.float32, device="cuda")
    ntx.ntx_dequant_q(qtype, dev, rows, cols, out)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy().view(np.uint32), orc.dequant(qtype, host, rows, cols).view(np.uint32))


def test_q5_k_tiled_dequant_and_layout(ntx, orc, syn):
    import tiling
    rows, cols = 32, 512
    host, dev = make(syn, Q5_K, rows, cols)
    W = tiled(ntx, Q5_K, dev, rows, cols)
    assert np.array_equal(W.cpu().numpy(), tiling.tile(Q5_K, host, rows, cols))
    out = torch.empty((rows, cols), dtype=torch.float32, device="cuda")
    ntx.ntx_dequant_q(Q5_K | T, W, rows, cols, out)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy().view(np.uint32), orc.dequant(Q5_K, host, rows, cols).view(np.uint32))


# (qtype, rows, cols, layout): several groups and a partial one, several chunks and a partial one,
# the Llama-8B layer shapes; F16 / F32 rows that are not 16-byte multiples take the simple kernel
GEMV = [(Q5_K, 48, 8192 + 256, "tiled"), (Q5_K, 4096, 4096, "tiled"), (Q5_K, 14336, 4096, "tiled"),
        (Q5_K, 4096, 14336, "tiled"), (Q5_K, 6144, 4096, "tiled"), (Q5_K, 37, 2304, "gguf"),
        (F16, 37, 4096 + 1024 + 8, "gguf"), (F16, 4096, 4096, "gguf"), (F16, 16, 28672, "gguf"),
        (F16, 5, 1003, "gguf"), (F32, 37, 4096 + 512 + 4, "gguf"), (F32, 4096, 4096, "gguf"),
        (F32, 16, 14336, "gguf"), (F32, 3, 31, "gguf")]


@pytest.mark.parametrize("qtype,rows,cols,layout", GEMV, ids=[f"{NAMES[q]}_{l}-{r}x{c}" for q, r, c, l in GEMV])
def test_gemv(ntx, orc, syn, qtype, rows, cols, layout):
    host, dev = make(syn, qtype, rows, cols)
    W, q = (tiled(ntx, qtype, dev, rows, cols), qtype | T) if layout == "tiled" else (dev, qtype)
    x = syn.normal_f32_host(1, 12, cols)
    y, o = gpu_gemv(ntx, q, W, rows, cols, x), orc.gemv(qtype, host, rows, cols, x)
    assert rel_err(y, o) <= GEMV_TIGHT
    assert elem_err(y, o) <= TOL
    assert ntx.ntx_device_error() == 0


@pytest.mark.parametrize("core", ["tc", "dp4a"], ids=["tensor-cores", "cuda-cores"])
@pytest.mark.parametrize("split", ["0", "1"], ids=["whole-rows", "column-halves"])
def test_q5_k_tiled_both_cluster_shapes_and_cores(ntx, orc, syn, monkeypatch, core, split):
    monkeypatch.setenv("NTX_GEMV_SPLIT", split)
    monkeypatch.setenv("NTX_GEMV_CORE", core)
    rows, cols = 1024, 8192 + 256
    host, dev = make(syn, Q5_K, rows, cols)
    W = tiled(ntx, Q5_K, dev, rows, cols)
    x = syn.normal_f32_host(7, 12, cols)
    assert rel_err(gpu_gemv(ntx, Q5_K | T, W, rows, cols, x), orc.gemv(Q5_K, host, rows, cols, x)) <= GEMV_TIGHT


@pytest.mark.parametrize("qtype", [Q5_K, F16, F32], ids=list(NAMES.values()))
def test_one_hot_input_returns_the_dequantized_column(ntx, syn, qtype):
    rows, cols = 32, 4096 + 256
    host, dev = make(syn, qtype, rows, cols)
    W, q = (tiled(ntx, qtype, dev, rows, cols), qtype | T) if qtype == Q5_K else (dev, qtype)
    dq = torch.empty((rows, cols), dtype=torch.float32, device="cuda")
    ntx.ntx_dequant_q(q, W, rows, cols, dq)
    for k in (0, 17, cols // 2 + 3, cols - 1):
        x = np.zeros(cols, dtype=np.float32)
        x[k] = 1.0
        assert np.array_equal(gpu_gemv(ntx, q, W, rows, cols, x), dq[:, k].cpu().numpy()), k


@pytest.mark.parametrize("qtype", [Q5_K, F16, F32], ids=list(NAMES.values()))
def test_outlier_channels(ntx, orc, syn, qtype):
    """Outlier input channels (1e3..1e4 times the rest): per-element error stays within the
    tolerance (the float formats have no fixed-point step at all)."""
    rows, cols = 64, 4096
    host, dev = make(syn, qtype, rows, cols, seed=5)
    W, q = (tiled(ntx, qtype, dev, rows, cols), qtype | T) if qtype == Q5_K else (dev, qtype)
    x = syn.normal_f32_host(31, 12, cols)
    for i, c in enumerate([5, 700, 1031, 2047, 2048, 3333, 3900, 4095]):
        x[c] = np.float32((1e4 if i >= 6 else 1e3) * (1.0 if i % 2 else -1.0))
    y, o = gpu_gemv(ntx, q, W, rows, cols, x), orc.gemv(qtype, host, rows, cols, x)
    assert rel_err(y, o) <= GEMV_TIGHT
    assert elem_err(y, o) <= TOL


@pytest.mark.parametrize("qtype", [Q5_K, F16], ids=["q5_k", "f16"])
def test_gemv_lm_head_sampled_rows(ntx, orc, syn, qtype):
    rows, cols = 128256, 4096
    qp = syn.sweep_qparams(qtype)
    dev = torch.empty(rows * syn.row_bytes(qtype, cols), dtype=torch.uint8, device="cuda")
    syn.blocks_dev(dev, qtype, 9, 21, rows, cols, qp)
    W, q = (tiled(ntx, qtype, dev, rows, cols), qtype | T) if qtype == Q5_K else (dev, qtype)
    x = syn.normal_f32_host(9, 22, cols)
    y = gpu_gemv(ntx, q, W, rows, cols, x)
    rng = np.random.default_rng(0)
    sample = np.unique(np.concatenate([[0, 15, 16, rows - 1], rng.integers(0, rows, 200)]))
    o = np.array([orc.gemv(qtype, syn.blocks_host(qtype, 9, 21, 1, cols, qp, row0=int(r)), 1, cols, x)[0]
                  for r in sample], dtype=np.float32)
    assert rel_err(y[sample], o) <= GEMV_TIGHT
    assert elem_err(y[sample], o) <= TOL
