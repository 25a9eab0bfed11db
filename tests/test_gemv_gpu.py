"""GPU parity of the quantized GEMV and dequantization (through the C ABI) with
the CPU oracle, on inputs from the seeded generator."""
import numpy as np
import pytest
import torch

from gpu_util import GEMV_TIGHT, TOL, elem_err, ntx_module, rel_err

pytestmark = pytest.mark.gpu

Q8_0, Q4_0, Q4_K, Q6_K = 0, 1, 2, 3
NAMES = {Q8_0: "q8_0", Q4_0: "q4_0", Q4_K: "q4_k", Q6_K: "q6_k"}


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


def gpu_gemv(ntx, qtype, W, rows, cols, x):
    xd = torch.from_numpy(x).cuda()
    y = torch.full((rows,), float("nan"), dtype=torch.float32, device="cuda")
    ntx.ntx_gemv_q(qtype, W, rows, cols, xd, y)
    torch.cuda.synchronize()
    return y.cpu().numpy()


# fast path: rows that are 16-byte multiples, several groups + a partial group,
# several chunks + a partial chunk
FAST = [(Q8_0, 37, 4096 + 256), (Q4_0, 37, 4096 + 256), (Q4_K, 37, 8192 + 256), (Q6_K, 37, 8192 + 2048),
        (Q8_0, 1, 32 * 8), (Q4_K, 3, 256), (Q6_K, 2, 2048), (Q8_0, 150, 4096), (Q4_0, 300, 1024)]


@pytest.mark.parametrize("qtype,rows,cols", FAST, ids=[f"{NAMES[q]}-{r}x{c}" for q, r, c in FAST])
def test_gemv_fast_path(ntx, orc, syn, qtype, rows, cols):
    host, dev = make(syn, qtype, rows, cols)
    x = syn.normal_f32_host(1, 12, cols)
    y = gpu_gemv(ntx, qtype, dev, rows, cols, x)
    o = orc.gemv(qtype, host, rows, cols, x)
    e = rel_err(y, o)
    assert e <= TOL and e <= GEMV_TIGHT, e
    assert elem_err(y, o) <= TOL
    assert ntx.ntx_device_error() == 0


# simple kernel: rows that are not 16-byte multiples, or W only 2-byte aligned
SIMPLE = [(Q8_0, 5, 96), (Q4_0, 9, 160), (Q6_K, 4, 256 * 3), (Q4_K, 5, 256 * 3)]


@pytest.mark.parametrize("qtype,rows,cols", SIMPLE, ids=[f"{NAMES[q]}-{r}x{c}" for q, r, c in SIMPLE])
def test_gemv_simple_path(ntx, orc, syn, qtype, rows, cols):
    host, dev = make(syn, qtype, rows, cols)
    if qtype == Q4_K:      # 144-byte rows take the fast path when aligned: offset W by 2 bytes
        buf = torch.zeros(dev.numel() + 16, dtype=torch.uint8, device="cuda")
        buf[2:2 + dev.numel()] = dev
        W = buf.data_ptr() + 2
    else:
        W = dev
    x = syn.normal_f32_host(2, 12, cols)
    y = gpu_gemv(ntx, qtype, W, rows, cols, x)
    o = orc.gemv(qtype, host, rows, cols, x)
    assert rel_err(y, o) <= GEMV_TIGHT


@pytest.mark.parametrize("qtype", [Q8_0, Q4_0, Q4_K, Q6_K], ids=list(NAMES.values()))
def test_one_hot_input_returns_the_dequantized_column(ntx, syn, qtype):
    """x = e_k: every product and the offset subtraction are exact, so y == W[:, k] bit for bit."""
    rows, cols = 24, 8192 + (2048 if qtype == Q6_K else 256)
    host, dev = make(syn, qtype, rows, cols)
    dq = torch.empty((rows, cols), dtype=torch.float32, device="cuda")
    ntx.ntx_dequant_q(qtype, dev, rows, cols, dq)
    for k in (0, 17, cols // 2 + 3, cols - 1):
        x = np.zeros(cols, dtype=np.float32)
        x[k] = 1.0
        y = gpu_gemv(ntx, qtype, dev, rows, cols, x)
        assert np.array_equal(y, dq[:, k].cpu().numpy()), k


@pytest.mark.parametrize("qtype", [Q8_0, Q4_K])
def test_gemv_input_edge_cases(ntx, orc, syn, qtype):
    rows, cols = 40, 8192
    host, dev = make(syn, qtype, rows, cols)
    zero = np.zeros(cols, dtype=np.float32)
    assert np.array_equal(gpu_gemv(ntx, qtype, dev, rows, cols, zero), np.zeros(rows, dtype=np.float32))
    # wide dynamic range: tiny and huge inputs mixed (exercises the input scaling)
    x = syn.normal_f32_host(3, 12, cols)
    x[::7] *= 1e20
    x[1::7] *= 1e-20
    assert rel_err(gpu_gemv(ntx, qtype, dev, rows, cols, x), orc.gemv(qtype, host, rows, cols, x)) <= GEMV_TIGHT
    for scale in (1e-30, 1e25):
        xs = (syn.normal_f32_host(4, 12, cols) * np.float32(scale)).astype(np.float32)
        assert rel_err(gpu_gemv(ntx, qtype, dev, rows, cols, xs), orc.gemv(qtype, host, rows, cols, xs)) <= GEMV_TIGHT


# ----------------------------------------------------------------- dequantization

DQ = [(Q8_0, 37, 4096 + 256), (Q4_0, 37, 4096 + 256), (Q4_K, 37, 8192 + 256), (Q6_K, 37, 8192 + 2048),
      (Q8_0, 3, 96), (Q6_K, 3, 768), (Q4_K, 4096, 4096), (Q4_0, 4096, 4096)]


@pytest.mark.parametrize("qtype,rows,cols", DQ, ids=[f"{NAMES[q]}-{r}x{c}" for q, r, c in DQ])
def test_dequant_bit_exact(ntx, orc, syn, qtype, rows, cols):
    host, dev = make(syn, qtype, rows, cols)
    out = torch.empty((rows, cols), dtype=torch.float32, device="cuda")
    ntx.ntx_dequant_q(qtype, dev, rows, cols, out)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy().view(np.uint32), orc.dequant(qtype, host, rows, cols).view(np.uint32))


def test_dequant_decode_recipe_subnormal_scales(ntx, orc, syn):
    """Q6_K at K = 28672 under the decode recipe has fp16-subnormal scales."""
    host, dev = make(syn, Q6_K, 8, 28672, decode=True)
    d = host.reshape(-1, 210)[:, 208:210].copy().view(np.uint16)
    assert np.any((d & 0x7C00) == 0)
    out = torch.empty((8, 28672), dtype=torch.float32, device="cuda")
    ntx.ntx_dequant_q(Q6_K, dev, 8, 28672, out)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy().view(np.uint32), orc.dequant(Q6_K, host, 8, 28672).view(np.uint32))


# ------------------------------------------------------- full-size workload shapes

# (K -> N): Llama-8B layer shapes of the GEMV sweep, and the Llama-70B shapes of the Q6_K decode
SWEEP = [(q, n, k) for q in (Q4_0, Q4_K) for (k, n) in ((4096, 6144), (4096, 4096), (4096, 14336), (14336, 4096))]
SWEEP += [(Q8_0, 4096, 4096), (Q8_0, 6144, 4096), (Q8_0, 4096, 14336), (Q6_K, 10240, 8192), (Q6_K, 8192, 28672),
          (Q6_K, 28672, 8192)]


@pytest.mark.parametrize("qtype,rows,cols", SWEEP, ids=[f"{NAMES[q]}-{r}x{c}" for q, r, c in SWEEP])
def test_gemv_full_shapes(ntx, orc, syn, qtype, rows, cols):
    host, dev = make(syn, qtype, rows, cols)
    x = syn.normal_f32_host(5, 12, cols)
    y = gpu_gemv(ntx, qtype, dev, rows, cols, x)
    o = orc.gemv(qtype, host, rows, cols, x)
    e = rel_err(y, o)
    assert e <= GEMV_TIGHT, e
    assert elem_err(y, o) <= TOL


@pytest.mark.parametrize("tiled", [False, True], ids=["gguf", "tiled"])
@pytest.mark.parametrize("qtype", [Q4_0, Q4_K, Q8_0, Q6_K], ids=["q4_0", "q4_k", "q8_0", "q6_k"])
def test_gemv_lm_head_sampled_rows(ntx, orc, syn, qtype, tiled):
    """The 4096 -> 128256 (8192 -> 128256 for Q6_K) LM-head GEMV at full size, in the GGUF-style
    and the tiled layout, checked on sampled rows the oracle computes one by one."""
    rows, cols = 128256, (8192 if qtype == Q6_K else 4096)
    qp = syn.sweep_qparams(qtype)
    dev = torch.empty(rows * syn.row_bytes(qtype, cols), dtype=torch.uint8, device="cuda")
    syn.blocks_dev(dev, qtype, 9, 21, rows, cols, qp)
    if tiled:
        t = torch.empty_like(dev)
        ntx.ntx_repack_q(qtype, dev, t, rows, cols)
        dev = t
    x = syn.normal_f32_host(9, 22, cols)
    y = gpu_gemv(ntx, qtype | (T if tiled else 0), dev, rows, cols, x)
    rng = np.random.default_rng(0)
    sample = np.unique(np.concatenate([[0, 1, 15, 16, rows // 2, rows - 17, rows - 2, rows - 1],
                                       rng.integers(0, rows, 300)]))
    o = np.empty(sample.size, dtype=np.float32)
    for i, r in enumerate(sample):
        Wr = syn.blocks_host(qtype, 9, 21, 1, cols, qp, row0=int(r))
        o[i] = orc.gemv(qtype, Wr, 1, cols, x)[0]
    assert rel_err(y[sample], o) <= GEMV_TIGHT
    assert elem_err(y[sample], o) <= TOL


# ------------------------------------------------------------ outlier channels

ZERO_CODE = {Q8_0: 0, Q4_0: 8, Q4_K: 0, Q6_K: 32}


def outlier_matrix(qtype, rows, cols, cols_out, seed):
    """Packed GGUF-style [rows, cols] with random fields, whose first rows // 2 rows hold a
    zero weight at every column of cols_out (the format's zero code; for Q4_K also a zero
    min for that sub-block), built with the test-side packer."""
    import blockpack as bp
    rng = np.random.default_rng(seed)
    be = 32 if qtype in (Q8_0, Q4_0) else 256
    out = bytearray()
    for r in range(rows):
        for b in range(cols // be):
            f = bp.random_fields(qtype, rng)
            if r < rows // 2:
                for c in cols_out:
                    if b * be <= c < (b + 1) * be:
                        f["q"] = np.array(f["q"])
                        f["q"][c - b * be] = ZERO_CODE[qtype]
                        if qtype == Q4_K:
                            f["m"] = np.array(f["m"])
                            f["m"][(c - b * be) // 32] = 0
            out += bp.pack(qtype, f)
    return np.frombuffer(bytes(out), dtype=np.uint8).reshape(rows, -1).copy()


def outlier_input(syn, cols, cols_out):
    """x ~ N(0, 1) with LLM-style outlier channels: six at 1e3 and two at 1e4 times the rest."""
    x = syn.normal_f32_host(31, 12, cols)
    for i, c in enumerate(cols_out):
        x[c] = np.float32((1e4 if i >= 6 else 1e3) * (1.0 if i % 2 else -1.0) * (1.0 + 0.1 * i))
    return x


@pytest.mark.parametrize("layout", ["gguf", "tiled-dp4a", "tiled-tc"])
@pytest.mark.parametrize("qtype", [Q8_0, Q4_0, Q4_K, Q6_K], ids=list(NAMES.values()))
def test_gemv_outlier_channels(ntx, orc, syn, monkeypatch, qtype, layout):
    """A few input channels 1e3..1e4 times the rest, and half of the rows with zero weight at
    those channels: those rows' outputs are far below the largest output, and must keep their
    own precision (per-element error against the oracle, floor 1e-3 max |o|), not only the
    normwise one."""
    rows, cols = 64, 4096
    cols_out = [5, 700, 1031, 2047, 2048, 3333, 3900, 4095]
    host = outlier_matrix(qtype, rows, cols, cols_out, seed=qtype + 40)
    dev = torch.from_numpy(host.reshape(-1)).cuda()
    q = qtype
    if layout != "gguf":
        monkeypatch.setenv("NTX_GEMV_CORE", "tc" if layout.endswith("tc") else "dp4a")
        t = torch.empty_like(dev)
        ntx.ntx_repack_q(qtype, dev, t, rows, cols)
        dev, q = t, qtype | T
    x = outlier_input(syn, cols, cols_out)
    y = gpu_gemv(ntx, q, dev, rows, cols, x)
    o = orc.gemv(qtype, host, rows, cols, x)
    # the rows that ignore the outliers are the small ones
    assert np.max(np.abs(o[: rows // 2])) < 0.05 * np.max(np.abs(o[rows // 2:]))
    assert rel_err(y, o) <= GEMV_TIGHT
    e = elem_err(y, o)
    print(f"outlier channels {NAMES[qtype]} {layout}: normwise {rel_err(y, o):.2e} per-element {e:.2e}")
    assert e <= TOL, e


# ------------------------------------------------------------------ tiled layouts

T = 16      # tiled flag


def make_tiled(ntx, syn, qtype, rows, cols, seed=1):
    host, dev = make(syn, qtype, rows, cols, seed)
    tiled = torch.empty_like(dev)
    ntx.ntx_repack_q(qtype, dev, tiled, rows, cols)
    torch.cuda.synchronize()
    return host, tiled


# 16-row groups: one group, fewer groups than SMs, several per SM; several 4096-column
# chunks and a partial one; a row shorter than one chunk
TILED_FAST = [(Q8_0, 48, 4096 + 256), (Q4_0, 48, 4096 + 256), (Q4_K, 48, 8192 + 256), (Q6_K, 48, 8192 + 256),
              (Q8_0, 48, 8192 + 1024 + 32), (Q4_0, 48, 8192 + 96),
              (Q8_0, 4096, 4096), (Q6_K, 16, 2048), (Q4_0, 304, 1024), (Q8_0, 16, 32), (Q4_K, 16, 256),
              (Q6_K, 4096, 1024 + 256), (Q4_0, 32, 96)]


@pytest.mark.parametrize("qtype,rows,cols", TILED_FAST, ids=[f"{NAMES[q]}_t-{r}x{c}" for q, r, c in TILED_FAST])
def test_gemv_tiled(ntx, orc, syn, qtype, rows, cols):
    host, W = make_tiled(ntx, syn, qtype, rows, cols)
    x = syn.normal_f32_host(1, 13, cols)
    y, o = gpu_gemv(ntx, qtype | T, W, rows, cols, x), orc.gemv(qtype, host, rows, cols, x)
    e = rel_err(y, o)
    assert e <= TOL and e <= GEMV_TIGHT, e
    assert elem_err(y, o) <= TOL


@pytest.mark.parametrize("qtype", [Q8_0, Q4_0, Q4_K, Q6_K], ids=list(NAMES.values()))
def test_tiled_dequant_bit_exact_and_simple_path(ntx, orc, syn, qtype):
    rows, cols = 32, 4096 if qtype != Q6_K else 6144
    host, W = make_tiled(ntx, syn, qtype, rows, cols)
    out = torch.empty((rows, cols), dtype=torch.float32, device="cuda")
    ntx.ntx_dequant_q(qtype | T, W, rows, cols, out)
    torch.cuda.synchronize()
    want = orc.dequant(qtype, host, rows, cols)
    assert np.array_equal(out.cpu().numpy().view(np.uint32), want.view(np.uint32))
    # the same tiled bytes at a 2-byte-aligned address take the simple kernel
    buf = torch.zeros(W.numel() + 16, dtype=torch.uint8, device="cuda")
    buf[2:2 + W.numel()] = W
    x = syn.normal_f32_host(2, 13, cols)
    y = gpu_gemv(ntx, qtype | T, buf.data_ptr() + 2, rows, cols, x)
    assert rel_err(y, orc.gemv(qtype, host, rows, cols, x)) <= GEMV_TIGHT


@pytest.mark.parametrize("qtype", [Q8_0, Q4_0, Q4_K, Q6_K], ids=list(NAMES.values()))
def test_tiled_one_hot_bit_exact(ntx, syn, qtype):
    rows, cols = 16, 8192 + (2048 if qtype == Q6_K else 256)
    host, W = make_tiled(ntx, syn, qtype, rows, cols)
    dq = torch.empty((rows, cols), dtype=torch.float32, device="cuda")
    ntx.ntx_dequant_q(qtype | T, W, rows, cols, dq)
    for k in (0, 33, cols // 2 + 5, cols - 1):
        x = np.zeros(cols, dtype=np.float32)
        x[k] = 1.0
        assert np.array_equal(gpu_gemv(ntx, qtype | T, W, rows, cols, x), dq[:, k].cpu().numpy()), k


TSWEEP = [(q, n, k) for q in (Q4_0, Q4_K, Q8_0) for (k, n) in ((4096, 6144), (4096, 4096), (4096, 14336),
                                                                 (14336, 4096))]
TSWEEP += [(Q6_K, 10240, 8192), (Q6_K, 8192, 8192), (Q6_K, 8192, 28672), (Q6_K, 28672, 8192)]


@pytest.mark.parametrize("qtype,rows,cols", TSWEEP, ids=[f"{NAMES[q]}_t-{r}x{c}" for q, r, c in TSWEEP])
def test_gemv_tiled_full_shapes(ntx, orc, syn, qtype, rows, cols):
    host, W = make_tiled(ntx, syn, qtype, rows, cols)
    x = syn.normal_f32_host(6, 12, cols)
    y, o = gpu_gemv(ntx, qtype | T, W, rows, cols, x), orc.gemv(qtype, host, rows, cols, x)
    assert rel_err(y, o) <= GEMV_TIGHT
    assert elem_err(y, o) <= TOL


@pytest.mark.parametrize("qtype,rows,cols", [(Q8_0, 32, 512), (Q4_0, 16, 256), (Q4_K, 32, 512), (Q6_K, 16, 768)],
                         ids=["q8_0", "q4_0", "q4_k", "q6_k"])
def test_repack_matches_documented_layout(ntx, syn, qtype, rows, cols):
    """The repack kernel's bytes equal the layout the header documents (an independent
    numpy model of it)."""
    import tiling
    host, W = make_tiled(ntx, syn, qtype, rows, cols)
    assert np.array_equal(W.cpu().numpy(), tiling.tile(qtype, host, rows, cols))


@pytest.mark.parametrize("core", ["tc", "dp4a"], ids=["tensor-cores", "cuda-cores"])
@pytest.mark.parametrize("split", ["0", "1"], ids=["whole-rows", "column-halves"])
@pytest.mark.parametrize("qtype,rows,cols", [(Q6_K, 1024, 8192 + 256), (Q8_0, 2048, 4096 + 32), (Q4_K, 160, 2304),
                                             (Q4_0, 32, 64)], ids=["q6_k", "q8_0", "q4_k", "q4_0"])
def test_gemv_tiled_both_cluster_shapes(ntx, orc, syn, monkeypatch, core, split, qtype, rows, cols):
    """Whole rows per CTA and CTA pairs that split the columns (forced either way), with
    the per-step sums on the tensor cores or on the CUDA cores: all match the oracle,
    including an odd number of units per row."""
    monkeypatch.setenv("NTX_GEMV_SPLIT", split)
    monkeypatch.setenv("NTX_GEMV_CORE", core)
    host, W = make_tiled(ntx, syn, qtype, rows, cols)
    x = syn.normal_f32_host(7, 12, cols)
    assert rel_err(gpu_gemv(ntx, qtype | T, W, rows, cols, x), orc.gemv(qtype, host, rows, cols, x)) <= GEMV_TIGHT


@pytest.mark.parametrize("core", ["tc", "dp4a"], ids=["tensor-cores", "cuda-cores"])
@pytest.mark.parametrize("qtype", [Q8_0, Q4_0, Q4_K, Q6_K], ids=list(NAMES.values()))
def test_tiled_one_hot_both_cores(ntx, syn, monkeypatch, core, qtype):
    """A one-hot x returns the dequantized column bit for bit on either unit."""
    monkeypatch.setenv("NTX_GEMV_CORE", core)
    rows, cols = 32, 4096 + (256 if qtype in (Q4_K, Q6_K) else 32)
    host, W = make_tiled(ntx, syn, qtype, rows, cols)
    dq = torch.empty((rows, cols), dtype=torch.float32, device="cuda")
    ntx.ntx_dequant_q(qtype | T, W, rows, cols, dq)
    for k in (0, 17, cols // 2 + 3, cols - 1):
        x = np.zeros(cols, dtype=np.float32)
        x[k] = 1.0
        assert np.array_equal(gpu_gemv(ntx, qtype | T, W, rows, cols, x), dq[:, k].cpu().numpy()), (core, k)


@pytest.mark.parametrize("core", ["tc", "dp4a"], ids=["tensor-cores", "cuda-cores"])
@pytest.mark.parametrize("qtype", [Q8_0, Q4_0, Q4_K, Q6_K], ids=list(NAMES.values()))
def test_tiled_input_edge_cases(ntx, orc, syn, monkeypatch, core, qtype):
    """The tiled path takes x as 24-bit fixed point relative to max |x|: a zero x gives
    exact zeros, and very small, very large and mixed-magnitude inputs stay within the
    tolerance (values far below max |x| round to zero, which the normwise error allows)."""
    monkeypatch.setenv("NTX_GEMV_CORE", core)
    rows, cols = 48, 8192 + 256
    host, W = make_tiled(ntx, syn, qtype, rows, cols)
    zero = np.zeros(cols, dtype=np.float32)
    assert np.array_equal(gpu_gemv(ntx, qtype | T, W, rows, cols, zero), np.zeros(rows, dtype=np.float32))
    x = syn.normal_f32_host(3, 12, cols)
    x[::7] *= 1e20
    x[1::7] *= 1e-20
    assert rel_err(gpu_gemv(ntx, qtype | T, W, rows, cols, x), orc.gemv(qtype, host, rows, cols, x)) <= GEMV_TIGHT
    for scale in (1e-30, 1e25):
        xs = (syn.normal_f32_host(4, 12, cols) * np.float32(scale)).astype(np.float32)
        assert rel_err(gpu_gemv(ntx, qtype | T, W, rows, cols, xs), orc.gemv(qtype, host, rows, cols, xs)) <= GEMV_TIGHT


@pytest.mark.parametrize("qtype", [Q8_0 | T, Q6_K | T, Q8_0], ids=["q8_0_t", "q6_k_t", "q8_0"])
def test_gemv_chain_without_sync(ntx, orc, syn, qtype):
    """Back-to-back GEMVs on one stream (programmatic dependent launch): the second
    reads the first's output, and a third overwrites the first's input; each matches the
    oracle on the values it actually read."""
    base = qtype & ~T
    K1, M1 = (8192 + 256, 512) if base == Q6_K else (4096 + 32, 512)
    M2 = M1
    h1, W1 = (make_tiled(ntx, syn, base, M1, K1, seed=3) if qtype & T else make(syn, base, M1, K1, 3))
    K2 = M1 if base != Q6_K else 512
    h2, W2 = (make_tiled(ntx, syn, base, M2, K2, seed=4) if qtype & T else make(syn, base, M2, K2, 4))
    h3, W3 = (make_tiled(ntx, syn, base, K1, M2, seed=5) if qtype & T else make(syn, base, K1, M2, 5))
    x = torch.from_numpy(syn.normal_f32_host(6, 12, K1)).cuda()
    x0 = x.cpu().numpy().copy()
    a = torch.empty(M1, dtype=torch.float32, device="cuda")
    b = torch.empty(M2, dtype=torch.float32, device="cuda")
    ntx.ntx_gemv_q(qtype, W1, M1, K1, x, a)      # a = W1 x
    ntx.ntx_gemv_q(qtype, W2, M2, K2, a, b)      # b = W2 a (reads the previous output)
    ntx.ntx_gemv_q(qtype, W3, K1, M2, b, x)      # x = W3 b (overwrites the first input)
    torch.cuda.synchronize()
    an, bn, xn = a.cpu().numpy(), b.cpu().numpy(), x.cpu().numpy()
    assert rel_err(an, orc.gemv(base, h1, M1, K1, x0)) <= GEMV_TIGHT
    assert rel_err(bn, orc.gemv(base, h2, M2, K2, an)) <= GEMV_TIGHT
    assert rel_err(xn, orc.gemv(base, h3, K1, M2, bn)) <= GEMV_TIGHT


def test_stream_read_probe(ntx):
    """The HBM read probe streams a buffer (larger than L2, with a ragged tail slice)
    without a device error."""
    buf = torch.empty((256 << 20) + 48, dtype=torch.uint8, device="cuda")
    ntx.ntx_stream_read_probe(buf, buf.numel())
    torch.cuda.synchronize()
    assert ntx.ntx_device_error() == 0
    with pytest.raises(ntx.NtxError):
        ntx.ntx_stream_read_probe(buf, 100)
