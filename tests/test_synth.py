"""The seeded input generator: determinism, ranges and the recipe's distributions."""
import numpy as np
import pytest

import blockpack  # noqa: F401  (keeps the tests directory importable)


def test_blocks_are_deterministic_and_addressable(syn):
    qp = syn.sweep_qparams(syn.Q8_0)
    a = syn.blocks_host(syn.Q8_0, 5, 1, 6, 256, qp)
    b = syn.blocks_host(syn.Q8_0, 5, 1, 6, 256, qp)
    assert np.array_equal(a, b)
    # rows generated on their own equal the same rows of the whole tensor
    c = syn.blocks_host(syn.Q8_0, 5, 1, 2, 256, qp, row0=3)
    assert np.array_equal(c, a[3:5])
    assert not np.array_equal(a, syn.blocks_host(syn.Q8_0, 6, 1, 6, 256, qp))


def test_generator_f16_conversion_matches_ieee(syn):
    rng = np.random.default_rng(0)
    ks = rng.integers(1, 2 ** 40, 5000, dtype=np.int64)
    es = rng.integers(-70, -20, 5000)
    for k, e in zip(ks, es):
        with np.errstate(over="ignore"):
            want = np.float16(float(k) * 2.0 ** int(e)).view(np.uint16)  # k*2^e is exact in double here
        assert syn.host().syn_f16_bits_of_scaled(int(k), int(e)) == want


@pytest.mark.parametrize("qtype", [0, 1, 2, 3, 4])
def test_sweep_distribution(orc, syn, qtype):
    qp = syn.sweep_qparams(qtype)
    W = syn.blocks_host(qtype, 1, 1, 64, 1024, qp)
    be, bb = syn.BLOCK[qtype]
    blocks = W.reshape(-1, bb)
    d_off = {0: 0, 1: 0, 2: 0, 3: 208, 4: 0}[qtype]
    d = blocks[:, d_off:d_off + 2].copy().view(np.float16).astype(np.float64).ravel()
    assert d.min() >= 0.999e-3 and d.max() <= 1.0001e-2
    if qtype == 0:
        q = blocks[:, 2:].view(np.int8)
        assert q.min() == -127 and q.max() == 127
    dense = orc.dequant(qtype, W, 64, 1024)
    assert np.all(np.isfinite(dense))


@pytest.mark.parametrize("qtype", [0, 1, 2, 3, 4])
def test_decode_recipe_is_unit_gain(orc, syn, qtype):
    """Decode tensors map a unit-RMS input to a roughly unit-RMS output."""
    K = 2048
    W = syn.blocks_host(qtype, 2, 3, 256, K, syn.decode_qparams(qtype, K))
    x = syn.normal_f32_host(2, 4, K)
    y = orc.gemv(qtype, W, 256, K, x)
    rms = float(np.sqrt(np.mean(y.astype(np.float64) ** 2)))
    assert 0.7 < rms < 1.4, rms


def test_normal_stand_in_moments(syn):
    x = syn.normal_f32_host(3, 9, 200000).astype(np.float64)
    assert abs(x.mean()) < 0.01 and abs(x.var() - 1) < 0.02 and np.abs(x).max() <= 6
    h = syn.normal_f16_host(3, 9, 1000).view(np.float16).astype(np.float32)
    assert np.array_equal(h, x[:1000].astype(np.float16).astype(np.float32))     # fp16 = RNE of the same value


def test_norm_weights_range(syn):
    w = syn.uniform_f32_host(1, 2, 10000, *syn.NORM_W)
    assert w.min() >= 0.9 and w.max() <= 1.1 + 1e-7
