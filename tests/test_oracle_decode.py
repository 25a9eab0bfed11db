"""Structural pins of the oracle's decode layer: special cases in which one Llama
layer reduces to a composition of the separately pinned pieces (GEMV, RMSNorm,
RoPE, attention, SwiGLU), so a swapped norm weight, a missing residual, a wrong
cache position or a rotated v fails."""
import numpy as np
import pytest

import blockpack as bp

HD, NQ, NKV, H, F, MAX_CTX = 32, 4, 2, 128, 96, 12
Q8 = 0


def _q8_matrix(rows, cols, rng, zero=False, identity=False):
    """Q8_0 [rows, cols]; d = 0 (zero), d = 1 with one-hot codes (identity), or random."""
    out = []
    dense = np.zeros((rows, cols))
    for r in range(rows):
        for b in range(cols // 32):
            if identity:
                q = np.zeros(32, dtype=np.int64)
                if r // 32 == b:
                    q[r % 32] = 1
                f = {"d": bp.f16_bits(1.0), "q": q}
            else:
                f = bp.random_fields(Q8, rng, d_range=(0.02, 0.05))
                if zero:
                    f["d"] = 0
            out.append(bp.pack(Q8, f))
            dense[r, b * 32:(b + 1) * 32] = [float(v) for v in bp.logical_weights(Q8, f)]
    return np.frombuffer(b"".join(out), dtype=np.uint8).reshape(rows, -1), dense


def _layer(rng, zero_attn=False, zero_ffn=False):
    qkv_rows = (NQ + 2 * NKV) * HD
    t = {"attn_norm": rng.uniform(0.5, 1.5, H).astype(np.float32),
         "ffn_norm": rng.uniform(0.5, 1.5, H).astype(np.float32)}
    t["w_qkv"], _ = _q8_matrix(qkv_rows, H, rng, zero=zero_attn)
    t["w_o"], _ = _q8_matrix(H, NQ * HD, rng, zero=zero_attn)
    t["w_gate"], _ = _q8_matrix(F, H, rng, zero=zero_ffn)
    t["w_up"], _ = _q8_matrix(F, H, rng, zero=zero_ffn)
    t["w_down"], _ = _q8_matrix(H, F, rng, zero=zero_ffn)
    t["k_cache"] = np.asarray(rng.standard_normal((NKV, MAX_CTX, HD)), dtype=np.float16).view(np.uint16)
    t["v_cache"] = np.asarray(rng.standard_normal((NKV, MAX_CTX, HD)), dtype=np.float16).view(np.uint16)
    return t


def _run(orc, t, h, pos):
    dims = orc.Dims(H, NQ, NKV, HD, F, MAX_CTX, 1e-5, 10000.0)
    h = h.copy()
    orc.decode_layer(dims, Q8, h, pos, t["attn_norm"], t["w_qkv"], t["w_o"], t["ffn_norm"], t["w_gate"],
                     t["w_up"], t["w_down"], t["k_cache"], t["v_cache"])
    return h


def test_zero_weights_pass_the_residual_through(orc):
    rng = np.random.default_rng(40)
    t = _layer(rng, zero_attn=True, zero_ffn=True)
    h0 = rng.standard_normal(H).astype(np.float32)
    h1 = _run(orc, t, h0, 5)
    assert np.array_equal(h1, h0)
    assert not np.any(t["k_cache"][:, 5].view(np.float16)) and not np.any(t["v_cache"][:, 5].view(np.float16))


def test_ffn_only_layer(orc):
    """Attention weights zero: h1 = h0 + W_down (silu(W_gate xn) * (W_up xn)), xn = RMSNorm(h0, ffn_norm)."""
    rng = np.random.default_rng(41)
    t = _layer(rng, zero_attn=True)
    h0 = rng.standard_normal(H).astype(np.float32)
    xn = orc.rmsnorm(h0, t["ffn_norm"], 1e-5)
    a = orc.swiglu(orc.gemv(Q8, t["w_gate"], F, H, xn), orc.gemv(Q8, t["w_up"], F, H, xn))
    want = h0 + orc.gemv(Q8, t["w_down"], H, F, a)
    assert np.array_equal(_run(orc, t, h0, 3), want)


def test_attention_only_layer_and_cache_write(orc):
    """FFN weights zero: h1 = h0 + W_o attn(RoPE(q), K, V) over positions 0..pos, with the
    new k (after RoPE) and v written to the caches at pos as fp16."""
    rng = np.random.default_rng(42)
    pos = 7
    t = _layer(rng, zero_ffn=True)
    kc0, vc0 = t["k_cache"].copy(), t["v_cache"].copy()
    # positions after pos hold values that must never be read
    t["k_cache"][:, pos + 1:] = np.float16(60000.0).view(np.uint16)
    t["v_cache"][:, pos + 1:] = np.float16(60000.0).view(np.uint16)
    h0 = rng.standard_normal(H).astype(np.float32)
    h1 = _run(orc, t, h0, pos)

    xn = orc.rmsnorm(h0, t["attn_norm"], 1e-5)
    qkv = orc.gemv(Q8, t["w_qkv"], (NQ + 2 * NKV) * HD, H, xn)
    q, k, v = qkv[:NQ * HD], qkv[NQ * HD:(NQ + NKV) * HD], qkv[(NQ + NKV) * HD:]
    q, k = orc.rope(q, k, NQ, NKV, HD, pos, 10000.0)
    k16 = np.asarray(k, dtype=np.float16).reshape(NKV, HD).view(np.uint16)
    v16 = np.asarray(v, dtype=np.float16).reshape(NKV, HD).view(np.uint16)
    assert np.array_equal(t["k_cache"][:, pos], k16)
    assert np.array_equal(t["v_cache"][:, pos], v16)
    assert np.array_equal(t["k_cache"][:, :pos], kc0[:, :pos]) and np.array_equal(t["v_cache"][:, :pos], vc0[:, :pos])
    kc, vc = kc0.copy(), vc0.copy()
    kc[:, pos], vc[:, pos] = k16, v16
    att = orc.attn_decode(q, kc, vc, NQ, NKV, HD, pos + 1, MAX_CTX)
    want = h0 + orc.gemv(Q8, t["w_o"], H, NQ * HD, att)
    assert np.array_equal(h1, want)


def test_lm_head_is_norm_then_gemv(orc):
    rng = np.random.default_rng(43)
    W, dense = _q8_matrix(64, H, rng)
    norm = rng.uniform(0.9, 1.1, H).astype(np.float32)
    h = rng.standard_normal(H).astype(np.float32)
    got = orc.lm_head(Q8, norm, W, 64, H, 1e-5, h)
    xn = orc.rmsnorm(h, norm, 1e-5)
    assert np.array_equal(got, orc.gemv(Q8, W, 64, H, xn))
    assert np.allclose(got, dense @ xn.astype(np.float64), rtol=1e-6, atol=1e-6)


@pytest.mark.parametrize("qtype", [0, 3])
def test_synthetic_model_stays_conditioned(orc, syn, qtype):
    """The decode recipe keeps the hidden state O(1) through the layers (no blow-up)."""
    from oracle import model
    spec = syn.ModelSpec(n_layers=3, hidden=256, n_q_heads=4, n_kv_heads=2, head_dim=64, ffn=512, vocab=300,
                         max_ctx=40, n_prefill=33, qtype=qtype, seed=7)
    logits, hidden = model.decode(spec, keep_hidden=True)
    rms = [float(np.sqrt(np.mean(h.astype(np.float64) ** 2))) for h in hidden]
    assert all(0.05 < r < 20 for r in rms), rms
    assert 0.2 < float(np.sqrt(np.mean(logits.astype(np.float64) ** 2))) < 5


def _tiny_spec(syn, **kw):
    base = dict(n_layers=3, hidden=256, n_q_heads=4, n_kv_heads=2, head_dim=128, ffn=512, vocab=64, max_ctx=24,
                n_prefill=16, qtype=syn.Q8_0, seed=5)
    base.update(kw)
    return syn.ModelSpec(**base)


def test_sequence_decode_structure(orc, syn):
    """The oracle's multi-token decode: one token equals the plain decode; earlier tokens'
    logits do not depend on later tokens (causality); a later token's logits depend on the
    earlier token (it attends to the K / V rows that token wrote)."""
    from oracle import model as om
    spec = _tiny_spec(syn)
    pos0 = spec.n_prefill
    one = om.decode_sequence(spec, [7], pos0)
    plain, _ = om.decode(spec, pos=pos0, token=7)
    assert np.array_equal(one[0], plain)
    ab = om.decode_sequence(spec, [7, 9, 3], pos0)
    assert np.array_equal(ab[0], plain)
    cb = om.decode_sequence(spec, [8, 9, 3], pos0)
    assert not np.array_equal(ab[1], cb[1]) and not np.array_equal(ab[2], cb[2])
    # the second token at pos0 + 1 with the prefilled row at pos0 (no first token) differs too
    alone, _ = om.decode(spec, pos=pos0 + 1, token=9)
    assert not np.array_equal(ab[1], alone)


def test_layer_skip_and_similarity(orc, syn):
    """Skipping a layer leaves h unchanged through it (the skipped model equals the model
    whose layer has zero residual contributions); a layer whose residual contributions are
    scaled by 2^-10 has a similarity within 1e-5 of 1 while ordinary layers are far below."""
    from oracle import model as om
    spec = _tiny_spec(syn, extra={"quiet_layers": [1]})
    cos = om.layer_similarity(spec)
    assert cos[1] > 1 - 1e-5 and max(cos[0], cos[2]) < 0.99
    _, hid = om.decode(spec, keep_hidden=True, skip={1})
    assert np.array_equal(hid[1], hid[0])
    full, hid_full = om.decode(spec, keep_hidden=True)
    assert np.array_equal(hid[0], hid_full[0]) and not np.array_equal(hid[2], hid_full[2])
