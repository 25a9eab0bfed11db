"""The C-ABI library: it builds for sm_100a, loads, exports every symbol that
include/ntx.h declares, and rejects bad arguments on the host before any launch
(no GPU needed: every call here returns before touching the device)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def ntx():
    from quantized_weight_gemv_block_b200 import build
    build.build()
    import quantized_weight_gemv_block_b200 as m
    m.lib()
    return m


def declared_functions():
    text = open(os.path.join(ROOT, "include", "ntx.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ntx_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(ntx):
    names = declared_functions()
    assert len(names) >= 20
    lib = ctypes.CDLL(ntx.LIB)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    assert sorted(ntx.EXPORTS) == names


def test_row_bytes_and_block_sizes(ntx):
    assert ntx.ntx_row_bytes(ntx.NTX_Q8_0, 4096) == 4352
    assert ntx.ntx_row_bytes(ntx.NTX_Q4_0, 4096) == 2304
    assert ntx.ntx_row_bytes(ntx.NTX_Q4_K, 14336) == 8064
    assert ntx.ntx_row_bytes(ntx.NTX_Q6_K, 28672) == 23520
    assert ntx.ntx_row_bytes(ntx.NTX_Q4_K, 128) == 0          # not a multiple of 256
    assert ntx.ntx_row_bytes(9, 256) == 0
    assert [ntx.ntx_block_elems(q) for q in range(7)] == [32, 32, 256, 256, 256, 1, 1]


def _status(ntx, fn, *args):
    return getattr(ntx.lib(), fn)(*args)


def test_gemv_rejects_bad_arguments(ntx):
    p = 0x10000          # never dereferenced: every call below fails validation first
    assert _status(ntx, "ntx_gemv_q", 7, p, 4, 256, p, p, None) == ntx.NTX_EINVAL
    assert _status(ntx, "ntx_gemv_q", 0, None, 4, 256, p, p, None) == ntx.NTX_EINVAL
    assert _status(ntx, "ntx_gemv_q", 0, p, 0, 256, p, p, None) == ntx.NTX_EINVAL
    assert _status(ntx, "ntx_gemv_q", 2, p, 4, 128, p, p, None) == ntx.NTX_EINVAL
    assert _status(ntx, "ntx_gemv_q", 0, p, 4, 256, p + 2, p, None) == ntx.NTX_EINVAL
    assert "aligned" in ntx.ntx_last_error()
    assert _status(ntx, "ntx_dequant_q", 3, p, 1, 100, p, None) == ntx.NTX_EINVAL
    # tiled layouts take whole 16-row groups
    assert _status(ntx, "ntx_gemv_q", 16, p, 40, 256, p, p, None) == ntx.NTX_EINVAL
    # unknown codes, and tiled forms that do not exist (F16, F32), are rejected, not misread
    for q in (7, 8, 15, 21, 22, 23):
        assert _status(ntx, "ntx_gemv_q", q, p, 16, 256, p, p, None) == ntx.NTX_EINVAL
        assert ntx.lib().ntx_row_bytes(q, 256) == 0
    assert ntx.lib().ntx_row_bytes(ntx.NTX_Q5_K, 256) == 176
    assert ntx.lib().ntx_row_bytes(ntx.NTX_Q5_K_T, 512) == 352
    assert ntx.lib().ntx_row_bytes(ntx.NTX_Q5_K, 128) == 0
    assert ntx.lib().ntx_row_bytes(ntx.NTX_F16, 3) == 6
    assert ntx.lib().ntx_row_bytes(ntx.NTX_F32, 7) == 28


def test_ops_reject_bad_arguments(ntx):
    p = 0x10000
    assert _status(ntx, "ntx_rmsnorm", None, p, p, 8, ctypes.c_float(1e-5), None) == ntx.NTX_EINVAL
    assert _status(ntx, "ntx_rmsnorm", p, p, p, 0, ctypes.c_float(1e-5), None) == ntx.NTX_EINVAL
    assert _status(ntx, "ntx_rope", p, p, 4, 2, 127, 0, ctypes.c_float(1e4), None) == ntx.NTX_EINVAL
    assert _status(ntx, "ntx_rope", p, p, 4, 2, 128, -1, ctypes.c_float(1e4), None) == ntx.NTX_EINVAL
    assert _status(ntx, "ntx_softmax", p, p, 0, None) == ntx.NTX_EINVAL
    assert _status(ntx, "ntx_swiglu", p, None, p, 4, None) == ntx.NTX_EINVAL
    assert _status(ntx, "ntx_argmax", p, 0, p, None) == ntx.NTX_EINVAL
    assert _status(ntx, "ntx_embed", 9, p, 10, 256, p, p, None) == ntx.NTX_EINVAL


def test_attention_rejects_bad_arguments(ntx):
    p = 0x10000
    f = ntx.lib().ntx_attn_decode
    ws = ntx.ntx_attn_workspace_bytes(32, 8, 128, 4097)
    assert ws > 0
    assert ntx.ntx_attn_workspace_bytes(30, 8, 128, 4097) == 0
    assert f(p, p, p, p, 32, 8, 64, 10, 4097, p, ws, None) == ntx.NTX_EUNSUPPORTED      # head_dim
    assert f(p, p, p, p, 24, 8, 128, 10, 4097, p, ws, None) == ntx.NTX_EUNSUPPORTED     # 3 q heads per kv head
    assert f(p, p, p, p, 32, 8, 128, 0, 4097, p, ws, None) == ntx.NTX_EINVAL            # n_ctx
    assert f(p, p, p, p, 32, 8, 128, 4098, 4097, p, ws, None) == ntx.NTX_EINVAL         # n_ctx > max_ctx
    assert f(p, p, p, p, 32, 8, 128, 10, 4097, p, 16, None) == ntx.NTX_EINVAL           # workspace too small
    assert f(p + 4, p, p, p, 32, 8, 128, 10, 4097, p, ws, None) == ntx.NTX_EINVAL       # alignment


def test_model_create_rejects_bad_descriptors(ntx):
    h = ctypes.c_void_p(0)
    assert ntx.lib().ntx_model_create(None, ctypes.byref(h)) == ntx.NTX_EINVAL
    layers = (ntx.LayerDesc * 1)()
    p = 0x10000
    layers[0] = ntx.LayerDesc(p, p, p, p, p, p, p, p, p)
    good = dict(n_layers=1, hidden=256, n_q_heads=2, n_kv_heads=1, head_dim=128, ffn=512, vocab=10, max_ctx=8,
                rms_eps=1e-5, rope_theta=1e4, qtype=0, tok_embd=p, out_norm=p, output=p,
                layers=ctypes.cast(layers, ctypes.POINTER(ntx.LayerDesc)), n_resident=1)

    def create(**kw):
        d = ntx.ModelDesc(**dict(good, **kw))
        return ntx.lib().ntx_model_create(ctypes.byref(d), ctypes.byref(h))

    assert create(head_dim=64) == ntx.NTX_EUNSUPPORTED
    assert create(n_q_heads=3, n_kv_heads=2) == ntx.NTX_EINVAL
    assert create(n_q_heads=3) == ntx.NTX_EUNSUPPORTED
    assert create(hidden=100) == ntx.NTX_EINVAL
    assert create(n_resident=2) == ntx.NTX_EINVAL
    assert create(qtype=9) == ntx.NTX_EINVAL
    assert create(tok_embd=p + 8) == ntx.NTX_EINVAL
    assert create(qtype=3, hidden=256, ffn=256) == ntx.NTX_EUNSUPPORTED      # Q6_K row of 210 B: not 16-byte multiple
    layers[0] = ntx.LayerDesc(p, p, None, p, p, p, p, p, p)
    assert create() == ntx.NTX_EINVAL
    assert h.value is None


def test_decode_entry_points_reject_null_model(ntx):
    assert ntx.lib().ntx_decode_step(None, 0, 0, 0x10000, None) == ntx.NTX_EINVAL
    assert ntx.lib().ntx_stream_layers(None, 0, 0, 0x10000, None, None, 0) == ntx.NTX_EINVAL
    assert ntx.lib().ntx_model_destroy(None) == ntx.NTX_EINVAL
    assert ntx.lib().ntx_device_error(None) == ntx.NTX_EINVAL


def test_read_probe_rejects_bad_arguments(ntx):
    p = 1 << 20
    assert _status(ntx, "ntx_stream_read_probe", None, 256, None) == ntx.NTX_EINVAL
    assert _status(ntx, "ntx_stream_read_probe", p, 100, None) == ntx.NTX_EINVAL       # not a multiple of 16
    assert _status(ntx, "ntx_stream_read_probe", p + 8, 256, None) == ntx.NTX_EINVAL   # not 16-byte aligned


def test_repack_rejects_bad_arguments(ntx):
    p = 0x10000
    f = ntx.lib().ntx_repack_q
    assert f(ntx.NTX_Q8_0_T, p, p * 4, 16, 256, None) == ntx.NTX_EINVAL     # already tiled
    assert f(ntx.NTX_Q8_0, p, p * 4, 16, 48, None) == ntx.NTX_EINVAL        # not whole blocks
    assert f(ntx.NTX_Q6_K, p, p * 4, 16, 128, None) == ntx.NTX_EINVAL       # Q6_K unit = 256
    assert f(ntx.NTX_Q8_0, p, p * 4, 8, 256, None) == ntx.NTX_EINVAL        # rows not a multiple of 16
    assert f(ntx.NTX_Q4_0, p, p + 100, 16, 256, None) == ntx.NTX_EINVAL     # overlap
    assert f(ntx.NTX_Q4_0, None, p, 16, 256, None) == ntx.NTX_EINVAL
    assert ntx.ntx_row_bytes(ntx.NTX_Q6_K_T, 2048) == 1680
    assert ntx.ntx_row_bytes(ntx.NTX_Q6_K_T, 256) == 210
    assert ntx.ntx_row_bytes(ntx.NTX_Q6_K_T, 128) == 0
    assert ntx.ntx_row_bytes(ntx.NTX_Q8_0_T, 32) == 34
    assert ntx.ntx_block_elems(ntx.NTX_Q4_K_T) == 256
