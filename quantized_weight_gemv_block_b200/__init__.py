"""Python binding of libntx, the sm_100a batch-1 quantized decode library.

Argument marshalling only: every function forwards to the C ABI of the same
name declared in include/ntx.h; all computation runs in the library's CUDA
kernels.  Tensors are passed as raw device pointers (torch tensors are accepted
and their data_ptr() is used); streams default to torch's current stream.
There is no fallback: if libntx.so is missing, importing a function raises.
"""
from __future__ import annotations

import ctypes
import os

from .build import LIB

NTX_OK, NTX_EINVAL, NTX_EUNSUPPORTED, NTX_ENOMEM, NTX_ECUDA, NTX_ETIMEOUT = range(6)
NTX_Q8_0, NTX_Q4_0, NTX_Q4_K, NTX_Q6_K, NTX_Q5_K, NTX_F16, NTX_F32 = range(7)
NTX_TILED = 16
NTX_Q8_0_T, NTX_Q4_0_T, NTX_Q4_K_T, NTX_Q6_K_T, NTX_Q5_K_T = 16, 17, 18, 19, 20
NTX_GEMV_QKV, NTX_GEMV_O, NTX_GEMV_GATE_UP, NTX_GEMV_DOWN, NTX_GEMV_HEAD = range(5)
NTX_HOST_PATH_NONE, NTX_HOST_PATH_PINNED, NTX_HOST_PATH_REGISTERED, NTX_HOST_PATH_PAGEABLE = range(4)
STATUS_NAMES = {0: "NTX_OK", 1: "NTX_EINVAL", 2: "NTX_EUNSUPPORTED", 3: "NTX_ENOMEM", 4: "NTX_ECUDA",
                5: "NTX_ETIMEOUT"}

# Every symbol of include/ntx.h.
EXPORTS = ("ntx_last_error", "ntx_version", "ntx_row_bytes", "ntx_block_elems", "ntx_device_error", "ntx_gemv_q",
           "ntx_stream_read_probe",
           "ntx_dequant_q", "ntx_repack_q", "ntx_rmsnorm", "ntx_rope", "ntx_attn_decode", "ntx_attn_decode_noalloc", "ntx_attn_workspace_bytes", "ntx_swiglu",
           "ntx_softmax", "ntx_argmax", "ntx_embed", "ntx_model_create", "ntx_model_destroy", "ntx_decode_step",
           "ntx_stream_layers", "ntx_stream_stats", "ntx_model_replay_gemv", "ntx_model_layer_similarity",
           "ntx_model_set_layer_skip", "ntx_plan_resident", "ntx_model_host_path", "ntx_verify_tokens",
           "ntx_speculative_step", "ntx_model_step_launches")


class NtxError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class LayerDesc(ctypes.Structure):
    _fields_ = [("attn_norm", ctypes.c_void_p), ("w_qkv", ctypes.c_void_p), ("w_o", ctypes.c_void_p),
                ("ffn_norm", ctypes.c_void_p), ("w_gate", ctypes.c_void_p), ("w_up", ctypes.c_void_p),
                ("w_down", ctypes.c_void_p), ("k_cache", ctypes.c_void_p), ("v_cache", ctypes.c_void_p)]


class ModelDesc(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int32), ("hidden", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("ffn", ctypes.c_int32),
                ("vocab", ctypes.c_int32), ("max_ctx", ctypes.c_int32), ("rms_eps", ctypes.c_float),
                ("rope_theta", ctypes.c_float), ("qtype", ctypes.c_int32), ("tok_embd", ctypes.c_void_p),
                ("out_norm", ctypes.c_void_p), ("output", ctypes.c_void_p), ("layers", ctypes.POINTER(LayerDesc)),
                ("n_resident", ctypes.c_int32), ("tensor_qtypes", ctypes.POINTER(ctypes.c_int32))]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libntx.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB):
            raise RuntimeError(f"{LIB} is missing: build it with `python -m quantized_weight_gemv_block_b200.build`")
        L = ctypes.CDLL(LIB)
        vp, i64, i32, ci, cf, sz = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int, ctypes.c_float,
                                    ctypes.c_size_t)
        sigs = {
            "ntx_last_error": ([], ctypes.c_char_p),
            "ntx_version": ([], ci),
            "ntx_row_bytes": ([ci, i64], sz),
            "ntx_block_elems": ([ci], ci),
            "ntx_device_error": ([ctypes.POINTER(ctypes.c_uint32)], ci),
            "ntx_gemv_q": ([ci, vp, i64, i64, vp, vp, vp], ci),
            "ntx_stream_read_probe": ([vp, sz, vp], ci),
            "ntx_dequant_q": ([ci, vp, i64, i64, vp, vp], ci),
            "ntx_repack_q": ([ci, vp, vp, i64, i64, vp], ci),
            "ntx_rmsnorm": ([vp, vp, vp, i64, cf, vp], ci),
            "ntx_rope": ([vp, vp, ci, ci, ci, i32, cf, vp], ci),
            "ntx_attn_decode": ([vp, vp, vp, vp, ci, ci, ci, i32, i32, vp, sz, vp], ci),
            "ntx_attn_workspace_bytes": ([ci, ci, ci, i32], sz),
            "ntx_attn_decode_noalloc": ([vp, vp, vp, vp, ci, ci, ci, i32, i32, vp], ci),
            "ntx_swiglu": ([vp, vp, vp, i64, vp], ci),
            "ntx_softmax": ([vp, vp, i64, vp], ci),
            "ntx_argmax": ([vp, i64, vp, vp], ci),
            "ntx_embed": ([ci, vp, i64, i64, vp, vp, vp], ci),
            "ntx_model_create": ([ctypes.POINTER(ModelDesc), ctypes.POINTER(vp)], ci),
            "ntx_model_destroy": ([vp], ci),
            "ntx_decode_step": ([vp, i32, i32, vp, vp], ci),
            "ntx_stream_layers": ([vp, i32, i32, vp, vp, vp, i64], ci),
            "ntx_stream_stats": ([vp, ctypes.POINTER(i64), ctypes.POINTER(cf)], ci),
            "ntx_model_replay_gemv": ([vp, ci, ci, vp, vp], ci),
            "ntx_model_layer_similarity": ([vp, i32, i32, ctypes.POINTER(cf), vp, vp], ci),
            "ntx_model_set_layer_skip": ([vp, ctypes.POINTER(ctypes.c_uint8)], ci),
            "ntx_plan_resident": ([ctypes.POINTER(ModelDesc), sz, ctypes.POINTER(i32), ctypes.POINTER(sz)], ci),
            "ntx_model_host_path": ([vp, ctypes.POINTER(i32)], ci),
            "ntx_verify_tokens": ([vp, ctypes.POINTER(i32), i32, i32, vp, vp, vp], ci),
            "ntx_model_step_launches": ([vp, ctypes.POINTER(i32)], ci),
            "ntx_speculative_step": ([vp, i32, i32, i32, ctypes.POINTER(ctypes.c_uint8), ctypes.POINTER(i32),
                                      ctypes.POINTER(i32), vp, vp, i64], ci),
        }
        for name, (args, res) in sigs.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def _p(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _s(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def check(status: int) -> None:
    if status != NTX_OK:
        raise NtxError(status, lib().ntx_last_error().decode())


def ntx_last_error() -> str:
    return lib().ntx_last_error().decode()


def ntx_version() -> int:
    return lib().ntx_version()


def ntx_row_bytes(qtype: int, cols: int) -> int:
    return lib().ntx_row_bytes(qtype, cols)


def ntx_block_elems(qtype: int) -> int:
    return lib().ntx_block_elems(qtype)


def ntx_device_error() -> int:
    code = ctypes.c_uint32(0)
    check(lib().ntx_device_error(ctypes.byref(code)))
    return code.value


def ntx_gemv_q(qtype, W, rows, cols, x, y, stream=None) -> None:
    check(lib().ntx_gemv_q(qtype, _p(W), rows, cols, _p(x), _p(y), _s(stream)))


def ntx_stream_read_probe(src, nbytes, stream=None) -> None:
    check(lib().ntx_stream_read_probe(_p(src), nbytes, _s(stream)))


def ntx_dequant_q(qtype, W, rows, cols, out, stream=None) -> None:
    check(lib().ntx_dequant_q(qtype, _p(W), rows, cols, _p(out), _s(stream)))


def ntx_repack_q(qtype, W, W_tiled, rows, cols, stream=None) -> None:
    check(lib().ntx_repack_q(qtype, _p(W), _p(W_tiled), rows, cols, _s(stream)))


def ntx_rmsnorm(x, w, y, n, eps, stream=None) -> None:
    check(lib().ntx_rmsnorm(_p(x), _p(w), _p(y), n, eps, _s(stream)))


def ntx_rope(q, k, n_q_heads, n_kv_heads, head_dim, pos, theta, stream=None) -> None:
    check(lib().ntx_rope(_p(q), _p(k), n_q_heads, n_kv_heads, head_dim, pos, theta, _s(stream)))


def ntx_attn_workspace_bytes(n_q_heads, n_kv_heads, head_dim, max_ctx) -> int:
    return lib().ntx_attn_workspace_bytes(n_q_heads, n_kv_heads, head_dim, max_ctx)


def ntx_attn_decode(q, k_cache, v_cache, out, n_q_heads, n_kv_heads, head_dim, n_ctx, max_ctx, workspace,
                    workspace_bytes, stream=None) -> None:
    check(lib().ntx_attn_decode(_p(q), _p(k_cache), _p(v_cache), _p(out), n_q_heads, n_kv_heads, head_dim, n_ctx,
                                max_ctx, _p(workspace), workspace_bytes, _s(stream)))


def ntx_attn_decode_noalloc(q, k_cache, v_cache, out, n_q_heads, n_kv_heads, head_dim, n_ctx, max_ctx,
                            stream=None) -> None:
    check(lib().ntx_attn_decode_noalloc(_p(q), _p(k_cache), _p(v_cache), _p(out), n_q_heads, n_kv_heads, head_dim,
                                        n_ctx, max_ctx, _s(stream)))


def ntx_swiglu(gate, up, out, n, stream=None) -> None:
    check(lib().ntx_swiglu(_p(gate), _p(up), _p(out), n, _s(stream)))


def ntx_softmax(x, y, n, stream=None) -> None:
    check(lib().ntx_softmax(_p(x), _p(y), n, _s(stream)))


def ntx_argmax(x, n, out_index, stream=None) -> None:
    check(lib().ntx_argmax(_p(x), n, _p(out_index), _s(stream)))


def ntx_embed(qtype, E, vocab, hidden, token_dev, h, stream=None) -> None:
    check(lib().ntx_embed(qtype, _p(E), vocab, hidden, _p(token_dev), _p(h), _s(stream)))


def ntx_model_create(desc: ModelDesc) -> int:
    handle = ctypes.c_void_p(0)
    check(lib().ntx_model_create(ctypes.byref(desc), ctypes.byref(handle)))
    return handle.value


def ntx_model_destroy(model: int) -> None:
    check(lib().ntx_model_destroy(model))


def ntx_decode_step(model: int, token: int, pos: int, logits, stream=None) -> None:
    check(lib().ntx_decode_step(model, token, pos, _p(logits), _s(stream)))


def ntx_stream_layers(model: int, token: int, pos: int, logits, compute=None, copy=None, timeout_ms: int = 0) -> None:
    check(lib().ntx_stream_layers(model, token, pos, _p(logits), _s(compute), _s(copy), timeout_ms))


def ntx_stream_stats(model: int):
    b = ctypes.c_int64(0)
    ms = ctypes.c_float(0)
    check(lib().ntx_stream_stats(model, ctypes.byref(b), ctypes.byref(ms)))
    return b.value, ms.value


def ntx_model_replay_gemv(model: int, kind: int, n_launches: int, logits=None, stream=None) -> None:
    check(lib().ntx_model_replay_gemv(model, kind, n_launches, _p(logits), _s(stream)))


def ntx_model_layer_similarity(model: int, token: int, pos: int, n_layers: int, compute=None, copy=None):
    """Cosine similarity of each layer's input and output hidden states (list of floats)."""
    out = (ctypes.c_float * n_layers)()
    check(lib().ntx_model_layer_similarity(model, token, pos, out, _s(compute), _s(copy) if copy is not None else None))
    return list(out)


def ntx_model_set_layer_skip(model: int, skip) -> None:
    """skip: sequence of n_layers flags (nonzero = leave the layer out), or None to clear."""
    if skip is None:
        check(lib().ntx_model_set_layer_skip(model, None))
        return
    arr = (ctypes.c_uint8 * len(skip))(*[1 if v else 0 for v in skip])
    check(lib().ntx_model_set_layer_skip(model, arr))


def ntx_plan_resident(desc: ModelDesc, hbm_budget: int):
    """(n_resident, hbm_bytes): the most leading layers that fit in hbm_budget bytes of HBM."""
    n = ctypes.c_int32(0)
    used = ctypes.c_size_t(0)
    check(lib().ntx_plan_resident(ctypes.byref(desc), hbm_budget, ctypes.byref(n), ctypes.byref(used)))
    return n.value, used.value


def ntx_model_host_path(model: int) -> int:
    p = ctypes.c_int32(0)
    check(lib().ntx_model_host_path(model, ctypes.byref(p)))
    return p.value


def ntx_verify_tokens(model: int, tokens, pos0: int, logits, compute=None, copy=None) -> None:
    """One pass of the full model over len(tokens) tokens at positions pos0..; logits [n, vocab]."""
    arr = (ctypes.c_int32 * len(tokens))(*[int(t) for t in tokens])
    check(lib().ntx_verify_tokens(model, arr, len(tokens), pos0, _p(logits), _s(compute),
                                  _s(copy) if copy is not None else None))


def ntx_speculative_step(model: int, token: int, pos: int, k: int, draft_skip=None, compute=None, copy=None,
                         timeout_ms: int = 0):
    """Draft k - 1 tokens, verify them in one pass; returns the accepted tokens (1..k of them)."""
    out = (ctypes.c_int32 * k)()
    n = ctypes.c_int32(0)
    skip = None if draft_skip is None else (ctypes.c_uint8 * len(draft_skip))(*[1 if v else 0 for v in draft_skip])
    check(lib().ntx_speculative_step(model, token, pos, k, skip, out, ctypes.byref(n), _s(compute),
                                     _s(copy) if copy is not None else None, timeout_ms))
    return list(out[:n.value])


def ntx_model_step_launches(model: int) -> int:
    n = ctypes.c_int32(0)
    check(lib().ntx_model_step_launches(model, ctypes.byref(n)))
    return n.value
