"""CPU oracle of the batch-1 quantized decode step (ctypes wrapper over oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the
benchmark's CPU-baseline / reference leg, never by the product path.  It shares
no code with the CUDA library; its inputs come from the seeded generator in
synth/ (or from the tests' own hand-built blocks).

Parity pins: every function here is checked against values fixed by its
definition or by the mathematics (tests/test_oracle_*.py): fp16 against the
IEEE tables, hand-built quant blocks, exact-integer GEMVs, closed forms and
invariants for RMSNorm, RoPE, softmax, SwiGLU and attention, and structural
special cases of the decode step.  The composed full-depth decode step has no
value printed by the pages; it is pinned through its parts and those special
cases only.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(_HERE, "liboracle.so")

Q8_0, Q4_0, Q4_K, Q6_K, Q5_K, F16, F32 = 0, 1, 2, 3, 4, 5, 6
BLOCK = {Q8_0: (32, 34), Q4_0: (32, 18), Q4_K: (256, 144), Q6_K: (256, 210), Q5_K: (256, 176), F16: (1, 2),
         F32: (1, 4)}


def build(force: bool = False) -> str:
    src = os.path.join(_HERE, "oracle.c")
    hdr = os.path.join(_HERE, "oracle.h")
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < max(os.path.getmtime(src),
                                                                      os.path.getmtime(hdr)):
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                               "-Wall", "-o", LIB, src, "-lm"])
    return LIB


class Dims(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("ffn", ctypes.c_int32), ("max_ctx", ctypes.c_int32),
                ("rms_eps", ctypes.c_float), ("rope_theta", ctypes.c_double)]


class Layer(ctypes.Structure):
    _fields_ = [("qtype", ctypes.c_int32 * 4), ("attn_norm", ctypes.c_void_p), ("w_qkv", ctypes.c_void_p),
                ("w_o", ctypes.c_void_p), ("ffn_norm", ctypes.c_void_p), ("w_gate", ctypes.c_void_p),
                ("w_up", ctypes.c_void_p), ("w_down", ctypes.c_void_p), ("k_cache", ctypes.c_void_p),
                ("v_cache", ctypes.c_void_p)]


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        vp, i64, i32, ci = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int
        L.orc_f16_to_f32.argtypes = [ctypes.c_uint16]
        L.orc_f16_to_f32.restype = ctypes.c_float
        L.orc_f32_to_f16.argtypes = [ctypes.c_float]
        L.orc_f32_to_f16.restype = ctypes.c_uint16
        L.orc_dequant.argtypes = [ci, vp, i64, i64, vp]
        L.orc_gemv.argtypes = [ci, vp, i64, i64, vp, vp]
        L.orc_rmsnorm.argtypes = [vp, vp, vp, i64, ctypes.c_float]
        L.orc_rmsnorm.restype = None
        L.orc_rope.argtypes = [vp, vp, ci, ci, ci, i32, ctypes.c_double]
        L.orc_rope.restype = None
        L.orc_attn_decode.argtypes = [vp, vp, vp, vp, ci, ci, ci, i32, i32]
        L.orc_attn_decode.restype = None
        L.orc_swiglu.argtypes = [vp, vp, vp, i64]
        L.orc_swiglu.restype = None
        L.orc_softmax.argtypes = [vp, vp, i64]
        L.orc_softmax.restype = None
        L.orc_decode_layer.argtypes = [ctypes.POINTER(Dims), ctypes.POINTER(Layer), vp, i32]
        L.orc_embed.argtypes = [ci, vp, i64, i32, vp]
        L.orc_lm_head.argtypes = [ci, vp, vp, i64, i64, ctypes.c_float, vp, vp]
        L.orc_set_threads.argtypes = [ci]
        L.orc_set_threads.restype = None
        L.orc_get_threads.restype = ci
        _lib = L
    return _lib


def _p(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be contiguous"
    return a.ctypes.data


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32)


def set_threads(n: int) -> None:
    lib().orc_set_threads(int(n))


def threads() -> int:
    return int(lib().orc_get_threads())


def f16_to_f32(bits: int) -> float:
    return float(lib().orc_f16_to_f32(int(bits)))


def f32_to_f16(x: float) -> int:
    return int(lib().orc_f32_to_f16(float(x)))


def f16_to_f32_array(bits: np.ndarray) -> np.ndarray:
    f = lib().orc_f16_to_f32
    return np.array([f(int(b)) for b in np.asarray(bits).ravel()], dtype=np.float32).reshape(np.shape(bits))


def f32_to_f16_array(x: np.ndarray) -> np.ndarray:
    f = lib().orc_f32_to_f16
    return np.array([f(float(v)) for v in np.asarray(x, dtype=np.float32).ravel()],
                    dtype=np.uint16).reshape(np.shape(x))


def dequant(qtype: int, W: np.ndarray, rows: int, cols: int) -> np.ndarray:
    W = np.ascontiguousarray(W, dtype=np.uint8)
    out = np.empty((rows, cols), dtype=np.float32)
    if lib().orc_dequant(qtype, _p(W), rows, cols, _p(out)) != 0:
        raise ValueError("bad qtype / cols")
    return out


def gemv(qtype: int, W: np.ndarray, rows: int, cols: int, x) -> np.ndarray:
    W = np.ascontiguousarray(W, dtype=np.uint8)
    x = _f32(x)
    assert x.size == cols
    y = np.empty(rows, dtype=np.float32)
    if lib().orc_gemv(qtype, _p(W), rows, cols, _p(x), _p(y)) != 0:
        raise ValueError("bad qtype / cols")
    return y


def rmsnorm(x, w, eps: float) -> np.ndarray:
    x, w = _f32(x), _f32(w)
    y = np.empty_like(x)
    lib().orc_rmsnorm(_p(x), _p(w), _p(y), x.size, eps)
    return y


def rope(q, k, n_q_heads: int, n_kv_heads: int, head_dim: int, pos: int, theta: float):
    q, k = _f32(q).copy(), _f32(k).copy()
    lib().orc_rope(_p(q), _p(k), n_q_heads, n_kv_heads, head_dim, pos, theta)
    return q, k


def attn_decode(q, k_cache: np.ndarray, v_cache: np.ndarray, n_q_heads: int, n_kv_heads: int, head_dim: int,
                n_ctx: int, max_ctx: int) -> np.ndarray:
    """k_cache / v_cache: fp16 bit patterns (uint16) [n_kv_heads, max_ctx, head_dim]."""
    q = _f32(q)
    kc = np.ascontiguousarray(k_cache, dtype=np.uint16)
    vc = np.ascontiguousarray(v_cache, dtype=np.uint16)
    out = np.empty(n_q_heads * head_dim, dtype=np.float32)
    lib().orc_attn_decode(_p(q), _p(kc), _p(vc), _p(out), n_q_heads, n_kv_heads, head_dim, n_ctx, max_ctx)
    return out


def swiglu(gate, up) -> np.ndarray:
    g, u = _f32(gate), _f32(up)
    out = np.empty_like(g)
    lib().orc_swiglu(_p(g), _p(u), _p(out), g.size)
    return out


def softmax(x) -> np.ndarray:
    x = _f32(x)
    y = np.empty_like(x)
    lib().orc_softmax(_p(x), _p(y), x.size)
    return y


def embed(qtype: int, E_row_or_table: np.ndarray, hidden: int, token: int) -> np.ndarray:
    E = np.ascontiguousarray(E_row_or_table, dtype=np.uint8)
    h = np.empty(hidden, dtype=np.float32)
    if lib().orc_embed(qtype, _p(E), hidden, token, _p(h)) != 0:
        raise ValueError("bad embedding arguments")
    return h


def lm_head(qtype: int, out_norm, W_out: np.ndarray, vocab: int, hidden: int, eps: float, h) -> np.ndarray:
    n, h = _f32(out_norm), _f32(h)
    W = np.ascontiguousarray(W_out, dtype=np.uint8)
    logits = np.empty(vocab, dtype=np.float32)
    if lib().orc_lm_head(qtype, _p(n), _p(W), vocab, hidden, eps, _p(h), _p(logits)) != 0:
        raise ValueError("bad lm head arguments")
    return logits


def decode_layer(dims: Dims, qtype, h: np.ndarray, pos: int, attn_norm, w_qkv, w_o, ffn_norm, w_gate, w_up,
                 w_down, k_cache: np.ndarray, v_cache: np.ndarray) -> None:
    """One layer in place on h (fp32) and on the fp16-bit caches (uint16).  qtype: the format
    of every matrix, or four formats (QKV, O, gate and up, down)."""
    keep = [_f32(attn_norm), np.ascontiguousarray(w_qkv), np.ascontiguousarray(w_o), _f32(ffn_norm),
            np.ascontiguousarray(w_gate), np.ascontiguousarray(w_up), np.ascontiguousarray(w_down)]
    assert h.dtype == np.float32 and h.flags["C_CONTIGUOUS"]
    assert k_cache.dtype == np.uint16 and v_cache.dtype == np.uint16
    qts = [int(qtype)] * 4 if np.isscalar(qtype) else [int(v) for v in qtype]
    assert len(qts) == 4
    L = Layer((ctypes.c_int32 * 4)(*qts), *[_p(a) for a in keep], _p(k_cache), _p(v_cache))
    if lib().orc_decode_layer(ctypes.byref(dims), ctypes.byref(L), _p(h), pos) != 0:
        raise ValueError("bad decode layer arguments")


def dims_of(spec) -> Dims:
    return Dims(spec.hidden, spec.n_q_heads, spec.n_kv_heads, spec.head_dim, spec.ffn, spec.max_ctx,
                spec.rms_eps, spec.rope_theta)
