"""Seeded synthetic inputs for the quantized decode path.

Input infrastructure shared by the tests, the CPU oracle harness and bench.py.
It produces bytes (packed quant blocks, fp16 / fp32 vectors) from
(seed, tensor id, index) with a counter-based SplitMix64 generator; the same C
header is compiled for the host (gcc) and for the device (nvcc), so a tensor
filled on the GPU is byte-identical to the one filled on the CPU.  No decode
arithmetic lives here.

Recipes (the workloads of the ntransformer news summary: Llama 8B Q8_0 and
Llama 70B Q6_K / Q4_K_M, "Hoja de ruta de desarrollo" and "Rendimiento y
estructura de caché" sections):
  * sweep tensors: every code uniform over its range, fp16 scales d (and dmin)
    uniform in [1e-3, 1e-2], Q4_K scales/mins uniform in 0..63, Q6_K sub-scales
    uniform in -127..127;
  * decode tensors: codes as above, but scales chosen so a GEMV maps a
    unit-RMS input to a roughly unit-RMS output: d uniform in
    [0.5 s, 1.5 s], s = 1 / sqrt(K * E[c^2] * 13/12) where c is the integer
    factor of d in one weight (Q4_K: scales 1..8, mins round(7.5 scale),
    dmin = d; Q6_K: sub-scales 1..16);
  * F16 / F32 weights: an Irwin-Hall(12) value times a power of two (1/4 for the
    sweep, the power of two nearest 1 / sqrt(K) for decode tensors);
  * vectors and the fp16 KV cache: Irwin-Hall(12) stand-in for N(0,1)
    (mean 0, variance 1, support [-6, 6], resolution 2^-16);
  * RMSNorm weights uniform in [0.9, 1.1].
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
HOST_LIB = os.path.join(_HERE, "libsynth_host.so")
DEV_LIB = os.path.join(_HERE, "libsynth_dev.so")

Q8_0, Q4_0, Q4_K, Q6_K, Q5_K, F16, F32 = 0, 1, 2, 3, 4, 5, 6
QTYPE_NAMES = {"q8_0": Q8_0, "q4_0": Q4_0, "q4_k": Q4_K, "q6_k": Q6_K, "q5_k": Q5_K, "f16": F16, "f32": F32}
# (elements per block, bytes per block)
BLOCK = {Q8_0: (32, 34), Q4_0: (32, 18), Q4_K: (256, 144), Q6_K: (256, 210), Q5_K: (256, 176), F16: (1, 2),
         F32: (1, 4)}


def qtype_of(name) -> int:
    if isinstance(name, int):
        return name
    return QTYPE_NAMES[name.lower()]


def row_bytes(qtype: int, cols: int) -> int:
    be, bb = BLOCK[qtype]
    assert cols % be == 0
    return cols // be * bb


class QParams(ctypes.Structure):
    _fields_ = [("d_lo", ctypes.c_uint64), ("d_hi", ctypes.c_uint64), ("d_exp", ctypes.c_int32),
                ("mode", ctypes.c_int32)]


def _scale_range(lo: float, hi: float, mode: int) -> QParams:
    e = math.floor(math.log2(hi)) - 31
    k_lo = math.ceil(lo / 2.0 ** e)
    k_hi = math.floor(hi / 2.0 ** e)
    assert 0 < k_lo <= k_hi and k_hi - k_lo < 2 ** 32
    return QParams(k_lo, k_hi, e, mode)


def sweep_qparams(qtype: int) -> QParams:
    """Scales of the GEMV sweep tensors: d (and dmin) uniform in [1e-3, 1e-2]; F16 / F32
    weights N(0, 1) / 4."""
    if qtype in (F16, F32):
        return QParams(0, 0, -2, 0)
    return _scale_range(1e-3, 1e-2, 0)


def _code_mean_square(qtype: int) -> float:
    """E[c^2] of the integer factor c multiplying d in one weight (decode recipe)."""
    if qtype == Q8_0:
        return float(np.mean(np.arange(-127, 128, dtype=np.float64) ** 2))
    if qtype == Q4_0:
        return float(np.mean((np.arange(16, dtype=np.float64) - 8) ** 2))
    if qtype == Q4_K:
        acc = []
        for s in range(1, 9):
            m = (15 * s + 1) // 2
            acc.append(np.mean((s * np.arange(16, dtype=np.float64) - m) ** 2))
        return float(np.mean(acc))
    if qtype == Q5_K:
        acc = []
        for s in range(1, 5):
            m = (31 * s + 1) // 2
            acc.append(np.mean((s * np.arange(32, dtype=np.float64) - m) ** 2))
        return float(np.mean(acc))
    if qtype == Q6_K:
        sc2 = np.mean(np.arange(1, 17, dtype=np.float64) ** 2)
        return float(sc2 * np.mean((np.arange(64, dtype=np.float64) - 32) ** 2))
    raise ValueError(qtype)


def decode_qparams(qtype: int, k: int) -> QParams:
    """Scales of a decode tensor whose rows have k columns (unit-RMS conditioning; F16 / F32
    weights N(0, 1) times the power of two nearest 1 / sqrt(k))."""
    if qtype in (F16, F32):
        return QParams(0, 0, -int(round(math.log2(math.sqrt(k)))), 1)
    s = 1.0 / math.sqrt(k * _code_mean_square(qtype) * 13.0 / 12.0)
    return _scale_range(0.5 * s, 1.5 * s, 1)


NORM_W = (7549747, 9227469, -23)    # k * 2^-23, k uniform: [0.9, 1.1]

# ---------------------------------------------------------------- libraries


def build_host(force: bool = False) -> str:
    src = os.path.join(_HERE, "synth_host.c")
    if force or not os.path.exists(HOST_LIB) or os.path.getmtime(HOST_LIB) < max(
            os.path.getmtime(src), os.path.getmtime(os.path.join(_HERE, "synth.h"))):
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                               "-Wall", "-o", HOST_LIB, src])
    return HOST_LIB


def build_dev(force: bool = False) -> str:
    src = os.path.join(_HERE, "synth_dev.cu")
    if force or not os.path.exists(DEV_LIB) or os.path.getmtime(DEV_LIB) < max(
            os.path.getmtime(src), os.path.getmtime(os.path.join(_HERE, "synth.h"))):
        subprocess.check_call(["nvcc", "-O2", "-std=c++17", "-shared", "-Xcompiler", "-fPIC", "-gencode",
                               "arch=compute_100a,code=sm_100a", "-fmad=false", "-o", DEV_LIB, src])
    return DEV_LIB


_host = None
_dev = None


def host():
    global _host
    if _host is None:
        lib = ctypes.CDLL(build_host())
        u64, i64, ci = ctypes.c_uint64, ctypes.c_int64, ctypes.c_int
        vp = ctypes.c_void_p
        lib.syn_fill_blocks.argtypes = [ci, u64, u64, i64, i64, ctypes.POINTER(QParams), vp]
        lib.syn_fill_normal_f32.argtypes = [u64, u64, i64, i64, vp]
        lib.syn_fill_normal_f16.argtypes = [u64, u64, i64, i64, vp]
        lib.syn_fill_uniform_f32.argtypes = [u64, u64, i64, i64, u64, u64, ci, vp]
        lib.syn_uniform_index.argtypes = [u64, u64, u64]
        lib.syn_uniform_index.restype = u64
        lib.syn_f16_bits_of_scaled.argtypes = [u64, ci]
        lib.syn_f16_bits_of_scaled.restype = ctypes.c_uint16
        _host = lib
    return _host


def dev():
    global _dev
    if _dev is None:
        lib = ctypes.CDLL(build_dev())
        u64, i64, ci, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
        lib.syn_fill_blocks_dev.argtypes = [ci, u64, u64, i64, i64, ctypes.POINTER(QParams), vp, vp]
        lib.syn_fill_normal_f32_dev.argtypes = [u64, u64, i64, i64, vp, vp]
        lib.syn_fill_normal_f16_dev.argtypes = [u64, u64, i64, i64, vp, vp]
        lib.syn_fill_uniform_f32_dev.argtypes = [u64, u64, i64, i64, u64, u64, ci, vp, vp]
        for f in (lib.syn_fill_blocks_dev, lib.syn_fill_normal_f32_dev, lib.syn_fill_normal_f16_dev,
                  lib.syn_fill_uniform_f32_dev):
            f.restype = ci
        _dev = lib
    return _dev


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


# ---------------------------------------------------------------- host fills

def blocks_host(qtype: int, seed: int, tid: int, rows: int, cols: int, qp: QParams, row0: int = 0) -> np.ndarray:
    """Rows [row0, row0+rows) of a packed [*, cols] tensor, as uint8 [rows, row_bytes]."""
    be, bb = BLOCK[qtype]
    nb_row = cols // be
    out = np.empty((rows, nb_row * bb), dtype=np.uint8)
    host().syn_fill_blocks(qtype, seed, tid, row0 * nb_row, rows * nb_row, ctypes.byref(qp), _ptr(out))
    return out


def normal_f32_host(seed: int, tid: int, n: int, i0: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    host().syn_fill_normal_f32(seed, tid, i0, n, _ptr(out))
    return out


def normal_f16_host(seed: int, tid: int, n: int, i0: int = 0) -> np.ndarray:
    """fp16 bit patterns (uint16)."""
    out = np.empty(n, dtype=np.uint16)
    host().syn_fill_normal_f16(seed, tid, i0, n, _ptr(out))
    return out


def uniform_f32_host(seed: int, tid: int, n: int, k_lo: int, k_hi: int, e: int, i0: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    host().syn_fill_uniform_f32(seed, tid, i0, n, k_lo, k_hi, e, _ptr(out))
    return out


def uniform_index(seed: int, tid: int, n_range: int) -> int:
    return int(host().syn_uniform_index(seed, tid, n_range))


# ---------------------------------------------------------------- device fills (torch tensors)

def _check(rc: int):
    if rc != 0:
        raise RuntimeError(f"synthetic fill kernel failed (cudaError {rc})")


def blocks_dev(out, qtype: int, seed: int, tid: int, rows: int, cols: int, qp: QParams, stream=None, row0=0):
    be, bb = BLOCK[qtype]
    nb_row = cols // be
    assert out.numel() * out.element_size() >= rows * nb_row * bb
    _check(dev().syn_fill_blocks_dev(qtype, seed, tid, row0 * nb_row, rows * nb_row, ctypes.byref(qp),
                                     out.data_ptr(), _stream(stream)))


def normal_f32_dev(out, seed: int, tid: int, stream=None):
    _check(dev().syn_fill_normal_f32_dev(seed, tid, 0, out.numel(), out.data_ptr(), _stream(stream)))


def normal_f16_dev(out, seed: int, tid: int, stream=None):
    _check(dev().syn_fill_normal_f16_dev(seed, tid, 0, out.numel(), out.data_ptr(), _stream(stream)))


def uniform_f32_dev(out, seed: int, tid: int, k_lo: int, k_hi: int, e: int, stream=None):
    _check(dev().syn_fill_uniform_f32_dev(seed, tid, 0, out.numel(), k_lo, k_hi, e, out.data_ptr(),
                                          _stream(stream)))


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream


# ---------------------------------------------------------------- model recipe

GLOBAL_LAYER = -1
KIND = {"tok_embd": 0, "out_norm": 1, "output": 2, "token": 3,
        "attn_norm": 10, "w_qkv": 11, "w_o": 12, "ffn_norm": 13, "w_gate": 14, "w_up": 15, "w_down": 16,
        "k_cache": 17, "v_cache": 18}


def tensor_id(layer: int, kind: str) -> int:
    """Stream id of one tensor of a synthetic model (layer -1 holds the global tensors)."""
    return (layer + 2) * 64 + KIND[kind]


@dataclass
class ModelSpec:
    """Shape and storage formats of a synthetic Llama-architecture model."""
    n_layers: int
    hidden: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    vocab: int
    max_ctx: int
    n_prefill: int          # positions 0..n_prefill-1 of the KV cache hold values; decode runs at pos = n_prefill
    qtype: int
    rms_eps: float = 1e-5
    rope_theta: float = 500000.0
    seed: int = 0
    tiled: bool = False       # weights handed to the library in the tiled layout (same bytes, regrouped)
    mix: str | None = None    # per-tensor formats: None (every tensor in qtype) or "q4_k_m" (below)
    # extra["quiet_layers"]: layers whose O and down projections are scaled by 2^-10 (their
    # output barely changes the hidden state: a planted candidate for the layer skip)
    extra: dict = field(default_factory=dict)

    def qtype_of(self, kind: str, layer: int = GLOBAL_LAYER) -> int:
        """Format of one tensor.  mix "q4_k_m" (a reading of the pages' "Q4_K_M" models, which
        mix formats per tensor without saying how): Q4_K everywhere except the LM head and the
        down projection of every even-numbered layer, which are Q6_K."""
        if self.mix == "q4_k_m":
            return Q6_K if kind == "output" or (kind == "w_down" and layer % 2 == 0) else Q4_K
        return self.qtype

    def lib_code(self, qtype: int) -> int:
        """The library's code of a tensor in `qtype` as this model hands it over (the tiled form
        when the model is tiled; F16 / F32 have none)."""
        return qtype | 16 if self.tiled and qtype not in (F16, F32) else qtype

    def tensor_qtypes(self):
        """Library codes of every tensor (tok_embd, output, then per layer w_qkv, w_o, w_gate and
        w_up, w_down), or None when every tensor has the model's format."""
        if self.mix is None:
            return None
        out = [self.lib_code(self.qtype_of("tok_embd")), self.lib_code(self.qtype_of("output"))]
        for l in range(self.n_layers):
            out += [self.lib_code(self.qtype_of(k, l)) for k in ("w_qkv", "w_o", "w_gate", "w_down")]
        return out

    @property
    def qkv_rows(self) -> int:
        return (self.n_q_heads + 2 * self.n_kv_heads) * self.head_dim

    @property
    def q_dim(self) -> int:
        return self.n_q_heads * self.head_dim

    def layer_weight_bytes(self, layer: int = 0) -> int:
        h, f, q = self.hidden, self.ffn, lambda k: self.qtype_of(k, layer)
        return (self.qkv_rows * row_bytes(q("w_qkv"), h) + h * row_bytes(q("w_o"), self.q_dim)
                + 2 * f * row_bytes(q("w_gate"), h) + h * row_bytes(q("w_down"), f))

    def kv_bytes_per_layer(self) -> int:
        return 2 * self.n_kv_heads * self.max_ctx * self.head_dim * 2

    def token(self) -> int:
        return uniform_index(self.seed, tensor_id(GLOBAL_LAYER, "token"), self.vocab)

    # (rows, cols, scale params, format) of each packed tensor
    def packed(self, kind: str, layer: int = GLOBAL_LAYER):
        h, f, q = self.hidden, self.ffn, self.qtype_of(kind, layer)
        shapes = {"tok_embd": (self.vocab, h, 1),
                  "output": (self.vocab, h, h),
                  "w_qkv": (self.qkv_rows, h, h),
                  "w_o": (h, self.q_dim, self.q_dim),
                  "w_gate": (f, h, h),
                  "w_up": (f, h, h),
                  "w_down": (h, f, f)}
        rows, cols, k = shapes[kind]
        qp = decode_qparams(q, k)
        if kind in ("w_o", "w_down") and layer in self.extra.get("quiet_layers", ()):
            # a near-identity layer: its two residual contributions scaled by 2^-10
            qp = QParams(qp.d_lo, qp.d_hi, qp.d_exp - 10, qp.mode)
        return rows, cols, qp, q


LLAMA_8B_Q8_0 = dict(n_layers=32, hidden=4096, n_q_heads=32, n_kv_heads=8, head_dim=128, ffn=14336,
                     vocab=128256, max_ctx=4097, n_prefill=4096, qtype=Q8_0, rope_theta=500000.0)
LLAMA_70B_Q6_K = dict(n_layers=80, hidden=8192, n_q_heads=64, n_kv_heads=8, head_dim=128, ffn=28672,
                      vocab=128256, max_ctx=8193, n_prefill=8192, qtype=Q6_K, rope_theta=500000.0)
LLAMA_70B_Q4_K = dict(LLAMA_70B_Q6_K, qtype=Q4_K)
LLAMA_70B_Q4_K_M = dict(LLAMA_70B_Q6_K, qtype=Q4_K, mix="q4_k_m")
