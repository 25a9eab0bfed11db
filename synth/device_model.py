"""Synthetic models placed on the GPU (and in pinned host memory for streamed
layers), filled by the device generator so every byte equals what the host
generator (and hence the CPU oracle) sees.  Input set-up only."""
from __future__ import annotations

import ctypes

import torch

from . import (GLOBAL_LAYER, NORM_W, BLOCK, ModelSpec, blocks_dev, normal_f16_dev, row_bytes, tensor_id,
               uniform_f32_dev)


def _alloc_packed(spec: ModelSpec, kind: str, layer: int, device, host: bool = False,
                  pinned: bool = True) -> torch.Tensor:
    rows, cols, qp, q = spec.packed(kind, layer)
    nbytes = rows * row_bytes(q, cols)
    t = torch.empty(nbytes, dtype=torch.uint8, device=device)
    blocks_dev(t, q, spec.seed, tensor_id(layer, kind), rows, cols, qp)
    if spec.lib_code(q) != q:
        import quantized_weight_gemv_block_b200 as ntx
        tt = torch.empty_like(t)
        ntx.ntx_repack_q(q, t, tt, rows, cols)
        t = tt
    if host:
        h = torch.empty(nbytes, dtype=torch.uint8, pin_memory=pinned)
        h.copy_(t)
        return h
    return t


class DeviceModel:
    """Tensors of a synthetic model and the ntx descriptor pointing at them.

    Layers >= n_resident keep their five packed matrices in host memory (page-locked
    unless host_pinned is False) and are streamed through the ring; everything else
    lives in HBM.
    """

    def __init__(self, spec: ModelSpec, n_resident: int | None = None, device="cuda", n_layers: int | None = None,
                 host_pinned: bool = True):
        import quantized_weight_gemv_block_b200 as ntx

        self.spec = spec
        self.n_layers = spec.n_layers if n_layers is None else n_layers
        self.n_resident = self.n_layers if n_resident is None else n_resident
        s = spec
        self.tok_embd = _alloc_packed(s, "tok_embd", GLOBAL_LAYER, device)
        self.output = _alloc_packed(s, "output", GLOBAL_LAYER, device)
        self.out_norm = torch.empty(s.hidden, dtype=torch.float32, device=device)
        uniform_f32_dev(self.out_norm, s.seed, tensor_id(GLOBAL_LAYER, "out_norm"), *NORM_W)
        self.layers = []
        for l in range(self.n_layers):
            host = l >= self.n_resident
            t = {k: _alloc_packed(s, k, l, device, host=host, pinned=host_pinned)
                 for k in ("w_qkv", "w_o", "w_gate", "w_up", "w_down")}
            for k in ("attn_norm", "ffn_norm"):
                t[k] = torch.empty(s.hidden, dtype=torch.float32, device=device)
                uniform_f32_dev(t[k], s.seed, tensor_id(l, k), *NORM_W)
            for k in ("k_cache", "v_cache"):
                t[k] = torch.empty(s.n_kv_heads * s.max_ctx * s.head_dim, dtype=torch.float16, device=device)
                normal_f16_dev(t[k], s.seed, tensor_id(l, k))
            self.layers.append(t)
        torch.cuda.synchronize()
        self._layer_descs = (ntx.LayerDesc * self.n_layers)()
        for l, t in enumerate(self.layers):
            self._layer_descs[l] = ntx.LayerDesc(*[t[k].data_ptr() for k in ("attn_norm", "w_qkv", "w_o", "ffn_norm",
                                                                            "w_gate", "w_up", "w_down", "k_cache",
                                                                            "v_cache")])
        qts = s.tensor_qtypes()
        if qts is not None:
            qts = qts[:2 + 4 * self.n_layers]
            self._qts = (ctypes.c_int32 * len(qts))(*qts)
            qts_p = ctypes.cast(self._qts, ctypes.POINTER(ctypes.c_int32))
        else:
            qts_p = None
        self.desc = ntx.ModelDesc(self.n_layers, s.hidden, s.n_q_heads, s.n_kv_heads, s.head_dim, s.ffn, s.vocab,
                                  s.max_ctx, s.rms_eps, s.rope_theta, s.lib_code(s.qtype),
                                  self.tok_embd.data_ptr(),
                                  self.out_norm.data_ptr(), self.output.data_ptr(),
                                  ctypes.cast(self._layer_descs, ctypes.POINTER(ntx.LayerDesc)), self.n_resident,
                                  qts_p)
        self.handle = ntx.ntx_model_create(self.desc)

    def reset_caches(self):
        """Restore the prefilled KV caches (the decode step writes position pos)."""
        s = self.spec
        for l, t in enumerate(self.layers):
            for k in ("k_cache", "v_cache"):
                normal_f16_dev(t[k], s.seed, tensor_id(l, k))

    def weight_bytes(self) -> int:
        n = self.tok_embd.numel() * 0 + self.output.numel()
        for t in self.layers:
            n += sum(t[k].numel() for k in ("w_qkv", "w_o", "w_gate", "w_up", "w_down"))
        return n

    def close(self):
        import quantized_weight_gemv_block_b200 as ntx
        if self.handle:
            ntx.ntx_model_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
