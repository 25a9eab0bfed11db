"""Oracle decode step of a whole synthetic model (TEST INFRASTRUCTURE ONLY).

Drives the C oracle layer by layer; each layer's packed weights, norm weights
and prefilled fp16 KV cache are regenerated on the host from the seed (synth/),
so host memory holds one layer at a time even for the 70B shapes.
"""
from __future__ import annotations

import numpy as np

import synth
from synth import GLOBAL_LAYER, ModelSpec, tensor_id

from . import decode_layer, dims_of, embed, lm_head


def layer_tensors(spec: ModelSpec, layer: int) -> dict:
    """Host copies of one layer's tensors, generated from the seed."""
    s, hd = spec.seed, spec.head_dim
    t = {}
    for kind in ("w_qkv", "w_o", "w_gate", "w_up", "w_down"):
        rows, cols, qp, q = spec.packed(kind, layer)
        t[kind] = synth.blocks_host(q, s, tensor_id(layer, kind), rows, cols, qp)
    for kind in ("attn_norm", "ffn_norm"):
        t[kind] = synth.uniform_f32_host(s, tensor_id(layer, kind), spec.hidden, *synth.NORM_W)
    n = spec.n_kv_heads * spec.max_ctx * hd
    for kind in ("k_cache", "v_cache"):
        t[kind] = synth.normal_f16_host(s, tensor_id(layer, kind), n).reshape(spec.n_kv_heads, spec.max_ctx, hd)
    return t


def embedding_row(spec: ModelSpec, token: int) -> np.ndarray:
    rows, cols, qp, q = spec.packed("tok_embd")
    row = synth.blocks_host(q, spec.seed, tensor_id(GLOBAL_LAYER, "tok_embd"), 1, cols, qp, row0=token)
    return embed(q, row, spec.hidden, 0)


def head_tensors(spec: ModelSpec, rows=None):
    """(out_norm, packed LM-head rows); rows = (row0, n) for a slice of the vocabulary."""
    vocab, cols, qp, q = spec.packed("output")
    row0, n = (0, vocab) if rows is None else rows
    W = synth.blocks_host(q, spec.seed, tensor_id(GLOBAL_LAYER, "output"), n, cols, qp, row0=row0)
    norm = synth.uniform_f32_host(spec.seed, tensor_id(GLOBAL_LAYER, "out_norm"), spec.hidden, *synth.NORM_W)
    return norm, W


def decode(spec: ModelSpec, pos: int | None = None, token: int | None = None, n_layers: int | None = None,
           head_rows=None, keep_hidden: bool = False, layer_hook=None, skip=()):
    """Logits of one decode step (token at position pos, default n_prefill).

    Returns (logits, hidden_states) where hidden_states[l] is h after layer l
    when keep_hidden is set.  layer_hook(l, tensors) may inspect the layer's
    tensors after the step (e.g. the KV rows written at pos).  Layers in `skip` are
    left out (h passes through them unchanged).
    """
    pos = spec.n_prefill if pos is None else pos
    token = spec.token() if token is None else token
    n_layers = spec.n_layers if n_layers is None else n_layers
    dims = dims_of(spec)
    h = embedding_row(spec, token).copy()
    hidden = []
    for layer in range(n_layers):
        if layer in skip:        # a skipped layer leaves h as it is
            if keep_hidden:
                hidden.append(h.copy())
            continue
        t = layer_tensors(spec, layer)
        qts = [spec.qtype_of(k, layer) for k in ("w_qkv", "w_o", "w_gate", "w_down")]
        decode_layer(dims, qts, h, pos, t["attn_norm"], t["w_qkv"], t["w_o"], t["ffn_norm"], t["w_gate"],
                     t["w_up"], t["w_down"], t["k_cache"], t["v_cache"])
        if keep_hidden:
            hidden.append(h.copy())
        if layer_hook is not None:
            layer_hook(layer, t)
    norm, W = head_tensors(spec, head_rows)
    n_rows = W.shape[0]
    logits = lm_head(spec.qtype_of("output"), norm, W, n_rows, spec.hidden, spec.rms_eps, h)
    return logits, hidden


def layer_similarity(spec: ModelSpec, pos: int | None = None, token: int | None = None):
    """Cosine similarity of each layer's input and output hidden states, in double, from the
    oracle's hidden states (every layer run)."""
    import numpy as np
    token = spec.token() if token is None else token
    h0 = embedding_row(spec, token).astype(np.float64)
    _, hidden = decode(spec, pos=pos, token=token, keep_hidden=True, head_rows=(0, 16))
    out, prev = [], h0
    for h in hidden:
        cur = h.astype(np.float64)
        out.append(float(prev @ cur / np.sqrt((prev @ prev) * (cur @ cur))))
        prev = cur
    return out


def decode_sequence(spec: ModelSpec, tokens, pos0: int):
    """Logits of each of `tokens` decoded one after another at positions pos0, pos0 + 1, ...
    (token i attends to the K / V rows tokens 0..i-1 wrote).  Keeps every layer's tensors in
    host memory: small models only."""
    import numpy as np
    dims = dims_of(spec)
    layers = [layer_tensors(spec, l) for l in range(spec.n_layers)]
    norm, W = head_tensors(spec)
    out = []
    for i, token in enumerate(tokens):
        h = embedding_row(spec, int(token)).copy()
        for layer, t in enumerate(layers):
            qts = [spec.qtype_of(k, layer) for k in ("w_qkv", "w_o", "w_gate", "w_down")]
            decode_layer(dims, qts, h, pos0 + i, t["attn_norm"], t["w_qkv"], t["w_o"], t["ffn_norm"], t["w_gate"],
                         t["w_up"], t["w_down"], t["k_cache"], t["v_cache"])
        out.append(lm_head(spec.qtype_of("output"), norm, W, W.shape[0], spec.hidden, spec.rms_eps, h))
    return np.stack(out)
