"""Shared helpers of the GPU parity tests."""
import numpy as np
import pytest

TOL = 2e-3            # max |gpu - oracle| / max |oracle| (normwise), the path's stated bound
GEMV_TIGHT = 1e-4     # fp32-accumulation GEMVs land far inside TOL; a dropped block would not
ELEM_FLOOR = 1e-3     # per-element errors are taken relative to max(|o_i|, ELEM_FLOOR * max |o|)


def rel_err(g, o) -> float:
    """Normwise relative error: max_i |g_i - o_i| / max_i |o_i|."""
    g = np.asarray(g, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    den = np.max(np.abs(o))
    return float(np.max(np.abs(g - o)) / den) if den > 0 else float(np.max(np.abs(g)))


def elem_err(g, o, floor: float = ELEM_FLOOR) -> float:
    """Per-element relative error: max_i |g_i - o_i| / max(|o_i|, floor * max_j |o_j|).

    An output far below the largest one is judged on its own size down to the floor, so
    bits lost on small outputs do not hide under the normwise figure; below the floor an
    output that is a near-cancellation of large terms is judged against the floor."""
    g = np.asarray(g, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    top = np.max(np.abs(o))
    if top == 0:
        return float(np.max(np.abs(g)))
    den = np.maximum(np.abs(o), floor * top)
    return float(np.max(np.abs(g - o) / den))


def need_gpu():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")


def ntx_module():
    need_gpu()
    from quantized_weight_gemv_block_b200 import build
    build.build()
    import synth
    synth.build_dev()
    import quantized_weight_gemv_block_b200 as ntx
    ntx.lib()
    return ntx
