"""Shared helpers of the GPU parity tests."""
import numpy as np
import pytest

TOL = 2e-3            # max |gpu - oracle| / max |oracle| (normwise), the path's stated bound
GEMV_TIGHT = 1e-4     # fp32-accumulation GEMVs land far inside TOL; a dropped block would not


def rel_err(g, o) -> float:
    g = np.asarray(g, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    den = np.max(np.abs(o))
    return float(np.max(np.abs(g - o)) / den) if den > 0 else float(np.max(np.abs(g)))


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
