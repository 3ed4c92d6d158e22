"""Helpers shared by the GPU parity tests."""
import numpy as np
import pytest
import torch

REL_L2_TOL = 5e-3     # per token row, layer outputs and logits
MARGIN_FLAG = 1e-4    # routing / argmax decisions closer than this are flagged, not failed


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from moe_decode_weight_router_b200 import build
    build.build()


def rel_l2_rows(got: np.ndarray, ref: np.ndarray) -> np.ndarray:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    return np.linalg.norm(got - ref, axis=-1) / np.maximum(np.linalg.norm(ref, axis=-1), 1e-300)


def assert_rows_close(got, ref, tol=REL_L2_TOL, what=""):
    r = rel_l2_rows(got, ref)
    assert np.all(np.isfinite(r)) and np.all(r <= tol), f"{what} relative L2 per row {r} > {tol}"
    return r
