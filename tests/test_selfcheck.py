"""The start-up self-check: its input generator, its compiled-in expected values, the
entry point's host-side validation, and (on a GPU) a passing run."""
import os
import subprocess
import sys
import warnings

import numpy as np
import pytest

from moe_decode_weight_router_b200 import _abi, build, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INC = os.path.join(ROOT, "moe_decode_weight_router_b200", "csrc", "selfcheck_expected.inc")


def test_splitmix64_matches_published_check_values():
    want = [int(l) for l in open(os.path.join(ROOT, "tests", "golden", "splitmix64_seed1234567.txt"))
            if l.strip() and not l.startswith("#")]
    gamma = np.uint64(0x9E3779B97F4A7C15)
    with warnings.catch_warnings():
        warnings.simplefilter("ignore")  # uint64 wrap-around is the definition
        got = [int(synth.splitmix64(np.uint64(1234567) + np.uint64(k) * gamma)) for k in range(len(want))]
    assert got == want


def test_selfcheck_inputs_follow_their_recipe():
    d = synth.selfcheck_inputs()
    S = synth.SELFCHECK
    assert d["x"].shape == (synth.SELFCHECK_M, S.H) and d["w13c"].shape == (S.E, 2 * S.I, S.H // 2)
    ex = (d["x"] >> 7) & 0xFF
    assert ex.min() >= 125 and ex.max() <= 128
    ew = (d["wr"] >> 7) & 0xFF
    assert ew.min() >= 119 and ew.max() <= 122
    assert d["w13s"].min() >= 120 and d["w13s"].max() <= 127
    assert not np.any((d["lm_q"] & 0x7F) == 0x7F)
    e = np.log2(d["lm_s"].astype(np.float64))
    assert np.all(e == np.round(e)) and e.min() >= -13 and e.max() <= -8
    # element 0 of the router weight is the generator's value at counter base + 2 * 2^32
    r = int(synth.splitmix64(np.uint64(synth.SELFCHECK_BASE + (2 << 32))))
    assert int(d["wr"][0, 0]) == ((r >> 63) << 15) | ((119 + ((r >> 56) & 3)) << 7) | (r & 0x7F)


def test_compiled_expected_values_come_from_the_oracle():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "oracle", "selfcheck_expected.py")],
                         capture_output=True, text=True, check=True).stdout
    assert out.strip() == open(INC).read().strip()


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _abi.load()


def test_selfcheck_validation(lib):
    need = lib.moe_selfcheck_workspace_bytes()
    assert need > 0 and need % 256 == 0
    fail, rel = _abi.ctypes.c_int(-1), _abi.ctypes.c_float(-1.0)
    ref = _abi.ctypes.byref
    assert lib.moe_selfcheck(None, need, None, ref(fail), ref(rel)) == 1
    assert fail.value == 0 and rel.value == 0.0
    A = 0x7f0000001000
    assert lib.moe_selfcheck(A + 8, need, None, None, None) == 3
    assert lib.moe_selfcheck(A, need - 1, None, None, None) == 4
    assert lib.moe_status_string(8).decode() == "MOE_ERR_SELFCHECK"


@pytest.mark.gpu
def test_selfcheck_passes_on_the_gpu():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from moe_decode_weight_router_b200 import moe_selfcheck
    st, fail, rel = moe_selfcheck()
    assert (st, fail) == (0, 0), (st, fail, rel)
    assert 0.0 <= rel <= 5e-3
    st2, fail2, _ = moe_selfcheck()  # a second run on fresh workspace agrees
    assert (st2, fail2) == (0, 0)
