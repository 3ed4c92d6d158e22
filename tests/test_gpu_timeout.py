"""The persistent step's bounded device waits, driven to expiry on purpose.

Every spin-wait in the decode step is bounded: after the limit it records
MOE_ERR_TIMEOUT in the workspace status word and the kernels return early instead of
hanging the GPU.  Here one layer's residual is held back (nothing ever publishes it)
and the wait limit is shortened to 1 ms, so the next layer's wait can only run out.
The call must come back with MOE_ERR_TIMEOUT, and the same workspace must then serve a
normal step that matches the oracle.  No fault is involved: the held counter simply
never reaches its target."""
import time

import pytest
import torch

from moe_decode_weight_router_b200 import decode_step, decode_step_launch_names, synth, workspace_status
from tests._gpu import need_gpu
from tests.test_gpu_decode_step import _check_step, _model

pytestmark = pytest.mark.gpu

MOE_ERR_TIMEOUT = 7


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


@pytest.mark.parametrize("M", [1, 4])
def test_persistent_step_wait_times_out_and_recovers(M):
    S = synth.TINY
    model = _model(S, 4, 1000, 61 + M)
    x = synth.tokens(M, S.H, 61 + M, device="cuda")
    assert decode_step_launch_names(model, M)[0] == "k_step"
    t0 = time.time()
    res = decode_step(model, x, wait_limit_ns=1_000_000, hold_layer=1)
    torch.cuda.synchronize()
    assert time.time() - t0 < 30.0  # the step returned (each wait gives up after 1 ms)
    assert workspace_status(res["ws"]) == MOE_ERR_TIMEOUT
    # the next call clears the control block: the same workspace serves a normal step
    ok = decode_step(model, x, trace=True, ws=res["ws"])
    torch.cuda.synchronize()
    assert workspace_status(ok["ws"]) == 0
    _check_step(model, S, x, ok, range(4))
