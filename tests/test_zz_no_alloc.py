"""The allocation-free LM-head entry point (lm_head_fp8_gemv_noalloc) against the
workspace entry point (lm_head_fp8_gemv), through the C ABI.

Callers that cannot provide scratch memory use the variant whose control block is a
static device array in the library; it must give the same logits and argmax, on a
first and a second call in a row (the second finds the block dirty from the first).
This file is collected last so that a failure here leaves every other test run."""
import ctypes

import numpy as np
import pytest
import torch

from moe_decode_weight_router_b200 import _abi, lm_head_fp8_gemv, synth
from tests._gpu import REL_L2_TOL, need_gpu, rel_l2_rows

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("V,H,M", [(4099, 512, 3), (synth.VOCAB, 2560, 4)])
def test_noalloc_matches_workspace_entry_on_two_calls(V, H, M):
    need_gpu()
    lib = _abi.load()
    q = synth.e4m3_codes((V, H), 77 + M, device="cuda")
    s = synth.row_scales(V, 77 + M, device="cuda")
    x = synth.tokens(M, H, 77 + M, device="cuda")
    ref_logits, ref_am = lm_head_fp8_gemv(x, q, s)
    stream = torch.cuda.current_stream()
    for call in range(2):
        logits = torch.full((M, V), float("nan"), dtype=torch.float32, device="cuda")
        am = torch.full((M,), -1, dtype=torch.int32, device="cuda")
        st = lib.lm_head_fp8_gemv_noalloc(ctypes.c_void_p(x.data_ptr()), M, V, H, ctypes.c_void_p(q.data_ptr()),
                                          ctypes.c_void_p(s.data_ptr()), ctypes.c_void_p(logits.data_ptr()),
                                          ctypes.c_void_p(am.data_ptr()), ctypes.c_void_p(stream.cuda_stream))
        assert st == 0, lib.moe_status_string(st)
        torch.cuda.synchronize()
        r = rel_l2_rows(logits.cpu().numpy(), ref_logits.cpu().numpy())
        assert np.all(r <= REL_L2_TOL), (call, r)
        assert np.array_equal(am.cpu().numpy(), ref_am.cpu().numpy()), call
    # sizes beyond the static block are refused before anything is launched
    assert lib.lm_head_fp8_gemv_noalloc(ctypes.c_void_p(x.data_ptr()), 9, V, H, ctypes.c_void_p(q.data_ptr()),
                                        ctypes.c_void_p(s.data_ptr()), None, ctypes.c_void_p(am.data_ptr()),
                                        ctypes.c_void_p(stream.cuda_stream)) == 2
