"""GPU parity of the FP8 LM head: the online quantiser (bit-exact bytes and
scales) and the GEMV + argmax (logits within tolerance, argmax exact)."""
import numpy as np
import pytest
import torch

import oracle
from moe_decode_weight_router_b200 import lm_head_fp8_gemv, lm_head_fp8_quantize, synth
from tests._gpu import MARGIN_FLAG, assert_rows_close, need_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def test_quantize_bit_exact_small_with_special_rows():
    V, H = 1000, 256
    w = synth.lm_head(V, H, 0, device="cuda")
    w[3].zero_()                                   # amax = 0 -> scale 1, codes 0
    w[4] = -w[4]
    w[5, 7] = 30.0                                 # one large outlier
    w[6] = torch.full((H,), -1e-30).to(torch.bfloat16)  # tiny negatives (rounding towards -0)
    q, s = lm_head_fp8_quantize(w)
    torch.cuda.synchronize()
    q_ref, s_ref = oracle.lmhead_quantize(synth.bits(w))
    np.testing.assert_array_equal(s.cpu().numpy(), s_ref)
    np.testing.assert_array_equal(q.cpu().numpy(), q_ref)


def test_quantize_bit_exact_full_size_sampled_rows():
    V, H = synth.VOCAB, 2560
    w = synth.lm_head(V, H, 1, device="cuda")
    q, s = lm_head_fp8_quantize(w)
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([np.random.default_rng(0).integers(0, V, 48), [0, 1, V - 2, V - 1]]))
    ridx = torch.from_numpy(rows).cuda()
    q_ref, s_ref = oracle.lmhead_quantize(synth.bits(w.index_select(0, ridx)))
    np.testing.assert_array_equal(s.index_select(0, ridx).cpu().numpy(), s_ref)
    np.testing.assert_array_equal(q.index_select(0, ridx).cpu().numpy(), q_ref)
    assert q.numel() * q.element_size() * 2 == w.numel() * w.element_size()  # half of the BF16 bytes


@pytest.mark.parametrize("V,H,M", [(1000, 256, 1), (1000, 256, 5), (4099, 512, 8), (synth.VOCAB, 2560, 1),
                                   (synth.VOCAB, 2560, 4)])
def test_gemv_parity(V, H, M):
    q = synth.e4m3_codes((V, H), V + M, device="cuda")
    s = synth.row_scales(V, V + M, device="cuda")
    x = synth.tokens(M, H, V + M, device="cuda")
    logits, am = lm_head_fp8_gemv(x, q, s)
    torch.cuda.synchronize()
    ref, am_ref, gap = oracle.lmhead_logits(synth.bits(x), synth.bits(q), s.cpu().numpy())
    assert_rows_close(logits.cpu().numpy(), ref, what="logits")
    am = am.cpu().numpy()
    for t in range(M):
        if gap[t] >= MARGIN_FLAG * max(1.0, abs(ref[t, am_ref[t]])):
            assert am[t] == am_ref[t], (t, am[t], am_ref[t])


def test_gemv_argmax_ties_and_no_logits():
    # small codes (|value| <= 1) everywhere except rows 123, 777, 1500, 1999, which all
    # hold 448 (0x7E); equal row scales and x = 1 make those four rows tie for the maximum
    V, H = 2000, 256
    q = synth.e4m3_codes((V, H), 3, device="cuda") & 0xBF   # clears the exponent MSB: |v| <= 1.875
    s = torch.full((V,), 1e-3, dtype=torch.float32, device="cuda")
    for r in (123, 777, 1500, 1999):
        q[r] = 0x7E
    x = torch.ones((1, H), dtype=torch.bfloat16, device="cuda")
    logits, am = lm_head_fp8_gemv(x, q, s)
    _, am2 = lm_head_fp8_gemv(x, q, s, want_logits=False)
    torch.cuda.synchronize()
    lg = logits.cpu().numpy()[0]
    assert lg[123] == lg[777] == lg[1500] == lg[1999] and lg.argmax() == 123
    assert am.item() == 123 and am2.item() == 123
    _, am_ref, _ = oracle.lmhead_logits(synth.bits(x), synth.bits(q), s.cpu().numpy())
    assert am_ref[0] == 123
