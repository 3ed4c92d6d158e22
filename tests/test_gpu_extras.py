"""GPU parity of the entry points beyond the step: the multi-token-prediction verify
window fused into the FP8 head's argmax tail, the BF16 head the FP8 head is compared
against, and temperature / top-k / top-p sampling.  Every expected value comes from
the oracle (verify rule, fp64 logits, fp64 sampler) on the same seeded inputs;
argmax and sampling decisions closer to a tie than the flag thresholds are flagged
rather than failed."""
import numpy as np
import pytest
import torch

import oracle
from moe_decode_weight_router_b200 import lm_head_bf16_gemv, lm_head_fp8_gemv, lm_head_fp8_verify, moe_sample, synth
from tests._gpu import MARGIN_FLAG, assert_rows_close, need_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


@pytest.mark.parametrize("V,H", [(4096, 256), (synth.VOCAB, 2560)])
def test_verify_window(V, H):
    M = 4
    q = synth.e4m3_codes((V, H), 21, device="cuda")
    s = synth.row_scales(V, 21, device="cuda")
    x = synth.tokens(M, H, 21, device="cuda")
    _, am = lm_head_fp8_gemv(x, q, s, want_logits=False)
    am = am.cpu().numpy()
    patterns = [list(am[:3]), [int(am[0]) ^ 1, int(am[1]), int(am[2])], [int(am[0]), int(am[1]) ^ 1, int(am[2])],
                [int(am[0]), int(am[1]), int(am[2]) ^ 1]]
    for d in patterns:
        _, am2, acc = lm_head_fp8_verify(x, q, s, torch.tensor(d, dtype=torch.int32))
        torch.cuda.synchronize()
        np.testing.assert_array_equal(am2.cpu().numpy(), am)
        want = oracle.mtp_accept(am, d)
        got = acc.cpu().numpy()[: len(want)]
        assert list(got) == want, (d, got, want)


@pytest.mark.parametrize("V,H,M", [(2048, 256, 1), (2048, 256, 4), (3001, 512, 8)])
def test_bf16_head_parity(V, H, M):
    w = synth.lm_head(V, H, 9, device="cuda")
    x = synth.tokens(M, H, 9, device="cuda")
    lg, am = lm_head_bf16_gemv(x, w)
    torch.cuda.synchronize()
    o_lg, o_am, gap = oracle.lmhead_logits_bf16(synth.bits(x), synth.bits(w))
    assert_rows_close(lg.cpu().numpy(), o_lg, what="bf16 head logits")
    am = am.cpu().numpy()
    for t in range(M):
        if gap[t] >= MARGIN_FLAG:
            assert am[t] == o_am[t]


def test_bf16_head_full_vocab_against_fp8_head_weights():
    # full vocabulary: argmax against the oracle on every row, logits on sampled columns
    V, H, M = synth.VOCAB, 2560, 4
    w = synth.lm_head(V, H, 10, device="cuda")
    x = synth.tokens(M, H, 10, device="cuda")
    lg, am = lm_head_bf16_gemv(x, w)
    torch.cuda.synchronize()
    o_lg, o_am, gap = oracle.lmhead_logits_bf16(synth.bits(x), synth.bits(w))
    assert_rows_close(lg.cpu().numpy(), o_lg, what="bf16 head logits (full vocabulary)")
    for t in range(M):
        if gap[t] >= MARGIN_FLAG:
            assert am.cpu().numpy()[t] == o_am[t]


@pytest.mark.parametrize("V,M,T,k,p", [(100, 4, 1.0, 29, 0.95), (synth.VOCAB, 4, 0.7, 29, 0.95),
                                       (synth.VOCAB, 2, 1.0, 1, 0.95), (5000, 8, 1.5, 32, 0.5)])
def test_sampling_parity(V, M, T, k, p):
    g = torch.Generator(device="cuda")
    g.manual_seed(V + M)
    logits = torch.randn((M, V), generator=g, device="cuda") * 4.0
    u = torch.rand((M,), generator=g, device="cuda")
    ids = moe_sample(logits, u, temperature=T, top_k=k, top_p=p)
    torch.cuda.synchronize()
    o_ids, margin = oracle.sample(logits.cpu().numpy().astype(np.float64), T, k, p, u.cpu().numpy().astype(np.float64))
    ids = ids.cpu().numpy()
    for t in range(M):
        if margin[t] < 1e-5:
            continue  # flagged: the draw sits on a cumulative boundary
        assert ids[t] == o_ids[t], (t, ids[t], o_ids[t])


def test_sampling_ties_take_lower_index():
    V = 1000
    logits = torch.zeros((2, V), device="cuda")
    logits[:, 100:140] = 5.0                     # 40 tied maxima: top-29 = indices 100..128
    u = torch.tensor([0.0, 0.999], device="cuda")
    ids = moe_sample(logits, u, temperature=1.0, top_k=29, top_p=1.0).cpu().numpy()
    assert ids[0] == 100 and ids[1] == 128
