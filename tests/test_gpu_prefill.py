"""GPU parity of the prefill chunk (one MoE layer for M tokens on the block-scaled
tensor cores) against the CPU oracle.

The MXFP8 quantiser is checked bit for bit; the chunk's routing (ids bit-exact
except flagged near-ties, weights, logits) and its layer output y (relative L2 per
token row <= 5e-3, the oracle evaluated with the GPU's own routing) on a small
shape, on a chunk whose tokens all pick the same experts (more than one 128-token
tile per expert), and at the Ling shape with M = 2048 on a seeded sample of tokens
plus every token of one expert.  Every expected value comes from the oracle on the
same seeded bytes."""
import numpy as np
import pytest
import torch

import oracle
from moe_decode_weight_router_b200 import (moe_experts_workspace_bytes, moe_mxfp4_experts, moe_mxfp8_quantize,
                                           moe_prefill_layer, synth, workspace_status)
from moe_decode_weight_router_b200.binding import moe_prefill_workspace_bytes
from tests._gpu import MARGIN_FLAG, assert_rows_close, need_gpu

pytestmark = pytest.mark.gpu

# Smallest shape the prefill path takes: H and I multiples of 128, E a multiple of 128.
SMALL = synth.LayerShape(H=256, I=128, E=128, k=4, Is=128, e_lo=120, e_hi=127)


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def _fetch(L):
    def fetch(lst):
        idx = torch.tensor(lst, dtype=torch.long, device="cuda")
        return {n: synth.bits(L[n].index_select(0, idx)) for n in ("w13c", "w13s", "w2c", "w2s")}
    return fetch


def _shared(L):
    return {"sw13": synth.bits(L["sw13"]), "sw2": synth.bits(L["sw2"])}


def _run(L, x, k):
    ws = torch.empty(moe_prefill_workspace_bytes(x.shape[0], x.shape[1], L["w13c"].shape[1] // 2,
                                                 L["w13c"].shape[0], k, L["sw13"].shape[0] // 2),
                     dtype=torch.uint8, device="cuda")
    y, ids, w, lg = moe_prefill_layer(x, L["wr"], L["w13c"], L["w13s"], L["w2c"], L["w2s"], L["sw13"], L["sw2"],
                                      top_k=k, ws=ws, want_logits=True)
    torch.cuda.synchronize()
    assert workspace_status(ws) == 0
    return y.cpu().numpy(), ids.cpu().numpy(), w.cpu().numpy(), lg.cpu().numpy()


def _check_routing(x, L, k, ids, w, lg):
    o_ids, o_w, o_lg, margin = oracle.route(synth.bits(x), synth.bits(L["wr"]), k)
    assert_rows_close(lg, o_lg, tol=1e-5, what="router logits")
    flagged = 0
    for t in range(x.shape[0]):
        if margin[t] < MARGIN_FLAG:
            flagged += 1
            continue
        assert list(ids[t]) == list(o_ids[t]), (t, ids[t], o_ids[t])
        np.testing.assert_allclose(w[t], o_w[t], rtol=1e-5, atol=1e-6)
    assert flagged <= max(2, x.shape[0] // 50)


def test_mxfp8_quantizer_bitexact():
    g = torch.Generator(device="cuda")
    g.manual_seed(11)
    v = torch.randn((64, 256), generator=g, device="cuda") * torch.exp2(torch.randint(-20, 20, (64, 1), device="cuda",
                                                                                    generator=g).float())
    v[0] = 0.0                                     # all-zero blocks: s = -127, codes 0
    v[1, :32] = 1e-40                              # subnormal block maximum
    v[2] = 3.0e38                                  # near the fp32 top: scale clamps at 127 - 8
    v[3] = torch.linspace(-448.0, 448.0, 256, device="cuda")
    v[4, :] = 0.0
    v[4, 5] = -2.0 ** -130                         # a lone subnormal
    v[5] = torch.arange(256, device="cuda").float() * 0.0625 + 0.03125  # e4m3 midpoints after scaling
    q, s = moe_mxfp8_quantize(v)
    torch.cuda.synchronize()
    oq, os_ = oracle.mxfp8_quantize(v.cpu().numpy())
    np.testing.assert_array_equal(s.cpu().numpy(), os_)
    np.testing.assert_array_equal(q.cpu().numpy(), oq)


@pytest.mark.parametrize("M,seed", [(128, 0), (256, 1), (384, 2)])
def test_prefill_small(M, seed):
    L = synth.layer(SMALL, seed, device="cuda")
    x = synth.tokens(M, SMALL.H, seed, device="cuda")
    y, ids, w, lg = _run(L, x, SMALL.k)
    _check_routing(x, L, SMALL.k, ids, w, lg)
    ref = oracle.moe_layer_prefill(synth.bits(x), ids, w.astype(np.float64), _fetch(L), _shared(L),
                                   np.arange(M))
    assert_rows_close(y, ref, what="prefill layer output")


def test_prefill_shared_tokens_span_several_tiles():
    # every token identical: each selected expert receives all M tokens (3 tiles of 128)
    M = 384
    L = synth.layer(SMALL, 7, device="cuda")
    x = synth.tokens(1, SMALL.H, 7, device="cuda").repeat(M, 1).contiguous()
    y, ids, w, lg = _run(L, x, SMALL.k)
    assert (ids == ids[0]).all()
    ref = oracle.moe_layer_prefill(synth.bits(x), ids, w.astype(np.float64), _fetch(L), _shared(L),
                                   np.array([0, 1, 127, 128, 255, 256, 383]))
    assert_rows_close(y[[0, 1, 127, 128, 255, 256, 383]], ref, what="prefill layer output")
    np.testing.assert_allclose(y, np.repeat(y[:1], M, axis=0), rtol=1e-5, atol=1e-6)


def test_prefill_ling_chunk():
    S = synth.LING
    M = 2048
    L = synth.layer(S, 3, device="cuda")
    x = synth.tokens(M, S.H, 3, device="cuda")
    y, ids, w, lg = _run(L, x, S.k)
    _check_routing(x, L, S.k, ids, w, lg)
    rng = np.random.default_rng(5)
    sample = set(rng.choice(M, 48, replace=False).tolist())
    e_star = int(ids[0, 0])
    sample |= set(np.nonzero((ids == e_star).any(axis=1))[0].tolist())  # every token of one expert
    toks = np.array(sorted(sample))
    ref = oracle.moe_layer_prefill(synth.bits(x), ids, w.astype(np.float64), _fetch(L), _shared(L), toks)
    assert_rows_close(y[toks], ref, what="prefill layer output (Ling)")


def test_experts_chunk_under_given_routing():
    # moe_mxfp4_experts with M a multiple of 128: the caller's routing (distinct random
    # experts per token, random positive weights, two ids outside [0, E) that must add
    # nothing, one token naming an expert twice) through the block-scaled path; every
    # token row against the oracle
    M = 256
    L = synth.layer(SMALL, 9, device="cuda")
    x = synth.tokens(M, SMALL.H, 9, device="cuda")
    rng = np.random.default_rng(9)
    ids = np.stack([rng.choice(SMALL.E, SMALL.k, replace=False) for _ in range(M)]).astype(np.int32)
    w = rng.uniform(0.05, 1.0, size=(M, SMALL.k)).astype(np.float32)
    ids[5, 2] = -1
    ids[7, 0] = SMALL.E
    ids[3, 1] = ids[3, 0]  # a token naming one expert twice gets both weights
    ws = torch.empty(moe_experts_workspace_bytes(M, SMALL.H, SMALL.I, SMALL.E, SMALL.k, SMALL.Is),
                     dtype=torch.uint8, device="cuda")
    y = moe_mxfp4_experts(x, torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda(), L["w13c"], L["w13s"],
                          L["w2c"], L["w2s"], L["sw13"], L["sw2"], ws=ws)
    torch.cuda.synchronize()
    assert workspace_status(ws) == 0
    ids_o, w_o = ids.copy(), w.astype(np.float64)
    bad = (ids_o < 0) | (ids_o >= SMALL.E)
    ids_o[bad] = 0
    w_o[bad] = 0.0
    ref = oracle.moe_layer_prefill(synth.bits(x), ids_o, w_o, _fetch(L), _shared(L), np.arange(M))
    assert_rows_close(y.cpu().numpy(), ref, what="experts chunk under given routing")
