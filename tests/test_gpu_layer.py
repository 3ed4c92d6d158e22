"""GPU parity of the router and the MXFP4 expert layer against the CPU oracle.

Tiny layer (H 256, I 64, 16 experts, top-2) and the Ling-shaped layer
(H 2560, I 768, 512 experts, top-8) at M = 1 and the M = 4 verify window with
random, identical and disjoint routings; plus edge cases.  Every expected value
comes from the oracle on the same seeded bytes."""
import numpy as np
import pytest
import torch

import oracle
from moe_decode_weight_router_b200 import moe_mxfp4_experts, moe_route, synth
from tests._gpu import MARGIN_FLAG, assert_rows_close, need_gpu, rel_l2_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def _layer(shape, seed, shared=True):
    L = synth.layer(shape, seed, device="cuda", shared=shared)
    return L


def _fetch(L):
    def fetch(lst):
        idx = torch.tensor(lst, dtype=torch.long, device="cuda")
        return {n: synth.bits(L[n].index_select(0, idx)) for n in ("w13c", "w13s", "w2c", "w2s")}
    return fetch


def _shared_np(L):
    return {"sw13": synth.bits(L["sw13"]), "sw2": synth.bits(L["sw2"])} if "sw13" in L else None


@pytest.mark.parametrize("shape,M,seed", [(synth.TINY, 1, 0), (synth.TINY, 4, 1), (synth.TINY, 8, 2),
                                          (synth.LING, 1, 0), (synth.LING, 4, 1), (synth.LING, 8, 2)])
def test_route_parity(shape, M, seed):
    wr = synth.normal_bf16((shape.E, shape.H), 0.02, seed, 1, "cuda")
    x = synth.tokens(M, shape.H, seed, device="cuda")
    ids, w, lg = moe_route(x, wr, shape.k, logits=True)
    torch.cuda.synchronize()
    o_ids, o_w, o_lg, margin = oracle.route(synth.bits(x), synth.bits(wr), shape.k)
    assert_rows_close(lg.cpu().numpy(), o_lg, tol=1e-5, what="router logits")
    ids, w = ids.cpu().numpy(), w.cpu().numpy()
    for t in range(M):
        if margin[t] < MARGIN_FLAG:
            continue  # flagged near-tie: the selection is decided below fp32 resolution
        assert list(ids[t]) == list(o_ids[t]), (t, ids[t], o_ids[t])
        np.testing.assert_allclose(w[t], o_w[t], rtol=1e-5, atol=1e-6)
        assert abs(w[t].sum() - 1) < 1e-5


def test_route_ties_go_to_lower_index():
    H, E, k = 256, 64, 8
    wr = synth.normal_bf16((E, H), 0.02, 5, 1, "cuda")
    for dup in (9, 17, 40, 63):
        wr[dup] = wr[3]
    x = (wr[3:4].float() * 50).to(torch.bfloat16)  # row 3 and its copies become the largest logits
    ids, w, lg = moe_route(x, wr, k, logits=True)
    torch.cuda.synchronize()
    l = lg.cpu().numpy()[0]
    assert l[3] == l[9] == l[17] == l[40] == l[63]
    assert list(ids.cpu().numpy()[0][:5]) == [3, 9, 17, 40, 63]
    o_ids, _, _, _ = oracle.route(synth.bits(x), synth.bits(wr), k)
    assert list(o_ids[0][:5]) == [3, 9, 17, 40, 63]


def _experts_check(shape, L, x, ids, w, what):
    y = moe_mxfp4_experts(x, ids, w, L["w13c"], L["w13s"], L["w2c"], L["w2s"], L.get("sw13"), L.get("sw2"))
    torch.cuda.synchronize()
    ref = oracle.moe_layer(synth.bits(x), ids.cpu().numpy(), w.cpu().numpy().astype(np.float64), _fetch(L),
                           _shared_np(L))
    return assert_rows_close(y.cpu().numpy(), ref, what=what)


@pytest.mark.parametrize("shape,M,seed", [(synth.TINY, 1, 0), (synth.TINY, 3, 3), (synth.TINY, 8, 4),
                                          (synth.LING, 1, 0), (synth.LING, 2, 5), (synth.LING, 4, 1),
                                          (synth.LING, 8, 2)])
def test_experts_random_routing(shape, M, seed):
    L = _layer(shape, seed)
    x = synth.tokens(M, shape.H, seed, device="cuda")
    ids, w, _ = moe_route(x, L["wr"], shape.k)
    _experts_check(shape, L, x, ids, w, f"experts M={M}")


def _forced(shape, L, x, mode, seed):
    M = x.shape[0]
    o_ids, o_w, o_lg, _ = oracle.route(synth.bits(x), synth.bits(L["wr"]), shape.k)
    if mode == "identical":
        ids = np.repeat(o_ids[0:1], M, axis=0)
    else:
        perm = synth.permutation(shape.E, seed).numpy()
        ids = perm[: M * shape.k].reshape(M, shape.k).astype(np.int32)
    w = oracle.softmax_weights_at(o_lg, ids)
    return (torch.from_numpy(ids.astype(np.int32)).cuda(), torch.from_numpy(w.astype(np.float32)).cuda())


@pytest.mark.parametrize("mode", ["identical", "disjoint"])
def test_experts_verify_window_forced_routing(mode):
    S = synth.LING
    L = _layer(S, 11)
    x = synth.tokens(4, S.H, 11, device="cuda")
    ids, w = _forced(S, L, x, mode, 11)
    n_distinct = len(set(ids.cpu().numpy().reshape(-1).tolist()))
    assert n_distinct == (8 if mode == "identical" else 32)
    _experts_check(S, L, x, ids, w, f"experts {mode}")


def test_experts_without_shared_expert():
    S = synth.LING
    L = _layer(S, 12, shared=False)
    x = synth.tokens(4, S.H, 12, device="cuda")
    ids, w, _ = moe_route(x, L["wr"], S.k)
    _experts_check(S, L, x, ids, w, "experts no shared")


def test_experts_duplicate_and_invalid_ids():
    # a token naming an expert twice gets both weights; ids outside [0, E) add nothing
    S = synth.TINY
    L = _layer(S, 13)
    x = synth.tokens(3, S.H, 13, device="cuda")
    ids = torch.tensor([[5, 5], [2, 99], [-1, 7]], dtype=torch.int32, device="cuda")
    w = torch.tensor([[0.25, 0.75], [0.6, 0.4], [0.3, 0.7]], dtype=torch.float32, device="cuda")
    y = moe_mxfp4_experts(x, ids, w, L["w13c"], L["w13s"], L["w2c"], L["w2s"], L["sw13"], L["sw2"])
    torch.cuda.synchronize()
    # oracle view: drop the invalid entries by giving them weight 0 on a valid expert
    ids_o = np.array([[5, 5], [2, 0], [0, 7]], np.int32)
    w_o = np.array([[0.25, 0.75], [0.6, 0.0], [0.0, 0.7]])
    ref = oracle.moe_layer(synth.bits(x), ids_o, w_o, _fetch(L), _shared_np(L))
    assert_rows_close(y.cpu().numpy(), ref, what="duplicate/invalid ids")


def test_experts_zero_codes_leave_shared_expert():
    S = synth.LING
    L = _layer(S, 14)
    L["w13c"].zero_()
    L["w2c"].zero_()
    x = synth.tokens(1, S.H, 14, device="cuda")
    ids, w, _ = moe_route(x, L["wr"], S.k)
    _experts_check(S, L, x, ids, w, "zero codes")


def test_experts_repeat_calls_are_stable():
    S = synth.LING
    L = _layer(S, 15)
    x = synth.tokens(4, S.H, 15, device="cuda")
    ids, w, _ = moe_route(x, L["wr"], S.k)
    ys = [moe_mxfp4_experts(x, ids, w, L["w13c"], L["w13s"], L["w2c"], L["w2s"], L["sw13"], L["sw2"]).clone()
          for _ in range(3)]
    torch.cuda.synchronize()
    for yy in ys[1:]:
        r = rel_l2_rows(yy.cpu().numpy(), ys[0].cpu().numpy())
        assert np.all(r < 1e-5)
