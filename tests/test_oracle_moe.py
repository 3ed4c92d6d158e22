"""Pins for the oracle's router and MoE layer: library routines, brute-force
dense-equivalent MoE, closed forms and invariants."""
import numpy as np
import pytest
import torch
from scipy.special import softmax

import oracle
from moe_decode_weight_router_b200 import synth
from tests._bruteforce import bf16_to_f64, dense_moe, silu


def _layer_np(shape, seed, M):
    L = synth.layer(shape, seed)
    Ln = {k: synth.bits(v) for k, v in L.items()}
    x = synth.bits(synth.tokens(M, shape.H, seed))
    return Ln, x


@pytest.mark.parametrize("M", [1, 4])
def test_route_matches_numpy(M):
    S = synth.TINY
    Ln, x = _layer_np(S, 0, M)
    ids, w, logits, margin = oracle.route(x, Ln["wr"], S.k)
    ref_logits = bf16_to_f64(x) @ bf16_to_f64(Ln["wr"]).T
    np.testing.assert_allclose(logits, ref_logits, rtol=1e-12, atol=1e-12)
    for t in range(M):
        order = np.argsort(-ref_logits[t], kind="stable")  # ties keep the lower index first
        assert list(ids[t]) == list(order[:S.k])
        np.testing.assert_allclose(w[t], softmax(ref_logits[t][order[:S.k]]), rtol=1e-12)
        assert abs(w[t].sum() - 1.0) <= 1e-12
        srt = np.sort(ref_logits[t])[::-1]
        assert margin[t] == pytest.approx(srt[S.k - 1] - srt[S.k], abs=1e-12)
    # the renormalised top-k weights equal the full softmax restricted to the top-k
    full = softmax(ref_logits, axis=1)
    for t in range(M):
        sel = full[t, ids[t]]
        np.testing.assert_allclose(w[t], sel / sel.sum(), rtol=1e-12)


def test_route_ties_go_to_lower_index():
    H, E, k = 64, 12, 3
    rng = np.random.default_rng(5)
    wr = torch.from_numpy(rng.standard_normal((E, H)).astype(np.float32)).to(torch.bfloat16)
    wr[7] = wr[2]
    wr[9] = wr[2]
    wr[4] = wr[2]
    x = wr[2:3].clone()  # makes row 2 (and its copies) the largest logit
    ids, w, _, margin = oracle.route(synth.bits(x), synth.bits(wr), k)
    assert list(ids[0]) == [2, 4, 7]
    np.testing.assert_allclose(w[0], [1 / 3] * 3, rtol=1e-12)
    assert margin[0] == 0.0  # the 4th copy (index 9) ties the 3rd pick


def test_route_distinct_experts_bounded_by_kM():
    S = synth.LING
    wr = synth.bits(synth.normal_bf16((S.E, S.H), 0.02, 3, 1))
    x = synth.bits(synth.tokens(4, S.H, 3))
    ids, w, _, _ = oracle.route(x, wr, S.k)
    for t in range(4):
        assert len(set(ids[t])) == S.k
    assert len(set(ids.reshape(-1))) <= S.k * 4
    assert np.all(np.abs(w.sum(1) - 1) <= 1e-12)


@pytest.mark.parametrize("M", [1, 4])
def test_moe_layer_equals_dense_equivalent(M):
    S = synth.TINY
    Ln, x = _layer_np(S, 0, M)
    ids, w, _, _ = oracle.route(x, Ln["wr"], S.k)
    y = oracle.moe_layer(x, ids, w, Ln, {"sw13": Ln["sw13"], "sw2": Ln["sw2"]})
    gate = np.zeros((M, S.E))
    for t in range(M):
        gate[t, ids[t]] = w[t]
    ref = dense_moe(x, gate, Ln)
    np.testing.assert_allclose(y, ref, rtol=1e-11, atol=1e-9 * np.abs(ref).max())


def test_moe_layer_zero_codes_leave_shared_expert():
    S = synth.TINY
    Ln, x = _layer_np(S, 1, 2)
    Lz = dict(Ln)
    Lz["w13c"] = np.zeros_like(Ln["w13c"])
    Lz["w2c"] = np.zeros_like(Ln["w2c"])
    ids, w, _, _ = oracle.route(x, Ln["wr"], S.k)
    y = oracle.moe_layer(x, ids, w, Lz, {"sw13": Ln["sw13"], "sw2": Ln["sw2"]})
    xs = bf16_to_f64(x)
    S13, S2 = bf16_to_f64(Ln["sw13"]), bf16_to_f64(Ln["sw2"])
    g = xs @ S13.T
    ref = (silu(g[:, :S.Is]) * g[:, S.Is:]) @ S2.T
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-15)


def test_moe_layer_constant_codes_closed_form():
    # every W13 and W2 code = 2 (E2M1 1.0) with scale exponent 127 (x1): each gate and
    # up row sums x, so a_r = silu(S) * S with S = sum_h x_h, and every output
    # element of every expert is I * silu(S) * S; the weights sum to 1.
    S = synth.TINY
    Ln, x = _layer_np(S, 2, 3)
    Lc = dict(Ln)
    Lc["w13c"] = np.full_like(Ln["w13c"], 0x22)
    Lc["w13s"] = np.full_like(Ln["w13s"], 127)
    Lc["w2c"] = np.full_like(Ln["w2c"], 0x22)
    Lc["w2s"] = np.full_like(Ln["w2s"], 127)
    ids, w, _, _ = oracle.route(x, Ln["wr"], S.k)
    y = oracle.moe_layer(x, ids, w, Lc, None)
    s = bf16_to_f64(x).sum(axis=1)
    ref = S.I * s / (1 + np.exp(-s)) * s
    np.testing.assert_allclose(y, np.repeat(ref[:, None], S.H, axis=1), rtol=1e-12)


def test_moe_layer_nibble_order_and_gate_up_split():
    # One expert, H = 64, I = 32.  Byte j of a row holds element 2j in its low nibble.
    # Gate rows carry code 2 (1.0) at element 0 only; up rows carry code 4 (2.0) at
    # element 1 only (a high nibble).  With x = (x0, x1, 0...) this gives
    # g = x0, u = 2 x1, a = silu(x0) * 2 x1 for every r, and W2 of code 2 (1.0)
    # sums a over r: y_h = I * silu(x0) * 2 x1.
    H, I = 64, 32
    w13c = np.zeros((1, 2 * I, H // 2), np.uint8)
    w13c[0, :I, 0] = 0x02
    w13c[0, I:, 0] = 0x40
    w13s = np.full((1, 2 * I, H // 32), 127, np.uint8)
    w2c = np.full((1, H, I // 2), 0x22, np.uint8)
    w2s = np.full((1, H, I // 32), 127, np.uint8)
    xv = torch.zeros((1, H), dtype=torch.bfloat16)
    xv[0, 0] = 0.75
    xv[0, 1] = -1.25
    x = synth.bits(xv)
    y = oracle.moe_layer(x, np.zeros((1, 1), np.int32), np.ones((1, 1)),
                         {"w13c": w13c, "w13s": w13s, "w2c": w2c, "w2s": w2s}, None)
    ref = I * (0.75 / (1 + np.exp(-0.75))) * 2 * -1.25
    np.testing.assert_allclose(y, np.full((1, H), ref), rtol=1e-14)


def test_moe_layer_scale_blocks_cover_32_elements():
    # A scale change in block 1 (elements 32..63) must affect exactly those elements.
    H, I = 64, 32
    rng = np.random.default_rng(9)
    w13c = rng.integers(0, 256, (1, 2 * I, H // 2), dtype=np.uint8)
    w13s = np.full((1, 2 * I, H // 32), 127, np.uint8)
    w2c = rng.integers(0, 256, (1, H, I // 2), dtype=np.uint8)
    w2s = np.full((1, H, I // 32), 127, np.uint8)
    L = {"w13c": w13c, "w13s": w13s, "w2c": w2c, "w2s": w2s}
    xv = torch.zeros((1, H), dtype=torch.bfloat16)
    xv[0, 40] = 1.0  # only element 40 (block 1) is non-zero
    x = synth.bits(xv)
    ids, w = np.zeros((1, 1), np.int32), np.ones((1, 1))
    y0 = oracle.moe_layer(x, ids, w, L, None)
    L2 = dict(L)
    L2["w13s"] = w13s.copy()
    L2["w13s"][..., 0] = 100  # block 0 only: no effect on element 40
    np.testing.assert_array_equal(oracle.moe_layer(x, ids, w, L2, None), y0)
    L3 = dict(L)
    L3["w13s"] = w13s.copy()
    L3["w13s"][..., 1] = 126  # block 1 halves g and u: a -> silu(g/2)(u/2)
    y3 = oracle.moe_layer(x, ids, w, L3, None)
    assert not np.allclose(y3, y0)
    gate = np.ones((1, 1))
    np.testing.assert_allclose(y3, dense_moe(x, gate, L3), rtol=1e-12, atol=1e-12)


def test_moe_layer_ling_shape_single_expert_matches_dense():
    # Full-size rows (H = 2560, I = 768) for two experts, dense numpy on the same bytes.
    S = synth.LING
    rng = np.random.default_rng(11)
    L = {
        "w13c": rng.integers(0, 256, (2, 2 * S.I, S.H // 2), dtype=np.uint8),
        "w13s": rng.integers(S.e_lo, S.e_hi + 1, (2, 2 * S.I, S.H // 32), dtype=np.uint8),
        "w2c": rng.integers(0, 256, (2, S.H, S.I // 2), dtype=np.uint8),
        "w2s": rng.integers(S.e_lo, S.e_hi + 1, (2, S.H, S.I // 32), dtype=np.uint8),
    }
    x = synth.bits(synth.tokens(1, S.H, 4))
    ids = np.array([[1, 0]], np.int32)
    w = np.array([[0.7, 0.3]])
    y = oracle.moe_layer(x, ids, w, L, None)
    ref = dense_moe(x, np.array([[0.3, 0.7]]), L)
    np.testing.assert_allclose(y, ref, rtol=1e-11, atol=1e-9 * np.abs(ref).max())


def test_moe_layer_fetch_callable_equals_arrays():
    S = synth.TINY
    Ln, x = _layer_np(S, 3, 4)
    ids, w, _, _ = oracle.route(x, Ln["wr"], S.k)
    calls = []

    def fetch(lst):
        calls.append(list(lst))
        return {n: Ln[n][lst] for n in ("w13c", "w13s", "w2c", "w2s")}

    y1 = oracle.moe_layer(x, ids, w, Ln, None)
    y2 = oracle.moe_layer(x, ids, w, fetch, None)
    np.testing.assert_array_equal(y1, y2)
    assert calls[0] == sorted(set(ids.reshape(-1).tolist()))
