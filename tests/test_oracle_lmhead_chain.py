"""Pins for the oracle's FP8 LM head, RMSNorm stand-in, MXFP8 quantiser,
prefill layer and the chained decode step."""
import numpy as np
import pytest
import torch

import oracle
from moe_decode_weight_router_b200 import synth
from tests._bruteforce import (bf16_to_f64, dense_moe, dequant_mxfp8, e4m3_to_f64, mxfp8_ref, silu)


def _lm(V, H, seed):
    return synth.bits(synth.lm_head(V, H, seed))


def test_lmhead_quantize_matches_torch_fp32_path():
    V, H = 96, 256
    wt = _lm(V, H, 0)
    wt[5] = 0  # an all-zero row: scale 1, codes 0
    q, s = oracle.lmhead_quantize(wt)
    w32 = bf16_to_f64(wt).astype(np.float32)
    amax = np.abs(w32).max(axis=1)
    s_ref = np.where(amax == 0, np.float32(1.0), (amax / np.float32(448.0)).astype(np.float32))
    np.testing.assert_array_equal(s, s_ref)
    scaled = (torch.from_numpy(w32) / torch.from_numpy(s_ref)[:, None])  # IEEE fp32 division
    scaled = torch.clamp(scaled, -448.0, 448.0)
    q_ref = scaled.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(q, q_ref)
    assert np.all(q[5] == 0) and s[5] == 1.0
    # the row maximum lands on the largest code (+-448)
    for v in range(V):
        if v == 5:
            continue
        h = int(np.argmax(np.abs(w32[v])))
        assert q[v, h] in (0x7E, 0xFE)


def test_lmhead_logits_match_numpy_and_argmax_ties():
    V, H, M = 200, 256, 4
    wt = _lm(V, H, 1)
    wt[150] = wt[37]  # duplicate rows give equal logits: the lower index must win
    q, s = oracle.lmhead_quantize(wt)
    x = synth.bits(synth.tokens(M, H, 1))
    xt = x.copy()
    logits, am, gap = oracle.lmhead_logits(xt, q, s)
    ref = (e4m3_to_f64(q) @ bf16_to_f64(xt).T).T * s.astype(np.float64)[None, :]
    np.testing.assert_allclose(logits, ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(am, np.argmax(ref, axis=1))  # numpy returns the first maximum
    # force the duplicated row to be the maximum for token 0
    x2 = synth.bits(torch.from_numpy(bf16_to_f64(wt[37:38]).astype(np.float32)).to(torch.bfloat16))
    l2, am2, gap2 = oracle.lmhead_logits(x2, q, s)
    assert am2[0] == 37 and l2[0, 150] == l2[0, 37] and gap2[0] == 0.0


def test_rmsnorm_bf16_matches_numpy():
    rng = np.random.default_rng(4)
    h = rng.standard_normal((3, 2560)) * np.array([[1e-3], [1.0], [1e5]])
    got = oracle.rmsnorm_bf16(h)
    ref = h / np.sqrt((h * h).mean(axis=1, keepdims=True) + 1e-6)
    # exactly representable in fp32 -> compare to torch's RNE bf16 cast within one ulp,
    # and exactly where the fp64 value is itself an fp32 value
    gv = bf16_to_f64(got)
    np.testing.assert_allclose(gv, ref, rtol=2 ** -8)
    r32 = ref.astype(np.float32)
    exact = r32.astype(np.float64) == ref
    tb = torch.from_numpy(r32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(got[exact], tb[exact])


def test_mxfp8_quantize_matches_reference():
    rng = np.random.default_rng(6)
    v = (rng.standard_normal((5, 256)) * np.array([[1e-4], [1.0], [3.0], [1e3], [0.0]])).astype(np.float32)
    v[1, 32:64] = 0.0                 # an all-zero block: scale 2^-127, codes 0
    v[2, 0:32] = np.linspace(-1.99, 1.99, 32, dtype=np.float32)  # amax 1.99 -> saturation at 448
    q, se = oracle.mxfp8_quantize(v)
    q_ref, se_ref = mxfp8_ref(v)
    np.testing.assert_array_equal(se, se_ref)
    np.testing.assert_array_equal(q, q_ref)
    assert se[1, 1] == 0 and np.all(q[1, 32:64] == 0)
    assert se[2, 0] == 127 + 0 - 8  # floor(log2 1.99) - 8
    # dequantised values stay within half an e4m3 step (or the 448 clip) of the input
    dq = dequant_mxfp8(q, se)
    err = np.abs(dq - v)
    assert np.all(err <= np.maximum(np.abs(v) * 2 ** -4 + 1e-30, np.abs(v) - 448 * 2.0 ** (se.repeat(32, 1).astype(int) - 127)))


def test_prefill_layer_matches_dense_mxfp8():
    S = synth.TINY
    M = 64
    L = {k: synth.bits(v) for k, v in synth.layer(S, 5).items()}
    x = synth.bits(synth.tokens(M, S.H, 5))
    ids, w, _, _ = oracle.route(x, L["wr"], S.k)
    toks = [0, 7, 31, 63]
    y = oracle.moe_layer_prefill(x, ids, w, L, {"sw13": L["sw13"], "sw2": L["sw2"]}, toks)
    # dense: MXFP8 of x and of fp32(a), evaluated for every expert
    from tests._bruteforce import dequant_mxfp4
    xq, xs = mxfp8_ref(bf16_to_f64(x).astype(np.float32))
    xd = dequant_mxfp8(xq, xs)
    W13 = dequant_mxfp4(L["w13c"], L["w13s"])
    W2 = dequant_mxfp4(L["w2c"], L["w2s"])
    S13, S2 = bf16_to_f64(L["sw13"]), bf16_to_f64(L["sw2"])
    for j, t in enumerate(toks):
        ref = np.zeros(S.H)
        for kk in range(S.k):
            e = ids[t, kk]
            gu = W13[e] @ xd[t]
            a = (silu(gu[:S.I]) * gu[S.I:]).astype(np.float32)
            aq, as_ = mxfp8_ref(a[None, :])
            ref += w[t, kk] * (W2[e] @ dequant_mxfp8(aq, as_)[0])
        g = S13 @ bf16_to_f64(x[t])
        a_s = silu(g[:S.Is]) * g[S.Is:]
        a_s = torch.from_numpy(a_s.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
        ref += S2 @ a_s
        np.testing.assert_allclose(y[j], ref, rtol=1e-9, atol=1e-9 * np.abs(ref).max())


def test_prefill_layer_close_to_decode_layer():
    # MXFP8 activations change the result by a few percent at most (relative L2).
    S = synth.TINY
    L = {k: synth.bits(v) for k, v in synth.layer(S, 6).items()}
    x = synth.bits(synth.tokens(8, S.H, 6))
    ids, w, _, _ = oracle.route(x, L["wr"], S.k)
    sh = {"sw13": L["sw13"], "sw2": L["sw2"]}
    yp = oracle.moe_layer_prefill(x, ids, w, L, sh, list(range(8)))
    yd = oracle.moe_layer(x, ids, w, L, sh)
    rel = np.linalg.norm(yp - yd, axis=1) / np.linalg.norm(yd, axis=1)
    assert np.all(rel < 0.1)


def test_decode_step_chain_matches_dense_chain():
    S = synth.TINY
    nL, M, V = 3, 2, 300
    layers_t = [synth.layer(S, 7, l) for l in range(nL)]
    layers = [{k: synth.bits(v) for k, v in L.items()} for L in layers_t]
    lm = _lm(V, S.H, 7)
    q, s = oracle.lmhead_quantize(lm)
    x0 = synth.bits(synth.tokens(M, S.H, 7))
    spec = [{"wr": L["wr"], "experts": L, "shared": {"sw13": L["sw13"], "sw2": L["sw2"]}} for L in layers]
    out = oracle.decode_step(x0, spec, q, s, S.k)
    # dense chain in numpy
    h = bf16_to_f64(x0)
    x = x0
    for L in layers:
        logits = bf16_to_f64(x) @ bf16_to_f64(L["wr"]).T
        gate = np.zeros((M, S.E))
        for t in range(M):
            top = np.argsort(-logits[t], kind="stable")[:S.k]
            z = np.exp(logits[t, top] - logits[t, top].max())
            gate[t, top] = z / z.sum()
        h = h + dense_moe(x, gate, L)
        xn = h / np.sqrt((h * h).mean(axis=1, keepdims=True) + 1e-6)
        x = torch.from_numpy(xn).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_allclose(out["h"], h, rtol=1e-9)
    ref_logits = (e4m3_to_f64(q) @ bf16_to_f64(out["x"][-1]).T).T * s.astype(np.float64)[None, :]
    np.testing.assert_allclose(out["logits"], ref_logits, rtol=1e-12, atol=1e-12)
    assert np.array_equal(out["argmax"], np.argmax(ref_logits, axis=1))
    # final bf16 input within one bf16 ulp of the dense chain's (double vs single rounding)
    np.testing.assert_allclose(bf16_to_f64(out["x"][-1]), bf16_to_f64(x), rtol=2 ** -7)
