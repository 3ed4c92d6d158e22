"""GPU parity of the whole decode step (L chained MoE layers + FP8 LM head).

Teacher-forced: each checked layer is recomputed by the oracle from the GPU's own
bf16 input of that layer (from the step's trace), so a near-tie routing flip in
one layer cannot make every later layer diverge; the residual update
h_{l+1} - h_l is compared with the oracle's layer output, the RMSNorm hand-off
x_{l+1} = bf16(RMSNorm(h_{l+1})) is checked against the oracle's, and the LM head
against the oracle on the GPU's final x."""
import numpy as np
import pytest
import torch

import oracle
from moe_decode_weight_router_b200 import (DecodeGraph, DecodeModel, decode_step, decode_step_launch_names,
                                           decode_step_workspace_bytes, synth, workspace_status)
from tests._bruteforce import bf16_to_f64
from tests._gpu import MARGIN_FLAG, assert_rows_close, need_gpu, rel_l2_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def _model(shape, n_layers, V, seed, path=0):
    layers = [synth.layer(shape, seed, l, device="cuda") for l in range(n_layers)]
    q = synth.e4m3_codes((V, shape.H), seed, device="cuda")
    s = synth.row_scales(V, seed, device="cuda")
    return DecodeModel(layers=layers, lm_q=q, lm_s=s, top_k=shape.k, step_path=path)


PATHS = {"persistent": 0, "per_layer": 1}


def _fetch(L):
    def fetch(lst):
        idx = torch.tensor(lst, dtype=torch.long, device="cuda")
        return {n: synth.bits(L[n].index_select(0, idx)) for n in ("w13c", "w13s", "w2c", "w2s")}
    return fetch


def _check_step(model, shape, x, res, layers_to_check):
    xt = res["x_trace"]
    ht = res["h_trace"].cpu().numpy()
    ids_t = res["ids_trace"].cpu().numpy()
    w_t = res["w_trace"].cpu().numpy()
    L = len(model.layers)
    M = x.shape[0]
    np.testing.assert_array_equal(synth.bits(xt[0]), synth.bits(x))
    np.testing.assert_array_equal(ht[0], bf16_to_f64(synth.bits(x)).astype(np.float32))
    for l in layers_to_check:
        Ly = model.layers[l]
        xl = synth.bits(xt[l])
        o_ids, o_w, o_lg, margin = oracle.route(xl, synth.bits(Ly["wr"]), shape.k)
        ids_use = o_ids.copy()
        for t in range(M):
            if margin[t] >= MARGIN_FLAG:
                assert list(ids_t[l, t]) == list(o_ids[t]), (l, t)
            else:
                ids_use[t] = ids_t[l, t]  # flagged near-tie: follow the GPU's choice
        w_use = oracle.softmax_weights_at(o_lg, ids_use)
        # the routing weights the step used, against the oracle's softmax at the same ids
        np.testing.assert_allclose(w_t[l], w_use, rtol=1e-5, atol=1e-6, err_msg=f"layer {l} routing weights")
        y_ref = oracle.moe_layer(xl, ids_use, w_use, _fetch(Ly),
                                 {"sw13": synth.bits(Ly["sw13"]), "sw2": synth.bits(Ly["sw2"])})
        dh = ht[l + 1].astype(np.float64) - ht[l].astype(np.float64)
        # the residual update is compared against the layer output; the fp32 residual sum
        # itself rounds at |h| * 2^-24, far below the tolerance
        assert_rows_close(dh, y_ref, what=f"layer {l} output")
        # hand-off: x_{l+1} = bf16(RMSNorm(h_{l+1})) within one bf16 step of the oracle's
        x_next = oracle.rmsnorm_bf16(ht[l + 1].astype(np.float64))
        got = bf16_to_f64(synth.bits(xt[l + 1]))
        ref = bf16_to_f64(x_next)
        assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -7 + 1e-30)
    # LM head on the GPU's final input
    logits_ref, am_ref, gap = oracle.lmhead_logits(synth.bits(xt[L]), synth.bits(model.lm_q), model.lm_s.cpu().numpy())
    assert_rows_close(res["logits"].cpu().numpy(), logits_ref, what="logits")
    am = res["argmax"].cpu().numpy()
    for t in range(M):
        if gap[t] >= MARGIN_FLAG * max(1.0, abs(logits_ref[t, am_ref[t]])):
            assert am[t] == am_ref[t]


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("M", [1, 4, 8])
def test_tiny_chain_all_layers(M, path):
    S = synth.TINY
    model = _model(S, 4, 1000, 21 + M, PATHS[path])
    x = synth.tokens(M, S.H, 21, device="cuda")
    names = decode_step_launch_names(model, M)
    assert names == (["k_step", "k_lm_gemv"] if path == "persistent" else
                     ["k_dense", "k_experts13", "k_experts2"] * 4 + ["k_final_norm", "k_lm_gemv"])
    res = decode_step(model, x, trace=True)
    torch.cuda.synchronize()
    assert workspace_status(res["ws"]) == 0
    _check_step(model, S, x, res, range(4))


def test_tiny_chain_free_running_matches_oracle_chain():
    """The step run free (no teacher forcing) against the oracle's own chain.  A
    near-tie routing decision anywhere in the chain would let the two follow different
    experts legitimately, so the seed is the first of a fixed list whose oracle chain
    has no decision closer than the flag margin; the test fails if none has."""
    S = synth.TINY
    for seed in range(31, 39):
        model = _model(S, 3, 1000, seed)
        x = synth.tokens(2, S.H, seed, device="cuda")
        spec = [{"wr": synth.bits(L["wr"]), "experts": _fetch(L),
                 "shared": {"sw13": synth.bits(L["sw13"]), "sw2": synth.bits(L["sw2"])}} for L in model.layers]
        out = oracle.decode_step(synth.bits(x), spec, synth.bits(model.lm_q), model.lm_s.cpu().numpy(), S.k)
        if all(np.all(m >= MARGIN_FLAG) for m in out["margin"]):
            break
    else:
        pytest.fail("no seed in 31..38 gives a chain without near-tie routing decisions")
    res = decode_step(model, x, trace=True)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(res["ids_trace"].cpu().numpy(), np.stack(out["ids"]))
    assert_rows_close(res["h_trace"][-1].cpu().numpy(), out["h"], what="free-running h_L")
    assert_rows_close(res["logits"].cpu().numpy(), out["logits"], what="free-running logits")
    # the same step with no trace or timeline runs the kernel instantiation that carries
    # no profiling or trace code (the one the benchmark times)
    lean = decode_step(model, x)
    torch.cuda.synchronize()
    assert_rows_close(lean["logits"].cpu().numpy(), out["logits"], what="free-running logits, untraced step")


@pytest.mark.parametrize("M", [1, 4])
def test_ling_shaped_untraced_step_matches_oracle_chain(M):
    """Three Ling-shaped layers run free with no trace (the instantiation without the
    profiling and trace code, as timed by the benchmark) against the oracle's own chain,
    on the first seed whose oracle chain has no routing decision within the flag margin."""
    S = synth.LING
    for seed in range(61, 71):
        model = _model(S, 3, 1000, seed)
        x = synth.tokens(M, S.H, seed, device="cuda")
        spec = [{"wr": synth.bits(L["wr"]), "experts": _fetch(L),
                 "shared": {"sw13": synth.bits(L["sw13"]), "sw2": synth.bits(L["sw2"])}} for L in model.layers]
        out = oracle.decode_step(synth.bits(x), spec, synth.bits(model.lm_q), model.lm_s.cpu().numpy(), S.k)
        if all(np.all(m >= MARGIN_FLAG) for m in out["margin"]):
            break
    else:
        pytest.fail("no seed in 61..70 gives a chain without near-tie routing decisions")
    res = decode_step(model, x)
    torch.cuda.synchronize()
    assert workspace_status(res["ws"]) == 0
    assert_rows_close(res["logits"].cpu().numpy(), out["logits"], what="untraced step logits")
    am_ref = np.argmax(out["logits"], axis=1)
    srt = np.sort(out["logits"], axis=1)
    for t in range(M):
        if srt[t, -1] - srt[t, -2] >= MARGIN_FLAG * max(1.0, abs(srt[t, -1])):
            assert int(res["argmax"][t]) == int(am_ref[t])


@pytest.mark.parametrize("M", [2, 3, 5, 8])
def test_ling_shaped_short_chain_every_window(M):
    """Three Ling-shaped layers (H 2560: the layer input of two or more tokens no longer
    fits the registers and is streamed; the top-k splits its warps into token groups x
    expert parts) at the verify-window sizes the tiny chain does not reach; every
    layer and the head are recomputed by the oracle."""
    S = synth.LING
    model = _model(S, 3, 1000, 51 + M)
    x = synth.tokens(M, S.H, 51 + M, device="cuda")
    assert decode_step_launch_names(model, M) == ["k_step", "k_lm_gemv"]
    res = decode_step(model, x, trace=True)
    torch.cuda.synchronize()
    assert workspace_status(res["ws"]) == 0
    _check_step(model, S, x, res, range(3))


@pytest.mark.parametrize("M,path", [(1, "persistent"), (4, "persistent"), (1, "per_layer")])
def test_ling_42_layers_sampled(M, path):
    """Full size: 42 distinct Ling-shaped layers (~67 GB MXFP4) and the 157,184 x 2,560
    FP8 LM head, in the same launch configuration the benchmark times; layers
    0, 1, 20 and 41 and the LM head are recomputed by the oracle."""
    S = synth.LING
    model = _model(S, synth.N_LAYERS, synth.VOCAB, 41 + M, PATHS[path])
    x = synth.tokens(M, S.H, 41 + M, device="cuda")
    res = decode_step(model, x, trace=True)
    torch.cuda.synchronize()
    assert workspace_status(res["ws"]) == 0
    _check_step(model, S, x, res, [0, 1, 20, 41])
    # the captured graph (one launch per step) is checked against the oracle the same way,
    # through the trace it fills; two runs need not agree bit for bit with each other
    # (fp32 atomic accumulation order), each must agree with the oracle
    ws = torch.empty(decode_step_workspace_bytes(model, M), dtype=torch.uint8, device="cuda")
    res_g = {"logits": torch.empty((M, synth.VOCAB), dtype=torch.float32, device="cuda"),
             "argmax": torch.empty((M,), dtype=torch.int32, device="cuda")}
    L = len(model.layers)
    res_g["x_trace"] = torch.empty((L + 1, M, S.H), dtype=torch.bfloat16, device="cuda")
    res_g["h_trace"] = torch.empty((L + 1, M, S.H), dtype=torch.float32, device="cuda")
    res_g["ids_trace"] = torch.empty((L, M, S.k), dtype=torch.int32, device="cuda")
    res_g["w_trace"] = torch.empty((L, M, S.k), dtype=torch.float32, device="cuda")
    g = DecodeGraph(model, x, res_g["logits"], res_g["argmax"], ws, trace=res_g)
    g.launch()
    g.launch()
    torch.cuda.synchronize()
    g.close()
    _check_step(model, S, x, res_g, [0, 41])
    del model
    torch.cuda.empty_cache()
