"""GPU parity of the MXFP4 products over the whole E8M0 range (2^-127 .. 2^127).

The synthetic layers elsewhere draw scale exponents from [118, 127]; these cases
draw them from wider ranges and build rows whose largest blocks meet a zero
activation, so a kernel that scaled blocks relative to a row's largest scale and
dropped the small ones would return zero where the oracle does not.  Every expected
value is the oracle's (fp64) on the same bytes; tolerance as everywhere: relative L2
per token row <= 5e-3.  MXFP4 and E8M0 are the OCP microscaling formats the DGX Spark
MoE knowledge card's routed experts use (知识卡片：NVIDIA DGX Spark 上提升 MoE 推理吞吐的
三种方法, 方法/产品要点 item 1)."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from moe_decode_weight_router_b200 import DecodeModel, decode_step, moe_mxfp4_experts, synth, workspace_status
from tests._gpu import assert_rows_close, need_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def _fetch(L):
    def fetch(lst):
        idx = torch.tensor(lst, dtype=torch.long, device="cuda")
        return {n: synth.bits(L[n].index_select(0, idx)) for n in ("w13c", "w13s", "w2c", "w2s")}
    return fetch


def _random_routing(S, M, seed):
    """Distinct experts per token from a seeded permutation, weights from a seeded
    softmax (the kernels take the routing as given)."""
    perm = synth.permutation(S.E, seed).numpy()
    ids = perm[: M * S.k].reshape(M, S.k).astype(np.int32)
    g = torch.Generator().manual_seed(seed)
    z = torch.randn((M, S.k), generator=g, dtype=torch.float64).numpy()
    w = np.exp(z - z.max(1, keepdims=True))
    w /= w.sum(1, keepdims=True)
    return ids, w.astype(np.float32)


def _check(S, L, x, ids, w, shared, what):
    ids_d = torch.from_numpy(ids).cuda()
    w_d = torch.from_numpy(w).cuda()
    y = moe_mxfp4_experts(x, ids_d, w_d, L["w13c"], L["w13s"], L["w2c"], L["w2s"],
                          L.get("sw13") if shared else None, L.get("sw2") if shared else None)
    torch.cuda.synchronize()
    sh = {"sw13": synth.bits(L["sw13"]), "sw2": synth.bits(L["sw2"])} if shared else None
    ref = oracle.moe_layer(synth.bits(x), ids, w.astype(np.float64), _fetch(L), sh)
    assert np.all(np.abs(ref) > 0.0), "the case must give every output a nonzero reference"
    return assert_rows_close(y.cpu().numpy(), ref, what=what)


@pytest.mark.parametrize("M", [1, 4])
@pytest.mark.parametrize("lo,hi", [(104, 127), (90, 127)])
def test_experts_wide_uniform_exponents(M, lo, hi):
    """Exponents uniform in [lo, hi]: a span of 23 is the widest the tensor-core path
    folds into f16 codes (subnormal codes included); 37 takes the exact per-block path."""
    S = dataclasses.replace(synth.LING, e_lo=lo, e_hi=hi)
    L = synth.layer(S, 60 + hi - lo, device="cuda")
    x = synth.tokens(M, S.H, 60 + M, device="cuda")
    ids, w = _random_routing(S, M, 60 + M)
    _check(S, L, x, ids, w, True, f"exponents [{lo},{hi}] M={M}")


@pytest.mark.parametrize("M", [1, 4])
def test_experts_largest_blocks_meet_zero_activation(M):
    """Every W13 row: blocks 0..39 at e = 254 (2^127), blocks 40..79 at e in [0, 100];
    x is zero on blocks 0..39, so only the small blocks contribute.  Gate rows of
    intermediate 0..383 have zero codes, so a = 0 there, which is where every W2 row
    has its e = 254 blocks (0..11); its blocks 12..23 are at e in [0, 100]."""
    S = synth.LING
    L = synth.layer(S, 70, device="cuda", shared=False)
    g13 = synth.uniform_ints_u8(L["w13s"].shape, 0, 100, 70, 51, "cuda")
    g13[:, :, :40] = 254
    L["w13s"] = g13
    L["w13c"][:, :384, :] = 0
    g2 = synth.uniform_ints_u8(L["w2s"].shape, 0, 100, 70, 52, "cuda")
    g2[:, :, :12] = 254
    L["w2s"] = g2
    x = synth.tokens(M, S.H, 70 + M, device="cuda")
    x[:, :1280] = 0
    ids, w = _random_routing(S, M, 70 + M)
    _check(S, L, x, ids, w, False, f"largest blocks at zero activation M={M}")


@pytest.mark.parametrize("M", [1, 4])
def test_experts_full_exponent_range_tiny_activations(M):
    """W13 exponents uniform over the whole finite E8M0 range [0, 254] against
    activations ~ N(0,1) * 2^-120 (bf16), W2 exponents in [0, 100]: block factors
    from 2^-127 (an fp32 subnormal) to 2^127, and an activation shift past 2^126."""
    S = synth.LING
    L = synth.layer(S, 80, device="cuda", shared=False)
    L["w13s"] = synth.uniform_ints_u8(L["w13s"].shape, 0, 254, 80, 51, "cuda")
    L["w2s"] = synth.uniform_ints_u8(L["w2s"].shape, 0, 100, 80, 52, "cuda")
    x = (synth.tokens(M, S.H, 80 + M, device="cuda").float() * 2.0 ** -120).to(torch.bfloat16)
    ids, w = _random_routing(S, M, 80 + M)
    _check(S, L, x, ids, w, False, f"full exponent range M={M}")


@pytest.mark.parametrize("M", [1, 4])
def test_decode_step_wide_exponents_three_layers(M):
    """Three chained Ling-shaped layers with exponents in [90, 127], teacher-forced
    against the oracle layer by layer, plus the LM head."""
    from tests.test_gpu_decode_step import _check_step
    S = dataclasses.replace(synth.LING, e_lo=90, e_hi=127)
    layers = [synth.layer(S, 90 + M, l, device="cuda") for l in range(3)]
    q = synth.e4m3_codes((1000, S.H), 90, device="cuda")
    s = synth.row_scales(1000, 90, device="cuda")
    model = DecodeModel(layers=layers, lm_q=q, lm_s=s, top_k=S.k)
    x = synth.tokens(M, S.H, 90 + M, device="cuda")
    res = decode_step(model, x, trace=True)
    torch.cuda.synchronize()
    assert workspace_status(res["ws"]) == 0
    _check_step(model, S, x, res, range(3))
