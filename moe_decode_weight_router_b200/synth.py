"""Seeded synthetic inputs at the shapes of the MoE decode workloads.

Random draws only: nothing here performs a step of the method (no decoding,
routing, quantisation or products).  Both the CUDA path and the CPU oracle are
fed from these tensors, so this module imports neither of them.

Shapes follow the DGX Spark MoE knowledge card ("知识卡片：NVIDIA DGX Spark 上提升
MoE 推理吞吐的三种方法"): 512 routed experts, top-8, 1 shared expert, hidden
2,560 (the LM head is 157,184 x 2,560), moe_intermediate_size 768, 42 layers.

Recipe (one torch generator per tensor, seeded from (seed, tensor id), on the
device the tensor lives on; BF16 tensors are an RNE cast of fp32 draws):
  x            bf16 [M,H]         ~ N(0, 1)
  router  Wr   bf16 [E,H]         ~ N(0, 0.02)
  W13 codes    u8   [E,2I,H/2]    uniform bytes (two uniform E2M1 nibbles each)
  W13 scales   u8   [E,2I,H/32]   uniform integers in [e_lo, e_hi]
  W2 codes     u8   [E,H,I/2]     uniform bytes
  W2 scales    u8   [E,H,I/32]    uniform integers in [e_lo, e_hi]
  shared W13   bf16 [2Is,H]       ~ N(0, 0.02)
  shared W2    bf16 [H,Is]        ~ N(0, 0.02)
  LM head      bf16 [V,H]         ~ N(0, 0.02)
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class LayerShape:
    H: int      # hidden size
    I: int      # routed expert intermediate size
    E: int      # routed experts
    k: int      # experts per token
    Is: int     # shared expert intermediate size
    e_lo: int   # E8M0 exponent range of the synthetic MXFP4 scales
    e_hi: int

    @property
    def expert_bytes(self) -> int:
        """MXFP4 bytes of one routed expert (codes + scales of W13 and W2)."""
        return (2 * self.I * (self.H // 2 + self.H // 32)) + (self.H * (self.I // 2 + self.I // 32))


# tiny layer: hidden 256, intermediate 64, 16 experts, top-2, shared 64, exponents 120..127
TINY = LayerShape(H=256, I=64, E=16, k=2, Is=64, e_lo=120, e_hi=127)
# Ling-shaped layer: hidden 2560, intermediate 768, 512 experts, top-8, shared 768, exponents 118..127
LING = LayerShape(H=2560, I=768, E=512, k=8, Is=768, e_lo=118, e_hi=127)
VOCAB = 157184
N_LAYERS = 42


def _gen(seed: int, tid: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 1_000_003 + int(tid))
    return g


def normal_bf16(shape, std: float, seed: int, tid: int, device="cpu") -> torch.Tensor:
    g = _gen(seed, tid, device)
    return (torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std).to(torch.bfloat16)


def uniform_bytes(shape, seed: int, tid: int, device="cpu") -> torch.Tensor:
    g = _gen(seed, tid, device)
    return torch.randint(0, 256, shape, generator=g, device=device, dtype=torch.uint8)


def uniform_ints_u8(shape, lo: int, hi: int, seed: int, tid: int, device="cpu") -> torch.Tensor:
    g = _gen(seed, tid, device)
    return torch.randint(lo, hi + 1, shape, generator=g, device=device, dtype=torch.uint8)


def tokens(M: int, H: int, seed: int, tid: int = 0, device="cpu") -> torch.Tensor:
    """Activations x bf16 [M,H] ~ N(0,1)."""
    return normal_bf16((M, H), 1.0, seed, 9_000 + tid, device)


def layer(shape: LayerShape, seed: int, layer_idx: int = 0, device="cpu", shared: bool = True) -> dict:
    """One MoE layer's weights, generated on ``device``."""
    S, b = shape, 100 * (layer_idx + 1)
    out = {
        "wr": normal_bf16((S.E, S.H), 0.02, seed, b + 1, device),
        "w13c": uniform_bytes((S.E, 2 * S.I, S.H // 2), seed, b + 2, device),
        "w13s": uniform_ints_u8((S.E, 2 * S.I, S.H // 32), S.e_lo, S.e_hi, seed, b + 3, device),
        "w2c": uniform_bytes((S.E, S.H, S.I // 2), seed, b + 4, device),
        "w2s": uniform_ints_u8((S.E, S.H, S.I // 32), S.e_lo, S.e_hi, seed, b + 5, device),
    }
    if shared:
        out["sw13"] = normal_bf16((2 * S.Is, S.H), 0.02, seed, b + 6, device)
        out["sw2"] = normal_bf16((S.H, S.Is), 0.02, seed, b + 7, device)
    return out


def lm_head(V: int, H: int, seed: int, device="cpu") -> torch.Tensor:
    """BF16 LM-head weight [V,H] ~ N(0, 0.02)."""
    return normal_bf16((V, H), 0.02, seed, 7_777, device)


def permutation(n: int, seed: int, tid: int = 4_242) -> torch.Tensor:
    """A seeded permutation of range(n) (for the forced disjoint routing)."""
    g = _gen(seed, tid, "cpu")
    return torch.randperm(n, generator=g)


def bits(t: torch.Tensor):
    """Host numpy view of a tensor's raw bits (bf16 -> uint16, uint8 as is)."""
    t = t.detach().to("cpu").contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view("uint16")
    return t.numpy()


def e4m3_codes(shape, seed: int, tid: int = 6_001, device="cpu") -> torch.Tensor:
    """Uniform E4M3 code bytes with the two NaN codes (0x7F, 0xFF) redrawn as 0x00
    -- for exercising the FP8 GEMV on its own, independent of any quantiser."""
    c = uniform_bytes(shape, seed, tid, device)
    return torch.where((c & 0x7F) == 0x7F, torch.zeros_like(c), c)


def row_scales(V: int, seed: int, tid: int = 6_002, device="cpu") -> torch.Tensor:
    """Positive fp32 row scales, log-uniform in [2^-14, 2^-8]."""
    g = _gen(seed, tid, device)
    u = torch.rand((V,), generator=g, device=device, dtype=torch.float32)
    return torch.exp2(-14.0 + 6.0 * u)


# ---------------------------------------------------------------------------
# Inputs of the library's start-up self-check: a counter-based generator
# (SplitMix64's output function, Steele, Lea & Flood, "Fast splittable pseudorandom
# number generators", OOPSLA 2014) that the library reimplements on the device from
# the same definition, so both sides hold the same bytes without sharing code.
# ---------------------------------------------------------------------------
SELFCHECK = LayerShape(H=256, I=64, E=16, k=2, Is=64, e_lo=120, e_hi=127)
SELFCHECK_V = 256
SELFCHECK_M = 4
SELFCHECK_LAYERS = 2
SELFCHECK_BASE = 0x5EED000000000000
SELFCHECK_TIDS = {"x": 1, "wr": 2, "w13c": 3, "w13s": 4, "w2c": 5, "w2s": 6, "sw13": 7, "sw2": 8,
                  "lm_q": 9, "lm_s": 10}


def splitmix64(counter):
    """SplitMix64 output function of uint64 counters (numpy, wrapping arithmetic)."""
    import numpy as np
    with np.errstate(over="ignore"):  # wrap-around modulo 2^64 is the definition
        z = np.asarray(counter, dtype=np.uint64) + np.uint64(0x9E3779B97F4A7C15)
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
        return z ^ (z >> np.uint64(31))


def selfcheck_inputs():
    """Raw bits of the self-check: a 4-token window x, one tiny MoE layer (used for every
    layer of the self-check's step) and its 256-row FP8 head.
    Element i of tensor `tid` draws r = splitmix64(BASE + tid * 2^32 + i):
      bf16  sign r>>63, exponent e0 + ((r>>56) & 3), mantissa r & 0x7F
            (e0 125 for x, 119 for the router and shared weights)
      MXFP4 codes r & 0xFF; E8M0 scales 120 + r % 8
      e4m3 head codes r & 0xFF with the NaN codes (0x7F, 0xFF) replaced by 0
      fp32 head row scales 2^-(8 + r % 6)."""
    import numpy as np
    S, V = SELFCHECK, SELFCHECK_V
    sizes = {"x": SELFCHECK_M * S.H, "wr": S.E * S.H, "w13c": S.E * 2 * S.I * S.H // 2, "w13s": S.E * 2 * S.I * S.H // 32,
             "w2c": S.E * S.H * S.I // 2, "w2s": S.E * S.H * S.I // 32, "sw13": 2 * S.Is * S.H,
             "sw2": S.H * S.Is, "lm_q": V * S.H, "lm_s": V}

    def r(name):
        i = np.arange(sizes[name], dtype=np.uint64)
        return splitmix64(np.uint64(SELFCHECK_BASE) + (np.uint64(SELFCHECK_TIDS[name]) << np.uint64(32)) + i)

    def bf16(name, e0):
        v = r(name)
        b = ((v >> np.uint64(63)) << np.uint64(15)) | ((np.uint64(e0) + ((v >> np.uint64(56)) & np.uint64(3)))
                                                       << np.uint64(7)) | (v & np.uint64(0x7F))
        return b.astype(np.uint16)

    out = {"x": bf16("x", 125).reshape(SELFCHECK_M, S.H), "wr": bf16("wr", 119).reshape(S.E, S.H),
           "sw13": bf16("sw13", 119).reshape(2 * S.Is, S.H), "sw2": bf16("sw2", 119).reshape(S.H, S.Is)}
    out["w13c"] = (r("w13c") & np.uint64(0xFF)).astype(np.uint8).reshape(S.E, 2 * S.I, S.H // 2)
    out["w13s"] = (np.uint64(120) + r("w13s") % np.uint64(8)).astype(np.uint8).reshape(S.E, 2 * S.I, S.H // 32)
    out["w2c"] = (r("w2c") & np.uint64(0xFF)).astype(np.uint8).reshape(S.E, S.H, S.I // 2)
    out["w2s"] = (np.uint64(120) + r("w2s") % np.uint64(8)).astype(np.uint8).reshape(S.E, S.H, S.I // 32)
    q = (r("lm_q") & np.uint64(0xFF)).astype(np.uint8)
    q[(q & 0x7F) == 0x7F] = 0
    out["lm_q"] = q.reshape(V, S.H)
    e = (np.uint64(127 - 8) - r("lm_s") % np.uint64(6)).astype(np.uint32) << np.uint32(23)
    out["lm_s"] = e.view(np.float32)
    return out
