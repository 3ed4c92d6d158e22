"""Independent dense numpy evaluations used to pin the oracle.

These never call the oracle: formats decode through the published E2M1 table
fixture, ``np.ldexp`` and torch's own bf16 / float8_e4m3fn types, and the MoE
is evaluated densely over *all* experts and mixed with a gate vector that is
zero off the selected experts (the dense-equivalent form of a sparse MoE).
"""
import math

import numpy as np
import torch
from scipy.special import expit

from tests._golden import e2m1_table

_E2M1 = e2m1_table()


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(bits).astype(np.uint16).view(np.int16)).view(
        torch.bfloat16).to(torch.float64).numpy()


def e4m3_to_f64(codes: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).view(
        torch.float8_e4m3fn).to(torch.float64).numpy()


def dequant_mxfp4(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """[..., R, C/2] codes + [..., R, C/32] scales -> float64 [..., R, C]."""
    lo = codes & 0x0F
    hi = codes >> 4
    nib = np.stack([lo, hi], axis=-1).reshape(*codes.shape[:-1], codes.shape[-1] * 2)
    vals = _E2M1[nib]
    sc = np.ldexp(1.0, scales.astype(np.int64) - 127)
    sc = np.repeat(sc, 32, axis=-1)
    return vals * sc


def dequant_mxfp8(q: np.ndarray, se: np.ndarray) -> np.ndarray:
    v = e4m3_to_f64(q)
    return v * np.repeat(np.ldexp(1.0, se.astype(np.int64) - 127), 32, axis=-1)


def silu(g):
    return g * expit(g)


def dense_moe(x_bits, gate, L):
    """y = sum_e gate[:, e] * W2_e (silu(Wg_e x) * Wu_e x) + shared(x), evaluated for every e."""
    x = bf16_to_f64(x_bits)
    W13 = dequant_mxfp4(L["w13c"], L["w13s"])  # [E, 2I, H]
    W2 = dequant_mxfp4(L["w2c"], L["w2s"])     # [E, H, I]
    E, twoI, H = W13.shape
    I = twoI // 2
    gu = np.einsum("erh,mh->emr", W13, x)        # [E, M, 2I]
    a = silu(gu[..., :I]) * gu[..., I:]
    ye = np.einsum("ehi,emi->emh", W2, a)        # [E, M, H]
    y = np.einsum("me,emh->mh", gate, ye)
    if "sw13" in L:
        S13 = bf16_to_f64(L["sw13"])
        S2 = bf16_to_f64(L["sw2"])
        Is = S13.shape[0] // 2
        g = x @ S13.T
        y = y + (silu(g[:, :Is]) * g[:, Is:]) @ S2.T
    return y


def mxfp8_ref(v: np.ndarray):
    """Reference MXFP8 conversion of fp32 rows: scale exponent from frexp,
    element codes from torch's float8_e4m3fn (RNE) with saturation at 448."""
    v = np.asarray(v, np.float32)
    M, K = v.shape
    q = np.zeros((M, K), np.uint8)
    se = np.zeros((M, K // 32), np.uint8)
    for t in range(M):
        for b in range(K // 32):
            blk = v[t, 32 * b:32 * b + 32]
            amax = float(np.max(np.abs(blk)))
            if amax == 0.0:
                s = -127
            else:
                s = min(127, max(-127, math.frexp(amax)[1] - 1 - 8))
            se[t, b] = s + 127
            sc = (blk.astype(np.float64) * 2.0 ** (-s)).astype(np.float32)
            sc = np.clip(sc, -448.0, 448.0)
            q[t, 32 * b:32 * b + 32] = torch.from_numpy(sc).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
            if amax == 0.0:
                q[t, 32 * b:32 * b + 32] = 0
    return q, se
