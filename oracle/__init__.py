"""CPU oracle for the batch-1 MXFP4 MoE decode step (fp64, plain loops in C).

TEST INFRASTRUCTURE ONLY: tests/, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package; the product library never
does, and this package imports nothing from it.

The arithmetic lives in ``moe_oracle.c`` (built on first use with gcc, OpenMP,
no fast-math, no FP contraction).  This wrapper only marshals numpy arrays and
composes per-layer calls into the chained decode step.  Tensors cross as raw
bits: BF16 as uint16, MXFP4/E4M3 codes and E8M0 scales as uint8.

Every function cites what it follows; the source pages are the DGX Spark MoE
knowledge card ("知识卡片：NVIDIA DGX Spark 上提升 MoE 推理吞吐的三种方法",
section 方法/产品要点) and the news retelling ("英伟达称不换芯片也能提速", section
不换卡，快在哪); the number formats follow the OCP Microscaling (MX) v1.0
specification.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")
_lock = threading.Lock()
_lib = None

GCC_FLAGS = ["-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
             "-fno-fast-math", "-fvisibility=hidden", "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into libmoe_oracle.so next to it (gcc)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *GCC_FLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_P = ctypes.c_void_p
_I = ctypes.c_int
_D = ctypes.c_double

_SIGS = {
    "orc_e2m1": (_D, [ctypes.c_uint]),
    "orc_e8m0": (_D, [ctypes.c_uint]),
    "orc_e4m3": (_D, [ctypes.c_uint]),
    "orc_bf16": (_D, [ctypes.c_uint16]),
    "orc_bf16_rne": (ctypes.c_uint16, [_D]),
    "orc_e4m3_encode": (ctypes.c_uint8, [ctypes.c_float]),
    "orc_route": (None, [_P, _I, _I, _P, _I, _I, _P, _P, _P, _P]),
    "orc_moe_layer": (None, [_P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _I, _P]),
    "orc_rmsnorm_bf16": (None, [_P, _I, _I, _D, _P]),
    "orc_lmhead_quantize": (None, [_P, _I, _I, _P, _P]),
    "orc_lmhead_logits": (None, [_P, _I, _I, _I, _P, _P, _P, _P, _P]),
    "orc_mxfp8_quantize": (None, [_P, _I, _I, _P, _P]),
    "orc_moe_layer_prefill": (None, [_P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _I,
                                     _P, _I, _P]),
    "orc_set_threads": (None, [_I]),
}


def set_threads(n: int) -> None:
    """Host threads of the oracle's parallel loops (timing only)."""
    lib().orc_set_threads(int(n))


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            for name, (res, args) in _SIGS.items():
                f = getattr(L, name)
                f.restype = res
                f.argtypes = args
            _lib = L
    return _lib


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


# --------------------------------------------------------------------------
# Formats (OCP MX v1.0 element and scale definitions)
# --------------------------------------------------------------------------

def e2m1(code: int) -> float:
    """FP4 E2M1 value of a 4-bit code (MXFP4 element; knowledge card, method 1)."""
    return lib().orc_e2m1(int(code))


def e8m0(e: int) -> float:
    """E8M0 shared-scale value 2^(e-127); NaN for 0xFF."""
    return lib().orc_e8m0(int(e))


def e4m3(code: int) -> float:
    """FP8 E4M3 (FN) value of a byte (FP8 LM head; knowledge card, method 2)."""
    return lib().orc_e4m3(int(code))


def bf16_value(bits: int) -> float:
    return lib().orc_bf16(int(bits))


def bf16_rne(v: float) -> int:
    """Nearest BF16 bits to v, ties to even."""
    return int(lib().orc_bf16_rne(float(v)))


def e4m3_encode(v: float) -> int:
    """e4m3 code of an fp32 value: nearest, ties to even, saturating at 448."""
    return int(lib().orc_e4m3_encode(float(v)))


# --------------------------------------------------------------------------
# Router (knowledge card, overview: 8 of 512 routed experts per token)
# --------------------------------------------------------------------------

def route(x: np.ndarray, wr: np.ndarray, k: int):
    """Softmax top-k routing of bf16 tokens x [M,H] against bf16 router rows wr [E,H].

    Returns ids int32 [M,k] (descending logit, ties to the lower index),
    renormalised weights fp64 [M,k], logits fp64 [M,E] and the decision margin
    l_(k) - l_(k+1) fp64 [M]."""
    x = _c(x, np.uint16)
    wr = _c(wr, np.uint16)
    M, H = x.shape
    E = wr.shape[0]
    assert wr.shape[1] == H and 0 < k <= E
    ids = np.zeros((M, k), np.int32)
    w = np.zeros((M, k), np.float64)
    logits = np.zeros((M, E), np.float64)
    margin = np.zeros((M,), np.float64)
    lib().orc_route(_p(x), M, H, _p(wr), E, k, _p(ids), _p(w), _p(logits), _p(margin))
    return ids, w, logits, margin


def softmax_weights_at(logits: np.ndarray, ids: np.ndarray) -> np.ndarray:
    """Renormalised routing weights of given (forced) expert ids: the softmax of
    the selected logits, as in the router (used for forced routings)."""
    out = np.zeros(ids.shape, np.float64)
    for t in range(ids.shape[0]):
        sel = logits[t, ids[t]]
        z = np.exp(sel - sel.max())
        out[t] = z / z.sum()
    return out


# --------------------------------------------------------------------------
# MoE layer (knowledge card, method 1; overview: 1 shared expert)
# --------------------------------------------------------------------------

def _compact(ids: np.ndarray, experts):
    """Map the expert ids used by ``ids`` onto a compact index space.

    ``experts`` is either a dict of full expert-indexed arrays
    (w13c [E,2I,H/2], w13s [E,2I,H/32], w2c [E,H,I/2], w2s [E,H,I/32]) or a
    callable ``fetch(list_of_ids) -> dict`` returning those arrays for the listed
    experts only (so a 512-expert layer never has to sit in host memory)."""
    uniq = sorted(set(int(e) for e in ids.reshape(-1)))
    remap = {e: i for i, e in enumerate(uniq)}
    cids = np.vectorize(lambda e: remap[int(e)], otypes=[np.int32])(ids) if ids.size else ids.astype(np.int32)
    if callable(experts):
        arrs = experts(uniq)
    else:
        arrs = {n: experts[n][uniq] for n in ("w13c", "w13s", "w2c", "w2s")}
    return _c(cids, np.int32), arrs, len(uniq)


def moe_layer(x: np.ndarray, ids: np.ndarray, w: np.ndarray, experts, shared=None) -> np.ndarray:
    """Decode MoE layer y [M,H] (fp64) for bf16 x [M,H] under the given routing.

    Routed experts: MXFP4 W13 (gate rows then up rows) and W2, SwiGLU, weighted
    sum with w; shared expert (dict sw13 [2Is,H], sw2 [H,Is] bf16 bits) added
    unweighted.  Activations stay BF16 (weights-only quantisation)."""
    x = _c(x, np.uint16)
    M, H = x.shape
    k = ids.shape[1]
    cids, arrs, nE = _compact(ids, experts)
    w13c = _c(arrs["w13c"], np.uint8)
    w13s = _c(arrs["w13s"], np.uint8)
    w2c = _c(arrs["w2c"], np.uint8)
    w2s = _c(arrs["w2s"], np.uint8)
    I = w13c.shape[1] // 2
    assert w13c.shape[2] * 2 == H and w2c.shape[1] == H and w2c.shape[2] * 2 == I
    sw13 = sw2 = None
    Is = 0
    if shared is not None:
        sw13 = _c(shared["sw13"], np.uint16)
        sw2 = _c(shared["sw2"], np.uint16)
        Is = sw13.shape[0] // 2
    y = np.zeros((M, H), np.float64)
    wd = _c(w, np.float64)
    lib().orc_moe_layer(_p(x), M, H, I, nE, k, _p(cids), _p(wd), _p(w13c), _p(w13s), _p(w2c),
                        _p(w2s), _p(sw13), _p(sw2), Is, _p(y))
    return y


def rmsnorm_bf16(h: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """bf16(h / sqrt(mean(h^2) + eps)) per row: the unit-weight RMSNorm stand-in
    that chains layers (attention is off this path)."""
    h = _c(h, np.float64)
    M, H = h.shape
    out = np.zeros((M, H), np.uint16)
    lib().orc_rmsnorm_bf16(_p(h), M, H, float(eps), _p(out))
    return out


# --------------------------------------------------------------------------
# LM head (knowledge card, method 2; retelling, 不换卡，快在哪)
# --------------------------------------------------------------------------

def lmhead_quantize(wt: np.ndarray):
    """BF16 [V,H] -> (e4m3 codes uint8 [V,H], fp32 row scales [V]); defined in fp32."""
    wt = _c(wt, np.uint16)
    V, H = wt.shape
    q = np.zeros((V, H), np.uint8)
    s = np.zeros((V,), np.float32)
    lib().orc_lmhead_quantize(_p(wt), V, H, _p(q), _p(s))
    return q, s


def lmhead_logits(x: np.ndarray, q: np.ndarray, s: np.ndarray):
    """fp64 logits [M,V] = s_v * sum_h e4m3(q[v,h]) x[t,h]; argmax (lowest index on
    ties) and the top1 - top2 gap per row."""
    x = _c(x, np.uint16)
    q = _c(q, np.uint8)
    s = _c(s, np.float32)
    M, H = x.shape
    V = q.shape[0]
    logits = np.zeros((M, V), np.float64)
    am = np.zeros((M,), np.int32)
    gap = np.zeros((M,), np.float64)
    lib().orc_lmhead_logits(_p(x), M, V, H, _p(q), _p(s), _p(logits), _p(am), _p(gap))
    return logits, am, gap


# --------------------------------------------------------------------------
# Prefill chunk: MXFP8 activations (OCP MX conversion rule)
# --------------------------------------------------------------------------

def mxfp8_quantize(v: np.ndarray):
    """fp32 [M,K] -> (e4m3 codes [M,K], E8M0 scales [M,K/32])."""
    v = _c(v, np.float32)
    M, K = v.shape
    q = np.zeros((M, K), np.uint8)
    se = np.zeros((M, K // 32), np.uint8)
    lib().orc_mxfp8_quantize(_p(v), M, K, _p(q), _p(se))
    return q, se


def moe_layer_prefill(x, ids, w, experts, shared, tokens) -> np.ndarray:
    """Prefill-chunk layer output y [len(tokens), H] (fp64) for the listed tokens."""
    x = _c(x, np.uint16)
    M, H = x.shape
    k = ids.shape[1]
    tokens = _c(np.asarray(tokens), np.int32)
    sub = ids[tokens]
    cids_sub, arrs, nE = _compact(sub, experts)
    cids = np.zeros_like(ids, dtype=np.int32)
    cids[tokens] = cids_sub
    w13c = _c(arrs["w13c"], np.uint8)
    w13s = _c(arrs["w13s"], np.uint8)
    w2c = _c(arrs["w2c"], np.uint8)
    w2s = _c(arrs["w2s"], np.uint8)
    I = w13c.shape[1] // 2
    sw13 = sw2 = None
    Is = 0
    if shared is not None:
        sw13 = _c(shared["sw13"], np.uint16)
        sw2 = _c(shared["sw2"], np.uint16)
        Is = sw13.shape[0] // 2
    y = np.zeros((len(tokens), H), np.float64)
    lib().orc_moe_layer_prefill(_p(x), M, H, I, nE, k, _p(_c(cids, np.int32)), _p(_c(w, np.float64)),
                                _p(w13c), _p(w13s), _p(w2c), _p(w2s), _p(sw13), _p(sw2), Is,
                                _p(tokens), len(tokens), _p(y))
    return y


# --------------------------------------------------------------------------
# The chained decode step (layers + LM head)
# --------------------------------------------------------------------------

def decode_step(x0: np.ndarray, layers, lm_q, lm_s, k: int, eps: float = 1e-6, teacher_x=None):
    """The whole decode step: for each layer route + MoE, h <- h + y,
    x <- bf16(RMSNorm(h)); then the FP8 LM head on the final x.

    ``layers`` is a sequence of dicts with 'wr' (bf16 bits [E,H]), 'experts'
    (arrays or fetch callable, see moe_layer) and 'shared'.  With
    ``teacher_x`` (sequence of bf16 [M,H], one per layer and one for the LM
    head) each layer reads the given input instead of the chained one, so a
    routing flip in one layer does not propagate (teacher forcing).
    Returns dict with ids, w, margin, y per layer, the final x, logits, argmax, gap."""
    x = _c(x0, np.uint16)
    h = np.vectorize(bf16_value, otypes=[np.float64])(x) if x.size else x.astype(np.float64)
    out = {"ids": [], "w": [], "margin": [], "y": [], "x": []}
    for li, L in enumerate(layers):
        if teacher_x is not None:
            x = _c(teacher_x[li], np.uint16)
        out["x"].append(x)
        ids, w, logits, margin = route(x, L["wr"], k)
        y = moe_layer(x, ids, w, L["experts"], L.get("shared"))
        out["ids"].append(ids)
        out["w"].append(w)
        out["margin"].append(margin)
        out["y"].append(y)
        h = h + y
        x = rmsnorm_bf16(h, eps)
    if teacher_x is not None and len(teacher_x) > len(layers):
        x = _c(teacher_x[len(layers)], np.uint16)
    out["x"].append(x)
    logits, am, gap = lmhead_logits(x, lm_q, lm_s)
    out.update(logits=logits, argmax=am, gap=gap, h=h)
    return out


# ---------------------------------------------------------------------------
# Beyond the step: the verify window, the BF16 head, sampling
# ---------------------------------------------------------------------------
def mtp_accept(argmax, drafts):
    """Multi-token-prediction verify (DGX Spark MoE knowledge card, 方法/产品要点 item 2:
    a window of the last accepted token plus draft tokens is verified in one step).
    The head's argmax at window position t is its prediction of the token after t;
    draft t+1 is accepted while it equals that prediction, and the head's own token
    at the first mismatch (or after the last draft) is accepted with them.
    Returns [count, token_1, ..., token_count]."""
    argmax = [int(a) for a in argmax]
    drafts = [int(d) for d in drafts]
    assert len(drafts) == len(argmax) - 1
    out = []
    n = 0
    while n < len(drafts) and drafts[n] == argmax[n]:
        out.append(drafts[n])
        n += 1
    out.append(argmax[n])
    return [n + 1] + out


def lmhead_logits_bf16(x: np.ndarray, w: np.ndarray):
    """The BF16 head the FP8 head is quantised from (same knowledge card, item 2):
    logits fp64 [M,V] = W x with bf16 -> fp64 exact operands (a library matmul of the
    exact values), argmax with ties to the lower index, and the top-2 gap [M]."""
    x = _c(x, np.uint16)
    w = _c(w, np.uint16)
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    wf = (w.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    logits = xf @ wf.T
    am = np.argmax(logits, axis=1).astype(np.int32)  # first occurrence = lowest index
    srt = np.sort(logits, axis=1)
    gap = srt[:, -1] - srt[:, -2] if logits.shape[1] > 1 else np.full(logits.shape[0], np.inf)
    return logits, am, gap


def sample(logits: np.ndarray, temperature: float, top_k: int, top_p: float, u: np.ndarray):
    """Temperature / top-k / top-p sampling of one token per row, the random draw
    u [M] in [0, 1) given (the knowledge card's serving settings: temperature,
    top-k 29, top-p 0.95).  Reading, step by step in fp64:
      z = logits / T; S = the top_k largest z (ties to the lower index);
      p_i = softmax of z over S; order S by (p desc, index asc);
      nucleus N = the shortest prefix of that order with sum p >= top_p;
      q = p renormalised over N; the sample is the first i of N (in order) whose
      cumulative q exceeds u (the last of N if rounding leaves none).
    Returns (ids int32 [M], margin fp64 [M]): margin = distance of u, and of top_p,
    to the nearest cumulative boundary -- below ~1e-6 the decision depends on
    rounding and a comparison is flagged rather than failed."""
    logits = np.asarray(logits, np.float64)
    M, V = logits.shape
    ids = np.zeros(M, np.int32)
    margin = np.zeros(M, np.float64)
    for t in range(M):
        z = logits[t] / float(temperature)
        order = sorted(range(V), key=lambda i: (-z[i], i))[:top_k]
        zm = z[order[0]]
        e = [np.exp(z[i] - zm) for i in order]
        den = sum(e)
        p = [v / den for v in e]
        # (p desc, index asc) is the z order already: p is monotone in z
        cum, n = 0.0, 0
        bounds_p = []
        while True:
            cum += p[n]
            bounds_p.append(cum)
            n += 1
            if cum >= top_p or n == len(p):
                break
        mass = cum
        q = [v / mass for v in p[:n]]
        c, pick = 0.0, n - 1
        bounds_q = []
        for j in range(n):
            c += q[j]
            bounds_q.append(c)
            if c > u[t]:
                pick = j
                break
        ids[t] = order[pick]
        m = min(abs(b - u[t]) for b in bounds_q)
        m = min(m, min(abs(b - top_p) for b in bounds_p))
        margin[t] = m
    return ids, margin
