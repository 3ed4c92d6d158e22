"""Writes the expected results of the library's start-up self-check.

The self-check (moe_selfcheck in the C ABI) generates, on the device, a 4-token window x,
one tiny MoE layer (hidden 256, intermediate 64, 16 experts, top-2, a shared expert of 64)
and a 256-row FP8 LM head from a counter-based generator, then runs the router and the
expert layer on token 0, the head and its verify window on the 4 tokens, and a 2-layer
decode step (the same layer twice) on
token 0 alone and on the whole window.  This script draws the same bytes
(moe_decode_weight_router_b200.synth.selfcheck_inputs), computes every expected result
with the CPU oracle only, and writes them as C constants:

    python oracle/selfcheck_expected.py > moe_decode_weight_router_b200/csrc/selfcheck_expected.inc

It refuses inputs whose routing or argmax would be decided within 1e-3 (the self-check
compares expert ids and argmaxes bit for bit)."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from moe_decode_weight_router_b200 import synth  # noqa: E402


def _floats(name, v):
    vals = [float(np.float32(a)).hex() + "f" for a in np.asarray(v).reshape(-1)]
    lines = [f"static const float {name}[{len(vals)}] = {{"]
    lines += ["    " + ", ".join(vals[i:i + 4]) + "," for i in range(0, len(vals), 4)]
    return lines + ["};"]


def _ints(name, v):
    v = np.asarray(v).reshape(-1)
    return [f"static const int {name}[{len(v)}] = {{{', '.join(str(int(a)) for a in v)}}};"]


def expected():
    S = synth.SELFCHECK
    d = synth.selfcheck_inputs()
    experts = {n: d[n] for n in ("w13c", "w13s", "w2c", "w2s")}
    shared = {"sw13": d["sw13"], "sw2": d["sw2"]}
    x0 = d["x"][:1]
    ids, w, _, margin = oracle.route(x0, d["wr"], S.k)
    y = oracle.moe_layer(x0, ids, w, experts, shared)
    _, am, gap = oracle.lmhead_logits(d["x"], d["lm_q"], d["lm_s"])
    layer = {"wr": d["wr"], "experts": experts, "shared": shared}
    st = oracle.decode_step(d["x"], [layer] * synth.SELFCHECK_LAYERS, d["lm_q"], d["lm_s"], S.k)
    margins = [float(margin[0])] + [float(m) for ml in st["margin"] for m in ml]
    assert min(margins) >= 1e-3, f"routing margin {min(margins)} too small for a bit-exact check"
    top = np.abs(st["logits"]).max(axis=1)
    assert np.all(gap >= 1e-3) and np.all(st["gap"] >= 1e-3 * np.maximum(top, 1.0)), "argmax gap too small"
    return ids, y, am, st


def main():
    ids, y, am, st = expected()
    out = ["// Expected results of moe_selfcheck, written by oracle/selfcheck_expected.py from the",
           "// CPU oracle (fp64) on the self-check inputs; do not edit."]
    out += _ints("kSelfcheckIds", ids[0])
    out += _ints("kSelfcheckHeadArgmax", am)
    out += _floats("kSelfcheckY", y[0])
    out += _ints("kSelfcheckStepArgmax", st["argmax"])
    out += _floats("kSelfcheckStepLogits", st["logits"])
    print("\n".join(out))


if __name__ == "__main__":
    main()
