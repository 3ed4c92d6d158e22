"""Pins of the oracle beyond the step: the multi-token-prediction verify rule, the
BF16 head, and temperature / top-k / top-p sampling.

The verify rule is pinned on its defining cases; the BF16 head against the FP8
head on weights the FP8 quantiser represents exactly (scale 1, codes exact); the
sampler by its special cases (top_k = 1 is the argmax, a tiny top_p keeps the top
token), the inverse-CDF law (over evenly spaced draws each token is picked with its
renormalised nucleus probability) and temperature invariance."""
import numpy as np

import oracle


def test_mtp_accept_cases():
    am = [11, 22, 33, 44]
    assert oracle.mtp_accept(am, [11, 22, 33]) == [4, 11, 22, 33, 44]   # every draft accepted + bonus
    assert oracle.mtp_accept(am, [99, 22, 33]) == [1, 11]               # first draft rejected
    assert oracle.mtp_accept(am, [11, 99, 33]) == [2, 11, 22]           # later drafts never rescue
    assert oracle.mtp_accept(am, [11, 22, 0]) == [3, 11, 22, 33]
    assert oracle.mtp_accept([7, 8], [7]) == [2, 7, 8]


def test_bf16_head_equals_fp8_head_on_exact_weights():
    rng = np.random.default_rng(3)
    V, H, M = 64, 128, 3
    codes = rng.integers(0, 256, size=(V, H)).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x01          # no NaN codes
    codes[:, 5] = 0x7E                             # every row reaches 448: scale exactly 1
    vals = np.array([[oracle.e4m3(int(c)) for c in row] for row in codes])
    w = np.array([[oracle.bf16_rne(v) for v in row] for row in vals], np.uint16)  # exact in bf16
    q, s = oracle.lmhead_quantize(w)
    assert np.all(s == 1.0)
    deq = np.array([[oracle.e4m3(int(c)) for c in row] for row in q]) * s[:, None]
    np.testing.assert_array_equal(deq, vals)        # the quantiser reproduces the exact codes' values
    x = np.array([[oracle.bf16_rne(v) for v in rng.normal(size=H)] for _ in range(M)], np.uint16)
    lg8, am8, _ = oracle.lmhead_logits(x, q, s)
    lgb, amb, _ = oracle.lmhead_logits_bf16(x, w)
    np.testing.assert_allclose(lgb, lg8, rtol=0, atol=1e-9 * np.abs(lg8).max())
    np.testing.assert_array_equal(amb, am8)


def test_bf16_head_one_hot():
    rng = np.random.default_rng(4)
    V, H = 40, 64
    w = np.array([[oracle.bf16_rne(v) for v in rng.normal(size=H)] for _ in range(V)], np.uint16)
    x = np.zeros((1, H), np.uint16)
    x[0, 17] = oracle.bf16_rne(1.0)
    lg, am, _ = oracle.lmhead_logits_bf16(x, w)
    col = np.array([oracle.bf16_value(int(w[v, 17])) for v in range(V)])
    np.testing.assert_array_equal(lg[0], col)
    assert am[0] == int(np.argmax(col))


def test_sample_special_cases():
    rng = np.random.default_rng(5)
    lg = rng.normal(size=(6, 50)) * 3
    u = rng.random(6)
    ids, _ = oracle.sample(lg, 0.8, 1, 0.95, u)
    np.testing.assert_array_equal(ids, np.argmax(lg, axis=1))          # top_k = 1: the argmax
    ids, _ = oracle.sample(lg, 1.3, 29, 1e-9, u)
    np.testing.assert_array_equal(ids, np.argmax(lg, axis=1))          # tiny top_p: the top token
    lg2 = lg.copy()
    lg2[0, 7] = lg2[0, 3] = lg2[0].max() + 1.0                          # tie at the top: lower index first
    ids, _ = oracle.sample(lg2[:1], 1.0, 1, 0.95, u[:1])
    assert ids[0] == 3


def test_sample_inverse_cdf_law_and_temperature():
    z = np.array([[2.0, 1.0, 0.5, 0.0, -1.0, -3.0, 1.0]])
    T, k, p = 0.9, 5, 0.9
    N = 4000
    us = (np.arange(N) + 0.5) / N
    counts = np.zeros(z.shape[1])
    for uu in us:
        i, _ = oracle.sample(z, T, k, p, np.array([uu]))
        counts[i[0]] += 1
    # the law, written independently: top-5 by (z desc, index asc), softmax, nucleus, renormalise
    order = sorted(range(z.shape[1]), key=lambda i: (-z[0, i], i))[:k]
    pr = np.exp(z[0, order] / T - z[0, order[0]] / T)
    pr /= pr.sum()
    n = int(np.searchsorted(np.cumsum(pr), p) + 1)
    want = np.zeros(z.shape[1])
    want[order[:n]] = pr[:n] / pr[:n].sum()
    np.testing.assert_allclose(counts / N, want, atol=1.0 / N + 1e-12)
    # temperature acts on the logits only through z = l / T
    u = np.array([0.37])
    a, _ = oracle.sample(z, 0.5, k, p, u)
    b, _ = oracle.sample(z * 2.0, 1.0, k, p, u)
    assert a[0] == b[0]
