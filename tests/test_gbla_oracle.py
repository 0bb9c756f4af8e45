"""Pins of the GBLA oracle (oracle/gbla.py) to things other than itself: element-by-element
loops of each reading on tiny inputs, the linear-time form of the same quantity (associativity),
closed forms and special cases, the order invariance of bidirectional attention, sequence
independence, soft forgetting, and planted mistakes each of which one of the pins catches.
CPU only."""

import math

import numpy as np
import pytest

import oracle.gbla as G


def rand_case(seed, lens=(5, 1, 7), H=2, d=3, W=4, scale=1.0):
    rng = np.random.default_rng(seed)
    T = int(sum(lens))
    so = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    x = {k: rng.normal(size=(T, H, d)) * scale for k in ("q", "k", "v", "z")}
    x["a"] = rng.normal(size=(T, H)) * 2
    for k in ("cq", "ck", "cv"):
        x[k] = rng.normal(size=(H, W, d)) * 0.7
    x["g"] = rng.normal(size=(H, d))
    return x, so


def brute(x, so, eps_a=G.EPS_ATTN, eps_n=G.EPS_NORM):
    """Every reading as nested loops over scalars (math module only)."""
    T, H, d = x["q"].shape
    W = x["cq"].shape[1]
    seq = [next(i for i in range(len(so) - 1) if so[i] <= t < so[i + 1]) for t in range(T)]

    def conv(name, c, t, h, i):
        tot = 0.0
        for j in range(W):
            if t - j >= so[seq[t]]:
                tot += x[c][h][j][i] * x[name][t - j][h][i]
        return tot

    phi = lambda u: u + 1.0 if u > 0 else math.exp(u)
    y = np.zeros((T, H, d))
    for t in range(T):
        for h in range(H):
            num = [0.0] * d
            den = 0.0
            for s in range(so[seq[t]], so[seq[t] + 1]):
                gate = 1.0 / (1.0 + math.exp(-x["a"][s][h]))
                sim = sum(phi(conv("q", "cq", t, h, i)) * phi(conv("k", "ck", s, h, i)) for i in range(d))
                for i in range(d):
                    num[i] += gate * sim * conv("v", "cv", s, h, i)
                den += gate * sim
            o = [num[i] / (den + eps_a) for i in range(d)]
            ms = sum(u * u for u in o) / d
            for i in range(d):
                zz = x["z"][t][h][i]
                y[t][h][i] = o[i] / math.sqrt(ms + eps_n) * x["g"][h][i] * zz / (1.0 + math.exp(-zz))
    return y


def run(x, so, rows=None):
    return G.gbla_forward(x["q"], x["k"], x["v"], x["a"], x["z"], x["cq"], x["ck"], x["cv"], x["g"], so, rows)


def linear_form(x, so):
    """o through the sequence state: S = sum_s w phi(k~) v~^T, n = sum_s w phi(k~), o = S^T phi(q~)/(n.phi(q~)+eps)."""
    qt = G.feature_map(G.causal_conv(x["q"], x["cq"], so))
    kt = G.feature_map(G.causal_conv(x["k"], x["ck"], so))
    vt = G.causal_conv(x["v"], x["cv"], so)
    w = G.key_gate(x["a"])
    o = np.zeros_like(vt)
    for i in range(len(so) - 1):
        sl = slice(so[i], so[i + 1])
        S = np.einsum("sh,shi,shj->hij", w[sl], kt[sl], vt[sl])
        n = np.einsum("sh,shi->hi", w[sl], kt[sl])
        o[sl] = np.einsum("thi,hij->thj", qt[sl], S) / (np.einsum("thi,hi->th", qt[sl], n)[..., None] + G.EPS_ATTN)
    return o


@pytest.mark.parametrize("seed", range(4))
def test_matches_elementwise_loops(seed):
    x, so = rand_case(seed)
    np.testing.assert_allclose(run(x, so), brute(x, so), rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("seed", range(4))
def test_quadratic_definition_equals_linear_time_form(seed):
    x, so = rand_case(10 + seed, lens=(40, 3, 65), H=3, d=8)
    o = G.gbla_attention(x["q"], x["k"], x["v"], x["a"], x["cq"], x["ck"], x["cv"], so)
    np.testing.assert_allclose(o, linear_form(x, so), rtol=1e-10, atol=1e-12)


def test_sampled_rows_equal_full_rows():
    x, so = rand_case(3, lens=(30, 20), H=2, d=4)
    rows = [29, 0, 31, 5]
    np.testing.assert_allclose(run(x, so, rows), run(x, so)[rows], rtol=1e-13)


def identity_conv(x):
    for k in ("cq", "ck", "cv"):
        x[k] = np.zeros_like(x[k])
        x[k][:, 0, :] = 1.0


def test_plain_kernelized_linear_attention_special_case():
    """Identity convolution, gates at 1, unit norm weight and a huge output gate (silu(z) = z):
    y is the RMS-normalised kernelized linear attention phi(Q)(phi(K)^T V)/(phi(Q) phi(K)^T 1)
    times z, written here with matrix products of the textbook form."""
    x, so = rand_case(5, lens=(12,), H=1, d=4)
    identity_conv(x)
    x["a"][:] = 60.0
    x["g"][:] = 1.0
    x["z"] = np.abs(x["z"]) + 50.0
    elu1 = lambda u: np.where(u > 0, u + 1, np.exp(np.minimum(u, 0)))
    q, k, v = elu1(x["q"][:, 0]), elu1(x["k"][:, 0]), x["v"][:, 0]
    o = (q @ (k.T @ v)) / ((q @ k.T).sum(1, keepdims=True) + G.EPS_ATTN)
    y = o / np.sqrt((o ** 2).mean(1, keepdims=True) + G.EPS_NORM) * x["z"][:, 0]
    np.testing.assert_allclose(run(x, so)[:, 0], y, rtol=1e-9)


def test_constant_values_come_out_unchanged():
    x, so = rand_case(6, lens=(9, 4), H=2, d=3)
    identity_conv(x)
    x["v"][:] = np.array([0.5, -2.0, 3.0])
    o = G.gbla_attention(x["q"], x["k"], x["v"], x["a"], x["cq"], x["ck"], x["cv"], so)
    np.testing.assert_allclose(o, np.broadcast_to(x["v"], o.shape), rtol=1e-5)


def test_single_token_sequence():
    x, so = rand_case(7, lens=(1,), H=1, d=5)
    o = G.gbla_attention(x["q"], x["k"], x["v"], x["a"], x["cq"], x["ck"], x["cv"], so)
    vt = x["cv"][0, 0] * x["v"][0, 0]
    qt, kt = G.feature_map(x["cq"][0, 0] * x["q"][0, 0]), G.feature_map(x["ck"][0, 0] * x["k"][0, 0])
    sim = G.key_gate(x["a"][0, 0]) * float(qt @ kt)
    np.testing.assert_allclose(o[0, 0], vt * sim / (sim + G.EPS_ATTN), rtol=1e-12)


def test_token_order_does_not_matter_without_the_convolution():
    """Bidirectional attention: with an identity convolution, permuting the tokens of a
    sequence permutes its outputs the same way."""
    x, so = rand_case(8, lens=(11,), H=2, d=4)
    identity_conv(x)
    perm = np.random.default_rng(0).permutation(11)
    xp = {k: (v[perm] if k in ("q", "k", "v", "z", "a") else v) for k, v in x.items()}
    np.testing.assert_allclose(run(xp, so), run(x, so)[perm], rtol=1e-12)


def test_convolution_is_causal_and_stays_inside_its_sequence():
    x, so = rand_case(9, lens=(6, 6), H=1, d=2)
    y0 = G.causal_conv(x["k"], x["ck"], so)
    x2 = dict(x)
    x2["k"] = x["k"].copy()
    x2["k"][3] += 5.0                       # a later token of sequence 0
    y1 = G.causal_conv(x2["k"], x["ck"], so)
    np.testing.assert_array_equal(y0[:3], y1[:3])
    assert not np.allclose(y0[3:6], y1[3:6])          # rows 3..5 see token 3
    np.testing.assert_array_equal(y0[6:], y1[6:])   # sequence 1 does not see sequence 0


def test_sequences_are_independent():
    x, so = rand_case(11, lens=(7, 9), H=2, d=3)
    full = run(x, so)
    for i in range(2):
        sl = slice(so[i], so[i + 1])
        xi = {k: (v[sl] if k in ("q", "k", "v", "z", "a") else v) for k, v in x.items()}
        np.testing.assert_allclose(run(xi, np.array([0, so[i + 1] - so[i]])), full[sl], rtol=1e-13)


def test_closed_gate_forgets_the_token():
    """A gate logit of -inf removes that token's key/value from every sum (soft forgetting in
    the limit), while the token still gets an output."""
    x, so = rand_case(12, lens=(8,), H=1, d=3)
    identity_conv(x)
    x["a"][2] = -800.0
    o = G.gbla_attention(x["q"], x["k"], x["v"], x["a"], x["cq"], x["ck"], x["cv"], so)
    keep = [t for t in range(8) if t != 2]
    w = G.key_gate(x["a"][keep, 0])
    for t in range(8):
        sim = w * (G.feature_map(x["k"][keep, 0]) @ G.feature_map(x["q"][t, 0]))
        np.testing.assert_allclose(o[t, 0], sim @ x["v"][keep, 0] / (sim.sum() + G.EPS_ATTN), rtol=1e-12)


def test_rmsnorm_output_has_unit_rms_before_the_gates():
    x, so = rand_case(13, lens=(10,), H=2, d=6)
    y = run(x, so)
    silu = x["z"] / (1 + np.exp(-x["z"]))
    r = y / (x["g"][None] * silu)
    rms = np.sqrt((r ** 2).mean(-1))
    o = G.gbla_attention(x["q"], x["k"], x["v"], x["a"], x["cq"], x["ck"], x["cv"], so)
    want = np.sqrt((o ** 2).mean(-1) / ((o ** 2).mean(-1) + G.EPS_NORM))
    np.testing.assert_allclose(rms, want, rtol=1e-10)


# Planted mistakes: each variant of the oracle must fail at least one pin above.

def _plant(monkeypatch, name):
    if name == "relu_feature_map":
        monkeypatch.setattr(G, "feature_map", lambda u: np.maximum(G._f64(u), 0.0))
    elif name == "no_gate":
        monkeypatch.setattr(G, "key_gate", lambda a: np.ones_like(G._f64(a)))
    elif name == "anticausal_conv":
        orig = G.causal_conv
        monkeypatch.setattr(G, "causal_conv", lambda x, c, so: orig(G._f64(x)[::-1], c, so)[::-1])
    elif name == "no_norm_eps":
        orig = G.gated_rmsnorm
        monkeypatch.setattr(G, "gated_rmsnorm", lambda o, z, g, eps=0.0: orig(o, z, g, 0.5))
    elif name == "sigmoid_output_gate":
        def bad(o, z, g, eps=G.EPS_NORM):
            o, z, g = G._f64(o), G._f64(z), G._f64(g)
            return o / np.sqrt((o * o).mean(-1, keepdims=True) + eps) * g[None] / (1 + np.exp(-z))
        monkeypatch.setattr(G, "gated_rmsnorm", bad)


@pytest.mark.parametrize("mistake", ["relu_feature_map", "no_gate", "anticausal_conv", "no_norm_eps",
                                     "sigmoid_output_gate"])
def test_planted_mistakes_are_caught(monkeypatch, mistake):
    x, so = rand_case(0)
    want = brute(x, so)
    _plant(monkeypatch, mistake)
    got = run(x, so)
    assert not np.allclose(got, want, rtol=1e-6, atol=1e-9), f"{mistake} not caught"
