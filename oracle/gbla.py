"""Plain fp64 definition of gated bidirectional linear attention, GBLA (TEST INFRASTRUCTURE ONLY).

Source: "Gated Bidirectional Linear Attention for Generative Retrieval" (the GBLA page),
sections "Abstract" and the AI summary above it.  The layer is bidirectional (every token of a
user history attends to every other one), linear-time, and "extends kernelized linear
attention" with three components: local causal mixing by a 1-D convolution, sequence-level key
gating for soft forgetting, and a gated RMSNorm on the output.  The page prints no formula;
the readings taken here (the plainest ones the text supports) are:

  1. Local causal mixing: a depthwise causal convolution of width W = 4 over the tokens of one
     sequence, applied to q, k and v separately, x~[t] = sum_{j<W} c[j] * x[t-j], with zero
     before the sequence's first token (no mixing across sequences).
  2. Kernelized attention with the positive feature map phi(x) = elu(x) + 1 (x + 1 for x > 0,
     exp(x) otherwise), no mask (bidirectional):
        o[t] = sum_s w[s] phi(q~[t]).phi(k~[s]) v~[s] / (sum_s w[s] phi(q~[t]).phi(k~[s]) + eps_a)
  3. Sequence-level key gating: every key's weight in that sum is w[s] = sigmoid(a[s]) in (0, 1),
     one gate logit per token and head (a gate near 0 softly forgets the token for the whole
     sequence).
  4. Gated RMSNorm output: y[t] = o[t] / sqrt(mean_i o[t,i]^2 + eps_n) * g * silu(z[t]), with a
     learned per-channel weight g and an output gate z (one value per token, head and channel).
  eps_a = eps_n = 1e-6.  Heads are independent (H heads of width d).

This module computes (2) as written, the quadratic sum over key tokens per output row: the
definition.  The linear-time form that makes the method fast (S = sum_s w[s] phi(k~[s]) v~[s]^T
and n = sum_s w[s] phi(k~[s]) per sequence and head, then o[t] = S^T phi(q~[t]) / (n.phi(q~[t]) +
eps_a)) is the same quantity by associativity; tests/test_gbla_oracle.py checks the two against
each other, against element-by-element loops and against closed forms.

Layout: token-major [T, H, d] tensors; sequence i owns rows seq_offsets[i] .. seq_offsets[i+1];
gate logits a [T, H]; conv kernels [H, W, d]; norm weight [H, d] (one per head).
"""

from __future__ import annotations

from typing import Iterable, Optional

import numpy as np

EPS_ATTN = 1e-6
EPS_NORM = 1e-6
CONV_WIDTH = 4


def _f64(x):
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().double().cpu().numpy()
    except ImportError:
        pass
    return np.asarray(x, dtype=np.float64)


def causal_conv(x, c, seq_offsets) -> np.ndarray:
    """Reading 1: y[t] = sum_j c[h, j] * x[t - j] over the same sequence (zero before its start).
    x [T, H, d], c [H, W, d]."""
    x, c = _f64(x), _f64(c)
    so = np.asarray(seq_offsets, np.int64)
    y = np.zeros_like(x)
    W = c.shape[1]
    for i in range(len(so) - 1):
        lo, hi = int(so[i]), int(so[i + 1])
        for j in range(W):
            if hi - lo - j <= 0:
                continue
            y[lo + j:hi] += c[None, :, j, :] * x[lo:hi - j]
    return y


def feature_map(x) -> np.ndarray:
    """Reading 2: phi(x) = elu(x) + 1."""
    x = _f64(x)
    return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def key_gate(a) -> np.ndarray:
    """Reading 3: w = sigmoid(a)."""
    a = _f64(a)
    return 0.5 * (1.0 + np.tanh(0.5 * a))   # = 1 / (1 + exp(-a)), without overflow for large |a|


def gbla_attention(q, k, v, a, cq, ck, cv, seq_offsets, rows: Optional[Iterable[int]] = None,
                   eps: float = EPS_ATTN) -> np.ndarray:
    """Reading 2 as written (quadratic in the sequence length): o [T, H, d] (or the rows asked
    for, in that order).  The rows of a sequence attend to every token of that sequence."""
    so = np.asarray(seq_offsets, np.int64)
    qt = feature_map(causal_conv(q, cq, so))
    kt = feature_map(causal_conv(k, ck, so))
    vt = causal_conv(v, cv, so)
    w = key_gate(a)
    T, H, d = qt.shape
    rows = np.arange(T) if rows is None else np.asarray(list(rows), np.int64)
    seq_of = np.searchsorted(so, rows, side="right") - 1
    out = np.zeros((len(rows), H, vt.shape[2]))
    for i, (t, sq) in enumerate(zip(rows, seq_of)):
        lo, hi = int(so[sq]), int(so[sq + 1])
        for h in range(H):
            sim = w[lo:hi, h] * (kt[lo:hi, h] @ qt[t, h])          # [L]
            out[i, h] = (sim @ vt[lo:hi, h]) / (sim.sum() + eps)
    return out


def gated_rmsnorm(o, z, g, eps: float = EPS_NORM) -> np.ndarray:
    """Reading 4: o / rms(o) * g * silu(z), per token and head over the d channels.
    o, z [n, H, d]; g [H, d]."""
    o, z, g = _f64(o), _f64(z), _f64(g)
    rms = np.sqrt((o * o).mean(axis=-1, keepdims=True) + eps)
    silu = z / (1.0 + np.exp(-z))
    return o / rms * g[None] * silu


def gbla_forward(q, k, v, a, z, cq, ck, cv, g, seq_offsets, rows: Optional[Iterable[int]] = None) -> np.ndarray:
    """The layer: gated RMSNorm of the gated kernelized attention.  Returns y for all rows (or
    the rows asked for, in that order)."""
    o = gbla_attention(q, k, v, a, cq, ck, cv, seq_offsets, rows)
    zz = _f64(z)
    if rows is not None:
        zz = zz[np.asarray(list(rows), np.int64)]
    return gated_rmsnorm(o, zz, g)
