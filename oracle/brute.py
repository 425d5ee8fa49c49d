"""Stdlib-Python brute force for tiny Differential Attention V2 cases.

TEST INFRASTRUCTURE ONLY (see the package docstring): never imported by the product path.

This is the second, independent implementation used to check the NumPy oracle. It uses
only lists, `math.exp` and explicit loops. Each attention weight is evaluated straight
from the weight formula of the "Differential Attention (V2)" lesson ("The noise floor of
softmax"), divided through by its own numerator: w_i = 1 / sum_j exp(x_j - x_i). The rows
of the two branches are subtracted as in "The differential concept" (A1 - lambda A2) and
multiplied by V. Causal attention lets query i see keys j <= i; the sliding window of the
"Attention variants" lesson keeps a query's last `window` keys. The V2 pairing of the
Hugging Face blog summary ("Differential Transformer V2 soll KI-Training stabiler machen",
shared-KV section) maps heads (2p, 2p+1) to KV head 2p*Hkv/Hq.

Inputs are nested Python lists of floats; it is meant for S <= 16, D <= 8 (the weights
cost O(n^2) exponentials per row).
"""
from __future__ import annotations

import math


def _dot(a, b):
    s = 0.0
    for x, y in zip(a, b):
        s += x * y
    return s


def _weights(logits):
    """w_i = e^{x_i} / sum_j e^{x_j} = 1 / sum_j e^{x_j - x_i}, one key at a time."""
    out = []
    for xi in logits:
        denom = 0.0
        for xj in logits:
            denom += math.exp(xj - xi)
        out.append(1.0 / denom)
    return out


def prefill(q, k, v, lam, causal=True, window=None):
    """q[b][i][h][d], k/v[b][j][g][d], lam[b][i][p] -> out[b][i][p][d] (lists of floats).

    window (causal only): query i sees its last `window` keys, i - window < j <= i."""
    B = len(q)
    S = len(q[0])
    Hq = len(q[0][0])
    Hkv = len(k[0][0])
    D = len(q[0][0][0])
    scale = math.sqrt(D)
    out = []
    for b in range(B):
        rows = []
        for i in range(S):
            heads = []
            visible = list(range(i + 1)) if causal else list(range(S))
            if window is not None:
                visible = [j for j in visible if i - j < window]
            for p in range(Hq // 2):
                h1, h2 = 2 * p, 2 * p + 1
                g = (h1 * Hkv) // Hq
                a1 = _weights([_dot(q[b][i][h1], k[b][j][g]) / scale for j in visible])
                a2 = _weights([_dot(q[b][i][h2], k[b][j][g]) / scale for j in visible])
                heads.append([sum((a1[n] - lam[b][i][p] * a2[n]) * v[b][j][g][d]
                                  for n, j in enumerate(visible)) for d in range(D)])
            rows.append(heads)
        out.append(rows)
    return out


def decode(q, kcache, vcache, seqlens, lam):
    """q[b][h][d], caches[b][j][g][d], seqlens[b], lam[b][p] -> out[b][p][d]."""
    B = len(q)
    Hq = len(q[0])
    Hkv = len(kcache[0][0])
    D = len(q[0][0])
    scale = math.sqrt(D)
    out = []
    for b in range(B):
        n = int(seqlens[b])
        heads = []
        for p in range(Hq // 2):
            if n == 0:
                heads.append([0.0] * D)
                continue
            h1, h2 = 2 * p, 2 * p + 1
            g = (h1 * Hkv) // Hq
            a1 = _weights([_dot(q[b][h1], kcache[b][j][g]) / scale for j in range(n)])
            a2 = _weights([_dot(q[b][h2], kcache[b][j][g]) / scale for j in range(n)])
            heads.append([sum((a1[j] - lam[b][p] * a2[j]) * vcache[b][j][g][d] for j in range(n))
                          for d in range(D)])
        out.append(heads)
    return out


def lambda_v1(lq1, lk1, lq2, lk2, lambda_init=0.8):
    """Per-pair V1 lambda from four lists of vectors (one vector per pair)."""
    return [math.exp(_dot(a, b)) - math.exp(_dot(c, e)) + lambda_init
            for a, b, c, e in zip(lq1, lk1, lq2, lk2)]
