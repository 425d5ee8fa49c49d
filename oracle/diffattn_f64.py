"""NumPy float64 oracle: the plain definition of forward Differential Attention V2.

TEST INFRASTRUCTURE ONLY (see the package docstring): never imported by the product path.

Sources (page title, then section / equation):
  [L16]  "Differential Attention (V2)" lesson (AI Engineering from Scratch, phase 10, 16):
         "The noise floor of softmax" -- the attention weight of key i,
         w_i = exp(q.k_i / sqrt(d)) / sum_j exp(q.k_j / sqrt(d));
         "The differential concept" -- A1 = softmax(Q1 K1^T / sqrt(d)),
         A2 = softmax(Q2 K2^T / sqrt(d)), DiffAttn = (A1 - lambda * A2) V, and the V1
         lambda re-parameterisation lambda = exp(lq1.lk1) - exp(lq2.lk2) + lambda_init;
         key-terms table ("lambda" may be negative; "Signal-to-noise ratio");
         "Exercises" 4 (lambda = 0 is the pure first softmax) and 5 (GQA + V2 cache size).
  [L07]  "Attention variants: sliding window, sparse, differential" lesson (phase 7, 15):
         "Sliding window attention" -- keys outside a query's window get -inf in the score
         matrix; its W = 4 figure and the key-terms table ("each query attends to its last
         W tokens"); causal attention lets query i see keys j <= i.
  [HF]   "Differential Transformer V2 soll KI-Training stabiler machen" (summary of the
         Hugging Face blog), section "Gemeinsamer KV-Cache statt Spezialkernel": two adjacent
         query heads inside one GQA group share K and V; section "Weniger Ausreisser und
         Gradientenspitzen": lambda is projected per token and per head and bounded by a
         sigmoid.

Readings of points the pages leave open (each also listed in the design notes):
  * head 2p of a pair is branch 1 (A1, +), head 2p+1 is branch 2 (A2, -lambda);
  * the KV head of pair p is g = (2p) // (Hq / Hkv);
  * lambda is one value per token and per output head (= pair): [B, S, Hq/2] for prefill,
    [B, Hq/2] for decode; it arrives already bounded (the model applies the sigmoid);
  * the score scale is 1/sqrt(D) for both branches;
  * causal means key j is visible from query i when j <= i, with Sq == Sk;
  * decode attends to keys [0, seqlen_b), the new token's key already appended.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "stable_softmax",
    "causal_mask",
    "window_mask",
    "pair_layout",
    "diff_attention_block",
    "prefill",
    "prefill_rows",
    "prefill_varlen",
    "prefill_backward",
    "prefill_backward_varlen",
    "prefill_branches",
    "decode",
    "decode_paged",
    "decode_multi",
    "lambda_v1",
    "lambda_v2_projection",
    "branch_weights",
    "snr",
]


def stable_softmax(x: np.ndarray) -> np.ndarray:
    """Softmax along the last axis: [L16] "The noise floor of softmax", w_i = e^{x_i} / sum_j e^{x_j}.

    Evaluated as w_i = exp(x_i - LSE(x)) with the log-sum-exp LSE(x) = c + log sum_j e^{x_j - c}
    for c = max_j x_j; the identity holds for every c, and this c keeps every exponent <= 0 so
    nothing overflows. Entries equal to -inf (masked keys) get weight exactly 0. A row must
    hold at least one finite entry.
    """
    x = np.asarray(x, dtype=np.float64)
    c = np.max(x, axis=-1, keepdims=True)
    lse = c + np.log(np.sum(np.exp(x - c), axis=-1, keepdims=True))
    return np.exp(x - lse)


def _additive(visible: np.ndarray) -> np.ndarray:
    """Additive mask of a visibility predicate: 0 where a key is visible, -inf elsewhere
    ([L07] "Sliding window attention": hidden keys get -inf in the score matrix)."""
    return np.where(visible, 0.0, -np.inf)


def causal_mask(n_q: int, n_k: int, q_offset: int = 0) -> np.ndarray:
    """Causal visibility: key j is visible from query i exactly when j <= i.

    Query rows are numbered q_offset .. q_offset + n_q - 1 (a row block of a longer
    sequence); keys are numbered 0 .. n_k - 1.
    """
    i = np.arange(q_offset, q_offset + n_q)[:, None]
    j = np.arange(n_k)[None, :]
    return _additive(j <= i)


def window_mask(n_q: int, n_k: int, window: int, q_offset: int = 0) -> np.ndarray:
    """Causal sliding window of [L07] ("Sliding window attention", its W = 4 figure and the
    key-terms table): query i sees its last `window` keys, i.e. key j with
    i - window < j <= i (the window holds the query's own key). window >= n gives the full
    causal mask; window = 1 leaves only j = i."""
    if window < 1:
        raise ValueError("window must be >= 1")
    i = np.arange(q_offset, q_offset + n_q)[:, None]
    j = np.arange(n_k)[None, :]
    return _additive((j <= i) & (i - j < window))


def pair_layout(Hq: int, Hkv: int):
    """V2 head pairing of [HF] (shared KV cache section) and [L16] "V1 vs V2".

    Returns a list of (p, h1, h2, g): pair p, its branch-1 head h1 = 2p, its branch-2 head
    h2 = 2p+1, and the KV head g both heads read. Both heads of a pair must sit in the same
    GQA group, which holds when Hq is a multiple of 2*Hkv.
    """
    if Hq % 2 != 0 or Hkv <= 0 or Hq % (2 * Hkv) != 0:
        raise ValueError(f"need Hq even and a multiple of 2*Hkv (Hq={Hq}, Hkv={Hkv})")
    G = Hq // Hkv
    out = []
    for p in range(Hq // 2):
        h1, h2 = 2 * p, 2 * p + 1
        g = h1 // G
        assert h2 // G == g
        out.append((p, h1, h2, g))
    return out


def diff_attention_block(q1, q2, k, v, lam, mask):
    """DiffAttn for one pair over a block of query rows: the equations of [L16] "The
    differential concept", A_b = softmax(Q_b K^T / sqrt(D) + mask), DiffAttn = (A_1 - lambda A_2) V.

    q1, q2: [n, D] the two heads of the pair; k, v: [m, D] their shared K/V head;
    lam: [n] one lambda per query row; mask: [n, m] additive (0 or -inf).
    Returns [n, D] = (softmax(q1 k^T / sqrt(D) + mask) - lam * softmax(q2 k^T / sqrt(D) + mask)) v.
    """
    D = q1.shape[-1]
    inv_sqrt_d = 1.0 / math.sqrt(D)
    a1 = stable_softmax(q1 @ k.T * inv_sqrt_d + mask)
    a2 = stable_softmax(q2 @ k.T * inv_sqrt_d + mask)
    w = a1 - lam[:, None] * a2
    return w @ v


def _f64(t) -> np.ndarray:
    """Exact upcast of a torch tensor or array (bf16/fp32 values) to float64."""
    if hasattr(t, "detach"):
        import torch  # local: only for the dtype conversion of inputs

        return t.detach().to(torch.float64).cpu().numpy()
    return np.asarray(t, dtype=np.float64)


def prefill(q, k, v, lam, causal: bool = True, row_block: int = 512, window=None) -> np.ndarray:
    """Forward prefill over the whole batch: out[B, S, Hq/2, D] in float64.

    q [B,S,Hq,D], k/v [B,S,Hkv,D], lam [B,S,Hq/2]. For every batch b and pair p the rows are
    processed in blocks of `row_block` (a memory bound only: every row is computed exactly
    as the definition states, over all its visible keys). `window` (causal only) restricts
    each query to its last `window` keys, the DiffAttn + sliding-window combination that the
    lesson's "Use it" section names for hybrid layers, with the window of `window_mask`.
    """
    if window is not None and not causal:
        raise ValueError("a sliding window is defined for causal attention")
    q, k, v, lam = _f64(q), _f64(k), _f64(v), _f64(lam)
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    out = np.zeros((B, S, Hq // 2, D), dtype=np.float64)
    for b in range(B):
        for p, h1, h2, g in pair_layout(Hq, Hkv):
            kk, vv = k[b, :, g], v[b, :, g]
            for r0 in range(0, S, row_block):
                r1 = min(S, r0 + row_block)
                n_k = r1 if causal else S
                if window is not None:
                    mask = window_mask(r1 - r0, n_k, window, r0)
                else:
                    mask = causal_mask(r1 - r0, n_k, r0) if causal else np.zeros((r1 - r0, S))
                out[b, r0:r1, p] = diff_attention_block(
                    q[b, r0:r1, h1], q[b, r0:r1, h2], kk[:n_k], vv[:n_k], lam[b, r0:r1, p], mask)
    return out


def prefill_varlen(q, k, v, lam, cu_seqlens, causal: bool = True, window=None) -> np.ndarray:
    """Prefill of sequences packed along the token axis: q [T,Hq,D], k/v [T,Hkv,D],
    lam [T,Hq/2], sequence b = tokens cu_seqlens[b] .. cu_seqlens[b+1]-1. Every sequence is an
    independent prefill (its queries see only its own keys); with `window` (causal only) the
    sliding window of the "Attention variants" lesson applies inside each sequence. Returns
    out [T,Hq/2,D]."""
    cu = [int(x) for x in cu_seqlens]
    T = int(q.shape[0])
    out = np.zeros((T, q.shape[1] // 2, q.shape[2]), dtype=np.float64)
    for b in range(len(cu) - 1):
        s0, s1 = cu[b], cu[b + 1]
        if s1 > s0:
            out[s0:s1] = prefill(q[None, s0:s1], k[None, s0:s1], v[None, s0:s1], lam[None, s0:s1], causal=causal,
                                 window=window)[0]
    return out


def prefill_backward(q, k, v, lam, dout, causal: bool = True, window=None):
    """Gradients of the prefill: returns (dq [B,S,Hq,D], dk, dv [B,S,Hkv,D], dlam [B,S,Hq/2])
    for an upstream gradient dout [B,S,Hq/2,D], all float64. With `window` (causal only) the
    mask is the sliding window of `window_mask`.

    The chain rule applied to the definition of `diff_attention_block`, per pair p (heads h1,
    h2 over KV head g) and batch b, with A_b = softmax(S_b), S_b = Q_b K^T / sqrt(D) + mask,
    O_b = A_b V and out = O_1 - lam * O_2:
      dlam_i  = -dout_i . O_2,i
      dV     += A_1^T dout - A_2^T (lam * dout)
      dA_1    = dout V^T,            dA_2 = -lam * (dout V^T)
      dS_b    = A_b * (dA_b - rowsum(A_b * dA_b))           (softmax backward)
      dQ_b    = dS_b K / sqrt(D),    dK += (dS_1^T Q_1 + dS_2^T Q_2) / sqrt(D)
    KV heads accumulate over every pair of their group.
    """
    q, k, v, lam, dout = _f64(q), _f64(k), _f64(v), _f64(lam), _f64(dout)
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    inv = 1.0 / math.sqrt(D)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    dlam = np.zeros_like(lam)
    if window is not None:
        mask = window_mask(S, S, int(window))
    else:
        mask = causal_mask(S, S) if causal else np.zeros((S, S))
    for b in range(B):
        for p, h1, h2, g in pair_layout(Hq, Hkv):
            kk, vv = k[b, :, g], v[b, :, g]
            a1 = stable_softmax(q[b, :, h1] @ kk.T * inv + mask)
            a2 = stable_softmax(q[b, :, h2] @ kk.T * inv + mask)
            lm = lam[b, :, p][:, None]
            do = dout[b, :, p]
            o2 = a2 @ vv
            dlam[b, :, p] = -np.sum(do * o2, axis=1)
            dv[b, :, g] += a1.T @ do - a2.T @ (lm * do)
            dpv = do @ vv.T
            for a, da, h in ((a1, dpv, h1), (a2, -lm * dpv, h2)):
                ds = a * (da - np.sum(a * da, axis=1, keepdims=True))
                dq[b, :, h] = ds @ kk * inv
                dk[b, :, g] += ds.T @ q[b, :, h] * inv
    return dq, dk, dv, dlam


def prefill_backward_varlen(q, k, v, lam, dout, cu_seqlens, causal: bool = True, window=None):
    """Gradients of `prefill_varlen` for packed sequences (q [T,Hq,D], k/v [T,Hkv,D],
    lam [T,Hq/2], dout [T,Hq/2,D]): every sequence is an independent prefill, so its
    gradients are those of its own prefill and no token of one sequence has a gradient
    through another; `window` (causal only) as in `prefill_varlen`. Returns (dq, dk, dv, dlam)
    in the packed layouts, float64."""
    cu = [int(x) for x in cu_seqlens]
    q, k, v, lam, dout = _f64(q), _f64(k), _f64(v), _f64(lam), _f64(dout)
    dq, dk, dv, dlam = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v), np.zeros_like(lam)
    for b in range(len(cu) - 1):
        s0, s1 = cu[b], cu[b + 1]
        if s1 > s0:
            g = prefill_backward(q[None, s0:s1], k[None, s0:s1], v[None, s0:s1], lam[None, s0:s1],
                                 dout[None, s0:s1], causal=causal, window=window)
            dq[s0:s1], dk[s0:s1], dv[s0:s1], dlam[s0:s1] = (x[0] for x in g)
    return dq, dk, dv, dlam


def prefill_branches(q, k, v, causal: bool = True):
    """Per-head pieces of the prefill that a training forward keeps for the backward pass:
    O_h = softmax(Q_h K_g^T / sqrt(D) + mask) V_g for every query head h (float64
    [B,S,Hq,D]), and the row log-sum-exp of the head's scaled scores in base 2,
    lse2_h[i] = log2(sum_j 2^(s_ij * log2(e))) with s = Q_h K_g^T / sqrt(D) (float64
    [B,S,Hq]), so that softmax row i equals 2^(s_ij * log2(e) - lse2_h[i]).

    Heads map to KV heads as in `pair_layout`; out = O_{2p} - lam * O_{2p+1} ("Differential
    Attention (V2)" lesson, "The differential concept")."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    inv = 1.0 / math.sqrt(D)
    mask = causal_mask(S, S) if causal else np.zeros((S, S))
    o = np.zeros_like(q)
    lse2 = np.zeros((B, S, Hq))
    for b in range(B):
        for p, h1, h2, g in pair_layout(Hq, Hkv):
            for h in (h1, h2):
                s_ = q[b, :, h] @ k[b, :, g].T * inv + mask
                o[b, :, h] = stable_softmax(s_) @ v[b, :, g]
                m = np.max(s_, axis=1, keepdims=True)
                lse2[b, :, h] = (m[:, 0] + np.log(np.sum(np.exp(s_ - m), axis=1))) / math.log(2.0)
    return o, lse2


def prefill_rows(q, k, v, lam, rows, causal: bool = True) -> np.ndarray:
    """Selected output rows of a prefill: rows is a list of (b, i, p); returns [len(rows), D].

    Each row is the definition applied to query i of pair p in batch b over keys j <= i
    (causal) or all keys. Used for sampled checks of full-size outputs. The K/V slice of a
    (b, g) is upcast once and shared by the rows that read it.
    """
    Hq = q.shape[2]
    Hkv = k.shape[2]
    layout = {p: (h1, h2, g) for p, h1, h2, g in pair_layout(Hq, Hkv)}
    S = q.shape[1]
    res = [None] * len(rows)
    by_slice = {}
    for n, (b, i, p) in enumerate(rows):
        by_slice.setdefault((b, layout[p][2]), []).append(n)
    for (b, g), idx in by_slice.items():
        n_max = max(rows[n][1] for n in idx) + 1 if causal else S
        kk = _f64(k[b, :n_max, g])
        vv = _f64(v[b, :n_max, g])
        for n in idx:
            _, i, p = rows[n]
            h1, h2, _ = layout[p]
            n_k = i + 1 if causal else S
            q1 = _f64(q[b, i, h1])[None, :]
            q2 = _f64(q[b, i, h2])[None, :]
            lm = np.array([float(lam[b, i, p])], dtype=np.float64)
            res[n] = diff_attention_block(q1, q2, kk[:n_k], vv[:n_k], lm, np.zeros((1, n_k)))[0]
    return np.stack(res) if res else np.zeros((0, q.shape[3]))


def decode(q, kcache, vcache, seqlens, lam, window=None) -> np.ndarray:
    """One decode step: out[B, Hq/2, D] in float64.

    q [B,Hq,D] is the new token's query; the caches [B,Smax,Hkv,D] already hold its key and
    value, and sequence b attends to keys [0, seqlens[b]), or with `window` to its last
    `window` keys [max(0, seqlens[b]-window), seqlens[b]) (the sliding window of the
    "Attention variants" lesson for the newest query). lam [B,Hq/2]. A sequence with
    seqlens[b] == 0 has no visible key; its output is defined as 0.
    """
    B, Hq, D = q.shape
    Hkv = kcache.shape[2]
    out = np.zeros((B, Hq // 2, D), dtype=np.float64)
    for b in range(B):
        n = int(seqlens[b])
        if n <= 0:
            continue
        n0 = max(0, n - int(window)) if window is not None else 0
        for g in range(Hkv):
            kk = _f64(kcache[b, n0:n, g])
            vv = _f64(vcache[b, n0:n, g])
            for p, h1, h2, gg in pair_layout(Hq, Hkv):
                if gg != g:
                    continue
                q1 = _f64(q[b, h1])[None, :]
                q2 = _f64(q[b, h2])[None, :]
                lm = np.array([float(lam[b, p])], dtype=np.float64)
                out[b, p] = diff_attention_block(q1, q2, kk, vv, lm, np.zeros((1, n - n0)))[0]
    return out


def decode_paged(q, kpages, vpages, block_table, seqlens, lam, window=None) -> np.ndarray:
    """Decode step over a paged cache: kpages/vpages [P, page_size, Hkv, D]; logical token t
    of sequence b lives in page block_table[b][t // page_size] at row t % page_size. The
    sequence's logical cache is gathered page by page, then `decode` (with `window`) applies
    as written."""
    page_size = int(kpages.shape[1])
    B = q.shape[0]
    outs = []
    for b in range(B):
        n = int(seqlens[b])
        n_pages = (n + page_size - 1) // page_size
        pages = [int(block_table[b][i]) for i in range(n_pages)]
        kc = np.concatenate([_f64(kpages[pg]) for pg in pages], axis=0)[:n] if n else np.zeros((0,) + tuple(kpages.shape[2:]))
        vc = np.concatenate([_f64(vpages[pg]) for pg in pages], axis=0)[:n] if n else np.zeros((0,) + tuple(vpages.shape[2:]))
        outs.append(decode(q[b:b + 1], kc[None], vc[None], [n], lam[b:b + 1], window=window)[0])
    return np.stack(outs)


def decode_multi(q, kcache, vcache, seqlens, lam) -> np.ndarray:
    """Decode of T new tokens per sequence (a speculative-decoding verification step):
    q [B,T,Hq,D], lam [B,T,Hq/2]; the caches already hold all T new keys, and new token t
    of sequence b attends to keys [0, seqlens[b] - T + t + 1) -- causal among the new tokens.
    Each token is one `decode` over its visible prefix. Returns out [B,T,Hq/2,D]."""
    B, T = q.shape[0], q.shape[1]
    out = np.zeros((B, T, q.shape[2] // 2, q.shape[3]), dtype=np.float64)
    for t in range(T):
        n_t = [max(0, int(seqlens[b]) - T + t + 1) for b in range(B)]
        out[:, t] = decode(q[:, t], kcache, vcache, n_t, lam[:, t])
    return out


def lambda_v1(lq1, lk1, lq2, lk2, lambda_init: float = 0.8) -> np.ndarray:
    """V1 lambda re-parameterisation of [L16] "The differential concept":
    lambda = exp(lq1 . lk1) - exp(lq2 . lk2) + lambda_init, one scalar per pair.

    Inputs are [n_pairs, d] (one set of four vectors per pair); returns [n_pairs] float64.
    The value may be negative or above 1 ([L16] key-terms table, "lambda").
    """
    a, b, c, e = (_f64(x) for x in (lq1, lk1, lq2, lk2))
    return np.exp(np.sum(a * b, axis=-1)) - np.exp(np.sum(c * e, axis=-1)) + float(lambda_init)


def lambda_v2_projection(x, w, bias=None) -> np.ndarray:
    """V2 lambda of [HF] (section "Weniger Ausreisser und Gradientenspitzen"): projected from
    each token's hidden state for each head (pair) and bounded by a sigmoid,
    lambda[t, p] = 1 / (1 + exp(-(x[t] . w[:, p] + bias[p]))). x [T, d_model], w [d_model,
    n_pairs], bias [n_pairs] or None (no bias). Returns [T, n_pairs] in (0, 1)."""
    z = _f64(x) @ _f64(w)
    if bias is not None:
        z = z + _f64(bias)[None, :]
    return 1.0 / (1.0 + np.exp(-z))


def branch_weights(q1, q2, k, lam, n_visible=None):
    """Attention weights of one query row: (a1, a2, a1 - lam * a2) over its visible keys.

    q1, q2: [D]; k: [m, D]. Keys n_visible.. are masked out (weight 0). The rows of A_1,
    A_2 and A_1 - lambda A_2 of [L16] "The differential concept" for one query.
    """
    q1, q2, k = _f64(q1), _f64(q2), _f64(k)
    m = k.shape[0] if n_visible is None else int(n_visible)
    D = q1.shape[-1]
    s1 = k[:m] @ q1 / math.sqrt(D)
    s2 = k[:m] @ q2 / math.sqrt(D)
    a1 = stable_softmax(s1)
    a2 = stable_softmax(s2)
    return a1, a2, a1 - float(lam) * a2


def snr(weights, signal_index: int) -> float:
    """Signal-to-noise ratio of one weight row ([L16] key-terms table, "Signal-to-noise
    ratio"): weight on the signal position over the average weight on the unrelated positions.

    Differential weights can be negative (A_1 - lambda A_2 is a difference of two
    distributions), so the average over unrelated positions is taken of the absolute weights.
    """
    w = np.asarray(weights, dtype=np.float64)
    others = np.delete(w, signal_index)
    return float(w[signal_index] / np.mean(np.abs(others)))
