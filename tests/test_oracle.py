"""Pins for the float64 oracle: checks against what the pages and the mathematics fix.

Every pin compares the oracle with something other than itself: a library routine
(torch scaled_dot_product_attention, scipy softmax), a closed form, an invariant, the
worked example printed on the pages, or the independent stdlib brute force. The
mutation tests in test_oracle_mutations.py plant plausible mistakes in the oracle and
check that these pins catch each one.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import brute
from oracle import diffattn_f64 as ora
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_prefill(B=2, S=37, Hq=8, Hkv=2, D=16, seed=0, lam_range=(-0.5, 1.5)):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, S, Hq, D))
    k = rng.standard_normal((B, S, Hkv, D))
    v = rng.standard_normal((B, S, Hkv, D))
    lam = rng.uniform(*lam_range, size=(B, S, Hq // 2))
    return q, k, v, lam


def _sdpa_head(q, k, v, h, g, causal=True):
    """Ordinary softmax attention of query head h over KV head g (torch, float64, CPU)."""
    qt = torch.from_numpy(q[:, :, h, :]).permute(0, 1, 2)[:, None]  # [B,1,S,D]
    kt = torch.from_numpy(k[:, :, g, :])[:, None]
    vt = torch.from_numpy(v[:, :, g, :])[:, None]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=causal)
    return o[:, 0].numpy()


# ----------------------------------------------------------------------------- pins
# Each pin_* returns True when the oracle satisfies it; the tests assert them and the
# mutation tests check that a planted mistake makes at least one of them False.

def pin_softmax_library(seed=0):
    from scipy.special import softmax as sp_softmax

    rng = np.random.default_rng(seed)
    x = rng.standard_normal((7, 33)) * 30.0
    ok = np.allclose(ora.stable_softmax(x), sp_softmax(x, axis=-1), rtol=1e-13, atol=1e-300)
    xm = x.copy()
    xm[:, 5:] = -np.inf
    ok &= np.allclose(ora.stable_softmax(xm)[:, :5], sp_softmax(x[:, :5], axis=-1), rtol=1e-13)
    ok &= bool(np.all(ora.stable_softmax(xm)[:, 5:] == 0.0))
    # shift invariance holds for logits far outside exp's range too
    ok &= np.allclose(ora.stable_softmax(x + 900.0), sp_softmax(x, axis=-1), rtol=1e-12)
    return bool(ok)


def pin_lambda0_is_softmax_attention(causal=True):
    """lambda = 0 leaves the pure first softmax ("Differential Attention (V2)" lesson,
    Exercise 4): pair p must equal ordinary attention of head 2p over its GQA KV head."""
    q, k, v, lam = _rand_prefill(seed=1)
    lam[:] = 0.0
    out = ora.prefill(q, k, v, lam, causal=causal, row_block=16)
    Hq, Hkv = q.shape[2], k.shape[2]
    G = Hq // Hkv
    ok = True
    for p in range(Hq // 2):
        ref = _sdpa_head(q, k, v, 2 * p, (2 * p) // G, causal=causal)
        ok &= np.allclose(out[:, :, p], ref, rtol=1e-11, atol=1e-12)
    return bool(ok)


def pin_second_branch_is_odd_head(causal=True):
    """O(0) - O(1) = A2 V: the subtracted branch is head 2p+1 over the same KV head."""
    q, k, v, lam = _rand_prefill(seed=2)
    o0 = ora.prefill(q, k, v, np.zeros_like(lam), causal=causal)
    o1 = ora.prefill(q, k, v, np.ones_like(lam), causal=causal)
    Hq, Hkv = q.shape[2], k.shape[2]
    G = Hq // Hkv
    ok = True
    for p in range(Hq // 2):
        ref = _sdpa_head(q, k, v, 2 * p + 1, (2 * p + 1) // G, causal=causal)
        ok &= np.allclose(o0[:, :, p] - o1[:, :, p], ref, rtol=1e-10, atol=1e-11)
    return bool(ok)


def pin_equal_queries_lambda1_zero():
    """Q1 = Q2 with lambda = 1 gives exactly zero (both branches computed identically)."""
    q, k, v, lam = _rand_prefill(seed=3)
    q[:, :, 1::2] = q[:, :, 0::2]
    out = ora.prefill(q, k, v, np.ones_like(lam))
    return bool(np.all(out == 0.0))


def pin_rows_sum_to_one_minus_lambda():
    """With V == 1 every output element is the row sum of A1 - lam*A2, which is 1 - lam."""
    q, k, v, lam = _rand_prefill(seed=4)
    v[:] = 1.0
    out = ora.prefill(q, k, v, lam)
    return bool(np.allclose(out, (1.0 - lam)[..., None], rtol=0, atol=1e-12))


def pin_causal_row0():
    """Causal row 0 sees only key 0, so out[b,0,p] = (1 - lam) * v[b,0,g]."""
    q, k, v, lam = _rand_prefill(seed=5)
    out = ora.prefill(q, k, v, lam)
    Hq, Hkv = q.shape[2], k.shape[2]
    G = Hq // Hkv
    ok = True
    for p in range(Hq // 2):
        g = (2 * p) // G
        ok &= np.allclose(out[:, 0, p], (1.0 - lam[:, 0, p])[:, None] * v[:, 0, g], atol=1e-13)
    return bool(ok)


def pin_linear_in_lambda():
    """O(lam) = O(0) - lam * (O(0) - O(1)) for three lambda values."""
    q, k, v, lam = _rand_prefill(seed=6)
    o0 = ora.prefill(q, k, v, np.zeros_like(lam))
    o1 = ora.prefill(q, k, v, np.ones_like(lam))
    ok = True
    for c in (-0.7, 0.37, 2.5):
        oc = ora.prefill(q, k, v, np.full_like(lam, c))
        ok &= np.allclose(oc, o0 - c * (o0 - o1), atol=1e-11)
    return bool(ok)


def pin_brute_force_prefill(causal=True):
    q, k, v, lam = _rand_prefill(B=2, S=9, Hq=8, Hkv=2, D=5, seed=7)
    ref = np.array(brute.prefill(q.tolist(), k.tolist(), v.tolist(), lam.tolist(), causal=causal))
    out = ora.prefill(q, k, v, lam, causal=causal, row_block=4)
    return bool(np.allclose(out, ref, rtol=0, atol=1e-12))


def pin_brute_force_decode():
    rng = np.random.default_rng(8)
    B, Smax, Hq, Hkv, D = 3, 11, 8, 2, 6
    q = rng.standard_normal((B, Hq, D))
    kc = rng.standard_normal((B, Smax, Hkv, D))
    vc = rng.standard_normal((B, Smax, Hkv, D))
    seqlens = np.array([11, 1, 0])
    lam = rng.uniform(-1, 2, size=(B, Hq // 2))
    ref = np.array(brute.decode(q.tolist(), kc.tolist(), vc.tolist(), seqlens.tolist(), lam.tolist()))
    out = ora.decode(q, kc, vc, seqlens, lam)
    return bool(np.allclose(out, ref, rtol=0, atol=1e-12))


def pin_decode_is_last_prefill_row():
    """A decode step over n cached keys equals row n-1 of a causal prefill of length n."""
    rng = np.random.default_rng(9)
    B, S, Hq, Hkv, D = 2, 21, 8, 2, 8
    q, k, v, lam = _rand_prefill(B=B, S=S, Hq=Hq, Hkv=Hkv, D=D, seed=9)
    seqlens = np.array([S, 13])
    qd = np.stack([q[0, S - 1], q[1, 12]])
    lamd = np.stack([lam[0, S - 1], lam[1, 12]])
    dec = ora.decode(qd, k, v, seqlens, lamd)
    full = ora.prefill(q, k, v, lam)
    ok = np.allclose(dec[0], full[0, S - 1], atol=1e-13)
    ok &= np.allclose(dec[1], ora.prefill(q[1:, :13], k[1:, :13], v[1:, :13], lam[1:, :13])[0, 12],
                      atol=1e-13)
    del rng
    return bool(ok)


def pin_decode_window_is_last_window_prefill_row():
    """A windowed decode step over n cached keys equals row n-1 of a windowed prefill of length
    n (windows 1, 5 and one longer than the sequence), and brute-force decode over the last
    `window` keys alone."""
    B, S, Hq, Hkv, D = 2, 21, 8, 2, 8
    q, k, v, lam = _rand_prefill(B=B, S=S, Hq=Hq, Hkv=Hkv, D=D, seed=31)
    seqlens = np.array([S, 13])
    qd = np.stack([q[0, S - 1], q[1, 12]])
    lamd = np.stack([lam[0, S - 1], lam[1, 12]])
    ok = True
    for w in (1, 5, 40):
        dec = ora.decode(qd, k, v, seqlens, lamd, window=w)
        ok &= np.allclose(dec[0], ora.prefill(q, k, v, lam, window=w)[0, S - 1], atol=1e-13)
        ok &= np.allclose(dec[1], ora.prefill(q[1:, :13], k[1:, :13], v[1:, :13], lam[1:, :13], window=w)[0, 12],
                          atol=1e-13)
    n0 = 13 - 5
    ref = np.array(brute.decode(qd[1:].tolist(), k[1:, n0:13].tolist(), v[1:, n0:13].tolist(), [5], lamd[1:].tolist()))
    ok &= np.allclose(ora.decode(qd, k, v, seqlens, lamd, window=5)[1], ref[0], atol=1e-12)
    return bool(ok)


def pin_prefill_rows_match_full():
    q, k, v, lam = _rand_prefill(seed=10)
    full = ora.prefill(q, k, v, lam)
    rows = [(0, 0, 0), (1, 36, 3), (0, 17, 2), (1, 5, 1)]
    sel = ora.prefill_rows(q, k, v, lam, rows)
    return bool(all(np.allclose(sel[n], full[b, i, p], atol=1e-13) for n, (b, i, p) in enumerate(rows)))


def pin_lambda_v1_closed_form():
    """lambda = exp(lq1.lk1) - exp(lq2.lk2) + lambda_init with dot products ln2 and 0 -> 1.8,
    and 0 and ln3 -> -1.2 (lambda may be negative)."""
    d = 4
    a = np.zeros((2, d)); b = np.zeros((2, d)); c = np.zeros((2, d)); e = np.zeros((2, d))
    a[0, 0], b[0, 0] = math.log(2.0), 1.0          # pair 0: a.b = ln 2, c.e = 0
    c[1, 1], e[1, 1] = math.log(3.0) / 2.0, 2.0    # pair 1: a.b = 0,    c.e = ln 3
    lam = ora.lambda_v1(a, b, c, e, 0.8)
    ok = abs(lam[0] - 1.8) < 1e-14 and abs(lam[1] - (-1.2)) < 1e-14
    rng = np.random.default_rng(11)
    vec = [rng.standard_normal((5, 7)) * 0.3 for _ in range(4)]
    ok &= np.allclose(ora.lambda_v1(*vec, 0.8), brute.lambda_v1(*(x.tolist() for x in vec), 0.8),
                      atol=1e-14)
    return bool(ok)


def pin_noise_mass_golden():
    """The 128k worked example of the lesson's "The problem" section (golden fixture)."""
    with open(os.path.join(GOLDEN, "noise_mass_128k.json")) as f:
        gold = json.load(f)
    n = gold["context_tokens"]
    w = gold["per_token_weight"]
    # one matching token with logit x and n-1 unrelated tokens with logit 0 such that each
    # unrelated token gets weight w: 1/(e^x + n - 1) = w
    x = math.log(1.0 / w - (n - 1))
    row = np.zeros(n)
    row[0] = x
    a = ora.stable_softmax(row)
    mass = float(np.sum(a[1:]))
    ok = abs(a[1] - w) < 1e-18 and abs(mass - gold["noise_mass"]) < 1e-12
    ok &= round(100 * mass) == gold["noise_mass_rounded_percent"]
    return bool(ok)


def pin_uniform_logits():
    """N equal logits give every token weight exactly-ish 1/N (the O(1/N) noise floor)."""
    ok = True
    for n in (1, 7, 4096):
        a = ora.stable_softmax(np.full(n, 3.25))
        ok &= np.allclose(a, 1.0 / n, rtol=1e-14)
    return bool(ok)


def pin_weights_rows_sum():
    rng = np.random.default_rng(12)
    k = rng.standard_normal((50, 16))
    ok = True
    for lam in (-0.3, 0.0, 0.8, 1.0):
        a1, a2, w = ora.branch_weights(rng.standard_normal(16), rng.standard_normal(16), k, lam, 31)
        ok &= abs(a1.sum() - 1) < 1e-14 and abs(a2.sum() - 1) < 1e-14
        ok &= abs(w.sum() - (1 - lam)) < 1e-13 and len(w) == 31
    return bool(ok)


def pin_branch_weights_library():
    """One query row's weights against the library: torch SDPA with V = I returns the row of
    softmax(q k^T / sqrt(D)) itself (D = 16, so a dropped or wrong 1/sqrt(D) changes it);
    keys past n_visible take no weight, which equals SDPA over the visible prefix."""
    rng = np.random.default_rng(24)
    D, m, n_vis = 16, 40, 29
    k = rng.standard_normal((m, D)) * 1.5
    q1, q2 = rng.standard_normal(D) * 1.5, rng.standard_normal(D) * 1.5

    def sdpa_row(q, n):
        eye = torch.eye(n, dtype=torch.float64)[None, None]
        kt = torch.from_numpy(k[:n])[None, None]
        qt = torch.from_numpy(q)[None, None, None]
        return torch.nn.functional.scaled_dot_product_attention(qt, kt, eye)[0, 0, 0].numpy()

    ok = True
    for lam, n in ((0.8, None), (-0.4, n_vis)):
        a1, a2, w = ora.branch_weights(q1, q2, k, lam, n)
        nn_ = m if n is None else n
        r1, r2 = sdpa_row(q1, nn_), sdpa_row(q2, nn_)
        ok &= len(a1) == nn_ and np.allclose(a1, r1, rtol=1e-12, atol=1e-15)
        ok &= np.allclose(a2, r2, rtol=1e-12, atol=1e-15)
        ok &= np.allclose(w, r1 - lam * r2, rtol=1e-12, atol=1e-15)
    return bool(ok)


def pin_snr_hand_values():
    """Signal-to-noise ratio (lesson key-terms table) on hand-computed rows with negative
    entries, where the mean of absolute weights differs from the signed mean:
    [0.5, -0.1, 0.1, -0.2] with the signal at 0 gives 0.5 / (0.4 / 3) = 3.75;
    [0.1, 0.6, -0.3] with the signal at 1 gives 0.6 / 0.2 = 3.0."""
    ok = math.isclose(ora.snr([0.5, -0.1, 0.1, -0.2], 0), 3.75, rel_tol=1e-14)
    ok &= math.isclose(ora.snr(np.array([0.1, 0.6, -0.3]), 1), 3.0, rel_tol=1e-14)
    return bool(ok)


def pin_window_reduces_to_causal_and_self():
    """A window at least S long is the causal mask; window 1 leaves each query only its own
    key, so out[b,i,p] = (1 - lam) v[b,i,g]."""
    q, k, v, lam = _rand_prefill(seed=13)
    S = q.shape[1]
    ok = np.allclose(ora.prefill(q, k, v, lam, window=S), ora.prefill(q, k, v, lam), atol=1e-13)
    ok &= np.allclose(ora.prefill(q, k, v, lam, window=10 * S), ora.prefill(q, k, v, lam), atol=1e-13)
    one = ora.prefill(q, k, v, lam, window=1)
    G = q.shape[2] // k.shape[2]
    for p in range(q.shape[2] // 2):
        ok &= np.allclose(one[:, :, p], (1.0 - lam[:, :, p])[..., None] * v[:, :, (2 * p) // G], atol=1e-13)
    return bool(ok)


def pin_window_brute_force():
    q, k, v, lam = _rand_prefill(B=1, S=11, Hq=4, Hkv=1, D=4, seed=14)
    ok = True
    for w in (2, 3, 7):
        ref = np.array(brute.prefill(q.tolist(), k.tolist(), v.tolist(), lam.tolist(), window=w))
        ok &= np.allclose(ora.prefill(q, k, v, lam, window=w, row_block=4), ref, atol=1e-12)
    return bool(ok)


def pin_window_mask_definition():
    """The lesson's worked picture: n = 8, window 4 keeps the last 4 keys of each row."""
    m = ora.window_mask(8, 8, 4)
    vis = (m == 0.0)
    ok = all(vis[i].sum() == min(i + 1, 4) for i in range(8))
    ok &= bool(vis[7, 4:].all() and not vis[7, :4].any() and vis[2, :3].all())
    return bool(ok)


def pin_varlen_is_per_sequence_prefill():
    """Packed sequences: each equals its own prefill, and a packing of equal lengths equals
    the batched prefill (the brute force checks the batched one)."""
    q, k, v, lam = _rand_prefill(B=3, S=13, Hq=8, Hkv=2, D=6, seed=15)
    flat = lambda t: t.reshape(-1, *t.shape[2:])
    cu = [0, 13, 26, 39]
    ok = np.allclose(ora.prefill_varlen(flat(q), flat(k), flat(v), flat(lam), cu).reshape(3, 13, 4, 6),
                     ora.prefill(q, k, v, lam), atol=1e-13)
    cu2 = [0, 5, 5, 20, 39]  # lengths 5, 0, 15, 19
    out = ora.prefill_varlen(flat(q), flat(k), flat(v), flat(lam), cu2)
    for a, b_ in zip(cu2[:-1], cu2[1:]):
        if b_ > a:
            ref = np.array(brute.prefill(*(flat(t)[None, a:b_].tolist() for t in (q, k, v, lam))))[0]
            ok &= np.allclose(out[a:b_], ref, atol=1e-12)
    return bool(ok)


def pin_varlen_window_is_per_sequence_window():
    """A sliding window over packed sequences: each sequence equals the brute force's windowed
    prefill of that sequence alone, and a window longer than every sequence is the causal
    packed prefill."""
    q, k, v, lam = _rand_prefill(B=1, S=39, Hq=4, Hkv=1, D=5, seed=17)
    flat = lambda t: t.reshape(-1, *t.shape[2:])
    cu = [0, 5, 5, 20, 39]  # lengths 5, 0, 15, 19
    ok = True
    for w in (1, 3, 7):
        out = ora.prefill_varlen(flat(q), flat(k), flat(v), flat(lam), cu, window=w)
        for a, b_ in zip(cu[:-1], cu[1:]):
            if b_ > a:
                ref = np.array(brute.prefill(*(flat(t)[None, a:b_].tolist() for t in (q, k, v, lam)), window=w))[0]
                ok &= np.allclose(out[a:b_], ref, atol=1e-12)
    ok &= np.allclose(ora.prefill_varlen(flat(q), flat(k), flat(v), flat(lam), cu, window=19),
                      ora.prefill_varlen(flat(q), flat(k), flat(v), flat(lam), cu), atol=1e-13)
    return bool(ok)


def pin_paged_decode_gathers_pages():
    """A paged cache with a shuffled block table decodes like the contiguous cache it holds
    (and, through `decode`, like the brute force)."""
    rng = np.random.default_rng(16)
    B, Hq, Hkv, D, ps = 3, 8, 2, 6, 4
    lens = [9, 1, 0]
    n_pages = 12
    kp = rng.standard_normal((n_pages, ps, Hkv, D))
    vp = rng.standard_normal((n_pages, ps, Hkv, D))
    perm = rng.permutation(n_pages)
    table = [perm[0:3].tolist(), perm[3:4].tolist() + [0, 0], [0, 0, 0]]
    q = rng.standard_normal((B, Hq, D))
    lam = rng.uniform(-1, 2, size=(B, Hq // 2))
    out = ora.decode_paged(q, kp, vp, table, lens, lam)
    ok = True
    for b in range(B):
        n = lens[b]
        kc = np.concatenate([kp[pg] for pg in table[b]], axis=0)[None, :max(n, 1)]
        vc = np.concatenate([vp[pg] for pg in table[b]], axis=0)[None, :max(n, 1)]
        ref = np.array(brute.decode(q[b:b + 1].tolist(), kc.tolist(), vc.tolist(), [n], lam[b:b + 1].tolist()))
        ok &= np.allclose(out[b], ref[0], atol=1e-12)
    return bool(ok)


def pin_paged_window_decode_gathers_pages():
    """The windowed decode over a paged cache equals the brute force over the last `window`
    keys of the gathered cache."""
    rng = np.random.default_rng(32)
    B, Hq, Hkv, D, ps = 2, 8, 2, 6, 4
    lens = [11, 3]
    n_pages = 8
    kp = rng.standard_normal((n_pages, ps, Hkv, D))
    vp = rng.standard_normal((n_pages, ps, Hkv, D))
    perm = rng.permutation(n_pages)
    table = [perm[0:3].tolist(), perm[3:4].tolist() + [0, 0]]
    q = rng.standard_normal((B, Hq, D))
    lam = rng.uniform(-1, 2, size=(B, Hq // 2))
    ok = True
    for w in (1, 5):
        out = ora.decode_paged(q, kp, vp, table, lens, lam, window=w)
        for b in range(B):
            n = lens[b]
            n0 = max(0, n - w)
            kc = np.concatenate([kp[pg] for pg in table[b]], axis=0)[None, n0:n]
            vc = np.concatenate([vp[pg] for pg in table[b]], axis=0)[None, n0:n]
            ref = np.array(brute.decode(q[b:b + 1].tolist(), kc.tolist(), vc.tolist(), [n - n0], lam[b:b + 1].tolist()))
            ok &= np.allclose(out[b], ref[0], atol=1e-12)
    return bool(ok)


def pin_lambda_v2_projection():
    """sigmoid(x W + b): W = 0 gives sigmoid(b) (0.5 without bias, 0.75 for b = ln 3); one
    nonzero weight gives sigmoid(x_k w_k); random inputs match torch.sigmoid(x @ W + b)."""
    rng = np.random.default_rng(17)
    x = rng.standard_normal((5, 12))
    w0 = np.zeros((12, 4))
    ok = np.allclose(ora.lambda_v2_projection(x, w0), 0.5, rtol=0, atol=0)
    ok &= np.allclose(ora.lambda_v2_projection(x, w0, np.full(4, math.log(3.0))), 0.75, atol=1e-15)
    w1 = w0.copy()
    w1[3, 2] = 0.7
    ok &= np.allclose(ora.lambda_v2_projection(x, w1)[:, 2], 1.0 / (1.0 + np.exp(-0.7 * x[:, 3])), atol=1e-15)
    w = rng.standard_normal((12, 4))
    b = rng.standard_normal(4)
    ref = torch.sigmoid(torch.from_numpy(x) @ torch.from_numpy(w) + torch.from_numpy(b)).numpy()
    lam = ora.lambda_v2_projection(x, w, b)
    ok &= np.allclose(lam, ref, atol=1e-14) and bool(np.all((lam > 0) & (lam < 1)))
    return bool(ok)


def pin_multi_token_decode_is_prefill_tail():
    """T new tokens decoded together equal the last T rows of a causal prefill."""
    q, k, v, lam = _rand_prefill(B=2, S=15, Hq=8, Hkv=2, D=6, seed=18)
    T = 3
    full = ora.prefill(q, k, v, lam)
    dec = ora.decode_multi(q[:, -T:], k, v, [15, 15], lam[:, -T:])
    return bool(np.allclose(dec, full[:, -T:], atol=1e-13))


def _torch_forward(q, k, v, lam, causal=True):
    """An independent float64 torch forward (for autograd): heads 2p and 2p+1 over KV head
    2p // G, scores / sqrt(D), causal mask, torch.softmax, out = A1 V - lam A2 V."""
    B, S, Hq, D = q.shape
    G = Hq // k.shape[2]
    kv = torch.arange(Hq) // G
    kk = k[:, :, kv].permute(0, 2, 1, 3)
    vv = v[:, :, kv].permute(0, 2, 1, 3)
    s_ = q.permute(0, 2, 1, 3) @ kk.transpose(-1, -2) / math.sqrt(D)
    if causal:
        s_ = s_.masked_fill(torch.triu(torch.ones(S, S, dtype=torch.bool), 1), float("-inf"))
    o = torch.softmax(s_, dim=-1) @ vv  # [B, Hq, S, D]
    return (o[:, 0::2] - lam.permute(0, 2, 1)[..., None] * o[:, 1::2]).permute(0, 2, 1, 3)


def pin_backward_matches_autograd(causal=True):
    q, k, v, lam = _rand_prefill(B=2, S=11, Hq=8, Hkv=2, D=6, seed=19)
    dout = np.random.default_rng(20).standard_normal((2, 11, 4, 6))
    ts = [torch.tensor(x, requires_grad=True) for x in (q, k, v, lam)]
    _torch_forward(*ts, causal=causal).backward(torch.tensor(dout))
    got = ora.prefill_backward(q, k, v, lam, dout, causal=causal)
    return bool(all(np.allclose(g, t.grad.numpy(), atol=1e-11) for g, t in zip(got, ts)))


def pin_backward_finite_differences():
    """Central differences of <dout, prefill(.)> on a few entries of every input."""
    q, k, v, lam = _rand_prefill(B=1, S=6, Hq=4, Hkv=1, D=3, seed=21)
    dout = np.random.default_rng(22).standard_normal((1, 6, 2, 3))
    grads = ora.prefill_backward(q, k, v, lam, dout)
    f = lambda q_, k_, v_, l_: float(np.sum(ora.prefill(q_, k_, v_, l_) * dout))
    eps = 1e-6
    ok = True
    for which, idx in ((0, (0, 4, 1, 2)), (1, (0, 3, 0, 1)), (2, (0, 5, 0, 0)), (3, (0, 2, 1))):
        args = [q.copy(), k.copy(), v.copy(), lam.copy()]
        args[which][idx] += eps
        up = f(*args)
        args[which][idx] -= 2 * eps
        dn = f(*args)
        ok &= abs((up - dn) / (2 * eps) - grads[which][idx]) < 1e-6
    return bool(ok)


def pin_branches_recombine_and_normalise():
    """O_{2p} - lam * O_{2p+1} is the prefill; 2^(s log2(e) - lse2) rows sum to one and
    equal the library softmax (scipy) of the scaled scores."""
    from scipy.special import softmax as sp_softmax
    q, k, v, lam = _rand_prefill(B=2, S=9, Hq=8, Hkv=2, D=5, seed=23)
    ok = True
    for causal in (True, False):
        o, lse2 = ora.prefill_branches(q, k, v, causal=causal)
        full = ora.prefill(q, k, v, lam, causal=causal)
        ok &= np.allclose(o[:, :, 0::2] - lam[..., None] * o[:, :, 1::2], full, atol=1e-13)
        # head 5 reads KV head 1 (group 4)
        s_ = q[1, :, 5] @ k[1, :, 1].T / math.sqrt(5)
        if causal:
            s_ = np.where(np.tril(np.ones((9, 9))) > 0, s_, -np.inf)
        a = np.exp2(s_ * math.log2(math.e) - lse2[1, :, 5][:, None])
        ok &= np.allclose(a.sum(axis=1), 1.0, atol=1e-13)
        ok &= np.allclose(a, sp_softmax(s_, axis=1), atol=1e-13)
    # the first causal row sees one key: its lse is that key's scaled score in base 2
    o, lse2 = ora.prefill_branches(q, k, v)
    ok &= math.isclose(lse2[0, 0, 3], float(q[0, 0, 3] @ k[0, 0, 0]) / math.sqrt(5) * math.log2(math.e),
                       rel_tol=1e-12, abs_tol=1e-12)
    return bool(ok)


def pin_backward_varlen_finite_differences():
    """Central differences of <dout, prefill_varlen(.)> for packed sequences of lengths
    3, 0, 5: entries inside a sequence match, and a key of the first sequence has exactly
    zero gradient through the second."""
    rng = np.random.default_rng(24)
    T, Hq, Hkv, D = 8, 4, 2, 3
    q, k, v = (rng.standard_normal((T, h, D)) for h in (Hq, Hkv, Hkv))
    lam = rng.uniform(0.2, 0.9, (T, Hq // 2))
    dout = rng.standard_normal((T, Hq // 2, D))
    cu = [0, 3, 3, 8]
    grads = ora.prefill_backward_varlen(q, k, v, lam, dout, cu)
    f = lambda q_, k_, v_, l_: float(np.sum(ora.prefill_varlen(q_, k_, v_, l_, cu) * dout))
    eps = 1e-6
    ok = True
    for which, idx in ((0, (6, 3, 1)), (1, (4, 1, 2)), (2, (2, 0, 0)), (3, (7, 1)), (1, (1, 0, 1))):
        args = [q.copy(), k.copy(), v.copy(), lam.copy()]
        args[which][idx] += eps
        up = f(*args)
        args[which][idx] -= 2 * eps
        dn = f(*args)
        ok &= abs((up - dn) / (2 * eps) - grads[which][idx]) < 1e-6
    # perturbing key 1 (first sequence) leaves the second sequence's outputs unchanged
    k2 = k.copy()
    k2[1] += 1.0
    ok &= np.array_equal(ora.prefill_varlen(q, k2, v, lam, cu)[3:], ora.prefill_varlen(q, k, v, lam, cu)[3:])
    return bool(ok)


def pin_backward_varlen_equal_lengths_is_batched():
    """Two packed sequences of equal length give the batched backward of the same data."""
    q, k, v, lam = _rand_prefill(B=2, S=6, Hq=8, Hkv=2, D=4, seed=25)
    dout = np.random.default_rng(26).standard_normal((2, 6, 4, 4))
    batched = ora.prefill_backward(q, k, v, lam, dout)
    packed = ora.prefill_backward_varlen(*(x.reshape((12,) + x.shape[2:]) for x in (q, k, v, lam, dout)), [0, 6, 12])
    return bool(all(np.allclose(a.reshape(p_.shape), p_, atol=1e-13) for a, p_ in zip(batched, packed)))


def pin_backward_window():
    """Sliding-window gradients: central differences of <dout, prefill(., window=3)>, and a
    window covering the whole sequence reduces to the causal backward."""
    q, k, v, lam = _rand_prefill(B=1, S=7, Hq=4, Hkv=2, D=3, seed=27)
    dout = np.random.default_rng(28).standard_normal((1, 7, 2, 3))
    grads = ora.prefill_backward(q, k, v, lam, dout, window=3)
    f = lambda q_, k_, v_, l_: float(np.sum(ora.prefill(q_, k_, v_, l_, window=3) * dout))
    eps = 1e-6
    ok = True
    for which, idx in ((0, (0, 6, 1, 2)), (1, (0, 4, 1, 0)), (1, (0, 1, 0, 1)), (2, (0, 3, 0, 2)), (3, (0, 5, 1))):
        args = [q.copy(), k.copy(), v.copy(), lam.copy()]
        args[which][idx] += eps
        up = f(*args)
        args[which][idx] -= 2 * eps
        dn = f(*args)
        ok &= abs((up - dn) / (2 * eps) - grads[which][idx]) < 1e-6
    full = ora.prefill_backward(q, k, v, lam, dout, window=7)
    causal = ora.prefill_backward(q, k, v, lam, dout)
    ok &= all(np.allclose(a, b, atol=1e-13) for a, b in zip(full, causal))
    return bool(ok)


def pin_backward_varlen_window():
    """Sliding-window gradients of packed sequences: central differences of
    <dout, prefill_varlen(., window=2)> (including a key of the first sequence, which the second
    never sees), and a window longer than every sequence reduces to the causal packed backward."""
    q, k, v, lam = _rand_prefill(B=1, S=9, Hq=4, Hkv=2, D=3, seed=29)
    q, k, v, lam = q[0], k[0], v[0], lam[0]
    dout = np.random.default_rng(30).standard_normal((9, 2, 3))
    cu = [0, 4, 9]
    grads = ora.prefill_backward_varlen(q, k, v, lam, dout, cu, window=2)
    f = lambda q_, k_, v_, l_: float(np.sum(ora.prefill_varlen(q_, k_, v_, l_, cu, window=2) * dout))
    eps = 1e-6
    ok = True
    for which, idx in ((0, (8, 1, 2)), (1, (2, 1, 0)), (1, (7, 0, 1)), (2, (5, 0, 2)), (3, (3, 1))):
        args = [q.copy(), k.copy(), v.copy(), lam.copy()]
        args[which][idx] += eps
        up = f(*args)
        args[which][idx] -= 2 * eps
        dn = f(*args)
        ok &= abs((up - dn) / (2 * eps) - grads[which][idx]) < 1e-6
    full = ora.prefill_backward_varlen(q, k, v, lam, dout, cu, window=5)
    causal = ora.prefill_backward_varlen(q, k, v, lam, dout, cu)
    ok &= all(np.allclose(a, b, atol=1e-13) for a, b in zip(full, causal))
    return bool(ok)


ALL_PINS = {
    "paged_window_decode_gathers_pages": pin_paged_window_decode_gathers_pages,
    "decode_window_is_last_window_prefill_row": pin_decode_window_is_last_window_prefill_row,
    "varlen_window_is_per_sequence_window": pin_varlen_window_is_per_sequence_window,
    "backward_varlen_window": pin_backward_varlen_window,
    "softmax_library": pin_softmax_library,
    "lambda0_is_softmax_attention": pin_lambda0_is_softmax_attention,
    "lambda0_noncausal": lambda: pin_lambda0_is_softmax_attention(causal=False),
    "second_branch_is_odd_head": pin_second_branch_is_odd_head,
    "equal_queries_lambda1_zero": pin_equal_queries_lambda1_zero,
    "rows_sum_to_one_minus_lambda": pin_rows_sum_to_one_minus_lambda,
    "causal_row0": pin_causal_row0,
    "linear_in_lambda": pin_linear_in_lambda,
    "brute_force_prefill": pin_brute_force_prefill,
    "brute_force_prefill_noncausal": lambda: pin_brute_force_prefill(causal=False),
    "brute_force_decode": pin_brute_force_decode,
    "decode_is_last_prefill_row": pin_decode_is_last_prefill_row,
    "prefill_rows_match_full": pin_prefill_rows_match_full,
    "lambda_v1_closed_form": pin_lambda_v1_closed_form,
    "noise_mass_golden": pin_noise_mass_golden,
    "uniform_logits": pin_uniform_logits,
    "weights_rows_sum": pin_weights_rows_sum,
    "branch_weights_library": pin_branch_weights_library,
    "snr_hand_values": pin_snr_hand_values,
    "window_reduces_to_causal_and_self": pin_window_reduces_to_causal_and_self,
    "window_brute_force": pin_window_brute_force,
    "window_mask_definition": pin_window_mask_definition,
    "varlen_is_per_sequence_prefill": pin_varlen_is_per_sequence_prefill,
    "paged_decode_gathers_pages": pin_paged_decode_gathers_pages,
    "lambda_v2_projection": pin_lambda_v2_projection,
    "multi_token_decode_is_prefill_tail": pin_multi_token_decode_is_prefill_tail,
    "backward_matches_autograd": pin_backward_matches_autograd,
    "backward_matches_autograd_noncausal": lambda: pin_backward_matches_autograd(causal=False),
    "backward_finite_differences": pin_backward_finite_differences,
    "branches_recombine_and_normalise": pin_branches_recombine_and_normalise,
    "backward_varlen_finite_differences": pin_backward_varlen_finite_differences,
    "backward_varlen_equal_lengths_is_batched": pin_backward_varlen_equal_lengths_is_batched,
    "backward_window": pin_backward_window,
}


@pytest.mark.parametrize("name", sorted(ALL_PINS))
def test_pin(name):
    assert ALL_PINS[name]()


# ------------------------------------------------------------ the noise-cancellation toy

def _planted_c1():
    case = workloads.CONFIGS["tiny_fp32_prefill_b1_s128"]
    inp = workloads.make_prefill(case)
    row, sig = workloads.plant_signal_row(inp)
    return inp, row, sig


def test_planted_row_noise_cancels():
    """"Differential Attention (V2)" lesson, Step 4: with a shared noise floor the difference
    map has a higher signal-to-noise ratio than the first softmax alone, for lambda in
    [0.5, 1]."""
    inp, row, sig = _planted_c1()
    q, k = inp["q"], inp["k"]
    for lam in (0.5, 0.75, 0.9, 1.0):
        a1, _, w = ora.branch_weights(q[0, row, 0], q[0, row, 1], k[0, :, 0], lam, row + 1)
        assert ora.snr(w, sig) > ora.snr(a1, sig)
    # lambda = 0 leaves the first softmax unchanged
    a1, _, w = ora.branch_weights(q[0, row, 0], q[0, row, 1], k[0, :, 0], 0.0, row + 1)
    assert np.array_equal(a1, w)


def test_planted_toy_length_1024_reports_ratio(capsys):
    """The lesson's length-1024 toy: report the SNR ratio diff/standard (the pages claim
    3x-10x qualitatively; this is reported, and only a ratio > 1 is asserted)."""
    case = workloads.PrefillCase(B=1, S=1024, Hq=2, Hkv=1, D=64, dtype="f32", seed=2024)
    inp = workloads.make_prefill(case)
    row, sig = workloads.plant_signal_row(inp, signal_key=300)
    q, k = inp["q"], inp["k"]
    a1, _, w = ora.branch_weights(q[0, row, 0], q[0, row, 1], k[0, :, 0], 0.9, row + 1)
    ratio = ora.snr(w, sig) / ora.snr(a1, sig)
    with capsys.disabled():
        print(f"\n[toy] length-1024 SNR diff/standard at lambda=0.9: {ratio:.2f}x")
    assert ratio > 1.0


def test_v2_kv_cache_matches_gqa_baseline():
    """Exercise 5 of the lesson: with 8 KV heads and 32 query heads the V2 cache is the
    same size as a baseline GQA cache -- it depends on Hkv, never on Hq."""
    a = workloads.make_decode(workloads.DecodeCase(B=2, Smax=16, Hq=32, Hkv=8, D=8,
                                                   len_lo=16, len_hi=16, seed=1))
    b = workloads.make_decode(workloads.DecodeCase(B=2, Smax=16, Hq=16, Hkv=8, D=8,
                                                   len_lo=16, len_hi=16, seed=1))
    nbytes = lambda t: t.numel() * t.element_size()
    assert nbytes(a["kcache"]) + nbytes(a["vcache"]) == 2 * 16 * 8 * 8 * 2 * 2
    assert nbytes(a["kcache"]) == nbytes(b["kcache"])


def test_pair_layout_rejects_straddling_pairs():
    with pytest.raises(ValueError):
        ora.pair_layout(6, 2)  # G = 3: pair (2,3) would straddle KV heads 0 and 1
    with pytest.raises(ValueError):
        ora.pair_layout(5, 1)
    assert ora.pair_layout(64, 8)[5] == (5, 10, 11, 1)
