"""Planted mistakes in the oracle (on the CPU) must each fail at least one pin.

Each mutant replaces one oracle function with a plausibly wrong version -- a dropped
term, a wrong sign, a swapped head, a wrong GQA index, an off-by-one mask -- and the test
checks that the pin suite of test_oracle.py notices. This shows the pins constrain every
part of the definition rather than only re-reading it.
"""
import math

import numpy as np
import pytest

from oracle import diffattn_f64 as ora
from tests.test_oracle import ALL_PINS


def _block_plus_sign(q1, q2, k, v, lam, mask):
    D = q1.shape[-1]
    a1 = ora.stable_softmax(q1 @ k.T / math.sqrt(D) + mask)
    a2 = ora.stable_softmax(q2 @ k.T / math.sqrt(D) + mask)
    return (a1 + lam[:, None] * a2) @ v


def _block_no_scale(q1, q2, k, v, lam, mask):
    a1 = ora.stable_softmax(q1 @ k.T + mask)
    a2 = ora.stable_softmax(q2 @ k.T + mask)
    return (a1 - lam[:, None] * a2) @ v


def _block_scale_d(q1, q2, k, v, lam, mask):
    D = q1.shape[-1]
    a1 = ora.stable_softmax(q1 @ k.T / D + mask)
    a2 = ora.stable_softmax(q2 @ k.T / D + mask)
    return (a1 - lam[:, None] * a2) @ v


def _block_lambda_on_first(q1, q2, k, v, lam, mask):
    D = q1.shape[-1]
    a1 = ora.stable_softmax(q1 @ k.T / math.sqrt(D) + mask)
    a2 = ora.stable_softmax(q2 @ k.T / math.sqrt(D) + mask)
    return (lam[:, None] * a1 - a2) @ v


def _block_shared_query(q1, q2, k, v, lam, mask):
    D = q1.shape[-1]
    a1 = ora.stable_softmax(q1 @ k.T / math.sqrt(D) + mask)
    return ((1.0 - lam[:, None]) * a1) @ v


def _block_softmax_wrong_axis(q1, q2, k, v, lam, mask):
    D = q1.shape[-1]
    s1 = q1 @ k.T / math.sqrt(D) + mask
    s2 = q2 @ k.T / math.sqrt(D) + mask
    a1 = np.nan_to_num(np.exp(s1) / np.sum(np.exp(s1), axis=0, keepdims=True))
    a2 = np.nan_to_num(np.exp(s2) / np.sum(np.exp(s2), axis=0, keepdims=True))
    return (a1 - lam[:, None] * a2) @ v


def _layout_swapped(Hq, Hkv):
    G = Hq // Hkv
    return [(p, 2 * p + 1, 2 * p, (2 * p) // G) for p in range(Hq // 2)]


def _layout_wrong_group(Hq, Hkv):
    return [(p, 2 * p, 2 * p + 1, p % Hkv) for p in range(Hq // 2)]


def _layout_split_heads(Hq, Hkv):
    # pairs (p, p + Hq/2) instead of adjacent heads
    G = Hq // Hkv
    return [(p, p, p + Hq // 2, p // G) for p in range(Hq // 2)]


def _mask_off_by_one(n_q, n_k, q_offset=0):
    # lets each query see one future key
    i = np.arange(q_offset, q_offset + n_q)[:, None]
    j = np.arange(n_k)[None, :]
    return np.where(j <= i + 1, 0.0, -np.inf)


def _mask_transposed(n_q, n_k, q_offset=0):
    i = np.arange(q_offset, q_offset + n_q)[:, None]
    j = np.arange(n_k)[None, :]
    return np.where(j >= i, 0.0, -np.inf)


def _window_off_by_one(n_q, n_k, window, q_offset=0):
    i = np.arange(q_offset, q_offset + n_q)[:, None]
    j = np.arange(n_k)[None, :]
    return np.where((j <= i) & (j >= i - window), 0.0, -np.inf)


def _softmax_no_max(x):
    x = np.asarray(x, dtype=np.float64)
    e = np.exp(x)
    return e / np.sum(e, axis=-1, keepdims=True)


def _softmax_off(x):
    x = np.asarray(x, dtype=np.float64)
    m = np.max(x, axis=-1, keepdims=True)
    e = np.exp(x - m)
    return e / (np.sum(e, axis=-1, keepdims=True) + 1e-6)


def _lambda_v1_plus(lq1, lk1, lq2, lk2, lambda_init=0.8):
    a, b, c, e = (np.asarray(x, dtype=np.float64) for x in (lq1, lk1, lq2, lk2))
    return np.exp(np.sum(a * b, -1)) + np.exp(np.sum(c * e, -1)) + lambda_init


def _lambda_v2_no_sigmoid(x, w, bias=None):
    z = np.asarray(x, dtype=np.float64) @ np.asarray(w, dtype=np.float64)
    return z if bias is None else z + np.asarray(bias)[None, :]


def _backward_variant(drop_rowsum=False, dlam_sign=-1.0, dk_first_only=False, dv_no_lambda=False,
                      dq_unscaled=False):
    """The chain rule of the prefill with one planted mistake (a flag set)."""
    def fn(q, k, v, lam, dout, causal=True, window=None):
        q, k, v, lam, dout = (np.asarray(x, dtype=np.float64) for x in (q, k, v, lam, dout))
        B, S, Hq, D = q.shape
        inv = 1.0 / math.sqrt(D)
        dq, dk, dv, dlam = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v), np.zeros_like(lam)
        if window is not None:
            mask = ora.window_mask(S, S, int(window))
        else:
            mask = ora.causal_mask(S, S) if causal else np.zeros((S, S))
        for b in range(B):
            for p, h1, h2, g in ora.pair_layout(Hq, k.shape[2]):
                kk, vv = k[b, :, g], v[b, :, g]
                a1 = ora.stable_softmax(q[b, :, h1] @ kk.T * inv + mask)
                a2 = ora.stable_softmax(q[b, :, h2] @ kk.T * inv + mask)
                lm = lam[b, :, p][:, None]
                do = dout[b, :, p]
                dlam[b, :, p] = dlam_sign * np.sum(do * (a2 @ vv), axis=1)
                dv[b, :, g] += a1.T @ do - a2.T @ ((1.0 if dv_no_lambda else lm) * do)
                dpv = do @ vv.T
                for a, da, h in ((a1, dpv, h1), (a2, -lm * dpv, h2)):
                    rs = 0.0 if drop_rowsum else np.sum(a * da, axis=1, keepdims=True)
                    ds = a * (da - rs)
                    dq[b, :, h] = ds @ kk * (1.0 if dq_unscaled else inv)
                    if not (dk_first_only and h == h2):
                        dk[b, :, g] += ds.T @ q[b, :, h] * inv
        return dq, dk, dv, dlam
    return fn


def _branches_natural_log(q, k, v, causal=True):
    o, lse2 = _ORIG_BRANCHES(q, k, v, causal)
    return o, lse2 * math.log(2.0)


def _branches_swapped(q, k, v, causal=True):
    o, lse2 = _ORIG_BRANCHES(q, k, v, causal)
    o2 = o.copy()
    o2[:, :, 0::2], o2[:, :, 1::2] = o[:, :, 1::2], o[:, :, 0::2]
    return o2, lse2


def _branch_weights_no_scale(q1, q2, k, lam, n_visible=None):
    q1, q2, k = (np.asarray(x, dtype=np.float64) for x in (q1, q2, k))
    m = k.shape[0] if n_visible is None else int(n_visible)
    a1 = ora.stable_softmax(k[:m] @ q1)
    a2 = ora.stable_softmax(k[:m] @ q2)
    return a1, a2, a1 - float(lam) * a2


def _snr_signed_mean(weights, signal_index):
    w = np.asarray(weights, dtype=np.float64)
    return float(w[signal_index] / np.mean(np.delete(w, signal_index)))


_ORIG_BRANCHES = ora.prefill_branches

def _varlen_window_ignored(q, k, v, lam, cu_seqlens, causal=True, window=None):
    return _VARLEN(q, k, v, lam, cu_seqlens, causal=causal)


_VARLEN = ora.prefill_varlen
_BWD_VARLEN = ora.prefill_backward_varlen
_DECODE = ora.decode


def _decode_window_off_by_one(q, kcache, vcache, seqlens, lam, window=None):
    return _DECODE(q, kcache, vcache, seqlens, lam, window=None if window is None else window + 1)


def _backward_varlen_window_ignored(q, k, v, lam, dout, cu_seqlens, causal=True, window=None):
    return _BWD_VARLEN(q, k, v, lam, dout, cu_seqlens, causal=causal)


MUTANTS = {
    "varlen_window_ignored": ("prefill_varlen", _varlen_window_ignored),
    "decode_window_off_by_one": ("decode", _decode_window_off_by_one),
    "backward_varlen_window_ignored": ("prefill_backward_varlen", _backward_varlen_window_ignored),
    "plus_sign": ("diff_attention_block", _block_plus_sign),
    "no_scale": ("diff_attention_block", _block_no_scale),
    "scale_by_d": ("diff_attention_block", _block_scale_d),
    "lambda_on_first_branch": ("diff_attention_block", _block_lambda_on_first),
    "second_branch_dropped": ("diff_attention_block", _block_shared_query),
    "softmax_wrong_axis": ("diff_attention_block", _block_softmax_wrong_axis),
    "heads_swapped": ("pair_layout", _layout_swapped),
    "wrong_gqa_group": ("pair_layout", _layout_wrong_group),
    "non_adjacent_pairs": ("pair_layout", _layout_split_heads),
    "mask_off_by_one": ("causal_mask", _mask_off_by_one),
    "mask_transposed": ("causal_mask", _mask_transposed),
    "softmax_unstable": ("stable_softmax", _softmax_no_max),
    "softmax_epsilon": ("stable_softmax", _softmax_off),
    "lambda_v1_plus": ("lambda_v1", _lambda_v1_plus),
    "window_off_by_one": ("window_mask", _window_off_by_one),
    "lambda_v2_no_sigmoid": ("lambda_v2_projection", _lambda_v2_no_sigmoid),
    "backward_no_softmax_rowsum": ("prefill_backward", _backward_variant(drop_rowsum=True)),
    "backward_dlambda_sign": ("prefill_backward", _backward_variant(dlam_sign=1.0)),
    "backward_dk_first_branch_only": ("prefill_backward", _backward_variant(dk_first_only=True)),
    "backward_dv_without_lambda": ("prefill_backward", _backward_variant(dv_no_lambda=True)),
    "backward_dq_unscaled": ("prefill_backward", _backward_variant(dq_unscaled=True)),
    "branches_lse_natural_log": ("prefill_branches", _branches_natural_log),
    "branches_heads_swapped": ("prefill_branches", _branches_swapped),
    "branch_weights_no_scale": ("branch_weights", _branch_weights_no_scale),
    "snr_signed_mean": ("snr", _snr_signed_mean),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(ora, attr, fn)
    failed = []
    with np.errstate(all="ignore"):
        for pin_name, pin in ALL_PINS.items():
            try:
                ok = pin()
            except Exception:  # a crash counts as a caught mutant
                ok = False
            if not ok:
                failed.append(pin_name)
    assert failed, f"mutant {name} passed every pin"
