"""GPU parity of the training forward and the backward pass against the float64 oracle
(through the C ABI)."""
import math

import numpy as np
import pytest
import torch

import workloads
from oracle import diffattn_f64 as ora
from tests.parity import bf16_close, grad_close, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def da():
    import differential_attention_v2_b200 as m

    assert torch.cuda.is_available()
    return m


def _case(B, S, Hq, Hkv, seed):
    case = workloads.PrefillCase(B=B, S=S, Hq=Hq, Hkv=Hkv, D=128, seed=seed)
    inp = workloads.make_prefill(case)
    inp["dout"] = workloads.make_prefill_grad(case)
    return inp


def _gpu_grads(da, inp, causal):
    d = {k: v.cuda() for k, v in inp.items()}
    out, ob, lse = da.prefill_train(d["q"], d["k"], d["v"], d["lam"], causal=causal)
    dq, dk, dv, dlam = da.backward(d["q"], d["k"], d["v"], d["lam"], ob, lse, d["dout"], causal=causal)
    torch.cuda.synchronize()
    assert da.device_error() == 0
    return (out, ob, lse), (dq, dk, dv, dlam)


def _check_grads(got, inp, causal, what):
    ref = ora.prefill_backward(inp["q"], inp["k"], inp["v"], inp["lam"], inp["dout"], causal=causal)
    for g, r, name in zip(got, ref, ("dq", "dk", "dv", "dlam")):
        grad_close(g, r, f"{what} {name}")


@pytest.mark.parametrize("B,S,Hq,Hkv,causal", [
    (1, 128, 4, 1, True),      # one tile, group of 4
    (2, 300, 8, 2, True),      # ragged tail (64-key and 32-row steps, 128-row forward tiles)
    (1, 1, 2, 1, True),        # a single token
    (1, 129, 16, 1, True),     # tile boundary + 1, group of 16
    (1, 640, 32, 4, True),     # several tiles, group of 8
    (2, 200, 8, 2, False),     # non-causal with ragged tiles
    (1, 513, 4, 2, False),     # non-causal, group of 2
])
def test_backward_matches_oracle(da, B, S, Hq, Hkv, causal):
    inp = _case(B, S, Hq, Hkv, seed=31 + S + Hq)
    _, grads = _gpu_grads(da, inp, causal)
    _check_grads(grads, inp, causal, f"B={B} S={S} Hq={Hq} Hkv={Hkv} causal={causal}")


def test_training_forward_outputs(da):
    """out equals the inference prefill bit for bit; O_b and lse match the oracle."""
    inp = _case(2, 300, 8, 2, seed=41)
    for causal in (True, False):
        (out, ob, lse), _ = _gpu_grads(da, inp, causal)
        d = {k: v.cuda() for k, v in inp.items()}
        assert torch.equal(out, da.prefill(d["q"], d["k"], d["v"], d["lam"], causal=causal))
        o_ref, lse_ref = ora.prefill_branches(inp["q"], inp["k"], inp["v"], causal=causal)
        bf16_close(ob, o_ref, f"o_branch causal={causal}")
        assert float(np.abs(to64(lse) - lse_ref).max()) < 1e-3, "lse"


def test_backward_lambda_edge_values(da):
    inp = _case(1, 200, 8, 1, seed=43)
    g = torch.Generator().manual_seed(4)
    inp["lam"] = (torch.rand(inp["lam"].shape, generator=g) * 4.0 - 1.5).float()
    inp["lam"][0, :10] = 0.0
    _, grads = _gpu_grads(da, inp, True)
    _check_grads(grads, inp, True, "lambda in [-1.5, 2.5]")


def test_backward_equal_branches_are_antisymmetric(da):
    """Q1 == Q2 and lambda == 1: the two heads of a pair get exactly opposite dQ."""
    inp = _case(1, 300, 8, 2, seed=47)
    inp["q"][:, :, 1::2] = inp["q"][:, :, 0::2]
    inp["lam"][:] = 1.0
    _, (dq, dk, dv, dlam) = _gpu_grads(da, inp, True)
    assert torch.equal(dq[:, :, 1::2], -dq[:, :, 0::2])


def test_backward_is_deterministic(da):
    inp = _case(2, 300, 16, 2, seed=53)
    _, g1 = _gpu_grads(da, inp, True)
    _, g2 = _gpu_grads(da, inp, True)
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)


def test_backward_full_size_one_group(da):
    """B=4 S=4096 Hq=64 Hkv=8: gradients of one (batch, KV group) slice against the oracle on
    that slice (dK, dV of the KV head; dQ of its 8 query heads; dlambda of its 4 pairs)."""
    case = workloads.CONFIGS["prefill_b4_s4096"]
    inp = workloads.make_prefill(case)
    inp["dout"] = workloads.make_prefill_grad(case)
    _, (dq, dk, dv, dlam) = _gpu_grads(da, inp, True)
    b, g = 3, 5
    G = case.Hq // case.Hkv
    heads = slice(g * G, (g + 1) * G)
    pairs = slice(g * G // 2, (g + 1) * G // 2)
    sl = {"q": inp["q"][b:b + 1, :, heads], "k": inp["k"][b:b + 1, :, g:g + 1],
          "v": inp["v"][b:b + 1, :, g:g + 1], "lam": inp["lam"][b:b + 1, :, pairs],
          "dout": inp["dout"][b:b + 1, :, pairs]}
    got = (dq[b:b + 1, :, heads], dk[b:b + 1, :, g:g + 1], dv[b:b + 1, :, g:g + 1], dlam[b:b + 1, :, pairs])
    _check_grads(got, sl, True, "B=4 S=4096 slice b=3 g=5")


def _packed(lens, Hq, Hkv, seed):
    T = sum(lens)
    case = workloads.PrefillCase(B=1, S=max(T, 1), Hq=Hq, Hkv=Hkv, D=128, seed=seed)
    inp = workloads.make_prefill(case)
    inp["dout"] = workloads.make_prefill_grad(case)
    packed = {k: v[0, :T].contiguous() for k, v in inp.items()}
    cu = [0]
    for L in lens:
        cu.append(cu[-1] + L)
    return packed, cu


def _gpu_varlen(da, inp, cu, causal):
    d = {k: v.cuda() for k, v in inp.items()}
    cu_t = torch.tensor(cu, dtype=torch.int32, device="cuda")
    mx = max(b - a for a, b in zip(cu[:-1], cu[1:]))
    out, ob, lse = da.prefill_varlen_train(d["q"], d["k"], d["v"], d["lam"], cu_t, mx, causal=causal)
    grads = da.backward_varlen(d["q"], d["k"], d["v"], d["lam"], ob, lse, d["dout"], cu_t, mx, causal=causal)
    torch.cuda.synchronize()
    assert da.device_error() == 0
    return (out, ob, lse), grads


@pytest.mark.parametrize("lens,Hq,Hkv,causal", [
    ([300, 1, 0, 200, 129], 8, 2, True),   # ragged, a single token, an empty sequence, tile + 1
    ([64, 65, 127, 128], 16, 2, True),     # offsets that are not multiples of 64 or 128
    ([513, 37], 4, 2, True),               # several tiles, group of 2
    ([300, 90, 200], 8, 1, False),         # full attention inside each sequence, group of 8
])
def test_backward_varlen_matches_oracle(da, lens, Hq, Hkv, causal):
    inp, cu = _packed(lens, Hq, Hkv, seed=61 + len(lens) + Hq)
    (out, ob, lse), grads = _gpu_varlen(da, inp, cu, causal)
    d = {k: v.cuda() for k, v in inp.items()}
    cu_t = torch.tensor(cu, dtype=torch.int32, device="cuda")
    mx = max(lens)
    assert torch.equal(out, da.prefill_varlen(d["q"], d["k"], d["v"], d["lam"], cu_t, mx, causal=causal))
    ref = ora.prefill_backward_varlen(inp["q"], inp["k"], inp["v"], inp["lam"], inp["dout"], cu, causal=causal)
    for g, r, name in zip(grads, ref, ("dq", "dk", "dv", "dlam")):
        grad_close(g, r, f"varlen {lens} causal={causal} {name}")


@pytest.mark.parametrize("lens,window,Hq,Hkv", [
    ([300, 1, 0, 200, 129], 64, 8, 2),     # ragged, single token, empty; window inside a tile
    ([513, 37, 260], 200, 16, 2),          # window wider than a tile
    ([300, 90], 1, 4, 2),                  # each query sees only itself
])
def test_backward_varlen_window_matches_oracle(da, lens, window, Hq, Hkv):
    inp, cu = _packed(lens, Hq, Hkv, seed=81 + window)
    d = {k: v.cuda() for k, v in inp.items()}
    cu_t = torch.tensor(cu, dtype=torch.int32, device="cuda")
    mx = max(lens)
    out, ob, lse = da.prefill_varlen_train(d["q"], d["k"], d["v"], d["lam"], cu_t, mx, window=window)
    assert torch.equal(out, da.prefill_varlen_window(d["q"], d["k"], d["v"], d["lam"], cu_t, mx, window))
    grads = da.backward_varlen(d["q"], d["k"], d["v"], d["lam"], ob, lse, d["dout"], cu_t, mx, window=window)
    torch.cuda.synchronize()
    assert da.device_error() == 0
    ref = ora.prefill_backward_varlen(inp["q"], inp["k"], inp["v"], inp["lam"], inp["dout"], cu, window=window)
    for g, r, name in zip(grads, ref, ("dq", "dk", "dv", "dlam")):
        grad_close(g, r, f"varlen window={window} {lens} {name}")


def test_backward_varlen_window_equal_lengths_equals_batched(da):
    """Packed sequences of equal length with a window: bit-identical to the batched window backward."""
    B, S, Hq, Hkv, W = 3, 300, 8, 2, 100
    case = workloads.PrefillCase(B=B, S=S, Hq=Hq, Hkv=Hkv, D=128, seed=87)
    inp = workloads.make_prefill(case)
    inp["dout"] = workloads.make_prefill_grad(case)
    d = {k: v.cuda() for k, v in inp.items()}
    out, ob, lse = da.prefill_train(d["q"], d["k"], d["v"], d["lam"], window=W)
    g_batched = da.backward(d["q"], d["k"], d["v"], d["lam"], ob, lse, d["dout"], window=W)
    flat = lambda t: t.reshape((B * S,) + t.shape[2:]).contiguous()
    cu = torch.tensor([0, S, 2 * S, 3 * S], dtype=torch.int32, device="cuda")
    outp, obp, lsep = da.prefill_varlen_train(flat(d["q"]), flat(d["k"]), flat(d["v"]), flat(d["lam"]), cu, S, window=W)
    assert torch.equal(outp.view(B, S, Hq // 2, 128), out)
    g_packed = da.backward_varlen(flat(d["q"]), flat(d["k"]), flat(d["v"]), flat(d["lam"]), obp, lsep, flat(d["dout"]),
                                  cu, S, window=W)
    assert da.device_error() == 0
    for a, b in zip(g_batched, g_packed):
        assert torch.equal(a.reshape(b.shape), b)


def test_backward_varlen_equal_lengths_equals_batched(da):
    """Packed sequences of equal (ragged) length give bit-identical gradients to the batch."""
    B, S, Hq, Hkv = 3, 300, 8, 2
    case = workloads.PrefillCase(B=B, S=S, Hq=Hq, Hkv=Hkv, D=128, seed=67)
    inp = workloads.make_prefill(case)
    inp["dout"] = workloads.make_prefill_grad(case)
    _, g_batched = _gpu_grads(da, inp, True)
    packed = {k: v.reshape((B * S,) + v.shape[2:]).contiguous() for k, v in inp.items()}
    _, g_packed = _gpu_varlen(da, packed, [0, S, 2 * S, 3 * S], True)
    for a, b in zip(g_batched, g_packed):
        assert torch.equal(a.reshape(b.shape), b)


@pytest.mark.parametrize("S,window,Hq,Hkv", [
    (300, 1, 8, 2),       # every query sees only itself
    (300, 64, 8, 2),      # window inside one 64-key block
    (700, 100, 16, 2),    # window across block and tile edges, several tiles
    (513, 300, 4, 2),     # window wider than a tile
])
def test_backward_window_matches_oracle(da, S, window, Hq, Hkv):
    inp = _case(1, S, Hq, Hkv, seed=71 + window)
    d = {k: v.cuda() for k, v in inp.items()}
    out, ob, lse = da.prefill_train(d["q"], d["k"], d["v"], d["lam"], window=window)
    assert torch.equal(out, da.prefill_window(d["q"], d["k"], d["v"], d["lam"], window))
    grads = da.backward(d["q"], d["k"], d["v"], d["lam"], ob, lse, d["dout"], window=window)
    torch.cuda.synchronize()
    assert da.device_error() == 0
    ref = ora.prefill_backward(inp["q"], inp["k"], inp["v"], inp["lam"], inp["dout"], window=window)
    for g, r, name in zip(grads, ref, ("dq", "dk", "dv", "dlam")):
        grad_close(g, r, f"window={window} S={S} {name}")


def test_backward_window_wider_than_sequence_is_causal(da):
    inp = _case(2, 300, 8, 2, seed=79)
    d = {k: v.cuda() for k, v in inp.items()}
    _, g_causal = _gpu_grads(da, inp, True)
    out, ob, lse = da.prefill_train(d["q"], d["k"], d["v"], d["lam"], window=300)
    g_win = da.backward(d["q"], d["k"], d["v"], d["lam"], ob, lse, d["dout"], window=300)
    for a, b in zip(g_causal, g_win):
        assert torch.equal(a, b)
