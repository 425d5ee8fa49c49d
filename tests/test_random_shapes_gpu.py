"""Seeded random shapes for every bf16 forward entry point, and the backward, against the
float64 oracle.

The fixed cases of the other files pin known edges; these draw sequence lengths, batch sizes,
GQA groups (2, 4, 8, 16), causal or full attention, window widths, packed-sequence length
mixes, decode lengths, page sizes and new-token counts from a fixed seed, so that shapes
nobody picked by hand (ragged tails at every position of a tile, items per CTA of every
count, partial last splits) run too. The prefill cases with a GQA group of a multiple of 4
run in both kernel forms (one CTA per item, and CTA pairs) and must agree bit for bit. The
backward cases draw causal, full or windowed attention and hold the gradients to the same
bounds as the fixed backward cases.
"""
import numpy as np
import pytest
import torch

import workloads
from oracle import diffattn_f64 as ora
from tests.parity import bf16_close

pytestmark = pytest.mark.gpu

_RNG = np.random.default_rng(20261203)
_GROUPS = [(4, 2), (8, 2), (16, 2), (32, 4), (16, 4), (64, 4), (8, 4)]  # (Hq, Hkv): groups 2, 4, 8, 16


def _prefill_cases(n):
    cases = []
    for i in range(n):
        Hq, Hkv = _GROUPS[int(_RNG.integers(len(_GROUPS)))]
        B = int(_RNG.integers(1, 4))
        S = int(_RNG.integers(1, 700))
        causal = bool(_RNG.integers(0, 4) > 0)
        window = int(_RNG.integers(1, S + 64)) if causal and _RNG.integers(0, 3) == 0 else 0
        cases.append((i, B, S, Hq, Hkv, causal, window))
    return cases


@pytest.fixture(scope="module")
def da():
    import differential_attention_v2_b200 as m

    assert torch.cuda.is_available()
    return m


@pytest.mark.parametrize("i,B,S,Hq,Hkv,causal,window", _prefill_cases(12))
def test_random_prefill(da, monkeypatch, i, B, S, Hq, Hkv, causal, window):
    inp = workloads.make_prefill(workloads.PrefillCase(B=B, S=S, Hq=Hq, Hkv=Hkv, D=128, seed=500 + i))
    d = {k: v.cuda() for k, v in inp.items()}

    def run():
        if window:
            o = da.prefill_window(d["q"], d["k"], d["v"], d["lam"], window)
        else:
            o = da.prefill(d["q"], d["k"], d["v"], d["lam"], causal=causal)
        assert da.device_error() == 0
        return o

    monkeypatch.setenv("DA2_PREFILL_CTA_PAIR", "0")
    out = run()
    ref = ora.prefill(inp["q"], inp["k"], inp["v"], inp["lam"], causal=causal, window=window or None)
    bf16_close(out, ref, f"random prefill {i}: B={B} S={S} Hq={Hq} Hkv={Hkv} causal={causal} window={window}")
    if (Hq // Hkv) % 4 == 0:
        monkeypatch.setenv("DA2_PREFILL_CTA_PAIR", "1")
        assert torch.equal(run(), out)


@pytest.mark.parametrize("i", range(4))
def test_random_packed_prefill(da, i):
    g = np.random.default_rng(600 + i)
    Hq, Hkv = _GROUPS[int(g.integers(len(_GROUPS)))]
    lens = [int(x) for x in g.integers(0, 400, size=int(g.integers(1, 7)))]
    T = max(1, sum(lens))
    if sum(lens) == 0:
        lens[0] = 1
    causal = bool(g.integers(0, 3) > 0)
    tg = torch.Generator().manual_seed(600 + i)
    q = torch.randn(T, Hq, 128, generator=tg).bfloat16()
    k = torch.randn(T, Hkv, 128, generator=tg).bfloat16()
    v = torch.randn(T, Hkv, 128, generator=tg).bfloat16()
    lam = torch.sigmoid(torch.randn(T, Hq // 2, generator=tg))
    cu = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32)
    out = da.prefill_varlen(q.cuda(), k.cuda(), v.cuda(), lam.cuda(), cu.cuda(), max(lens), causal=causal)
    assert da.device_error() == 0
    bf16_close(out, ora.prefill_varlen(q, k, v, lam, cu.tolist(), causal=causal), f"random packed {i}: {lens}")


@pytest.mark.parametrize("i", range(6))
def test_random_decodes(da, i):
    g = np.random.default_rng(700 + i)
    Hq, Hkv = _GROUPS[int(g.integers(len(_GROUPS)))]
    B = int(g.integers(1, 6))
    Smax = int(g.integers(64, 5000))
    lens = [int(x) for x in g.integers(0, Smax + 1, size=B)]
    case = workloads.DecodeCase(B=B, Smax=Smax, Hq=Hq, Hkv=Hkv, D=128, len_lo=1, len_hi=Smax, seed=700 + i)
    inp = workloads.make_decode(case)
    inp["seqlens"] = torch.tensor(lens, dtype=torch.int32)
    d = {k: inp[k].cuda() for k in ("q", "kcache", "vcache", "seqlens", "lam")}
    out = da.decode(d["q"], d["kcache"], d["vcache"], d["seqlens"], d["lam"])
    assert da.device_error() == 0
    ref = ora.decode(inp["q"], inp["kcache"], inp["vcache"], inp["seqlens"], inp["lam"])
    bf16_close(out, ref, f"random decode {i}: B={B} Smax={Smax} Hq={Hq} Hkv={Hkv} lens={lens}")
    # the same step over a shuffled paged copy of the cache
    ps = int(2 ** g.integers(3, 9))
    n_pg = (Smax + ps - 1) // ps
    tg = torch.Generator().manual_seed(800 + i)
    perm = torch.randperm(B * n_pg, generator=tg)
    pad = n_pg * ps - Smax
    kc = torch.nn.functional.pad(inp["kcache"], (0, 0, 0, 0, 0, pad))
    vc = torch.nn.functional.pad(inp["vcache"], (0, 0, 0, 0, 0, pad))
    kp = torch.empty(B * n_pg, ps, Hkv, 128, dtype=torch.bfloat16)
    vp = torch.empty_like(kp)
    kp[perm] = kc.reshape(B * n_pg, ps, Hkv, 128)
    vp[perm] = vc.reshape(B * n_pg, ps, Hkv, 128)
    table = perm.view(B, n_pg).to(torch.int32)
    outp = da.decode_paged(d["q"], kp.cuda(), vp.cuda(), table.cuda(), d["seqlens"], d["lam"])
    assert da.device_error() == 0
    bf16_close(outp, ref, f"random paged decode {i}: page size {ps}")
    # multi-token verification when the group leaves room for it (T x group <= 16)
    T = int(g.integers(2, 16 // (Hq // Hkv) + 1)) if Hq // Hkv <= 8 else 1
    if T > 1:
        qm = torch.randn(B, T, Hq, 128, generator=tg).bfloat16()
        lm = torch.sigmoid(torch.randn(B, T, Hq // 2, generator=tg))
        outm = da.decode_multi(qm.cuda(), d["kcache"], d["vcache"], d["seqlens"], lm.cuda())
        assert da.device_error() == 0
        bf16_close(outm, ora.decode_multi(qm, inp["kcache"], inp["vcache"], lens, lm), f"random multi-token {i}: T={T}")


def _backward_cases(n):
    g = np.random.default_rng(20261204)
    cases = []
    for i in range(n):
        Hq, Hkv = _GROUPS[int(g.integers(len(_GROUPS)))]
        B = int(g.integers(1, 3))
        S = int(g.integers(1, 450))
        mode = ("causal", "full", "window")[int(g.integers(0, 3))]
        window = int(g.integers(1, max(2, S // 2))) if mode == "window" else 0
        cases.append((i, B, S, Hq, Hkv, mode, window))
    return cases


@pytest.mark.parametrize("i,B,S,Hq,Hkv,mode,window", _backward_cases(6))
def test_random_backward(da, i, B, S, Hq, Hkv, mode, window):
    from tests.parity import grad_close

    case = workloads.PrefillCase(B=B, S=S, Hq=Hq, Hkv=Hkv, D=128, seed=1100 + i)
    inp = workloads.make_prefill(case)
    inp["dout"] = workloads.make_prefill_grad(case)
    d = {k: v.cuda() for k, v in inp.items()}
    causal = mode != "full"
    out, ob, lse = da.prefill_train(d["q"], d["k"], d["v"], d["lam"], causal=causal, window=window or None)
    grads = da.backward(d["q"], d["k"], d["v"], d["lam"], ob, lse, d["dout"], causal=causal, window=window or None)
    torch.cuda.synchronize()
    assert da.device_error() == 0
    ref = ora.prefill_backward(inp["q"], inp["k"], inp["v"], inp["lam"], inp["dout"], causal=causal,
                               window=window or None)
    for got, r, name in zip(grads, ref, ("dq", "dk", "dv", "dlam")):
        grad_close(got, r, f"random backward {i}: B={B} S={S} Hq={Hq} Hkv={Hkv} {mode} window={window} {name}")
