"""GPU parity of the CTA-pair form of the prefill (two CTAs of a cluster share every MMA).

The pair form is chosen with DA2_PREFILL_CTA_PAIR=1 for GQA groups of a multiple of 4. Every
work item of it computes its rows with the same fp32 operations in the same order as the
one-CTA form, so the two must agree bit for bit; one case of each entry point is also checked
against the float64 oracle directly.
"""
import numpy as np
import pytest
import torch

import workloads
from oracle import diffattn_f64 as ora
from tests.parity import bf16_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def da():
    import differential_attention_v2_b200 as m

    assert torch.cuda.is_available()
    return m


def _dev(inp):
    return {k: v.cuda() for k, v in inp.items()}


def _both(monkeypatch, fn):
    monkeypatch.setenv("DA2_PREFILL_CTA_PAIR", "0")
    one = fn()
    monkeypatch.setenv("DA2_PREFILL_CTA_PAIR", "1")
    pair = fn()
    return one, pair


@pytest.mark.parametrize("B,S,Hq,Hkv,causal,window", [
    (1, 300, 8, 2, True, 0),      # one cluster per item, ragged tail, group of 4
    (8, 1024, 32, 4, True, 0),    # 512 items over the clusters: several per cluster, both parities
    (6, 700, 16, 2, False, 0),    # non-causal, group of 8, ragged last key tile
    (2, 257, 64, 4, True, 0),     # group of 16: four pair-pairs per KV head
    (8, 1024, 32, 4, True, 200),  # sliding window
])
def test_pair_form_equals_one_cta(da, monkeypatch, B, S, Hq, Hkv, causal, window):
    inp = workloads.make_prefill(workloads.PrefillCase(B=B, S=S, Hq=Hq, Hkv=Hkv, D=128, seed=31 + S + window))
    d = _dev(inp)

    def run():
        if window:
            o = da.prefill_window(d["q"], d["k"], d["v"], d["lam"], window)
        else:
            o = da.prefill(d["q"], d["k"], d["v"], d["lam"], causal=causal)
        assert da.device_error() == 0
        return o

    one, pair = _both(monkeypatch, run)
    assert torch.equal(one, pair)
    if B * S <= 4096:
        ref = ora.prefill(inp["q"], inp["k"], inp["v"], inp["lam"], causal=causal, window=window or None)
        bf16_close(pair, ref, f"pair form B={B} S={S} Hq={Hq} Hkv={Hkv} causal={causal} window={window}")


def test_pair_form_varlen_and_train(da, monkeypatch):
    """Packed sequences (ragged, empty, single-token) and the training forward's O_b and lse."""
    lens = [300, 1, 0, 129, 700, 77]
    T = sum(lens)
    g = torch.Generator().manual_seed(T)
    q = torch.randn(T, 16, 128, generator=g).bfloat16().cuda()
    k = torch.randn(T, 4, 128, generator=g).bfloat16().cuda()
    v = torch.randn(T, 4, 128, generator=g).bfloat16().cuda()
    lam = torch.sigmoid(torch.randn(T, 8, generator=g)).cuda()
    cu = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32, device="cuda")

    def varlen():
        o = da.prefill_varlen(q, k, v, lam, cu, max(lens))
        assert da.device_error() == 0
        return o

    one, pair = _both(monkeypatch, varlen)
    assert torch.equal(one, pair)
    ref = ora.prefill_varlen(q.cpu(), k.cpu(), v.cpu(), lam.cpu(), cu.tolist())
    bf16_close(pair, ref, "pair form, packed sequences")

    inp = workloads.make_prefill(workloads.PrefillCase(B=4, S=1024, Hq=16, Hkv=4, D=128, seed=78))
    d = _dev(inp)

    def train():
        r = da.prefill_train(d["q"], d["k"], d["v"], d["lam"])
        assert da.device_error() == 0
        return r

    (o1, ob1, l1), (o2, ob2, l2) = _both(monkeypatch, train)
    assert torch.equal(o1, o2) and torch.equal(ob1, ob2) and torch.equal(l1, l2)
