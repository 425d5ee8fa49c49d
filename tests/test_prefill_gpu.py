"""GPU parity of the prefill entry points against the float64 oracle (through the C ABI)."""
import numpy as np
import pytest
import torch

import workloads
from oracle import diffattn_f64 as ora
from tests.parity import bf16_close, f32_close, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def da():
    import differential_attention_v2_b200 as m

    assert torch.cuda.is_available()
    return m


def _dev(inp):
    return {k: (v.cuda() if hasattr(v, "cuda") else v) for k, v in inp.items()}


def _run_bf16(da, inp, causal=True):
    d = _dev(inp)
    out = da.prefill(d["q"], d["k"], d["v"], d["lam"], causal=causal)
    assert da.device_error() == 0
    return out


@pytest.mark.parametrize("B,S,Hq,Hkv,causal", [
    (1, 128, 4, 1, True),      # one tile, group of 4
    (2, 300, 8, 2, True),      # three tiles with a ragged tail
    (1, 1, 2, 1, True),        # a single token, the smallest pairing
    (1, 129, 16, 1, True),     # tile boundary + 1, group of 16
    (2, 257, 16, 4, True),     # group of 4
    (1, 640, 32, 4, True),     # five full tiles, group of 8
    (2, 300, 8, 2, False),     # full (non-causal) attention with a ragged key tile
    (1, 513, 4, 2, False),     # non-causal, group of 2
])
def test_prefill_bf16_matches_oracle(da, B, S, Hq, Hkv, causal):
    inp = workloads.make_prefill(workloads.PrefillCase(B=B, S=S, Hq=Hq, Hkv=Hkv, D=128, seed=7 + S + Hq))
    out = _run_bf16(da, inp, causal)
    ref = ora.prefill(inp["q"], inp["k"], inp["v"], inp["lam"], causal=causal)
    bf16_close(out, ref, f"prefill B={B} S={S} Hq={Hq} Hkv={Hkv} causal={causal}")


def test_prefill_bf16_lambda_edge_values(da):
    """lambda negative, zero and above one (V1 values may be any real number)."""
    inp = workloads.make_prefill(workloads.PrefillCase(B=1, S=200, Hq=8, Hkv=1, D=128, seed=5))
    g = torch.Generator().manual_seed(3)
    inp["lam"] = (torch.rand(inp["lam"].shape, generator=g) * 4.0 - 1.5).float()
    inp["lam"][0, :10] = 0.0
    out = _run_bf16(da, inp)
    ref = ora.prefill(inp["q"], inp["k"], inp["v"], inp["lam"])
    bf16_close(out, ref, "lambda in [-1.5, 2.5]")


def test_prefill_bf16_equal_heads_cancel_exactly(da):
    """Q1 = Q2 with lambda = 1: both branches run the same arithmetic, so the output is 0."""
    inp = workloads.make_prefill(workloads.PrefillCase(B=1, S=260, Hq=8, Hkv=2, D=128, seed=9))
    inp["q"][:, :, 1::2] = inp["q"][:, :, 0::2]
    inp["lam"].fill_(1.0)
    out = _run_bf16(da, inp)
    assert torch.count_nonzero(out).item() == 0


def test_prefill_bf16_value_ones(da):
    """V == 1: every output element is 1 - lambda (row sums of A1 - lambda A2)."""
    inp = workloads.make_prefill(workloads.PrefillCase(B=1, S=384, Hq=4, Hkv=1, D=128, seed=11))
    inp["v"].fill_(1.0)
    out = _run_bf16(da, inp)
    expect = (1.0 - inp["lam"].double())[..., None].expand(out.shape).numpy()
    bf16_close(out, expect, "V == 1")


def test_prefill_bf16_repeatable(da):
    inp = workloads.make_prefill(workloads.PrefillCase(B=1, S=384, Hq=8, Hkv=2, D=128, seed=13))
    a = _run_bf16(da, inp)
    b = _run_bf16(da, inp)
    assert torch.equal(a, b)


@pytest.mark.parametrize("name,n_rows", [("c2_bf16_prefill", 1024), ("c3_long_bf16_prefill", 1024)])
def test_prefill_bf16_full_size_sampled(da, name, n_rows):
    """Full-size workloads in the benchmark's launch configuration; a seeded stratified
    sample of rows (tile boundaries, first/last rows, every pair) checked against the oracle
    row by row, plus finiteness of the whole output."""
    case = workloads.CONFIGS[name]
    inp = workloads.make_prefill(case)
    out = _run_bf16(da, inp).cpu()
    assert torch.isfinite(out.float()).all()
    rows = sample_rows(case.B, case.S, case.Hq // 2, n=n_rows, seed=case.seed)
    ref = ora.prefill_rows(inp["q"], inp["k"], inp["v"], inp["lam"], rows)
    got = torch.stack([out[b, i, p] for b, i, p in rows])
    bf16_close(got, ref, f"{name} sampled rows")


def test_prefill_f32_c1_with_planted_row(da):
    """The tiny fp32 workload with the planted signal row: the whole output within 1e-5."""
    inp = workloads.make_prefill(workloads.CONFIGS["c1_tiny_fp32_prefill"])
    row, sig = workloads.plant_signal_row(inp)
    d = _dev(inp)
    out = da.prefill_f32(d["q"], d["k"], d["v"], d["lam"])
    ref = ora.prefill(inp["q"], inp["k"], inp["v"], inp["lam"])
    f32_close(out, ref, "c1 fp32")
    f32_close(out[0, row, 0], ref[0, row, 0], "c1 planted row")


@pytest.mark.parametrize("B,S,Hq,Hkv,D,causal", [
    (2, 77, 8, 2, 128, True), (1, 200, 4, 1, 64, False), (1, 1, 2, 1, 64, True)])
def test_prefill_f32_matches_oracle(da, B, S, Hq, Hkv, D, causal):
    inp = workloads.make_prefill(workloads.PrefillCase(B=B, S=S, Hq=Hq, Hkv=Hkv, D=D, dtype="f32", seed=S))
    d = _dev(inp)
    out = da.prefill_f32(d["q"], d["k"], d["v"], d["lam"], causal=causal)
    ref = ora.prefill(inp["q"], inp["k"], inp["v"], inp["lam"], causal=causal)
    f32_close(out, ref, f"fp32 prefill S={S} D={D}")


def test_prefill_rejects_bad_arguments_on_gpu(da):
    q = torch.zeros(1, 16, 6, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 16, 2, 128, dtype=torch.bfloat16, device="cuda")
    lam = torch.zeros(1, 16, 3, device="cuda")
    with pytest.raises(da.DiffAttnError):
        da.prefill(q, k, k, lam)  # group of 3 heads: pairs would straddle KV heads
    assert da.device_error() == 0
