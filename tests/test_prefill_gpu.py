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


# Launches with several work items per CTA (one persistent CTA per SM on 148 SMs): item
# boundaries, both parities of the per-item barriers and row-sum buffers, odd and even bands.
@pytest.mark.parametrize("B,S,Hq,Hkv,causal,window", [
    (8, 1024, 32, 4, True, 0),     # 1024 items, ~7 per CTA, causal work 1..8 KV tiles
    (6, 700, 16, 2, False, 0),     # 288 items, all of equal work, ragged last key tile
    (8, 1024, 32, 4, True, 200),   # sliding window over many items
])
def test_prefill_many_items_per_cta(da, B, S, Hq, Hkv, causal, window):
    inp = workloads.make_prefill(workloads.PrefillCase(B=B, S=S, Hq=Hq, Hkv=Hkv, D=128, seed=3 * S + window))
    d = _dev(inp)
    if window:
        out = da.prefill_window(d["q"], d["k"], d["v"], d["lam"], window)
    else:
        out = da.prefill(d["q"], d["k"], d["v"], d["lam"], causal=causal)
    assert da.device_error() == 0
    ref = ora.prefill(inp["q"], inp["k"], inp["v"], inp["lam"], causal=causal, window=window or None)
    bf16_close(out, ref, f"many items B={B} S={S} Hq={Hq} causal={causal} window={window}")


def test_prefill_train_many_items_per_cta(da):
    """The training forward's per-head O_b and row lse over 256 items (~2 per CTA)."""
    inp = workloads.make_prefill(workloads.PrefillCase(B=4, S=1024, Hq=16, Hkv=2, D=128, seed=77))
    d = _dev(inp)
    out, ob, lse = da.prefill_train(d["q"], d["k"], d["v"], d["lam"])
    assert da.device_error() == 0
    assert torch.equal(out, da.prefill(d["q"], d["k"], d["v"], d["lam"]))
    o_ref, lse_ref = ora.prefill_branches(inp["q"], inp["k"], inp["v"])
    bf16_close(ob, o_ref, "o_branch, many items")
    assert float(np.abs(lse.double().cpu().numpy() - lse_ref).max()) < 1e-3, "lse"


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


@pytest.mark.parametrize("name,n_rows", [("prefill_b4_s4096", 1024), ("prefill_b1_s32768", 1024)])
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
    inp = workloads.make_prefill(workloads.CONFIGS["tiny_fp32_prefill_b1_s128"])
    row, sig = workloads.plant_signal_row(inp)
    d = _dev(inp)
    out = da.prefill_f32(d["q"], d["k"], d["v"], d["lam"])
    ref = ora.prefill(inp["q"], inp["k"], inp["v"], inp["lam"])
    f32_close(out, ref, "tiny fp32 prefill")
    f32_close(out[0, row, 0], ref[0, row, 0], "tiny fp32 planted row")


@pytest.mark.parametrize("B,S,Hq,Hkv,D,causal", [
    (2, 77, 8, 2, 128, True), (1, 200, 4, 1, 64, False), (1, 1, 2, 1, 64, True)])
def test_prefill_f32_matches_oracle(da, B, S, Hq, Hkv, D, causal):
    inp = workloads.make_prefill(workloads.PrefillCase(B=B, S=S, Hq=Hq, Hkv=Hkv, D=D, dtype="f32", seed=S))
    d = _dev(inp)
    out = da.prefill_f32(d["q"], d["k"], d["v"], d["lam"], causal=causal)
    ref = ora.prefill(inp["q"], inp["k"], inp["v"], inp["lam"], causal=causal)
    f32_close(out, ref, f"fp32 prefill S={S} D={D}")


@pytest.mark.parametrize("B,S,Hq,Hkv,window", [
    (1, 300, 8, 2, 1),       # each query sees only itself
    (1, 300, 8, 2, 17),      # window inside one tile
    (2, 700, 8, 1, 128),     # exactly one tile wide
    (1, 700, 16, 2, 129),    # one more than a tile
    (1, 1000, 8, 2, 300),    # spans several tiles, ragged sequence
    (1, 257, 8, 2, 5000),    # wider than the sequence: plain causal
])
def test_prefill_window_matches_oracle(da, B, S, Hq, Hkv, window):
    inp = workloads.make_prefill(workloads.PrefillCase(B=B, S=S, Hq=Hq, Hkv=Hkv, D=128, seed=window + S))
    d = _dev(inp)
    out = da.prefill_window(d["q"], d["k"], d["v"], d["lam"], window)
    assert da.device_error() == 0
    ref = ora.prefill(inp["q"], inp["k"], inp["v"], inp["lam"], window=window)
    bf16_close(out, ref, f"window={window} S={S}")


def test_prefill_window_at_full_size_sampled(da):
    """The 4 x 4k workload with a 1024-key window (a hybrid sliding-window layer), sampled rows."""
    case = workloads.CONFIGS["prefill_b4_s4096"]
    inp = workloads.make_prefill(case)
    out = da.prefill_window(*(inp[x].cuda() for x in ("q", "k", "v", "lam")), 1024).cpu()
    assert da.device_error() == 0
    rows = sample_rows(case.B, case.S, case.Hq // 2, n=512, seed=5)
    # the row's window is the causal prefix of the slice that ends at the row
    ref = np.concatenate([ora.prefill_rows(*(inp[x][b:b + 1, max(0, i - 1023):i + 1] for x in ("q", "k", "v", "lam")),
                                           [(0, i - max(0, i - 1023), p)]) for b, i, p in rows])
    got = torch.stack([out[b, i, p] for b, i, p in rows])
    bf16_close(got, ref, "window 1024 sampled rows")


_MANY_LENS = [int(x) for x in np.random.default_rng(300).integers(0, 41, size=300)]


@pytest.mark.parametrize("lens,Hq,Hkv,causal,extra", [
    ([300, 1, 0, 129, 128, 77], 8, 2, True, 0),       # ragged, single token, empty, tile edges
    ([1000, 513], 16, 2, True, 0),
    ([200, 64, 390], 8, 1, False, 0),                 # non-causal packed sequences
    # longest length declared above the true one: the top row tiles hold no sequence
    ([700, 5, 0, 1300, 260, 129], 8, 2, True, 400),
    # more sequences than the kernel sorts in shared memory: one CTA per item
    (_MANY_LENS, 4, 2, True, 0),
])
def test_prefill_varlen_matches_oracle(da, lens, Hq, Hkv, causal, extra):
    T = sum(lens)
    g = torch.Generator().manual_seed(T)
    q = torch.randn(T, Hq, 128, generator=g).bfloat16()
    k = torch.randn(T, Hkv, 128, generator=g).bfloat16()
    v = torch.randn(T, Hkv, 128, generator=g).bfloat16()
    lam = torch.sigmoid(torch.randn(T, Hq // 2, generator=g))
    cu = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32)
    out = da.prefill_varlen(q.cuda(), k.cuda(), v.cuda(), lam.cuda(), cu.cuda(), max(lens) + extra, causal=causal)
    assert da.device_error() == 0
    ref = ora.prefill_varlen(q, k, v, lam, cu.tolist(), causal=causal)
    bf16_close(out, ref, f"varlen {lens}")


@pytest.mark.parametrize("lens,window,Hq,Hkv", [
    ([300, 1, 0, 200, 129, 700], 64, 8, 2),     # ragged, single token, empty; window inside a tile
    ([300, 1, 0, 200, 129, 700], 200, 16, 2),   # window wider than a tile
    ([513, 37, 260], 1, 4, 2),                  # each query sees only itself
    ([513, 37, 260], 1000, 8, 4),               # window past every sequence: plain causal
])
def test_prefill_varlen_window_matches_oracle(da, lens, window, Hq, Hkv):
    T = sum(lens)
    g = torch.Generator().manual_seed(T + window)
    q = torch.randn(T, Hq, 128, generator=g).bfloat16()
    k = torch.randn(T, Hkv, 128, generator=g).bfloat16()
    v = torch.randn(T, Hkv, 128, generator=g).bfloat16()
    lam = torch.sigmoid(torch.randn(T, Hq // 2, generator=g))
    cu = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32)
    out = da.prefill_varlen_window(q.cuda(), k.cuda(), v.cuda(), lam.cuda(), cu.cuda(), max(lens), window)
    assert da.device_error() == 0
    ref = ora.prefill_varlen(q, k, v, lam, cu.tolist(), window=window)
    bf16_close(out, ref, f"varlen window {window} {lens}")


@pytest.mark.parametrize("B,S", [(3, 333), (300, 150)])
def test_prefill_varlen_window_equals_batched_window(da, B, S):
    """Equal-length packed sequences with a window give the batched window prefill bit for bit
    (300 sequences: the one-CTA-per-item launch)."""
    case = workloads.PrefillCase(B=B, S=S, Hq=8, Hkv=2, D=128, seed=10 + B)
    inp = workloads.make_prefill(case)
    d = _dev(inp)
    batched = da.prefill_window(d["q"], d["k"], d["v"], d["lam"], 100)
    flat = lambda t: t.reshape(-1, *t.shape[2:]).contiguous()
    cu = torch.arange(0, (B + 1) * S, S, dtype=torch.int32, device="cuda")
    packed = da.prefill_varlen_window(flat(d["q"]), flat(d["k"]), flat(d["v"]), flat(d["lam"]), cu, S, 100)
    assert da.device_error() == 0
    assert torch.equal(packed.view(B, S, 4, 128), batched)


def test_prefill_varlen_equals_batched(da):
    """Equal-length packed sequences give the batched prefill's output bit for bit."""
    case = workloads.PrefillCase(B=3, S=333, Hq=16, Hkv=2, D=128, seed=8)
    inp = workloads.make_prefill(case)
    d = _dev(inp)
    batched = da.prefill(d["q"], d["k"], d["v"], d["lam"])
    flat = lambda t: t.reshape(-1, *t.shape[2:]).contiguous()
    cu = torch.tensor([0, 333, 666, 999], dtype=torch.int32, device="cuda")
    packed = da.prefill_varlen(flat(d["q"]), flat(d["k"]), flat(d["v"]), flat(d["lam"]), cu, 333)
    assert torch.equal(packed.view(3, 333, 8, 128), batched)


def test_prefill_varlen_many_sequences_equals_batched(da):
    """300 equal-length packed sequences (one CTA per item) give the batched output bit for bit."""
    case = workloads.PrefillCase(B=300, S=150, Hq=4, Hkv=2, D=128, seed=9)
    inp = workloads.make_prefill(case)
    d = _dev(inp)
    batched = da.prefill(d["q"], d["k"], d["v"], d["lam"])
    flat = lambda t: t.reshape(-1, *t.shape[2:]).contiguous()
    cu = torch.arange(0, 301 * 150, 150, dtype=torch.int32, device="cuda")
    packed = da.prefill_varlen(flat(d["q"]), flat(d["k"]), flat(d["v"]), flat(d["lam"]), cu, 150)
    assert da.device_error() == 0
    assert torch.equal(packed.view(300, 150, 2, 128), batched)


def test_prefill_rejects_bad_arguments_on_gpu(da):
    q = torch.zeros(1, 16, 6, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 16, 2, 128, dtype=torch.bfloat16, device="cuda")
    lam = torch.zeros(1, 16, 3, device="cuda")
    with pytest.raises(da.DiffAttnError):
        da.prefill(q, k, k, lam)  # group of 3 heads: pairs would straddle KV heads
    assert da.device_error() == 0
