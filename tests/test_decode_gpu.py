"""GPU parity of the decode and lambda entry points against the float64 oracle."""
import numpy as np
import pytest
import torch

import workloads
from oracle import diffattn_f64 as ora
from tests.parity import bf16_close, f32_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def da():
    import differential_attention_v2_b200 as m

    assert torch.cuda.is_available()
    return m


def _decode_case(B, Smax, Hq, Hkv, lens, seed, dtype="bf16"):
    inp = workloads.make_decode(workloads.DecodeCase(B=B, Smax=Smax, Hq=Hq, Hkv=Hkv, D=128, len_lo=1,
                                                     len_hi=Smax, dtype=dtype, seed=seed))
    inp["seqlens"] = torch.tensor(lens, dtype=torch.int32)
    return inp


def _run(da, inp):
    out = da.decode(inp["q"].cuda(), inp["kcache"].cuda(), inp["vcache"].cuda(), inp["seqlens"].cuda(),
                    inp["lam"].cuda())
    assert da.device_error() == 0
    return out


@pytest.mark.parametrize("B,Smax,Hq,Hkv,lens", [
    (3, 300, 16, 2, [300, 1, 0]),            # full, single key, empty sequence
    (4, 1000, 64, 8, [1000, 999, 64, 65]),    # group of 8, stage boundaries
    (2, 700, 8, 4, [700, 129]),               # group of 2
    (2, 700, 16, 4, [511, 700]),              # group of 4
    (2, 900, 32, 2, [900, 333]),              # group of 16 (two head tiles)
    (1, 5000, 8, 1, [5000]),                  # several splits
])
def test_decode_bf16_matches_oracle(da, B, Smax, Hq, Hkv, lens):
    inp = _decode_case(B, Smax, Hq, Hkv, lens, seed=B * Smax + Hq)
    out = _run(da, inp)
    ref = ora.decode(inp["q"], inp["kcache"], inp["vcache"], inp["seqlens"], inp["lam"])
    bf16_close(out, ref, f"decode B={B} Smax={Smax} Hq={Hq} Hkv={Hkv}")
    for b, n in enumerate(lens):
        if n == 0:
            assert torch.count_nonzero(out[b]).item() == 0


@pytest.mark.parametrize("B,Smax,Hq,Hkv,lens,window", [
    (4, 3000, 64, 8, [3000, 1, 0, 2100], 1),         # only the newest key; an empty sequence
    (4, 3000, 64, 8, [3000, 130, 64, 2100], 64),     # window of one stage, lengths at stage edges
    (3, 5000, 32, 2, [5000, 4097, 700], 700),        # group of 16, window starting mid-stage
    (2, 9000, 16, 4, [9000, 1500], 4096),            # a window spanning several splits
    (3, 800, 16, 2, [800, 100, 799], 5000),          # window wider than every sequence
])
def test_decode_window_matches_oracle(da, B, Smax, Hq, Hkv, lens, window):
    inp = _decode_case(B, Smax, Hq, Hkv, lens, seed=40 + window)
    out = da.decode(inp["q"].cuda(), inp["kcache"].cuda(), inp["vcache"].cuda(), inp["seqlens"].cuda(),
                    inp["lam"].cuda(), window=window)
    assert da.device_error() == 0
    ref = ora.decode(inp["q"], inp["kcache"], inp["vcache"], inp["seqlens"], inp["lam"], window=window)
    bf16_close(out, ref, f"decode window={window} lens={lens}")
    if window >= Smax:
        # the plain decode, bit for bit
        assert torch.equal(out, _run(da, inp))


@pytest.mark.parametrize("page_size,window", [(16, 100), (64, 64), (256, 700)])
def test_decode_paged_window_matches_contiguous(da, page_size, window):
    """The windowed decode over a shuffled paged copy of the cache: parity with the oracle and
    bit-identity with the contiguous windowed decode (same Smax, same splits)."""
    B, Smax, Hq, Hkv = 3, 2048, 32, 4
    lens = [2048, 700, 90]
    inp = _decode_case(B, Smax, Hq, Hkv, lens, seed=60 + page_size)
    n_pg = Smax // page_size
    g = torch.Generator().manual_seed(61)
    perm = torch.randperm(B * n_pg, generator=g)
    kp = torch.empty(B * n_pg, page_size, Hkv, 128, dtype=torch.bfloat16)
    vp = torch.empty_like(kp)
    kp[perm] = inp["kcache"].reshape(B * n_pg, page_size, Hkv, 128)
    vp[perm] = inp["vcache"].reshape(B * n_pg, page_size, Hkv, 128)
    table = perm.view(B, n_pg).to(torch.int32)
    d = {k: inp[k].cuda() for k in ("q", "kcache", "vcache", "seqlens", "lam")}
    out = da.decode_paged(d["q"], kp.cuda(), vp.cuda(), table.cuda(), d["seqlens"], d["lam"], window=window)
    assert da.device_error() == 0
    ref = ora.decode_paged(inp["q"], kp, vp, table.tolist(), inp["seqlens"], inp["lam"], window=window)
    bf16_close(out, ref, f"paged decode window={window} page_size={page_size}")
    contiguous = da.decode(d["q"], d["kcache"], d["vcache"], d["seqlens"], d["lam"], window=window)
    assert torch.equal(out, contiguous)


def test_decode_matches_last_prefill_row(da):
    """One decode step over n cached keys equals row n-1 of a prefill of length n."""
    case = workloads.PrefillCase(B=1, S=333, Hq=16, Hkv=2, D=128, seed=21)
    inp = workloads.make_prefill(case)
    pre = da.prefill(inp["q"].cuda(), inp["k"].cuda(), inp["v"].cuda(), inp["lam"].cuda()).cpu()
    dec = da.decode(inp["q"][:, -1].contiguous().cuda(), inp["k"].cuda(), inp["v"].cuda(),
                    torch.tensor([333], dtype=torch.int32, device="cuda"), inp["lam"][:, -1].contiguous().cuda()).cpu()
    ref = ora.prefill_rows(inp["q"], inp["k"], inp["v"], inp["lam"], [(0, 332, p) for p in range(8)])
    bf16_close(dec[0], ref, "decode row")
    bf16_close(pre[0, -1], ref, "prefill row")


def test_decode_c4_full_size(da):
    """The 64-sequence decode workload (lengths uniform in [1024, 8192]) in full."""
    inp = workloads.make_decode(workloads.CONFIGS["decode_b64_s8192"])
    out = _run(da, inp)
    ref = ora.decode(inp["q"], inp["kcache"], inp["vcache"], inp["seqlens"], inp["lam"])
    bf16_close(out, ref, "decode B=64 Smax=8192")


def test_decode_c5_needle_with_v1_lambda(da):
    """The 128k needle workload with the V1 lambda computed on the GPU, in full."""
    case = workloads.CONFIGS["needle_decode_b8_s131072"]
    inp = workloads.make_decode(case)
    B, n_pairs = case.B, case.Hq // 2
    lam = da.lambda_v1(inp["lq1"].cuda(), inp["lk1"].cuda(), inp["lq2"].cuda(), inp["lk2"].cuda(),
                       inp["lambda_init"], rows=B)
    lam_ref = ora.lambda_v1(inp["lq1"], inp["lk1"], inp["lq2"], inp["lk2"], inp["lambda_init"])
    np.testing.assert_allclose(lam.cpu().double().numpy(), np.broadcast_to(lam_ref, (B, n_pairs)), rtol=2e-6, atol=2e-6)
    inp["lam"] = lam.cpu()
    out = _run(da, inp)
    ref = ora.decode(inp["q"], inp["kcache"], inp["vcache"], inp["seqlens"], inp["lam"])
    bf16_close(out, ref, "needle decode B=8 L=131072")


def test_lambda_v1_matches_oracle(da):
    g = torch.Generator().manual_seed(4)
    vec = [torch.randn(32, 128, generator=g) * 0.3 for _ in range(4)]
    for init in (0.8, 0.0, -0.2):
        got = da.lambda_v1(*(x.cuda() for x in vec), lambda_init=init, rows=5)
        ref = ora.lambda_v1(*vec, init)
        np.testing.assert_allclose(got.cpu().double().numpy(), np.broadcast_to(ref, (5, 32)), rtol=1e-5, atol=1e-6)


@pytest.mark.parametrize("lens,D", [([300, 1, 0], 128), ([77, 200], 64)])
def test_decode_f32_matches_oracle(da, lens, D):
    B, Smax, Hq, Hkv = len(lens), max(lens), 8, 2
    inp = workloads.make_decode(workloads.DecodeCase(B=B, Smax=Smax, Hq=Hq, Hkv=Hkv, D=D, len_lo=1, len_hi=Smax,
                                                     dtype="f32", seed=D))
    inp["seqlens"] = torch.tensor(lens, dtype=torch.int32)
    out = da.decode_f32(inp["q"].cuda(), inp["kcache"].cuda(), inp["vcache"].cuda(), inp["seqlens"].cuda(),
                        inp["lam"].cuda())
    ref = ora.decode(inp["q"], inp["kcache"], inp["vcache"], inp["seqlens"], inp["lam"])
    f32_close(out, ref, "fp32 decode")


def test_decode_equal_heads_cancel_exactly(da):
    """Q1 = Q2 with lambda = 1 cancels exactly in the decode path too."""
    inp = _decode_case(3, 700, 16, 2, [700, 5, 380], seed=31)
    inp["q"][:, 1::2] = inp["q"][:, 0::2]
    inp["lam"].fill_(1.0)
    out = _run(da, inp)
    assert torch.count_nonzero(out).item() == 0


def _paged(kc, vc, page_size, seed):
    """Scatter contiguous caches [B,Smax,Hkv,D] into shuffled pages; returns pages + table."""
    B, Smax = kc.shape[:2]
    max_pages = Smax // page_size
    n_pages = B * max_pages + 3
    perm = torch.randperm(n_pages, generator=torch.Generator().manual_seed(seed))[: B * max_pages]
    table = perm.view(B, max_pages).to(torch.int32)
    kp = torch.zeros(n_pages, page_size, *kc.shape[2:], dtype=kc.dtype)
    vp = torch.zeros_like(kp)
    for b in range(B):
        for i in range(max_pages):
            kp[table[b, i]] = kc[b, i * page_size:(i + 1) * page_size]
            vp[table[b, i]] = vc[b, i * page_size:(i + 1) * page_size]
    return kp, vp, table


@pytest.mark.parametrize("page_size,lens", [(16, [1024, 17, 0, 1000]), (64, [1024, 640, 65, 1]),
                                            (256, [1024, 1023, 300, 257]), (8, [512, 9, 100, 511])])
def test_decode_paged_matches_contiguous_and_oracle(da, page_size, lens):
    B, Hq, Hkv = len(lens), 16, 2
    Smax = ((max(lens) + page_size - 1) // page_size) * page_size
    inp = _decode_case(B, Smax, Hq, Hkv, lens, seed=page_size)
    kp, vp, table = _paged(inp["kcache"], inp["vcache"], page_size, seed=page_size)
    got = da.decode_paged(inp["q"].cuda(), kp.cuda(), vp.cuda(), table.cuda(), inp["seqlens"].cuda(),
                          inp["lam"].cuda())
    assert da.device_error() == 0
    contiguous = _run(da, inp)
    assert torch.equal(got, contiguous)  # same splits, same arithmetic
    ref = ora.decode_paged(inp["q"], kp, vp, table.tolist(), inp["seqlens"], inp["lam"])
    bf16_close(got, ref, f"paged decode page_size={page_size}")


@pytest.mark.parametrize("T,d_model,n_pairs,with_bias", [
    (1, 64, 8, False), (100, 256, 32, True), (4096, 4096, 32, True), (333, 512, 64, False), (70, 128, 40, True),
    # ragged last 32-token tiles, one 64-wide chunk of d_model, the bench's 16k x 4096 shape
    (193, 256, 8, False), (20000, 2048, 24, True), (16384, 4096, 32, False),
    # d_model an odd multiple of 64: the kernel's last 128-wide chunk is half past the end
    (257, 192, 16, True), (130, 320, 8, False)])
def test_lambda_v2_projection_matches_oracle(da, T, d_model, n_pairs, with_bias):
    g = torch.Generator().manual_seed(T + n_pairs)
    x = torch.randn(T, d_model, generator=g).bfloat16()
    w = (torch.randn(d_model, n_pairs, generator=g) / d_model ** 0.5).bfloat16()
    bias = torch.randn(n_pairs, generator=g) if with_bias else None
    got = da.lambda_v2(x.cuda(), w.cuda(), None if bias is None else bias.cuda())
    ref = ora.lambda_v2_projection(x, w, bias)
    np.testing.assert_allclose(got.cpu().double().numpy(), ref, rtol=0, atol=1e-5)
    assert torch.all((got > 0) & (got < 1))


@pytest.mark.parametrize("B,T,Smax,Hq,Hkv,lens", [
    (3, 2, 700, 16, 2, [700, 2, 301]),       # group 8, two tokens (two column tiles)
    (2, 4, 900, 8, 2, [900, 65]),            # group 4, four tokens
    (2, 8, 500, 4, 2, [500, 8]),             # group 2, eight tokens
    (2, 1, 600, 16, 2, [600, 1]),            # one token: the plain decode
])
def test_decode_multi_matches_oracle(da, B, T, Smax, Hq, Hkv, lens):
    inp = _decode_case(B, Smax, Hq, Hkv, lens, seed=T * 100 + Smax)
    g = torch.Generator().manual_seed(T)
    q = torch.randn(B, T, Hq, 128, generator=g).bfloat16()
    lam = torch.sigmoid(torch.randn(B, T, Hq // 2, generator=g))
    out = da.decode_multi(q.cuda(), inp["kcache"].cuda(), inp["vcache"].cuda(), inp["seqlens"].cuda(), lam.cuda())
    assert da.device_error() == 0
    ref = ora.decode_multi(q, inp["kcache"], inp["vcache"], inp["seqlens"], lam)
    bf16_close(out, ref, f"decode_multi T={T}")
    if T == 1:
        single = da.decode(q[:, 0].contiguous().cuda(), inp["kcache"].cuda(), inp["vcache"].cuda(),
                           inp["seqlens"].cuda(), lam[:, 0].contiguous().cuda())
        assert torch.equal(out[:, 0], single)
