"""The bounds-checking build of the library on small parity cases.

libdiffattn_v2_debug.so is the library compiled with -DDA2_DEBUG_BOUNDS: its kernels compare
every checked shared-memory offset, tensor-memory column and global index with the extent it
addresses, and on a violation record code 4 in the device error word and skip the access.
These tests run the small cases of the prefill (one-CTA and CTA-pair forms, sliding window,
packed sequences with and without a window, training outputs, lambda computed in the kernel), the decode (GQA groups 8 and 16, paged cache,
multi-token) and the backward through it, and require both a zero error word and the usual
agreement with the float64 oracle. (No case here is meant to violate a bound.)
"""
import numpy as np
import pytest
import torch

import workloads
from oracle import diffattn_f64 as ora
from tests.parity import bf16_close, grad_close

pytestmark = pytest.mark.gpu

ERR_BOUNDS = 4


@pytest.fixture(scope="module")
def dbg():
    """The binding's wrappers, calling into the bounds-checking library for this module."""
    import differential_attention_v2_b200 as da
    from differential_attention_v2_b200 import _lib
    from differential_attention_v2_b200.build import DEBUG_LIB_PATH, build

    assert torch.cuda.is_available()
    build(debug_bounds=True)  # a no-op when the library is up to date
    saved = _lib.LIB
    _lib.LIB = _lib.load(DEBUG_LIB_PATH)
    try:
        yield da
    finally:
        _lib.LIB = saved


def _clean(da):
    torch.cuda.synchronize()
    code = da.device_error()
    assert code != ERR_BOUNDS, "a kernel reported an index outside its extent"
    assert code == 0, f"device error {code}"


def test_prefill_fused_lambda_in_bounds(dbg):
    B, S, Hq, Hkv, d_model = 2, 300, 8, 2, 256
    inp = workloads.make_prefill(workloads.PrefillCase(B=B, S=S, Hq=Hq, Hkv=Hkv, D=128, seed=57))
    g = torch.Generator().manual_seed(58)
    x = torch.randn(B, S, d_model, generator=g).bfloat16()
    w = (torch.randn(d_model, Hq // 2, generator=g) / d_model ** 0.5).bfloat16()
    d = {k: v.cuda() for k, v in inp.items()}
    lam = torch.empty(B, S, Hq // 2, device="cuda")
    out = dbg.prefill_fused_lambda(d["q"], d["k"], d["v"], x.cuda(), w.t().contiguous().cuda(), lambda_out=lam)
    _clean(dbg)
    lam_ref = ora.lambda_v2_projection(x.reshape(B * S, d_model), w).reshape(B, S, Hq // 2)
    np.testing.assert_allclose(lam.cpu().double().numpy(), lam_ref, rtol=0, atol=1e-5)
    bf16_close(out, ora.prefill(inp["q"], inp["k"], inp["v"], torch.from_numpy(lam_ref).float()),
               "debug fused-lambda prefill")


@pytest.mark.parametrize("pair", ["0", "1"])
def test_prefill_forms_window_and_train_in_bounds(dbg, monkeypatch, pair):
    monkeypatch.setenv("DA2_PREFILL_CTA_PAIR", pair)
    inp = workloads.make_prefill(workloads.PrefillCase(B=2, S=300, Hq=8, Hkv=2, D=128, seed=51))
    d = {k: v.cuda() for k, v in inp.items()}
    out = dbg.prefill(d["q"], d["k"], d["v"], d["lam"])
    _clean(dbg)
    bf16_close(out, ora.prefill(inp["q"], inp["k"], inp["v"], inp["lam"]), f"debug prefill pair={pair}")
    out = dbg.prefill_window(d["q"], d["k"], d["v"], d["lam"], 100)
    _clean(dbg)
    bf16_close(out, ora.prefill(inp["q"], inp["k"], inp["v"], inp["lam"], window=100), f"debug window pair={pair}")
    out, ob, lse = dbg.prefill_train(d["q"], d["k"], d["v"], d["lam"], causal=False)
    _clean(dbg)
    bf16_close(out, ora.prefill(inp["q"], inp["k"], inp["v"], inp["lam"], causal=False), f"debug train pair={pair}")
    # many items per CTA (and per cluster), both item parities
    inp = workloads.make_prefill(workloads.PrefillCase(B=8, S=1024, Hq=32, Hkv=4, D=128, seed=52))
    d = {k: v.cuda() for k, v in inp.items()}
    out = dbg.prefill(d["q"], d["k"], d["v"], d["lam"])
    _clean(dbg)
    rows = [(b, i, p) for b in (0, 7) for i in (0, 127, 128, 1023) for p in (0, 15)]
    got = np.stack([out[b, i, p].double().cpu().numpy() for b, i, p in rows])
    bf16_close(got, ora.prefill_rows(inp["q"], inp["k"], inp["v"], inp["lam"], rows), f"debug many items pair={pair}")


def test_prefill_packed_sequences_in_bounds(dbg):
    lens = [300, 1, 0, 129, 700, 77]
    T = sum(lens)
    g = torch.Generator().manual_seed(T)
    q = torch.randn(T, 8, 128, generator=g).bfloat16()
    k = torch.randn(T, 2, 128, generator=g).bfloat16()
    v = torch.randn(T, 2, 128, generator=g).bfloat16()
    lam = torch.sigmoid(torch.randn(T, 4, generator=g))
    cu = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32)
    out = dbg.prefill_varlen(q.cuda(), k.cuda(), v.cuda(), lam.cuda(), cu.cuda(), max(lens) + 200)
    _clean(dbg)
    bf16_close(out, ora.prefill_varlen(q, k, v, lam, cu.tolist()), "debug packed prefill")
    out = dbg.prefill_varlen_window(q.cuda(), k.cuda(), v.cuda(), lam.cuda(), cu.cuda(), max(lens), 90)
    _clean(dbg)
    bf16_close(out, ora.prefill_varlen(q, k, v, lam, cu.tolist(), window=90), "debug packed window prefill")


@pytest.mark.parametrize("B,Smax,Hq,Hkv,lens", [
    (4, 3000, 16, 2, [3000, 2000, 1, 0]),   # group 8, splits, an empty sequence
    (3, 2500, 64, 4, [2500, 333, 1]),       # group 16: two 8-column MMA tiles
])
def test_decode_in_bounds(dbg, B, Smax, Hq, Hkv, lens):
    inp = workloads.make_decode(workloads.DecodeCase(B=B, Smax=Smax, Hq=Hq, Hkv=Hkv, D=128, len_lo=1, len_hi=Smax,
                                                     seed=53 + Hq))
    inp["seqlens"] = torch.tensor(lens, dtype=torch.int32)
    d = {k: inp[k].cuda() for k in ("q", "kcache", "vcache", "seqlens", "lam")}
    out = dbg.decode(d["q"], d["kcache"], d["vcache"], d["seqlens"], d["lam"])
    _clean(dbg)
    ref = ora.decode(inp["q"], inp["kcache"], inp["vcache"], inp["seqlens"], inp["lam"])
    bf16_close(out, ref, f"debug decode group {Hq // Hkv}")


def test_paged_and_multi_token_decode_in_bounds(dbg):
    B, Hq, Hkv, ps, max_pages = 3, 16, 2, 16, 40
    lens = [640, 17, 0]
    g = torch.Generator().manual_seed(54)
    n_pages = B * max_pages
    kp = torch.randn(n_pages, ps, Hkv, 128, generator=g).bfloat16()
    vp = torch.randn(n_pages, ps, Hkv, 128, generator=g).bfloat16()
    table = torch.randperm(n_pages, generator=g).view(B, max_pages).to(torch.int32)
    q = torch.randn(B, Hq, 128, generator=g).bfloat16()
    lam = torch.sigmoid(torch.randn(B, Hq // 2, generator=g))
    sl = torch.tensor(lens, dtype=torch.int32)
    out = dbg.decode_paged(q.cuda(), kp.cuda(), vp.cuda(), table.cuda(), sl.cuda(), lam.cuda())
    _clean(dbg)
    bf16_close(out, ora.decode_paged(q, kp, vp, table.tolist(), lens, lam), "debug paged decode")
    # two new tokens per sequence over a contiguous cache
    Smax, T = 700, 2
    kc = torch.randn(B, Smax, Hkv, 128, generator=g).bfloat16()
    vc = torch.randn(B, Smax, Hkv, 128, generator=g).bfloat16()
    qm = torch.randn(B, T, Hq, 128, generator=g).bfloat16()
    lm = torch.sigmoid(torch.randn(B, T, Hq // 2, generator=g))
    sl = torch.tensor([700, 2, 300], dtype=torch.int32)
    out = dbg.decode_multi(qm.cuda(), kc.cuda(), vc.cuda(), sl.cuda(), lm.cuda())
    _clean(dbg)
    bf16_close(out, ora.decode_multi(qm, kc, vc, sl.tolist(), lm), "debug multi-token decode")


def test_backward_in_bounds(dbg):
    case = workloads.PrefillCase(B=2, S=300, Hq=8, Hkv=2, D=128, seed=55)
    inp = workloads.make_prefill(case)
    dout = workloads.make_prefill_grad(case)
    d = {k: v.cuda() for k, v in inp.items()}
    out, ob, lse = dbg.prefill_train(d["q"], d["k"], d["v"], d["lam"])
    grads = dbg.backward(d["q"], d["k"], d["v"], d["lam"], ob, lse, dout.cuda())
    _clean(dbg)
    ref = ora.prefill_backward(inp["q"], inp["k"], inp["v"], inp["lam"], dout)
    for gpu, r, name in zip(grads, ref, ("dq", "dk", "dv", "dlam")):
        grad_close(gpu, r, f"debug backward {name}")


def test_backward_packed_window_in_bounds(dbg):
    lens, W, Hq, Hkv = [300, 1, 0, 129], 70, 8, 2
    T = sum(lens)
    case = workloads.PrefillCase(B=1, S=T, Hq=Hq, Hkv=Hkv, D=128, seed=59)
    inp = {k: v[0].contiguous() for k, v in workloads.make_prefill(case).items()}
    dout = workloads.make_prefill_grad(case)[0].contiguous()
    d = {k: v.cuda() for k, v in inp.items()}
    cu = [0] + list(np.cumsum(lens))
    cu_t = torch.tensor(cu, dtype=torch.int32, device="cuda")
    out, ob, lse = dbg.prefill_varlen_train(d["q"], d["k"], d["v"], d["lam"], cu_t, max(lens), window=W)
    grads = dbg.backward_varlen(d["q"], d["k"], d["v"], d["lam"], ob, lse, dout.cuda(), cu_t, max(lens), window=W)
    _clean(dbg)
    ref = ora.prefill_backward_varlen(inp["q"], inp["k"], inp["v"], inp["lam"], dout, cu, window=W)
    for gpu, r, name in zip(grads, ref, ("dq", "dk", "dv", "dlam")):
        grad_close(gpu, r, f"debug packed window backward {name}")


def test_decode_wait_that_expires_reports_and_leaves_the_gpu_usable(dbg):
    """A bounded wait that runs out: the debug build's test hook makes one decode CTA
    announce a ring stage and never copy it. Its consumer warps give up after the wait limit,
    the kernel returns with the decode-wait code in the device error word, and the next call
    on the same context is correct again."""
    import ctypes

    from differential_attention_v2_b200 import _lib

    hook = _lib.LIB.diffattn_v2_test_withhold_decode_stage
    hook.restype = ctypes.c_int
    hook.argtypes = [ctypes.c_int]
    inp = workloads.make_decode(workloads.DecodeCase(B=2, Smax=2000, Hq=16, Hkv=2, D=128, len_lo=2000, len_hi=2000,
                                                     seed=56))
    d = {k: inp[k].cuda() for k in ("q", "kcache", "vcache", "seqlens", "lam")}
    _clean(dbg)
    assert hook(1) == 0  # withhold the first stage of CTA (0, 0, 0)
    try:
        dbg.decode(d["q"], d["kcache"], d["vcache"], d["seqlens"], d["lam"])
        torch.cuda.synchronize()
        assert dbg.device_error() == 2  # a pipeline wait expired in a decode kernel
    finally:
        assert hook(0) == 0
    out = dbg.decode(d["q"], d["kcache"], d["vcache"], d["seqlens"], d["lam"])
    _clean(dbg)
    bf16_close(out, ora.decode(inp["q"], inp["kcache"], inp["vcache"], inp["seqlens"], inp["lam"]),
               "decode after an expired wait")
