"""The prefill writes no output row past the last valid one.

The epilogue stages each warp's 32 rows x 32 columns of out in shared memory and writes them
with one tensor store. A [B,S] launch relies on the tensor map's extent to drop rows past S;
with packed sequences a warp whose 32 rows reach past its sequence's end stores its valid rows
itself, and those per-thread stores (and the training forward's per-head outputs) are 256-bit
where the row is 32-byte aligned, 128-bit otherwise. Each case places the output inside a
larger buffer filled with a sentinel, at a 32-byte aligned offset and at one that is only
16-byte aligned, with lengths whose last row tile ends inside a 32-row slab: the rows past
the end must keep the sentinel and the valid rows must match the float64 oracle.
"""
import numpy as np
import pytest
import torch

import workloads
from oracle import diffattn_f64 as ora
from tests.parity import bf16_close

pytestmark = pytest.mark.gpu

SENTINEL = 7.0
PAD_ROWS = 40


@pytest.fixture(scope="module")
def da():
    import differential_attention_v2_b200 as m

    assert torch.cuda.is_available()
    return m


def _padded(n_rows, row_shape, offset_elems):
    """A contiguous [n_rows, *row_shape] bf16 view inside a sentinel-filled buffer that holds
    PAD_ROWS more rows, starting offset_elems elements into it."""
    row = int(np.prod(row_shape))
    big = torch.full((offset_elems + (n_rows + PAD_ROWS) * row,), SENTINEL, dtype=torch.bfloat16, device="cuda")
    view = big[offset_elems:offset_elems + n_rows * row].view(n_rows, *row_shape)
    tail = big[offset_elems + n_rows * row:]
    return view, tail


@pytest.mark.parametrize("offset", [0, 8], ids=["aligned32", "aligned16"])
@pytest.mark.parametrize("S", [1, 33, 300, 1000])
def test_dense_rows_past_s_untouched(da, S, offset):
    Hq, Hkv, D = 4, 2, 128
    inp = workloads.make_prefill(workloads.PrefillCase(B=1, S=S, Hq=Hq, Hkv=Hkv, D=D, seed=900 + S))
    d = {k: v.cuda() for k, v in inp.items()}
    out, tail = _padded(S, (Hq // 2, D), offset)
    da.prefill(d["q"], d["k"], d["v"], d["lam"], out=out.view(1, S, Hq // 2, D))
    assert da.device_error() == 0
    assert torch.all(tail == SENTINEL), "rows past S were written"
    bf16_close(out.view(1, S, Hq // 2, D), ora.prefill(inp["q"], inp["k"], inp["v"], inp["lam"]), f"dense S={S}")


@pytest.mark.parametrize("offset", [0, 8], ids=["aligned32", "aligned16"])
@pytest.mark.parametrize("lens", [[130, 45], [31], [1], [97, 200, 33]])
def test_packed_rows_past_end_untouched(da, lens, offset):
    Hq, Hkv, D = 8, 2, 128
    T = sum(lens)
    g = torch.Generator().manual_seed(910 + T)
    q = torch.randn(T, Hq, D, generator=g).bfloat16()
    k = torch.randn(T, Hkv, D, generator=g).bfloat16()
    v = torch.randn(T, Hkv, D, generator=g).bfloat16()
    lam = torch.sigmoid(torch.randn(T, Hq // 2, generator=g))
    cu = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32)
    out, tail = _padded(T, (Hq // 2, D), offset)
    da.prefill_varlen(q.cuda(), k.cuda(), v.cuda(), lam.cuda(), cu.cuda(), max(lens), out=out)
    assert da.device_error() == 0
    assert torch.all(tail == SENTINEL), "rows past the last sequence were written"
    bf16_close(out, ora.prefill_varlen(q, k, v, lam, cu.tolist()), f"packed {lens}")


@pytest.mark.parametrize("offset", [0, 8], ids=["aligned32", "aligned16"])
def test_training_outputs_rows_past_s_untouched(da, offset):
    B, S, Hq, Hkv, D = 1, 161, 4, 2, 128
    inp = workloads.make_prefill(workloads.PrefillCase(B=B, S=S, Hq=Hq, Hkv=Hkv, D=D, seed=930))
    d = {k: v.cuda() for k, v in inp.items()}
    out, out_tail = _padded(S, (Hq // 2, D), offset)
    ob, ob_tail = _padded(S, (Hq, D), offset)
    out4, ob4 = out.view(B, S, Hq // 2, D), ob.view(B, S, Hq, D)
    _, ob_ret, lse = da.prefill_train(d["q"], d["k"], d["v"], d["lam"], out=out4, o_branch=ob4)
    assert da.device_error() == 0
    assert torch.all(out_tail == SENTINEL) and torch.all(ob_tail == SENTINEL), "rows past S were written"
    bf16_close(out4, ora.prefill(inp["q"], inp["k"], inp["v"], inp["lam"]), "training forward out")
    # per-head normalised outputs O_h = A_h V and the base-2 row log-sum-exp
    ref_ob, ref_lse = ora.prefill_branches(inp["q"], inp["k"], inp["v"])
    bf16_close(ob_ret, ref_ob, "training forward per-head outputs")
    assert np.abs(lse.cpu().double().numpy() - ref_lse).max() < 1e-3
