"""The no-allocation decode entry point against the regular decode entry point and the oracle.

diffattn_v2_decode_noalloc serves callers that cannot allocate device memory (a KV-cache
pool or caching allocator that owns nearly all HBM, plugin interfaces without a workspace):
its split partials live in the library's fixed 16 MiB device array. Here it is called
through the C ABI on three inputs in a row (GQA groups of 4, 8 and 16; the group of 16 runs
the kernel form with two 8-column MMA tiles), and each output is compared with
diffattn_v2_decode (caller-provided workspace) and with the float64 oracle, within the bf16
tolerance of the other tests. Each call reuses the array the previous one left behind. This
file is named so that pytest collects it last.
"""
import ctypes

import pytest
import torch

import workloads
from oracle import diffattn_f64 as ora
from tests.parity import bf16_close

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 16 << 20


@pytest.fixture(scope="module")
def da():
    import differential_attention_v2_b200 as m

    assert torch.cuda.is_available()
    return m


def _inputs(B, Smax, Hq, Hkv, lens, seed):
    """CPU inputs of one decode step (the oracle reads these; the calls get device copies)."""
    inp = workloads.make_decode(workloads.DecodeCase(B=B, Smax=Smax, Hq=Hq, Hkv=Hkv, D=128, len_lo=1, len_hi=Smax,
                                                     seed=seed))
    inp["seqlens"] = torch.tensor(lens, dtype=torch.int32)
    return {k: v for k, v in inp.items() if k in ("q", "kcache", "vcache", "seqlens", "lam")}


def _noalloc(da, d, out):
    B, Hq, D = d["q"].shape
    Smax, Hkv = d["kcache"].shape[1], d["kcache"].shape[2]
    stream = torch.cuda.current_stream().cuda_stream
    return da.LIB.diffattn_v2_decode_noalloc(d["q"].data_ptr(), d["kcache"].data_ptr(), d["vcache"].data_ptr(),
                                             d["seqlens"].data_ptr(), d["lam"].data_ptr(), out.data_ptr(), B, Smax,
                                             Hq, Hkv, D, ctypes.c_void_p(stream))


def test_noalloc_decode_matches_decode_and_oracle_on_three_calls(da):
    cases = [
        _inputs(4, 3000, 16, 2, [3000, 2000, 1, 0], seed=41),           # group 8, several splits, an empty sequence
        _inputs(8, 6000, 64, 8, [6000, 17, 4096, 1, 5999, 64, 65, 3000], seed=42),
        _inputs(3, 5000, 64, 4, [5000, 333, 4097], seed=43),            # group 16: two 8-column MMA tiles
        _inputs(5, 2500, 8, 2, [2500, 1, 1200, 0, 64], seed=44),         # group 4
    ]
    for n, h in enumerate(cases):
        d = {k: v.cuda() for k, v in h.items()}
        need = da.decode_workspace_size(d["q"].shape[0], d["kcache"].shape[1], d["q"].shape[1], d["kcache"].shape[2],
                                        128)
        assert 0 < need <= SCRATCH_BYTES
        ref = da.decode(d["q"], d["kcache"], d["vcache"], d["seqlens"], d["lam"])
        out = torch.full_like(ref, float("nan"))
        assert _noalloc(da, d, out) == 0
        torch.cuda.synchronize()
        assert da.device_error() == 0
        bf16_close(out, ref.double().cpu().numpy(), f"no-alloc decode vs decode, call {n + 1}")
        oracle = ora.decode(h["q"], h["kcache"], h["vcache"], h["seqlens"], h["lam"])
        bf16_close(out, oracle, f"no-alloc decode vs oracle, call {n + 1}")


def test_noalloc_decode_refuses_sizes_beyond_the_array(da):
    # 64 sequences x 64 heads at 128k context need about 68 MB of partials
    B, Smax, Hq, Hkv = 64, 131072, 64, 8
    assert da.decode_workspace_size(B, Smax, Hq, Hkv, 128) > SCRATCH_BYTES
    base = 1 << 20  # aligned placeholders: the call must refuse before touching them
    st = da.LIB.diffattn_v2_decode_noalloc(base, base, base, base, base, base, B, Smax, Hq, Hkv, 128, None)
    assert st == -2
