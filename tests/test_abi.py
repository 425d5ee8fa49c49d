"""The C-ABI library without a GPU: it loads, exports every declared entry point, and its
host-side argument checks reject bad input before touching CUDA."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "diffattn_v2.h")


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"DA2_API\s+[\w\s\*]+?\b(diffattn_v2_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from differential_attention_v2_b200.build import build

    build()
    import differential_attention_v2_b200 as da

    return da.LIB


def test_header_declares_entry_points():
    names = _declared()
    assert "diffattn_v2_prefill" in names and "diffattn_v2_decode" in names
    assert len(names) >= 9


def test_library_exports_every_declared_symbol(lib):
    import differential_attention_v2_b200 as da

    for name in _declared():
        assert hasattr(lib, name), name
        assert name in da.EXPORTED, f"binding lacks {name}"


def test_bounds_checking_build_exports_every_declared_symbol():
    """The debug-bounds twin of the library (same sources, -DDA2_DEBUG_BOUNDS) loads and
    exports the same entry points."""
    from differential_attention_v2_b200 import _lib
    from differential_attention_v2_b200.build import DEBUG_LIB_PATH, build

    build(debug_bounds=True)
    dbg = _lib.load(DEBUG_LIB_PATH)
    for name in _declared():
        assert hasattr(dbg, name), name
    assert dbg.diffattn_v2_version() == 100


def test_version_and_status_strings(lib):
    assert lib.diffattn_v2_version() == 100
    for code in (0, -1, -2, -3, -4, 7):
        assert lib.diffattn_v2_status_string(code)


# Fake, never dereferenced, 16-byte aligned device addresses: every call below must be
# rejected (or be a no-op) by the host-side checks, before any CUDA call.
P = 1 << 20
Q = P + 4096
K = P + 8192
V = P + 12288
L = P + 16384
O = P + 20480


@pytest.mark.parametrize("args,expect", [
    ((Q, K, V, L, O, 2, 256, 7, 1, 128, 1), -1),        # odd Hq
    ((Q, K, V, L, O, 2, 256, 6, 2, 128, 1), -1),        # a pair would straddle KV heads
    ((Q, K, V, L, O, 2, 256, 8, 0, 128, 1), -1),        # Hkv = 0
    ((Q, K, V, L, O, -1, 256, 8, 2, 128, 1), -1),       # negative B
    ((Q, K, V, L, O, 2, 256, 8, 2, 0, 1), -1),          # D = 0
    ((None, K, V, L, O, 2, 256, 8, 2, 128, 1), -1),     # null q
    ((Q, K, V, None, O, 2, 256, 8, 2, 128, 1), -1),     # null lambda
    ((Q + 2, K, V, L, O, 2, 256, 8, 2, 128, 1), -1),    # misaligned q
    ((Q, K, V, L, O, 2, 256, 8, 2, 128, 2), -1),        # causal flag not 0/1
    ((Q, K, V, L, O, 2, 256, 8, 2, 64, 1), -2),         # bf16 path implements D = 128 only
    ((Q, K, V, L, O, 0, 256, 8, 2, 128, 1), 0),         # B = 0: no-op
    ((Q, K, V, L, O, 2, 0, 8, 2, 128, 1), 0),           # S = 0: no-op
    ((None, None, None, None, None, 0, 0, 8, 2, 128, 1), 0),
])
def test_prefill_host_checks(lib, args, expect):
    assert lib.diffattn_v2_prefill(*args, None) == expect


def test_prefill_window_host_checks(lib):
    assert lib.diffattn_v2_prefill_window(Q, K, V, L, O, 1, 64, 8, 2, 128, 0, None) == -1   # window 0
    assert lib.diffattn_v2_prefill_window(Q, K, V, L, O, 1, 64, 6, 2, 128, 8, None) == -1   # straddling pair
    assert lib.diffattn_v2_prefill_window(Q, K, V, L, O, 1, 64, 8, 2, 64, 8, None) == -2    # D = 64
    assert lib.diffattn_v2_prefill_window(Q, K, V, L, O, 0, 64, 8, 2, 128, 8, None) == 0    # B = 0


def test_prefill_varlen_host_checks(lib):
    C = P + 28672
    assert lib.diffattn_v2_prefill_varlen(Q, K, V, L, O, None, 2, 64, 100, 8, 2, 128, 1, None) == -1  # no cu_seqlens
    assert lib.diffattn_v2_prefill_varlen(Q, K, V, L, O, C, 2, 64, 100, 8, 2, 64, 1, None) == -2      # D = 64
    assert lib.diffattn_v2_prefill_varlen(Q, K, V, L, O, C, 2, 64, 100, 6, 2, 128, 1, None) == -1     # straddling
    assert lib.diffattn_v2_prefill_varlen(Q, K, V, L, O, C, 0, 64, 100, 8, 2, 128, 1, None) == 0      # no sequences
    assert lib.diffattn_v2_prefill_varlen(Q, K, V, L, O, C, 2, 64, 100, 8, 2, 128, 3, None) == -1     # causal flag


def test_prefill_varlen_window_host_checks(lib):
    C = P + 28672
    f = lib.diffattn_v2_prefill_varlen_window
    assert f(Q, K, V, L, O, C, 2, 64, 100, 8, 2, 128, 0, None) == -1       # window 0
    assert f(Q, K, V, L, O, None, 2, 64, 100, 8, 2, 128, 16, None) == -1   # no cu_seqlens
    assert f(Q, K, V, L, O, C, 2, 64, 100, 6, 2, 128, 16, None) == -1      # straddling pair
    assert f(Q, K, V, L, O, C, 2, 64, 100, 8, 2, 64, 16, None) == -2       # D = 64
    assert f(Q, K, V, L, O, C, 0, 64, 100, 8, 2, 128, 16, None) == 0       # no sequences


def test_varlen_window_training_host_checks(lib):
    C, W = P + 28672, P + 32768
    ft = lib.diffattn_v2_prefill_varlen_window_train
    assert ft(Q, K, V, L, O, O, L, C, 2, 64, 100, 8, 2, 128, 0, None) == -1        # window 0
    assert ft(Q, K, V, L, O, O, L, None, 2, 64, 100, 8, 2, 128, 16, None) == -1    # no cu_seqlens
    assert ft(Q, K, V, L, O, O, L, C, 2, 64, 100, 8, 2, 64, 16, None) == -2        # D = 64
    assert ft(Q, K, V, L, O, O, L, C, 0, 64, 100, 8, 2, 128, 16, None) == 0        # no sequences
    fb = lib.diffattn_v2_backward_varlen_window
    args = (Q, K, V, L, O, L, O, Q, K, V, L, C, 2, 64, 100, 8, 2, 128)
    assert fb(*args, 0, W, 1 << 30, None) == -1                                   # window 0
    assert fb(*args, 16, W, 0, None) == -1                                        # workspace too small
    assert fb(Q, K, V, L, O, L, O, Q, K, V, L, C, 2, 64, 100, 8, 2, 64, 16, W, 1 << 30, None) == -2  # D = 64


def test_prefill_f32_host_checks(lib):
    assert lib.diffattn_v2_prefill_f32(Q, K, V, L, O, 1, 16, 4, 1, 96, 1, None) == -2
    assert lib.diffattn_v2_prefill_f32(Q, K, V, L, O, 1, 16, 4, 3, 64, 1, None) == -1
    assert lib.diffattn_v2_prefill_f32(None, K, V, L, O, 1, 16, 4, 1, 64, 1, None) == -1


def test_decode_workspace_size(lib):
    import differential_attention_v2_b200 as da

    assert da.decode_workspace_size(0, 8192, 64, 8, 128) == 0
    assert da.decode_workspace_size(4, 8192, 6, 2, 128) == 0
    ws = da.decode_workspace_size(64, 8192, 64, 8, 128)
    assert ws > 0 and ws % 16 == 0
    # fp32 (m, l, O[D]) per (b, head, split), a multiple of B*Hq*(D+2)*4, then one int32
    # split counter per (b, KV head) padded to 16 bytes
    counters = (64 * 8 * 4 + 15) // 16 * 16
    assert (ws - counters) % (64 * 64 * 130 * 4) == 0
    # grows with Smax (more splits), never with nothing
    assert da.decode_workspace_size(64, 65536, 64, 8, 128) >= ws


def test_decode_window_host_checks(lib):
    W = P + 32768
    f = lib.diffattn_v2_decode_window
    assert f(Q, K, V, L, L, O, 2, 256, 8, 2, 128, 0, W, 1 << 30, None) == -1      # window 0
    assert f(Q, K, V, L, L, O, 2, 256, 8, 2, 128, 16, W, 0, None) == -1           # workspace too small
    assert f(Q, K, V, L, L, O, 2, 256, 8, 2, 64, 16, W, 1 << 30, None) == -2      # D = 64
    assert f(Q, K, V, L, L, O, 0, 256, 8, 2, 128, 16, W, 1 << 30, None) == 0      # B = 0


def test_decode_paged_window_host_checks(lib):
    W, T = P + 32768, P + 36864
    f = lib.diffattn_v2_decode_paged_window
    assert f(Q, K, V, T, L, L, O, 2, 8, 64, 16, 8, 2, 128, 0, W, 1 << 30, None) == -1      # window 0
    assert f(Q, K, V, T, L, L, O, 2, 8, 12, 16, 8, 2, 128, 16, W, 1 << 30, None) == -1     # page size not 2^k
    assert f(Q, K, V, T, L, L, O, 2, 8, 64, 16, 8, 2, 64, 16, W, 1 << 30, None) == -2      # D = 64
    assert f(Q, K, V, T, L, L, O, 0, 8, 64, 16, 8, 2, 128, 16, W, 1 << 30, None) == 0      # B = 0


def test_decode_host_checks(lib):
    ws = lib.diffattn_v2_decode_workspace_size(2, 1024, 16, 2, 128)
    S = P + 24576
    W = P + 65536
    args = (Q, K, V, S, L, O, 2, 1024, 16, 2, 128, W, ws, None)
    bad_ws = args[:12] + (ws - 16,) + args[13:]
    assert lib.diffattn_v2_decode(*bad_ws) == -1                       # workspace too small
    no_ws = args[:11] + (None,) + args[12:]
    assert lib.diffattn_v2_decode(*no_ws) == -1                        # null workspace
    odd = (Q, K, V, S, L, O, 2, 1024, 10, 1, 128, W, ws, None)
    assert lib.diffattn_v2_decode(*odd) == -2                          # group size 10
    d64 = (Q, K, V, S, L, O, 2, 1024, 16, 2, 64, W, 1 << 30, None)
    assert lib.diffattn_v2_decode(*d64) == -2
    b0 = (None, None, None, None, None, None, 0, 1024, 16, 2, 128, None, 0, None)
    assert lib.diffattn_v2_decode(*b0) == 0
    assert lib.diffattn_v2_decode(Q, K, V, S, L, O, 2, 0, 16, 2, 128, W, ws, None) == -1
    assert lib.diffattn_v2_decode_f32(Q, K, V, S, L, O, 2, 1024, 16, 3, 64, None) == -1


def test_decode_paged_host_checks(lib):
    T = P + 32768
    W = P + 65536
    S_ = P + 24576
    ws = lib.diffattn_v2_decode_workspace_size(2, 1024, 16, 2, 128)
    ok = (Q, K, V, T, S_, L, O, 2, 16, 64, 40, 16, 2, 128, W, ws, None)
    bad_ps = ok[:9] + (48,) + ok[10:]
    assert lib.diffattn_v2_decode_paged(*bad_ps) == -1                  # page size not a power of two
    small = ok[:9] + (4,) + ok[10:]
    assert lib.diffattn_v2_decode_paged(*small) == -1                   # page size below 8
    no_table = ok[:3] + (None,) + ok[4:]
    assert lib.diffattn_v2_decode_paged(*no_table) == -1
    short_ws = ok[:15] + (ws - 16,) + ok[16:]
    assert lib.diffattn_v2_decode_paged(*short_ws) == -1
    d64 = ok[:13] + (64,) + ok[14:]
    assert lib.diffattn_v2_decode_paged(*d64[:15] + (1 << 30,) + d64[16:]) == -2


def test_decode_multi_host_checks(lib):
    W = P + 65536
    S_ = P + 24576
    ws = lib.diffattn_v2_decode_multi_workspace_size(2, 2, 1024, 16, 2, 128)
    assert ws >= lib.diffattn_v2_decode_workspace_size(2, 1024, 16, 2, 128)
    assert lib.diffattn_v2_decode_multi(Q, K, V, S_, L, O, 2, 4, 1024, 16, 2, 128, W, 1 << 30, None) == -2  # T*G > 16
    assert lib.diffattn_v2_decode_multi(Q, K, V, S_, L, O, 2, 0, 1024, 16, 2, 128, W, ws, None) == -1       # T = 0
    assert lib.diffattn_v2_decode_multi(Q, K, V, S_, L, O, 2, 2, 1024, 16, 2, 128, W, ws - 16, None) == -1  # workspace


def test_lambda_v2_host_checks(lib):
    assert lib.diffattn_v2_lambda_v2(Q, K, None, 10, 100, 32, O, None) == -2   # d_model % 64
    assert lib.diffattn_v2_lambda_v2(Q, K, None, 10, 128, 20, O, None) == -2   # n_pairs % 8
    assert lib.diffattn_v2_lambda_v2(Q, K, None, 10, 128, 72, O, None) == -2   # n_pairs > 64
    assert lib.diffattn_v2_lambda_v2(None, K, None, 10, 128, 32, O, None) == -1
    assert lib.diffattn_v2_lambda_v2(Q, K, None, 0, 128, 32, O, None) == 0


def test_prefill_fused_lambda_host_checks(lib):
    X, W = P + 24576, P + 28672
    f = lib.diffattn_v2_prefill_fused_lambda
    assert f(Q, K, V, X, W, None, O, None, 1, 64, 8, 2, 128, 100, 1, None) == -1       # d_model % 8
    assert f(Q, K, V, X, W, None, O, None, 1, 64, 8, 2, 128, 0, 1, None) == -1         # d_model = 0
    assert f(Q, K, V, None, W, None, O, None, 1, 64, 8, 2, 128, 256, 1, None) == -1    # null x
    assert f(Q, K, V, X, None, None, O, None, 1, 64, 8, 2, 128, 256, 1, None) == -1    # null w_lambda_t
    assert f(Q, K, V, X, W, L + 4, O, None, 1, 64, 8, 2, 128, 256, 1, None) == -1      # misaligned bias
    assert f(Q, K, V, X, W, None, O, L + 8, 1, 64, 8, 2, 128, 256, 1, None) == -1      # misaligned lambda_out
    assert f(Q, K, V, X, W, None, O, None, 1, 64, 6, 2, 128, 256, 1, None) == -1       # straddling pair
    assert f(Q, K, V, X, W, None, O, None, 1, 64, 8, 2, 64, 256, 1, None) == -2        # D = 64
    assert f(Q, K, V, X, W, None, O, None, 1, 64, 8, 2, 128, 256, 2, None) == -1       # causal flag
    assert f(Q, K, V, X, W, None, O, None, 0, 64, 8, 2, 128, 256, 1, None) == 0        # B = 0


def test_lambda_v1_host_checks(lib):
    assert lib.diffattn_v2_lambda_v1(Q, K, V, L, 0.8, 0, 128, 1, O, None) == -1
    assert lib.diffattn_v2_lambda_v1(Q, K, V, L, 0.8, 4, 0, 1, O, None) == -1
    assert lib.diffattn_v2_lambda_v1(Q, K, V, L, 0.8, 4, 128, 0, O, None) == 0
    assert lib.diffattn_v2_lambda_v1(None, K, V, L, 0.8, 4, 128, 1, O, None) == -1


def test_package_exposes_every_binding_name(lib):
    """Each wrapper of the binding module is reachable from the package namespace."""
    import differential_attention_v2_b200 as da
    from differential_attention_v2_b200 import _lib

    public = [n for n in dir(_lib) if not n.startswith("_") and callable(getattr(_lib, n))
              and getattr(getattr(_lib, n), "__module__", "") == _lib.__name__ and n != "DiffAttnError"]
    for name in public:
        assert getattr(da, name) is getattr(_lib, name), name


def test_prefill_train_host_checks(lib):
    OB, LS = P + 32768, P + 40960
    assert lib.diffattn_v2_prefill_train(Q, K, V, L, O, OB, LS, 2, 256, 7, 1, 128, 1, None) == -1  # odd Hq
    assert lib.diffattn_v2_prefill_train(Q, K, V, L, O, None, LS, 2, 256, 8, 1, 128, 1, None) == -1  # no o_branch
    assert lib.diffattn_v2_prefill_train(Q, K, V, L, O, OB, LS + 4, 2, 256, 8, 1, 128, 1, None) == -1  # unaligned
    assert lib.diffattn_v2_prefill_train(Q, K, V, L, O, OB, LS, 2, 256, 8, 1, 64, 1, None) == -2  # D = 64
    assert lib.diffattn_v2_prefill_train(Q, K, V, L, O, OB, LS, 0, 256, 8, 1, 128, 1, None) == 0   # empty


def test_backward_host_checks(lib):
    OB, LS, DO, DQ, DK, DV, DL, W = (P + 32768 * i for i in range(1, 9))
    ws = lib.diffattn_v2_backward_workspace_size(2, 256, 8)
    assert ws == 2 * (8 // 2) * 256 * 20                   # five fp32 row terms per (b, pair, row)
    assert lib.diffattn_v2_backward_workspace_size(1, 300, 8) == 4 * 384 * 20  # rows padded to 128
    assert lib.diffattn_v2_backward_workspace_size(0, 256, 8) == 0
    ok = (Q, K, V, L, OB, LS, DO, DQ, DK, DV, DL, 2, 256, 8, 2, 128, 1, W, ws, None)
    assert lib.diffattn_v2_backward(*ok[:18], ws - 4, None) == -1                  # short workspace
    assert lib.diffattn_v2_backward(*ok[:6], None, *ok[7:]) == -1                  # no dout
    assert lib.diffattn_v2_backward(*ok[:9], DV + 8, *ok[10:]) == -1               # unaligned dv
    assert lib.diffattn_v2_backward(*ok[:13], 6, *ok[14:]) == -1                   # pair straddles KV heads
    assert lib.diffattn_v2_backward(*ok[:16], 2, *ok[17:]) == -1                   # causal not 0/1
    assert lib.diffattn_v2_backward(*ok[:15], 64, *ok[16:]) == -2                  # D = 64
    assert lib.diffattn_v2_backward(*ok[:11], 0, *ok[12:]) == 0                    # B = 0


def test_varlen_training_host_checks(lib):
    OB, LS, CU = P + 32768, P + 40960, P + 49152
    args = (Q, K, V, L, O, OB, LS, CU, 2, 256, 300, 8, 2, 128, 1, None)
    assert lib.diffattn_v2_prefill_varlen_train(*args[:7], None, *args[8:]) == -1   # no cu_seqlens
    assert lib.diffattn_v2_prefill_varlen_train(*args[:11], 6, *args[12:]) == -1    # pair straddles KV heads
    assert lib.diffattn_v2_prefill_varlen_train(*args[:13], 64, *args[14:]) == -2   # D = 64
    assert lib.diffattn_v2_prefill_varlen_train(*args[:8], 0, *args[9:]) == 0       # no sequences
    ws = lib.diffattn_v2_backward_varlen_workspace_size(3, 500, 8)
    assert ws >= 4 * (500 + 3 * 128) * 20                                            # padded row terms
    assert lib.diffattn_v2_backward_varlen_workspace_size(0, 500, 8) == 0
    DO, DQ, DK, DV, DL, W = (P + 65536 + 32768 * i for i in range(6))
    ok = (Q, K, V, L, OB, LS, DO, DQ, DK, DV, DL, CU, 3, 256, 500, 8, 2, 128, 1, W, ws, None)
    assert lib.diffattn_v2_backward_varlen(*ok[:20], ws - 16, None) == -1            # short workspace
    assert lib.diffattn_v2_backward_varlen(*ok[:11], None, *ok[12:]) == -1           # no cu_seqlens
    assert lib.diffattn_v2_backward_varlen(*ok[:18], 2, *ok[19:]) == -1              # causal not 0/1
    assert lib.diffattn_v2_backward_varlen(*ok[:17], 64, *ok[18:]) == -2             # D = 64
    assert lib.diffattn_v2_backward_varlen(*ok[:12], 0, *ok[13:]) == 0               # B = 0


def test_window_training_host_checks(lib):
    OB, LS, DO, DQ, DK, DV, DL, W = (P + 32768 * i for i in range(1, 9))
    assert lib.diffattn_v2_prefill_window_train(Q, K, V, L, O, OB, LS, 2, 256, 8, 2, 128, 0, None) == -1  # window < 1
    assert lib.diffattn_v2_prefill_window_train(Q, K, V, L, O, OB, LS, 2, 256, 8, 2, 64, 64, None) == -2  # D = 64
    assert lib.diffattn_v2_prefill_window_train(Q, K, V, L, O, OB, LS, 0, 256, 8, 2, 128, 64, None) == 0   # empty
    ws = lib.diffattn_v2_backward_workspace_size(2, 256, 8)
    ok = (Q, K, V, L, OB, LS, DO, DQ, DK, DV, DL, 2, 256, 8, 2, 128, 64, W, ws, None)
    assert lib.diffattn_v2_backward_window(*ok[:16], 0, *ok[17:]) == -1           # window < 1
    assert lib.diffattn_v2_backward_window(*ok[:18], ws - 4, None) == -1          # short workspace
    assert lib.diffattn_v2_backward_window(*ok[:15], 64, *ok[16:]) == -2          # D = 64
