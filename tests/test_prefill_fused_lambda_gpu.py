"""The prefill with the V2 lambda computed inside the kernel against the float64 oracle.

lambda[t, p] = sigmoid(x[t] . w[:, p] + bias[p]) ("Differential Transformer V2 soll
KI-Training stabiler machen", "Weniger Ausreisser und Gradientenspitzen") feeds the operator
of the "Differential Attention (V2)" lesson; the oracle composes its projection and its
prefill. The kernel's lambda copy is held to the projection's own 1e-5 bound, the output to
the bf16 contract, and both are compared with the two-launch path (projection, then prefill).
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


@pytest.mark.parametrize("B,S,Hq,Hkv,d_model,with_bias,causal", [
    (2, 300, 8, 2, 256, True, True),      # ragged last tile, lanes all full
    (1, 129, 16, 2, 200, False, True),    # d_model not a multiple of 256: partly idle lanes
    (1, 640, 32, 4, 1024, True, True),    # several tiles and items per CTA
    (2, 200, 4, 2, 512, True, False),     # full attention
    (1, 1, 2, 1, 64, False, True),        # a single token
])
def test_fused_lambda_matches_oracle(da, B, S, Hq, Hkv, d_model, with_bias, causal):
    inp = workloads.make_prefill(workloads.PrefillCase(B=B, S=S, Hq=Hq, Hkv=Hkv, D=128, seed=1200 + S + d_model))
    g = torch.Generator().manual_seed(1300 + d_model)
    x = torch.randn(B, S, d_model, generator=g).bfloat16()
    w = (torch.randn(d_model, Hq // 2, generator=g) / d_model ** 0.5).bfloat16()
    bias = torch.randn(Hq // 2, generator=g) if with_bias else None
    wt = w.t().contiguous()

    d = {k: v.cuda() for k, v in inp.items()}
    lam_out = torch.full((B, S, Hq // 2), -1.0, device="cuda")
    out = da.prefill_fused_lambda(d["q"], d["k"], d["v"], x.cuda(), wt.cuda(),
                                  None if bias is None else bias.cuda(), lambda_out=lam_out, causal=causal)
    assert da.device_error() == 0

    lam_ref = ora.lambda_v2_projection(x.reshape(B * S, d_model), w, bias).reshape(B, S, Hq // 2)
    np.testing.assert_allclose(lam_out.cpu().double().numpy(), lam_ref, rtol=0, atol=1e-5)
    ref = ora.prefill(inp["q"], inp["k"], inp["v"], torch.from_numpy(lam_ref).float(), causal=causal)
    bf16_close(out, ref, f"fused lambda B={B} S={S} Hq={Hq} d_model={d_model} causal={causal}")

    # the two-launch path: lambda_v2 (tensor cores) then prefill; lambda differs by rounding only
    if d_model % 64 == 0 and (Hq // 2) % 8 == 0:
        lam2 = da.lambda_v2(x.reshape(B * S, d_model).cuda(), w.cuda(), None if bias is None else bias.cuda())
        assert float((lam2.reshape(B, S, Hq // 2) - lam_out).abs().max()) < 2e-6
        out2 = da.prefill(d["q"], d["k"], d["v"], lam2.reshape(B, S, Hq // 2), causal=causal)
        bf16_close(out2, ref, "two-launch path")


def test_fused_lambda_without_copy_equals_with_copy(da):
    B, S, Hq, Hkv, d_model = 1, 256, 8, 2, 512
    inp = workloads.make_prefill(workloads.PrefillCase(B=B, S=S, Hq=Hq, Hkv=Hkv, D=128, seed=1400))
    g = torch.Generator().manual_seed(1401)
    x = torch.randn(B, S, d_model, generator=g).bfloat16().cuda()
    wt = (torch.randn(Hq // 2, d_model, generator=g) / d_model ** 0.5).bfloat16().cuda()
    d = {k: v.cuda() for k, v in inp.items()}
    lam = torch.empty(B, S, Hq // 2, device="cuda")
    a = da.prefill_fused_lambda(d["q"], d["k"], d["v"], x, wt, lambda_out=lam)
    b = da.prefill_fused_lambda(d["q"], d["k"], d["v"], x, wt)
    assert da.device_error() == 0
    assert torch.equal(a, b)
    # and equal, bit for bit, to the plain prefill fed the same lambda
    assert torch.equal(a, da.prefill(d["q"], d["k"], d["v"], lam))
