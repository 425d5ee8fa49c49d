"""Seeded synthetic inputs for the Differential Attention V2 forward operator.

This module only draws random numbers and arranges them into the shapes the operator
consumes. It holds none of the operator's arithmetic (no softmax, no scores, no lambda
formula), so both the float64 oracle and the CUDA path can take their inputs from here
without sharing any of the method.

Shapes and distributions follow the long-context workloads the pages motivate
("Differential Attention (V2)" lesson, section "When to reach for it", workload table:
long-context RAG 64k+, needle-in-haystack past 32k). No benchmark items are reproduced;
the named public suites are stood in for by these synthetic tensors.

Layout ("BSHD", row-major, contiguous):
  prefill  q [B,S,Hq,D], k/v [B,S,Hkv,D], lam fp32 [B,S,Hq/2]
  decode   q [B,Hq,D], kcache/vcache [B,Smax,Hkv,D], seqlens int32 [B], lam fp32 [B,Hq/2]
Every generator uses a torch CPU generator seeded per config, so results are identical
on every host.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

__all__ = [
    "CONFIGS",
    "PrefillCase",
    "DecodeCase",
    "make_prefill",
    "make_decode",
    "plant_signal_row",
    "plant_needles",
    "v1_lambda_params",
    "config_case",
]


@dataclass(frozen=True)
class PrefillCase:
    B: int
    S: int
    Hq: int
    Hkv: int
    D: int
    dtype: str = "bf16"  # "bf16" or "f32"
    causal: bool = True
    seed: int = 0


@dataclass(frozen=True)
class DecodeCase:
    B: int
    Smax: int
    Hq: int
    Hkv: int
    D: int
    len_lo: int
    len_hi: int
    dtype: str = "bf16"
    seed: int = 0
    needle: bool = False
    lambda_kind: str = "v2"  # "v2": sigmoid(N(0,1)); "v1": exp(a.b) - exp(c.e) + 0.8 params


# The five workloads of the operator's scope, with their seeds (1000 + index).
CONFIGS = {
    # tiny fp32 causal prefill, with the planted signal-plus-noise row in pair 0
    "tiny_fp32_prefill_b1_s128": PrefillCase(B=1, S=128, Hq=4, Hkv=1, D=64, dtype="f32", seed=1000),
    # bf16 causal prefill at 4 x 4k
    "prefill_b4_s4096": PrefillCase(B=4, S=4096, Hq=64, Hkv=8, D=128, seed=1001),
    # long-context bf16 causal prefill at 32k
    "prefill_b1_s32768": PrefillCase(B=1, S=32768, Hq=64, Hkv=8, D=128, seed=1002),
    # bf16 decode, one new token per sequence, lengths uniform in [1024, 8192]
    "decode_b64_s8192": DecodeCase(B=64, Smax=8192, Hq=64, Hkv=8, D=128, len_lo=1024, len_hi=8192,
                                 seed=1003),
    # long-context decode with one planted needle key per sequence and V1-style lambda
    "needle_decode_b8_s131072": DecodeCase(B=8, Smax=131072, Hq=64, Hkv=8, D=128, len_lo=131072,
                                   len_hi=131072, seed=1004, needle=True, lambda_kind="v1"),
}

_DT = {"bf16": torch.bfloat16, "f32": torch.float32}


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def _randn(shape, gen, dtype, chunk_elems=1 << 26):
    """N(0,1) samples drawn in fp32 and rounded once to `dtype`, in bounded chunks."""
    n = 1
    for s in shape:
        n *= int(s)
    out = torch.empty(n, dtype=dtype)
    for lo in range(0, n, chunk_elems):
        hi = min(n, lo + chunk_elems)
        out[lo:hi] = torch.randn(hi - lo, generator=gen, dtype=torch.float32).to(dtype)
    return out.view(*shape)


def _sigmoid_normal(shape, gen):
    """lambda input values of the V2 kind: a sigmoid-bounded draw in (0, 1), fp32."""
    return torch.sigmoid(torch.randn(*shape, generator=gen, dtype=torch.float32))


def make_prefill(case: PrefillCase):
    """Return dict(q, k, v, lam) as CPU tensors for a prefill case."""
    if case.Hq % 2 or case.Hq % (2 * case.Hkv):
        raise ValueError("Hq must be even and a multiple of 2*Hkv")
    gen = _gen(case.seed)
    dt = _DT[case.dtype]
    q = _randn((case.B, case.S, case.Hq, case.D), gen, dt)
    k = _randn((case.B, case.S, case.Hkv, case.D), gen, dt)
    v = _randn((case.B, case.S, case.Hkv, case.D), gen, dt)
    lam = _sigmoid_normal((case.B, case.S, case.Hq // 2), gen)
    return {"q": q, "k": k, "v": v, "lam": lam}


def make_prefill_grad(case: PrefillCase):
    """Upstream gradient dL/d(out) for a prefill case: standard normal, shape [B,S,Hq/2,D],
    in the case's dtype, from its own seeded stream (seed + 7919)."""
    gen = _gen(case.seed + 7919)
    return _randn((case.B, case.S, case.Hq // 2, case.D), gen, _DT[case.dtype])


def plant_signal_row(inp, b=0, row=None, pair=0, signal_key=7, logit_gain=4.0, seed=77):
    """Plant the signal-plus-shared-noise query row of the lesson's noise-cancellation toy.

    Follows "Differential Attention (V2)" lesson, section "Build it", Step 4: one known
    signal position, the rest noise. Query row `row` of pair `pair` is rewritten so that
    branch 2 holds a noise vector n ~ N(0,1)^D and branch 1 holds
    n + logit_gain * sqrt(D) * k_s / |k_s|^2, where k_s is key `signal_key` of the pair's
    K/V head. Both branches then share the noise logits n.k_j / sqrt(D); at the signal key
    branch 1's logit is larger by exactly `logit_gain`, elsewhere by a small amount that
    depends on how far k_j is from orthogonal to k_s. Keys and values are left as they are.
    Modifies `inp` in place and returns (row, signal_key).
    """
    q, k = inp["q"], inp["k"]
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    h1, h2 = 2 * pair, 2 * pair + 1
    g = h1 // G
    if row is None:
        row = S - 1
    gen = _gen(seed)
    key = k[b, signal_key, g].to(torch.float64)
    n = torch.randn(D, generator=gen, dtype=torch.float32).to(torch.float64)
    q[b, row, h1] = (n + logit_gain * math.sqrt(D) * key / key.dot(key)).to(q.dtype)
    q[b, row, h2] = n.to(q.dtype)
    return row, signal_key


def v1_lambda_params(n_pairs: int, D: int, gen: torch.Generator, std=0.1):
    """The four V1 re-parameterisation vectors per pair, each ~ N(0, std^2), fp32 [n_pairs, D]."""
    return {
        name: (torch.randn(n_pairs, D, generator=gen, dtype=torch.float32) * std)
        for name in ("lq1", "lk1", "lq2", "lk2")
    }


def plant_needles(inp, gen):
    """Set one key per sequence (same position for every KV head) to a needle.

    For KV head g the needle key is 4 * q1/|q1| * sqrt(D), where q1 is the query of the
    first head of the first pair in g's GQA group. Returns the positions (int64 [B]).
    """
    q, kc, seqlens = inp["q"], inp["kcache"], inp["seqlens"]
    B, Hq, D = q.shape
    Hkv = kc.shape[2]
    G = Hq // Hkv
    pos = torch.empty(B, dtype=torch.int64)
    for b in range(B):
        n = int(seqlens[b])
        pos[b] = int(torch.randint(0, n, (1,), generator=gen))
        for g in range(Hkv):
            h = g * G  # first head of the first pair in group g
            q1 = q[b, h].to(torch.float64)
            kc[b, pos[b], g] = (4.0 * q1 / q1.norm() * math.sqrt(D)).to(kc.dtype)
    return pos


def make_decode(case: DecodeCase):
    """Return dict(q, kcache, vcache, seqlens, lam[, v1 params, needle_pos]) as CPU tensors."""
    if case.Hq % 2 or case.Hq % (2 * case.Hkv):
        raise ValueError("Hq must be even and a multiple of 2*Hkv")
    gen = _gen(case.seed)
    dt = _DT[case.dtype]
    seqlens = torch.randint(case.len_lo, case.len_hi + 1, (case.B,), generator=gen,
                            dtype=torch.int64).to(torch.int32)
    q = _randn((case.B, case.Hq, case.D), gen, dt)
    kc = _randn((case.B, case.Smax, case.Hkv, case.D), gen, dt)
    vc = _randn((case.B, case.Smax, case.Hkv, case.D), gen, dt)
    out = {"q": q, "kcache": kc, "vcache": vc, "seqlens": seqlens}
    if case.lambda_kind == "v1":
        out.update(v1_lambda_params(case.Hq // 2, case.D, gen))
        out["lambda_init"] = 0.8
        out["lam"] = None  # produced by the operator's V1 lambda step
    else:
        out["lam"] = _sigmoid_normal((case.B, case.Hq // 2), gen)
    if case.needle:
        out["needle_pos"] = plant_needles(out, gen)
    return out


def config_case(name: str):
    return CONFIGS[name]


def prefill_flops(B, S, Hq, D, causal=True):
    """Algorithmic FLOPs of one forward prefill: 2 GEMMs (QK^T, PV) x 2 flop per MAC for every
    (query head, visible key) pair: 4*D per visible (query, key) pair and head."""
    visible = S * (S + 1) // 2 if causal else S * S
    return 4 * D * Hq * B * visible


def decode_bytes(seqlens, Hkv, D, Hq, elem=2):
    """Bytes a decode step must move: every visible K and V row once, plus q, lambda and out."""
    kv = int(sum(int(x) for x in seqlens)) * Hkv * D * 2 * elem
    B = len(seqlens)
    return kv + B * Hq * D * elem + B * (Hq // 2) * 4 + B * (Hq // 2) * D * elem
