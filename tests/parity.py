"""Helpers for the GPU parity tests: tolerances and comparisons against the oracle.

Every comparison records the error it measured (max-abs, relative Frobenius, the bound it
was held to): printed as a `[parity]` line (shown with `pytest -s`), and appended as one JSON
line to the file named by DA2_PARITY_LOG when that variable is set, so that a GPU run leaves
the achieved margins of every test behind.
"""
import json
import os

import numpy as np
import torch


def _record(kind, what, **vals):
    test = os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0]
    line = {"kind": kind, "what": what, "test": test, **vals}
    print(f"[parity] {kind} {what}: " + " ".join(f"{k}={v:.3e}" for k, v in vals.items()))
    path = os.environ.get("DA2_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(line) + "\n")

# Tolerances of the operator's contract: fp32 paths max-abs 1e-5; bf16 paths max-abs 2e-2
# and relative Frobenius 5e-3 (output rounded once to bf16 from an fp32 epilogue, P rounded
# to bf16 for the PV product).
F32_MAX_ABS = 1e-5
BF16_MAX_ABS = 2e-2
BF16_REL_FRO = 5e-3


def to64(t):
    return t.detach().to(torch.float64).cpu().numpy()


def bf16_close(got, ref, what=""):
    got = to64(got) if hasattr(got, "detach") else np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    max_abs = float(err.max()) if err.size else 0.0
    den = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(got - ref) / den) if den > 0 else float(np.linalg.norm(got))
    _record("bf16", what, max_abs=max_abs, rel_fro=rel, max_abs_bound=BF16_MAX_ABS, rel_fro_bound=BF16_REL_FRO)
    assert max_abs <= BF16_MAX_ABS, f"{what}: max-abs {max_abs:.3e} > {BF16_MAX_ABS}"
    assert rel <= BF16_REL_FRO, f"{what}: rel-Frobenius {rel:.3e} > {BF16_REL_FRO}"
    return max_abs, rel


def f32_close(got, ref, what=""):
    got = to64(got) if hasattr(got, "detach") else np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    err = float(np.abs(got - ref).max()) if got.size else 0.0
    _record("f32", what, max_abs=err, max_abs_bound=F32_MAX_ABS)
    assert err <= F32_MAX_ABS, f"{what}: max-abs {err:.3e} > {F32_MAX_ABS}"
    return err


def sample_rows(B, S, n_pairs, n=1024, seed=0, tile=128):
    """Seeded stratified sample of (b, i, p): tile boundaries, first and last rows, every pair."""
    rng = np.random.default_rng(seed)
    special = sorted({0, 1, tile - 1, tile, tile + 1, 2 * tile - 1, S // 2, S - 2, S - 1} & set(range(S)))
    rows = []
    for b in range(B):
        for p in range(n_pairs):
            for i in special:
                rows.append((b, i, p))
    while len(rows) < n + len(special) * B * n_pairs:
        rows.append((int(rng.integers(B)), int(rng.integers(S)), int(rng.integers(n_pairs))))
    return rows


# Gradients (bf16 backward): relative Frobenius and max-abs relative to the largest
# reference entry. P and dS are rounded to bf16 before their products (relative 2^-9 each),
# the branch outputs O_b that E = dO . O_b reads are stored in bf16, and every gradient is
# rounded once to bf16: each term is ~2e-3 relative. The bounds are set at about twice the
# worst errors measured on B200 over the whole backward test set (the kernels are
# deterministic: no atomics, fixed summation order): relative Frobenius 3.15e-3 (dV of a
# one-token sequence) and max-abs 4.86e-3 of the largest entry (dV with a one-key window).
GRAD_REL_FRO = 6e-3
GRAD_MAX_REL = 9.5e-3
# A reference that is identically zero (e.g. dQ with a one-key window: P = 1, dS = dP - E = 0)
# has no scale for a relative bound; the GPU's result there is fp32 rounding of O(1) terms
# (dP from the MMA against E from a dot product). Measured worst: 2.79e-6 (dK with a one-key
# window over 300 tokens); the bound is just under twice that.
GRAD_ZERO_ABS = 5.5e-6


def grad_close(got, ref, what=""):
    got = to64(got) if hasattr(got, "detach") else np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite gradient"
    scale = float(np.abs(ref).max()) if ref.size else 0.0
    max_abs = float(np.abs(got - ref).max()) if ref.size else 0.0
    if scale == 0.0:
        _record("grad_zero_ref", what, max_abs=max_abs, max_abs_bound=GRAD_ZERO_ABS)
        assert max_abs <= GRAD_ZERO_ABS, f"{what}: zero reference, max-abs {max_abs:.3e} > {GRAD_ZERO_ABS}"
        return max_abs, 0.0
    den = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(got - ref) / den) if den > 0 else float(np.linalg.norm(got))
    _record("grad", what, max_abs_over_scale=max_abs / scale, rel_fro=rel, max_abs_over_scale_bound=GRAD_MAX_REL,
            rel_fro_bound=GRAD_REL_FRO)
    assert max_abs <= GRAD_MAX_REL * max(scale, 1e-30), f"{what}: max-abs {max_abs:.3e} > {GRAD_MAX_REL} x {scale:.3e}"
    assert rel <= GRAD_REL_FRO, f"{what}: rel-Frobenius {rel:.3e} > {GRAD_REL_FRO}"
    return max_abs, rel
