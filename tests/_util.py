"""Helpers shared by the GPU parity tests (no attention arithmetic here)."""

import numpy as np


def to_dev(bits):
    """uint16 bf16 bits (numpy) -> bf16 CUDA tensor with the same bits."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def to_f64(t):
    """CUDA/CPU tensor -> float64 numpy array (exact for bf16/fp32)."""
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_fro(got, ref):
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / den) if den > 0 else float(np.linalg.norm(got))


def check_o(got, ref, what=""):
    """Forward output tolerance: max-abs <= 1e-2 and relative Frobenius <= 5e-3."""
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = float(np.max(np.abs(got - ref))) if ref.size else 0.0
    rf = rel_fro(got, ref)
    assert err <= 1e-2, f"{what}: O max-abs error {err:.3e}"
    assert rf <= 5e-3, f"{what}: O relative Frobenius error {rf:.3e}"
    return err, rf


def check_lse(got, ref, what=""):
    """|dLSE| <= 1e-5 * max(1, |LSE|); rows with no visible key must be -inf on both sides."""
    dead = np.isneginf(ref)
    assert np.array_equal(np.isneginf(got), dead), f"{what}: -inf rows differ"
    live = ~dead
    tol = 1e-5 * np.maximum(1.0, np.abs(ref[live]))
    bad = np.abs(got[live] - ref[live]) > tol
    assert not bad.any(), f"{what}: LSE error {np.max(np.abs(got[live]-ref[live])):.3e} at {np.argwhere(bad)[:3]}"


def check_grad(got, ref, what=""):
    """Gradient tolerance: relative Frobenius <= 2e-2."""
    assert np.all(np.isfinite(got)), f"{what}: non-finite gradient"
    rf = rel_fro(got, ref)
    assert rf <= 2e-2, f"{what}: relative Frobenius error {rf:.3e}"
    return rf
