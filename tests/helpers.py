"""Shared tolerance checks and row samplers for the GPU parity tests.

Tolerances (stated in the design notes and applied everywhere):

* fp32 path: max |gpu - oracle| <= 1e-5 (unnormalised).
* bf16 path: rel-L2 = ||gpu - oracle|| / ||oracle|| <= 5e-3, and
  max over elements of (|gpu - oracle| - 2^-8 |oracle|) <= 1e-2 * max(1, rms(oracle)):
  the literal max-abs 1e-2 for outputs of unit scale, measured in units of
  the oracle's RMS for larger outputs (a window of 4096 sigmoid weights gives
  |o| ~ 64, where one bf16 ulp is 0.25), after allowing the half
  unit-in-the-last-place of the final bf16 output cast (2^-8 relative).
"""
from __future__ import annotations

import numpy as np

BF16_REL_L2 = 5e-3
BF16_MAX_NORM = 1e-2
F32_MAX_ABS = 1e-5


def to_np(t) -> np.ndarray:
    import torch
    if isinstance(t, torch.Tensor):
        return t.detach().float().cpu().numpy().astype(np.float64)
    return np.asarray(t, dtype=np.float64)


def bf16_errors(got, ref):
    got, ref = to_np(got), to_np(ref)
    diff = got - ref
    nref = np.linalg.norm(ref)
    rel_l2 = np.linalg.norm(diff) / max(nref, 1e-30)
    rms = np.sqrt(np.mean(ref * ref)) if ref.size else 0.0
    excess = np.max(np.abs(diff) - 2.0 ** -8 * np.abs(ref)) if ref.size else 0.0
    max_norm = max(excess, 0.0) / max(rms, 1.0)
    return rel_l2, max_norm, float(np.max(np.abs(diff))) if ref.size else 0.0


def assert_bf16_close(got, ref, what="", allowance=None):
    """allowance: optional per-element slack added to the max-abs check (the
    deviation that bf16 storage of the rotated Q/K operands causes by itself,
    see quantized_operand_bwd); rel-L2 is always against the exact oracle."""
    if allowance is not None:
        got_np, ref_np = to_np(got), to_np(ref)
        excess = np.abs(got_np - ref_np) - np.asarray(allowance, dtype=np.float64)
        clipped = ref_np + np.sign(got_np - ref_np) * np.maximum(excess, 0.0)
        rel_l2, _, max_abs = bf16_errors(got_np, ref_np)
        _, max_norm, _ = bf16_errors(clipped, ref_np)
        assert np.all(np.isfinite(got_np)), f"{what}: non-finite output"
        assert rel_l2 <= BF16_REL_L2 and max_norm <= BF16_MAX_NORM, \
            f"{what}: rel_l2={rel_l2:.3e} max_norm(beyond allowance)={max_norm:.3e} max_abs={max_abs:.3e}"
        return rel_l2, max_norm
    rel_l2, max_norm, max_abs = bf16_errors(got, ref)
    assert np.all(np.isfinite(to_np(got))), f"{what}: non-finite output"
    assert rel_l2 <= BF16_REL_L2 and max_norm <= BF16_MAX_NORM, \
        f"{what}: rel_l2={rel_l2:.3e} max_norm={max_norm:.3e} max_abs={max_abs:.3e}"
    return rel_l2, max_norm


def assert_f32_close(got, ref, what="", tol=F32_MAX_ABS):
    got, ref = to_np(got), to_np(ref)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = float(np.max(np.abs(got - ref))) if ref.size else 0.0
    assert err <= tol, f"{what}: max abs err {err:.3e} > {tol:.1e}"
    return err


def sample_rows(B, H, N, window, n_random=256, seed=0, tile=128):
    """(b, h, i) rows: the first rows (partial windows), rows around every
    tile edge near the start and end, the last row, and random rows."""
    rng = np.random.default_rng(seed)
    picks = set()
    firsts = list(range(min(N, 3))) + [min(N - 1, window - 1), min(N - 1, window), min(N - 1, 2 * window - 1)]
    edges = []
    for e in list(range(tile, min(N, 4 * tile + 1), tile)) + [N - tile, N - 1]:
        for di in (-1, 0, 1):
            if 0 <= e + di < N:
                edges.append(e + di)
    for b in range(B):
        for h in range(H):
            for i in firsts + edges[:6]:
                if rng.random() < 0.35:
                    picks.add((b, h, int(i)))
    for _ in range(n_random):
        picks.add((int(rng.integers(B)), int(rng.integers(H)), int(rng.integers(N))))
    picks.add((B - 1, H - 1, N - 1))
    picks.add((0, 0, 0))
    return np.array(sorted(picks), dtype=np.int64)


def round_bf16(x) -> np.ndarray:
    """Round to the nearest bf16 value (ties to even), returned as fp64."""
    f = np.asarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def quantized_operand_bwd(q, k, v, do, *, window, n_sink, mode, slopes, rope_base, exact):
    """Per-element deviation of the gradients caused only by the bf16
    precision of the tensor-core operands (rotated Q and K, P, dS): the
    dense numpy oracle's backward with those four matrices rounded to bf16,
    minus the exact oracle's gradients. Returns |d dq|, |d dk|, |d dv|."""
    from oracle import ref_numpy
    got = ref_numpy.swat_bwd(q, k, v, do, window=window, n_sink=n_sink, mode=mode,
                             slopes=slopes, rope_base=rope_base, operand_round=round_bf16)
    return tuple(np.abs(g - e) for g, e in zip(got, exact))
