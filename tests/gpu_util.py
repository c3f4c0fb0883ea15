"""Helpers shared by the GPU tests: tolerance checks against the oracle and
row sampling.  No PatchEmbed arithmetic lives here."""
from __future__ import annotations

import numpy as np
import torch


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    """One bf16 ulp at |v| (8 significant bits), with the subnormal floor."""
    a = np.abs(np.asarray(v, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return np.exp2(e - 7)


def assert_within_tolerance(gpu: torch.Tensor, ref: np.ndarray, absdot: np.ndarray,
                            rows=None, what: str = "", rel: float = 1e-3) -> float:
    """|gpu - oracle| <= rel * sum_k |x_k w_k| per element (fp32 output; rel = 1e-3
    unless a test states its own bound), plus one bf16 ulp of the oracle value
    for bf16 output.  Returns the worst ratio err/tol."""
    g = gpu.detach().to("cpu").double().numpy()
    if rows is not None:
        g = g[rows]
        ref = ref[rows]
        absdot = absdot[rows]
    assert g.shape == ref.shape, (g.shape, ref.shape)
    tol = rel * absdot
    if gpu.dtype == torch.bfloat16:
        tol = tol + bf16_ulp(ref)
    err = np.abs(g - ref)
    bad = ~(err <= tol)
    if bad.any():
        idx = np.argwhere(bad)[:5]
        det = [(tuple(int(x) for x in i), float(g[tuple(i)]), float(ref[tuple(i)]), float(tol[tuple(i)]))
               for i in idx]
        raise AssertionError(f"{what}: {int(bad.sum())} elements out of tolerance; first: {det}")
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(tol > 0, err / tol, 0.0)
    return float(ratio.max()) if ratio.size else 0.0


def sample_rows(N: int, k: int, seed: int, extra=()) -> np.ndarray:
    """k random rows plus the first/last rows of every 128-row tile boundary
    pair near the ends and any `extra` rows (item boundaries)."""
    rng = np.random.default_rng(seed)
    s = set(rng.choice(N, size=min(k, N), replace=False).tolist())
    for r in (0, 1, 127, 128, 129, N - 129, N - 128, N - 1):
        if 0 <= r < N:
            s.add(r)
    for r in extra:
        if 0 <= r < N:
            s.add(int(r))
    return np.array(sorted(s), dtype=np.int64)


def mask_of(rows: np.ndarray, N: int) -> np.ndarray:
    m = np.zeros(N, dtype=np.uint8)
    m[rows] = 1
    return m
