"""Helpers shared by the GPU tests: host<->device bf16 transfers and the
parity metrics.  No attention arithmetic lives here."""
from __future__ import annotations

import numpy as np

import synth

# Bars of the parity contract: permutations bit-exact; attention within
# max-abs 2e-2 and mean-abs 2e-3 of the fp64 oracle; in addition a relative
# L2 error per head of at most 1e-2 (at N >= 32k the outputs are ~1e-2 in
# magnitude, below the absolute bar, so the relative bar is the sharp one).
MAX_ABS = 2e-2
MEAN_ABS = 2e-3
REL_L2 = 1e-2


def to_dev(a: np.ndarray, device="cuda"):
    import torch
    assert a.dtype == np.uint16
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device).view(torch.bfloat16)


def to_host(t) -> np.ndarray:
    import torch
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


def compare(gpu_rows_bf16: np.ndarray, oracle_rows: np.ndarray, heads: np.ndarray):
    """gpu_rows_bf16: [R][D] uint16; oracle_rows: [R][D] float64; heads: [R]
    (rel-L2 is taken per head).  Returns a dict of metrics."""
    g = synth.bf16_to_f32(gpu_rows_bf16).astype(np.float64)
    d = np.abs(g - oracle_rows)
    rel = 0.0
    for h in np.unique(heads):
        m = heads == h
        den = np.linalg.norm(oracle_rows[m])
        rel = max(rel, float(np.linalg.norm(g[m] - oracle_rows[m]) / max(den, 1e-300)))
    return {"max_abs": float(d.max()), "mean_abs": float(d.mean()), "rel_l2": rel,
            "finite": bool(np.isfinite(g).all())}


def assert_parity(metrics, where=""):
    assert metrics["finite"], f"{where}: non-finite outputs"
    assert metrics["max_abs"] <= MAX_ABS, f"{where}: {metrics}"
    assert metrics["mean_abs"] <= MEAN_ABS, f"{where}: {metrics}"
    assert metrics["rel_l2"] <= REL_L2, f"{where}: {metrics}"
