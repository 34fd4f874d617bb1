"""Helpers of the GPU parity tests: move synthetic inputs to the device, compare with the oracle.

The comparison is the layer's stated tolerance, elementwise over every compared output:
``|y - y_ref| <= 2^-10 |y_ref| + 1e-3 sum_k |a_k w_k|`` with ``y_ref`` the fp64 oracle.
NaN or Inf in the CUDA output always fails.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth

DEV = "cuda"


def to_dev(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x)).to(DEV)


def half_bits_to_f64(Y: torch.Tensor) -> np.ndarray:
    return Y.float().cpu().numpy().astype(np.float64)


def compare(y: np.ndarray, y_ref: np.ndarray, absdot: np.ndarray, what: str = "") -> float:
    """Assert the tolerance; return the worst err/bound ratio (for the record)."""
    assert y.shape == y_ref.shape, (y.shape, y_ref.shape)
    assert np.all(np.isfinite(y)), f"{what}: non-finite output"
    bound = oracle.tolerance(y_ref, absdot)
    err = np.abs(y - y_ref)
    bad = err > bound
    ratio = float(np.max(err / np.maximum(bound, 1e-300))) if err.size else 0.0
    if bad.any():
        idx = np.argwhere(bad)[:5].tolist()
        raise AssertionError(f"{what}: {int(bad.sum())}/{bad.size} outside tolerance, worst ratio {ratio:.3g}, "
                             f"first {idx}: got {[y[tuple(i)] for i in idx]} ref {[y_ref[tuple(i)] for i in idx]}")
    return ratio


def w4a16_case(K, N, g, M, seed=0):
    """Inputs, prepacked weights and the CUDA output of one W4A16 layer."""
    import bit_weight_quantized_prepack_b200 as wq
    d = synth.w4a16_inputs(K, N, g, M, seed=seed)
    Q, s, A = to_dev(d["Q"]), to_dev(d["s"]), to_dev(d["A"])
    Wp = wq.wq_prepack(Q, s, g)
    Y = wq.wq_gemm_w4a16(A, Wp, N, g)
    torch.cuda.synchronize()
    return d, Wp, Y


def check_w4a16_full(d, Y, what=""):
    y_ref = oracle.w4a16(d["A"], d["Q"], d["s"], d["g"])
    ad = oracle.w4a16_absdot(d["A"], d["Q"], d["s"], d["g"])
    return compare(half_bits_to_f64(Y), y_ref, ad, what)


def check_w4a16_cols(d, Y, cols, rows=None, what=""):
    """Compare the given output columns (and rows) only; the oracle computes just those."""
    cols = np.asarray(cols)
    A = d["A"] if rows is None else d["A"][rows]
    Qc, sc = d["Q"][:, cols], d["s"][:, cols]
    y_ref = oracle.w4a16(A, Qc, sc, d["g"])
    ad = oracle.w4a16_absdot(A, Qc, sc, d["g"])
    y = half_bits_to_f64(Y)[:, cols]
    if rows is not None:
        y = y[rows]
    return compare(y, y_ref, ad, what)


def sample_cols(N, n, seed=0):
    rng = np.random.default_rng(seed)
    # always include both edges and the last (possibly ragged) tile
    cols = set(rng.choice(N, size=min(n, N), replace=False).tolist()) | {0, N - 1}
    return np.array(sorted(cols))
