"""Seeded synthetic inputs for the 4-bit weight-quantised linear layer.

This module only draws random numbers and lays them out in the input formats
the layer consumes. It holds none of the layer's arithmetic: no
dequantisation, no product, no kernel layout. The CPU oracle's tests, the CUDA
path's tests and the benchmark all take their inputs from here, so both sides
see identical bytes.

Value distributions follow the workloads of the MARLIN page (4-bit weights,
fp16 activations, one linear layer) and the OdysseyLLM page (W4A8):

* codes ``q``: integers uniform in 0..15, shape ``[K, N]``;
* W4A16 group scales: fp16 ``0.002 + 0.01*|N(0,1)|`` per ``(K/g, N)``;
* W4A16 activations: fp16 ``N(0,1)``, shape ``[M, K]``;
* W4A8 activations: int8 uniform in ``[-127, 127]`` (both ends included);
* W4A8 per-token scale: fp32 ``0.01 + 0.05*|N(0,1)|`` per row;
* W4A8 per-channel weight scale: fp32 ``0.002 + 0.01*|N(0,1)|`` per column.

Draw order for one seed (one ``numpy.random.default_rng(seed)`` per layer):
codes, then weight scales, then activations (then, for W4A8, the per-token
scales). ``numpy`` draws sequentially, so the first ``M`` rows of the
activations are the same for every ``M``: the weights stay identical across an
``M`` sweep with the same seed.

The input format of ``Q`` (the packed codes the layer receives) is 8 codes per
int32 along K: code ``q[8*i + j, n]`` sits in bits ``4*j .. 4*j+3`` of
``Q[i, n]`` (lowest nibble first).
"""
from __future__ import annotations

import numpy as np

__all__ = ["pack_q", "w4a16_inputs", "w4a8_inputs", "w4a16_sparse24_inputs", "w4a16_mixed_inputs"]


def pack_q(q: np.ndarray) -> np.ndarray:
    """Encode codes ``q[K, N]`` (values 0..15) into the packed int32 input ``Q[K/8, N]``."""
    q = np.asarray(q)
    K, N = q.shape
    if K % 8:
        raise ValueError("K must be a multiple of 8 to pack 8 codes per int32")
    q32 = q.astype(np.uint32).reshape(K // 8, 8, N)
    word = np.zeros((K // 8, N), dtype=np.uint32)
    for j in range(8):
        word |= q32[:, j, :] << np.uint32(4 * j)
    return word.view(np.int32)


def _codes(rng: np.random.Generator, K: int, N: int) -> np.ndarray:
    return rng.integers(0, 16, size=(K, N), dtype=np.uint8)


def w4a16_inputs(K: int, N: int, g: int, M: int, seed: int = 0) -> dict:
    """Inputs of one W4A16 layer: codes, packed codes, fp16 group scales, fp16 activations."""
    if K % g:
        raise ValueError("g must divide K")
    rng = np.random.default_rng(seed)
    q = _codes(rng, K, N)
    s = (0.002 + 0.01 * np.abs(rng.standard_normal((K // g, N)))).astype(np.float16)
    A = rng.standard_normal((M, K)).astype(np.float16)
    return {"q": q, "Q": pack_q(q), "s": s, "A": A, "K": K, "N": N, "g": g, "M": M}


def w4a8_inputs(K: int, N: int, M: int, seed: int = 0) -> dict:
    """Inputs of one W4A8 layer: codes, packed codes, fp32 channel scales, int8 activations, fp32 token scales."""
    rng = np.random.default_rng(seed)
    q = _codes(rng, K, N)
    sw = (0.002 + 0.01 * np.abs(rng.standard_normal(N))).astype(np.float32)
    A = rng.integers(-127, 128, size=(M, K), dtype=np.int8)
    sa = (0.01 + 0.05 * np.abs(rng.standard_normal(M))).astype(np.float32)
    return {"q": q, "Q": pack_q(q), "sw": sw, "A": A, "sa": sa, "K": K, "N": N, "M": M}


def w4a16_sparse24_inputs(K: int, N: int, g: int, M: int, seed: int = 0) -> dict:
    """The inputs of ``w4a16_inputs`` with the codes pruned 2:4: in every run of 4 rows
    (4i .. 4i+3) of every column, two rows drawn uniformly keep their code and the other two
    get code 8 (a zero weight). The pattern is drawn after the activations."""
    d = w4a16_inputs(K, N, g, M, seed=seed)
    rng = np.random.default_rng(seed + 1)
    q = d["q"].reshape(K // 4, 4, N).copy()
    keep = np.argsort(rng.random((K // 4, 4, N)), axis=1)[:, :2, :]  # two distinct rows per group
    mask = np.zeros((K // 4, 4, N), dtype=bool)
    np.put_along_axis(mask, keep, True, axis=1)
    q[~mask] = 8
    q = q.reshape(K, N)
    d.update(q=q, Q=pack_q(q))
    return d


def w4a16_mixed_inputs(K: int, N: int, g: int, M: int, seed: int = 0, frac4: float = 0.15) -> dict:
    """The inputs of ``w4a16_inputs`` for mixed 2/4-bit weights: a width per block of 32 rows
    and 128 columns, 4 with probability ``frac4`` and 2 otherwise (``widths`` uint8
    [K/32, ceil(N/128)]); the codes of 2-bit blocks are the 4-bit draws reduced mod 4."""
    d = w4a16_inputs(K, N, g, M, seed=seed)
    rng = np.random.default_rng(seed + 2)
    nt = -(-N // 128)
    widths = np.where(rng.random((K // 32, nt)) < frac4, 4, 2).astype(np.uint8)
    per = np.repeat(np.repeat(widths, 32, axis=0), 128, axis=1)[:, :N]
    q = np.where(per == 2, d["q"] % 4, d["q"]).astype(np.uint8)
    d.update(q=q, Q=pack_q(q), widths=widths)
    return d
