"""CPU fp64 oracle of the 4-bit weight-quantised linear layer (W4A16 and W4A8).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
legs of ``bench.py`` may import this module. The library never does: it has no
CPU path, and it shares no code, table or helper with this file.

What it computes, and where that comes from:

* "MARLIN: Mixed-Precision Auto-Regressive Parallel Inference on Large Language
  Models", Abstract: a linear layer whose weights are quantised to 4 bits per
  element and whose activations stay in fp16. The layer is
  ``Y[M,N] = A[M,K] . W[K,N]``.
* "Atom: Low-bit Quantization for Efficient and Accurate LLM Serving",
  proposed method (fine-grained group quantisation): one scale per group of
  ``g`` consecutive rows of ``W`` and output column. The zero point is fixed at
  8, so ``W[k,n] = (q[k,n] - 8) * s[k // g, n]``.
* "A Speed Odyssey for Deployable Quantization of LLMs", Abstract (FastGEMM,
  W4A8): int8 activations times the same 4-bit weights, with a per-token scale
  (Atom, dynamic activation quantisation) and a per-channel weight scale:
  ``Y[m,n] = sa[m] * sw[n] * sum_k A[m,k] * (q[k,n] - 8)``.

Around the layer (each function's docstring gives its reading of the pages):

* per-token activation quantisation (``quantize_act``; Atom, method: dynamic
  activation quantisation), 8-bit for W4A8 and 4-bit for W4A4 numerics;
* asymmetric groups (``dequant_zp``, ``w4a16_zp``): a 4-bit zero point per group
  and column instead of the fixed 8;
* act order (``dequant_gidx``, ``w4a16_gidx``, ``act_order_perm``,
  ``reorder_rows``): groups whose rows are scattered along K by ``g_idx``;
* 2:4 sparse weights (``is_sparse24``, ``prepack_w4a16_sparse24``): the layer is
  ``w4a16`` of the pruned weight; only the prepacked format differs;
* mixed 2/4-bit weights (``dequant_mixed``, ``w4a16_mixed``, ``prepack_mixed``): a bit width
  per aligned 32-row x 128-column block, zero point 2 or 8.

Every function here is pinned by ``tests/oracle_pins.py`` (hand-worked golden
values, exact rational brute force, closed forms and invariants); none is
"parity unpinned".

The pages do not fix the packing of the codes; the reading used here is the
plainest one for "8 codes per int32" of a K x N weight: ``Q`` is ``[K/8, N]``
and code ``k = 8*i + j`` of column ``n`` sits in bits ``4j .. 4j+3`` of
``Q[i, n]``.

The layer reaches the exact product up to rounding, so the oracle is that
definition written out in float64: unpack, dequantise exactly in fp64, then one
fp64 matrix product (a library primitive). The W4A8 integer accumulator is
computed exactly as well (see ``w4a8_acc``).

The prepacked weight format (``prepack_w4a16`` / ``prepack_w4a8``) is this
library's own design: the "Efficient Arbitrary Precision Acceleration for Large
Language Models on GPU Tensor Cores" page names a matrix preprocessing step
that reorders the weights for the kernel, but gives no layout. The functions
below restate the documented layout plainly, so that the CUDA prepack can be
compared with it byte for byte.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "unpack_codes", "dequant", "w4a16", "w4a16_absdot", "w4a16_entry",
    "tolerance", "w4a8_acc", "w4a8", "w4a8_absdot", "quantize_act",
    "dequant_gidx", "w4a16_gidx", "w4a16_gidx_absdot", "act_order_perm", "pack_codes", "reorder_rows",
    "prepack_w4a16_act_order",
    "dequant_zp", "w4a16_zp", "w4a16_zp_absdot", "prepack_w4a16_zp", "prepacked_bytes_w4a16_zp", "unprepack_w4a16_zp",
    "TILE_N", "TILE_K", "prepack_w4a16", "prepack_w4a8",
    "is_sparse24", "MIXED_BLOCK_ROWS", "mixed_zero_points", "dequant_mixed", "w4a16_mixed", "w4a16_mixed_absdot",
    "prepacked_bytes_mixed", "prepack_mixed", "unprepack_mixed", "prepacked_bytes_w4a16_sparse24", "prepack_w4a16_sparse24",
    "unprepack_w4a16_sparse24",
    "prepacked_bytes_w4a16", "prepacked_bytes_w4a8", "unprepack_w4a16", "unprepack_w4a8",
]

ZERO_POINT = 8          # w = (q - 8) * s  (fixed symmetric zero point)
REL_TOL = 2.0 ** -10    # |y - y_ref| <= 2^-10 |y_ref| + 1e-3 sum_k |a_k w_k|
ABS_DOT_TOL = 1e-3


# --------------------------------------------------------------------------
# the layer
# --------------------------------------------------------------------------
def unpack_codes(Q: np.ndarray) -> np.ndarray:
    """Codes ``q[K, N]`` from the packed ``Q[K/8, N]``: ``q[8i+j, n] = (Q[i,n] >> 4j) & 15``."""
    Qu = np.asarray(Q).view(np.uint32)
    K8, N = Qu.shape
    q = np.empty((K8, 8, N), dtype=np.uint8)
    for j in range(8):
        q[:, j, :] = (Qu >> np.uint32(4 * j)) & np.uint32(0xF)
    return q.reshape(K8 * 8, N)


def dequant(q: np.ndarray, s: np.ndarray, g: int) -> np.ndarray:
    """``W[k,n] = (q[k,n] - 8) * s[k // g, n]`` in float64 (exact: an int times an fp16)."""
    K, N = q.shape
    if K % g:
        raise ValueError("g must divide K")
    group = np.arange(K) // g
    return (q.astype(np.float64) - ZERO_POINT) * np.asarray(s, dtype=np.float64)[group, :]


def _w_columns(Q, s, g, n0, n1):
    return dequant(unpack_codes(np.asarray(Q)[:, n0:n1]), np.asarray(s)[:, n0:n1], g)


def w4a16(A: np.ndarray, Q: np.ndarray, s: np.ndarray, g: int, chunk: int = 4096) -> np.ndarray:
    """``Y = A . W`` in float64, with ``W`` dequantised in float64; chunked along N to bound memory."""
    A64 = np.asarray(A, dtype=np.float64)
    N = np.asarray(Q).shape[1]
    Y = np.empty((A64.shape[0], N), dtype=np.float64)
    for n0 in range(0, N, chunk):
        n1 = min(N, n0 + chunk)
        Y[:, n0:n1] = A64 @ _w_columns(Q, s, g, n0, n1)
    return Y


def w4a16_absdot(A: np.ndarray, Q: np.ndarray, s: np.ndarray, g: int, chunk: int = 4096) -> np.ndarray:
    """``sum_k |A[m,k] * W[k,n]|`` in float64: the scale of the tolerance's second term."""
    A64 = np.abs(np.asarray(A, dtype=np.float64))
    N = np.asarray(Q).shape[1]
    out = np.empty((A64.shape[0], N), dtype=np.float64)
    for n0 in range(0, N, chunk):
        n1 = min(N, n0 + chunk)
        out[:, n0:n1] = A64 @ np.abs(_w_columns(Q, s, g, n0, n1))
    return out


def w4a16_entry(A: np.ndarray, Q: np.ndarray, s: np.ndarray, g: int, m: int, n: int):
    """One output ``(y[m,n], sum_k |a w|)`` computed on its own, for sampled checks of large layers."""
    w = _w_columns(Q, s, g, n, n + 1)[:, 0]
    a = np.asarray(A[m], dtype=np.float64)
    return float(a @ w), float(np.abs(a) @ np.abs(w))


def tolerance(y_ref: np.ndarray, absdot: np.ndarray) -> np.ndarray:
    """Allowed error: ``2^-10 |y_ref| + 1e-3 sum_k |a_k w_k|``."""
    return REL_TOL * np.abs(y_ref) + ABS_DOT_TOL * absdot


def w4a8_acc(A: np.ndarray, Q: np.ndarray, chunk: int = 4096) -> np.ndarray:
    """Exact integer accumulator ``sum_k A[m,k] * (q[k,n] - 8)`` as int64.

    The product runs in float64 through BLAS: every operand is an integer of
    magnitude <= 127 or <= 8 and every partial sum stays far below 2^53, so
    each float64 operation is exact and the order of summation cannot change
    the result.
    """
    A64 = np.asarray(A, dtype=np.float64)
    K = A64.shape[1]
    if 127 * 8 * K >= 2 ** 53:
        raise ValueError("K too large for an exact float64 accumulation")
    N = np.asarray(Q).shape[1]
    acc = np.empty((A64.shape[0], N), dtype=np.int64)
    for n0 in range(0, N, chunk):
        n1 = min(N, n0 + chunk)
        wq = unpack_codes(np.asarray(Q)[:, n0:n1]).astype(np.float64) - ZERO_POINT
        acc[:, n0:n1] = (A64 @ wq).astype(np.int64)
    return acc


def w4a8(A: np.ndarray, sa: np.ndarray, Q: np.ndarray, sw: np.ndarray):
    """``(acc, Y)``: the exact int64 accumulator and ``Y = acc * sa[m] * sw[n]`` in float64."""
    acc = w4a8_acc(A, Q)
    Y = acc.astype(np.float64) * np.asarray(sa, np.float64)[:, None] * np.asarray(sw, np.float64)[None, :]
    return acc, Y


def w4a8_absdot(A: np.ndarray, sa: np.ndarray, Q: np.ndarray, sw: np.ndarray, chunk: int = 4096) -> np.ndarray:
    """``sa[m] * sw[n] * sum_k |A[m,k] * (q[k,n] - 8)|`` in float64."""
    A64 = np.abs(np.asarray(A, dtype=np.float64))
    N = np.asarray(Q).shape[1]
    out = np.empty((A64.shape[0], N), dtype=np.float64)
    for n0 in range(0, N, chunk):
        n1 = min(N, n0 + chunk)
        wq = np.abs(unpack_codes(np.asarray(Q)[:, n0:n1]).astype(np.float64) - ZERO_POINT)
        out[:, n0:n1] = A64 @ wq
    return out * np.asarray(sa, np.float64)[:, None] * np.asarray(sw, np.float64)[None, :]


# --------------------------------------------------------------------------
# act order: groups that are not contiguous along K
# --------------------------------------------------------------------------
def dequant_gidx(q: np.ndarray, s: np.ndarray, z, g_idx: np.ndarray) -> np.ndarray:
    """``W[k,n] = (q[k,n] - z[g_idx[k], n]) * s[g_idx[k], n]`` in float64 (exact).

    Group quantisation whose groups are not runs of consecutive rows: row ``k`` belongs to
    group ``g_idx[k]`` (the "act order" of GPTQ-style checkpoints, where the rows were
    quantised in an order of decreasing activation importance and each run of ``g`` rows in
    that order shares one scale and zero point). The pages fix groups only as "fine-grained"
    (Atom, method); this reading keeps their per-group scale and zero point and lets the rows
    of a group lie anywhere. ``z = None`` is the fixed zero point 8.
    """
    g_idx = np.asarray(g_idx)
    zz = ZERO_POINT if z is None else np.asarray(z, dtype=np.float64)[g_idx, :]
    return (q.astype(np.float64) - zz) * np.asarray(s, dtype=np.float64)[g_idx, :]


def w4a16_gidx(A: np.ndarray, Q: np.ndarray, s: np.ndarray, z, g_idx: np.ndarray, chunk: int = 4096) -> np.ndarray:
    """``Y = A . W`` with ``W = dequant_gidx(...)``, in float64, chunked along N."""
    A64 = np.asarray(A, dtype=np.float64)
    N = np.asarray(Q).shape[1]
    Y = np.empty((A64.shape[0], N), dtype=np.float64)
    for n0 in range(0, N, chunk):
        n1 = min(N, n0 + chunk)
        zc = None if z is None else np.asarray(z)[:, n0:n1]
        Y[:, n0:n1] = A64 @ dequant_gidx(unpack_codes(np.asarray(Q)[:, n0:n1]), np.asarray(s)[:, n0:n1], zc, g_idx)
    return Y


def w4a16_gidx_absdot(A: np.ndarray, Q: np.ndarray, s: np.ndarray, z, g_idx: np.ndarray,
                      chunk: int = 4096) -> np.ndarray:
    """``sum_k |A[m,k] * W[k,n]|`` for the act-order weights."""
    A64 = np.abs(np.asarray(A, dtype=np.float64))
    N = np.asarray(Q).shape[1]
    out = np.empty((A64.shape[0], N), dtype=np.float64)
    for n0 in range(0, N, chunk):
        n1 = min(N, n0 + chunk)
        zc = None if z is None else np.asarray(z)[:, n0:n1]
        out[:, n0:n1] = A64 @ np.abs(dequant_gidx(unpack_codes(np.asarray(Q)[:, n0:n1]), np.asarray(s)[:, n0:n1],
                                                  zc, g_idx))
    return out


def act_order_perm(g_idx: np.ndarray, g: int) -> np.ndarray:
    """The row order that makes the groups contiguous: ``perm`` with ``g_idx[perm[i]] == i // g``.

    Rows are sorted by group, keeping their order inside a group. Every group must hold
    exactly ``g`` rows (as it does when the groups are runs of ``g`` rows of some order);
    otherwise no such ``perm`` exists and ``ValueError`` is raised.
    """
    g_idx = np.asarray(g_idx)
    K = g_idx.shape[0]
    if g <= 0 or K % g:
        raise ValueError("g must divide K")
    perm = np.argsort(g_idx, kind="stable")
    if not np.array_equal(g_idx[perm], np.arange(K) // g):
        raise ValueError("every group must hold exactly g rows")
    return perm


def pack_codes(q: np.ndarray) -> np.ndarray:
    """``Q[K/8, N]`` int32 from codes ``q[K, N]``: code ``8i + j`` in bits ``4j .. 4j+3`` of ``Q[i]``."""
    K, N = q.shape
    q32 = np.asarray(q, dtype=np.uint32).reshape(K // 8, 8, N)
    word = np.zeros((K // 8, N), dtype=np.uint32)
    for j in range(8):
        word |= q32[:, j, :] << np.uint32(4 * j)
    return word.view(np.int32)


def reorder_rows(Q: np.ndarray, perm: np.ndarray) -> np.ndarray:
    """The packed codes of the weight whose row ``i`` is row ``perm[i]`` of ``Q``'s weight."""
    return pack_codes(unpack_codes(Q)[np.asarray(perm)])


def prepack_w4a16_act_order(Q: np.ndarray, s: np.ndarray, z, perm: np.ndarray, g: int) -> np.ndarray:
    """The prepacked buffer of an act-order weight: its rows taken in the order ``perm`` (so that
    group ``i // g`` holds rows ``i``), then the contiguous-group layout (with zero points when
    ``z`` is given). The layer then reads the activations in the same order."""
    Qr = reorder_rows(Q, perm)
    return prepack_w4a16(Qr, s, g) if z is None else prepack_w4a16_zp(Qr, s, z, g)


# --------------------------------------------------------------------------
# asymmetric groups: a zero point per group and column
# --------------------------------------------------------------------------
def dequant_zp(q: np.ndarray, s: np.ndarray, z: np.ndarray, g: int) -> np.ndarray:
    """``W[k,n] = (q[k,n] - z[k // g, n]) * s[k // g, n]`` in float64 (exact).

    "Atom: Low-bit Quantization for Efficient and Accurate LLM Serving", method
    (fine-grained group quantisation), read with an asymmetric zero point per group and
    column (the GPTQ-style format the pages leave open): a 4-bit code ``q`` and a 4-bit zero
    ``z`` (0..15) per group, so that a group's weights need not be centred on code 8.
    ``z = 8`` everywhere is the symmetric layer of ``dequant``.
    """
    K, N = q.shape
    if K % g:
        raise ValueError("g must divide K")
    group = np.arange(K) // g
    zz = np.asarray(z, dtype=np.float64)[group, :]
    return (q.astype(np.float64) - zz) * np.asarray(s, dtype=np.float64)[group, :]


def w4a16_zp(A: np.ndarray, Q: np.ndarray, s: np.ndarray, z: np.ndarray, g: int, chunk: int = 4096) -> np.ndarray:
    """``Y = A . W`` with ``W = dequant_zp(...)``, in float64, chunked along N."""
    A64 = np.asarray(A, dtype=np.float64)
    N = np.asarray(Q).shape[1]
    Y = np.empty((A64.shape[0], N), dtype=np.float64)
    for n0 in range(0, N, chunk):
        n1 = min(N, n0 + chunk)
        Y[:, n0:n1] = A64 @ dequant_zp(unpack_codes(np.asarray(Q)[:, n0:n1]), np.asarray(s)[:, n0:n1],
                                       np.asarray(z)[:, n0:n1], g)
    return Y


def w4a16_zp_absdot(A: np.ndarray, Q: np.ndarray, s: np.ndarray, z: np.ndarray, g: int, chunk: int = 4096) -> np.ndarray:
    """``sum_k |A[m,k] * W[k,n]|`` for the asymmetric weights."""
    A64 = np.abs(np.asarray(A, dtype=np.float64))
    N = np.asarray(Q).shape[1]
    out = np.empty((A64.shape[0], N), dtype=np.float64)
    for n0 in range(0, N, chunk):
        n1 = min(N, n0 + chunk)
        out[:, n0:n1] = A64 @ np.abs(dequant_zp(unpack_codes(np.asarray(Q)[:, n0:n1]), np.asarray(s)[:, n0:n1],
                                                np.asarray(z)[:, n0:n1], g))
    return out


# --------------------------------------------------------------------------
# dynamic per-token activation quantisation (the step before W4A8)
# --------------------------------------------------------------------------
def quantize_act(A: np.ndarray, bits: int = 8):
    """``(q, sa)``: integer codes ``q[M,K]`` (int8) and fp32 per-token scales ``sa[M]`` of fp16 activations.

    "Atom: Low-bit Quantization for Efficient and Accurate LLM Serving", method: the
    activations' quantisation parameters are computed from the activation matrix itself at
    inference time, one scale per token (row); the activations are 8-bit for W4A8 and 4-bit
    for W4A4. The pages fix neither the rounding nor the range; the reading used here is the
    plainest symmetric one with ``L = 2^(bits-1) - 1`` levels each side (127 for 8 bits, 7 for
    4), written in fp32 so that the integer codes are decided in one stated precision:

    * ``amax[m] = max_k |A[m,k]|`` (exact: fp16 values);
    * ``inv = fp32(L / amax)``, ``q = rint(fp32(A[m,k] * inv))`` with ties to even, clamped
      to ``[-L, L]`` (-L - 1 is never produced);
    * ``sa[m] = fp32(amax / L)``, so ``A[m,k] ~ q[m,k] * sa[m]``;
    * a row of zeros gives ``q = 0`` and ``sa = 0``.
    """
    if bits not in (4, 8):
        raise ValueError("bits must be 4 or 8")
    L = np.float32(2 ** (bits - 1) - 1)
    A32 = np.asarray(A, dtype=np.float16).astype(np.float32)
    amax = np.max(np.abs(A32), axis=1)
    q = np.zeros(A32.shape, dtype=np.int8)
    sa = np.zeros(A32.shape[0], dtype=np.float32)
    for m in range(A32.shape[0]):
        if amax[m] == 0:
            continue
        inv = L / amax[m]                                  # fp32 division, round to nearest
        t = A32[m] * inv                                   # fp32 products, round to nearest
        q[m] = np.clip(np.rint(t), -L, L).astype(np.int8)  # ties to even
        sa[m] = amax[m] / L
    return q, sa


# --------------------------------------------------------------------------
# the prepacked weight format (this library's layout, restated plainly)
# --------------------------------------------------------------------------
TILE_N = 128      # output columns per tile
TILE_K = 128      # rows of W per k-block
# nibble position of code j (j = 0..7 within a word) in a prepacked word
NIBBLE_POS_W4A16 = (0, 4, 1, 5, 2, 6, 3, 7)
NIBBLE_POS_W4A8 = (0, 2, 4, 6, 1, 3, 5, 7)


def _check_kn(K, N):
    if K <= 0 or K % TILE_K:
        raise ValueError("K must be a positive multiple of 128")
    if N <= 0 or N % 8:
        raise ValueError("N must be a positive multiple of 8")


def _group_slots(K: int, g: int) -> int:
    """Scale rows stored per blob: ``128/g`` for g in {32, 64, 128}; 1 for g a multiple of 128 below K; 0 for g == K."""
    if g == K:
        return 0
    if g in (32, 64, 128):
        return TILE_K // g
    if g % TILE_K == 0 and K % g == 0:
        return 1
    raise ValueError("unsupported group size")


def prepacked_bytes_w4a16(K: int, N: int, g: int) -> int:
    _check_kn(K, N)
    nt, kt = -(-N // TILE_N), K // TILE_K
    slots = _group_slots(K, g)
    blob = TILE_N * TILE_K // 2 + 2 * TILE_N * slots
    tail = 0 if slots else ((2 * nt * TILE_N + 15) // 16) * 16
    return nt * kt * blob + tail


def prepacked_bytes_w4a8(K: int, N: int) -> int:
    _check_kn(K, N)
    return -(-N // TILE_N) * (K // TILE_K) * (TILE_N * TILE_K // 2)


def _blob_words(q: np.ndarray, nibble_pos) -> np.ndarray:
    """Code words of every blob: ``[NT, KT, h=2, v=2, r=128, i=4]`` uint32.

    Word ``(nt, kt, h, v, r, i)`` holds the 8 codes of column ``nt*128 + r``,
    rows ``kt*128 + 64h + 32v + 8i + j`` for ``j = 0..7``; code ``j`` sits at
    nibble ``nibble_pos[j]``. Columns past N hold code 8 (a zero weight).
    """
    K, N = q.shape
    nt, kt = -(-N // TILE_N), K // TILE_K
    qp = np.full((K, nt * TILE_N), ZERO_POINT, dtype=np.uint32)
    qp[:, :N] = q
    # [kt, h, v, i, j, nt, r]
    qv = qp.reshape(kt, 2, 2, 4, 8, nt, TILE_N)
    words = np.zeros((kt, 2, 2, 4, nt, TILE_N), dtype=np.uint32)
    for j in range(8):
        words |= qv[:, :, :, :, j, :, :] << np.uint32(4 * nibble_pos[j])
    # -> [nt, kt, h, v, r, i]
    return np.ascontiguousarray(words.transpose(4, 0, 1, 2, 5, 3))


def prepack_w4a16(Q: np.ndarray, s: np.ndarray, g: int) -> np.ndarray:
    """The W4A16 prepacked buffer as bytes (uint8), following the library's documented layout.

    Blob ``(nt, kt)`` starts at byte ``(nt*KT + kt) * blob_bytes``: 8192 bytes
    of code words (``_blob_words`` order) followed by ``slots`` rows of 128
    fp16 scales, row ``u`` holding ``s[(kt*128 + u*g) // g, nt*128 + r]`` for
    ``g <= 128`` and ``s[(kt*128) // g, ...]`` for larger ``g``. For ``g == K``
    the blobs hold codes only and one fp16 scale per (padded) column follows
    all blobs. Scales of padded columns are 0.
    """
    q = unpack_codes(Q)
    K, N = q.shape
    slots = _group_slots(K, g)
    nt, kt = -(-N // TILE_N), K // TILE_K
    words = _blob_words(q, NIBBLE_POS_W4A16).reshape(nt, kt, -1)
    s = np.asarray(s, dtype=np.float16)
    sp = np.zeros((s.shape[0], nt * TILE_N), dtype=np.float16)
    sp[:, :N] = s
    parts = []
    if slots:
        krow = np.arange(kt)[:, None] * TILE_K + np.arange(slots)[None, :] * g   # first row of each slot
        grp = krow // g                                                          # [kt, slots]
        sc = sp[grp]                                                             # [kt, slots, nt*128]
        sc = sc.reshape(kt, slots, nt, TILE_N).transpose(2, 0, 1, 3).reshape(nt, kt, -1)
        blob = np.concatenate([words.view(np.uint8), sc.view(np.uint8)], axis=2)
        parts.append(blob.reshape(-1))
    else:
        parts.append(words.view(np.uint8).reshape(-1))
        tail = np.zeros(prepacked_bytes_w4a16(K, N, g) - words.nbytes, dtype=np.uint8)
        tail[: 2 * nt * TILE_N] = sp[0].view(np.uint8)
        parts.append(tail)
    out = np.concatenate(parts)
    assert out.nbytes == prepacked_bytes_w4a16(K, N, g)
    return out


def prepack_w4a8(Q: np.ndarray) -> np.ndarray:
    """The W4A8 prepacked buffer as bytes: the code blobs only, with the W4A8 nibble order."""
    q = unpack_codes(Q)
    out = _blob_words(q, NIBBLE_POS_W4A8).view(np.uint8).reshape(-1)
    assert out.nbytes == prepacked_bytes_w4a8(*q.shape)
    return out


def _codes_from_words(words: np.ndarray, nibble_pos, K: int, N: int) -> np.ndarray:
    nt, kt = words.shape[:2]
    w = words.reshape(nt, kt, 2, 2, TILE_N, 4)
    q = np.zeros((kt, 2, 2, 4, 8, nt, TILE_N), dtype=np.uint8)
    wt = w.transpose(1, 2, 3, 5, 0, 4)  # [kt, h, v, i, nt, r]
    for j in range(8):
        q[:, :, :, :, j, :, :] = (wt >> np.uint32(4 * nibble_pos[j])) & np.uint32(0xF)
    return q.reshape(K, nt * TILE_N)[:, :N]


def unprepack_w4a16(Wp: np.ndarray, K: int, N: int, g: int):
    """Inverse of ``prepack_w4a16``: ``(q[K,N] uint8, s[K/g, N] fp16)``."""
    slots = _group_slots(K, g)
    nt, kt = -(-N // TILE_N), K // TILE_K
    code_bytes = TILE_N * TILE_K // 2
    Wp = np.asarray(Wp, dtype=np.uint8)
    if slots:
        blob = Wp.reshape(nt, kt, code_bytes + 2 * TILE_N * slots)
        words = np.ascontiguousarray(blob[:, :, :code_bytes]).view(np.uint32)
        sc = np.ascontiguousarray(blob[:, :, code_bytes:]).view(np.float16).reshape(nt, kt, slots, TILE_N)
        sc = sc.transpose(1, 2, 0, 3).reshape(kt * slots, nt * TILE_N)  # rows in k order
        krow = (np.arange(kt)[:, None] * TILE_K + np.arange(slots)[None, :] * g).reshape(-1)
        s = np.zeros((K // g, nt * TILE_N), dtype=np.float16)
        s[krow // g] = sc
        s = s[:, :N]
    else:
        words = np.ascontiguousarray(Wp[: nt * kt * code_bytes]).view(np.uint32).reshape(nt, kt, -1)
        s = np.ascontiguousarray(Wp[nt * kt * code_bytes: nt * kt * code_bytes + 2 * nt * TILE_N]).view(np.float16)
        s = s[None, :N].copy()
    return _codes_from_words(words, NIBBLE_POS_W4A16, K, N), s


def unprepack_w4a8(Wp: np.ndarray, K: int, N: int) -> np.ndarray:
    """Inverse of ``prepack_w4a8``: codes ``q[K,N]`` uint8."""
    nt, kt = -(-N // TILE_N), K // TILE_K
    words = np.ascontiguousarray(np.asarray(Wp, dtype=np.uint8)).view(np.uint32).reshape(nt, kt, -1)
    return _codes_from_words(words, NIBBLE_POS_W4A8, K, N)


# --------------------------------------------------------------------------
# the asymmetric prepacked format: the W4A16 blob followed by the blob's zero points
# --------------------------------------------------------------------------
def prepacked_bytes_w4a16_zp(K: int, N: int, g: int) -> int:
    """Blobs of ``8192 + 256 * slots + 128 * slots`` bytes (codes, fp16 scales, uint8 zeros);
    ``g`` below ``K`` (one scale and one zero per group and column)."""
    _check_kn(K, N)
    slots = _group_slots(K, g)
    if slots == 0:
        raise ValueError("zero points need g < K")
    nt, kt = -(-N // TILE_N), K // TILE_K
    return nt * kt * (TILE_N * TILE_K // 2 + 3 * TILE_N * slots)


def prepack_w4a16_zp(Q: np.ndarray, s: np.ndarray, z: np.ndarray, g: int) -> np.ndarray:
    """Blob ``(nt, kt)`` = the W4A16 blob of ``prepack_w4a16`` (codes, then ``slots`` rows of 128
    fp16 scales) followed by ``slots`` rows of 128 uint8 zero points, row ``u`` holding
    ``z[(kt*128 + u*g) // g, nt*128 + r]`` for ``g <= 128`` and ``z[(kt*128) // g, ...]`` for
    larger ``g``. Padded columns get zero point 8 and scale 0."""
    K = np.asarray(Q).shape[0] * 8
    N = np.asarray(Q).shape[1]
    slots = _group_slots(K, g)
    if slots == 0:
        raise ValueError("zero points need g < K")
    nt, kt = -(-N // TILE_N), K // TILE_K
    base = prepack_w4a16(Q, s, g).reshape(nt, kt, -1)
    zp = np.full((np.asarray(z).shape[0], nt * TILE_N), ZERO_POINT, dtype=np.uint8)
    zp[:, :N] = np.asarray(z, dtype=np.uint8)
    krow = np.arange(kt)[:, None] * TILE_K + np.arange(slots)[None, :] * g
    zz = zp[krow // g]                                                   # [kt, slots, nt*128]
    zz = zz.reshape(kt, slots, nt, TILE_N).transpose(2, 0, 1, 3).reshape(nt, kt, -1)
    out = np.concatenate([base, zz], axis=2).reshape(-1)
    assert out.nbytes == prepacked_bytes_w4a16_zp(K, N, g)
    return out


def unprepack_w4a16_zp(Wp: np.ndarray, K: int, N: int, g: int):
    """Inverse of ``prepack_w4a16_zp``: ``(q[K,N], s[K/g,N] fp16, z[K/g,N] uint8)``."""
    slots = _group_slots(K, g)
    nt, kt = -(-N // TILE_N), K // TILE_K
    base_bytes = TILE_N * TILE_K // 2 + 2 * TILE_N * slots
    blob = np.asarray(Wp, dtype=np.uint8).reshape(nt, kt, base_bytes + TILE_N * slots)
    q, s = unprepack_w4a16(np.ascontiguousarray(blob[:, :, :base_bytes]).reshape(-1), K, N, g)
    zz = blob[:, :, base_bytes:].reshape(nt, kt, slots, TILE_N).transpose(1, 2, 0, 3).reshape(kt * slots, nt * TILE_N)
    krow = (np.arange(kt)[:, None] * TILE_K + np.arange(slots)[None, :] * g).reshape(-1)
    z = np.zeros((K // g, nt * TILE_N), dtype=np.uint8)
    z[krow // g] = zz
    return q, s, z[:, :N]


# --------------------------------------------------------------------------
# 2:4 sparse weights (the library's prepacked format for them)
# --------------------------------------------------------------------------
# A 2:4 sparse weight has, in every run of 4 consecutive rows of a column (a pruning group,
# rows 4i .. 4i+3), at most 2 codes other than 8 (weight 0). The layer is the W4A16 layer of
# that weight (``w4a16``): sparsity changes the storage, not the result. ("MARLIN:
# Mixed-Precision Auto-Regressive Parallel Inference on Large Language Models", Abstract: the
# kernel extends to NVIDIA 2:4 sparsity; the format below is this library's own.)
#
# Blob (nt, kt) of a 128-column tile and a 128-row k-block: 4096 bytes of code words, 2048 bytes
# of metadata words, then the group scales as in the dense blob (``slots`` rows of 128 fp16).
# Within the k-block, 32-row block b (rows 32b .. 32b+31) holds pruning groups j = 0..7. Column
# c of the tile is in row tile rt = c // 16, with g = c % 8 and half = (c % 16) // 8.
#   code word (b*8 + rt)*32 + 4g + (j % 4) holds the kept codes of groups j and j+4 of the two
#     columns 16rt + g (half 0) and 16rt + g + 8 (half 1) (``_sparse_code_nibble``);
#   metadata word ((b*8 + rt)*8 + g)*2 + j // 4 holds each group's two kept positions, bits 0-1
#     the lower, bits 2-3 the higher (``_sparse_meta_place``).
# The kept rows of a group are its rows whose code is not 8, made up to two with the lowest
# remaining rows (code 8).


def _sparse_code_nibble(half: int, j: int, kept_index: int) -> int:
    """Nibble of a code word that holds kept code ``kept_index`` (0 lower, 1 higher row) of
    group j of the column in ``half``."""
    return half + 2 * (j >= 4) + 4 * kept_index


def _sparse_meta_place(b: int, rt: int, g: int, half: int, j: int):
    """(word, nibble) of the metadata of group j of column 16rt + 8half + g in 32-row block b."""
    return ((b * 8 + rt) * 8 + g) * 2 + j // 4, (j % 4) + 4 * half


def is_sparse24(q: np.ndarray) -> bool:
    """True when every run of 4 rows (4i .. 4i+3) of every column has at most 2 codes other than 8."""
    q = np.asarray(q)
    K, N = q.shape
    return K % 4 == 0 and bool(((q.reshape(K // 4, 4, N) != ZERO_POINT).sum(axis=1) <= 2).all())


def _kept_rows(col_group: np.ndarray):
    """The two kept positions (ascending) of a pruning group's 4 codes."""
    keep = [p for p in range(4) if col_group[p] != ZERO_POINT]
    for p in range(4):
        if len(keep) == 2:
            break
        if p not in keep:
            keep.append(p)
    return sorted(keep)


def prepacked_bytes_w4a16_sparse24(K: int, N: int, g: int) -> int:
    _check_kn(K, N)
    nt, kt = -(-N // TILE_N), K // TILE_K
    slots = _group_slots(K, g)
    blob = 4096 + 2048 + 2 * TILE_N * slots
    tail = 0 if slots else ((2 * nt * TILE_N + 15) // 16) * 16
    return nt * kt * blob + tail


def prepack_w4a16_sparse24(Q: np.ndarray, s: np.ndarray, g: int) -> np.ndarray:
    """The 2:4 sparse prepacked buffer as bytes, following the layout above (loops over the
    documented indices, one code at a time)."""
    q = unpack_codes(Q)
    K, N = q.shape
    if not is_sparse24(q):
        raise ValueError("not 2:4 sparse")
    slots = _group_slots(K, g)
    nt, kt = -(-N // TILE_N), K // TILE_K
    qp = np.full((K, nt * TILE_N), ZERO_POINT, dtype=np.uint8)
    qp[:, :N] = q
    blob_bytes = 4096 + 2048 + 2 * TILE_N * slots
    out = np.zeros(prepacked_bytes_w4a16_sparse24(K, N, g), dtype=np.uint8)
    sp = np.zeros((np.asarray(s).shape[0], nt * TILE_N), dtype=np.float16)
    sp[:, :N] = np.asarray(s, dtype=np.float16)
    for n_t in range(nt):
        for k_t in range(kt):
            codes = np.zeros(1024, dtype=np.uint32)
            meta = np.zeros(512, dtype=np.uint32)
            for c in range(TILE_N):
                col = n_t * TILE_N + c
                rt, gg, half = c // 16, c % 8, (c % 16) // 8
                for b in range(4):
                    for j in range(8):
                        r0 = k_t * TILE_K + 32 * b + 4 * j
                        keep = _kept_rows(qp[r0:r0 + 4, col])
                        w = (b * 8 + rt) * 32 + 4 * gg + j % 4
                        for ki, pos in enumerate(keep):
                            codes[w] |= np.uint32(int(qp[r0 + pos, col]) << (4 * _sparse_code_nibble(half, j, ki)))
                        mw, mn = _sparse_meta_place(b, rt, gg, half, j)
                        meta[mw] |= np.uint32((keep[0] | (keep[1] << 2)) << (4 * mn))
            start = (n_t * kt + k_t) * blob_bytes
            out[start:start + 4096] = codes.view(np.uint8)
            out[start + 4096:start + 6144] = meta.view(np.uint8)
            for u in range(slots):
                grp = (k_t * TILE_K + u * g) // g
                out[start + 6144 + 256 * u:start + 6144 + 256 * (u + 1)] = \
                    sp[grp, n_t * TILE_N:(n_t + 1) * TILE_N].view(np.uint8)
    if not slots:
        tail = nt * kt * blob_bytes
        out[tail:tail + 2 * nt * TILE_N] = sp[0].view(np.uint8)
    return out


def unprepack_w4a16_sparse24(Wp: np.ndarray, K: int, N: int, g: int):
    """Inverse of ``prepack_w4a16_sparse24``: ``(q[K,N] uint8, s[K/g, N] fp16)``, pruned rows as 8."""
    slots = _group_slots(K, g)
    nt, kt = -(-N // TILE_N), K // TILE_K
    Wp = np.asarray(Wp, dtype=np.uint8)
    blob_bytes = 4096 + 2048 + 2 * TILE_N * slots
    q = np.full((K, nt * TILE_N), ZERO_POINT, dtype=np.uint8)
    s = np.zeros((K // g, nt * TILE_N), dtype=np.float16)
    for n_t in range(nt):
        for k_t in range(kt):
            start = (n_t * kt + k_t) * blob_bytes
            codes = Wp[start:start + 4096].copy().view(np.uint32)
            meta = Wp[start + 4096:start + 6144].copy().view(np.uint32)
            for c in range(TILE_N):
                col = n_t * TILE_N + c
                rt, gg, half = c // 16, c % 8, (c % 16) // 8
                for b in range(4):
                    for j in range(8):
                        r0 = k_t * TILE_K + 32 * b + 4 * j
                        mw, mn = _sparse_meta_place(b, rt, gg, half, j)
                        m = (int(meta[mw]) >> (4 * mn)) & 0xF
                        w = (b * 8 + rt) * 32 + 4 * gg + j % 4
                        for ki, pos in enumerate((m & 3, m >> 2)):
                            q[r0 + pos, col] = (int(codes[w]) >> (4 * _sparse_code_nibble(half, j, ki))) & 0xF
            for u in range(slots):
                grp = (k_t * TILE_K + u * g) // g
                s[grp, n_t * TILE_N:(n_t + 1) * TILE_N] = \
                    Wp[start + 6144 + 256 * u:start + 6144 + 256 * (u + 1)].copy().view(np.float16)
    if not slots:
        tail = nt * kt * blob_bytes
        s = Wp[tail:tail + 2 * nt * TILE_N].copy().view(np.float16)[None, :]
    return q[:, :N], s[:, :N]


# --------------------------------------------------------------------------
# Mixed 2/4-bit weights
# --------------------------------------------------------------------------
# "Enabling Fast 2-bit LLM on GPUs: Memory Alignment and Asynchronous Dequantization", Abstract:
# most groups of weights are quantised to 2 bits and only the small fraction of groups with a
# large range to 4 bits, the 4-bit groups placed with the GPU's memory alignment in mind.
# Reading (the page gives no format): the bit width is chosen per aligned block of 32 rows
# (32i .. 32i+31) and 128 columns (the n-tile), ``widths[K/32, ceil(N/128)]`` in {2, 4}; a
# b-bit code q in 0 .. 2^b - 1 stands for q - 2^(b-1) (zero point 2 or 8) times the group
# scale, ``W[k,n] = (q[k,n] - z(k,n)) * s[k // g, n]``. Codes of every width travel in the usual
# 4-bit packing of Q.
MIXED_BLOCK_ROWS = 32


def mixed_zero_points(widths: np.ndarray, K: int, N: int) -> np.ndarray:
    """z[K, N]: 2 in 2-bit blocks, 8 in 4-bit blocks."""
    w = np.asarray(widths)
    if w.shape != (K // MIXED_BLOCK_ROWS, -(-N // TILE_N)) or not np.isin(w, (2, 4)).all():
        raise ValueError("widths must be [K/32, ceil(N/128)] with values 2 or 4")
    per = np.repeat(np.repeat(w, MIXED_BLOCK_ROWS, axis=0), TILE_N, axis=1)[:, :N]
    return np.where(per == 2, 2, 8).astype(np.int64)


def dequant_mixed(q: np.ndarray, s: np.ndarray, g: int, widths: np.ndarray) -> np.ndarray:
    """``W[k,n] = (q[k,n] - z[k,n]) * s[k // g, n]`` in float64, z from the block's width."""
    K, N = q.shape
    if K % g:
        raise ValueError("g must divide K")
    z = mixed_zero_points(widths, K, N)
    if (q.astype(np.int64) >= 2 * z).any():
        raise ValueError("a code does not fit its block's width")
    return (q.astype(np.float64) - z) * np.asarray(s, dtype=np.float64)[np.arange(K) // g, :]


def w4a16_mixed(A: np.ndarray, Q: np.ndarray, s: np.ndarray, g: int, widths: np.ndarray) -> np.ndarray:
    """``Y = A . W`` in float64 for mixed 2/4-bit weights."""
    return np.asarray(A, dtype=np.float64) @ dequant_mixed(unpack_codes(Q), s, g, widths)


def w4a16_mixed_absdot(A: np.ndarray, Q: np.ndarray, s: np.ndarray, g: int, widths: np.ndarray) -> np.ndarray:
    """``sum_k |A[m,k] * W[k,n]|`` for the tolerance of the mixed layer."""
    return np.abs(np.asarray(A, dtype=np.float64)) @ np.abs(dequant_mixed(unpack_codes(Q), s, g, widths))


# Prepacked mixed buffer (the library's own format):
#   a table of NT*KT + 1 uint32 entries (padded to 128 bytes): entry nt*KT + kt = (byte offset of
#     blob (nt, kt) / 16) << 4 | wbits, bit v of wbits set when 32-row block v of the blob is
#     4-bit; the last entry = (end of the blobs / 16) << 4;
#   for g == K the column scales (NT*128 fp16, padded to 16 bytes) right after the table;
#   then the blobs, nt-major: blocks v = 0..3 (rows 32v .. of the k-block), each 2048 bytes
#   (4-bit: word r*4 + i holds rows 32v + 8i + j of column r, code j at nibble
#   NIBBLE_POS_W4A16[j], as in the dense blob) or 1024 bytes (2-bit: word rt*32 + 4gc + t holds
#   rows 32v + 8t + r of columns 16rt + gc + 8j at the 2-bit field ``_mixed_field(r, j)``), then
#   the ``slots`` rows of 128 fp16 group scales.
def _mixed_field(r: int, j: int) -> int:
    """2-bit field (bits 2f, 2f+1 of the word) of row 8t + r of column 16rt + gc + 8j."""
    return r // 2 + 4 * j + 8 * (r % 2)


def _mixed_table_bytes(nblob: int) -> int:
    return ((nblob + 1) * 4 + 127) // 128 * 128


def prepacked_bytes_mixed(K: int, N: int, g: int, widths: np.ndarray) -> int:
    _check_kn(K, N)
    nt, kt = -(-N // TILE_N), K // TILE_K
    slots = _group_slots(K, g)
    w = np.asarray(widths)
    code = int(np.where(w == 4, 2048, 1024).sum())
    tail = 0 if slots else ((2 * nt * TILE_N + 15) // 16) * 16
    return _mixed_table_bytes(nt * kt) + tail + code + nt * kt * 2 * TILE_N * slots


def prepack_mixed(Q: np.ndarray, s: np.ndarray, g: int, widths: np.ndarray) -> np.ndarray:
    """The mixed 2/4-bit prepacked buffer as bytes, following the layout above (loops over the
    documented indices)."""
    q = unpack_codes(Q)
    K, N = q.shape
    dequant_mixed(q, np.zeros((K // g, N)), g, widths)  # checks the widths and the code ranges
    w = np.asarray(widths)
    slots = _group_slots(K, g)
    nt_n, kt_n = -(-N // TILE_N), K // TILE_K
    qp = np.full((K, nt_n * TILE_N), 0, dtype=np.uint8)
    qp[:, :N] = q
    for nt in range(nt_n):  # padded columns: the zero point of their block (weight 0)
        for b in range(K // MIXED_BLOCK_ROWS):
            if nt * TILE_N + TILE_N > N:
                qp[32 * b:32 * b + 32, max(N, nt * TILE_N):(nt + 1) * TILE_N] = 2 if w[b, nt] == 2 else 8
    sp = np.zeros((np.asarray(s).shape[0], nt_n * TILE_N), dtype=np.float16)
    sp[:, :N] = np.asarray(s, dtype=np.float16)
    nblob = nt_n * kt_n
    head = _mixed_table_bytes(nblob) + (0 if slots else ((2 * nt_n * TILE_N + 15) // 16) * 16)
    out = np.zeros(prepacked_bytes_mixed(K, N, g, w), dtype=np.uint8)
    table = np.zeros(nblob + 1, dtype=np.uint32)
    pos = head
    for nt in range(nt_n):
        for kt in range(kt_n):
            wbits = sum(1 << v for v in range(4) if w[4 * kt + v, nt] == 4)
            table[nt * kt_n + kt] = ((pos // 16) << 4) | wbits
            for v in range(4):
                r0 = kt * TILE_K + 32 * v
                if w[4 * kt + v, nt] == 4:
                    words = np.zeros(TILE_N * 4, dtype=np.uint32)
                    for r in range(TILE_N):
                        for i in range(4):
                            for j in range(8):
                                code = int(qp[r0 + 8 * i + j, nt * TILE_N + r])
                                words[r * 4 + i] |= np.uint32(code << (4 * NIBBLE_POS_W4A16[j]))
                else:
                    words = np.zeros(256, dtype=np.uint32)
                    for rt in range(8):
                        for gc in range(8):
                            for t in range(4):
                                for j in range(2):
                                    for r in range(8):
                                        code = int(qp[r0 + 8 * t + r, nt * TILE_N + 16 * rt + gc + 8 * j])
                                        words[rt * 32 + 4 * gc + t] |= np.uint32(code << (2 * _mixed_field(r, j)))
                out[pos:pos + words.nbytes] = words.view(np.uint8)
                pos += words.nbytes
            for u in range(slots):
                grp = (kt * TILE_K + u * g) // g
                out[pos:pos + 256] = sp[grp, nt * TILE_N:(nt + 1) * TILE_N].view(np.uint8)
                pos += 256
    table[nblob] = (pos // 16) << 4
    out[:table.nbytes] = table.view(np.uint8)
    if not slots:
        t0 = _mixed_table_bytes(nblob)
        out[t0:t0 + 2 * nt_n * TILE_N] = sp[0].view(np.uint8)
    assert pos == out.nbytes
    return out


def unprepack_mixed(Wp: np.ndarray, K: int, N: int, g: int):
    """Inverse of ``prepack_mixed``: ``(q[K,N] uint8, s[K/g, N] fp16, widths[K/32, NT] uint8)``."""
    Wp = np.asarray(Wp, dtype=np.uint8)
    slots = _group_slots(K, g)
    nt_n, kt_n = -(-N // TILE_N), K // TILE_K
    nblob = nt_n * kt_n
    table = Wp[:(nblob + 1) * 4].copy().view(np.uint32)
    q = np.zeros((K, nt_n * TILE_N), dtype=np.uint8)
    s = np.zeros((K // g, nt_n * TILE_N), dtype=np.float16)
    widths = np.zeros((K // MIXED_BLOCK_ROWS, nt_n), dtype=np.uint8)
    for nt in range(nt_n):
        for kt in range(kt_n):
            e = int(table[nt * kt_n + kt])
            pos, wbits = (e >> 4) * 16, e & 0xF
            for v in range(4):
                r0 = kt * TILE_K + 32 * v
                if (wbits >> v) & 1:
                    widths[4 * kt + v, nt] = 4
                    words = Wp[pos:pos + 2048].copy().view(np.uint32)
                    for r in range(TILE_N):
                        for i in range(4):
                            for j in range(8):
                                q[r0 + 8 * i + j, nt * TILE_N + r] = (int(words[r * 4 + i]) >> (4 * NIBBLE_POS_W4A16[j])) & 0xF
                    pos += 2048
                else:
                    widths[4 * kt + v, nt] = 2
                    words = Wp[pos:pos + 1024].copy().view(np.uint32)
                    for rt in range(8):
                        for gc in range(8):
                            for t in range(4):
                                for j in range(2):
                                    for r in range(8):
                                        q[r0 + 8 * t + r, nt * TILE_N + 16 * rt + gc + 8 * j] = \
                                            (int(words[rt * 32 + 4 * gc + t]) >> (2 * _mixed_field(r, j))) & 0x3
                    pos += 1024
            for u in range(slots):
                grp = (kt * TILE_K + u * g) // g
                s[grp, nt * TILE_N:(nt + 1) * TILE_N] = Wp[pos:pos + 256].copy().view(np.float16)
                pos += 256
    if not slots:
        t0 = _mixed_table_bytes(nblob)
        s = Wp[t0:t0 + 2 * nt_n * TILE_N].copy().view(np.float16)[None, :]
    return q[:, :N], s[:, :N], widths
