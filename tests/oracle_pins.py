"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each ``pin_*`` takes the oracle module (so that a test can hand it a copy with
a planted mistake) and raises ``AssertionError`` when the oracle disagrees
with the fact it is pinned to:

* hand-worked examples (``tests/golden``), exact in binary;
* exact rational brute force (``fractions.Fraction``) on tiny layers, using the
  raw codes from the generator rather than the oracle's unpacking;
* closed forms of special cases: identity activations reproduce the
  dequantised weights, all-8 codes give zero, all-0 codes give
  ``-8 * sum_k a_k s_k``;
* invariants: power-of-two scale homogeneity, row permutation, linearity;
* W4A8: the integer accumulator against Python integer loops;
* per-token activation quantisation: hand-worked rows (``tests/golden/act_quant.txt``)
  and exact rational bounds;
* asymmetric groups (zero points): hand-worked layers (``tests/golden/zp_examples.txt``),
  exact rational brute force, and zero point 8 reproducing the symmetric layer;
* act order (groups not contiguous along K): hand-worked layers, row orders and reordered
  words (``tests/golden/act_order_examples.txt``), exact rational brute force, contiguous
  groups reproducing the grouped layers, and the reordering identity the library relies on;
* the prepacked layout: single codes and scales placed by hand-worked byte
  offsets (``tests/golden/blob_layout.txt``), independent of the oracle's own
  inverse of its layout.
"""
from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np
import pytest

import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line


def golden_words():
    out = []
    for line in _rows("unpack_words.txt"):
        w, codes = line.split(":")
        out.append((int(w, 16), [int(c) for c in codes.split()]))
    return out


def golden_hand():
    out = []
    for line in _rows("hand_examples.txt"):
        kind, words, scales, g, acts, sasw, expect = [p.strip() for p in line.split("|")]
        words = [int(w, 16) for w in words.split()]
        out.append({
            "kind": kind,
            "Q": np.array(words, dtype=np.uint32).view(np.int32).reshape(-1, 1),
            "s": None if scales == "-" else np.array([float(x) for x in scales.split()], dtype=np.float16).reshape(-1, 1),
            "g": None if g == "-" else int(g),
            "A": np.array([float(x) for x in acts.split()]).reshape(1, -1),
            "sasw": None if sasw == "-" else [float(x) for x in sasw.split()],
            "expect": [float(x) for x in expect.split()],
        })
    return out


# ---------------------------------------------------------------- unpacking
def pin_unpack_golden(o):
    for word, codes in golden_words():
        Q = np.array([[word]], dtype=np.uint32).view(np.int32)
        got = o.unpack_codes(Q)[:, 0].tolist()
        assert got == codes, (hex(word), got, codes)


def pin_unpack_matches_generator(o):
    d = synth.w4a16_inputs(64, 24, 32, 1, seed=3)
    assert np.array_equal(o.unpack_codes(d["Q"]), d["q"])


# ---------------------------------------------------------------- W4A16
def pin_hand_examples(o):
    for ex in golden_hand():
        if ex["kind"] == "w4a16":
            A = ex["A"].astype(np.float16)
            y = o.w4a16(A, ex["Q"], ex["s"], ex["g"])
            assert y.shape == (1, 1)
            assert y[0, 0] == ex["expect"][0], (y, ex)
        else:
            A = ex["A"].astype(np.int8)
            sa = np.array([ex["sasw"][0]], np.float32)
            sw = np.array([ex["sasw"][1]], np.float32)
            acc, y = o.w4a8(A, sa, ex["Q"], sw)
            assert int(acc[0, 0]) == int(ex["expect"][1]), (acc, ex)
            assert y[0, 0] == ex["expect"][0], (y, ex)


def _exact_w4a16(A, q, s, g):
    M, K = A.shape
    N = q.shape[1]
    y = [[Fraction(0)] * N for _ in range(M)]
    for m in range(M):
        for n in range(N):
            acc = Fraction(0)
            for k in range(K):
                acc += Fraction(float(A[m, k])) * (int(q[k, n]) - 8) * Fraction(float(s[k // g, n]))
            y[m][n] = acc
    return y


def pin_bruteforce_w4a16(o):
    # M, K, N all different so that a transposed operand cannot pass
    for (M, K, N, g, seed) in [(3, 64, 5, 16, 1), (2, 48, 7, 48, 2), (4, 32, 3, 8, 3), (1, 128, 9, 32, 4)]:
        d = synth.w4a16_inputs(K, N, g, M, seed=seed)
        y = o.w4a16(d["A"], d["Q"], d["s"], g)
        assert y.shape == (M, N)
        ex = _exact_w4a16(d["A"], d["q"], d["s"], g)
        for m in range(M):
            for n in range(N):
                absdot = sum(abs(float(d["A"][m, k]) * (int(d["q"][k, n]) - 8) * float(d["s"][k // g, n]))
                             for k in range(K))
                err = abs(Fraction(float(y[m, n])) - ex[m][n])
                assert err <= Fraction(K * 2.0 ** -52 * absdot + 1e-300), (M, K, N, g, m, n, float(err))


def pin_absdot(o):
    d = synth.w4a16_inputs(64, 6, 16, 2, seed=5)
    got = o.w4a16_absdot(d["A"], d["Q"], d["s"], 16)
    for m in range(2):
        for n in range(6):
            ref = math.fsum(abs(float(d["A"][m, k]) * (int(d["q"][k, n]) - 8) * float(d["s"][k // 16, n]))
                            for k in range(64))
            assert abs(got[m, n] - ref) <= 1e-12 * ref
    y1, a1 = o.w4a16_entry(d["A"], d["Q"], d["s"], 16, 1, 4)
    assert abs(a1 - got[1, 4]) <= 1e-12 * got[1, 4]
    assert abs(y1 - o.w4a16(d["A"], d["Q"], d["s"], 16)[1, 4]) <= 1e-12 * a1


def pin_identity_activation(o):
    # A = I reproduces W exactly; W[k,n] = (q-8)*s written out per element
    for (K, N, g) in [(64, 5, 16), (32, 3, 32), (128, 2, 64)]:
        d = synth.w4a16_inputs(K, N, g, 1, seed=7)
        A = np.eye(K, dtype=np.float16)
        y = o.w4a16(A, d["Q"], d["s"], g)
        for k in range(K):
            for n in range(N):
                assert y[k, n] == (int(d["q"][k, n]) - 8) * float(d["s"][k // g, n]), (K, N, g, k, n)


def pin_all_eight(o):
    K, N, g = 64, 6, 16
    d = synth.w4a16_inputs(K, N, g, 3, seed=8)
    Q = synth.pack_q(np.full((K, N), 8, np.uint8))
    y = o.w4a16(d["A"], Q, d["s"], g)
    assert np.all(y == 0.0)


def pin_all_zero_codes(o):
    K, N, g = 64, 6, 16
    d = synth.w4a16_inputs(K, N, g, 3, seed=9)
    Q = synth.pack_q(np.zeros((K, N), np.uint8))
    y = o.w4a16(d["A"], Q, d["s"], g)
    for m in range(3):
        for n in range(N):
            ref = -8.0 * math.fsum(float(d["A"][m, k]) * float(d["s"][k // g, n]) for k in range(K))
            scale = 8.0 * math.fsum(abs(float(d["A"][m, k]) * float(d["s"][k // g, n])) for k in range(K))
            assert abs(y[m, n] - ref) <= K * 2.0 ** -52 * scale


def pin_scale_homogeneity(o):
    d = synth.w4a16_inputs(128, 10, 32, 4, seed=10)
    y1 = o.w4a16(d["A"], d["Q"], d["s"], 32)
    y2 = o.w4a16(d["A"], d["Q"], (d["s"].astype(np.float32) * 2).astype(np.float16), 32)
    assert np.array_equal(y2, 2 * y1)


def pin_row_permutation(o):
    d = synth.w4a16_inputs(128, 10, 32, 6, seed=11)
    perm = np.array([3, 0, 5, 1, 4, 2])
    y = o.w4a16(d["A"], d["Q"], d["s"], 32)
    yp = o.w4a16(d["A"][perm], d["Q"], d["s"], 32)
    ad = o.w4a16_absdot(d["A"], d["Q"], d["s"], 32)
    assert np.all(np.abs(yp - y[perm]) <= 128 * 2.0 ** -52 * ad[perm])


def pin_linearity(o):
    d = synth.w4a16_inputs(128, 10, 32, 4, seed=12)
    e = synth.w4a16_inputs(128, 10, 32, 4, seed=13)
    A1, A2 = d["A"].astype(np.float64), e["A"].astype(np.float64)
    y12 = o.w4a16(A1 + A2, d["Q"], d["s"], 32)
    y1 = o.w4a16(A1, d["Q"], d["s"], 32)
    y2 = o.w4a16(A2, d["Q"], d["s"], 32)
    ad = o.w4a16_absdot(np.abs(A1) + np.abs(A2), d["Q"], d["s"], 32)
    assert np.all(np.abs(y12 - (y1 + y2)) <= 4 * 128 * 2.0 ** -52 * ad)


def pin_tolerance_formula(o):
    y = np.array([1.0, -2.0, 0.0])
    ad = np.array([2.0, 0.5, 3.0])
    t = o.tolerance(y, ad)
    assert np.allclose(t, [2.0 ** -10 + 2e-3, 2.0 ** -9 + 5e-4, 3e-3], rtol=1e-15, atol=0)


# ---------------------------------------------------------------- W4A8
def pin_bruteforce_w4a8(o):
    for (M, K, N, seed) in [(3, 64, 5, 1), (2, 40, 7, 2), (5, 16, 3, 3)]:
        d = synth.w4a8_inputs(K, N, M, seed=seed)
        acc, y = o.w4a8(d["A"], d["sa"], d["Q"], d["sw"])
        assert acc.shape == (M, N) and acc.dtype == np.int64
        for m in range(M):
            for n in range(N):
                ref = sum(int(d["A"][m, k]) * (int(d["q"][k, n]) - 8) for k in range(K))
                assert int(acc[m, n]) == ref, (m, n)
                yex = Fraction(ref) * Fraction(float(d["sa"][m])) * Fraction(float(d["sw"][n]))
                assert abs(Fraction(float(y[m, n])) - yex) <= abs(yex) * Fraction(2.0 ** -51)
        ad = o.w4a8_absdot(d["A"], d["sa"], d["Q"], d["sw"])
        for m in range(M):
            for n in range(N):
                ref = sum(abs(int(d["A"][m, k]) * (int(d["q"][k, n]) - 8)) for k in range(K))
                exp = ref * float(d["sa"][m]) * float(d["sw"][n])
                assert abs(ad[m, n] - exp) <= 1e-12 * max(exp, 1e-30)


def pin_w4a8_extremes(o):
    # the largest accumulator magnitude: a = -127 everywhere, all codes 0 -> 8*127*K
    K, N = 1024, 3
    A = np.full((1, K), -127, np.int8)
    Q = synth.pack_q(np.zeros((K, N), np.uint8))
    acc = o.w4a8_acc(A, Q)
    assert np.all(acc == 8 * 127 * K)
    Q = synth.pack_q(np.full((K, N), 15, np.uint8))
    assert np.all(o.w4a8_acc(A, Q) == -7 * 127 * K)


# ---------------------------------------------------------------- prepacked layout
def golden_layout():
    out = []
    for line in _rows("blob_layout.txt"):
        parts = [p.strip() for p in line.split("|")]
        kind, what = parts[0].split()
        dims = parts[1].split()
        K, N = int(dims[0]), int(dims[1])
        g = None if dims[2] == "-" else int(dims[2])
        a, b = (int(x) for x in parts[2].split())
        offs = [int(x) for x in parts[3].split()]
        half = parts[4] if len(parts) > 4 else None
        out.append((kind, what, K, N, g, a, b, offs, half))
    return out


# a scale bit pattern whose two bytes are both non-zero and different
_SCALE_BITS = 0x4A3C


def pin_blob_layout_golden(o):
    # one code (value 3 among 8s) or one scale (among zeros) at a time: exactly the bytes the
    # hand-worked table names change, to exactly the values it implies
    for kind, what, K, N, g, a, b, offs, half in golden_layout():
        if what == "zero":
            q = np.full((K, N), 8, np.uint8)
            s = np.zeros((K // g, N), np.float16)
            z = np.full((K // g, N), 8, np.uint8)
            base = o.prepack_w4a16_zp(synth.pack_q(q), s, z, g)
            z[a, b] = 3
            Wp = o.prepack_w4a16_zp(synth.pack_q(q), s, z, g)
            diff = np.nonzero(Wp != base)[0].tolist()
            assert diff == offs, (K, N, g, a, b, diff, offs)
            assert all(int(Wp[x]) == 3 for x in offs)
            continue
        if what == "code":
            q = np.full((K, N), 8, np.uint8)
            base_q = q.copy()
            q[a, b] = 3
            if kind == "w4a16":
                s = np.zeros((K // g, N), np.float16)
                Wp, base = o.prepack_w4a16(synth.pack_q(q), s, g), o.prepack_w4a16(synth.pack_q(base_q), s, g)
            elif kind == "w4a16zp":
                s = np.zeros((K // g, N), np.float16)
                z = np.full((K // g, N), 8, np.uint8)
                Wp, base = o.prepack_w4a16_zp(synth.pack_q(q), s, z, g), o.prepack_w4a16_zp(synth.pack_q(base_q), s, z, g)
            else:
                Wp, base = o.prepack_w4a8(synth.pack_q(q)), o.prepack_w4a8(synth.pack_q(base_q))
            diff = np.nonzero(Wp != base)[0].tolist()
            assert diff == offs, (kind, K, N, g, a, b, diff, offs)
            want = 0x83 if half == "lo" else 0x38
            assert int(Wp[offs[0]]) == want, (kind, a, b, hex(int(Wp[offs[0]])))
        else:
            q = np.full((K, N), 8, np.uint8)
            s = np.zeros((K // g, N), np.float16)
            base = o.prepack_w4a16(synth.pack_q(q), s, g)
            s[a, b] = np.array([_SCALE_BITS], np.uint16).view(np.float16)[0]
            Wp = o.prepack_w4a16(synth.pack_q(q), s, g)
            diff = np.nonzero(Wp != base)[0].tolist()
            assert diff == sorted(x for off in offs for x in (off, off + 1)), (K, N, g, a, b, diff, offs)
            for off in offs:
                assert int(Wp[off]) | (int(Wp[off + 1]) << 8) == _SCALE_BITS


# ---------------------------------------------------------------- per-token activation quantisation
def golden_act_quant(bits=8):
    out = []
    for line in _rows("act_quant.txt"):
        parts = [x.strip() for x in line.split("|")]
        row_bits = 8
        if parts[0].startswith("bits="):
            row_bits = int(parts[0][5:])
            parts = parts[1:]
        if row_bits != bits:
            continue
        acts, codes, sa = parts
        out.append((np.array([float(x) for x in acts.split()], np.float16),
                    [int(x) for x in codes.split()], None if sa == "-" else float(sa)))
    return out


def pin_act_quant_golden(o):
    for bits in (8, 4):
        rows = golden_act_quant(bits)
        assert rows
        q, sa = o.quantize_act(np.stack([r[0] for r in rows]), bits=bits)
        assert q.dtype == np.int8 and sa.dtype == np.float32
        for i, (a, codes, s) in enumerate(rows):
            assert q[i].tolist() == codes, (bits, i, q[i].tolist(), codes)
            if s is not None:
                assert float(sa[i]) == s, (bits, i, float(sa[i]), s)


def pin_act_quant_bounds(o):
    # against exact rational arithmetic: each code is within 1/2 (plus the two fp32 roundings)
    # of a * 127 / max|a|, never beyond +-127, equal to +-127 at the row's largest magnitude,
    # of the activation's sign; and sa is max|a| / 127 to fp32 precision
    rng = np.random.default_rng(4)
    A = (rng.standard_normal((6, 96)) * np.array([[1e-3], [1.0], [30.0], [1e3], [0.5], [7.0]])).astype(np.float16)
    A[4, :] = 0
    A[4, 17] = -0.25
    for bits, L in ((8, 127), (4, 7)):
        q, sa = o.quantize_act(A, bits=bits)
        for m in range(A.shape[0]):
            amax = max(abs(Fraction(float(x))) for x in A[m])
            assert abs(Fraction(float(sa[m])) - amax / L) <= amax / L * Fraction(2.0 ** -24)
            for k in range(A.shape[1]):
                a = Fraction(float(A[m, k]))
                exact = a * L / amax
                assert abs(int(q[m, k])) <= L
                assert abs(Fraction(int(q[m, k])) - exact) <= Fraction(1, 2) + 2 * L * Fraction(2.0 ** -24), (bits, m, k)
                if abs(a) == amax:
                    assert abs(int(q[m, k])) == L
                if q[m, k] != 0:
                    assert (q[m, k] > 0) == (a > 0)


# ---------------------------------------------------------------- asymmetric groups (zero points)
def golden_zp():
    out = []
    for line in _rows("zp_examples.txt"):
        words, scales, zeros, g, acts, expect = [p.strip() for p in line.split("|")]
        out.append({"Q": np.array([int(w, 16) for w in words.split()], np.uint32).view(np.int32).reshape(-1, 1),
                    "s": np.array([float(x) for x in scales.split()], np.float16).reshape(-1, 1),
                    "z": np.array([int(x) for x in zeros.split()], np.uint8).reshape(-1, 1),
                    "g": int(g), "A": np.array([float(x) for x in acts.split()], np.float16).reshape(1, -1),
                    "y": float(expect)})
    return out


def pin_zp_golden(o):
    for ex in golden_zp():
        y = o.w4a16_zp(ex["A"], ex["Q"], ex["s"], ex["z"], ex["g"])
        assert y.shape == (1, 1) and y[0, 0] == ex["y"], (y, ex["y"])


def pin_zp_bruteforce(o):
    # exact rationals from the raw codes and zeros of the generator, M, K, N all different
    for (M, K, N, g, seed) in [(3, 64, 5, 16, 1), (2, 48, 7, 48, 2), (1, 128, 9, 32, 4)]:
        d = synth.w4a16_inputs(K, N, g, M, seed=seed)
        z = np.random.default_rng(seed + 100).integers(0, 16, (K // g, N)).astype(np.uint8)
        y = o.w4a16_zp(d["A"], d["Q"], d["s"], z, g)
        ad = o.w4a16_zp_absdot(d["A"], d["Q"], d["s"], z, g)
        assert y.shape == (M, N)
        for m in range(M):
            for n in range(N):
                exact = Fraction(0)
                absdot = Fraction(0)
                for k in range(K):
                    t = Fraction(float(d["A"][m, k])) * (int(d["q"][k, n]) - int(z[k // g, n])) * Fraction(float(d["s"][k // g, n]))
                    exact += t
                    absdot += abs(t)
                assert abs(Fraction(float(y[m, n])) - exact) <= Fraction(K * 2.0 ** -52) * absdot + Fraction(1e-300)
                assert abs(Fraction(float(ad[m, n])) - absdot) <= Fraction(K * 2.0 ** -52) * absdot + Fraction(1e-300)


def pin_zp_eight_is_symmetric(o):
    # zero point 8 everywhere is the symmetric layer, bit for bit
    d = synth.w4a16_inputs(256, 40, 64, 3, seed=14)
    z = np.full((4, 40), 8, np.uint8)
    assert np.array_equal(o.w4a16_zp(d["A"], d["Q"], d["s"], z, 64), o.w4a16(d["A"], d["Q"], d["s"], 64))


# ---------------------------------------------------------------- act order
def golden_act_order(kind):
    out = []
    for line in _rows("act_order_examples.txt"):
        parts = [p.strip() for p in line.split("|")]
        if parts[0] != kind:
            continue
        if kind == "layer":
            words, scales, zeros, gidx, acts, expect = parts[1:]
            out.append({"Q": np.array([int(w, 16) for w in words.split()], np.uint32).view(np.int32).reshape(-1, 1),
                        "s": np.array([float(x) for x in scales.split()], np.float16).reshape(-1, 1),
                        "z": None if zeros == "-" else np.array([int(x) for x in zeros.split()], np.uint8).reshape(-1, 1),
                        "g_idx": np.array([int(x) for x in gidx.split()]),
                        "A": np.array([float(x) for x in acts.split()], np.float16).reshape(1, -1),
                        "y": float(expect)})
        elif kind == "perm":
            g, gidx, perm = parts[1:]
            out.append((int(g), np.array([int(x) for x in gidx.split()]), [int(x) for x in perm.split()]))
        else:
            words, perm, expect = parts[1:]
            out.append((np.array([int(w, 16) for w in words.split()], np.uint32).view(np.int32).reshape(-1, 1),
                        np.array([int(x) for x in perm.split()]), [int(w, 16) for w in expect.split()]))
    return out


def pin_act_order_golden(o):
    for ex in golden_act_order("layer"):
        y = o.w4a16_gidx(ex["A"], ex["Q"], ex["s"], ex["z"], ex["g_idx"])
        assert y.shape == (1, 1) and y[0, 0] == ex["y"], (y, ex["y"])
    for g, gidx, perm in golden_act_order("perm"):
        assert o.act_order_perm(gidx, g).tolist() == perm
    for Q, perm, words in golden_act_order("reorder"):
        assert o.reorder_rows(Q, perm).view(np.uint32)[:, 0].tolist() == words


def pin_act_order_unequal_groups_refused(o):
    for g, gidx in [(2, [0, 0, 0, 1]), (2, [0, 1, 2, 2]), (3, [0, 0, 1, 1])]:
        try:
            o.act_order_perm(np.array(gidx), g)
        except ValueError:
            continue
        raise AssertionError(f"g_idx {gidx} with g = {g} has no contiguous order but was accepted")


def _random_gidx(rng, K, g):
    return rng.permutation(np.arange(K) // g)


def pin_act_order_bruteforce(o):
    # exact rationals from the raw codes of the generator; groups scattered at random along K
    for (M, K, N, g, zp, seed) in [(3, 64, 5, 16, True, 1), (2, 48, 7, 8, False, 2), (1, 128, 9, 32, True, 4)]:
        d = synth.w4a16_inputs(K, N, g, M, seed=seed)
        rng = np.random.default_rng(seed + 200)
        gidx = _random_gidx(rng, K, g)
        z = rng.integers(0, 16, (K // g, N)).astype(np.uint8) if zp else None
        y = o.w4a16_gidx(d["A"], d["Q"], d["s"], z, gidx)
        ad = o.w4a16_gidx_absdot(d["A"], d["Q"], d["s"], z, gidx)
        assert y.shape == (M, N)
        for m in range(M):
            for n in range(N):
                exact = Fraction(0)
                absdot = Fraction(0)
                for k in range(K):
                    zk = 8 if z is None else int(z[gidx[k], n])
                    t = Fraction(float(d["A"][m, k])) * (int(d["q"][k, n]) - zk) * Fraction(float(d["s"][gidx[k], n]))
                    exact += t
                    absdot += abs(t)
                assert abs(Fraction(float(y[m, n])) - exact) <= Fraction(K * 2.0 ** -52) * absdot + Fraction(1e-300)
                assert abs(Fraction(float(ad[m, n])) - absdot) <= Fraction(K * 2.0 ** -52) * absdot + Fraction(1e-300)


def pin_act_order_contiguous_is_grouped(o):
    # g_idx = k // g is the grouped layer, bit for bit (same weights, same product)
    d = synth.w4a16_inputs(256, 40, 64, 3, seed=15)
    z = np.random.default_rng(15).integers(0, 16, (4, 40)).astype(np.uint8)
    gidx = np.arange(256) // 64
    assert np.array_equal(o.w4a16_gidx(d["A"], d["Q"], d["s"], z, gidx), o.w4a16_zp(d["A"], d["Q"], d["s"], z, 64))
    assert np.array_equal(o.w4a16_gidx(d["A"], d["Q"], d["s"], None, gidx), o.w4a16(d["A"], d["Q"], d["s"], 64))


def pin_act_order_reordering_identity(o):
    # taking the weight's rows and the activations' columns in the order perm turns scattered
    # groups into contiguous ones and leaves y unchanged (up to the order of the fp64 sums)
    for (M, K, N, g, zp, seed) in [(4, 512, 24, 128, True, 21), (3, 256, 16, 32, False, 22), (2, 384, 8, 64, True, 23)]:
        d = synth.w4a16_inputs(K, N, g, M, seed=seed)
        rng = np.random.default_rng(seed)
        gidx = _random_gidx(rng, K, g)
        z = rng.integers(0, 16, (K // g, N)).astype(np.uint8) if zp else None
        perm = o.act_order_perm(gidx, g)
        assert sorted(perm.tolist()) == list(range(K))
        assert np.array_equal(gidx[perm], np.arange(K) // g)
        y = o.w4a16_gidx(d["A"], d["Q"], d["s"], z, gidx)
        ad = o.w4a16_gidx_absdot(d["A"], d["Q"], d["s"], z, gidx)
        Qr = o.reorder_rows(d["Q"], perm)
        assert np.array_equal(o.unpack_codes(Qr), d["q"][perm])
        Ar = d["A"][:, perm]
        yr = o.w4a16(Ar, Qr, d["s"], g) if z is None else o.w4a16_zp(Ar, Qr, d["s"], z, g)
        assert np.all(np.abs(yr - y) <= 1e-12 * ad)


def pin_pack_codes(o):
    d = synth.w4a16_inputs(64, 12, 64, 1, seed=16)
    assert np.array_equal(o.pack_codes(d["q"]), d["Q"])
    assert np.array_equal(o.pack_codes(o.unpack_codes(d["Q"])), d["Q"])


# ---------------------------------------------------------------- 2:4 sparse prepacked layout
def golden_sparse24():
    out = []
    for line in _rows("sparse24_layout.txt"):
        parts = [p.strip() for p in line.split("|")]
        K, N, g = (int(x) for x in parts[1].split())
        a, b = (int(x) for x in parts[2].split())
        offs = [int(x) for x in parts[3].split()]
        vals = [int(x, 16) for x in parts[4].split()] if len(parts) > 4 else None
        out.append((parts[0], K, N, g, a, b, offs, vals))
    return out


def pin_sparse24_layout_golden(o):
    # one code 3 among 8s (its code byte and, where the kept rows move, its metadata byte) or one
    # scale among zeros: exactly the bytes the hand-worked table names change, to its values
    bases = {}
    for what, K, N, g, a, b, offs, vals in golden_sparse24():
        q = np.full((K, N), 8, np.uint8)
        s = np.zeros((K // g, N), np.float16)
        if (K, N, g) not in bases:
            bases[K, N, g] = o.prepack_w4a16_sparse24(synth.pack_q(q), s, g)
        base = bases[K, N, g]
        assert np.all(base[:4096] == 0x88) and np.all(base[4096:6144] == 0x44)
        if what == "code":
            q[a, b] = 3
            Wp = o.prepack_w4a16_sparse24(synth.pack_q(q), s, g)
            diff = np.nonzero(Wp != base)[0].tolist()
            assert diff == offs, (K, N, g, a, b, diff, offs)
            assert [int(Wp[x]) for x in offs] == vals, (a, b, [hex(int(Wp[x])) for x in offs])
        else:
            s[a, b] = np.array([_SCALE_BITS], np.uint16).view(np.float16)[0]
            Wp = o.prepack_w4a16_sparse24(synth.pack_q(q), s, g)
            diff = np.nonzero(Wp != base)[0].tolist()
            assert diff == sorted(x for off in offs for x in (off, off + 1)), (K, N, g, a, b, diff, offs)
            for off in offs:
                assert int(Wp[off]) | (int(Wp[off + 1]) << 8) == _SCALE_BITS


def pin_sparse24_two_kept_codes(o):
    # both kept rows of one group non-zero, at positions 2 and 3 (the worked example's column
    # and group): nibble 2 (byte 3157, low half) takes pos 2, nibble 6 (byte 3159) pos 3;
    # metadata 2 | 3 << 2
    q = np.full((384, 296), 8, np.uint8)
    q[118, 5], q[119, 5] = 5, 3
    s = np.zeros((3, 296), np.float16)
    Wp = o.prepack_w4a16_sparse24(synth.pack_q(q), s, 128)
    base = o.prepack_w4a16_sparse24(synth.pack_q(np.full((384, 296), 8, np.uint8)), s, 128)
    assert np.nonzero(Wp != base)[0].tolist() == [3157, 3159, 5676]
    assert [int(Wp[x]) for x in (3157, 3159, 5676)] == [0x85, 0x83, 0xE4]


def pin_sparse24_definition(o):
    # is_sparse24 against its definition, brute force over every 4-row pattern of one column
    for bits in range(16):
        q = np.full((8, 1), 8, np.uint8)
        for p in range(4):
            if bits >> p & 1:
                q[4 + p, 0] = 1 + p
        assert o.is_sparse24(q) == (bin(bits).count("1") <= 2)
    assert not o.is_sparse24(np.full((6, 1), 8, np.uint8))  # K not a multiple of 4
    q = np.full((128, 8), 8, np.uint8)
    q[0:3, 2] = 1
    with pytest.raises(ValueError):
        o.prepack_w4a16_sparse24(synth.pack_q(q), np.zeros((1, 8), np.float16), 128)
    d = synth.w4a16_sparse24_inputs(256, 24, 64, 1, seed=3)
    nz = (d["q"].reshape(64, 4, 24) != 8).sum(axis=1)
    assert o.is_sparse24(d["q"]) and nz.max() <= 2


# ---------------------------------------------------------------- mixed 2/4-bit weights
MIXED_GOLDEN_WIDTHS = np.array([[2, 4], [4, 4], [2, 4], [2, 4], [2, 2], [2, 2], [2, 2], [2, 4]], np.uint8)


def golden_mixed():
    out = []
    for line in _rows("mixed_layout.txt"):
        parts = [p.strip() for p in line.split("|")]
        K, N, g = (int(x) for x in parts[1].split())
        ab = None if parts[2] == "-" else tuple(int(x) for x in parts[2].split())
        offs = [int(x) for x in parts[3].split()]
        vals = parts[4].split() if len(parts) > 4 else None
        out.append((parts[0], K, N, g, ab, offs, vals))
    return out


def pin_mixed_layout_golden(o):
    # the blob table, one code 3 among codes at their zero points, or one scale among zeros:
    # exactly the bytes and values the hand-worked table names
    W = MIXED_GOLDEN_WIDTHS
    bases = {}
    for what, K, N, g, ab, offs, vals in golden_mixed():
        z = o.mixed_zero_points(W, K, N).astype(np.uint8)
        s = np.zeros((K // g, N), np.float16)
        if (K, N, g) not in bases:
            bases[K, N, g] = o.prepack_mixed(synth.pack_q(z), s, g, W)
        base = bases[K, N, g]
        if what == "table":
            assert base[:4 * len(offs)].view(np.uint32).tolist() == [int(v) for v in vals]
            continue
        q = z.copy()
        if what == "code":
            q[ab] = 3
        else:
            s[ab] = np.array([_SCALE_BITS], np.uint16).view(np.float16)[0]
        Wp = o.prepack_mixed(synth.pack_q(q), s, g, W)
        diff = np.nonzero(Wp != base)[0].tolist()
        if what == "code":
            assert diff == offs, (K, N, g, ab, diff, offs)
            assert [int(Wp[x]) for x in offs] == [int(v, 16) for v in vals], (ab, [hex(int(Wp[x])) for x in offs])
        else:
            assert diff == sorted(x for off in offs for x in (off, off + 1)), (K, N, g, ab, diff, offs)
            for off in offs:
                assert int(Wp[off]) | (int(Wp[off + 1]) << 8) == _SCALE_BITS


def pin_mixed_all_four_bit_is_w4a16(o):
    # every block 4-bit: the layer is w4a16 bit for bit, and each blob is the dense blob
    d = synth.w4a16_inputs(256, 200, 64, 3, seed=17)
    W4 = np.full((256 // 32, 2), 4, np.uint8)
    assert np.array_equal(o.w4a16_mixed(d["A"], d["Q"], d["s"], 64, W4), o.w4a16(d["A"], d["Q"], d["s"], 64))
    mixed = o.prepack_mixed(d["Q"], d["s"], 64, W4)
    dense = o.prepack_w4a16(d["Q"], d["s"], 64)
    head = (4 * (2 * 2 + 1) + 127) // 128 * 128
    assert np.array_equal(mixed[head:], dense)


def pin_mixed_bruteforce(o):
    # exact rational sums on a tiny mixed case (one block of each width per column tile)
    rng = np.random.default_rng(19)
    K, N, g, M = 64, 8, 32, 2
    W = np.array([[2], [4]], np.uint8)
    q = np.vstack([rng.integers(0, 4, (32, N)), rng.integers(0, 16, (32, N))]).astype(np.uint8)
    s = (0.01 + 0.02 * rng.random((K // g, N))).astype(np.float16)
    A = rng.standard_normal((M, K)).astype(np.float16)
    y = o.w4a16_mixed(A, synth.pack_q(q), s, g, W)
    for m in range(M):
        for n in range(N):
            ex = sum(Fraction(float(A[m, k])) * (int(q[k, n]) - (2 if k < 32 else 8)) * Fraction(float(s[k // g, n]))
                     for k in range(K))
            assert abs(Fraction(y[m, n]) - ex) <= abs(ex) * Fraction(1, 2 ** 40) + Fraction(1, 2 ** 60)


def pin_mixed_two_bit_closed_form(o):
    # every block 2-bit and every code 0: W = -2 s, so y = -2 sum_k a_k s[k // g]
    d = synth.w4a16_inputs(128, 24, 32, 2, seed=23)
    W2 = np.full((4, 1), 2, np.uint8)
    y = o.w4a16_mixed(d["A"], synth.pack_q(np.zeros((128, 24), np.uint8)), d["s"], 32, W2)
    want = -2.0 * (d["A"].astype(np.float64) @ d["s"].astype(np.float64)[np.arange(128) // 32])
    assert np.allclose(y, want, rtol=1e-12, atol=1e-12)
    with pytest.raises(ValueError):  # a 2-bit block holds codes 0..3 only
        q = np.zeros((128, 24), np.uint8)
        q[5, 3] = 4
        o.w4a16_mixed(d["A"], synth.pack_q(q), d["s"], 32, W2)
    with pytest.raises(ValueError):  # widths are 2 or 4
        o.w4a16_mixed(d["A"], d["Q"], d["s"], 32, np.full((4, 1), 3, np.uint8))


ALL_PINS = [
    pin_unpack_golden, pin_unpack_matches_generator, pin_hand_examples, pin_bruteforce_w4a16,
    pin_absdot, pin_identity_activation, pin_all_eight, pin_all_zero_codes, pin_scale_homogeneity,
    pin_row_permutation, pin_linearity, pin_tolerance_formula, pin_bruteforce_w4a8, pin_w4a8_extremes,
    pin_blob_layout_golden, pin_act_quant_golden, pin_act_quant_bounds, pin_zp_golden, pin_zp_bruteforce,
    pin_zp_eight_is_symmetric, pin_act_order_golden, pin_act_order_unequal_groups_refused,
    pin_act_order_bruteforce, pin_act_order_contiguous_is_grouped, pin_act_order_reordering_identity,
    pin_pack_codes, pin_sparse24_layout_golden, pin_sparse24_two_kept_codes, pin_sparse24_definition,
    pin_mixed_layout_golden, pin_mixed_all_four_bit_is_w4a16, pin_mixed_bruteforce, pin_mixed_two_bit_closed_form,
]
