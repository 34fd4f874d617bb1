"""CPU tests of the oracle: its pins, its prepack-layout restatement, and that the pins catch planted mistakes."""
import numpy as np
import pytest

import oracle
import synth
from oracle import wq_oracle as O

from oracle_pins import ALL_PINS, pin_blob_layout_golden, pin_mixed_layout_golden, pin_sparse24_layout_golden



@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(O)


# ------------------------------------------------------------ planted mistakes
def _mut_zero_point(mp):
    mp.setattr(O, "ZERO_POINT", 7)


def _mut_group_mod(mp):
    def dequant(q, s, g):
        K = q.shape[0]
        G = np.asarray(s).shape[0]
        return (q.astype(np.float64) - 8) * np.asarray(s, np.float64)[np.arange(K) % G, :]
    mp.setattr(O, "dequant", dequant)


def _mut_group_off_by_one(mp):
    def dequant(q, s, g):
        K = q.shape[0]
        G = np.asarray(s).shape[0]
        return (q.astype(np.float64) - 8) * np.asarray(s, np.float64)[(np.arange(K) // g + 1) % G, :]
    mp.setattr(O, "dequant", dequant)


def _mut_scale_dropped(mp):
    mp.setattr(O, "dequant", lambda q, s, g: q.astype(np.float64) - 8)


def _mut_nibbles_reversed(mp):
    def unpack_codes(Q):
        Qu = np.asarray(Q).view(np.uint32)
        K8, N = Qu.shape
        q = np.empty((K8, 8, N), np.uint8)
        for j in range(8):
            q[:, j, :] = (Qu >> np.uint32(4 * (7 - j))) & np.uint32(15)
        return q.reshape(K8 * 8, N)
    mp.setattr(O, "unpack_codes", unpack_codes)


def _mut_k_reversed(mp):
    orig = O._w_columns
    mp.setattr(O, "_w_columns", lambda Q, s, g, n0, n1: orig(Q, s, g, n0, n1)[::-1])


def _mut_sign_flipped(mp):
    mp.setattr(O, "dequant", lambda q, s, g: (8 - q.astype(np.float64)) *
               np.asarray(s, np.float64)[np.arange(q.shape[0]) // g, :])


def _mut_w4a8_no_zero_point(mp):
    def w4a8_acc(A, Q, chunk=4096):
        return (np.asarray(A, np.float64) @ O.unpack_codes(Q).astype(np.float64)).astype(np.int64)
    mp.setattr(O, "w4a8_acc", w4a8_acc)


def _mut_w4a8_sw_dropped(mp):
    def w4a8(A, sa, Q, sw):
        acc = O.w4a8_acc(A, Q)
        return acc, acc.astype(np.float64) * np.asarray(sa, np.float64)[:, None]
    mp.setattr(O, "w4a8", w4a8)


def _mut_absdot_signed(mp):
    def absdot(A, Q, s, g, chunk=4096):
        return np.abs(np.asarray(A, np.float64)) @ O.dequant(O.unpack_codes(Q), s, g)
    mp.setattr(O, "w4a16_absdot", absdot)


def _mut_tolerance_rel_dropped(mp):
    mp.setattr(O, "tolerance", lambda y, ad: 1e-3 * ad)


def _mut_act_round_half_up(mp):
    orig = O.quantize_act

    def quantize_act(A, bits=8):
        A32 = np.asarray(A, np.float16).astype(np.float32)
        amax = np.max(np.abs(A32), axis=1)
        q = np.zeros(A32.shape, np.int8)
        sa = np.zeros(A32.shape[0], np.float32)
        L = np.float32(2 ** (bits - 1) - 1)
        for m in range(A32.shape[0]):
            if amax[m]:
                t = A32[m] * (L / amax[m])
                q[m] = np.clip(np.floor(t + np.float32(0.5)), -L, L).astype(np.int8)
                sa[m] = amax[m] / L
        return q, sa
    del orig
    mp.setattr(O, "quantize_act", quantize_act)


def _mut_act_range_128(mp):
    def quantize_act(A, bits=8):
        A32 = np.asarray(A, np.float16).astype(np.float32)
        amax = np.max(np.abs(A32), axis=1)
        q = np.zeros(A32.shape, np.int8)
        sa = np.zeros(A32.shape[0], np.float32)
        for m in range(A32.shape[0]):
            if amax[m]:
                q[m] = np.clip(np.rint(A32[m] * (np.float32(128.0) / amax[m])), -128, 127).astype(np.int8)
                sa[m] = amax[m] / np.float32(128.0)
        return q, sa
    mp.setattr(O, "quantize_act", quantize_act)


def _mut_act_scale_per_tensor(mp):
    def quantize_act(A, bits=8):
        A32 = np.asarray(A, np.float16).astype(np.float32)
        amax = np.float32(np.max(np.abs(A32)))
        if amax == 0:
            return np.zeros(A32.shape, np.int8), np.zeros(A32.shape[0], np.float32)
        q = np.clip(np.rint(A32 * (np.float32(127.0) / amax)), -127, 127).astype(np.int8)
        return q, np.full(A32.shape[0], amax / np.float32(127.0), np.float32)
    mp.setattr(O, "quantize_act", quantize_act)


def _mut_act_4bit_8_levels(mp):
    orig = O.quantize_act

    def quantize_act(A, bits=8):
        if bits == 8:
            return orig(A, 8)
        A32 = np.asarray(A, np.float16).astype(np.float32)
        amax = np.max(np.abs(A32), axis=1)
        q = np.zeros(A32.shape, np.int8)
        sa = np.zeros(A32.shape[0], np.float32)
        for m in range(A32.shape[0]):
            if amax[m]:
                q[m] = np.clip(np.rint(A32[m] * (np.float32(8.0) / amax[m])), -8, 7).astype(np.int8)
                sa[m] = amax[m] / np.float32(8.0)
        return q, sa
    mp.setattr(O, "quantize_act", quantize_act)


def _mut_zp_ignored(mp):
    mp.setattr(O, "dequant_zp", lambda q, s, z, g: O.dequant(q, s, g))


def _mut_zp_sign(mp):
    def dequant_zp(q, s, z, g):
        grp = np.arange(q.shape[0]) // g
        return (q.astype(np.float64) + np.asarray(z, np.float64)[grp, :] - 16) * np.asarray(s, np.float64)[grp, :]
    mp.setattr(O, "dequant_zp", dequant_zp)


def _mut_gidx_ignored(mp):
    def dequant_gidx(q, s, z, g_idx):  # groups read as contiguous runs instead of g_idx
        G = np.asarray(s).shape[0]
        grp = np.arange(q.shape[0]) // (q.shape[0] // G)
        zz = 8 if z is None else np.asarray(z, np.float64)[grp, :]
        return (q.astype(np.float64) - zz) * np.asarray(s, np.float64)[grp, :]
    mp.setattr(O, "dequant_gidx", dequant_gidx)


def _mut_gidx_zero_contiguous(mp):
    def dequant_gidx(q, s, z, g_idx):  # the scale follows g_idx, the zero point does not
        G = np.asarray(s).shape[0]
        grp = np.arange(q.shape[0]) // (q.shape[0] // G)
        zz = 8 if z is None else np.asarray(z, np.float64)[grp, :]
        return (q.astype(np.float64) - zz) * np.asarray(s, np.float64)[np.asarray(g_idx), :]
    mp.setattr(O, "dequant_gidx", dequant_gidx)


def _mut_perm_inverse(mp):
    real = O.act_order_perm
    mp.setattr(O, "act_order_perm", lambda g_idx, g: np.argsort(real(g_idx, g)))


def _mut_reorder_within_word(mp):
    def reorder_rows(Q, perm):  # the order applied to whole words, codes kept inside them
        q = O.unpack_codes(Q)
        return O.pack_codes(q.reshape(-1, 8, q.shape[1])[np.asarray(perm)[::8] // 8].reshape(q.shape))
    mp.setattr(O, "reorder_rows", reorder_rows)


def _mut_mixed_two_bit_zero_one(mp):
    real = O.mixed_zero_points
    mp.setattr(O, "mixed_zero_points", lambda w, K, N: np.where(real(w, K, N) == 2, 1, 8))


MUTATIONS = [_mut_mixed_two_bit_zero_one, _mut_gidx_ignored, _mut_gidx_zero_contiguous, _mut_perm_inverse, _mut_reorder_within_word, _mut_zp_ignored, _mut_zp_sign, _mut_act_4bit_8_levels, _mut_act_round_half_up, _mut_act_range_128, _mut_act_scale_per_tensor, _mut_zero_point, _mut_group_mod, _mut_group_off_by_one, _mut_scale_dropped, _mut_nibbles_reversed,
             _mut_k_reversed, _mut_sign_flipped, _mut_w4a8_no_zero_point, _mut_w4a8_sw_dropped,
             _mut_absdot_signed, _mut_tolerance_rel_dropped]


@pytest.mark.parametrize("mutate", MUTATIONS, ids=lambda f: f.__name__[5:])
def test_pins_catch_planted_mistake(mutate, monkeypatch):
    mutate(monkeypatch)
    caught = []
    for pin in ALL_PINS:
        try:
            pin(O)
        except (AssertionError, ValueError, IndexError):
            caught.append(pin.__name__)
    assert caught, "no pin caught the planted mistake"


# ------------------------------------------------------------ prepack layout (the library's own format)
SHAPES = [(128, 128, 128), (256, 200, 64), (384, 136, 32), (512, 8, 256), (256, 264, 256), (1024, 392, 128)]


@pytest.mark.parametrize("K,N,g", SHAPES)
def test_prepack_roundtrip(K, N, g):
    d = synth.w4a16_inputs(K, N, g, 1, seed=K + N + g)
    Wp = O.prepack_w4a16(d["Q"], d["s"], g)
    assert Wp.nbytes == O.prepacked_bytes_w4a16(K, N, g)
    q, s = O.unprepack_w4a16(Wp, K, N, g)
    assert np.array_equal(q, d["q"])
    assert np.array_equal(s.view(np.uint16), d["s"].view(np.uint16))


@pytest.mark.parametrize("K,N,g", [(256, 128, 128), (256, 200, 64), (384, 136, 32), (512, 8, 256)])
def test_prepack_zp_roundtrip(K, N, g):
    d = synth.w4a16_inputs(K, N, g, 1, seed=K + N + g)
    z = np.random.default_rng(K).integers(0, 16, (K // g, N)).astype(np.uint8)
    Wp = O.prepack_w4a16_zp(d["Q"], d["s"], z, g)
    assert Wp.nbytes == O.prepacked_bytes_w4a16_zp(K, N, g)
    q, s, zz = O.unprepack_w4a16_zp(Wp, K, N, g)
    assert np.array_equal(q, d["q"]) and np.array_equal(zz, z)
    assert np.array_equal(s.view(np.uint16), d["s"].view(np.uint16))


@pytest.mark.parametrize("K,N", [(128, 128), (256, 200), (640, 24)])
def test_prepack_w4a8_roundtrip(K, N):
    d = synth.w4a8_inputs(K, N, 1, seed=K + N)
    Wp = O.prepack_w4a8(d["Q"])
    assert Wp.nbytes == O.prepacked_bytes_w4a8(K, N)
    assert np.array_equal(O.unprepack_w4a8(Wp, K, N), d["q"])


def test_prepack_blob_locality():
    # a code of column n and row k lands inside blob (n // 128, k // 128), and nowhere else
    K, N, g = 384, 296, 128
    nt, kt = 3, 3
    blob = O.prepacked_bytes_w4a16(K, N, g) // (nt * kt)
    rng = np.random.default_rng(0)
    for _ in range(20):
        k, n = int(rng.integers(K)), int(rng.integers(N))
        q = np.full((K, N), 8, np.uint8)
        q[k, n] = 3
        s = np.zeros((K // g, N), np.float16)
        Wp = O.prepack_w4a16(synth.pack_q(q), s, g)
        base = O.prepack_w4a16(synth.pack_q(np.full((K, N), 8, np.uint8)), s, g)
        diff = np.nonzero(Wp != base)[0]
        assert diff.size == 1
        assert diff[0] // blob == (n // 128) * kt + (k // 128)


def test_prepack_padding_is_zero_weight():
    K, N, g = 256, 72, 64
    d = synth.w4a16_inputs(K, N, g, 1, seed=1)
    Wp = O.prepack_w4a16(d["Q"], d["s"], g)
    full = O.unprepack_w4a16(Wp, K, 128, g)
    assert np.all(full[0][:, N:] == 8)
    assert np.all(full[1][:, N:] == 0)


# Layout mistakes made in both directions at once (prepack and its inverse): the round trip and
# the blob-locality test cannot see them; only the hand-worked byte offsets can.
def _mut_layout_h_v_swapped(mp):
    def blob_words(q, nibble_pos):
        w = _ORIG_BLOB_WORDS(q, nibble_pos)           # [nt, kt, h, v, r, i]
        return np.ascontiguousarray(w.transpose(0, 1, 3, 2, 4, 5))

    def codes_from_words(words, nibble_pos, K, N):
        nt, kt = words.shape[:2]
        w = words.reshape(nt, kt, 2, 2, O.TILE_N, 4).transpose(0, 1, 3, 2, 4, 5)
        return _ORIG_CODES_FROM_WORDS(np.ascontiguousarray(w).reshape(nt, kt, -1), nibble_pos, K, N)
    mp.setattr(O, "_blob_words", blob_words)
    mp.setattr(O, "_codes_from_words", codes_from_words)


def _mut_layout_i_reversed(mp):
    def blob_words(q, nibble_pos):
        return np.ascontiguousarray(_ORIG_BLOB_WORDS(q, nibble_pos)[..., ::-1])

    def codes_from_words(words, nibble_pos, K, N):
        nt, kt = words.shape[:2]
        w = words.reshape(nt, kt, 2, 2, O.TILE_N, 4)[..., ::-1]
        return _ORIG_CODES_FROM_WORDS(np.ascontiguousarray(w).reshape(nt, kt, -1), nibble_pos, K, N)
    mp.setattr(O, "_blob_words", blob_words)
    mp.setattr(O, "_codes_from_words", codes_from_words)


def _mut_layout_nibble_table(mp):
    mp.setattr(O, "NIBBLE_POS_W4A16", (0, 1, 2, 3, 4, 5, 6, 7))


_ORIG_BLOB_WORDS = O._blob_words
_ORIG_CODES_FROM_WORDS = O._codes_from_words
LAYOUT_MUTATIONS = [_mut_layout_h_v_swapped, _mut_layout_i_reversed, _mut_layout_nibble_table]


@pytest.mark.parametrize("mutate", LAYOUT_MUTATIONS, ids=lambda f: f.__name__[5:])
def test_layout_mistake_caught_only_by_the_golden_offsets(mutate, monkeypatch):
    mutate(monkeypatch)
    # the self-consistency checks still pass with the mistake in place ...
    for K, N, g in SHAPES[:3]:
        test_prepack_roundtrip(K, N, g)
    test_prepack_w4a8_roundtrip(256, 200)
    test_prepack_blob_locality()
    # ... and the hand-worked byte offsets catch it
    with pytest.raises(AssertionError):
        pin_blob_layout_golden(O)


@pytest.mark.parametrize("K,N,g", [(128, 128, 128), (256, 200, 64), (384, 136, 32), (512, 8, 256), (256, 40, 256)])
def test_prepack_sparse24_roundtrip(K, N, g):
    d = synth.w4a16_sparse24_inputs(K, N, g, 1, seed=K + N + g)
    Wp = O.prepack_w4a16_sparse24(d["Q"], d["s"], g)
    assert Wp.nbytes == O.prepacked_bytes_w4a16_sparse24(K, N, g)
    q, s = O.unprepack_w4a16_sparse24(Wp, K, N, g)
    assert np.array_equal(q, d["q"])
    assert np.array_equal(s.view(np.uint16), d["s"].view(np.uint16))


def test_prepack_sparse24_padding_is_zero_weight():
    d = synth.w4a16_sparse24_inputs(256, 72, 64, 1, seed=2)
    q, s = O.unprepack_w4a16_sparse24(O.prepack_w4a16_sparse24(d["Q"], d["s"], 64), 256, 128, 64)
    assert np.all(q[:, 72:] == 8) and np.all(s[:, 72:] == 0)


# Sparse layout mistakes made in both directions: the round trip passes, the offsets catch them.
def _mut_sparse_code_nibble_bits_swapped(mp):
    mp.setattr(O, "_sparse_code_nibble", lambda half, j, ki: 2 * half + (j >= 4) + 4 * ki)


def _mut_sparse_meta_half_and_word_swapped(mp):
    mp.setattr(O, "_sparse_meta_place",
               lambda b, rt, g, half, j: (((b * 8 + rt) * 8 + g) * 2 + half, (j % 4) + 4 * (j // 4)))


def _mut_sparse_fill_highest(mp):
    def kept_rows(col_group):
        keep = [p for p in range(4) if col_group[p] != 8]
        for p in (3, 2, 1, 0):
            if len(keep) == 2:
                break
            if p not in keep:
                keep.append(p)
        return sorted(keep)
    mp.setattr(O, "_kept_rows", kept_rows)


@pytest.mark.parametrize("mutate", [_mut_sparse_code_nibble_bits_swapped, _mut_sparse_meta_half_and_word_swapped,
                                    _mut_sparse_fill_highest],
                         ids=lambda f: f.__name__[5:])
def test_sparse_layout_mistake_caught_only_by_the_golden_offsets(mutate, monkeypatch):
    mutate(monkeypatch)
    test_prepack_sparse24_roundtrip(256, 200, 64)
    with pytest.raises(AssertionError):
        pin_sparse24_layout_golden(O)


@pytest.mark.parametrize("K,N,g,frac4", [(128, 128, 128, 0.5), (256, 200, 64, 0.3), (384, 136, 32, 0.2),
                                         (256, 40, 256, 0.5), (512, 8, 128, 1.0), (256, 136, 128, 0.0)])
def test_prepack_mixed_roundtrip(K, N, g, frac4):
    d = synth.w4a16_mixed_inputs(K, N, g, 1, seed=K + N + g, frac4=frac4)
    Wp = O.prepack_mixed(d["Q"], d["s"], g, d["widths"])
    assert Wp.nbytes == O.prepacked_bytes_mixed(K, N, g, d["widths"])
    q, s, w = O.unprepack_mixed(Wp, K, N, g)
    assert np.array_equal(q, d["q"]) and np.array_equal(w, d["widths"])
    assert np.array_equal(s.view(np.uint16), d["s"].view(np.uint16))


# Mixed layout mistakes made in both directions: the round trip passes, the offsets catch them.
def _mut_mixed_field_halves_swapped(mp):
    mp.setattr(O, "_mixed_field", lambda r, j: r // 2 + 8 * j + 4 * (r % 2))


def _mut_mixed_table_padded_twice(mp):
    mp.setattr(O, "_mixed_table_bytes", lambda nblob: ((nblob + 1) * 4 + 127) // 128 * 128 + 16)


@pytest.mark.parametrize("mutate", [_mut_mixed_field_halves_swapped, _mut_mixed_table_padded_twice],
                         ids=lambda f: f.__name__[5:])
def test_mixed_layout_mistake_caught_only_by_the_golden_offsets(mutate, monkeypatch):
    mutate(monkeypatch)
    test_prepack_mixed_roundtrip(256, 200, 64, 0.3)
    with pytest.raises(AssertionError):
        pin_mixed_layout_golden(O)


def test_package_reexports():
    assert oracle.w4a16 is O.w4a16
