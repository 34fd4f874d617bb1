"""GPU tests of mixed 2/4-bit weights: the CUDA layout pass against the oracle's restatement of
the mixed format byte for byte, its inverse, the checks of widths and codes, and the layer on the
register-operand kernel against the fp64 oracle for every tile height (1, 2, 4, 8, 16 rows), every
scale mode (groups of 32, 64, 128, 256 rows and one scale per column), ragged N, stream-K
splits, the full layer sizes (sampled columns) and bitwise determinism; with every block at 4
bits the layer equals the dense W4A16 layer bit for bit. A buffer whose blob table does not fit
the format is refused by the kernel before any copy, and reported through the status word."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
from wq_check import compare, half_bits_to_f64, sample_cols, to_dev

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _wq():
    import bit_weight_quantized_prepack_b200 as wq
    return wq


def _prepack(wq, d, g):
    return wq.wq_prepack_mixed(to_dev(d["Q"]), to_dev(d["s"]), to_dev(d["widths"]), g)


def _check(d, Y, g, what, cols=None):
    """Compare with the fp64 oracle, on every column or on the given ones (one oracle call per
    sampled column: that column alone, with the width of its n-tile)."""
    Q, s, A, W = d["Q"], d["s"], d["A"], d["widths"]
    if cols is None:
        return compare(half_bits_to_f64(Y), oracle.w4a16_mixed(A, Q, s, g, W),
                       oracle.w4a16_mixed_absdot(A, Q, s, g, W), what)
    ref = np.stack([oracle.w4a16_mixed(A, Q[:, [n]], s[:, [n]], g, W[:, [n // 128]])[:, 0] for n in cols], axis=1)
    ad = np.stack([oracle.w4a16_mixed_absdot(A, Q[:, [n]], s[:, [n]], g, W[:, [n // 128]])[:, 0] for n in cols], axis=1)
    return compare(half_bits_to_f64(Y)[:, cols], ref, ad, what)


LAYOUT = [(128, 128, 128, 0.5), (256, 136, 128, 0.4), (384, 296, 32, 0.2), (256, 200, 64, 0.3), (512, 136, 256, 0.5),
          (384, 296, 384, 0.3), (128, 8, 64, 1.0), (640, 1000, 128, 0.0)]


@pytest.mark.parametrize("K,N,g,frac4", LAYOUT)
def test_mixed_prepack_matches_oracle_bytes(K, N, g, frac4):
    wq = _wq()
    d = synth.w4a16_mixed_inputs(K, N, g, 1, seed=K * 3 + N + g, frac4=frac4)
    got = _prepack(wq, d, g).cpu().numpy()
    ref = oracle.prepack_mixed(d["Q"], d["s"], g, d["widths"])
    assert got.nbytes == ref.nbytes
    assert np.array_equal(got, ref), f"first difference at byte {int(np.argmax(got != ref))}"


@pytest.mark.parametrize("K,N,g,frac4", LAYOUT)
def test_mixed_unpack_roundtrip(K, N, g, frac4):
    wq = _wq()
    d = synth.w4a16_mixed_inputs(K, N, g, 1, seed=K + 5 * N + g, frac4=frac4)
    Q2, s2, w2 = wq.wq_unpack_mixed(_prepack(wq, d, g), K, N, g)
    assert np.array_equal(Q2.cpu().numpy(), d["Q"])
    assert np.array_equal(s2.cpu().numpy().view(np.uint16), d["s"].view(np.uint16))
    assert np.array_equal(w2.cpu().numpy(), d["widths"])


def test_mixed_prepack_refuses_bad_widths_codes_and_short_buffers():
    wq = _wq()
    K, N, g = 256, 136, 128
    d = synth.w4a16_mixed_inputs(K, N, g, 1, seed=3, frac4=0.3)
    bad_w = d["widths"].copy()
    bad_w[1, 1] = 3
    with pytest.raises(wq.WqError) as e:
        wq.wq_prepack_mixed(to_dev(d["Q"]), to_dev(d["s"]), to_dev(bad_w), g)
    assert e.value.status == wq.WQ_ERR_INVALID_ARG
    q = d["q"].copy()
    b2 = np.argwhere(d["widths"] == 2)[0]
    q[32 * b2[0] + 7, 128 * b2[1] + 5] = 9  # a 4-bit code in a 2-bit block
    with pytest.raises(wq.WqError) as e:
        wq.wq_prepack_mixed(to_dev(synth.pack_q(q)), to_dev(d["s"]), to_dev(d["widths"]), g)
    assert e.value.status == wq.WQ_ERR_INVALID_ARG
    # the C call itself refuses a buffer smaller than the widths need
    n4 = int((d["widths"] == 4).sum())
    need = wq.wq_prepacked_bytes_mixed(K, N, g, n4)
    Wp = torch.empty(need, dtype=torch.uint8, device="cuda")
    Qd, sd, wd = to_dev(d["Q"]), to_dev(d["s"]), to_dev(d["widths"])
    P = ctypes.c_void_p
    assert wq.lib.wq_prepack_mixed(P(Qd.data_ptr()), P(sd.data_ptr()), P(wd.data_ptr()), K, N, g, P(Wp.data_ptr()),
                                   need - 16, None) == wq.WQ_ERR_INVALID_ARG
    assert wq.lib.wq_prepack_mixed(P(Qd.data_ptr()), P(sd.data_ptr()), P(wd.data_ptr()), K, N, g, P(Wp.data_ptr()),
                                   need, None) == wq.WQ_OK


SHAPES = [(128, 8), (4096, 264), (4096, 4096), (11008, 392)]


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8, 9, 16])
@pytest.mark.parametrize("K,N", SHAPES)
@pytest.mark.parametrize("g", [32, 64, 128, 256, "K"])
def test_mixed_vs_oracle(M, K, N, g):
    wq = _wq()
    g = K if g == "K" else g
    if K % g:
        pytest.skip("group size must divide K")
    plan = wq.wq_plan(6, M, N, K, g)
    assert plan["threads"] == 576 and plan["tile_m"] >= M
    d = synth.w4a16_mixed_inputs(K, N, g, M, seed=K + N + M + g, frac4=0.3)
    Y = wq.wq_gemm_w4a16_mixed(to_dev(d["A"]), _prepack(wq, d, g), N, g)
    torch.cuda.synchronize()
    assert wq.wq_get_device_status() == wq.WQ_OK
    _check(d, Y, g, f"mixed K={K} N={N} g={g} M={M}")


@pytest.mark.parametrize("M", [1, 5, 16])
@pytest.mark.parametrize("g", [32, 128, "K"])
def test_mixed_all_four_bit_equals_dense_bitwise(M, g):
    wq = _wq()
    K, N = 4096, 1032
    g = K if g == "K" else g
    d = synth.w4a16_mixed_inputs(K, N, g, M, seed=M + 40, frac4=1.0)
    A = to_dev(d["A"])
    Ym = wq.wq_gemm_w4a16_mixed(A, _prepack(wq, d, g), N, g)
    Yd = wq.wq_gemm_w4a16(A, wq.wq_prepack(to_dev(d["Q"]), to_dev(d["s"]), g), N, g)
    assert torch.equal(Ym.view(torch.int16), Yd.view(torch.int16))


@pytest.mark.parametrize("K,N,g", [(4096, 12288, 128), (4096, 22016, 128), (11008, 4096, 128), (8192, 57344, 128),
                                   (8192, 57344, 8192)])
@pytest.mark.parametrize("M", [1, 16])
def test_mixed_full_layer_sizes_sampled(K, N, g, M):
    wq = _wq()
    d = synth.w4a16_mixed_inputs(K, N, g, M, seed=N + M, frac4=0.15)
    Y = wq.wq_gemm_w4a16_mixed(to_dev(d["A"]), _prepack(wq, d, g), N, g)
    torch.cuda.synchronize()
    assert wq.wq_get_device_status() == wq.WQ_OK
    _check(d, Y, g, f"mixed full K={K} N={N} g={g} M={M}", cols=sample_cols(N, 96, seed=M))


def test_mixed_is_deterministic():
    wq = _wq()
    K, N, g, M = 4096, 4096, 128, 3
    d = synth.w4a16_mixed_inputs(K, N, g, M, seed=11, frac4=0.3)
    A, Wp = to_dev(d["A"]), _prepack(wq, d, g)
    Y0 = wq.wq_gemm_w4a16_mixed(A, Wp, N, g)
    for _ in range(5):
        assert torch.equal(wq.wq_gemm_w4a16_mixed(A, Wp, N, g).view(torch.int16), Y0.view(torch.int16))


def test_mixed_table_outside_the_buffer_is_refused_by_the_kernel():
    # One table entry points past the end of the buffer: the weight producer checks every blob
    # against the buffer's size and the widths before copying it, copies nothing of that chunk,
    # and records WQ_ERR_INVALID_ARG; the context stays usable and a repaired buffer gives the
    # oracle's result again. (Waits of the other CTAs on the stopped one end at a short limit.)
    wq = _wq()
    K, N, g, M = 1024, 392, 128, 2
    d = synth.w4a16_mixed_inputs(K, N, g, M, seed=29, frac4=0.3)
    Wp = _prepack(wq, d, g)
    good = Wp[:64].clone()
    table = Wp[:64].view(torch.int32)
    table[5] = (Wp.numel() // 16 + 8) << 4  # blob 5 now starts 128 bytes past the end
    A = to_dev(d["A"])
    wq.wq_debug_set_wait_timeout_ns(50_000_000)
    try:
        wq.wq_gemm_w4a16_mixed(A, Wp, N, g)
        torch.cuda.synchronize()
        assert wq.wq_get_device_status() == wq.WQ_ERR_INVALID_ARG
    finally:
        wq.wq_debug_set_wait_timeout_ns(0)
    Wp[:64] = good
    Y = wq.wq_gemm_w4a16_mixed(A, Wp, N, g)
    torch.cuda.synchronize()
    assert wq.wq_get_device_status() == wq.WQ_OK
    _check(d, Y, g, "mixed after a refused table")


def test_mixed_shape_limits():
    wq = _wq()
    K, N, g = 256, 136, 128
    d = synth.w4a16_mixed_inputs(K, N, g, 17, seed=2)
    Wp = _prepack(wq, d, g)
    with pytest.raises(wq.WqError) as e:
        wq.wq_gemm_w4a16_mixed(to_dev(d["A"]), Wp, N, g)
    assert e.value.status == wq.WQ_ERR_UNSUPPORTED_SHAPE
    assert wq.wq_gemm_w4a16_mixed(to_dev(d["A"][:0]), Wp, N, g).shape == (0, N)
    assert wq.wq_workspace_bytes(6, 17, N, K) == 0 and wq.wq_workspace_bytes(6, 16, N, K) > 0
