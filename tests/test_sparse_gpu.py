"""GPU tests of 2:4 sparse weights: the CUDA layout pass against the oracle's restatement of
the sparse format byte for byte, its inverse, the device-side check of the 2:4 pattern, and
the sparse warp-MMA layer against the fp64 oracle (the W4A16 layer of the pruned weight) for
every tile height (1, 2, 4, 8, 16 rows), every scale mode (groups of 32, 64, 128, 256 rows and
one scale per column), ragged N, stream-K splits, the full layer sizes (sampled columns) and
bitwise determinism."""
import numpy as np
import pytest
import torch

import oracle
import synth
from wq_check import check_w4a16_cols, check_w4a16_full, sample_cols, to_dev

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _wq():
    import bit_weight_quantized_prepack_b200 as wq
    return wq


LAYOUT = [(128, 128, 128), (384, 296, 128), (384, 296, 32), (256, 200, 64), (512, 136, 256), (384, 296, 384),
          (128, 8, 64), (640, 1000, 128)]


@pytest.mark.parametrize("K,N,g", LAYOUT)
def test_sparse_prepack_matches_oracle_bytes(K, N, g):
    wq = _wq()
    d = synth.w4a16_sparse24_inputs(K, N, g, 1, seed=K * 5 + N + g)
    Wp = wq.wq_prepack_sparse24(to_dev(d["Q"]), to_dev(d["s"]), g)
    ref = oracle.prepack_w4a16_sparse24(d["Q"], d["s"], g)
    got = Wp.cpu().numpy()
    assert got.nbytes == ref.nbytes == wq.wq_prepacked_bytes_sparse24(K, N, g)
    assert np.array_equal(got, ref), f"first difference at byte {int(np.argmax(got != ref))}"


@pytest.mark.parametrize("K,N,g", LAYOUT)
def test_sparse_unpack_roundtrip(K, N, g):
    wq = _wq()
    d = synth.w4a16_sparse24_inputs(K, N, g, 1, seed=K + 3 * N + g)
    Q, s = to_dev(d["Q"]), to_dev(d["s"])
    Q2, s2 = wq.wq_unpack_sparse24(wq.wq_prepack_sparse24(Q, s, g), K, N, g)
    assert torch.equal(Q2, Q)
    assert torch.equal(s2.view(torch.int16), s.view(torch.int16))


def test_sparse_prepack_fewer_kept_codes_and_extremes():
    # groups with 0, 1 or 2 codes other than 8, at every pair of positions, codes 0 and 15
    wq = _wq()
    K, N, g = 256, 136, 128
    rng = np.random.default_rng(5)
    q = np.full((K, N), 8, np.uint8)
    for grp in range(K // 4):
        for n in range(N):
            k = int(rng.integers(0, 3))
            pos = rng.choice(4, size=k, replace=False)
            q[4 * grp + pos, n] = rng.choice([0, 15, 1, 14, 7, 9], size=k)
    s = (0.01 + 0.01 * rng.random((K // g, N))).astype(np.float16)
    Q = synth.pack_q(q)
    Wp = wq.wq_prepack_sparse24(to_dev(Q), to_dev(s), g)
    assert np.array_equal(Wp.cpu().numpy(), oracle.prepack_w4a16_sparse24(Q, s, g))
    Q2, _ = wq.wq_unpack_sparse24(Wp, K, N, g)
    assert np.array_equal(Q2.cpu().numpy(), Q)


@pytest.mark.parametrize("where", [(0, 0), (125, 135), (64, 77)])
def test_sparse_prepack_refuses_three_weights_in_a_group(where):
    wq = _wq()
    K, N, g = 256, 136, 128
    d = synth.w4a16_sparse24_inputs(K, N, g, 1, seed=9)
    q = d["q"].copy()
    k0, n = where[0] // 4 * 4, where[1]
    q[k0:k0 + 4, n] = [1, 2, 3, 8]
    assert not oracle.is_sparse24(q)
    with pytest.raises(wq.WqError) as e:
        wq.wq_prepack_sparse24(to_dev(synth.pack_q(q)), to_dev(d["s"]), g)
    assert e.value.status == wq.WQ_ERR_NOT_SPARSE
    # the device's check word is reset by each call: a valid weight afterwards passes
    wq.wq_prepack_sparse24(to_dev(d["Q"]), to_dev(d["s"]), g)


# (K, N): one k-block and one tile; 3 ragged tiles of 32 k-blocks over 96 CTAs; 148 CTAs over
# 1024 units; a long K
SHAPES = [(128, 8), (4096, 264), (4096, 4096), (11008, 392)]


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8, 9, 16])
@pytest.mark.parametrize("K,N", SHAPES)
@pytest.mark.parametrize("g", [32, 64, 128, 256, "K"])
def test_sparse_vs_oracle(M, K, N, g):
    wq = _wq()
    g = K if g == "K" else g
    if K % g:
        pytest.skip("group size must divide K")
    plan = wq.wq_plan(5, M, N, K, g)
    assert plan["threads"] == 576 and plan["tile_m"] >= M
    d = synth.w4a16_sparse24_inputs(K, N, g, M, seed=K + N + M + g)
    Wp = wq.wq_prepack_sparse24(to_dev(d["Q"]), to_dev(d["s"]), g)
    Y = wq.wq_gemm_w4a16_sparse24(to_dev(d["A"]), Wp, N, g)
    torch.cuda.synchronize()
    assert wq.wq_get_device_status() == wq.WQ_OK
    check_w4a16_full(d, Y, f"sparse K={K} N={N} g={g} M={M}")


@pytest.mark.parametrize("K,N,g", [(4096, 12288, 128), (4096, 22016, 128), (11008, 4096, 128), (8192, 57344, 128),
                                   (8192, 57344, 8192)])
@pytest.mark.parametrize("M", [1, 16])
def test_sparse_full_layer_sizes_sampled(K, N, g, M):
    wq = _wq()
    d = synth.w4a16_sparse24_inputs(K, N, g, M, seed=N + M)
    Wp = wq.wq_prepack_sparse24(to_dev(d["Q"]), to_dev(d["s"]), g)
    Y = wq.wq_gemm_w4a16_sparse24(to_dev(d["A"]), Wp, N, g)
    torch.cuda.synchronize()
    assert wq.wq_get_device_status() == wq.WQ_OK
    check_w4a16_cols(d, Y, sample_cols(N, 96, seed=M), what=f"sparse full K={K} N={N} g={g} M={M}")


def test_sparse_identity_activation_gives_the_pruned_weights():
    # A = I (128 rows of a 128-row K): y[m, n] = (q[m, n] - 8) * s, with zeros where pruned
    wq = _wq()
    K, N, g = 128, 264, 32
    d = synth.w4a16_sparse24_inputs(K, N, g, 1, seed=4)
    for m0 in range(0, K, 16):
        A = np.zeros((16, K), np.float16)
        A[np.arange(16), m0 + np.arange(16)] = 1
        Wp = wq.wq_prepack_sparse24(to_dev(d["Q"]), to_dev(d["s"]), g)
        Y = wq.wq_gemm_w4a16_sparse24(to_dev(A), Wp, N, g).cpu().numpy()
        rows = m0 + np.arange(16)
        want = ((d["q"][rows].astype(np.float64) - 8) * d["s"][rows // g].astype(np.float64)).astype(np.float16)
        assert np.array_equal(Y.view(np.uint16), want.view(np.uint16))


def test_sparse_is_deterministic():
    wq = _wq()
    K, N, g, M = 4096, 4096, 128, 3
    d = synth.w4a16_sparse24_inputs(K, N, g, M, seed=11)
    A, Wp = to_dev(d["A"]), wq.wq_prepack_sparse24(to_dev(d["Q"]), to_dev(d["s"]), g)
    Y0 = wq.wq_gemm_w4a16_sparse24(A, Wp, N, g)
    for _ in range(5):
        assert torch.equal(wq.wq_gemm_w4a16_sparse24(A, Wp, N, g).view(torch.int16), Y0.view(torch.int16))


def test_sparse_and_dense_layers_agree_on_the_pruned_weight():
    # the same pruned weight through the dense and the sparse buffer: both within the oracle's
    # tolerance, and close to each other
    wq = _wq()
    K, N, g, M = 4096, 1024, 128, 4
    d = synth.w4a16_sparse24_inputs(K, N, g, M, seed=21)
    A = to_dev(d["A"])
    Yd = wq.wq_gemm_w4a16(A, wq.wq_prepack(to_dev(d["Q"]), to_dev(d["s"]), g), N, g)
    Ys = wq.wq_gemm_w4a16_sparse24(A, wq.wq_prepack_sparse24(to_dev(d["Q"]), to_dev(d["s"]), g), N, g)
    check_w4a16_full(d, Yd, "dense on pruned")
    check_w4a16_full(d, Ys, "sparse on pruned")


def test_sparse_shape_limits():
    wq = _wq()
    K, N, g = 256, 136, 128
    d = synth.w4a16_sparse24_inputs(K, N, g, 17, seed=2)
    Wp = wq.wq_prepack_sparse24(to_dev(d["Q"]), to_dev(d["s"]), g)
    with pytest.raises(wq.WqError) as e:  # the sparse path serves M <= 16
        wq.wq_gemm_w4a16_sparse24(to_dev(d["A"]), Wp, N, g)
    assert e.value.status == wq.WQ_ERR_UNSUPPORTED_SHAPE
    Y = wq.wq_gemm_w4a16_sparse24(to_dev(d["A"][:0]), Wp, N, g)  # M = 0: nothing launched
    assert Y.shape == (0, N)
    assert wq.wq_workspace_bytes(5, 17, N, K) == 0 and wq.wq_workspace_bytes(5, 16, N, K) > 0
