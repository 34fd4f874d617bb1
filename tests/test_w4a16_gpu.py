"""GPU parity of the W4A16 layer against the fp64 oracle.

Small layers are compared on every output; the full-size layer configurations on every
output where the oracle is cheap and on sampled columns (all rows) otherwise. Exact special
cases (identity activations, all-8 codes, power-of-two scales, row permutation, repeat
calls) are compared bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from wq_check import (check_w4a16_cols, check_w4a16_full, compare, half_bits_to_f64, sample_cols, to_dev,
                      w4a16_case)

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _wq():
    import bit_weight_quantized_prepack_b200 as wq
    return wq


# (K, N, g, M): several tiles, ragged N (not a multiple of 128), ragged M (not a multiple of 16),
# M across tile_m choices (16..256) and above 256 (several m-tiles), every group-size kind
SMALL = [
    (128, 128, 128, 1), (256, 256, 64, 3), (384, 136, 32, 16), (1024, 264, 128, 17), (1024, 1024, 128, 33),
    (512, 392, 256, 100), (640, 520, 640, 129), (1024, 512, 1024, 256), (2048, 256, 128, 300),
    (1280, 1000, 128, 64), (4096, 128, 4096, 5), (256, 8, 128, 2), (768, 2056, 32, 48), (512, 640, 512, 513),
    (2048, 2048, 64, 1), (3072, 1536, 128, 8), (512, 264, 128, 32), (1024, 136, 1024, 32), (1024, 392, 128, 65),
]


@pytest.mark.parametrize("K,N,g,M", SMALL)
def test_small_layers_vs_oracle(K, N, g, M):
    d, Wp, Y = w4a16_case(K, N, g, M, seed=K + N + g + M)
    check_w4a16_full(d, Y, f"K={K} N={N} g={g} M={M}")


@pytest.mark.parametrize("K,g", [(128, 128), (256, 256), (1024, 128), (1024, 32), (512, 64)])
def test_identity_activation_reproduces_weights_bitwise(K, g):
    # A = I: Y[k, n] is one weight times 1.0 plus exact zeros, so it must equal the kernel's
    # documented weight rounding bit for bit: fp16_rn((q-8) * s) for g < K, fp16_rn(fp32((q-8) * s)) for g == K.
    wq = _wq()
    N = 136
    d = synth.w4a16_inputs(K, N, g, 1, seed=K + g)
    A = np.eye(K, dtype=np.float16)
    Wp = wq.wq_prepack(to_dev(d["Q"]), to_dev(d["s"]), g)
    Y = wq.wq_gemm_w4a16(to_dev(A), Wp, N, g).cpu().numpy()
    qm8 = d["q"].astype(np.float32) - 8
    s_full = d["s"][np.arange(K) // g].astype(np.float32)
    if g < K:
        exp = (qm8.astype(np.float16) * d["s"][np.arange(K) // g]).astype(np.float16)
    else:
        exp = (qm8 * s_full).astype(np.float16)
    assert np.array_equal(Y.astype(np.float32), exp.astype(np.float32)), \
        f"{int((Y.astype(np.float32) != exp.astype(np.float32)).sum())} weights differ"


@pytest.mark.parametrize("K,g,M", [(1024, 128, 16), (1024, 1024, 16), (2048, 256, 32), (512, 64, 16), (1024, 32, 9)])
def test_unit_rows_reproduce_weights_bitwise(K, g, M):
    # small batches (one tile of <= 32 rows): row i of A is the unit vector e_{k_i}, so
    # Y[i, n] = fp16_rn((q[k_i, n] - 8) * s[k_i // g, n]) bit for bit, whichever of the two
    # scale placements the kernel uses (a single exact product, one rounding)
    wq = _wq()
    N = 264
    d = synth.w4a16_inputs(K, N, g, 1, seed=K + g + M)
    ks = np.random.default_rng(M).choice(K, size=M, replace=False)
    A = np.zeros((M, K), np.float16)
    A[np.arange(M), ks] = 1
    Wp = wq.wq_prepack(to_dev(d["Q"]), to_dev(d["s"]), g)
    Y = wq.wq_gemm_w4a16(to_dev(A), Wp, N, g).cpu().numpy()
    exact = (d["q"][ks].astype(np.float64) - 8) * d["s"][ks // g].astype(np.float64)
    exp = exact.astype(np.float16)  # one round-to-nearest-even of the exact product
    assert np.array_equal(Y.astype(np.float32), exp.astype(np.float32)), \
        f"{int((Y.astype(np.float32) != exp.astype(np.float32)).sum())} weights differ"


@pytest.mark.parametrize("g", [128, 1024])
def test_all_eight_codes_give_zero(g):
    wq = _wq()
    K, N, M = 1024, 264, 33
    d = synth.w4a16_inputs(K, N, g, M, seed=5)
    Q = synth.pack_q(np.full((K, N), 8, np.uint8))
    Wp = wq.wq_prepack(to_dev(Q), to_dev(d["s"]), g)
    Y = wq.wq_gemm_w4a16(to_dev(d["A"]), Wp, N, g)
    assert torch.all(Y.float() == 0)


@pytest.mark.parametrize("g", [64, 2048])
def test_all_zero_codes_closed_form(g):
    wq = _wq()
    K, N, M = 2048, 392, 7
    d = synth.w4a16_inputs(K, N, g, M, seed=6)
    d["Q"] = synth.pack_q(np.zeros((K, N), np.uint8))
    Wp = wq.wq_prepack(to_dev(d["Q"]), to_dev(d["s"]), g)
    Y = wq.wq_gemm_w4a16(to_dev(d["A"]), Wp, N, g)
    # y = -8 * sum_k a[m,k] * s[k//g, n]
    A64 = d["A"].astype(np.float64)
    S = d["s"].astype(np.float64)[np.arange(K) // g]
    y_ref = -8.0 * (A64 @ S)
    ad = 8.0 * (np.abs(A64) @ S)
    compare(half_bits_to_f64(Y), y_ref, ad, "all-zero codes")


@pytest.mark.parametrize("g", [128, 4096])
def test_power_of_two_scale_homogeneity_bitwise(g):
    wq = _wq()
    K, N, M = 4096, 520, 16
    d = synth.w4a16_inputs(K, N, g, M, seed=7)
    A = to_dev(d["A"])
    Y1 = wq.wq_gemm_w4a16(A, wq.wq_prepack(to_dev(d["Q"]), to_dev(d["s"]), g), N, g)
    s2 = (d["s"].astype(np.float32) * 2).astype(np.float16)
    Y2 = wq.wq_gemm_w4a16(A, wq.wq_prepack(to_dev(d["Q"]), to_dev(s2), g), N, g)
    assert torch.equal((Y1.float() * 2).half().view(torch.int16), Y2.view(torch.int16))


@pytest.mark.parametrize("M", [5, 16, 100, 256])
def test_row_permutation_bitwise(M):
    wq = _wq()
    K, N, g = 2048, 392, 128
    d = synth.w4a16_inputs(K, N, g, M, seed=8)
    Wp = wq.wq_prepack(to_dev(d["Q"]), to_dev(d["s"]), g)
    perm = np.random.default_rng(M).permutation(M)
    Y = wq.wq_gemm_w4a16(to_dev(d["A"]), Wp, N, g)
    Yp = wq.wq_gemm_w4a16(to_dev(d["A"][perm]), Wp, N, g)
    assert torch.equal(Yp.view(torch.int16), Y[torch.from_numpy(perm).cuda()].view(torch.int16))


def test_repeat_calls_are_bitwise_identical():
    wq = _wq()
    K, N, g, M = 4096, 4096, 128, 7
    d = synth.w4a16_inputs(K, N, g, M, seed=9)
    A = to_dev(d["A"])
    Wp = wq.wq_prepack(to_dev(d["Q"]), to_dev(d["s"]), g)
    Y1 = wq.wq_gemm_w4a16(A, Wp, N, g)
    for _ in range(3):
        assert torch.equal(wq.wq_gemm_w4a16(A, Wp, N, g).view(torch.int16), Y1.view(torch.int16))


def test_output_guard_regions_untouched():
    wq = _wq()
    K, N, g, M = 1024, 264, 128, 19
    d = synth.w4a16_inputs(K, N, g, M, seed=10)
    Wp = wq.wq_prepack(to_dev(d["Q"]), to_dev(d["s"]), g)
    guard = 4096
    buf = torch.full((guard + M * N + guard,), 12345, dtype=torch.int16, device="cuda")
    Y = buf[guard:guard + M * N].view(torch.float16).view(M, N)
    wq.wq_gemm_w4a16(to_dev(d["A"]), Wp, N, g, Y=Y)
    assert torch.all(buf[:guard] == 12345) and torch.all(buf[guard + M * N:] == 12345)
    check_w4a16_full(d, Y, "guarded output")


def test_empty_batch_is_a_no_op():
    wq = _wq()
    K, N, g = 256, 128, 128
    d = synth.w4a16_inputs(K, N, g, 1, seed=11)
    Wp = wq.wq_prepack(to_dev(d["Q"]), to_dev(d["s"]), g)
    Y = wq.wq_gemm_w4a16(torch.empty((0, K), dtype=torch.float16, device="cuda"), Wp, N, g)
    assert Y.shape == (0, N)


# ------------------------------------------------------------------ the layer configurations
LLAMA7B = [(4096, 12288), (4096, 4096), (4096, 22016), (11008, 4096)]
M_SWEEP = [1, 2, 4, 8, 16, 32, 64, 128]


def test_single_layer_4096_m1():
    d, Wp, Y = w4a16_case(4096, 4096, 128, 1, seed=0)
    check_w4a16_full(d, Y, "4096x4096 M=1 g=128")


@pytest.mark.parametrize("K,N", LLAMA7B)
def test_llama7b_layers_m_sweep(K, N):
    wq = _wq()
    g = 128
    d = synth.w4a16_inputs(K, N, g, max(M_SWEEP), seed=0)
    Wp = wq.wq_prepack(to_dev(d["Q"]), to_dev(d["s"]), g)
    A = to_dev(d["A"])
    y_ref = oracle.w4a16(d["A"], d["Q"], d["s"], g)
    ad = oracle.w4a16_absdot(d["A"], d["Q"], d["s"], g)
    for M in M_SWEEP:
        Y = wq.wq_gemm_w4a16(A[:M].contiguous(), Wp, N, g)
        compare(half_bits_to_f64(Y), y_ref[:M], ad[:M], f"K={K} N={N} M={M}")


LLAMA70B = [(8192, 10240), (8192, 8192), (8192, 57344), (28672, 8192)]


@pytest.mark.parametrize("K,N", LLAMA70B)
@pytest.mark.parametrize("gkind", ["g128", "channel"])
def test_llama70b_layers_sampled(K, N, gkind):
    wq = _wq()
    g = 128 if gkind == "g128" else K
    d = synth.w4a16_inputs(K, N, g, 128, seed=0)
    Wp = wq.wq_prepack(to_dev(d["Q"]), to_dev(d["s"]), g)
    A = to_dev(d["A"])
    cols = sample_cols(N, 768, seed=K + N)
    Qc, sc = d["Q"][:, cols], d["s"][:, cols]
    y_ref = oracle.w4a16(d["A"], Qc, sc, g)
    ad = oracle.w4a16_absdot(d["A"], Qc, sc, g)
    for M in (1, 16, 64, 128):
        Y = wq.wq_gemm_w4a16(A[:M].contiguous(), Wp, N, g)
        compare(half_bits_to_f64(Y)[:, cols], y_ref[:M], ad[:M], f"K={K} N={N} g={g} M={M}")


def test_compute_bound_sweep_sampled():
    wq = _wq()
    K = N = 8192
    g = 128
    d = synth.w4a16_inputs(K, N, g, 4096, seed=0)
    Wp = wq.wq_prepack(to_dev(d["Q"]), to_dev(d["s"]), g)
    A = to_dev(d["A"])
    cols = sample_cols(N, 192, seed=1)
    Qc, sc = d["Q"][:, cols], d["s"][:, cols]
    y_ref = oracle.w4a16(d["A"], Qc, sc, g)
    ad = oracle.w4a16_absdot(d["A"], Qc, sc, g)
    for M in (256, 512, 1024, 4096):
        Y = wq.wq_gemm_w4a16(A[:M].contiguous(), Wp, N, g)
        compare(half_bits_to_f64(Y)[:, cols], y_ref[:M], ad[:M], f"8192^2 M={M}")
