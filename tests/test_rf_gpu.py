"""GPU parity of the register-operand kernel (calls of at most 16 rows: weights
dequantised in registers feed warp-level m16n8k16 MMAs, no tensor memory) against the fp64
oracle: every scale mode (groups of 32, 64, 128 and 256 rows, one scale per column, zero
points), every tile height (1, 2, 4, 8, 16 rows, rows past M zero), ragged N, stream-K splits from
whole tiles to 32 CTAs per tile, the full layer sizes, bitwise determinism, and identity
activations reproducing (q - 8) * s."""
import numpy as np
import pytest
import torch

import oracle
import synth
from wq_check import check_w4a16_full, check_w4a16_cols, compare, half_bits_to_f64, sample_cols, to_dev

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _wq():
    import bit_weight_quantized_prepack_b200 as wq
    return wq


# (K, N): one k-block and one tile; 3 ragged tiles of 32 k-blocks over 96 CTAs (each tile split
# 32 ways); 148 CTAs over 1024 units; a long K
SHAPES = [(128, 8), (4096, 264), (4096, 4096), (11008, 392)]


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8, 9, 16])
@pytest.mark.parametrize("K,N", SHAPES)
@pytest.mark.parametrize("g", [32, 64, 128, 256, "K"])
def test_rf_vs_oracle(M, K, N, g):
    wq = _wq()
    g = K if g == "K" else g
    if K % g:
        pytest.skip("group size must divide K")
    plan = wq.wq_plan(0, M, N, K, g)
    assert plan["threads"] == 576 and plan["tile_m"] >= M
    d = synth.w4a16_inputs(K, N, g, M, seed=K + N + M + g)
    Wp = wq.wq_prepack(to_dev(d["Q"]), to_dev(d["s"]), g)
    Y = wq.wq_gemm_w4a16(to_dev(d["A"]), Wp, N, g)
    torch.cuda.synchronize()
    assert wq.wq_get_device_status() == wq.WQ_OK
    check_w4a16_full(d, Y, f"rf K={K} N={N} g={g} M={M}")


@pytest.mark.parametrize("M", [1, 2, 4, 7, 13])
@pytest.mark.parametrize("K,N,g", [(4096, 264, 64), (4096, 4096, 128), (11008, 392, 32), (2048, 136, 256)])
def test_rf_zero_points_vs_oracle(M, K, N, g):
    wq = _wq()
    d = synth.w4a16_inputs(K, N, g, M, seed=K + M)
    z = np.random.default_rng(K + N).integers(0, 16, (K // g, N)).astype(np.uint8)
    Wp = wq.wq_prepack_zp(to_dev(d["Q"]), to_dev(d["s"]), to_dev(z), g)
    Y = wq.wq_gemm_w4a16_zp(to_dev(d["A"]), Wp, N, g)
    torch.cuda.synchronize()
    assert wq.wq_get_device_status() == wq.WQ_OK
    compare(half_bits_to_f64(Y), oracle.w4a16_zp(d["A"], d["Q"], d["s"], z, g),
            oracle.w4a16_zp_absdot(d["A"], d["Q"], d["s"], z, g), f"rf zp K={K} N={N} g={g} M={M}")


@pytest.mark.parametrize("K,N,g", [(4096, 12288, 128), (4096, 22016, 128), (11008, 4096, 128), (8192, 57344, 128),
                                   (8192, 57344, 8192), (28672, 8192, 128)])
@pytest.mark.parametrize("M", [1, 2, 8, 16])
def test_rf_full_layer_sizes_sampled(K, N, g, M):
    # the bench's launch configuration at full size; the oracle computes sampled columns
    wq = _wq()
    d = synth.w4a16_inputs(K, N, g, M, seed=N + M)
    Wp = wq.wq_prepack(to_dev(d["Q"]), to_dev(d["s"]), g)
    Y = wq.wq_gemm_w4a16(to_dev(d["A"]), Wp, N, g)
    torch.cuda.synchronize()
    assert wq.wq_get_device_status() == wq.WQ_OK
    check_w4a16_cols(d, Y, sample_cols(N, 96, seed=M), what=f"rf full K={K} N={N} g={g} M={M}")


def test_rf_is_deterministic():
    wq = _wq()
    K, N, g, M = 4096, 4096, 128, 2
    d = synth.w4a16_inputs(K, N, g, M, seed=11)
    A, Wp = to_dev(d["A"]), wq.wq_prepack(to_dev(d["Q"]), to_dev(d["s"]), g)
    Y0 = wq.wq_gemm_w4a16(A, Wp, N, g)
    for _ in range(5):
        assert torch.equal(wq.wq_gemm_w4a16(A, Wp, N, g).view(torch.int16), Y0.view(torch.int16))


@pytest.mark.parametrize("K,g", [(128, 32), (256, 64), (256, 128), (512, 256)])
def test_rf_identity_rows_reproduce_weights(K, g):
    # rows e_k, four at a time (M = 4): y[m, n] = (q[k, n] - 8) * s[k // g, n] (for g = 32 the
    # weight rounded to fp16 once, otherwise exact in fp32), then one fp16 rounding: either way
    # the weight's own fp16 value
    wq = _wq()
    N = 136
    d = synth.w4a16_inputs(K, N, g, 1, seed=K + g)
    Wp = wq.wq_prepack(to_dev(d["Q"]), to_dev(d["s"]), g)
    eye = np.eye(K, dtype=np.float16)
    W = np.concatenate([wq.wq_gemm_w4a16(to_dev(eye[k:k + 4]), Wp, N, g).cpu().numpy() for k in range(0, K, 4)])
    exp = ((d["q"].astype(np.float32) - 8) * d["s"][np.arange(K) // g].astype(np.float32)).astype(np.float16)
    assert np.array_equal(W.view(np.uint16), exp.view(np.uint16))


# ---------------------------------------------------------------- W4A8 on the register-operand kernel
def _w4a8(d, with_acc=True):
    wq = _wq()
    M, N = d["M"], d["N"]
    Wp = wq.wq_prepack_w4a8(to_dev(d["Q"]))
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda") if with_acc else None
    Y = wq.wq_gemm_w4a8(to_dev(d["A"]), to_dev(d["sa"]), Wp, to_dev(d["sw"]), N, acc_out=acc)
    torch.cuda.synchronize()
    assert wq.wq_get_device_status() == wq.WQ_OK
    return Y, acc


@pytest.mark.parametrize("M", [1, 2, 3, 5, 8, 11, 16])
@pytest.mark.parametrize("K,N", [(128, 8), (4096, 264), (4096, 4096), (11008, 392)])
def test_rf_w4a8_exact_acc(M, K, N):
    wq = _wq()
    assert wq.wq_plan(1, M, N, K, K)["threads"] == 576
    d = synth.w4a8_inputs(K, N, M, seed=K + N + M)
    Y, acc = _w4a8(d)
    acc_ref, y_ref = oracle.w4a8(d["A"], d["sa"], d["Q"], d["sw"])
    got = acc.cpu().numpy().astype(np.int64)
    assert np.array_equal(got, acc_ref), f"{int((got != acc_ref).sum())} accumulators differ"
    compare(half_bits_to_f64(Y), y_ref, oracle.w4a8_absdot(d["A"], d["sa"], d["Q"], d["sw"]), f"rf w4a8 {K}x{N} M={M}")


def test_rf_w4a8_extremes():
    # a = -128 (the int8 minimum) against codes 0 and 15 over K = 16384, and a = 127: the largest sums
    K, N, M = 16384, 256, 2
    d = synth.w4a8_inputs(K, N, M, seed=1)  # two rows: the register-operand kernel's 2-row tile
    q = np.zeros((K, N), np.uint8)
    q[:, N // 2:] = 15
    d["Q"] = synth.pack_q(q)
    d["A"] = np.stack([np.full(K, -128, np.int8), np.full(K, 127, np.int8)])
    _, acc = _w4a8(d)
    got = acc.cpu().numpy()
    assert np.all(got[0, : N // 2] == 8 * 128 * K) and np.all(got[0, N // 2:] == -7 * 128 * K)
    assert np.all(got[1, : N // 2] == -8 * 127 * K) and np.all(got[1, N // 2:] == 7 * 127 * K)


@pytest.mark.parametrize("K,N", [(4096, 11008), (11008, 4096)])
@pytest.mark.parametrize("M", [1, 8, 16])
def test_rf_w4a8_full_sizes_sampled(K, N, M):
    d = synth.w4a8_inputs(K, N, M, seed=N + M)
    Y, acc = _w4a8(d)
    cols = sample_cols(N, 96, seed=M)
    acc_ref = oracle.w4a8_acc(d["A"], d["Q"][:, cols])
    assert np.array_equal(acc.cpu().numpy()[:, cols].astype(np.int64), acc_ref)


@pytest.mark.parametrize("M,bits", [(1, 8), (4, 8), (8, 4), (16, 8)])
def test_rf_w4a8_on_fp16_activations(M, bits):
    # the one-call quantise-then-multiply path on the register-operand kernel: accumulators
    # bit-exact against the oracle's quantiser and exact integer sums
    wq = _wq()
    K, N = 4096, 1032
    rng = np.random.default_rng(M + bits)
    A = rng.standard_normal((M, K)).astype(np.float16)
    d = synth.w4a8_inputs(K, N, M, seed=M)
    Wp = wq.wq_prepack_w4a8(to_dev(d["Q"]))
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    wq.wq_gemm_w4a8_fp16act(to_dev(A), Wp, to_dev(d["sw"]), N, acc_out=acc, act_bits=bits)
    torch.cuda.synchronize()
    q, sa = oracle.quantize_act(A, bits=bits)
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), oracle.w4a8_acc(q, d["Q"]))
