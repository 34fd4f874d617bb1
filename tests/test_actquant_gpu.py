"""GPU parity of the per-token activation quantisation and of the W4A8 layer on fp16
activations (wq_gemm_w4a8_fp16act) against the oracle: int8 codes and fp32 scales bit for bit
(both sides take the rounding decisions in the same fp32 operations), the fused call's int32
accumulators bit for bit, Y within the tolerance."""
import numpy as np
import pytest
import torch

import oracle
import synth
from oracle_pins import golden_act_quant
from wq_check import compare, half_bits_to_f64, sample_cols, to_dev

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _wq():
    import bit_weight_quantized_prepack_b200 as wq
    return wq


def _acts(M, K, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((M, K)) * scale).astype(np.float16)


@pytest.mark.parametrize("bits", [8, 4])
def test_hand_worked_rows_bitwise(bits):
    wq = _wq()
    rows = golden_act_quant(bits)
    A = np.zeros((len(rows), 8), np.float16)
    for i, (a, _, _) in enumerate(rows):
        A[i] = a
    # K must be a multiple of 8: the worked rows are exactly 8 long
    q, sa = wq.wq_quantize_act(to_dev(A), bits=bits)
    torch.cuda.synchronize()
    for i, (_, codes, s) in enumerate(rows):
        assert q[i].cpu().tolist() == codes, (i, q[i].cpu().tolist(), codes)
        if s is not None:
            assert float(sa[i]) == s


@pytest.mark.parametrize("M,K,scale,bits", [(1, 4096, 1.0, 8), (16, 11008, 3.0, 8), (128, 4096, 0.01, 8),
                                            (3, 8, 1.0, 8), (300, 1024, 100.0, 8), (64, 28672, 1.0, 8),
                                            (16, 11008, 3.0, 4), (300, 1024, 100.0, 4)])
def test_codes_and_scales_bitwise(M, K, scale, bits):
    wq = _wq()
    A = _acts(M, K, M + K, scale)
    A[0, :] = 0  # a zero row
    if M > 2:
        A[2, : K // 2] = np.float16(0.5)  # ties: amax 0.5, 0.25 * inv is exactly half of the top level
        A[2, K // 2:] = np.float16(0.25) * np.where(np.arange(K - K // 2) % 2 == 0, 1, -1).astype(np.float16)
    q, sa = wq.wq_quantize_act(to_dev(A), bits=bits)
    torch.cuda.synchronize()
    q_ref, sa_ref = oracle.quantize_act(A, bits=bits)
    assert np.array_equal(q.cpu().numpy(), q_ref), int((q.cpu().numpy() != q_ref).sum())
    assert np.array_equal(sa.cpu().numpy().view(np.uint32), sa_ref.view(np.uint32))


@pytest.mark.parametrize("K,N", [(4096, 11008), (11008, 4096)])
@pytest.mark.parametrize("M", [1, 16, 128])
def test_w4a8_on_fp16_activations_vs_oracle(K, N, M):
    wq = _wq()
    d = synth.w4a8_inputs(K, N, 1, seed=K + M)
    A = _acts(M, K, seed=N + M)
    Wp = wq.wq_prepack_w4a8(to_dev(d["Q"]))
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    sa = torch.empty((M,), dtype=torch.float32, device="cuda")
    Y = wq.wq_gemm_w4a8_fp16act(to_dev(A), Wp, to_dev(d["sw"]), N, acc_out=acc, sa_out=sa)
    torch.cuda.synchronize()
    assert wq.wq_get_device_status() == wq.WQ_OK
    q_ref, sa_ref = oracle.quantize_act(A)
    assert np.array_equal(sa.cpu().numpy().view(np.uint32), sa_ref.view(np.uint32))
    acc_ref, y_ref = oracle.w4a8(q_ref, sa_ref, d["Q"], d["sw"])
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), acc_ref)
    compare(half_bits_to_f64(Y), y_ref, oracle.w4a8_absdot(q_ref, sa_ref, d["Q"], d["sw"]), f"K={K} N={N} M={M}")


def test_w4a8_on_fp16_activations_large_m_sampled():
    wq = _wq()
    K, N, M = 4096, 11008, 1024
    d = synth.w4a8_inputs(K, N, 1, seed=5)
    A = _acts(M, K, seed=6)
    Wp = wq.wq_prepack_w4a8(to_dev(d["Q"]))
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    Y = wq.wq_gemm_w4a8_fp16act(to_dev(A), Wp, to_dev(d["sw"]), N, acc_out=acc)
    torch.cuda.synchronize()
    cols = sample_cols(N, 40, seed=1)
    q_ref, sa_ref = oracle.quantize_act(A)
    acc_ref, y_ref = oracle.w4a8(q_ref, sa_ref, d["Q"][:, cols], d["sw"][cols])
    assert np.array_equal(acc.cpu().numpy()[:, cols].astype(np.int64), acc_ref)
    compare(half_bits_to_f64(Y)[:, cols], y_ref, oracle.w4a8_absdot(q_ref, sa_ref, d["Q"][:, cols], d["sw"][cols]))


def test_fused_call_matches_the_two_step_path_bitwise():
    # quantise, then the int8 layer, through the separate entry points: the same bits as the one call
    wq = _wq()
    K, N, M = 4096, 4096, 40
    d = synth.w4a8_inputs(K, N, 1, seed=8)
    A = to_dev(_acts(M, K, seed=9))
    Wp = wq.wq_prepack_w4a8(to_dev(d["Q"]))
    sw = to_dev(d["sw"])
    q, sa = wq.wq_quantize_act(A)
    Y2 = wq.wq_gemm_w4a8(q, sa, Wp, sw, N)
    Y1 = wq.wq_gemm_w4a8_fp16act(A, Wp, sw, N)
    torch.cuda.synchronize()
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))


@pytest.mark.parametrize("K,N,M", [(4096, 11008, 16), (11008, 4096, 128)])
def test_w4a4_numerics_vs_oracle(K, N, M):
    # 4-bit per-token activations, held one per int8, on the int8 tensor cores
    wq = _wq()
    d = synth.w4a8_inputs(K, N, 1, seed=K + 4 * M)
    A = _acts(M, K, seed=N + 4 * M)
    Wp = wq.wq_prepack_w4a8(to_dev(d["Q"]))
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    sa = torch.empty((M,), dtype=torch.float32, device="cuda")
    Y = wq.wq_gemm_w4a8_fp16act(to_dev(A), Wp, to_dev(d["sw"]), N, acc_out=acc, sa_out=sa, act_bits=4)
    torch.cuda.synchronize()
    q_ref, sa_ref = oracle.quantize_act(A, bits=4)
    assert np.abs(q_ref).max() <= 7
    assert np.array_equal(sa.cpu().numpy().view(np.uint32), sa_ref.view(np.uint32))
    acc_ref, y_ref = oracle.w4a8(q_ref, sa_ref, d["Q"], d["sw"])
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), acc_ref)
    compare(half_bits_to_f64(Y), y_ref, oracle.w4a8_absdot(q_ref, sa_ref, d["Q"], d["sw"]), f"W4A4 K={K} N={N} M={M}")
