"""GPU parity of the W4A8 layer: int32 accumulators bit-exact against the oracle's exact
integer sums, fp16 outputs within the tolerance of the scale epilogue."""
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


def _run(d, with_acc=True):
    wq = _wq()
    M, N = d["M"], d["N"]
    Wp = wq.wq_prepack_w4a8(to_dev(d["Q"]))
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda") if with_acc else None
    Y = wq.wq_gemm_w4a8(to_dev(d["A"]), to_dev(d["sa"]), Wp, to_dev(d["sw"]), N, acc_out=acc)
    torch.cuda.synchronize()
    return Wp, Y, acc


SMALL = [(128, 128, 1), (256, 136, 3), (1024, 264, 17), (2048, 1000, 129), (512, 512, 256), (1280, 392, 300),
         (384, 8, 2), (4096, 256, 64), (512, 264, 16), (1024, 392, 32)]


@pytest.mark.parametrize("K,N,M", SMALL)
def test_small_layers_exact_acc(K, N, M):
    d = synth.w4a8_inputs(K, N, M, seed=K + N + M)
    _, Y, acc = _run(d)
    acc_ref, y_ref = oracle.w4a8(d["A"], d["sa"], d["Q"], d["sw"])
    got = acc.cpu().numpy().astype(np.int64)
    assert np.array_equal(got, acc_ref), f"{int((got != acc_ref).sum())} accumulators differ"
    compare(half_bits_to_f64(Y), y_ref, oracle.w4a8_absdot(d["A"], d["sa"], d["Q"], d["sw"]), f"{K}x{N} M={M}")


def test_accumulator_extremes():
    # |acc| at its largest: a = -127 everywhere against codes 0 (q-8 = -8) and 15 (q-8 = 7)
    K, N, M = 16384, 256, 3
    d = synth.w4a8_inputs(K, N, M, seed=1)
    q = np.zeros((K, N), np.uint8)
    q[:, N // 2:] = 15
    d["Q"] = synth.pack_q(q)
    d["A"] = np.full((M, K), -127, np.int8)
    _, Y, acc = _run(d)
    got = acc.cpu().numpy()
    assert np.all(got[:, : N // 2] == 8 * 127 * K) and np.all(got[:, N // 2:] == -7 * 127 * K)


def test_acc_out_optional_and_same_output():
    d = synth.w4a8_inputs(1024, 520, 33, seed=2)
    _, Y1, _ = _run(d, with_acc=True)
    _, Y2, _ = _run(d, with_acc=False)
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))


@pytest.mark.parametrize("K,N", [(4096, 11008), (11008, 4096)])
def test_w4a8_layers(K, N):
    wq = _wq()
    d = synth.w4a8_inputs(K, N, 1024, seed=0)
    Wp = wq.wq_prepack_w4a8(to_dev(d["Q"]))
    A, sa, sw = to_dev(d["A"]), to_dev(d["sa"]), to_dev(d["sw"])
    acc_ref128, y_ref128 = oracle.w4a8(d["A"][:128], d["sa"][:128], d["Q"], d["sw"])
    ad128 = oracle.w4a8_absdot(d["A"][:128], d["sa"][:128], d["Q"], d["sw"])
    cols = sample_cols(N, 512, seed=K)
    accc, yc = oracle.w4a8(d["A"], d["sa"], d["Q"][:, cols], d["sw"][cols])
    adc = oracle.w4a8_absdot(d["A"], d["sa"], d["Q"][:, cols], d["sw"][cols])
    for M in (1, 16, 128, 1024):
        acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
        Y = wq.wq_gemm_w4a8(A[:M].contiguous(), sa[:M].contiguous(), Wp, sw, N, acc_out=acc)
        got = acc.cpu().numpy().astype(np.int64)
        y = half_bits_to_f64(Y)
        if M <= 128:  # every output
            assert np.array_equal(got, acc_ref128[:M]), f"M={M}: {int((got != acc_ref128[:M]).sum())} differ"
            compare(y, y_ref128[:M], ad128[:M], f"W4A8 {K}x{N} M={M}")
        else:  # sampled columns, every row
            assert np.array_equal(got[:, cols], accc), f"M={M}: {int((got[:, cols] != accc).sum())} differ"
            compare(y[:, cols], yc, adc, f"W4A8 {K}x{N} M={M}")
