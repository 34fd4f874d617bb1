"""GPU parity of the layer with a zero point per group and column (asymmetric groups):
the prepacked buffer byte for byte against the oracle's layout, every output against the
fp64 oracle, zero point 8 bit for bit against the symmetric layer, and identity activations
reproducing fp16_rn((q - z) * s) bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import synth
from wq_check import compare, half_bits_to_f64, to_dev

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _wq():
    import bit_weight_quantized_prepack_b200 as wq
    return wq


def _zeros(K, N, g, seed):
    return np.random.default_rng(seed).integers(0, 16, (K // g, N)).astype(np.uint8)


@pytest.mark.parametrize("K,N,g", [(256, 200, 64), (384, 136, 32), (512, 264, 256), (1024, 392, 128)])
def test_prepack_zp_matches_oracle_bytes_and_roundtrips(K, N, g):
    wq = _wq()
    d = synth.w4a16_inputs(K, N, g, 1, seed=K + N)
    z = _zeros(K, N, g, K)
    Wp = wq.wq_prepack_zp(to_dev(d["Q"]), to_dev(d["s"]), to_dev(z), g)
    torch.cuda.synchronize()
    assert np.array_equal(Wp.cpu().numpy(), oracle.prepack_w4a16_zp(d["Q"], d["s"], z, g))
    Q, s, zz = wq.wq_unpack_zp(Wp, K, N, g)
    assert np.array_equal(Q.cpu().numpy(), d["Q"]) and np.array_equal(zz.cpu().numpy(), z)
    assert np.array_equal(s.cpu().numpy().view(np.uint16), d["s"].view(np.uint16))


# register-operand tiles, 32-row small tiles, large tiles, several m-tiles; group sizes below, at and above 128
CASES = [(1024, 264, 128, 1), (512, 392, 64, 5), (384, 136, 32, 16), (1024, 1024, 128, 17), (2048, 256, 256, 33),
         (1024, 512, 32, 100), (512, 640, 128, 300), (4096, 4096, 128, 16)]


@pytest.mark.parametrize("K,N,g,M", CASES)
def test_zp_layers_vs_oracle(K, N, g, M):
    wq = _wq()
    d = synth.w4a16_inputs(K, N, g, M, seed=K + N + M)
    z = _zeros(K, N, g, M)
    Wp = wq.wq_prepack_zp(to_dev(d["Q"]), to_dev(d["s"]), to_dev(z), g)
    Y = wq.wq_gemm_w4a16_zp(to_dev(d["A"]), Wp, N, g)
    torch.cuda.synchronize()
    assert wq.wq_get_device_status() == wq.WQ_OK
    compare(half_bits_to_f64(Y), oracle.w4a16_zp(d["A"], d["Q"], d["s"], z, g),
            oracle.w4a16_zp_absdot(d["A"], d["Q"], d["s"], z, g), f"zp K={K} N={N} g={g} M={M}")


@pytest.mark.parametrize("K,N,g,M", [(1024, 264, 128, 1), (384, 136, 32, 16), (1024, 1024, 128, 17), (512, 640, 64, 300)])
def test_zero_point_eight_is_the_symmetric_layer_bitwise(K, N, g, M):
    wq = _wq()
    d = synth.w4a16_inputs(K, N, g, M, seed=3 * K + M)
    A, Q, s = to_dev(d["A"]), to_dev(d["Q"]), to_dev(d["s"])
    Wz = wq.wq_prepack_zp(Q, s, torch.full((K // g, N), 8, dtype=torch.uint8, device="cuda"), g)
    Y1 = wq.wq_gemm_w4a16_zp(A, Wz, N, g)
    Y2 = wq.wq_gemm_w4a16(A, wq.wq_prepack(Q, s, g), N, g)
    torch.cuda.synchronize()
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))


@pytest.mark.parametrize("K,g", [(128, 32), (256, 128), (256, 64), (512, 256)])
def test_identity_activation_reproduces_asymmetric_weights_bitwise(K, g):
    wq = _wq()
    N = 136
    d = synth.w4a16_inputs(K, N, g, 1, seed=K + g)
    z = _zeros(K, N, g, g)
    Wp = wq.wq_prepack_zp(to_dev(d["Q"]), to_dev(d["s"]), to_dev(z), g)
    Y = wq.wq_gemm_w4a16_zp(to_dev(np.eye(K, dtype=np.float16)), Wp, N, g).cpu().numpy()
    grp = np.arange(K) // g
    exp = ((d["q"].astype(np.float32) - z[grp].astype(np.float32)) * d["s"][grp].astype(np.float32)).astype(np.float16)
    assert np.array_equal(Y.view(np.uint16), exp.view(np.uint16)), int((Y != exp).sum())
