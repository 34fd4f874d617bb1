"""GPU parity of act order (groups scattered along K by g_idx): the reordered buffer byte for
byte against the oracle's layout, the activation gather bit for bit, and the one-call layer
against the fp64 oracle of the definition with g_idx."""
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


def _case(K, N, g, M, zp, seed):
    d = synth.w4a16_inputs(K, N, g, M, seed=seed)
    rng = np.random.default_rng(seed + 7)
    gidx = rng.permutation(np.arange(K) // g)
    z = rng.integers(0, 16, (K // g, N)).astype(np.uint8) if zp else None
    perm = oracle.act_order_perm(gidx, g).astype(np.int32)
    return d, gidx, z, perm


@pytest.mark.parametrize("K,N,g,zp", [(256, 200, 64, False), (384, 136, 32, True), (512, 264, 256, True),
                                      (1024, 392, 128, False), (512, 136, 512, False)])
def test_prepack_act_order_matches_oracle_bytes(K, N, g, zp):
    wq = _wq()
    d, gidx, z, perm = _case(K, N, g, 1, zp, K + N)
    Wp = wq.wq_prepack_act_order(to_dev(d["Q"]), to_dev(d["s"]), to_dev(perm), g, z=None if z is None else to_dev(z))
    torch.cuda.synchronize()
    assert np.array_equal(Wp.cpu().numpy(), oracle.prepack_w4a16_act_order(d["Q"], d["s"], z, perm, g))


@pytest.mark.parametrize("M,K", [(1, 128), (3, 4096), (40, 11008), (257, 1024)])
def test_permute_act_bitwise(M, K):
    wq = _wq()
    rng = np.random.default_rng(M + K)
    A = rng.standard_normal((M, K)).astype(np.float16)
    perm = rng.permutation(K).astype(np.int32)
    out = wq.wq_permute_act(to_dev(A), to_dev(perm))
    torch.cuda.synchronize()
    assert wq.wq_get_device_status() == wq.WQ_OK
    assert np.array_equal(out.cpu().numpy().view(np.uint16), A[:, perm].view(np.uint16))


# register-operand tiles, 32-row small tiles, large tiles, ragged N, group sizes below, at and above 128
CASES = [(1024, 264, 128, 1, False), (1024, 264, 128, 1, True), (512, 392, 64, 5, True), (384, 136, 32, 16, False),
         (1024, 1024, 128, 33, True), (2048, 256, 256, 17, False), (1024, 640, 32, 300, True),
         (4096, 4096, 128, 8, True)]


@pytest.mark.parametrize("K,N,g,M,zp", CASES)
def test_act_order_layer_vs_oracle(K, N, g, M, zp):
    wq = _wq()
    d, gidx, z, perm = _case(K, N, g, M, zp, K + N + M)
    p = to_dev(perm)
    Wp = wq.wq_prepack_act_order(to_dev(d["Q"]), to_dev(d["s"]), p, g, z=None if z is None else to_dev(z))
    Y = wq.wq_gemm_w4a16_act_order(to_dev(d["A"]), p, Wp, N, g, zero_points=zp)
    torch.cuda.synchronize()
    assert wq.wq_get_device_status() == wq.WQ_OK
    compare(half_bits_to_f64(Y), oracle.w4a16_gidx(d["A"], d["Q"], d["s"], z, gidx),
            oracle.w4a16_gidx_absdot(d["A"], d["Q"], d["s"], z, gidx), f"act order K={K} N={N} g={g} M={M} zp={zp}")


def test_act_order_equals_gather_then_grouped_layer_bitwise():
    # the one-call layer is the gather followed by the grouped layer, bit for bit
    wq = _wq()
    K, N, g, M = 2048, 512, 128, 24
    d, gidx, z, perm = _case(K, N, g, M, True, 5)
    p = to_dev(perm)
    Wp = wq.wq_prepack_act_order(to_dev(d["Q"]), to_dev(d["s"]), p, g, z=to_dev(z))
    A = to_dev(d["A"])
    Y1 = wq.wq_gemm_w4a16_act_order(A, p, Wp, N, g, zero_points=True)
    Y2 = wq.wq_gemm_w4a16_zp(wq.wq_permute_act(A, p), Wp, N, g)
    torch.cuda.synchronize()
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))


def test_prepack_refuses_a_perm_that_is_not_a_permutation():
    wq = _wq()
    K, N, g = 256, 128, 64
    d = synth.w4a16_inputs(K, N, g, 1, seed=3)
    for bad in (np.zeros(K, np.int32), np.r_[np.arange(K - 1), K].astype(np.int32),
                np.r_[np.arange(K - 1), -1].astype(np.int32)):
        with pytest.raises(wq.WqError):
            wq.wq_prepack_act_order(to_dev(d["Q"]), to_dev(d["s"]), to_dev(bad), g)
    assert wq.wq_get_device_status() == wq.WQ_OK


def test_gather_index_out_of_range_is_reported_not_read():
    # the kernel's own bounds check: the element becomes 0 and the status word records it
    wq = _wq()
    M, K = 2, 256
    A = np.ones((M, K), np.float16)
    perm = np.arange(K, dtype=np.int32)
    perm[5] = K
    perm[9] = -3
    out = wq.wq_permute_act(to_dev(A), to_dev(perm)).cpu().numpy()
    assert wq.wq_get_device_status() == wq.WQ_ERR_INVALID_ARG
    assert wq.wq_get_device_status() == wq.WQ_OK
    exp = np.ones((M, K), np.float16)
    exp[:, [5, 9]] = 0
    assert np.array_equal(out, exp)
