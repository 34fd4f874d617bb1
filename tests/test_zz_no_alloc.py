"""GPU test of wq_gemm_w4a16_noalloc, the W4A16 call that allocates no device memory.

Some callers cannot allocate device memory when they run the layer: an inference engine that
hands all free memory to its own pool at start-up, a plugin whose host framework owns every
allocation, a latency-critical loop that must not risk the implicit synchronisation of an
allocation. For them the library keeps the stream-K scratch of the W4A16 kernels in one fixed
8 MiB device array instead of a cudaMalloc'd workspace.

The test calls the entry point through the C ABI (ctypes, raw device pointers) twice in a
row with different activations, so that the second call runs on the scratch the first one
left behind. Each output is compared with the fp64 oracle within the parity tolerance of the
other tests and, since both entry points run the same deterministic kernels, bit for bit with
the regular entry point on the same inputs. The cases cover register-operand tiles, 32-row tiles, a
large tile and per-column scales (g = K). The test also checks that the second call leaves
the device's free memory unchanged, that a call needing more scratch than the array holds is
refused without a launch, and that an expired device-side wait of the fixed-scratch call is
reported by wq_get_device_status. The file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _c_abi(wq, A, Wp, Y, N, g):
    M, K = A.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return wq.lib.wq_gemm_w4a16_noalloc(ctypes.c_void_p(A.data_ptr()), ctypes.c_void_p(Wp.data_ptr()),
                                        ctypes.c_void_p(Y.data_ptr()), M, N, K, g, stream)


# (K, N, g, M): register-operand tiles (M = 5, 12); 32-row tiles; a 48-row large tile; per-column
# scales on the register-operand kernel (M = 3) and 32-row tiles; g = 64 at M = 1
CASES = [(4096, 1032, 128, 5), (4096, 1032, 128, 12), (1024, 1032, 128, 28), (2048, 2056, 64, 40),
         (2048, 520, 2048, 3), (1024, 264, 1024, 24), (4096, 1032, 64, 1)]


@pytest.mark.parametrize("K,N,g,M", CASES)
def test_noalloc_matches_the_oracle_twice_in_a_row(K, N, g, M):
    import bit_weight_quantized_prepack_b200 as wq
    import oracle
    import synth
    from wq_check import compare
    d = synth.w4a16_inputs(K, N, g, M, seed=11)
    Q = torch.from_numpy(d["Q"]).cuda()
    s = torch.from_numpy(d["s"]).cuda()
    Wp = wq.wq_prepack(Q, s, g)
    rng = np.random.default_rng(5)
    Y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    for call in range(2):
        A_np = d["A"] if call == 0 else rng.standard_normal((M, K)).astype(np.float16)
        A = torch.from_numpy(A_np).cuda()
        Y.fill_(float("nan"))
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        rc = _c_abi(wq, A, Wp, Y, N, g)
        assert rc == wq.WQ_OK, wq.status_string(rc)
        torch.cuda.synchronize()
        if call == 1:  # the first call on a device may load the library's device code
            assert torch.cuda.mem_get_info()[0] == free_before, "the call changed free device memory"
        assert wq.wq_get_device_status() == wq.WQ_OK
        y = Y.float().cpu().numpy().astype(np.float64)
        y_ref = oracle.w4a16(A_np, d["Q"], d["s"], g)
        compare(y, y_ref, oracle.w4a16_absdot(A_np, d["Q"], d["s"], g), f"call {call}")
        Y_alloc = wq.wq_gemm_w4a16(A, Wp, N, g)
        torch.cuda.synchronize()
        assert torch.equal(Y.view(torch.int16), Y_alloc.view(torch.int16)), f"call {call}: bits differ"


def test_noalloc_refuses_a_plan_beyond_its_scratch():
    import bit_weight_quantized_prepack_b200 as wq
    K, N, g, M = 1024, 1024, 128, 512  # 256-row tiles on every SM: about 19 MB of scratch
    Wp = torch.zeros(wq.wq_prepacked_bytes(K, N, g), dtype=torch.uint8, device="cuda")
    A = torch.zeros((M, K), dtype=torch.float16, device="cuda")
    Y = torch.full((M, N), 7.0, dtype=torch.float16, device="cuda")
    torch.cuda.synchronize()
    rc = _c_abi(wq, A, Wp, Y, N, g)
    assert rc == wq.WQ_ERR_SCRATCH_LIMIT, wq.status_string(rc)
    torch.cuda.synchronize()
    assert bool((Y == 7.0).all()), "a refused call must launch nothing"


def test_noalloc_expired_wait_is_reported_and_cleared():
    # CTA 0 skips publishing its partial, so the owner of tile 0 waits on a flag that nothing
    # sets; with a 20 ms limit the wait expires. wq_get_device_status reports it from the fixed
    # array's own status word, clears it, and the next call is correct.
    import bit_weight_quantized_prepack_b200 as wq
    import oracle
    import synth
    from wq_check import compare
    K, N, g, M = 4096, 4096, 128, 1
    plan = wq.wq_plan(0, M, N, K, g)
    assert plan["units"] > plan["grid"] > 1 and plan["units"] % plan["grid"] != 0
    d = synth.w4a16_inputs(K, N, g, M, seed=3)
    A = torch.from_numpy(d["A"]).cuda()
    Wp = wq.wq_prepack(torch.from_numpy(d["Q"]).cuda(), torch.from_numpy(d["s"]).cuda(), g)
    Y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    assert wq.wq_get_device_status() == wq.WQ_OK
    wq.wq_debug_set_wait_timeout_ns(20_000_000)
    wq.wq_debug_skip_publish(0)
    try:
        assert _c_abi(wq, A, Wp, Y, N, g) == wq.WQ_OK
        assert wq.wq_get_device_status() == wq.WQ_ERR_TIMEOUT
    finally:
        wq.wq_debug_skip_publish(-1)
        wq.wq_debug_set_wait_timeout_ns(0)
    assert wq.wq_get_device_status() == wq.WQ_OK
    assert _c_abi(wq, A, Wp, Y, N, g) == wq.WQ_OK
    assert wq.wq_get_device_status() == wq.WQ_OK
    y = Y.float().cpu().numpy().astype(np.float64)
    compare(y, oracle.w4a16(d["A"], d["Q"], d["s"], g), oracle.w4a16_absdot(d["A"], d["Q"], d["s"], g),
            "after an expired wait")
