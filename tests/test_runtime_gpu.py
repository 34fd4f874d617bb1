"""GPU tests of the runtime around the kernels: bounded waits that expire, CUDA-graph capture
with a reserved workspace, and concurrent calls on two streams."""
import numpy as np
import pytest
import torch

import synth
from wq_check import check_w4a16_full, to_dev

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _wq():
    import bit_weight_quantized_prepack_b200 as wq
    return wq


@pytest.mark.parametrize("M", [1, 24])  # the register-operand and the small-tile kernel
def test_expired_wait_reports_timeout_and_context_survives(M):
    # CTA 0 holds the first k-blocks of tile 0 and skips publishing its partial, so the CTA
    # that finishes tile 0 waits on a flag nothing sets. With a 20 ms limit the wait expires,
    # the call reports WQ_ERR_TIMEOUT, and the next call is correct.
    wq = _wq()
    K, N, g = 4096, 4096, 128
    plan = wq.wq_plan(0, M, N, K, g)
    assert plan["units"] > plan["grid"] > 1 and plan["units"] % plan["grid"] != 0
    d = synth.w4a16_inputs(K, N, g, M, seed=3)
    A = to_dev(d["A"])
    Wp = wq.wq_prepack(to_dev(d["Q"]), to_dev(d["s"]), g)
    assert wq.wq_get_device_status() == wq.WQ_OK
    wq.wq_debug_set_wait_timeout_ns(20_000_000)
    wq.wq_debug_skip_publish(0)
    try:
        wq.wq_gemm_w4a16(A, Wp, N, g)
        assert wq.wq_get_device_status() == wq.WQ_ERR_TIMEOUT
    finally:
        wq.wq_debug_skip_publish(-1)
        wq.wq_debug_set_wait_timeout_ns(0)
    assert wq.wq_get_device_status() == wq.WQ_OK
    Y = wq.wq_gemm_w4a16(A, Wp, N, g)
    assert wq.wq_get_device_status() == wq.WQ_OK
    check_w4a16_full(d, Y, "after an expired wait")


def test_graph_capture_with_reserved_workspace():
    wq = _wq()
    K, N, g, M = 4096, 4096, 128, 16
    d = synth.w4a16_inputs(K, N, g, M, seed=4)
    A = to_dev(d["A"])
    Wp = wq.wq_prepack(to_dev(d["Q"]), to_dev(d["s"]), g)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    Y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    with torch.cuda.stream(s):
        wq.wq_workspace_reserve(wq.wq_workspace_bytes(0, M, N, K), stream=s)
        Y_eager = wq.wq_gemm_w4a16(A, Wp, N, g, stream=s)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=s):
            wq.wq_gemm_w4a16(A, Wp, N, g, Y=Y, stream=s)
    for _ in range(3):
        Y.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(Y.view(torch.int16), Y_eager.view(torch.int16))
    check_w4a16_full(d, Y, "graph replay")


def test_capture_without_reserved_workspace_is_refused():
    wq = _wq()
    K, N, g, M = 1024, 1024, 128, 200
    d = synth.w4a16_inputs(K, N, g, M, seed=5)
    A = to_dev(d["A"])
    Wp = wq.wq_prepack(to_dev(d["Q"]), to_dev(d["s"]), g)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with pytest.raises(wq.WqError) as ei:
        with torch.cuda.stream(s):
            with torch.cuda.graph(graph, stream=s):
                wq.wq_gemm_w4a16(A, Wp, N, g, stream=s)
    assert ei.value.status == wq.WQ_ERR_CAPTURING


def test_two_streams_concurrently():
    # Three layers of different shapes and kernels (register-operand, 32-row and large tiles) on
    # three streams, 50 rounds: the kernels may run side by side, so a stream-K owner may find
    # the CTAs it waits for not yet resident; its waits are bounded and no round may time out.
    # Every round must report WQ_OK and match the oracle.
    import oracle
    from wq_check import compare, half_bits_to_f64
    wq = _wq()
    K, g = 4096, 128
    cases = [synth.w4a16_inputs(K, 4096, g, 3, seed=6), synth.w4a16_inputs(K, 2048, g, 40, seed=7),
             synth.w4a16_inputs(K, 3072, g, 24, seed=8)]
    refs = [(oracle.w4a16(d["A"], d["Q"], d["s"], g), oracle.w4a16_absdot(d["A"], d["Q"], d["s"], g)) for d in cases]
    dev = [(to_dev(d["A"]), wq.wq_prepack(to_dev(d["Q"]), to_dev(d["s"]), g)) for d in cases]
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream() for _ in cases]
    for it in range(50):
        outs = [None] * len(cases)
        for i, (st, (A, Wp)) in enumerate(zip(streams, dev)):
            with torch.cuda.stream(st):
                outs[i] = wq.wq_gemm_w4a16(A, Wp, cases[i]["N"], g, stream=st)
        torch.cuda.synchronize()
        for st in streams:
            assert wq.wq_get_device_status(st) == wq.WQ_OK, f"round {it}"
        for (y_ref, ad), Y in zip(refs, outs):
            compare(half_bits_to_f64(Y), y_ref, ad, f"two streams, round {it}")


@pytest.mark.parametrize("M", [3, 24])  # register-operand and 32-row tiles
def test_graph_capture_of_the_one_call_entry_points(M):
    # the act-order layer (gather + layer) and W4A8 on fp16 activations (quantise + layer) keep
    # their intermediate buffers in the stream's workspace: with the workspace of their kind
    # reserved, a captured call replays the eager call bit for bit
    import oracle
    wq = _wq()
    K, N, g = 2048, 1032, 128
    d = synth.w4a16_inputs(K, N, g, M, seed=M)
    rng = np.random.default_rng(M)
    gidx = rng.permutation(np.arange(K) // g)
    perm = to_dev(oracle.act_order_perm(gidx, g).astype(np.int32))
    A = to_dev(d["A"])
    Wa = wq.wq_prepack_act_order(to_dev(d["Q"]), to_dev(d["s"]), perm, g)
    W8 = wq.wq_prepack_w4a8(to_dev(d["Q"]))
    sw = to_dev(np.full(N, 0.01, np.float32))
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    Y1 = torch.empty((M, N), dtype=torch.float16, device="cuda")
    Y2 = torch.empty((M, N), dtype=torch.float16, device="cuda")
    with torch.cuda.stream(s):
        wq.wq_workspace_reserve(max(wq.wq_workspace_bytes(4, M, N, K), wq.wq_workspace_bytes(2, M, N, K)), stream=s)
        E1 = wq.wq_gemm_w4a16_act_order(A, perm, Wa, N, g, stream=s)
        E2 = wq.wq_gemm_w4a8_fp16act(A, W8, sw, N, stream=s)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=s):
            wq.wq_gemm_w4a16_act_order(A, perm, Wa, N, g, Y=Y1, stream=s)
            wq.wq_gemm_w4a8_fp16act(A, W8, sw, N, Y=Y2, stream=s)
    for _ in range(3):
        Y1.zero_()
        Y2.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(Y1.view(torch.int16), E1.view(torch.int16))
        assert torch.equal(Y2.view(torch.int16), E2.view(torch.int16))
    assert wq.wq_get_device_status(s) == wq.WQ_OK
