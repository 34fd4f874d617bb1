"""GPU tests of the layout pass: the CUDA prepack must equal the oracle's restatement of the
documented layout byte for byte, and unpack(prepack(Q, s)) must give (Q, s) back bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import synth
from wq_check import to_dev

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

SMALL = [(128, 128, 128), (256, 200, 64), (384, 136, 32), (512, 8, 256), (256, 264, 256), (1024, 392, 128),
         (128, 8, 32), (640, 1000, 128), (1280, 520, 640)]


@pytest.mark.parametrize("K,N,g", SMALL)
def test_prepack_matches_oracle_bytes(K, N, g):
    import bit_weight_quantized_prepack_b200 as wq
    d = synth.w4a16_inputs(K, N, g, 1, seed=K * 7 + N + g)
    Wp = wq.wq_prepack(to_dev(d["Q"]), to_dev(d["s"]), g)
    ref = oracle.prepack_w4a16(d["Q"], d["s"], g)
    got = Wp.cpu().numpy()
    assert got.nbytes == ref.nbytes
    assert np.array_equal(got, ref), f"first difference at byte {int(np.argmax(got != ref))}"


@pytest.mark.parametrize("K,N,g", SMALL)
def test_unpack_roundtrip(K, N, g):
    import bit_weight_quantized_prepack_b200 as wq
    d = synth.w4a16_inputs(K, N, g, 1, seed=K + 3 * N + g)
    Q, s = to_dev(d["Q"]), to_dev(d["s"])
    Q2, s2 = wq.wq_unpack(wq.wq_prepack(Q, s, g), K, N, g)
    assert torch.equal(Q2, Q)
    assert torch.equal(s2.view(torch.int16), s.view(torch.int16))


@pytest.mark.parametrize("K,N", [(128, 128), (256, 200), (640, 24), (1024, 1000)])
def test_prepack_w4a8_matches_oracle_and_roundtrips(K, N):
    import bit_weight_quantized_prepack_b200 as wq
    d = synth.w4a8_inputs(K, N, 1, seed=K + N)
    Q = to_dev(d["Q"])
    Wp = wq.wq_prepack_w4a8(Q)
    assert np.array_equal(Wp.cpu().numpy(), oracle.prepack_w4a8(d["Q"]))
    assert torch.equal(wq.wq_unpack_w4a8(Wp, K, N), Q)


# every weight shape of the layer configurations, round trip on the device (bit-exact)
FULL = [(4096, 4096), (4096, 12288), (4096, 22016), (11008, 4096), (8192, 10240), (8192, 8192),
        (8192, 57344), (28672, 8192)]


@pytest.mark.parametrize("K,N", FULL)
def test_full_size_roundtrip(K, N):
    import bit_weight_quantized_prepack_b200 as wq
    gen = torch.Generator(device="cuda").manual_seed(K + N)
    Q = torch.randint(-2 ** 31, 2 ** 31 - 1, (K // 8, N), dtype=torch.int32, device="cuda", generator=gen)
    for g in (128, K):
        s = torch.randn((K // g, N), device="cuda", generator=gen).to(torch.float16)
        Q2, s2 = wq.wq_unpack(wq.wq_prepack(Q, s, g), K, N, g)
        assert torch.equal(Q2, Q)
        assert torch.equal(s2.view(torch.int16), s.view(torch.int16))
    assert torch.equal(wq.wq_unpack_w4a8(wq.wq_prepack_w4a8(Q), K, N), Q)
