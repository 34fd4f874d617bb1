"""CPU tests of the binding's argument checks: a wrongly sized buffer is refused in Python,
before any call reaches the library (where it would become an out-of-bounds copy or store
on the device). The library object is replaced by a recorder, so the tests also show that
nothing was called; size queries are answered by the real library (host arithmetic only)."""
import pytest
import torch

import bit_weight_quantized_prepack_b200 as wq


class _Recorder:
    """Stands in for the loaded library: records every entry point called, except the pure size
    queries, which it forwards to the real library."""
    PURE = {"wq_prepacked_bytes", "wq_prepacked_bytes_w4a8", "wq_prepacked_bytes_zp", "wq_prepacked_bytes_sparse24",
            "wq_prepacked_bytes_mixed", "wq_status_string"}

    def __init__(self, real):
        self.real, self.calls = real, []

    def __getattr__(self, name):
        if name in self.PURE:
            return getattr(self.real, name)

        def f(*args):
            self.calls.append(name)
            return 0
        return f


@pytest.fixture
def rec(monkeypatch):
    r = _Recorder(wq.lib)
    monkeypatch.setattr(wq, "lib", r)
    return r


K, N, g, M = 256, 136, 128, 3


def _w4a16(**over):
    a = {"A": torch.zeros((M, K), dtype=torch.float16),
         "Wp": torch.zeros(wq.wq_prepacked_bytes(K, N, g), dtype=torch.uint8),
         "Y": torch.zeros((M, N), dtype=torch.float16)}
    a.update(over)
    return a


@pytest.mark.parametrize("what,over", [
    ("Wp too small", {"Wp": torch.zeros(wq.wq_prepacked_bytes(K, N, g) - 1, dtype=torch.uint8)}),
    ("Y rows", {"Y": torch.zeros((M + 1, N), dtype=torch.float16)}),
    ("Y cols", {"Y": torch.zeros((M, N - 8), dtype=torch.float16)}),
    ("A not 2-D", {"A": torch.zeros((M * K,), dtype=torch.float16)}),
])
def test_gemm_w4a16_refuses_wrong_sizes(rec, what, over):
    a = _w4a16(**over)
    with pytest.raises(ValueError):
        wq.wq_gemm_w4a16(a["A"], a["Wp"], N, g, Y=a["Y"])
    with pytest.raises(ValueError):
        wq.wq_gemm_w4a16_noalloc(a["A"], a["Wp"], N, g, a["Y"])
    assert rec.calls == []


def test_gemm_w4a16_wrong_dtype_and_device(rec):
    a = _w4a16(Y=torch.zeros((M, N), dtype=torch.float32))
    with pytest.raises(TypeError):
        wq.wq_gemm_w4a16(a["A"], a["Wp"], N, g, Y=a["Y"])
    a = _w4a16()  # right sizes, but host tensors: refused as not CUDA
    with pytest.raises(TypeError, match="CUDA"):
        wq.wq_gemm_w4a16(a["A"], a["Wp"], N, g, Y=a["Y"])
    with pytest.raises(wq.WqError):  # g does not divide K
        wq.wq_gemm_w4a16(a["A"], a["Wp"], N, 96, Y=a["Y"])
    with pytest.raises(ValueError):  # the fixed-scratch call allocates nothing: Y is required
        wq.wq_gemm_w4a16_noalloc(a["A"], a["Wp"], N, g, None)
    assert rec.calls == []


def _w4a8(**over):
    a = {"A": torch.zeros((M, K), dtype=torch.int8), "sa": torch.ones(M, dtype=torch.float32),
         "Wp": torch.zeros(wq.wq_prepacked_bytes_w4a8(K, N), dtype=torch.uint8),
         "sw": torch.ones(N, dtype=torch.float32), "Y": torch.zeros((M, N), dtype=torch.float16),
         "acc": torch.zeros((M, N), dtype=torch.int32)}
    a.update(over)
    return a


@pytest.mark.parametrize("over", [
    {"sa": torch.ones(M - 1, dtype=torch.float32)},
    {"sw": torch.ones(N + 8, dtype=torch.float32)},
    {"Wp": torch.zeros(wq.wq_prepacked_bytes_w4a8(K, N) // 2, dtype=torch.uint8)},
    {"Y": torch.zeros((M, N + 8), dtype=torch.float16)},
    {"acc": torch.zeros((M - 1, N), dtype=torch.int32)},
])
def test_gemm_w4a8_refuses_wrong_sizes(rec, over):
    a = _w4a8(**over)
    with pytest.raises(ValueError):
        wq.wq_gemm_w4a8(a["A"], a["sa"], a["Wp"], a["sw"], N, Y=a["Y"], acc_out=a["acc"])
    assert rec.calls == []


def test_prepack_and_unpack_refuse_wrong_sizes(rec):
    Q = torch.zeros((K // 8, N), dtype=torch.int32)
    with pytest.raises(ValueError):  # s must be [K/g, N]
        wq.wq_prepack(Q, torch.zeros((K // g + 1, N), dtype=torch.float16), g)
    with pytest.raises(ValueError):  # caller-given Wp too small
        wq.wq_prepack(Q, torch.zeros((K // g, N), dtype=torch.float16), g,
                      Wp=torch.zeros(16, dtype=torch.uint8))
    with pytest.raises(ValueError):
        wq.wq_prepack_w4a8(Q, Wp=torch.zeros(16, dtype=torch.uint8))
    with pytest.raises(ValueError):
        wq.wq_unpack(torch.zeros(16, dtype=torch.uint8), K, N, g)
    with pytest.raises(ValueError):
        wq.wq_unpack_w4a8(torch.zeros(16, dtype=torch.uint8), K, N)
    assert rec.calls == []


def test_zero_point_calls_refuse_wrong_sizes(rec):
    Q = torch.zeros((K // 8, N), dtype=torch.int32)
    s = torch.zeros((K // g, N), dtype=torch.float16)
    with pytest.raises(ValueError):  # z must be [K/g, N]
        wq.wq_prepack_zp(Q, s, torch.zeros((K // g, N + 8), dtype=torch.uint8), g)
    with pytest.raises(TypeError):  # z must be uint8
        wq.wq_prepack_zp(Q, s, torch.zeros((K // g, N), dtype=torch.int32), g)
    with pytest.raises(wq.WqError):  # zero points need g < K
        wq.wq_prepack_zp(Q, torch.zeros((1, N), dtype=torch.float16), torch.zeros((1, N), dtype=torch.uint8), K)
    with pytest.raises(ValueError):  # the zero-point buffer is larger than the symmetric one
        wq.wq_gemm_w4a16_zp(torch.zeros((M, K), dtype=torch.float16),
                            torch.zeros(wq.wq_prepacked_bytes(K, N, g), dtype=torch.uint8), N, g)
    assert rec.calls == []


def test_act_order_calls_refuse_wrong_sizes(rec):
    Q = torch.zeros((K // 8, N), dtype=torch.int32)
    s = torch.zeros((K // g, N), dtype=torch.float16)
    perm = torch.arange(K, dtype=torch.int32)
    with pytest.raises(ValueError):  # perm must be [K]
        wq.wq_prepack_act_order(Q, s, perm[:-8], g)
    with pytest.raises(TypeError):  # perm must be int32
        wq.wq_prepack_act_order(Q, s, perm.long(), g)
    with pytest.raises(ValueError):  # z must be [K/g, N]
        wq.wq_prepack_act_order(Q, s, perm, g, z=torch.zeros((K // g + 1, N), dtype=torch.uint8))
    A = torch.zeros((M, K), dtype=torch.float16)
    with pytest.raises(ValueError):
        wq.wq_permute_act(A, perm, A_out=torch.zeros((M, K + 8), dtype=torch.float16))
    with pytest.raises(ValueError):  # the zero-point buffer is larger than the symmetric one
        wq.wq_gemm_w4a16_act_order(A, perm, torch.zeros(wq.wq_prepacked_bytes(K, N, g), dtype=torch.uint8), N, g,
                                   zero_points=True)
    assert rec.calls == []


def test_sparse_calls_refuse_wrong_sizes(rec):
    Q = torch.zeros((K // 8, N), dtype=torch.int32)
    with pytest.raises(ValueError):  # s must be [K/g, N]
        wq.wq_prepack_sparse24(Q, torch.zeros((K // g + 1, N), dtype=torch.float16), g)
    with pytest.raises(ValueError):  # caller-given Wp too small
        wq.wq_prepack_sparse24(Q, torch.zeros((K // g, N), dtype=torch.float16), g,
                               Wp=torch.zeros(wq.wq_prepacked_bytes_sparse24(K, N, g) - 16, dtype=torch.uint8))
    with pytest.raises(wq.WqError):  # g does not divide K
        wq.wq_prepack_sparse24(Q, torch.zeros((2, N), dtype=torch.float16), 96)
    with pytest.raises(ValueError):  # the dense buffer is larger, the sparse one must hold its own size
        wq.wq_gemm_w4a16_sparse24(torch.zeros((M, K), dtype=torch.float16),
                                  torch.zeros(wq.wq_prepacked_bytes_sparse24(K, N, g) - 1, dtype=torch.uint8), N, g)
    with pytest.raises(ValueError):
        wq.wq_gemm_w4a16_sparse24(torch.zeros((M, K), dtype=torch.float16),
                                  torch.zeros(wq.wq_prepacked_bytes_sparse24(K, N, g), dtype=torch.uint8), N, g,
                                  Y=torch.zeros((M, N + 8), dtype=torch.float16))
    with pytest.raises(ValueError):
        wq.wq_unpack_sparse24(torch.zeros(16, dtype=torch.uint8), K, N, g)
    assert rec.calls == []


def test_mixed_calls_refuse_wrong_sizes(rec):
    Q = torch.zeros((K // 8, N), dtype=torch.int32)
    s = torch.zeros((K // g, N), dtype=torch.float16)
    W = torch.full((K // 32, 2), 2, dtype=torch.uint8)
    with pytest.raises(ValueError):  # widths must be [K/32, ceil(N/128)]
        wq.wq_prepack_mixed(Q, s, W[:, :1], g)
    with pytest.raises(TypeError):  # widths must be uint8
        wq.wq_prepack_mixed(Q, s, W.int(), g)
    with pytest.raises(ValueError):  # s must be [K/g, N]
        wq.wq_prepack_mixed(Q, s[:1], W, g)
    least = wq.wq_prepacked_bytes_mixed(K, N, g, 0)
    with pytest.raises(ValueError):  # smaller than any mixed buffer of this shape
        wq.wq_gemm_w4a16_mixed(torch.zeros((M, K), dtype=torch.float16), torch.zeros(least - 1, dtype=torch.uint8), N, g)
    with pytest.raises(ValueError):
        wq.wq_gemm_w4a16_mixed(torch.zeros((M, K), dtype=torch.float16), torch.zeros(least, dtype=torch.uint8), N, g,
                               Y=torch.zeros((M + 1, N), dtype=torch.float16))
    with pytest.raises(ValueError):
        wq.wq_unpack_mixed(torch.zeros(16, dtype=torch.uint8), K, N, g)
    assert rec.calls == []
