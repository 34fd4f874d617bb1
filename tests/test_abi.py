"""CPU tests of the C ABI: the library loads, exports every function include/wq.h declares,
agrees with the oracle on buffer sizes, and rejects bad arguments on the host (these calls
return before touching a device, so they run without a GPU)."""
import ctypes
import os
import re

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"^WQ_API\s+[\w\s\*]+?\b(wq_\w+)\s*\(", text, flags=re.M)
    return names


@pytest.fixture(scope="module")
def wq():
    import bit_weight_quantized_prepack_b200 as wq
    return wq


def test_header_declares_the_entry_points():
    names = set(_declared_functions())
    for must in ("wq_prepack", "wq_gemm_w4a16", "wq_gemm_w4a8", "wq_prepacked_bytes", "wq_unpack",
                 "wq_get_device_status", "wq_workspace_reserve", "wq_prepack_zp", "wq_gemm_w4a16_zp",
                 "wq_prepack_act_order", "wq_gemm_w4a16_act_order", "wq_quantize_act", "wq_gemm_w4a8_fp16act",
                 "wq_prepack_sparse24", "wq_gemm_w4a16_sparse24", "wq_prepack_mixed", "wq_gemm_w4a16_mixed",
                 "wq_gemm_w4a16_noalloc"):
        assert must in names


def test_library_exports_every_declared_symbol(wq):
    raw = ctypes.CDLL(wq.LIB_PATH)
    missing = [n for n in _declared_functions() if not hasattr(raw, n)]
    assert not missing, missing


def test_version_and_status_strings(wq):
    assert wq.wq_version() >= 10000
    seen = set()
    for st in range(11):
        s = wq.status_string(st)
        assert s.startswith("WQ_") and s not in seen
        seen.add(s)
    assert wq.status_string(1234).startswith("WQ_ERR")


@pytest.mark.parametrize("K,N,g", [(128, 8, 128), (4096, 4096, 128), (4096, 4096, 4096), (11008, 4096, 128),
                                   (28672, 8192, 28672), (256, 200, 32), (512, 1000, 64), (1280, 520, 640)])
def test_prepacked_bytes_agree_with_oracle(wq, K, N, g):
    assert wq.wq_prepacked_bytes(K, N, g) == oracle.prepacked_bytes_w4a16(K, N, g)
    assert wq.wq_prepacked_bytes_w4a8(K, N) == oracle.prepacked_bytes_w4a8(K, N)


@pytest.mark.parametrize("K,N,g", [(128, 8, 128), (384, 296, 128), (384, 296, 32), (4096, 4096, 4096),
                                   (256, 200, 64), (1280, 520, 640)])
def test_sparse_prepacked_bytes_agree_with_oracle(wq, K, N, g):
    assert wq.wq_prepacked_bytes_sparse24(K, N, g) == oracle.prepacked_bytes_w4a16_sparse24(K, N, g)


@pytest.mark.parametrize("K,N,g,frac4", [(128, 8, 128, 0.5), (256, 136, 128, 0.4), (384, 296, 32, 0.2),
                                         (4096, 4096, 4096, 0.3), (1280, 520, 640, 1.0), (256, 200, 64, 0.0)])
def test_mixed_prepacked_bytes_agree_with_oracle(wq, K, N, g, frac4):
    import synth
    w = synth.w4a16_mixed_inputs(K, N, g, 1, seed=K, frac4=frac4)["widths"]
    assert wq.wq_prepacked_bytes_mixed(K, N, g, int((w == 4).sum())) == oracle.prepacked_bytes_mixed(K, N, g, w)
    assert wq.wq_prepacked_bytes_mixed(K, N, g, -1) == 0
    assert wq.wq_prepacked_bytes_mixed(K, N, g, w.size + 1) == 0


@pytest.mark.parametrize("K,N,g", [(100, 128, 100), (128, 12, 128), (0, 128, 128), (256, 128, 48),
                                   (256, 128, 96), (384, 128, 256), (256, -8, 128)])
def test_unsupported_shapes_have_no_size(wq, K, N, g):
    assert wq.wq_prepacked_bytes(K, N, g) == 0


def test_host_side_argument_checks(wq):
    L = wq.lib
    P = ctypes.c_void_p
    good = P(0x10000)  # never dereferenced: every call below fails a host-side check first
    # shapes
    assert L.wq_gemm_w4a16(good, good, good, 1, 128, 100, 128, None) == wq.WQ_ERR_UNSUPPORTED_SHAPE
    assert L.wq_gemm_w4a16(good, good, good, 1, 12, 128, 128, None) == wq.WQ_ERR_UNSUPPORTED_SHAPE
    assert L.wq_gemm_w4a16(good, good, good, 1, 128, 0, 128, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_gemm_w4a16(good, good, good, -1, 128, 128, 128, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_gemm_w4a16(good, good, good, (1 << 24) + 1, 128, 128, 128, None) == wq.WQ_ERR_UNSUPPORTED_SHAPE
    assert L.wq_gemm_w4a8(good, good, good, good, good, None, 1, 128, 262144, None) == wq.WQ_ERR_UNSUPPORTED_SHAPE
    # W4A8 sums a * 16(q - 8) in int32, up to 16384 per term (a = -128): K = 131072 would wrap
    assert L.wq_gemm_w4a8(good, good, good, good, good, None, 1, 128, 131072, None) == wq.WQ_ERR_UNSUPPORTED_SHAPE
    assert L.wq_gemm_w4a8(good, good, good, good, good, None, 0, 128, 130944, None) == wq.WQ_OK
    assert 130944 * 16384 < 2 ** 31 <= 131072 * 16384
    # group size
    assert L.wq_gemm_w4a16(good, good, good, 1, 128, 256, 48, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_prepack(good, good, 256, 128, 96, good, None) == wq.WQ_ERR_INVALID_ARG
    # null pointers
    assert L.wq_gemm_w4a16(good, None, good, 1, 128, 128, 128, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_gemm_w4a16(None, good, good, 1, 128, 128, 128, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_gemm_w4a8(good, None, good, good, good, None, 1, 128, 128, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_prepack(None, good, 128, 128, 128, good, None) == wq.WQ_ERR_INVALID_ARG
    # alignment
    odd = P(0x10008)
    assert L.wq_gemm_w4a16(odd, good, good, 1, 128, 128, 128, None) == wq.WQ_ERR_MISALIGNED
    assert L.wq_gemm_w4a16(good, odd, good, 1, 128, 128, 128, None) == wq.WQ_ERR_MISALIGNED
    assert L.wq_gemm_w4a16(good, good, odd, 1, 128, 128, 128, None) == wq.WQ_ERR_MISALIGNED
    assert L.wq_gemm_w4a8(good, P(0x10002), good, good, good, None, 1, 128, 128, None) == wq.WQ_ERR_MISALIGNED
    assert L.wq_prepack(odd, good, 128, 128, 128, good, None) == wq.WQ_ERR_MISALIGNED
    # 2:4 sparse: the sparse warp MMA serves M <= 16; the same shape, group and pointer checks
    assert L.wq_gemm_w4a16_sparse24(good, good, good, 17, 128, 128, 128, None) == wq.WQ_ERR_UNSUPPORTED_SHAPE
    assert L.wq_gemm_w4a16_sparse24(good, good, good, 1, 128, 100, 128, None) == wq.WQ_ERR_UNSUPPORTED_SHAPE
    assert L.wq_gemm_w4a16_sparse24(good, good, good, 1, 128, 256, 48, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_gemm_w4a16_sparse24(good, odd, good, 1, 128, 128, 128, None) == wq.WQ_ERR_MISALIGNED
    assert L.wq_gemm_w4a16_sparse24(None, good, None, 0, 128, 128, 128, None) == wq.WQ_OK
    assert L.wq_prepack_sparse24(good, good, 256, 128, 96, good, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_prepack_sparse24(odd, good, 128, 128, 128, good, None) == wq.WQ_ERR_MISALIGNED
    assert L.wq_prepack_sparse24(good, None, 128, 128, 128, good, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_unpack_sparse24(good, 128, 128, 128, good, odd, None) == wq.WQ_ERR_MISALIGNED
    assert wq.wq_prepacked_bytes_sparse24(256, 128, 96) == 0
    # mixed 2/4-bit: M <= 16, the caller's buffer size, the usual checks
    least = wq.wq_prepacked_bytes_mixed(128, 128, 128, 0)
    assert L.wq_gemm_w4a16_mixed(good, good, least, good, 17, 128, 128, 128, None) == wq.WQ_ERR_UNSUPPORTED_SHAPE
    assert L.wq_gemm_w4a16_mixed(good, good, least - 16, good, 1, 128, 128, 128, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_gemm_w4a16_mixed(good, odd, least, good, 1, 128, 128, 128, None) == wq.WQ_ERR_MISALIGNED
    assert L.wq_gemm_w4a16_mixed(None, good, least, None, 0, 128, 128, 128, None) == wq.WQ_OK
    assert L.wq_prepack_mixed(good, good, None, 128, 128, 128, good, least, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_prepack_mixed(good, good, good, 256, 128, 96, good, least, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_unpack_mixed(good, 128, 128, 128, good, good, None, None) == wq.WQ_ERR_INVALID_ARG
    # an empty batch is a no-op that needs no activation or output pointer
    assert L.wq_gemm_w4a16(None, good, None, 0, 128, 128, 128, None) == wq.WQ_OK
    assert L.wq_gemm_w4a8(None, None, good, None, None, None, 0, 128, 128, None) == wq.WQ_OK


def test_binding_raises_on_error_status(wq):
    with pytest.raises(wq.WqError) as ei:
        wq._check(wq.WQ_ERR_MISALIGNED, "x")
    assert ei.value.status == wq.WQ_ERR_MISALIGNED and "MISALIGNED" in str(ei.value)
