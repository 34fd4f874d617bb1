"""CPU tests of the launch planner through wq_plan_for (host arithmetic, no GPU): for a B200's
148 SMs and 227 KB of opt-in shared memory, every supported shape gets a plan whose tiles
cover M, whose ring and barriers fit shared memory, and whose stream-K split gives every CTA
work. Calls of at most 16 rows (W4A16 and W4A8) get the register-operand plan: one tile of 1, 2,
4, 8 or 16 rows, 576 threads, and the residue sums in shared memory after the ring."""
import itertools

import pytest

SMS, SMEM = 148, 232448


def _rf(kind, M):
    return M <= 16


def _red(p):  # bytes of the register-operand kernel's residue sums
    return 4 * p["tile_m"] * 128 * 4


@pytest.fixture(scope="module")
def wq():
    return pytest.importorskip("bit_weight_quantized_prepack_b200")


MS = [1, 2, 5, 15, 16, 17, 31, 32, 33, 48, 63, 64, 65, 100, 127, 128, 129, 200, 255, 256, 257, 511, 1024, 4096]
SHAPES = [(128, 8), (1024, 136), (4096, 4096), (4096, 22016), (11008, 4096), (8192, 57344), (131072, 8)]


@pytest.mark.parametrize("K,N", SHAPES)
@pytest.mark.parametrize("kind,g", [(0, 32), (0, 64), (0, 128), (0, 256), (0, None), (1, None)])
def test_plan_invariants(wq, K, N, kind, g):
    if g is None:
        g = K
    if kind == 0 and K % g:
        pytest.skip("group size must divide K")
    for M in MS:
        p = wq.wq_plan_for(kind, M, N, K, g, SMS, SMEM)
        tm = p["tile_m"]
        if _rf(kind, M):
            assert tm == (1 if M == 1 else 2 if M == 2 else 4 if M <= 4 else 8 if M <= 8 else 16), (M, p)
        else:
            assert tm % 16 == 0 and 16 <= tm <= 256, (M, p)
        assert p["m_tiles"] == -(-M // tm), (M, p)                     # the tiles cover M ...
        assert (p["m_tiles"] - 1) * tm < M, (M, p)                      # ... with no empty tile
        assert p["n_tiles"] == -(-N // 128) and p["k_blocks"] == K // 128
        assert p["units"] == p["n_tiles"] * p["m_tiles"] * p["k_blocks"]
        assert p["grid"] == min(SMS, p["units"])                        # every CTA has a unit
        assert 2 <= p["stages"] <= 32
        act = tm * (256 if kind == 0 else 128)
        blob = 8192 + (256 * (128 // min(g, 128)) if kind == 0 and g < K else 0)
        red = _red(p) if _rf(kind, M) else 0
        assert p["smem_bytes"] == p["stages"] * (act + blob) + 1024 + red  # ring + alignment slack
        assert p["smem_bytes"] + 2048 <= SMEM                           # room for the static barriers
        assert p["threads"] == (576 if _rf(kind, M) else 704)


@pytest.mark.parametrize("K,N", SHAPES)
@pytest.mark.parametrize("g", [32, 64, 128, 256, None])
def test_sparse_plan_invariants(wq, K, N, g):
    # 2:4 sparse W4A16 (kind 5): the register-operand kernel only; activation slots of at
    # least 8 rows (one 1024-byte swizzle atom per 64-column piece); blobs of 6144 bytes of
    # codes and metadata plus the scale rows
    g = K if g is None else g
    if K % g:
        pytest.skip("group size must divide K")
    for M in [m for m in MS if m <= 16]:
        p = wq.wq_plan_for(5, M, N, K, g, SMS, SMEM)
        dense = wq.wq_plan_for(0, M, N, K, g, SMS, SMEM)
        tm = p["tile_m"]
        assert tm == dense["tile_m"] and p["grid"] == dense["grid"] and p["units"] == dense["units"]
        assert p["threads"] == 576 and p["m_tiles"] == 1
        act = max(tm, 8) * 256
        blob = 6144 + (256 * (128 // min(g, 128)) if g < K else 0)
        assert p["smem_bytes"] == p["stages"] * (act + blob) + 1024 + _red(p)
        assert p["smem_bytes"] + 2048 <= SMEM
        more = (p["stages"] + 1) * (act + blob) + 1024 + _red(p)
        assert p["stages"] == 32 or more + 2048 > SMEM
    for M in (17, 32, 100):
        with pytest.raises(wq.WqError) as e:
            wq.wq_plan_for(5, M, N, K, g, SMS, SMEM)
        assert e.value.status == wq.WQ_ERR_UNSUPPORTED_SHAPE


@pytest.mark.parametrize("K,N", SHAPES)
@pytest.mark.parametrize("g", [32, 128, None])
def test_mixed_plan_is_the_dense_register_operand_plan(wq, K, N, g):
    # mixed 2/4-bit (kind 6): the slots hold the largest blob (every block 4-bit) and shared memory
    # also holds the CTA's table entries (at most ceil(units / grid) + 1, widened to 16-byte
    # boundaries); otherwise the dense register-operand plan. M > 16 is refused
    g = K if g is None else g
    if K % g:
        pytest.skip("group size must divide K")
    for M in [m for m in MS if m <= 16]:
        p = wq.wq_plan_for(6, M, N, K, g, SMS, SMEM)
        d = wq.wq_plan_for(0, M, N, K, g, SMS, SMEM)
        for key in ("grid", "tile_m", "m_tiles", "n_tiles", "k_blocks", "threads", "units"):
            assert p[key] == d[key], key
        tbl = ((-(-p["units"] // SMS) + 7) * 4 + 15) // 16 * 16
        act = p["tile_m"] * 256
        blob = 8192 + (256 * (128 // min(g, 128)) if g < K else 0)
        assert p["smem_bytes"] == p["stages"] * (act + blob) + 1024 + _red(p) + tbl
        assert p["smem_bytes"] + 2048 <= SMEM and p["stages"] <= d["stages"]
    with pytest.raises(wq.WqError):
        wq.wq_plan_for(6, 17, N, K, g, SMS, SMEM)


def test_plan_uses_the_largest_ring_that_fits(wq):
    for M, kind in itertools.product([1, 16, 32, 64, 256], [0, 1]):
        p = wq.wq_plan_for(kind, M, 4096, 4096, 128 if kind == 0 else 4096, SMS, SMEM)
        act = p["tile_m"] * (256 if kind == 0 else 128)
        blob = 8192 + (256 if kind == 0 else 0)
        more = (p["stages"] + 1) * (act + blob) + 1024 + (_red(p) if _rf(kind, M) else 0)
        assert p["stages"] == 32 or more + 2048 > SMEM, p


def test_plan_scales_with_the_device(wq):
    small = wq.wq_plan_for(0, 1, 4096, 4096, 128, 20, SMEM)
    assert small["grid"] == 20
    tight = wq.wq_plan_for(0, 64, 4096, 4096, 128, SMS, 100 * 1024)
    assert tight["stages"] >= 2 and tight["smem_bytes"] + 2048 <= 100 * 1024
    with pytest.raises(wq.WqError):  # 256-row tiles need two 72 KB stages
        wq.wq_plan_for(0, 256, 4096, 4096, 128, SMS, 100 * 1024)


def test_plan_rejects_bad_arguments(wq):
    bad = [(2, 1, 4096, 4096, 128, SMS, SMEM), (0, 0, 4096, 4096, 128, SMS, SMEM),
           (0, 1, 4096, 4000, 128, SMS, SMEM), (0, 1, 4096, 4096, 100, SMS, SMEM),
           (0, 1, 4096, 4096, 128, 0, SMEM), (0, 1, 4096, 4096, 128, SMS, 0)]
    for args in bad:
        with pytest.raises(wq.WqError):
            wq.wq_plan_for(*args)
    with pytest.raises(wq.WqError):
        wq.wq_plan_for(0, 1, 4096, 4096, 128, SMS, 16 * 1024)  # not even two stages fit
