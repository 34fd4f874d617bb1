"""CPU test: the small-tile kernel's barrier protocol cannot deadlock for the launch plans it
uses (every layer shape of the configurations, every ring size the planner can pick, short
and ragged stream-K ranges). The model lives in schedule_model.py."""
import pytest

from schedule_model import simulate

SHAPES = [(4096, 4096), (4096, 12288), (4096, 22016), (11008, 4096), (8192, 10240), (8192, 8192),
          (8192, 57344), (28672, 8192), (128, 128), (384, 1000), (1024, 136)]


def _plan(K, N):
    kbs = K // 128
    units = -(-N // 128) * kbs
    return units, min(148, units), kbs


@pytest.mark.parametrize("K,N", SHAPES)
@pytest.mark.parametrize("slots", [5, 9, 13, 16, 17, 18])
def test_no_deadlock(K, N, slots):
    units, grid, kbs = _plan(K, N)
    if K * N > 8192 * 10240 and slots not in (16, 17):
        pytest.skip("large shapes: the ring sizes the planner picks for them")
    stuck = simulate(units, grid, kbs, min(4, slots // 2), slots)
    assert not stuck, stuck[:5]


def test_model_catches_slot_indexed_barrier_hazard():
    # the earlier protocol indexed chunk barriers by ring slot; the same model with that
    # indexing deadlocks on the 8192 x 10240 layer with a 17-slot ring (seen on the GPU as an
    # expired wait on 4 tiles)
    import schedule_model as sm
    orig = sm.chunks

    def slot_indexed(beg, end, kbs, chunk, slots):
        uses = [0] * slots
        for seg, pos, c, it0, ch in orig(beg, end, kbs, chunk, slots):
            if pos is None:
                yield seg, pos, c, it0, ch
                continue
            # barrier number = slot + 33 * (uses of that slot), so that mod 33 is the slot and
            # the phase parity is the slot's use count
            yield seg, pos, c, it0, pos + sm.NCB * uses[pos]
            uses[pos] += 1
    sm.chunks = slot_indexed
    try:
        units, grid, kbs = _plan(8192, 10240)
        assert simulate(units, grid, kbs, 4, 17)
    finally:
        sm.chunks = orig
