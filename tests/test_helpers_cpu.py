"""Host logic of the parity tests: the seeded row sample of the full-size GEMM checks
reaches every 128-row M tile and every 32-row group of the scale atom."""
import numpy as np
import pytest

from helpers import tile_covering_rows


@pytest.mark.parametrize("M", [1, 31, 128, 333, 4096, 8192])
def test_tile_covering_rows(M):
    r = tile_covering_rows(M, 256, seed=0)
    assert r.dtype == np.int64 and np.all(np.diff(r) > 0)
    assert r[0] == 0 and r[-1] == M - 1
    assert set((r // 32).tolist()) == set(range(-(-M // 32)))          # every 32-row group
    assert set((r // 128).tolist()) == set(range(-(-M // 128)))        # every M tile
    assert len(r) >= min(M, 256)
    assert np.array_equal(r, tile_covering_rows(M, 256, seed=0))       # seeded
