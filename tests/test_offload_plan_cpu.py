"""CPU tests of the dense offload's segment plan (no GPU needed)."""
import pytest

from paged_kv_chunk_query_b200 import _lib as L
from paged_kv_chunk_query_b200.offload import plan_segments


@pytest.mark.parametrize("n_past,window", [(0, 4), (3, 4), (4, 4), (5, 4), (17, 4), (4032, 512),
                                           (64, 512), (1024, 512)])
def test_plan_covers_the_past_once_in_order(n_past, window):
    plan = plan_segments(n_past, window)
    covered = []
    for mode, a, n in plan:
        assert 0 <= n <= window
        covered += list(range(a, a + n))
    assert covered == list(range(n_past))
    if n_past <= window:
        assert [m for m, _, _ in plan] == [L.SEG_WHOLE]
    else:
        modes = [m for m, _, _ in plan]
        assert modes[0] == L.SEG_FIRST and modes[-1] == L.SEG_LAST
        assert all(m == L.SEG_NEXT for m in modes[1:-1])
        assert all(n == window for _, _, n in plan[:-1])
