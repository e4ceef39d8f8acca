"""Host-side checks of the seeded input and row-sampling helpers."""
import pytest

import bd_inputs


@pytest.mark.parametrize("B,H,L,b", [(4, 32, 2048, 32), (1, 32, 8192, 256),
                                     (1, 2, 64, 8), (2, 3, 100, 25)])
def test_fwd_sample_rows_covers_edge_blocks_of_sampled_heads(B, H, L, b):
    rows = bd_inputs.fwd_sample_rows(B, H, L, b, 200, heads=8, per_block=16)
    assert rows == sorted(set(rows))
    assert all(0 <= r < B * H * 2 * L for r in rows)
    got = set(rows)
    starts = (0, L - b, L, 2 * L - b)

    def covers(h):
        base = h * 2 * L
        return all(base + s0 in got and base + s0 + b - 1 in got for s0 in starts)

    # the first and last head always, and min(8, B * H) heads in all
    assert covers(0) and covers(B * H - 1)
    assert sum(covers(h) for h in range(B * H)) >= min(8, B * H)
    # small blocks are taken whole
    if b <= 16:
        assert all(h * 2 * L + s0 + i in got for h in (0, B * H - 1)
                   for s0 in starts for i in range(b))


def test_fwd_sample_rows_is_seeded():
    a = bd_inputs.fwd_sample_rows(4, 32, 2048, 32, 100, seed=3)
    assert a == bd_inputs.fwd_sample_rows(4, 32, 2048, 32, 100, seed=3)
    assert a != bd_inputs.fwd_sample_rows(4, 32, 2048, 32, 100, seed=4)
