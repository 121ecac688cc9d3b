"""Host-side check of the chained launch's task queue (no GPU).

The kernel decodes task q into (layer, row tile, out-channel tile) with the lag
order described in csrc/eql_tc_chain.cu; this test restates that order from its
description (not from the kernel source) and checks the properties the kernel's
deadlock-freedom rests on: every task appears once, and every layer-1 tile of a
row precedes every layer-2 tile of that row.  The lag rule (0.6 of the row tiles,
at least one wave of layer-1 tiles, at most all rows) is checked on the shapes
the tests and the bench use.
"""
import pytest


def lag_of(n_rt, n_dt1, grid):
    lag = (3 * n_rt + 2) // 5
    wave = (grid + n_dt1 - 1) // n_dt1
    return min(max(lag, wave), n_rt)


def queue(n_rt, n1, n2, lag):
    q = [(0, r, j) for r in range(lag) for j in range(n1)]
    for k in range(lag, n_rt):
        q += [(0, k, j) for j in range(n1)] + [(1, k - lag, j) for j in range(n2)]
    q += [(1, r, j) for r in range(n_rt - lag, n_rt) for j in range(n2)]
    return q


SHAPES = [
    # N, C1 (layer-1 out-channels), C2 (layer-2 out-channels), SMs
    (12608, 768, 192, 148), (333, 768, 192, 148), (1, 64, 48, 148), (129, 16, 32, 148),
    (4097, 208, 16, 148), (1000, 384, 64, 148), (777, 128, 64, 148), (12608, 768, 192, 8),
]


@pytest.mark.parametrize("N,C1,C2,sms", SHAPES)
def test_queue_covers_every_tile_once_with_layer1_first(N, C1, C2, sms):
    n_rt = (N + 127) // 128
    n1, n2 = (C1 + 127) // 128, (C2 + 127) // 128
    total = n_rt * (n1 + n2)
    grid = min(total, sms)
    lag = lag_of(n_rt, n1, grid)
    assert 0 <= lag <= n_rt
    q = queue(n_rt, n1, n2, lag)
    assert len(q) == total and len(set(q)) == total
    pos = {t: i for i, t in enumerate(q)}
    for r in range(n_rt):
        last_l1 = max(pos[(0, r, j)] for j in range(n1))
        first_l2 = min(pos[(1, r, j)] for j in range(n2))
        assert last_l1 < first_l2
    # the first wave of CTAs takes layer-1 tiles only (when there are enough)
    first_wave = q[:grid]
    if lag * n1 >= grid:
        assert all(layer == 0 for layer, _, _ in first_wave)
