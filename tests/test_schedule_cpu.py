"""Host-side checks of the causal forward's unit-to-CTA assignment (fa_fwd_schedule; no GPU).

A unit is one pair of 128-row query tiles of one (b, h), numbered level-major; its work is the key
blocks its two tiles visit under the causal mask ("FlashAttention-2 GPU work partitioning",
section 4: causal tiles skip the blocks above the diagonal).  The checks: every unit runs exactly
once, the modelled per-CTA work is as even as the plain snake deal's, and far fewer heads are
live at once (the point of the table: their K and V stay in L2).
"""
import numpy as np
import pytest

import exact_attention_158_b200 as fa

SMS = 148


def unit_work(u, BH, N):
    """Key blocks (128 keys each) visited by the two query tiles of unit u, plus one for the unit's
    own start-up."""
    pairs = (N + 255) // 256
    p = pairs - 1 - u // BH
    blocks = 0
    for i in (0, 1):
        q0 = 256 * p + 128 * i
        if q0 < N:
            blocks += (min(q0 + 128, N) - 1) // 128 + 1
    return blocks + 1


def snake_lists(units, G):
    lists = [[] for _ in range(G)]
    for u in range(units):
        r, c = divmod(u, G)
        lists[G - 1 - c if r % 2 else c].append(u)
    return lists


def table_lists(start, unit, G):
    return [list(unit[start[c]:start[c + 1]]) for c in range(G)]


def imbalance(lists, BH, N):
    loads = [sum(unit_work(u, BH, N) for u in lst) for lst in lists]
    return max(loads) / (sum(loads) / len(loads))


def mean_live_heads(lists, BH, N, samples=400):
    """Heads live at once, averaged over the modelled run, a head being live from the start of its
    first unit to the end of its last: the heads whose K and V L2 has to hold for them to be read
    from DRAM once."""
    first, last = {}, {}
    for lst in lists:
        t = 0
        for u in lst:
            w, h = unit_work(u, BH, N), u % BH
            first[h] = min(first.get(h, t), t)
            last[h] = max(last.get(h, t + w), t + w)
            t += w
    end = max(last.values())
    return float(np.mean([sum(1 for h in first if first[h] <= x < last[h])
                          for x in np.linspace(0, end, samples, endpoint=False)]))


# (B, H, N, d): the causal shapes of the forward's benchmark and its sequence-length sweep
TABLE_SHAPES = [(8, 16, 2048, 128), (4, 16, 4096, 128), (32, 16, 512, 128), (16, 16, 1024, 128),
                (2, 16, 8192, 128), (1, 32, 16384, 128),
                # ragged N: the last pair's second tile is short or empty
                (8, 16, 1900, 128), (3, 32, 4000, 128), (6, 16, 3000, 128)]


@pytest.mark.parametrize("shape", TABLE_SHAPES, ids=lambda s: "B{}H{}N{}d{}".format(*s))
def test_table_covers_every_unit_once_and_balances(shape):
    B, H, N, d = shape
    BH = B * H
    units = BH * ((N + 255) // 256)
    sched = fa.fwd_schedule(B, H, N, d, SMS)
    assert sched is not None, "this shape should take a table"
    start, unit = sched
    G = min(units, SMS)
    assert start[0] == 0 and start[G] == units and np.all(np.diff(start[:G + 1]) >= 0)
    assert np.all(start[G:] == units)
    assert np.array_equal(np.sort(unit), np.arange(units)), "a unit is missing or repeated"
    lists = table_lists(start, unit, G)
    snake = snake_lists(units, G)
    assert imbalance(lists, BH, N) <= max(1.06, imbalance(snake, BH, N) + 0.02)
    # the level-major snake keeps most heads live (every head has a unit in each pair level); the
    # table about a group's worth
    assert mean_live_heads(lists, BH, N) <= 0.6 * mean_live_heads(snake, BH, N)


@pytest.mark.parametrize("shape", [(1, 16, 16384, 128), (2, 3, 2048, 128), (1, 1, 300, 64),
                                   (149, 1, 256, 128), (8, 32, 2048, 64), (4, 32, 4096, 64)],
                         ids=lambda s: "B{}H{}N{}d{}".format(*s))
def test_no_table_for_few_heads_or_units(shape):
    # under 32 heads (no two groups of 16), no more units than CTAs, or d = 64: the snake deal
    assert fa.fwd_schedule(*shape, SMS) is None


def test_table_depends_on_the_cta_count():
    a = fa.fwd_schedule(8, 16, 2048, 128, 148)
    b = fa.fwd_schedule(8, 16, 2048, 128, 132)
    assert a is not None and b is not None
    assert np.all(b[0][132:] == 1024) and not np.array_equal(a[0][:133], b[0][:133])


def test_schedule_rejections():
    import ctypes
    lib = fa.load_library()
    f = lib.fa_fwd_schedule
    ip = ctypes.POINTER(ctypes.c_int)
    f.argtypes = [ctypes.c_int] * 5 + [ip, ip, ctypes.c_int, ip]
    f.restype = ctypes.c_int
    start = np.zeros(149, dtype=np.int32)
    unit = np.zeros(1024, dtype=np.int32)
    cnt = ctypes.c_int(0)
    sp, up = start.ctypes.data_as(ip), unit.ctypes.data_as(ip)
    assert f(8, 16, 2048, 128, 148, sp, up, 1023, ctypes.byref(cnt)) == 1  # capacity too small
    assert f(8, 16, 2048, 96, 148, sp, up, 1024, ctypes.byref(cnt)) == 2   # head dim
    assert f(0, 16, 2048, 128, 148, sp, up, 1024, ctypes.byref(cnt)) == 1
    assert f(8, 16, 2048, 128, 0, sp, up, 1024, ctypes.byref(cnt)) == 1
    assert f(8, 16, 2048, 128, 148, None, up, 1024, ctypes.byref(cnt)) == 1
    assert f(8, 16, 2048, 128, 148, sp, up, 1024, ctypes.byref(cnt)) == 0 and cnt.value == 1024
