"""CPU models of two pieces of index logic in the backward kernels, checked
against brute force (the GPU parity tests check the kernels themselves):

- merge_shared_corners: which corners of a level's 4 points share a pixel, and
  who keeps the summed weight.  Partner cells at (dx, dy) with |dx|, |dy| <= 1
  share this point's corner c = i + 2j with the partner's corner c - dx - 2 dy,
  restricted by the column mask (dx) and the row mask (dy).
- reduce_pair3 / pair_lane_point: two points' partial sums reduced over a
  sub-warp of LANES lanes, the first exchange a reduce-scatter; which lane ends
  with which point's totals.

- level_of: a point's level floor(j / K) by one multiply-high with
  m = ceil(2^32 / K), in every kernel that maps points to levels.

These restate the kernels' arithmetic in Python; they are not the oracle."""
import random

import pytest


def merge_model(cells):
    """cells: 4 tuples (x0, y0, vm, w[4]) in lane order.  Returns per lane the
    four scatter weights, None for a corner merged into a lower lane."""
    out = []
    for me in range(4):
        x0, y0, vm, w = cells[me]
        total = list(w)
        merged = 0
        for o in (1, 2, 3):
            p = me ^ o
            px, py, pvm, pw = cells[p]
            dx, dy = px - x0, py - y0
            if abs(dx) > 1 or abs(dy) > 1:
                continue
            sh = dx + 2 * dy
            mx = 15 if dx == 0 else (0xA if dx > 0 else 0x5)
            my = 15 if dy == 0 else (0xC if dy > 0 else 0x3)
            m = mx & my & vm & ((pvm << sh) if sh >= 0 else (pvm >> -sh)) & 15
            if p < me:
                merged |= m
            else:
                for c in range(4):
                    if (m >> c) & 1:
                        total[c] += pw[c - sh]
        out.append([None if (merged >> c) & 1 else total[c] for c in range(4)])
    return out


def test_merge_masks_match_pixel_equality():
    rng = random.Random(7)
    for _ in range(20000):
        W, H = rng.randint(1, 5), rng.randint(1, 5)
        cells = []
        for _ in range(4):
            x0, y0 = rng.randint(-1, W - 1), rng.randint(-1, H - 1)
            vm = 0
            for c in range(4):
                xi, yj = x0 + (c & 1), y0 + (c >> 1)
                if 0 <= xi < W and 0 <= yj < H and rng.random() < 0.9:  # zero weights drop out
                    vm |= 1 << c
            cells.append((x0, y0, vm, [rng.randint(1, 1000) for _ in range(4)]))
        got = {}
        for (x0, y0, vm, _), ws in zip(cells, merge_model(cells)):
            for c in range(4):
                if (vm >> c) & 1 and ws[c] is not None:
                    key = (x0 + (c & 1), y0 + (c >> 1))
                    assert key not in got, "a pixel kept by two lanes"
                    got[key] = ws[c]
        want = {}
        for x0, y0, vm, w in cells:
            for c in range(4):
                if (vm >> c) & 1:
                    key = (x0 + (c & 1), y0 + (c >> 1))
                    want[key] = want.get(key, 0) + w[c]
        assert got == want


def test_merge_never_touches_corners_outside_the_mask():
    # Two points in the same cell, one with a corner masked off (zero weight or
    # outside the map): that corner must keep its own (unmerged) weight path.
    cells = [(3, 3, 0b1111, [1, 2, 3, 4]), (3, 3, 0b0111, [10, 20, 30, 40]),
             (9, 9, 0b1111, [5, 5, 5, 5]), (0, 9, 0b1111, [6, 6, 6, 6])]
    out = merge_model(cells)
    assert out[0] == [11, 22, 33, 4]      # corner 3 of lane 1 is masked: no merge there
    assert out[1] == [None, None, None, 40]


def pair_reduce_model(lanes, ta, tb):
    """ta, tb: per lane one partial value of points A and B.  Returns per lane
    the value after reduce_pair3's exchanges (one of the three sums)."""
    half = lanes // 2
    v = []
    for lane in range(lanes):
        upper = bool(lane & half)
        partner = lane ^ half
        send_from_partner = ta[partner] if (partner & half) else tb[partner]
        mine = tb[lane] if upper else ta[lane]
        v.append(mine + send_from_partner)
    sh = half // 2
    while sh > 0:
        v = [v[l] + v[l ^ sh] for l in range(lanes)]
        sh //= 2
    return v


def pair_lane_point(lanes, lane):
    if lanes == 1:
        return 0
    half = lanes // 2
    return 2 * (lane - half) + 1 if lane & half else 2 * lane


@pytest.mark.parametrize("lanes", [2, 4, 8, 16, 32])
def test_pair_reduction_places_each_point_total_once(lanes):
    rng = random.Random(lanes)
    ta = [rng.randint(-50, 50) for _ in range(lanes)]
    tb = [rng.randint(-50, 50) for _ in range(lanes)]
    v = pair_reduce_model(lanes, ta, tb)
    half = lanes // 2
    assert all(x == sum(ta) for x in v[:half])
    assert all(x == sum(tb) for x in v[half:])
    # A batch of LANES points reduced in pairs (2u, 2u + 1): lane u keeps pair u's
    # A, lane half + u its B, and that is exactly pair_lane_point's mapping.
    kept = {}
    for u in range(half):
        for lane in range(lanes):
            if (lane & (half - 1)) == u:
                kept[lane] = 2 * u + (1 if lane & half else 0)
    assert kept == {lane: pair_lane_point(lanes, lane) for lane in range(lanes)}
    assert sorted(kept.values()) == list(range(lanes))


def test_level_of_is_exact_integer_division():
    """floor(j m / 2^32) with m = floor((2^32 - 1) / K) + 1 equals j // K for every
    j < 2^16 and every K the op accepts (1 <= K <= 64; m = 0 stands for K = 1),
    exhaustively."""
    import numpy as np

    j = np.arange(1 << 16, dtype=np.uint64)
    for K in range(1, 65):
        m = 0 if K == 1 else (0xFFFFFFFF // K) + 1
        assert m < (1 << 32)
        got = j if m == 0 else (j * np.uint64(m)) >> np.uint64(32)
        assert np.array_equal(got, j // np.uint64(K)), K
