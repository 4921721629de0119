"""Each pass of the GPU radix select picks the digit of the kr-th largest remaining key from a
256-bin histogram h: the largest d with (sum of h above d) + h[d] >= kr, else 0, and the rank
left within that digit. The device finds it with one warp: lane l owns bins 8l .. 8l+7, a
suffix sum over lanes finds the lane that holds the digit, and that lane scans its 8 bins.
This checks on the CPU that the lane form returns what the bin-by-bin scan returns."""
import numpy as np


def digit_serial(h, kr):
    cum, d = 0, 255
    while d > 0:
        if cum + h[d] >= kr:
            break
        cum += h[d]
        d -= 1
    return d, kr - cum


def digit_lanes(h, kr):
    v = np.asarray(h).reshape(32, 8)
    s = v.sum(axis=1)
    incl = np.cumsum(s[::-1])[::-1]          # sum over lanes >= l
    hit = np.flatnonzero(incl >= kr)
    if hit.size == 0:
        return 0, kr - (incl[0] - v[0, 0])
    L = int(hit.max())
    cum = int(incl[L] - s[L])
    d = 8 * L + 7
    for i in range(7, 0, -1):
        if cum + v[L, i] >= kr:
            break
        cum += v[L, i]
        d -= 1
    return d, kr - cum


def test_lane_form_matches_bin_scan():
    rng = np.random.default_rng(5)
    for trial in range(4000):
        kind = trial % 4
        if kind == 0:
            h = rng.integers(0, 20, 256)
        elif kind == 1:  # sparse: most bins empty
            h = np.where(rng.random(256) < 0.05, rng.integers(1, 500, 256), 0)
        elif kind == 2:  # everything in one bin
            h = np.zeros(256, np.int64)
            h[int(rng.integers(0, 256))] = int(rng.integers(1, 5000))
        else:
            h = rng.integers(0, 3, 256)
        total = int(h.sum())
        for kr in {1, max(1, total // 2), max(1, total), total + 1, int(rng.integers(1, total + 2))}:
            assert digit_lanes(h, kr) == digit_serial(h, kr), (trial, kr)
