"""The decode step keeps an entry of a caller's block list when it is in range, above the
entry before it in the list and above every entry kept so far (an invalid list is skipped
entry by entry and flagged). The device-side check evaluates the same rule with two prefix
scans: an entry is kept when it is in range, in order with its predecessor, and above the
largest such entry before it. This checks on the CPU that the two forms keep the same
entries, for random lists with swaps, repeats and out-of-range values."""
import numpy as np


def kept_serial(lst, nblk):
    kept, prev = [], -1
    for k, v in enumerate(lst):
        if v < 0 or v >= nblk or (k > 0 and lst[k - 1] >= v):
            continue
        if v > prev:
            kept.append(int(v))
            prev = v
    return kept


def kept_scan(lst, nblk):
    lst = np.asarray(lst, dtype=np.int64)
    n = len(lst)
    if n == 0:
        return []
    in_range = (lst >= 0) & (lst < nblk)
    in_order = np.ones(n, bool)
    in_order[1:] = lst[:-1] < lst[1:]
    elig = in_range & in_order
    vals = np.where(elig, lst, -1)
    before = np.concatenate(([-1], np.maximum.accumulate(vals)[:-1]))  # exclusive prefix max
    take = elig & (lst > before)
    return [int(v) for v in lst[take]]


def test_scan_form_keeps_the_same_entries():
    rng = np.random.default_rng(11)
    for trial in range(3000):
        nblk = int(rng.integers(1, 200))
        n = int(rng.integers(0, 120))
        lst = np.sort(rng.integers(-3, nblk + 3, n))
        for _ in range(int(rng.integers(0, 6))):  # swaps
            if n > 1:
                i = int(rng.integers(0, n - 1))
                lst[i], lst[i + 1] = lst[i + 1], lst[i]
        for _ in range(int(rng.integers(0, 4))):  # arbitrary values, repeats
            if n > 0:
                lst[int(rng.integers(0, n))] = int(rng.integers(-5, nblk + 5))
        assert kept_scan(lst, nblk) == kept_serial(lst, nblk), (list(lst), nblk)


def test_valid_list_is_kept_whole():
    lst = [0, 3, 4, 9, 15]
    assert kept_scan(lst, 16) == lst == kept_serial(lst, 16)
