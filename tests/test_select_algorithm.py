"""The radix top-P scheme of the one-launch selection (csrc/topp_select.cuh), restated
in numpy, against the oracle's selection (oracle/spava_oracle.py select_passing).

The kernel resolves the P-th largest ordered key in digits that start right below
the leading bits every key shares (from the block's min and max), 11 bits at a time,
and then takes keys above it plus the lowest-index keys equal to it.  These checks
pin that scheme itself -- the digit boundaries, the descending bin search, the
count of tied keys to take -- on random scores, heavy ties, all-equal blocks, mixed
signs and narrow ranges, at P = 1 and P = n among others.  The GPU tests check the
CUDA code of the same scheme against the oracle bit for bit.
"""

import numpy as np
import pytest

from oracle import spava_oracle as orc


def ordered_keys(scores):
    b = np.asarray(scores, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = np.where(b == 0x80000000, 0, b)  # -0 -> +0
    return np.where(b & 0x80000000, (~b) & 0xFFFFFFFF, b | 0x80000000).astype(np.uint64)


def digit_select(scores, passing, threads=256):
    """Indices of the top `passing` scores, ascending, by the kernel's scheme."""
    keys = ordered_keys(scores)
    kmin, kmax = int(keys.min()), int(keys.max())
    cp = 32 if kmin == kmax else 32 - (kmin ^ kmax).bit_length()  # shared leading bits
    pmask = 0xFFFFFFFF if cp == 32 else (~(0xFFFFFFFF >> cp)) & 0xFFFFFFFF
    prefix, k, shift = kmax & pmask, passing, 32 - cp
    while shift > 0:
        wd = min(11, shift)
        shift -= wd
        nb = 1 << wd
        match = (keys & pmask) == prefix
        hist = np.bincount(((keys[match] >> shift) & (nb - 1)).astype(np.int64), minlength=nb)
        bpt = nb // threads if nb >= threads else 1
        found, excl = False, 0
        for t in range(threads):  # thread t owns the bins top .. top - bpt + 1
            top = nb - 1 - t * bpt
            own = [int(hist[top - q]) for q in range(bpt) if top - q >= 0]
            if not found and excl < k <= excl + sum(own):
                acc = excl
                for q, cb in enumerate(own):
                    if acc + cb >= k:
                        prefix, k, found = prefix | ((top - q) << shift), k - acc, True
                        break
                    acc += cb
            excl += sum(own)
        assert found
        pmask |= (nb - 1) << shift
    T, take_eq = prefix, k
    eq_rank = np.cumsum(keys == T) - 1
    win = (keys > T) | ((keys == T) & (eq_rank < take_eq))
    assert int(win.sum()) == passing
    return np.nonzero(win)[0]


def _cases():
    rng = np.random.default_rng(123)
    out = []
    for trial in range(60):
        n = int(rng.integers(1, 12000))
        p = [1, n, int(rng.integers(1, n + 1))][trial % 3]
        kind = trial % 6
        if kind == 0:
            s = rng.standard_normal(n)
        elif kind == 1:
            s = rng.integers(0, 5, n).astype(np.float64)  # heavy ties
        elif kind == 2:
            s = np.full(n, 1.5)  # every key equal
        elif kind == 3:
            s = rng.standard_normal(n) * 1e-3 + 3.0  # narrow range: many shared leading bits
        elif kind == 4:
            s = np.where(rng.random(n) < 0.5, -0.0, 0.0)  # signed zeros only
        else:
            s = rng.standard_normal(n) * 1e30  # wide range, both signs
        out.append((s.astype(np.float32), p))
    return out


@pytest.mark.parametrize("scores,passing", _cases())
def test_digit_select_equals_oracle(scores, passing):
    n = len(scores)
    off = np.array([0, n, n + 1])  # one candidate block, then a last host
    want = orc.select_passing(scores[None, :], off, 0, passing)[0, 0]
    np.testing.assert_array_equal(digit_select(scores, passing), want)


def test_digit_select_with_a_1024_thread_group():
    rng = np.random.default_rng(7)
    s = rng.standard_normal(16384).astype(np.float32)
    off = np.array([0, 16384, 16385])
    want = orc.select_passing(s[None, :], off, 0, 1024)[0, 0]
    np.testing.assert_array_equal(digit_select(s, 1024, threads=1024), want)
