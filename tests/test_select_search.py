"""The threshold search of the register selection kernel, restated on the
host and checked against the oracle's top-p selection (oracle/topp.py,
oracle/reuse.py).

The kernel (select_reg_kernel in csrc/select.cu) finds the largest key tau
with S(tau) = sum_{key >= tau} u >= T bit by bit, and takes two shortcuts
whose exactness rests on an argument rather than on the arithmetic being the
same as the oracle's:
  * a step is first decided on coarse masses a = floor(P * 2^21) = u >> 19:
    with A = sum_{key >= c} a, S(c) lies in [A 2^19, (A + NB) 2^19), so
    A 2^19 >= T or (A + NB) 2^19 <= T settles it; only in between is the
    exact sum needed;
  * after every odd bit from bit 15 down, the search stops when the bracket
    [tau, tau + 2^b) holds a single key value with mass: that key is the
    threshold.
This test restates those steps with numpy integers (one row at a time, the
warp's lanes as an array), checks every coarse decision against the exact
one and the early threshold against the full 29-step search, and compares
the kept set with the oracle on rows with ties, NaN, P > 1, masses below
2^-40, near-equal keys and candidate restrictions.  The GPU kernel itself is
compared with the oracle in tests/test_gpu_parity.py and test_gpu_reuse.py.
"""

import numpy as np
import pytest

from oracle import reuse as oreu
from oracle import topp as otop

SHIFT = 19
MIN_MASS_KEY = 0x2B800000  # P = 2^-40, the smallest key with u > 0
TOP = 0x20000000           # bits 30 and 29 of any threshold with T > 0


def _keys(P):
    """float32 bits of clamp(P, 0, 1); NaN and P <= 0 give 0."""
    P = np.asarray(P, np.float32)
    ok = P > 0
    k = np.minimum(np.where(ok, P, np.float32(0)), np.float32(1)).astype(np.float32).view(np.uint32)
    return np.where(ok, k, 0).astype(np.uint32)


def _mass(key):
    """floor(P * 2^40) from the exponent e and the 24-bit significand m."""
    e = (key >> 23).astype(np.int64)
    m = ((key & 0x7FFFFF) | 0x800000).astype(np.int64)
    out = np.zeros(key.shape, np.int64)
    up = (e > 0) & (e >= 110)
    out[up] = m[up] << (e[up] - 110)
    dn = (e > 0) & (e < 110) & (110 - e < 24)
    out[dn] = m[dn] >> (110 - e[dn])
    return out


def _coarse(key):
    """floor(P * 2^21) from the same bits: m * 2^(e - 129)."""
    e = (key >> 23).astype(np.int64)
    m = ((key & 0x7FFFFF) | 0x800000).astype(np.int64)
    sh = 129 - e
    return np.where((e == 0) | (sh >= 24), 0, m >> np.clip(sh, 0, 63))


def _full_search(key, u, T):
    tau = TOP
    for b in range(28, -1, -1):
        c = tau | (1 << b)
        if int(u[key >= c].sum()) >= T:
            tau = c
    return tau


def kernel_select(P, p, cand=None):
    """The register kernel's steps on one row; returns the 0/1 mask."""
    NB = len(P)
    key = _keys(P)
    if cand is not None:
        key = np.where(np.asarray(cand).astype(bool), key, 0).astype(np.uint32)
    if p == np.float32(1.0):
        return np.ones(NB, np.uint8) if cand is None else np.asarray(cand).astype(bool).astype(np.uint8)
    u = _mass(key)
    total = int(u.sum())
    T = int(np.ceil(np.float64(p) * np.float64(total)))
    if T == 0:  # keep the first block of the order among the eligible ones
        elig = np.ones(NB, bool) if cand is None else np.asarray(cand).astype(bool)
        out = np.zeros(NB, np.uint8)
        if elig.any():
            out[int(np.argmax(np.where(elig, key.astype(np.int64), -1)))] = 1
        return out
    a = _coarse(key)
    assert np.array_equal(a, u >> SHIFT)
    assert int(a.sum()) < 2 ** 31  # one 32-bit warp reduction
    tau = TOP
    for b in range(28, -1, -1):
        c = tau | (1 << b)
        A = int(a[key >= c].sum())
        exact = int(u[key >= c].sum()) >= T
        if (A << SHIFT) >= T:
            ge = True
        elif ((A + NB) << SHIFT) <= T:
            ge = False
        else:
            ge = exact
        assert ge == exact
        if ge:
            tau = c
        if (b & 1) and b <= 15:
            lo, hi = max(tau, MIN_MASS_KEY), tau + (1 << b)
            inb = key[(key >= lo) & (key < hi)]
            if inb.size and inb.min() == inb.max():
                tau = int(inb.min())
                break
    assert tau == _full_search(key, u, T)
    need = T - int(u[key > tau].sum())
    assert need > 0
    sel = key > tau
    carry = 0
    for j in np.flatnonzero(key == tau):  # ascending index order
        if carry < need:
            sel[j] = True
        carry += int(u[j])
    return sel.astype(np.uint8)


def _oracle(P, p, cand=None):
    kept, k = otop.select_row(P, p) if cand is None else oreu.select_row_restricted(P, p, cand)
    out = np.zeros(len(P), np.uint8)
    out[np.asarray(kept[:k], dtype=np.int64)] = 1
    return out


def _rows(NB, rng):
    x = rng.standard_normal(NB) * rng.uniform(0.5, 6)
    soft = np.exp(x - x.max())
    yield (soft / soft.sum()).astype(np.float32)                                    # softmax row
    yield rng.choice(np.array([0.1, 0.05, 0.05, 0.2, 0.0, 1e-3], np.float32), NB)  # ties
    yield np.full(NB, np.float32(1.0 / NB))                                         # all equal
    junk = (rng.uniform(0, 1, NB) ** 30).astype(np.float32)                         # tiny masses, junk
    junk[rng.integers(0, NB, max(1, NB // 10))] = np.nan
    junk[rng.integers(0, NB, max(1, NB // 10))] = 2.0
    junk[rng.integers(0, NB, max(1, NB // 10))] = -1.0
    yield junk
    base = np.float32(rng.uniform(1e-4, 1e-2))                                      # keys 1-7 ulps apart
    yield (base.view(np.uint32) + rng.integers(0, 8, NB).astype(np.uint32)).view(np.float32)


@pytest.mark.parametrize("NB", [1, 2, 7, 33, 255, 591, 1024])
def test_search_matches_oracle(NB):
    rng = np.random.default_rng(NB)
    for P in _rows(NB, rng):
        for p in (0.5, 0.886, 0.97, 0.999, 1e-6, 1.0):
            assert np.array_equal(kernel_select(P, np.float32(p)), _oracle(P, p)), (NB, p)
        cand = (rng.uniform(size=NB) < 0.3).astype(np.uint8)
        for p in (0.5, 0.9, 1.0):
            assert np.array_equal(kernel_select(P, np.float32(p), cand), _oracle(P, p, cand)), (NB, p)


def test_early_stop_and_coarse_steps_are_taken():
    """On a 591-block softmax row the shortcuts do fire (the test above would
    pass vacuously if they never did): the search stops early and most steps
    are settled on coarse masses."""
    rng = np.random.default_rng(1)
    x = rng.standard_normal(591) * 3
    P = np.exp(x - x.max())
    P = (P / P.sum()).astype(np.float32)
    key = _keys(P)
    u = _mass(key)
    T = int(np.ceil(np.float64(np.float32(0.886)) * np.float64(int(u.sum()))))
    a = _coarse(key)
    tau, steps, coarse = TOP, 0, 0
    for b in range(28, -1, -1):
        c = tau | (1 << b)
        steps += 1
        A = int(a[key >= c].sum())
        coarse += (A << SHIFT) >= T or ((A + 591) << SHIFT) <= T
        if int(u[key >= c].sum()) >= T:
            tau = c
        if (b & 1) and b <= 15:
            inb = key[(key >= max(tau, MIN_MASS_KEY)) & (key < tau + (1 << b))]
            if inb.size and inb.min() == inb.max():
                break
    assert steps < 29 and coarse >= steps - 2
