"""Interval (skip-list) encoding of the kept key blocks -- oracle (test
infrastructure only).

Source: CalibAtt (calibrated sparse attention), appendix Fig. S9 (number of
intervals per skip-list row at N = 75,600; 95% of rows need at most 50, out
of a theoretical maximum of 295), Fig. S10 (each row stores interval pairs;
(b) per-layer trimming to the widest row; (c) merging outlier rows lowers the
layer's width) and Table S3 (skip-list memory for Wan-T2V 14B at 720p by
"Merge %": 100 = no merge, 99, 95; merging at 95% lowers the sparsity from
62.50% to 62.41%, i.e. merging adds computed blocks).

Definitions (readings: the pages give no formulas):

  runs of a row: the maximal runs of consecutive kept key-block indices,
      each an interval pair (start, end) with end exclusive, in ascending
      order.  Consecutive runs are separated by a gap of
      start_{r+1} - end_r >= 1 skipped blocks.  A row of NB blocks has at
      most ceil(NB / 2) runs.
  merge to width W (W >= 1): while the row has more than W intervals, fill
      the smallest gap between neighbouring intervals (the leftmost of equal
      gaps), joining the two into one.  Filling a gap adds its blocks to the
      kept set, so a merged row keeps a superset of its blocks; smallest gaps
      first adds the fewest blocks.
  width for a merge percentage q (Table S3's "Merge %" as a fraction,
      0 < q <= 1): the smallest W >= 1 such that at least ceil(q * rows)
      rows (IEEE float64 product) have at most W runs; q = 1 gives the
      widest row (Fig. S10 (b)), q = 0.95 merges the 5% widest rows
      (Fig. S10 (c)).
  padding: pairs beyond a row's count are (-1, -1).

Pinned by (tests/test_oracle.py): the theoretical maximum (alternating rows
reach ceil(NB / 2); NB = 590 full blocks of N = 75,600 gives the pages' 295);
brute force over every subset of tiny rows (runs are maximal, disjoint,
ascending, and decode back to the subset); brute force over every choice of
gaps to fill (fewest added blocks, then leftmost gaps: the lexicographically
smallest choice); hand-worked rows in tests/golden/interval_cases.json;
closed forms of the width for two-valued run counts.
"""

import math

import numpy as np


def max_intervals(NB):
    """Most runs a row of NB key blocks can have (every other block kept)."""
    return (NB + 1) // 2


def runs_of(kept):
    """Maximal runs of an ascending list of distinct block indices:
    list of (start, end) with end exclusive."""
    out = []
    for j in kept:
        j = int(j)
        if out and out[-1][1] == j:
            out[-1] = (out[-1][0], j + 1)
        else:
            out.append((j, j + 1))
    return out


def merge_runs(runs, W):
    """Fill the smallest gap (leftmost on ties) until at most W intervals."""
    assert W >= 1
    iv = list(runs)
    while len(iv) > W:
        gaps = [iv[r + 1][0] - iv[r][1] for r in range(len(iv) - 1)]
        r = gaps.index(min(gaps))   # list.index: the leftmost smallest gap
        iv[r:r + 2] = [(iv[r][0], iv[r + 1][1])]
    return iv


def decode_row(pairs):
    """Ascending block indices covered by a row's interval pairs."""
    out = []
    for s, e in pairs:
        out.extend(range(int(s), int(e)))
    return out


def kept_to_intervals(kept_idx, kept_cnt, W):
    """Encode every row: (intervals int32 [..., W, 2] padded with -1,
    n_int int32 [...], n_runs int32 [...]), where n_runs counts the runs
    before merging and n_int = min(n_runs, W)."""
    kept_idx = np.asarray(kept_idx)
    kept_cnt = np.asarray(kept_cnt)
    lead = kept_cnt.shape
    iv = np.full(lead + (W, 2), -1, dtype=np.int32)
    n_int = np.zeros(lead, dtype=np.int32)
    n_runs = np.zeros(lead, dtype=np.int32)
    for pos in np.ndindex(*lead):
        r = runs_of(kept_idx[pos][: int(kept_cnt[pos])])
        m = merge_runs(r, W)
        n_runs[pos] = len(r)
        n_int[pos] = len(m)
        for t, (s, e) in enumerate(m):
            iv[pos + (t,)] = (s, e)
    return iv, n_int, n_runs


def intervals_to_kept(intervals, n_int, NB):
    """Decode every row: (mask uint8 [..., NB], kept_idx int32 [..., NB]
    padded with -1, kept_cnt int32 [...])."""
    intervals = np.asarray(intervals)
    n_int = np.asarray(n_int)
    lead = n_int.shape
    mask = np.zeros(lead + (NB,), dtype=np.uint8)
    idx = np.full(lead + (NB,), -1, dtype=np.int32)
    cnt = np.zeros(lead, dtype=np.int32)
    for pos in np.ndindex(*lead):
        k = decode_row(intervals[pos][: int(n_int[pos])])
        if k:
            mask[pos + (k,)] = 1
        idx[pos][: len(k)] = k
        cnt[pos] = len(k)
    return mask, idx, cnt


def run_histogram(n_runs, NB):
    """Number of rows with r runs, r = 0 .. max_intervals(NB)."""
    return np.bincount(np.asarray(n_runs).reshape(-1), minlength=max_intervals(NB) + 1).astype(np.int64)


def width_for_merge(hist, q):
    """Smallest W >= 1 such that at least ceil(q * rows) rows have <= W runs."""
    hist = [int(x) for x in hist]
    rows = sum(hist)
    need = math.ceil(float(q) * float(rows))
    covered = hist[0]
    for W in range(1, len(hist)):
        covered += hist[W]
        if covered >= need:
            return W
    return max(1, len(hist) - 1)


def list_bytes(rows, NB):
    """Bytes of the padded index-list form (int32 [rows, NB] + int32 counts)."""
    return rows * NB * 4 + rows * 4


def interval_bytes(rows, W):
    """Bytes of the interval form (int32 pairs [rows, W, 2] + int32 counts)."""
    return rows * W * 8 + rows * 4
