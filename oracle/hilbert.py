"""Hilbert-curve token order of a (T, Hh, W) latent grid -- oracle.

Source: "Ride the Wave: Precision-Allocated Sparse Attention for Smooth Video
Generation" (DFSAttn), abstract: tokens are reordered along a Hilbert curve so
that spatially close tokens become contiguous and block sparsity becomes finer
grained.  The page names no curve variant.

Reading taken (the pages are silent): the n-dimensional Hilbert curve of
J. Skilling, "Programming the Hilbert curve", AIP Conf. Proc. 707 (2004),
in its "axes -> transpose" direction, on the smallest 2^k cube that holds the
grid (k = ceil(log2(max(T, Hh, W))), at least 1), with axis order (t, y, x),
t being the first (most significant) axis of every bit group.  Grid points
are flattened row-major, n = (t*Hh + y)*W + x.  perm lists the flat token
indices in increasing Hilbert index; cube points outside the grid are simply
absent.  inv is the inverse permutation: inv[perm[i]] = i.

Pinned by (tests/test_oracle.py): bijection on every grid; unit Manhattan
steps and origin start on full 2^k cubes; every aligned 8^m run of indices
fills an aligned 2^m sub-cube; the 2-D restriction reproduces the textbook
quadrant-rotation Hilbert curve on 2^k squares; inverse scatter restores the
token order.
"""

import numpy as np


def bits_for(extent):
    """Smallest k >= 1 with 2**k >= extent."""
    k = 1
    while (1 << k) < extent:
        k += 1
    return k


def axes_to_transpose(coords, k):
    """Skilling's axes -> transposed Hilbert index, vectorised over points.

    coords: int64 array [n_dims, n_points], each entry in [0, 2**k).
    Returns the "transposed" index: n_dims words whose bits, read level by
    level from the top, spell the Hilbert index.
    """
    x = np.array(coords, dtype=np.int64, copy=True)
    n = x.shape[0]
    top = 1 << (k - 1)
    # Inverse undo of the excess work: walk the bit levels from the top.
    q = top
    while q > 1:
        p = q - 1
        for i in range(n):
            hit = (x[i] & q) != 0
            # where the level bit is set: invert the low bits of axis 0
            x[0] = np.where(hit, x[0] ^ p, x[0])
            # otherwise: exchange the low bits of axis 0 and axis i
            t = (x[0] ^ x[i]) & p
            t = np.where(hit, 0, t)
            x[0] ^= t
            x[i] ^= t
        q >>= 1
    # Gray encode.
    for i in range(1, n):
        x[i] ^= x[i - 1]
    t = np.zeros_like(x[0])
    q = top
    while q > 1:
        t = np.where((x[n - 1] & q) != 0, t ^ (q - 1), t)
        q >>= 1
    for i in range(n):
        x[i] ^= t
    return x


def transpose_to_index(xt, k):
    """Interleave the transposed words into one integer Hilbert index.

    At every level b (from k-1 down to 0) the bits of axes 0..n-1 are
    appended in that order, so axis 0 is the most significant of each group.
    """
    n = xt.shape[0]
    h = np.zeros(xt.shape[1], dtype=np.int64)
    for b in range(k - 1, -1, -1):
        for i in range(n):
            h = (h << 1) | ((xt[i] >> b) & 1)
    return h


def hilbert_index(coords, k):
    """Hilbert index of points given as int array [n_dims, n_points]."""
    return transpose_to_index(axes_to_transpose(coords, k), k)


def grid_hilbert_keys(T, Hh, W):
    """Hilbert index of every grid token in row-major (t, y, x) order."""
    k = bits_for(max(T, Hh, W))
    t, y, x = np.meshgrid(np.arange(T), np.arange(Hh), np.arange(W), indexing="ij")
    coords = np.stack([t.ravel(), y.ravel(), x.ravel()]).astype(np.int64)
    return hilbert_index(coords, k), k


def hilbert_perm(T, Hh, W):
    """perm[i] = flat token index at Hilbert rank i; inv[perm[i]] = i.

    Both are int32 arrays of length L = T*Hh*W.  The Hilbert indices of grid
    points are distinct, so the (stable) argsort has no ties.
    """
    keys, _ = grid_hilbert_keys(T, Hh, W)
    perm = np.argsort(keys, kind="stable").astype(np.int32)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size, dtype=np.int32)
    return perm, inv


def permute_rows(x, perm, inverse=False):
    """Reorder the token axis (axis -2) of x.

    forward:  y[..., i, :] = x[..., perm[i], :]   (gather into Hilbert order)
    inverse:  y[..., perm[i], :] = x[..., i, :]   (scatter back to grid order)
    """
    x = np.asarray(x)
    if not inverse:
        return x[..., perm, :]
    y = np.empty_like(x)
    y[..., perm, :] = x
    return y
