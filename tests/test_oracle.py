"""Pins of the CPU oracle to things other than itself (CPU only).

Each test ties one oracle function to a closed form, a textbook or library
routine, a brute-force enumeration or an invariant, so that a dropped term,
a wrong sign or index or a transposed operand fails at least one of them.
The last group plants such mistakes in copies of oracle functions and checks
that the pins catch them.
"""

import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import attention as oatt
from oracle import correction as ocor
from oracle import hilbert as ohil
from oracle import intervals as oint
from oracle import refresh as oref
from oracle import reuse as oreu
from oracle import scoring as osco
from oracle import tail as otail
from oracle import topp as otop

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------- Hilbert

def _cube_points(k, n=3):
    side = 1 << k
    grids = np.meshgrid(*[np.arange(side)] * n, indexing="ij")
    return np.stack([g.ravel() for g in grids]).astype(np.int64)


@pytest.mark.parametrize("k", [1, 2, 3])
def test_hilbert_full_cube_is_a_continuous_bijection(k):
    pts = _cube_points(k)
    d = ohil.hilbert_index(pts, k)
    assert sorted(d.tolist()) == list(range(8 ** k))
    walk = pts[:, np.argsort(d)]
    steps = np.abs(np.diff(walk, axis=1)).sum(axis=0)
    assert np.all(steps == 1), "consecutive curve points must be unit neighbours"
    assert np.all(walk[:, 0] == 0), "curve starts at the origin"


@pytest.mark.parametrize("k", [2, 3])
def test_hilbert_aligned_runs_fill_aligned_subcubes(k):
    pts = _cube_points(k)
    d = ohil.hilbert_index(pts, k)
    walk = pts[:, np.argsort(d)]
    for m in range(1, k):
        run = 8 ** m
        side = 1 << m
        for start in range(0, 8 ** k, run):
            seg = walk[:, start:start + run]
            lo = seg.min(axis=1)
            assert np.all(lo % side == 0)
            assert np.all(seg.max(axis=1) - lo == side - 1)
            assert len({tuple(c) for c in seg.T}) == run


def _textbook_d2xy(n, d):
    """Classic quadrant-rotation Hilbert curve on an n x n square (n = 2^k)."""
    x = y = 0
    s = 1
    t = d
    while s < n:
        rx = 1 & (t // 2)
        ry = 1 & (t ^ rx)
        if ry == 0:
            if rx == 1:
                x, y = s - 1 - x, s - 1 - y
            x, y = y, x
        x += s * rx
        y += s * ry
        t //= 4
        s *= 2
    return x, y


@pytest.mark.parametrize("k", [1, 2, 3, 4])
def test_hilbert_2d_matches_textbook_curve(k):
    n = 1 << k
    pts = _cube_points(k, n=2)
    d = ohil.hilbert_index(pts, k)
    table = {_textbook_d2xy(n, i): i for i in range(n * n)}
    for j in range(n * n):
        assert table[(int(pts[0, j]), int(pts[1, j]))] == d[j]


@pytest.mark.parametrize("grid", [(2, 32, 32), (3, 5, 7), (1, 1, 1), (21, 30, 52)])
def test_hilbert_perm_bijection_and_inverse(grid):
    perm, inv = ohil.hilbert_perm(*grid)
    L = int(np.prod(grid))
    assert perm.dtype == np.int32 and perm.size == L
    assert np.array_equal(np.sort(perm), np.arange(L))
    assert np.array_equal(perm[inv], np.arange(L))
    x = np.random.default_rng(0).standard_normal((1, 2, L, 3))
    y = ohil.permute_rows(x, perm)
    assert np.array_equal(ohil.permute_rows(y, perm, inverse=True), x)


def test_hilbert_grid_is_restriction_of_cube_order():
    T, Hh, W = 3, 5, 6
    perm, _ = ohil.hilbert_perm(T, Hh, W)
    k = ohil.bits_for(max(T, Hh, W))
    cube = _cube_points(k)
    order = cube[:, np.argsort(ohil.hilbert_index(cube, k))]
    inside = (order[0] < T) & (order[1] < Hh) & (order[2] < W)
    flat = (order[0] * Hh + order[1]) * W + order[2]
    assert np.array_equal(flat[inside], perm)


# ------------------------------------------------------------------ scoring

def test_pool_golden_ramps():
    cases = json.load(open(os.path.join(GOLDEN, "pool_cases.json")))["cases"]
    for c in cases:
        L, blk = c["L"], c["blk"]
        x = np.broadcast_to(np.arange(L, dtype=np.float64)[None, None, :, None], (1, 1, L, 2))
        got = osco.pool_blocks(x, blk)[0, 0, :, 0]
        assert np.allclose(got, c["means"], rtol=0, atol=1e-6), c


def test_pool_constant_and_linearity():
    rng = np.random.default_rng(1)
    x = np.full((1, 2, 70, 8), 3.25)
    assert np.all(osco.pool_blocks(x, 16) == np.float32(3.25))
    a = rng.standard_normal((1, 2, 70, 8))
    b = rng.standard_normal((1, 2, 70, 8))
    lhs = osco.pool_blocks(2 * a - b, 16)
    rhs = 2 * osco.pool_blocks(a, 16).astype(np.float64) - osco.pool_blocks(b, 16)
    assert np.allclose(lhs, rhs, atol=1e-5)


def test_block_probs_rows_sum_to_one_and_match_scipy():
    from scipy.special import softmax
    rng = np.random.default_rng(2)
    q = rng.standard_normal((1, 3, 300, 16)).astype(np.float32)
    k = rng.standard_normal((1, 3, 300, 16)).astype(np.float32)
    qbar, kbar, P = osco.score_blocks(q, k, 64)
    assert P.shape == (1, 3, 5, 5) and P.dtype == np.float32
    assert np.allclose(P.sum(-1), 1, atol=1e-6)
    # logits formed independently: loop over pairs, explicit 1/sqrt(D)
    S = np.zeros((1, 3, 5, 5))
    for h in range(3):
        for i in range(5):
            for j in range(5):
                S[0, h, i, j] = float(np.dot(qbar[0, h, i].astype(np.float64),
                                             kbar[0, h, j].astype(np.float64))) / 4.0
    assert np.allclose(P, softmax(S, axis=-1), rtol=1e-6, atol=1e-9)
    # rows are not symmetric in general: the query side is the row
    assert not np.allclose(P, np.swapaxes(P, -1, -2))


def test_block_probs_uniform_for_constant_keys():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((1, 1, 256, 8))
    k = np.ones((1, 1, 256, 8)) * 0.7
    _, _, P = osco.score_blocks(q, k, 32)
    assert np.allclose(P, 1.0 / 8, atol=1e-7)


def test_block_probs_prefers_aligned_key():
    # one key block aligned with the query mean must get the largest share
    q = np.zeros((1, 1, 4, 2)); q[..., 0] = 1.0
    k = np.zeros((1, 1, 4, 2)); k[0, 0, 2:, 0] = 5.0; k[0, 0, :2, 0] = -5.0
    _, _, P = osco.score_blocks(q, k, 2)
    expect = np.exp([-5 / math.sqrt(2), 5 / math.sqrt(2)])
    expect /= expect.sum()
    assert np.allclose(P[0, 0, 0], expect, rtol=1e-6)


# -------------------------------------------------------------------- top-p

def test_topp_golden_rows():
    cases = json.load(open(os.path.join(GOLDEN, "topp_cases.json")))["cases"]
    for c in cases:
        P = np.array([np.nan if v == "nan" else v for v in c["P"]], dtype=np.float32)
        kept, k = otop.select_row(P, c["p"])
        assert kept.tolist() == c["kept"], c["name"]
        assert k == len(c["kept"])


def _brute_force_row(P, p):
    """Smallest subset reaching T; among equal sizes the ordered top-k."""
    P = otop.clamp_probs(P)
    nb = P.size
    u = [int(math.floor(float(x) * 2 ** 40)) for x in P]
    U = sum(u)
    T = math.ceil(float(np.float64(np.float32(p)) * np.float64(U)))
    if np.float32(p) == 1:
        return list(range(nb))
    for size in range(1, nb + 1):
        best = None
        for sub in itertools.combinations(range(nb), size):
            if sum(u[j] for j in sub) >= T:
                key = sorted(sub, key=lambda j: (-float(P[j]), j))
                if best is None or [(-float(P[j]), j) for j in key] < [(-float(P[j]), j) for j in best]:
                    best = key
        if best is not None:
            return sorted(best)
    raise AssertionError("unreachable")


@pytest.mark.parametrize("seed", range(12))
def test_topp_matches_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    nb = int(rng.integers(1, 11))
    z = rng.standard_normal(nb) * rng.uniform(0.2, 3)
    if seed % 3 == 0:
        z = np.round(z)  # ties
    P = (np.exp(z) / np.exp(z).sum()).astype(np.float32)
    for p in (0.3, 0.5, 0.9, 0.97, 1.0):
        kept, _ = otop.select_row(P, p)
        assert kept.tolist() == _brute_force_row(P, p), (P, p)


def test_topp_mass_and_minimality_on_random_rows():
    from block_sparse_attention_logits_b200.synthetic import random_probs
    P = random_probs(1, 2, 37, seed=5, temperature=2.0)
    p = np.array([0.9, 0.5], dtype=np.float32)
    mask, idx, cnt = otop.select_topp_mask(P, p)
    for h in range(2):
        for i in range(37):
            row = otop.clamp_probs(P[0, h, i])
            u = np.floor(row.astype(np.float64) * 2 ** 40)
            U = u.sum()
            T = math.ceil(float(p[h]) * U)
            kept = idx[0, h, i, :cnt[0, h, i]]
            assert np.array_equal(np.nonzero(mask[0, h, i])[0], kept)
            assert u[kept].sum() >= T
            smallest = kept[np.lexsort((-kept, row[kept]))[0]]  # least P, highest index
            assert u[kept].sum() - u[smallest] < T
            # every dropped block is ordered after every kept block
            dropped = np.setdiff1d(np.arange(37), kept)
            if dropped.size:
                worst_kept = min((row[j], -j) for j in kept)
                best_dropped = max((row[j], -j) for j in dropped)
                assert best_dropped < worst_kept


def test_topp_p_one_and_equal_rows():
    P = np.full((1, 1, 9, 9), 1 / 9, dtype=np.float32)
    mask, idx, cnt = otop.select_topp_mask(P, [1.0])
    assert np.all(mask == 1) and np.all(cnt == 9)
    P = np.full((1, 1, 8, 8), 0.125, dtype=np.float32)
    mask, idx, cnt = otop.select_topp_mask(P, [0.5])
    assert np.all(cnt == 4) and np.all(idx[..., :4] == np.arange(4))


def test_topp_fast_equals_loop():
    from block_sparse_attention_logits_b200.synthetic import random_probs
    for ties in (False, True):
        P = random_probs(2, 3, 29, seed=9, temperature=1.5, ties=ties)
        p = np.array([0.9, 0.35, 1.0], dtype=np.float32)
        a = otop.select_topp_mask(P, p)
        b = otop.select_topp_mask_fast(P, p)
        for x, y in zip(a, b):
            assert np.array_equal(x, y)


def test_topp_rejects_bad_p():
    P = np.full((1, 1, 2, 2), 0.5, dtype=np.float32)
    for bad in (0.0, -0.1, 1.5, float("nan")):
        with pytest.raises(ValueError):
            otop.select_topp_mask(P, [bad])


# ---------------------------------------------------------------- attention

def _naive_attention(q, k, v):
    L, D = q.shape
    O = np.zeros((L, D))
    lse = np.zeros(L)
    for r in range(L):
        s = [sum(q[r, d] * k[c, d] for d in range(D)) / math.sqrt(D) for c in range(L)]
        m = max(s)
        z = sum(math.exp(x - m) for x in s)
        lse[r] = m + math.log(z)
        for c in range(L):
            w = math.exp(s[c] - lse[r])
            for d in range(D):
                O[r, d] += w * v[c, d]
    return O, lse


def test_keep_all_equals_naive_triple_loop():
    rng = np.random.default_rng(7)
    L, D, blk = 11, 4, 4
    q, k, v = (rng.standard_normal((1, 1, L, D)) for _ in range(3))
    nb = 3
    idx = np.tile(np.arange(nb, dtype=np.int32), (1, 1, nb, 1))
    cnt = np.full((1, 1, nb), nb, dtype=np.int32)
    O, lse = oatt.masked_attention(q, k, v, idx, cnt, blk)
    On, lsen = _naive_attention(q[0, 0], k[0, 0], v[0, 0])
    assert np.allclose(O[0, 0], On, atol=1e-12)
    assert np.allclose(lse[0, 0], lsen, atol=1e-12)


def test_keep_all_equals_torch_sdpa_float64():
    rng = np.random.default_rng(8)
    B, H, L, D, blk = 1, 2, 200, 16, 64
    q, k, v = (rng.standard_normal((B, H, L, D)) for _ in range(3))
    nb = 4
    idx = np.tile(np.arange(nb, dtype=np.int32), (B, H, nb, 1))
    cnt = np.full((B, H, nb), nb, dtype=np.int32)
    O, lse = oatt.masked_attention(q, k, v, idx, cnt, blk)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v)).numpy()
    assert np.allclose(O, ref, atol=1e-12)
    Od, lsed = oatt.dense_attention(q, k, v)
    assert np.allclose(Od, ref, atol=1e-12) and np.allclose(lsed, lse, atol=1e-12)
    # LSE against torch.logsumexp of independently formed logits
    s = torch.from_numpy(q) @ torch.from_numpy(k).transpose(-1, -2) / math.sqrt(D)
    assert np.allclose(lse, torch.logsumexp(s, dim=-1).numpy(), atol=1e-12)


def test_masked_attention_weights_sum_to_one_and_respect_mask():
    rng = np.random.default_rng(9)
    B, H, L, D, blk = 1, 1, 150, 8, 32
    q, k, v = (rng.standard_normal((B, H, L, D)) for _ in range(3))
    kept = np.array([0, 4])  # 4 is the partial last block (22 tokens)
    o, lse = oatt.masked_attention_block(q, k, v, kept, blk, 0, 0, 1)
    cols = np.r_[0:32, 128:150]
    s = q[0, 0, 32:64] @ k[0, 0, cols].T / math.sqrt(D)
    w = np.exp(s - lse[:, None])
    assert np.allclose(w.sum(1), 1, atol=1e-12)
    assert np.allclose(o, w @ v[0, 0, cols], atol=1e-12)
    # changing a value in a dropped block changes nothing
    v2 = v.copy(); v2[0, 0, 40] += 100.0
    o2, _ = oatt.masked_attention_block(q, k, v2, kept, blk, 0, 0, 1)
    assert np.array_equal(o, o2)


def test_single_block_constant_keys_closed_form():
    rng = np.random.default_rng(10)
    B, H, L, D, blk = 1, 1, 100, 8, 32
    q = rng.standard_normal((B, H, L, D))
    k = np.tile(rng.standard_normal(D), (B, H, L, 1))
    v = rng.standard_normal((B, H, L, D))
    for j, n in ((1, 32), (3, 4)):  # a full block and the partial last block
        o, lse = oatt.masked_attention_block(q, k, v, [j], blk, 0, 0, 0)
        expect = q[0, 0, :32] @ k[0, 0, 0] / math.sqrt(D) + math.log(n)
        assert np.allclose(lse, expect, atol=1e-12)
        assert np.allclose(o, v[0, 0, j * 32:j * 32 + n].mean(0), atol=1e-12)


def test_empty_kept_set():
    z = np.zeros((1, 1, 4, 2))
    o, lse = oatt.masked_attention_block(z, z, z, [], 4, 0, 0, 0)
    assert np.all(o == 0) and np.all(np.isneginf(lse))


# --------------------------------------------------------------- correction

def test_bf16_round_matches_torch_cast():
    rng = np.random.default_rng(11)
    x = np.concatenate([rng.standard_normal(5000) * 10 ** rng.uniform(-30, 30, 5000),
                        [0.0, -0.0, np.inf, -np.inf, 3.3895314e38, 1e-40]]).astype(np.float32)
    ours = ocor.bf16_round(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    assert np.array_equal(ours.view(np.uint32), ref.view(np.uint32))


def test_correction_identities():
    rng = np.random.default_rng(12)
    to_bf16 = lambda a: torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16).float().numpy()
    od = to_bf16(rng.standard_normal((1, 3, 40, 8)))
    osp = to_bf16(od + 0.05 * rng.standard_normal(od.shape))
    R = ocor.refresh_refinement(od, osp)
    assert np.allclose(ocor.apply_correction(osp, R, np.zeros(3)), osp)
    full = ocor.apply_correction(osp, R, np.ones(3))
    # one bf16 rounding of R: |err| <= half an ulp of |R| (2^-9 relative)
    assert np.all(np.abs(full - od) <= np.abs(od - osp) * 2.0 ** -8 + 1e-30)
    half = ocor.apply_correction(osp, R, np.array([0.0, 0.5, 1.0]))
    assert np.allclose(half[:, 1], osp[:, 1] + 0.5 * R[:, 1])
    assert np.allclose(half[:, 2], full[:, 2]) and np.allclose(half[:, 0], osp[:, 0])


# ------------------------------------------------------------ fused refresh

def _refresh_case(seed, B=1, H=2, L=150, D=8, blk=32):
    rng = np.random.default_rng(seed)
    q, k, v = (rng.standard_normal((B, H, L, D)) for _ in range(3))
    NB = (L + blk - 1) // blk
    idx = np.zeros((B, H, NB, NB), np.int32)
    cnt = np.zeros((B, H, NB), np.int32)
    for b in range(B):
        for h in range(H):
            for i in range(NB):
                kept = np.sort(rng.choice(NB, rng.integers(1, NB + 1), replace=False))
                idx[b, h, i, :len(kept)] = kept
                cnt[b, h, i] = len(kept)
    return q, k, v, idx, cnt, NB


def test_refresh_keep_all_gives_unit_mass_and_zero_refinement():
    q, k, v, _, _, NB = _refresh_case(21)
    fi, fc = oref.full_lists(1, 2, NB)
    Od, Ld, Os, Ls, R, mass = oref.fused_refresh(q, k, v, fi, fc, 32)
    assert np.array_equal(Od, Os) and np.array_equal(Ld, Ls)
    assert np.all(R == 0) and np.all(mass == 1.0)


def test_refresh_mass_closed_form_for_constant_keys():
    rng = np.random.default_rng(22)
    B, H, L, D, blk = 1, 1, 150, 8, 32   # 5 blocks, the last one holds 22 tokens
    q = rng.standard_normal((B, H, L, D))
    k = np.tile(rng.standard_normal(D), (B, H, L, 1))
    v = rng.standard_normal((B, H, L, D))
    NB = 5
    idx = np.zeros((B, H, NB, NB), np.int32)
    cnt = np.zeros((B, H, NB), np.int32)
    idx[0, 0, :, :2] = [0, 4]
    cnt[:] = 2
    *_, mass = oref.fused_refresh(q, k, v, idx, cnt, blk)
    assert np.allclose(mass, (32 + 22) / 150, atol=1e-12)


def test_refresh_dense_is_mass_weighted_mixture_of_kept_and_complement():
    q, k, v, idx, cnt, NB = _refresh_case(23)
    Od, Ld, Os, Ls, R, mass = oref.fused_refresh(q, k, v, idx, cnt, 32)
    ci, cc = oref.complement_lists(idx, cnt, NB)
    Oc, Lc = oatt.masked_attention(q, k, v, ci, cc, 32)
    full = cc == 0  # rows that keep every block have an empty complement
    fullr = np.repeat(full, 32, axis=2)[:, :, :150]
    Oc = np.where(fullr[..., None], 0.0, Oc)
    mix = mass[..., None] * Os + (1 - mass[..., None]) * Oc
    assert np.allclose(Od, mix, atol=1e-12)
    assert np.allclose(Ld, np.logaddexp(Ls, np.where(fullr, -np.inf, Lc)), atol=1e-12)
    assert np.all((mass > 0) & (mass <= 1 + 1e-15))


def test_refresh_refinement_matches_torch_rounding():
    q, k, v, idx, cnt, _ = _refresh_case(24)
    Od, _, Os, _, R, _ = oref.fused_refresh(q, k, v, idx, cnt, 32)
    t = lambda a: torch.from_numpy(np.asarray(a, np.float64)).to(torch.bfloat16).float()
    ref = (t(Od) - t(Os)).to(torch.bfloat16).float().numpy()
    assert np.array_equal(R.view(np.uint32), ref.view(np.uint32))


def test_refresh_empty_kept_row():
    q, k, v, idx, cnt, _ = _refresh_case(25)
    cnt[0, 1, 2] = 0
    _, _, Os, Ls, _, mass = oref.fused_refresh(q, k, v, idx, cnt, 32)
    rows = slice(64, 96)
    assert np.all(Os[0, 1, rows] == 0) and np.all(np.isneginf(Ls[0, 1, rows])) and np.all(mass[0, 1, rows] == 0)


def test_planted_mistake_inverted_mass_is_caught(monkeypatch):
    monkeypatch.setattr(oref, "kept_mass", lambda ls, ld: np.exp(np.asarray(ld) - np.asarray(ls)))
    with pytest.raises(AssertionError):
        test_refresh_mass_closed_form_for_constant_keys()


# ------------------------------------------------------------- mask reuse

def test_drift_closed_forms():
    rng = np.random.default_rng(31)
    qb, kb = rng.standard_normal((2, 3, 7, 8)), rng.standard_normal((2, 3, 7, 8))
    assert np.all(oreu.block_drift(qb, kb, qb, kb) == 0)
    # uniform scaling of the query means by c: drift |c - 1|
    for c in (0.5, 1.1, 3.0):
        assert np.allclose(oreu.block_drift(qb, kb, c * qb, kb), abs(c - 1), atol=1e-12)
    # one perturbed entry: its size over the reference norm; the larger side wins
    kq = kb.copy()
    kq[1, 2, 3, 4] += 0.25
    d = oreu.block_drift(qb, kb, qb, kq)
    assert np.isclose(d[1, 2], 0.25 / np.sqrt((kb[1, 2] ** 2).sum()), atol=1e-12)
    assert np.all(np.delete(d.ravel(), 1 * 3 + 2) == 0)
    both = oreu.block_drift(qb, kb, 1.2 * qb, kq)
    assert np.isclose(both[1, 2], max(0.2, d[1, 2]))
    z = np.zeros_like(qb)
    assert np.all(oreu.block_drift(z, z, z, z) == 0) and np.all(np.isinf(oreu.block_drift(z, kb, qb, kb)))


def test_restricted_scoring_all_candidates_and_scipy():
    import scipy.special
    rng = np.random.default_rng(32)
    B, H, L, D, blk = 1, 2, 300, 16, 32
    q, k = rng.standard_normal((B, H, L, D)), rng.standard_normal((B, H, L, D))
    qb, kb, P = osco.score_blocks(q, k, blk)
    NB = qb.shape[2]
    allc = np.ones((B, H, NB, NB), np.uint8)
    assert np.allclose(oreu.restricted_probs(qb, kb, allc), P, rtol=1e-6, atol=0)
    cand = rng.random((B, H, NB, NB)) < 0.4
    cand[0, 1, 3] = False  # a row without candidates
    Pr = oreu.restricted_probs(qb, kb, cand)
    assert np.all(Pr[~cand] == 0) and np.all(Pr[0, 1, 3] == 0)
    s = osco.block_logits(qb, kb)
    for (b, h, i) in [(0, 0, 0), (0, 1, 5), (0, 0, NB - 1)]:
        sel = cand[b, h, i]
        if sel.any():
            ref = scipy.special.softmax(s[b, h, i, sel])
            assert np.allclose(Pr[b, h, i, sel], ref, rtol=1e-6)
            assert abs(Pr[b, h, i].astype(np.float64).sum() - 1) < 1e-6


def test_restricted_selection_all_candidates_equals_unrestricted():
    rng = np.random.default_rng(33)
    P = rng.dirichlet(np.ones(12), size=(1, 2, 12)).astype(np.float32)
    pv = np.array([0.7, 0.95], np.float32)
    allc = np.ones(P.shape, np.uint8)
    a = otop.select_topp_mask_fast(P, pv)
    b = oreu.select_topp_mask_restricted(P, pv, allc)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_restricted_selection_golden_row_and_edges():
    P = np.array([0.4, 0.3, 0.2, 0.1], np.float32)
    cand = np.array([0, 1, 0, 1], np.uint8)
    # target 0.7 of the candidates' mass 0.4: block 1 alone (0.3) reaches it
    kept, k = oreu.select_row_restricted(P, 0.7, cand)
    assert k == 1 and list(kept) == [1]
    kept, k = oreu.select_row_restricted(P, 0.9, cand)
    assert k == 2 and list(kept) == [1, 3]
    kept, k = oreu.select_row_restricted(P, 1.0, cand)
    assert list(kept) == [1, 3]
    kept, k = oreu.select_row_restricted(P, 0.5, np.zeros(4, np.uint8))
    assert k == 0 and kept.size == 0


@pytest.mark.parametrize("seed", [34, 35, 36])
def test_restricted_selection_matches_brute_force(seed):
    rng = np.random.default_rng(seed)
    nb = 9
    P = rng.dirichlet(np.ones(nb)).astype(np.float32)
    cand = np.flatnonzero(rng.random(nb) < 0.6)
    if cand.size == 0:
        cand = np.array([0])
    cm = np.zeros(nb, np.uint8)
    cm[cand] = 1
    p = np.float32(rng.uniform(0.3, 0.95))
    kept, k = oreu.select_row_restricted(P, p, cm)
    u = otop.fixed_point_mass(otop.clamp_probs(P))
    T = int(np.ceil(np.float64(p) * np.float64(int(u[cand].sum()))))
    assert set(kept) <= set(cand)
    assert int(u[kept].sum()) >= T
    for r in range(1, k):   # no smaller candidate subset reaches T
        for sub in itertools.combinations(cand, r):
            assert int(u[list(sub)].sum()) < T
    # the kept set is the ordered top-k of the candidates
    order = sorted(cand, key=lambda j: (-float(P[j]), j))
    assert sorted(order[:k]) == list(kept)


def test_planted_mistake_restricted_target_is_caught(monkeypatch):
    def full_row_target(P_row, p, cand_row):
        cand = np.flatnonzero(np.asarray(cand_row).astype(bool))
        Pc = otop.clamp_probs(P_row)
        u = otop.fixed_point_mass(Pc)
        T = int(np.ceil(np.float64(np.float32(p)) * np.float64(int(u.sum()))))   # wrong total
        order = sorted(cand, key=lambda j: (-float(Pc[j]), j))
        csum = np.cumsum(u[order])
        k = int(np.argmax(csum >= T)) + 1 if csum[-1] >= T else len(order)
        return np.sort(np.array(order[:k], np.int32)), k
    monkeypatch.setattr(oreu, "select_row_restricted", full_row_target)
    with pytest.raises(AssertionError):
        test_restricted_selection_golden_row_and_edges()


# ----------------------------------------------------- interval skip lists

def _as_lists(pairs):
    return [[int(a), int(b)] for a, b in pairs]


def test_intervals_golden_rows_and_widths():
    cases = json.load(open(os.path.join(GOLDEN, "interval_cases.json")))
    for row in cases["rows"]:
        runs = oint.runs_of(row["kept"])
        assert _as_lists(runs) == row["runs"], row["name"]
        for W, want in row["merged"].items():
            assert _as_lists(oint.merge_runs(runs, int(W))) == want, (row["name"], W)
    for w in cases["widths"]:
        hist = oint.run_histogram(w["n_runs"], 16)
        assert oint.width_for_merge(hist, w["q"]) == w["W"], w["why"]


def test_intervals_theoretical_maximum():
    # every other block kept reaches ceil(NB / 2) runs; the 590 full blocks
    # of N = 75,600 at 128 tokens give the pages' 295 (Fig. S9)
    for NB in range(1, 40):
        assert len(oint.runs_of(range(0, NB, 2))) == oint.max_intervals(NB) == math.ceil(NB / 2)
    assert 75600 // 128 == 590 and oint.max_intervals(590) == 295
    NB = 9
    most = max(len(oint.runs_of([j for j in range(NB) if m >> j & 1])) for m in range(1 << NB))
    assert most == oint.max_intervals(NB)


def test_intervals_brute_force_round_trip():
    NB = 10
    rows = [[j for j in range(NB) if m >> j & 1] for m in range(1 << NB)]
    for kept in rows:
        runs = oint.runs_of(kept)
        for s, e in runs:
            assert 0 <= s < e <= NB
        for (s0, e0), (s1, e1) in zip(runs, runs[1:]):
            assert s1 - e0 >= 1          # maximal: a skipped block between runs
        assert oint.decode_row(runs) == kept
    # the array forms, every subset at once, W = the theoretical maximum
    W = oint.max_intervals(NB)
    idx = np.full((len(rows), NB), -1, np.int32)
    cnt = np.zeros(len(rows), np.int32)
    for r, kept in enumerate(rows):
        idx[r, :len(kept)] = kept
        cnt[r] = len(kept)
    iv, n_int, n_runs = oint.kept_to_intervals(idx, cnt, W)
    assert np.array_equal(n_int, n_runs)
    assert np.all(iv[np.arange(W)[None, :] >= n_int[:, None]] == -1)
    mask, idx2, cnt2 = oint.intervals_to_kept(iv, n_int, NB)
    assert np.array_equal(cnt2, cnt) and np.array_equal(idx2, idx)
    for r, kept in enumerate(rows):
        assert np.flatnonzero(mask[r]).tolist() == kept


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_merge_is_fewest_added_blocks_then_leftmost(seed):
    """Brute force over every choice of gaps to fill: the merged row adds the
    fewest blocks, and among such choices fills the lexicographically
    smallest set of gaps (the leftmost)."""
    rng = np.random.default_rng(seed)
    NB = 24
    for _ in range(60):
        kept = np.flatnonzero(rng.random(NB) < rng.uniform(0.2, 0.7)).tolist()
        runs = oint.runs_of(kept)
        n = len(runs)
        gaps = [runs[r + 1][0] - runs[r][1] for r in range(n - 1)]
        for W in range(1, n):
            best = min(itertools.combinations(range(n - 1), n - W),
                       key=lambda c: (sum(gaps[g] for g in c), c))
            iv = [list(runs[0])]
            for r in range(n - 1):
                if r in best:
                    iv[-1][1] = runs[r + 1][1]
                else:
                    iv.append(list(runs[r + 1]))
            got = oint.merge_runs(runs, W)
            assert _as_lists(got) == iv
            dec = oint.decode_row(got)
            assert set(kept) <= set(dec) and len(dec) - len(kept) == sum(gaps[g] for g in best)


def test_width_for_merge_closed_forms():
    # a rows with x runs and b rows with y > x runs: the width is max(x, 1)
    # while ceil(q * (a + b)) <= a, else y
    for a, b, x, y in [(95, 5, 3, 40), (99, 1, 0, 7), (10, 30, 2, 5), (1, 1, 1, 2)]:
        n_runs = [x] * a + [y] * b
        hist = oint.run_histogram(n_runs, 2 * y)
        for q in (0.5, 0.9, 0.95, 0.99, 1.0):
            want = max(x, 1) if math.ceil(q * (a + b)) <= a else y
            assert oint.width_for_merge(hist, q) == want, (a, b, x, y, q)
    assert oint.list_bytes(10, 591) == 10 * 591 * 4 + 40
    assert oint.interval_bytes(10, 50) == 10 * 50 * 8 + 40


def test_planted_mistake_rightmost_gap_first_is_caught(monkeypatch):
    def rightmost(runs, W):
        iv = list(runs)
        while len(iv) > W:
            gaps = [iv[r + 1][0] - iv[r][1] for r in range(len(iv) - 1)]
            r = len(gaps) - 1 - gaps[::-1].index(min(gaps))
            iv[r:r + 2] = [(iv[r][0], iv[r + 1][1])]
        return iv
    monkeypatch.setattr(oint, "merge_runs", rightmost)
    with pytest.raises(AssertionError):
        test_intervals_golden_rows_and_widths()


def test_planted_mistake_inclusive_end_is_caught(monkeypatch):
    orig = oint.runs_of
    monkeypatch.setattr(oint, "runs_of", lambda kept: [(s, e - 1) for s, e in orig(kept)])
    with pytest.raises(AssertionError):
        test_intervals_golden_rows_and_widths()


# ------------------------------------------------ coarse tail (RECAP section 3.2)

def _random_lists(rng, B, H, NB, keep=0.4):
    idx = np.full((B, H, NB, NB), -1, np.int32)
    cnt = np.zeros((B, H, NB), np.int32)
    for pos in np.ndindex(B, H, NB):
        kept = np.flatnonzero(rng.random(NB) < keep)
        idx[pos][: kept.size] = kept
        cnt[pos] = kept.size
    idx[0, 0, 0] = np.arange(NB)      # a row keeping everything (empty tail)
    cnt[0, 0, 0] = NB
    cnt[0, 0, 1] = 0                   # a row keeping nothing
    return idx, cnt


def test_tail_is_exact_for_constant_blocks():
    """Keys and values constant within every block: zero key variance and zero
    value-key covariance, so the coarse tail equals the exact tail (closed
    form n_j exp(a . k_j) for the block masses)."""
    rng = np.random.default_rng(31)
    B, H, D, blk = 1, 2, 8, 16
    L = 5 * blk + 7
    NB = (L + blk - 1) // blk
    kap = rng.standard_normal((B, H, NB, D))
    nu = rng.standard_normal((B, H, NB, D))
    blocks = np.minimum(np.arange(L) // blk, NB - 1)
    k, v = kap[:, :, blocks], nu[:, :, blocks]
    q = rng.standard_normal((B, H, L, D)) * 2.0
    idx, cnt = _random_lists(rng, B, H, NB)
    stats = otail.block_stats(k, v, blk)
    assert np.all(stats[1] < 1e-24) and np.all(np.abs(stats[4]) < 1e-12)
    lbar, obar = otail.coarse_tail(q, stats, idx, cnt, blk)
    l_T, o_T = otail.exact_tail(q, k, v, idx, cnt, blk)
    fin = np.isfinite(l_T)
    assert np.array_equal(fin, np.isfinite(lbar))
    assert np.allclose(lbar[fin], l_T[fin], rtol=0, atol=1e-10)
    assert np.allclose(obar[fin], o_T[fin], rtol=0, atol=1e-10)
    assert np.all(np.isneginf(lbar[0, 0, :blk])) and np.all(obar[0, 0, :blk] == 0)


def _gaussian_block_case(seed):
    """One large block of Gaussian keys (diagonal covariance) with values
    v = M k + noise, followed by a short query block that keeps only itself,
    so that its tail is exactly the large block."""
    rng = np.random.default_rng(seed)
    D, blk, nq = 4, 65536, 8
    L = blk + nq
    mu = np.array([0.3, -0.2, 0.5, 0.1])
    sd = np.array([0.5, 0.8, 0.3, 0.6])
    M = np.array([[1.0, 0.5, 0.0, -0.3], [0.2, -1.0, 0.4, 0.0], [0.0, 0.3, 0.8, 0.5], [-0.6, 0.0, 0.2, 1.0]])
    k = np.empty((1, 1, L, D))
    k[0, 0, :blk] = mu + sd * rng.standard_normal((blk, D))
    k[0, 0, blk:] = rng.standard_normal((nq, D))
    v = np.empty((1, 1, L, D))
    v[0, 0] = k[0, 0] @ M.T + 0.3 * rng.standard_normal((L, D))
    q = np.zeros((1, 1, L, D))
    q[0, 0, blk:] = np.array([1.2, -0.9, 1.5, 0.8]) * (1 + 0.1 * rng.standard_normal((nq, D)))
    idx = np.full((1, 1, 2, 2), -1, np.int32)
    cnt = np.ones((1, 1, 2), np.int32)
    idx[0, 0, 0, 0], idx[0, 0, 1, 0] = 0, 1     # block 0 keeps itself, block 1 keeps itself
    return q, k, v, idx, cnt, blk, mu, sd, M


def test_tail_mass_is_the_gaussian_limit():
    """COBS reading: for Gaussian keys log mean_c exp(a . k_c) tends to
    a . mu + 1/2 sum_d a_d^2 sd_d^2.  The coarse log-mass matches the exact
    tail's within Monte Carlo error (~2e-3 at 65536 keys); dropping the
    variance term or doubling it misses by ~0.15."""
    q, k, v, idx, cnt, blk, mu, sd, M = _gaussian_block_case(41)
    lbar, _ = otail.coarse_tail(q, otail.block_stats(k, v, blk), idx, cnt, blk)
    l_T, _ = otail.exact_tail(q, k, v, idx, cnt, blk)
    rows = slice(blk, None)
    a = q[0, 0, rows] / 2.0
    err = np.abs(lbar[0, 0, rows] - l_T[0, 0, rows])
    assert err.max() < 0.02
    half_var = 0.5 * (a * a) @ (sd * sd)
    assert half_var.min() > 0.1                    # the variance term is not negligible here
    limit = np.log(blk) + a @ mu + half_var        # the population-moment closed form
    assert np.abs(l_T[0, 0, rows] - limit).max() < 0.03


def test_tail_value_is_the_gaussian_limit():
    """PISA reading: for jointly Gaussian keys and values the exp-weighted
    value mean is vbar + Cov(v, k) a.  The coarse output matches the exact
    tail output within Monte Carlo error; without C, or with C transposed, it
    misses by more than 0.1."""
    q, k, v, idx, cnt, blk, mu, sd, M = _gaussian_block_case(42)
    stats = otail.block_stats(k, v, blk)
    _, obar = otail.coarse_tail(q, stats, idx, cnt, blk)
    _, o_T = otail.exact_tail(q, k, v, idx, cnt, blk)
    rows = slice(blk, None)
    a = q[0, 0, rows] / 2.0
    assert np.abs(obar[0, 0, rows] - o_T[0, 0, rows]).max() < 0.03
    comp = a @ (M @ np.diag(sd * sd)).T            # M Sigma a, the population closed form
    assert np.abs(comp).max() > 0.1
    assert np.abs(o_T[0, 0, rows] - (mu @ M.T + comp)).max() < 0.04
    wrong = a @ (M @ np.diag(sd * sd))             # transposed covariance
    assert np.abs(wrong - comp).max() > 0.1


def test_reconstruction_with_same_step_refinement_is_dense():
    """A refinement taken at the step itself makes the reconstructed tail exact,
    so sparse part + tail is dense attention (the LSE merge of a partition of
    the keys); a row keeping every block returns its sparse output."""
    rng = np.random.default_rng(43)
    B, H, D, blk = 1, 2, 16, 16
    L = 6 * blk + 5
    NB = (L + blk - 1) // blk
    q, k, v = (rng.standard_normal((B, H, L, D)) for _ in range(3))
    idx, cnt = _random_lists(rng, B, H, NB)
    O_S, l_S = oatt.masked_attention(q, k, v, idx, cnt, blk)
    lbar, obar = otail.coarse_tail(q, otail.block_stats(k, v, blk), idx, cnt, blk)
    l_T, o_T = otail.exact_tail(q, k, v, idx, cnt, blk)
    d_l, d_o = otail.refinement(l_T, o_T, lbar, obar)
    O, lse = otail.reconstruct(l_S, O_S, lbar, obar, d_l, d_o)
    O_d, l_d = oatt.dense_attention(q, k, v)
    assert np.allclose(O, O_d, rtol=0, atol=1e-10) and np.allclose(lse, l_d, rtol=1e-12, atol=0)
    assert np.array_equal(O[0, 0, :blk], O_S[0, 0, :blk])       # all kept: the tail is empty
    # a stale refinement still leaves the all-kept row untouched and keeps the
    # output a convex combination in weight (the weights sum to 1)
    O2, lse2 = otail.reconstruct(l_S, O_S, lbar, obar, 0.5 * d_l, 0.5 * d_o)
    assert np.array_equal(O2[0, 0, :blk], O_S[0, 0, :blk])
    ws = np.exp(np.nan_to_num(l_S, neginf=-np.inf) - lse2)
    wt = np.exp(lbar + 0.5 * d_l - lse2)
    assert np.allclose(np.where(np.isneginf(l_S), 0, ws) + np.where(np.isneginf(lbar), 0, wt), 1.0, atol=1e-12)


def test_planted_mistake_variance_factor_is_caught(monkeypatch):
    orig = otail.block_stats

    def doubled(k, v, blk):
        kbar, s2, vbar, n, C = orig(k, v, blk)
        return kbar, 2 * s2, vbar, n, C     # as if the second-order term had no 1/2
    monkeypatch.setattr(otail, "block_stats", doubled)
    with pytest.raises(AssertionError):
        test_tail_mass_is_the_gaussian_limit()


def test_planted_mistake_transposed_covariance_is_caught(monkeypatch):
    orig = otail.block_stats

    def transposed(k, v, blk):
        kbar, s2, vbar, n, C = orig(k, v, blk)
        return kbar, s2, vbar, n, np.swapaxes(C, -1, -2)
    monkeypatch.setattr(otail, "block_stats", transposed)
    with pytest.raises(AssertionError):
        test_tail_value_is_the_gaussian_limit()


# ------------------------------------------------- planted mistakes are caught

def test_planted_mistake_strict_inequality_is_caught(monkeypatch):
    def strict(P_row, p):
        P_row = otop.clamp_probs(P_row)
        nb = P_row.shape[0]
        if np.float32(p) == 1:
            return np.arange(nb, dtype=np.int32), nb
        order = np.lexsort((np.arange(nb), -P_row.astype(np.float64)))
        u = otop.fixed_point_mass(P_row)
        T = int(np.ceil(np.float64(np.float32(p)) * float(u.sum())))
        csum = np.cumsum(u[order])
        k = int(np.argmax(csum > T)) + 1  # planted: ">" instead of ">="
        return np.sort(order[:k]).astype(np.int32), k
    monkeypatch.setattr(otop, "select_row", strict)
    with pytest.raises(AssertionError):
        test_topp_golden_rows()


def test_planted_mistake_tie_order_is_caught(monkeypatch):
    orig = otop.select_row

    def highest_index_first(P_row, p):
        kept, k = orig(np.asarray(P_row)[::-1].copy(), p)
        return np.sort(len(P_row) - 1 - kept).astype(np.int32), k
    monkeypatch.setattr(otop, "select_row", highest_index_first)
    with pytest.raises(AssertionError):
        test_topp_golden_rows()


def test_planted_mistake_pool_divisor_is_caught(monkeypatch):
    def full_divisor(x, blk):
        x = np.asarray(x, dtype=np.float64)
        B, H, L, D = x.shape
        nb = (L + blk - 1) // blk
        out = np.zeros((B, H, nb, D))
        for i in range(nb):
            out[:, :, i] = x[:, :, i * blk:(i + 1) * blk].sum(2) / blk  # planted
        return out.astype(np.float32)
    monkeypatch.setattr(osco, "pool_blocks", full_divisor)
    with pytest.raises(AssertionError):
        test_pool_golden_ramps()


def test_planted_mistake_transposed_logits_is_caught(monkeypatch):
    orig = osco.block_logits
    monkeypatch.setattr(osco, "block_logits", lambda a, b: np.swapaxes(orig(a, b), -1, -2))
    with pytest.raises(AssertionError):
        test_block_probs_prefers_aligned_key()


def test_planted_mistake_attention_scale_is_caught(monkeypatch):
    def no_scale(q_rows, k, v, cols):
        kc = np.asarray(k, dtype=np.float64)[cols]
        s = np.asarray(q_rows, dtype=np.float64) @ kc.T  # planted: no 1/sqrt(D)
        m = s.max(1, keepdims=True)
        lse = m[:, 0] + np.log(np.exp(s - m).sum(1))
        return np.exp(s - lse[:, None]) @ np.asarray(v, dtype=np.float64)[cols], lse
    monkeypatch.setattr(oatt, "attend_rows", no_scale)
    with pytest.raises(AssertionError):
        test_keep_all_equals_torch_sdpa_float64()


def test_planted_mistake_hilbert_axis_order_is_caught(monkeypatch):
    orig = ohil.hilbert_index
    monkeypatch.setattr(ohil, "hilbert_index", lambda c, k: orig(np.asarray(c)[::-1], k))
    with pytest.raises(AssertionError):
        test_hilbert_2d_matches_textbook_curve(2)
