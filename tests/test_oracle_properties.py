"""Property-based checks of the oracle (CPU): random inputs drawn by
hypothesis, each checked against what the definitions imply -- top-p
selection is the shortest ordered prefix reaching the target, interval
encoding decodes back and merging adds the fewest blocks, the drift does not
depend on the scale of the means, a refinement taken at the same step
turns the coarse tail into the exact one, E4M3 encoding is the nearest
value, monotone, and bounded in its block quantization error, and the masked
attention depends on the kept set only (not its order), is affine in V and
moves its LSE by exactly q.c/sqrt(D) when every key is shifted by c."""

import itertools

import numpy as np
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

from oracle import attention as oatt
from oracle import fp8 as ofp8
from oracle import intervals as oint
from oracle import reuse as oreu
from oracle import tail as otail
from oracle import topp as otop

SETTINGS = settings(max_examples=60, deadline=None, suppress_health_check=[HealthCheck.too_slow])


@SETTINGS
@given(st.lists(st.floats(0.0, 1.0, width=32), min_size=1, max_size=40),
       st.floats(0.0078125, 1.0, width=32))
def test_topp_is_the_shortest_ordered_prefix(row, p):
    P = np.asarray(row, np.float32)
    kept, k = otop.select_row(P, np.float32(p))
    assert k == len(kept) >= 1 and list(kept) == sorted(kept)
    if np.float32(p) == 1:
        assert k == P.size
        return
    u = otop.fixed_point_mass(otop.clamp_probs(P))
    T = int(np.ceil(np.float64(np.float32(p)) * np.float64(int(u.sum()))))
    order = sorted(range(P.size), key=lambda j: (-float(otop.clamp_probs(P)[j]), j))
    assert sorted(order[:k]) == list(kept)              # a prefix of the order
    if T > 0:
        assert int(u[kept].sum()) >= T                   # reaches the target
        assert int(u[order[:k - 1]].sum()) < T           # one block fewer does not


@SETTINGS
@given(st.integers(1, 48).flatmap(lambda nb: st.tuples(st.just(nb), st.sets(st.integers(0, nb - 1)),
                                                       st.integers(1, nb))))
def test_intervals_round_trip_and_fewest_added_blocks(args):
    nb, kept_set, W = args
    kept = sorted(kept_set)
    runs = oint.runs_of(kept)
    assert len(runs) <= oint.max_intervals(nb)
    merged = oint.merge_runs(runs, W)
    assert len(merged) == min(len(runs), W)
    dec = oint.decode_row(merged)
    assert set(kept) <= set(dec) and dec == sorted(set(dec))
    if len(runs) <= W:
        assert dec == kept
    gaps = sorted(runs[r + 1][0] - runs[r][1] for r in range(len(runs) - 1))
    assert len(dec) - len(kept) == sum(gaps[:max(0, len(runs) - W)])   # the smallest gaps are filled


@SETTINGS
@given(st.integers(0, 2 ** 31 - 1), st.floats(0.01, 100.0))
def test_drift_does_not_depend_on_the_scale_of_the_means(seed, c):
    rng = np.random.default_rng(seed)
    ref_q, ref_k = rng.standard_normal((1, 2, 5, 8)), rng.standard_normal((1, 2, 5, 8))
    q = ref_q + 0.1 * rng.standard_normal(ref_q.shape)
    k = ref_k + 0.2 * rng.standard_normal(ref_k.shape)
    d1 = oreu.block_drift(ref_q, ref_k, q, k)
    d2 = oreu.block_drift(c * ref_q, c * ref_k, c * q, c * k)
    assert np.allclose(d1, d2, rtol=1e-9, atol=0)


@settings(max_examples=15, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(st.integers(0, 2 ** 31 - 1), st.integers(1, 5), st.integers(0, 15))
def test_same_step_refinement_makes_the_tail_exact(seed, nblocks, ragged):
    rng = np.random.default_rng(seed)
    blk, D = 8, 4
    L = nblocks * blk + ragged
    NB = (L + blk - 1) // blk
    q, k, v = (rng.standard_normal((1, 1, L, D)) for _ in range(3))
    idx = np.full((1, 1, NB, NB), -1, np.int32)
    cnt = np.zeros((1, 1, NB), np.int32)
    for i in range(NB):
        sel = np.flatnonzero(rng.random(NB) < 0.5)
        idx[0, 0, i, :sel.size] = sel
        cnt[0, 0, i] = sel.size
    O_S, l_S = oatt.masked_attention(q, k, v, idx, cnt, blk)
    lbar, obar = otail.coarse_tail(q, otail.block_stats(k, v, blk), idx, cnt, blk)
    l_T, o_T = otail.exact_tail(q, k, v, idx, cnt, blk)
    O, lse = otail.reconstruct(l_S, O_S, lbar, obar, *otail.refinement(l_T, o_T, lbar, obar))
    O_d, l_d = oatt.dense_attention(q, k, v)
    assert np.allclose(O, O_d, atol=1e-10) and np.allclose(lse, l_d, rtol=1e-12, atol=1e-12)


@SETTINGS
@given(st.integers(1, 12), st.integers(1, 12), st.integers(1, 12))
def test_hilbert_order_is_a_bijection_on_any_grid(T, Hh, W):
    from oracle import hilbert as ohil
    perm, inv = ohil.hilbert_perm(T, Hh, W)
    L = T * Hh * W
    assert sorted(perm.tolist()) == list(range(L))
    assert np.array_equal(perm[inv], np.arange(L)) and np.array_equal(inv[perm], np.arange(L))
    x = np.arange(L * 2, dtype=np.float64).reshape(1, L, 2)
    assert np.array_equal(ohil.permute_rows(ohil.permute_rows(x, perm), perm, inverse=True), x)


@settings(max_examples=15, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(st.integers(0, 2 ** 31 - 1), st.integers(1, 4), st.integers(0, 7))
def test_refresh_kept_share_is_a_mixture_weight(seed, nblocks, ragged):
    from oracle import refresh as oref
    rng = np.random.default_rng(seed)
    blk, D = 8, 4
    L = nblocks * blk + ragged
    NB = (L + blk - 1) // blk
    q, k, v = (rng.standard_normal((1, 1, L, D)) for _ in range(3))
    idx = np.full((1, 1, NB, NB), -1, np.int32)
    cnt = np.zeros((1, 1, NB), np.int32)
    for i in range(NB):
        sel = np.flatnonzero(rng.random(NB) < 0.5)
        idx[0, 0, i, :sel.size] = sel
        cnt[0, 0, i] = sel.size
    Od, Ld, Os, Ls, R, mass = oref.fused_refresh(q, k, v, idx, cnt, blk)
    assert np.all((mass >= 0) & (mass <= 1 + 1e-12))
    ci, cc = oref.complement_lists(idx, cnt, NB)
    Oc, Lc = oatt.masked_attention(q, k, v, ci, cc, blk)
    mix = mass[..., None] * np.nan_to_num(Os) + (1 - mass)[..., None] * np.nan_to_num(Oc)
    assert np.allclose(mix, Od, atol=1e-10)


_E4M3_CODES = np.array([c for c in range(256) if not np.isnan(ofp8.e4m3_value(np.uint8(c)))], np.uint8)
_E4M3_VALUES = ofp8.e4m3_value(_E4M3_CODES)


@SETTINGS
@given(st.lists(st.floats(-600.0, 600.0, width=32), min_size=1, max_size=64))
def test_e4m3_is_the_nearest_value_and_monotone(xs):
    x = np.asarray(xs, np.float32)
    v = ofp8.e4m3_value(ofp8.e4m3_encode(x))
    xc = np.clip(x.astype(np.float64), -448.0, 448.0)
    best = np.abs(xc[:, None] - _E4M3_VALUES[None, :]).min(axis=1)
    assert np.array_equal(np.abs(v - xc), best)          # no representable value is nearer
    order = np.argsort(x, kind="stable")
    assert np.all(np.diff(v[order]) >= 0)                 # encoding keeps the order


@SETTINGS
@given(st.integers(0, 2 ** 31 - 1), st.integers(1, 300), st.floats(1e-3, 1e3))
def test_block_quantization_error_is_one_e4m3_rounding(seed, L, spread):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((1, 1, L, 8)) * spread).astype(np.float32)
    codes, scales = ofp8.quantize_blocks(x, 128)
    deq = ofp8.dequantize_blocks(codes, scales, 128)
    s = np.broadcast_to(np.repeat(scales.astype(np.float64), 128, axis=2)[:, :, :L, None], x.shape)
    err = np.abs(deq - x)
    normal = np.abs(x) >= 2.0 ** -6 * s
    # half a unit in the last place: 2^-4 relative for normal codes, 2^-10
    # of the scale for subnormal ones, plus the float32 rounding of x * (448 / amax)
    assert np.all(err[normal] <= (2.0 ** -4 + 2.0 ** -20) * np.abs(x[normal]))
    assert np.all(err[~normal] <= (2.0 ** -10 + 2.0 ** -20) * s[~normal])


def _attention_case(seed, nblocks, ragged, blk=8, D=8):
    rng = np.random.default_rng(seed)
    L = max(1, nblocks * blk - ragged)
    nb = (L + blk - 1) // blk
    q, k, v = (rng.standard_normal((1, 1, L, D)) for _ in range(3))
    idx = np.full((1, 1, nb, nb), -1, np.int32)
    cnt = np.zeros((1, 1, nb), np.int32)
    for i in range(nb):
        kept = np.flatnonzero(rng.uniform(size=nb) < 0.6)
        idx[0, 0, i, :len(kept)] = kept
        cnt[0, 0, i] = len(kept)
    return q, k, v, idx, cnt, blk, rng


@SETTINGS
@given(st.integers(0, 2 ** 31 - 1), st.integers(1, 5), st.integers(0, 7))
def test_masked_attention_depends_on_the_kept_set_not_its_order(seed, nblocks, ragged):
    q, k, v, idx, cnt, blk, rng = _attention_case(seed, nblocks, ragged)
    shuffled = idx.copy()
    for i in range(idx.shape[2]):
        c = cnt[0, 0, i]
        shuffled[0, 0, i, :c] = rng.permutation(idx[0, 0, i, :c])
    O1, L1 = oatt.masked_attention(q, k, v, idx, cnt, blk)
    O2, L2 = oatt.masked_attention(q, k, v, shuffled, cnt, blk)
    np.testing.assert_allclose(np.nan_to_num(O2), np.nan_to_num(O1), rtol=0, atol=1e-12)
    np.testing.assert_allclose(np.nan_to_num(L2, neginf=0), np.nan_to_num(L1, neginf=0), rtol=0, atol=1e-12)


@SETTINGS
@given(st.integers(0, 2 ** 31 - 1), st.integers(1, 5), st.integers(0, 7), st.floats(-3.0, 3.0), st.floats(-3.0, 3.0))
def test_masked_attention_is_affine_in_v_and_shift_invariant_in_k(seed, nblocks, ragged, a, b):
    """Softmax weights sum to one per row: O(a V + b) = a O + b.  Adding one
    vector c to every key adds q.c / sqrt(D) to every logit of a query row:
    O is unchanged and LSE moves by exactly that amount."""
    q, k, v, idx, cnt, blk, rng = _attention_case(seed, nblocks, ragged)
    O, LSE = oatt.masked_attention(q, k, v, idx, cnt, blk)
    rows = np.isfinite(LSE)  # rows that keep at least one block
    Oa, _ = oatt.masked_attention(q, k, a * v + b, idx, cnt, blk)
    np.testing.assert_allclose(Oa[rows], (a * O + b)[rows], rtol=0, atol=1e-9)
    c = rng.standard_normal(q.shape[-1])
    Os, Ls = oatt.masked_attention(q, k + c, v, idx, cnt, blk)
    np.testing.assert_allclose(Os[rows], O[rows], rtol=0, atol=1e-9)
    shift = (q @ c)[..., :] / np.sqrt(q.shape[-1])
    np.testing.assert_allclose(Ls[rows], (LSE + shift)[rows], rtol=0, atol=1e-9)
