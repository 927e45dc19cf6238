"""Pins for the CPU oracle, independent of the oracle's own code.

Each test checks the oracle against something the pages or the mathematics
fix: closed forms of the Sobol prefix counts, the full-period invariant,
brute force over every level pair, special cases, hand-derived examples, the
linear cost identity, library routines for the quantiser, and exhaustive
search for the tilt apportionment.  No GPU is needed.
"""
import math
import os

import numpy as np
import pytest

GOLD = os.path.join(os.path.dirname(__file__), "golden")
P = 8
Q = 1 << P


def _bitrev(l, p=P):
    return int(format(l, f"0{p}b")[::-1], 2)


def _prefix_counts(K):
    """C[b, m] = #{l < m : K[b, l] = 1}, m = 0..Q."""
    return np.concatenate([np.zeros((K.shape[0], 1), np.int64), np.cumsum(K, axis=1)], axis=1)


def _closed_form_T(C, L):
    """Two-counter closed form: count = C[b, n] + (L - n) - C[b, L - n], n = C[a, L]."""
    n = C[:, L]                                  # ones in A's stream, per level a
    b = np.arange(C.shape[0])
    return C[b[None, :], n[:, None]] + (L - n)[:, None] - C[b[None, :], (L - n)[:, None]]


# ---------------------------------------------------------------- Sobol-8 --

def test_sobol_direction_numbers_equal_bit_reversal(orc):
    # First Sobol dimension in natural order = van der Corput radical inverse.
    for p in range(1, 9):
        r = orc.sobol_r(p)
        assert [int(v) - 1 for v in r] == [_bitrev(l, p) for l in range(1 << p)]


def test_prefix_count_closed_forms(orc):
    K = orc.indicator(P).astype(np.int64)
    C = _prefix_counts(K)
    b = np.arange(Q + 1)
    for k in range(P + 1):
        assert np.array_equal(C[:, 1 << k], -(-b // (1 << (P - k)))), k
    assert np.array_equal(C[:, 96], -(-b // 4) + -(-np.maximum(b - 2, 0) // 8))
    assert np.array_equal(C[:, 192], -(-b // 2) + -(-np.maximum(b - 1, 0) // 4))


def test_full_period_reproduces_level(orc):
    # A full-period stream (L = 2^p) holds exactly b ones: the decoded value
    # 2 b / 2^p - 1 is the level's own value x / 2^(p-1).
    for p in range(1, 9):
        K = orc.indicator(p)
        assert np.array_equal(K.sum(axis=1), np.arange((1 << p) + 1))


def test_indicator_is_monotone_in_level(orc):
    K = orc.indicator(P).astype(int)
    assert np.all(np.diff(K, axis=0) >= 0)


# ------------------------------------------------------------------ C-BSG --

@pytest.mark.slow
def test_cbsg_bit_by_bit_equals_closed_form_all_pairs_all_lengths(orc):
    K = orc.indicator(P).astype(np.int64)
    C = _prefix_counts(K)
    for L in range(0, Q + 1):
        T = orc.cbsg_table(L)
        assert np.array_equal(T, _closed_form_T(C, L)), L


def test_cbsg_special_cases(orc):
    K = orc.indicator(P).astype(np.int64)
    C = _prefix_counts(K)
    for L in (1, 2, 63, 64, 96, 128, 191, 192, 255, 256):
        T = orc.cbsg_table(L)
        if L % 2 == 0:
            assert np.all(T[128, :] == L // 2)          # x_A = 0: zero product
            assert np.all(T[:, 128] == L // 2)          # x_B = 0: zero product
        assert np.array_equal(T[0, :], L - C[:, L])     # A all zeros: counts B's zeros
        assert np.array_equal(T[Q, :], C[:, L])         # A all ones: counts B's ones
        assert T.min() >= 0 and T.max() <= L


def test_cbsg_streams_follow_two_enable_counters(orc):
    K = orc.indicator(P)
    for a, b, L in [(192, 77, 256), (3, 250, 96), (200, 200, 64)]:
        za, zb = orc.cbsg_streams(a, b, L)
        assert np.array_equal(za, K[a, :L])
        # B's bits at A's ones are K[b]'s prefix, and likewise at A's zeros
        assert np.array_equal(zb[za == 1], K[b, : int(za.sum())])
        assert np.array_equal(zb[za == 0], K[b, : int(L - za.sum())])
        assert orc.cbsg_count(a, b, L) == int(np.sum(za == zb))


def test_enable_window_matches_why_it_works(orc):
    rows = [l.split() for l in open(os.path.join(GOLD, "enable_window_vit.txt"))
            if l.strip() and not l.startswith("#")]
    p, L = map(int, rows[0])
    K = orc.indicator(p)
    for x, want in ((int(u), int(v)) for u, v in rows[1:]):
        za, _ = orc.cbsg_streams(x + (1 << (p - 1)), 128, L, p)
        n_one = int(za.sum())
        assert abs(n_one - (L - n_one)) == want


def test_hand_derived_counts(orc):
    for line in open(os.path.join(GOLD, "decode_examples.txt")):
        if line.startswith("#") or not line.strip():
            continue
        a, b, L, want = map(int, line.split())
        assert orc.cbsg_count(a, b, L) == want, (a, b, L)


def test_decode_at_full_period_is_exact_on_a_worked_pair(orc):
    # a = b = 192 (x = 64), L = 256: count 160, 2*160/256 - 1 = 1/4 = 64*64/128^2.
    a_lv = np.full((1, 1, 1), 192, np.uint8)
    b_lv = np.full((1, 1, 1), 192, np.uint8)
    counts, out, steps = orc.matmul(a_lv, np.ones((1, 1), np.float32), b_lv,
                                    np.ones((1, 1), np.float32), np.zeros((1, 1), np.int32), [256])
    assert counts.ravel()[0] == 160 and out.ravel()[0] == 4096.0 and steps == 256


# -------------------------------------------------------------- quantiser --

def test_quantize_integer_rows_round_trip(orc):
    rng = np.random.default_rng(0)
    x = rng.integers(-127, 128, size=(33, 70)).astype(np.float32)
    x[:, 0] = 127.0                                     # amax = 127 -> s = 1
    lv, s = orc.quantize(x, axis=0)
    assert np.all(s == 1.0)
    assert np.array_equal(lv.astype(int), x.astype(int) + 128)


def test_quantize_matches_float32_library_rounding(orc):
    rng = np.random.default_rng(1)
    x = (rng.standard_normal((50, 257)) * rng.uniform(0.01, 30, (50, 1))).astype(np.float32)
    x[3] = 0.0
    lv, s = orc.quantize(x, axis=0)
    amax = np.abs(x).max(axis=1).astype(np.float32)
    s_ref = amax / np.float32(127.0)
    assert np.array_equal(s, s_ref)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.where(s_ref[:, None] > 0, np.rint(x / s_ref[:, None]), 0.0)
    ref = np.clip(q, -127, 127).astype(int) + 128
    assert np.array_equal(lv.astype(int), ref)
    # the row maximum maps to +-127, a zero row to level 128 with scale 0
    i = np.abs(x[0]).argmax()
    assert abs(int(lv[0, i]) - 128) == 127
    assert s[3] == 0.0 and np.all(lv[3] == 128)


def test_quantize_ties_round_half_to_even(orc):
    x = np.array([[127.0, 2.5, 3.5, -2.5, -0.5, 0.5, 1.5]], np.float32)
    lv, _ = orc.quantize(x)
    assert list(lv[0].astype(int) - 128) == [127, 2, 4, -2, 0, 0, 2]


def test_quantize_axis1_is_axis0_of_transpose(orc):
    rng = np.random.default_rng(2)
    x = rng.standard_normal((67, 45)).astype(np.float32)
    lv1, s1 = orc.quantize(x, axis=1)
    lv0, s0 = orc.quantize(np.ascontiguousarray(x.T), axis=0)
    assert np.array_equal(lv1, lv0) and np.array_equal(s1, s0)


def test_quantize_flags_nonfinite(orc):
    x = np.array([[1.0, np.nan, 2.0]], np.float32)
    with pytest.raises(orc.OracleError) as e:
        orc.quantize(x)
    assert e.value.code == orc.ERR_NONFINITE


# ------------------------------------------------------------------ rungs --

def test_row_stat_modes(orc):
    x = np.array([[-3.0, 1.0, 2.0], [0.1, 0.7, 0.2]], np.float32)
    assert list(orc.row_stat(x, orc.STAT_AMAX)) == [3.0, np.float32(0.7)]
    assert list(orc.row_stat(x, orc.STAT_ROWMAX)) == [2.0, np.float32(0.7)]


def test_rungs_by_definition(orc):
    tau = np.array([0.8, 0.6, 0.4, 0.2], np.float32)
    stat = np.array([1.0, 0.8, 0.6, 0.4, 0.2, 0.19, 0.0, 0.79999], np.float32)
    assert list(orc.assign_rungs(stat, tau, 5)) == [4, 4, 3, 2, 1, 0, 0, 3]
    # brute force on random groups: rung = #{k : g/max >= tau_k}
    rng = np.random.default_rng(3)
    st = rng.exponential(size=(7, 100)).astype(np.float32)
    r = orc.assign_rungs(st, tau, 5)
    gt = st / st.max(axis=1, keepdims=True)
    assert np.array_equal(r, (gt[..., None] >= tau).sum(-1))
    assert np.all(orc.assign_rungs(np.zeros((2, 5), np.float32), tau, 5) == 0)
    assert np.all(orc.assign_rungs(st, tau[:0], 1) == 0)


def test_rungs_reject_unsorted_tau(orc):
    with pytest.raises(orc.OracleError):
        orc.assign_rungs(np.ones(4, np.float32), np.array([0.2, 0.8], np.float32), 3)


# ----------------------------------------------------------------- matmul --

def _small_problem(rng, batch, M, N, D):
    a_lv = rng.integers(1, 256, (batch, M, D)).astype(np.uint8)
    b_lv = rng.integers(1, 256, (batch, N, D)).astype(np.uint8)
    a_s = rng.uniform(0.01, 1, (batch, M)).astype(np.float32)
    b_s = rng.uniform(0.01, 1, (batch, N)).astype(np.float32)
    rung = rng.integers(0, 5, (batch, M)).astype(np.int32)
    return a_lv, a_s, b_lv, b_s, rung


def test_matmul_counts_equal_table_sum_and_cost_identity(orc):
    rng = np.random.default_rng(4)
    ladder = np.array([64, 96, 128, 192, 256], np.int32)
    a_lv, a_s, b_lv, b_s, rung = _small_problem(rng, 2, 9, 7, 13)
    counts, out, steps = orc.matmul(a_lv, a_s, b_lv, b_s, rung, ladder)
    C = _prefix_counts(orc.indicator(P).astype(np.int64))
    tables = {int(L): _closed_form_T(C, int(L)) for L in ladder}
    for g in range(2):
        for i in range(9):
            T = tables[int(ladder[rung[g, i]])]
            want = T[a_lv[g, i][None, :], b_lv[g][:, :]].sum(axis=1)
            assert np.array_equal(counts[g, i, :, 0], want)
    # early termination: simulated XNORs = sum_i L_i * N * D
    assert steps == int(ladder[rung].sum()) * 7 * 13
    # decode from the exact integers
    L = ladder[rung][..., None].astype(np.float64)
    ref = (a_s[..., None].astype(np.float64) * b_s[:, None, :] * 128.0 ** 2
           * (2.0 * counts[..., 0] / L - 13))
    np.testing.assert_array_equal(out, ref.astype(np.float32))


def test_matmul_selected_outputs_match_full(orc):
    rng = np.random.default_rng(5)
    ladder = np.array([64, 96, 128, 192, 256], np.int32)
    a_lv, a_s, b_lv, b_s, rung = _small_problem(rng, 3, 5, 6, 11)
    c_all, o_all, _ = orc.matmul(a_lv, a_s, b_lv, b_s, rung, ladder)
    sel = np.array([[0, 0, 0], [2, 4, 5], [1, 3, 2]], np.int64)
    c, o, steps = orc.matmul(a_lv, a_s, b_lv, b_s, rung, ladder, sel=sel)
    for k, (g, i, j) in enumerate(sel):
        assert c[k, 0] == c_all[g, i, j, 0] and o[k] == o_all[g, i, j]
    assert steps == sum(int(ladder[rung[g, i]]) * 11 for g, i, _ in sel)


def _pool3():
    from mixed_precision_vit_b200.workloads import sobol_pool
    return sobol_pool(3, P)


def test_memo_matmul_equals_bit_by_bit_matmul(orc):
    """The memoised oracle (each (a, b, L) count read from a table of
    bit-by-bit counts) gives the literal oracle's counts, outputs and cost on
    every variant: ladder rows, K-bands with a tilt, per-band scales, the
    unipolar mode, seed-bank variants of B, all outputs and selected ones."""
    rng = np.random.default_rng(21)
    ladder = np.array([64, 96, 128, 192, 256], np.int32)
    a_lv, a_s, b_lv, b_s, rung = _small_problem(rng, 2, 7, 6, 32)
    a_lv[0, 0, :5] = 0                                     # the level range's ends
    b_lv[1, 2, :7] = 255
    bl = orc.kband_tilt(ladder, 4, 0.25, 256)
    a_sb = rng.uniform(0.01, 1, (2, 7, 4)).astype(np.float32)
    b_sb = rng.uniform(0.01, 1, (2, 6, 4)).astype(np.float32)
    sel = np.array([[0, 0, 0], [1, 6, 5], [1, 2, 2], [0, 3, 4]], np.int64)
    cases = [dict(), dict(band_len=bl, chunk_d=8), dict(band_len=bl, chunk_d=8, band_scales=True),
             dict(unipolar=True), dict(b_shift=37), dict(b_antithetic=True, b_shift=5),
             dict(sel=sel), dict(sel=sel, band_len=bl, chunk_d=8), dict(gray=True),
             dict(pool=_pool3()), dict(pool=_pool3(), band_len=bl, chunk_d=8),
             dict(pool=_pool3(), unipolar=True)]
    for kw in cases:
        sa, sb = (a_sb, b_sb) if kw.get("band_scales") else (a_s, b_s)
        want = orc.matmul(a_lv, sa, b_lv, sb, rung, ladder, **kw)
        got = orc.matmul(a_lv, sa, b_lv, sb, rung, ladder, memo=True, **kw)
        assert np.array_equal(got[0], want[0]), kw
        np.testing.assert_array_equal(got[1], want[1])
        assert got[2] == want[2], kw


def test_matmul_zero_operand_gives_zero(orc):
    rng = np.random.default_rng(6)
    a_lv, a_s, b_lv, b_s, rung = _small_problem(rng, 1, 4, 4, 9)
    a_lv[0, 2, :] = 128                                    # x = 0 row
    _, out, _ = orc.matmul(a_lv, a_s, b_lv, b_s, rung, [64, 96, 128, 192, 256])
    assert np.all(out[0, 2] == 0.0)


def test_matmul_bands_tilt_zero_is_parent(orc):
    gate = dict(l.split() for l in open(os.path.join(GOLD, "kband_gates.txt"))
                if l.strip() and not l.startswith("#"))
    rng = np.random.default_rng(7)
    ladder = np.array([64, 96, 128, 192, 256], np.int32)
    n_bands, chunk = 4, 8
    a_lv, a_s, b_lv, b_s, rung = _small_problem(rng, 1, 6, 5, n_bands * chunk)
    c0, o0, s0 = orc.matmul(a_lv, a_s, b_lv, b_s, rung, ladder)
    bl = orc.kband_tilt(ladder, n_bands, 0.0, 256)
    c1, o1, s1 = orc.matmul(a_lv, a_s, b_lv, b_s, rung, ladder, band_len=bl, chunk_d=chunk)
    assert np.array_equal(c1.sum(-1), c0[..., 0]) and s1 == s0
    rel = np.linalg.norm(o1 - o0) / np.linalg.norm(o0)
    assert rel < float(gate["parent_rel_err_max"])
    bt = orc.kband_tilt(ladder, n_bands, 0.25, 256)
    c2, o2, s2 = orc.matmul(a_lv, a_s, b_lv, b_s, rung, ladder, band_len=bt, chunk_d=chunk)
    assert s2 == s0                                        # iso-compute identity
    rel = np.linalg.norm(o2 - o0) / np.linalg.norm(o0)
    assert rel > float(gate["tilted_rel_err_min"])


def test_matmul_rejects_band_width_mismatch(orc):
    rng = np.random.default_rng(8)
    a_lv, a_s, b_lv, b_s, rung = _small_problem(rng, 1, 2, 2, 10)
    bl = np.full((3, 5), 64, np.int32)
    with pytest.raises(orc.OracleError) as e:
        orc.matmul(a_lv, a_s, b_lv, b_s, rung, [64, 96, 128, 192, 256], band_len=bl, chunk_d=4)
    assert e.value.code == orc.ERR_TABLE


# ------------------------------------------------- per-(row, band) scales --
# [K-band pull request, "Summary": the contraction axis is partitioned into
# bands of whole quantisation chunks]; here one chunk per band.

def test_quantize_chunked_hand_values(orc):
    # chunk 0: amax 127 -> s = 1; chunk 1: amax 254 -> s = 2 (both exact in fp32)
    x = np.array([[127.0, -64.0, 0.5, 0.0, 254.0, -127.0, 3.0, 1.0]], np.float32)
    lv, sc = orc.quantize_chunked(x, 4)
    assert sc.tolist() == [[1.0, 2.0]]
    # 0.5 -> 0 and -63.5 -> -64 and 1.5 -> 2 and 0.5 -> 0 (ties to even), level = x + 128
    assert lv.tolist() == [[255, 64, 128, 128, 255, 64, 130, 128]]


def test_quantize_chunked_chunks_are_independent_rows(orc):
    rng = np.random.default_rng(31)
    x = (rng.standard_normal((5, 24)) * np.array([1.0, 10.0, 0.1])[np.arange(24) // 8]).astype(np.float32)
    lv, sc = orc.quantize_chunked(x, 8)
    for c in range(3):
        lvc, scc = orc.quantize(np.ascontiguousarray(x[:, 8 * c:8 * c + 8]), axis=0)
        assert np.array_equal(lv[:, 8 * c:8 * c + 8], lvc) and np.array_equal(sc[:, c], scc)
    lv1, sc1 = orc.quantize_chunked(x, 24)                  # one chunk = the row scale
    lv0, sc0 = orc.quantize(x, axis=0)
    assert np.array_equal(lv1, lv0) and np.array_equal(sc1[:, 0], sc0)


def test_matmul_band_scales_decode_by_hand(orc):
    # every band's term carries its own scales: C = q^2 sum_b s_ib s_jb (2 c_b / L_b - D_b)
    from fractions import Fraction
    rng = np.random.default_rng(32)
    n_bands, chunk = 3, 4
    ladder = np.array([64, 128], np.int32)
    bl = np.array([[48, 128], [64, 128], [80, 128]], np.int32)    # per (band, rung) lengths
    a_lv = rng.integers(1, 256, (1, 2, n_bands * chunk)).astype(np.uint8)
    b_lv = rng.integers(1, 256, (1, 3, n_bands * chunk)).astype(np.uint8)
    a_s = np.array([[[0.5, 0.25, 2.0], [1.5, 0.75, 0.125]]], np.float32)
    b_s = np.array([[[0.5, 1.0, 4.0], [0.25, 2.0, 0.5], [1.0, 1.0, 1.0]]], np.float32)
    rung = np.array([[0, 1]], np.int32)
    counts, out, _ = orc.matmul(a_lv, a_s, b_lv, b_s, rung, ladder, band_len=bl, chunk_d=chunk,
                                band_scales=True)
    for i in range(2):
        for j in range(3):
            acc = Fraction(0)
            for b in range(n_bands):
                L = int(bl[b, rung[0, i]])
                c = sum(orc.cbsg_count(int(a_lv[0, i, d]), int(b_lv[0, j, d]), L)
                        for d in range(b * chunk, (b + 1) * chunk))
                assert counts[0, i, j, b] == c
                acc += (Fraction(float(a_s[0, i, b])) * Fraction(float(b_s[0, j, b]))
                        * (Fraction(2 * c, L) - chunk))
            assert out[0, i, j] == np.float32(float(128 * 128 * acc))


def test_matmul_band_scales_equal_row_scales_is_plain_decode(orc):
    rng = np.random.default_rng(33)
    ladder = np.array([64, 96, 128, 192, 256], np.int32)
    n_bands, chunk = 4, 8
    a_lv, a_s, b_lv, b_s, rung = _small_problem(rng, 2, 6, 5, n_bands * chunk)
    bl = orc.kband_tilt(ladder, n_bands, 0.25, 256)
    c0, o0, _ = orc.matmul(a_lv, a_s, b_lv, b_s, rung, ladder, band_len=bl, chunk_d=chunk)
    a_sb = np.repeat(a_s[..., None], n_bands, axis=-1)
    b_sb = np.repeat(b_s[..., None], n_bands, axis=-1)
    c1, o1, _ = orc.matmul(a_lv, a_sb, b_lv, b_sb, rung, ladder, band_len=bl, chunk_d=chunk,
                           band_scales=True)
    assert np.array_equal(c0, c1)
    np.testing.assert_allclose(o1, o0, rtol=1e-6, atol=0)


def test_matmul_band_scales_need_bands(orc):
    rng = np.random.default_rng(34)
    a_lv, a_s, b_lv, b_s, rung = _small_problem(rng, 1, 2, 2, 8)
    with pytest.raises(orc.OracleError) as e:
        orc.matmul(a_lv, a_s, b_lv, b_s, rung, [64], band_scales=True)
    assert e.value.code == orc.ERR_ARG


# ------------------------------------------------- fraction-based fixed MP --
# ["scmp_vit" README, MP flags: levels get a given fraction of the rows (or
# heads), the longest level the largest statistic]

def test_assign_fraction_hand_example(orc):
    # order by statistic: row 4 (5), row 0 (3), row 2 (2), row 3 (2, tie -> after
    # row 2), row 1 (1), row 5 (0).  Rung 2 takes floor(6 * 0.2 + 1/2) = 1 row,
    # rungs >= 1 take floor(6 * 0.5 + 1/2) = 3 rows.
    stat = np.array([3.0, 1.0, 2.0, 2.0, 5.0, 0.0], np.float32)
    rung = orc.assign_fraction(stat, [0.5, 0.3, 0.2])
    assert rung.tolist() == [1, 0, 1, 0, 2, 0]


def test_assign_fraction_per_head_hand_example(orc):
    # 4 heads of 3 rows, ranked in sets of 2 by their max statistic
    stat = np.array([[1, 4, 2], [7, 0, 0], [3, 3, 1], [2, 3, 0]], np.float32)
    rung = orc.assign_fraction(stat, [0.5, 0.5], set_size=2)
    # set 0: head 1 (7) above head 0 (4); set 1: equal maxima, head 2 first
    assert rung.tolist() == [[0, 0, 0], [1, 1, 1], [1, 1, 1], [0, 0, 0]]


def test_assign_fraction_nan_as_minus_inf_and_one_rung(orc):
    # NaN counts as -inf: order row 3 (2), row 1 (1), row 0 (NaN, tie with
    # row 2's -inf, lower index first), row 2.  Rung 2 takes floor(4 * 0.5 +
    # 1/2) = 2 rows, rungs >= 1 floor(4 * 0.75 + 1/2) = 3.
    stat = np.array([np.nan, 1.0, -np.inf, 2.0], np.float32)
    assert orc.assign_fraction(stat, [0.25, 0.25, 0.5]).tolist() == [1, 2, 0, 2]
    assert orc.assign_fraction(stat, [1.0]).tolist() == [0, 0, 0, 0]


def test_assign_fraction_counts_and_monotone(orc):
    rng = np.random.default_rng(40)
    for n, fr in [(16, [1 / 3, 1 / 3, 1 / 3]), (257, [0.05, 0.225, 0.575, 0.15]),
                  (1000, [0.1, 0.2, 0.3, 0.4]), (7, [0.0, 1.0, 0.0])]:
        stat = rng.integers(0, 20, n).astype(np.float32)   # many ties
        rung = orc.assign_fraction(stat, fr)
        for k in range(1, len(fr)):
            want = int(np.floor(n * sum(fr[k:]) + 0.5))
            assert int((rung >= k).sum()) == want
        # a larger statistic never has a shorter length; among equal statistics
        # the lower index never has a shorter length
        for i in range(n):
            for j in range(n):
                if stat[i] > stat[j] or (stat[i] == stat[j] and i < j):
                    assert rung[i] >= rung[j]


def test_assign_fraction_rejects_bad_fractions(orc):
    stat = np.ones((2, 4), np.float32)
    for fr, ss in [([0.5, 0.4], 0), ([1.2, -0.2], 0), ([0.5, 0.5], 3)]:
        with pytest.raises(orc.OracleError):
            orc.assign_fraction(stat, fr, set_size=ss)


# ------------------------------------------------------ unipolar AND mode --
# ["scmp_vit" README, the comp matmul's unipolar quant mode; "Precision As You
# Need", the unipolar AND gate]: sign-magnitude streams of magnitude level
# 2|x|, one enable-gated counter on B advanced at A's ones.

def test_and_count_hand_values(orc):
    # x_a = 32: magnitude level 64, a full period (L = 256) holds exactly 64
    # ones, so B emits its first 64 bits: C[100][64] = ceil(100 / 4) = 25 for
    # x_b = 50 (magnitude level 100), by the prefix-count closed form.
    assert orc.and_count(128 + 32, 128 + 50, 256) == 25
    assert orc.and_count(128 - 32, 128 + 50, 256) == -25
    assert orc.and_count(128 - 32, 128 - 50, 256) == 25
    assert orc.and_count(128, 128 + 50, 256) == 0          # x_a = 0: no ones
    assert orc.and_count(128 + 32, 128, 256) == 0          # x_b = 0
    assert orc.and_count(128 + 32, 128 + 50, 0) == 0


def test_and_count_equals_prefix_count_closed_form(orc):
    # count = sign * C[2|x_b|][C[2|x_a|][L]]: B's first n bits, n = A's ones
    K = orc.indicator(P).astype(np.int64)
    C = _prefix_counts(K)
    rng = np.random.default_rng(41)
    for _ in range(3000):
        a, b = (int(v) for v in rng.integers(1, Q, 2))
        L = int(rng.choice([1, 7, 64, 96, 128, 192, 255, 256]))
        xa, xb = a - Q // 2, b - Q // 2
        want = int(np.sign(xa) * np.sign(xb)) * int(C[2 * abs(xb), C[2 * abs(xa), L]])
        assert orc.and_count(a, b, L) == want, (a, b, L)


def test_unipolar_matmul_decode_by_hand(orc):
    from fractions import Fraction
    rng = np.random.default_rng(42)
    a_lv, a_s, b_lv, b_s, rung = _small_problem(rng, 1, 3, 4, 9)
    ladder = np.array([64, 96, 128, 192, 256], np.int32)
    counts, out, steps = orc.matmul(a_lv, a_s, b_lv, b_s, rung, ladder, unipolar=True)
    for i in range(3):
        L = int(ladder[rung[0, i]])
        for j in range(4):
            c = sum(orc.and_count(int(a_lv[0, i, d]), int(b_lv[0, j, d]), L) for d in range(9))
            assert counts[0, i, j, 0] == c
            want = (Fraction(float(a_s[0, i])) * Fraction(float(b_s[0, j])) * 128 * 128
                    * Fraction(c, L))
            assert out[0, i, j] == np.float32(float(want))


def test_unipolar_estimates_the_product(orc):
    # statistical sanity (not parity): at L = 256 the signed AND estimate
    # tracks sum_d x_a x_b of the quantised values
    rng = np.random.default_rng(43)
    xa = rng.integers(-127, 128, (1, 16, 64))
    xb = rng.integers(-127, 128, (1, 16, 64))
    a_lv, b_lv = (xa + 128).astype(np.uint8), (xb + 128).astype(np.uint8)
    one = np.full((1, 16), 1.0 / 128, np.float32)
    rung = np.zeros((1, 16), np.int32)
    _, out, _ = orc.matmul(a_lv, one, b_lv, one, rung, [256], unipolar=True)
    exact = np.einsum("gid,gjd->gij", xa, xb).astype(np.float64) / 128 ** 2  # scales 1/128
    err = np.linalg.norm(out - exact) / np.linalg.norm(exact)
    assert err < 0.05, err


# --------------------------------------------- Sobol seed-bank variants --
# ["scmp_vit" README, Sobol-seed bank: default, antithetic, alternative seeds
# on the K side]: digital shift of the integer points and the antithetic 1 - u
# for the second operand's sequence.

def test_sobol_variant_hand_values(orc):
    r = orc.sobol_r(P)
    assert orc.sobol_r_variant(0, False).tolist() == r.tolist()
    # l = 0, 1, 2: u = 0, 128, 64
    assert orc.sobol_r_variant(5, False)[:3].tolist() == [5 + 1, (128 ^ 5) + 1, (64 ^ 5) + 1]
    assert orc.sobol_r_variant(0, True)[:3].tolist() == [256, 128, 192]
    assert orc.sobol_r_variant(5, True)[:3].tolist() == [256 - 5, 256 - (128 ^ 5), 256 - (64 ^ 5)]


def test_sobol_variants_keep_the_full_period(orc):
    for s, anti in [(0, True), (1, False), (77, True), (255, False)]:
        r = orc.sobol_r_variant(s, anti)
        assert sorted(r.tolist()) == list(range(1, Q + 1))
        K = orc.indicator_variant(s, anti)
        assert np.array_equal(K.sum(axis=1), np.arange(Q + 1))


def test_antithetic_indicator_is_the_complement(orc):
    # 1[Q - u <= b] = 1 - 1[u + 1 <= Q - b]: K'[b] = 1 - K[Q - b]
    K = orc.indicator(P).astype(int)
    Ka = orc.indicator_variant(0, True).astype(int)
    assert np.array_equal(Ka, 1 - K[::-1])


def test_matmul_with_b_variant_matches_two_table_closed_form(orc):
    # count = C_B[b][n] + (L - n) - C_B[b][L - n], n = C_A[a][L]
    rng = np.random.default_rng(44)
    CA = _prefix_counts(orc.indicator(P).astype(np.int64))
    for s, anti in [(0, True), (91, False), (200, True)]:
        CB = _prefix_counts(orc.indicator_variant(s, anti).astype(np.int64))
        a_lv, a_s, b_lv, b_s, rung = _small_problem(rng, 1, 4, 3, 11)
        ladder = np.array([64, 96, 128, 192, 256], np.int32)
        counts, _, _ = orc.matmul(a_lv, a_s, b_lv, b_s, rung, ladder, b_shift=s, b_antithetic=anti)
        for i in range(4):
            L = int(ladder[rung[0, i]])
            for j in range(3):
                want = 0
                for d in range(11):
                    n = int(CA[a_lv[0, i, d], L])
                    b = int(b_lv[0, j, d])
                    want += int(CB[b, n]) + (L - n) - int(CB[b, L - n])
                assert counts[0, i, j, 0] == want
    c0, o0, _ = orc.matmul(a_lv, a_s, b_lv, b_s, rung, ladder)
    c1, o1, _ = orc.matmul(a_lv, a_s, b_lv, b_s, rung, ladder, b_shift=0, b_antithetic=False)
    assert np.array_equal(c0, c1) and np.array_equal(o0, o1)


# ------------------------------------------- Gray order and Sobol pools --

def test_gray_order_hand_values(orc):
    """First dimension in Gray-code order: point l is the XOR of the direction
    numbers 2^(8-k) over the bits k-1 of g = l ^ (l >> 1):
    g = 0, 1, 3, 2, 6, 7, 5, 4 -> u = 0, 128, 192, 64, 96, 224, 160, 32."""
    r = orc.sobol_r_gray(P)
    assert list(r[:8] - 1) == [0, 128, 192, 64, 96, 224, 160, 32]
    # point l + 1 differs from point l by one direction number: the one of the
    # lowest zero bit of l
    u = r - 1
    for l in range(255):
        k = (~l & (l + 1)).bit_length()          # 1-based position of l's lowest zero bit
        assert u[l] ^ u[l + 1] == 1 << (P - k)


def test_gray_order_keeps_dyadic_prefixes_and_the_full_period(orc):
    """The first 2^k points of either order are the same set (the Gray code
    permutes each block of 2^k indices), so prefix counts agree at every
    power-of-two length and the full-period invariant holds; at L = 96 and 192
    the two orders differ."""
    Cn = _prefix_counts(orc.indicator(P).astype(np.int64))
    Kg = orc.indicator_points(orc.sobol_r_gray(P) - 1)
    Cg = _prefix_counts(Kg.astype(np.int64))
    for k in range(P + 1):
        assert np.array_equal(Cn[:, 1 << k], Cg[:, 1 << k])
    assert np.array_equal(Cg[:, 256], np.arange(257))
    assert not np.array_equal(Cn[:, 96], Cg[:, 96])
    assert not np.array_equal(Cn[:, 192], Cg[:, 192])


def test_indicator_points_rejects_a_non_permutation(orc):
    u = np.arange(256, dtype=np.int32)
    u[7] = u[8]
    with pytest.raises(orc.OracleError) as e:
        orc.indicator_points(u)
    assert e.value.code == orc.ERR_TABLE


def test_pool_generator_is_sobol_in_gray_order():
    """The seeded pool generator (inputs, not SC arithmetic): every sequence
    is a permutation of the period, dimension 1 is the first Sobol dimension
    in Gray-code order, and dimension 2 follows the direction numbers of the
    polynomial x + 1 (v_k = v_{k-1} XOR v_{k-1} / 2, v_1 = 1/2)."""
    import oracle
    from mixed_precision_vit_b200.workloads import sobol_pool
    u = sobol_pool(64, P)
    assert all(sorted(row) == list(range(256)) for row in u)
    assert np.array_equal(u[0], oracle.sobol_r_gray(P) - 1)
    V = [0] * (P + 1)
    V[1] = 1 << (P - 1)
    for k in range(2, P + 1):
        V[k] = V[k - 1] ^ (V[k - 1] >> 1)
    want = []
    for l in range(256):
        g, x = l ^ (l >> 1), 0
        for k in range(1, P + 1):
            if (g >> (k - 1)) & 1:
                x ^= V[k]
        want.append(x)
    assert list(u[1]) == want
    assert len({tuple(r) for r in u}) == 64


def _closed_form_T_of(C, L):
    """Two-counter closed form with one sequence's prefix counts C."""
    n = C[:, L]
    a = np.arange(C.shape[0])
    return C[:, n].T + (L - n)[:, None] - C[:, L - n].T


def test_pool_counts_follow_each_index_sequence(orc):
    """With a pool, index d streams both operands from sequence d mod P: the
    bit-by-bit counts equal the sum over d of the two-counter closed form of
    that index's own prefix counts."""
    from mixed_precision_vit_b200.workloads import sobol_pool
    rng = np.random.default_rng(31)
    ladder = np.array([64, 96, 128, 192, 256], np.int32)
    a_lv, a_s, b_lv, b_s, rung = _small_problem(rng, 1, 6, 5, 11)
    pool = sobol_pool(4, P)
    counts, _, steps = orc.matmul(a_lv, a_s, b_lv, b_s, rung, ladder, pool=pool)
    Cs = [_prefix_counts(orc.indicator_points(pool[q]).astype(np.int64)) for q in range(4)]
    for i in range(6):
        L = int(ladder[rung[0, i]])
        want = np.zeros(5, np.int64)
        for d in range(11):
            T = _closed_form_T_of(Cs[d % 4], L)
            want += T[a_lv[0, i, d], b_lv[0, :, d]]
        assert np.array_equal(counts[0, i, :, 0], want)
    assert steps == int(ladder[rung].sum()) * 5 * 11


def test_pool_of_one_sequence_reduces_to_a_single_table(orc):
    """A pool whose every row is the natural-order sequence gives the default
    result; one whose every row is the Gray-order sequence gives gray=True."""
    rng = np.random.default_rng(32)
    ladder = np.array([64, 96, 128, 192, 256], np.int32)
    a_lv, a_s, b_lv, b_s, rung = _small_problem(rng, 2, 5, 4, 9)
    nat = np.tile(orc.sobol_r(P) - 1, (3, 1))
    gry = np.tile(orc.sobol_r_gray(P) - 1, (2, 1))
    c0, o0, _ = orc.matmul(a_lv, a_s, b_lv, b_s, rung, ladder)
    c1, o1, _ = orc.matmul(a_lv, a_s, b_lv, b_s, rung, ladder, pool=nat)
    assert np.array_equal(c0, c1) and np.array_equal(o0, o1)
    c2, o2, _ = orc.matmul(a_lv, a_s, b_lv, b_s, rung, ladder, gray=True)
    c3, o3, _ = orc.matmul(a_lv, a_s, b_lv, b_s, rung, ladder, pool=gry)
    assert np.array_equal(c2, c3) and np.array_equal(o2, o3)
    assert not np.array_equal(c0, c2)                   # the orders differ at 96 and 192
    with pytest.raises(orc.OracleError):
        orc.matmul(a_lv, a_s, b_lv, b_s, rung, ladder, pool=nat, gray=True)


def test_pool_full_period_invariant_per_sequence(orc):
    """Every sequence of a pool keeps the full-period invariant: a full period
    of K_s[b, .] holds exactly b ones, so a full-length stream reproduces its
    level; at L = 2^p the A operand's count of ones n = C_s[a][2^p] = a."""
    from mixed_precision_vit_b200.workloads import sobol_pool
    pool = sobol_pool(64, P)
    for q in range(64):
        K = orc.indicator_points(pool[q])
        assert np.array_equal(K.sum(axis=1), np.arange(257))
    # the unipolar count at full length is sign * C_s[2|x_b|][C_s[2|x_a|][256]]
    # = sign * C_s[2|x_b|][2|x_a|]: levels a = b = 255 (x = 127, magnitude
    # level 254) on one contraction index, which streams from sequence 0
    a_lv = np.array([[[255]]], np.uint8)
    b_lv = np.array([[[255]]], np.uint8)
    c, _, _ = orc.matmul(a_lv, np.ones((1, 1), np.float32), b_lv, np.ones((1, 1), np.float32),
                         np.zeros((1, 1), np.int32), [256], pool=pool, unipolar=True)
    C0 = _prefix_counts(orc.indicator_points(pool[0]).astype(np.int64))
    assert c[0, 0, 0, 0] == C0[254, 254]


def test_estimator_sanity_on_gaussian_inputs(orc):
    # Not parity: at L = 256 the SC product of Gaussian matrices has about the
    # norm of the exact product ("Why it works": ~1.005x on Gaussian inputs),
    # and the error shrinks as L grows.
    rng = np.random.default_rng(9)
    A = rng.standard_normal((24, 64)).astype(np.float32)
    B = rng.standard_normal((64, 20)).astype(np.float32)
    a_lv, a_s = orc.quantize(A, axis=0)
    b_lv, b_s = orc.quantize(B, axis=1)
    exact = A.astype(np.float64) @ B.astype(np.float64)
    errs = []
    for L in (64, 128, 256):
        _, out, _ = orc.matmul(a_lv, a_s, b_lv, b_s, np.zeros(24, np.int32), [L])
        errs.append(np.linalg.norm(out[0] - exact) / np.linalg.norm(exact))
        if L == 256:
            ratio = np.linalg.norm(out[0]) / np.linalg.norm(exact)
            assert 0.95 < ratio < 1.1
    assert errs[0] > errs[1] > errs[2]


# ------------------------------------------------------------------- tilt --

def _best_apportionment(raw, target):
    """Exhaustive: among vectors with each entry floor or ceil of raw and the
    given sum, the one closest to raw in squared distance (ties: earlier
    bands take the extra unit first)."""
    n = len(raw)
    fl = [math.floor(r) for r in raw]
    need = target - sum(fl)
    best, best_key = None, None
    for mask in range(1 << n):
        if bin(mask).count("1") != need:
            continue
        v = [fl[b] + ((mask >> b) & 1) for b in range(n)]
        key = (round(sum((v[b] - raw[b]) ** 2 for b in range(n)), 9),
               [-((mask >> b) & 1) for b in range(n)])
        if best_key is None or key < best_key:
            best, best_key = v, key
    return best


def test_tilt_identity_parent_and_exhaustive_rounding(orc):
    ladder = [64, 96, 128, 192, 256]
    assert np.all(orc.kband_tilt(ladder, 16, 0.0, 256) == np.array(ladder))
    for n_bands, tilt in [(4, 0.25), (5, -0.3), (7, 0.1), (10, 0.45), (2, 0.2)]:
        bl = orc.kband_tilt(ladder, n_bands, tilt, 256)
        for k, Lk in enumerate(ladder):
            assert bl[:, k].sum() == n_bands * Lk              # never overspent
            pos = [(2 * b - (n_bands - 1)) / (n_bands - 1) for b in range(n_bands)]
            raw = [Lk * (1 + tilt * p) for p in pos]
            if max(raw) > 256:
                assert np.all(bl[:, k] == Lk)                  # rung cannot be tilted
            else:
                assert list(bl[:, k]) == _best_apportionment(raw, n_bands * Lk)


def test_tilt_sixteen_bands_shape(orc):
    bl = orc.kband_tilt([64, 96, 128, 192, 256], 16, 0.25, 256)
    assert np.all(bl[:, 4] == 256)                              # top rung at the ceiling
    for k in range(4):
        assert np.all(np.diff(bl[:, k]) >= 0)                   # later bands longer
        assert bl[0, k] < bl[-1, k]
    assert bl.max() <= 256 and bl.min() >= 1


def test_tilt_rejects_ladder_above_ceiling(orc):
    with pytest.raises(orc.OracleError) as e:
        orc.kband_tilt([64, 300], 4, 0.0, 256)
    assert e.value.code == orc.ERR_TABLE
