"""Pins for the oracle's NF4 codebook, quantiser and dequantiser (CPU only).

Each check ties the oracle to something other than itself: the normal CDF
evaluated through math.erf with bisection (not the inverse CDF the oracle
calls), scipy's ndtri, brute-force nearest-level search, exact round trips
and the error bound of a nearest-level quantiser.
"""

import math

import numpy as np
import pytest

from oracle import nf4

C = nf4.codebook()


def _phi(x):
    return 0.5 * (1.0 + math.erf(x / math.sqrt(2.0)))


def _quantile_by_bisection(p):
    lo, hi = -10.0, 10.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if _phi(mid) < p:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def test_codebook_shape_and_exact_points():
    assert C.dtype == np.float32 and C.shape == (16,)
    assert np.all(np.diff(C) > 0), "levels strictly increasing"
    assert C[0] == np.float32(-1.0) and C[15] == np.float32(1.0) and C[7] == np.float32(0.0)
    assert np.sum(C < 0) == 7 and np.sum(C > 0) == 8


def test_codebook_is_normal_quantiles_by_cdf_bisection():
    # Rebuild the levels from the forward CDF (bisection on erf), not inv_cdf.
    d = nf4.DELTA
    top = _quantile_by_bisection(d)
    pos = [_quantile_by_bisection(d + i * (0.5 - d) / 8) / top for i in range(8)]
    neg = [-_quantile_by_bisection(d + i * (0.5 - d) / 7) / top for i in range(7)]
    ref = np.array(sorted(pos + neg + [0.0]), np.float32)
    assert np.array_equal(ref.view(np.uint32), C.view(np.uint32))


def test_codebook_matches_scipy_ndtri():
    from scipy.special import ndtri
    d = nf4.DELTA
    top = ndtri(d)
    pos = ndtri(d + np.arange(8) * (0.5 - d) / 8) / top
    neg = -ndtri(d + np.arange(7) * (0.5 - d) / 7) / top
    ref = np.sort(np.concatenate([pos, neg, [0.0]])).astype(np.float32)
    assert np.array_equal(ref.view(np.uint32), C.view(np.uint32))


def test_codebook_golden_fixture():
    # tests/golden/nf4_codebook.txt is written by tests/golden/make_golden.py,
    # which calls only the oracle; this catches accidental changes to it.
    path = __file__.replace("test_oracle_nf4.py", "golden/nf4_codebook.txt")
    rows = [ln.split() for ln in open(path) if ln.strip() and not ln.startswith("#")]
    bits = np.array([int(r[1], 16) for r in rows], np.uint32)
    assert np.array_equal(bits, C.view(np.uint32))


def test_midpoints_between_levels():
    m = nf4.midpoints()
    assert m.shape == (15,)
    assert np.all(C[:-1] < m) and np.all(m < C[1:])
    assert np.all(np.abs(m.astype(np.float64) - (C[:-1].astype(np.float64) + C[1:]) / 2) <= 6e-8)


def _brute_codes(W, block=64):
    blocks = W.reshape(-1, block).astype(np.float32)
    am = np.max(np.abs(blocks), axis=1)
    out = np.full(blocks.shape, 7, np.uint8)
    near_tie = np.zeros(blocks.shape, bool)
    m = nf4.midpoints().astype(np.float64)
    for b in range(blocks.shape[0]):
        if am[b] == 0:
            continue
        v = (blocks[b] / am[b]).astype(np.float32).astype(np.float64)
        dist = np.abs(v[:, None] - C.astype(np.float64)[None, :])
        out[b] = np.argmin(dist, axis=1)      # argmin takes the lower index on ties
        near_tie[b] = np.min(np.abs(v[:, None] - m[None, :]), axis=1) < 1.2e-7
    return out.reshape(-1), near_tie.reshape(-1)


def test_quantize_matches_brute_force_nearest_level():
    g = np.random.default_rng(11)
    W = (g.standard_normal((96, 320)) * 0.02).astype(np.float32)
    W[5, 64:128] = 0.0                        # one all-zero block
    codes, absmax = nf4.quantize(W)
    got = nf4.unpack(codes, W.size)
    ref, near = _brute_codes(W)
    assert np.array_equal(got[~near], ref[~near])
    assert np.all(np.abs(got[near].astype(int) - ref[near].astype(int)) <= 1)
    assert np.array_equal(absmax, np.max(np.abs(W.reshape(-1, 64)), axis=1))


def test_absmax_element_maps_to_an_end_code():
    g = np.random.default_rng(12)
    W = (g.standard_normal((16, 256)) * 0.02).astype(np.float32)
    codes, absmax = nf4.quantize(W)
    flat = nf4.unpack(codes, W.size).reshape(-1, 64)
    blocks = W.reshape(-1, 64)
    for b in range(blocks.shape[0]):
        j = int(np.argmax(np.abs(blocks[b])))
        assert flat[b, j] == (15 if blocks[b, j] > 0 else 0)


def test_codebook_round_trip_and_packing_order():
    # A block holding 1.0 (sets absmax = 1) and every level exactly: code i for c_i.
    row = np.concatenate([C, C, C, C]).astype(np.float32)         # 64 values, absmax 1
    W = np.stack([row, row * np.float32(0.25)])                     # power-of-two scale is exact
    codes, absmax = nf4.quantize(W)
    assert np.array_equal(absmax, np.array([1.0, 0.25], np.float32))
    expect = np.tile(np.arange(16, dtype=np.uint8), 8)
    assert np.array_equal(nf4.unpack(codes, W.size), expect)
    # high nibble = even element: (0,1) -> 0x01, (2,3) -> 0x23, ...
    assert codes[0] == 0x01 and codes[1] == 0x23 and codes[7] == 0xEF
    back = nf4.dequantize(codes, absmax, 2, 64)
    assert np.array_equal(back, W)


def test_midpoint_ties_go_to_the_lower_code():
    m = nf4.midpoints()
    row = np.zeros(64, np.float32)
    row[0] = 1.0
    row[1:16] = m
    row[16:31] = np.nextafter(m, np.float32(np.inf))
    codes, _ = nf4.quantize(row[None, :])
    got = nf4.unpack(codes, 64)
    assert np.array_equal(got[1:16], np.arange(15))
    assert np.array_equal(got[16:31], np.arange(1, 16))


def test_zero_block_and_nonfinite_rejected():
    W = np.zeros((2, 64), np.float32)
    codes, absmax = nf4.quantize(W)
    assert np.all(absmax == 0) and np.all(codes == 0x77)
    assert np.all(nf4.dequantize(codes, absmax, 2, 64) == 0)
    W[0, 3] = np.nan
    with pytest.raises(AssertionError):
        nf4.quantize(W)


def test_dequantize_is_level_times_absmax_and_error_bound():
    g = np.random.default_rng(13)
    W = (g.standard_normal((64, 192)) * 0.02).astype(np.float32)
    codes, absmax = nf4.quantize(W)
    Wt = nf4.dequantize(codes, absmax, 64, 192)
    idx = nf4.unpack(codes, W.size).reshape(-1, 64)
    assert np.array_equal(Wt.reshape(-1, 64), (C[idx] * absmax[:, None]).astype(np.float32))
    gap = float(np.max(np.diff(C.astype(np.float64)))) / 2
    err = np.abs(W.reshape(-1, 64).astype(np.float64) - Wt.reshape(-1, 64))
    assert np.all(err <= absmax[:, None] * (gap + 1e-6))


# ----------------------------------------------------------------- absmax, 8 bit


def test_absmax8_exact_on_its_own_grid():
    # a run whose values are j * 2^-10 (max 255 * 2^-10): s = 2^-10 exactly, q = j
    j = np.array(list(range(256)), dtype=np.float32)
    a = (j * np.float32(2.0 ** -10)).astype(np.float32)
    q, s = nf4.quantize_absmax8(a)
    assert s.tolist() == [2.0 ** -10]
    assert np.array_equal(q, j.astype(np.uint8))
    assert np.array_equal(nf4.dequantize_absmax8(q, s), a)


def test_absmax8_nearest_step_and_bound():
    rng = np.random.default_rng(5)
    a = np.abs(rng.normal(0.0, 0.06, 256 * 7 + 100)).astype(np.float32)   # ragged last run
    q, s = nf4.quantize_absmax8(a)
    assert s.size == 8 and q.dtype == np.uint8
    idx = np.arange(a.size) // 256
    for g in range(8):
        run = a[idx == g]
        assert q[idx == g][np.argmax(run)] == 255, "each run's max takes the top code"
        # s is max/255 to within half an fp32 ulp
        assert abs(float(s[g]) - float(run.max()) / 255.0) <= 2.0 ** -24 * float(s[g])
    # q is the nearest integer to a / s (checked in fp64), so |a~ - a| <= s/2 (+ rounding)
    sd = s[idx].astype(np.float64)
    ratio = a.astype(np.float64) / sd
    assert np.all(np.abs(q - ratio) <= 0.5 + 1e-5)
    back = nf4.dequantize_absmax8(q, s).astype(np.float64)
    assert np.all(np.abs(back - a) <= 0.5 * sd * (1 + 1e-5) + 2.0 ** -23 * a)
    # order is kept inside a run
    for g in range(8):
        m = idx == g
        o = np.argsort(a[m], kind="stable")
        assert np.all(np.diff(q[m][o].astype(int)) >= 0)


def test_absmax8_zero_run_and_tie_to_even():
    a = np.zeros(300, dtype=np.float32)
    a[256:] = np.float32(2.0 ** -10) * np.float32(255.0)
    a[257] = np.float32(2.5 * 2.0 ** -10)    # exactly q = 2.5 -> even 2
    a[258] = np.float32(3.5 * 2.0 ** -10)    # exactly q = 3.5 -> even 4
    q, s = nf4.quantize_absmax8(a)
    assert s[0] == 0 and np.all(q[:256] == 0)
    assert np.all(nf4.dequantize_absmax8(q, s)[:256] == 0)
    assert s[1] == np.float32(2.0 ** -10) and q[257] == 2 and q[258] == 4


def test_dequantize_dq_is_codes_times_rounded_absmax():
    rng = np.random.default_rng(6)
    N, K = 8, 256 * 4
    W = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    codes, am = nf4.quantize(W)
    q, s = nf4.quantize_absmax8(am)
    got = nf4.dequantize_dq(codes, q, s, N, K)
    a2 = nf4.dequantize_absmax8(q, s)
    # brute force per element: level[code] * a~ of its block
    idx = nf4.unpack(codes, N * K)
    want = np.array([np.float32(C[idx[i]] * a2[i // 64]) for i in range(N * K)], np.float32)
    assert np.array_equal(got.reshape(-1), want)
    # and the double-quantised weight stays within half an absmax step of the fp32 one
    ref = nf4.dequantize(codes, am, N, K)
    step = np.repeat(s[np.arange(am.size) // 256], 64).reshape(N, K)
    assert np.all(np.abs(got - ref) <= 0.5 * step * (1 + 1e-5) + 2.0 ** -22 * np.abs(ref))
