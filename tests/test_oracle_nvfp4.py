"""Pins of the oracle's NVFP4 quantisation (e2m1 elements, e4m3 block scales
of 16, a float32 scale per row): the e2m1 grid and its ties from an
independent nearest-value search, exact reconstruction of rows built on the
grid, the error bound the two roundings allow, zero rows and blocks, and the
block-scaled dot product against the product of the dequantised rows."""
import numpy as np
import pytest

from oracle import dlm_oracle as O

# e2m1 magnitudes in order, with their mantissa bit
GRID = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
MANT = [0, 1, 0, 1, 0, 1, 0, 1]


def nearest_e2m1(x: float) -> float:
    """Nearest grid magnitude by search; a tie goes to the value whose
    mantissa bit is 0; beyond 6 the value saturates."""
    a = abs(x)
    if a >= 6.0:
        r = 6.0
    else:
        d = [abs(a - g) for g in GRID]
        best = min(d)
        cands = [i for i, di in enumerate(d) if di == best]
        i = cands[0] if len(cands) == 1 else [c for c in cands if MANT[c] == 0][0]
        r = GRID[i]
    return -r if x < 0 else r


def test_e2m1_grid_values_are_fixed_points():
    g = np.array(GRID + [-v for v in GRID[1:]])
    assert np.array_equal(O.round_to_e2m1(g), g)


def test_e2m1_midpoints_tie_to_even_mantissa():
    for lo, hi, mlo in zip(GRID[:-1], GRID[1:], MANT[:-1]):
        mid = (lo + hi) / 2
        want = lo if mlo == 0 else hi
        assert O.round_to_e2m1(mid) == want, (lo, hi)
        assert O.round_to_e2m1(-mid) == -want


def test_e2m1_matches_nearest_search_and_saturates():
    xs = np.linspace(-9.0, 9.0, 36001)
    got = O.round_to_e2m1(xs)
    want = np.array([nearest_e2m1(float(x)) for x in xs])
    assert np.array_equal(got, want)
    assert O.round_to_e2m1(1e6) == 6.0 and O.round_to_e2m1(-7.0) == -6.0


def test_on_grid_rows_reconstruct_exactly():
    rng = np.random.default_rng(3)
    rows, cols = 6, 128
    nb = cols // O.NVFP4_BLOCK
    grid = np.array(GRID + [-v for v in GRID[1:]])
    q = rng.choice(grid, size=(rows, cols))
    qb = q.reshape(rows, nb, O.NVFP4_BLOCK)
    qb[:, :, 0] = 6.0                      # every block reaches the e2m1 maximum
    e4m3 = np.unique(np.abs(O.round_to_e4m3(np.linspace(0.02, 448.0, 4001))))
    sb = rng.choice(e4m3[e4m3 >= 2.0 ** -6], size=(rows, nb))
    sb[:, 0] = 448.0                       # the row's largest block scale
    sr = np.ldexp(1.0, rng.integers(-14, -6, size=rows))   # powers of two: exact products
    x = (q * np.repeat(sb, O.NVFP4_BLOCK, axis=1) * sr[:, None]).astype(np.float32)
    assert np.array_equal(x.astype(np.float64), q * np.repeat(sb, O.NVFP4_BLOCK, axis=1)
                          * sr[:, None])   # the construction itself is exact in float32
    q2, sb2, sr2 = O.quantize_rows_nvfp4(x)
    assert np.array_equal(sr2, sr.astype(np.float32))
    assert np.array_equal(sb2, sb)
    assert np.array_equal(q2, q)
    assert np.array_equal(O.dequantize_rows_nvfp4(q2, sb2, sr2), x.astype(np.float64))


def test_error_within_the_rounding_bound():
    """With s = sb*sr and sb the e4m3 rounding of amax_b/(6 sr) (relative
    error <= 2^-4 for normal scales), x/s lies within 6/(1 - 2^-4) and the
    e2m1 rounding moves it by at most 1 (half the spacing of [4, 6], or the
    saturation beyond 6): |x - q s| <= s <= (1 + 2^-4) amax_b / 6."""
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((64, 256)) * rng.uniform(0.1, 10.0, size=(64, 1))).astype(np.float32)
    q, sb, sr = O.quantize_rows_nvfp4(x)
    assert np.array_equal(O.round_to_e4m3(sb), sb)        # block scales on the e4m3 grid
    assert np.array_equal(O.round_to_e2m1(q), q)          # elements on the e2m1 grid
    err = np.abs(O.dequantize_rows_nvfp4(q, sb, sr) - x.astype(np.float64))
    amax_b = np.abs(x.astype(np.float64)).reshape(64, -1, O.NVFP4_BLOCK).max(axis=2)
    bound = (1.0 + 2.0 ** -4) * amax_b / 6.0 * (1.0 + 1e-6)
    assert (err.reshape(64, -1, O.NVFP4_BLOCK) <= bound[:, :, None]).all()
    # and the quantisation is not trivially coarse: most elements move by
    # less than an eighth of their block's maximum
    assert np.mean(err.reshape(64, -1, O.NVFP4_BLOCK) < amax_b[:, :, None] / 8) > 0.9


def test_zero_rows_and_blocks():
    x = np.zeros((3, 32), np.float32)
    x[1, 16:] = np.linspace(-1, 1, 16)
    q, sb, sr = O.quantize_rows_nvfp4(x)
    assert sr[0] == 1.0 and not sb[0].any() and not q[0].any()
    assert sb[1, 0] == 0.0 and not q[1, :16].any() and sb[1, 1] == 448.0
    assert np.abs(q[1, 16:]).max() == 6.0


def test_block_scaled_dot_equals_the_dequantised_product():
    rng = np.random.default_rng(7)
    a = rng.standard_normal((5, 64)).astype(np.float32)
    b = rng.standard_normal((9, 64)).astype(np.float32)
    qa, sba, sra = O.quantize_rows_nvfp4(a)
    qb, sbb, srb = O.quantize_rows_nvfp4(b)
    got = O.nvfp4_dot(qa, sba, sra, qb, sbb, srb)
    want = O.dequantize_rows_nvfp4(qa, sba, sra) @ O.dequantize_rows_nvfp4(qb, sbb, srb).T
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12)


def test_columns_must_fill_blocks():
    with pytest.raises(ValueError):
        O.quantize_rows_nvfp4(np.ones((2, 24), np.float32))


def test_blocked_quantisation_equals_whole_matrix():
    """Rows are independent: quantising in row blocks gives the same codes,
    block scales and row scales as one call over the whole matrix."""
    r = np.random.default_rng(21)
    x = r.standard_normal((37, 96)).astype(np.float32) * 0.02
    q, sb, sr = O.quantize_rows_nvfp4(x)
    qb, sbb, srb = O.quantize_rows_nvfp4_blocked(x, rows_per_block=8)
    assert np.array_equal(qb, q) and np.array_equal(sbb, sb) and np.array_equal(srb, sr)


def test_head_logits_equal_dequantised_product_with_f32_row_factor():
    """The NVFP4 head's logits: the block-scaled sums times the two row
    scales' product rounded to float32 -- equal to the product of the rows
    dequantised without their row scales, times that factor."""
    r = np.random.default_rng(22)
    a = r.standard_normal((5, 64)).astype(np.float32)
    b = r.standard_normal((33, 64)).astype(np.float32) * 0.02
    qa, sba, sra = O.quantize_rows_nvfp4(a)
    qb, sbb, srb = O.quantize_rows_nvfp4(b)
    got = O.nvfp4_head_logits(qa, sba, sra, qb, sbb, srb, rows_per_block=7)
    da = O.dequantize_rows_nvfp4(qa, sba, np.ones(5))
    db = O.dequantize_rows_nvfp4(qb, sbb, np.ones(33))
    f = (sra[:, None] * srb[None, :]).astype(np.float32).astype(np.float64)
    want = (da @ db.T) * f
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12)
    # and it stays within float32 rounding of the f64 row-scale product
    assert np.allclose(got, O.nvfp4_dot(qa, sba, sra, qb, sbb, srb), rtol=2 ** -23)
