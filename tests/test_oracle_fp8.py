"""Pins of the oracle's e4m3 LM head (NLD tutorial section 8.6, FP8 weight
quantisation; course section 15, low-bit weights on Blackwell).  CPU only.

The rounding is written from the format's definition; here it is held
against torch's float8_e4m3fn cast (an independent implementation), against
the format's own grid, and the quantised head against the exact logits in
the special case where quantisation loses nothing."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from oracle import dlm_oracle as O


def _grid():
    """Every finite non-negative e4m3 value, from the bit patterns."""
    vals = []
    for e in range(16):
        for m in range(8):
            if e == 15 and m == 7:
                continue                      # the NaN pattern
            vals.append(m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7))
    return np.array(sorted(set(vals)))


def _torch_e4m3(x):
    return torch.tensor(x, dtype=torch.float64).to(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_grid_is_fixed_points():
    g = _grid()
    assert len(g) == 127 and g[-1] == 448.0 and g[1] == 2.0 ** -9
    for v in (g, -g):
        assert np.array_equal(O.round_to_e4m3(v), v)


def test_midpoints_round_to_even():
    g = _grid()
    mid = (g[:-1] + g[1:]) / 2
    got = O.round_to_e4m3(mid)
    # the neighbour whose mantissa is even (bit pattern index even)
    idx = np.arange(len(g))
    want = np.where(idx[:-1] % 2 == 0, g[:-1], g[1:])
    assert np.array_equal(got, want)
    assert np.array_equal(got, _torch_e4m3(mid))


def test_matches_torch_cast_on_random_values():
    r = np.random.default_rng(0)
    x = np.concatenate([r.uniform(-448, 448, 20000),
                        r.standard_normal(20000) * 0.01,          # subnormal range
                        np.exp(r.uniform(-12, 6, 20000)) * r.choice([-1, 1], 20000)])
    x = x[np.abs(x) <= 448]
    assert np.array_equal(O.round_to_e4m3(x), _torch_e4m3(x))


def test_saturates_beyond_the_largest_value():
    x = np.array([448.0, 463.9, 464.0, 500.0, 1e30, -1e30])
    assert np.array_equal(O.round_to_e4m3(x), [448, 448, 448, 448, 448, -448])


def test_row_quantisation_bounds():
    r = np.random.default_rng(1)
    x = (r.standard_normal((64, 300)) * np.exp(r.uniform(-8, 8, (64, 1)))).astype(np.float32)
    x[5] = 0.0
    q, s = O.quantize_rows_e4m3(x)
    assert s.dtype == np.float32 and s[5] == 1.0 and (q[5] == 0).all()
    g = _grid()
    assert np.isin(np.abs(q), g).all()
    nz = [i for i in range(64) if i != 5]
    assert (np.abs(q[nz]).max(axis=1) == 448.0).all()
    # dequantised error at most half a grid step: 2^-4 relative for normal
    # values, 2^-10 * s absolute in the subnormal range
    err = np.abs(q * s[:, None].astype(np.float64) - x)
    bound = np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10 * s[:, None]) * (1 + 1e-6)
    assert (err <= bound).all()


def test_fp8_head_is_exact_when_quantisation_is():
    """Rows that are e4m3 values times a power of two quantise without loss
    (the row maximum is 448 * 2^k), so the e4m3 head gives the exact logits."""
    r = np.random.default_rng(2)
    g = _grid()

    def rows(n, d):
        v = r.choice(np.concatenate([g, -g]), size=(n, d))
        v[:, 0] = 448.0
        return v * np.ldexp(1.0, r.integers(-12, -4, size=(n, 1)))

    V, d = 300, 64
    w = rows(V, d)
    y = rows(5, d)
    dims = O.ModelDims(d_model=d, n_heads=1, n_kv_heads=1, head_dim=d, vocab=V, dtype="f32",
                       lm_fp8=True)
    zeros = np.zeros((d, d), np.float32)
    m = O.OracleModel(dims, {"emb": np.zeros((V, d), np.float32), "w_q": zeros, "w_k": zeros,
                             "w_v": zeros, "w_o": zeros, "w_lm": w.astype(np.float32)})
    assert np.array_equal(m.lm_q * m.lm_scale[:, None].astype(np.float64), w)
    assert np.array_equal(m.logits(y), y @ w.T)
