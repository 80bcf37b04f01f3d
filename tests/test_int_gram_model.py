"""The integer Gram leaf's arithmetic, modelled in exact integers on the CPU (numpy and
Python integers; nothing here imports the CUDA path or the oracle).

The leaf reads each column of an item as 32-bit fixed point: the column is scaled by
2^(31 - E), E = the exponent of its largest magnitude over the item's first 128 rows + 2
(that magnitude lies below 2^(E - 2)), and truncated toward zero to an integer N.  Flipping the sign bit (U = N + 2^31) makes the four bytes
of U unsigned digits whose top digit is the signed top digit + 128, so N^T N is a sum of
16 Grams of unsigned byte matrices, weighted by powers of 256, with column-sum
corrections for the +128.  These tests check that this reading reproduces N^T N exactly,
that every digit-pair Gram of an item fits an int32 accumulator, and that the
fixed-point image moves each value by less than 2^-27 of its column's largest magnitude.
"""
import numpy as np
import pytest

MAX_ITEM_ROWS = 24576   # rows per leaf item


def fixed_point(X, lead=128):
    """(N, E): N = trunc(X 2^(31 - E)) per column as int64; E from the first `lead` rows."""
    m = np.max(np.abs(X[:lead]), axis=0)
    _, e = np.frexp(m)                  # m = f 2^e with f in [0.5, 1)
    E = np.where(m > 0, e + 2, -90)     # a column whose lead rows are zero: any later nonzero value is out of range
    assert np.all(np.abs(X) < np.ldexp(1.0, E)), "a value at or above 2^E leaves the integer leaf"
    N = np.trunc(np.ldexp(X, 31 - E)).astype(np.int64)
    assert np.all(np.abs(N) < 2 ** 31)
    return N, E


def byte_digits(N):
    """The four unsigned bytes of U = N + 2^31, least significant first."""
    U = (N + 2 ** 31).astype(np.uint64)
    return [((U >> np.uint64(8 * i)) & np.uint64(255)).astype(np.int64) for i in range(4)]


def gram_from_digits(N):
    """N^T N from the 16 unsigned digit-pair Grams and the digits' column sums, combined in
    Python integers (the leaf combines them exactly in int64 per weight)."""
    rows, c = N.shape
    u = byte_digits(N)
    P = [[u[i].T @ u[j] for j in range(4)] for i in range(4)]   # each entry <= 255^2 rows
    s = [d.sum(axis=0) for d in u]
    G = [[0] * c for _ in range(c)]
    for a in range(c):
        for b in range(c):
            acc = 0
            for i in range(4):
                for j in range(4):
                    t = int(P[i][j][a, b])
                    if j == 3:                   # D_3 = u_3 - 128 on the right
                        t -= 128 * int(s[i][a])
                    if i == 3:                   # and on the left
                        t -= 128 * int(s[j][b])
                    if i == 3 and j == 3:
                        t += 128 * 128 * rows
                    acc += t << (8 * (i + j))
            G[a][b] = acc
    return G


def exact_gram(N):
    rows, c = N.shape
    cols = [[int(v) for v in N[:, a]] for a in range(c)]
    return [[sum(x * y for x, y in zip(cols[a], cols[b])) for b in range(c)] for a in range(c)]


def test_digit_pair_grams_fit_int32_accumulators():
    assert 255 * 255 * MAX_ITEM_ROWS < 2 ** 31
    assert 255 * 255 * 33026 >= 2 ** 31   # 33 025 rows is the most any item could hold


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_digit_split_reproduces_the_fixed_point_gram_exactly(seed):
    rng = np.random.default_rng(seed)
    rows, c = 300, 6
    scales = np.ldexp(1.0, rng.integers(-20, 20, size=c))   # columns of very different magnitude
    X = (rng.standard_normal((rows, c)) * scales).astype(np.float32).astype(np.float64)
    X[:, 0] = 0.0                                             # an all-zero column
    X[:, 1] = -np.abs(X[:, 1])                                # a column of one sign
    N, E = fixed_point(X)
    assert gram_from_digits(N) == exact_gram(N)


def test_extreme_fixed_point_values_split_exactly():
    N = np.array([[2 ** 31 - 1, -(2 ** 31) + 1, 0, -1, 1, 255, -256, 2 ** 24, -(2 ** 24)]], dtype=np.int64)
    N = np.repeat(N, 3, axis=0)
    assert gram_from_digits(N) == exact_gram(N)
    u = byte_digits(N)   # the digits read back as N with the top one signed
    recon = u[0] + (u[1] << 8) + (u[2] << 16) + ((u[3] - 128) << 24)
    assert np.array_equal(recon, N)


@pytest.mark.parametrize("seed", [3, 4])
def test_fixed_point_image_error_bound(seed):
    rng = np.random.default_rng(seed)
    rows, c = 2048, 5
    X = (rng.standard_normal((rows, c)) * np.ldexp(1.0, rng.integers(-10, 10, size=c))).astype(np.float32)
    X = X.astype(np.float64)
    N, E = fixed_point(X)
    Xt = np.ldexp(N.astype(np.float64), E - 31)
    colmax = np.max(np.abs(X), axis=0)
    assert np.all(np.abs(Xt - X) < np.ldexp(colmax, -27))
    assert np.all(np.abs(Xt) <= np.abs(X))                     # truncation moves values toward zero
