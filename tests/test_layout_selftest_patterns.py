"""The tensor-core layout self-test (dsa_selftest_mma_layout) can only catch a
layout mistake if its test matrices make that mistake change the product.
These CPU checks plant each mistake in a host model of the self-test's
matrices and show that the product changes: a transposed operand, a missing or
wrong swizzle, swapped K chunks, a wrong P swizzle, an accumulator row or
column read from the wrong lane, and a wrong e4m3 code. The matrices are the
self-test's own (the same hash of row and column as csrc/layout_selftest.cu)."""
import numpy as np


_M32 = 0xFFFFFFFF


def _mix(r, c, seed):
    """The self-test's 32-bit hash of (row, column)."""
    r = np.asarray(r, dtype=np.uint64)
    c = np.asarray(c, dtype=np.uint64)
    x = ((r * 0x9E3779B1) & _M32) ^ ((c * 0x85EBCA77) & _M32) ^ seed
    x = x ^ (x >> 15)
    x = (x * 0x2C1B3C6D) & _M32
    return x ^ (x >> 12)


def a_val(m, k):
    return (_mix(m, k, 0x1234) % 7).astype(np.int64) - 3


def b_val(n, k):
    return (_mix(n, k, 0x5678) % 5).astype(np.int64) - 2


def _mat(f, rows, cols):
    r = np.arange(rows)[:, None]
    c = np.arange(cols)[None, :]
    return f(r, c).astype(np.int64)


A = _mat(a_val, 128, 128)          # [m][k]
B256 = _mat(b_val, 256, 128)       # [n][k], the indexer forms
B32 = _mat(b_val, 32, 128)         # [n][k], the attention forms


def _changed(wrong, right):
    return int(np.count_nonzero(wrong != right))


def test_values_fit_the_formats_exactly():
    assert A.min() >= -3 and A.max() <= 3 and B256.min() >= -2 and B256.max() <= 2
    d = A @ B256.T
    assert np.abs(d).max() < 2 ** 24  # every partial sum is exact in float32


def test_no_two_rows_or_columns_coincide():
    # a mix-up of two operand rows, or of two accumulator rows or columns, is
    # invisible if they hold the same values
    for mat in (A, B256, A @ B256.T, (A @ B256.T).T, A @ B32.T, (A @ B32.T).T):
        assert len({row.tobytes() for row in mat}) == mat.shape[0]


def test_a_transposed_is_caught():
    right = A @ B256.T
    assert _changed(A.T @ B256.T, right) > 1000


def test_missing_or_wrong_128_byte_swizzle_is_caught():
    # element (m, k) of a 128-byte row lives in 16-byte unit (k % 64) // 8 ^ (m % 8);
    # reading without the swizzle takes unit u from where unit u ^ (m % 8) was written
    right = A @ B256.T
    m = np.arange(128)[:, None]
    k = np.arange(128)[None, :]
    unit = (k % 64) // 8
    k_read = (k // 64) * 64 + ((unit ^ (m % 8)) * 8) + k % 8
    a_read = A[np.broadcast_to(m, k_read.shape), k_read]
    assert _changed(a_read @ B256.T, right) > 1000
    # the swizzle taken from the wrong row bits (r / 8 instead of r % 8)
    k_read2 = (k // 64) * 64 + ((unit ^ ((m // 8) % 8)) * 8) + k % 8
    a_read2 = A[np.broadcast_to(m, k_read2.shape), k_read2]
    assert _changed(a_read2 @ B256.T, right) > 1000


def test_swapped_k_chunks_are_caught():
    right = A @ B256.T
    assert _changed(A[:, np.arange(128) ^ 64] @ B256.T, right) > 1000


def test_wrong_p_swizzle_is_caught():
    # P row k holds 32 heads in 64 bytes; unit c (8 heads) at c ^ ((k >> 1) & 3)
    right = A @ B32.T
    n = np.arange(32)[:, None]
    k = np.arange(128)[None, :]
    n_read = ((n // 8) ^ ((k >> 1) & 3)) * 8 + n % 8       # read unswizzled
    b_read = B32[n_read, np.broadcast_to(k, n_read.shape)]
    assert _changed(A @ b_read.T, right) > 500
    n_read2 = ((n // 8) ^ ((k >> 2) & 1)) * 8 + n % 8      # the 32-byte-row rule instead
    b_read2 = B32[n_read2 % 32, np.broadcast_to(k, n_read2.shape)]
    assert _changed(A @ b_read2.T, right) > 500


def test_wrong_accumulator_lane_or_column_is_caught():
    right = A @ B32.T
    assert _changed(np.roll(right, 1, axis=0), right) > 1000   # row m read from lane m + 1
    assert _changed(np.roll(right, 1, axis=1), right) > 1000   # column n from column n + 1
    # the M = 64 half-subpartition mapping (row r in lane r % 16 + 32 (r // 16))
    lanes = np.array([(r % 16) + 32 * (r // 16) for r in range(64)])
    assert _changed(right[lanes], right[:64]) > 1000


def _e4m3_value(code):
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 7
    if e == 0:
        return s * (m / 8.0) * 2.0 ** -6
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def test_e4m3_codes_of_the_selftest_decode_to_their_integers():
    # the codes the self-test writes for -3 .. 3, decoded with the e4m3
    # definition (sign, 4 exponent bits biased by 7, 3 mantissa bits)
    codes = {0: 0x00, 1: 0x38, 2: 0x40, 3: 0x44}
    for v in range(-3, 4):
        c = codes[abs(v)] | (0x80 if v < 0 else 0)
        assert _e4m3_value(c) == v
