"""The integer identity behind the Q1_0_g128 tensor-core product's bit
planes, checked exhaustively on the host (no GPU, no oracle).

Per packed byte, weight i (0..7) is bit b_i.  Plane 0 multiplies the whole
byte w = sum_i b_i 2^i, plane i >= 1 multiplies b_i 2^i, and the activation
side carries Y_0 = 2^7 X_0 and Y_i = 2^(7-i) X_i - 2^7 X_0 (X: 24-bit fixed
point, |X| <= 2^23), so that
    w Y_0 + sum_{i>=1} (b_i 2^i) Y_i = 2^7 sum_i b_i X_i
exactly.  Each Y is split into four signed 8-bit limbs; the u8 x s8 products
of one 128-weight group (16 k-slots per plane, 8 planes) sum below 2^20 per
limb column, so the int32 accumulators are exact and the limb pair
D_lo + 256 D_hi stays below 2^29.
"""
import numpy as np


def plane_values(X):
    """Y_0..Y_7 of one byte from the fixed-point x of its eight weights."""
    Y = np.empty(8, dtype=np.int64)
    Y[0] = 128 * X[0]
    for i in range(1, 8):
        Y[i] = X[i] * (1 << (7 - i)) - 128 * X[0]
    return Y


def limbs(y):
    """Balanced base-256 digits l0..l3 (each in [-128, 127] but the last)."""
    out = []
    r = int(y)
    for _ in range(3):
        lo = ((r & 0xFF) ^ 0x80) - 0x80
        out.append(lo)
        r = (r - lo) >> 8
    out.append(r)
    return out


def test_identity_every_byte():
    rng = np.random.default_rng(7)
    for w in range(256):
        bits = [(w >> i) & 1 for i in range(8)]
        for _ in range(8):
            X = rng.integers(-(1 << 23), (1 << 23) + 1, size=8)
            Y = plane_values(X)
            lhs = w * int(Y[0]) + sum(bits[i] * (1 << i) * int(Y[i]) for i in range(1, 8))
            assert lhs == 128 * sum(bits[i] * int(X[i]) for i in range(8))


def test_identity_at_the_extremes():
    for w in (0, 1, 0x80, 0xFF, 0x55, 0xAA):
        bits = [(w >> i) & 1 for i in range(8)]
        for X in (np.full(8, 1 << 23), np.full(8, -(1 << 23)),
                  np.array([(1 << 23) if i % 2 else -(1 << 23) for i in range(8)])):
            Y = plane_values(X)
            lhs = w * int(Y[0]) + sum(bits[i] * (1 << i) * int(Y[i]) for i in range(1, 8))
            assert lhs == 128 * sum(bits[i] * int(X[i]) for i in range(8))


def test_limbs_fit_and_reassemble():
    bound = (1 << 30) + (1 << 29)
    rng = np.random.default_rng(8)
    cases = [bound, -bound, bound - 1, -bound + 1, 0, 1, -1, 127, -128, 1 << 24, -(1 << 24)]
    cases += list(rng.integers(-bound, bound + 1, size=2000))
    for y in cases:
        l0, l1, l2, l3 = limbs(y)
        assert all(-128 <= v <= 127 for v in (l0, l1, l2))
        assert -97 <= l3 <= 97
        assert l0 + 256 * l1 + 65536 * l2 + (1 << 24) * l3 == y
    # every plane value stays inside that bound
    ext = np.array([1 << 23, -(1 << 23)])
    for x0 in ext:
        for xi in ext:
            X = np.array([x0] + [xi] * 7)
            assert np.abs(plane_values(X)).max() <= bound


def test_group_accumulator_headroom():
    """One limb column of one group: 16 k-slots x 8 planes of u8 A times s8
    limbs.  |A| sums to 255 (plane 0) + 2 + 4 + ... + 128 per slot."""
    per_slot = 255 + sum(1 << i for i in range(1, 8))
    assert per_slot == 509
    d_max = 16 * per_slot * 128
    assert d_max < (1 << 20)
    assert d_max * 257 < (1 << 29)           # D_lo + 256 D_hi
    assert d_max * 257 < (1 << 31)
