"""The order keys of the top-k, and the raw-bit candidate test built on them.

The top-k ranks FP32 scores by order-preserving 32-bit keys: -0.0 is folded
onto +0.0, a negative float maps to the complement of its bits and a
non-negative one to its bits with the top bit set.  Its single pass over a
row takes every score whose key is at or above a sampled bound `lo`; for a
bound above the key of +0.0 it tests the raw bits instead, as one signed
compare with lo & 0x7FFFFFFF.  These tests check, on the CPU and for every
class of bit pattern (zeros of both signs, denormals, normals, infinities,
NaNs of both signs), that the keys order the floats as the comparison does
and that the raw-bit test accepts exactly the scores the key test accepts.
"""

import numpy as np
import pytest

KEY_POS_ZERO = 0x80000000


def order_key(bits: np.ndarray) -> np.ndarray:
    u = bits.astype(np.uint32).copy()
    u[u == 0x80000000] = 0
    neg = (u & 0x80000000) != 0
    return np.where(neg, ~u, u | np.uint32(0x80000000)).astype(np.uint32)


def raw_test(bits: np.ndarray, lo: int) -> np.ndarray:
    assert lo > KEY_POS_ZERO
    return bits.astype(np.uint32).view(np.int32) >= np.int32(lo & 0x7FFFFFFF)


def special_patterns() -> np.ndarray:
    f = np.array([0.0, -0.0, np.inf, -np.inf, 1.0, -1.0, np.finfo(np.float32).max,
                  -np.finfo(np.float32).max, np.finfo(np.float32).tiny, -np.finfo(np.float32).tiny],
                 dtype=np.float32).view(np.uint32)
    extra = np.array([0x00000001, 0x80000001, 0x007FFFFF, 0x807FFFFF,   # denormals
                      0x7FC00000, 0xFFC00000, 0x7F800001, 0xFF800001,   # quiet / signalling NaNs
                      0x7FFFFFFF, 0xFFFFFFFF], dtype=np.uint32)
    return np.concatenate([f, extra])


def test_keys_order_floats_as_comparison():
    rng = np.random.default_rng(11)
    bits = rng.integers(0, 2**32, size=200_000, dtype=np.uint64).astype(np.uint32)
    bits = np.concatenate([bits, special_patterns()])
    f = bits.view(np.float32)
    finite = bits[~np.isnan(f)]
    ff = finite.view(np.float32)
    k = order_key(finite)
    i = rng.integers(0, finite.size, size=100_000)
    j = rng.integers(0, finite.size, size=100_000)
    assert np.array_equal(k[i] < k[j], ff[i] < ff[j])
    assert np.array_equal(k[i] == k[j], ff[i] == ff[j])          # -0.0 == +0.0 included
    # positive NaNs rank above +inf, negative NaNs below -inf
    nan = bits[np.isnan(f)]
    kn = order_key(nan)
    pos = (nan & 0x80000000) == 0
    k_inf = order_key(np.array([0x7F800000, 0xFF800000], dtype=np.uint32))
    assert np.all(kn[pos] > k_inf[0]) and np.all(kn[~pos] < k_inf[1])


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_raw_bit_test_equals_key_test_for_positive_bounds(seed):
    rng = np.random.default_rng(seed)
    bits = rng.integers(0, 2**32, size=300_000, dtype=np.uint64).astype(np.uint32)
    bits = np.concatenate([bits, special_patterns()])
    keys = order_key(bits)
    los = [KEY_POS_ZERO + 1, int(order_key(np.array([0x3F800000], dtype=np.uint32))[0]),
           int(order_key(np.array([0x7F800000], dtype=np.uint32))[0]),          # +inf
           int(order_key(np.array([0x7F800000], dtype=np.uint32))[0]) + 1,      # just above +inf
           0xFFFFFFFF]
    los += [int(x) for x in rng.integers(KEY_POS_ZERO + 1, 2**32, size=20, dtype=np.uint64)]
    # bounds as the single pass forms them: a sampled key with its low 10 bits cleared
    sampled = keys[keys > KEY_POS_ZERO + 1024][:20]
    los += [int(x) & ~0x3FF for x in sampled if (int(x) & ~0x3FF) > KEY_POS_ZERO]
    for lo in los:
        assert np.array_equal(raw_test(bits, lo), keys >= lo), hex(lo)


def test_bound_at_positive_zero_key_is_left_to_the_key_test():
    # at lo = key(+0.0) the raw test would drop -0.0, whose key equals +0.0's:
    # the kernel only takes the raw test strictly above that key
    bits = np.array([0x80000000, 0x00000000], dtype=np.uint32)
    assert np.all(order_key(bits) >= KEY_POS_ZERO)
    assert not (bits.view(np.int32) >= np.int32(KEY_POS_ZERO & 0x7FFFFFFF))[0]
