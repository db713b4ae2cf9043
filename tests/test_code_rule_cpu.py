"""The codec's code decision by buckets (quant4.cuh, code_bucket) against
the count rule code = #{k : v > t_k}, on the CPU, for both codebooks.

The kernel splits |v| into 64 buckets over [2^-8, 1) by the bits above bit
20 (exponent and three mantissa bits), each holding at most one positive
threshold, plus one bucket below and one from 1 up (Inf and NaN included),
and uses the codebooks' symmetry t_{14-k} = -t_k, t_7 = 0.  This test
restates that rule from its description and checks it on every fp32
pattern within 2^16 of each threshold (both signs), on 4M random values of
[-1, 1] and on the special values.  (Run once over all 2.1e9 fp32 values of
[-1, 1]: no mismatch.)"""
import numpy as np
import pytest

from oracle import shampoo4_oracle as O

BASE = int(np.float32(2.0 ** -8).view(np.uint32)) >> 20


def _table(t):
    pos = t[8:]
    nb = np.zeros(66, np.int32)
    tb = np.full(66, np.nan, np.float32)
    nb[65] = 7
    for i in range(64):
        lo = np.uint32((BASE + i) << 20).view(np.float32)
        hi = np.uint32((BASE + i + 1) << 20).view(np.float32)
        inside = pos[(pos >= lo) & (pos < hi)]
        assert inside.size <= 1
        nb[i + 1] = int(np.sum(pos < lo))
        if inside.size:
            tb[i + 1] = inside[0]
    return nb, tb


def _bucket_codes(v, nb, tb):
    ab = v.view(np.uint32) & np.uint32(0x7FFFFFFF)
    i = (np.minimum(np.maximum(ab >> 20, BASE - 1), BASE + 64) - (BASE - 1)).astype(np.int64)
    a = ab.view(np.float32)
    with np.errstate(invalid="ignore"):
        return np.where(v > 0, 8 + nb[i] + (a > tb[i]), 7 - nb[i] - (a >= tb[i]))


def _rule(v, t):
    c = np.zeros(v.shape, np.int64)
    with np.errstate(invalid="ignore"):
        for tk in t:
            c += v > tk
    return c


@pytest.mark.parametrize("cbk", [O.LINEAR_SQUARE, O.DYNAMIC_TREE])
def test_bucket_rule_equals_the_count_rule(cbk):
    t = O.thresholds_f32(cbk)
    assert t[7] == 0.0 and np.array_equal(t[:7], -t[::-1][:7]) and t[8:].min() >= 2.0 ** -8
    nb, tb = _table(t)
    vals = []
    for tk in np.concatenate([t[8:], np.float32([2.0 ** -8, 1.0, 0.0])]):
        b = int(np.float32(tk).view(np.uint32))
        bits = np.clip(b + np.arange(-65536, 65536), 0, 0x3F800000).astype(np.uint32)
        vals.append(bits.view(np.float32))
    rng = np.random.default_rng(3)
    vals.append(rng.uniform(-1, 1, 4 << 20).astype(np.float32))
    v = np.concatenate(vals).astype(np.float32)
    v = np.concatenate([v, -v, np.float32([np.nan, -np.nan, np.inf, -np.inf, 0.0, -0.0, 1.0, -1.0])])
    assert np.array_equal(_bucket_codes(v, nb, tb), _rule(v, t))


# ---- the signed buckets of the common case (quant4.cuh, quantize8_signed) --
#
# For q in [-1, 1]: qb = float32(q + 3) in [2, 4]; bucket k = (bits(qb) >>
# SHIFT) - (bits(2.0) >> SHIFT); c0[k] = the number of thresholds whose own
# bucket is below k; code = c0 + (q > t[c0]) with t[15] = +Inf.  SHIFT is
# 16 for linear square and 14 for the dynamic tree.  (Run once over all
# 2.1e9 fp32 values of [-1, 1] for both codebooks: no mismatch.)

SHIFTS = {O.LINEAR_SQUARE: 16, O.DYNAMIC_TREE: 14}


def _signed_bucket(q, shift):
    qb = (q.astype(np.float32) + np.float32(3.0)).astype(np.float32)
    return (qb.view(np.uint32) >> shift).astype(np.int64) - (0x40000000 >> shift)


def _signed_codes(q, t, shift):
    kb = _signed_bucket(t, shift)
    assert np.all(np.diff(kb) > 0), "two thresholds share a bucket"
    count = (0x40800000 >> shift) - (0x40000000 >> shift) + 1
    c0 = np.array([int(np.sum(kb < k)) for k in range(count)], np.int64)
    t16 = np.concatenate([t, np.float32([np.inf])]).astype(np.float32)
    c = c0[_signed_bucket(q, shift)]
    return c + (q > t16[c])


@pytest.mark.parametrize("cbk", [O.LINEAR_SQUARE, O.DYNAMIC_TREE])
def test_signed_bucket_rule_equals_the_count_rule(cbk):
    shift = SHIFTS[cbk]
    t = O.thresholds_f32(cbk)
    # the bucket width stays below the smallest gap between thresholds
    assert 2.0 ** (shift - 22) < np.min(np.diff(t.astype(np.float64)))
    vals = []
    for tk in t:                                   # every pattern near each threshold
        b = int(np.float32(tk).view(np.uint32))
        vals.append((b + np.arange(-65536, 65536)).astype(np.uint32).view(np.float32))
    off = 0x40000000 >> shift
    count = (0x40800000 >> shift) - off + 1
    for k in range(count + 1):                     # values on both sides of each bucket edge
        edge = np.uint32((off + k) << shift).view(np.float32) - np.float32(3.0)
        vals.append(np.float32(edge) + np.arange(-2000, 2000, dtype=np.float32) * np.float32(2.0 ** -24))
    rng = np.random.default_rng(5)
    vals.append(rng.uniform(-1, 1, 4 << 20).astype(np.float32))
    vals.append(np.float32([0.0, -0.0, 1.0, -1.0, 1e-38, -1e-38, 1e-45, -1e-45, 2.0 ** -30, -(2.0 ** -30)]))
    q = np.concatenate(vals).astype(np.float32)
    q = q[np.abs(q) <= 1]
    q = np.concatenate([q, -q])
    assert np.array_equal(_signed_codes(q, t, shift), _rule(q, t))
