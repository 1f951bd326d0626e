"""The fixed-point arithmetic of the tensor-core decodes, checked on the CPU.

The kernels' integer contractions are exact; what they round is stated in include/kvq.h
and used by the decode bound of tests/_helpers.py.  These tests emulate each rounding
step in numpy float32 (the kernels' fp32 operations, each rounded to nearest even) and
check the stated bounds on many random and edge-case inputs:
  * query digits (INT8 keys): E from the exponent of max |q| (max |q| 2^E in [2^21,
    2^22)), q_fix = rint(q 2^E), three balanced base-256 digits in [-128, 127] that
    recombine to q_fix exactly, |q - q_fix 2^-E| <= 2^-22 max |q|, exact for entries within
    2^11 of max |q|, and digit sums of 128 int8 codes that fit in int32;
  * value weights (both kernels): W = rint(fl(p v) 2^E'), smax 2^E' in [2^23, 2^24) from
    smax's exponent, never above 2^24 - 1, |W 2^-E' - p v| < 2^-23 smax per token;
  * softmax sums: sum rint(p 2^24) 2^-24 within n 2^-25 of sum p over n tokens.
"""
import numpy as np
import pytest

F32 = np.float32


def _exp_bits(x):
    return (np.asarray(x, F32).view(np.uint32) >> 23).astype(np.int64)


def _digits(q16):
    """The kernel's digit scheme for one head's query (fp16 [128])."""
    q = q16.astype(F32)
    amax = F32(np.abs(q).max())
    E = 21 - (int(_exp_bits(amax)) - 127) if amax > 0 else 0
    qf = np.rint(q * F32(2.0 ** E)).astype(np.int64)        # q 2^E is exact (fp16 times 2^E)
    d0 = ((qf + 128) & 255) - 128
    r1 = (qf - d0) >> 8
    d1 = ((r1 + 128) & 255) - 128
    d2 = (r1 - d1) >> 8
    return E, qf, d0, d1, d2, amax


def _queries(rng, n):
    out = [rng.standard_normal(128).astype(np.float16) for _ in range(n)]
    out += [(rng.standard_normal(128) * 10.0 ** rng.uniform(-6, 4)).astype(np.float16) for _ in range(n)]
    edge = np.zeros(128, np.float16)
    out.append(edge.copy())                                   # all zero
    one = edge.copy(); one[5] = np.float16(65504.0); out.append(one)        # fp16 max
    tiny = edge.copy(); tiny[3] = np.float16(2.0 ** -24); tiny[7] = -np.float16(2.0 ** -24)
    out.append(tiny)                                          # fp16 subnormals only
    mix = rng.standard_normal(128).astype(np.float16); mix[0] = np.float16(-65504.0); out.append(mix)
    top = np.full(128, np.float16(1.9990234375)); top[::2] *= -1; out.append(top)   # mantissas at the top
    return out


def test_query_digits_exact_and_bounded():
    rng = np.random.default_rng(11)
    for q16 in _queries(rng, 300):
        E, qf, d0, d1, d2, amax = _digits(q16)
        for d in (d0, d1, d2):
            assert d.min() >= -128 and d.max() <= 127
        assert np.array_equal(d0 + 256 * d1 + 65536 * d2, qf)
        assert np.abs(qf).max() < 2 ** 22
        q = q16.astype(np.float64)
        err = np.abs(q - qf.astype(np.float64) * 2.0 ** -E)
        assert np.all(err <= 2.0 ** -22 * float(amax))
        near = np.abs(q) >= float(amax) * 2.0 ** -11
        assert np.all(err[near] == 0.0)
        # digit sums over 128 int8 codes stay in int32 (|D_k| < 2^21)
        c = rng.integers(-127, 128, size=(64, 128))
        for d in (d0, d1, d2):
            assert np.abs(c @ d).max() < 2 ** 21
        assert np.array_equal(c @ d0 + 256 * (c @ d1) + 65536 * (c @ d2), c @ qf)


def _weights(p, v):
    """W, the unit 2^-E' and smax for one slice or chunk (p, v float32 arrays)."""
    smax = F32(v.max())
    sexp = int(_exp_bits(smax))
    assert sexp >= 28
    rscale = F32(2.0 ** (150 - sexp))
    prod = (p * v).astype(F32) * rscale                      # fl(p v), then the exact 2^E' scaling
    W = np.minimum(np.rint(prod.astype(np.float64)), 2 ** 24 - 1).astype(np.int64)
    return W, 2.0 ** (sexp - 150), float(smax), prod


@pytest.mark.parametrize("scale_exp", [-30, -8, 0, 5, 40])
def test_value_weights_bounded(scale_exp):
    rng = np.random.default_rng(100 + scale_exp)
    for trial in range(200):
        n = int(rng.integers(1, 129))
        p = rng.uniform(0.0, 1.0, n).astype(F32)
        p[rng.integers(0, n)] = F32(1.0)                      # the slice's max logit
        v = (rng.uniform(0.0, 1.0, n) * 2.0 ** scale_exp).astype(F32)
        if trial % 7 == 0:                                    # the largest scale with a full mantissa
            v[0] = F32(np.nextafter(F32(2.0 ** (scale_exp + 1)), F32(0)))
        W, unit, smax, prod = _weights(p, v)
        assert np.all(np.rint(prod.astype(np.float64)) <= 2 ** 24 - 1)   # the clamp never binds
        err = np.abs(W * unit - p.astype(np.float64) * v.astype(np.float64))
        assert np.all(err < 2.0 ** -23 * smax)
        assert 2.0 ** 23 <= smax / unit < 2.0 ** 24


def test_softmax_sum_fixed_point():
    rng = np.random.default_rng(7)
    for n in (1, 32, 128):
        for _ in range(500):
            p = rng.uniform(0.0, 1.0, n).astype(F32)
            lq = np.rint((p * F32(2.0 ** 24)).astype(np.float64)).astype(np.int64)   # p 2^24 exact
            assert lq.sum() < 2 ** 32                         # the warp's unsigned reduction
            L = float(lq.sum()) * 2.0 ** -24
            assert abs(L - float(p.astype(np.float64).sum())) <= n * 2.0 ** -25
