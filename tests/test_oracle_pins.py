"""Pins for the CPU oracle: each test checks it against something other than itself --
hand-worked examples from the pages' equations, invariants, closed forms, library
routines for special cases, and fp64 brute force on tiny inputs.  CPU only.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from kv_cache_quantization_absmax_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ----------------------------------------------------------------------------------
# fp16 conversions (IEEE binary16) against numpy's own conversions
# ----------------------------------------------------------------------------------

def test_half_to_double_all_patterns():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.half_to_double(int(b)) for b in bits])
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite], ref[finite])
    assert np.array_equal(np.isinf(got), np.isinf(ref))
    assert np.array_equal(np.isnan(got), np.isnan(ref))


def test_double_to_half_round_to_nearest_even():
    rng = np.random.default_rng(123)
    xs = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.uniform(-9, 5, 20000),
        # exact midpoints between neighbouring halves exercise ties-to-even
        (np.arange(0, 4096, dtype=np.float64) + 0.5) * 2.0 ** -24,
        (np.arange(1024, 2048, dtype=np.float64) + 0.5) * 2.0 ** -3,
        [0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e9, -1e9, 2.0 ** -25, 2.0 ** -25 * 1.0001],
    ])
    with np.errstate(over="ignore"):
        ref = xs.astype(np.float16).view(np.uint16)
    got = np.array([oracle.double_to_half(float(x)) for x in xs], dtype=np.uint16)
    assert np.array_equal(got, ref)


# ----------------------------------------------------------------------------------
# INT8 absmax quantization (Q-TensorFormer section 6, INT8 equation)
# ----------------------------------------------------------------------------------

def _fl32_nearest(fr: Fraction) -> Fraction:
    """Nearest fp32 value (ties to even) of an exact rational, by exact arithmetic;
    used only to validate the hand-worked fixture values themselves."""
    if fr == 0:
        return Fraction(0)
    sign = -1 if fr < 0 else 1
    a = abs(fr)
    e = math.floor(math.log2(a.numerator) - math.log2(a.denominator))
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, -126)
    quantum = Fraction(2) ** (e - 23)
    n = round(a / quantum)          # Python rounds Fractions half to even
    return sign * n * quantum


@pytest.mark.parametrize("case", _golden("int8_worked_examples.json")["cases"],
                         ids=lambda c: c["name"])
def test_int8_worked_examples(case):
    dt = np.float32 if case["dtype"] == "f32" else np.float16
    x = np.array([float.fromhex(v) for v in case["x"]]).astype(dt)
    assert np.array_equal(x.astype(np.float64), [float.fromhex(v) for v in case["x"]])
    codes, scales = oracle.quantize_int8(x[None, :])
    assert float(scales[0]) == float.fromhex(case["scale"])
    assert codes[0].tolist() == case["codes"]
    # the fixture's scale is the fp32 value nearest to a / 127 (exact rational check)
    a = max(abs(Fraction(float(v))) for v in x)
    assert _fl32_nearest(a / 127) == Fraction(float.fromhex(case["scale"]))
    # dequantized values are the exact product c * s (formed in fp64, where 8 + 24
    # significant bits fit) rounded once to fp32
    xh = oracle.dequantize_int8(codes, scales)
    exact = np.array(case["codes"], np.float64) * float.fromhex(case["scale"])
    assert np.array_equal(xh[0], exact.astype(np.float32))


def _sweep_like(n, d, dtype, seed):
    x, _, _ = inputs.sweep_matrix(n * d, d, dtype, seed, n_rows=n)
    return x


@pytest.mark.parametrize("dtype", [np.float32, np.float16])
@pytest.mark.parametrize("d", [16, 128, 1024])
def test_int8_invariants(dtype, d):
    x = _sweep_like(256, d, dtype, seed=d)
    x[7] = 0                       # a zero row
    x[9, :] = x[9, 0]              # an all-equal row
    codes, s = oracle.quantize_int8(x)
    xf = x.astype(np.float64)
    a = np.abs(xf).max(axis=1)
    # zero row: zero scale, zero codes
    assert s[7] == 0 and not codes[7].any()
    nz = a > 0
    # |c| <= 127 and the absmax element maps to exactly +-127 with its sign
    assert np.abs(codes.astype(np.int32)).max() <= 127
    j = np.abs(xf).argmax(axis=1)
    rows = np.nonzero(nz)[0]
    assert np.array_equal(codes[rows, j[rows]].astype(np.int32),
                          np.where(xf[rows, j[rows]] > 0, 127, -127))
    # all-equal row maps every element to the same +-127
    assert np.all(codes[9] == codes[9, 0]) and abs(int(codes[9, 0])) == 127
    # round-trip error bound |x - x_hat| <= s/2 (checked in fp64, one fp32 ulp of slack)
    xh = oracle.dequantize_int8(codes, s).astype(np.float64)
    err = np.abs(xf - xh)
    slack = np.spacing(np.abs(xh).astype(np.float32)).astype(np.float64)
    assert np.all(err <= s.astype(np.float64)[:, None] / 2 + slack)
    # the scale sits within half an fp32 ulp of a / 127
    s64 = s.astype(np.float64)
    assert np.all(np.abs(s64[nz] - a[nz] / 127) <= np.spacing(s[nz]).astype(np.float64) / 2)


def test_int8_symmetry_and_power_of_two_scaling():
    x = _sweep_like(64, 128, np.float32, seed=5)
    c, s = oracle.quantize_int8(x)
    cn, sn = oracle.quantize_int8(-x)            # round-half-even is odd-symmetric
    assert np.array_equal(cn, -c) and np.array_equal(sn, s)
    c4, s4 = oracle.quantize_int8(x * np.float32(4.0))   # exact rescale by 2^2
    assert np.array_equal(c4, c) and np.array_equal(s4, s * np.float32(4.0))


def test_dequant_fp16_is_rounded_fp32_product():
    x = _sweep_like(64, 128, np.float16, seed=6)
    c, s = oracle.quantize_int8(x)
    f32 = oracle.dequantize_int8(c, s, np.float32)
    f16 = oracle.dequantize_int8(c, s, np.float16)
    assert np.array_equal(f16.view(np.uint16), f32.astype(np.float16).view(np.uint16))


def test_int8_scores_against_fp64_brute_force():
    x, q, _ = inputs.sweep_matrix(128 * 1024, 1024, np.float32, 1, n_rows=128)
    c, s = oracle.quantize_int8(x)
    got = oracle.int8_scores(q, c, s).astype(np.float64)
    xh = (c.astype(np.float64) * s.astype(np.float64)[:, None]).astype(np.float32)
    terms = xh.astype(np.float64) * q.astype(np.float64)[None, :]
    ref = terms.sum(axis=1)
    d = x.shape[1]
    bound = 2 * d * 2.0 ** -24 * np.abs(terms).sum(axis=1)
    assert np.all(np.abs(got - ref) <= bound)
    # fp16 query: the same scores as the widened fp32 query
    q16 = q.astype(np.float16)
    assert np.array_equal(oracle.int8_scores(q16, c, s), oracle.int8_scores(q16.astype(np.float32), c, s))


# ----------------------------------------------------------------------------------
# QJL sketch and estimator (QJL abstract)
# ----------------------------------------------------------------------------------

def _tiny_sketch(g):
    r = np.array(g["rows_0_7"], np.float64)
    r16 = np.concatenate([r, -r])
    return np.concatenate([r16, r16])


def test_qjl_hand_worked_example():
    g = _golden("qjl_tiny_example.json")
    S = _tiny_sketch(g)
    k = np.array(g["key"], np.float16)[None, :]
    words, norms, u = oracle.qjl_encode(k, S, want_u=True)
    assert np.array_equal(u[0, :16], g["projections_0_15"])
    assert int(words[0, 0]) == int(g["word"], 16)
    assert int(norms.view(np.uint16)[0]) == int(g["norm_f16_bits"], 16)
    assert float(norms[0]) == 3.775390625
    q = np.array(g["query"], np.float16)[None, :]
    v64, v32 = oracle.qjl_query_sketch(q, S)
    assert np.array_equal(v64[0, :16], g["query_sketch_0_15"])
    est = oracle.qjl_estimate(v64[0], words[0], float(norms[0]))
    expect = math.sqrt(math.pi / 2) / 32 * 3.775390625 * g["signed_sum"]
    assert est == pytest.approx(expect, rel=1e-15)
    sc = oracle.qjl_scores(v64, words, norms)
    assert sc[0, 0] == np.float32(expect)


def test_qjl_projection_matches_matmul():
    S = inputs.sketch_matrix(256, 128)
    keys = inputs.lognormal_cache(11, 1, 2, 64)[0].reshape(-1, 128)
    words, norms, u = oracle.qjl_encode(keys, S, want_u=True)
    ref = keys.astype(np.float64) @ S.astype(np.float64).T
    assert np.allclose(u, ref, rtol=0, atol=1e-12 * np.abs(ref).max())
    bits = (u >= 0).astype(np.uint64)
    packed = np.zeros((keys.shape[0], 8), np.uint64)
    for i in range(256):
        packed[:, i // 32] |= bits[:, i] << np.uint64(i % 32)
    assert np.array_equal(words.astype(np.uint64), packed)
    nref = np.sqrt((keys.astype(np.float64) ** 2).sum(axis=1)).astype(np.float16)
    assert np.array_equal(norms.view(np.uint16), nref.view(np.uint16))
    q = inputs.gaussian_queries(12, 1, 3)[0]
    v64, v32 = oracle.qjl_query_sketch(q, S)
    vref = q.astype(np.float64) @ S.astype(np.float64).T
    assert np.allclose(v64, vref, rtol=0, atol=1e-12 * np.abs(vref).max())
    assert np.array_equal(v32, v64.astype(np.float32))


def test_qjl_estimator_unbiased_over_2000_sketches():
    """Mean over 2000 independent Gaussian sketches lies within 3 standard errors of the
    exact inner product (fp64 sketches, seeds 10000..11999)."""
    k = inputs.lognormal_cache(4, 1, 1, 1)[0].reshape(1, 128)
    q = inputs.gaussian_queries(40, 1, 1)[0]
    exact = float(k[0].astype(np.float64) @ q[0].astype(np.float64))
    est = []
    for seed in range(10000, 12000):
        S = inputs.sketch_matrix_f64(256, 128, seed)
        words, norms = oracle.qjl_encode(k, S)
        v64, _ = oracle.qjl_query_sketch(q, S)
        est.append(oracle.qjl_estimate(v64[0], words[0], float(norms[0])))
    est = np.array(est)
    se = est.std(ddof=1) / math.sqrt(len(est))
    assert abs(est.mean() - exact) <= 3 * se, (est.mean(), exact, se)
    # the 1/m scaling: the spread shrinks like 1/sqrt(m) -- variance is O(|q|^2 |k|^2 / m)
    assert est.std() < 2.0 * np.linalg.norm(q[0].astype(np.float64)) * np.linalg.norm(
        k[0].astype(np.float64)) / math.sqrt(256)


def test_qjl_parallel_key_and_scaling():
    S = inputs.sketch_matrix(256, 128)
    q = inputs.gaussian_queries(13, 1, 1)[0]
    # k parallel to q (k = q exactly): every bit agrees with the sign of v, so the
    # estimate is sqrt(pi/2)/m * |k| * sum |v_i| >= 0
    k = q.copy()
    words, norms = oracle.qjl_encode(k, S)
    v64, _ = oracle.qjl_query_sketch(q, S)
    est = oracle.qjl_estimate(v64[0], words[0], float(norms[0]))
    assert est == pytest.approx(math.sqrt(math.pi / 2) / 256 * float(norms[0]) * np.abs(v64[0]).sum(),
                                rel=1e-12)
    # scaling the key by 4 (exact in fp16) leaves the bits unchanged and scales the estimate
    k4 = (k.astype(np.float32) * 4).astype(np.float16)
    w4, n4 = oracle.qjl_encode(k4, S)
    assert np.array_equal(w4, words)
    assert float(n4[0]) == 4 * float(norms[0])
    assert oracle.qjl_estimate(v64[0], w4[0], float(n4[0])) == pytest.approx(4 * est, rel=1e-12)
    # a zero key: every projection is 0 >= 0, so all bits are set, and the norm is 0
    wz, nz = oracle.qjl_encode(np.zeros((1, 128), np.float16), S)
    assert np.all(wz == 0xFFFFFFFF) and float(nz[0]) == 0.0



def tie_keys():
    """Keys whose exact norm is an fp16 rounding midpoint (ulp 2 at 2048, 2^-7 at 8)."""
    rows = np.zeros((6, 128), np.float16)
    rows[0, :3] = [2048, 64, 1]                 # 2048^2 + 64^2 + 1 = 2049^2: tie -> even 2048
    rows[1, :4] = [2048, 110, 14, 1]            # = 2051^2: tie between 2050 and 2052 -> 2052
    rows[2, :3] = [8, 0.25, 2.0 ** -8]          # = 8.00390625^2: tie -> 8
    rows[3] = rows[2]
    rows[3, 3:10] = 2.0 ** -24                  # seven 2^-48 squares after 64: each below
    #                                             half an ulp of the partial sum, dropped
    rows[4, 100:103] = [8, 0.25, 2.0 ** -8]
    rows[4, 0:7] = 2.0 ** -24                   # the same squares first: 7 * 2^-48 is exact,
    #                                             then 64 + 7 * 2^-48 rounds to 64 + 2^-45
    rows[5] = rows[2]
    rows[5, 3] = 2.0 ** -12                     # a 2^-24 square is kept: above the midpoint
    return rows


def test_qjl_norm_fp64_index_order_and_ties():
    """The stored norm is the fp16 rounding (nearest, ties to even) of the root of the
    fp64 sum of squares taken in index order: exact midpoints pin the tie rule; the same
    multiset of squares in two orders pins the order (the exact norm would round up in
    both); a kept small square pins that the sum is not a coarser one."""
    S = inputs.sketch_matrix(32, 128)
    _, norms = oracle.qjl_encode(tie_keys(), S)
    assert [float(x) for x in norms] == [2048.0, 2052.0, 8.0, 8.0, 8.0078125, 8.0078125]

# ----------------------------------------------------------------------------------
# Decode step: softmax invariants, special cases, fp64 brute force with the page's GQA
# broadcast (unsqueeze(2).expand(...).reshape(...))
# ----------------------------------------------------------------------------------

def _tiny_cache(T, D=8, B=1, Hq=4, Hkv=2, seed=0):
    rng = np.random.default_rng(seed)
    k = rng.standard_normal((B, Hkv, T, D)).astype(np.float16)
    v = rng.standard_normal((B, Hkv, T, D)).astype(np.float16)
    q = rng.standard_normal((B, Hq, D)).astype(np.float16)
    kc, ks = oracle.quantize_int8(k.reshape(-1, D))
    vc, vs = oracle.quantize_int8(v.reshape(-1, D))
    return (k, q, kc.reshape(B, Hkv, T, D), ks.reshape(B, Hkv, T),
            vc.reshape(B, Hkv, T, D), vs.reshape(B, Hkv, T))


def _fl32_product(c, s):
    """fl32(c * s): the exact fp64 product rounded once to fp32, returned in fp64."""
    return (c.astype(np.float64) * s.astype(np.float64)[..., None]).astype(np.float32).astype(np.float64)


def _brute_force(q, kdeq_or_scores, vdeq, Hq, sigma, scores_given=False):
    """fp64 attention with the GQA broadcast written as the page's tensor idiom."""
    import torch
    qt = torch.tensor(q.astype(np.float64))
    V = torch.tensor(vdeq)
    B, Hkv, T, D = V.shape
    G = Hq // Hkv
    Ve = V.unsqueeze(2).expand(B, Hkv, G, T, D).reshape(B, Hq, T, D)
    if scores_given:
        sc = torch.tensor(kdeq_or_scores)
    else:
        K = torch.tensor(kdeq_or_scores)
        Ke = K.unsqueeze(2).expand(B, Hkv, G, T, D).reshape(B, Hq, T, D)
        sc = torch.einsum("bhd,bhtd->bht", qt, Ke)
    p = torch.softmax(sigma * sc, dim=-1)
    out = torch.einsum("bht,bhtd->bhd", p, Ve)
    return out.numpy(), sc.numpy(), p.numpy()


@pytest.mark.parametrize("T", [1, 5, 33])
def test_decode_int8_brute_force(T):
    k, q, kc, ks, vc, vs = _tiny_cache(T)
    r = oracle.decode_attention(q, k_codes=kc, k_scales=ks, v_codes=vc, v_scales=vs,
                                want_scores=True, want_probs=True)
    kdeq = _fl32_product(kc, ks)
    vdeq = _fl32_product(vc, vs)
    sigma = float(np.float32(1.0) / np.sqrt(np.float32(8)))
    out, sc, p = _brute_force(q, kdeq, vdeq, 4, sigma)
    assert np.allclose(r["scores"], sc, rtol=0, atol=1e-5)
    assert np.allclose(r["probs"], p, rtol=0, atol=1e-6)
    assert np.allclose(r["out"], out, rtol=0, atol=1e-5)
    # softmax rows sum to one
    assert np.all(np.abs(r["probs"].astype(np.float64).sum(-1) - 1) <= T * 2.0 ** -23)
    if T == 1:   # a single token: p = 1 exactly and the output is that token's values
        assert np.array_equal(r["out"], np.repeat(
            (vc.astype(np.float32) * vs[..., None])[:, :, 0], 2, axis=1))


@pytest.mark.parametrize("T", [1, 5, 33])
def test_decode_qjl_brute_force(T):
    k, q, _, _, vc, vs = _tiny_cache(T, D=8)
    S = inputs.sketch_matrix(32, 8, seed=3)
    B, Hkv, _, D = k.shape
    words, norms = oracle.qjl_encode(k.reshape(-1, D), S)
    words = words.reshape(B, Hkv, T, 1)
    norms = norms.reshape(B, Hkv, T)
    r = oracle.decode_attention(q, k_words=words, k_norms=norms, S=S, v_codes=vc, v_scales=vs,
                                want_scores=True, want_probs=True)
    # brute-force estimator scores from the definition, fp64, per (b, h, t)
    G = 4 // Hkv
    v = q.astype(np.float64) @ S.astype(np.float64).T                    # [B, Hq, m]
    v = v.astype(np.float32).astype(np.float64)                           # stored fp32
    bits = ((words[..., 0][..., None] >> np.arange(32, dtype=np.uint32)) & 1).astype(np.float64)
    sgn = 2 * bits - 1                                                   # [B, Hkv, T, 32]
    sgn_e = np.repeat(sgn, G, axis=1)
    nrm_e = np.repeat(norms.astype(np.float64), G, axis=1)
    sc = math.sqrt(math.pi / 2) / 32 * nrm_e * np.einsum("bhm,bhtm->bht", v, sgn_e)
    vdeq = _fl32_product(vc, vs)
    sigma = float(np.float32(1.0) / np.sqrt(np.float32(8)))
    out, _, p = _brute_force(q, sc, vdeq, 4, sigma, scores_given=True)
    assert np.allclose(r["scores"], sc, rtol=1e-6, atol=1e-6)
    assert np.allclose(r["probs"], p, rtol=0, atol=1e-6)
    assert np.allclose(r["out"], out, rtol=0, atol=1e-5)


@pytest.mark.parametrize("T,Hq,Hkv", [(1, 4, 2), (5, 4, 2), (33, 4, 1), (40, 6, 3)])
def test_decode_from_scores_pins(T, Hq, Hkv):
    """The fp64 definition after the scores (used as the reference of the arithmetic
    bound): equals the page's GQA broadcast in fp64 brute force; T = 1 gives the value
    row; equal scores give the mean of the values; it agrees with decode_attention's fp32
    output on the same scores within the fp32 summation error."""
    rng = np.random.default_rng(T + Hq)
    D = 8
    sc = rng.standard_normal((1, Hq, T)) * 30
    vdeq = rng.standard_normal((1, Hkv, T, D))
    sigma = float(np.float32(1.0) / np.sqrt(np.float32(D)))
    out, p = oracle.decode_from_scores(sc, vdeq)
    ref, _, pr = _brute_force(np.zeros((1, Hq, D)), sc, vdeq, Hq, sigma, scores_given=True)
    assert np.allclose(out, ref, rtol=0, atol=1e-13) and np.allclose(p, pr, rtol=0, atol=1e-15)
    if T == 1:
        assert np.array_equal(out[0], np.repeat(vdeq[0, :, 0], Hq // Hkv, axis=0))
    flat, _ = oracle.decode_from_scores(np.full((1, Hq, T), 2.5), vdeq)
    assert np.allclose(flat[0], np.repeat(vdeq[0].mean(axis=1), Hq // Hkv, axis=0), rtol=0, atol=1e-14)
    # against the C oracle's fp32 decode of an INT8 cache, on the C oracle's own scores
    k, q, kc, ks, vc, vs = _tiny_cache(T, D=D, Hq=Hq, Hkv=Hkv, seed=T)
    r = oracle.decode_attention(q, k_codes=kc, k_scales=ks, v_codes=vc, v_scales=vs, want_scores=True)
    o64, p64 = oracle.decode_from_scores(r["scores"], _fl32_product(vc, vs))
    vabs = np.repeat(np.abs(_fl32_product(vc, vs)), Hq // Hkv, axis=1)
    tol = (T + 4) * 2.0 ** -23 * np.einsum("bht,bhtd->bhd", p64, vabs) + 1e-30
    assert np.all(np.abs(r["out"] - o64) <= tol)


def test_decode_equal_logits_give_mean_of_values():
    T = 40
    _, q, kc, ks, vc, vs = _tiny_cache(T)
    q = np.zeros_like(q)                       # every score is 0
    r = oracle.decode_attention(q, k_codes=kc, k_scales=ks, v_codes=vc, v_scales=vs,
                                want_probs=True)
    assert np.all(r["probs"] == np.float32(1.0) / np.float32(T))
    vdeq = vc.astype(np.float64) * vs.astype(np.float64)[..., None]
    mean = np.repeat(vdeq.mean(axis=2), 2, axis=1)
    assert np.allclose(r["out"], mean, rtol=0, atol=1e-5)


def test_decode_gqa_group_mapping():
    """Query head h reads KV head h // G: give the two KV heads very different values."""
    T = 6
    k, q, kc, ks, vc, vs = _tiny_cache(T)
    vc = vc.copy()
    vc[:, 0] = 10
    vc[:, 1] = -10
    vs = np.ones_like(vs)
    r = oracle.decode_attention(q, k_codes=kc, k_scales=ks, v_codes=vc, v_scales=vs)
    assert np.allclose(r["out"][0, :2], 10) and np.allclose(r["out"][0, 2:], -10)


# ---- append-on-decode ----

def _append_case(T, cap, D=8, B=1, Hq=4, Hkv=2, seed=5):
    """A cache of `cap` rows per head holding T tokens (rows >= T filled with a sentinel)
    and a new token's key / value rows."""
    rng = np.random.default_rng(seed)
    full_k = rng.standard_normal((B, Hkv, T + 1, D)).astype(np.float16)
    full_v = rng.standard_normal((B, Hkv, T + 1, D)).astype(np.float16)
    q = rng.standard_normal((B, Hq, D)).astype(np.float16)
    kc = np.full((B, Hkv, cap, D), 77, np.int8)
    ks = np.full((B, Hkv, cap), 3.5, np.float32)
    vc = np.full((B, Hkv, cap, D), -77, np.int8)
    vs = np.full((B, Hkv, cap), 2.5, np.float32)
    if T > 0:
        c, s = oracle.quantize_int8(full_k[:, :, :T].reshape(-1, D))
        kc[:, :, :T], ks[:, :, :T] = c.reshape(B, Hkv, T, D), s.reshape(B, Hkv, T)
        c, s = oracle.quantize_int8(full_v[:, :, :T].reshape(-1, D))
        vc[:, :, :T], vs[:, :, :T] = c.reshape(B, Hkv, T, D), s.reshape(B, Hkv, T)
    return q, full_k, full_v, kc, ks, vc, vs


def test_decode_append_to_empty_cache_returns_the_new_value_row():
    """T = 0: one token, p = 1 exactly, so every query head returns its KV head's
    dequantized new value row, bit for bit."""
    q, fk, fv, kc, ks, vc, vs = _append_case(0, 3)
    r = oracle.decode_append(q, fk[:, :, 0], fv[:, :, 0], T=0, k_codes=kc, k_scales=ks,
                             v_codes=vc, v_scales=vs)
    c, s = oracle.quantize_int8(fv[:, :, 0].reshape(-1, 8))
    vhat = (c.astype(np.float32) * s[:, None]).reshape(1, 2, 8)
    assert np.array_equal(r["out"], np.repeat(vhat, 2, axis=1))


@pytest.mark.parametrize("T,cap", [(1, 2), (5, 9), (33, 34)])
def test_decode_append_int8_against_brute_force(T, cap):
    q, fk, fv, kc, ks, vc, vs = _append_case(T, cap)
    r = oracle.decode_append(q, fk[:, :, T], fv[:, :, T], T=T, k_codes=kc, k_scales=ks,
                             v_codes=vc, v_scales=vs, want_scores=True)
    # the appended rows are the per-row quantization of the new rows; nothing else moves
    c, s = oracle.quantize_int8(fk[:, :, T].reshape(-1, 8))
    assert np.array_equal(r["k_codes"][:, :, T], c.reshape(1, 2, 8))
    assert np.array_equal(r["k_scales"][:, :, T], s.reshape(1, 2))
    keep = np.ones(cap, bool)
    keep[T] = False
    assert np.array_equal(r["k_codes"][:, :, keep], kc[:, :, keep])
    assert np.array_equal(r["v_scales"][:, :, keep], vs[:, :, keep])
    # fp64 attention over all T + 1 tokens quantized from scratch
    kc_all, ks_all = oracle.quantize_int8(fk.reshape(-1, 8))
    vc_all, vs_all = oracle.quantize_int8(fv.reshape(-1, 8))
    kdeq = _fl32_product(kc_all.reshape(1, 2, T + 1, 8), ks_all.reshape(1, 2, T + 1))
    vdeq = _fl32_product(vc_all.reshape(1, 2, T + 1, 8), vs_all.reshape(1, 2, T + 1))
    sigma = float(np.float32(1.0) / np.sqrt(np.float32(8)))
    out, sc, _ = _brute_force(q, kdeq, vdeq, 4, sigma)
    assert np.allclose(r["scores"], sc, rtol=0, atol=1e-5)
    assert np.allclose(r["out"], out, rtol=0, atol=1e-5)


def test_decode_append_qjl_against_brute_force():
    T, cap = 7, 8
    q, fk, fv, _, _, vc, vs = _append_case(T, cap, seed=9)
    S = inputs.sketch_matrix(32, 8, seed=3)
    w, n = oracle.qjl_encode(fk[:, :, :T].reshape(-1, 8), S)
    kw = np.zeros((1, 2, cap, 1), np.uint32)
    kn = np.zeros((1, 2, cap), np.float16)
    kw[:, :, :T] = w.reshape(1, 2, T, 1)
    kn[:, :, :T] = n.reshape(1, 2, T)
    r = oracle.decode_append(q, fk[:, :, T], fv[:, :, T], T=T, k_words=kw, k_norms=kn, S=S,
                             v_codes=vc, v_scales=vs, want_scores=True)
    # estimator scores from the definition over all T + 1 keys, sketched from scratch
    w_all, n_all = oracle.qjl_encode(fk.reshape(-1, 8), S)
    assert np.array_equal(r["k_words"][:, :, :T + 1].reshape(-1), w_all.reshape(-1))
    assert np.array_equal(r["k_norms"][:, :, :T + 1].reshape(-1).view(np.uint16),
                          n_all.reshape(-1).view(np.uint16))
    v = (q.astype(np.float64) @ S.astype(np.float64).T).astype(np.float32).astype(np.float64)
    bits = ((w_all.reshape(1, 2, T + 1)[..., None] >> np.arange(32, dtype=np.uint32)) & 1)
    sgn = np.repeat(2.0 * bits - 1, 2, axis=1)
    nrm = np.repeat(n_all.reshape(1, 2, T + 1).astype(np.float64), 2, axis=1)
    sc = math.sqrt(math.pi / 2) / 32 * nrm * np.einsum("bhm,bhtm->bht", v, sgn)
    assert np.allclose(r["scores"], sc, rtol=1e-6, atol=1e-6)


# ---- channel-wise INT8 and group-wise INT4 ----

@pytest.mark.parametrize("dtype", [np.float16, np.float32])
def test_channelwise_int8_is_the_row_rule_on_the_transpose(dtype):
    """One scale per column of each block = the pinned per-row rule applied to the
    block's transpose (codes and scales bit for bit; dequantized values too)."""
    rng = np.random.default_rng(21)
    x = (rng.standard_normal((3, 37, 24)) * rng.lognormal(0, 1, (3, 1, 24))).astype(dtype)
    x[1, :, 5] = 0                                   # an all-zero column: scale 0, codes 0
    codes, scales = oracle.quantize_int8_channelwise(x)
    deq = oracle.dequantize_int8_channelwise(codes, scales)
    for b in range(3):
        c_t, s_t = oracle.quantize_int8(np.ascontiguousarray(x[b].T))
        assert np.array_equal(codes[b], c_t.T)
        assert np.array_equal(scales[b].view(np.uint32), s_t.view(np.uint32))
        assert np.array_equal(deq[b].view(np.uint32), oracle.dequantize_int8(c_t, s_t).T.view(np.uint32))
    assert np.all(codes[1, :, 5] == 0) and scales[1, 5] == 0


def _hex32(h):
    return np.float32(float.fromhex(h))


def test_int4_worked_examples():
    spec = json.load(open(os.path.join(GOLDEN, "int4_worked_examples.json")))
    for ex in spec["examples"]:
        x = np.array([ex["x"]], np.float32)
        g = ex["group"]
        packed, s, z = oracle.quantize_int4_group(x, g)
        assert s[0, 0] == _hex32(ex["scale_hex"]), ex["name"]
        assert z[0, 0] == np.float32(ex["zero"]), ex["name"]
        assert list(packed[0]) == ex["packed"], ex["name"]
        lo, hi = packed[0] & 0xF, packed[0] >> 4
        assert list(np.stack([lo, hi], 1).reshape(-1)) == ex["codes"], ex["name"]
        xh = oracle.dequantize_int4_group(packed, s, z, g)[0]
        want = ([_hex32(h) for h in ex["x_hat_hex"]] if "x_hat_hex" in ex
                else [np.float32(v) for v in ex["x_hat"]])
        assert np.array_equal(xh, np.array(want, np.float32)), ex["name"]
    # the tie case: the exact quotient 1.5 / s4 is below 7.5, the fp32 one is 7.5
    s4 = float(_hex32("0x1.99999ap-3"))
    assert Fraction(3, 2) / Fraction(s4) < Fraction(15, 2)
    assert np.float32(np.float32(1.5) / np.float32(s4)) == np.float32(7.5)


@pytest.mark.parametrize("dtype,g", [(np.float16, 32), (np.float32, 64), (np.float16, 128)])
def test_int4_invariants(dtype, g):
    rng = np.random.default_rng(31)
    x = (rng.standard_normal((50, 256)) * 3 + rng.standard_normal((50, 1))).astype(dtype)
    packed, s, z = oracle.quantize_int4_group(x, g)
    codes = np.stack([packed & 0xF, packed >> 4], -1).reshape(50, 256)
    xg = x.astype(np.float64).reshape(50, -1, g)
    cg = codes.reshape(50, -1, g)
    # the minimum maps to 0, the maximum to 15, the zero point is the minimum
    assert np.all(np.take_along_axis(cg, xg.argmin(-1)[..., None], -1) == 0)
    assert np.all(np.take_along_axis(cg, xg.argmax(-1)[..., None], -1) == 15)
    assert np.array_equal(z, xg.min(-1).astype(np.float32))
    # reconstruction error: half a step, plus the fp32 roundings of the quotient and of
    # the reconstruction (a few ulps of the group's magnitude)
    xh = oracle.dequantize_int4_group(packed, s, z, g).astype(np.float64).reshape(50, -1, g)
    mag = np.abs(xg).max(-1, keepdims=True)
    slack = s.astype(np.float64)[..., None] * 2.0 ** -19 + 4 * mag * 2.0 ** -23
    assert np.all(np.abs(xh - xg) <= s.astype(np.float64)[..., None] / 2 + slack)
    # groups are independent: each group quantized as a row of its own
    p1, s1, z1 = oracle.quantize_int4_group(np.ascontiguousarray(x.reshape(-1, g)), g)
    assert np.array_equal(p1.reshape(packed.shape), packed)
    assert np.array_equal(s1.reshape(s.shape), s) and np.array_equal(z1.reshape(z.shape), z)


def test_decode_int4_values_against_brute_force():
    T, g = 9, 4
    _, q, kc, ks, _, _ = _tiny_cache(T)
    rng = np.random.default_rng(12)
    v = rng.standard_normal((1, 2, T, 8)).astype(np.float16)
    packed, s, z = oracle.quantize_int4_group(v.reshape(-1, 8), g)
    v4 = (packed.reshape(1, 2, T, 4), s.reshape(1, 2, T, 2), z.reshape(1, 2, T, 2), g)
    r = oracle.decode_attention(q, k_codes=kc, k_scales=ks, v4=v4)
    vdeq = oracle.dequantize_int4_group(packed, s, z, g).astype(np.float64).reshape(1, 2, T, 8)
    kdeq = _fl32_product(kc, ks)
    sigma = float(np.float32(1.0) / np.sqrt(np.float32(8)))
    out, _, _ = _brute_force(q, kdeq, vdeq, 4, sigma)
    assert np.allclose(r["out"], out, rtol=0, atol=1e-5)


# ---- attention-sink eviction ----

def test_eviction_worked_examples():
    spec = json.load(open(os.path.join(GOLDEN, "eviction_example.json")))
    for ex in spec["examples"]:
        mass = np.array([ex["mass"]], np.float32)
        kept = oracle.evict_select(mass, ex["n_sink"], ex["n_keep"])
        assert list(kept[0]) == ex["kept"], ex["name"]


def test_eviction_invariants():
    rng = np.random.default_rng(41)
    mass = rng.exponential(1.0, (5, 300)).astype(np.float32)
    mass[:, 100:110] = mass[:, 100:101]            # runs of equal masses
    kept = oracle.evict_select(mass, 4, 120)
    for b in range(5):
        k = kept[b]
        assert np.all(np.diff(k) > 0) and list(k[:4]) == [0, 1, 2, 3]
        evicted = np.setdiff1d(np.arange(4, 300), k)
        assert mass[b, k[4:]].min() >= mass[b, evicted].max()
        # at the cut, the kept equal masses are the smallest indices
        cut = mass[b, k[4:]].min()
        eq_kept = k[4:][mass[b, k[4:]] == cut]
        eq_evicted = evicted[mass[b, evicted] == cut]
        assert eq_evicted.size == 0 or eq_kept.max() < eq_evicted.min()


def test_attention_mass_sums_to_heads():
    """Each query head's probabilities sum to one, so one step's mass sums to Hq."""
    T = 33
    _, q, kc, ks, vc, vs = _tiny_cache(T)
    m = oracle.attention_mass(q, k_codes=kc, k_scales=ks)
    assert m.shape == (1, T)
    assert abs(m.sum() - 4) <= 4 * T * 2.0 ** -23
    # equal logits: every token gets Hq / T
    m0 = oracle.attention_mass(np.zeros_like(q), k_codes=kc, k_scales=ks)
    assert np.allclose(m0, 4.0 / T, rtol=1e-6)


def test_gather_rows_keeps_order():
    cache = np.arange(2 * 3 * 8 * 2).reshape(2, 3, 8, 2)
    kept = np.array([[0, 1, 5], [2, 3, 7]], np.int32)
    g = oracle.gather_rows(cache, kept)
    assert g.shape == (2, 3, 3, 2)
    assert np.array_equal(g[1, 2, 2], cache[1, 2, 7])


# ---- QJL as the 1-bit residual of group-wise INT4 ("TurboQuant" news page) ----

def _grid_keys(n, d=128, g=32, seed=0):
    """Keys exactly on an INT4 grid: per group z + c * s with s a power of two, codes
    0..15 and both ends present, all representable in fp16."""
    rng = np.random.default_rng(seed)
    keys = np.empty((n, d), np.float64)
    for r in range(n):
        for k in range(d // g):
            z = rng.integers(-64, 64) / 16.0
            s = 2.0 ** rng.integers(-5, 0)
            c = rng.integers(0, 16, g)
            c[rng.integers(0, g)] = 0
            c[(rng.integers(1, g) + np.argmin(c)) % g] = 15
            keys[r, k * g:(k + 1) * g] = z + c * s
    k16 = keys.astype(np.float16)
    assert np.array_equal(k16.astype(np.float64), keys)
    return k16


def test_qjlres_zero_residual_closed_form():
    """Keys on the INT4 grid: the residual is exactly 0, its norm is 0, every sign bit is
    set (bit = [u >= 0]) and the score is the exact dot product <q, k> in fp32."""
    k = _grid_keys(6)
    S = inputs.sketch_matrix(256, 128)
    e = oracle.qjl_residual_encode(k, 32, S, want_r=True)
    assert not np.any(e["r"].astype(np.float64))
    assert not np.any(e["rnorms"].astype(np.float64))
    assert np.all(e["words"] == 0xFFFFFFFF)
    q = inputs.gaussian_queries(9, 1, 2)
    k4 = (e["packed"].reshape(1, 1, 6, 64), e["scales"].reshape(1, 1, 6, 4), e["zeros"].reshape(1, 1, 6, 4), 32)
    r = oracle.decode_attention(q, k4=k4, k_words=e["words"].reshape(1, 1, 6, 8), k_norms=e["rnorms"].reshape(1, 1, 6),
                                S=S, want_out=False, want_scores=True)
    exact = (q.astype(np.float64)[0] @ k.astype(np.float64).T).astype(np.float32)
    assert np.array_equal(r["scores"][0], exact)


@pytest.mark.parametrize("g", [32, 64, 128])
def test_qjlres_decomposition(g):
    """The INT4 stage is the standalone group-wise INT4 quantizer; k_hat + r reproduces k
    to within half an fp16 ulp of r; the stored norm is fp16 of numpy's norm of r; the
    sign bits are those of numpy's S @ r away from zero."""
    k, = inputs.lognormal_cache(21, 1, 2, 40, n_tensors=1)
    k = k.reshape(-1, 128)
    S = inputs.sketch_matrix(256, 128)
    e = oracle.qjl_residual_encode(k, g, S, want_r=True)
    p, s, z = oracle.quantize_int4_group(k, g)
    assert np.array_equal(e["packed"], p) and np.array_equal(e["scales"], s) and np.array_equal(e["zeros"], z)
    khat = oracle.dequantize_int4_group(p, s, z, g).astype(np.float64)
    r = e["r"].astype(np.float64)
    half_ulp = np.spacing(np.abs(e["r"]).astype(np.float16)).astype(np.float64) / 2
    assert np.all(np.abs(k.astype(np.float64) - khat - r) <= half_ulp + 2.0 ** -24 * np.abs(k.astype(np.float64)))
    assert np.any(r)
    assert np.array_equal(e["rnorms"], np.linalg.norm(r, axis=1).astype(np.float16))
    u = r @ S.astype(np.float64).T
    bits = ((e["words"][:, :, None] >> np.arange(32, dtype=np.uint32)) & 1).reshape(len(k), -1).astype(bool)
    far = np.abs(u) > 1e-9 * np.linalg.norm(r, axis=1, keepdims=True)
    assert np.array_equal(bits[far], (u >= 0)[far])


def test_qjlres_unbiased_and_tighter_than_plain_qjl():
    """Over 1000 independent Gaussian sketches the residual score's mean lies within 3
    standard errors of <q, k_hat + r> (about <q, k>), and its spread is at most
    1.3 * ||r|| / ||k|| of the plain QJL estimator's on the same sketches."""
    k, = inputs.lognormal_cache(31, 1, 1, 1, n_tensors=1)
    k = k.reshape(1, 128)
    q = inputs.gaussian_queries(41, 1, 1)
    e0 = oracle.qjl_residual_encode(k, 32, inputs.sketch_matrix(256, 128), want_r=True)
    khat = oracle.dequantize_int4_group(e0["packed"], e0["scales"], e0["zeros"], 32).astype(np.float64)
    r = e0["r"].astype(np.float64)
    target = float(q[0, 0].astype(np.float64) @ (khat[0] + r[0]))
    exact = float(q[0, 0].astype(np.float64) @ k[0].astype(np.float64))
    assert abs(target - exact) <= 1e-3 * np.abs(q[0, 0].astype(np.float64) * k[0]).sum()
    res, plain = [], []
    for seed in range(20000, 21000):
        S = inputs.sketch_matrix_f64(256, 128, seed)
        e = oracle.qjl_residual_encode(k, 32, S)
        k4 = (e["packed"].reshape(1, 1, 1, 64), e["scales"].reshape(1, 1, 1, 4), e["zeros"].reshape(1, 1, 1, 4), 32)
        sc = oracle.decode_attention(q, k4=k4, k_words=e["words"].reshape(1, 1, 1, 8),
                                     k_norms=e["rnorms"].reshape(1, 1, 1), S=S, want_out=False, want_scores=True)
        res.append(float(sc["scores"][0, 0, 0]))
        w, n = oracle.qjl_encode(k, S)
        v64, _ = oracle.qjl_query_sketch(q[0], S)
        plain.append(oracle.qjl_estimate(v64[0], w[0], float(n[0])))
    res, plain = np.array(res), np.array(plain)
    se = res.std(ddof=1) / math.sqrt(len(res))
    assert abs(res.mean() - target) <= 3 * se, (res.mean(), target, se)
    ratio = np.linalg.norm(r[0]) / np.linalg.norm(k[0].astype(np.float64))
    assert ratio < 0.5
    assert res.std() <= 1.3 * ratio * plain.std(), (res.std(), plain.std(), ratio)
