"""GPU parity of QJL as the 1-bit residual of group-wise INT4 (keys: INT4 codes + the
residual's sign sketch; the "TurboQuant" news page's two stages) against the CPU oracle.

- Encode: INT4 codes, scales, zero points, the fp16 residual and its fp16 norm
  bit-exact; sign bits exact except where the oracle's |(S r)_i| < 1e-4 ||r|| (the GPU
  projects in fp32 on the tensor cores).
- Decode (same encoded cache on both sides): outputs max-abs <= 2e-3 and within the
  arithmetic bound (tests/_helpers.py, check_decode_bound); scores within
  32 * 2^-24 * sum_j |q_j| (|c_j s_g| + |z_g|) (fp32 factored INT4 dot against the
  oracle's fp64 sum of rounded reconstructions) + 1e-4 * c ||r|| ||S q||_2 (the
  residual estimator's natural scale, as for QJL keys).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from kv_cache_quantization_absmax_b200 import inputs
from tests import _oracle_pool
from tests._helpers import (check_decode_bound, check_decode_unit, decode_chain, sm_count, softmax_scale, to_np,
                            words_u32)

pytestmark = pytest.mark.gpu

OUT_TOL = 2e-3


@pytest.fixture(scope="module")
def kvq():
    from kv_cache_quantization_absmax_b200 import kvq as m
    return m


def _cuda(*arrs):
    return [torch.from_numpy(np.ascontiguousarray(a)).cuda() for a in arrs]


@pytest.mark.parametrize("n,g,m", [(1, 32, 256), (127, 32, 256), (1000, 64, 256), (300, 128, 128),
                                   (4097, 32, 128), (70000, 32, 256)])
def test_qjlres_encode_parity(kvq, n, g, m):
    k, = inputs.lognormal_cache(800 + n, 1, 1, n, n_tensors=1)
    k = k.reshape(n, 128)
    S = inputs.sketch_matrix(m, 128)
    ref = oracle.qjl_residual_encode(k, g, S, want_r=True, want_u=True)
    kg, Sg = _cuda(k, S)
    o = kvq.kvq_qjl_residual_encode(kg, g, Sg)
    assert np.array_equal(to_np(o["packed"]), ref["packed"])
    assert np.array_equal(to_np(o["scales"]), ref["scales"])
    assert np.array_equal(to_np(o["zeros"]), ref["zeros"])
    assert np.array_equal(to_np(o["residual"]).view(np.uint16), ref["r"].view(np.uint16))
    assert np.array_equal(to_np(o["rnorms"]).view(np.uint16), ref["rnorms"].view(np.uint16))
    gw = words_u32(o["words"])
    diff = gw ^ ref["words"]
    bits = ((diff[:, :, None] >> np.arange(32, dtype=np.uint32)) & 1).reshape(n, m).astype(bool)
    band = np.abs(ref["u"]) < 1e-4 * np.linalg.norm(ref["r"].astype(np.float64), axis=1, keepdims=True)
    assert not np.any(bits & ~band)
    assert kvq.kvq_device_error() == 0


def _res_cache(seed, B, Hkv, T, Hq, g=32, m=256):
    k, v = inputs.lognormal_cache(seed, B, Hkv, T, n_tensors=2)
    q = inputs.gaussian_queries(seed + 1, B, Hq)
    S = inputs.sketch_matrix(m, 128)
    e = oracle.qjl_residual_encode(k.reshape(-1, 128), g, S)
    vc, vs = oracle.quantize_int8(v.reshape(-1, 128))
    shp = (B, Hkv, T)
    c = dict(k4=(e["packed"].reshape(shp + (64,)), e["scales"].reshape(shp + (128 // g,)),
                 e["zeros"].reshape(shp + (128 // g,)), g),
             k_words=e["words"].reshape(shp + (m // 32,)), k_norms=e["rnorms"].reshape(shp), S=S,
             v_codes=vc.reshape(shp + (128,)), v_scales=vs.reshape(shp))
    return q, c


def _gpu(c):
    p4, s4, z4, g = c["k4"]
    pg, sg, zg, wg, ng, Sg, vcg, vsg = _cuda(p4, s4, z4, c["k_words"].view(np.int32), c["k_norms"], c["S"],
                                            c["v_codes"], c["v_scales"])
    return dict(k_packed4=pg, k_scales4=sg, k_zeros4=zg, k_group=g, k_words=wg, k_norms=ng, sketch=Sg,
                v_codes=vcg, v_scales=vsg)


def _score_tol(q, c, Hq):
    p4, s4, z4, g = c["k4"]
    B, Hkv, T, _ = p4.shape
    G = Hq // Hkv
    codes = np.stack([p4 & 0xF, p4 >> 4], axis=-1).reshape(B, Hkv, T, 128).astype(np.float64)
    sc = np.repeat(s4.astype(np.float64), g, axis=-1)
    zr = np.repeat(np.abs(z4.astype(np.float64)), g, axis=-1)
    mag = np.abs(codes * sc) + zr                                   # [B, Hkv, T, D]
    qa = np.abs(q.astype(np.float64))                               # [B, Hq, D]
    t_int4 = 32 * 2.0 ** -24 * np.einsum("bhd,bhtd->bht", qa, np.repeat(mag, G, axis=1))
    m = c["S"].shape[0]
    v64, _ = oracle.qjl_query_sketch(q.reshape(-1, 128), c["S"])
    vn = np.linalg.norm(v64, axis=1).reshape(B, Hq, 1)
    rn = np.repeat(c["k_norms"].astype(np.float64), G, axis=1)
    t_res = 1e-4 * math.sqrt(math.pi / 2) / m * rn * vn
    return t_int4 + t_res


@pytest.mark.parametrize("B,Hq,Hkv,T,g,m", [(1, 1, 1, 1, 32, 256), (1, 4, 1, 7, 32, 256), (2, 8, 2, 1500, 32, 256),
                                            (1, 32, 8, 2049, 64, 256), (1, 4, 4, 700, 128, 128),
                                            (1, 2, 1, 333, 32, 128), (16, 32, 8, 3, 32, 256),
                                            (4, 8, 4, 100, 64, 256), (2, 4, 4, 4100, 32, 256)])
def test_decode_qjlres_parity(kvq, B, Hq, Hkv, T, g, m):
    q, c = _res_cache(900 + T, B, Hkv, T, Hq, g, m)
    ref = oracle.decode_attention(q, want_scores=True, **c)
    out, scores = kvq.kvq_decode_attention_qjlres(_cuda(q)[0], want_scores=True, **_gpu(c))
    assert np.abs(to_np(out) - ref["out"]).max() <= OUT_TOL
    err = np.abs(to_np(scores).astype(np.float64) - ref["scores"])
    tol = _score_tol(q, c, Hq)
    assert np.all(err <= tol), float((err / tol).max())
    vc, vs = c["v_codes"], c["v_scales"]
    vals = oracle.dequantize_int8(vc.reshape(-1, 128), vs.reshape(-1)).reshape(vc.shape)
    check_decode_bound(to_np(out), to_np(scores), ref["scores"], vals, qjl=True)
    assert kvq.kvq_device_error() == 0


def test_decode_qjlres_scores_only(kvq):
    q, c = _res_cache(950, 2, 4, 3000, 8)
    ref = oracle.decode_attention(q, want_out=False, want_scores=True, **c)
    gk = _gpu(c)
    gk.pop("v_codes"), gk.pop("v_scales")
    for _ in range(2):
        out, scores = kvq.kvq_decode_attention_qjlres(_cuda(q)[0], want_out=False, want_scores=True, **gk)
        assert out is None
        err = np.abs(to_np(scores).astype(np.float64) - ref["scores"])
        assert np.all(err <= _score_tol(q, c, 8))


def test_decode_qjlres_beats_plain_qjl_on_scores(kvq):
    """The residual estimator's scores are closer to the exact <q, k> than plain QJL's on
    the same sketch matrix (GPU encode and decode, mean absolute error)."""
    B, Hq, Hkv, T = 1, 8, 2, 2048
    k, v = inputs.lognormal_cache(960, B, Hkv, T, n_tensors=2)
    q = inputs.gaussian_queries(961, B, Hq)
    S = torch.from_numpy(inputs.sketch_matrix(256, 128)).cuda()
    kg, qg = _cuda(k, q)
    vc, vs = kvq.kvq_quantize_int8(_cuda(v)[0])
    e = kvq.kvq_qjl_residual_encode(kg, 32, S)
    _, s_res = kvq.kvq_decode_attention_qjlres(qg, k_packed4=e["packed"], k_scales4=e["scales"],
                                               k_zeros4=e["zeros"], k_group=32, k_words=e["words"],
                                               k_norms=e["rnorms"], sketch=S, v_codes=vc, v_scales=vs,
                                               want_scores=True)
    w, n = kvq.kvq_qjl_encode(kg, S)
    _, s_qjl = kvq.kvq_decode_attention(qg, k_words=w, k_norms=n, sketch=S, v_codes=vc, v_scales=vs,
                                        want_scores=True)
    exact = np.einsum("bhd,bhtd->bht", np.repeat(q.astype(np.float64), 1, axis=1),
                      np.repeat(k.astype(np.float64), Hq // Hkv, axis=1))
    e_res = np.abs(to_np(s_res) - exact).mean()
    e_qjl = np.abs(to_np(s_qjl) - exact).mean()
    assert e_res < 0.5 * e_qjl, (e_res, e_qjl)


def test_qjlres_gqa_long_context_all_units(kvq):
    """Long-context GQA cache (batch 4, 32 query / 8 KV heads, 131072 tokens): keys
    encoded as INT4 + residual sketch and values INT8-quantized on the GPU, one decode
    step.  Every one of the 32 KV units is re-done end to end by the oracle from the fp16
    cache (in spawned worker processes): the INT4 stage and residual norms bit-exact, sign
    bits exact outside the band, scores within their tolerance wherever both sides hold
    the same bits, outputs within 2e-3 and within the arithmetic bound."""
    B, Hq, Hkv, T = 4, 32, 8, 131072
    G = Hq // Hkv
    kv = inputs.lognormal_cache_device(5, (2, B, Hkv, T, 128), n_sigma_dims=(0, 2, 4), device="cuda")
    q = inputs.gaussian_queries_device(50, (B, Hq, 128), "cuda")
    S_np = inputs.sketch_matrix(256, 128)
    S = torch.from_numpy(S_np).cuda()
    e = kvq.kvq_qjl_residual_encode(kv[0], 32, S)
    vc, vs = kvq.kvq_quantize_int8(kv[1])
    out, scores = kvq.kvq_decode_attention_qjlres(q, k_packed4=e["packed"], k_scales4=e["scales"],
                                                  k_zeros4=e["zeros"], k_group=32, k_words=e["words"],
                                                  k_norms=e["rnorms"], sketch=S, v_codes=vc, v_scales=vs,
                                                  want_scores=True)
    out, scores = to_np(out), to_np(scores)
    assert kvq.kvq_device_error() == 0
    q_np = to_np(q)
    units = [(b, g) for b in range(B) for g in range(Hkv)]
    jobs = [(to_np(kv[0, b, g]), to_np(kv[1, b, g]), q_np[b, g * G:(g + 1) * G], S_np, 32) for b, g in units]
    del kv
    refs = _oracle_pool.run_units(_oracle_pool.qjlres_unit, jobs)
    n_chain, n_rescale = decode_chain(B, Hkv, T, Hq, sm_count(), qjl=True)
    for (b, g), job, r in zip(units, jobs, refs):
        assert np.array_equal(to_np(e["packed"][b, g]), r["packed"])
        assert np.array_equal(to_np(e["scales"][b, g]).view(np.uint32), r["scales"].view(np.uint32))
        assert np.array_equal(to_np(e["zeros"][b, g]).view(np.uint32), r["zeros"].view(np.uint32))
        assert np.array_equal(to_np(e["rnorms"][b, g]).view(np.uint16), r["rnorms"].view(np.uint16))
        assert np.array_equal(to_np(e["residual"][b, g]).view(np.uint16), r["r"].view(np.uint16))
        assert np.array_equal(to_np(vc[b, g]), r["v_codes"])
        assert np.array_equal(to_np(vs[b, g]).view(np.uint32), r["v_scales"].view(np.uint32))
        gw = words_u32(e["words"][b, g])
        same = np.all(gw == r["words"], axis=1)
        if not np.all(same):
            t_diff = np.flatnonzero(~same)
            resid = r["r"][t_diff]
            u = resid.astype(np.float64) @ S_np.astype(np.float64).T
            n64 = np.linalg.norm(resid.astype(np.float64), axis=1)
            band = np.abs(u) < 1e-4 * n64[:, None]
            diff = gw[t_diff] ^ r["words"][t_diff]
            bits = ((diff[:, :, None] >> np.arange(32, dtype=np.uint32)) & 1).reshape(len(t_diff), 256).astype(bool)
            assert not np.any(bits & ~band)
        hs = slice(g * G, (g + 1) * G)
        c = dict(k4=(r["packed"][None, None], r["scales"].reshape(1, 1, T, 4), r["zeros"].reshape(1, 1, T, 4), 32),
                 k_words=r["words"][None, None], k_norms=r["rnorms"][None, None], S=S_np)
        tol = _score_tol(job[2][None], c, G)[0]
        err = np.abs(scores[b, hs].astype(np.float64) - r["scores"])
        assert np.all(err[:, same] <= tol[:, same])
        assert np.abs(out[b, hs] - r["out"]).max() <= OUT_TOL
        check_decode_unit(out[b, hs], scores[b, hs], r["scores"], oracle.dequantize_int8(r["v_codes"], r["v_scales"]),
                          softmax_scale(), n_chain, n_rescale)
