"""GPU parity of the fused decode step (scores -> softmax -> sum of INT8 values) against
the CPU oracle, for INT8 keys and QJL keys, MHA, GQA and MQA.

Decode outputs, two bars for every element:
  * the spec line: max-abs error <= 2e-3 against the oracle's fp32-accumulated result;
  * the bound derived from the kernels' arithmetic (tests/_helpers.py, check_decode_bound)
    against the oracle's fp64 softmax-weighted sum over the oracle's scores, which a lost
    or misplaced 128-token chunk exceeds even at 131072 tokens.
INT8 raw scores: the fp32 summation bound.  QJL estimator scores (same sign words and
norms on both sides): 1e-4 relative to max(|score|, c ||k|| ||S q||_2).
"""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_quantization_absmax_b200 import inputs
from tests import _oracle_pool
from tests._helpers import (bit_mismatch_outside_band, check_decode_bound, check_decode_unit, decode_chain,
                            score_tolerance, sm_count, softmax_scale, to_np, words_u32)

pytestmark = pytest.mark.gpu

OUT_TOL = 2e-3


@pytest.fixture(scope="module")
def kvq():
    from kv_cache_quantization_absmax_b200 import kvq as m
    return m


def _vals(vc, vs):
    """Dequantized value rows [B, Hkv, T, D] (the oracle's fl32(c * s))."""
    return oracle.dequantize_int8(vc.reshape(-1, vc.shape[-1]), vs.reshape(-1)).reshape(vc.shape)


def _int8_cache(seed, B, Hkv, T, Hq):
    k, v = inputs.lognormal_cache(seed, B, Hkv, T, n_tensors=2)
    q = inputs.gaussian_queries(seed + 1, B, Hq)
    kc, ks = oracle.quantize_int8(k.reshape(-1, 128))
    vc, vs = oracle.quantize_int8(v.reshape(-1, 128))
    shp = (B, Hkv, T)
    return q, kc.reshape(shp + (128,)), ks.reshape(shp), vc.reshape(shp + (128,)), vs.reshape(shp)


def _cuda(*arrs):
    return [torch.from_numpy(np.ascontiguousarray(a)).cuda() for a in arrs]


def _int8_score_bound(q, kc, ks, G):
    xh = kc.astype(np.float64) * ks.astype(np.float64)[..., None]
    terms = np.abs(np.repeat(xh, G, axis=1) * q.astype(np.float64)[:, :, None, :]).sum(-1)
    return 2 * 128 * 2.0 ** -24 * terms + 1e-30


# MHA, GQA (G = 2, 4, 8, and G = 3, 6 that are not powers of two), MQA (Hkv = 1, G up to
# 32: query heads split over several CTAs per token range).  Contexts of 512 tokens and
# more take the tensor-core kernel (128-token chunks, partial chunks at range and unit
# edges, ranges over up to four units): G = 1 .. 8 and MQA among them.
@pytest.mark.parametrize("B,Hq,Hkv,T", [(1, 1, 1, 1), (1, 4, 4, 5), (2, 8, 2, 33), (1, 8, 1, 1000),
                                        (2, 16, 4, 4097), (1, 8, 8, 300), (1, 16, 2, 2500),
                                        (16, 16, 8, 3), (4, 8, 8, 100), (3, 24, 3, 70),
                                        (1, 16, 1, 1000), (2, 32, 1, 700), (1, 32, 2, 3000),
                                        (1, 12, 2, 500), (2, 6, 2, 301), (2, 4, 4, 1030),
                                        (1, 2, 1, 777), (3, 6, 3, 2000), (8, 8, 8, 600)])
def test_decode_int8_parity(kvq, B, Hq, Hkv, T, flags=0):
    q, kc, ks, vc, vs = _int8_cache(10 + T, B, Hkv, T, Hq)
    ref = oracle.decode_attention(q, k_codes=kc, k_scales=ks, v_codes=vc, v_scales=vs,
                                  want_scores=True)
    qg, kcg, ksg, vcg, vsg = _cuda(q, kc, ks, vc, vs)
    out, scores = kvq.kvq_decode_attention(qg, k_codes=kcg, k_scales=ksg, v_codes=vcg,
                                           v_scales=vsg, want_scores=True, flags=flags)
    out, scores = to_np(out), to_np(scores)
    assert np.abs(out - ref["out"]).max() <= OUT_TOL
    # raw scores: fp32 summation bound on the same codes (the tensor-core kernel's exact
    # fixed-point sums, from a query rounded by at most 2^-22 max |q|, stay well inside it)
    assert np.all(np.abs(scores.astype(np.float64) - ref["scores"]) <= _int8_score_bound(q, kc, ks, Hq // Hkv))
    check_decode_bound(out, scores, ref["scores"], _vals(vc, vs), qjl=False)


@pytest.mark.parametrize("B,Hq,Hkv,T", [(2, 16, 4, 4097), (1, 16, 1, 1000), (2, 4, 4, 1030)])
def test_decode_int8_cuda_cores_flag_parity(kvq, B, Hq, Hkv, T):
    """KVQ_DECODE_CUDA_CORES on shapes that would take the tensor-core kernel: scores and
    weighted sum in fp32 on the CUDA cores, against the same oracle and bounds."""
    test_decode_int8_parity(kvq, B, Hq, Hkv, T, flags=kvq.KVQ_DECODE_CUDA_CORES)


def test_decode_scores_only_outlier_layer(kvq):
    """The one-layer INT8 cache with outlier channels: scores of one fp16 query per head
    against the dequantized keys (no value pass)."""
    k, v, q = inputs.outlier_layer(seed=0)
    kc, ks = oracle.quantize_int8(k.reshape(-1, 128))
    kc, ks = kc.reshape(k.shape), ks.reshape(k.shape[:-1])
    ref = oracle.decode_attention(q, k_codes=kc, k_scales=ks, want_out=False, want_scores=True)
    qg, kcg, ksg = _cuda(q, kc, ks)
    out, scores = kvq.kvq_decode_attention(qg, k_codes=kcg, k_scales=ksg, want_out=False,
                                           want_scores=True)
    assert out is None
    assert np.all(np.abs(to_np(scores).astype(np.float64) - ref["scores"]) <= _int8_score_bound(q, kc, ks, 1))


def _qjl_cache(seed, B, Hkv, T, Hq, m=256):
    k, v = inputs.lognormal_cache(seed, B, Hkv, T, n_tensors=2)
    q = inputs.gaussian_queries(seed + 1, B, Hq)
    S = inputs.sketch_matrix(m, 128)
    w, n = oracle.qjl_encode(k.reshape(-1, 128), S)
    vc, vs = oracle.quantize_int8(v.reshape(-1, 128))
    shp = (B, Hkv, T)
    return q, S, w.reshape(shp + (m // 32,)), n.reshape(shp), vc.reshape(shp + (128,)), vs.reshape(shp)


@pytest.mark.parametrize("B,Hq,Hkv,T,m", [(1, 1, 1, 1, 256), (1, 4, 1, 7, 256), (2, 8, 2, 1500, 256),
                                          (1, 32, 8, 2049, 256), (1, 4, 4, 700, 128), (1, 2, 1, 333, 32),
                                          (16, 32, 8, 3, 256), (4, 8, 4, 100, 256),
                                          (2, 16, 1, 1000, 256), (1, 12, 2, 801, 256), (1, 3, 1, 257, 64)])
def test_decode_qjl_parity(kvq, B, Hq, Hkv, T, m, flags=0):
    q, S, w, n, vc, vs = _qjl_cache(100 + T, B, Hkv, T, Hq, m)
    ref = oracle.decode_attention(q, k_words=w, k_norms=n, S=S, v_codes=vc, v_scales=vs,
                                  want_scores=True)
    qg, Sg, wg, ng, vcg, vsg = _cuda(q, S, w.view(np.int32), n, vc, vs)
    out, scores = kvq.kvq_decode_attention(qg, k_words=wg, k_norms=ng, sketch=Sg, v_codes=vcg,
                                           v_scales=vsg, want_scores=True, flags=flags)
    out, scores = to_np(out), to_np(scores)
    assert np.abs(out - ref["out"]).max() <= OUT_TOL
    v64, _ = oracle.qjl_query_sketch(q.reshape(-1, 128), S)
    G = Hq // Hkv
    tol = score_tolerance(ref["scores"].reshape(B * Hq, T),
                          np.repeat(n, G, axis=1).reshape(B * Hq, T), v64, m)
    err = np.abs(scores.astype(np.float64) - ref["scores"]).reshape(B * Hq, T)
    assert np.all(err <= tol), float((err / tol).max())
    check_decode_bound(out, scores, ref["scores"], _vals(vc, vs), qjl=True, v_scales=vs)


# Shapes whose token count and capacity are multiples of 8 take the tensor-core value
# pass (chunks of 128 tokens): one partial chunk, several chunks with a partial tail,
# CTA ranges that span many short units (several segments and table builds per CTA),
# one, two and four query heads per CTA, m = 32, 128 and 256, and groups of 8, 16 and 32
# query heads per KV head (two to eight CTAs per token range).
@pytest.mark.parametrize("B,Hq,Hkv,T,m", [(1, 4, 1, 8, 256), (2, 8, 2, 1504, 256), (1, 32, 8, 2048, 256),
                                          (1, 4, 4, 704, 128), (1, 2, 1, 336, 32), (16, 32, 8, 8, 256),
                                          (4, 8, 4, 96, 256), (3, 12, 3, 5000, 256),
                                          (1, 8, 1, 1504, 256), (1, 16, 2, 2048, 256), (1, 32, 1, 4096, 256)])
def test_decode_qjl_tc_parity(kvq, B, Hq, Hkv, T, m):
    test_decode_qjl_parity(kvq, B, Hq, Hkv, T, m)


@pytest.mark.parametrize("B,Hq,Hkv,T,m", [(2, 8, 2, 1504, 256), (1, 32, 8, 2048, 256), (16, 32, 8, 8, 256),
                                          (1, 16, 2, 2048, 256), (1, 4, 4, 704, 128)])
def test_decode_qjl_cuda_cores_flag_parity(kvq, B, Hq, Hkv, T, m):
    """KVQ_DECODE_CUDA_CORES on shapes that would take the tensor-core value pass: the
    weighted sum runs in fp32 on the CUDA cores, against the same oracle and bounds."""
    test_decode_qjl_parity(kvq, B, Hq, Hkv, T, m, flags=kvq.KVQ_DECODE_CUDA_CORES)


@pytest.mark.parametrize("key_format,T", [("int8", 4096), ("qjl", 4096), ("qjl", 1000)])
def test_decode_output_independent_of_scores_request(kvq, key_format, T):
    """Asking for the raw scores only adds their stores: the output is bit-identical with
    and without them (the arithmetic bound of the other tests reads the scores of the
    same call)."""
    B, Hq, Hkv = 2, 16, 4
    if key_format == "int8":
        q, kc, ks, vc, vs = _int8_cache(600, B, Hkv, T, Hq)
        qg, kcg, ksg, vcg, vsg = _cuda(q, kc, ks, vc, vs)
        keys = dict(k_codes=kcg, k_scales=ksg)
    else:
        q, S, w, n, vc, vs = _qjl_cache(601, B, Hkv, T, Hq)
        qg, Sg, wg, ng, vcg, vsg = _cuda(q, S, w.view(np.int32), n, vc, vs)
        keys = dict(k_words=wg, k_norms=ng, sketch=Sg)
    a, _ = kvq.kvq_decode_attention(qg, v_codes=vcg, v_scales=vsg, **keys)
    b, _ = kvq.kvq_decode_attention(qg, v_codes=vcg, v_scales=vsg, want_scores=True, **keys)
    assert np.array_equal(to_np(a).view(np.uint32), to_np(b).view(np.uint32))


def test_decode_qjl_tc_zero_value_chunk(kvq):
    """Value rows that are all zero (scale 0) over whole 128-token chunks and over a
    partial one: those chunks add nothing to the weighted sum but still to the softmax
    sum.  Against the oracle on the same codes and scales."""
    B, Hq, Hkv, T, m = 1, 8, 2, 1000, 256
    q, S, w, n, vc, vs = _qjl_cache(900, B, Hkv, T, Hq, m)
    vc[0, 0, 128:384] = 0
    vs[0, 0, 128:384] = 0.0
    vc[0, 1, 900:] = 0
    vs[0, 1, 900:] = 0.0
    ref = oracle.decode_attention(q, k_words=w, k_norms=n, S=S, v_codes=vc, v_scales=vs, want_scores=True)
    qg, Sg, wg, ng, vcg, vsg = _cuda(q, S, w.view(np.int32), n, vc, vs)
    out, scores = kvq.kvq_decode_attention(qg, k_words=wg, k_norms=ng, sketch=Sg, v_codes=vcg, v_scales=vsg,
                                           want_scores=True)
    assert np.abs(to_np(out) - ref["out"]).max() <= OUT_TOL
    check_decode_bound(to_np(out), to_np(scores), ref["scores"], _vals(vc, vs), qjl=True, v_scales=vs)
    assert kvq.kvq_device_error() == 0


def test_decode_int8_llama7b_layer_sampled(kvq):
    """One layer of the 7B-shaped cache (batch 8, 32 heads, 4096 tokens): GPU quantize
    then GPU decode; 6 sampled (batch, head) units re-done by the oracle from the fp16
    cache."""
    B, H, T = 8, 32, 4096
    kv = inputs.lognormal_cache_device(3, (2, B, H, T, 128), n_sigma_dims=(0, 2, 4), device="cuda")
    q = inputs.gaussian_queries_device(33, (B, H, 128), "cuda")
    kc, ks = kvq.kvq_quantize_int8(kv[0])
    vc, vs = kvq.kvq_quantize_int8(kv[1])
    out, scores = kvq.kvq_decode_attention(q, k_codes=kc, k_scales=ks, v_codes=vc, v_scales=vs,
                                           want_scores=True)
    out, scores = to_np(out), to_np(scores)
    rng = np.random.default_rng(3)
    for b, h in zip(rng.integers(0, B, 6), rng.integers(0, H, 6)):
        kc_r, ks_r = oracle.quantize_int8(to_np(kv[0, b, h]))
        vc_r, vs_r = oracle.quantize_int8(to_np(kv[1, b, h]))
        ref = oracle.decode_attention(to_np(q[b, h])[None, None], k_codes=kc_r[None, None],
                                      k_scales=ks_r[None, None], v_codes=vc_r[None, None],
                                      v_scales=vs_r[None, None], want_scores=True)
        assert np.abs(out[b, h] - ref["out"][0, 0]).max() <= OUT_TOL
        # the unit's bound, with the chain lengths of the whole layer's launch
        n_chain, n_rescale = decode_chain(B, H, T, H, sm_count(), qjl=False)
        check_decode_unit(out[b, h][None], scores[b, h][None], ref["scores"][0], _vals(vc_r, vs_r),
                          softmax_scale(), n_chain, n_rescale, tc_smax=float(vs_r.max()))


def test_decode_qjl_gqa_long_context_all_units(kvq):
    """Long-context GQA cache: batch 4, 32 query / 8 KV heads, 131072 tokens; keys
    QJL-encoded and values INT8-quantized on the GPU, then one fused decode step (the
    launch the benchmark times).  Every one of the 32 KV units is re-done end to end by
    the oracle from the fp16 cache (in spawned worker processes): sign words exact
    outside the band, value codes and scales bit-exact, estimator scores within their
    tolerance wherever both sides hold the same bits, outputs within 2e-3 and within the
    arithmetic bound."""
    B, Hq, Hkv, T = 4, 32, 8, 131072
    G = Hq // Hkv
    kv = inputs.lognormal_cache_device(5, (2, B, Hkv, T, 128), n_sigma_dims=(0, 2, 4), device="cuda")
    q = inputs.gaussian_queries_device(50, (B, Hq, 128), "cuda")
    S_np = inputs.sketch_matrix(256, 128)
    S = torch.from_numpy(S_np).cuda()
    words, norms = kvq.kvq_qjl_encode(kv[0], S)
    vc, vs = kvq.kvq_quantize_int8(kv[1])
    out, scores = kvq.kvq_decode_attention(q, k_words=words, k_norms=norms, sketch=S, v_codes=vc,
                                           v_scales=vs, want_scores=True)
    out, scores = to_np(out), to_np(scores)
    assert kvq.kvq_device_error() == 0
    q_np = to_np(q)
    units = [(b, g) for b in range(B) for g in range(Hkv)]
    jobs = [(to_np(kv[0, b, g]), to_np(kv[1, b, g]), q_np[b, g * G:(g + 1) * G], S_np) for b, g in units]
    refs = _oracle_pool.run_units(_oracle_pool.qjl_unit, jobs)
    n_chain, n_rescale = decode_chain(B, Hkv, T, Hq, sm_count(), qjl=True)
    sigma = softmax_scale()
    worst = 0.0
    for (b, g), job, r in zip(units, jobs, refs):
        gw = words_u32(words[b, g])
        assert np.array_equal(to_np(norms[b, g]).view(np.uint16), r["norms"].view(np.uint16))
        same = np.all(gw == r["words"], axis=1)                       # tokens with identical bits
        if not np.all(same):
            t_diff = np.flatnonzero(~same)
            _, _, u = oracle.qjl_encode(job[0][t_diff], S_np, want_u=True)
            n64 = np.linalg.norm(job[0][t_diff].astype(np.float64), axis=1)
            bad, _ = bit_mismatch_outside_band(gw[t_diff], r["words"][t_diff], u, n64)
            assert bad == 0
        assert np.array_equal(to_np(vc[b, g]), r["v_codes"])
        assert np.array_equal(to_np(vs[b, g]).view(np.uint32), r["v_scales"].view(np.uint32))
        hs = slice(g * G, (g + 1) * G)
        v64, _ = oracle.qjl_query_sketch(job[2], S_np)
        tol = score_tolerance(r["scores"], np.repeat(r["norms"][None], G, axis=0), v64, 256)
        err = np.abs(scores[b, hs].astype(np.float64) - r["scores"])
        assert np.all(err[:, same] <= tol[:, same])
        assert np.abs(out[b, hs] - r["out"]).max() <= OUT_TOL
        vals = oracle.dequantize_int8(r["v_codes"], r["v_scales"])
        worst = max(worst, check_decode_unit(out[b, hs], scores[b, hs], r["scores"], vals, sigma, n_chain,
                                             n_rescale, tc_smax=float(r["v_scales"].max())))
    print(f"long-context GQA decode: largest error / arithmetic bound over 32 units = {worst:.3g}")


def test_decode_rejects_bad_workspace(kvq):
    q, kc, ks, vc, vs = _int8_cache(1, 1, 2, 64, 2)
    qg, kcg, ksg, vcg, vsg = _cuda(q, kc, ks, vc, vs)
    out = torch.empty((1, 2, 128), dtype=torch.float32, device="cuda")
    a = kvq.make_decode_args(qg, k_codes=kcg, k_scales=ksg, v_codes=vcg, v_scales=vsg, out=out)
    need = kvq.kvq_decode_workspace_bytes(a)
    assert need > 0
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    a.workspace, a.workspace_bytes = ws.data_ptr(), need - 1
    import ctypes
    assert kvq.lib.kvq_decode_attention(ctypes.byref(a), None) == kvq.KVQ_ERR_WORKSPACE
    a.workspace_bytes = need
    assert kvq.lib.kvq_decode_attention(ctypes.byref(a), None) == kvq.KVQ_OK
    torch.cuda.synchronize()


def test_decode_workspace_reused_across_calls_and_shapes(kvq):
    """One workspace serves a sequence of calls of different shapes and key formats
    (units split over several CTAs, units inside one range, query heads split over two
    CTAs per range), twice over: every result matches the oracle, whatever an earlier
    call left in the workspace."""
    cases = []
    for (B, Hq, Hkv, T) in [(1, 8, 1, 1000), (16, 16, 8, 3), (2, 16, 4, 4097), (1, 16, 1, 999)]:
        q, kc, ks, vc, vs = _int8_cache(200 + T, B, Hkv, T, Hq)
        ref = oracle.decode_attention(q, k_codes=kc, k_scales=ks, v_codes=vc, v_scales=vs, want_scores=True)
        qg, kcg, ksg, vcg, vsg = _cuda(q, kc, ks, vc, vs)
        cases.append((ref, _vals(vc, vs), None, False,
                      dict(q=qg, k_codes=kcg, k_scales=ksg, v_codes=vcg, v_scales=vsg)))
    q, S, w, n, vc, vs = _qjl_cache(300, 4, 8, 100, 8)
    ref = oracle.decode_attention(q, k_words=w, k_norms=n, S=S, v_codes=vc, v_scales=vs, want_scores=True)
    qg, Sg, wg, ng, vcg, vsg = _cuda(q, S, w.view(np.int32), n, vc, vs)
    cases.append((ref, _vals(vc, vs), vs, True,
                  dict(q=qg, k_words=wg, k_norms=ng, sketch=Sg, v_codes=vcg, v_scales=vsg)))
    need = 0
    for *_, c in cases:
        rest = {k: v for k, v in c.items() if k != "q"}
        need = max(need, kvq.kvq_decode_workspace_bytes(kvq.make_decode_args(
            c["q"], out=torch.empty(c["q"].shape, dtype=torch.float32, device="cuda"), **rest)))
    ws = torch.full((need,), 0xA5, dtype=torch.uint8, device="cuda")
    for rep in range(2):
        for ref, vals, vsc, qjl, c in cases:
            rest = {k: v for k, v in c.items() if k != "q"}
            out, scores = kvq.kvq_decode_attention(c["q"], workspace=ws, want_scores=True, **rest)
            assert np.abs(to_np(out) - ref["out"]).max() <= OUT_TOL
            check_decode_bound(to_np(out), to_np(scores), ref["scores"], vals, qjl=qjl, v_scales=vsc)
    assert kvq.kvq_device_error() == 0


def test_decode_qjl_scores_only(kvq):
    """A QJL scores-only call (no values, no output), twice on one workspace: the
    estimator scores match the oracle's."""
    q, S, w, n, vc, vs = _qjl_cache(400, 2, 4, 3000, 8)
    qg, Sg, wg, ng = _cuda(q, S, w.view(np.int32), n)
    scores = torch.empty((2, 8, 3000), dtype=torch.float32, device="cuda")
    a = kvq.make_decode_args(qg, k_words=wg, k_norms=ng, sketch=Sg, scores_out=scores)
    need = kvq.kvq_decode_workspace_bytes(a)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    for _ in range(2):
        _, sc = kvq.kvq_decode_attention(qg, k_words=wg, k_norms=ng, sketch=Sg, want_out=False,
                                         want_scores=True, workspace=ws)
        torch.cuda.synchronize()
    ref = oracle.decode_attention(q, k_words=w, k_norms=n, S=S, want_out=False, want_scores=True)
    v64, _ = oracle.qjl_query_sketch(q.reshape(-1, 128), S)
    tol = score_tolerance(ref["scores"].reshape(16, 3000), np.repeat(n, 2, axis=1).reshape(16, 3000), v64, 256)
    err = np.abs(to_np(sc).astype(np.float64) - ref["scores"]).reshape(16, 3000)
    assert np.all(err <= tol)
