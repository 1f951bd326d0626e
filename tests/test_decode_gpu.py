"""GPU parity of the fused decode step (scores -> softmax -> sum of INT8 values) against
the CPU oracle, for INT8 keys and QJL keys, MHA and GQA.

Decode outputs: max-abs error <= 2e-3 against the oracle's fp32-accumulated result.
INT8 raw scores: the fp32 summation bound.  QJL estimator scores (same sign words and
norms on both sides): 1e-4 relative to max(|score|, c ||k|| ||S q||_2).
"""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_quantization_absmax_b200 import inputs
from tests._helpers import score_tolerance, to_np

pytestmark = pytest.mark.gpu

OUT_TOL = 2e-3


@pytest.fixture(scope="module")
def kvq():
    from kv_cache_quantization_absmax_b200 import kvq as m
    return m


def _int8_cache(seed, B, Hkv, T, Hq):
    k, v = inputs.lognormal_cache(seed, B, Hkv, T, n_tensors=2)
    q = inputs.gaussian_queries(seed + 1, B, Hq)
    kc, ks = oracle.quantize_int8(k.reshape(-1, 128))
    vc, vs = oracle.quantize_int8(v.reshape(-1, 128))
    shp = (B, Hkv, T)
    return q, kc.reshape(shp + (128,)), ks.reshape(shp), vc.reshape(shp + (128,)), vs.reshape(shp)


def _cuda(*arrs):
    return [torch.from_numpy(np.ascontiguousarray(a)).cuda() for a in arrs]


@pytest.mark.parametrize("B,Hq,Hkv,T", [(1, 1, 1, 1), (1, 4, 4, 5), (2, 8, 2, 33), (1, 8, 1, 1000),
                                        (2, 16, 4, 4097), (1, 8, 8, 300), (1, 16, 2, 2500),
                                        (16, 16, 8, 3), (4, 8, 8, 100), (3, 24, 3, 70)])
def test_decode_int8_parity(kvq, B, Hq, Hkv, T):
    q, kc, ks, vc, vs = _int8_cache(10 + T, B, Hkv, T, Hq)
    ref = oracle.decode_attention(q, k_codes=kc, k_scales=ks, v_codes=vc, v_scales=vs,
                                  want_scores=True)
    qg, kcg, ksg, vcg, vsg = _cuda(q, kc, ks, vc, vs)
    out, scores = kvq.kvq_decode_attention(qg, k_codes=kcg, k_scales=ksg, v_codes=vcg,
                                           v_scales=vsg, want_scores=True)
    assert np.abs(to_np(out) - ref["out"]).max() <= OUT_TOL
    # raw scores: fp32 summation bound on the same codes
    G = Hq // Hkv
    xh = (kc.astype(np.float64) * ks.astype(np.float64)[..., None])
    terms = np.abs(np.repeat(xh, G, axis=1) * q.astype(np.float64)[:, :, None, :]).sum(-1)
    assert np.all(np.abs(to_np(scores).astype(np.float64) - ref["scores"]) <= 2 * 128 * 2.0 ** -24 * terms + 1e-30)


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
    xh = kc.astype(np.float64) * ks.astype(np.float64)[..., None]
    terms = np.abs(xh * q.astype(np.float64)[:, :, None, :]).sum(-1)
    assert np.all(np.abs(to_np(scores).astype(np.float64) - ref["scores"]) <= 2 * 128 * 2.0 ** -24 * terms)


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
                                          (16, 32, 8, 3, 256), (4, 8, 4, 100, 256)])
def test_decode_qjl_parity(kvq, B, Hq, Hkv, T, m):
    q, S, w, n, vc, vs = _qjl_cache(100 + T, B, Hkv, T, Hq, m)
    ref = oracle.decode_attention(q, k_words=w, k_norms=n, S=S, v_codes=vc, v_scales=vs,
                                  want_scores=True)
    qg, Sg, wg, ng, vcg, vsg = _cuda(q, S, w.view(np.int32), n, vc, vs)
    out, scores = kvq.kvq_decode_attention(qg, k_words=wg, k_norms=ng, sketch=Sg, v_codes=vcg,
                                           v_scales=vsg, want_scores=True)
    assert np.abs(to_np(out) - ref["out"]).max() <= OUT_TOL
    v64, _ = oracle.qjl_query_sketch(q.reshape(-1, 128), S)
    G = Hq // Hkv
    tol = score_tolerance(ref["scores"].reshape(B * Hq, T),
                          np.repeat(n, G, axis=1).reshape(B * Hq, T), v64, m)
    err = np.abs(to_np(scores).astype(np.float64) - ref["scores"]).reshape(B * Hq, T)
    assert np.all(err <= tol), float((err / tol).max())


# Shapes whose token count and capacity are multiples of 8 take the tensor-core value
# pass (chunks of 128 tokens): one partial chunk, several chunks with a partial tail,
# CTA ranges that span many short units (several segments and table builds per CTA),
# one, two and four query heads per KV head, m = 32, 128 and 256.
@pytest.mark.parametrize("B,Hq,Hkv,T,m", [(1, 4, 1, 8, 256), (2, 8, 2, 1504, 256), (1, 32, 8, 2048, 256),
                                          (1, 4, 4, 704, 128), (1, 2, 1, 336, 32), (16, 32, 8, 8, 256),
                                          (4, 8, 4, 96, 256), (3, 12, 3, 5000, 256)])
def test_decode_qjl_tc_parity(kvq, B, Hq, Hkv, T, m):
    test_decode_qjl_parity(kvq, B, Hq, Hkv, T, m)


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
    ref = oracle.decode_attention(q, k_words=w, k_norms=n, S=S, v_codes=vc, v_scales=vs)
    qg, Sg, wg, ng, vcg, vsg = _cuda(q, S, w.view(np.int32), n, vc, vs)
    out, _ = kvq.kvq_decode_attention(qg, k_words=wg, k_norms=ng, sketch=Sg, v_codes=vcg, v_scales=vsg)
    assert np.abs(to_np(out) - ref["out"]).max() <= OUT_TOL
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
    out, _ = kvq.kvq_decode_attention(q, k_codes=kc, k_scales=ks, v_codes=vc, v_scales=vs)
    out = to_np(out)
    rng = np.random.default_rng(3)
    for b, h in zip(rng.integers(0, B, 6), rng.integers(0, H, 6)):
        k_np = to_np(kv[0, b, h])
        v_np = to_np(kv[1, b, h])
        kc_r, ks_r = oracle.quantize_int8(k_np)
        vc_r, vs_r = oracle.quantize_int8(v_np)
        ref = oracle.decode_attention(to_np(q[b, h])[None, None], k_codes=kc_r[None, None],
                                      k_scales=ks_r[None, None], v_codes=vc_r[None, None],
                                      v_scales=vs_r[None, None])
        assert np.abs(out[b, h] - ref["out"][0, 0]).max() <= OUT_TOL


def test_decode_qjl_gqa_long_context_sampled(kvq):
    """Long-context GQA cache: batch 4, 32 query / 8 KV heads, 131072 tokens; keys
    QJL-encoded and values INT8-quantized on the GPU, then one fused decode step.  One
    sampled KV unit (4 query heads) is re-done end to end by the oracle."""
    B, Hq, Hkv, T = 4, 32, 8, 131072
    kv = inputs.lognormal_cache_device(5, (2, B, Hkv, T, 128), n_sigma_dims=(0, 2, 4), device="cuda")
    q = inputs.gaussian_queries_device(50, (B, Hq, 128), "cuda")
    S_np = inputs.sketch_matrix(256, 128)
    S = torch.from_numpy(S_np).cuda()
    words, norms = kvq.kvq_qjl_encode(kv[0], S)
    vc, vs = kvq.kvq_quantize_int8(kv[1])
    out, _ = kvq.kvq_decode_attention(q, k_words=words, k_norms=norms, sketch=S, v_codes=vc,
                                      v_scales=vs)
    out = to_np(out)
    assert kvq.kvq_device_error() == 0
    b, g = 2, 5
    k_np = to_np(kv[0, b, g])
    v_np = to_np(kv[1, b, g])
    w_r, n_r = oracle.qjl_encode(k_np, S_np)
    vc_r, vs_r = oracle.quantize_int8(v_np)
    qs = to_np(q[b, g * 4:(g + 1) * 4])[None]
    ref = oracle.decode_attention(qs, k_words=w_r[None, None], k_norms=n_r[None, None], S=S_np,
                                  v_codes=vc_r[None, None], v_scales=vs_r[None, None])
    assert np.abs(out[b, g * 4:(g + 1) * 4] - ref["out"][0]).max() <= OUT_TOL


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
    (units split over several CTAs, units inside one range), twice over: every result
    matches the oracle, whatever an earlier call left in the workspace."""
    cases = []
    for (B, Hq, Hkv, T) in [(1, 8, 1, 1000), (16, 16, 8, 3), (2, 16, 4, 4097)]:
        q, kc, ks, vc, vs = _int8_cache(200 + T, B, Hkv, T, Hq)
        ref = oracle.decode_attention(q, k_codes=kc, k_scales=ks, v_codes=vc, v_scales=vs)["out"]
        qg, kcg, ksg, vcg, vsg = _cuda(q, kc, ks, vc, vs)
        cases.append((ref, dict(q=qg, k_codes=kcg, k_scales=ksg, v_codes=vcg, v_scales=vsg)))
    q, S, w, n, vc, vs = _qjl_cache(300, 4, 8, 100, 8)
    ref = oracle.decode_attention(q, k_words=w, k_norms=n, S=S, v_codes=vc, v_scales=vs)["out"]
    qg, Sg, wg, ng, vcg, vsg = _cuda(q, S, w.view(np.int32), n, vc, vs)
    cases.append((ref, dict(q=qg, k_words=wg, k_norms=ng, sketch=Sg, v_codes=vcg, v_scales=vsg)))
    need = 0
    for _, c in cases:
        rest = {k: v for k, v in c.items() if k != "q"}
        need = max(need, kvq.kvq_decode_workspace_bytes(kvq.make_decode_args(
            c["q"], out=torch.empty(c["q"].shape, dtype=torch.float32, device="cuda"), **rest)))
    ws = torch.full((need,), 0xA5, dtype=torch.uint8, device="cuda")
    for rep in range(2):
        for ref, c in cases:
            rest = {k: v for k, v in c.items() if k != "q"}
            out, _ = kvq.kvq_decode_attention(c["q"], workspace=ws, **rest)
            assert np.abs(to_np(out) - ref).max() <= OUT_TOL
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
