"""GPU parity of append-on-decode (kvq_decode_append) against the CPU oracle.

The new token's key / value rows are encoded inside the decode kernel and stored at
token T of caches with a per-head capacity above T + 1.  Checked: the appended INT8
codes and scales and the QJL norms bit-exact; QJL sign bits exact outside the band
|(S k)_i| < 1e-4 ||k||; every other cache row untouched; decode outputs within 2e-3
max-abs of the oracle and within the arithmetic bound (tests/_helpers.py,
check_decode_bound); raw scores within the fp32 summation bound (INT8 keys) or the
estimator bound on the same stored bits (QJL keys).
"""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_quantization_absmax_b200 import inputs
from tests._helpers import bit_mismatch_outside_band, check_decode_bound, score_tolerance, to_np, words_u32

pytestmark = pytest.mark.gpu

OUT_TOL = 2e-3


@pytest.fixture(scope="module")
def kvq():
    from kv_cache_quantization_absmax_b200 import kvq as m
    return m


def _case(seed, B, Hq, Hkv, T, cap):
    """INT8-quantized cache holding T tokens in `cap` rows per head (sentinels beyond),
    and the new token's fp16 key / value rows."""
    k, v = inputs.lognormal_cache(seed, B, Hkv, T + 1, n_tensors=2)
    q = inputs.gaussian_queries(seed + 1, B, Hq)
    D = 128
    kc = np.full((B, Hkv, cap, D), 55, np.int8)
    ks = np.full((B, Hkv, cap), 7.25, np.float32)
    vc = np.full((B, Hkv, cap, D), -55, np.int8)
    vs = np.full((B, Hkv, cap), 9.5, np.float32)
    if T > 0:
        c, s = oracle.quantize_int8(k[:, :, :T].reshape(-1, D))
        kc[:, :, :T], ks[:, :, :T] = c.reshape(B, Hkv, T, D), s.reshape(B, Hkv, T)
        c, s = oracle.quantize_int8(v[:, :, :T].reshape(-1, D))
        vc[:, :, :T], vs[:, :, :T] = c.reshape(B, Hkv, T, D), s.reshape(B, Hkv, T)
    return q, k[:, :, T].copy(), v[:, :, T].copy(), k[:, :, :T], kc, ks, vc, vs


def _vals(vc, vs):
    """Dequantized value rows [B, Hkv, T, D]."""
    vc, vs = np.ascontiguousarray(vc), np.ascontiguousarray(vs)
    return oracle.dequantize_int8(vc.reshape(-1, 128), vs.reshape(-1)).reshape(vc.shape)


def _cuda(*arrs):
    return [torch.from_numpy(np.ascontiguousarray(a)).cuda() for a in arrs]


# T + 1 >= 512 takes the tensor-core decode, with the append encoded by a kernel of its
# own first; the shorter contexts encode inside the CUDA-core kernel.
@pytest.mark.parametrize("B,Hq,Hkv,T,cap", [(1, 4, 4, 0, 8), (2, 8, 2, 33, 40), (1, 8, 1, 999, 1000),
                                            (2, 16, 4, 4095, 4096), (16, 16, 8, 2, 3),
                                            (3, 24, 3, 70, 77), (1, 8, 8, 1500, 1501)])
def test_append_int8(kvq, B, Hq, Hkv, T, cap):
    q, kn, vn, _, kc, ks, vc, vs = _case(40 + T, B, Hq, Hkv, T, cap)
    ref = oracle.decode_append(q, kn, vn, T=T, k_codes=kc, k_scales=ks, v_codes=vc, v_scales=vs,
                               want_scores=True)
    qg, kng, vng, kcg, ksg, vcg, vsg = _cuda(q, kn, vn, kc, ks, vc, vs)
    out, scores = kvq.kvq_decode_append(qg, kng, vng, T=T, k_codes=kcg, k_scales=ksg, v_codes=vcg,
                                        v_scales=vsg, want_scores=True)
    assert np.array_equal(to_np(kcg), ref["k_codes"])
    assert np.array_equal(to_np(ksg).view(np.uint32), ref["k_scales"].view(np.uint32))
    assert np.array_equal(to_np(vcg), ref["v_codes"])
    assert np.array_equal(to_np(vsg).view(np.uint32), ref["v_scales"].view(np.uint32))
    assert np.abs(to_np(out) - ref["out"]).max() <= OUT_TOL
    G = Hq // Hkv
    kfull = ref["k_codes"][:, :, :T + 1].astype(np.float64) * ref["k_scales"][:, :, :T + 1, None]
    terms = np.abs(np.repeat(kfull, G, axis=1) * q.astype(np.float64)[:, :, None, :]).sum(-1)
    err = np.abs(to_np(scores).astype(np.float64) - ref["scores"])
    assert np.all(err <= 2 * 128 * 2.0 ** -24 * terms + 1e-30)
    vals = _vals(ref["v_codes"][:, :, :T + 1], ref["v_scales"][:, :, :T + 1])
    check_decode_bound(to_np(out), to_np(scores), ref["scores"], vals, qjl=False)
    assert kvq.kvq_device_error() == 0


def test_append_int8_scores_only(kvq):
    """No output: only the key row is appended (no value pointers), scores over T + 1."""
    B, Hq, Hkv, T, cap = 2, 8, 4, 300, 304
    q, kn, _, _, kc, ks, _, _ = _case(7, B, Hq, Hkv, T, cap)
    ref = oracle.decode_append(q, kn, None, T=T, k_codes=kc, k_scales=ks, want_out=False,
                               want_scores=True)
    qg, kng, kcg, ksg = _cuda(q, kn, kc, ks)
    out, scores = kvq.kvq_decode_append(qg, kng, None, T=T, k_codes=kcg, k_scales=ksg,
                                        want_out=False, want_scores=True)
    assert out is None
    assert np.array_equal(to_np(kcg), ref["k_codes"])
    assert np.array_equal(to_np(ksg).view(np.uint32), ref["k_scales"].view(np.uint32))
    kfull = ref["k_codes"][:, :, :T + 1].astype(np.float64) * ref["k_scales"][:, :, :T + 1, None]
    terms = np.abs(np.repeat(kfull, Hq // Hkv, axis=1) * q.astype(np.float64)[:, :, None, :]).sum(-1)
    assert np.all(np.abs(to_np(scores).astype(np.float64) - ref["scores"]) <= 2 * 128 * 2.0 ** -24 * terms)


# T + 1 and the capacity multiples of 8 take the tensor-core decode, with the append
# encoded by a kernel of its own first: (1, 32, 8, 2047, 2048), (2, 16, 2, 1535, 1536),
# (1, 8, 4, 4095, 4104, m = 128); the others encode inside the CUDA-core kernel.
@pytest.mark.parametrize("B,Hq,Hkv,T,cap,m", [(1, 4, 1, 0, 4, 256), (2, 8, 2, 100, 128, 256),
                                              (1, 32, 8, 2047, 2048, 256), (1, 4, 4, 333, 400, 128),
                                              (4, 8, 4, 5000, 5001, 64), (2, 16, 2, 1535, 1536, 256),
                                              (1, 8, 4, 4095, 4104, 128)])
def test_append_qjl(kvq, B, Hq, Hkv, T, cap, m):
    q, kn, vn, kprev, _, _, vc, vs = _case(90 + T, B, Hq, Hkv, T, cap)
    S = inputs.sketch_matrix(m, 128)
    kw = np.full((B, Hkv, cap, m // 32), 0x5A5A5A5A, np.uint32)
    knorm = np.full((B, Hkv, cap), 3.0, np.float16)
    if T > 0:
        w, n = oracle.qjl_encode(kprev.reshape(-1, 128), S)
        kw[:, :, :T] = w.reshape(B, Hkv, T, m // 32)
        knorm[:, :, :T] = n.reshape(B, Hkv, T)
    ref = oracle.decode_append(q, kn, vn, T=T, k_words=kw, k_norms=knorm, S=S, v_codes=vc,
                               v_scales=vs)
    qg, kng, vng, Sg, kwg, kng2, vcg, vsg = _cuda(q, kn, vn, S, kw.view(np.int32), knorm, vc, vs)
    out, scores = kvq.kvq_decode_append(qg, kng, vng, T=T, k_words=kwg, k_norms=kng2, sketch=Sg,
                                        v_codes=vcg, v_scales=vsg, want_scores=True)
    got_w = words_u32(kwg)
    # the new row's bits: exact outside the band around zero
    _, _, u = oracle.qjl_encode(kn.reshape(-1, 128), S, want_u=True)
    new_w = got_w[:, :, T].reshape(-1, m // 32)
    norms64 = np.linalg.norm(kn.reshape(-1, 128).astype(np.float64), axis=1)
    bad, _ = bit_mismatch_outside_band(new_w, ref["k_words"][:, :, T].reshape(-1, m // 32), u, norms64)
    assert bad == 0
    keep = np.ones(cap, bool)
    keep[T] = False
    assert np.array_equal(got_w[:, :, keep], kw[:, :, keep])
    assert np.array_equal(to_np(kng2).view(np.uint16), ref["k_norms"].view(np.uint16))
    assert np.array_equal(to_np(vcg), ref["v_codes"])
    assert np.array_equal(to_np(vsg).view(np.uint32), ref["v_scales"].view(np.uint32))
    # decode on the stored bits (the band's bits may legitimately differ)
    ref2 = oracle.decode_attention(q, k_words=got_w[:, :, :T + 1], k_norms=ref["k_norms"][:, :, :T + 1],
                                   S=S, v_codes=ref["v_codes"][:, :, :T + 1],
                                   v_scales=ref["v_scales"][:, :, :T + 1], want_scores=True)
    assert np.abs(to_np(out) - ref2["out"]).max() <= OUT_TOL
    v64, _ = oracle.qjl_query_sketch(q.reshape(-1, 128), S)
    G = Hq // Hkv
    tol = score_tolerance(ref2["scores"].reshape(B * Hq, T + 1),
                          np.repeat(ref["k_norms"][:, :, :T + 1], G, axis=1).reshape(B * Hq, T + 1),
                          v64, m)
    err = np.abs(to_np(scores).astype(np.float64) - ref2["scores"]).reshape(B * Hq, T + 1)
    assert np.all(err <= tol)
    vs1 = ref["v_scales"][:, :, :T + 1]
    check_decode_bound(to_np(out), to_np(scores), ref2["scores"], _vals(ref["v_codes"][:, :, :T + 1], vs1),
                       qjl=True, v_scales=vs1)
    assert kvq.kvq_device_error() == 0


def test_append_rejects_bad_capacity(kvq):
    import ctypes
    B, Hq, Hkv, T, cap = 1, 4, 4, 10, 10      # capacity must be >= T + 1
    q, kn, vn, _, kc, ks, vc, vs = _case(3, B, Hq, Hkv, T, cap)
    qg, kng, vng, kcg, ksg, vcg, vsg = _cuda(q, kn, vn, kc, ks, vc, vs)
    out = torch.empty((B, Hq, 128), dtype=torch.float32, device="cuda")
    a = kvq.make_decode_append_args(qg, kng, vng, T=T, k_codes=kcg, k_scales=ksg, v_codes=vcg,
                                    v_scales=vsg, out=out)
    assert kvq.lib.kvq_decode_append_workspace_bytes(ctypes.byref(a)) == 0
    assert kvq.lib.kvq_decode_append(ctypes.byref(a), None) == kvq.KVQ_ERR_INVALID_ARG
