"""kvq_decode_attention_noalloc: the decode step with the library's built-in scratch.

It serves callers that can neither allocate device memory nor lend a workspace (an
engine that has reserved all device memory through its own allocator, or a path where
an allocation is not allowed).  The test calls it through the C ABI twice in a row --
an INT8 GQA step, then a QJL GQA step, both sharing the one scratch array -- and
checks each result against kvq_decode_attention with a caller-owned workspace and
against the oracle, within the decode tolerance the other tests use (2e-3 max-abs), and
against the oracle within the arithmetic bound of tests/_helpers.py.  It also checks
that a request larger than the scratch is refused before anything is launched.  This
file is collected last so that a failure here cannot hide the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from kv_cache_quantization_absmax_b200 import inputs
from tests._helpers import check_decode_bound, to_np

pytestmark = pytest.mark.gpu

TOL = 2e-3


@pytest.fixture(scope="module")
def kvq():
    from kv_cache_quantization_absmax_b200 import kvq as m
    return m


def _int8_case(B=2, Hq=16, Hkv=4, T=3001):
    k, v = inputs.lognormal_cache(71, B, Hkv, T, n_tensors=2)
    q = inputs.gaussian_queries(72, B, Hq)
    kc, ks = oracle.quantize_int8(k.reshape(-1, 128))
    vc, vs = oracle.quantize_int8(v.reshape(-1, 128))
    shp = (B, Hkv, T)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    ref = oracle.decode_attention(q, k_codes=kc.reshape(shp + (128,)), k_scales=ks.reshape(shp),
                                  v_codes=vc.reshape(shp + (128,)), v_scales=vs.reshape(shp), want_scores=True)
    ref.update(vals=oracle.dequantize_int8(vc, vs).reshape(shp + (128,)), qjl=False, vs=None)
    return ref, dict(q=t(q), k_codes=t(kc.reshape(shp + (128,))), k_scales=t(ks.reshape(shp)),
                     v_codes=t(vc.reshape(shp + (128,))), v_scales=t(vs.reshape(shp)))


def _qjl_case(B=1, Hq=32, Hkv=8, T=5000):
    k, v = inputs.lognormal_cache(73, B, Hkv, T, n_tensors=2)
    q = inputs.gaussian_queries(74, B, Hq)
    S = inputs.sketch_matrix(256, 128)
    w, n = oracle.qjl_encode(k.reshape(-1, 128), S)
    vc, vs = oracle.quantize_int8(v.reshape(-1, 128))
    shp = (B, Hkv, T)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    ref = oracle.decode_attention(q, k_words=w.reshape(shp + (8,)), k_norms=n.reshape(shp), S=S,
                                  v_codes=vc.reshape(shp + (128,)), v_scales=vs.reshape(shp), want_scores=True)
    ref.update(vals=oracle.dequantize_int8(vc, vs).reshape(shp + (128,)), qjl=True, vs=vs.reshape(shp))
    return ref, dict(q=t(q), k_words=t(w.view(np.int32).reshape(shp + (8,))), k_norms=t(n.reshape(shp)),
                     sketch=t(S), v_codes=t(vc.reshape(shp + (128,))), v_scales=t(vs.reshape(shp)))


def _noalloc(kvq, case):
    q = case["q"]
    out = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
    rest = {k: v for k, v in case.items() if k != "q"}
    T = rest["v_codes"].shape[2]
    scores = torch.full((q.shape[0], q.shape[1], T), float("nan"), dtype=torch.float32, device="cuda")
    a = kvq.make_decode_args(q, out=out, scores_out=scores, **rest)
    st = kvq.lib.kvq_decode_attention_noalloc(ctypes.byref(a), None)
    assert st == kvq.KVQ_OK, kvq.lib.kvq_status_string(st)
    return out, scores


def _check_oracle(got, ref):
    out, scores = to_np(got[0]), to_np(got[1])
    assert np.abs(out - ref["out"]).max() <= TOL
    check_decode_bound(out, scores, ref["scores"], ref["vals"], qjl=ref["qjl"], v_scales=ref["vs"])


def _with_workspace(kvq, case):
    rest = {k: v for k, v in case.items() if k != "q"}
    out, _ = kvq.kvq_decode_attention(case["q"], **rest)
    return out


def test_noalloc_matches_workspace_entry_point_two_calls(kvq):
    (o1, c1), (o2, c2) = _int8_case(), _qjl_case()
    ref1, ref2 = _with_workspace(kvq, c1), _with_workspace(kvq, c2)
    got1 = _noalloc(kvq, c1)            # first call on this device sets the scratch up
    got2 = _noalloc(kvq, c2)            # second call reuses the same scratch
    torch.cuda.synchronize()
    assert kvq.kvq_device_error() == 0
    assert torch.isfinite(got1[0]).all() and torch.isfinite(got2[0]).all()
    assert (got1[0] - ref1).abs().max().item() <= TOL
    assert (got2[0] - ref2).abs().max().item() <= TOL
    _check_oracle(got1, o1)
    _check_oracle(got2, o2)
    got1b = _noalloc(kvq, c1)           # and once more, after the other case used it
    torch.cuda.synchronize()
    assert (got1b[0] - ref1).abs().max().item() <= TOL
    _check_oracle(got1b, o1)


def test_noalloc_refuses_requests_larger_than_its_scratch(kvq):
    # 64 x 64 KV units x 8 query heads each: far more split states than 8 MiB holds.
    B, Hkv, G, T = 64, 64, 8, 16
    cap = kvq.lib.kvq_decode_noalloc_max_workspace_bytes()
    case = dict(q=torch.zeros((B, Hkv * G, 128), dtype=torch.float16, device="cuda"),
                k_codes=torch.zeros((B, Hkv, T, 128), dtype=torch.int8, device="cuda"),
                k_scales=torch.zeros((B, Hkv, T), dtype=torch.float32, device="cuda"),
                v_codes=torch.zeros((B, Hkv, T, 128), dtype=torch.int8, device="cuda"),
                v_scales=torch.zeros((B, Hkv, T), dtype=torch.float32, device="cuda"))
    out = torch.empty((B, Hkv * G, 128), dtype=torch.float32, device="cuda")
    a = kvq.make_decode_args(case["q"], out=out, **{k: v for k, v in case.items() if k != "q"})
    assert kvq.kvq_decode_workspace_bytes(a) > cap
    assert kvq.lib.kvq_decode_attention_noalloc(ctypes.byref(a), None) == kvq.KVQ_ERR_WORKSPACE
