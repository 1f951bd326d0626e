"""The failure path of the tensor-core decode kernels, on the GPU, without a fault.

With KVQ_DECODE_TEST_EXPIRE the kernels' key producer issues no loads, so every role
that consumes key tiles waits on an mbarrier phase that never completes.  Each such wait
is bounded (about 2 s): the first one to give up records its code in the library's error
word and raises the CTA's abort flag, the other roles leave at their next wait, copies
already in flight are drained, and the launch completes.  The combine kernel then writes
NaN for every output.  The test checks exactly that: the call returns, kvq_device_error()
reports one code of that kernel (and reading it clears it), every output is NaN, and the
next call on the same device, without the flag, is correct again.
"""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_quantization_absmax_b200 import inputs

pytestmark = pytest.mark.gpu

OUT_TOL = 2e-3
# the bounded waits' codes: tensor-core INT8 kernel (producer, MMA, softmax, merge) and
# tensor-core QJL kernel (producer, MMA, scorer, accumulator)
INT8_TC_CODES = (0x221, 0x222, 0x223, 0x224)
QJL_TC_CODES = (0x211, 0x212, 0x213, 0x214)


@pytest.fixture(scope="module")
def kvq():
    from kv_cache_quantization_absmax_b200 import kvq as m
    return m


def _cuda(*arrs):
    return [torch.from_numpy(np.ascontiguousarray(a)).cuda() for a in arrs]


def test_int8_tensor_core_wait_expiry(kvq):
    B, Hq, Hkv, T = 1, 8, 2, 1024           # 1024 tokens: the tensor-core INT8 kernel
    k, v = inputs.lognormal_cache(501, B, Hkv, T, n_tensors=2)
    q = inputs.gaussian_queries(502, B, Hq)
    kc, ks = oracle.quantize_int8(k.reshape(-1, 128))
    vc, vs = oracle.quantize_int8(v.reshape(-1, 128))
    shp = (B, Hkv, T)
    qg, kcg, ksg, vcg, vsg = _cuda(q, kc.reshape(shp + (128,)), ks.reshape(shp), vc.reshape(shp + (128,)),
                                   vs.reshape(shp))
    assert kvq.kvq_device_error() == 0
    out, _ = kvq.kvq_decode_attention(qg, k_codes=kcg, k_scales=ksg, v_codes=vcg, v_scales=vsg,
                                      flags=kvq.KVQ_DECODE_TEST_EXPIRE)
    torch.cuda.synchronize()
    assert kvq.kvq_device_error() in INT8_TC_CODES
    assert kvq.kvq_device_error() == 0       # read and cleared
    assert torch.isnan(out).all()
    out2, _ = kvq.kvq_decode_attention(qg, k_codes=kcg, k_scales=ksg, v_codes=vcg, v_scales=vsg)
    torch.cuda.synchronize()
    assert kvq.kvq_device_error() == 0
    ref = oracle.decode_attention(q, k_codes=kc.reshape(shp + (128,)), k_scales=ks.reshape(shp),
                                  v_codes=vc.reshape(shp + (128,)), v_scales=vs.reshape(shp))
    assert np.abs(out2.cpu().numpy() - ref["out"]).max() <= OUT_TOL


def test_qjl_tensor_core_wait_expiry(kvq):
    B, Hq, Hkv, T = 1, 8, 2, 1024           # a multiple of 8: the tensor-core QJL kernel
    k, v = inputs.lognormal_cache(503, B, Hkv, T, n_tensors=2)
    q = inputs.gaussian_queries(504, B, Hq)
    S = inputs.sketch_matrix(256, 128)
    w, n = oracle.qjl_encode(k.reshape(-1, 128), S)
    vc, vs = oracle.quantize_int8(v.reshape(-1, 128))
    shp = (B, Hkv, T)
    qg, Sg, wg, ng, vcg, vsg = _cuda(q, S, w.view(np.int32).reshape(shp + (8,)), n.reshape(shp),
                                     vc.reshape(shp + (128,)), vs.reshape(shp))
    assert kvq.kvq_device_error() == 0
    out, _ = kvq.kvq_decode_attention(qg, k_words=wg, k_norms=ng, sketch=Sg, v_codes=vcg, v_scales=vsg,
                                      flags=kvq.KVQ_DECODE_TEST_EXPIRE)
    torch.cuda.synchronize()
    assert kvq.kvq_device_error() in QJL_TC_CODES
    assert kvq.kvq_device_error() == 0
    assert torch.isnan(out).all()
    out2, _ = kvq.kvq_decode_attention(qg, k_words=wg, k_norms=ng, sketch=Sg, v_codes=vcg, v_scales=vsg)
    torch.cuda.synchronize()
    assert kvq.kvq_device_error() == 0
    ref = oracle.decode_attention(q, k_words=w.reshape(shp + (8,)), k_norms=n.reshape(shp), S=S,
                                  v_codes=vc.reshape(shp + (128,)), v_scales=vs.reshape(shp))
    assert np.abs(out2.cpu().numpy() - ref["out"]).max() <= OUT_TOL
