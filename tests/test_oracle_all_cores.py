"""The all-cores build of the oracle (the same C source compiled with OpenMP, used for the
all-cores CPU baseline) gives results identical to the single-threaded oracle: every row,
key or (batch, head) unit is computed by one thread with the same arithmetic."""
import numpy as np
import pytest

import oracle
from kv_cache_quantization_absmax_b200 import inputs


@pytest.fixture
def both():
    def run(fn):
        oracle.use_all_cores(False)
        a = fn()
        oracle.use_all_cores(True)
        try:
            b = fn()
        finally:
            oracle.use_all_cores(False)
        return a, b
    return run


def _same(a, b):
    if isinstance(a, dict):
        assert a.keys() == b.keys()
        for k in a:
            _same(a[k], b[k])
    elif isinstance(a, (tuple, list)):
        for x, y in zip(a, b):
            _same(x, y)
    elif a is None:
        assert b is None
    else:
        a, b = np.asarray(a), np.asarray(b)
        assert a.dtype == b.dtype and a.shape == b.shape
        assert np.array_equal(a.view(np.uint8), b.view(np.uint8))


def test_all_cores_build_runs_threads():
    oracle.use_all_cores(True)
    try:
        n = oracle.threads()
    finally:
        oracle.use_all_cores(False)
    assert n >= 1 and oracle.threads() == 1


def test_all_cores_results_identical(both):
    k, v = inputs.lognormal_cache(31, 2, 3, 257, n_tensors=2)
    q = inputs.gaussian_queries(32, 2, 6)
    S = inputs.sketch_matrix(256, 128)
    x = k.reshape(-1, 128)
    _same(*both(lambda: oracle.quantize_int8(x)))
    c, s = oracle.quantize_int8(x)
    _same(*both(lambda: oracle.dequantize_int8(c, s, np.float16)))
    _same(*both(lambda: oracle.int8_scores(q[0, 0], c, s)))
    _same(*both(lambda: oracle.qjl_encode(x, S, want_u=True)))
    _same(*both(lambda: oracle.qjl_residual_encode(x, 32, S, want_r=True, want_u=True)))
    _same(*both(lambda: oracle.quantize_int4_group(x, 32)))
    p4, s4, z4 = oracle.quantize_int4_group(x, 32)
    _same(*both(lambda: oracle.dequantize_int4_group(p4, s4, z4, 32, np.float16)))
    blocks = k.reshape(6, 257, 128)
    _same(*both(lambda: oracle.quantize_int8_channelwise(blocks)))
    cc, cs = oracle.quantize_int8_channelwise(blocks)
    _same(*both(lambda: oracle.dequantize_int8_channelwise(cc, cs, np.float32)))
    vc, vs = oracle.quantize_int8(v.reshape(-1, 128))
    kc = c.reshape(2, 3, 257, 128)
    ks = s.reshape(2, 3, 257)
    vc, vs = vc.reshape(2, 3, 257, 128), vs.reshape(2, 3, 257)
    _same(*both(lambda: oracle.decode_attention(q, k_codes=kc, k_scales=ks, v_codes=vc, v_scales=vs,
                                                want_scores=True, want_probs=True)))
    w, n = oracle.qjl_encode(x, S)
    _same(*both(lambda: oracle.decode_attention(q, k_words=w.reshape(2, 3, 257, 8), k_norms=n.reshape(2, 3, 257),
                                                S=S, v_codes=vc, v_scales=vs, want_scores=True)))
