"""Parity at the workloads' full sizes, in the launch configurations the benchmark uses;
outputs are sampled and re-done one by one by the oracle (from the same fp16/fp32
inputs, copied back to the host).

  * throughput sweep: 1e9 elements at D = 128, 1024, 8192, fp32 and fp16;
  * the 7B-shaped cache: all 32 layers x {K, V} quantized in one launch, decode sampled
    (outputs within 2e-3 and within the arithmetic bound of tests/_helpers.py);
  * the key-sketch workload: estimator scores of one query per head over 32768 keys.
"""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_quantization_absmax_b200 import inputs
from tests._helpers import check_decode_unit, decode_chain, score_tolerance, sm_count, softmax_scale, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvq():
    from kv_cache_quantization_absmax_b200 import kvq as m
    return m


@pytest.mark.parametrize("dtype", [np.float32, np.float16])
@pytest.mark.parametrize("d", [128, 1024, 8192])
def test_sweep_1e9_sampled(kvq, d, dtype):
    x, q, cols = inputs.sweep_matrix_device(10 ** 9, d, dtype, 30 + d % 7, "cuda")
    n = x.shape[0]
    codes, scales = kvq.kvq_quantize_int8(x)
    xh = kvq.kvq_dequantize_int8(codes, scales, torch.float32)
    scores = kvq.kvq_int8_scores(torch.from_numpy(q).cuda(), codes, scales)
    torch.cuda.synchronize()
    rng = np.random.default_rng(d)
    rows = np.unique(np.concatenate([rng.integers(0, n, 64), [0, n - 1]]))
    ridx = torch.from_numpy(rows).cuda()
    x_s = to_np(x[ridx])
    c_ref, s_ref = oracle.quantize_int8(x_s)
    assert np.array_equal(to_np(codes[ridx]), c_ref)
    assert np.array_equal(to_np(scales[ridx]).view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(to_np(xh[ridx]), oracle.dequantize_int8(c_ref, s_ref))
    ref = oracle.int8_scores(q, c_ref, s_ref).astype(np.float64)
    xh64 = oracle.dequantize_int8(c_ref, s_ref).astype(np.float64)
    bound = 2 * d * 2.0 ** -24 * np.abs(xh64 * q.astype(np.float64)[None, :]).sum(1)
    assert np.all(np.abs(to_np(scores[ridx]).astype(np.float64) - ref) <= bound)


def test_llama7b_cache_full_sampled(kvq):
    L, B, H, T = 32, 8, 32, 4096
    cache = inputs.lognormal_cache_device(3, (L, 2, B, H, T, 128), n_sigma_dims=(0, 1, 3, 5), device="cuda")
    q = inputs.gaussian_queries_device(30, (L, B, H, 128), "cuda")
    codes, scales = kvq.kvq_quantize_int8(cache)          # one launch over 134M rows
    outs, scs = [], []
    for l in (0, 17, 31):
        out, sc = kvq.kvq_decode_attention(q[l], k_codes=codes[l, 0], k_scales=scales[l, 0],
                                           v_codes=codes[l, 1], v_scales=scales[l, 1], want_scores=True)
        outs.append(to_np(out))
        scs.append(to_np(sc))
    torch.cuda.synchronize()
    rng = np.random.default_rng(7)
    flat = cache.view(-1, 128)
    rows = np.unique(np.concatenate([rng.integers(0, flat.shape[0], 512), [0, flat.shape[0] - 1]]))
    ridx = torch.from_numpy(rows).cuda()
    c_ref, s_ref = oracle.quantize_int8(to_np(flat[ridx]))
    assert np.array_equal(to_np(codes.view(-1, 128)[ridx]), c_ref)
    assert np.array_equal(to_np(scales.view(-1)[ridx]), s_ref)
    for i, l in enumerate((0, 17, 31)):
        b, h = int(rng.integers(0, B)), int(rng.integers(0, H))
        kc, ks = oracle.quantize_int8(to_np(cache[l, 0, b, h]))
        vc, vs = oracle.quantize_int8(to_np(cache[l, 1, b, h]))
        ref = oracle.decode_attention(to_np(q[l, b, h])[None, None], k_codes=kc[None, None],
                                      k_scales=ks[None, None], v_codes=vc[None, None],
                                      v_scales=vs[None, None], want_scores=True)
        assert np.abs(outs[i][b, h] - ref["out"][0, 0]).max() <= 2e-3
        n_chain, n_rescale = decode_chain(B, H, T, H, sm_count(), qjl=False)
        check_decode_unit(outs[i][b, h][None], scs[i][b, h][None], ref["scores"][0],
                          oracle.dequantize_int8(vc, vs), softmax_scale(), n_chain, n_rescale,
                          tc_smax=float(vs.max()))


def test_key_sketch_scores_full_size(kvq):
    """keys [1, 32, 32768, 128], S [256, 128] (seed 7), one query per head: the GPU
    encodes all keys; for two sampled heads the oracle's sign words replace the GPU's so
    that both sides score the same bits."""
    H, T = 32, 32768
    keys = inputs.lognormal_cache_device(4, (1, H, T, 128), n_sigma_dims=(1, 3), device="cuda")
    q = torch.from_numpy(inputs.gaussian_queries(40, 1, H)).cuda()
    S_np = inputs.sketch_matrix(256, 128)
    S = torch.from_numpy(S_np).cuda()
    words, norms = kvq.kvq_qjl_encode(keys, S)
    for h in (3, 29):
        w_r, n_r = oracle.qjl_encode(to_np(keys[0, h]), S_np)
        words[0, h].copy_(torch.from_numpy(w_r.view(np.int32)))
        norms[0, h].copy_(torch.from_numpy(n_r))
        _, scores = kvq.kvq_decode_attention(q, k_words=words, k_norms=norms, sketch=S,
                                             want_out=False, want_scores=True)
        v64, _ = oracle.qjl_query_sketch(to_np(q[0, h])[None], S_np)
        ref = oracle.qjl_scores(v64, w_r, n_r)[0].astype(np.float64)
        got = to_np(scores[0, h]).astype(np.float64)
        tol = score_tolerance(ref[None], n_r[None], v64, 256)[0]
        assert np.all(np.abs(got - ref) <= tol), float((np.abs(got - ref) / tol).max())
