"""GPU parity of channel-wise INT8 and group-wise INT4 quantize / dequantize against the
CPU oracle: codes, packed nibbles, scales, zero points and dequantized values bit-exact.
Decode over INT4 values: outputs within 2e-3 max-abs of the oracle and within the
arithmetic bound (tests/_helpers.py, check_decode_bound), on the INT4 reconstructions."""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_quantization_absmax_b200 import inputs
from tests._helpers import (check_decode_bound, check_decode_unit, decode_chain, sm_count, softmax_scale,
                            to_np)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvq():
    from kv_cache_quantization_absmax_b200 import kvq as m
    return m


def _rows(seed, n, d, dtype):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, d)) * rng.lognormal(0, 1.5, (n, 1)) + rng.standard_normal((n, 1))
    x = x.astype(dtype)
    if n > 3:
        x[1] = 0                     # all-zero row
        x[2] = dtype(1.25)           # constant row: scale 0 in every group
        x[3, : d // 2] = dtype(-7)   # half constant
    return x


@pytest.mark.parametrize("dtype", [np.float16, np.float32])
@pytest.mark.parametrize("n,d,g", [(1, 128, 32), (7, 128, 64), (1000, 128, 32), (33, 256, 128),
                                   (5, 1024, 64), (300, 8192, 32)])
def test_int4_quantize_dequantize_bit_exact(kvq, dtype, n, d, g):
    x = _rows(n * 7 + d + g, n, d, dtype)
    p_r, s_r, z_r = oracle.quantize_int4_group(x, g)
    xg = torch.from_numpy(x).cuda()
    p, s, z = kvq.kvq_quantize_int4(xg, g)
    assert np.array_equal(to_np(p), p_r)
    assert np.array_equal(to_np(s).view(np.uint32), s_r.view(np.uint32))
    assert np.array_equal(to_np(z).view(np.uint32), z_r.view(np.uint32))
    for od, tod in ((np.float32, torch.float32), (np.float16, torch.float16)):
        ref = oracle.dequantize_int4_group(p_r, s_r, z_r, g, out_dtype=od)
        got = to_np(kvq.kvq_dequantize_int4(p, s, z, g, out_dtype=tod))
        assert np.array_equal(got.view(np.uint16 if od == np.float16 else np.uint32),
                              ref.view(np.uint16 if od == np.float16 else np.uint32))


def test_int4_full_7b_layer_sampled(kvq):
    """One 7B-shaped layer of K ([8, 32, 4096, 128] fp16, groups of 32) on the GPU;
    2000 sampled rows re-done by the oracle."""
    x = inputs.lognormal_cache_device(11, (8, 32, 4096, 128), n_sigma_dims=(1, 3), device="cuda")
    p, s, z = kvq.kvq_quantize_int4(x, 32)
    rows = x.reshape(-1, 128)
    idx = torch.from_numpy(np.random.default_rng(4).choice(rows.shape[0], 2000, replace=False)).cuda()
    xs = to_np(rows[idx])
    p_r, s_r, z_r = oracle.quantize_int4_group(xs, 32)
    assert np.array_equal(to_np(p.reshape(-1, 64)[idx]), p_r)
    assert np.array_equal(to_np(s.reshape(-1, 4)[idx]).view(np.uint32), s_r.view(np.uint32))
    assert np.array_equal(to_np(z.reshape(-1, 4)[idx]).view(np.uint32), z_r.view(np.uint32))


@pytest.mark.parametrize("dtype", [np.float16, np.float32])
@pytest.mark.parametrize("nb,rows,d", [(1, 1, 64), (3, 37, 64), (4, 4096, 128), (2, 1000, 192)])
def test_channelwise_int8_bit_exact(kvq, dtype, nb, rows, d):
    rng = np.random.default_rng(nb * 100 + rows)
    x = (rng.standard_normal((nb, rows, d)) * rng.lognormal(0, 1.5, (nb, 1, d))).astype(dtype)
    x[0, :, 3] = 0                                   # an all-zero column
    c_r, s_r = oracle.quantize_int8_channelwise(x)
    xg = torch.from_numpy(x).cuda()
    c, s = kvq.kvq_quantize_int8_channelwise(xg)
    assert np.array_equal(to_np(c), c_r)
    assert np.array_equal(to_np(s).view(np.uint32), s_r.view(np.uint32))
    for od, tod in ((np.float32, torch.float32), (np.float16, torch.float16)):
        ref = oracle.dequantize_int8_channelwise(c_r, s_r, out_dtype=od)
        got = to_np(kvq.kvq_dequantize_int8_channelwise(c, s, out_dtype=tod))
        assert np.array_equal(got.view(np.uint16 if od == np.float16 else np.uint32),
                              ref.view(np.uint16 if od == np.float16 else np.uint32))


OUT_TOL = 2e-3


def _vals4(vp, vs4, vz4, g):
    """The INT4 reconstructions [..., T, D] of packed values [..., T, D/2]."""
    lead = vp.shape[:-1]
    return oracle.dequantize_int4_group(vp.reshape(-1, 64), vs4.reshape(-1, 128 // g),
                                        vz4.reshape(-1, 128 // g), g).reshape(lead + (128,))


def _abs4(vp, vs4, vz4, g):
    """|c s| + |z| per element [..., T, D]: the two parts the kernel sums separately."""
    lead = vp.shape[:-1]
    p = vp.reshape(-1, 64)
    c = np.empty((p.shape[0], 128), np.float64)
    c[:, 0::2] = p & 15
    c[:, 1::2] = p >> 4
    s = np.repeat(vs4.reshape(-1, 128 // g).astype(np.float64), g, axis=1)
    z = np.repeat(vz4.reshape(-1, 128 // g).astype(np.float64), g, axis=1)
    return (np.abs(c * s) + np.abs(z)).reshape(lead + (128,))


@pytest.mark.parametrize("B,Hq,Hkv,T,g", [(1, 4, 4, 5, 32), (2, 8, 2, 33, 64), (1, 8, 1, 1000, 128),
                                          (2, 16, 4, 4097, 32), (16, 16, 8, 3, 32), (1, 8, 8, 1501, 32),
                                          (4, 8, 8, 100, 64)])
def test_decode_int4_values(kvq, B, Hq, Hkv, T, g):
    k, v = inputs.lognormal_cache(60 + T, B, Hkv, T, n_tensors=2)
    q = inputs.gaussian_queries(61 + T, B, Hq)
    kc, ks = oracle.quantize_int8(k.reshape(-1, 128))
    vp, vs4, vz4 = oracle.quantize_int4_group(v.reshape(-1, 128), g)
    shp = (B, Hkv, T)
    kc, ks = kc.reshape(shp + (128,)), ks.reshape(shp)
    vp, vs4, vz4 = vp.reshape(shp + (64,)), vs4.reshape(shp + (-1,)), vz4.reshape(shp + (-1,))
    ref = oracle.decode_attention(q, k_codes=kc, k_scales=ks, v4=(vp, vs4, vz4, g), want_scores=True)
    qg, kcg, ksg, vpg, vsg, vzg = [torch.from_numpy(np.ascontiguousarray(a)).cuda()
                                   for a in (q, kc, ks, vp, vs4, vz4)]
    out, scores = kvq.kvq_decode_attention_int4v(qg, k_codes=kcg, k_scales=ksg, v_packed=vpg,
                                                 v_scales4=vsg, v_zeros4=vzg, v_group=g, want_scores=True)
    assert np.abs(to_np(out) - ref["out"]).max() <= OUT_TOL
    xh = kc.astype(np.float64) * ks.astype(np.float64)[..., None]
    terms = np.abs(np.repeat(xh, Hq // Hkv, axis=1) * q.astype(np.float64)[:, :, None, :]).sum(-1)
    assert np.all(np.abs(to_np(scores).astype(np.float64) - ref["scores"]) <= 2 * 128 * 2.0 ** -24 * terms + 1e-30)
    check_decode_bound(to_np(out), to_np(scores), ref["scores"], _vals4(vp, vs4, vz4, g), qjl=False,
                       vabs=_abs4(vp, vs4, vz4, g))
    assert kvq.kvq_device_error() == 0


def test_decode_int4_values_7b_layer_sampled(kvq):
    """One 7B-shaped layer: K INT8 and V INT4 (groups of 32) quantized on the GPU, one
    decode step; 6 sampled (batch, head) units re-done by the oracle."""
    B, H, T = 8, 32, 4096
    kv = inputs.lognormal_cache_device(13, (2, B, H, T, 128), n_sigma_dims=(0, 2, 4), device="cuda")
    q = inputs.gaussian_queries_device(31, (B, H, 128), "cuda")
    kc, ks = kvq.kvq_quantize_int8(kv[0])
    vp, vs4, vz4 = kvq.kvq_quantize_int4(kv[1], 32)
    out, scores = kvq.kvq_decode_attention_int4v(q, k_codes=kc, k_scales=ks, v_packed=vp, v_scales4=vs4,
                                                 v_zeros4=vz4, v_group=32, want_scores=True)
    out, scores = to_np(out), to_np(scores)
    n_chain, n_rescale = decode_chain(B, H, T, H, sm_count(), qjl=False)
    rng = np.random.default_rng(8)
    for b, h in zip(rng.integers(0, B, 6), rng.integers(0, H, 6)):
        kc_r, ks_r = oracle.quantize_int8(to_np(kv[0, b, h]))
        vp_r, vs_r, vz_r = oracle.quantize_int4_group(to_np(kv[1, b, h]), 32)
        ref = oracle.decode_attention(to_np(q[b, h])[None, None], k_codes=kc_r[None, None],
                                      k_scales=ks_r[None, None],
                                      v4=(vp_r[None, None], vs_r[None, None], vz_r[None, None], 32),
                                      want_scores=True)
        assert np.abs(out[b, h] - ref["out"][0, 0]).max() <= OUT_TOL
        check_decode_unit(out[b, h][None], scores[b, h][None], ref["scores"][0], _vals4(vp_r, vs_r, vz_r, 32),
                          softmax_scale(), n_chain, n_rescale, vabs=_abs4(vp_r, vs_r, vz_r, 32))


def test_decode_int4_values_unaligned_group_params(kvq):
    """Group parameters that are only 4-byte aligned take the direct-load path."""
    B, Hq, Hkv, T, g = 2, 8, 4, 257, 32
    k, v = inputs.lognormal_cache(77, B, Hkv, T, n_tensors=2)
    q = inputs.gaussian_queries(78, B, Hq)
    kc, ks = oracle.quantize_int8(k.reshape(-1, 128))
    vp, vs4, vz4 = oracle.quantize_int4_group(v.reshape(-1, 128), g)
    shp = (B, Hkv, T)
    ref = oracle.decode_attention(q, k_codes=kc.reshape(shp + (128,)), k_scales=ks.reshape(shp),
                                  v4=(vp.reshape(shp + (64,)), vs4.reshape(shp + (4,)), vz4.reshape(shp + (4,)), g),
                                  want_scores=True)
    # copy the parameters into buffers offset by one float
    sbuf = torch.zeros(vs4.size + 1, dtype=torch.float32, device="cuda")
    zbuf = torch.zeros(vz4.size + 1, dtype=torch.float32, device="cuda")
    sbuf[1:] = torch.from_numpy(vs4.reshape(-1)).cuda()
    zbuf[1:] = torch.from_numpy(vz4.reshape(-1)).cuda()
    qg, kcg, ksg, vpg = [torch.from_numpy(np.ascontiguousarray(a)).cuda() for a in
                         (q, kc.reshape(shp + (128,)), ks.reshape(shp), vp.reshape(shp + (64,)))]
    out, scores = kvq.kvq_decode_attention_int4v(qg, k_codes=kcg, k_scales=ksg, v_packed=vpg,
                                                 v_scales4=sbuf[1:], v_zeros4=zbuf[1:], v_group=g, want_scores=True)
    assert np.abs(to_np(out) - ref["out"]).max() <= OUT_TOL
    check_decode_bound(to_np(out), to_np(scores), ref["scores"],
                       _vals4(vp.reshape(shp + (64,)), vs4, vz4, g), qjl=False,
                       vabs=_abs4(vp.reshape(shp + (64,)), vs4, vz4, g))
