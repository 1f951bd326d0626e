"""GPU parity of channel-wise INT8 and group-wise INT4 quantize / dequantize against the
CPU oracle: codes, packed nibbles, scales, zero points and dequantized values bit-exact."""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_quantization_absmax_b200 import inputs
from tests._helpers import to_np

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
