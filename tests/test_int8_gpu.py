"""GPU parity of the INT8 path (quantize, dequantize, scores) against the CPU oracle.

Codes, scales and dequantized values must be bit-exact; scores must agree within the
fp32 summation bound 2 * D * 2^-24 * sum_j |q_j x_hat_j| (the two sides sum in
different orders).  All calls go through the C ABI.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from kv_cache_quantization_absmax_b200 import inputs
from tests._helpers import to_np

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def kvq():
    from kv_cache_quantization_absmax_b200 import kvq as m
    return m


def _check_quant(kvq, x_np):
    x = torch.from_numpy(x_np).cuda()
    codes, scales = kvq.kvq_quantize_int8(x)
    c_ref, s_ref = oracle.quantize_int8(x_np.reshape(-1, x_np.shape[-1]))
    c_gpu, s_gpu = to_np(codes).reshape(c_ref.shape), to_np(scales).reshape(s_ref.shape)
    assert np.array_equal(s_gpu.view(np.uint32), s_ref.view(np.uint32))
    bad = np.nonzero(c_gpu != c_ref)
    assert bad[0].size == 0, f"{bad[0].size} codes differ, first at {bad[0][:3]}, {bad[1][:3]}"
    return codes, scales, c_ref, s_ref


@pytest.mark.parametrize("case", json.load(open(os.path.join(GOLDEN, "int8_worked_examples.json")))["cases"],
                         ids=lambda c: c["name"])
def test_worked_examples_on_gpu(kvq, case):
    dt = np.float32 if case["dtype"] == "f32" else np.float16
    row = np.array([float.fromhex(v) for v in case["x"]]).astype(dt)
    x = np.zeros((3, 16), dt)   # the kernels take rows of >= 16 elements: pad with zeros
    x[1, :4] = row
    x[2, :4] = -row
    codes, scales, _, _ = _check_quant(kvq, x)
    assert to_np(codes)[1, :4].tolist() == case["codes"]
    assert float(to_np(scales)[1]) == float.fromhex(case["scale"])


@pytest.mark.parametrize("dtype", [np.float16, np.float32])
@pytest.mark.parametrize("d", [16, 32, 48, 64, 128, 256, 512, 1024, 2048, 4096, 8192, 2000 * 16 // 16])
def test_quantize_dequant_parity(kvq, dtype, d):
    if d % 16:
        pytest.skip("d must be a multiple of 16")
    n = max(3, min(5000, (1 << 20) // d)) + 7          # ragged row count
    x, _, _ = inputs.sweep_matrix(n * d, d, dtype, 99, n_rows=n)
    x[1] = 0                                            # zero row
    x[2] = x[2, 0]                                      # all-equal row
    if dtype == np.float32:                             # subnormal scale, clamp binds
        tiny = np.float32(2.0) ** -149
        x[3] = 0
        x[3, :3] = [190 * tiny, -190 * tiny, tiny]
    codes, scales, c_ref, s_ref = _check_quant(kvq, x)
    for out_dt, np_dt in ((torch.float32, np.float32), (torch.float16, np.float16)):
        xh = to_np(kvq.kvq_dequantize_int8(codes, scales, out_dt))
        ref = oracle.dequantize_int8(c_ref, s_ref, np_dt)
        assert np.array_equal(xh.view(np.uint32 if np_dt == np.float32 else np.uint16),
                              ref.view(np.uint32 if np_dt == np.float32 else np.uint16))


@pytest.mark.parametrize("d", [128, 1024, 8192])
@pytest.mark.parametrize("qdtype", [np.float32, np.float16])
def test_int8_scores_parity(kvq, d, qdtype):
    n = 3001
    x, q, _ = inputs.sweep_matrix(n * d, d, np.float32, 7, n_rows=n)
    q = q.astype(qdtype)
    c_ref, s_ref = oracle.quantize_int8(x)
    codes = torch.from_numpy(c_ref).cuda()
    scales = torch.from_numpy(s_ref).cuda()
    got = to_np(kvq.kvq_int8_scores(torch.from_numpy(q).cuda(), codes, scales)).astype(np.float64)
    ref = oracle.int8_scores(q, c_ref, s_ref).astype(np.float64)
    xh = oracle.dequantize_int8(c_ref, s_ref).astype(np.float64)
    bound = 2 * d * 2.0 ** -24 * np.abs(xh * q.astype(np.float64)[None, :]).sum(1)
    assert np.all(np.abs(got - ref) <= bound)


def test_zero_rows_is_a_no_op(kvq):
    x = torch.empty((0, 128), dtype=torch.float16, device="cuda")
    codes, scales = kvq.kvq_quantize_int8(x)
    assert codes.shape == (0, 128) and scales.shape == (0,)
    out = kvq.kvq_dequantize_int8(codes, scales)
    assert out.shape == (0, 128)


def test_outlier_layer_roundtrip(kvq):
    """The one-layer cache with outlier channels 3 and 77 (x10), K and V."""
    k, v, q = inputs.outlier_layer(seed=0)
    for t in (k, v):
        codes, scales, c_ref, s_ref = _check_quant(kvq, t)
        xh = to_np(kvq.kvq_dequantize_int8(codes, scales)).reshape(-1, 128).astype(np.float64)
        err = np.abs(xh - t.reshape(-1, 128).astype(np.float64))
        slack = np.spacing(np.abs(xh).astype(np.float32)).astype(np.float64)
        assert np.all(err <= s_ref[:, None].astype(np.float64) / 2 + slack)


@pytest.mark.parametrize("dtype", [np.float16, np.float32])
def test_sweep_sampled_rows_large(kvq, dtype):
    """1e8 elements at D = 1024 in the launch configuration of the benchmark; rows are
    sampled and checked bit-exactly against the oracle."""
    d = 1024
    total = 10 ** 8
    n = total // d
    x_np, _, _ = inputs.sweep_matrix(total, d, dtype, 3)
    x = torch.from_numpy(x_np).cuda()
    codes, scales = kvq.kvq_quantize_int8(x)
    xh = kvq.kvq_dequantize_int8(codes, scales, torch.float32)
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([rng.integers(0, n, 400), [0, n - 1]]))
    c_ref, s_ref = oracle.quantize_int8(x_np[rows])
    assert np.array_equal(to_np(codes)[rows], c_ref)
    assert np.array_equal(to_np(scales)[rows], s_ref)
    assert np.array_equal(to_np(xh)[rows], oracle.dequantize_int8(c_ref, s_ref))
