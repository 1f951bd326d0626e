"""GPU parity of the QJL sketch (tcgen05 encode, query sketch) against the CPU oracle.

Sign words: bit-exact except at coordinates where the oracle's fp64 |(S k)_i| is below
1e-4 ||k||.  Norms: the correctly rounded fp16 of the fp64 norm (bit-exact).  Query
sketch: within the fp32 accumulation bound 128 * 2^-23 * sum_j |S_ij q_j|.
"""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_quantization_absmax_b200 import inputs
from tests._helpers import bit_mismatch_outside_band, to_np, words_u32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvq():
    from kv_cache_quantization_absmax_b200 import kvq as m
    return m


def _encode_and_compare(kvq, keys_np, S_np, max_band_frac=1e-3):
    keys = torch.from_numpy(keys_np).cuda()
    S = torch.from_numpy(S_np).cuda()
    words, norms = kvq.kvq_qjl_encode(keys, S)
    flat = keys_np.reshape(-1, 128)
    w_ref, n_ref, u = oracle.qjl_encode(flat, S_np, want_u=True)
    n64 = np.sqrt((flat.astype(np.float64) ** 2).sum(1))
    outside, total = bit_mismatch_outside_band(words_u32(words).reshape(w_ref.shape), w_ref, u, n64)
    assert outside == 0, f"{outside} sign bits differ outside the 1e-4*||k|| band ({total} total)"
    assert total <= max_band_frac * u.size
    assert np.array_equal(to_np(norms).reshape(-1).view(np.uint16), n_ref.view(np.uint16))
    return words, norms, w_ref, n_ref


@pytest.mark.parametrize("n", [1, 127, 128, 129, 1000, 4096 + 77])
@pytest.mark.parametrize("m", [256, 128, 32])
def test_encode_parity_small(kvq, n, m):
    keys = inputs.lognormal_cache(4, 1, 1, n)[0].reshape(n, 128)
    S = inputs.sketch_matrix(m, 128)
    _encode_and_compare(kvq, keys, S)


def test_encode_special_keys(kvq):
    S = inputs.sketch_matrix(256, 128)
    keys = inputs.lognormal_cache(8, 1, 1, 300)[0].reshape(300, 128)
    keys[0] = 0                                 # zero key: all bits set, norm 0
    keys[1] = keys[2] * np.float16(4)           # scaled copy: same bits
    keys[3, :] = np.float16(65504)              # largest fp16 values
    keys[4, :] = np.float16(2.0 ** -24)         # smallest subnormals
    words, norms, w_ref, n_ref = _encode_and_compare(kvq, keys, S)
    w = words_u32(words)
    assert np.all(w[0] == 0xFFFFFFFF) and float(to_np(norms)[0]) == 0.0
    assert np.array_equal(w[1], w[2])


def _near_midpoint_pairs(scale, count, rng, within):
    """fp16 pairs (a, b) whose fp64 norm lies within `within` (relative) of a midpoint
    between two fp16 values."""
    out = []
    while len(out) < count:
        a = rng.uniform(0.5, 1.0, 4096).astype(np.float16) * np.float16(scale)
        b = rng.uniform(0.5, 1.0, 4096).astype(np.float16) * np.float16(scale)
        n = np.hypot(a.astype(np.float64), b.astype(np.float64))
        lo = n.astype(np.float16).astype(np.float64)
        nxt = np.nextafter(n.astype(np.float16), np.float16(np.inf)).astype(np.float64)
        prv = np.nextafter(n.astype(np.float16), np.float16(-np.inf)).astype(np.float64)
        mid = np.where(n >= lo, (lo + nxt) / 2, (lo + prv) / 2)
        hit = np.abs(n / mid - 1) < within
        out += list(zip(a[hit], b[hit]))
    return out[:count]


def test_encode_norm_slow_paths(kvq):
    """Norms near fp16 rounding midpoints, bit-exact against the oracle: two large
    components within 2^-20 of a midpoint (either side of the fp32 fast path's 2^-21
    margin); the same at 2^-19 with subnormal components added, whose squares span more
    than 53 bits; exact midpoints (the tie rule); and exact midpoints with small squares
    that the index-order fp64 sum drops or keeps depending on their position, scaled by
    powers of two."""
    from tests.test_oracle_pins import tie_keys
    rng = np.random.default_rng(77)
    keys = np.zeros((256, 128), np.float16)
    for i, (a, b) in enumerate(_near_midpoint_pairs(1.0, 128, rng, 2.0 ** -20)):
        keys[i, 3], keys[i, 90] = a, b
    for i, (a, b) in enumerate(_near_midpoint_pairs(256.0, 128, rng, 2.0 ** -19)):
        keys[128 + i, 0], keys[128 + i, 127] = a, b
        keys[128 + i, 1:120:7] = np.float16(2.0 ** -24) * (1 + i % 5)
    ties = tie_keys()
    scaled = [ties[:2] * np.float16(2.0 ** k) for k in range(-8, 5)]
    scaled += [ties[2:] * np.float16(2.0 ** k) for k in range(0, 8)]
    keys = np.concatenate([keys] + scaled)
    S = inputs.sketch_matrix(256, 128)
    _encode_and_compare(kvq, keys, S)


def test_encode_norm_slow_queue_overflow(kvq):
    """Every key takes the slow norm and each CTA gets three tiles (384 such keys, more
    than its 256-entry queue): queued keys and the overflow computed inline, all
    bit-exact against the oracle."""
    from tests.test_oracle_pins import tie_keys
    rng = np.random.default_rng(78)
    base = np.zeros((96, 128), np.float16)
    for i, (a, b) in enumerate(_near_midpoint_pairs(4.0, 96, rng, 2.0 ** -22)):
        base[i, i % 128], base[i, (i * 37 + 5) % 128] = a, b   # distinct: 36 i != -5 mod 128
    ties = tie_keys()
    base = np.concatenate([base] + [ties * np.float16(2.0 ** k) for k in range(0, 5)])
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    n = sms * 128 * 3
    keys = np.ascontiguousarray(np.resize(base, (n, 128)))
    S = inputs.sketch_matrix(256, 128)
    _encode_and_compare(kvq, keys, S)


def test_encode_full_size_sampled(kvq):
    """The key-sketch workload: keys [1, 32, 32768, 128] (1,048,576 keys, per-channel
    LogNormal std), S [256, 128] from seed 7; 2048 sampled keys checked against the oracle."""
    keys = inputs.lognormal_cache_device(4, (1, 32, 32768, 128), n_sigma_dims=(1, 3), device="cuda")
    S_np = inputs.sketch_matrix(256, 128)
    S = torch.from_numpy(S_np).cuda()
    words, norms = kvq.kvq_qjl_encode(keys, S)
    torch.cuda.synchronize()
    assert kvq.kvq_device_error() == 0
    flat = keys.view(-1, 128)
    rng = np.random.default_rng(1)
    idx = np.unique(np.concatenate([rng.integers(0, flat.shape[0], 2048), [0, flat.shape[0] - 1]]))
    sel = to_np(flat[torch.from_numpy(idx).cuda()])
    w_ref, n_ref, u = oracle.qjl_encode(sel, S_np, want_u=True)
    n64 = np.sqrt((sel.astype(np.float64) ** 2).sum(1))
    w_gpu = words_u32(words).reshape(-1, 8)[idx]
    outside, _ = bit_mismatch_outside_band(w_gpu, w_ref, u, n64)
    assert outside == 0
    assert np.array_equal(to_np(norms).reshape(-1)[idx].view(np.uint16), n_ref.view(np.uint16))


@pytest.mark.parametrize("n_q", [1, 32, 128, 200])
@pytest.mark.parametrize("m", [256, 64])
def test_query_sketch_parity(kvq, n_q, m):
    q = inputs.gaussian_queries(40, 1, n_q)[0]
    S = inputs.sketch_matrix(m, 128)
    v = to_np(kvq.kvq_qjl_query_sketch(torch.from_numpy(q).cuda(), torch.from_numpy(S).cuda()))
    v64, _ = oracle.qjl_query_sketch(q, S)
    bound = 128 * 2.0 ** -23 * (np.abs(q.astype(np.float64))[:, None, :] *
                                np.abs(S.astype(np.float64))[None, :, :]).sum(-1)
    assert np.all(np.abs(v.astype(np.float64) - v64) <= bound)
