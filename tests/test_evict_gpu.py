"""GPU parity of attention-sink eviction ("Q-TensorFormer" model card, section 6,
Attention-Sink Dynamic Eviction) against the CPU oracle.

- Mass decode: the decode output as the plain decode step (max-abs 2e-3 and the
  arithmetic bound of tests/_helpers.py, check_decode_bound); the added
  attention mass within 2e-5 relative + 1e-7 per head of the oracle's (fp32 scores
  and exp2 on the GPU against the oracle's exactly summed scores).
- Selection: bit-exact (same int32 indices) against the oracle run on the same fp32
  mass array.
- Compaction: byte-exact.
"""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_quantization_absmax_b200 import inputs
from tests._helpers import check_decode_bound, to_np

pytestmark = pytest.mark.gpu

OUT_TOL = 2e-3


@pytest.fixture(scope="module")
def kvq():
    from kv_cache_quantization_absmax_b200 import kvq as m
    return m


def _cuda(*arrs):
    return [torch.from_numpy(np.ascontiguousarray(a)).cuda() for a in arrs]


def _int8_cache(seed, B, Hkv, T, Hq):
    k, v = inputs.lognormal_cache(seed, B, Hkv, T, n_tensors=2)
    q = inputs.gaussian_queries(seed + 1, B, Hq)
    kc, ks = oracle.quantize_int8(k.reshape(-1, 128))
    vc, vs = oracle.quantize_int8(v.reshape(-1, 128))
    shp = (B, Hkv, T)
    return q, dict(k_codes=kc.reshape(shp + (128,)), k_scales=ks.reshape(shp),
                   v_codes=vc.reshape(shp + (128,)), v_scales=vs.reshape(shp))


def _qjl_cache(seed, B, Hkv, T, Hq, m=256):
    k, v = inputs.lognormal_cache(seed, B, Hkv, T, n_tensors=2)
    q = inputs.gaussian_queries(seed + 1, B, Hq)
    S = inputs.sketch_matrix(m, 128)
    w, n = oracle.qjl_encode(k.reshape(-1, 128), S)
    vc, vs = oracle.quantize_int8(v.reshape(-1, 128))
    shp = (B, Hkv, T)
    return q, dict(k_words=w.reshape(shp + (m // 32,)), k_norms=n.reshape(shp), S=S,
                   v_codes=vc.reshape(shp + (128,)), v_scales=vs.reshape(shp))


def _gpu_kwargs(c):
    g = {}
    for k, v in c.items():
        if k == "S":
            g["sketch"] = _cuda(v)[0]
        elif k == "k_words":
            g[k] = _cuda(v.view(np.int32))[0]
        else:
            g[k] = _cuda(v)[0]
    return g


def _vals(c):
    """The cache's dequantized value rows [B, Hkv, T, D]."""
    vc, vs = c["v_codes"], c["v_scales"]
    return oracle.dequantize_int8(vc.reshape(-1, 128), vs.reshape(-1)).reshape(vc.shape)


def _mass_tol(ref, Hq):
    return 2e-5 * np.abs(ref) + 1e-7 * Hq


@pytest.mark.parametrize("fmt,B,Hq,Hkv,T", [("int8", 1, 1, 1, 1), ("int8", 2, 8, 2, 33),
                                            ("int8", 1, 8, 1, 1000), ("int8", 2, 16, 4, 4097),
                                            ("int8", 3, 24, 3, 70), ("qjl", 1, 4, 1, 7),
                                            ("qjl", 2, 8, 2, 1500), ("qjl", 1, 32, 8, 2049),
                                            ("qjl", 1, 4, 1, 8), ("qjl", 2, 8, 2, 1504)])
@pytest.mark.parametrize("want_scores", [False, True])
def test_mass_decode_parity(kvq, fmt, B, Hq, Hkv, T, want_scores):
    make = _int8_cache if fmt == "int8" else _qjl_cache
    q, c = make(500 + T, B, Hkv, T, Hq)
    ref = oracle.decode_attention(q, want_scores=True, **c)
    ref_out = ref["out"]
    ref_mass = oracle.attention_mass(q, **c)
    init = np.random.default_rng(T).random((B, T), dtype=np.float32)
    mass = _cuda(init)[0]
    g = _gpu_kwargs(c)
    out, scores = kvq.kvq_decode_attention_mass(_cuda(q)[0], mass, want_scores=want_scores, **g)
    assert np.abs(to_np(out) - ref_out).max() <= OUT_TOL
    if scores is None:   # the same kernel's scores, from the plain decode step
        _, scores = kvq.kvq_decode_attention(_cuda(q)[0], want_scores=True, **g)
    check_decode_bound(to_np(out), to_np(scores), ref["scores"], _vals(c), qjl=fmt == "qjl",
                       v_scales=c["v_scales"] if fmt == "qjl" else None)
    if not want_scores:
        scores = None
    err = np.abs(to_np(mass).astype(np.float64) - (init.astype(np.float64) + ref_mass))
    assert np.all(err <= _mass_tol(ref_mass, Hq) + 2.0 ** -23 * (init + ref_mass)), float(err.max())
    assert (scores is not None) == want_scores
    assert kvq.kvq_device_error() == 0


def test_mass_accumulates_over_steps(kvq):
    """Three decode steps (three queries) add up: mass = sum of the oracle's masses."""
    B, Hq, Hkv, T = 2, 8, 2, 777
    _, c = _int8_cache(610, B, Hkv, T, Hq)
    g = _gpu_kwargs(c)
    mass = torch.zeros((B, T), dtype=torch.float32, device="cuda")
    ref = np.zeros((B, T))
    for step in range(3):
        q = inputs.gaussian_queries(620 + step, B, Hq)
        kvq.kvq_decode_attention_mass(_cuda(q)[0], mass, **g)
        ref += oracle.attention_mass(q, **c)
    err = np.abs(to_np(mass).astype(np.float64) - ref)
    assert np.all(err <= 3 * _mass_tol(ref, Hq)), float(err.max())
    # each step's probabilities sum to one per head
    assert abs(float(to_np(mass).astype(np.float64).sum()) - 3 * B * Hq) <= 1e-3


def test_mass_rejects_missing_output_and_mass(kvq):
    import ctypes
    q, c = _int8_cache(630, 1, 2, 50, 2)
    g = _gpu_kwargs(c)
    qg = _cuda(q)[0]
    out = torch.empty((1, 2, 128), dtype=torch.float32, device="cuda")
    mass = torch.zeros((1, 50), dtype=torch.float32, device="cuda")
    a = kvq.make_decode_mass_args(qg, mass, out=out, **g)
    need = int(kvq.lib.kvq_decode_mass_workspace_bytes(ctypes.byref(a)))
    assert need > 0
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    a.base.workspace, a.base.workspace_bytes = ws.data_ptr(), need - 1
    assert kvq.lib.kvq_decode_attention_mass(ctypes.byref(a), None) == kvq.KVQ_ERR_WORKSPACE
    a.base.workspace_bytes = need
    a.attn_mass = None
    assert kvq.lib.kvq_decode_attention_mass(ctypes.byref(a), None) == kvq.KVQ_ERR_INVALID_ARG
    a.attn_mass = mass.data_ptr()
    a.base.out = None
    assert kvq.lib.kvq_decode_attention_mass(ctypes.byref(a), None) == kvq.KVQ_ERR_INVALID_ARG
    a.base.out = out.data_ptr()
    assert kvq.lib.kvq_decode_attention_mass(ctypes.byref(a), None) == kvq.KVQ_OK
    torch.cuda.synchronize()


def _mass_cases():
    rng = np.random.default_rng(7)
    yield "uniform", rng.random((3, 5000), dtype=np.float32), 4, 1000
    yield "ties", rng.integers(0, 6, (2, 4099)).astype(np.float32), 4, 2048
    yield "signed", np.where(rng.random((2, 3000)) < 0.3, 0.0,
                             rng.standard_normal((2, 3000))).astype(np.float32), 2, 1500
    neg0 = np.zeros((1, 2000), np.float32)
    neg0[0, ::3] = -0.0
    neg0[0, 5::7] = 1e-38  # subnormal-adjacent values above zero
    yield "zeros", neg0, 4, 900
    yield "equal", np.full((2, 1025), 0.25, np.float32), 4, 512
    yield "keep_all", rng.random((2, 300), dtype=np.float32), 4, 300
    yield "sinks_only", rng.random((2, 300), dtype=np.float32), 16, 16
    yield "no_sinks", rng.random((4, 1024), dtype=np.float32), 0, 100
    yield "one_token", rng.random((5, 1), dtype=np.float32), 0, 1
    yield "keep_one", rng.random((2, 2000), dtype=np.float32), 0, 1
    yield "keep_all_but_one", rng.random((2, 2000), dtype=np.float32), 4, 1999
    yield "long", rng.random((4, 131072), dtype=np.float32), 4, 65536
    yield "tiny_spread", (1.0 + rng.integers(0, 3, (1, 70000)) * 2.0 ** -23).astype(np.float32), 4, 20000


@pytest.mark.parametrize("name,mass,n_sink,n_keep", list(_mass_cases()), ids=[c[0] for c in _mass_cases()])
def test_evict_select_exact(kvq, name, mass, n_sink, n_keep):
    ref = oracle.evict_select(mass, n_sink, n_keep)
    kept = kvq.kvq_evict_select(_cuda(mass)[0], n_sink, n_keep)
    assert np.array_equal(to_np(kept), ref)


def test_evict_select_zero_keep_and_bad_args(kvq):
    m = torch.rand((2, 100), device="cuda")
    k = kvq.kvq_evict_select(m, 0, 0)
    assert k.shape == (2, 0)
    for n_sink, n_keep in [(5, 4), (0, 101), (-1, 3)]:
        with pytest.raises(kvq.KvqError):
            kvq.kvq_evict_select(m, n_sink, max(n_keep, 0), kept=torch.empty((2, 200), dtype=torch.int32,
                                                                             device="cuda"))


@pytest.mark.parametrize("shape,dtype", [((2, 3, 100, 128), torch.int8), ((2, 3, 100), torch.float32),
                                         ((1, 8, 257, 8), torch.int32), ((3, 2, 50), torch.float16),
                                         ((2, 2, 90, 3), torch.uint8), ((2, 4, 64, 2), torch.float32),
                                         ((1, 1, 4096, 64), torch.uint8)])
def test_gather_rows_exact(kvq, shape, dtype):
    B, H, T = shape[:3]
    g = torch.Generator().manual_seed(int(np.prod(shape)))
    src_cpu = torch.randint(-100, 100, shape, generator=g).to(dtype)
    mass = np.random.default_rng(T).random((B, T), dtype=np.float32)
    n_keep = max(1, T // 2)
    kept = oracle.evict_select(mass, min(4, n_keep), n_keep)
    ref = oracle.gather_rows(src_cpu.numpy(), kept)
    # dst with spare rows: rows from n_keep on are left as they are
    dst = torch.full((B, H, n_keep + 3) + tuple(shape[3:]), 7, dtype=dtype, device="cuda")
    kvq.kvq_gather_rows(src_cpu.cuda(), _cuda(kept)[0], dst=dst)
    d = dst.cpu().numpy()
    assert np.array_equal(d[:, :, :n_keep], ref)
    assert np.all(d[:, :, n_keep:] == 7)


def test_gather_rows_unaligned_views(kvq):
    """Base addresses off every alignment (1-byte offsets) take the byte path, exactly."""
    B, H, T, R = 2, 3, 200, 40
    raw = torch.randint(0, 255, (B * H * T * R + 1,), dtype=torch.uint8, device="cuda")
    src = raw[1:].view(B, H, T, R)
    kept = torch.from_numpy(oracle.evict_select(np.random.default_rng(1).random((B, T), dtype=np.float32),
                                                4, 50)).cuda()
    out_raw = torch.zeros((B * H * 50 * R + 3,), dtype=torch.uint8, device="cuda")
    dst = out_raw[3:].view(B, H, 50, R)
    kvq.kvq_gather_rows(src, kept, dst=dst)
    assert np.array_equal(to_np(dst), oracle.gather_rows(to_np(src), to_np(kept)))


def test_gather_rows_bad_index_records_error(kvq):
    """A kept index outside the source rows is skipped by the kernel's bounds check and
    reported through kvq_device_error (code 0x301); the other rows are copied."""
    src = torch.arange(2 * 1 * 10, dtype=torch.float32, device="cuda").view(2, 1, 10)
    kept = torch.tensor([[0, 3, 10], [1, 2, 9]], dtype=torch.int32, device="cuda")
    dst = torch.full((2, 1, 3), -1.0, device="cuda")
    kvq.kvq_gather_rows(src, kept, dst=dst)
    assert kvq.kvq_device_error() == 0x301
    assert to_np(dst).tolist() == [[[0.0, 3.0, -1.0]], [[11.0, 12.0, 19.0]]]
    assert kvq.kvq_device_error() == 0


@pytest.mark.parametrize("fmt", ["int8", "qjl"])
def test_evict_pipeline_end_to_end(kvq, fmt):
    """Two mass decode steps, selection of 4 sinks + 300 tokens, compaction of every cache
    array, then a decode over the compacted cache: equal to the oracle's decode over the
    oracle's compaction of the same selection."""
    B, Hq, Hkv, T, n_sink, n_keep = 2, 8, 2, 1000, 4, 304
    make = _int8_cache if fmt == "int8" else _qjl_cache
    _, c = make(700, B, Hkv, T, Hq)
    g = _gpu_kwargs(c)
    mass = torch.zeros((B, T), dtype=torch.float32, device="cuda")
    for step in range(2):
        q = inputs.gaussian_queries(710 + step, B, Hq)
        kvq.kvq_decode_attention_mass(_cuda(q)[0], mass, **g)
    kept = kvq.kvq_evict_select(mass, n_sink, n_keep)
    ref_kept = oracle.evict_select(to_np(mass), n_sink, n_keep)
    assert np.array_equal(to_np(kept), ref_kept)
    gc = {k: (kvq.kvq_gather_rows(v, kept) if k != "sketch" else v) for k, v in g.items()}
    cc = {k: (oracle.gather_rows(v, ref_kept) if k != "S" else v) for k, v in c.items()}
    for k in gc:
        if k != "sketch":
            want = cc["k_words"].view(np.int32) if k == "k_words" else cc[k]
            assert np.array_equal(to_np(gc[k]), want), k
    q = inputs.gaussian_queries(720, B, Hq)
    out, scores = kvq.kvq_decode_attention(_cuda(q)[0], want_scores=True, **gc)
    ref = oracle.decode_attention(q, want_scores=True, **cc)
    assert np.abs(to_np(out) - ref["out"]).max() <= OUT_TOL
    check_decode_bound(to_np(out), to_np(scores), ref["scores"], _vals(cc), qjl=fmt == "qjl",
                       v_scales=cc["v_scales"] if fmt == "qjl" else None)
    assert kvq.kvq_device_error() == 0


def test_evict_llama7b_layer_sampled(kvq):
    """One layer of the 7B-shaped cache (batch 8, 32 heads, 4096 tokens) keeping 4 sinks
    + 2044 tokens: GPU quantize, mass decode, selection, compaction.  Mass of two sampled
    batch rows re-done by the oracle from the GPU codes; selection exact on the GPU mass;
    compaction exact on two sampled (batch, head) units."""
    B, H, T, n_sink, n_keep = 8, 32, 4096, 4, 2048
    kv = inputs.lognormal_cache_device(3, (2, B, H, T, 128), n_sigma_dims=(0, 2, 4), device="cuda")
    q = inputs.gaussian_queries_device(33, (B, H, 128), "cuda")
    kc, ks = kvq.kvq_quantize_int8(kv[0])
    vc, vs = kvq.kvq_quantize_int8(kv[1])
    del kv
    mass = torch.zeros((B, T), dtype=torch.float32, device="cuda")
    kvq.kvq_decode_attention_mass(q, mass, k_codes=kc, k_scales=ks, v_codes=vc, v_scales=vs)
    kept = kvq.kvq_evict_select(mass, n_sink, n_keep)
    kc2 = kvq.kvq_gather_rows(kc, kept)
    ks2 = kvq.kvq_gather_rows(ks, kept)
    m_np = to_np(mass)
    assert np.array_equal(to_np(kept), oracle.evict_select(m_np, n_sink, n_keep))
    for b in (1, 6):
        ref = oracle.attention_mass(to_np(q[b:b + 1]), k_codes=to_np(kc[b:b + 1]), k_scales=to_np(ks[b:b + 1]))
        err = np.abs(m_np[b].astype(np.float64) - ref[0])
        assert np.all(err <= _mass_tol(ref[0], H)), float(err.max())
    k_np = to_np(kept)
    for b, h in ((0, 5), (7, 31)):
        assert np.array_equal(to_np(kc2[b, h]), to_np(kc[b, h])[k_np[b]])
        assert np.array_equal(to_np(ks2[b, h]), to_np(ks[b, h])[k_np[b]])
    assert kvq.kvq_device_error() == 0


def test_gather_rows_multi_exact(kvq):
    """One launch compacts arrays of different row sizes and alignments (INT8 codes,
    fp32 scales, int32 sign words, fp16 norms, odd-byte rows at an odd offset) exactly as
    the oracle's compaction of each."""
    B, H, T = 3, 4, 700
    g = torch.Generator().manual_seed(5)
    shapes = [((B, H, T, 128), torch.int8), ((B, H, T), torch.float32), ((B, H, T, 8), torch.int32),
              ((B, H, T), torch.float16), ((B, H, T, 3), torch.uint8)]
    srcs = [torch.randint(-100, 100, sh, generator=g).to(dt).cuda() for sh, dt in shapes]
    raw = torch.randint(0, 255, (B * H * T * 5 + 1,), dtype=torch.uint8).cuda()
    srcs.append(raw[1:].view(B, H, T, 5))                                  # 1-byte aligned rows
    mass = np.random.default_rng(11).random((B, T), dtype=np.float32)
    kept = oracle.evict_select(mass, 4, 333)
    dsts = kvq.kvq_gather_rows_multi(srcs, _cuda(kept)[0])
    for x, y in zip(srcs, dsts):
        assert np.array_equal(to_np(y), oracle.gather_rows(to_np(x), kept))
    assert kvq.kvq_device_error() == 0


def test_gather_rows_multi_matches_single_calls_at_layer_size(kvq):
    """The 7B-shaped layer's K/V codes and scales [8, 32, 4096] compacted to 2048 tokens:
    one multi-array launch equals four single-array launches, byte for byte."""
    B, H, T = 8, 32, 4096
    g = torch.Generator(device="cuda").manual_seed(3)
    codes = [torch.randint(-127, 128, (B, H, T, 128), generator=g, device="cuda", dtype=torch.int32).to(torch.int8)
             for _ in range(2)]
    scales = [torch.rand((B, H, T), generator=g, device="cuda") for _ in range(2)]
    mass = torch.rand((B, T), generator=g, device="cuda")
    kept = kvq.kvq_evict_select(mass, 4, 2048)
    multi = kvq.kvq_gather_rows_multi(codes + scales, kept)
    for x, y in zip(codes + scales, multi):
        assert torch.equal(y, kvq.kvq_gather_rows(x, kept))
    assert kvq.kvq_device_error() == 0
