"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every
entry point include/kvq.h declares, and rejects bad arguments before launching anything.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def kvq():
    from kv_cache_quantization_absmax_b200 import kvq as m
    return m


def _declared():
    src = open(os.path.join(ROOT, "include", "kvq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kvq_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol(kvq):
    names = _declared()
    assert {"kvq_quantize_int8", "kvq_dequantize_int8", "kvq_qjl_encode",
            "kvq_decode_attention"} <= set(names)
    for n in names:
        assert hasattr(kvq.lib, n), n
    assert kvq.lib.kvq_abi_version() == kvq.ABI_VERSION == 2


def test_status_strings(kvq):
    for s in range(6):
        assert kvq.lib.kvq_status_string(s)


def _p(v):
    return ctypes.c_void_p(v)


A16 = 0x10000          # a 16-byte aligned dummy address (never dereferenced: checks fail first)


def test_quantize_rejects_bad_arguments(kvq):
    L = kvq.lib
    E = kvq.KVQ_ERR_INVALID_ARG
    assert L.kvq_quantize_int8(_p(A16), 1, 10, 100, _p(A16), _p(A16), None) == E   # d % 16
    assert L.kvq_quantize_int8(_p(A16), 1, -1, 128, _p(A16), _p(A16), None) == E   # n < 0
    assert L.kvq_quantize_int8(_p(A16), 7, 10, 128, _p(A16), _p(A16), None) == E   # dtype
    assert L.kvq_quantize_int8(None, 1, 10, 128, _p(A16), _p(A16), None) == E      # null
    assert L.kvq_quantize_int8(_p(A16 + 8), 1, 10, 128, _p(A16), _p(A16), None) == E  # misaligned
    assert L.kvq_quantize_int8(_p(A16), 1, 10, 128, _p(A16), _p(A16 + 2), None) == E
    assert L.kvq_quantize_int8(_p(A16), 1, 10, 1 << 20, _p(A16), _p(A16), None) == E  # too wide
    assert L.kvq_quantize_int8(None, 1, 0, 128, None, None, None) == kvq.KVQ_OK     # no rows
    assert L.kvq_dequantize_int8(_p(A16), _p(A16), 10, 24, _p(A16), 0, None) == E
    assert L.kvq_dequantize_int8(_p(A16), _p(A16), 10, 128, _p(A16 + 4), 0, None) == E
    assert L.kvq_int8_scores(_p(A16), 0, _p(A16), _p(A16), 10, 16384, _p(A16), None) == E


def test_qjl_rejects_bad_arguments(kvq):
    L = kvq.lib
    assert L.kvq_qjl_encode(_p(A16), 10, 64, _p(A16), 256, _p(A16), _p(A16), None) == kvq.KVQ_ERR_UNSUPPORTED
    assert L.kvq_qjl_encode(_p(A16), 10, 128, _p(A16), 512, _p(A16), _p(A16), None) == kvq.KVQ_ERR_UNSUPPORTED
    assert L.kvq_qjl_encode(_p(A16), 10, 128, _p(A16), 100, _p(A16), _p(A16), None) == kvq.KVQ_ERR_INVALID_ARG
    assert L.kvq_qjl_encode(_p(A16), 10, 128, _p(A16), 256, _p(A16 + 4), _p(A16), None) == kvq.KVQ_ERR_INVALID_ARG
    assert L.kvq_qjl_encode(_p(A16), 0, 128, _p(A16), 256, None, None, None) == kvq.KVQ_OK
    assert L.kvq_qjl_query_sketch(_p(A16), 4, 128, _p(A16), 256, _p(A16 + 4), None) == kvq.KVQ_ERR_INVALID_ARG


def _args(kvq, **kw):
    a = kvq.DecodeArgs()
    a.batch, a.n_q_heads, a.n_kv_heads, a.seq_len, a.head_dim = 1, 8, 2, 100, 128
    a.key_format = kvq.KVQ_KEYS_INT8
    a.q_f16 = a.k_codes = a.k_scales = a.v_codes = a.v_scales = a.out = A16
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def test_decode_rejects_bad_arguments(kvq):
    L = kvq.lib
    call = lambda a: L.kvq_decode_attention(ctypes.byref(a), None)
    E, U = kvq.KVQ_ERR_INVALID_ARG, kvq.KVQ_ERR_UNSUPPORTED
    assert call(_args(kvq, n_kv_heads=3)) == E                 # Hq % Hkv
    assert call(_args(kvq, seq_len=0)) == E                    # softmax over nothing
    assert call(_args(kvq, head_dim=64)) == U
    assert call(_args(kvq, head_dim=100)) == E
    assert call(_args(kvq, out=None)) == E                     # nothing requested
    assert call(_args(kvq, key_format=5)) == E
    # any group size is served (here valid arguments without a workspace)
    for hq, hkv in ((6, 2), (16, 1), (32, 1), (24, 2)):
        assert call(_args(kvq, n_q_heads=hq, n_kv_heads=hkv)) == kvq.KVQ_ERR_WORKSPACE
        assert L.kvq_decode_workspace_bytes(ctypes.byref(_args(kvq, n_q_heads=hq, n_kv_heads=hkv))) > 0
    assert call(_args(kvq, k_codes=A16 + 1)) == E
    assert call(_args(kvq, q_f16=None)) == E
    assert call(_args(kvq, sm_scale=-1.0)) == E
    assert call(_args(kvq, flags=4)) == E                      # unknown flag bit
    assert call(_args(kvq, flags=kvq.KVQ_DECODE_CUDA_CORES)) == kvq.KVQ_ERR_WORKSPACE
    assert call(_args(kvq, flags=kvq.KVQ_DECODE_TEST_EXPIRE)) == kvq.KVQ_ERR_WORKSPACE
    qjl = dict(key_format=kvq.KVQ_KEYS_QJL, k_words=A16, k_norms_f16=A16, sketch_f16=A16)
    assert call(_args(kvq, sketch_dim=100, **qjl)) == E
    assert call(_args(kvq, sketch_dim=512, **qjl)) == U
    for hq in (16, 32, 6):                                              # QJL with G = 8, 16, 3
        assert call(_args(kvq, sketch_dim=256, n_q_heads=hq, **qjl)) == kvq.KVQ_ERR_WORKSPACE
    assert call(_args(kvq, sketch_dim=256, sketch_f16=A16 + 2,
                      **{k: v for k, v in qjl.items() if k != "sketch_f16"})) == E
    # valid arguments but no workspace
    assert call(_args(kvq)) == kvq.KVQ_ERR_WORKSPACE
    assert L.kvq_decode_workspace_bytes(ctypes.byref(_args(kvq))) > 0
    assert L.kvq_decode_workspace_bytes(ctypes.byref(_args(kvq, seq_len=0))) == 0
    # batch 0: nothing to do
    assert call(_args(kvq, batch=0)) == kvq.KVQ_OK


def test_product_path_has_no_cpu_fallback():
    """The binding loads only libkvq and never the oracle."""
    src = open(os.path.join(ROOT, "kv_cache_quantization_absmax_b200", "kvq.py")).read()
    assert "oracle" not in src.replace("never the oracle", "")
    for f in os.listdir(os.path.join(ROOT, "kv_cache_quantization_absmax_b200", "csrc")):
        assert "oracle" not in open(os.path.join(ROOT, "kv_cache_quantization_absmax_b200", "csrc", f)).read()


def test_lowbit_rejects_bad_arguments(kvq):
    L = kvq.lib
    E, U = kvq.KVQ_ERR_INVALID_ARG, kvq.KVQ_ERR_UNSUPPORTED
    assert L.kvq_quantize_int4(_p(A16), 1, 4, 128, 48, _p(A16), _p(A16), _p(A16), None) == E  # d % group
    assert L.kvq_quantize_int4(_p(A16), 1, 4, 128, 16, _p(A16), _p(A16), _p(A16), None) == U  # group size
    assert L.kvq_quantize_int4(_p(A16 + 8), 1, 4, 128, 32, _p(A16), _p(A16), _p(A16), None) == E
    assert L.kvq_quantize_int4(None, 1, 0, 128, 32, None, None, None, None) == kvq.KVQ_OK    # no rows
    assert L.kvq_dequantize_int4(_p(A16), _p(A16), _p(A16), 4, 128, 32, _p(A16 + 4), 0, None) == E
    assert L.kvq_quantize_int8_channelwise(_p(A16), 1, 2, 10, 96, _p(A16), _p(A16), None) == E  # d % 64
    assert L.kvq_quantize_int8_channelwise(_p(A16), 1, 2, 0, 128, _p(A16), _p(A16), None) == E  # rows
    assert L.kvq_quantize_int8_channelwise(_p(A16), 1, 0, 10, 128, _p(A16), _p(A16), None) == kvq.KVQ_OK
    assert L.kvq_dequantize_int8_channelwise(_p(A16), _p(A16 + 2), 2, 10, 128, _p(A16), 1, None) == E


def test_eviction_rejects_bad_arguments(kvq):
    L = kvq.lib
    E = kvq.KVQ_ERR_INVALID_ARG
    sel = L.kvq_evict_select
    assert sel(_p(A16), 2, 100, 5, 4, _p(A16), None) == E          # n_keep < n_sink
    assert sel(_p(A16), 2, 100, 0, 101, _p(A16), None) == E        # n_keep > seq_len
    assert sel(_p(A16), 2, 100, -1, 4, _p(A16), None) == E
    assert sel(_p(A16), 2, 1 << 31, 4, 8, _p(A16), None) == E      # seq_len >= 2^31
    assert sel(_p(A16 + 2), 2, 100, 4, 8, _p(A16), None) == E      # misaligned mass
    assert sel(None, 2, 100, 4, 8, _p(A16), None) == E
    assert sel(None, 0, 100, 4, 8, None, None) == kvq.KVQ_OK        # no rows
    assert sel(None, 2, 100, 0, 0, None, None) == kvq.KVQ_OK        # nothing kept
    g = L.kvq_gather_rows
    assert g(_p(A16), _p(A16), 2, 4, 100, 10, 0, _p(A16), 10, None) == E          # row_bytes
    assert g(_p(A16), _p(A16), 2, 4, 100, 9, 128, _p(A16), 10, None) == E         # dst_rows < n_keep
    assert g(_p(A16), _p(A16), 2, 4, 100, 1 << 25, 128, _p(A16), 1 << 24, None) == E  # too many bytes
    assert g(_p(A16), _p(A16), 2, 4, 100, 10, 128, _p(A16 + 1), 10, None) == E    # kept alignment
    assert g(None, _p(A16), 2, 4, 100, 10, 128, _p(A16), 10, None) == E
    assert g(None, None, 2, 4, 100, 10, 128, None, 0, None) == kvq.KVQ_OK         # nothing kept
    m = kvq.DecodeMassArgs()
    m.base = _args(kvq)
    assert L.kvq_decode_attention_mass(ctypes.byref(m), None) == E   # no attn_mass
    m.attn_mass = A16 + 2
    assert L.kvq_decode_attention_mass(ctypes.byref(m), None) == E   # misaligned
    m.attn_mass = A16
    m.base = _args(kvq, out=None, scores_out=A16)
    assert L.kvq_decode_attention_mass(ctypes.byref(m), None) == E   # no output
    m.base = _args(kvq)
    assert L.kvq_decode_attention_mass(ctypes.byref(m), None) == kvq.KVQ_ERR_WORKSPACE
    assert L.kvq_decode_mass_workspace_bytes(ctypes.byref(m)) > L.kvq_decode_workspace_bytes(ctypes.byref(m.base))


def test_qjlres_rejects_bad_arguments(kvq):
    L = kvq.lib
    E, U = kvq.KVQ_ERR_INVALID_ARG, kvq.KVQ_ERR_UNSUPPORTED
    enc = L.kvq_qjl_residual_encode
    ok = [_p(A16)] * 0
    args = lambda **kw: [kw.get("keys", _p(A16)), kw.get("n", 10), kw.get("d", 128), kw.get("g", 32),
                         kw.get("S", _p(A16)), kw.get("m", 256), kw.get("packed", _p(A16)), _p(A16), _p(A16),
                         kw.get("resid", _p(A16)), _p(A16), _p(A16), None]
    assert enc(*args(g=16)) == U
    assert enc(*args(g=48)) == E                     # d % group
    assert enc(*args(d=64, g=32)) == U               # d != 128
    assert enc(*args(m=100)) == E
    assert enc(*args(packed=_p(A16 + 4))) == E       # packed must be 16-byte aligned
    assert enc(*args(resid=_p(A16 + 2))) == E
    assert enc(*args(keys=None)) == E
    assert enc(*args(n=0, keys=None)) == kvq.KVQ_OK
    assert L.kvq_quantize_int4(_p(A16), 1, 4, 128, 32, _p(A16 + 4), _p(A16), _p(A16), None) == E
    r = kvq.DecodeQjlresArgs()
    r.base = _args(kvq, key_format=kvq.KVQ_KEYS_QJL, k_words=A16, k_norms_f16=A16, sketch_f16=A16, sketch_dim=256)
    r.k_packed4, r.k_scales4, r.k_zeros4, r.k_group = A16, A16, A16, 32
    call = lambda: L.kvq_decode_attention_qjlres(ctypes.byref(r), None)
    assert call() == kvq.KVQ_ERR_WORKSPACE
    assert L.kvq_decode_qjlres_workspace_bytes(ctypes.byref(r)) > 0
    r.k_group = 16
    assert call() == U
    r.k_group = 32
    r.k_packed4 = A16 + 8
    assert call() == E
    r.k_packed4 = A16
    r.base.sketch_dim = 64
    assert call() == U
    r.base.sketch_dim = 256
    r.base.key_format = kvq.KVQ_KEYS_INT8
    assert call() == E


def test_gather_multi_rejects_bad_arguments(kvq):
    L = kvq.lib
    E = kvq.KVQ_ERR_INVALID_ARG
    arr = (kvq.GatherArray * 9)()
    for i in range(9):
        arr[i] = kvq.GatherArray(A16, A16, 100, 10, 128)
    assert L.kvq_gather_rows_multi(arr, 9, 2, 4, _p(A16), 10, None) == E          # too many arrays
    assert L.kvq_gather_rows_multi(None, 2, 2, 4, _p(A16), 10, None) == E
    arr[1] = kvq.GatherArray(A16, A16, 100, 9, 128)                             # dst_rows < n_keep
    assert L.kvq_gather_rows_multi(arr, 2, 2, 4, _p(A16), 10, None) == E
    arr[1] = kvq.GatherArray(A16, A16, 100, 10, 0)                              # row_bytes
    assert L.kvq_gather_rows_multi(arr, 2, 2, 4, _p(A16), 10, None) == E
    arr[1] = kvq.GatherArray(A16, A16, 100, 10, 4)
    assert L.kvq_gather_rows_multi(arr, 2, 2, 4, _p(A16 + 2), 10, None) == E    # kept alignment
    assert L.kvq_gather_rows_multi(arr, 0, 2, 4, None, 10, None) == kvq.KVQ_OK
    assert L.kvq_gather_rows_multi(arr, 2, 2, 4, None, 0, None) == kvq.KVQ_OK


def test_decode_plan_takes_the_tensor_core_int8_kernel_from_512_tokens(kvq):
    """The INT8 decode's plan (host side, no GPU: the library then assumes 148 SMs): from
    512 tokens, with 16-byte aligned code arrays and an output, it runs the tensor-core
    kernel, one CTA per SM, so its partial states take less workspace than the CUDA-core
    plan's three CTAs per SM that KVQ_DECODE_CUDA_CORES selects; below 512 tokens, or
    without an output, both plans are the CUDA-core one."""
    ws = lambda **kw: kvq.lib.kvq_decode_workspace_bytes(ctypes.byref(_args(kvq, **kw)))
    cc = kvq.KVQ_DECODE_CUDA_CORES
    llama = dict(batch=8, n_q_heads=32, n_kv_heads=32, seq_len=4096)      # one 7B-shaped layer
    assert 0 < ws(**llama) < ws(flags=cc, **llama)
    assert ws(**llama) == ws(flags=kvq.KVQ_DECODE_TEST_EXPIRE, **llama)
    short = dict(batch=8, n_q_heads=32, n_kv_heads=32, seq_len=511)
    assert ws(**short) == ws(flags=cc, **short) > 0
    # scores only (no output): the CUDA-core kernel
    assert ws(out=None, scores_out=A16, **llama) == ws(out=None, scores_out=A16, flags=cc, **llama)
