"""The CPU oracle for the KV-cache compression path -- TEST INFRASTRUCTURE.

A plain, slow, obviously correct restatement of what the path computes (the C source
``kvq_oracle.c`` holds the arithmetic; this module only marshals numpy arrays through
ctypes).  Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import it.  It shares no code with the CUDA library.

Pinned by ``tests/test_oracle_pins.py`` against worked examples, invariants, closed forms
and brute force (see that file); no function here is "parity unpinned".
"""
import ctypes
import os

import numpy as np

from . import build as _build

F32, F16 = 0, 1
KEYS_INT8, KEYS_QJL, KEYS_QJLRES = 0, 1, 2

_libs = {}
_all_cores = False


def use_all_cores(on: bool = True) -> None:
    """Run the calls that follow on the all-cores build of the same C source (OpenMP over
    rows, keys or (batch, head) units; every result identical), or, with on=False, on the
    single-threaded build (the default)."""
    global _all_cores
    _all_cores = bool(on)


def threads() -> int:
    """Threads the current build runs its outer loops on (1 for the single-threaded one)."""
    return int(_load().ora_max_threads())


def _load():
    key = _all_cores
    if key not in _libs:
        path = _build.build(all_cores=key)
        lib = ctypes.CDLL(path)
        lib.ora_max_threads.restype = ctypes.c_int
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        I32 = ctypes.c_int
        lib.ora_half_to_double.argtypes = [ctypes.c_uint16]
        lib.ora_half_to_double.restype = ctypes.c_double
        lib.ora_double_to_half.argtypes = [ctypes.c_double]
        lib.ora_double_to_half.restype = ctypes.c_uint16
        lib.ora_quantize_int8.argtypes = [P, I32, I64, I64, P, P]
        lib.ora_dequantize_int8.argtypes = [P, P, I64, I64, P, I32]
        lib.ora_int8_scores.argtypes = [P, I32, P, P, I64, I64, P]
        lib.ora_qjl_encode.argtypes = [P, I64, I32, P, I32, P, P, P]
        lib.ora_qjl_query_sketch.argtypes = [P, I32, I64, I32, P, I32, P, P]
        lib.ora_qjl_estimate.argtypes = [P, P, ctypes.c_double, I32]
        lib.ora_qjl_estimate.restype = ctypes.c_double
        lib.ora_qjl_scores.argtypes = [P, I64, P, P, I64, I32, P]
        lib.ora_decode_attention.argtypes = [I64, I64, I64, I64, I32, P, I32, P, P, P, P, P,
                                             I32, P, P, P, I32, P, P, P, P, P, I32, ctypes.c_float,
                                             P, P, P]
        lib.ora_qjlres_encode.argtypes = [P, I64, I32, I32, P, I32, P, P, P, P, P, P, P]
        lib.ora_qjlres_encode.restype = I32
        lib.ora_quantize_int8_channelwise.argtypes = [P, I32, I64, I64, I64, P, P]
        lib.ora_dequantize_int8_channelwise.argtypes = [P, P, I64, I64, I64, P, I32]
        lib.ora_quantize_int4_group.argtypes = [P, I32, I64, I64, I32, P, P, P]
        lib.ora_dequantize_int4_group.argtypes = [P, P, P, I64, I64, I32, P, I32]
        for f in ("ora_quantize_int8_channelwise", "ora_dequantize_int8_channelwise",
                  "ora_quantize_int4_group", "ora_dequantize_int4_group"):
            getattr(lib, f).restype = I32
        for f in ("ora_quantize_int8", "ora_dequantize_int8", "ora_int8_scores",
                  "ora_qjl_encode", "ora_qjl_query_sketch", "ora_qjl_scores",
                  "ora_decode_attention"):
            getattr(lib, f).restype = ctypes.c_int
        _libs[key] = lib
    return _libs[key]


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _dtype_code(a):
    if a.dtype == np.float16:
        return F16
    if a.dtype == np.float32:
        return F32
    raise TypeError(f"unsupported dtype {a.dtype}")


def _check(rc, name):
    if rc != 0:
        raise ValueError(f"{name} returned {rc}")


def half_to_double(bits: int) -> float:
    return _load().ora_half_to_double(int(bits))


def double_to_half(x: float) -> int:
    return _load().ora_double_to_half(float(x))


def quantize_int8(x: np.ndarray):
    """Per-row absmax INT8: returns (codes int8 [n, d], scales fp32 [n])."""
    x = np.ascontiguousarray(x)
    n, d = x.shape
    codes = np.empty((n, d), np.int8)
    scales = np.empty((n,), np.float32)
    _check(_load().ora_quantize_int8(_ptr(x), _dtype_code(x), n, d, _ptr(codes), _ptr(scales)),
           "ora_quantize_int8")
    return codes, scales


def dequantize_int8(codes: np.ndarray, scales: np.ndarray, out_dtype=np.float32):
    codes = np.ascontiguousarray(codes, np.int8)
    scales = np.ascontiguousarray(scales, np.float32)
    n, d = codes.shape
    out = np.empty((n, d), out_dtype)
    _check(_load().ora_dequantize_int8(_ptr(codes), _ptr(scales), n, d, _ptr(out),
                                       _dtype_code(out)), "ora_dequantize_int8")
    return out


def int8_scores(q: np.ndarray, codes: np.ndarray, scales: np.ndarray):
    q = np.ascontiguousarray(q)
    codes = np.ascontiguousarray(codes, np.int8)
    scales = np.ascontiguousarray(scales, np.float32)
    n, d = codes.shape
    assert q.shape == (d,)
    out = np.empty((n,), np.float32)
    _check(_load().ora_int8_scores(_ptr(q), _dtype_code(q), _ptr(codes), _ptr(scales), n, d,
                                   _ptr(out)), "ora_int8_scores")
    return out


def qjl_encode(keys_f16: np.ndarray, S: np.ndarray, want_u: bool = False):
    """Sign sketch of fp16 keys [n, d] with sketch matrix S [m, d] (any float dtype, used
    in fp64).  Returns (words uint32 [n, m/32], norms fp16 [n][, u fp64 [n, m]])."""
    keys = np.ascontiguousarray(keys_f16, np.float16)
    S64 = np.ascontiguousarray(S, np.float64)
    n, d = keys.shape
    m = S64.shape[0]
    assert S64.shape[1] == d
    words = np.empty((n, m // 32), np.uint32)
    norms = np.empty((n,), np.float16)
    u = np.empty((n, m), np.float64) if want_u else None
    _check(_load().ora_qjl_encode(_ptr(keys), n, d, _ptr(S64), m, _ptr(words), _ptr(norms),
                                  _ptr(u)), "ora_qjl_encode")
    return (words, norms, u) if want_u else (words, norms)


def qjl_query_sketch(q: np.ndarray, S: np.ndarray):
    """v = S q for each row of q [n, d]; returns (v64 [n, m], v32 [n, m])."""
    q = np.ascontiguousarray(q)
    S64 = np.ascontiguousarray(S, np.float64)
    n, d = q.shape
    m = S64.shape[0]
    v64 = np.empty((n, m), np.float64)
    v32 = np.empty((n, m), np.float32)
    _check(_load().ora_qjl_query_sketch(_ptr(q), _dtype_code(q), n, d, _ptr(S64), m, _ptr(v64),
                                        _ptr(v32)), "ora_qjl_query_sketch")
    return v64, v32


def qjl_estimate(v: np.ndarray, key_words: np.ndarray, key_norm: float) -> float:
    v = np.ascontiguousarray(v, np.float64)
    w = np.ascontiguousarray(key_words, np.uint32)
    return _load().ora_qjl_estimate(_ptr(v), _ptr(w), float(key_norm), v.shape[0])


def qjl_scores(v: np.ndarray, words: np.ndarray, norms_f16: np.ndarray):
    v = np.ascontiguousarray(np.atleast_2d(v), np.float64)
    words = np.ascontiguousarray(words, np.uint32)
    norms = np.ascontiguousarray(norms_f16, np.float16)
    nq, m = v.shape
    nk = words.shape[0]
    out = np.empty((nq, nk), np.float32)
    _check(_load().ora_qjl_scores(_ptr(v), nq, _ptr(words), _ptr(norms), nk, m, _ptr(out)),
           "ora_qjl_scores")
    return out


def qjl_residual_encode(keys_f16: np.ndarray, group: int, S: np.ndarray, want_r: bool = False,
                        want_u: bool = False):
    """QJL as the 1-bit residual of group-wise INT4 (the "TurboQuant" news page: a first
    quantizer, then a 1-bit QJL correction of its residual error).  keys fp16 [n, d];
    returns a dict: packed uint8 [n, d/2], scales, zeros fp32 [n, d/group] (the INT4
    stage, as quantize_int4_group), words uint32 [n, m/32] and rnorms fp16 [n] (the QJL
    sketch of r = fp16(fl32(k - k_hat)), k_hat the INT4 reconstruction), and optionally
    r fp16 [n, d] and u fp64 [n, m] = S r."""
    keys = np.ascontiguousarray(keys_f16, np.float16)
    S64 = np.ascontiguousarray(S, np.float64)
    n, d = keys.shape
    m = S64.shape[0]
    assert S64.shape[1] == d
    out = dict(packed=np.zeros((n, d // 2), np.uint8), scales=np.empty((n, d // group), np.float32),
               zeros=np.empty((n, d // group), np.float32), words=np.empty((n, m // 32), np.uint32),
               rnorms=np.empty((n,), np.float16))
    r = np.empty((n, d), np.float16) if want_r else None
    u = np.empty((n, m), np.float64) if want_u else None
    _check(_load().ora_qjlres_encode(_ptr(keys), n, d, group, _ptr(S64), m, _ptr(out["packed"]),
                                     _ptr(out["scales"]), _ptr(out["zeros"]), _ptr(out["words"]),
                                     _ptr(out["rnorms"]), _ptr(r), _ptr(u)), "ora_qjlres_encode")
    if want_r:
        out["r"] = r
    if want_u:
        out["u"] = u
    return out


def decode_attention(q_f16, *, k_codes=None, k_scales=None, k_words=None, k_norms=None,
                     S=None, k4=None, v_codes=None, v_scales=None, v4=None, sm_scale=0.0,
                     want_out=True, want_scores=False, want_probs=False):
    """One decode step.  q [B, Hq, D] fp16; INT8 keys [B, Hkv, T, D] + [B, Hkv, T] or
    QJL keys words [B, Hkv, T, m/32] + norms [B, Hkv, T] + S [m, D], or residual keys:
    k4 = (packed [B, Hkv, T, D/2], scales, zeros [B, Hkv, T, D/g], g) with the residual's
    words and norms in k_words / k_norms; INT8 values, or group-wise INT4 values
    v4 = (packed [B, Hkv, T, D/2], scales, zeros [B, Hkv, T, D/g], g).
    Returns a dict with 'out' [B, Hq, D], 'scores' / 'probs' [B, Hq, T] as requested."""
    q = np.ascontiguousarray(q_f16, np.float16)
    B, Hq, D = q.shape
    qjl = k_words is not None
    k4p = k4s = k4z = None
    k4g = 0
    if k4 is not None:
        k4p = np.ascontiguousarray(k4[0], np.uint8)
        k4s = np.ascontiguousarray(k4[1], np.float32)
        k4z = np.ascontiguousarray(k4[2], np.float32)
        k4g = int(k4[3])
    if qjl:
        k_words = np.ascontiguousarray(k_words, np.uint32)
        k_norms = np.ascontiguousarray(k_norms, np.float16)
        Hkv, T = k_words.shape[1], k_words.shape[2]
        S64 = np.ascontiguousarray(S, np.float64)
        m = S64.shape[0]
    else:
        k_codes = np.ascontiguousarray(k_codes, np.int8)
        k_scales = np.ascontiguousarray(k_scales, np.float32)
        Hkv, T = k_codes.shape[1], k_codes.shape[2]
        S64, m = None, 0
    v4p = v4s = v4z = None
    v4g = 0
    if want_out and v4 is not None:
        v4p = np.ascontiguousarray(v4[0], np.uint8)
        v4s = np.ascontiguousarray(v4[1], np.float32)
        v4z = np.ascontiguousarray(v4[2], np.float32)
        v4g = int(v4[3])
    elif want_out:
        v_codes = np.ascontiguousarray(v_codes, np.int8)
        v_scales = np.ascontiguousarray(v_scales, np.float32)
    out = np.empty((B, Hq, D), np.float32) if want_out else None
    scores = np.empty((B, Hq, T), np.float32) if want_scores else None
    probs = np.empty((B, Hq, T), np.float32) if want_probs else None
    rc = _load().ora_decode_attention(
        B, Hq, Hkv, T, D, _ptr(q), (KEYS_QJLRES if k4 is not None else KEYS_QJL) if qjl else KEYS_INT8,
        _ptr(k_codes) if not qjl else None, _ptr(k_scales) if not qjl else None,
        _ptr(k_words) if qjl else None, _ptr(k_norms) if qjl else None, _ptr(S64), m,
        _ptr(k4p), _ptr(k4s), _ptr(k4z), k4g,
        _ptr(v_codes) if (want_out and v4 is None) else None,
        _ptr(v_scales) if (want_out and v4 is None) else None,
        _ptr(v4p), _ptr(v4s), _ptr(v4z), v4g,
        float(sm_scale), _ptr(out), _ptr(scores), _ptr(probs))
    _check(rc, "ora_decode_attention")
    return {"out": out, "scores": scores, "probs": probs}


def decode_from_scores(scores, values, sm_scale=0.0):
    """The decode step after its scores, in fp64 ("QJL" abstract and "GPU-Accelerated INT8
    Quantization ..." abstract: attention over the compressed cache; "Q-TensorFormer" model
    card, section 4: query head h reads KV head h // G).  For each (b, h):
        p_t = exp(sigma s_t - max_t sigma s_t) / sum_t exp(...),   out = sum_t p_t v_t,
    sigma = sm_scale, or the fp32 value of 1/sqrt(D) when 0 (as decode_attention).
    scores [B, Hq, T] (any float dtype, used in fp64); values [B, Hkv, T, D] (the
    dequantized value rows, used in fp64).  Returns (out fp64 [B, Hq, D], p fp64
    [B, Hq, T])."""
    s = np.asarray(scores, np.float64)
    v = np.asarray(values, np.float64)
    B, Hq, T = s.shape
    Hkv, D = v.shape[1], v.shape[3]
    assert v.shape == (B, Hkv, T, D) and Hq % Hkv == 0
    G = Hq // Hkv
    # the fp32 value of 1/sqrt(D) that decode_attention uses
    sigma = float(sm_scale) if sm_scale != 0.0 else float(np.float32(1.0) / np.sqrt(np.float32(D)))
    lg = sigma * s
    e = np.exp(lg - lg.max(axis=-1, keepdims=True))
    p = e / e.sum(axis=-1, keepdims=True)
    out = np.empty((B, Hq, D), np.float64)
    for b in range(B):
        for h in range(Hq):
            out[b, h] = p[b, h] @ v[b, h // G]
    return out, p


def decode_append(q_f16, k_new_f16, v_new_f16, *, T, k_codes=None, k_scales=None, k_words=None,
                  k_norms=None, S=None, v_codes=None, v_scales=None, sm_scale=0.0,
                  want_out=True, want_scores=False):
    """Append-on-decode ("Quantum-Inspired GPU & J-Space VRAM Optimizer" page, section 4:
    the cache writes are intercepted and the compressed representation stored): the new
    token's key row [B, Hkv, D] is quantized (INT8 keys: quantize_int8) or sign-sketched
    (QJL keys: qjl_encode) and its value row INT8-quantized, both stored at token T of
    copies of the cache arrays ([B, Hkv, capacity, ...], capacity >= T + 1); then one
    decode step over the T + 1 tokens.  Returns a dict with the decode outputs and the
    updated cache copies."""
    kn = np.ascontiguousarray(k_new_f16, np.float16)
    B, Hkv, D = kn.shape
    qjl = k_words is not None
    res = {}
    if qjl:
        w, n = qjl_encode(kn.reshape(-1, D), S)
        kw = np.array(k_words, np.uint32, copy=True)
        kno = np.array(k_norms, np.float16, copy=True)
        kw[:, :, T] = w.reshape(B, Hkv, -1)
        kno[:, :, T] = n.reshape(B, Hkv)
        res.update(k_words=kw, k_norms=kno)
        keys = dict(k_words=kw[:, :, :T + 1], k_norms=kno[:, :, :T + 1], S=S)
    else:
        c, s = quantize_int8(kn.reshape(-1, D))
        kc = np.array(k_codes, np.int8, copy=True)
        ks = np.array(k_scales, np.float32, copy=True)
        kc[:, :, T] = c.reshape(B, Hkv, D)
        ks[:, :, T] = s.reshape(B, Hkv)
        res.update(k_codes=kc, k_scales=ks)
        keys = dict(k_codes=kc[:, :, :T + 1], k_scales=ks[:, :, :T + 1])
    vals = {}
    if want_out:
        c, s = quantize_int8(np.ascontiguousarray(v_new_f16, np.float16).reshape(-1, D))
        vc = np.array(v_codes, np.int8, copy=True)
        vs = np.array(v_scales, np.float32, copy=True)
        vc[:, :, T] = c.reshape(B, Hkv, D)
        vs[:, :, T] = s.reshape(B, Hkv)
        res.update(v_codes=vc, v_scales=vs)
        vals = dict(v_codes=vc[:, :, :T + 1], v_scales=vs[:, :, :T + 1])
    res.update(decode_attention(q_f16, sm_scale=sm_scale, want_out=want_out,
                                want_scores=want_scores, **keys, **vals))
    return res


def quantize_int8_channelwise(x: np.ndarray):
    """Channel-wise INT8 of blocks x [n_blocks, rows, d]: returns (codes int8 like x,
    scales fp32 [n_blocks, d]), one scale per column of each block."""
    x = np.ascontiguousarray(x)
    nb, rows, d = x.shape
    codes = np.empty(x.shape, np.int8)
    scales = np.empty((nb, d), np.float32)
    _check(_load().ora_quantize_int8_channelwise(_ptr(x), _dtype_code(x), nb, rows, d, _ptr(codes),
                                                 _ptr(scales)), "ora_quantize_int8_channelwise")
    return codes, scales


def dequantize_int8_channelwise(codes: np.ndarray, scales: np.ndarray, out_dtype=np.float32):
    codes = np.ascontiguousarray(codes, np.int8)
    scales = np.ascontiguousarray(scales, np.float32)
    nb, rows, d = codes.shape
    out = np.empty(codes.shape, out_dtype)
    _check(_load().ora_dequantize_int8_channelwise(_ptr(codes), _ptr(scales), nb, rows, d, _ptr(out),
                                                   F16 if out_dtype == np.float16 else F32),
           "ora_dequantize_int8_channelwise")
    return out


def quantize_int4_group(x: np.ndarray, g: int):
    """Group-wise asymmetric INT4 of rows x [n, d] (fp16 or fp32), groups of g: returns
    (packed uint8 [n, d/2], scales fp32 [n, d/g], zeros fp32 [n, d/g])."""
    x = np.ascontiguousarray(x)
    n, d = x.shape
    packed = np.zeros((n, d // 2), np.uint8)
    scales = np.empty((n, d // g), np.float32)
    zeros = np.empty((n, d // g), np.float32)
    _check(_load().ora_quantize_int4_group(_ptr(x), _dtype_code(x), n, d, g, _ptr(packed), _ptr(scales),
                                           _ptr(zeros)), "ora_quantize_int4_group")
    return packed, scales, zeros


def dequantize_int4_group(packed, scales, zeros, g: int, out_dtype=np.float32):
    packed = np.ascontiguousarray(packed, np.uint8)
    scales = np.ascontiguousarray(scales, np.float32)
    zeros = np.ascontiguousarray(zeros, np.float32)
    n, half = packed.shape
    d = 2 * half
    out = np.empty((n, d), out_dtype)
    _check(_load().ora_dequantize_int4_group(_ptr(packed), _ptr(scales), _ptr(zeros), n, d, g, _ptr(out),
                                             F16 if out_dtype == np.float16 else F32),
           "ora_dequantize_int4_group")
    return out


def attention_mass(q_f16, **decode_kwargs):
    """Attention mass of one decode step ("Q-TensorFormer" model card, section 6,
    Attention-Sink Dynamic Eviction: sum over heads h of alpha_{h,j}): the oracle's
    softmax probabilities [B, Hq, T] summed over the query heads -> [B, T] (fp64 sum of
    the fp32 probabilities)."""
    r = decode_attention(q_f16, want_out=False, want_probs=True, **decode_kwargs)
    return r["probs"].astype(np.float64).sum(axis=1)


def evict_select(mass, n_sink: int, n_keep: int):
    """Tokens retained per batch row of mass [B, T] (same section): the first n_sink
    tokens, plus the n_keep - n_sink tokens of largest mass among the others (equal
    masses: the smaller token index first); returned in token order, int32 [B, n_keep]."""
    mass = np.asarray(mass)
    B, T = mass.shape
    assert 0 <= n_sink <= n_keep <= T
    out = np.empty((B, n_keep), np.int32)
    for b in range(B):
        rest = np.arange(n_sink, T)
        # primary key: larger mass first; secondary: smaller index first
        order = rest[np.lexsort((rest, -mass[b, n_sink:]))]
        kept = np.concatenate([np.arange(n_sink), order[: n_keep - n_sink]])
        out[b] = np.sort(kept)
    return out


def gather_rows(cache, kept):
    """Compaction of a cache [B, H, T, ...] to the kept tokens [B, n_keep] (in order):
    out[b, h, j] = cache[b, h, kept[b, j]]."""
    cache = np.asarray(cache)
    B = cache.shape[0]
    return np.stack([cache[b][:, kept[b]] for b in range(B)])
