"""Thin Python binding over libkvq (include/kvq.h): argument marshalling only.

Every function has the name of the C entry point it calls, takes torch CUDA tensors,
allocates its outputs with torch (device memory is torch's job; the library allocates
nothing) and enqueues the work on the current torch stream.  All arithmetic happens in
the library's CUDA kernels.  There is no fallback: if the library cannot be built or
loaded, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import build as _build

KVQ_OK, KVQ_ERR_INVALID_ARG, KVQ_ERR_UNSUPPORTED, KVQ_ERR_CUDA, KVQ_ERR_WORKSPACE, KVQ_ERR_DEVICE = range(6)
KVQ_F32, KVQ_F16 = 0, 1
KVQ_KEYS_INT8, KVQ_KEYS_QJL = 0, 1
KVQ_DECODE_CUDA_CORES = 1
KVQ_DECODE_TEST_EXPIRE = 2
ABI_VERSION = 2

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I32 = ctypes.c_int32


class DecodeArgs(ctypes.Structure):
    """Mirror of ``kvq_decode_args``."""
    _fields_ = [
        ("batch", _I64), ("n_q_heads", _I64), ("n_kv_heads", _I64), ("seq_len", _I64),
        ("head_dim", _I32), ("key_format", _I32),
        ("q_f16", _P), ("k_codes", _P), ("k_scales", _P), ("k_words", _P), ("k_norms_f16", _P),
        ("sketch_f16", _P), ("sketch_dim", _I32), ("sm_scale", ctypes.c_float),
        ("v_codes", _P), ("v_scales", _P), ("out", _P), ("scores_out", _P),
        ("workspace", _P), ("workspace_bytes", ctypes.c_size_t), ("flags", ctypes.c_uint32),
    ]


class DecodeAppendArgs(ctypes.Structure):
    """Mirror of ``kvq_decode_append_args``."""
    _fields_ = [("base", DecodeArgs), ("capacity", _I64), ("k_new_f16", _P), ("v_new_f16", _P)]


class DecodeInt4vArgs(ctypes.Structure):
    """Mirror of ``kvq_decode_int4v_args``."""
    _fields_ = [("base", DecodeArgs), ("v_packed", _P), ("v_scales4", _P), ("v_zeros4", _P),
                ("v_group", _I32)]


class GatherArray(ctypes.Structure):
    """Mirror of ``kvq_gather_array``."""
    _fields_ = [("src", _P), ("dst", _P), ("src_rows", _I64), ("dst_rows", _I64), ("row_bytes", _I64)]


class DecodeQjlresArgs(ctypes.Structure):
    """Mirror of ``kvq_decode_qjlres_args``."""
    _fields_ = [("base", DecodeArgs), ("k_packed4", _P), ("k_scales4", _P), ("k_zeros4", _P),
                ("k_group", _I32)]


class DecodeMassArgs(ctypes.Structure):
    """Mirror of ``kvq_decode_mass_args``."""
    _fields_ = [("base", DecodeArgs), ("attn_mass", _P)]


class KvqError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn} failed: {lib.kvq_status_string(status).decode()} (status {status})")


def _load():
    path = _build.build()
    so = ctypes.CDLL(path)
    so.kvq_abi_version.restype = ctypes.c_int
    so.kvq_status_string.argtypes = [ctypes.c_int]
    so.kvq_status_string.restype = ctypes.c_char_p
    so.kvq_quantize_int8.argtypes = [_P, ctypes.c_int, _I64, _I64, _P, _P, _P]
    so.kvq_dequantize_int8.argtypes = [_P, _P, _I64, _I64, _P, ctypes.c_int, _P]
    so.kvq_int8_scores.argtypes = [_P, ctypes.c_int, _P, _P, _I64, _I64, _P, _P]
    so.kvq_qjl_encode.argtypes = [_P, _I64, _I32, _P, _I32, _P, _P, _P]
    so.kvq_qjl_query_sketch.argtypes = [_P, _I64, _I32, _P, _I32, _P, _P]
    so.kvq_decode_attention.argtypes = [ctypes.POINTER(DecodeArgs), _P]
    so.kvq_decode_workspace_bytes.argtypes = [ctypes.POINTER(DecodeArgs)]
    so.kvq_decode_workspace_bytes.restype = ctypes.c_size_t
    so.kvq_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint32)]
    so.kvq_decode_attention_noalloc.argtypes = [ctypes.POINTER(DecodeArgs), _P]
    so.kvq_decode_attention_noalloc.restype = ctypes.c_int
    so.kvq_decode_noalloc_max_workspace_bytes.argtypes = []
    so.kvq_decode_noalloc_max_workspace_bytes.restype = ctypes.c_size_t
    so.kvq_quantize_int8_channelwise.argtypes = [_P, ctypes.c_int, _I64, _I64, _I64, _P, _P, _P]
    so.kvq_dequantize_int8_channelwise.argtypes = [_P, _P, _I64, _I64, _I64, _P, ctypes.c_int, _P]
    so.kvq_quantize_int4.argtypes = [_P, ctypes.c_int, _I64, _I64, _I32, _P, _P, _P, _P]
    so.kvq_dequantize_int4.argtypes = [_P, _P, _P, _I64, _I64, _I32, _P, ctypes.c_int, _P]
    for f in ("kvq_quantize_int8_channelwise", "kvq_dequantize_int8_channelwise", "kvq_quantize_int4",
              "kvq_dequantize_int4"):
        getattr(so, f).restype = ctypes.c_int
    so.kvq_decode_attention_int4v.argtypes = [ctypes.POINTER(DecodeInt4vArgs), _P]
    so.kvq_decode_attention_int4v.restype = ctypes.c_int
    so.kvq_decode_int4v_workspace_bytes.argtypes = [ctypes.POINTER(DecodeInt4vArgs)]
    so.kvq_decode_int4v_workspace_bytes.restype = ctypes.c_size_t
    so.kvq_decode_append.argtypes = [ctypes.POINTER(DecodeAppendArgs), _P]
    so.kvq_decode_append.restype = ctypes.c_int
    so.kvq_decode_append_workspace_bytes.argtypes = [ctypes.POINTER(DecodeAppendArgs)]
    so.kvq_decode_append_workspace_bytes.restype = ctypes.c_size_t
    so.kvq_decode_attention_mass.argtypes = [ctypes.POINTER(DecodeMassArgs), _P]
    so.kvq_decode_attention_mass.restype = ctypes.c_int
    so.kvq_decode_mass_workspace_bytes.argtypes = [ctypes.POINTER(DecodeMassArgs)]
    so.kvq_decode_mass_workspace_bytes.restype = ctypes.c_size_t
    so.kvq_evict_select.argtypes = [_P, _I64, _I64, _I64, _I64, _P, _P]
    so.kvq_evict_select.restype = ctypes.c_int
    so.kvq_gather_rows.argtypes = [_P, _P, _I64, _I64, _I64, _I64, _I64, _P, _I64, _P]
    so.kvq_gather_rows.restype = ctypes.c_int
    so.kvq_gather_rows_multi.argtypes = [ctypes.POINTER(GatherArray), _I32, _I64, _I64, _P, _I64, _P]
    so.kvq_gather_rows_multi.restype = ctypes.c_int
    so.kvq_decode_attention_qjlres.argtypes = [ctypes.POINTER(DecodeQjlresArgs), _P]
    so.kvq_decode_attention_qjlres.restype = ctypes.c_int
    so.kvq_decode_qjlres_workspace_bytes.argtypes = [ctypes.POINTER(DecodeQjlresArgs)]
    so.kvq_decode_qjlres_workspace_bytes.restype = ctypes.c_size_t
    so.kvq_qjl_residual_encode.argtypes = [_P, _I64, _I32, _I32, _P, _I32, _P, _P, _P, _P, _P, _P, _P]
    so.kvq_qjl_residual_encode.restype = ctypes.c_int
    for f in ("kvq_quantize_int8", "kvq_dequantize_int8", "kvq_int8_scores", "kvq_qjl_encode",
              "kvq_qjl_query_sketch", "kvq_decode_attention", "kvq_device_error"):
        getattr(so, f).restype = ctypes.c_int
    if so.kvq_abi_version() != ABI_VERSION:
        raise RuntimeError(f"libkvq ABI version {so.kvq_abi_version()} != {ABI_VERSION}")
    return so


lib = _load()
LIBRARY_PATH = os.path.abspath(_build.LIB)


def _check(fn, status):
    if status != KVQ_OK:
        raise KvqError(fn, status)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    """The stream to enqueue on: torch's current stream, or the one given.  A given stream
    first waits for the current one, where the inputs were made and the outputs
    allocated (torch may hand an output a block that work on the current stream still
    touches)."""
    cur = torch.cuda.current_stream()
    if stream is None:
        return ctypes.c_void_p(cur.cuda_stream)
    if stream.cuda_stream != cur.cuda_stream:
        stream.wait_stream(cur)
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t):
    if t.dtype == torch.float16:
        return KVQ_F16
    if t.dtype == torch.float32:
        return KVQ_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _need_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("inputs must be contiguous CUDA tensors")


def _u16(t):
    return t.view(torch.int16) if t.dtype == torch.float16 else t


# --------------------------------------------------------------------------------------

def kvq_quantize_int8(x, codes=None, scales=None, stream=None):
    """Per-row absmax INT8 of x [..., D] (fp16/fp32): returns (codes int8 [..., D],
    scales fp32 [...])."""
    _need_cuda(x)
    d = x.shape[-1]
    n = x.numel() // d if d else 0
    if codes is None:
        codes = torch.empty(x.shape, dtype=torch.int8, device=x.device)
    if scales is None:
        scales = torch.empty(x.shape[:-1], dtype=torch.float32, device=x.device)
    _check("kvq_quantize_int8", lib.kvq_quantize_int8(_ptr(x), _dtype_code(x), n, d, _ptr(codes),
                                                      _ptr(scales), _stream(stream)))
    return codes, scales


def kvq_dequantize_int8(codes, scales, out_dtype=torch.float32, out=None, stream=None):
    _need_cuda(codes, scales)
    d = codes.shape[-1]
    n = codes.numel() // d if d else 0
    if out is None:
        out = torch.empty(codes.shape, dtype=out_dtype, device=codes.device)
    _check("kvq_dequantize_int8", lib.kvq_dequantize_int8(_ptr(codes), _ptr(scales), n, d, _ptr(out),
                                                          _dtype_code(out), _stream(stream)))
    return out


def kvq_int8_scores(q, codes, scales, out=None, stream=None):
    """scores_r = sum_j q_j * x_hat_rj for one query q [D] against rows [..., D]."""
    _need_cuda(q, codes, scales)
    d = codes.shape[-1]
    n = codes.numel() // d if d else 0
    if out is None:
        out = torch.empty(codes.shape[:-1], dtype=torch.float32, device=codes.device)
    _check("kvq_int8_scores", lib.kvq_int8_scores(_ptr(q), _dtype_code(q), _ptr(codes), _ptr(scales),
                                                  n, d, _ptr(out), _stream(stream)))
    return out


def kvq_qjl_encode(keys, sketch, words=None, norms=None, stream=None):
    """QJL sign sketch of fp16 keys [..., 128] with fp16 S [m, 128]: returns
    (words uint32-as-int32 [..., m/32], norms fp16 [...])."""
    _need_cuda(keys, sketch)
    d = keys.shape[-1]
    n = keys.numel() // d if d else 0
    m = sketch.shape[0]
    if words is None:
        words = torch.empty(keys.shape[:-1] + (m // 32,), dtype=torch.int32, device=keys.device)
    if norms is None:
        norms = torch.empty(keys.shape[:-1], dtype=torch.float16, device=keys.device)
    _check("kvq_qjl_encode", lib.kvq_qjl_encode(_ptr(keys), n, d, _ptr(sketch), m, _ptr(words),
                                                _ptr(norms), _stream(stream)))
    return words, norms


def kvq_qjl_query_sketch(q, sketch, out=None, stream=None):
    _need_cuda(q, sketch)
    d = q.shape[-1]
    n = q.numel() // d if d else 0
    m = sketch.shape[0]
    if out is None:
        out = torch.empty(q.shape[:-1] + (m,), dtype=torch.float32, device=q.device)
    _check("kvq_qjl_query_sketch", lib.kvq_qjl_query_sketch(_ptr(q), n, d, _ptr(sketch), m,
                                                            _ptr(out), _stream(stream)))
    return out


def make_decode_args(q, *, k_codes=None, k_scales=None, k_words=None, k_norms=None, sketch=None,
                     v_codes=None, v_scales=None, out=None, scores_out=None, sm_scale=0.0,
                     workspace=None, flags=0):
    """Fill a ``kvq_decode_args`` from tensors (q [B, Hq, D] fp16; cache [B, Hkv, T, ...])."""
    B, Hq, D = q.shape
    a = DecodeArgs()
    a.batch, a.n_q_heads, a.head_dim = B, Hq, D
    qjl = k_words is not None
    ref = k_words if qjl else k_codes
    a.n_kv_heads, a.seq_len = ref.shape[1], ref.shape[2]
    a.key_format = KVQ_KEYS_QJL if qjl else KVQ_KEYS_INT8
    a.q_f16 = q.data_ptr()
    if qjl:
        a.k_words, a.k_norms_f16, a.sketch_f16 = k_words.data_ptr(), k_norms.data_ptr(), sketch.data_ptr()
        a.sketch_dim = sketch.shape[0]
    else:
        a.k_codes, a.k_scales = k_codes.data_ptr(), k_scales.data_ptr()
    if v_codes is not None:
        a.v_codes, a.v_scales = v_codes.data_ptr(), v_scales.data_ptr()
    a.out = out.data_ptr() if out is not None else None
    a.scores_out = scores_out.data_ptr() if scores_out is not None else None
    a.sm_scale = float(sm_scale)
    a.flags = int(flags)
    if workspace is not None:
        a.workspace, a.workspace_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    return a


def kvq_decode_workspace_bytes(args: DecodeArgs) -> int:
    return int(lib.kvq_decode_workspace_bytes(ctypes.byref(args)))


def kvq_decode_attention(q, *, k_codes=None, k_scales=None, k_words=None, k_norms=None, sketch=None,
                         v_codes=None, v_scales=None, want_out=True, want_scores=False,
                         sm_scale=0.0, workspace=None, out=None, scores_out=None, stream=None, flags=0):
    """One decode step; returns (out [B, Hq, D] fp32 or None, scores [B, Hq, T] or None).
    flags: KVQ_DECODE_CUDA_CORES keeps the scores and the weighted value sum on the CUDA
    cores (no tensor-core kernel)."""
    _need_cuda(q, k_codes, k_scales, k_words, k_norms, sketch, v_codes, v_scales)
    B, Hq, D = q.shape
    ref = k_words if k_words is not None else k_codes
    T = ref.shape[2]
    if want_out and out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float32, device=q.device)
    if want_scores and scores_out is None:
        scores_out = torch.empty((B, Hq, T), dtype=torch.float32, device=q.device)
    a = make_decode_args(q, k_codes=k_codes, k_scales=k_scales, k_words=k_words, k_norms=k_norms,
                         sketch=sketch, v_codes=v_codes if want_out else None,
                         v_scales=v_scales if want_out else None, out=out if want_out else None,
                         scores_out=scores_out if want_scores else None, sm_scale=sm_scale, flags=flags)
    need = kvq_decode_workspace_bytes(a)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    a.workspace, a.workspace_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    _check("kvq_decode_attention", lib.kvq_decode_attention(ctypes.byref(a), _stream(stream)))
    return (out if want_out else None), (scores_out if want_scores else None)


def kvq_decode_attention_noalloc(q, *, k_codes=None, k_scales=None, k_words=None, k_norms=None,
                                 sketch=None, v_codes=None, v_scales=None, want_out=True,
                                 want_scores=False, sm_scale=0.0, out=None, scores_out=None,
                                 stream=None):
    """The decode step using the library's built-in scratch instead of a workspace
    (for callers that cannot allocate device memory); see include/kvq.h."""
    _need_cuda(q, k_codes, k_scales, k_words, k_norms, sketch, v_codes, v_scales)
    B, Hq, D = q.shape
    ref = k_words if k_words is not None else k_codes
    T = ref.shape[2]
    if want_out and out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float32, device=q.device)
    if want_scores and scores_out is None:
        scores_out = torch.empty((B, Hq, T), dtype=torch.float32, device=q.device)
    a = make_decode_args(q, k_codes=k_codes, k_scales=k_scales, k_words=k_words, k_norms=k_norms,
                         sketch=sketch, v_codes=v_codes if want_out else None,
                         v_scales=v_scales if want_out else None, out=out if want_out else None,
                         scores_out=scores_out if want_scores else None, sm_scale=sm_scale)
    _check("kvq_decode_attention_noalloc", lib.kvq_decode_attention_noalloc(ctypes.byref(a), _stream(stream)))
    return (out if want_out else None), (scores_out if want_scores else None)


def kvq_device_error() -> int:
    code = ctypes.c_uint32(0)
    _check("kvq_device_error", lib.kvq_device_error(ctypes.byref(code)))
    return int(code.value)


def make_decode_append_args(q, k_new, v_new, *, T, k_codes=None, k_scales=None, k_words=None,
                            k_norms=None, sketch=None, v_codes=None, v_scales=None, out=None,
                            scores_out=None, sm_scale=0.0, workspace=None):
    """Fill a ``kvq_decode_append_args``: cache tensors [B, Hkv, capacity, ...] holding T
    tokens; k_new / v_new [B, Hkv, D] fp16."""
    a = DecodeAppendArgs()
    a.base = make_decode_args(q, k_codes=k_codes, k_scales=k_scales, k_words=k_words,
                              k_norms=k_norms, sketch=sketch, v_codes=v_codes, v_scales=v_scales,
                              out=out, scores_out=scores_out, sm_scale=sm_scale, workspace=workspace)
    ref = k_words if k_words is not None else k_codes
    a.capacity = ref.shape[2]
    a.base.seq_len = T
    a.k_new_f16 = k_new.data_ptr()
    a.v_new_f16 = v_new.data_ptr() if v_new is not None else None
    return a


def kvq_decode_append(q, k_new, v_new, *, T, k_codes=None, k_scales=None, k_words=None,
                      k_norms=None, sketch=None, v_codes=None, v_scales=None, want_out=True,
                      want_scores=False, sm_scale=0.0, workspace=None, out=None, scores_out=None,
                      stream=None):
    """Append-on-decode (see include/kvq.h): writes the new token's encoded key / value
    rows at position T of the cache tensors (in place) and returns the decode step over
    the T + 1 tokens: (out [B, Hq, D] fp32 or None, scores [B, Hq, T + 1] or None)."""
    _need_cuda(q, k_new, v_new, k_codes, k_scales, k_words, k_norms, sketch, v_codes, v_scales)
    B, Hq, D = q.shape
    if want_out and out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float32, device=q.device)
    if want_scores and scores_out is None:
        scores_out = torch.empty((B, Hq, T + 1), dtype=torch.float32, device=q.device)
    a = make_decode_append_args(q, k_new, v_new if want_out else None, T=T, k_codes=k_codes,
                                k_scales=k_scales, k_words=k_words, k_norms=k_norms, sketch=sketch,
                                v_codes=v_codes if want_out else None,
                                v_scales=v_scales if want_out else None,
                                out=out if want_out else None,
                                scores_out=scores_out if want_scores else None, sm_scale=sm_scale)
    need = int(lib.kvq_decode_append_workspace_bytes(ctypes.byref(a)))
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    a.base.workspace, a.base.workspace_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    _check("kvq_decode_append", lib.kvq_decode_append(ctypes.byref(a), _stream(stream)))
    return (out if want_out else None), (scores_out if want_scores else None)


def kvq_quantize_int8_channelwise(x, codes=None, scales=None, stream=None):
    """Channel-wise INT8 of x [..., rows, d] (fp16/fp32): each leading index is a block
    with one scale per column; returns (codes int8 like x, scales fp32 [..., d])."""
    _need_cuda(x)
    rows, d = x.shape[-2], x.shape[-1]
    nb = x.numel() // (rows * d)
    if codes is None:
        codes = torch.empty(x.shape, dtype=torch.int8, device=x.device)
    if scales is None:
        scales = torch.empty(x.shape[:-2] + (d,), dtype=torch.float32, device=x.device)
    _check("kvq_quantize_int8_channelwise",
           lib.kvq_quantize_int8_channelwise(x.data_ptr(), _dtype_code(x), nb, rows, d, codes.data_ptr(),
                                             scales.data_ptr(), _stream(stream)))
    return codes, scales


def kvq_dequantize_int8_channelwise(codes, scales, out=None, out_dtype=torch.float16, stream=None):
    _need_cuda(codes, scales)
    rows, d = codes.shape[-2], codes.shape[-1]
    nb = codes.numel() // (rows * d)
    if out is None:
        out = torch.empty(codes.shape, dtype=out_dtype, device=codes.device)
    _check("kvq_dequantize_int8_channelwise",
           lib.kvq_dequantize_int8_channelwise(codes.data_ptr(), scales.data_ptr(), nb, rows, d,
                                               out.data_ptr(), _dtype_code(out), _stream(stream)))
    return out


def kvq_quantize_int4(x, group, packed=None, scales=None, zeros=None, stream=None):
    """Group-wise asymmetric INT4 of x [..., d]: returns (packed uint8 [..., d/2], scales,
    zeros fp32 [..., d/group])."""
    _need_cuda(x)
    d = x.shape[-1]
    n = x.numel() // d
    if packed is None:
        packed = torch.empty(x.shape[:-1] + (d // 2,), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(x.shape[:-1] + (d // group,), dtype=torch.float32, device=x.device)
    if zeros is None:
        zeros = torch.empty(x.shape[:-1] + (d // group,), dtype=torch.float32, device=x.device)
    _check("kvq_quantize_int4",
           lib.kvq_quantize_int4(x.data_ptr(), _dtype_code(x), n, d, group, packed.data_ptr(), scales.data_ptr(),
                                 zeros.data_ptr(), _stream(stream)))
    return packed, scales, zeros


def kvq_dequantize_int4(packed, scales, zeros, group, out=None, out_dtype=torch.float16, stream=None):
    _need_cuda(packed, scales, zeros)
    d = packed.shape[-1] * 2
    n = packed.numel() * 2 // d
    if out is None:
        out = torch.empty(packed.shape[:-1] + (d,), dtype=out_dtype, device=packed.device)
    _check("kvq_dequantize_int4",
           lib.kvq_dequantize_int4(packed.data_ptr(), scales.data_ptr(), zeros.data_ptr(), n, d, group,
                                   out.data_ptr(), _dtype_code(out), _stream(stream)))
    return out


def make_decode_int4v_args(q, *, k_codes, k_scales, v_packed, v_scales4, v_zeros4, v_group, out=None,
                           scores_out=None, sm_scale=0.0, workspace=None):
    """Fill a ``kvq_decode_int4v_args`` (INT8 keys, group-wise INT4 values)."""
    a = DecodeInt4vArgs()
    a.base = make_decode_args(q, k_codes=k_codes, k_scales=k_scales, out=out, scores_out=scores_out,
                              sm_scale=sm_scale, workspace=workspace)
    a.v_packed = v_packed.data_ptr() if v_packed is not None else None
    a.v_scales4 = v_scales4.data_ptr() if v_scales4 is not None else None
    a.v_zeros4 = v_zeros4.data_ptr() if v_zeros4 is not None else None
    a.v_group = v_group
    return a


def kvq_decode_attention_int4v(q, *, k_codes, k_scales, v_packed, v_scales4, v_zeros4, v_group,
                               want_scores=False, sm_scale=0.0, workspace=None, out=None,
                               scores_out=None, stream=None):
    """Decode step with INT8 keys and group-wise INT4 values; returns (out, scores or None)."""
    _need_cuda(q, k_codes, k_scales, v_packed, v_scales4, v_zeros4)
    B, Hq, D = q.shape
    T = k_codes.shape[2]
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float32, device=q.device)
    if want_scores and scores_out is None:
        scores_out = torch.empty((B, Hq, T), dtype=torch.float32, device=q.device)
    a = make_decode_int4v_args(q, k_codes=k_codes, k_scales=k_scales, v_packed=v_packed,
                               v_scales4=v_scales4, v_zeros4=v_zeros4, v_group=v_group, out=out,
                               scores_out=scores_out if want_scores else None, sm_scale=sm_scale)
    need = int(lib.kvq_decode_int4v_workspace_bytes(ctypes.byref(a)))
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    a.base.workspace, a.base.workspace_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    _check("kvq_decode_attention_int4v", lib.kvq_decode_attention_int4v(ctypes.byref(a), _stream(stream)))
    return out, (scores_out if want_scores else None)


def make_decode_mass_args(q, attn_mass, *, k_codes=None, k_scales=None, k_words=None, k_norms=None,
                          sketch=None, v_codes, v_scales, out, scores_out=None, sm_scale=0.0,
                          workspace=None):
    """Fill a ``kvq_decode_mass_args``."""
    a = DecodeMassArgs()
    a.base = make_decode_args(q, k_codes=k_codes, k_scales=k_scales, k_words=k_words, k_norms=k_norms,
                              sketch=sketch, v_codes=v_codes, v_scales=v_scales, out=out,
                              scores_out=scores_out, sm_scale=sm_scale, workspace=workspace)
    a.attn_mass = attn_mass.data_ptr() if attn_mass is not None else None
    return a


def kvq_decode_attention_mass(q, attn_mass, *, k_codes=None, k_scales=None, k_words=None, k_norms=None,
                              sketch=None, v_codes, v_scales, want_scores=False, sm_scale=0.0,
                              workspace=None, out=None, scores_out=None, stream=None):
    """Decode step that also adds its attention mass (summed over query heads) into
    ``attn_mass`` [B, T] fp32 in place; returns (out, scores or None)."""
    _need_cuda(q, attn_mass, k_codes, k_scales, k_words, k_norms, sketch, v_codes, v_scales)
    B, Hq, D = q.shape
    ref = k_words if k_words is not None else k_codes
    T = ref.shape[2]
    if attn_mass.dtype != torch.float32 or tuple(attn_mass.shape) != (B, T):
        raise ValueError("attn_mass must be fp32 [batch, seq_len]")
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float32, device=q.device)
    if want_scores and scores_out is None:
        scores_out = torch.empty((B, Hq, T), dtype=torch.float32, device=q.device)
    a = make_decode_mass_args(q, attn_mass, k_codes=k_codes, k_scales=k_scales, k_words=k_words,
                              k_norms=k_norms, sketch=sketch, v_codes=v_codes, v_scales=v_scales, out=out,
                              scores_out=scores_out if want_scores else None, sm_scale=sm_scale)
    need = int(lib.kvq_decode_mass_workspace_bytes(ctypes.byref(a)))
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    a.base.workspace, a.base.workspace_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    _check("kvq_decode_attention_mass", lib.kvq_decode_attention_mass(ctypes.byref(a), _stream(stream)))
    return out, (scores_out if want_scores else None)


def kvq_evict_select(mass, n_sink, n_keep, kept=None, stream=None):
    """Tokens to keep per batch row of ``mass`` [B, T] fp32: int32 [B, n_keep], increasing."""
    _need_cuda(mass, kept)
    if mass.dtype != torch.float32 or mass.dim() != 2:
        raise ValueError("mass must be fp32 [batch, seq_len]")
    B, T = mass.shape
    if kept is None:
        kept = torch.empty((B, max(int(n_keep), 0)), dtype=torch.int32, device=mass.device)
    _check("kvq_evict_select", lib.kvq_evict_select(_ptr(mass), B, T, int(n_sink), int(n_keep), _ptr(kept),
                                                    _stream(stream)))
    return kept


def kvq_gather_rows(src, kept, dst=None, stream=None):
    """Compact ``src`` [B, H, T, ...] to the kept tokens (int32 [B, n_keep]):
    dst[b, h, j] = src[b, h, kept[b, j]]; ``dst`` [B, H, R >= n_keep, ...] if given."""
    _need_cuda(src, kept, dst)
    if kept.dtype != torch.int32:
        raise ValueError("kept must be int32")
    B, H, T = src.shape[:3]
    n_keep = kept.shape[1]
    row_bytes = src[0, 0, 0].numel() * src.element_size() if src.numel() else 0
    if dst is None:
        dst = torch.empty((B, H, n_keep) + tuple(src.shape[3:]), dtype=src.dtype, device=src.device)
    if dst.dtype != src.dtype or dst.shape[:2] != src.shape[:2] or dst.shape[3:] != src.shape[3:]:
        raise ValueError("dst must match src except along the token axis")
    _check("kvq_gather_rows", lib.kvq_gather_rows(_ptr(src), _ptr(dst), B, H, T, dst.shape[2], row_bytes,
                                                  _ptr(kept), n_keep, _stream(stream)))
    return dst


def kvq_qjl_residual_encode(keys, group, sketch, stream=None):
    """Keys fp16 [..., D] -> group-wise INT4 + the residual's 1-bit QJL sketch: a dict of
    packed [..., D/2] uint8, scales / zeros [..., D/group] fp32, residual [..., D] fp16,
    words [..., m/32] (int32 view of uint32) and rnorms [...] fp16."""
    _need_cuda(keys, sketch)
    if keys.dtype != torch.float16:
        raise ValueError("keys must be fp16")
    D = keys.shape[-1]
    lead = tuple(keys.shape[:-1])
    n = keys.numel() // D
    m = sketch.shape[0]
    dev = keys.device
    o = dict(packed=torch.empty(lead + (D // 2,), dtype=torch.uint8, device=dev),
             scales=torch.empty(lead + (D // group,), dtype=torch.float32, device=dev),
             zeros=torch.empty(lead + (D // group,), dtype=torch.float32, device=dev),
             residual=torch.empty(lead + (D,), dtype=torch.float16, device=dev),
             words=torch.empty(lead + (m // 32,), dtype=torch.int32, device=dev),
             rnorms=torch.empty(lead, dtype=torch.float16, device=dev))
    _check("kvq_qjl_residual_encode", lib.kvq_qjl_residual_encode(
        _ptr(keys), n, D, int(group), _ptr(sketch), m, _ptr(o["packed"]), _ptr(o["scales"]), _ptr(o["zeros"]),
        _ptr(o["residual"]), _ptr(o["words"]), _ptr(o["rnorms"]), _stream(stream)))
    return o


def make_decode_qjlres_args(q, *, k_packed4, k_scales4, k_zeros4, k_group, k_words, k_norms, sketch,
                            v_codes=None, v_scales=None, out=None, scores_out=None, sm_scale=0.0,
                            workspace=None):
    """Fill a ``kvq_decode_qjlres_args`` (residual keys, INT8 values)."""
    a = DecodeQjlresArgs()
    a.base = make_decode_args(q, k_words=k_words, k_norms=k_norms, sketch=sketch, v_codes=v_codes,
                              v_scales=v_scales, out=out, scores_out=scores_out, sm_scale=sm_scale,
                              workspace=workspace)
    a.k_packed4 = k_packed4.data_ptr() if k_packed4 is not None else None
    a.k_scales4 = k_scales4.data_ptr() if k_scales4 is not None else None
    a.k_zeros4 = k_zeros4.data_ptr() if k_zeros4 is not None else None
    a.k_group = int(k_group)
    return a


def kvq_decode_attention_qjlres(q, *, k_packed4, k_scales4, k_zeros4, k_group, k_words, k_norms, sketch,
                                v_codes=None, v_scales=None, want_out=True, want_scores=False,
                                sm_scale=0.0, workspace=None, out=None, scores_out=None, stream=None):
    """Decode step over residual keys (kvq_qjl_residual_encode) and INT8 values; returns
    (out [B, Hq, D] fp32 or None, scores [B, Hq, T] or None)."""
    _need_cuda(q, k_packed4, k_scales4, k_zeros4, k_words, k_norms, sketch, v_codes, v_scales)
    B, Hq, D = q.shape
    T = k_words.shape[2]
    if want_out and out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float32, device=q.device)
    if want_scores and scores_out is None:
        scores_out = torch.empty((B, Hq, T), dtype=torch.float32, device=q.device)
    a = make_decode_qjlres_args(q, k_packed4=k_packed4, k_scales4=k_scales4, k_zeros4=k_zeros4,
                                k_group=k_group, k_words=k_words, k_norms=k_norms, sketch=sketch,
                                v_codes=v_codes if want_out else None,
                                v_scales=v_scales if want_out else None, out=out if want_out else None,
                                scores_out=scores_out if want_scores else None, sm_scale=sm_scale)
    need = int(lib.kvq_decode_qjlres_workspace_bytes(ctypes.byref(a)))
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    a.base.workspace, a.base.workspace_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    _check("kvq_decode_attention_qjlres", lib.kvq_decode_attention_qjlres(ctypes.byref(a), _stream(stream)))
    return (out if want_out else None), (scores_out if want_scores else None)


def kvq_gather_rows_multi(srcs, kept, dsts=None, stream=None):
    """kvq_gather_rows for several arrays [B, H, T, ...] of one cache in one launch;
    returns the list of compacted arrays."""
    _need_cuda(kept, *srcs)
    if kept.dtype != torch.int32:
        raise ValueError("kept must be int32")
    B, H = srcs[0].shape[:2]
    n_keep = kept.shape[1]
    if dsts is None:
        dsts = [torch.empty((B, H, n_keep) + tuple(x.shape[3:]), dtype=x.dtype, device=x.device) for x in srcs]
    arr = (GatherArray * max(1, len(srcs)))()
    for i, (x, y) in enumerate(zip(srcs, dsts)):
        _need_cuda(y)
        if tuple(x.shape[:2]) != (B, H) or y.dtype != x.dtype or y.shape[:2] != x.shape[:2] or y.shape[3:] != x.shape[3:]:
            raise ValueError("every array is [B, H, T, ...] with dst matching src except along the token axis")
        arr[i] = GatherArray(x.data_ptr(), y.data_ptr(), x.shape[2], y.shape[2],
                             x[0, 0, 0].numel() * x.element_size())
    _check("kvq_gather_rows_multi", lib.kvq_gather_rows_multi(arr, len(srcs), B, H, _ptr(kept), n_keep,
                                                              _stream(stream)))
    return dsts
