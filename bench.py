#!/usr/bin/env python
"""Throughput of the KV-cache compression + compressed-cache decode path on B200.

One step is one pass of the whole path over one batch of synthetic input:
  7B-shaped cache  (32 layers x {K, V} x [batch 8, 32 heads, 4096 tokens, 128] fp16)
    1. INT8 per-token absmax quantize of the whole cache            (1 launch)
    2. one decode step per layer: INT8 scores, softmax, sum of INT8
       values, one fp16 query per head                              (32 x 2 launches)
    3. INT8 dequantize of the whole cache back to fp16               (1 launch)
  long-context GQA cache (batch 4, 32 query / 8 KV heads, 131072 tokens, 128)
    4. QJL sign sketch of K (m = 256, Gaussian S from seed 7)        (1 launch)
    5. INT8 quantize of V                                            (1 launch)
    6. one fused GQA decode step: query sketch, estimator scores,
       softmax, sum of INT8 values                                   (3 launches)
The reported value is the algorithmic bytes of the step (each input read once, each
output written once) divided by the device time of the step, in GB/s; decode keys/s and
per-row figures are reported beside it.  Inputs (~47 GB resident) are far larger than
the 126 MB L2, so no flush is needed between steps.

Also on the line, outside the step: the widened rows (next_rows, including the step's
GQA decode with the weighted value sum kept on the CUDA cores), the one-layer INT8
cache's latencies (one_layer), the key-sketch workload's encode and estimator scores
over 1M keys (key_sketch), the INT8 quantize/dequantize throughput sweep, an end-to-end
step from pinned host memory (e2e), and the C oracle's rate on the host cores, with its
all-cores build and single-threaded (cpu_baseline).  Per-row figures come last on the
line, as [ms, GB/s, fraction of the measured HBM peak(, oracle GB/s)].
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "KV quantize/dequant GB/s and compressed-cache decode keys/s; % of HBM peak"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_TC_TFLOPS = 1590.0

# ---------------------------------------------------------------------------------
# Workload geometry and algorithmic bytes (host logic; no GPU needed)
# ---------------------------------------------------------------------------------
LLAMA = dict(layers=32, batch=8, heads=32, seq=4096, dim=128)
GQA = dict(batch=4, q_heads=32, kv_heads=8, seq=131072, dim=128, m=256)


def row_bytes(llama=LLAMA, gqa=GQA):
    """Algorithmic bytes of each row of the step (read once + written once)."""
    D = llama["dim"]
    rows_a = llama["layers"] * 2 * llama["batch"] * llama["heads"] * llama["seq"]
    keys_layer = llama["batch"] * llama["heads"] * llama["seq"]
    q_layer = llama["batch"] * llama["heads"] * D
    n_g = gqa["batch"] * gqa["kv_heads"] * gqa["seq"]
    m = gqa["m"]
    q_g = gqa["batch"] * gqa["q_heads"] * D
    return {
        "quantize_cache": rows_a * (2 * D + D + 4),
        "decode_int8": llama["layers"] * (keys_layer * 2 * (D + 4) + q_layer * 2 + q_layer * 4),
        "dequantize_cache": rows_a * (D + 4 + 2 * D),
        "qjl_encode": n_g * (2 * D + m // 8 + 2) + m * D * 2,
        "quantize_v": n_g * (2 * D + D + 4),
        "decode_qjl": n_g * (m // 8 + 2 + D + 4) + m * D * 2 + q_g * 2 + q_g * 4,
    }


def decode_keys(llama=LLAMA, gqa=GQA):
    return (llama["layers"] * llama["batch"] * llama["heads"] * llama["seq"]
            + gqa["batch"] * gqa["kv_heads"] * gqa["seq"])


# quantize; per layer the INT8 decode and its combine; dequantize; QJL encode; value
# quantize; the tensor-core QJL decode (which projects the queries itself) and its combine
LAUNCHES_PER_STEP = 1 + LLAMA["layers"] * 2 + 1 + 1 + 1 + 2


def max_over_ranks(value: float, group=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    backend = dist.get_backend(group)
    dev = torch.device("cuda", torch.cuda.current_device()) if backend == "nccl" else torch.device("cpu")
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def aggregate(bytes_per_rank: float, n_ranks: int, step_ms_max: float, steps: int) -> float:
    """Whole-job GB/s: bytes all ranks processed / the slowest rank's time."""
    return bytes_per_rank * n_ranks * steps / (step_ms_max * steps * 1e-3) / 1e9


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def load_tc_peak():
    """Dense fp16/bf16 tensor-core TFLOP/s for a kernel timed alone (the burst figure)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"])
    except Exception:
        return FALLBACK_TC_TFLOPS


# ---------------------------------------------------------------------------------
# Clock sampling during the timed region
# ---------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="kvq_clocks_", suffix=".csv")
            os.close(fd)
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                   "-lms", "100"]
            if self.gpu_id:
                cmd += ["-i", self.gpu_id]
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 8:
                    continue
                try:
                    rows.append((float(parts[0]), float(parts[1]), parts[4:8]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for _, _, flags in rows for n, fl in zip(names, flags) if fl == "Active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons, "samples": len(rows)}


def gpu_id_for(device_index: int):
    import torch
    try:
        uuid = str(torch.cuda.get_device_properties(device_index).uuid)
        return uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    except Exception:
        return None


# ---------------------------------------------------------------------------------
# The device workload
# ---------------------------------------------------------------------------------
class Workload:
    def __init__(self, device, seed_offset=0):
        import torch
        from kv_cache_quantization_absmax_b200 import inputs, kvq

        self.kvq = kvq
        self.torch = torch
        L, B, H, T, D = (LLAMA[k] for k in ("layers", "batch", "heads", "seq", "dim"))
        gb, gq, gk, gt, m = (GQA[k] for k in ("batch", "q_heads", "kv_heads", "seq", "m"))
        dev = device
        # 7B-shaped cache [L, 2, B, H, T, D] fp16: one sigma per (layer, K/V, head, channel)
        self.cache = inputs.lognormal_cache_device(3 + seed_offset, (L, 2, B, H, T, D),
                                                   n_sigma_dims=(0, 1, 3, 5), device=dev)
        self.q7 = inputs.gaussian_queries_device(30 + seed_offset, (L, B, H, D), dev)
        self.codes = torch.empty((L, 2, B, H, T, D), dtype=torch.int8, device=dev)
        self.scales = torch.empty((L, 2, B, H, T), dtype=torch.float32, device=dev)
        self.deq = torch.empty((L, 2, B, H, T, D), dtype=torch.float16, device=dev)
        self.out7 = torch.empty((L, B, H, D), dtype=torch.float32, device=dev)
        # long-context GQA cache [2, B, Hkv, T, D] fp16
        self.gcache = inputs.lognormal_cache_device(5 + seed_offset, (2, gb, gk, gt, D),
                                                    n_sigma_dims=(0, 2, 4), device=dev)
        self.qg = inputs.gaussian_queries_device(50 + seed_offset, (gb, gq, D), dev)
        self.S = torch.from_numpy(inputs.sketch_matrix(m, D)).to(dev)
        self.words = torch.empty((gb, gk, gt, m // 32), dtype=torch.int32, device=dev)
        self.norms = torch.empty((gb, gk, gt), dtype=torch.float16, device=dev)
        self.vcodes = torch.empty((gb, gk, gt, D), dtype=torch.int8, device=dev)
        self.vscales = torch.empty((gb, gk, gt), dtype=torch.float32, device=dev)
        self.outg = torch.empty((gb, gq, D), dtype=torch.float32, device=dev)
        # decode argument structs and caller-owned workspaces (sized once)
        self.args7 = []
        for l in range(L):
            a = kvq.make_decode_args(self.q7[l], k_codes=self.codes[l, 0], k_scales=self.scales[l, 0],
                                     v_codes=self.codes[l, 1], v_scales=self.scales[l, 1],
                                     out=self.out7[l])
            self.args7.append(a)
        ws7 = kvq.kvq_decode_workspace_bytes(self.args7[0])
        self.ws7 = torch.empty(ws7, dtype=torch.uint8, device=dev)
        for a in self.args7:
            a.workspace, a.workspace_bytes = self.ws7.data_ptr(), ws7
        self.argsg = kvq.make_decode_args(self.qg, k_words=self.words, k_norms=self.norms, sketch=self.S,
                                          v_codes=self.vcodes, v_scales=self.vscales, out=self.outg)
        wsg = kvq.kvq_decode_workspace_bytes(self.argsg)
        self.wsg = torch.empty(wsg, dtype=torch.uint8, device=dev)
        self.argsg.workspace, self.argsg.workspace_bytes = self.wsg.data_ptr(), wsg
        # the same step with the weighted value sum kept on the CUDA cores
        self.argsg_cc = kvq.make_decode_args(self.qg, k_words=self.words, k_norms=self.norms, sketch=self.S,
                                             v_codes=self.vcodes, v_scales=self.vscales, out=self.outg,
                                             flags=kvq.KVQ_DECODE_CUDA_CORES)
        self.argsg_cc.workspace, self.argsg_cc.workspace_bytes = self.wsg.data_ptr(), wsg
        torch.cuda.synchronize()

    def step(self, stream, ev=None):
        """Launch the whole path on `stream`; if `ev` (7 events) is given, record row
        boundaries."""
        import ctypes
        kvq = self.kvq
        lib = kvq.lib
        s = ctypes.c_void_p(stream.cuda_stream)
        rec = (lambda i: ev[i].record(stream)) if ev is not None else (lambda i: None)
        rec(0)
        kvq.kvq_quantize_int8(self.cache, self.codes, self.scales, stream=stream)
        rec(1)
        for a in self.args7:
            st = lib.kvq_decode_attention(ctypes.byref(a), s)
            if st != kvq.KVQ_OK:
                raise kvq.KvqError("kvq_decode_attention", st)
        rec(2)
        kvq.kvq_dequantize_int8(self.codes, self.scales, out=self.deq, stream=stream)
        rec(3)
        kvq.kvq_qjl_encode(self.gcache[0], self.S, self.words, self.norms, stream=stream)
        rec(4)
        kvq.kvq_quantize_int8(self.gcache[1], self.vcodes, self.vscales, stream=stream)
        rec(5)
        st = lib.kvq_decode_attention(ctypes.byref(self.argsg), s)
        if st != kvq.KVQ_OK:
            raise kvq.KvqError("kvq_decode_attention", st)
        rec(6)

    def host_buffers(self):
        """Pinned host copies of the step's inputs, for the end-to-end measurement."""
        t = self.torch
        hb = {}
        for name in ("cache", "q7", "gcache", "qg"):
            dv = getattr(self, name)
            h = t.empty(dv.shape, dtype=dv.dtype, pin_memory=True)
            h.copy_(dv)
            hb[name] = h
        hb["out7"] = t.empty(self.out7.shape, dtype=t.float32, pin_memory=True)
        hb["outg"] = t.empty(self.outg.shape, dtype=t.float32, pin_memory=True)
        return hb


ROW_NAMES = ["quantize_cache", "decode_int8", "dequantize_cache", "qjl_encode", "quantize_v",
             "decode_qjl"]


SWEEP_D = (128, 1024, 8192)
SWEEP_TOTALS = (10 ** 6, 10 ** 7, 10 ** 8, 10 ** 9)


def measure_sweep(stream, reps=3):
    """The INT8 quantize/dequantize throughput sweep (fp32 and fp16 [N x D] tensors, D in
    {128, 1024, 8192}, N = total // D for total in {1e6 .. 1e9}; N(0,1) values with 1% of
    the columns x20): per point the device time of each kernel (the L2 flushed before
    every timed launch), the reconstruction error max |x - x_hat| and mean |x - x_hat|,
    and the attention-score error of one fp32 N(0,1) query, |q.x - q.x_hat| over all rows
    (scores of the codes by kvq_int8_scores against the fp32 dot product of x)."""
    import numpy as np
    import torch
    from kv_cache_quantization_absmax_b200 import inputs, kvq
    dev = torch.device("cuda", torch.cuda.current_device())
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    peak, _ = load_peaks()
    out = []
    idx = -1
    for dtype in (np.float32, np.float16):
        for d in SWEEP_D:
            for total in SWEEP_TOTALS:
                idx += 1                                   # sweep index 0 .. 23: seed 2000 + index
                x, q, _ = inputs.sweep_matrix_device(total, d, dtype, idx, dev)
                n = x.shape[0]
                codes = torch.empty((n, d), dtype=torch.int8, device=dev)
                scales = torch.empty((n,), dtype=torch.float32, device=dev)
                xh = torch.empty_like(x)
                # x is drawn on torch's current stream, whose freed temporaries the
                # outputs above may reuse: the kernels on `stream` start after it is done
                torch.cuda.synchronize()

                def timed(fn):
                    with torch.cuda.stream(stream):
                        fn()                                   # warm-up
                    ms = 0.0
                    for _ in range(reps):
                        with torch.cuda.stream(stream):
                            flush.fill_(idx & 0xFF)
                            e0 = torch.cuda.Event(enable_timing=True)
                            e1 = torch.cuda.Event(enable_timing=True)
                            e0.record(stream)
                            fn()
                            e1.record(stream)
                        torch.cuda.synchronize()
                        ms += e0.elapsed_time(e1)
                    return ms / reps
                b = x.element_size()
                qms = timed(lambda: kvq.kvq_quantize_int8(x, codes, scales, stream=stream))
                dms = timed(lambda: kvq.kvq_dequantize_int8(codes, scales, out=xh, stream=stream))
                bytes_q = n * d * (b + 1) + 4 * n
                # errors, in row chunks of at most 2^26 elements
                qd = torch.from_numpy(q).to(dev)
                sc = kvq.kvq_int8_scores(qd, codes, scales)
                rmax = rsum = smax = ssum = 0.0
                step = max(1, (1 << 26) // d)
                for r0 in range(0, n, step):
                    xs = x[r0:r0 + step].float()
                    e = (xs - xh[r0:r0 + step].float()).abs_()
                    rmax = max(rmax, float(e.max()))
                    rsum += float(e.double().sum())
                    se = (xs @ qd - sc[r0:r0 + step]).abs_()
                    smax = max(smax, float(se.max()))
                    ssum += float(se.double().sum())
                torch.cuda.synchronize()
                # below 1e8 elements (at most 80 MB moved) a launch is a few microseconds:
                # latency and L2, not HBM, set its time, so no HBM fraction is claimed
                hbm = total >= 10 ** 8
                out.append({"dtype": "f16" if dtype == np.float16 else "f32", "d": d, "total": total, "rows": n,
                            "regime": "hbm" if hbm else "latency",
                            "quantize_ms": round(qms, 4), "quantize_GBps": round(bytes_q / (qms * 1e-3) / 1e9, 1),
                            "quantize_frac": round(bytes_q / (qms * 1e-3) / 1e9 / peak, 4) if hbm else None,
                            "dequantize_ms": round(dms, 4), "dequantize_GBps": round(bytes_q / (dms * 1e-3) / 1e9, 1),
                            "dequantize_frac": round(bytes_q / (dms * 1e-3) / 1e9 / peak, 4) if hbm else None,
                            "recon_max_abs": round(rmax, 6), "recon_mean_abs": round(rsum / (n * d), 7),
                            "score_max_abs": round(smax, 6), "score_mean_abs": round(ssum / n, 7)})
                del x, codes, scales, xh, sc
    del flush
    torch.cuda.empty_cache()
    if kvq.kvq_device_error() != 0:
        raise RuntimeError("device-side error recorded during the sweep")
    return out


def measure_small_configs(stream, reps=20):
    """The two workloads that are not part of the step.

    one-layer INT8 cache with outlier channels (K, V fp16 [1, 8, 512, 128], seed 0; 3.2 MB,
    L2-resident): the latency of quantizing K and V, dequantizing them back to fp16, and
    the decode scores of one fp16 query per head against the INT8 keys (no roofline claim).

    key sketch (keys fp16 [1, 32, 32768, 128] seed 4, m = 256, S seed 7, one N(0,1)
    query per head seed 40): the encode, and the asymmetric-estimator scores of the query
    against all 1,048,576 sketched keys (query sketch + score pass, 34 B read and 4 B
    written per key); the L2 is flushed before every timed launch."""
    import ctypes

    import numpy as np
    import torch
    from kv_cache_quantization_absmax_b200 import inputs, kvq
    dev = torch.device("cuda", torch.cuda.current_device())
    peak, _ = load_peaks()
    tc_peak = load_tc_peak()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def timed(fn, n, do_flush):
        with torch.cuda.stream(stream):
            fn()
        torch.cuda.synchronize()
        ms = 0.0
        for i in range(n):
            with torch.cuda.stream(stream):
                if do_flush:
                    flush.fill_(i & 0xFF)
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                fn()
                e1.record(stream)
            torch.cuda.synchronize()
            ms += e0.elapsed_time(e1)
        return ms / n

    out = {}
    # ---- one-layer cache, latency ----
    k, v, q = inputs.outlier_layer(seed=0)
    kv = torch.from_numpy(np.stack([k, v])).to(dev)                  # [2, 1, 8, 512, 128]
    qg = torch.from_numpy(q).to(dev)
    codes = torch.empty(kv.shape, dtype=torch.int8, device=dev)
    scales = torch.empty(kv.shape[:-1], dtype=torch.float32, device=dev)
    deq = torch.empty_like(kv)
    scores = torch.empty((1, 8, 512), dtype=torch.float32, device=dev)
    torch.cuda.synchronize()
    sa = kvq.make_decode_args(qg, k_codes=codes[0], k_scales=scales[0], scores_out=scores)
    ws = torch.empty(kvq.kvq_decode_workspace_bytes(sa), dtype=torch.uint8, device=dev)
    sa.workspace, sa.workspace_bytes = ws.data_ptr(), ws.numel()
    s = ctypes.c_void_p(stream.cuda_stream)

    def score_call():
        st = kvq.lib.kvq_decode_attention(ctypes.byref(sa), s)
        if st != kvq.KVQ_OK:
            raise kvq.KvqError("kvq_decode_attention", st)
    q_us = timed(lambda: kvq.kvq_quantize_int8(kv, codes, scales, stream=stream), reps, False) * 1e3
    d_us = timed(lambda: kvq.kvq_dequantize_int8(codes, scales, out=deq, stream=stream), reps, False) * 1e3
    s_us = timed(score_call, reps, False) * 1e3
    out["one_layer"] = {"quantize_kv_us": round(q_us, 2), "dequantize_kv_us": round(d_us, 2),
                        "scores_us": round(s_us, 2), "regime": "latency"}
    del kv, codes, scales, deq, scores, ws
    # ---- key sketch: encode and estimator scores over 1M keys ----
    H, T, D, m = 32, 32768, 128, GQA["m"]
    keys = inputs.lognormal_cache_device(4, (1, H, T, D), n_sigma_dims=(1, 3), device=dev)
    qk = torch.from_numpy(inputs.gaussian_queries(40, 1, H)).to(dev)
    S = torch.from_numpy(inputs.sketch_matrix(m, D)).to(dev)
    words = torch.empty((1, H, T, m // 32), dtype=torch.int32, device=dev)
    norms = torch.empty((1, H, T), dtype=torch.float16, device=dev)
    sc = torch.empty((1, H, T), dtype=torch.float32, device=dev)
    torch.cuda.synchronize()
    n_keys = H * T
    e_ms = timed(lambda: kvq.kvq_qjl_encode(keys, S, words, norms, stream=stream), 5, True)
    e_bytes = n_keys * (2 * D + m // 8 + 2) + m * D * 2
    e_flops = 2.0 * n_keys * m * D
    ka = kvq.make_decode_args(qk, k_words=words, k_norms=norms, sketch=S, scores_out=sc)
    kws = torch.empty(kvq.kvq_decode_workspace_bytes(ka), dtype=torch.uint8, device=dev)
    ka.workspace, ka.workspace_bytes = kws.data_ptr(), kws.numel()

    def key_scores():
        st = kvq.lib.kvq_decode_attention(ctypes.byref(ka), s)
        if st != kvq.KVQ_OK:
            raise kvq.KvqError("kvq_decode_attention", st)
    s_ms = timed(key_scores, reps, True)
    s_bytes = n_keys * (m // 8 + 2 + 4) + m * D * 2 + H * D * 2
    bound_us = max(e_bytes / (peak * 1e9), e_flops / (tc_peak * 1e12)) * 1e6
    out["key_sketch"] = {
        "encode_ms": round(e_ms, 4), "encode_GBps": round(e_bytes / (e_ms * 1e-3) / 1e9, 1),
        "encode_roofline_frac": round(bound_us / (e_ms * 1e3), 4),
        "scores_ms": round(s_ms, 4), "scores_keys_per_s": round(n_keys / (s_ms * 1e-3), 1),
        "scores_GBps": round(s_bytes / (s_ms * 1e-3) / 1e9, 1),
        "scores_frac_hbm": round(s_bytes / (s_ms * 1e-3) / 1e9 / peak, 4)}
    del keys, words, norms, sc, kws, flush
    torch.cuda.empty_cache()
    if kvq.kvq_device_error() != 0:
        raise RuntimeError("device-side error recorded during the small workloads")
    return out


def measure_next_rows(wl, stream, reps=3):
    """Device time of the widened rows (not part of the step): append-on-decode on the
    same caches, whose last row each call re-appends (the new key / value rows are the
    cache's own fp16 rows at that position, so the cache does not change)."""
    import ctypes
    import torch
    kvq = wl.kvq
    lib = kvq.lib
    L, B, H, T, D = (LLAMA[k] for k in ("layers", "batch", "heads", "seq", "dim"))
    gb, gq, gk, gt, m = (GQA[k] for k in ("batch", "q_heads", "kv_heads", "seq", "m"))
    s = ctypes.c_void_p(stream.cuda_stream)
    knew = wl.cache[:, :, :, :, T - 1].contiguous()          # [L, 2, B, H, D]
    gnew = wl.gcache[:, :, :, gt - 1].contiguous()            # [2, gb, gk, D]
    torch.cuda.synchronize()   # made on torch's current stream, used on `stream`
    a7 = [kvq.make_decode_append_args(wl.q7[l], knew[l, 0], knew[l, 1], T=T - 1,
                                      k_codes=wl.codes[l, 0], k_scales=wl.scales[l, 0],
                                      v_codes=wl.codes[l, 1], v_scales=wl.scales[l, 1],
                                      out=wl.out7[l], workspace=wl.ws7) for l in range(L)]
    ag = kvq.make_decode_append_args(wl.qg, gnew[0], gnew[1], T=gt - 1, k_words=wl.words,
                                     k_norms=wl.norms, sketch=wl.S, v_codes=wl.vcodes,
                                     v_scales=wl.vscales, out=wl.outg, workspace=wl.wsg)
    # the append entry point keeps the CUDA-core kernels (more CTAs per SM than the
    # tensor-core decode): its workspace is sized on its own, once
    need = max(lib.kvq_decode_append_workspace_bytes(ctypes.byref(a)) for a in a7 + [ag])
    wsa = torch.empty(int(need), dtype=torch.uint8, device=wl.cache.device)
    for a in a7 + [ag]:
        a.base.workspace, a.base.workspace_bytes = wsa.data_ptr(), int(need)

    def run(args_list):
        for a in args_list:
            st = lib.kvq_decode_append(ctypes.byref(a), s)
            if st != kvq.KVQ_OK:
                raise kvq.KvqError("kvq_decode_append", st)

    out = {}
    for name, args_list, units, key_bytes, per_new_written in (
            ("append_int8", a7, B * H, 2 * (D + 4), 2 * (D + 4)),
            ("append_qjl", [ag], gb * gk, m // 8 + 2 + D + 4, m // 8 + 2 + D + 4)):
        with torch.cuda.stream(stream):
            run(args_list)                                    # warm-up
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        with torch.cuda.stream(stream):
            for _ in range(reps):
                run(args_list)
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / reps / len(args_list)
        seq = T if name == "append_int8" else gt
        q_heads = H if name == "append_int8" else gq
        sketch = 0 if name == "append_int8" else m * D * 2
        per_call = (units * seq * key_bytes            # T - 1 cached rows + the appended row, read
                    + units * 2 * D * 2                # new fp16 key and value rows, read
                    + units * per_new_written          # appended encoded rows, written
                    + (gb if name == "append_qjl" else B) * q_heads * D * (2 + 4) + sketch)
        out[name] = {"ms": round(ms, 4), "GB/s": round(per_call / (ms * 1e-3) / 1e9, 1),
                     "bytes_per_call": int(per_call),
                     "workload": ("7B-shaped layer: append 1 token to [8, 32, 4095 + 1, 128] INT8 K/V, "
                                  "decode over 4096 (per layer, 32 layers)") if name == "append_int8" else
                                 ("GQA [4, 32q/8kv]: append 1 token to 131071 QJL keys (m = 256) + "
                                  "INT8 V, decode over 131072")}
    # ---- group-wise INT4 (groups of 32) and channel-wise INT8 over the 7B-shaped cache ----
    g = 32
    elems = L * 2 * B * H * T * D
    v4p = torch.empty((L, 2, B, H, T, D // 2), dtype=torch.uint8, device=wl.cache.device)
    v4s = torch.empty((L, 2, B, H, T, D // g), dtype=torch.float32, device=wl.cache.device)
    v4z = torch.empty_like(v4s)
    cws = torch.empty((L, 2, B, H, D), dtype=torch.float32, device=wl.cache.device)

    def timed(fn, n=reps):
        with torch.cuda.stream(stream):
            fn()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        with torch.cuda.stream(stream):
            for _ in range(n):
                fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n

    def row(name, ms, nbytes, workload):
        out[name] = {"ms": round(ms, 4), "GB/s": round(nbytes / (ms * 1e-3) / 1e9, 1),
                     "bytes_per_call": int(nbytes), "workload": workload}

    cache_desc = "7B-shaped cache, 32 L x {K, V} x [8, 32, 4096, 128] fp16"

    # ---- the long-context GQA decode with the weighted value sum on the CUDA cores ----
    def dec_cc():
        st = lib.kvq_decode_attention(ctypes.byref(wl.argsg_cc), s)
        if st != kvq.KVQ_OK:
            raise kvq.KvqError("kvq_decode_attention", st)
    ms = timed(dec_cc)
    row("decode_qjl_cuda_cores", ms, row_bytes()["decode_qjl"],
        "GQA [4, 32q/8kv, 131072]: the decode_qjl row of the step with KVQ_DECODE_CUDA_CORES")
    # ---- the 7B-shaped INT8 decode with scores and value sum on the CUDA cores ----
    a7cc = [kvq.make_decode_args(wl.q7[l], k_codes=wl.codes[l, 0], k_scales=wl.scales[l, 0],
                                 v_codes=wl.codes[l, 1], v_scales=wl.scales[l, 1], out=wl.out7[l],
                                 flags=kvq.KVQ_DECODE_CUDA_CORES) for l in range(L)]
    wscc = torch.empty(int(lib.kvq_decode_workspace_bytes(ctypes.byref(a7cc[0]))), dtype=torch.uint8,
                       device=wl.cache.device)
    for a in a7cc:
        a.workspace, a.workspace_bytes = wscc.data_ptr(), wscc.numel()

    def dec8_cc():
        for a in a7cc:
            st = lib.kvq_decode_attention(ctypes.byref(a), s)
            if st != kvq.KVQ_OK:
                raise kvq.KvqError("kvq_decode_attention", st)
    ms = timed(dec8_cc) / L
    row("decode_int8_cuda_cores", ms, row_bytes()["decode_int8"] / L,
        "7B-shaped layer [8, 32, 4096, 128]: the decode_int8 row of the step with KVQ_DECODE_CUDA_CORES, per layer")
    del wscc
    ms = timed(lambda: kvq.kvq_quantize_int4(wl.cache, g, v4p, v4s, v4z, stream=stream))
    row("int4_quantize", ms, elems * (2 + 0.5) + elems // g * 8, cache_desc + ", groups of 32")
    ms = timed(lambda: kvq.kvq_dequantize_int4(v4p, v4s, v4z, g, out=wl.deq, stream=stream))
    row("int4_dequantize", ms, elems * (0.5 + 2) + elems // g * 8, cache_desc + " -> fp16")
    a4 = [kvq.make_decode_int4v_args(wl.q7[l], k_codes=wl.codes[l, 0], k_scales=wl.scales[l, 0],
                                     v_packed=v4p[l, 1], v_scales4=v4s[l, 1], v_zeros4=v4z[l, 1],
                                     v_group=g, out=wl.out7[l]) for l in range(L)]
    ws4 = torch.empty(int(lib.kvq_decode_int4v_workspace_bytes(ctypes.byref(a4[0]))), dtype=torch.uint8,
                      device=wl.cache.device)
    for a in a4:
        a.base.workspace, a.base.workspace_bytes = ws4.data_ptr(), ws4.numel()

    def dec4():
        for a in a4:
            st = lib.kvq_decode_attention_int4v(ctypes.byref(a), s)
            if st != kvq.KVQ_OK:
                raise kvq.KvqError("kvq_decode_attention_int4v", st)
    ms = timed(dec4) / L
    keys = B * H * T
    row("decode_int8k_int4v", ms, keys * (D + 4 + D // 2 + (D // g) * 8) + B * H * D * 6,
        "7B-shaped layer: INT8 K + INT4 V (groups of 32) [8, 32, 4096, 128], one decode step per layer")
    ms = timed(lambda: kvq.kvq_quantize_int8_channelwise(wl.cache, wl.codes, cws, stream=stream))
    row("int8_channelwise_quantize", ms, elems * 3 + cws.numel() * 4,
        cache_desc + ", one scale per (layer, K/V, batch, head, channel)")
    ms = timed(lambda: kvq.kvq_dequantize_int8_channelwise(wl.codes, cws, out=wl.deq, stream=stream))
    row("int8_channelwise_dequantize", ms, elems * 3 + cws.numel() * 4, cache_desc + " -> fp16")
    del v4p, v4s, v4z, cws

    # ---- attention-sink eviction over one 7B-shaped layer: 4 sinks + 2044 of 4096 kept ----
    n_sink, n_keep = 4, T // 2
    mass = torch.zeros((B, T), dtype=torch.float32, device=wl.cache.device)
    torch.cuda.synchronize()   # zero-filled on torch's current stream, used on `stream`
    am = [kvq.make_decode_mass_args(wl.q7[l], mass, k_codes=wl.codes[l, 0], k_scales=wl.scales[l, 0],
                                    v_codes=wl.codes[l, 1], v_scales=wl.scales[l, 1], out=wl.out7[l])
          for l in range(L)]
    mws = torch.empty(int(lib.kvq_decode_mass_workspace_bytes(ctypes.byref(am[0]))), dtype=torch.uint8,
                      device=wl.cache.device)
    for a in am:
        a.base.workspace, a.base.workspace_bytes = mws.data_ptr(), mws.numel()

    def dec_mass():
        for a in am:
            st = lib.kvq_decode_attention_mass(ctypes.byref(a), s)
            if st != kvq.KVQ_OK:
                raise kvq.KvqError("kvq_decode_attention_mass", st)
    ms = timed(dec_mass) / L
    row("decode_int8_mass", ms, keys * 2 * (D + 4) + B * H * D * 6 + keys * 4 * 2 + B * T * 8,
        "7B-shaped layer: INT8 K/V [8, 32, 4096, 128] decode step that also adds its attention mass "
        "(scores written and re-read, [8, 4096] mass updated)")
    kept = torch.empty((B, n_keep), dtype=torch.int32, device=wl.cache.device)
    P = ctypes.c_void_p

    def select():  # direct C-ABI call: the Python wrapper's checks would dominate a 10 us launch
        st = lib.kvq_evict_select(P(mass.data_ptr()), B, T, n_sink, n_keep, P(kept.data_ptr()), s)
        if st != kvq.KVQ_OK:
            raise kvq.KvqError("kvq_evict_select", st)
    ms = timed(select)
    row("evict_select", ms, B * T * 4 + B * n_keep * 4,
        "mass [8, 4096] fp32 -> 4 sinks + top 2044 per batch row (int32 [8, 2048])")
    kdst = torch.empty((2, B, H, n_keep, D), dtype=torch.int8, device=wl.cache.device)
    sdst = torch.empty((2, B, H, n_keep), dtype=torch.float32, device=wl.cache.device)

    garr = (kvq.GatherArray * 4)()
    for t in range(2):
        garr[2 * t] = kvq.GatherArray(wl.codes[0, t].data_ptr(), kdst[t].data_ptr(), T, n_keep, D)
        garr[2 * t + 1] = kvq.GatherArray(wl.scales[0, t].data_ptr(), sdst[t].data_ptr(), T, n_keep, 4)

    def compact():
        st = lib.kvq_gather_rows_multi(garr, 4, B, H, P(kept.data_ptr()), n_keep, s)
        if st != kvq.KVQ_OK:
            raise kvq.KvqError("kvq_gather_rows_multi", st)
    ms = timed(compact)
    row("evict_compact", ms, 2 * 2 * B * H * n_keep * (D + 4) + B * n_keep * 4,
        "7B-shaped layer: INT8 K/V codes + scales [8, 32, 4096] -> the 2048 kept tokens (one launch)")
    del mass, mws, kdst, sdst

    # ---- QJL as the 1-bit residual of group-wise INT4 (groups of 32), GQA cache keys ----
    dev = wl.cache.device
    n_keys = gb * gk * gt
    kshape = (gb, gk, gt)
    rp = torch.empty(kshape + (D // 2,), dtype=torch.uint8, device=dev)
    rs = torch.empty(kshape + (D // 32,), dtype=torch.float32, device=dev)
    rz = torch.empty_like(rs)
    rr = torch.empty(kshape + (D,), dtype=torch.float16, device=dev)
    rw = torch.empty(kshape + (m // 32,), dtype=torch.int32, device=dev)
    rn = torch.empty(kshape, dtype=torch.float16, device=dev)
    enc_args = [P(wl.gcache[0].data_ptr()), n_keys, D, 32, P(wl.S.data_ptr()), m, P(rp.data_ptr()),
                P(rs.data_ptr()), P(rz.data_ptr()), P(rr.data_ptr()), P(rw.data_ptr()), P(rn.data_ptr()), s]

    def res_encode():
        st = lib.kvq_qjl_residual_encode(*enc_args)
        if st != kvq.KVQ_OK:
            raise kvq.KvqError("kvq_qjl_residual_encode", st)
    ms = timed(res_encode)
    # algorithmic: fp16 keys read; INT4 codes, group scales and zeros, the fp16 residual
    # (an output), sign words and norms written (the residual's re-read by the sketch
    # stage is not counted)
    row("qjlres_encode", ms, n_keys * (2 * D + D // 2 + 8 * (D // 32) + 2 * D + m // 8 + 2),
        "GQA cache keys [4, 8, 131072, 128] fp16 -> INT4 (groups of 32) + residual sign sketch (m = 256)")
    ar = kvq.make_decode_qjlres_args(wl.qg, k_packed4=rp, k_scales4=rs, k_zeros4=rz, k_group=32, k_words=rw,
                                     k_norms=rn, sketch=wl.S, v_codes=wl.vcodes, v_scales=wl.vscales,
                                     out=wl.outg)
    rws = torch.empty(int(lib.kvq_decode_qjlres_workspace_bytes(ctypes.byref(ar))), dtype=torch.uint8, device=dev)
    ar.base.workspace, ar.base.workspace_bytes = rws.data_ptr(), rws.numel()

    def dec_res():
        st = lib.kvq_decode_attention_qjlres(ctypes.byref(ar), s)
        if st != kvq.KVQ_OK:
            raise kvq.KvqError("kvq_decode_attention_qjlres", st)
    ms = timed(dec_res)
    row("decode_qjlres", ms, n_keys * (D // 2 + 8 * (D // 32) + m // 8 + 2 + D + 4) + gb * gq * D * (2 + 4) + m * D * 2,
        "GQA [4, 32q/8kv, 131072]: INT4 keys + residual sign sketch (m = 256) + INT8 V, one fused decode step")
    del rp, rs, rz, rr, rw, rn, rws

    if kvq.kvq_device_error() != 0:
        raise RuntimeError("device-side error recorded during the widened rows")
    return out


# ---------------------------------------------------------------------------------
# CPU oracle baseline (bounded sample of the same workload, single thread)
# ---------------------------------------------------------------------------------
class CpuSample:
    """A bounded sample of each row of the step, drawn once (outside any timing), that
    the C oracle is timed on: single-threaded, or with its all-cores build (OpenMP over
    rows, keys or (batch, head) units, identical results)."""

    def __init__(self, scale: float = 1.0):
        import numpy as np

        import oracle
        from kv_cache_quantization_absmax_b200 import inputs

        D, m = 128, GQA["m"]
        self.D, self.m = D, m
        self.n_rows = max(1024, int(131072 * scale))      # quantize / dequantize rows
        self.n_units = max(1, int(8 * scale))             # INT8 decode: units of 4096 tokens
        self.n_keys = max(512, int(16384 * scale))        # QJL encode keys
        self.n_gunits = 16                                # QJL GQA decode: 16 KV units x 4 query heads
        self.n_gtok = max(256, int(2048 * scale))         # tokens per QJL decode unit
        self.x = inputs.lognormal_cache(3, 1, 1, self.n_rows)[0].reshape(self.n_rows, D)
        self.c, self.s = oracle.quantize_int8(self.x)
        T = LLAMA["seq"]
        kk, vv = inputs.lognormal_cache(31, self.n_units, 1, T, n_tensors=2)
        kc, ks = oracle.quantize_int8(kk.reshape(-1, D))
        vc, vs = oracle.quantize_int8(vv.reshape(-1, D))
        shp = (self.n_units, 1, T)
        self.dec8 = dict(k_codes=kc.reshape(shp + (D,)), k_scales=ks.reshape(shp),
                         v_codes=vc.reshape(shp + (D,)), v_scales=vs.reshape(shp))
        self.q8 = inputs.gaussian_queries(32, self.n_units, 1)
        self.S = inputs.sketch_matrix(m, D)
        self.kq = inputs.lognormal_cache(41, 1, 1, self.n_keys)[0].reshape(self.n_keys, D)
        # the estimator's cost does not depend on the bit values: seeded random sign
        # words and norms stand in for encoded keys
        rng = np.random.default_rng(51)
        gs = (self.n_gunits, 1, self.n_gtok)
        w = rng.integers(0, 2 ** 32, gs + (m // 32,), dtype=np.uint32)
        n = (np.abs(rng.standard_normal(gs)) * 11 + 1).astype(np.float16)
        vg = inputs.lognormal_cache(52, self.n_gunits, 1, self.n_gtok)[0]
        vgc, vgs = oracle.quantize_int8(vg.reshape(-1, D))
        self.decq = dict(k_words=w, k_norms=n, S=self.S, v_codes=vgc.reshape(gs + (D,)), v_scales=vgs.reshape(gs))
        self.qg = inputs.gaussian_queries(53, self.n_gunits, 4)
        self.np = np
        self.description = (
            f"C oracle on a bounded sample of each row: quantize/dequantize "
            f"{self.n_rows} rows x 128 fp16, INT8 decode {self.n_units} units x {T} tokens, QJL "
            f"encode {self.n_keys} keys, QJL GQA decode {self.n_gunits} KV units x {self.n_gtok} tokens x 4 "
            f"query heads; each row's GB/s is applied to that row's bytes in the full step")

    def rates(self, all_cores: bool = False):
        """GB/s of each row of the step on this sample; returns (rates, threads used)."""
        import oracle

        D, m = self.D, self.m
        r = {}

        def timed(fn):
            t0 = time.perf_counter()
            fn()
            return time.perf_counter() - t0

        oracle.use_all_cores(all_cores)
        try:
            threads = oracle.threads()
            dt = timed(lambda: oracle.quantize_int8(self.x))
            r["quantize_cache"] = r["quantize_v"] = self.n_rows * (3 * D + 4) / dt / 1e9
            dt = timed(lambda: oracle.dequantize_int8(self.c, self.s, self.np.float16))
            r["dequantize_cache"] = self.n_rows * (3 * D + 4) / dt / 1e9
            dt = timed(lambda: oracle.decode_attention(self.q8, **self.dec8))
            r["decode_int8"] = self.n_units * LLAMA["seq"] * 2 * (D + 4) / dt / 1e9
            dt = timed(lambda: oracle.qjl_encode(self.kq, self.S))
            r["qjl_encode"] = self.n_keys * (2 * D + m // 8 + 2) / dt / 1e9
            dt = timed(lambda: oracle.decode_attention(self.qg, **self.decq))
            r["decode_qjl"] = self.n_gunits * self.n_gtok * (m // 8 + 2 + D + 4) / dt / 1e9
        finally:
            oracle.use_all_cores(False)
        return r, threads


def cpu_next_rates():
    """The single-threaded C oracle on a bounded sample of each widened row (a few seconds
    in all), as GB/s by the same byte counts per unit as the GPU rows in `next_rows`."""
    import numpy as np

    import oracle
    from kv_cache_quantization_absmax_b200 import inputs

    D, m, T = 128, GQA["m"], LLAMA["seq"]
    r = {}

    def timed(fn):
        t0 = time.perf_counter()
        fn()
        return time.perf_counter() - t0

    # INT8 cache of 2 units x 4096 tokens; appended token at T - 1
    k, v = inputs.lognormal_cache(61, 2, 1, T, n_tensors=2)
    kc, ks = oracle.quantize_int8(k.reshape(-1, D))
    vc, vs = oracle.quantize_int8(v.reshape(-1, D))
    shp = (2, 1, T)
    c8 = dict(k_codes=kc.reshape(shp + (D,)), k_scales=ks.reshape(shp), v_codes=vc.reshape(shp + (D,)),
              v_scales=vs.reshape(shp))
    q = inputs.gaussian_queries(62, 2, 1)
    kn = k[:, :, T - 1].copy()
    vn = v[:, :, T - 1].copy()
    dt = timed(lambda: oracle.decode_append(q, kn, vn, T=T - 1, **c8))
    r["append_int8"] = 2 * T * 2 * (D + 4) / dt / 1e9
    dt = timed(lambda: (oracle.decode_attention(q, **c8), oracle.attention_mass(q, **c8)))
    r["decode_int8_mass"] = 2 * T * (2 * (D + 4) + 12) / dt / 1e9
    mass = oracle.attention_mass(q, **c8).astype(np.float32)
    dt = timed(lambda: oracle.evict_select(mass, 4, T // 2))
    r["evict_select"] = 2 * (T * 4 + (T // 2) * 4) / dt / 1e9
    kept = oracle.evict_select(mass, 4, T // 2)
    cache = kc.reshape(2, 1, T, D)
    dt = timed(lambda: oracle.gather_rows(cache, kept))
    r["evict_compact"] = 2 * (T // 2) * D * 2 / dt / 1e9
    # group-wise INT4 and channel-wise INT8 on 65536 rows of 128 fp16
    x = inputs.lognormal_cache(63, 1, 16, 4096)[0].reshape(-1, D)
    n = x.shape[0]
    dt = timed(lambda: oracle.quantize_int4_group(x, 32))
    r["int4_quantize"] = n * (D * 2.5 + 32) / dt / 1e9
    p4, s4, z4 = oracle.quantize_int4_group(x, 32)
    dt = timed(lambda: oracle.dequantize_int4_group(p4, s4, z4, 32, np.float16))
    r["int4_dequantize"] = n * (D * 2.5 + 32) / dt / 1e9
    blocks = x.reshape(16, 4096, D)
    dt = timed(lambda: oracle.quantize_int8_channelwise(blocks))
    r["int8_channelwise_quantize"] = n * D * 3 / dt / 1e9
    cwc, cws = oracle.quantize_int8_channelwise(blocks)
    dt = timed(lambda: oracle.dequantize_int8_channelwise(cwc, cws, np.float16))
    r["int8_channelwise_dequantize"] = n * D * 3 / dt / 1e9
    pv, sv, zv = oracle.quantize_int4_group(v.reshape(-1, D), 32)
    v4 = (pv.reshape(shp + (D // 2,)), sv.reshape(shp + (4,)), zv.reshape(shp + (4,)), 32)
    dt = timed(lambda: oracle.decode_attention(q, k_codes=c8["k_codes"], k_scales=c8["k_scales"], v4=v4))
    r["decode_int8k_int4v"] = 2 * T * (D + 4 + D // 2 + 32) / dt / 1e9
    # QJL-family rows on 8192 keys of one GQA unit (4 query heads)
    gt = 8192
    kg, vg = inputs.lognormal_cache(64, 1, 1, gt, n_tensors=2)
    S = inputs.sketch_matrix(m, D)
    w, nr = oracle.qjl_encode(kg.reshape(-1, D), S)
    vgc, vgs = oracle.quantize_int8(vg.reshape(-1, D))
    gs = (1, 1, gt)
    cq = dict(k_words=w.reshape(gs + (m // 32,)), k_norms=nr.reshape(gs), S=S, v_codes=vgc.reshape(gs + (D,)),
              v_scales=vgs.reshape(gs))
    qg = inputs.gaussian_queries(65, 1, 4)
    dt = timed(lambda: oracle.decode_append(qg, kg[:, :, gt - 1].copy(), vg[:, :, gt - 1].copy(), T=gt - 1, **cq))
    r["append_qjl"] = gt * (m // 8 + 2 + D + 4) / dt / 1e9
    dt = timed(lambda: oracle.qjl_residual_encode(kg.reshape(-1, D), 32, S))
    r["qjlres_encode"] = gt * (2 * D + D // 2 + 32 + 2 * D + m // 8 + 2) / dt / 1e9
    e = oracle.qjl_residual_encode(kg.reshape(-1, D), 32, S)
    cr = dict(k4=(e["packed"].reshape(gs + (D // 2,)), e["scales"].reshape(gs + (4,)), e["zeros"].reshape(gs + (4,)), 32),
              k_words=e["words"].reshape(gs + (m // 32,)), k_norms=e["rnorms"].reshape(gs), S=S,
              v_codes=cq["v_codes"], v_scales=cq["v_scales"])
    dt = timed(lambda: oracle.decode_attention(qg, **cr))
    r["decode_qjlres"] = gt * (D // 2 + 32 + m // 8 + 2 + D + 4) / dt / 1e9
    return r


def cpu_step_gbs(rates):
    rb = row_bytes()
    t = sum(rb[k] / 1e9 / rates[k] for k in rb)
    return sum(rb.values()) / 1e9 / t, t


# ---------------------------------------------------------------------------------
# Arms
# ---------------------------------------------------------------------------------
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    smp = CpuSample(args.ref_scale)
    for _ in range(args.warmup):
        smp.rates(all_cores=True)
    times, per_step = [], []
    threads = 1
    for _ in range(args.steps):
        t0 = time.perf_counter()
        rates, threads = smp.rates(all_cores=True)
        times.append(time.perf_counter() - t0)
        per_step.append(cpu_step_gbs(rates))
    value = statistics.median(v for v, _ in per_step)
    step_s = statistics.median(t for _, t in per_step)
    sample = smp.description
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(step_s * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": workload_config(),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads,
                         "host_cores": os.cpu_count(), "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "sample_wall_s_per_step": round(statistics.median(times), 3),
        "note": "the CPU oracle as it stands, its all-cores build on the host's cores; ms_per_step "
                "is the full step extrapolated from per-row sample rates",
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config():
    return {
        "workload": "llama7b_kv_cache_int8 (32L x {K,V} x [8,32,4096,128] fp16: quantize, 32 decode "
                    "steps, dequantize) + gqa_long_context_qjl ([4, 32q/8kv, 131072, 128] fp16: QJL "
                    "encode m=256, INT8 V, fused GQA decode)",
        "llama_cache": dict(LLAMA), "gqa_cache": dict(GQA),
        "l2": "inputs larger than L2 (about 47 GB resident per GPU), no flush",
        "parallelism": "weak-scaled replicas, one per GPU",
    }


def run_gpu(args):
    import torch
    import torch.distributed as dist

    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", device_id=torch.device("cuda", local),
                                timeout=__import__("datetime").timedelta(seconds=300))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    from kv_cache_quantization_absmax_b200 import kvq
    wl = Workload(dev)
    stream = torch.cuda.Stream(device=dev)
    rb = row_bytes()
    step_bytes = float(sum(rb.values()))

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            wl.step(stream)
    torch.cuda.synchronize()
    if kvq.kvq_device_error() != 0:
        raise RuntimeError("device-side error recorded during warm-up")

    # ---- device-timed region ----
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(7)] for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(gpu_id_for(dev.index))
    barrier()
    sampler.start()
    time.sleep(0.3)
    t_start.record(stream)
    with torch.cuda.stream(stream):
        for k in range(args.steps):
            wl.step(stream, evs[k])
    t_end.record(stream)
    barrier()
    clocks = sampler.stop()
    total_ms = t_start.elapsed_time(t_end)
    total_ms_max = max_over_ranks(total_ms)
    ms_step = total_ms_max / args.steps
    row_ms = {n: statistics.mean(evs[k][i].elapsed_time(evs[k][i + 1]) for k in range(args.steps))
              for i, n in enumerate(ROW_NAMES)}
    if kvq.kvq_device_error() != 0:
        raise RuntimeError("device-side error recorded during the timed region")

    # ---- end to end: pinned host inputs -> device, step, outputs -> host ----
    e2e = None
    try:
        hb = wl.host_buffers()
        h2d = sum(hb[n].numel() * hb[n].element_size() for n in ("cache", "q7", "gcache", "qg"))
        d2h = sum(hb[n].numel() * hb[n].element_size() for n in ("out7", "outg"))
        e_steps = max(1, min(args.steps, args.e2e_steps))
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        with torch.cuda.stream(stream):
            for _ in range(e_steps):
                wl.cache.copy_(hb["cache"], non_blocking=True)
                wl.q7.copy_(hb["q7"], non_blocking=True)
                wl.gcache.copy_(hb["gcache"], non_blocking=True)
                wl.qg.copy_(hb["qg"], non_blocking=True)
                wl.step(stream)
                hb["out7"].copy_(wl.out7, non_blocking=True)
                hb["outg"].copy_(wl.outg, non_blocking=True)
        e1.record(stream)
        barrier()
        e_ms = max_over_ranks(e0.elapsed_time(e1)) / e_steps
        e2e = {"value": round(aggregate(step_bytes, world, e_ms, 1), 2), "unit": "GB/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": round(e_ms, 3), "steps": e_steps}
        del hb
    except RuntimeError as exc:  # pinned allocation can fail on a small host
        e2e = {"value": None, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0,
               "unavailable": str(exc)[:200]}

    next_rows = measure_next_rows(wl, stream)
    small = measure_small_configs(stream)
    sweep = measure_sweep(stream) if not args.no_sweep else None
    barrier()

    if rank == 0:
        peak, peak_kind = load_peaks()
        for v in next_rows.values():
            v["frac_hbm"] = round(v["GB/s"] / peak, 4)
        dom = max(("quantize_cache", "dequantize_cache"), key=lambda n: row_ms[n])
        achieved = rb[dom] / (row_ms[dom] * 1e-3) / 1e9
        traffic = load_traffic(dom)
        dec_ms = row_ms["decode_int8"] + row_ms["decode_qjl"]
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            smp = CpuSample(args.cpu_scale)
            r1, _ = smp.rates(all_cores=False)
            rn, threads = smp.rates(all_cores=True)
            v1, _ = cpu_step_gbs(r1)
            vn, _ = cpu_step_gbs(rn)
            cpu = {"value": round(vn, 4), "unit": "GB/s", "cores": threads, "host_cores": os.cpu_count(),
                   "kind": "oracle", "sample": smp.description + "; all-cores build of the oracle",
                   "single_thread": {"value": round(v1, 4), "unit": "GB/s", "cores": 1}}
            # the widened rows: the single-threaded oracle on small samples of each
            for k, g in cpu_next_rates().items():
                if k in next_rows:
                    next_rows[k]["cpu_oracle_GBps"] = round(g, 5)
        fields = ["ms", "GB/s", "frac_hbm", "cpu_oracle_GBps"]
        # the per-row figures come last, compactly, so that a reader of the line's tail sees them
        line = {
            "metric": METRIC, "value": round(aggregate(step_bytes, world, ms_step, args.steps), 2),
            "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "storage": "fp16 in; int8 codes + fp32 scales; "
            "1-bit sign words + fp16 norms", "data": "synthetic", "config": workload_config(),
            "sweep": sweep,
            "e2e": e2e,
            "gpu_launches": LAUNCHES_PER_STEP * args.steps,
            "clocks": clocks,
            "cpu_baseline": cpu,
            "roofline": {"bound": "hbm", "kernel": dom, "achieved": round(achieved, 1),
                         "peak": peak, "unit": "GB/s", "frac": round(achieved / peak, 4),
                         "traffic": traffic, "peak_source": f"{peak_kind} hbm_gbs"},
            "frac_hbm_step": round(aggregate(step_bytes, 1, ms_step, 1) / peak, 4),
            "decode_keys_per_s": round(decode_keys() * world / (dec_ms * 1e-3), 1),
            "one_layer": small["one_layer"],
            "key_sketch": small["key_sketch"],
            "row_fields": fields,
            "next_rows": {n: [v.get(f) for f in fields] for n, v in next_rows.items()},
            "rows": {n: [round(row_ms[n], 4), round(rb[n] / (row_ms[n] * 1e-3) / 1e9, 1),
                         round(rb[n] / (row_ms[n] * 1e-3) / 1e9 / peak, 4)] for n in ROW_NAMES},
        }
        if cpu is None:
            del line["cpu_baseline"]
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def load_traffic(kernel_row: str):
    """DRAM bytes per launch of the dominant kernel from the committed ncu summary, if the
    kernel's source file is unchanged since the counters were taken (else null)."""
    import hashlib

    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            tr = json.load(f)
        h = hashlib.sha256()
        for rel in tr["kernel_sources"]:
            with open(os.path.join(ROOT, rel), "rb") as f:
                h.update(f.read())
        if tr.get("sources_hash") != h.hexdigest():
            return None
        v = tr.get("rows", {}).get(kernel_row)
        return None if v is None else float(v)
    except Exception:
        return None


def run_profile_case(case: str, reps: int = 3, layers: int = 1):
    """Small single-kernel cases for ncu captures (inputs larger than L2, a few GB at most).
    quantize / dequantize take `layers` layers of the 7B-shaped cache (K and V each)."""
    import torch
    from kv_cache_quantization_absmax_b200 import inputs, kvq

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(0)
    B, H, T, D = LLAMA["batch"], LLAMA["heads"], LLAMA["seq"], LLAMA["dim"]
    if case in ("quantize", "dequantize", "decode_int8", "decode_int8_cuda_cores"):
        shape = (2 * (layers if not case.startswith("decode_int8") else 1), B, H, T, D)
        kv = inputs.lognormal_cache_device(3, shape, n_sigma_dims=(0, 2, 4), device=dev)
        codes, scales = kvq.kvq_quantize_int8(kv)
        out = torch.empty_like(kv)
        q = inputs.gaussian_queries_device(30, (B, H, D), dev)
        for _ in range(reps):
            if case == "quantize":
                kvq.kvq_quantize_int8(kv, codes, scales)
            elif case == "dequantize":
                kvq.kvq_dequantize_int8(codes, scales, out=out)
            else:
                kvq.kvq_decode_attention(q, k_codes=codes[0], k_scales=scales[0], v_codes=codes[1],
                                         v_scales=scales[1],
                                         flags=kvq.KVQ_DECODE_CUDA_CORES if case.endswith("cores") else 0)
    elif case in ("qjl_encode", "decode_qjl"):
        gb, gq, gk, gt, m = (GQA[k] for k in ("batch", "q_heads", "kv_heads", "seq", "m"))
        if case == "qjl_encode":
            gb = 1
        kv = inputs.lognormal_cache_device(5, (2, gb, gk, gt, D), n_sigma_dims=(0, 2, 4), device=dev)
        S = torch.from_numpy(inputs.sketch_matrix(m, D)).to(dev)
        words, norms = kvq.kvq_qjl_encode(kv[0], S)
        vc, vs = kvq.kvq_quantize_int8(kv[1])
        q = inputs.gaussian_queries_device(50, (gb, gq, D), dev)
        for _ in range(reps):
            if case == "qjl_encode":
                kvq.kvq_qjl_encode(kv[0], S, words, norms)
            else:
                kvq.kvq_decode_attention(q, k_words=words, k_norms=norms, sketch=S, v_codes=vc,
                                         v_scales=vs)
    elif case in ("int4_quantize", "int4_dequantize", "cw_quantize", "cw_dequantize", "decode_int4v"):
        kv = inputs.lognormal_cache_device(3, (2, B, H, T, D), n_sigma_dims=(0, 2, 4), device=dev)
        p4, s4, z4 = kvq.kvq_quantize_int4(kv, 32)
        cwc, cws = kvq.kvq_quantize_int8_channelwise(kv)
        out = torch.empty_like(kv)
        kc, ks = kvq.kvq_quantize_int8(kv[0])
        q = inputs.gaussian_queries_device(30, (B, H, D), dev)
        for _ in range(reps):
            if case == "int4_quantize":
                kvq.kvq_quantize_int4(kv, 32, p4, s4, z4)
            elif case == "int4_dequantize":
                kvq.kvq_dequantize_int4(p4, s4, z4, 32, out=out)
            elif case == "cw_quantize":
                kvq.kvq_quantize_int8_channelwise(kv, cwc, cws)
            elif case == "cw_dequantize":
                kvq.kvq_dequantize_int8_channelwise(cwc, cws, out=out)
            else:
                kvq.kvq_decode_attention_int4v(q, k_codes=kc, k_scales=ks, v_packed=p4[1], v_scales4=s4[1],
                                               v_zeros4=z4[1], v_group=32)
    elif case in ("qjlres_encode", "decode_qjlres"):
        gb, gq, gk, gt, m = (GQA[k] for k in ("batch", "q_heads", "kv_heads", "seq", "m"))
        if case == "qjlres_encode":
            gb = 1
        kv = inputs.lognormal_cache_device(5, (2, gb, gk, gt, D), n_sigma_dims=(0, 2, 4), device=dev)
        S = torch.from_numpy(inputs.sketch_matrix(m, D)).to(dev)
        e = kvq.kvq_qjl_residual_encode(kv[0], 32, S)
        vc, vs = kvq.kvq_quantize_int8(kv[1])
        q = inputs.gaussian_queries_device(50, (gb, gq, D), dev)
        for _ in range(reps):
            if case == "qjlres_encode":
                kvq.kvq_qjl_residual_encode(kv[0], 32, S)
            else:
                kvq.kvq_decode_attention_qjlres(q, k_packed4=e["packed"], k_scales4=e["scales"],
                                                k_zeros4=e["zeros"], k_group=32, k_words=e["words"],
                                                k_norms=e["rnorms"], sketch=S, v_codes=vc, v_scales=vs)
    elif case in ("decode_mass", "evict_select", "evict_compact"):
        kv = inputs.lognormal_cache_device(3, (2, B, H, T, D), n_sigma_dims=(0, 2, 4), device=dev)
        codes, scales = kvq.kvq_quantize_int8(kv)
        del kv
        q = inputs.gaussian_queries_device(30, (B, H, D), dev)
        mass = torch.zeros((B, T), dtype=torch.float32, device=dev)
        kvq.kvq_decode_attention_mass(q, mass, k_codes=codes[0], k_scales=scales[0], v_codes=codes[1],
                                      v_scales=scales[1])
        kept = kvq.kvq_evict_select(mass, 4, T // 2)
        dst = torch.empty((B, H, T // 2, D), dtype=torch.int8, device=dev)
        for _ in range(reps):
            if case == "decode_mass":
                kvq.kvq_decode_attention_mass(q, mass, k_codes=codes[0], k_scales=scales[0], v_codes=codes[1],
                                              v_scales=scales[1])
            elif case == "evict_select":
                kvq.kvq_evict_select(mass, 4, T // 2, kept=kept)
            else:
                kvq.kvq_gather_rows(codes[0], kept, dst=dst)
    else:
        raise SystemExit(f"unknown profile case {case}")
    torch.cuda.synchronize()
    if kvq.kvq_device_error() != 0:
        raise RuntimeError("device-side error recorded")
    return 0


def main(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["kvq", "reference"], default="kvq")
    p.add_argument("--e2e-steps", type=int, default=3)
    p.add_argument("--ref-scale", type=float, default=2.0,
                   help="size of the oracle's per-step sample in the reference arm")
    p.add_argument("--cpu-scale", type=float, default=8.0,
                   help="size of the oracle sample for the cpu_baseline key")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-sweep", action="store_true", help="skip the quantize/dequantize throughput sweep")
    p.add_argument("--profile-case", default=None,
                   help="run one small single-kernel case (quantize, dequantize, decode_int8, "
                        "decode_int8_cuda_cores, qjl_encode, decode_qjl, int4_quantize, int4_dequantize, cw_quantize, "
                        "cw_dequantize, decode_int4v, decode_mass, evict_select, evict_compact, qjlres_encode, "
                        "decode_qjlres) for an ncu "
                        "capture, then exit")
    p.add_argument("--profile-layers", type=int, default=1,
                   help="layers of the 7B-shaped cache in the quantize / dequantize profile cases")
    args = p.parse_args(argv)
    if args.profile_case:
        return run_profile_case(args.profile_case, layers=args.profile_layers)
    if args.warmup < 3 and args.impl == "kvq":
        print("note: warm-up raised to 3 steps", file=sys.stderr)
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
