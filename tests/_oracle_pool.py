"""Oracle work on whole KV units, run in a pool of spawned processes by the full-size GPU
tests (numpy and the oracle only: a spawned worker never touches the GPU)."""
import concurrent.futures as cf
import multiprocessing as mp
import os

import numpy as np


def qjl_unit(k16, v16, q16, S, sm_scale=0.0):
    """One KV unit with QJL keys and INT8 values, from its fp16 keys / values [T, D] and the
    unit's fp16 queries [G, D]: the oracle's sign words and norms, value codes and scales,
    and its decode (raw scores [G, T] and output [G, D])."""
    import oracle
    T, D = k16.shape
    w, n = oracle.qjl_encode(k16, S)
    vc, vs = oracle.quantize_int8(v16)
    r = oracle.decode_attention(q16[None], k_words=w[None, None], k_norms=n[None, None], S=S,
                                v_codes=vc[None, None], v_scales=vs[None, None], sm_scale=sm_scale,
                                want_scores=True)
    return dict(words=w, norms=n, v_codes=vc, v_scales=vs, scores=r["scores"][0], out=r["out"][0])


def qjlres_unit(k16, v16, q16, S, group, sm_scale=0.0):
    """One KV unit with residual keys (group-wise INT4 + the residual's sign sketch) and
    INT8 values: the oracle's encode of both (with the fp16 residual r) and its decode
    (scores [G, T], out [G, D])."""
    import oracle
    T, D = k16.shape
    e = oracle.qjl_residual_encode(k16, group, S, want_r=True)
    vc, vs = oracle.quantize_int8(v16)
    ng = D // group
    k4 = (e["packed"][None, None], e["scales"].reshape(1, 1, T, ng), e["zeros"].reshape(1, 1, T, ng), group)
    r = oracle.decode_attention(q16[None], k4=k4, k_words=e["words"][None, None],
                                k_norms=e["rnorms"][None, None], S=S, v_codes=vc[None, None],
                                v_scales=vs[None, None], sm_scale=sm_scale, want_scores=True)
    e.update(v_codes=vc, v_scales=vs, scores=r["scores"][0], out=r["out"][0])
    return e


def run_units(fn, jobs):
    """fn(*job) for every job, in spawned worker processes; results in job order."""
    n = max(1, min(len(jobs), os.cpu_count() or 1, 16))
    with cf.ProcessPoolExecutor(max_workers=n, mp_context=mp.get_context("spawn")) as ex:
        return list(ex.map(fn, *zip(*jobs)))
