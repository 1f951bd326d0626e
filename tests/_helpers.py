"""Shared test helpers (no arithmetic of the method lives here)."""
import numpy as np


def to_np(t):
    return t.detach().cpu().numpy()


def words_u32(t):
    """uint32 view of a words tensor stored as int32."""
    return to_np(t).view(np.uint32)


def bit_mismatch_outside_band(gpu_words, ora_words, u, norms64, band=1e-4):
    """Return the number of sign bits that differ where the oracle's |u_i| >= band*||k||.

    gpu_words/ora_words: uint32 [n, m/32]; u: fp64 [n, m]; norms64: fp64 [n] (||k||)."""
    n, nw = ora_words.shape
    diff = gpu_words ^ ora_words
    bits = ((diff[:, :, None] >> np.arange(32, dtype=np.uint32)) & 1).reshape(n, nw * 32).astype(bool)
    allowed = np.abs(u) < band * norms64[:, None]
    return int(np.count_nonzero(bits & ~allowed)), int(np.count_nonzero(bits))


def score_tolerance(ref, norms, v, m, rel=1e-4):
    """Estimator-score tolerance: rel * max(|ref|, c * ||k|| * ||S q||_2), c = sqrt(pi/2)/m.

    The second term is the score's natural scale (its standard deviation over sign
    patterns), so scores that cancel to near zero are held to rel times that scale."""
    c = np.sqrt(np.pi / 2) / m
    scale = c * norms.astype(np.float64) * np.linalg.norm(v.astype(np.float64), axis=-1)[..., None]
    return rel * np.maximum(np.abs(ref.astype(np.float64)), scale)


# ---------------------------------------------------------------------------------------
# Decode outputs: a bound derived from the arithmetic of the GPU kernels
# ---------------------------------------------------------------------------------------
# The spec line for a decode output is 2e-3 max-abs against the oracle.  At long
# context a typical output is a few 1e-3 and losing a whole 128-token chunk moves it by
# less than that, so every decode test also holds each output element to the error the
# kernels' arithmetic can produce, against the oracle's fp64 softmax-weighted sum over the
# oracle's own scores (oracle.decode_from_scores):
#
#   |out_gpu - out_ref| <= e^(2 Dm) [ sum_t P_t (rho_t + expm1(delta_t)) |v_t - out_ref| ]
#                          + (n_chain + 66) 2^-24 (sum_t P_t |v_t| + |out_ref|)
#                          + [tensor-core value pass] 2^-23 * 128 * 127 * smax + 2^-18 |out_ref|
#
#  * P_t, out_ref: fp64 softmax and weighted sum of the oracle's scores;
#  * delta_t = sigma |s_gpu,t - s_ref,t|: the GPU's own score deviation (itself held to the
#    score tolerance by the caller), which moves p_t by a factor e^(+-delta_t);
#  * rho_t: relative error of the GPU's weight of token t: the fp32 logit (the scale
#    constant, the product and the subtraction of the running max: ln2 2^-24 (3|lg_t| +
#    |lg_t - M|), lg in the log2 domain) and the hardware 2^x, taken as 2^-21 relative per
#    use, applied once to the token and once per later rescale of its accumulator (at most
#    one per pipeline step of 64 tokens in a CTA range, plus the merges);
#  * n_chain: the longest sequential fp32 accumulation in any kernel: a CTA range of W
#    tokens is split over at least 16 lane groups / warps / chunks, then the lane, warp and
#    range merges (W <= ceil(B Hkv T nsub / SMs), rounded up to 64);
#  * the tensor-core value pass rounds each weight of a 128-token chunk (or 32-token
#    slice) to an integer multiple of 2^-E with smax 2^E in [2^23, 2^24), after rounding
#    the product p * s to fp32 (below 2^-23 smax |c| per token, |c| <= 127), and each
#    token's share of the softmax sum to 2^-24 (at most 2^-25 per token, 2^-18 relative
#    for a chunk, whose sum is at least 1); both are relative to the chunk's maximum
#    weight 1, so their share of the output is at most the largest chunk's
#    (tests/test_fixedpoint_cpu.py checks these roundings).
# Dm = max_t (delta_t + rho_t).  Every term is a worst case, not an estimate.

EX2_REL = 2.0 ** -21


def decode_chain(batch, n_kv_heads, seq_len, n_q_heads, n_sm, qjl=False):
    """(n_chain, n_rescale) for the bound above.  A CTA range holds at most
    W = ceil(units * T * nsub / SMs) tokens (rounded up to 64), nsub = head subgroups per
    KV head (G / 8 for INT8 keys, G / 4 for QJL keys, at least 1).  Within a range:
      INT8 keys: on the CUDA cores 32 lane groups (16 from four heads per CTA up) each
                 sum their own tokens and rescale at most once per pipeline stage (64 or 128
                 tokens); on the tensor cores one running state per range takes one exact
                 32-token slice sum at a time (one rescale per slice); the bound takes the
                 larger of the two;
      QJL keys:  32 (warp, token parity) chains on the CUDA cores, or one running state per
                 128-token chunk on the tensor cores; at most one rescale per 128 tokens."""
    G = n_q_heads // n_kv_heads
    cap = 4 if qjl else 8
    g = cap
    while g > 1 and G % g:
        g //= 2
    nsub = G // g
    total = batch * n_kv_heads * seq_len
    W = -(-total * nsub // n_sm)
    W = -(-W // 64) * 64
    if qjl:
        groups, stage = 32, 128
    else:
        groups, stage = 16, 32
    n_chain = W // groups + 64 + (-(-seq_len // W)) + 2
    n_rescale = W // stage + 8
    return n_chain, n_rescale


def decode_out_bound(out_ref, p, vals, s_gpu, s_ref, sigma, n_chain, n_rescale, tc_smax=None, vabs=None,
                     chunk=16384):
    """Per-element bound (see above) for one KV unit: out_ref [H, D] fp64, p [H, T] fp64,
    vals [T, D] fp64 (the unit's dequantized values), s_gpu / s_ref [H, T] raw scores,
    sigma the softmax scale; tc_smax: the unit's largest value scale when the tensor-core
    value pass may run (else None); vabs [T, D]: the magnitudes the kernel accumulates
    when it sums a value in parts (INT4 values: |c s| + |z|), else |vals|.
    Returns [H, D]."""
    s_gpu = np.asarray(s_gpu, np.float64)
    s_ref = np.asarray(s_ref, np.float64)
    delta = sigma * np.abs(s_gpu - s_ref)
    lg = s_gpu * sigma * 1.4426950408889634
    M = lg.max(axis=-1, keepdims=True)
    rho = np.log(2.0) * 2.0 ** -24 * (3 * np.abs(lg) + np.abs(lg - M)) + (n_rescale + 2) * EX2_REL
    w = p * (rho + np.expm1(delta))                                   # [H, T]
    Ew = np.zeros_like(out_ref)
    for t0 in range(0, vals.shape[0], chunk):
        v = vals[t0:t0 + chunk]                                        # [t, D]
        for h in range(out_ref.shape[0]):
            Ew[h] += w[h, t0:t0 + chunk] @ np.abs(v - out_ref[h][None, :])
    Ew *= np.exp(2 * float((delta + rho).max()))
    acc = (n_chain + 66) * 2.0 ** -24 * (p @ (np.abs(vals) if vabs is None else vabs) + np.abs(out_ref))
    b = Ew + acc + 1e-30
    if tc_smax is not None:
        b += 2.0 ** -23 * 128 * 127 * float(tc_smax) + 2.0 ** -18 * np.abs(out_ref)
    return b


def check_decode_unit(out_gpu, s_gpu, s_ref, vals, sigma, n_chain, n_rescale, tc_smax=None, vabs=None):
    """Assert the bound for one KV unit: out_gpu [H, D], s_gpu / s_ref [H, T], vals [T, D].
    The reference is the oracle's fp64 softmax-weighted sum of s_ref.  Returns
    max(err / bound)."""
    import oracle
    s_ref = np.asarray(s_ref, np.float64)
    out64, p = oracle.decode_from_scores(s_ref[None], np.asarray(vals, np.float64)[None, None],
                                         sm_scale=sigma)
    ref, p = out64[0], p[0]
    bound = decode_out_bound(ref, p, np.asarray(vals, np.float64), s_gpu, s_ref, sigma, n_chain,
                             n_rescale, tc_smax, None if vabs is None else np.asarray(vabs, np.float64))
    err = np.abs(np.asarray(out_gpu, np.float64) - ref)
    ratio = float((err / bound).max())
    assert np.all(err <= bound), f"decode output off by {ratio:.3g} x its arithmetic bound"
    return ratio


def sm_count():
    import torch
    return torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count


def softmax_scale(sm_scale=0.0, head_dim=128):
    """The decode's softmax scale: sm_scale, or the fp32 value of 1/sqrt(head_dim)."""
    return float(sm_scale) if sm_scale else float(np.float32(1.0) / np.sqrt(np.float32(head_dim)))


def check_decode_bound(out_gpu, s_gpu, s_ref, vals, *, qjl, v_scales=None, sm_scale=0.0, n_sm=None, vabs=None):
    """check_decode_unit for every (batch, KV head) of a decode step: out_gpu [B, Hq, D],
    s_gpu / s_ref [B, Hq, T] raw scores, vals [B, Hkv, T, D] dequantized values (fp32 or
    fp64); v_scales [B, Hkv, T] when the tensor-core value pass may run (QJL keys; for
    INT8 values without it, the unit's largest value scale is max |vals| / 127, which the
    largest code of absmax rows makes exact); vabs [B, Hkv, T, D] as for decode_out_bound
    (INT4 values, which never take the tensor-core pass).  Returns the largest err / bound."""
    out_gpu, s_gpu, s_ref = (np.asarray(a) for a in (out_gpu, s_gpu, s_ref))
    B, Hq, T = s_ref.shape
    Hkv = vals.shape[1]
    G = Hq // Hkv
    n_chain, n_rescale = decode_chain(B, Hkv, T, Hq, n_sm or sm_count(), qjl=qjl)
    sigma = softmax_scale(sm_scale, vals.shape[-1])
    worst = 0.0
    for b in range(B):
        for g in range(Hkv):
            hs = slice(g * G, (g + 1) * G)
            if v_scales is not None:
                smax = float(np.asarray(v_scales)[b, g].max())
            elif not qjl and vabs is None:
                smax = float(np.abs(np.asarray(vals[b, g])).max()) / 127.0
            else:
                smax = None
            worst = max(worst, check_decode_unit(out_gpu[b, hs], s_gpu[b, hs], s_ref[b, hs],
                                                 np.asarray(vals[b, g], np.float64), sigma, n_chain,
                                                 n_rescale, smax, None if vabs is None else vabs[b, g]))
    return worst
