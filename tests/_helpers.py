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
