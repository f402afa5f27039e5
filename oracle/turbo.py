"""TurboQuant-style vector quantizer and attention, float64.  Test
infrastructure only.

What the pages fix:
* a random orthogonal rotation makes the coordinates of a vector behave like
  independent Gaussians and spreads outlier channels (zubnet.ai survey,
  "Famille deux ..."; "La compression du cache KV est une decision
  d'infrastructure ...", section "TurboQuant est le choix de portabilite ...";
  "Quantification du KV-Cache ...", "TurboQuant : les cinq innovations"
  item 1, where the inverse rotation does not amplify the error because it is
  orthogonal);
* each rotated coordinate goes through a precomputed scalar quantizer, a
  Lloyd-Max codebook for a Gaussian fixed at deployment (same page, item 2);
* a 1-bit Johnson-Lindenstrauss (QJL) transform of the residual corrects inner
  products (survey and the encorp.ai section above).

Readings where the pages are silent (the workload fixes 3-bit codes, a QJL
sketch of m = 128 Gaussian rows on keys only, per-vector fp16 norms):
* x -> n = ||x||, u = x / n (u = 0 when n = 0), y = Pi u;
* code of y_c = number of thresholds strictly below y_c (a tie goes to the lower
  index); the 8 levels are the Lloyd-Max levels for N(0, 1) scaled by 1/sqrt(d)
  (the law of a coordinate of a rotated unit vector) and rounded to fp16, the
  form the table is deployed in; thresholds are midpoints of adjacent levels;
* keys: e = y - c_hat (residual in rotated coordinates), gamma = n ||e||, sign
  bit i = 1 iff (S e)_i >= 0; stored n and gamma are fp16;
* score_t = scale (n_t <Pi q, c_hat_t> + gamma_t sqrt(pi/2)/m <S Pi q, sign_t>),
  sign_t in {-1, +1}: E[g sign(g')] for correlated standard normals makes the
  sketch term unbiased for n <Pi q, e> (pinned by Monte Carlo);
* values: v_hat = n Pi^T c_hat, so sum_t p_t v_hat_t = Pi^T sum_t p_t n_t c_hat_t;
* Pi is the Q factor of the QR decomposition of a seeded N(0, 1) d x d draw with
  the signs fixed so that diag(R) > 0 (unique); S is a seeded N(0, 1) m x d draw.
* Walsh-Hadamard variant ("TurboQuant : les cinq innovations", item 1 names a
  Walsh-Hadamard transform as the rotation): Pi = H_d / sqrt(d) with H_d the
  Sylvester-order Hadamard matrix, no random sign flips (the page describes the
  plain transform); every other step is unchanged.
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import ndtr

from .numerics import decode16, fp16_round


# ------------------------------------------------------------------ codebook
def lloyd_max_gaussian(levels: int = 8, iters: int = 10000, tol: float = 1e-15):
    """Lloyd-Max quantizer of N(0, 1): alternately thresholds = midpoints of the
    levels and levels = conditional means E[X | cell].  Returns (levels,
    thresholds), both float64 and ascending."""
    c = np.linspace(-2.0, 2.0, levels)
    phi = lambda x: np.exp(-0.5 * x * x) / math.sqrt(2 * math.pi)
    for _ in range(iters):
        t = 0.5 * (c[1:] + c[:-1])
        lo = np.concatenate([[-np.inf], t])
        hi = np.concatenate([t, [np.inf]])
        mass = ndtr(hi) - ndtr(lo)
        new = (phi(lo) - phi(hi)) / mass
        if np.max(np.abs(new - c)) < tol:
            c = new
            break
        c = new
    return c, 0.5 * (c[1:] + c[:-1])


def deployed_codebook(d: int, levels: int = 8):
    """Levels for N(0, 1/d) rounded to fp16 (float64 values) and the midpoint
    thresholds between them (exact in float64)."""
    c, _ = lloyd_max_gaussian(levels)
    cf = fp16_round(c / math.sqrt(d))
    return cf, 0.5 * (cf[1:] + cf[:-1])


def gaussian_mse(levels: np.ndarray, thresholds: np.ndarray) -> float:
    """E[(X - Q(X))^2] for X ~ N(0, 1), in closed form per cell."""
    lo = np.concatenate([[-np.inf], thresholds])
    hi = np.concatenate([thresholds, [np.inf]])
    phi = lambda x: np.where(np.isinf(x), 0.0, np.exp(-0.5 * np.where(np.isinf(x), 0, x) ** 2) / math.sqrt(2 * math.pi))
    xphi = lambda x: np.where(np.isinf(x), 0.0, np.where(np.isinf(x), 0, x) * phi(x))
    m0 = ndtr(hi) - ndtr(lo)                       # P(cell)
    m1 = phi(lo) - phi(hi)                         # E[X; cell]
    m2 = m0 + xphi(lo) - xphi(hi)                  # E[X^2; cell]
    return float(np.sum(m2 - 2 * levels * m1 + levels ** 2 * m0))


# ------------------------------------------------------------------ rotation
def rotation(gauss: np.ndarray) -> np.ndarray:
    """Q factor of QR(gauss) with diag(R) > 0, float64."""
    q, r = np.linalg.qr(np.asarray(gauss, np.float64))
    sgn = np.sign(np.diag(r))
    sgn[sgn == 0] = 1.0
    return q * sgn[None, :]


def rotation_wht(d: int) -> np.ndarray:
    """Walsh-Hadamard rotation H_d / sqrt(d), float64, with H_1 = [1] and
    H_2n = [[H_n, H_n], [H_n, -H_n]] (Sylvester order); d a power of two."""
    if d < 1 or d & (d - 1):
        raise ValueError("d must be a power of two")
    h = np.ones((1, 1))
    while h.shape[0] < d:
        h = np.block([[h, h], [h, -h]])
    return h / math.sqrt(d)


# ------------------------------------------------------------------ quantizer
def codes_of(y: np.ndarray, thresholds: np.ndarray) -> np.ndarray:
    """Number of thresholds strictly below each value (ties go low)."""
    return np.sum(np.asarray(y)[..., None] > thresholds, axis=-1).astype(np.uint8)


def quantize(x: np.ndarray, Pi: np.ndarray, levels: np.ndarray, thresholds: np.ndarray,
             S: np.ndarray = None):
    """Vectors x [T][d] (float64) -> dict with codes [T][d], n (fp16 values),
    y (rotated unit vectors, float64), and for keys (S given) gamma (fp16
    values) and sign bits [T][m] (uint8 0/1) with the raw S e for diagnostics."""
    x = np.asarray(x, np.float64)
    n = np.sqrt(np.sum(x * x, axis=1))
    safe = np.where(n > 0, n, 1.0)
    u = np.where(n[:, None] > 0, x / safe[:, None], 0.0)
    y = u @ Pi.T
    c = codes_of(y, thresholds)
    out = {"codes": c, "n": fp16_round(n), "n_exact": n, "y": y}
    if S is not None:
        e = y - levels[c]
        out["gamma_exact"] = n * np.sqrt(np.sum(e * e, axis=1))
        out["gamma"] = fp16_round(out["gamma_exact"])
        se = e @ np.asarray(S, np.float64).T
        out["se"] = se
        out["signs"] = (se >= 0).astype(np.uint8)
    return out


def qjl_constant(m: int) -> float:
    return math.sqrt(math.pi / 2.0) / m


# ------------------------------------------------------------------ attention
def scores_quantized(q: np.ndarray, Pi: np.ndarray, S: np.ndarray, levels: np.ndarray, kq: dict,
                     scale: float) -> np.ndarray:
    """q [g][d] against quantized keys -> scaled scores [g][T]."""
    qr = np.asarray(q, np.float64) @ Pi.T                      # Pi q
    qs = qr @ np.asarray(S, np.float64).T                      # S Pi q
    chat = levels[kq["codes"]]                                 # [T][d]
    sgn = 2.0 * kq["signs"].astype(np.float64) - 1.0           # [T][m]
    m = sgn.shape[1]
    main = (qr @ chat.T) * kq["n"][None, :]
    corr = (qs @ sgn.T) * (kq["gamma"][None, :] * qjl_constant(m))
    return scale * (main + corr)


def attention(q, Pi, S, levels, kq: dict, vq: dict, wk: np.ndarray, wv: np.ndarray, scale: float) -> np.ndarray:
    """Decode attention over T_q quantized tokens (kq, vq) and the exact window
    tokens wk, wv [r][d] (float64).  Returns [g][d]."""
    q = np.asarray(q, np.float64)
    s_q = scores_quantized(q, Pi, S, levels, kq, scale) if kq["codes"].shape[0] else np.zeros((q.shape[0], 0))
    s_w = scale * (q @ np.asarray(wk, np.float64).T)
    s = np.concatenate([s_q, s_w], axis=1)
    mx = s.max(axis=1, keepdims=True)
    p = np.exp(s - mx)
    pq, pw = p[:, :s_q.shape[1]], p[:, s_q.shape[1]:]
    o_rot = pq @ (levels[vq["codes"]] * vq["n"][:, None]) if s_q.shape[1] else np.zeros_like(q)
    o = o_rot @ Pi + pw @ np.asarray(wv, np.float64)
    return o / p.sum(axis=1, keepdims=True)


def dequantize_values(vq: dict, Pi: np.ndarray, levels: np.ndarray) -> np.ndarray:
    """v_hat = n Pi^T c_hat, [T][d]."""
    return (levels[vq["codes"]] * vq["n"][:, None]) @ Pi
