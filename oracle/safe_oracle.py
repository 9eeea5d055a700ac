"""Plain fp64 CPU oracle for the SAFE-DiT attention hot path.

TEST INFRASTRUCTURE ONLY. Nothing in the product path may import, call or
execute this module: only the test suite, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it. It shares
no code with the CUDA library (``mask_free_b200``) and imports nothing from it.

Every function follows one passage of the paper *SAFE-DiT: Semantics-Aware
Fast-path Execution for High-Resolution Diffusion Transformers* (arXiv
2606.29360, HTML version of the paper body), cited by equation number. The
code is the definition written out: fp64 arithmetic, a library matmul or sort
as a single step where noted, no blocking, fusion or reordering beyond what
the equations state.

Layouts (shared with the CUDA path only through the test harness):
  image tensors Q, K, V, O   [B, N, H, d]   (token-major)
  text tensors  K_y, V_y     [B, M, H, d]
  valid_len                  [B] int, keys j < valid_len[b] are valid
  scores                     [B, N]
  S, C                       [B, k], [B, N-k] int, each strictly ascending

Readings of the paper where it is silent:
  * the padding mask m_text keeps a prefix of valid keys (right padding);
  * scores are kept per sample b (Eq. (10) has no batch index);
  * top-k ties go to the lower token index; -0.0 is treated as +0.0;
  * a mask dimension with stride 0 is a broadcast dimension and is scanned
    once (its rows are the same stored row);
  * the context cache holds post-projection K/V rows (projection is
    row-wise, so selecting rows commutes with it: Eq. (1), Eq. (14)).
"""

from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np

# ----------------------------------------------------------------------------
# bf16 helpers (exact widening only; rounding of inputs happens in the
# seeded input generator, not here)
# ----------------------------------------------------------------------------


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 values stored as uint16 bit patterns to float64 (exact)."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def f16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen fp16 values stored as uint16 bit patterns to float64 (exact)."""
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


# ----------------------------------------------------------------------------
# Row-constant mask class R  (Eq. (6), with the per-broadcast-row rule and the
# special cases stated after Eq. (7))
# ----------------------------------------------------------------------------

DTYPE_BOOL, DTYPE_U8, DTYPE_F32, DTYPE_F16, DTYPE_BF16 = 0, 1, 2, 3, 4


def _mask_values(flat: np.ndarray, dtype_code: int) -> np.ndarray:
    if dtype_code in (DTYPE_BOOL, DTYPE_U8):
        return np.asarray(flat).astype(np.uint8)
    if dtype_code == DTYPE_F32:
        return np.asarray(flat, dtype=np.float32).astype(np.float64)
    if dtype_code == DTYPE_F16:
        return f16_bits_to_f64(flat)
    if dtype_code == DTYPE_BF16:
        return bf16_bits_to_f64(flat)
    raise ValueError(f"unknown mask dtype code {dtype_code}")


def row_in_R(row: np.ndarray, dtype_code: int) -> bool:
    """Is one mask row a row-constant shift (Eq. (6))?

    Boolean/byte masks: true means "may attend". A row is removable only when
    every key is visible (the all-valid Boolean mask is the special case named
    after Eq. (7)); any blocked key keeps the mask.

    Additive masks: the row must equal c_i * 1 for a real c_i, i.e. every
    entry finite and equal (by value) to the row's first entry. Infinite or
    NaN entries are not real constants, so such rows are never in R.
    """
    if dtype_code in (DTYPE_BOOL, DTYPE_U8):
        return bool(np.all(row != 0))
    if row.size == 0:
        return True
    if not np.all(np.isfinite(row)):
        return False
    return bool(np.all(row == row[0]))


def classify_mask(storage: np.ndarray, dtype_code: int, sizes: Sequence[int],
                  strides: Sequence[int], offset: int = 0):
    """Classify a 4-D mask view [B, H, n_q, n_k] given in element strides.

    ``storage`` is the flat 1-D array of stored elements (bf16/fp16 as uint16
    bit patterns). A dimension whose stride is 0 is a broadcast dimension: its
    rows are the same stored row, so it counts once (size treated as 1).

    Returns ``(verdict, nfail, first_fail)``: verdict 1 iff every distinct
    row is in R (Eq. (6), applied per broadcast row); nfail = number of rows
    not in R; first_fail = smallest flat row index b*H'*Q' + h*Q' + i over
    the distinct-row extents (H', Q'), or -1 if none fails.
    """
    sizes = [int(s) for s in sizes]
    strides = [int(s) for s in strides]
    eff = [1 if strides[a] == 0 else sizes[a] for a in range(3)]
    nk = 1 if strides[3] == 0 else sizes[3]
    vals = _mask_values(storage, dtype_code)
    nfail = 0
    first_fail = -1
    for b in range(eff[0]):
        for h in range(eff[1]):
            for i in range(eff[2]):
                start = offset + b * strides[0] + h * strides[1] + i * strides[2]
                idx = start + np.arange(nk, dtype=np.int64) * strides[3]
                if sizes[3] == 0:
                    idx = idx[:0]
                if not row_in_R(vals[idx], dtype_code):
                    nfail += 1
                    if first_fail < 0:
                        first_fail = (b * eff[1] + h) * eff[2] + i
    return (1 if nfail == 0 else 0), nfail, first_fail


# ----------------------------------------------------------------------------
# Scaled dot-product attention  (Eq. (2), with Eq. (5) as the per-row
# distribution)
# ----------------------------------------------------------------------------


def softmax_rows(logits: np.ndarray) -> np.ndarray:
    """Row-wise softmax, Eq. (5): exp(l - max l) / sum exp(l - max l).

    Entries equal to -inf get probability 0. Subtracting the row maximum is
    the row-constant shift of Eq. (7) and does not change the result.
    """
    m = np.max(logits, axis=-1, keepdims=True)
    e = np.exp(logits - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def sdpa_masked(q: np.ndarray, k: np.ndarray, v: np.ndarray, m: Optional[np.ndarray],
                scale: Optional[float] = None, dtype=np.float64) -> np.ndarray:
    """Eq. (2) for one head, literally: Softmax(q k^T / sqrt(d_h) + m) v.

    q [n_q, d], k [n_k, d], v [n_k, d_v], m [n_q, n_k] additive (None = no
    mask argument, i.e. a zero bias). ``dtype`` selects the arithmetic
    (float64 by default; float32 gives the "explicit FP32 reference").
    """
    q = np.asarray(q, dtype=dtype)
    k = np.asarray(k, dtype=dtype)
    v = np.asarray(v, dtype=dtype)
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    logits = (q @ k.T) * dtype(scale)
    if m is not None:
        logits = logits + np.asarray(m, dtype=dtype)
    return softmax_rows(logits) @ v


def attention(Q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float,
              kv_len: Optional[Sequence[int]] = None,
              q_rows: Optional[np.ndarray] = None,
              with_lse: bool = False):
    """Mask-free or padded attention over [B, n, H, d] tensors (Eq. (2)-(4)).

    For every (b, h) and selected query row i:
        l_j = scale * sum_c q_ic k_jc   for valid keys j
        p_j = exp(l_j - max l) / sum_j exp(l_j - max l)
        o_i = sum_j p_j v_j
    Valid keys are all keys (self-attention, Eq. (3)) or j < kv_len[b]
    (image->text cross-attention keeping the text padding mask, Eq. (4)).

    q_rows: None (all rows), a 1-D array of row indices shared by all b, or a
    2-D array [B, r] of per-sample row indices (the sensitive set S for
    Eq. (16)/(17)). Returns O [B, r, H, d] (and lse [B, H, r], natural log).
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    B, N, H, d = Q.shape
    if q_rows is None:
        rows = np.broadcast_to(np.arange(N), (B, N))
    else:
        rows = np.asarray(q_rows)
        if rows.ndim == 1:
            rows = np.broadcast_to(rows, (B, rows.shape[0]))
    r = rows.shape[1]
    O = np.zeros((B, r, H, V.shape[-1]), dtype=np.float64)
    lse = np.zeros((B, H, r), dtype=np.float64)
    for b in range(B):
        L = K.shape[1] if kv_len is None else int(kv_len[b])
        for h in range(H):
            q = Q[b, rows[b], h, :]
            k = K[b, :L, h, :]
            v = V[b, :L, h, :]
            logits = (q @ k.T) * scale
            mx = np.max(logits, axis=1, keepdims=True)
            e = np.exp(logits - mx)
            s = np.sum(e, axis=1, keepdims=True)
            O[b, :, h, :] = (e / s) @ v
            lse[b, h, :] = (mx + np.log(s))[:, 0]
    if with_lse:
        return O, lse
    return O


def cross_attention(Q, Ky, Vy, valid_len, scale, q_rows=None):
    """Eq. (4) (and Eq. (17) with q_rows = S): image queries attend to the
    first valid_len[b] text keys of sample b; padding keys get zero weight."""
    return attention(Q, Ky, Vy, scale, kv_len=valid_len, q_rows=q_rows)


def srsu_attention(Q, S, Kc, Vc, scale):
    """Eq. (16): O^S = SDPA(Q_S, K_{S u C}, V_{S u C}, no mask).

    Kc/Vc are the global keys/values in original token order, assembled from
    the current sensitive rows and the cached context rows (i.e. the cache
    after ``cache_scatter``). Query rows are Q[b, S[b, r]]."""
    return attention(Q, Kc, Vc, scale, kv_len=None, q_rows=np.asarray(S))


# ----------------------------------------------------------------------------
# PCSP  (Eq. (9)-(12))
# ----------------------------------------------------------------------------


def text_probabilities(Q, Ky, valid_len, scale, b: int, h: int) -> np.ndarray:
    """Eq. (9): A[i, j] = image->text attention probability after the
    padding mask and normalisation, for sample b and head h; shape
    [N, valid_len[b]] (padding columns are zero and omitted)."""
    Q = np.asarray(Q, dtype=np.float64)
    Ky = np.asarray(Ky, dtype=np.float64)
    L = int(valid_len[b])
    logits = (Q[b, :, h, :] @ Ky[b, :L, h, :].T) * scale
    return softmax_rows(logits)


def pcsp_scores(Q, Ky, valid_len, w, scale, heads: Optional[Sequence[int]] = None) -> np.ndarray:
    """Eq. (10) for one step t and one layer l, per sample b:

        s~[b, i] = (1/|H|) * sum_{h in H} sum_{j in T_b} w[b, j] * A_{b,h}[i, j]

    with T_b the valid (non-padding) keys j < valid_len[b]. w[b, j] >= 0 are
    the content weights (zero on padding). The mean over the warm-up steps and
    layers of Eq. (10) is the caller's sum of such calls divided by |W||L|
    (a positive constant, irrelevant to the top-k of Eq. (12)).
    """
    Q = np.asarray(Q, dtype=np.float64)
    B, N, H, _ = Q.shape
    hs = list(range(H)) if heads is None else list(heads)
    w = np.asarray(w, dtype=np.float64)
    out = np.zeros((B, N), dtype=np.float64)
    for b in range(B):
        L = int(valid_len[b])
        acc = np.zeros(N, dtype=np.float64)
        for h in hs:
            A = text_probabilities(Q, Ky, valid_len, scale, b, h)
            acc += A @ w[b, :L]
        out[b] = acc / len(hs)
    return out


def ceil_k(rho_num: int, rho_den: int, N: int) -> int:
    """k = ceil(rho * N) for rho = rho_num / rho_den, in exact integers
    (Eq. (12))."""
    return -((-rho_num * N) // rho_den)


def topk_partition(scores: np.ndarray, k: int):
    """Eq. (12): S = TopK(s, k), C = complement.

    Ordering: score descending, then token index ascending (ties go to the
    lower index); -0.0 is the same score as +0.0. A library sort is the one
    step used. Returns S [B, k] and C [B, N-k], each sorted ascending.
    """
    scores = np.asarray(scores, dtype=np.float64) + 0.0  # -0.0 -> +0.0
    B, N = scores.shape
    S = np.zeros((B, k), dtype=np.int64)
    C = np.zeros((B, N - k), dtype=np.int64)
    for b in range(B):
        order = np.lexsort((np.arange(N), -scores[b]))  # primary: -score, secondary: index
        S[b] = np.sort(order[:k])
        C[b] = np.sort(order[k:])
    return S, C


# ----------------------------------------------------------------------------
# Context cache  (Eq. (14), (16), (19))
# ----------------------------------------------------------------------------


def cache_scatter(cache: np.ndarray, src: np.ndarray, S: Optional[np.ndarray],
                  src_compact: bool) -> np.ndarray:
    """Return the cache after writing the current sensitive rows into it.

    cache [B, N, H, d]; S [B, k] (None = full refresh, Eq. (19): the cache
    becomes the source). With S given, row S[b, r] of the cache takes
    src[b, r] (compact source, [B, k, H, d]) or src[b, S[b, r]] (full-size
    source). Every other row is unchanged: this assembles K_{S u C} in the
    original token order from current sensitive and cached context rows
    (Eq. (16)). Works on any dtype (copies are exact).
    """
    out = np.array(cache, copy=True)
    if S is None:
        out[...] = src
        return out
    S = np.asarray(S)
    for b in range(out.shape[0]):
        for r in range(S.shape[1]):
            out[b, S[b, r]] = src[b, r] if src_compact else src[b, S[b, r]]
    return out


# ----------------------------------------------------------------------------
# Sensitivity field on the latent grid  (Eq. (11))
# ----------------------------------------------------------------------------


def gaussian_taps(sigma: float, truncate: float = 4.0) -> np.ndarray:
    """The 1-D Gaussian G_sigma of Eq. (11) at integer offsets t = -r..r.

    Weights exp(-t^2 / (2 sigma^2)) normalised to sum 1, cut at radius
    r = floor(truncate * sigma + 1/2). The paper gives no sigma and no
    cut-off; a cut at 4 sigma is the usual choice. sigma = 0 is the identity.
    """
    if sigma <= 0.0:
        return np.ones(1, dtype=np.float64)
    r = int(math.floor(truncate * sigma + 0.5))
    t = np.arange(-r, r + 1, dtype=np.float64)
    g = np.exp(-(t * t) / (2.0 * sigma * sigma))
    return g / np.sum(g)


def reflect_index(idx: np.ndarray, n: int) -> np.ndarray:
    """Index into [0, n) of the half-sample symmetric extension of a line of
    n values: ... x1 x0 | x0 x1 ... x_{n-1} | x_{n-1} x_{n-2} ... (period 2n)."""
    m = np.mod(np.asarray(idx), 2 * n)
    return np.where(m < n, m, 2 * n - 1 - m)


def smooth_scores(scores: np.ndarray, grid_h: int, grid_w: int, sigma: float,
                  truncate: float = 4.0) -> np.ndarray:
    """G_sigma * s~ of Eq. (11), per sample.

    The N = grid_h * grid_w scores of a sample lie on the latent token grid
    in row-major order (token i = y * grid_w + x). The 2-D Gaussian is
    separable: convolve every row with the 1-D taps, then every column.
    Borders: half-sample reflection (the paper names no border rule).
    """
    s = np.asarray(scores, dtype=np.float64)
    B, N = s.shape
    assert N == grid_h * grid_w
    g = gaussian_taps(sigma, truncate)
    r = (g.size - 1) // 2
    f = s.reshape(B, grid_h, grid_w)
    xs, ys = np.arange(grid_w), np.arange(grid_h)
    rows = np.zeros_like(f)
    for t in range(-r, r + 1):
        rows += g[t + r] * f[:, :, reflect_index(xs + t, grid_w)]
    out = np.zeros_like(f)
    for t in range(-r, r + 1):
        out += g[t + r] * rows[:, reflect_index(ys + t, grid_h), :]
    return out.reshape(B, N)


def norm01(x: np.ndarray) -> np.ndarray:
    """Norm of Eq. (11): per-sample min-max map onto [0, 1]. A flat field
    (max = min) maps to 0, a reading: the paper does not define that case."""
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    for b in range(x.shape[0]):
        lo, hi = np.min(x[b]), np.max(x[b])
        if hi > lo:
            out[b] = (x[b] - lo) / (hi - lo)
    return out


def sensitivity_field(scores: np.ndarray, grid_h: int, grid_w: int, sigma: float,
                      truncate: float = 4.0) -> np.ndarray:
    """s = Norm(G_sigma * s~), Eq. (11). [B, N] -> [B, N] in [0, 1]."""
    return norm01(smooth_scores(scores, grid_h, grid_w, sigma, truncate))


# ----------------------------------------------------------------------------
# Sensitivity-weighted CFG  (Eq. (20), (21))
# ----------------------------------------------------------------------------


def partition_indicator(S: np.ndarray, N: int) -> np.ndarray:
    """The binary variant after Eq. (21): s_i = 1 for tokens of S, 0 for C."""
    S = np.asarray(S)
    out = np.zeros((S.shape[0], N), dtype=np.float64)
    for b in range(S.shape[0]):
        out[b, S[b]] = 1.0
    return out


def sw_cfg(f_c: np.ndarray, f_u: np.ndarray, s: np.ndarray, gamma_ctx: float,
           gamma_sens: float) -> np.ndarray:
    """Eq. (20): gamma_i = gamma_ctx + (gamma_sens - gamma_ctx) * s_i, then
    Eq. (21): f^_i = f_u,i + gamma_i * (f_c,i - f_u,i).

    f_c, f_u: conditional / unconditional predictions [B, N, C] (token-major,
    C values per token); s: [B, N]. Returns [B, N, C] in fp64.
    """
    fc = np.asarray(f_c, dtype=np.float64)
    fu = np.asarray(f_u, dtype=np.float64)
    gamma = gamma_ctx + (gamma_sens - gamma_ctx) * np.asarray(s, dtype=np.float64)
    return fu + gamma[:, :, None] * (fc - fu)


# ----------------------------------------------------------------------------
# Row-selective block: row-wise layers on the rows of S  (Eq. (13), (15))
# ----------------------------------------------------------------------------


def gelu_tanh(x: np.ndarray) -> np.ndarray:
    """GELU in its tanh form (Hendrycks and Gimpel, "Gaussian Error Linear
    Units (GELUs)", the tanh approximation of x * Phi(x)):
        0.5 x (1 + tanh( sqrt(2 / pi) (x + 0.044715 x^3) )).
    The paper names no activation; this is the form DiT-family MLPs use."""
    x = np.asarray(x, dtype=np.float64)
    return 0.5 * x * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (x + 0.044715 * x ** 3)))


def gathered_linear(X: np.ndarray, S: Optional[np.ndarray], Wt: np.ndarray,
                    bias: Optional[np.ndarray] = None, act: str = "none") -> np.ndarray:
    """A row-wise layer of the row-selective block B^S (Eq. (15)) evaluated
    only on the sensitive rows: with the row selection P_S of Eq. (13),

        Y[b, r, :] = act( X[b, S[b, r], :] @ Wt^T + bias ),

    X [B, N, D_in] (token-major), Wt [D_out, D_in] (the weight of a linear
    layer y = x W^T + b), bias [D_out] or None, act "none" or "gelu_tanh".
    S = None selects every row in order (the dense block of Eq. (18)). One
    library matmul per sample, fp64. Returns [B, k or N, D_out]."""
    X = np.asarray(X, dtype=np.float64)
    Wt = np.asarray(Wt, dtype=np.float64)
    out = []
    for b in range(X.shape[0]):
        rows = X[b] if S is None else X[b, np.asarray(S)[b]]   # P_S H (Eq. (13))
        y = rows @ Wt.T
        if bias is not None:
            y = y + np.asarray(bias, dtype=np.float64)[None, :]
        if act == "gelu_tanh":
            y = gelu_tanh(y)
        elif act != "none":
            raise ValueError(f"unknown activation {act!r}")
        out.append(y)
    return np.stack(out)
