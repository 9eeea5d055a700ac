"""Pins of the fp64 oracle against facts fixed by the paper and by mathematics.

Each test checks the oracle against something other than itself: closed
forms derived by hand (tests/golden), invariants the equations state, special
cases that reduce to a textbook result, and brute force on tiny inputs. A
plausible slip in the oracle (a dropped scale, a sign, a transposed operand,
a wrong padding side, an off-by-one in k) fails at least one of them.
"""

import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _num(s):
    return {"0": 0.0, "ln2": math.log(2), "ln3": math.log(3), "ln4": math.log(4), "-inf": -math.inf}.get(s, None) \
        if s in ("0", "ln2", "ln3", "ln4", "-inf") else float(s)


# ---------------------------------------------------------------- attention: closed forms


@pytest.mark.parametrize("case", json.load(open(os.path.join(GOLDEN, "softmax_closed_form.json")))["cases"],
                         ids=lambda c: c["name"])
def test_sdpa_closed_form_golden(case):
    # Eq. (2) with d_h = 1 and an explicit scale of 1: q = [1], k_j = [logit_j],
    # V = identity, so the output row is the distribution pi_i itself.
    logits = np.array([_num(s) for s in case["logits"]])
    n = len(logits)
    q = np.ones((1, 1))
    k = logits.reshape(n, 1)
    v = np.eye(n)
    m = None if case["mask"] is None else np.array([[_num(s) for s in case["mask"]]])
    out = O.sdpa_masked(q, k, v, m, scale=1.0)[0]
    expected = np.array([a / b for a, b in case["expected"]])
    np.testing.assert_allclose(out, expected, rtol=0, atol=1e-15)


def _brute_attention(Q, K, V, scale, kv_len=None, rows=None):
    """Pure-Python loops over the definition (tiny inputs only)."""
    B, N, H, d = Q.shape
    out = {}
    for b in range(B):
        L = K.shape[1] if kv_len is None else kv_len[b]
        rr = range(N) if rows is None else rows[b]
        for h in range(H):
            for r, i in enumerate(rr):
                logits = []
                for j in range(L):
                    logits.append(scale * sum(float(Q[b, i, h, c]) * float(K[b, j, h, c]) for c in range(d)))
                mx = max(logits)
                e = [math.exp(x - mx) for x in logits]
                s = math.fsum(e)
                for c in range(V.shape[-1]):
                    out[(b, r, h, c)] = math.fsum(e[j] / s * float(V[b, j, h, c]) for j in range(L))
    return out


def test_attention_brute_force_tiny():
    rng = np.random.default_rng(7)
    B, N, M, H, d = 2, 6, 5, 2, 3
    Q = rng.standard_normal((B, N, H, d))
    K = rng.standard_normal((B, N, H, d))
    V = rng.standard_normal((B, N, H, d))
    Ky = rng.standard_normal((B, M, H, d))
    Vy = rng.standard_normal((B, M, H, d))
    scale = 1 / math.sqrt(d)
    # self-attention, all rows
    got = O.attention(Q, K, V, scale)
    for (b, r, h, c), val in _brute_attention(Q, K, V, scale).items():
        assert abs(got[b, r, h, c] - val) < 1e-13
    # cross-attention with padding and a row selection
    lens = [3, 5]
    rows = np.array([[0, 2, 5], [1, 3, 4]])
    got = O.cross_attention(Q, Ky, Vy, lens, scale, q_rows=rows)
    for (b, r, h, c), val in _brute_attention(Q, Ky, Vy, scale, kv_len=lens, rows=rows).items():
        assert abs(got[b, r, h, c] - val) < 1e-13


def test_attention_scale_is_one_over_sqrt_dh():
    # With q = k = e_0 * a, the logit between identical rows is a^2 / sqrt(d).
    d = 16
    a = 3.0
    Q = np.zeros((1, 1, 1, d)); Q[0, 0, 0, 0] = a
    K = np.zeros((1, 2, 1, d)); K[0, 0, 0, 0] = a  # key 1 is zero -> logit 0
    V = np.zeros((1, 2, 1, d)); V[0, 0, 0, 0] = 1.0
    out = O.attention(Q, K, V, 1 / math.sqrt(d))
    l0 = a * a / math.sqrt(d)
    assert abs(out[0, 0, 0, 0] - 1 / (1 + math.exp(-l0))) < 1e-15


def test_lse_closed_form():
    # identical keys: every logit equals c, so lse = c + ln(L)
    d, L = 8, 7
    rng = np.random.default_rng(3)
    q = rng.standard_normal(d)
    k = rng.standard_normal(d)
    Q = q.reshape(1, 1, 1, d)
    K = np.broadcast_to(k, (1, L, 1, d)).copy()
    V = rng.standard_normal((1, L, 1, d))
    out, lse = O.attention(Q, K, V, 0.5, with_lse=True)
    c = 0.5 * float(q @ k)
    assert abs(lse[0, 0, 0] - (c + math.log(L))) < 1e-12
    np.testing.assert_allclose(out[0, 0, 0], V[0, :, 0].mean(axis=0), atol=1e-14)


# ---------------------------------------------------------------- Eq. (7): invariance and necessity


def test_row_constant_shift_invariance_fp64():
    rng = np.random.default_rng(11)
    n_q, n_k, d = 9, 13, 8
    q, k, v = (rng.standard_normal((n, d)) for n in (n_q, n_k, n_k))
    c = rng.uniform(-5, 5, size=(n_q, 1))
    masked = O.sdpa_masked(q, k, v, np.broadcast_to(c, (n_q, n_k)))
    plain = O.sdpa_masked(q, k, v, None)
    assert np.max(np.abs(masked - plain)) <= 1e-12


def test_non_constant_row_changes_distribution():
    # With zero logits the distribution is softmax(m_i) itself, which is not
    # uniform for a non-constant row (necessity half of Eq. (7)).
    n_k = 5
    m = np.array([[0.0, 1.0, 0.0, -2.0, 0.5]])
    pi = O.sdpa_masked(np.zeros((1, 1)), np.zeros((n_k, 1)), np.eye(n_k), m, scale=1.0)[0]
    e = np.exp(m[0])
    np.testing.assert_allclose(pi, e / e.sum(), atol=1e-15)
    assert np.max(np.abs(pi - 1.0 / n_k)) > 1e-3
    # and on random logits the masked and mask-free outputs differ
    rng = np.random.default_rng(5)
    q, k, v = rng.standard_normal((4, 6)), rng.standard_normal((n_k, 6)), rng.standard_normal((n_k, 6))
    mm = np.zeros((4, n_k)); mm[2] = m[0]
    assert np.max(np.abs(O.sdpa_masked(q, k, v, mm) - O.sdpa_masked(q, k, v, None))) > 1e-3


def test_fp32_reference_agreement_certified_masks():
    # The explicit FP32 reference with a certified-removable mask agrees with
    # the mask-free FP32 result within 9e-8 (the paper's exactness result).
    rng = np.random.default_rng(2)
    n, d = 256, 64
    q, k, v = (rng.standard_normal((n, d)).astype(np.float32) for _ in range(3))
    zero = np.zeros((n, n), dtype=np.float32)
    a = O.sdpa_masked(q, k, v, zero, dtype=np.float32)
    b = O.sdpa_masked(q, k, v, None, dtype=np.float32)
    assert np.max(np.abs(a - b)) <= 9e-8
    # fp32 vs fp64: the fp32 mode is a genuine fp32 evaluation (not exact)
    c64 = O.sdpa_masked(q, k, v, None)
    err = np.max(np.abs(b - c64))
    assert 0 < err < 1e-5


# ---------------------------------------------------------------- classifier (Eq. (6))


def _classify(t, code):
    a = np.ascontiguousarray(t)
    st = [s // a.itemsize for s in a.strides]
    return O.classify_mask(a.reshape(-1), code, a.shape, st)


def test_classifier_six_tiny_masks():
    from mask_free_b200 import synth
    masks = synth.tiny_masks(N=256, H=2, valid_len=11, M=16, seed=42)
    assert _classify(masks["all_true"].numpy(), O.DTYPE_BOOL) == (1, 0, -1)
    assert _classify(masks["all_zero"].numpy(), O.DTYPE_F32) == (1, 0, -1)
    assert _classify(masks["row_constant"].numpy(), O.DTYPE_F32) == (1, 0, -1)
    i = masks["_nonconst_row"]
    assert _classify(masks["one_nonconstant_row"].numpy(), O.DTYPE_F32) == (0, 1, i)  # head 0, row i
    v, nf, ff = _classify(masks["text_padding"].numpy(), O.DTYPE_BOOL)
    assert (v, nf, ff) == (0, 256, 0)
    v, nf, ff = _classify(masks["nan_entry"].numpy(), O.DTYPE_F32)
    assert v == 0 and nf == 1


def test_classifier_verdict_matches_effect_on_attention():
    # A mask is in R exactly when attention with it equals attention without
    # it for arbitrary logits: check the verdict against the effect.
    rng = np.random.default_rng(9)
    n, d = 16, 8
    q, k, v = (rng.standard_normal((n, d)) for _ in range(3))
    cases = {
        "zero": np.zeros((n, n)),
        "rowconst": np.broadcast_to(rng.uniform(-5, 5, (n, 1)), (n, n)).copy(),
        "nonconst": np.where(np.arange(n)[None, :] == 3, 0.7, 0.0) * (np.arange(n)[:, None] == 5),
        "bias": rng.standard_normal((n, n)) * 0.1,
    }
    for name, m in cases.items():
        verdict = O.classify_mask(m.astype(np.float32).reshape(-1), O.DTYPE_F32, (1, 1, n, n), (0, 0, n, 1))[0]
        diff = np.max(np.abs(O.sdpa_masked(q, k, v, m) - O.sdpa_masked(q, k, v, None)))
        assert (diff < 1e-12) == (verdict == 1), name


def test_classifier_special_values_and_dtypes():
    f = np.float32
    assert O.row_in_R(np.array([-0.0, 0.0, 0.0], dtype=f).astype(np.float64), O.DTYPE_F32)
    assert not O.row_in_R(np.array([-np.inf] * 4), O.DTYPE_F32)       # all -inf gives NaN in SDPA
    assert not O.row_in_R(np.array([np.inf] * 4), O.DTYPE_F32)
    assert not O.row_in_R(np.array([1.0, np.nan]), O.DTYPE_F32)
    assert not O.row_in_R(np.array([1.0, 1.0 + 2 ** -20]), O.DTYPE_F32)
    assert O.row_in_R(np.array([2, 1, 255], dtype=np.uint8), O.DTYPE_U8)
    assert not O.row_in_R(np.array([2, 0, 255], dtype=np.uint8), O.DTYPE_U8)
    # bf16 / fp16 bit patterns: 0x3F80 = 1.0 (bf16), 0x3C00 = 1.0 (fp16)
    assert O.classify_mask(np.array([0x3F80] * 4, np.uint16), O.DTYPE_BF16, (1, 1, 1, 4), (0, 0, 0, 1))[0] == 1
    assert O.classify_mask(np.array([0x3F80, 0x3F81, 0x3F80, 0x3F80], np.uint16), O.DTYPE_BF16,
                           (1, 1, 1, 4), (0, 0, 0, 1))[0] == 0
    assert O.classify_mask(np.array([0x7FC0, 0x7FC0], np.uint16), O.DTYPE_BF16, (1, 1, 1, 2), (0, 0, 0, 1))[0] == 0
    assert O.classify_mask(np.array([0x3C00] * 3, np.uint16), O.DTYPE_F16, (1, 1, 1, 3), (0, 0, 0, 1))[0] == 1
    assert O.classify_mask(np.array([0x3C00, 0x8000, 0x3C00], np.uint16), O.DTYPE_F16,
                           (1, 1, 1, 3), (0, 0, 0, 1))[0] == 0
    # -0 and +0 in fp16 are the same real value
    assert O.classify_mask(np.array([0x0000, 0x8000], np.uint16), O.DTYPE_F16, (1, 1, 1, 2), (0, 0, 0, 1))[0] == 1


def test_classifier_broadcast_rows_and_first_fail():
    # [B=2, H=3 (stride 0), n_q=4, n_k=5]: 8 distinct rows; rows (b=1, i=2) and
    # (b=1, i=3) are non-constant -> nfail 2, first_fail = 1*4 + 2 = 6.
    st = np.zeros((2, 4, 5), dtype=np.float32)
    st[1, 2, 4] = 1.0
    st[1, 3, 0] = -1.0
    v, nf, ff = O.classify_mask(st.reshape(-1), O.DTYPE_F32, (2, 3, 4, 5), (20, 0, 5, 1))
    assert (v, nf, ff) == (0, 2, 6)
    # key-broadcast rows (n_k stride 0) are constant: removable iff finite
    vals = np.array([1.0, -3.0, 7.5], dtype=np.float32)
    assert O.classify_mask(vals, O.DTYPE_F32, (1, 1, 3, 1000), (0, 0, 1, 0))[0] == 1
    vals[1] = -np.inf
    assert O.classify_mask(vals, O.DTYPE_F32, (1, 1, 3, 1000), (0, 0, 1, 0)) == (0, 1, 1)
    # brute force over all 2^6 boolean 2x3 masks
    for bits in itertools.product([0, 1], repeat=6):
        m = np.array(bits, dtype=np.uint8)
        v, nf, ff = O.classify_mask(m, O.DTYPE_BOOL, (1, 1, 2, 3), (0, 0, 3, 1))
        rows_ok = [all(bits[0:3]), all(bits[3:6])]
        assert nf == rows_ok.count(False) and v == int(all(rows_ok))
        assert ff == (-1 if all(rows_ok) else rows_ok.index(False))


# ---------------------------------------------------------------- padding, special cases


def test_padding_keys_get_zero_weight():
    rng = np.random.default_rng(1)
    B, N, M, H, d = 2, 8, 10, 2, 4
    Q = rng.standard_normal((B, N, H, d))
    Ky = rng.standard_normal((B, M, H, d))
    Vy = rng.standard_normal((B, M, H, d))
    lens = [3, 7]
    ref = O.cross_attention(Q, Ky, Vy, lens, 0.5)
    for fill in (np.nan, 1e30, -1e30):
        Ky2, Vy2 = Ky.copy(), Vy.copy()
        for b, L in enumerate(lens):
            Ky2[b, L:] = fill
            Vy2[b, L:] = fill
        out = O.cross_attention(Q, Ky2, Vy2, lens, 0.5)
        assert np.all(np.isfinite(out))
        assert np.array_equal(out, ref)
    # right padding, not left: padding at the front changes the result
    Vy3 = Vy.copy(); Vy3[0, 0] += 1.0
    assert not np.array_equal(O.cross_attention(Q, Ky, Vy3, lens, 0.5), ref)


def test_single_valid_key_returns_its_value():
    rng = np.random.default_rng(4)
    Q = rng.standard_normal((1, 5, 2, 4))
    Ky = rng.standard_normal((1, 6, 2, 4))
    Vy = rng.standard_normal((1, 6, 2, 4))
    out = O.cross_attention(Q, Ky, Vy, [1], 0.5)
    for i in range(5):
        assert np.array_equal(out[0, i], Vy[0, 0])


def test_identical_keys_give_mean_of_values():
    rng = np.random.default_rng(6)
    Q = rng.standard_normal((1, 4, 1, 8))
    K = np.broadcast_to(rng.standard_normal(8), (1, 9, 1, 8)).copy()
    V = rng.standard_normal((1, 9, 1, 8))
    out = O.cross_attention(Q, K, V, [6], 0.3)
    np.testing.assert_allclose(out[0, :, 0], np.broadcast_to(V[0, :6, 0].mean(0), (4, 8)), atol=1e-14)


# ---------------------------------------------------------------- SRSU (Eq. (16)) and cache


def test_srsu_all_rows_equals_dense():
    rng = np.random.default_rng(8)
    B, N, H, d = 2, 12, 2, 4
    Q, K, V = (rng.standard_normal((B, N, H, d)) for _ in range(3))
    S = np.broadcast_to(np.arange(N), (B, N))
    cache_k = O.cache_scatter(np.zeros_like(K), K, S, src_compact=False)
    cache_v = O.cache_scatter(np.zeros_like(V), V, S, src_compact=False)
    dense = O.attention(Q, K, V, 0.5)
    assert np.max(np.abs(O.srsu_attention(Q, S, cache_k, cache_v, 0.5) - dense)) < 1e-14


def test_srsu_unchanged_context_reproduces_dense_rows():
    rng = np.random.default_rng(12)
    B, N, H, d = 2, 16, 3, 5
    Q, K, V = (rng.standard_normal((B, N, H, d)) for _ in range(3))
    S = np.array([[1, 4, 5, 11], [0, 2, 3, 15]])
    dense = O.attention(Q, K, V, 0.4)
    out = O.srsu_attention(Q, S, K, V, 0.4)
    for b in range(B):
        np.testing.assert_allclose(out[b], dense[b, S[b]], atol=1e-14)
    # stale context changes the result (queries still see all keys)
    Kc = K.copy(); Kc[:, 7] += 0.5
    assert np.max(np.abs(O.srsu_attention(Q, S, Kc, V, 0.4) - out)) > 1e-6


def test_cache_scatter_properties():
    rng = np.random.default_rng(13)
    B, N, H, d, k = 2, 10, 2, 3, 4
    cache = rng.standard_normal((B, N, H, d))
    src_full = rng.standard_normal((B, N, H, d))
    S = np.array([[0, 3, 4, 9], [2, 5, 6, 7]])
    C = np.array([[i for i in range(N) if i not in S[b]] for b in range(B)])
    out = O.cache_scatter(cache, src_full, S, src_compact=False)
    compact = np.stack([src_full[b, S[b]] for b in range(B)])
    out2 = O.cache_scatter(cache, compact, S, src_compact=True)
    assert np.array_equal(out, out2)
    for b in range(B):
        assert np.array_equal(out[b, S[b]], src_full[b, S[b]])
        assert np.array_equal(out[b, C[b]], cache[b, C[b]])
    assert np.array_equal(O.cache_scatter(cache, src_full, None, False), src_full)
    # the input cache is not modified
    assert not np.array_equal(out, cache)


# ---------------------------------------------------------------- PCSP (Eq. (9)-(12))


def test_pcsp_uniform_weights_degenerate_closed_form():
    # w uniform over the valid keys: sum_j A_ij = 1, so every score is 1/len_b.
    rng = np.random.default_rng(14)
    B, N, M, H, d = 2, 20, 12, 3, 8
    Q = rng.standard_normal((B, N, H, d))
    Ky = rng.standard_normal((B, M, H, d))
    lens = [5, 12]
    w = np.zeros((B, M))
    for b, L in enumerate(lens):
        w[b, :L] = 1.0 / L
    s = O.pcsp_scores(Q, Ky, lens, w, 1 / math.sqrt(d))
    for b, L in enumerate(lens):
        np.testing.assert_allclose(s[b], np.full(N, 1.0 / L), rtol=1e-12)


def test_pcsp_one_hot_weight_brute_force():
    rng = np.random.default_rng(15)
    B, N, M, H, d = 1, 6, 5, 2, 3
    Q = rng.standard_normal((B, N, H, d))
    Ky = rng.standard_normal((B, M, H, d))
    lens = [4]
    j0 = 2
    w = np.zeros((B, M)); w[0, j0] = 1.0
    s = O.pcsp_scores(Q, Ky, lens, w, 0.7)
    for i in range(N):
        acc = 0.0
        for h in range(H):
            logits = [0.7 * sum(Q[0, i, h, c] * Ky[0, j, h, c] for c in range(d)) for j in range(4)]
            e = [math.exp(x) for x in logits]
            acc += e[j0] / sum(e)
        assert abs(s[0, i] - acc / H) < 1e-14
    # padding keys do not matter
    Ky2 = Ky.copy(); Ky2[0, 4:] = np.nan
    assert np.array_equal(O.pcsp_scores(Q, Ky2, lens, w, 0.7), s)


def test_pcsp_identical_text_keys():
    rng = np.random.default_rng(16)
    B, N, M, H, d = 1, 7, 9, 2, 4
    Q = rng.standard_normal((B, N, H, d))
    Ky = np.broadcast_to(rng.standard_normal(d), (B, M, H, d)).copy()
    w = rng.random((B, M)); w[0, 6:] = 0; w /= w.sum()
    s = O.pcsp_scores(Q, Ky, [6], w, 0.5)
    np.testing.assert_allclose(s[0], np.full(N, 1.0 / 6), rtol=1e-13)


@pytest.mark.parametrize("case", json.load(open(os.path.join(GOLDEN, "topk_k_values.json")))["cases"],
                         ids=lambda c: f"{c['rho'][0]}/{c['rho'][1]}x{c['N']}")
def test_ceil_k_golden(case):
    assert O.ceil_k(case["rho"][0], case["rho"][1], case["N"]) == case["k"]


def test_topk_rank_characterisation_brute_force():
    rng = np.random.default_rng(17)
    for trial in range(200):
        N = int(rng.integers(1, 12))
        k = int(rng.integers(1, N + 1))
        scores = rng.integers(0, 4, size=(2, N)).astype(np.float64) * 0.25  # many ties
        scores[scores == 0.0] = -0.0 if trial % 2 else 0.0
        S, C = O.topk_partition(scores, k)
        for b in range(2):
            chosen = set()
            for i in range(N):
                rank = sum(1 for j in range(N)
                           if scores[b, j] > scores[b, i] or (scores[b, j] == scores[b, i] and j < i))
                if rank < k:
                    chosen.add(i)
            assert list(S[b]) == sorted(chosen)
            assert list(C[b]) == sorted(set(range(N)) - chosen)


def test_topk_all_equal_and_signed_zero():
    S, C = O.topk_partition(np.zeros((1, 10)), 4)
    assert list(S[0]) == [0, 1, 2, 3] and list(C[0]) == list(range(4, 10))
    sc = np.array([[0.0, -0.0, 0.0, -0.0, 1.0]])
    S, _ = O.topk_partition(sc, 3)
    assert list(S[0]) == [0, 1, 4]
    S, C = O.topk_partition(np.arange(6, dtype=float).reshape(1, 6), 6)
    assert list(S[0]) == list(range(6)) and C.shape == (1, 0)


# ---------------------------------------------------------------- Eq. (11): smoothing and Norm


@pytest.mark.parametrize("shape,sigma", [((16, 16), 0.5), ((12, 20), 1.0), ((20, 12), 2.5), ((9, 7), 7.0)])
def test_smoothing_matches_library_gaussian_filter(shape, sigma):
    # an independent implementation of the same operator: scipy's separable
    # Gaussian filter, half-sample reflection at the borders, cut at 4 sigma
    # (non-square grids catch a swapped axis; sigma = 7 on a 9 x 7 grid needs
    # repeated reflections)
    from scipy.ndimage import gaussian_filter
    gh, gw = shape
    rng = np.random.default_rng(11)
    s = rng.random((2, gh * gw))
    got = O.smooth_scores(s, gh, gw, sigma)
    for b in range(2):
        ref = gaussian_filter(s[b].reshape(gh, gw), sigma, mode="reflect", truncate=4.0)
        np.testing.assert_allclose(got[b].reshape(gh, gw), ref, rtol=0, atol=1e-13)


def test_smoothing_identity_constant_and_interior_impulse():
    rng = np.random.default_rng(12)
    s = rng.random((1, 35))
    np.testing.assert_array_equal(O.smooth_scores(s, 5, 7, 0.0), s)  # sigma = 0: no smoothing
    c = np.full((1, 48), 0.37)
    np.testing.assert_allclose(O.smooth_scores(c, 6, 8, 1.3), c, atol=1e-15)  # a flat field stays flat
    # an impulse far from the borders spreads into the sampled 2-D Gaussian:
    # value at offset (dy, dx) = exp(-(dy^2 + dx^2) / (2 sigma^2)) / Z^2, total 1
    gh = gw = 33
    sigma = 1.5
    d = np.zeros((1, gh * gw))
    d[0, 16 * gw + 16] = 1.0
    out = O.smooth_scores(d, gh, gw, sigma).reshape(gh, gw)
    z = sum(math.exp(-t * t / (2 * sigma * sigma)) for t in range(-6, 7))  # radius floor(4 * 1.5 + 0.5) = 6
    for dy, dx in [(0, 0), (1, 0), (0, 2), (3, -4), (-6, 6)]:
        want = math.exp(-(dy * dy + dx * dx) / (2 * sigma * sigma)) / (z * z)
        assert abs(out[16 + dy, 16 + dx] - want) < 1e-15
    assert out[16 + 7, 16] == 0.0 and abs(out.sum() - 1.0) < 1e-13


def test_norm_maps_onto_unit_interval_preserving_order():
    rng = np.random.default_rng(13)
    x = rng.normal(size=(3, 50)) * 7 + 2
    y = O.norm01(x)
    for b in range(3):
        assert y[b].min() == 0.0 and y[b].max() == 1.0
        assert np.array_equal(np.argsort(x[b], kind="stable"), np.argsort(y[b], kind="stable"))
        i, j = np.argmin(x[b]), np.argmax(x[b])
        k = (i + 1) % 50 if (i + 1) % 50 != j else (i + 2) % 50
        # affine: the relative position of any value between min and max
        assert abs(y[b, k] - (x[b, k] - x[b, i]) / (x[b, j] - x[b, i])) < 1e-15
    assert np.array_equal(O.norm01(np.full((1, 4), 5.0)), np.zeros((1, 4)))
    # top-k is unchanged by Norm (a strictly increasing map)
    S1, _ = O.topk_partition(x, 9)
    S2, _ = O.topk_partition(y, 9)
    assert np.array_equal(S1, S2)


# ---------------------------------------------------------------- Eq. (20), (21): SW-CFG


def test_sw_cfg_special_cases_and_interpolation():
    rng = np.random.default_rng(14)
    fc, fu = rng.normal(size=(2, 6, 3)), rng.normal(size=(2, 6, 3))
    s = rng.random((2, 6))
    # gamma = 1 everywhere returns the conditional prediction, 0 the
    # unconditional one (whatever s is)
    np.testing.assert_allclose(O.sw_cfg(fc, fu, s, 1.0, 1.0), fc, atol=1e-15)
    np.testing.assert_allclose(O.sw_cfg(fc, fu, s, 0.0, 0.0), fu, atol=1e-15)
    # s = 0 uses the context scale, s = 1 the sensitive scale: with the other
    # scale arbitrary, the conditional / unconditional prediction comes back
    np.testing.assert_allclose(O.sw_cfg(fc, fu, np.zeros((2, 6)), 1.0, 9.0), fc, atol=1e-15)
    np.testing.assert_allclose(O.sw_cfg(fc, fu, np.ones((2, 6)), -3.0, 0.0), fu, atol=1e-15)
    # the guided prediction is the extrapolation (1 - g) f_u + g f_c, affine in s
    g_ctx, g_sens = 4.0, 7.5
    out = O.sw_cfg(fc, fu, s, g_ctx, g_sens)
    g = g_ctx * (1 - s) + g_sens * s
    np.testing.assert_allclose(out, (1 - g)[..., None] * fu + g[..., None] * fc, atol=1e-12)
    mid = O.sw_cfg(fc, fu, np.full((2, 6), 0.5), g_ctx, g_sens)
    ends = 0.5 * (O.sw_cfg(fc, fu, np.zeros((2, 6)), g_ctx, g_sens) + O.sw_cfg(fc, fu, np.ones((2, 6)), g_ctx, g_sens))
    np.testing.assert_allclose(mid, ends, atol=1e-12)


def test_partition_indicator_binary_variant():
    S = np.array([[0, 3, 4], [1, 2, 5]])
    ind = O.partition_indicator(S, 6)
    assert ind.tolist() == [[1, 0, 0, 1, 1, 0], [0, 1, 1, 0, 0, 1]]
    rng = np.random.default_rng(15)
    fc, fu = rng.normal(size=(2, 6, 2)), rng.normal(size=(2, 6, 2))
    out = O.sw_cfg(fc, fu, ind, 1.0, 0.0)  # C tokens keep f_c, S tokens get f_u
    for b in range(2):
        for i in range(6):
            np.testing.assert_allclose(out[b, i], fu[b, i] if i in S[b] else fc[b, i], atol=1e-15)


# ---------------------------------------------------------------- row-selective block (Eq. (13), (15))


def test_gathered_linear_hand_computed():
    # X rows [1, 2], [3, 4], [5, 6]; W^T maps (a, b) to (a, b, a + b); bias
    # (0.5, 0, -1). Rows S = (2, 0): (5, 6) -> (5.5, 6, 10), (1, 2) -> (1.5, 2, 2)
    X = np.array([[[1.0, 2.0], [3.0, 4.0], [5.0, 6.0]]])
    Wt = np.array([[1.0, 0.0], [0.0, 1.0], [1.0, 1.0]])
    got = O.gathered_linear(X, np.array([[2, 0]]), Wt, np.array([0.5, 0.0, -1.0]))
    assert np.array_equal(got, np.array([[[5.5, 6.0, 10.0], [1.5, 2.0, 2.0]]]))
    # without S: every row, in order
    assert np.array_equal(O.gathered_linear(X, None, Wt)[0, 1], np.array([3.0, 4.0, 7.0]))


def test_gathered_linear_brute_force_with_activation():
    import torch
    rng = np.random.default_rng(3)
    B, N, Din, Dout = 2, 7, 5, 3
    X = rng.standard_normal((B, N, Din))
    Wt = rng.standard_normal((Dout, Din))
    bias = rng.standard_normal(Dout)
    S = np.array([[6, 1, 3], [0, 2, 5]])
    got = O.gathered_linear(X, S, Wt, bias, act="gelu_tanh")
    for b, r, n in itertools.product(range(B), range(S.shape[1]), range(Dout)):
        acc = bias[n]
        for c in range(Din):
            acc += X[b, S[b, r], c] * Wt[n, c]
        want = torch.nn.functional.gelu(torch.tensor(acc, dtype=torch.float64), approximate="tanh").item()
        assert abs(got[b, r, n] - want) <= 1e-12 * max(1.0, abs(want))


def test_gathered_linear_row_selection_commutes():
    # P_S (X W^T) = (P_S X) W^T: the selected rows of the dense layer
    rng = np.random.default_rng(4)
    X = rng.standard_normal((2, 40, 16))
    Wt = rng.standard_normal((24, 16))
    S = np.stack([np.sort(rng.choice(40, 11, replace=False)) for _ in range(2)])
    dense = O.gathered_linear(X, None, Wt, act="gelu_tanh")
    sel = O.gathered_linear(X, S, Wt, act="gelu_tanh")
    for b in range(2):
        assert np.allclose(sel[b], dense[b, S[b]], rtol=0, atol=1e-12)


def test_gelu_tanh_library_odd_part_and_exact_gelu():
    import torch
    x = np.linspace(-8.0, 8.0, 3201)
    g = O.gelu_tanh(x)
    lib = torch.nn.functional.gelu(torch.from_numpy(x), approximate="tanh").numpy()
    assert np.max(np.abs(g - lib)) <= 1e-12
    # odd part: gelu(x) - gelu(-x) = x for x * s(x) with s(x) + s(-x) = 1
    assert np.max(np.abs((g - O.gelu_tanh(-x)) - x)) <= 1e-12
    assert O.gelu_tanh(np.array([0.0]))[0] == 0.0
    # within 1e-3 of the exact x * Phi(x) everywhere (the approximation's
    # deviation is a few 1e-4 at most)
    exact = np.array([0.5 * v * (1.0 + math.erf(v / math.sqrt(2.0))) for v in x])
    assert np.max(np.abs(g - exact)) <= 1e-3
