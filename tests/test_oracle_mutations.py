"""Plant plausible mistakes in the oracle (on the CPU) and check that the pins
in test_oracle_pins.py catch every one of them."""

import math

import numpy as np
import pytest

import oracle.safe_oracle as S
import tests.test_oracle_pins as P


def _attention_no_scale(Q, K, V, scale, kv_len=None, q_rows=None, with_lse=False):
    return _ORIG["attention"](Q, K, V, 1.0, kv_len, q_rows, with_lse)


def _attention_left_padding(Q, K, V, scale, kv_len=None, q_rows=None, with_lse=False):
    if kv_len is None:
        return _ORIG["attention"](Q, K, V, scale, None, q_rows, with_lse)
    M = K.shape[1]
    Kf = np.flip(np.asarray(K, dtype=np.float64), axis=1)
    Vf = np.flip(np.asarray(V, dtype=np.float64), axis=1)
    return _ORIG["attention"](Q, Kf, Vf, scale, kv_len, q_rows, with_lse) if M else None


def _attention_swapped_qk(Q, K, V, scale, kv_len=None, q_rows=None, with_lse=False):
    # uses value rows as keys (a transposed/swapped operand)
    return _ORIG["attention"](Q, V, V, scale, kv_len, q_rows, with_lse)


def _softmax_no_exp(logits):
    e = logits - np.max(logits, axis=-1, keepdims=True) + 10.0
    return e / np.sum(e, axis=-1, keepdims=True)


def _ceil_k_floor(rho_num, rho_den, N):
    return (rho_num * N) // rho_den


def _topk_ties_high(scores, k):
    scores = np.asarray(scores, dtype=np.float64) + 0.0
    B, N = scores.shape
    Sx = np.zeros((B, k), dtype=np.int64)
    Cx = np.zeros((B, N - k), dtype=np.int64)
    for b in range(B):
        order = np.lexsort((-np.arange(N), -scores[b]))
        Sx[b] = np.sort(order[:k])
        Cx[b] = np.sort(order[k:])
    return Sx, Cx


def _row_in_R_no_finite(row, dtype_code):
    if dtype_code in (S.DTYPE_BOOL, S.DTYPE_U8):
        return bool(np.all(row != 0))
    return bool(np.all(row == row[0])) if row.size else True


def _pcsp_no_mean(Q, Ky, valid_len, w, scale, heads=None):
    H = np.asarray(Q).shape[2]
    return _ORIG["pcsp_scores"](Q, Ky, valid_len, w, scale, heads) * H


def _scatter_off_by_one(cache, src, Sidx, src_compact):
    out = np.array(cache, copy=True)
    if Sidx is None:
        out[...] = src
        return out
    for b in range(out.shape[0]):
        for r in range(Sidx.shape[1]):
            j = min(Sidx[b, r] + 1, out.shape[1] - 1)
            out[b, j] = src[b, r] if src_compact else src[b, Sidx[b, r]]
    return out


def _reflect_whole_sample(idx, n):
    # mirror about the edge sample itself (x1 x0 | x0 is not repeated): a
    # different border rule
    if n == 1:
        return np.zeros_like(np.asarray(idx))
    m = np.mod(np.asarray(idx), 2 * n - 2)
    return np.where(m < n, m, 2 * n - 2 - m)


def _taps_unnormalised(sigma, truncate=4.0):
    g = _ORIG["gaussian_taps"](sigma, truncate)
    return g / g.max()


def _smooth_swapped_axes(scores, grid_h, grid_w, sigma, truncate=4.0):
    # grid height and width exchanged (rows of the wrong length)
    return _ORIG["smooth_scores"](scores, grid_w, grid_h, sigma, truncate)


def _norm_no_min(x):
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    for b in range(x.shape[0]):
        hi = np.max(x[b])
        if hi != 0:
            out[b] = x[b] / hi
    return out


def _sw_cfg_swapped(f_c, f_u, s, gamma_ctx, gamma_sens):
    return _ORIG["sw_cfg"](f_u, f_c, s, gamma_ctx, gamma_sens)


def _sw_cfg_scales_swapped(f_c, f_u, s, gamma_ctx, gamma_sens):
    return _ORIG["sw_cfg"](f_c, f_u, s, gamma_sens, gamma_ctx)


def _indicator_complement(S, N):
    return 1.0 - _ORIG["partition_indicator"](S, N)


def _linear_transposed_weight(X, Sidx, Wt, bias=None, act="none"):
    return _ORIG["gathered_linear"](X, Sidx, np.asarray(Wt).T, bias, act)


def _linear_bias_after_activation(X, Sidx, Wt, bias=None, act="none"):
    y = _ORIG["gathered_linear"](X, Sidx, Wt, None, act)
    return y if bias is None else y + np.asarray(bias)[None, None, :]


def _linear_ignores_rows(X, Sidx, Wt, bias=None, act="none"):
    if Sidx is None:
        return _ORIG["gathered_linear"](X, None, Wt, bias, act)
    k = np.asarray(Sidx).shape[1]
    return _ORIG["gathered_linear"](np.asarray(X)[:, :k], None, Wt, bias, act)


def _gelu_cubic_coefficient_slip(x):
    x = np.asarray(x, dtype=np.float64)
    return 0.5 * x * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (x + 0.44715 * x ** 3)))


_ORIG = {n: getattr(S, n) for n in ("attention", "softmax_rows", "ceil_k", "topk_partition", "row_in_R",
                                    "pcsp_scores", "cache_scatter", "gaussian_taps", "smooth_scores", "sw_cfg",
                                    "partition_indicator", "gathered_linear")}

MUTATIONS = {
    "attention_no_scale": ("attention", _attention_no_scale),
    "attention_left_padding": ("attention", _attention_left_padding),
    "attention_swapped_operand": ("attention", _attention_swapped_qk),
    "softmax_without_exp": ("softmax_rows", _softmax_no_exp),
    "ceil_k_as_floor": ("ceil_k", _ceil_k_floor),
    "topk_ties_to_higher_index": ("topk_partition", _topk_ties_high),
    "classifier_ignores_nonfinite": ("row_in_R", _row_in_R_no_finite),
    "pcsp_missing_head_mean": ("pcsp_scores", _pcsp_no_mean),
    "scatter_off_by_one": ("cache_scatter", _scatter_off_by_one),
    "smoothing_whole_sample_reflection": ("reflect_index", _reflect_whole_sample),
    "smoothing_unnormalised_taps": ("gaussian_taps", _taps_unnormalised),
    "smoothing_swapped_grid_axes": ("smooth_scores", _smooth_swapped_axes),
    "norm_without_min": ("norm01", _norm_no_min),
    "sw_cfg_swapped_predictions": ("sw_cfg", _sw_cfg_swapped),
    "sw_cfg_swapped_scales": ("sw_cfg", _sw_cfg_scales_swapped),
    "indicator_complement": ("partition_indicator", _indicator_complement),
    "linear_transposed_weight": ("gathered_linear", _linear_transposed_weight),
    "linear_bias_after_activation": ("gathered_linear", _linear_bias_after_activation),
    "linear_ignores_selected_rows": ("gathered_linear", _linear_ignores_rows),
    "gelu_cubic_coefficient_slip": ("gelu_tanh", _gelu_cubic_coefficient_slip),
}


def _run_all_pins():
    """Run every pin; return the number that failed."""
    import json
    import os
    failures = 0
    golden = os.path.join(os.path.dirname(P.__file__), "golden")
    fns = [getattr(P, n) for n in dir(P) if n.startswith("test_")]
    for fn in fns:
        params = []
        if fn.__name__ == "test_sdpa_closed_form_golden":
            params = json.load(open(os.path.join(golden, "softmax_closed_form.json")))["cases"]
        elif fn.__name__ == "test_ceil_k_golden":
            params = json.load(open(os.path.join(golden, "topk_k_values.json")))["cases"]
        calls = [(c,) for c in params] if params else [()]
        for mark in getattr(fn, "pytestmark", []):
            if mark.name == "parametrize" and not params:
                multi = "," in mark.args[0]
                calls = [tuple(v) if multi else (v,) for v in mark.args[1]]
        for args in calls:
            try:
                fn(*args)
            except Exception:  # AssertionError or a crash both count as caught
                failures += 1
    return failures


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, monkeypatch):
    attr, bad = MUTATIONS[name]
    monkeypatch.setattr(S, attr, bad)
    # the package namespace re-exports the functions: patch it too
    import oracle
    monkeypatch.setattr(oracle, attr, bad)
    assert _run_all_pins() > 0, f"no pin caught the planted mistake {name}"


def test_pins_pass_unmutated():
    assert _run_all_pins() == 0
