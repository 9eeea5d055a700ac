"""GPU parity of the row-wise layers of the row-selective block (Eq. (13),
(15)): Y[b, r] = act(X[b, S[b, r]] W^T + bias), against the fp64 oracle,
through the C ABI."""

import numpy as np
import pytest
import torch

import oracle as O
from mask_free_b200 import ops, synth
from tests.helpers import to64

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(autouse=True)
def _status_clean():
    ops.device_status()
    yield


def _layer(B, N, d_in, d_out, seed, with_bias=True):
    X = synth.normal_bf16((B, N, d_in), seed)
    Wt = (synth.normal_bf16((d_out, d_in), seed + 1).float() / np.sqrt(d_in)).to(torch.bfloat16)
    bias = (0.1 * torch.randn(d_out, generator=torch.Generator().manual_seed(seed + 2))) if with_bias else None
    return X, Wt, bias


def _rows(B, N, k, seed):
    return np.stack([np.sort(np.random.default_rng(seed + b).choice(N, k, replace=False))
                     for b in range(B)]).astype(np.int32)


def _check(got, Xsel64, Wt64, bias64, act):
    """|GPU - oracle| per element within the bound of its arithmetic: the
    bf16 rounding of the result (2^-9 of it; 2^-8 taken) plus an fp32
    accumulation bound d_in 2^-24 sum_c |x_c w_c| (scaled by 1.13, GELU's
    largest slope, when it follows), and 1e-6 for tanh and the bias add."""
    ref = O.gathered_linear(Xsel64, None, Wt64, bias64, act)
    d_in = Wt64.shape[1]
    absprod = np.abs(Xsel64) @ np.abs(Wt64).T
    slope = 1.13 if act == "gelu_tanh" else 1.0
    tol = 2.0 ** -8 * np.abs(ref) + slope * d_in * 2.0 ** -24 * absprod + 1e-6
    g = to64(got)
    err = np.abs(g - ref)
    assert np.all(np.isfinite(g))
    assert np.all(err <= tol), (float(err.max()), float((err - tol).max()))
    assert err.mean() <= 2.0 ** -9 * np.abs(ref).mean() + 1e-6
    return ref


@pytest.mark.parametrize("B,N,d_in,d_out,k,act,with_bias", [
    (2, 300, 200, 264, 77, "none", True),          # ragged rows, K chunk and column tile
    (1, 1000, 2304, 512, 333, "gelu_tanh", True),  # the block's width
    (2, 129, 64, 256, None, "none", False),        # every row (dense block)
    (1, 50, 64, 8, 5, "gelu_tanh", True),          # one K chunk, fewer rows and columns than a tile
    (2, 4096, 128, 1000, 1229, "gelu_tanh", False),
    (2, 8192, 256, 2048, 4096, "gelu_tanh", True),  # 512 tiles: several per CTA, both accumulators
])
@pytest.mark.parametrize("compact_copy", [True, False])
def test_gather_linear_parity(B, N, d_in, d_out, k, act, with_bias, compact_copy):
    # compact_copy: the rows of S copied into the workspace first (the
    # default); else gathered by the GEMM itself (no workspace)
    if k is None and not compact_copy:
        pytest.skip("every row: no gather either way")
    X, Wt, bias = _layer(B, N, d_in, d_out, seed=N + d_out)
    S = _rows(B, N, k, seed=k) if k is not None else None
    got = ops.gather_linear(X.to(DEV), Wt.to(DEV), None if S is None else torch.from_numpy(S).to(DEV),
                            None if bias is None else bias.to(DEV), act=act, ws=None if compact_copy else False)
    X64 = to64(X)
    Xsel = X64 if S is None else np.stack([X64[b, S[b]] for b in range(B)])
    _check(got, Xsel, to64(Wt), None if bias is None else bias.numpy().astype(np.float64), act)
    assert ops.device_status() == 0


def test_gelu_over_the_whole_pre_activation_range():
    # pre-activations from -12 to 12 through the bias: GELU's tails (y -> -0
    # for very negative inputs, y -> x for large ones) against the oracle's
    # tanh form, on both kernels (every row: CTA pairs; rows of S gathered
    # by the GEMM: one CTA per tile)
    B, N, d_in, d_out = 1, 300, 64, 512
    X, Wt, _ = _layer(B, N, d_in, d_out, seed=31)
    bias = torch.linspace(-12.0, 12.0, d_out)
    Xd, Wd, bd = X.to(DEV), Wt.to(DEV), bias.to(DEV)
    S = _rows(B, N, 150, seed=4)
    X64 = to64(X)
    got = ops.gather_linear(Xd, Wd, bias=bd, act="gelu_tanh")
    _check(got, X64, to64(Wt), bias.numpy().astype(np.float64), "gelu_tanh")
    got = ops.gather_linear(Xd, Wd, S=torch.from_numpy(S).to(DEV), bias=bd, act="gelu_tanh", ws=False)
    _check(got, np.stack([X64[0, S[0]]]), to64(Wt), bias.numpy().astype(np.float64), "gelu_tanh")
    assert ops.device_status() == 0


def test_gathered_rows_equal_dense_rows_bitwise():
    B, N, d_in, d_out, k = 2, 700, 320, 520, 211
    X, Wt, bias = _layer(B, N, d_in, d_out, seed=17)
    Xd, Wd, bd = X.to(DEV), Wt.to(DEV), bias.to(DEV)
    S = torch.from_numpy(_rows(B, N, k, seed=3)).to(DEV)
    dense = ops.gather_linear(Xd, Wd, bias=bd, act="gelu_tanh")
    for ws in (None, False):  # compact copy first / gathered by the GEMM
        sel = ops.gather_linear(Xd, Wd, S=S, bias=bd, act="gelu_tanh", ws=ws)
        for b in range(B):
            assert torch.equal(sel[b], dense[b, S[b].long()])
        # rows in any order, repeated rows included
        Sr = torch.tensor([[5, 5, 699, 0], [3, 2, 1, 0]], dtype=torch.int32, device=DEV)
        sel = ops.gather_linear(Xd, Wd, S=Sr, bias=bd, act="gelu_tanh", ws=ws)
        for b in range(B):
            assert torch.equal(sel[b], dense[b, Sr[b].long()])
    assert ops.device_status() == 0


def test_gather_linear_block_width_full_size_sampled():
    # the benchmark's layer: 2 x 6400 sensitive rows of a 25600-token image,
    # width 2304 -> QKV 6912; sampled output rows against the oracle
    B, N, d_in, d_out, k = 2, 25600, 2304, 6912, 6400
    X, Wt, bias = _layer(B, N, d_in, d_out, seed=5)
    S = _rows(B, N, k, seed=11)
    got = ops.gather_linear(X.to(DEV), Wt.to(DEV), torch.from_numpy(S).to(DEV), bias.to(DEV))
    pick = np.random.default_rng(2).choice(k, 48, replace=False)
    Xsel = np.stack([to64(X[b, torch.from_numpy(S[b, pick]).long()]) for b in range(B)])
    _check(got[:, torch.from_numpy(pick).long().to(DEV)], Xsel, to64(Wt), bias.numpy().astype(np.float64), "none")
    assert ops.device_status() == 0


def test_gather_linear_out_of_range_row_flagged_not_faulted():
    B, N, d_in, d_out = 1, 200, 64, 64
    X, Wt, _ = _layer(B, N, d_in, d_out, seed=23)
    Xd, Wd = X.to(DEV), Wt.to(DEV)
    S = torch.tensor([[7, 200, -1, 3]], dtype=torch.int32, device=DEV)
    dense = ops.gather_linear(Xd, Wd)
    for ws in (None, False):  # compact copy first / gathered by the GEMM
        got = ops.gather_linear(Xd, Wd, S=S, ws=ws)
        assert ops.device_status() & (1 << ops.SAFE_ERR_DEVICE_CHECK)
        assert torch.equal(got[0, 0], dense[0, 7]) and torch.equal(got[0, 3], dense[0, 3])
        assert torch.equal(got[0, 1], dense[0, 0]) and torch.equal(got[0, 2], dense[0, 0])  # replaced by row 0
