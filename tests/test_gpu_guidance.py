"""GPU parity of the sensitivity field (Eq. (11)), the binary partition field
and sensitivity-weighted CFG (Eq. (20), (21)) against the fp64 oracle,
through the C ABI."""

import math

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
    assert ops.device_status() == 0


def _scores(B, N, seed):
    # PCSP-like scores: positive, smooth-ish variation plus noise
    rng = np.random.default_rng(seed)
    return (rng.random((B, N)) * 0.02 + 0.004).astype(np.float32)


# ---------------------------------------------------------------- Eq. (11)


def _field_tol(sc64, gh, gw, sigma):
    """Per-sample bound on |GPU - oracle| of the normalised field: fp32 taps
    and two passes of (2r+1)-term sums err by <= 2 (2r+1) u max|G*s| (u =
    2^-24) before Norm, which divides that by the field's range, so a
    strongly smoothed (nearly flat) field is the least well conditioned."""
    sm = O.smooth_scores(sc64, gh, gw, sigma)
    taps = O.gaussian_taps(sigma).size
    return [1e-6 + 2 * taps * 2.0 ** -24 * np.abs(sm[b]).max() / (sm[b].max() - sm[b].min())
            for b in range(sm.shape[0])]


@pytest.mark.parametrize("B,gh,gw,sigma", [(2, 64, 64, 1.5), (1, 40, 24, 2.5), (2, 9, 7, 7.0), (2, 33, 17, 0.0),
                                           (1, 160, 160, 2.0), (1, 1, 300, 3.0)])
def test_sensitivity_field_parity(B, gh, gw, sigma):
    sc = _scores(B, gh * gw, 101)
    got = ops.sensitivity_field(torch.from_numpy(sc).to(DEV), gh, gw, sigma).cpu().numpy()
    ref = O.sensitivity_field(sc.astype(np.float64), gh, gw, sigma)
    tol = _field_tol(sc.astype(np.float64), gh, gw, sigma)
    for b in range(B):
        assert np.max(np.abs(got[b] - ref[b])) <= tol[b], (b, np.max(np.abs(got[b] - ref[b])), tol[b])
        assert got[b].min() == 0.0 and got[b].max() == 1.0


def test_sensitivity_field_flat_and_impulse():
    flat = torch.full((1, 48), 0.37, device=DEV)
    assert torch.equal(ops.sensitivity_field(flat, 6, 8, 1.3), torch.zeros_like(flat))
    # interior impulse: normalised field equals the normalised 2-D Gaussian
    d = np.zeros((1, 33 * 33), dtype=np.float32)
    d[0, 16 * 33 + 16] = 1.0
    got = ops.sensitivity_field(torch.from_numpy(d).to(DEV), 33, 33, 1.5).cpu().numpy()
    np.testing.assert_allclose(got, O.sensitivity_field(d.astype(np.float64), 33, 33, 1.5), atol=1e-6)
    assert got[0, 16 * 33 + 16] == 1.0


def test_pcsp_smoothing_topk_pipeline():
    # PCSP scores on the GPU -> sensitivity field -> top-k: the GPU split is
    # exactly the oracle's top-k of the GPU's own field, and the field is
    # within tolerance of the oracle's field of the GPU's scores
    B, gh, gw, M, H, d, k = 2, 48, 40, 128, 4, 96, 577
    N = gh * gw
    Q = synth.normal_bf16((B, N, H, d), 111)
    Ky = synth.normal_bf16((B, M, H, d), 112)
    lens = torch.tensor([70, 128], dtype=torch.int32)
    w = synth.content_weights(lens, M, 113)
    sc, _, _ = ops.pcsp_topk(Q.to(DEV), Ky.to(DEV), lens.to(DEV), w.to(DEV))
    s = ops.sensitivity_field(sc, gh, gw, 2.0)
    S, C = ops.topk_partition(s, k)
    s_host = s.cpu().numpy().astype(np.float64)
    S_ref, C_ref = O.topk_partition(s_host, k)
    assert np.array_equal(S.cpu().numpy(), S_ref) and np.array_equal(C.cpu().numpy(), C_ref)
    sc64 = sc.cpu().numpy().astype(np.float64)
    ref = O.sensitivity_field(sc64, gh, gw, 2.0)
    tol = _field_tol(sc64, gh, gw, 2.0)
    for b in range(B):
        assert np.max(np.abs(s_host[b] - ref[b])) <= tol[b]


# ---------------------------------------------------------------- Eq. (20), (21)


def test_partition_indicator_exact_and_flagged():
    N = 1000
    rng = np.random.default_rng(7)
    S = np.stack([np.sort(rng.choice(N, 333, replace=False)) for _ in range(2)]).astype(np.int32)
    got = ops.partition_indicator(torch.from_numpy(S).to(DEV), N).cpu().numpy()
    assert np.array_equal(got, O.partition_indicator(S, N))
    bad = torch.tensor([[3, 2, 9]], dtype=torch.int32, device=DEV)  # not ascending
    ops.partition_indicator(bad, 16)
    torch.cuda.synchronize()
    assert ops.device_status() & (1 << ops.SAFE_ERR_DEVICE_CHECK)


def _cfg_inputs(B, N, C, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    fc = torch.randn((B, N, C), generator=g).to(dtype)
    fu = torch.randn((B, N, C), generator=g).to(dtype)
    s = torch.rand((B, N), generator=g)
    return fc, fu, s


@pytest.mark.parametrize("B,N,C", [(1, 25600, 16), (2, 999, 3), (2, 4096, 64)])
def test_sw_cfg_fp32_parity(B, N, C):
    fc, fu, s = _cfg_inputs(B, N, C, torch.float32, 201)
    out = ops.sw_cfg(fc.to(DEV), fu.to(DEV), s.to(DEV), 4.0, 7.5).cpu().numpy().astype(np.float64)
    ref = O.sw_cfg(fc.numpy(), fu.numpy(), s.numpy(), 4.0, 7.5)
    scale = np.abs(fu.numpy()) + 7.5 * np.abs(fc.numpy() - fu.numpy())
    assert np.all(np.abs(out - ref) <= 4e-7 * scale + 1e-30)


@pytest.mark.parametrize("B,N,C", [(1, 25600, 16), (2, 777, 12)])
def test_sw_cfg_bf16_parity(B, N, C):
    fc, fu, s = _cfg_inputs(B, N, C, torch.bfloat16, 202)
    out = ops.sw_cfg(fc.to(DEV), fu.to(DEV), s.to(DEV), 1.0, 5.0).cpu().float().numpy().astype(np.float64)
    ref = O.sw_cfg(to64(fc), to64(fu), s.numpy(), 1.0, 5.0)
    # one bf16 rounding of the fp32 result: within one bf16 step of the fp64 value
    assert np.all(np.abs(out - ref) <= 2.0 ** -7 * np.abs(ref) + 1e-6)


def test_sw_cfg_in_place_equal_scales_and_binary_variant():
    B, N, C = 2, 512, 8
    fc, fu, s = _cfg_inputs(B, N, C, torch.float32, 203)
    # in place on f_c
    want = ops.sw_cfg(fc.to(DEV), fu.to(DEV), s.to(DEV), 3.0, 6.0)
    buf = fc.to(DEV)
    ops.sw_cfg(buf, fu.to(DEV), s.to(DEV), 3.0, 6.0, out=buf)
    assert torch.equal(buf, want)
    # equal scales: standard CFG whatever s is
    a = ops.sw_cfg(fc.to(DEV), fu.to(DEV), s.to(DEV), 4.5, 4.5)
    b = ops.sw_cfg(fc.to(DEV), fu.to(DEV), torch.zeros_like(s).to(DEV), 4.5, 4.5)
    assert torch.equal(a, b)
    # binary variant: gamma_sens on S, gamma_ctx on C
    S = torch.stack([torch.sort(torch.randperm(N, generator=torch.Generator().manual_seed(b))[:100])[0]
                     for b in range(B)]).to(torch.int32)
    ind = ops.partition_indicator(S.to(DEV), N)
    out = ops.sw_cfg(fc.to(DEV), fu.to(DEV), ind, 2.0, 9.0).cpu().numpy().astype(np.float64)
    ref = O.sw_cfg(fc.numpy(), fu.numpy(), O.partition_indicator(S.numpy(), N), 2.0, 9.0)
    np.testing.assert_allclose(out, ref, rtol=1e-6, atol=1e-6)


def test_shared_cfg_pair_partition():
    # the conditional sample's split, applied to both halves of the pair;
    # bit-exact against the oracle's top-k of that sample's scores
    N, k = 3000, 751
    sc = torch.from_numpy(_scores(2, N, 301)).to(DEV)
    S, C = ops.shared_partition(sc, k)
    S_ref, C_ref = O.topk_partition(sc[:1].cpu().numpy().astype(np.float64), k)
    for b in range(2):
        assert np.array_equal(S[b].cpu().numpy(), S_ref[0]) and np.array_equal(C[b].cpu().numpy(), C_ref[0])
    # SRSU of both samples then gathers the same rows
    Sb, _ = ops.shared_partition(sc, k, sample=1)
    S1_ref, _ = O.topk_partition(sc[1:].cpu().numpy().astype(np.float64), k)
    assert np.array_equal(Sb[0].cpu().numpy(), S1_ref[0])

