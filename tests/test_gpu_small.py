"""GPU parity on small and edge-case inputs: every call of the C ABI against
the fp64 oracle (attention: max-abs 1e-2, mean-abs 1e-3, rel-RMS 1e-2;
classifier, top-k, scatter: bit-exact)."""

import math

import numpy as np
import pytest
import torch

import oracle as O
from mask_free_b200 import ops, synth
from tests.helpers import (assert_attn_close, bits, storage_view_for_oracle, to64, to_device_view)

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(autouse=True)
def _status_clean():
    ops.device_status()
    yield


def rnd_bf16(shape, seed):
    return synth.normal_bf16(shape, seed)


# ---------------------------------------------------------------- classifier


def oracle_classify(v_cpu, code):
    arr, sizes, strides, off = storage_view_for_oracle(v_cpu)
    return O.classify_mask(arr, code, sizes, strides, off)


CODES = {torch.bool: O.DTYPE_BOOL, torch.uint8: O.DTYPE_U8, torch.float32: O.DTYPE_F32,
         torch.float16: O.DTYPE_F16, torch.bfloat16: O.DTYPE_BF16}


def check_classify(v_cpu):
    want = oracle_classify(v_cpu, CODES[v_cpu.dtype])
    got = ops.mask_classify(to_device_view(v_cpu))
    assert got == want, (got, want)
    return got


def test_classify_tiny_masks():
    m = synth.tiny_masks(N=256, H=2, valid_len=11, M=16, seed=42)
    assert check_classify(m["all_true"]) == (1, 0, -1)
    assert check_classify(m["all_zero"]) == (1, 0, -1)
    assert check_classify(m["row_constant"]) == (1, 0, -1)
    assert check_classify(m["one_nonconstant_row"]) == (0, 1, m["_nonconst_row"])
    assert check_classify(m["text_padding"])[0] == 0
    assert check_classify(m["nan_entry"])[:2] == (0, 1)


@pytest.mark.parametrize("dtype", [torch.bool, torch.uint8, torch.float32, torch.float16, torch.bfloat16])
def test_classify_dtypes_strides_and_broadcast(dtype):
    g = torch.Generator().manual_seed(3)
    for trial in range(6):
        B, H, nq, nk = 2, 3, 37, 1 + int(torch.randint(1, 300, (1,), generator=g))
        if dtype in (torch.bool, torch.uint8):
            base = torch.ones((B, H, nq, nk + 5), dtype=torch.uint8)
            base[torch.rand(base.shape, generator=g) < 0.002] = 0
            base = base.to(dtype)
        else:
            c = torch.randn((B, H, nq, 1), generator=g) * 3
            base = c.expand(B, H, nq, nk + 5).contiguous()
            hit = torch.rand(base.shape, generator=g) < 0.001
            base[hit] = base[hit] + 0.5
            base = base.to(dtype)
            if trial == 1:
                base[0, 1, 5, 7] = float("inf")
            if trial == 2:
                base[1, 2, 9] = float("-inf")  # all -inf row: not removable
            if trial == 3:
                base[1, 0, 3] = 0.0
                base[1, 0, 3, ::2] = -0.0   # -0 == +0: removable
        views = [base[..., :nk], base[..., 3:3 + nk],  # unaligned row starts
                 base[:, :1].expand(B, H, nq, nk + 5)[..., :nk],  # stride-0 head dim
                 base.transpose(2, 3)[..., :nq][:, :, :nk],  # non-unit key stride
                 base[..., :1].expand(B, H, nq, nk)]  # key-broadcast rows
        for v in views:
            check_classify(v)


def test_classify_large_all_valid_with_planted_failures():
    N = 4096
    m = torch.ones((2, 1, N, N), dtype=torch.bool, device=DEV)
    assert ops.mask_classify(m) == (1, 0, -1)
    m[1, 0, 777, 4095] = False
    m[0, 0, 4000, 0] = False
    assert ops.mask_classify(m) == (0, 2, 4000)
    mf = torch.zeros((2, 24, 512, 4096), dtype=torch.bfloat16, device=DEV)
    assert ops.mask_classify(mf) == (1, 0, -1)
    mf[1, 23, 511, 17] = 1.0
    assert ops.mask_classify(mf) == (0, 1, (1 * 24 + 23) * 512 + 511)


# ---------------------------------------------------------------- attention


def rand_qkv(B, N, H, d, seed):
    return [rnd_bf16((B, N, H, d), seed + i) for i in range(3)]


@pytest.mark.parametrize("B,N,H,d", [(1, 256, 2, 64), (2, 384, 3, 96), (1, 512, 2, 128), (3, 200, 2, 96),
                                     (1, 129, 1, 64), (1, 1, 2, 96), (2, 1000, 1, 128), (1, 300, 4, 96)])
def test_attn_self_parity(B, N, H, d):
    Q, K, V = rand_qkv(B, N, H, d, seed=B * 1000 + N + d)
    scale = 1 / math.sqrt(d)
    out, lse = ops.attn_self(Q.to(DEV), K.to(DEV), V.to(DEV), return_lse=True)
    ref, ref_lse = O.attention(to64(Q), to64(K), to64(V), scale, with_lse=True)
    assert_attn_close(out, ref, f"self {B,N,H,d}")
    np.testing.assert_allclose(to64(lse), ref_lse, atol=2e-3, rtol=0)
    assert ops.device_status() == 0


def test_attn_self_scale_argument():
    Q, K, V = rand_qkv(1, 256, 2, 96, seed=77)
    out = ops.attn_self(Q.to(DEV), K.to(DEV), V.to(DEV), scale=0.37)
    assert_attn_close(out, O.attention(to64(Q), to64(K), to64(V), 0.37), "scale", magnitude_scaled=True)


def test_attn_self_row_constant_mask_elision_matches_masked_oracle():
    # Eq. (7)/(8): the mask-free GPU result equals the oracle WITH the
    # row-constant mask (applied literally, Eq. (2)).
    N, d = 256, 64
    Q, K, V = rand_qkv(1, N, 2, d, seed=5)
    m = synth.tiny_masks(N=N, H=2, valid_len=11, M=16, seed=42)["row_constant"].numpy()
    out = ops.attn_self(Q.to(DEV), K.to(DEV), V.to(DEV))
    for h in range(2):
        ref = O.sdpa_masked(to64(Q)[0, :, h], to64(K)[0, :, h], to64(V)[0, :, h], m[0, h].astype(np.float64))
        assert_attn_close(out[:, :, h:h + 1], ref[None, :, None, :], f"masked-oracle head {h}")


# ---------------------------------------------------------------- cross-attention


@pytest.mark.parametrize("B,N,M,H,d,lens", [(1, 256, 16, 2, 64, [11]), (2, 512, 128, 3, 96, [8, 128]),
                                            (2, 300, 256, 2, 96, [16, 256]), (3, 129, 100, 2, 128, [1, 33, 100]),
                                            (1, 64, 40, 1, 64, [32])])
def test_attn_cross_parity_and_padding(B, N, M, H, d, lens):
    Q = rnd_bf16((B, N, H, d), 11)
    Ky = rnd_bf16((B, M, H, d), 12)
    Vy = rnd_bf16((B, M, H, d), 13)
    L = torch.tensor(lens, dtype=torch.int32)
    scale = 1 / math.sqrt(d)
    out = ops.attn_cross(Q.to(DEV), Ky.to(DEV), Vy.to(DEV), L.to(DEV))
    ref = O.cross_attention(to64(Q), to64(Ky), to64(Vy), lens, scale)
    assert_attn_close(out, ref, "cross")
    # padding rows poisoned with NaN / huge values: bitwise the same output
    Kp, Vp = Ky.clone(), Vy.clone()
    for b, l in enumerate(lens):
        Kp[b, l:] = float("nan")
        Vp[b, l:] = 1e30
    out2 = ops.attn_cross(Q.to(DEV), Kp.to(DEV), Vp.to(DEV), L.to(DEV))
    assert torch.isfinite(out2.float()).all()
    assert np.array_equal(bits(out), bits(out2))
    assert ops.device_status() == 0


def test_attn_cross_single_valid_key_returns_value_row():
    Q = rnd_bf16((2, 256, 2, 96), 21)
    Ky = rnd_bf16((2, 128, 2, 96), 22)
    Vy = rnd_bf16((2, 128, 2, 96), 23)
    L = torch.tensor([1, 1], dtype=torch.int32)
    out = ops.attn_cross(Q.to(DEV), Ky.to(DEV), Vy.to(DEV), L.to(DEV)).cpu()
    for b in range(2):
        for h in range(2):
            assert torch.equal(out[b, :, h], Vy[b, 0, h].expand(256, 96))


def test_attn_cross_row_selection_equals_dense_rows():
    B, N, M, H, d = 2, 640, 128, 2, 96
    Q = rnd_bf16((B, N, H, d), 31)
    Ky, Vy = rnd_bf16((B, M, H, d), 32), rnd_bf16((B, M, H, d), 33)
    L = torch.tensor([50, 128], dtype=torch.int32, device=DEV)
    S = torch.stack([torch.from_numpy(np.sort(np.random.default_rng(b).choice(N, 301, replace=False)))
                     for b in range(B)]).to(torch.int32)
    dense = ops.attn_cross(Q.to(DEV), Ky.to(DEV), Vy.to(DEV), L)
    sel = ops.attn_cross(Q.to(DEV), Ky.to(DEV), Vy.to(DEV), L, q_idx=S.to(DEV))
    for b in range(B):
        assert torch.equal(sel[b].cpu(), dense[b, S[b].long()].cpu())
    ref = O.cross_attention(to64(Q), to64(Ky), to64(Vy), [50, 128], 1 / math.sqrt(d), q_rows=S.numpy())
    assert_attn_close(sel, ref, "cross rows")


# More (b, h) pairs than SMs: one CTA per (b, h) streams every query tile of
# its head, so the query-slot ring wraps several times and both softmax
# warpgroups see several tiles (odd and even counts, both softmax forms).
@pytest.mark.parametrize("B,N,M,H,d,lens,rows", [(2, 2000, 128, 80, 96, [77, 128], None),
                                                 (1, 1700, 256, 150, 128, [200], None),
                                                 (2, 3000, 128, 80, 64, [8, 96], 1500),
                                                 (1, 2200, 40, 160, 96, [33], 1111)])
def test_attn_cross_many_tiles_per_cta(B, N, M, H, d, lens, rows):
    Q = rnd_bf16((B, N, H, d), 71)
    Ky, Vy = rnd_bf16((B, M, H, d), 72), rnd_bf16((B, M, H, d), 73)
    L = torch.tensor(lens, dtype=torch.int32, device=DEV)
    S = None
    if rows is not None:
        S = torch.stack([torch.from_numpy(np.sort(np.random.default_rng(70 + b).choice(N, rows, replace=False)))
                         for b in range(B)]).to(torch.int32)
    out = ops.attn_cross(Q.to(DEV), Ky.to(DEV), Vy.to(DEV), L, q_idx=None if S is None else S.to(DEV))
    torch.cuda.synchronize()
    assert ops.device_status() == 0  # no wait of the pipeline ran out
    ref = O.cross_attention(to64(Q), to64(Ky), to64(Vy), lens, 1 / math.sqrt(d),
                            q_rows=None if S is None else S.numpy())
    # valid lengths from 8 keys, the workloads' shortest text: the plain bar
    assert_attn_close(out, ref, "cross many tiles")


def test_attn_cross_very_short_text_magnitude_bar():
    """Valid lengths below the workloads' minimum of 8 (5 keys): the softmax
    averages so few values that output rows reach magnitude ~4, where half a
    bf16 step of the output alone is ~1e-2. This case (and only the scale
    test above) takes the absolute bounds times the output magnitude."""
    B, N, M, H, d, lens = 2, 3000, 128, 80, 64, [5, 96]
    Q = rnd_bf16((B, N, H, d), 74)
    Ky, Vy = rnd_bf16((B, M, H, d), 75), rnd_bf16((B, M, H, d), 76)
    L = torch.tensor(lens, dtype=torch.int32, device=DEV)
    out = ops.attn_cross(Q.to(DEV), Ky.to(DEV), Vy.to(DEV), L)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    ref = O.cross_attention(to64(Q), to64(Ky), to64(Vy), lens, 1 / math.sqrt(d))
    assert_attn_close(out, ref, "cross with 5 valid keys", magnitude_scaled=True)


def test_pcsp_scores_many_tiles_per_cta():
    B, N, M, H, d = 2, 2000, 128, 80, 96
    Q = rnd_bf16((B, N, H, d), 81)
    Ky = rnd_bf16((B, M, H, d), 82)
    lens = [100, 17]
    w = synth.content_weights(torch.tensor(lens), M, 83)
    sc, _, _ = ops.pcsp_topk(Q.to(DEV), Ky.to(DEV), torch.tensor(lens, dtype=torch.int32, device=DEV), w.to(DEV))
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    ref = O.pcsp_scores(to64(Q), to64(Ky), lens, w.numpy().astype(np.float64), 1 / math.sqrt(d))
    np.testing.assert_allclose(sc.cpu().numpy(), ref, rtol=2e-5, atol=1e-8)


def test_attn_cross_invalid_length_is_flagged_not_faulted():
    Q = rnd_bf16((1, 128, 1, 64), 1).to(DEV)
    Ky = rnd_bf16((1, 16, 1, 64), 2).to(DEV)
    out = ops.attn_cross(Q, Ky, Ky, torch.tensor([0], dtype=torch.int32, device=DEV))
    torch.cuda.synchronize()
    assert ops.device_status() & (1 << ops.SAFE_ERR_DEVICE_CHECK)
    assert torch.isfinite(out.float()).all()


# ---------------------------------------------------------------- PCSP and top-k


def test_pcsp_scores_parity_uniform_and_accumulate():
    B, N, M, H, d = 2, 512, 64, 3, 96
    Q = rnd_bf16((B, N, H, d), 41)
    Ky = rnd_bf16((B, M, H, d), 42)
    lens = [9, 64]
    L = torch.tensor(lens, dtype=torch.int32, device=DEV)
    w = synth.content_weights(torch.tensor(lens), M, 43)
    scale = 1 / math.sqrt(d)
    sc, _, _ = ops.pcsp_topk(Q.to(DEV), Ky.to(DEV), L, w.to(DEV))
    ref = O.pcsp_scores(to64(Q), to64(Ky), lens, w.numpy().astype(np.float64), scale)
    np.testing.assert_allclose(sc.cpu().numpy(), ref, rtol=2e-5, atol=1e-8)
    # accumulate: two identical calls give exactly twice the scores
    sc2 = sc.clone()
    ops.pcsp_topk(Q.to(DEV), Ky.to(DEV), L, w.to(DEV), scores=sc2, accumulate=True)
    assert torch.equal(sc2, sc * 2)
    # uniform weights over valid keys: every score is 1/len (closed form)
    su, _, _ = ops.pcsp_topk(Q.to(DEV), Ky.to(DEV), L, None)
    for b, l in enumerate(lens):
        np.testing.assert_allclose(su[b].cpu().numpy(), 1.0 / l, rtol=1e-5)
    # padding keys do not matter
    Kp = Ky.clone()
    Kp[0, 9:] = float("nan")
    sp, _, _ = ops.pcsp_topk(Q.to(DEV), Kp.to(DEV), L, w.to(DEV))
    assert torch.equal(sp, sc)


def test_fused_cross_pcsp_equals_separate_calls_bitwise():
    B, N, M, H, d, k = 2, 1000, 128, 3, 96, 301
    Q = rnd_bf16((B, N, H, d), 51)
    Ky, Vy = rnd_bf16((B, M, H, d), 52), rnd_bf16((B, M, H, d), 53)
    lens = torch.tensor([29, 128], dtype=torch.int32, device=DEV)
    w = synth.content_weights(lens.cpu(), M, 54).to(DEV)
    Qd, Kd, Vd = Q.to(DEV), Ky.to(DEV), Vy.to(DEV)
    O_sep = ops.attn_cross(Qd, Kd, Vd, lens)
    sc_sep, S_sep, C_sep = ops.pcsp_topk(Qd, Kd, lens, w, k=k)
    O_f, sc_f, S_f, C_f = ops.attn_cross_pcsp(Qd, Kd, Vd, lens, w, k=k)
    assert torch.equal(O_f, O_sep) and torch.equal(sc_f, sc_sep)
    assert torch.equal(S_f, S_sep) and torch.equal(C_f, C_sep)
    # and against the oracle
    ref = O.pcsp_scores(to64(Q), to64(Ky), [29, 128], w.cpu().numpy().astype(np.float64), 1 / math.sqrt(d))
    np.testing.assert_allclose(sc_f.cpu().numpy(), ref, rtol=2e-5, atol=1e-8)
    assert_attn_close(O_f, O.cross_attention(to64(Q), to64(Ky), to64(Vy), [29, 128], 1 / math.sqrt(d)), "fused")
    assert ops.device_status() == 0


def _valid_topk(S, C, scores64, k, tol):
    S, C = S.cpu().numpy(), C.cpu().numpy()
    for b in range(S.shape[0]):
        assert np.all(np.diff(S[b]) > 0) and np.all(np.diff(C[b]) > 0)
        assert np.array_equal(np.sort(np.r_[S[b], C[b]]), np.arange(scores64.shape[1]))
        sel = np.zeros(scores64.shape[1], dtype=bool)
        sel[S[b]] = True
        if 0 < k < scores64.shape[1]:
            assert scores64[b][sel].min() >= scores64[b][~sel].max() - tol


def test_pcsp_topk_pipeline_valid_against_oracle_scores():
    B, N, M, H, d, k = 2, 1024, 128, 4, 96, 307
    Q = rnd_bf16((B, N, H, d), 51)
    Ky = rnd_bf16((B, M, H, d), 52)
    lens = [77, 128]
    w = synth.content_weights(torch.tensor(lens), M, 53)
    sc, S, C = ops.pcsp_topk(Q.to(DEV), Ky.to(DEV), torch.tensor(lens, dtype=torch.int32, device=DEV),
                             w.to(DEV), k=k)
    ref = O.pcsp_scores(to64(Q), to64(Ky), lens, w.numpy().astype(np.float64), 1 / math.sqrt(d))
    _valid_topk(S, C, ref, k, tol=1e-5 * np.abs(ref).max())
    S_ref, _ = O.topk_partition(ref, k)
    agree = np.mean([len(set(S[b].cpu().numpy()) & set(S_ref[b])) / k for b in range(B)])
    assert agree > 0.99


@pytest.mark.parametrize("B,N,k,kind", [(2, 4096, 1229, "normal"), (3, 1000, 1, "ties"), (1, 777, 777, "normal"),
                                        (2, 36864, 7373, "ties"), (1, 1, 1, "normal"), (2, 2049, 1024, "zeros"),
                                        (1, 5000, 2500, "signed_zero"), (2, 25600, 6400, "few_values"),
                                        (1, 40960, 10240, "normal"), (2, 40961, 9999, "ties"),
                                        (1, 65536, 16384, "few_values")])
def test_topk_partition_bit_exact(B, N, k, kind):
    """Keys in shared memory up to N = 40960, read from global memory above."""
    rng = np.random.default_rng(N + k)
    if kind == "normal":
        s = rng.standard_normal((B, N)).astype(np.float32)
    elif kind == "ties":
        s = rng.integers(0, 7, size=(B, N)).astype(np.float32) / 8
    elif kind == "zeros":
        s = np.zeros((B, N), dtype=np.float32)
    elif kind == "signed_zero":
        s = np.where(rng.random((B, N)) < 0.5, -0.0, 0.0).astype(np.float32)
        s[:, ::97] = -1e-30
    else:
        s = rng.choice(np.array([-3.5, 0.25, 1e-3, 7.0], dtype=np.float32), size=(B, N))
    S, C = ops.topk_partition(torch.from_numpy(s).to(DEV), k)
    S_ref, C_ref = O.topk_partition(s.astype(np.float64), k)
    assert np.array_equal(S.cpu().numpy(), S_ref)
    assert np.array_equal(C.cpu().numpy(), C_ref)


def test_topk_nan_is_flagged():
    s = torch.zeros((1, 100), device=DEV)
    s[0, 5] = float("nan")
    ops.topk_partition(s, 10)
    assert ops.device_status() & (1 << ops.SAFE_ERR_DEVICE_CHECK)


# ---------------------------------------------------------------- cache scatter


@pytest.mark.parametrize("compact", [True, False])
def test_cache_scatter_bit_exact(compact):
    B, N, H, d, k = 2, 1000, 3, 96, 333
    cache_k, cache_v = rnd_bf16((B, N, H, d), 61), rnd_bf16((B, N, H, d), 62)
    S = np.stack([np.sort(np.random.default_rng(b + 7).choice(N, k, replace=False)) for b in range(B)])
    rows = k if compact else N
    src_k, src_v = rnd_bf16((B, rows, H, d), 63), rnd_bf16((B, rows, H, d), 64)
    Kc, Vc = cache_k.to(DEV), cache_v.to(DEV)
    ops.ctx_cache_scatter(src_k.to(DEV), src_v.to(DEV), torch.from_numpy(S.astype(np.int32)).to(DEV), Kc, Vc,
                          src_compact=compact)
    shape = (B, N, H, d)
    want_k = O.cache_scatter(synth.bf16_bits(cache_k).reshape(shape),
                             synth.bf16_bits(src_k).reshape(src_k.shape), S, compact)
    want_v = O.cache_scatter(synth.bf16_bits(cache_v).reshape(shape),
                             synth.bf16_bits(src_v).reshape(src_v.shape), S, compact)
    assert np.array_equal(synth.bf16_bits(Kc.cpu()).reshape(shape), want_k)
    assert np.array_equal(synth.bf16_bits(Vc.cpu()).reshape(shape), want_v)
    assert ops.device_status() == 0


def test_cache_full_refresh_and_bad_indices():
    B, N, H, d = 2, 500, 2, 64
    src_k, src_v = rnd_bf16((B, N, H, d), 71).to(DEV), rnd_bf16((B, N, H, d), 72).to(DEV)
    Kc, Vc = torch.zeros_like(src_k), torch.zeros_like(src_v)
    ops.ctx_cache_scatter(src_k, src_v, None, Kc, Vc)
    assert torch.equal(Kc, src_k) and torch.equal(Vc, src_v)
    # an out-of-range index is skipped and flagged; the other rows still land
    S = torch.tensor([[3, 10, 600], [0, 1, 499]], dtype=torch.int32, device=DEV)
    Kc2, Vc2 = torch.zeros_like(src_k), torch.zeros_like(src_v)
    ops.ctx_cache_scatter(src_k, src_v, S, Kc2, Vc2, src_compact=False)
    assert ops.device_status() & (1 << ops.SAFE_ERR_DEVICE_CHECK)
    assert torch.equal(Kc2[0, 10], src_k[0, 10]) and torch.equal(Kc2[1, 499], src_k[1, 499])
    assert torch.count_nonzero(Kc2[0, 11:]) == 0


# ---------------------------------------------------------------- SRSU


@pytest.mark.parametrize("B,N,H,d,k", [(1, 256, 2, 64, 64), (2, 512, 3, 96, 200), (2, 1000, 2, 128, 333),
                                       (1, 384, 2, 96, 1), (1, 300, 2, 96, 300)])
def test_srsu_parity_gather_and_compact(B, N, H, d, k):
    Q, K, V = rand_qkv(B, N, H, d, seed=N + k)
    Kc = synth.drifted_bf16(K, 0.05, 9)
    Vc = synth.drifted_bf16(V, 0.05, 10)
    S = np.stack([np.sort(np.random.default_rng(b + N).choice(N, k, replace=False)) for b in range(B)])
    Sd = torch.from_numpy(S.astype(np.int32)).to(DEV)
    scale = 1 / math.sqrt(d)
    out, lse = ops.srsu_attn(Q.to(DEV), Sd, Kc.to(DEV), Vc.to(DEV), return_lse=True)
    ref, ref_lse = O.attention(to64(Q), to64(Kc), to64(Vc), scale, q_rows=S, with_lse=True)
    assert_attn_close(out, ref, "srsu")
    np.testing.assert_allclose(to64(lse), ref_lse, atol=2e-3, rtol=0)
    Qc = torch.stack([Q[b, S[b]] for b in range(B)]).contiguous()
    out_c = ops.srsu_attn(Qc.to(DEV), Sd, Kc.to(DEV), Vc.to(DEV), q_compact=True)
    assert torch.equal(out_c, out)
    assert ops.device_status() == 0


def test_srsu_all_rows_equals_dense_bitwise():
    B, N, H, d = 2, 512, 2, 96
    Q, K, V = rand_qkv(B, N, H, d, seed=88)
    Qd, Kd, Vd = Q.to(DEV), K.to(DEV), V.to(DEV)
    S = torch.arange(N, dtype=torch.int32, device=DEV).expand(B, N).contiguous()
    assert torch.equal(ops.srsu_attn(Qd, S, Kd, Vd), ops.attn_self(Qd, Kd, Vd))
    # unchanged context: SRSU rows equal the dense rows of S
    Ss = torch.tensor([[0, 5, 77, 300, 511], [1, 2, 3, 128, 256]], dtype=torch.int32, device=DEV)
    dense = ops.attn_self(Qd, Kd, Vd)
    sr = ops.srsu_attn(Qd, Ss, Kd, Vd)
    for b in range(B):
        assert torch.equal(sr[b], dense[b, Ss[b].long()])


def test_srsu_bad_index_flagged():
    Q = rnd_bf16((1, 256, 1, 64), 1).to(DEV)
    S = torch.tensor([[0, 3, 999]], dtype=torch.int32, device=DEV)
    ops.srsu_attn(Q, S, Q, Q)
    assert ops.device_status() & (1 << ops.SAFE_ERR_DEVICE_CHECK)


@pytest.mark.parametrize("B,N,H,d,k", [(1, 4096, 2, 96, 4096), (2, 3000, 3, 64, 1500), (1, 4096, 1, 128, 777),
                                       (2, 4096, 3, 96, 1229)])
def test_key_split_wave_balancing_matches_oracle(B, N, H, d, k):
    # the last partial wave of CTAs is split along the keys and merged by
    # the last part; the workspace needs no initialisation (filled with NaN)
    Q, K, V = rand_qkv(B, N, H, d, seed=N + 3 * k)
    Qd, Kd, Vd = Q.to(DEV), K.to(DEV), V.to(DEV)
    nbytes = ops.attn_workspace_bytes(B, k, N, H, d)
    assert nbytes > 0
    ws = torch.full((nbytes // 4,), float("nan"), dtype=torch.float32, device=DEV).view(torch.uint8)
    scale = 1 / math.sqrt(d)
    if k == N:
        out, lse = ops.attn_self(Qd, Kd, Vd, return_lse=True, ws=ws)
        out_whole, lse_whole = ops.attn_self(Qd, Kd, Vd, return_lse=True, ws=False)
        ref, ref_lse = O.attention(to64(Q), to64(K), to64(V), scale, with_lse=True)
    else:
        S = np.stack([np.sort(np.random.default_rng(b + 5).choice(N, k, replace=False)) for b in range(B)])
        Sd = torch.from_numpy(S.astype(np.int32)).to(DEV)
        out, lse = ops.srsu_attn(Qd, Sd, Kd, Vd, return_lse=True, ws=ws)
        out_whole, lse_whole = ops.srsu_attn(Qd, Sd, Kd, Vd, return_lse=True, ws=False)
        ref, ref_lse = O.attention(to64(Q), to64(K), to64(V), scale, q_rows=S, with_lse=True)
    assert_attn_close(out, ref, "split")
    assert_attn_close(out_whole, ref, "whole")
    np.testing.assert_allclose(to64(lse), ref_lse, atol=2e-3, rtol=0)
    np.testing.assert_allclose(to64(lse_whole), ref_lse, atol=2e-3, rtol=0)
    # a second call reuses the workspace
    out2 = ops.attn_self(Qd, Kd, Vd, ws=ws) if k == N else ops.srsu_attn(Qd, Sd, Kd, Vd, ws=ws)
    assert torch.equal(out2, out)
    assert ops.device_status() == 0


@pytest.mark.parametrize("B,N,H,d,k", [(2, 4096, 3, 96, 1229), (1, 1000, 2, 64, 333), (2, 700, 2, 128, 700)])
def test_srsu_compact_query_copy_is_bit_identical(B, N, H, d, k):
    # with room for the compact query rows the entry point copies the rows of
    # S out of Q first and loads compact tiles; the attention-only workspace
    # and no workspace gather them in the kernel: the same bits either way,
    # and the same as a caller-compacted Q
    Q, K, V = rand_qkv(B, N, H, d, seed=2 * N + k)
    Qd, Kd, Vd = Q.to(DEV), K.to(DEV), V.to(DEV)
    S = np.stack([np.sort(np.random.default_rng(b + 11).choice(N, k, replace=False)) for b in range(B)])
    Sd = torch.from_numpy(S.astype(np.int32)).to(DEV)
    full = ops.srsu_workspace_bytes(B, k, N, H, d)
    split = ops.attn_workspace_bytes(B, k, N, H, d)
    assert full >= split + B * k * H * d * 2
    ws = torch.full((full // 4,), float("nan"), dtype=torch.float32, device=DEV).view(torch.uint8)
    out_copy = ops.srsu_attn(Qd, Sd, Kd, Vd, ws=ws)
    out_gather = ops.srsu_attn(Qd, Sd, Kd, Vd, ws=ws[:max(split, 1)] if split else False)
    out_none = ops.srsu_attn(Qd, Sd, Kd, Vd, ws=False)
    Qc = torch.stack([Qd[b, Sd[b].long()] for b in range(B)]).contiguous()
    out_caller = ops.srsu_attn(Qc, Sd, Kd, Vd, q_compact=True, ws=ws)
    assert torch.equal(out_copy, out_gather) and torch.equal(out_copy, out_caller)
    if split == 0:
        assert torch.equal(out_copy, out_none)
    ref = O.attention(to64(Q), to64(K), to64(V), 1 / math.sqrt(d), q_rows=S)
    assert_attn_close(out_copy, ref, "srsu, compact query copy")
    assert ops.device_status() == 0


# ---------------------------------------------------------------- failure detection


def test_bounded_wait_timeout_reports_status():
    ops.selftest_wait_timeout(2_000_000)  # 2 ms limit on a barrier nothing arrives on
    st = ops.device_status()
    assert st & (1 << ops.SAFE_ERR_TIMEOUT)
    assert ops.device_status() == 0  # the read cleared it
    # the context is still usable
    Q = rnd_bf16((1, 128, 1, 64), 3).to(DEV)
    out = ops.attn_self(Q, Q, Q)
    assert torch.isfinite(out.float()).all() and ops.device_status() == 0


def test_invalid_arguments_raise():
    Q = rnd_bf16((1, 128, 1, 80), 3).to(DEV)
    with pytest.raises(ops.SafeError) as e:
        ops.attn_self(Q, Q, Q)
    assert e.value.status == ops.SAFE_ERR_UNSUPPORTED
    x = torch.empty((0, 128, 1, 64), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(ops.SafeError) as e:
        ops.attn_self(x, x, x)
    assert e.value.status == ops.SAFE_ERR_INVALID_ARG
