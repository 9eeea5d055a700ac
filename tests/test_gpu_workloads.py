"""GPU parity on the Lumina-Next-scale workloads.

N = 4096 (dense block, SRSU step): full comparison of every output;
N = 25600 / 36864: 512 seeded sampled query rows per head for the attention
outputs, whole-buffer bitwise checks for the cache, and the 20-call anchor /
SRSU sequence at N = 36864 replayed by the oracle.
The partition S used by the GPU calls is the oracle's own (from its fp64 PCSP
scores); the GPU's PCSP split is checked separately for validity.
"""

import math

import numpy as np
import pytest
import torch

import oracle as O
from mask_free_b200 import ops, synth
from tests.helpers import assert_attn_close, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"
SAMPLE = 512


@pytest.fixture(autouse=True)
def _status_clean():
    ops.device_status()
    yield
    assert ops.device_status() == 0


def load(workload):
    s = synth.WORKLOADS[workload]
    inp = synth.make_inputs(workload)
    host64 = {n: synth.bf16_to_f64(inp[n]) for n in ("Q", "K", "V", "Ky", "Vy", "Kc", "Vc")}
    dev = {n: v.to(DEV) for n, v in inp.items()}
    return s, inp, host64, dev


def oracle_partition(s, inp, h64, scale):
    lens = inp["valid_len"].numpy()
    sc = O.pcsp_scores(h64["Q"], h64["Ky"], lens, inp["w"].numpy().astype(np.float64), scale)
    S, C = O.topk_partition(sc, s.k)
    return sc, S, C


def check_gpu_partition(s, dev, ref_scores):
    sc, S, C = ops.pcsp_topk(dev["Q"], dev["Ky"], dev["valid_len"], dev["w"], k=s.k)
    np.testing.assert_allclose(sc.cpu().numpy(), ref_scores, rtol=3e-5, atol=1e-8)
    S, C = S.cpu().numpy(), C.cpu().numpy()
    tol = 3e-5 * np.abs(ref_scores).max()
    for b in range(s.B):
        assert np.all(np.diff(S[b]) > 0) and np.all(np.diff(C[b]) > 0)
        sel = np.zeros(s.N, dtype=bool)
        sel[S[b]] = True
        assert sel.sum() == s.k and not np.any(sel[C[b]])
        assert ref_scores[b][sel].min() >= ref_scores[b][~sel].max() - tol


@pytest.mark.parametrize("workload", ["n4096", "n4096_srsu"])
def test_n4096_full(workload):
    s, inp, h, d = load(workload)
    scale = 1 / math.sqrt(s.d)
    lens = inp["valid_len"].numpy()
    if workload == "n4096":
        assert_attn_close(ops.attn_self(d["Q"], d["K"], d["V"]), O.attention(h["Q"], h["K"], h["V"], scale),
                          "n4096 self")
        assert_attn_close(ops.attn_cross(d["Q"], d["Ky"], d["Vy"], d["valid_len"]),
                          O.cross_attention(h["Q"], h["Ky"], h["Vy"], lens, scale), "n4096 cross")
        mask = torch.ones((s.B, 1, s.N, s.N), dtype=torch.bool, device=DEV)
        assert ops.mask_classify(mask) == (1, 0, -1)
        return
    ref_scores, S_ref, _ = oracle_partition(s, inp, h, scale)
    check_gpu_partition(s, d, ref_scores)
    S_dev = torch.from_numpy(S_ref.astype(np.int32)).to(DEV)
    # sensitive rows of the current K/V go into the drifted cache (Eq. (16))
    Kc, Vc = d["Kc"].clone(), d["Vc"].clone()
    ops.ctx_cache_scatter(d["K"], d["V"], S_dev, Kc, Vc, src_compact=False)
    shape = tuple(inp["K"].shape)
    Kc_ref = O.cache_scatter(synth.bf16_bits(inp["Kc"]).reshape(shape), synth.bf16_bits(inp["K"]).reshape(shape),
                             S_ref, False)
    Vc_ref = O.cache_scatter(synth.bf16_bits(inp["Vc"]).reshape(shape), synth.bf16_bits(inp["V"]).reshape(shape),
                             S_ref, False)
    assert np.array_equal(synth.bf16_bits(Kc.cpu()).reshape(shape), Kc_ref)
    assert np.array_equal(synth.bf16_bits(Vc.cpu()).reshape(shape), Vc_ref)
    out = ops.srsu_attn(d["Q"], S_dev, Kc, Vc)
    assert_attn_close(out, O.srsu_attention(h["Q"], S_ref, O.bf16_bits_to_f64(Kc_ref), O.bf16_bits_to_f64(Vc_ref),
                                            scale), "n4096 srsu")
    outx = ops.attn_cross(d["Q"], d["Ky"], d["Vy"], d["valid_len"], q_idx=S_dev)
    assert_attn_close(outx, O.cross_attention(h["Q"], h["Ky"], h["Vy"], lens, scale, q_rows=S_ref), "n4096 cross S")


def test_n25600_sampled():
    s, inp, h, d = load("n25600")
    scale = 1 / math.sqrt(s.d)
    lens = inp["valid_len"].numpy()
    rows = synth.sample_rows(s.N, SAMPLE, seed=4004)
    # dense anchor self-attention
    out = ops.attn_self(d["Q"], d["K"], d["V"])
    assert_attn_close(out[:, rows], O.attention(h["Q"], h["K"], h["V"], scale, q_rows=rows), "n25600 self")
    del out
    # cross-attention
    outx = ops.attn_cross(d["Q"], d["Ky"], d["Vy"], d["valid_len"])
    assert_attn_close(outx[:, rows], O.cross_attention(h["Q"], h["Ky"], h["Vy"], lens, scale, q_rows=rows),
                      "n25600 cross")
    del outx
    # PCSP -> (oracle) partition -> scatter -> SRSU over the drifted cache
    ref_scores, S_ref, _ = oracle_partition(s, inp, h, scale)
    check_gpu_partition(s, d, ref_scores)
    S_dev = torch.from_numpy(S_ref.astype(np.int32)).to(DEV)
    Kc, Vc = d["Kc"].clone(), d["Vc"].clone()
    ops.ctx_cache_scatter(d["K"], d["V"], S_dev, Kc, Vc, src_compact=False)
    shape = tuple(inp["K"].shape)
    Kc_ref = O.cache_scatter(synth.bf16_bits(inp["Kc"]).reshape(shape), synth.bf16_bits(inp["K"]).reshape(shape),
                             S_ref, False)
    Vc_ref = O.cache_scatter(synth.bf16_bits(inp["Vc"]).reshape(shape), synth.bf16_bits(inp["V"]).reshape(shape),
                             S_ref, False)
    assert np.array_equal(synth.bf16_bits(Kc.cpu()).reshape(shape), Kc_ref)
    assert np.array_equal(synth.bf16_bits(Vc.cpu()).reshape(shape), Vc_ref)
    out = ops.srsu_attn(d["Q"], S_dev, Kc, Vc)
    rsel = synth.sample_rows(s.k, SAMPLE, seed=4005)
    ref = O.attention(h["Q"], O.bf16_bits_to_f64(Kc_ref), O.bf16_bits_to_f64(Vc_ref), scale,
                      q_rows=S_ref[:, rsel])
    assert_attn_close(out[:, rsel], ref, "n25600 srsu")


def test_n36864_twenty_call_sequence():
    """Anchor (dense + full refresh, Eq. (18)/(19)) at calls 0, 5, 10, 15;
    otherwise scatter of the sensitive rows + SRSU (Eq. (15)/(16)), with the
    cache updated in place. Call t uses the seeded base fields shifted along
    the tokens by (1009 t, 2003 t, 3001 t) for (Q, K, V) (exact copies)."""
    s = synth.WORKLOADS["n36864_seq"]
    inp = synth.make_inputs("n36864_seq")
    scale = 1 / math.sqrt(s.d)
    lens = inp["valid_len"].numpy()
    h64 = {n: synth.bf16_to_f64(inp[n]) for n in ("Q", "Ky")}
    ref_scores, S_ref, _ = oracle_partition(s, inp, {"Q": h64["Q"], "Ky": h64["Ky"]}, scale)
    d = {n: inp[n].to(DEV) for n in ("Q", "K", "V", "Ky", "w", "valid_len")}
    check_gpu_partition(s, d, ref_scores)
    S_dev = torch.from_numpy(S_ref.astype(np.int32)).to(DEV)
    shape = tuple(inp["K"].shape)
    base = {n: synth.bf16_bits(inp[n]).reshape(shape) for n in ("Q", "K", "V")}
    shifts = {"Q": 1009, "K": 2003, "V": 3001}
    cache_k = np.zeros(shape, dtype=np.uint16)
    cache_v = np.zeros(shape, dtype=np.uint16)
    Kc = torch.zeros(shape, dtype=torch.bfloat16, device=DEV)
    Vc = torch.zeros(shape, dtype=torch.bfloat16, device=DEV)
    rows = synth.sample_rows(s.N, SAMPLE, seed=5005)
    rsel = synth.sample_rows(s.k, SAMPLE, seed=5006)
    for t in range(20):
        cur = {n: torch.roll(d[n], shifts[n] * t, dims=1) for n in ("Q", "K", "V")}
        cur_h = {n: np.roll(base[n], shifts[n] * t, axis=1) for n in ("Q", "K", "V")}
        if t % 5 == 0:
            out = ops.attn_self(cur["Q"], cur["K"], cur["V"])
            ops.ctx_cache_scatter(cur["K"], cur["V"], None, Kc, Vc)
            cache_k = O.cache_scatter(cache_k, cur_h["K"], None, False)
            cache_v = O.cache_scatter(cache_v, cur_h["V"], None, False)
            if t in (0, 15):
                ref = O.attention(O.bf16_bits_to_f64(cur_h["Q"]), O.bf16_bits_to_f64(cur_h["K"]),
                                  O.bf16_bits_to_f64(cur_h["V"]), scale, q_rows=rows)
                assert_attn_close(out[:, rows], ref, f"n36864 anchor call {t}")
        else:
            ops.ctx_cache_scatter(cur["K"], cur["V"], S_dev, Kc, Vc, src_compact=False)
            out = ops.srsu_attn(cur["Q"], S_dev, Kc, Vc)
            cache_k = O.cache_scatter(cache_k, cur_h["K"], S_ref, False)
            cache_v = O.cache_scatter(cache_v, cur_h["V"], S_ref, False)
            if t in (1, 19):
                ref = O.attention(O.bf16_bits_to_f64(cur_h["Q"]), O.bf16_bits_to_f64(cache_k),
                                  O.bf16_bits_to_f64(cache_v), scale, q_rows=S_ref[:, rsel])
                assert_attn_close(out[:, rsel], ref, f"n36864 srsu call {t}")
        assert np.array_equal(synth.bf16_bits(Kc.cpu()).reshape(shape), cache_k), f"K cache differs at call {t}"
        assert np.array_equal(synth.bf16_bits(Vc.cpu()).reshape(shape), cache_v), f"V cache differs at call {t}"
        del out, cur
    # cross-attention at M = 256 on sampled rows
    Ky, Vy = d["Ky"], inp["Vy"].to(DEV)
    outx = ops.attn_cross(d["Q"], Ky, Vy, d["valid_len"])
    assert_attn_close(outx[:, rows], O.cross_attention(h64["Q"], h64["Ky"], synth.bf16_to_f64(inp["Vy"]), lens,
                                                      scale, q_rows=rows), "n36864 cross")
