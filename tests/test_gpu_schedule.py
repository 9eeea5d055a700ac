"""The run schedule's block executor (mask_free_b200.schedule.BlockAttention)
on the GPU, replayed call by call by the fp64 oracle.

A 7-call run with two warm-up anchors and an anchor every 5th call (anchors
0, 1, 5; row-selective calls 2, 3, 4, 6; Eq. (14)) at N = 4096, H = 4,
d = 96, k = 1229: N = 4096 gives 16 query blocks per head, so the flash
kernel runs its key-split tail, and k = 1229 leaves a ragged last query tile.
Every call draws fresh Q, K, V. The oracle keeps its own copy of the context
cache and of the accumulated PCSP scores and checks, on every call:
  - the cache, whole buffer, bit for bit (refresh at anchors, Eq. (19);
    scatter of the rows of S otherwise, Eq. (16); untouched between anchors
    in the assembled form);
  - the warm-up scores (Eq. (9), (10), accumulated over the warm-up calls) and
    the split taken after the last warm-up call (Eq. (12)), for validity;
  - the outputs on sampled rows: dense self-attention and cross-attention at
    anchors, SRSU over S u C (Eq. (16)) and cross-attention on S (Eq. (17))
    otherwise, with full-size and (call 6) compact current rows.
"""

import math

import numpy as np
import pytest
import torch

import oracle as O
from mask_free_b200 import ops, synth
from mask_free_b200.schedule import AnchorSchedule, BlockAttention
from tests.helpers import assert_attn_close

pytestmark = pytest.mark.gpu
DEV = "cuda"
B, N, H, d, M, k = 2, 4096, 4, 96, 128, 1229
T, EVERY, WARMUP = 7, 5, 2
SAMPLE = 256


@pytest.fixture(autouse=True)
def _status_clean():
    ops.device_status()
    yield
    assert ops.device_status() == 0


def _call_inputs(t):
    return {n: synth.normal_bf16((B, N, H, d), 9100 + 10 * t + i) for i, n in enumerate(("Q", "K", "V"))}


@pytest.mark.parametrize("assembled", [False, True])
def test_block_attention_run_matches_oracle_replay(assembled):
    scale = 1.0 / math.sqrt(d)
    lens = synth.uniform_lengths(B, 8, M, 9201)
    w = synth.content_weights(lens, M, 9202)
    Ky = synth.normal_bf16((B, M, H, d), 9203)
    Vy = synth.normal_bf16((B, M, H, d), 9204)
    lens_np, w_np = lens.numpy(), w.numpy().astype(np.float64)
    Ky64, Vy64 = synth.bf16_to_f64(Ky), synth.bf16_to_f64(Vy)
    dKy, dVy, dlens, dw = Ky.to(DEV), Vy.to(DEV), lens.to(DEV), w.to(DEV)

    sched = AnchorSchedule(T, EVERY, warmup=WARMUP)
    assert sched.anchors() == [0, 1, 5]
    blk = BlockAttention(sched, B, N, H, d, k, DEV, w=dw, assembled=assembled)
    shape = (B, N, H, d)
    cache_k = np.zeros(shape, dtype=np.uint16)
    cache_v = np.zeros(shape, dtype=np.uint16)
    ref_scores = np.zeros((B, N))
    S = None
    rows = synth.sample_rows(N, SAMPLE, seed=9205)
    rsel = synth.sample_rows(k, SAMPLE, seed=9206)
    for t in range(T):
        cur = _call_inputs(t)
        bits = {n: synth.bf16_bits(cur[n]).reshape(shape) for n in cur}
        h64 = {n: synth.bf16_to_f64(cur[n]) for n in cur}
        if sched.is_anchor(t):
            dcur = {n: cur[n].to(DEV) for n in cur}
            out = blk(t, dcur["Q"], dcur["K"], dcur["V"], dKy, dVy, dlens)
            cache_k, cache_v = bits["K"].copy(), bits["V"].copy()
            assert_attn_close(out["self"][:, rows], O.attention(h64["Q"], h64["K"], h64["V"], scale, q_rows=rows),
                              f"call {t} dense self")
            assert_attn_close(out["cross"][:, rows],
                              O.cross_attention(h64["Q"], Ky64, Vy64, lens_np, scale, q_rows=rows),
                              f"call {t} dense cross")
            if t < WARMUP:
                ref_scores = ref_scores + O.pcsp_scores(h64["Q"], Ky64, lens_np, w_np, scale)
                np.testing.assert_allclose(blk.scores.cpu().numpy(), ref_scores, rtol=3e-5, atol=1e-8)
            if t == WARMUP - 1:
                # the split of the accumulated scores: a valid top-k of the
                # oracle's scores (a near-tie at the k-boundary may go
                # either way); the replay below uses the GPU's own S
                S, C = blk.S.cpu().numpy(), blk.C.cpu().numpy()
                tol = 3e-5 * np.abs(ref_scores).max()
                for b in range(B):
                    assert np.all(np.diff(S[b]) > 0) and np.all(np.diff(C[b]) > 0)
                    sel = np.zeros(N, dtype=bool)
                    sel[S[b]] = True
                    assert sel.sum() == k and not np.any(sel[C[b]])
                    assert ref_scores[b][sel].min() >= ref_scores[b][~sel].max() - tol
        else:
            compact = t == T - 1
            if compact:
                idx = torch.from_numpy(S).long()
                dcur = {n: torch.stack([cur[n][b, idx[b]] for b in range(B)]).to(DEV) for n in cur}
            else:
                dcur = {n: cur[n].to(DEV) for n in cur}
            out = blk(t, dcur["Q"], dcur["K"], dcur["V"], dKy, dVy, dlens)
            assert torch.equal(out["S"].cpu(), torch.from_numpy(S.astype(np.int32)))
            # K and V of S u C: current rows of S over the cached context rows
            kv_k = O.cache_scatter(cache_k, bits["K"], S, False)
            kv_v = O.cache_scatter(cache_v, bits["V"], S, False)
            if not assembled:
                cache_k, cache_v = kv_k, kv_v
            ref_self = O.attention(h64["Q"], O.bf16_bits_to_f64(kv_k), O.bf16_bits_to_f64(kv_v), scale,
                                   q_rows=S[:, rsel])
            assert_attn_close(out["self"][:, rsel], ref_self, f"call {t} srsu (compact={compact})")
            ref_cross = O.cross_attention(h64["Q"], Ky64, Vy64, lens_np, scale, q_rows=S[:, rsel])
            assert_attn_close(out["cross"][:, rsel], ref_cross, f"call {t} cross on S (compact={compact})")
        assert np.array_equal(synth.bf16_bits(blk.Kc.cpu()).reshape(shape), cache_k), f"K cache at call {t}"
        assert np.array_equal(synth.bf16_bits(blk.Vc.cpu()).reshape(shape), cache_v), f"V cache at call {t}"
        del out, dcur
