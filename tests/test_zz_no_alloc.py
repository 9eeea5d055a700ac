"""The allocation-free PCSP entry point (safe_pcsp_topk_noalloc).

It serves callers that cannot allocate device memory (hosted plugins with no
workspace, loops with a fixed memory plan): its per-head scratch is a fixed
array inside the library instead of a caller workspace. This file is
collected last on purpose, so a run that stops at the first failure has
already run every other test; it also passes on its own in a fresh process.

Checked through the C ABI against safe_pcsp_topk (the workspace entry point)
on two calls in a row: both run the same kernels on the same inputs, only
the scratch address differs, so scores, S and C must be bit-identical. The
scores are also compared with the fp64 oracle at the PCSP score tolerance of
the other tests, and the size limit is checked.
"""

import ctypes
import math

import numpy as np
import pytest
import torch

import oracle as O
from mask_free_b200 import ops, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"
SCRATCH_FLOATS = 1 << 21


def _noalloc(Q, Ky, lens, w, scores, accumulate, k, S, C):
    B, N, H, d = Q.shape
    M = Ky.shape[1]
    return ops.lib().safe_pcsp_topk_noalloc(
        ctypes.c_void_p(Q.data_ptr()), ctypes.c_void_p(Ky.data_ptr()), ctypes.c_void_p(lens.data_ptr()),
        ctypes.c_void_p(w.data_ptr()), B, N, M, H, d, 1.0 / math.sqrt(d), ctypes.c_void_p(scores.data_ptr()),
        accumulate, k, ctypes.c_void_p(S.data_ptr()), ctypes.c_void_p(C.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_pcsp_matches_workspace_entry_point_on_two_calls():
    B, N, M, H, d, k = 2, 4096, 128, 24, 96, 1229
    lens = torch.tensor([37, 128], dtype=torch.int32)
    w = synth.content_weights(lens, M, 7).to(DEV)
    lens = lens.to(DEV)
    scores_new = torch.zeros((B, N), dtype=torch.float32, device=DEV)
    scores_ref = torch.zeros_like(scores_new)
    ref = np.zeros((B, N))
    for call in range(2):
        Q = synth.normal_bf16((B, N, H, d), 900 + call).to(DEV)
        Ky = synth.normal_bf16((B, M, H, d), 910 + call).to(DEV)
        accumulate = call  # second call adds to the first call's scores
        S_new = torch.empty((B, k), dtype=torch.int32, device=DEV)
        C_new = torch.empty((B, N - k), dtype=torch.int32, device=DEV)
        st = _noalloc(Q, Ky, lens, w, scores_new, accumulate, k, S_new, C_new)
        assert st == ops.SAFE_OK
        _, S_ref, C_ref = ops.pcsp_topk(Q, Ky, lens, w, scores=scores_ref, accumulate=bool(accumulate), k=k)
        torch.cuda.synchronize()
        assert torch.equal(scores_new, scores_ref), f"call {call}: scores differ from the workspace entry point"
        assert torch.equal(S_new, S_ref) and torch.equal(C_new, C_ref), f"call {call}: partition differs"
        assert ops.device_status() == 0
        ref = ref + O.pcsp_scores(synth.bf16_to_f64(Q.cpu()), synth.bf16_to_f64(Ky.cpu()), lens.cpu().numpy(),
                                  w.cpu().numpy(), 1.0 / math.sqrt(d))
        np.testing.assert_allclose(scores_new.cpu().numpy(), ref, rtol=3e-5, atol=1e-8)


def test_noalloc_pcsp_rejects_sizes_beyond_the_scratch():
    # B * H * N = 2 * 24 * 43691 > 2^21: refused on the host, nothing launched
    B, H, N, d, M = 2, 24, 43691, 96, 16
    assert B * H * N > SCRATCH_FLOATS
    fake = ctypes.c_void_p(0x10000)
    st = ops.lib().safe_pcsp_topk_noalloc(fake, fake, fake, None, B, N, M, H, d, 0.1, fake, 0, 0, None, None,
                                          None)
    assert st == ops.SAFE_ERR_UNSUPPORTED
