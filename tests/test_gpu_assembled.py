"""SRSU with the global keys assembled in the kernel (Eq. (14), (16)): rows of
S from the current K/V, all other rows from the context cache, which is only
read. Checked against the fp64 oracle (the cache after the scatter of the
current rows, then Eq. (16)) and bit for bit against the two-launch form
(safe_ctx_cache_scatter into a copy of the cache, then safe_srsu_attn)."""

import math

import numpy as np
import pytest
import torch

import oracle as O
from mask_free_b200 import ops, synth
from tests.helpers import assert_attn_close, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(autouse=True)
def _status_clean():
    ops.device_status()
    yield


def _inputs(B, N, H, d, k, seed, pattern="random"):
    Q = synth.normal_bf16((B, N, H, d), seed)
    Kc = synth.normal_bf16((B, N, H, d), seed + 1)   # cache (anchor rows)
    Vc = synth.normal_bf16((B, N, H, d), seed + 2)
    Kn = synth.normal_bf16((B, N, H, d), seed + 3)   # current rows, full size
    Vn = synth.normal_bf16((B, N, H, d), seed + 4)
    rows = []
    for b in range(B):
        rng = np.random.default_rng(seed + 10 * b)
        if pattern == "random":
            s = np.sort(rng.choice(N, k, replace=False))
        elif pattern == "block":
            # one contiguous region: whole key tiles of S between partial ones
            start = int(rng.integers(0, N - k + 1))
            s = np.arange(start, start + k)
        else:  # "ends": the first and last tokens plus random rows between
            mid = np.sort(rng.choice(np.arange(1, N - 1), k - 2, replace=False))
            s = np.concatenate([[0], mid, [N - 1]])
        rows.append(s)
    S = np.stack(rows).astype(np.int32)
    return Q, Kc, Vc, Kn, Vn, S


def _compact(t, S):
    return torch.stack([t[b, torch.from_numpy(S[b]).long()] for b in range(t.shape[0])]).contiguous()


def _two_launch(Qd, Sd, Kcur, Vcur, Kc, Vc, q_compact, cur_compact, ws=None):
    K2, V2 = Kc.clone(), Vc.clone()
    ops.ctx_cache_scatter(Kcur, Vcur, Sd, K2, V2, src_compact=cur_compact)
    return ops.srsu_attn(Qd, Sd, K2, V2, q_compact=q_compact, return_lse=True, ws=ws)


@pytest.mark.parametrize("B,N,H,d,k", [(1, 256, 2, 64, 64), (2, 512, 3, 96, 200), (2, 1000, 2, 128, 333),
                                       (1, 384, 2, 96, 1), (1, 300, 2, 96, 300)])
def test_assembled_parity_with_oracle(B, N, H, d, k):
    Q, Kc, Vc, Kn, Vn, S = _inputs(B, N, H, d, k, seed=7 * N + k)
    Sd = torch.from_numpy(S).to(DEV)
    Kc_d, Vc_d = Kc.to(DEV), Vc.to(DEV)
    out, lse = ops.srsu_attn_assembled(Q.to(DEV), Sd, Kn.to(DEV), Vn.to(DEV), Kc_d, Vc_d, return_lse=True)
    K_asm = O.cache_scatter(to64(Kc), to64(Kn), S, src_compact=False)
    V_asm = O.cache_scatter(to64(Vc), to64(Vn), S, src_compact=False)
    ref, ref_lse = O.attention(to64(Q), K_asm, V_asm, 1 / math.sqrt(d), q_rows=S, with_lse=True)
    assert_attn_close(out, ref, "assembled srsu")
    np.testing.assert_allclose(to64(lse), ref_lse, atol=2e-3, rtol=0)
    # the cache is only read
    assert torch.equal(Kc_d.cpu(), Kc) and torch.equal(Vc_d.cpu(), Vc)
    assert ops.device_status() == 0


@pytest.mark.parametrize("q_compact", [False, True])
@pytest.mark.parametrize("cur_compact", [False, True])
@pytest.mark.parametrize("B,N,H,d,k,pattern", [(2, 1000, 2, 96, 333, "random"), (1, 2000, 2, 96, 700, "block"),
                                               (2, 777, 3, 64, 50, "ends"), (1, 640, 2, 128, 640, "random"),
                                               (2, 513, 1, 96, 129, "block")])
def test_assembled_equals_scatter_then_srsu_bitwise(B, N, H, d, k, pattern, q_compact, cur_compact):
    Q, Kc, Vc, Kn, Vn, S = _inputs(B, N, H, d, k, seed=N + 3 * k, pattern=pattern)
    Sd = torch.from_numpy(S).to(DEV)
    Qd = (_compact(Q, S) if q_compact else Q).to(DEV)
    Kcur = (_compact(Kn, S) if cur_compact else Kn).to(DEV)
    Vcur = (_compact(Vn, S) if cur_compact else Vn).to(DEV)
    Kc_d, Vc_d = Kc.to(DEV), Vc.to(DEV)
    want, want_lse = _two_launch(Qd, Sd, Kcur, Vcur, Kc_d, Vc_d, q_compact, cur_compact)
    got, got_lse = ops.srsu_attn_assembled(Qd, Sd, Kcur, Vcur, Kc_d, Vc_d, q_compact=q_compact,
                                           cur_compact=cur_compact, return_lse=True)
    assert torch.equal(got, want) and torch.equal(got_lse, want_lse)
    assert torch.equal(Kc_d.cpu(), Kc) and torch.equal(Vc_d.cpu(), Vc)
    assert ops.device_status() == 0


@pytest.mark.parametrize("B,N,H,d,k", [(2, 4096, 3, 96, 1229), (1, 4096, 1, 128, 777), (2, 3000, 3, 64, 1500)])
def test_assembled_key_split_plan_bitwise(B, N, H, d, k):
    # the last wave is split along the keys: a part starts at key tile kv0 > 0
    # and finds its first row of S by binary search
    assert ops.attn_workspace_bytes(B, k, N, H, d) > 0
    Q, Kc, Vc, Kn, Vn, S = _inputs(B, N, H, d, k, seed=N + k)
    Sd = torch.from_numpy(S).to(DEV)
    Qd, Kn_d, Vn_d, Kc_d, Vc_d = Q.to(DEV), Kn.to(DEV), Vn.to(DEV), Kc.to(DEV), Vc.to(DEV)
    want, want_lse = _two_launch(Qd, Sd, Kn_d, Vn_d, Kc_d, Vc_d, False, False)
    got, got_lse = ops.srsu_attn_assembled(Qd, Sd, Kn_d, Vn_d, Kc_d, Vc_d, return_lse=True)
    assert torch.equal(got, want) and torch.equal(got_lse, want_lse)
    whole = ops.srsu_attn_assembled(Qd, Sd, Kn_d, Vn_d, Kc_d, Vc_d, ws=False)
    ref = O.attention(to64(Q), O.cache_scatter(to64(Kc), to64(Kn), S, False),
                      O.cache_scatter(to64(Vc), to64(Vn), S, False), 1 / math.sqrt(d), q_rows=S)
    assert_attn_close(got, ref, "split")
    assert_attn_close(whole, ref, "whole")
    assert ops.device_status() == 0


def test_assembled_all_rows_current_is_dense_on_current():
    # S = every token: no cached row is visible, the result is dense
    # self-attention on the current K/V
    B, N, H, d = 2, 512, 2, 96
    Q, Kc, Vc, Kn, Vn, _ = _inputs(B, N, H, d, 1, seed=5)
    S = torch.arange(N, dtype=torch.int32, device=DEV).expand(B, N).contiguous()
    Qd, Kn_d, Vn_d = Q.to(DEV), Kn.to(DEV), Vn.to(DEV)
    got = ops.srsu_attn_assembled(Qd, S, Kn_d, Vn_d, Kc.to(DEV), Vc.to(DEV))
    assert torch.equal(got, ops.attn_self(Qd, Kn_d, Vn_d))


def test_assembled_out_of_order_rows_flagged():
    # S not ascending across key tiles: the rows met out of order are skipped
    # and flagged; every copy stays inside the tile it belongs to
    B, N, H, d = 1, 512, 1, 64
    Q, Kc, Vc, Kn, Vn, _ = _inputs(B, N, H, d, 1, seed=9)
    S = torch.tensor([[3, 300, 10, 400]], dtype=torch.int32, device=DEV)
    ops.srsu_attn_assembled(Q.to(DEV), S, Kn.to(DEV), Vn.to(DEV), Kc.to(DEV), Vc.to(DEV))
    assert ops.device_status() & (1 << ops.SAFE_ERR_DEVICE_CHECK)
