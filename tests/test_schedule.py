"""Host-side checks of the run schedule (no GPU): the anchor set of Eq. (14),
and the library calls one block makes on each call of a 20-call run. The
library is replaced by a recorder and CPU tensors stand in for device
tensors; the calls themselves are parity-tested on the GPU elsewhere."""

import pytest
import torch

from mask_free_b200 import ops
from mask_free_b200.schedule import AnchorSchedule, BlockAttention


class _Recorder:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def fn(*args):
            if not name.endswith("workspace_bytes"):
                assert len(args) == len(ops._SIGS[name]), name
                self.calls.append((name, args))
                return ops.SAFE_OK
            return 0
        return fn

    def take(self):
        c, self.calls = self.calls, []
        return c


@pytest.fixture
def rec(monkeypatch):
    r = _Recorder()
    monkeypatch.setattr(ops, "lib", lambda: r)
    monkeypatch.setattr(ops, "_on_device", lambda t: True)
    monkeypatch.setattr(ops, "_stream", lambda: None)
    return r


def test_anchor_set_and_last_anchor():
    s = AnchorSchedule(T=20, every=5)
    assert s.anchors() == [0, 5, 10, 15]
    assert [s.last_anchor(t) for t in (1, 4, 5, 6, 19)] == [0, 0, 0, 5, 15]
    w = AnchorSchedule(T=12, every=5, warmup=3)
    assert w.anchors() == [0, 1, 2, 5, 10]
    assert w.last_anchor(3) == 2
    for bad in (dict(T=0, every=5), dict(T=5, every=0), dict(T=5, every=2, warmup=0), dict(T=5, every=2, warmup=6)):
        with pytest.raises(ValueError):
            AnchorSchedule(**bad)
    with pytest.raises(ValueError):
        s.is_anchor(20)
    with pytest.raises(ValueError):
        s.last_anchor(0)


B, N, H, d, M, k = 2, 64, 2, 64, 16, 16


def _inputs(rows=N):
    z = lambda *sh, dt=torch.bfloat16: torch.zeros(sh, dtype=dt)
    return z(B, rows, H, d), z(B, rows, H, d), z(B, rows, H, d), z(B, M, H, d), z(B, M, H, d), z(B, dt=torch.int32)


def _names(calls):
    return [n for n, _ in calls]


def test_twenty_call_run_makes_the_expected_calls(rec):
    sched = AnchorSchedule(T=20, every=5)
    blk = BlockAttention(sched, B, N, H, d, k, device="cpu")
    Q, K, V, Ky, Vy, lens = _inputs()
    for t in range(20):
        out = blk(t, Q, K, V, Ky, Vy, lens)
        calls = rec.take()
        if t == 0:
            # dense block, full refresh, cross-attention with the PCSP scores, the split
            assert _names(calls) == ["safe_attn_self", "safe_ctx_cache_scatter", "safe_attn_cross_pcsp",
                                     "safe_topk_partition"]
            sc = calls[1][1]
            assert sc[3] is None and sc[2] == 0                   # S = NULL: refresh from the full rows
            assert calls[2][1][13] == 0                           # accumulate off on the first call
            assert calls[3][1][3] == k
            assert tuple(out["self"].shape) == (B, N, H, d) and tuple(out["cross"].shape) == (B, N, H, d)
        elif t % 5 == 0:
            assert _names(calls) == ["safe_attn_self", "safe_ctx_cache_scatter", "safe_attn_cross"]
            assert calls[1][1][3] is None
        else:
            assert _names(calls) == ["safe_ctx_cache_scatter", "safe_srsu_attn", "safe_attn_cross"]
            s_ptr = blk.S.data_ptr()
            sc, sr, cr = calls[0][1], calls[1][1], calls[2][1]
            assert sc[3].value == s_ptr and sc[4] == k and sc[2] == 0     # scatter of the current rows of S
            assert sr[2].value == s_ptr and sr[3] == k and sr[1] == 0     # SRSU gathers the rows of S from Q
            assert sr[4].value == blk.Kc.data_ptr()                       # ... against the cache
            assert cr[1].value == s_ptr and cr[2] == k                    # cross-attention on the rows of S
            assert tuple(out["self"].shape) == (B, k, H, d) and tuple(out["cross"].shape) == (B, k, H, d)


def test_warmup_accumulates_scores_and_smooths_before_the_split(rec):
    sched = AnchorSchedule(T=8, every=4, warmup=2)
    blk = BlockAttention(sched, B, N, H, d, k, device="cpu", w=torch.zeros((B, M)), sigma=1.5, grid_h=8, grid_w=8)
    Q, K, V, Ky, Vy, lens = _inputs()
    blk(0, Q, K, V, Ky, Vy, lens)
    c0 = rec.take()
    assert _names(c0) == ["safe_attn_self", "safe_ctx_cache_scatter", "safe_attn_cross_pcsp"]
    assert c0[2][1][13] == 0 and c0[2][1][4] is not None                 # weights passed, no accumulation
    blk(1, Q, K, V, Ky, Vy, lens)
    c1 = rec.take()
    assert _names(c1) == ["safe_attn_self", "safe_ctx_cache_scatter", "safe_attn_cross_pcsp",
                          "safe_sensitivity_field", "safe_topk_partition"]
    assert c1[2][1][13] == 1                                             # second warm-up call accumulates
    assert c1[2][1][12].value == blk.scores.data_ptr() == c1[3][1][0].value
    assert c1[4][1][0].value == c1[3][1][1].value                        # the split reads the smoothed field
    blk(2, Q, K, V, Ky, Vy, lens)
    assert _names(rec.take()) == ["safe_ctx_cache_scatter", "safe_srsu_attn", "safe_attn_cross"]


def test_assembled_and_compact_forms(rec):
    sched = AnchorSchedule(T=3, every=5)
    Q, K, V, Ky, Vy, lens = _inputs()
    blk = BlockAttention(sched, B, N, H, d, k, device="cpu", assembled=True)
    blk(0, Q, K, V, Ky, Vy, lens)
    rec.take()
    blk(1, Q, K, V, Ky, Vy, lens)
    calls = rec.take()
    assert _names(calls) == ["safe_srsu_attn_assembled", "safe_attn_cross"]   # no scatter: the cache is only read
    assert calls[0][1][6] == 0
    # compact current rows [B, k, H, d]
    Qs, Ks, Vs, _, _, _ = _inputs(rows=k)
    blk(2, Qs, Ks, Vs, Ky, Vy, lens)
    calls = rec.take()
    assert calls[0][1][1] == 1 and calls[0][1][6] == 1                        # q_compact, cur_compact
    assert calls[1][1][1] is None and calls[1][1][2] == k                     # cross over the compact rows
    plain = BlockAttention(sched, B, N, H, d, k, device="cpu")
    plain(0, Q, K, V, Ky, Vy, lens)
    rec.take()
    plain(1, Qs, Ks, Vs, Ky, Vy, lens)
    calls = rec.take()
    assert _names(calls) == ["safe_ctx_cache_scatter", "safe_srsu_attn", "safe_attn_cross"]
    assert calls[0][1][2] == 1 and calls[1][1][1] == 1                       # compact source, compact Q


def test_selective_call_before_warmup_is_refused(rec):
    sched = AnchorSchedule(T=6, every=5)
    blk = BlockAttention(sched, B, N, H, d, k, device="cpu")
    Q, K, V, Ky, Vy, lens = _inputs()
    with pytest.raises(RuntimeError):
        blk(1, Q, K, V, Ky, Vy, lens)
    with pytest.raises(ValueError):
        BlockAttention(sched, B, N, H, d, N + 1, device="cpu")
    with pytest.raises(ValueError):
        BlockAttention(sched, B, N, H, d, k, device="cpu", sigma=1.0, grid_h=7, grid_w=8)
