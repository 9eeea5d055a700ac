"""Host-side checks of the Python binding (no GPU): every entry point reaches
its C function with the declared number of arguments and the expected sizes,
and a tensor whose shape or device does not match the others is refused
with ValueError before anything is launched (the library trusts the sizes it
is given). The library is replaced by a recorder and CPU tensors stand in
for device tensors."""

import pytest
import torch

from mask_free_b200 import ops

bf16, f32, i32 = torch.bfloat16, torch.float32, torch.int32


class _Recorder:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def fn(*args):
            self.calls.append((name, args))
            if name.endswith("workspace_bytes"):
                return 0
            return ops.SAFE_OK
        return fn


@pytest.fixture
def rec(monkeypatch):
    r = _Recorder()
    monkeypatch.setattr(ops, "lib", lambda: r)
    monkeypatch.setattr(ops, "_on_device", lambda t: True)
    monkeypatch.setattr(ops, "_stream", lambda: None)
    return r


def _last(rec, name):
    calls = [a for n, a in rec.calls if n == name]
    assert calls, f"{name} was not called"
    args = calls[-1]
    assert len(args) == len(ops._SIGS[name]), (name, len(args), len(ops._SIGS[name]))
    return args


def t(*shape, dtype=bf16):
    return torch.zeros(shape, dtype=dtype)


B, N, H, d, M, k = 2, 300, 3, 64, 40, 70


def test_valid_calls_reach_the_abi_with_their_sizes(rec):
    Q = t(B, N, H, d)
    ops.attn_self(Q, Q, Q, return_lse=True)
    a = _last(rec, "safe_attn_self")
    assert a[5:9] == (B, N, H, d)
    Ky, lens, w = t(B, M, H, d), t(B, dtype=i32), t(B, M, dtype=f32)
    S = t(B, k, dtype=i32)
    ops.attn_cross(Q, Ky, Ky, lens, q_idx=S)
    a = _last(rec, "safe_attn_cross")
    assert a[2] == k and a[7:12] == (B, N, M, H, d)
    ops.pcsp_topk(Q, Ky, lens, w, k=k)
    a = _last(rec, "safe_pcsp_topk")
    assert a[4:9] == (B, N, M, H, d) and a[12] == k
    ops.attn_cross_pcsp(Q, Ky, Ky, lens, w, k=k)
    _last(rec, "safe_attn_cross_pcsp")
    ops.topk_partition(t(B, N, dtype=f32), k)
    assert _last(rec, "safe_topk_partition")[1:4] == (B, N, k)
    ops.srsu_attn(Q, S, Q, Q)
    a = _last(rec, "safe_srsu_attn")
    assert a[1] == 0 and a[3] == k and a[8:12] == (B, N, H, d)
    ops.srsu_attn(t(B, k, H, d), S, Q, Q, q_compact=True)
    assert _last(rec, "safe_srsu_attn")[1] == 1
    ops.srsu_attn_assembled(Q, S, t(B, k, H, d), t(B, k, H, d), Q, Q, cur_compact=True)
    a = _last(rec, "safe_srsu_attn_assembled")
    assert a[6] == 1 and a[3] == k and a[11:15] == (B, N, H, d)
    ops.ctx_cache_scatter(t(B, k, H, d), t(B, k, H, d), S, Q, Q, src_compact=True)
    a = _last(rec, "safe_ctx_cache_scatter")
    assert a[2] == 1 and a[4] == k
    ops.ctx_cache_scatter(Q, Q, None, Q, Q)  # anchor refresh: full-size source
    assert _last(rec, "safe_ctx_cache_scatter")[2] == 0
    ops.sensitivity_field(t(B, 15 * 20, dtype=f32), 15, 20, 2.0)
    assert _last(rec, "safe_sensitivity_field")[2:5] == (B, 15, 20)
    ops.partition_indicator(S, N)
    assert _last(rec, "safe_partition_indicator")[3:5] == (B, N)
    ops.sw_cfg(t(B, N, 4, dtype=f32), t(B, N, 4, dtype=f32), t(B, N, dtype=f32), 1.0, 5.0)
    assert _last(rec, "safe_sw_cfg")[4:8] == (2, B, N, 4)
    ops.mask_classify(torch.ones((B, 1, N, N), dtype=torch.bool), sync=False)
    _last(rec, "safe_mask_classify")
    ops.gather_linear(t(B, N, 64), t(40, 64), S=S, bias=t(40, dtype=f32), act="gelu_tanh")
    a = _last(rec, "safe_gather_linear")
    assert a[2] == k and a[5] == 1 and a[7:11] == (B, N, 64, 40)
    ops.gather_linear(t(B, N, 64), t(40, 64))
    a = _last(rec, "safe_gather_linear")
    assert a[1] is None and a[2] == 0 and a[5] == 0


def _refused(fn, *args, **kw):
    with pytest.raises(ValueError):
        fn(*args, **kw)


def test_mismatched_shapes_are_refused_before_any_launch(rec):
    Q = t(B, N, H, d)
    Ky, lens, w = t(B, M, H, d), t(B, dtype=i32), t(B, M, dtype=f32)
    S = t(B, k, dtype=i32)
    # self-attention: K / V / out / lse
    _refused(ops.attn_self, Q, t(B, N + 1, H, d), Q)
    _refused(ops.attn_self, Q, Q, t(B, N, H, d + 8))
    _refused(ops.attn_self, Q, Q, Q, out=t(B, N - 1, H, d))
    _refused(ops.attn_self, Q, Q, Q, return_lse=True, lse=t(B, N, H, dtype=f32))
    # cross: text K / V, lengths, query rows, output
    _refused(ops.attn_cross, Q, t(B, M, H + 1, d), t(B, M, H + 1, d), lens)
    _refused(ops.attn_cross, Q, Ky, t(B, M + 1, H, d), lens)
    _refused(ops.attn_cross, Q, Ky, Ky, t(B + 1, dtype=i32))
    _refused(ops.attn_cross, Q, Ky, Ky, lens, q_idx=t(B + 1, k, dtype=i32))
    _refused(ops.attn_cross, Q, Ky, Ky, lens, q_idx=S, out=t(B, N, H, d))
    # PCSP: weights, scores, split buffers, k > N
    _refused(ops.pcsp_topk, Q, Ky, lens, t(B, M + 1, dtype=f32))
    _refused(ops.pcsp_topk, Q, Ky, lens, w, scores=t(B, N + 1, dtype=f32))
    _refused(ops.pcsp_topk, Q, Ky, lens, w, k=k, S=t(B, k + 1, dtype=i32))
    _refused(ops.pcsp_topk, Q, Ky, lens, w, k=k, C=t(B, N - k + 1, dtype=i32))
    _refused(ops.attn_cross_pcsp, Q, Ky, Ky, lens, w, out=t(B, N, H, d + 8))
    _refused(ops.topk_partition, t(B, N, dtype=f32), N + 1)
    # SRSU: Q compact or not, S batch, cache pair, current rows, output
    _refused(ops.srsu_attn, t(B, k, H, d), S, Q, Q)                  # compact Q without q_compact
    _refused(ops.srsu_attn, Q, S, Q, Q, q_compact=True)
    _refused(ops.srsu_attn, Q, t(B + 1, k, dtype=i32), Q, Q)
    _refused(ops.srsu_attn, Q, S, Q, t(B, N + 1, H, d))
    _refused(ops.srsu_attn, Q, S, Q, Q, out=t(B, N, H, d))
    _refused(ops.srsu_attn_assembled, Q, S, t(B, k - 1, H, d), t(B, k - 1, H, d), Q, Q, cur_compact=True)
    _refused(ops.srsu_attn_assembled, Q, S, t(B, k, H, d), t(B, k, H, d), Q, Q, cur_compact=False)
    # scatter: source extent follows src_compact
    _refused(ops.ctx_cache_scatter, Q, Q, S, Q, Q, src_compact=True)
    _refused(ops.ctx_cache_scatter, t(B, k, H, d), t(B, k, H, d), S, Q, Q, src_compact=False)
    _refused(ops.ctx_cache_scatter, Q, Q, S, Q, t(B, N, H + 1, d), src_compact=False)
    # guidance: the grid must cover the scores; SW-CFG operands agree
    _refused(ops.sensitivity_field, t(B, 301, dtype=f32), 15, 20, 2.0)
    _refused(ops.sensitivity_field, t(B, 300, dtype=f32), 15, 20, 2.0, out=t(B, 299, dtype=f32))
    _refused(ops.partition_indicator, S, N, out=t(B, N - 1, dtype=f32))
    fc = t(B, N, 4, dtype=f32)
    _refused(ops.sw_cfg, fc, t(B, N, 5, dtype=f32), t(B, N, dtype=f32), 1.0, 5.0)
    _refused(ops.sw_cfg, fc, fc, t(B, N - 1, dtype=f32), 1.0, 5.0)
    _refused(ops.sw_cfg, fc, fc, t(B, N, dtype=f32), 1.0, 5.0, out=t(B, N, 4, dtype=bf16))
    _refused(ops.mask_classify, torch.ones((B, 1, N, N), dtype=torch.bool), result=t(4, dtype=torch.int64))
    # row-wise layer: weight width, rows, bias, activation, output
    X = t(B, N, 24)
    _refused(ops.gather_linear, X, t(40, 32))
    _refused(ops.gather_linear, X, t(40, 24), S=t(B + 1, k, dtype=i32))
    _refused(ops.gather_linear, X, t(40, 24), bias=t(41, dtype=f32))
    _refused(ops.gather_linear, X, t(40, 24), act="relu")
    _refused(ops.gather_linear, X, t(40, 24), S=S, out=t(B, N, 40))
    assert rec.calls == []  # nothing reached the library


def test_tensors_on_another_device_are_refused(rec):
    Q = t(B, N, H, d)
    other = torch.zeros((B, N, H, d), dtype=bf16, device="meta")
    _refused(ops.attn_self, Q, other, Q)
    _refused(ops.srsu_attn, Q, t(B, k, dtype=i32), Q, other)
    assert rec.calls == []
