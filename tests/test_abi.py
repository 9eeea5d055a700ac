"""CPU-side checks of the C ABI: the library loads, exports every entry point
declared in include/safe_attn.h, and rejects bad arguments on the host before
touching the GPU."""

import ctypes
import os
import re
import subprocess

import pytest

from mask_free_b200 import build as B
from mask_free_b200 import ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "safe_attn.h")


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(safe_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return ops.lib()


def test_library_exports_every_declared_symbol(lib):
    names = header_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), f"{n} declared in safe_attn.h but not exported"
    nm = subprocess.run(["nm", "-D", "--defined-only", B.LIB], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (safe_[a-z0-9_]+)", nm))
    assert set(names) <= exported
    # the binding knows the signature of every declared entry point
    assert set(names) == set(ops.exported_symbols())


def test_library_is_built_for_sm100a_only():
    flags = " ".join(B.NVCC_FLAGS)
    assert "arch=compute_100a,code=sm_100a" in flags
    assert flags.count("-gencode") == 1


def test_abi_version_and_status_strings(lib):
    assert lib.safe_abi_version() == 7
    assert lib.safe_status_string(0) == b"ok"
    assert lib.safe_status_string(1) == b"invalid argument"
    assert lib.safe_status_string(99) == b"unknown status"


def test_attn_workspace_plan(lib):
    # wave-balancing workspace: needed when the last wave of 256-row units
    # is partial, none when the units fill whole waves or keys are too few
    lib.safe_attn_workspace_bytes.restype = ctypes.c_size_t
    assert lib.safe_attn_workspace_bytes(2, 6400, 25600, 24, 96) > 0      # 1200 units: 8.1 waves
    assert lib.safe_attn_workspace_bytes(1, 256, 256, 2, 64) == 0         # 2 key tiles: no split
    # SRSU: the key split's workspace (256-byte aligned) plus the compact query rows
    lib.safe_srsu_workspace_bytes.restype = ctypes.c_size_t
    split = lib.safe_attn_workspace_bytes(2, 6400, 25600, 24, 96)
    assert lib.safe_srsu_workspace_bytes(2, 6400, 25600, 24, 96) == ((split + 255) // 256) * 256 + 2 * 6400 * 24 * 96 * 2
    assert lib.safe_srsu_workspace_bytes(1, 64, 256, 2, 64) == 64 * 2 * 64 * 2
    assert lib.safe_srsu_workspace_bytes(1, 64, 256, 2, 80) == 0
    assert lib.safe_attn_workspace_bytes(0, 256, 256, 2, 64) == 0
    assert lib.safe_attn_workspace_bytes(1, 256, 256, 2, 80) == 0
    # dense N = 4096 on 148 SMs: 768 units, the last 28 split into 4 key
    # parts; a part keeps 256 rows of bf16 O / l and 256 (m, l) pairs
    slots = 28 * 4 * 256
    assert lib.safe_attn_workspace_bytes(2, 4096, 4096, 24, 96) == \
        -(-slots * 96 * 2 // 256) * 256 + -(-slots * 8 // 256) * 256


def test_workspace_size(lib):
    assert lib.safe_pcsp_workspace_bytes(2, 25600, 24) == 2 * 25600 * 24 * 4
    assert lib.safe_pcsp_workspace_bytes(0, 10, 1) == 0


def test_host_validation_rejects_bad_arguments_without_gpu(lib):
    null = None
    # null / misaligned tensors, empty sizes, unsupported head dims
    assert lib.safe_attn_self(null, null, null, null, null, 1, 1, 1, 96, 1.0, null, 0, null) == 1
    fake = ctypes.c_void_p(0x10000)
    odd = ctypes.c_void_p(0x10008)
    assert lib.safe_attn_self(odd, fake, fake, fake, null, 1, 16, 1, 96, 1.0, null, 0, null) == 1
    assert lib.safe_attn_self(fake, fake, fake, fake, null, 0, 16, 1, 96, 1.0, null, 0, null) == 1
    assert lib.safe_attn_self(fake, fake, fake, fake, null, 1, 0, 1, 96, 1.0, null, 0, null) == 1
    assert lib.safe_attn_self(fake, fake, fake, fake, null, 1, 16, 1, 80, 1.0, null, 0, null) == 2
    assert lib.safe_attn_self(fake, fake, fake, fake, null, 1, 16, 1, 96, float("nan"), null, 0, null) == 1
    # the logit scale must be positive (the kernels scale each row's maximum)
    for bad in (0.0, -0.1, float("-inf")):
        assert lib.safe_attn_self(fake, fake, fake, fake, null, 1, 16, 1, 96, bad, null, 0, null) == 1
        assert lib.safe_srsu_attn(fake, 0, fake, 4, fake, fake, fake, null, 1, 16, 1, 96, bad, null, 0, null) == 1
        assert lib.safe_attn_cross(fake, null, 16, fake, fake, fake, fake, 1, 16, 16, 1, 96, bad, null) == 1
        assert lib.safe_pcsp_topk(fake, fake, fake, null, 1, 16, 16, 1, 96, bad, fake, 0, 4, fake, null, fake,
                                  4096, null) == 1
    # SRSU: k out of range
    assert lib.safe_srsu_attn(fake, 0, fake, 0, fake, fake, fake, null, 1, 16, 1, 96, 1.0, null, 0, null) == 1
    assert lib.safe_srsu_attn(fake, 0, fake, 17, fake, fake, fake, null, 1, 16, 1, 96, 1.0, null, 0, null) == 1
    # assembled-key SRSU: S and the current rows are required; k, d as above
    asm = lib.safe_srsu_attn_assembled
    assert asm(fake, 0, null, 4, fake, fake, 1, fake, fake, fake, null, 1, 16, 1, 96, 1.0, null, 0, null) == 1
    assert asm(fake, 0, fake, 4, null, fake, 1, fake, fake, fake, null, 1, 16, 1, 96, 1.0, null, 0, null) == 1
    assert asm(fake, 0, fake, 4, fake, odd, 1, fake, fake, fake, null, 1, 16, 1, 96, 1.0, null, 0, null) == 1
    assert asm(fake, 0, fake, 0, fake, fake, 1, fake, fake, fake, null, 1, 16, 1, 96, 1.0, null, 0, null) == 1
    assert asm(fake, 0, fake, 17, fake, fake, 1, fake, fake, fake, null, 1, 16, 1, 96, 1.0, null, 0, null) == 1
    assert asm(fake, 0, fake, 4, fake, fake, 1, fake, fake, fake, null, 1, 16, 1, 80, 1.0, null, 0, null) == 2
    # row-wise layer: widths multiples of 8, act 0/1, k in [1, N] with S, aligned bias
    lib.safe_gather_linear_workspace_bytes.restype = ctypes.c_size_t
    assert lib.safe_gather_linear_workspace_bytes(2, 6400, 2304) == 2 * 6400 * 2304 * 2
    assert lib.safe_gather_linear_workspace_bytes(0, 6400, 2304) == 0
    gl = lib.safe_gather_linear
    assert gl(fake, null, 0, fake, null, 0, fake, 1, 16, 60, 64, null, 0, null) == 1
    assert gl(fake, null, 0, fake, null, 0, fake, 1, 16, 56, 64, null, 0, null) == 1
    assert gl(fake, null, 0, fake, null, 0, fake, 1, 16, 64, 4, null, 0, null) == 1
    assert gl(fake, null, 0, fake, null, 2, fake, 1, 16, 64, 64, null, 0, null) == 1
    assert gl(fake, fake, 0, fake, null, 0, fake, 1, 16, 64, 64, null, 0, null) == 1
    assert gl(fake, fake, 17, fake, null, 0, fake, 1, 16, 64, 64, null, 0, null) == 1
    assert gl(fake, null, 0, fake, ctypes.c_void_p(0x10002), 0, fake, 1, 16, 64, 64, null, 0, null) == 1
    assert gl(odd, null, 0, fake, null, 0, fake, 1, 16, 64, 64, null, 0, null) == 1
    # cross: M > 256 unsupported, nq must equal N without q_idx
    assert lib.safe_attn_cross(fake, null, 16, fake, fake, fake, fake, 1, 16, 257, 1, 96, 1.0, null) == 2
    assert lib.safe_attn_cross(fake, null, 8, fake, fake, fake, fake, 1, 16, 16, 1, 96, 1.0, null) == 1
    # PCSP: k > N, missing / short workspace
    assert lib.safe_pcsp_topk(fake, fake, fake, null, 1, 16, 16, 1, 96, 1.0, fake, 0, 17, fake, null, fake, 4096,
                              null) == 1
    assert lib.safe_pcsp_topk(fake, fake, fake, null, 1, 16, 16, 1, 96, 1.0, fake, 0, 4, fake, null, null, 0,
                              null) == 1
    assert lib.safe_pcsp_topk(fake, fake, fake, null, 1, 16, 16, 2, 96, 1.0, fake, 0, 4, fake, null, fake, 64,
                              null) == 1
    # top-k: k = 0
    assert lib.safe_topk_partition(fake, 1, 16, 0, fake, null, null) == 1
    # scatter: compact source needs S; k > N
    assert lib.safe_ctx_cache_scatter(fake, fake, 1, null, 0, fake, fake, 1, 16, 1, 96, null) == 1
    assert lib.safe_ctx_cache_scatter(fake, fake, 1, fake, 17, fake, fake, 1, 16, 1, 96, null) == 1
    # classifier: negative stride, zero size, bad dtype
    sizes = (ctypes.c_int64 * 4)(1, 1, 4, 4)
    bad_sizes = (ctypes.c_int64 * 4)(1, 1, 0, 4)
    strides = (ctypes.c_int64 * 4)(16, 16, 4, 1)
    neg = (ctypes.c_int64 * 4)(16, 16, 4, -1)
    assert lib.safe_mask_classify(fake, 0, sizes, neg, fake, null) == 1
    assert lib.safe_mask_classify(fake, 0, bad_sizes, strides, fake, null) == 1
    assert lib.safe_mask_classify(fake, 7, sizes, strides, fake, null) == 1
    assert lib.safe_mask_classify(ctypes.c_void_p(0x10002), 2, sizes, strides, fake, null) == 1
    # timeout self-test: limit out of range
    assert lib.safe_selftest_wait_timeout(0, null) == 1
    assert lib.safe_get_device_status(null, null) == 1


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros((1, 16, 1, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        ops.attn_self(x, x, x)


def test_guidance_entry_points_validate_on_host(lib):
    null = None
    fake = ctypes.c_void_p(0x10000)
    other = ctypes.c_void_p(0x20000)
    ws_ok = lib.safe_sensitivity_workspace_bytes(2, 64 * 64)
    assert ws_ok == 2 * 4096 * 4 + 256  # row-pass field + min/max keys, each 256-byte aligned
    assert lib.safe_sensitivity_workspace_bytes(0, 5) == 0
    # sensitivity field: aliasing, negative sigma, bad truncate, short / misaligned workspace, radius > 128
    assert lib.safe_sensitivity_field(fake, fake, 2, 64, 64, 1.0, 4.0, other, ws_ok, null) == 1
    assert lib.safe_sensitivity_field(fake, other, 2, 64, 64, -1.0, 4.0, fake, ws_ok, null) == 1
    assert lib.safe_sensitivity_field(fake, other, 2, 64, 64, 1.0, 0.0, fake, ws_ok, null) == 1
    assert lib.safe_sensitivity_field(fake, other, 2, 64, 64, float("inf"), 4.0, fake, ws_ok, null) == 1
    assert lib.safe_sensitivity_field(fake, other, 2, 64, 64, 1.0, 4.0, fake, ws_ok - 4, null) == 1
    assert lib.safe_sensitivity_field(fake, other, 2, 64, 64, 1.0, 4.0, ctypes.c_void_p(0x10080), ws_ok, null) == 1
    assert lib.safe_sensitivity_field(fake, other, 2, 0, 64, 1.0, 4.0, fake, ws_ok, null) == 1
    assert lib.safe_sensitivity_field(fake, other, 2, 64, 64, 32.2, 4.0, fake, ws_ok, null) == 2  # r = 129
    # partition indicator: k out of range
    assert lib.safe_partition_indicator(fake, 0, other, 1, 16, null) == 1
    assert lib.safe_partition_indicator(fake, 17, other, 1, 16, null) == 1
    # SW-CFG: dtype fp16 unsupported, misaligned fp32, non-finite scale, empty
    assert lib.safe_sw_cfg(fake, fake, fake, fake, 3, 1, 16, 4, 1.0, 2.0, null) == 2
    assert lib.safe_sw_cfg(ctypes.c_void_p(0x10002), fake, fake, fake, 2, 1, 16, 4, 1.0, 2.0, null) == 1
    assert lib.safe_sw_cfg(fake, fake, fake, fake, 2, 1, 16, 4, float("nan"), 2.0, null) == 1
    assert lib.safe_sw_cfg(fake, fake, fake, fake, 4, 1, 16, 0, 1.0, 2.0, null) == 1


def test_fused_cross_pcsp_validates_on_host(lib):
    null = None
    fake = ctypes.c_void_p(0x10000)
    ws_ok = lib.safe_pcsp_workspace_bytes(1, 16, 1)
    args = lambda M, k, ws, wsb: (fake, fake, fake, fake, null, fake, 1, 16, M, 1, 96, 1.0, fake, 0, k, fake, null,
                                  ws, wsb, null)
    assert lib.safe_attn_cross_pcsp(*args(16, 4, null, 0)) == 1             # no workspace
    assert lib.safe_attn_cross_pcsp(*args(16, 4, fake, ws_ok - 4)) == 1     # short workspace
    assert lib.safe_attn_cross_pcsp(*args(16, 17, fake, ws_ok)) == 1        # k > N
    assert lib.safe_attn_cross_pcsp(*args(257, 4, fake, ws_ok)) == 2        # M > 256



def test_graft_entry_build_loads_the_library():
    # the build entry point compiles (if needed), loads the library and
    # checks the ABI version it was written against
    import __graft_entry__ as g
    g.build()
    assert ops.abi_version() == 7
