"""Comparison helpers shared by the GPU parity tests (test code only)."""

from __future__ import annotations

import numpy as np
import torch

# Tolerances for attention outputs (bf16-rounded inputs, fp32 accumulation,
# bf16 output) against the fp64 oracle.
MAX_ABS = 1e-2
MEAN_ABS = 1e-3
REL_RMS = 1e-2


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def attn_errors(gpu: torch.Tensor, ref: np.ndarray):
    g = to64(gpu)
    assert g.shape == ref.shape, (g.shape, ref.shape)
    diff = np.abs(g - ref)
    rel_rms = float(np.sqrt(np.mean(diff ** 2)) / max(np.sqrt(np.mean(ref ** 2)), 1e-30))
    return float(diff.max()), float(diff.mean()), rel_rms


def assert_attn_close(gpu: torch.Tensor, ref: np.ndarray, label: str = "", magnitude_scaled: bool = False):
    """Attention parity bar. With magnitude_scaled, the absolute bounds are
    multiplied by max(1, max|ref|) (max-abs) and max(1, rms(ref)) (mean-abs):
    for peaked softmaxes the outputs approach single value rows of size ~1-4,
    where bf16 output rounding alone is 2^-9 of the magnitude."""
    g = to64(gpu)
    assert np.all(np.isfinite(g)), f"{label}: non-finite output"
    mx, mean, rr = attn_errors(gpu, ref)
    amax, amean = MAX_ABS, MEAN_ABS
    if magnitude_scaled:
        amax *= max(1.0, float(np.abs(ref).max()))
        amean *= max(1.0, float(np.sqrt(np.mean(ref ** 2))))
    assert mx <= amax and mean <= amean and rr <= REL_RMS, \
        f"{label}: max_abs {mx:.3e} mean_abs {mean:.3e} rel_rms {rr:.3e}"
    return mx, mean, rr


def bits(t: torch.Tensor) -> np.ndarray:
    """Raw bytes of a tensor (for bit-exact comparisons)."""
    return t.detach().contiguous().cpu().view(torch.uint8).numpy()


def storage_view_for_oracle(v: torch.Tensor):
    """(flat storage array, sizes, strides, offset) of a CPU view, for
    oracle.classify_mask; 16-bit floats as uint16 bit patterns."""
    st = v.untyped_storage()
    flat = torch.empty(0, dtype=v.dtype).set_(st, 0, (st.nbytes() // v.element_size(),), (1,))
    if v.dtype == torch.bool:
        arr = flat.view(torch.uint8).numpy()
    elif v.dtype in (torch.float16, torch.bfloat16):
        arr = flat.view(torch.int16).numpy().view(np.uint16)
    else:
        arr = flat.numpy()
    return arr, tuple(v.shape), tuple(v.stride()), v.storage_offset()


def to_device_view(v: torch.Tensor, device="cuda") -> torch.Tensor:
    """The same strided view over a device copy of the whole storage."""
    st = v.untyped_storage()
    flat = torch.empty(0, dtype=v.dtype).set_(st, 0, (st.nbytes() // v.element_size(),), (1,))
    dflat = flat.to(device)
    return torch.as_strided(dflat, v.shape, v.stride(), v.storage_offset())
