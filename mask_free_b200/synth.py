"""Seeded synthetic inputs for the SAFE-DiT attention hot path.

This module only draws random numbers and rounds them to the storage types:
it holds none of the method's arithmetic. Both the CUDA path and the fp64
oracle consume exactly the values produced here (bf16 tensors are widened
exactly by the oracle).

Recipe (workload shapes of the paper's Lumina-Next runs at 1024^2, 2560^2
and 3072^2, with a 16x spatial reduction from pixels to latent tokens):
  * Q, K, V, K_y, V_y: fp32 standard normals from numpy PCG64(seed), rounded
    to bf16 with round-to-nearest-even; seed = 1000 * (workload seed id) +
    100 * call + tensor id.
  * text valid lengths: uniform integers in [lo, hi] per sample.
  * content weights w: U(0, 1) on valid keys, 0 on padding, normalised to
    sum 1 per sample in fp64, stored as fp32.
  * context drift: cache = bf16(K + std * z), z standard normal (fp32).
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

# tensor ids used in seeds
T_Q, T_K, T_V, T_KY, T_VY, T_LEN, T_W, T_DK, T_DV, T_MASK = range(10)


def seed_for(seed_id: int, tensor_id: int, call: int = 0) -> int:
    return 1000 * seed_id + 100 * call + tensor_id


def normal_f32(shape, seed: int) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.standard_normal(size=shape, dtype=np.float32)


def normal_bf16(shape, seed: int) -> torch.Tensor:
    """Standard normals rounded to bf16 (RNE), as a CPU torch tensor."""
    return torch.from_numpy(normal_f32(shape, seed)).to(torch.bfloat16)


def uniform_lengths(B: int, lo: int, hi: int, seed: int) -> torch.Tensor:
    rng = np.random.Generator(np.random.PCG64(seed))
    return torch.from_numpy(rng.integers(lo, hi + 1, size=B).astype(np.int32))


def content_weights(valid_len: torch.Tensor, M: int, seed: int) -> torch.Tensor:
    rng = np.random.Generator(np.random.PCG64(seed))
    B = valid_len.shape[0]
    w = np.zeros((B, M), dtype=np.float64)
    for b in range(B):
        L = int(valid_len[b])
        u = rng.random(L)
        w[b, :L] = u / u.sum()
    return torch.from_numpy(w.astype(np.float32))


def drifted_bf16(base: torch.Tensor, std: float, seed: int) -> torch.Tensor:
    z = normal_f32(tuple(base.shape), seed)
    return (base.float() + std * torch.from_numpy(z)).to(torch.bfloat16)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Raw uint16 bit patterns of a bf16 CPU tensor (for the oracle)."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact widening of a bf16 tensor to float64 numpy."""
    return t.float().numpy().astype(np.float64)


@dataclass(frozen=True)
class Shape:
    seed_id: int  # distinguishes the workloads' random streams
    B: int
    N: int
    H: int
    d: int
    M: int
    len_lo: int
    len_hi: int
    k: int


# The workloads, by what they are: a tiny check; the 1024^2 (N = 4096)
# dense block and SRSU step; the 2560^2 (N = 25600) anchor + SRSU step; the
# 3072^2 (N = 36864) 20-call anchor / SRSU sequence.
WORKLOADS = {
    "tiny": Shape(seed_id=1, B=1, N=256, H=2, d=64, M=16, len_lo=11, len_hi=11, k=64),
    "n4096": Shape(seed_id=2, B=2, N=4096, H=24, d=96, M=128, len_lo=8, len_hi=128, k=1229),
    "n4096_srsu": Shape(seed_id=3, B=2, N=4096, H=24, d=96, M=128, len_lo=8, len_hi=128, k=1229),
    "n25600": Shape(seed_id=4, B=2, N=25600, H=24, d=96, M=128, len_lo=8, len_hi=128, k=6400),
    "n36864_seq": Shape(seed_id=5, B=2, N=36864, H=24, d=96, M=256, len_lo=16, len_hi=256, k=7373),
}


def make_inputs(workload: str, shape: Shape = None, call: int = 0, drift_std: float = 0.05):
    """All tensors of one hot-path step of `workload` (CPU, bf16 / int32 / fp32)."""
    s = shape or WORKLOADS[workload]
    c = WORKLOADS[workload].seed_id
    inp = {
        "Q": normal_bf16((s.B, s.N, s.H, s.d), seed_for(c, T_Q, call)),
        "K": normal_bf16((s.B, s.N, s.H, s.d), seed_for(c, T_K, call)),
        "V": normal_bf16((s.B, s.N, s.H, s.d), seed_for(c, T_V, call)),
        "Ky": normal_bf16((s.B, s.M, s.H, s.d), seed_for(c, T_KY)),
        "Vy": normal_bf16((s.B, s.M, s.H, s.d), seed_for(c, T_VY)),
        "valid_len": uniform_lengths(s.B, s.len_lo, s.len_hi, seed_for(c, T_LEN)),
    }
    inp["w"] = content_weights(inp["valid_len"], s.M, seed_for(c, T_W))
    inp["Kc"] = drifted_bf16(inp["K"], drift_std, seed_for(c, T_DK, call))
    inp["Vc"] = drifted_bf16(inp["V"], drift_std, seed_for(c, T_DV, call))
    return inp


def sample_rows(N: int, count: int, seed: int) -> np.ndarray:
    """Sorted distinct query rows drawn uniformly (for sampled parity at large N)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return np.sort(rng.choice(N, size=min(count, N), replace=False))


def tiny_masks(N: int, H: int, valid_len: int, M: int, seed: int):
    """The masks of the tiny check, as CPU tensors shaped [1, H|1, n_q, n_k]:
    all-true bool, all-zero additive, row-constant additive c_i ~ U(-5, 5),
    one non-constant row, text padding (valid_len of M keys), one NaN entry."""
    rng = np.random.Generator(np.random.PCG64(seed))
    c = rng.uniform(-5.0, 5.0, size=(1, H, N, 1)).astype(np.float32)
    rowconst = np.broadcast_to(c, (1, H, N, N)).copy()
    nonconst = np.zeros((1, H, N, N), dtype=np.float32)
    i = int(rng.integers(0, N))
    nonconst[0, 0, i, int(rng.integers(0, N))] = 1.0
    pad = np.zeros((1, 1, N, M), dtype=bool)
    pad[..., :valid_len] = True
    withnan = np.zeros((1, 1, N, N), dtype=np.float32)
    withnan[0, 0, int(rng.integers(0, N)), int(rng.integers(0, N))] = np.nan
    return {
        "all_true": torch.ones((1, 1, N, N), dtype=torch.bool),
        "all_zero": torch.zeros((1, 1, N, N), dtype=torch.float32),
        "row_constant": torch.from_numpy(rowconst),
        "one_nonconstant_row": torch.from_numpy(nonconst),
        "text_padding": torch.from_numpy(pad),
        "nan_entry": torch.from_numpy(withnan),
        "_nonconst_row": i,
    }
