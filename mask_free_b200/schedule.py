"""Host-side sequencing of SAFE-DiT's attention calls over a denoising run.

The anchor set and the latest anchor a(t) follow Eq. (14); anchor calls run
the dense block and refresh the context cache (Eq. (18), (19)); the calls
between anchors run the row-selective form on the fixed partition (Eq. (15)
to (17)); the partition comes from the PCSP scores accumulated over the
warm-up calls (Eq. (9), (10)), optionally smoothed (Eq. (11)), split by
top-k (Eq. (12)). This module only decides which library calls to make and
owns the buffers they share; every computation runs in the library's CUDA
kernels through ``mask_free_b200.ops``.
"""

from __future__ import annotations

import math
from typing import Optional

import torch

from mask_free_b200 import ops


class AnchorSchedule:
    """Anchor set A over T calls: the first `warmup` calls (dense; they build
    the partition and the cache) and after them every call t with
    t % every == 0. a(t) = max{tau in A : tau < t} (Eq. (14))."""

    def __init__(self, T: int, every: int, warmup: int = 1):
        if T < 1 or every < 1 or not 1 <= warmup <= T:
            raise ValueError("need T >= 1, every >= 1 and 1 <= warmup <= T")
        self.T, self.every, self.warmup = T, every, warmup

    def is_anchor(self, t: int) -> bool:
        if not 0 <= t < self.T:
            raise ValueError(f"call index {t} outside [0, {self.T})")
        return t < self.warmup or t % self.every == 0

    def anchors(self):
        return [t for t in range(self.T) if self.is_anchor(t)]

    def last_anchor(self, t: int) -> int:
        """a(t): the latest anchor strictly before call t (t >= 1)."""
        if not 1 <= t < self.T:
            raise ValueError(f"a(t) is defined for 1 <= t < {self.T}")
        return max(a for a in range(t) if self.is_anchor(a))


class BlockAttention:
    """The attention calls of one DiT block across a run.

    Owns the context cache (K/V rows of every token, [B, N, H, d] bf16) and the
    PCSP scores / partition. ``__call__(t, Q, K, V, Ky, Vy, valid_len)``
    returns a dict:
      anchor calls:  "self" [B, N, H, d], "cross" [B, N, H, d] (the dense block)
      other calls:   "self" [B, k, H, d], "cross" [B, k, H, d] for the rows "S"
    On other calls Q, K, V may be full-size [B, N, H, d] or compact
    [B, k, H, d] (the current rows of S in the order of S).

      k          size of the sensitive set (Eq. (12)), e.g. ceil(rho N)
      w          text-token weights [B, M] fp32 of Eq. (10), or None (uniform)
      sigma      Eq. (11) smoothing before the split (None: raw scores), on
                 the grid_h x grid_w latent grid
      assembled  SRSU with K/V of S u C assembled in the kernel (no scatter;
                 the cache is only read between anchors). Off by default: at
                 the 2560^2 workload this form is measured slower than the
                 scatter followed by SRSU that the default runs.
    """

    def __init__(self, schedule: AnchorSchedule, B: int, N: int, H: int, d: int, k: int, device,
                 w: Optional[torch.Tensor] = None, sigma: Optional[float] = None, grid_h: Optional[int] = None,
                 grid_w: Optional[int] = None, assembled: bool = False, scale: Optional[float] = None):
        if not 1 <= k <= N:
            raise ValueError(f"k = {k} outside [1, N = {N}]")
        if sigma is not None and (grid_h is None or grid_w is None or grid_h * grid_w != N):
            raise ValueError("smoothing needs grid_h * grid_w == N")
        self.sched, self.B, self.N, self.H, self.d, self.k = schedule, B, N, H, d, k
        self.w, self.sigma, self.grid, self.assembled = w, sigma, (grid_h, grid_w), assembled
        self.scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
        self.Kc = torch.zeros((B, N, H, d), dtype=torch.bfloat16, device=device)
        self.Vc = torch.zeros_like(self.Kc)
        self.scores = torch.zeros((B, N), dtype=torch.float32, device=device)
        self.S: Optional[torch.Tensor] = None
        self.C: Optional[torch.Tensor] = None

    def _fix_partition(self):
        s = self.scores
        if self.sigma is not None:
            s = ops.sensitivity_field(s, self.grid[0], self.grid[1], self.sigma)
        self.S, self.C = ops.topk_partition(s, self.k)

    def __call__(self, t: int, Q, K, V, Ky, Vy, valid_len):
        if self.sched.is_anchor(t):
            # dense block (Eq. (18)) and cache refresh (Eq. (19))
            out_self = ops.attn_self(Q, K, V, scale=self.scale)
            ops.ctx_cache_scatter(K, V, None, self.Kc, self.Vc)
            if t < self.sched.warmup:
                # warm-up: the PCSP scores from the cross-attention's own
                # probabilities, accumulated over the warm-up calls
                out_cross, _, _, _ = ops.attn_cross_pcsp(Q, Ky, Vy, valid_len, self.w, scores=self.scores,
                                                         accumulate=t > 0, scale=self.scale)
                if t == self.sched.warmup - 1:
                    self._fix_partition()
            else:
                out_cross = ops.attn_cross(Q, Ky, Vy, valid_len, scale=self.scale)
            return {"self": out_self, "cross": out_cross}
        if self.S is None:
            raise RuntimeError("no partition: the warm-up calls have not run")
        compact = Q.shape[1] == self.k and self.k != self.N
        if self.assembled:
            out_self = ops.srsu_attn_assembled(Q, self.S, K, V, self.Kc, self.Vc, q_compact=compact,
                                               cur_compact=compact, scale=self.scale)
        else:
            ops.ctx_cache_scatter(K, V, self.S, self.Kc, self.Vc, src_compact=compact)
            out_self = ops.srsu_attn(Q, self.S, self.Kc, self.Vc, q_compact=compact, scale=self.scale)
        if compact:
            # the cross-attention's query rows are Q itself
            out_cross = ops.attn_cross(Q, Ky, Vy, valid_len, scale=self.scale)
        else:
            out_cross = ops.attn_cross(Q, Ky, Vy, valid_len, q_idx=self.S, scale=self.scale)
        return {"self": out_self, "cross": out_cross, "S": self.S}
