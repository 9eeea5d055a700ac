"""fp64 CPU oracle for the SAFE-DiT attention hot path (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline legs may import this package. See ``safe_oracle`` for the
definitions and the equations they follow.
"""

from .safe_oracle import *  # noqa: F401,F403
from .safe_oracle import (DTYPE_BF16, DTYPE_BOOL, DTYPE_F16, DTYPE_F32, DTYPE_U8,  # noqa: F401
                          attention, cache_scatter, ceil_k, classify_mask, cross_attention,
                          pcsp_scores, row_in_R, sdpa_masked, softmax_rows, srsu_attention,
                          text_probabilities, topk_partition, gaussian_taps, reflect_index, smooth_scores,
                          norm01, sensitivity_field, partition_indicator, sw_cfg, gelu_tanh,
                          gathered_linear)
