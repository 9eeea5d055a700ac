"""Run one kernel of the hot path a few times on one workload, for profilers.

    python -m mask_free_b200.profile_case --kernel self --workload n4096 --launches 3

Kernels: self, srsu, cross, pcsp, topk, scatter, classify, linear (the
row-selective block's QKV layer: the k rows of S of a [B, N, H*d] hidden
state, H*d -> 3*H*d). Inputs are
generated on the device (standard normals in bf16, like the benchmark), so
the process holds only the tensors of that one call (n4096: ~0.2 GB).
"""

from __future__ import annotations

import argparse

import torch

from mask_free_b200 import ops, synth


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--kernel", required=True, choices=["self", "srsu", "cross", "pcsp", "topk", "scatter",
                                                        "classify", "linear"])
    ap.add_argument("--workload", default="n4096", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--launches", type=int, default=3)
    a = ap.parse_args()
    s = synth.WORKLOADS[a.workload]
    dev = torch.device("cuda")
    g = torch.Generator(device=dev).manual_seed(s.seed_id)

    def bf(rows):
        return torch.randn((s.B, rows, s.H, s.d), generator=g, device=dev).to(torch.bfloat16)

    lens = synth.uniform_lengths(s.B, s.len_lo, s.len_hi, 1).to(dev)
    S = torch.sort(torch.randperm(s.N, device=dev, generator=g)[:s.k])[0].to(torch.int32)
    S = S.expand(s.B, s.k).contiguous()
    if a.kernel in ("self", "srsu", "cross", "pcsp", "scatter"):
        Q, K, V = bf(s.N), bf(s.N), bf(s.N)
    if a.kernel in ("cross", "pcsp"):
        Ky, Vy = bf(s.M), bf(s.M)
    if a.kernel == "linear":
        dm = s.H * s.d
        X = torch.randn((s.B, s.N, dm), generator=g, device=dev).to(torch.bfloat16)
        Wt = (torch.randn((3 * dm, dm), generator=g, device=dev) / dm ** 0.5).to(torch.bfloat16)
    for _ in range(a.launches):
        if a.kernel == "self":
            ops.attn_self(Q, K, V)
        elif a.kernel == "srsu":
            ops.srsu_attn(Q, S, K, V)
        elif a.kernel == "cross":
            ops.attn_cross(Q, Ky, Vy, lens)
        elif a.kernel == "pcsp":
            ops.pcsp_topk(Q, Ky, lens, None)
        elif a.kernel == "topk":
            sc = torch.randn((s.B, s.N), generator=g, device=dev)
            ops.topk_partition(sc, s.k)
        elif a.kernel == "scatter":
            ops.ctx_cache_scatter(K, V, S, Q, Q.clone(), src_compact=False)
        elif a.kernel == "linear":
            ops.gather_linear(X, Wt, S=S)
        elif a.kernel == "classify":
            m = torch.ones((s.B, 1, s.N, s.N), dtype=torch.bool, device=dev)
            ops.mask_classify(m)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    print("ok", a.kernel, a.workload, a.launches)


if __name__ == "__main__":
    main()
