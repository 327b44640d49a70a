"""A small, self-contained run of one kernel of libgdn2 for profilers (ncu).

    python -m gated_delta_rule_160_b200.profile_case --kernel chunk --n-seq 2 --iters 3
    python -m gated_delta_rule_160_b200.profile_case --kernel decode --n-seq 64 --iters 3

``chunk`` runs gdn2_chunk_fwd on the first ``n-seq`` sequences of the 16-head, T=4096,
d=128 bf16 prefill workload (2 sequences: 268 MB of inputs, larger than L2); ``decode``
runs gdn2_decode_step on ``n-seq`` sequences of the 32-head decode workload. Each kernel
is launched ``iters`` times; profile the last launches (ncu -s / -c).
"""
import argparse

import torch

import gated_delta_rule_160_b200 as G
from gated_delta_rule_160_b200 import workloads as W


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--kernel", choices=["chunk", "decode"], default="chunk")
    ap.add_argument("--n-seq", type=int, default=2)
    ap.add_argument("--iters", type=int, default=3)
    a = ap.parse_args()
    G.load_library()
    if a.kernel == "chunk":
        wl = W.WORKLOADS["prefill_b8_h16_t4096"]
        d = W.prefill_inputs(wl, "cuda", n_seq=a.n_seq)
        o = torch.empty(d["v"].shape, dtype=torch.float32, device="cuda")
        for _ in range(a.iters):
            G.gdn2_chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], n_seq=a.n_seq, o=o)
    else:
        wl = W.WORKLOADS["decode_256seq_h32"]
        S = W.decode_state(wl, "cuda", n_seq=a.n_seq)
        d = W.decode_inputs(wl, 0, "cuda", n_seq=a.n_seq)
        o = torch.empty(d["v"].shape, dtype=torch.float32, device="cuda")
        for _ in range(a.iters):
            G.gdn2_decode_step(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], S, o=o)
    torch.cuda.synchronize()
    print("profile_case done:", a.kernel, a.n_seq, a.iters)


if __name__ == "__main__":
    main()
