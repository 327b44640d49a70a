"""A small, self-contained run of one kernel of libgdn2 for profilers (ncu).

    python -m gated_delta_rule_160_b200.profile_case --kernel chunk --n-seq 2 --iters 3
    python -m gated_delta_rule_160_b200.profile_case --kernel prologue --n-seq 2 --iters 3
    python -m gated_delta_rule_160_b200.profile_case --kernel decode --n-seq 64 --iters 3
    python -m gated_delta_rule_160_b200.profile_case --kernel bwd --n-seq 2 --T 1024 --iters 2
    python -m gated_delta_rule_160_b200.profile_case --kernel grouped --n-seq 2 --T 8192 --iters 3
    python -m gated_delta_rule_160_b200.profile_case --kernel serving --n-seq 64 --iters 3

``chunk`` runs gdn2_chunk_fwd on the first ``n-seq`` sequences of the 16-head, T=4096,
d=128 bf16 prefill workload (2 sequences: 268 MB of inputs, larger than L2; ``T`` cuts them);
``prologue`` runs gdn2_chunk_fwd_prologue on raw projections of the same shapes (seeded
normal pre-activations, as the benchmark's fused pre-processing leg makes them); ``decode``
runs gdn2_decode_step on ``n-seq`` sequences of the 32-head decode workload; ``bwd`` runs
gdn2_chunk_bwd (gradients of sum(o * dO)) on the prefill workload's first ``n-seq``
sequences; ``grouped`` runs gdn2_chunk_fwd on the grouped-head workload (16 query/key heads
shared by 32 value heads, with an initial state), its sequences cut to ``T`` tokens;
``serving`` runs gdn2_decode_multi (4 tokens per sequence) on ``n-seq`` sequences of the
32-head decode workload whose states sit at seeded-random slots of a pool twice as large. Each
kernel is launched ``iters`` times; profile the last launches (ncu -s / -c).
"""
import argparse

import torch

import gated_delta_rule_160_b200 as G
from gated_delta_rule_160_b200 import workloads as W


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--kernel", choices=["chunk", "prologue", "decode", "bwd", "grouped", "serving"], default="chunk")
    ap.add_argument("--n-seq", type=int, default=2)
    ap.add_argument("--T", type=int, default=None, help="tokens per sequence (chunk, bwd, grouped)")
    ap.add_argument("--iters", type=int, default=3)
    a = ap.parse_args()
    G.load_library()
    if a.kernel in ("chunk", "bwd"):
        wl = W.WORKLOADS["prefill_b8_h16_t4096"]
        d = W.prefill_inputs(wl, "cuda", n_seq=a.n_seq, T=a.T)
        o = torch.empty(d["v"].shape, dtype=torch.float32, device="cuda")
        if a.kernel == "chunk":
            for _ in range(a.iters):
                G.gdn2_chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], n_seq=a.n_seq, o=o)
        else:
            dO = torch.randn(o.shape, generator=torch.Generator(device="cuda").manual_seed(wl.seed + 29),
                             device="cuda")
            ws = None
            for _ in range(a.iters):
                G.gdn2_chunk_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], dO, n_seq=a.n_seq,
                                 want_dS0=False, workspace=ws)
    elif a.kernel == "prologue":
        wl = W.WORKLOADS["prefill_b8_h16_t4096"]
        d = W.prefill_inputs(wl, "cuda", n_seq=a.n_seq, T=a.T)
        T_all = d["v"].shape[0]
        gen = torch.Generator(device="cuda").manual_seed(wl.seed + 17)
        rn = lambda *shp: torch.randn(*shp, generator=gen, device="cuda").to(wl.dtype)
        raw = dict(q=rn(T_all, wl.h_qk, wl.dk), k=rn(T_all, wl.h_qk, wl.dk), a=rn(T_all, wl.h_v, wl.dk),
                   b=rn(T_all, wl.h_v, wl.dk), w=rn(T_all, wl.h_v, wl.dv))
        o = torch.empty(d["v"].shape, dtype=torch.float32, device="cuda")
        for _ in range(a.iters):
            G.gdn2_chunk_fwd(raw["q"], raw["k"], d["v"], raw["a"], raw["b"], raw["w"], n_seq=a.n_seq, o=o,
                             prologue=True)
    elif a.kernel == "grouped":
        wl = W.WORKLOADS["grouped_b2_qk16_v32_t32768"]
        d = W.prefill_inputs(wl, "cuda", n_seq=a.n_seq, T=a.T)
        o = torch.empty(d["v"].shape, dtype=torch.float32, device="cuda")
        S_T = torch.empty_like(d["S0"])
        for _ in range(a.iters):
            G.gdn2_chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], S0=d["S0"], n_seq=a.n_seq,
                             o=o, S_T=S_T)
    elif a.kernel == "serving":
        wl = W.WORKLOADS["decode_256seq_h32"]
        N, n_tok = a.n_seq, 4
        pool = torch.zeros((2 * N, wl.h_v, wl.dk, wl.dv), dtype=torch.float32, device="cuda")
        perm = torch.randperm(2 * N, generator=torch.Generator().manual_seed(wl.seed))[:N]
        pool[perm.to("cuda")] = W.decode_state(wl, "cuda", n_seq=N)
        slots = perm.to(torch.int32).to("cuda")
        t_ = W.token_inputs(N * n_tok, wl.h_qk, wl.h_v, wl.dk, wl.dv, wl.dtype, "cuda", wl.seed * 7919)
        x = {k: t.view(N, n_tok, *t.shape[1:]) for k, t in t_.items()}
        o = torch.empty((N, n_tok, wl.h_v, wl.dv), dtype=torch.float32, device="cuda")
        for _ in range(a.iters):
            G.gdn2_decode_multi(*(x[k] for k in ("q", "k", "v", "log_alpha", "b", "w")), pool, slots=slots, o=o)
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
