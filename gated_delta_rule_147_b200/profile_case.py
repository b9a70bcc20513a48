"""Runs one chunk-forward workload a few times (for ncu captures).

    python -m gated_delta_rule_147_b200.profile_case --workload gdn --launches 3
    python -m gated_delta_rule_147_b200.profile_case --decode --launches 3
    python -m gated_delta_rule_147_b200.profile_case --workload gdn --bwd --launches 2

Workloads are the seeded ones of gated_delta_rule_147_b200.inputs; --heads
and --seq shrink a workload (B=1, H=heads, T=seq) for small captures.
"""
from __future__ import annotations

import argparse


def main():
    import torch

    from gated_delta_rule_147_b200 import TIED, chunk_fwd, decode_step
    from gated_delta_rule_147_b200.inputs import DECODE, WORKLOADS, make_chunk_inputs, \
        make_decode_state, make_decode_step

    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="gdn", choices=sorted(WORKLOADS))
    ap.add_argument("--launches", type=int, default=3)
    ap.add_argument("--heads", type=int, default=0)
    ap.add_argument("--seq", type=int, default=0)
    ap.add_argument("--decode", action="store_true")
    ap.add_argument("--bwd", action="store_true", help="run the backward pass (chunk_bwd)")
    a = ap.parse_args()
    dev = torch.device("cuda:0")
    if a.decode:
        S = make_decode_state(DECODE).to(dev)
        st = {k: v.to(dev) for k, v in make_decode_step(DECODE, 0).items()}
        for _ in range(a.launches):
            decode_step(st["q"], st["k"], st["v"], st["alpha"], st["b"], st["w"], S)
        torch.cuda.synchronize()
        return
    wl = WORKLOADS[a.workload]
    if a.heads:
        wl = wl.with_(B=1, H=a.heads)
    if a.seq:
        wl = wl.with_(T=a.seq)
    inp = make_chunk_inputs(wl)
    d = {k: (v.to(dev) if hasattr(v, "to") else v) for k, v in inp.items()}
    w = TIED if wl.w == "tied" else d["w"]
    o = torch.empty((wl.B, wl.T, wl.H, wl.dv), dtype=d["v"].dtype, device=dev)
    ST = torch.empty((wl.B, wl.H, wl.dk, wl.dv), dtype=torch.float32, device=dev)
    if a.bwd:
        from gated_delta_rule_147_b200 import chunk_bwd, gdr_chunk_bwd_workspace_size
        from gated_delta_rule_147_b200.inputs import make_cotangents
        cot = make_cotangents(wl)
        dO, dST = cot["dO"].to(dev), cot["dS_T"].to(dev)
        ws = torch.empty(gdr_chunk_bwd_workspace_size(wl.B, wl.T, wl.H, wl.dk, wl.dv),
                         dtype=torch.uint8, device=dev)
        for _ in range(a.launches):
            chunk_bwd(d["q"], d["k"], d["v"], d["alpha"], d["b"], w, d["S0"], dO=dO, dS_T=dST,
                      workspace=ws)
        torch.cuda.synchronize()
        return
    for _ in range(a.launches):
        chunk_fwd(d["q"], d["k"], d["v"], d["alpha"], d["b"], w, d["S0"], out=o, S_T=ST)
    torch.cuda.synchronize()


if __name__ == "__main__":
    main()
