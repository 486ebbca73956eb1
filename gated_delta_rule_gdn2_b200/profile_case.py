"""One workload of the benchmark, run on its own for an ncu capture.

    python -m gated_delta_rule_gdn2_b200.profile_case {train,prefill,decode,long} [--batch B] [--T T] [--reps N]

train: gdn2_chunk_fwd_save then gdn2_chunk_bwd_saved (B x T4096 x H16, d 128),
N times each; prefill: gdn2_chunk_fwd at that shape; decode: gdn2_decode_step
at B256 H16 (fp32 state in place); long: gdn2_chunk_fwd at B1 H16 and the given
T.  Inputs are drawn on the device from the benchmark's distributions, so a
capture starts within seconds.  Launch order per rep: train = forward, then
backward; the others one kernel (the segmented long forward: its passes).
"""
from __future__ import annotations

import argparse


def main():
    import torch
    import gated_delta_rule_gdn2_b200 as g
    from gated_delta_rule_gdn2_b200.inputs import make_inputs_device

    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=["train", "prefill", "decode", "long"])
    ap.add_argument("--batch", type=int, default=8)
    ap.add_argument("--T", type=int, default=4096)
    ap.add_argument("--reps", type=int, default=2)
    a = ap.parse_args()
    dev = torch.device("cuda", 0)
    D, H = 128, 16
    sh = torch.cuda.current_stream().cuda_stream
    names = ("q", "k", "v", "log_alpha", "b", "w")
    if a.case == "decode":
        B = 256
        x = make_inputs_device(B, 1, H, D, D, seed=1002, device=dev)
        toks = [x[n][:, 0].contiguous() for n in names]
        S = x["S0"].clone()
        o = torch.empty((B, H, D), dtype=torch.bfloat16, device=dev)
        for _ in range(a.reps):
            assert g.gdn2_decode_step(*toks, S, o, B, H, D, D, g.GDN2_BF16, sh) == 0
    else:
        B, T = (1, a.T) if a.case == "long" else (a.batch, a.T)
        x = make_inputs_device(B, T, H, D, D, seed=1004, device=dev, alpha_mu=4.0 if a.case == "long" else 3.0)
        toks = [x[n] for n in names]
        o = torch.empty((B, T, H, D), dtype=torch.bfloat16, device=dev)
        ST = torch.empty((B, H, D, D), dtype=torch.float32, device=dev)
        nfw = g.gdn2_chunk_fwd_workspace(B, T, H, D, D, g.GDN2_BF16)
        wsf = torch.empty(max(nfw, 16), dtype=torch.uint8, device=dev)
        if a.case == "train":
            dO = torch.randn((B, T, H, D), device=dev).to(torch.bfloat16)
            nst = g.gdn2_chunk_states_bytes(B, T, H, D, D, g.GDN2_BF16)
            nbw = g.gdn2_chunk_bwd_saved_workspace(B, T, H, D, D, g.GDN2_BF16)
            states = torch.empty(nst, dtype=torch.uint8, device=dev)
            wsb = torch.empty(max(nbw, 16), dtype=torch.uint8, device=dev)
            grads = [torch.empty_like(toks[0]) for _ in range(6)]
            dS0 = torch.empty_like(ST)
            for _ in range(a.reps):
                assert g.gdn2_chunk_fwd_save(*toks, x["S0"], o, ST, states, B, T, H, D, D, g.GDN2_BF16, wsf, nfw,
                                             sh) == 0
                assert g.gdn2_chunk_bwd_saved(*toks, x["S0"], dO, None, states, *grads, dS0, B, T, H, D, D,
                                              g.GDN2_BF16, wsb, nbw, sh) == 0
        else:
            for _ in range(a.reps):
                assert g.gdn2_chunk_fwd(*toks, x["S0"], o, ST, B, T, H, D, D, g.GDN2_BF16, wsf, nfw, sh) == 0
    torch.cuda.synchronize()
    assert g.gdn2_get_device_status() == 0
    print("ok", a.case)


if __name__ == "__main__":
    main()
