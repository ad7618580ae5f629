"""Runs a few launches of one hot kernel on a synthetic workload, for profilers.

    python -m vector_quantized_mx_b200.profile_case decode|decode_native|prefill|prefill_native|moe|quant [--reps 3]

decode          mxc_linear, PostScale E4M3-B16, M=16, K=4096, N=9216 (split-K decode path)
decode_native   mxc_native_linear on the same decoded weights
prefill         mxc_linear, PreScale E8M0-B32, M=2048 (--rows), K=4096, N=9216 (BF16 out)
prefill_native  mxc_native_linear on the same decoded weights
moe             mxc_moe_linear, PreScale+ E4M3-B16, gate/up 3072x4096, 128 experts, Zipf(1.1) top-8
swiglu          mxc_moe_gate_up_swiglu on the same gate/up weights and rows
quant           mxc_quantize_act, E8M0-B32, 8192 x 4096 BF16
Each case checks the device error word after its launches.
"""
from __future__ import annotations

import argparse

import numpy as np
import torch

from . import build, mxc, synth


def _dev_bf16(bits, dev):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(torch.bfloat16)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=["decode", "decode_native", "decode_long", "prefill", "prefill_native", "moe",
                                     "swiglu", "quant"])
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--rows", type=int, default=2048, help="prefill cases: activation rows (at most 8192)")
    args = ap.parse_args(argv)
    build.build()
    dev = torch.device("cuda", 0)
    if args.case == "decode_long":
        # K = N = 8192 at M = 16 (PostScale E4M3-B16, 256 x 256 QBlocks): two rounds a CTA
        w = synth.config5_weight(256, "postscale", "e4m3_b16")
        x = synth.config5_activations(16)
        pw = mxc.pack_weight(w, dev)
        a = mxc.quantize_act(_dev_bf16(x, dev), w.fmt)
        for _ in range(args.reps):
            mxc.linear(a, pw)
    elif args.case.startswith("decode"):
        w, x = synth.config2(16)
        pw = mxc.pack_weight(w, dev)
        a = mxc.quantize_act(_dev_bf16(x, dev), w.fmt)
        nat = mxc.decode_weight(pw) if args.case == "decode_native" else None
        for _ in range(args.reps):
            mxc.linear(a, pw) if nat is None else mxc.native_linear(a, nat)
    elif args.case.startswith("prefill"):
        w, x = synth.config3()
        pw = mxc.pack_weight(w, dev)
        a = mxc.quantize_act(_dev_bf16(x[:args.rows], dev), w.fmt)
        nat = mxc.decode_weight(pw) if args.case == "prefill_native" else None
        for _ in range(args.reps):
            if nat is None:
                mxc.linear(a, pw, torch.bfloat16)
            else:
                mxc.native_linear(a, nat, torch.bfloat16)
    elif args.case in ("moe", "swiglu"):
        row_tok, off = synth.config4_routing()
        xg = synth.config4_activations("gate_up", row_tok)
        experts = [mxc.pack_weight(synth.config4_expert(e, "gate_up"), dev) for e in range(synth.MOE_EXPERTS)]
        offd = torch.from_numpy(off.astype(np.int32)).to(dev)
        a = mxc.quantize_act_grouped(_dev_bf16(xg, dev), "e4m3_b16", offd)
        h_ts = torch.tensor([0.01], dtype=torch.float32, device=dev)
        for _ in range(args.reps):
            if args.case == "moe":
                mxc.moe_linear(a, offd, experts, torch.bfloat16)
            else:
                mxc.moe_gate_up_swiglu(a, offd, experts, h_tscale=h_ts)
    else:
        x = synth.make_activations(3, 8192, 4096, outliers=True)
        xd = _dev_bf16(x, dev)
        out = mxc.empty_act(8192, 4096, "e8m0_b32", dev)
        for _ in range(args.reps):
            mxc.quantize_act(xd, "e8m0_b32", out=out)
    torch.cuda.synchronize()
    status = mxc.get_device_error()
    if status != 0:
        raise SystemExit(f"device error {status}")
    print("ok", args.case)


if __name__ == "__main__":
    main()
