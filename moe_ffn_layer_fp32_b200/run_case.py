"""Runs one synthetic workload through the layer and prints per-stage device times.

    python -m moe_ffn_layer_fp32_b200.run_case --workload c2 --iters 3
    python -m moe_ffn_layer_fp32_b200.run_case --workload c4 --tokens 64 --iters 3     # decode batch
    python -m moe_ffn_layer_fp32_b200.run_case --workload c1 --chain 24 --iters 3      # stack of 24 layers

Meant as a fixed, small command line for profilers (one handle, `--iters`
forwards after one warm-up forward, nothing else on the device).  Weights and
x are the seeded synthetic draws of `synth.WORKLOADS`; the weights are
quantised on the device by the library's Eq. (6) kernel.
"""
from __future__ import annotations

import argparse

import numpy as np
import torch

from . import synth
from .layer import MoELayer, quantize_int4


def quantized_weights(w: synth.Workload, device: torch.device, layer: int = 0):
    lw = synth.workload_layer(w, layer)
    gu_w, gu_s, dn_w, dn_s = [], [], [], []
    for g in range(w.E + 1):
        p, s = quantize_int4(torch.from_numpy(lw.w_gate_up[g]).to(device))
        gu_w.append(p.reshape(-1))
        gu_s.append(s.reshape(-1))
        p, s = quantize_int4(torch.from_numpy(lw.w_down[g]).to(device))
        dn_w.append(p.reshape(-1))
        dn_s.append(s.reshape(-1))
    wr = torch.from_numpy(lw.w_router).to(device)
    bias = None if lw.router_bias is None else torch.from_numpy(lw.router_bias).to(device)
    return (wr, bias, torch.cat(gu_w), torch.cat(gu_s), torch.cat(dn_w), torch.cat(dn_s)), lw


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--workload", default="c2", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--tokens", type=int, default=None, help="tokens per forward (default: the workload's T)")
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--no-decode", action="store_true", help="keep T <= 64 on the prefill kernels")
    ap.add_argument("--cuda-cores", action="store_true")
    ap.add_argument("--deterministic", action="store_true")
    ap.add_argument("--tc-int8", action="store_true", help="prefill GEMMs on the kind::i8 tensor-core kernels")
    ap.add_argument("--chain", type=int, default=0,
                    help="run a stack of this many layers (layer l's weights seeded as the workload's layer l) "
                         "through mmoe_forward_chain")
    args = ap.parse_args(argv)
    if args.chain:
        return chain(args)

    dev = torch.device("cuda", 0)
    w = synth.WORKLOADS[args.workload]
    T = w.T if args.tokens is None else args.tokens
    tensors, lw = quantized_weights(w, dev)
    L = MoELayer(w.d, w.h, shared_hidden=w.hs, n_experts=w.E, top_k=w.k, max_tokens=T,
                 has_router_bias=lw.router_bias is not None, decode=not args.no_decode,
                 cuda_cores=args.cuda_cores, deterministic=args.deterministic, tc_int8=args.tc_int8)
    L.load(*tensors)
    del tensors
    x = torch.from_numpy(synth.workload_x(w, T=T).view(np.int16)).to(dev).view(torch.bfloat16)
    y = torch.empty((T, w.d), dtype=torch.float32, device=dev)
    L.forward(x, y)
    torch.cuda.synchronize()
    L.profile(True)
    for _ in range(args.iters):
        L.forward(x, y)
    stages = L.profile_read()
    L.profile(False)
    L.close()
    per = {k: round(v[1] * 1e3 / max(args.iters, 1), 2) for k, v in stages.items() if v[0] or v[1]}
    print(f"{w.name} T={T}: per forward, us by stage: {per}", flush=True)
    return 0


def chain(args) -> int:
    dev = torch.device("cuda", 0)
    w = synth.WORKLOADS[args.workload]
    T = w.T if args.tokens is None else args.tokens
    layers = []
    for l in range(args.chain):
        tensors, lw = quantized_weights(w, dev, l)
        L = MoELayer(w.d, w.h, shared_hidden=w.hs, n_experts=w.E, top_k=w.k, max_tokens=T,
                     has_router_bias=lw.router_bias is not None)
        L.load(*tensors)
        layers.append(L)
        del tensors
    x = torch.from_numpy(synth.workload_x(w, T=T).view(np.int16)).to(dev).view(torch.bfloat16)
    ys = [torch.empty((T, w.d), dtype=torch.float32, device=dev) for _ in layers]
    MoELayer.forward_chain(layers, x, ys)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.iters):
        MoELayer.forward_chain(layers, x, ys)
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / max(args.iters, 1)
    print(f"{w.name} T={T}, {len(layers)} layers: {us:.1f} us per stack, {us / len(layers):.2f} us per layer",
          flush=True)
    for L in layers:
        L.close()
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
