"""Run one layer (or one stage of it) on seeded device-resident inputs.

    python -m post_weight_quantization_20_b200.run_layer --rows 768 --cols 3072 \
        --tokens 16384 [--op layer|hessian|prepare|quantize] [--repeat 3] [--bits 4 --group 128]

Inputs are drawn on the GPU (X ~ N(0, 1) in fp16, W ~ N(0, 0.02^2) in fp16, one
fixed seed; ``quantize`` times the sweep and packing alone, on a U and order
prepared once beforehand), every op runs ``--repeat`` times untimed and then ``--repeat`` times
between CUDA events, and one line with the mean time per call is printed.  Meant
for quick timings of a shape and as a small, fixed command line to put under a
profiler (the untimed calls are the warm-up a profiler can skip with ``-s``).
"""
from __future__ import annotations

import argparse

import torch

from . import gptq as G


def main(argv=None) -> None:
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--rows", type=int, default=768)
    ap.add_argument("--cols", type=int, default=3072)
    ap.add_argument("--tokens", type=int, default=16384)
    ap.add_argument("--op", choices=["layer", "hessian", "prepare", "quantize"], default="layer")
    ap.add_argument("--repeat", type=int, default=3)
    ap.add_argument("--bits", type=int, default=4)
    ap.add_argument("--group", type=int, default=128)
    ap.add_argument("--act-order", action="store_true")
    a = ap.parse_args(argv)

    dev = torch.device("cuda", torch.cuda.current_device())
    G.load_library()
    gen = torch.Generator(device=dev)
    gen.manual_seed(0)
    R, C, T = a.rows, a.cols, a.tokens
    X = torch.randn(T, C, device=dev, generator=gen).half()
    W = (0.02 * torch.randn(R, C, device=dev, generator=gen)).half()
    cfg = G.make_config(a.bits, a.group, act_order=a.act_order)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    H = torch.empty(C, C, device=dev)
    U = torch.empty(C, C, device=dev)
    perm = torch.empty(C, dtype=torch.int32, device=dev)
    wsp = G.alloc_workspace(G.GPTQ_OP_PREPARE, R, C, cfg, dev)
    G.gptq_hessian_accumulate(H, 0, X, status)

    if a.op == "hessian":
        def run():
            G.gptq_hessian_accumulate(H, 0, X, status)
        work = f"{float(T) * C * (C + 1) / 1e12:.4f} TFLOP per call"
    elif a.op == "prepare":
        def run():
            G.gptq_prepare(H, cfg, U, perm, wsp, status)
        work = f"{2.0 * C ** 3 / 3e12:.4f} TFLOP per call (2/3 C^3)"
    elif a.op == "quantize":
        G.gptq_prepare(H, cfg, U, perm, wsp, status)
        Gn = G.n_groups(C, cfg.group_size)
        codes = torch.empty(R, C, dtype=torch.uint8, device=dev)
        scales = torch.empty(R, Gn, device=dev)
        zeros = torch.empty(R, Gn, device=dev)
        g_idx = torch.empty(C, dtype=torch.int32, device=dev)
        losses = torch.empty(C, device=dev)
        packed = torch.empty(R, G.packed_words(C, cfg.bits), dtype=torch.int32, device=dev)
        wsq = G.alloc_workspace(G.GPTQ_OP_QUANTIZE, R, C, cfg, dev)

        def run():
            G.gptq_quantize_layer(W, U, perm, cfg, codes, scales, zeros, g_idx, losses, wsq, status)
            G.gptq_pack(codes, cfg.bits, packed)
        work = f"sweep + lazy updates + pack, {float(R) * C * C / 1e12:.4f} TFLOP of update per call"
    else:
        def run():
            G.quantize_layer(W, X, cfg, check=False)
        work = "Hessian + prepare + sweep + pack, with their allocations"

    for _ in range(a.repeat):
        run()
    torch.cuda.synchronize(dev)
    G.check_status(status, a.op)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(a.repeat):
        run()
    e1.record()
    torch.cuda.synchronize(dev)
    G.check_status(status, a.op)
    ms = e0.elapsed_time(e1) / a.repeat
    print(f"op={a.op} rows={R} cols={C} tokens={T}: {ms:.3f} ms per call ({work})")


if __name__ == "__main__":
    main()
