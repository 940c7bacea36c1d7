"""GPTQ against round-to-nearest on the synthetic workloads: the calibration
objective of each quantized layer.

    python -m post_weight_quantization_20_b200.compare_rtn [--workloads opt125m llama7b]
        [--tokens 262144]

For every layer both quantizers run on the GPU (quantize_layer and quantize_rtn,
same grids and packing); the objective is the quadratic term of the layer's loss,
tr((W - Q) H (W - Q)^T) with the undamped H = 2 X^T X / n (GPTQ量化算法深度解析
§2.1), evaluated in float64 from the layer's own Hessian.  One line per layer:
both objectives, their ratio, and each relative to tr(W H W^T).
"""
from __future__ import annotations

import argparse

import torch

from . import gptq as G
from . import synthetic as S
from .workloads import ORDER, WORKLOADS


def dequantize(codes: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor,
               g_idx: torch.Tensor) -> torch.Tensor:
    """Q[r, c] = scales[r, g_idx[c]] (codes[r, c] - zeros[r, g_idx[c]]) in float64."""
    g = g_idx.long()
    s = scales.double()[:, g]
    z = zeros.double()[:, g]
    return s * (codes.double() - z)


def objective(W: torch.Tensor, Q: torch.Tensor, H: torch.Tensor) -> float:
    """tr((W - Q) H (W - Q)^T) in float64; H symmetric, given by its upper triangle."""
    Hu = torch.triu(H.double())
    Hs = Hu + Hu.T - torch.diag(torch.diagonal(Hu))
    D = W.double() - Q
    return float(((D @ Hs) * D).sum())


def _device(a, dt, dev):
    if dt == S.BF16:
        return torch.from_numpy(a.view("int16")).view(torch.bfloat16).to(dev)
    return torch.from_numpy(a).to(dev)


def main(argv=None) -> None:
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--workloads", nargs="+", default=["opt125m", "llama7b"],
                    choices=list(ORDER))
    ap.add_argument("--tokens", type=int, default=None, help="calibration tokens per layer")
    a = ap.parse_args(argv)
    dev = torch.device("cuda", torch.cuda.current_device())
    print(f"{'workload':10} {'layer':18} {'quantizer':16} {'GPTQ':>11} {'RTN':>11} {'ratio':>6} "
          f"{'GPTQ rel':>9} {'RTN rel':>9}")
    for wname in a.workloads:
        wl = WORKLOADS[wname]
        T = a.tokens or wl.tokens
        for l in wl.layers:
            W = _device(S.gen_weight(l.rows, l.cols, wl.wdtype, wl.wspec, seed=1234, tag=l.tag),
                        wl.wdtype, dev)
            X = _device(S.gen_activations(T, l.cols, wl.xdtype, wl.xspec, seed=1234, tag=l.tag),
                        wl.xdtype, dev)
            for q in wl.quant:
                cfg = G.make_config(q.bits, q.group_size, q.sym, q.act_order, q.damp,
                                    q.block_size)
                gq = G.quantize_layer(W, X, cfg)
                rt = G.quantize_rtn(W, cfg)
                H = gq.H
                e_g = objective(W, dequantize(gq.codes, gq.scales, gq.zeros, gq.g_idx), H)
                e_r = objective(W, dequantize(rt.codes, rt.scales, rt.zeros, rt.g_idx), H)
                base = objective(W, torch.zeros_like(W, dtype=torch.float64), H)
                print(f"{wname:10} {l.name:18} {q.label():16} {e_g:11.4e} {e_r:11.4e} "
                      f"{e_g / e_r:6.3f} {e_g / base:9.2e} {e_r / base:9.2e}", flush=True)
            del X, W
            torch.cuda.empty_cache()


if __name__ == "__main__":
    main()
