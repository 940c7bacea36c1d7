"""Canary margins around every buffer the library writes.

Each output, both workspaces and the status word are views into larger byte
buffers whose margins hold a fixed pattern (tests/guards.py).  A layer is run
through the four C calls on odd shapes that take the single-panel, SIMT-fallback,
tensor-core and two-level update paths; afterwards every margin must be intact,
and the outputs must equal those of the same calls on plain buffers given the
same Hessian (H is reproducible only to fp32 addition order between runs, so the
reference factors a copy of the guarded run's H).
"""
import pytest
import torch

from post_weight_quantization_20_b200 import gptq as G
from post_weight_quantization_20_b200 import synthetic as S
from tests.guards import Guarded

pytestmark = pytest.mark.gpu
DEV = "cuda"

CASES = [  # R, C, bits, group, act-order
    (1, 33, 4, 0, False),        # one panel, unaligned rows of X (SIMT Hessian)
    (17, 129, 3, 32, True),      # C % 4 != 0: SIMT trailing update
    (33, 200, 4, 64, False),     # tensor-core trailing update, ragged panel
    (40, 384, 2, 128, True),
    (5, 1400, 4, 128, True),     # more than 1024 columns: the two-level update
]


@pytest.mark.parametrize("R,C,bits,group,act", CASES,
                         ids=[f"{c[0]}x{c[1]}-{c[2]}b-g{c[3]}{'-act' if c[4] else ''}" for c in CASES])
def test_outputs_stay_inside_their_buffers(R, C, bits, group, act):
    X = torch.from_numpy(S.gen_activations(3 * C + 100, C, S.F16, S.ActSpec(mix_rank=4),
                                           seed=C)).to(DEV)
    W = torch.from_numpy(S.gen_weight(R, C, S.F16, S.WeightSpec(), seed=R + C)).to(DEV)
    cfg = G.make_config(bits, group, act_order=act)
    Gn = G.n_groups(C, group)
    shapes = {
        "H": ((C, C), torch.float32), "U": ((C, C), torch.float32), "perm": ((C,), torch.int32),
        "wsp": ((G.gptq_workspace_size(G.GPTQ_OP_PREPARE, R, C, cfg),), torch.uint8),
        "wsq": ((G.gptq_workspace_size(G.GPTQ_OP_QUANTIZE, R, C, cfg),), torch.uint8),
        "codes": ((R, C), torch.uint8), "scales": ((R, Gn), torch.float32),
        "zeros": ((R, Gn), torch.float32), "g_idx": ((C,), torch.int32),
        "losses": ((C,), torch.float32), "packed": ((R, G.packed_words(C, bits)), torch.int32),
    }
    bufs = {k: Guarded(s, dt, DEV) for k, (s, dt) in shapes.items()}
    bufs["status"] = Guarded((1,), torch.int32, DEV, fill=torch.zeros(1, dtype=torch.int32))
    b = {k: v.t for k, v in bufs.items()}
    G.gptq_hessian_accumulate(b["H"], 0, X, b["status"])
    G.gptq_prepare(b["H"], cfg, b["U"], b["perm"], b["wsp"], b["status"])
    G.gptq_quantize_layer(W, b["U"], b["perm"], cfg, b["codes"], b["scales"], b["zeros"],
                          b["g_idx"], b["losses"], b["wsq"], b["status"])
    G.gptq_pack(b["codes"], bits, b["packed"])
    torch.cuda.synchronize()
    assert int(b["status"].item()) == 0
    broken = [k for k, v in bufs.items() if not v.intact()]
    assert not broken, f"writes past the end of {broken}"

    # the same calls on plain buffers, from a copy of the same H
    H = torch.triu(b["H"]).clone()
    U = torch.empty(C, C, device=DEV)
    perm = torch.empty(C, dtype=torch.int32, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    G.gptq_prepare(H, cfg, U, perm, G.alloc_workspace(G.GPTQ_OP_PREPARE, R, C, cfg, DEV), st)
    out = {k: torch.empty(s, dtype=dt, device=DEV) for k, (s, dt) in shapes.items()
           if k in ("codes", "scales", "zeros", "g_idx", "losses", "packed")}
    G.gptq_quantize_layer(W, U, perm, cfg, out["codes"], out["scales"], out["zeros"],
                          out["g_idx"], out["losses"],
                          G.alloc_workspace(G.GPTQ_OP_QUANTIZE, R, C, cfg, DEV), st)
    G.gptq_pack(out["codes"], bits, out["packed"])
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert torch.equal(perm, b["perm"]) and torch.equal(U, b["U"])
    for k, v in out.items():
        assert torch.equal(v, b[k]), k
