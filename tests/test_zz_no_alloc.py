"""gptq_prepare_static: the prepare step for callers that cannot allocate device memory.

Such callers (a plugin inside a framework whose caching allocator already holds
the device memory, code with a fixed memory budget, a service that must not
allocate after start-up) cannot hand the library a workspace; this entry point
uses a scratch array compiled into the library instead.  The test calls it
through the C ABI twice in a row, on two different layers, and checks each result
against gptq_prepare with a caller workspace.  It lives in its own file, collected
last, and passes both alone in a fresh process and after the other tests.
"""
import numpy as np
import pytest
import torch

from post_weight_quantization_20_b200 import gptq as G
from post_weight_quantization_20_b200 import synthetic as S

pytestmark = pytest.mark.gpu
DEV = "cuda"
U_TOL = 1e-3   # the relative Frobenius tolerance the U parity tests use


def _hessian(cols, seed):
    X = S.gen_activations(4 * cols + 256, cols, S.F16, S.ActSpec(mix_rank=4), seed=seed)
    H = torch.empty(cols, cols, device=DEV)
    G.gptq_hessian_accumulate(H, 0, torch.from_numpy(X).to(DEV))
    return H


def _with_workspace(H, cfg):
    C = H.shape[0]
    U = torch.empty(C, C, device=DEV)
    perm = torch.empty(C, dtype=torch.int32, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    ws = G.alloc_workspace(G.GPTQ_OP_PREPARE, 0, C, cfg, DEV)
    G.gptq_prepare(H, cfg, U, perm, ws, st)
    return U, perm, st


def _static(H, cfg):
    C = H.shape[0]
    U = torch.full((C, C), float("nan"), device=DEV)
    perm = torch.full((C,), -1, dtype=torch.int32, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    G.gptq_prepare_static(H, cfg, U, perm, st)
    return U, perm, st


def _rel(a, b):
    return float(torch.linalg.norm(a - b) / torch.linalg.norm(b))


def test_static_scratch_matches_workspace_on_two_calls_in_a_row():
    layers = [(_hessian(640, 1), G.make_config(4, 128, act_order=True)),
              (_hessian(G.GPTQ_STATIC_MAX_COLS, 2), G.make_config(3, 0, act_order=False))]
    static = [_static(H, cfg) for H, cfg in layers]           # two calls back to back
    ref = [_with_workspace(H, cfg) for H, cfg in layers]
    torch.cuda.synchronize()
    for (Us, ps, ss), (Ur, pr, sr) in zip(static, ref):
        assert int(ss.item()) == 0 and int(sr.item()) == 0
        assert torch.equal(ps, pr)
        assert _rel(Us, Ur) <= U_TOL
        assert torch.isfinite(Us).all()


def test_static_scratch_refuses_layers_above_its_limit():
    C = G.GPTQ_STATIC_MAX_COLS + 1
    H = torch.eye(C, device=DEV)
    U = torch.empty(C, C, device=DEV)
    perm = torch.empty(C, dtype=torch.int32, device=DEV)
    with pytest.raises(G.GPTQError) as e:
        G.gptq_prepare_static(H, G.make_config(4, 128), U, perm)
    assert e.value.code == G.GPTQ_ERR_WORKSPACE
