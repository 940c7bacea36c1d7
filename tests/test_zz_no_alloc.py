"""gptq_prepare_static: the prepare step for callers that cannot allocate device memory.

Such callers (a plugin inside a framework whose caching allocator already holds
the device memory, code with a fixed memory budget, a service that must not
allocate after start-up) cannot hand the library a workspace; this entry point
uses a scratch array compiled into the library instead.  The test calls it
through the C ABI twice in a row, on two different layers, and checks each result
against gptq_prepare with a caller workspace; that a call after a warm-up one
changes neither the device's free memory nor torch's reserved memory; and that a
call with a caller-given order right after a descending-diagonal call (whose
leftovers share the array) still checks and uses the given order.  It lives in its own file, collected
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


def test_static_scratch_allocates_nothing():
    H = _hessian(512, 3)
    cfg = G.make_config(4, 128, act_order=True)
    U = torch.empty(512, 512, device=DEV)
    perm = torch.empty(512, dtype=torch.int32, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    G.gptq_prepare_static(H, cfg, U, perm, st)          # warm-up: the one-time set-up
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    reserved0 = torch.cuda.memory_reserved()
    G.gptq_prepare_static(H, cfg, U, perm, st)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    assert torch.cuda.memory_reserved() == reserved0
    assert int(st.item()) == 0


def test_static_scratch_given_order_after_descending_order():
    C = 384
    H = _hessian(C, 4)
    _static(H, G.make_config(4, 128, act_order=True))     # leaves its counts in the array
    given = torch.from_numpy(np.random.default_rng(5).permutation(C).astype(np.int32)).to(DEV)
    cfg = G.make_config(4, 128, act_order=G.GPTQ_ORDER_GIVEN)
    U = torch.empty(C, C, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    G.gptq_prepare_static(H, cfg, U, given.clone(), st)
    ref_perm = given.clone()
    Uw = torch.empty(C, C, device=DEV)
    sw = torch.zeros(1, dtype=torch.int32, device=DEV)
    G.gptq_prepare(H, cfg, Uw, ref_perm, G.alloc_workspace(G.GPTQ_OP_PREPARE, 0, C, cfg, DEV), sw)
    torch.cuda.synchronize()
    assert int(st.item()) == 0 and int(sw.item()) == 0
    assert _rel(U, Uw) <= U_TOL
    # a bad permutation is still caught after a call that left other counts behind
    bad = given.clone()
    bad[3] = bad[4]
    st2 = torch.zeros(1, dtype=torch.int32, device=DEV)
    G.gptq_prepare_static(H, cfg, U, bad, st2)
    torch.cuda.synchronize()
    assert int(st2.item()) & G.GPTQ_ERR_INVALID_ARG
