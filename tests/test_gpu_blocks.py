"""Shared-input groups and the round-to-nearest path.

* Layers that read the same input (q/k/v, gate/up) share one Hessian and one
  factorization: quantize_layers_shared must give exactly what separate
  quantize_layer calls give, and every weight of the group must match the
  float64 oracle on the shared Hessian at the stated tolerances.
* Round-to-nearest is the sweep with U = I (no error is fed forward): its codes
  must be the oracle's round-to-nearest on the same grids, computed from the
  original weights, except at entries whose x/s is within a hair of a rounding
  tie (the kernel forms x * (1/s), within 2 ulp of the quotient).
* On a layer with correlated inputs GPTQ's calibration objective
  tr((W - Q) H (W - Q)^T) must beat round-to-nearest's.
"""
import numpy as np
import pytest
import torch

from oracle import gptq_ref as o
from post_weight_quantization_20_b200 import gptq as G
from post_weight_quantization_20_b200 import synthetic as S
from tests.parity import compare_layer

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _dev(a, dt):
    if dt == S.BF16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(DEV)
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def test_shared_input_group_matches_separate_layers():
    C = 384
    X = S.gen_activations(3000, C, S.F16, S.ActSpec(mix_rank=6), seed=11)
    Ws = [S.gen_weight(R, C, S.F16, S.WeightSpec(), seed=20 + R) for R in (96, 160, 64)]
    cfg = G.make_config(4, 128, act_order=True)
    Xd = _dev(X, S.F16)
    shared = G.quantize_layers_shared([_dev(W, S.F16) for W in Ws], Xd, cfg)
    torch.cuda.synchronize()
    assert len(shared) == 3
    # one Hessian for the group: equal to a fresh one up to fp32 accumulation order
    # (token splits are added into H atomically, so H is reproducible only to that)
    fresh = G.quantize_layer(_dev(Ws[0], S.F16), Xd, cfg)
    torch.cuda.synchronize()
    Hs, Hf = torch.triu(shared[0].H), torch.triu(fresh.H)
    assert (torch.linalg.norm(Hs - Hf) / torch.linalg.norm(Hf)).item() <= 1e-6
    # each weight: exactly what a standalone sweep over the same U and order gives
    for W, r in zip(Ws, shared):
        R = W.shape[0]
        G_ = G.n_groups(C, cfg.group_size)
        codes = torch.empty(R, C, dtype=torch.uint8, device=DEV)
        scales = torch.empty(R, G_, device=DEV)
        zeros = torch.empty(R, G_, device=DEV)
        g_idx = torch.empty(C, dtype=torch.int32, device=DEV)
        losses = torch.empty(C, device=DEV)
        ws = G.alloc_workspace(G.GPTQ_OP_QUANTIZE, R, C, cfg, DEV)
        G.gptq_quantize_layer(_dev(W, S.F16), r.U, r.perm, cfg, codes, scales, zeros, g_idx,
                              losses, ws)
        torch.cuda.synchronize()
        assert r.U is shared[0].U and r.perm is shared[0].perm
        for k, v in (("codes", codes), ("scales", scales), ("zeros", zeros), ("g_idx", g_idx),
                     ("losses", losses)):
            assert torch.equal(getattr(r, k), v), k


def test_shared_input_group_matches_oracle():
    """q/k/v-shaped group (three weights, one input): one Hessian and one factor on the
    GPU; each weight against the oracle's sweep on the oracle's own float64 Hessian of
    the same calibration tokens, in the same (given) act-order."""
    C = 512
    X = S.gen_activations(5000, C, S.F16, S.ActSpec(outlier_frac=0.02, mix_rank=4), seed=21)
    Ws = [S.gen_weight(R, C, S.F16, S.WeightSpec(outlier_frac=0.001), seed=30 + R)
          for R in (160, 96, 64)]
    H64, n = o.hessian(S.to_f64(X, S.F16))
    perm = o.act_order_perm(H64)
    cfg = G.make_config(4, 128, act_order=G.GPTQ_ORDER_GIVEN)
    out = G.quantize_layers_shared([_dev(W, S.F16) for W in Ws], _dev(X, S.F16), cfg,
                                   perm=torch.from_numpy(perm.astype(np.int32)).to(DEV))
    torch.cuda.synchronize()
    prepared = o.prepare(H64, 0.01, False, perm)
    for k, (W, r) in enumerate(zip(Ws, out)):
        gpu = {"codes": r.codes.cpu().numpy().astype(np.int64), "scales": r.scales.cpu().numpy(),
               "zeros": r.zeros.cpu().numpy(), "losses": r.losses.cpu().numpy(),
               "g_idx": r.g_idx.cpu().numpy().astype(np.int64)}
        p, ref = compare_layer(S.to_f64(W, S.F16), H64, n, perm, gpu, 4, 128, False,
                               prepared=prepared)
        p.assert_bars(f"shared-input group, weight {k} ({W.shape[0]}x{C})")
        np.testing.assert_array_equal(r.packed.cpu().numpy().view(np.uint32),
                                      o.pack(gpu["codes"], 4))


def _oracle_rtn(W64, bits, group, sym):
    """Round-to-nearest with the oracle's grids from the original weights; also the
    pre-rounding x/s of every entry."""
    R, C = W64.shape
    codes = np.empty((R, C), dtype=np.int64)
    pre = np.empty((R, C), dtype=np.float64)
    g = group if group > 0 else C
    scales, zeros = [], []
    for j0 in range(0, C, g):
        s, z, _ = o.grid(W64[:, j0:j0 + g], bits, sym)
        c, _, t = o.quantize(W64[:, j0:j0 + g], s[:, None], z[:, None], bits)
        codes[:, j0:j0 + g] = c
        pre[:, j0:j0 + g] = t
        scales.append(s)
        zeros.append(z)
    return codes, pre, np.stack(scales, 1), np.stack(zeros, 1)


@pytest.mark.parametrize("bits,group,sym", [(4, 128, False), (3, 0, False), (4, 64, True), (2, 32, False)])
def test_rtn_matches_oracle(bits, group, sym):
    R, C = 150, 384
    W = S.gen_weight(R, C, S.F16, S.WeightSpec(outlier_frac=0.002), seed=bits * 7 + group)
    cfg = G.make_config(bits, group, sym)
    res = G.quantize_rtn(_dev(W, S.F16), cfg)
    torch.cuda.synchronize()
    codes = res.codes.cpu().numpy().astype(np.int64)
    ref, pre, s_ref, z_ref = _oracle_rtn(S.to_f64(W, S.F16), bits, group, sym)
    diff = codes != ref
    # only near-ties may round the other way, and only to the neighbouring code (a
    # symmetric grid puts each group's largest magnitude exactly on a tie, +-(maxq/2),
    # so there one entry per row and group may differ)
    dist = np.abs(pre - np.floor(pre) - 0.5)
    assert np.all(dist[diff] < 1e-5), dist[diff]
    assert np.all(np.abs(codes - ref) <= 1)
    n_groups = (C // group) if group > 0 else 1
    assert diff.sum() <= (R * n_groups if sym else 1e-3 * R * C)
    np.testing.assert_array_equal(res.zeros.cpu().numpy(), z_ref.astype(np.float32))
    np.testing.assert_allclose(res.scales.cpu().numpy(), s_ref, rtol=1e-6)
    np.testing.assert_array_equal(res.packed.cpu().numpy().view(np.uint32), o.pack(codes, bits))


def test_gptq_beats_rtn_on_the_calibration_objective():
    R, C = 128, 512
    X = S.gen_activations(4000, C, S.F16, S.ActSpec(mix_rank=8), seed=3)
    W = S.gen_weight(R, C, S.F16, S.WeightSpec(), seed=4)
    cfg = G.make_config(3, 128)
    Wd = _dev(W, S.F16)
    gq = G.quantize_layer(Wd, _dev(X, S.F16), cfg)
    rt = G.quantize_rtn(Wd, cfg)
    torch.cuda.synchronize()
    H64, _ = o.hessian(S.to_f64(X, S.F16))
    W64 = S.to_f64(W, S.F16)

    def objective(r):
        sc = r.scales.cpu().numpy().astype(np.float64)
        zc = r.zeros.cpu().numpy().astype(np.float64)
        gi = r.g_idx.cpu().numpy().astype(np.int64)
        Q = sc[:, gi] * (r.codes.cpu().numpy().astype(np.float64) - zc[:, gi])
        D = W64 - Q
        return float(np.sum((D @ H64) * D))

    e_gptq, e_rtn = objective(gq), objective(rt)
    print(f"calibration objective: GPTQ {e_gptq:.4e}, RTN {e_rtn:.4e}, ratio {e_gptq / e_rtn:.3f}")
    assert e_gptq < 0.9 * e_rtn
