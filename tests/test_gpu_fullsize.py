"""Full-size layers of the five workloads, in the launch configuration bench.py uses.

Every layer is quantized whole on the GPU (262144 calibration tokens).  What the
float64 oracle can afford decides the check:
  * sampled Hessian entries H[i][j], each computed by the oracle from the two
    columns alone (all layers);
  * the permutation is a permutation, and with act-order it is descending in the
    oracle's diagonal (computed per column) up to fp32 accumulation error;
  * codes lie on the grid, packed words equal the oracle's packing of the codes,
    and (codes, scales, zeros, g_idx) dequantize consistently;
  * layers with cols <= 4096: the oracle forms H in float64, factors it, and sweeps
    a sample of rows with the near-tie replay -- codes must match exactly on those
    rows (forced near-ties <= 0.1%), scales within 1e-4, zeros equal;
  * larger layers: properties that hold at any size -- the per-column losses sum
    to 1/2 tr((W-Q) Hp (W-Q)^T) on the GPU's own Hessian (1e-3 relative), and
    GPTQ's calibration objective tr((W-Q) H (W-Q)^T) on sampled rows is no worse
    than round-to-nearest's.
The 12288 x 49152 fc2 layer of the OPT-175B-shaped workload (a 26 GB fp16
calibration set) is too large for this harness and is not run here.
"""
import numpy as np
import pytest
import torch

from oracle import gptq_ref as o
from post_weight_quantization_20_b200 import gptq as G
from post_weight_quantization_20_b200 import synthetic as S
from post_weight_quantization_20_b200.workloads import ORDER, WORKLOADS
from tests.parity import compare_layer

pytestmark = [pytest.mark.gpu, pytest.mark.slow]
DEV = "cuda"
TAU = 2e-3
SAMPLE_ROWS = 48
ORACLE_FULL_MAX_COLS = 4096


def _cases():
    out = []
    for wname in ORDER:
        wl = WORKLOADS[wname]
        for l in wl.layers:
            if l.cols * wl.tokens > 262144 * 16384:
                continue                           # the 12288 x 49152 layer
            settings = wl.quant if l is wl.layers[0] else wl.quant[:1]
            for qi, q in enumerate(settings):
                out.append(pytest.param(wname, l.name, qi, id=f"{wname}-{l.name}-{q.label()}"))
    return out


_DATA = {}


def _data(wname, lname):
    key = (wname, lname)
    if key not in _DATA:
        _DATA.clear()                              # keep one layer's inputs in memory
        wl = WORKLOADS[wname]
        l = [x for x in wl.layers if x.name == lname][0]
        W = S.gen_weight(l.rows, l.cols, wl.wdtype, wl.wspec, seed=1234, tag=l.tag)
        X = S.gen_activations(wl.tokens, l.cols, wl.xdtype, wl.xspec, seed=1234, tag=l.tag)
        _DATA[key] = (wl, l, W, X)
    return _DATA[key]


def _dev(a, dt):
    if dt == S.BF16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(DEV)
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


@pytest.mark.parametrize("wname,lname,qi", _cases())
def test_full_size_layer(wname, lname, qi):
    wl, l, W, X = _data(wname, lname)
    q = wl.quant[qi]
    R, C = l.rows, l.cols
    cfg = G.make_config(q.bits, q.group_size, q.sym, q.act_order, q.damp, q.block_size)
    res = G.quantize_layer(_dev(W, wl.wdtype), _dev(X, wl.xdtype), cfg)
    torch.cuda.synchronize()
    Hg = res.H.cpu().numpy()
    codes = res.codes.cpu().numpy().astype(np.int64)
    scales = res.scales.cpu().numpy()
    zeros = res.zeros.cpu().numpy()
    g_idx = res.g_idx.cpu().numpy().astype(np.int64)
    perm = res.perm.cpu().numpy().astype(np.int64)
    losses = res.losses.cpu().numpy().astype(np.float64)
    packed = res.packed.cpu().numpy().view(np.uint32)
    rng = np.random.default_rng(C)

    # Hessian entries, one by one
    pairs = [(i, i) for i in rng.integers(0, C, 8)] + \
            [tuple(sorted(p)) for p in rng.integers(0, C, size=(24, 2))] + [(0, C - 1)]
    for i, j in pairs:
        Hij, _ = o.hessian(S.to_f64(X[:, [i, j]], wl.xdtype))
        assert abs(Hg[i, j] - Hij[0, 1]) <= 1e-5 * np.sqrt(Hij[0, 0] * Hij[1, 1]), (i, j)

    # ordering
    assert np.array_equal(np.sort(perm), np.arange(C))
    if q.act_order:
        d = np.empty(C)
        for c0 in range(0, C, 512):
            Xc = S.to_f64(X[:, c0:c0 + 512], wl.xdtype)
            d[c0:c0 + 512] = 2.0 * np.einsum("ij,ij->j", Xc, Xc) / Xc.shape[0]
        dp = d[perm]
        assert np.all(dp[:-1] >= dp[1:] - 1e-5 * np.abs(dp[1:]))
    else:
        assert np.array_equal(perm, np.arange(C))

    # codes, packing, dequantization
    maxq = 2 ** q.bits - 1
    assert codes.min() >= 0 and codes.max() <= maxq
    np.testing.assert_array_equal(packed, o.pack(codes, q.bits))
    g = q.group_size
    if g > 0:
        inv = np.empty(C, dtype=np.int64)
        inv[perm] = np.arange(C)
        np.testing.assert_array_equal(g_idx, inv // g)
    else:
        assert np.all(g_idx == 0)
    assert np.all(zeros == np.rint(zeros)) and zeros.min() >= 0 and zeros.max() <= maxq
    assert np.all(scales > 0) and np.all(np.isfinite(losses)) and np.all(losses >= 0)

    W64 = S.to_f64(W, wl.wdtype)
    rows = np.sort(rng.choice(R, size=min(SAMPLE_ROWS, R), replace=False))
    if C <= ORACLE_FULL_MAX_COLS:
        H64, n = np.zeros((C, C)), 0
        for t0 in range(0, X.shape[0], 32768):
            H64, n = o.hessian_accumulate(H64, n, S.to_f64(X[t0:t0 + 32768], wl.xdtype))
        # the oracle's own order; where it differs from the GPU's the keys must be
        # near-tied (validated above), and the GPU's order is then used for the sweep
        use_perm = o.act_order_perm(H64) if q.act_order else np.arange(C)
        if not np.array_equal(use_perm, perm):
            dd = np.diag(H64)
            diff = np.nonzero(use_perm != perm)[0]
            assert np.all(np.abs(dd[use_perm[diff]] - dd[perm[diff]]) <= 1e-5 * dd[perm[diff]])
            print(f"{wname} {lname}: {len(diff)} positions of the order differ at near-tied keys")
            use_perm = perm
        gpu = {"codes": codes[rows], "scales": scales[rows], "zeros": zeros[rows],
               "losses": np.zeros(C), "g_idx": g_idx}
        p, ref = compare_layer(W64[rows], H64, n, use_perm, gpu, q.bits, q.group_size, q.sym, TAU,
                               damp=q.damp, block_size=q.block_size)
        print(f"{wname} {lname} {q.label()} rows={len(rows)}: {p.summary()}")
        assert p.bad_hints == 0 and p.code_mismatch == 0
        assert p.forced_frac <= 1e-3
        assert p.zero_diff == 0.0 and p.scale_rel <= 1e-4
        assert p.recon_rel <= 5e-3
    else:
        # loss identity on the GPU's own Hessian (all rows)
        Hd = np.triu(Hg.astype(np.float64)) + np.triu(Hg.astype(np.float64), 1).T
        lam = q.damp * np.mean(np.diag(Hd))
        Hp = Hd[np.ix_(perm, perm)] + lam * np.eye(C)
        Qg = scales[:, g_idx].astype(np.float64) * (codes - zeros[:, g_idx].astype(np.float64))
        D = (W64 - Qg)[:, perm]
        total = 0.5 * float(np.sum((D @ Hp) * D))
        assert abs(float(losses.sum()) - total) <= 1e-3 * total
        # GPTQ's calibration objective tr(dW H dW^T) (undamped H, sampled rows) is no
        # worse than round-to-nearest's on the same grids' rule
        Wp = W64[rows][:, perm]
        if g > 0:
            Qr = np.empty_like(Wp)
            for j0 in range(0, C, g):
                s_, z_, _ = o.grid(Wp[:, j0:j0 + g], q.bits, q.sym)
                _, Qr[:, j0:j0 + g], _ = o.quantize(Wp[:, j0:j0 + g], s_[:, None], z_[:, None], q.bits)
        else:
            s_, z_, _ = o.grid(Wp, q.bits, q.sym)
            _, Qr, _ = o.quantize(Wp, s_[:, None], z_[:, None], q.bits)
        Hpu = Hd[np.ix_(perm, perm)]
        Dg = D[rows]
        Dr = Wp - Qr
        err_gptq = float(np.sum((Dg @ Hpu) * Dg))
        err_rtn = float(np.sum((Dr @ Hpu) * Dr))
        print(f"{wname} {lname} {q.label()}: objective gptq/rtn on sampled rows = {err_gptq / err_rtn:.3f}")
        assert err_gptq <= err_rtn
