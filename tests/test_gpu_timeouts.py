"""Failure detection without a GPU fault: bounded device waits that are made to run out.

Each case launches a kernel whose wait can never be satisfied (an mbarrier nothing
arrives on; a grid barrier a CTA leaves without arriving at) and checks that the
wait gives up, that GPTQ_ERR_TIMEOUT reaches the caller's status word, and that
the context still computes correct results afterwards.
"""
import time

import numpy as np
import pytest
import torch

from oracle import gptq_ref as o
from post_weight_quantization_20_b200 import gptq as G

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _context_still_works():
    # a packing call whose result is known exactly
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 16, size=(3, 70), dtype=np.uint8)
    c = torch.from_numpy(codes).to(DEV)
    packed = torch.empty(3, G.packed_words(70, 4), dtype=torch.int32, device=DEV)
    G.gptq_pack(c, 4, packed)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(packed.cpu().numpy().view(np.uint32), o.pack(codes.astype(np.int64), 4))


@pytest.mark.parametrize("which,limit_s", [(G.GPTQ_SELFTEST_MBARRIER, 5.0),
                                           (G.GPTQ_SELFTEST_GRID_BARRIER, 30.0)])
def test_bounded_wait_reports_timeout(which, limit_s):
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    G.gptq_selftest_timeout(which, status)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    code = int(status.item())
    print(f"selftest {which}: gave up after {dt:.3f} s, status {G.status_names(code)}")
    assert code & G.GPTQ_ERR_TIMEOUT
    assert dt < limit_s
    _context_still_works()


def test_selftest_rejects_bad_arguments():
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    with pytest.raises(G.GPTQError):
        G.gptq_selftest_timeout(7, status)


def _hessian_matches_oracle(X16):
    H = torch.empty(X16.shape[1], X16.shape[1], device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    G.gptq_hessian_accumulate(H, 0, X16, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    H64, _ = o.hessian(X16.cpu().numpy().astype(np.float64))
    iu = np.triu_indices(X16.shape[1])
    Hg = H.cpu().numpy().astype(np.float64)
    assert np.linalg.norm(Hg[iu] - H64[iu]) <= 1e-5 * np.linalg.norm(H64[iu])


@pytest.mark.parametrize("kernel", ["hessian", "gemm3"])
def test_pipeline_waits_give_up_and_drain(kernel):
    """The tensor-core kernels' own waits run out (a limit of two polls, shorter than
    any copy takes): each CTA stops, waits for its copies and MMAs in flight, frees
    its TMEM, and the call reports GPTQ_ERR_TIMEOUT; afterwards, with the default
    limit, the same kernels compute correct results."""
    rng = np.random.default_rng(3)
    X = torch.from_numpy(rng.standard_normal((8192, 1024)).astype(np.float16)).to(DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    G.gptq_debug_set_wait_limit(2)
    try:
        if kernel == "hessian":
            H = torch.empty(1024, 1024, device=DEV)
            G.gptq_hessian_accumulate(H, 0, X, st)
        else:
            # the sweep's lazy updates of a 2048-column layer run on the 3xTF32 products
            C, R = 2048, 256
            cfg = G.make_config(4, 128)
            W = torch.from_numpy((0.02 * rng.standard_normal((R, C))).astype(np.float16)).to(DEV)
            U = torch.eye(C, device=DEV)
            perm = torch.arange(C, dtype=torch.int32, device=DEV)
            Gn = G.n_groups(C, 128)
            G.gptq_quantize_layer(W, U, perm, cfg, torch.empty(R, C, dtype=torch.uint8, device=DEV),
                                  torch.empty(R, Gn, device=DEV), torch.empty(R, Gn, device=DEV),
                                  torch.empty(C, dtype=torch.int32, device=DEV),
                                  torch.empty(C, device=DEV),
                                  G.alloc_workspace(G.GPTQ_OP_QUANTIZE, R, C, cfg, DEV), st)
        torch.cuda.synchronize()
    finally:
        G.gptq_debug_set_wait_limit(0)
    code = int(st.item())
    print(f"{kernel} with a two-poll wait limit: status {G.status_names(code)}")
    assert code & G.GPTQ_ERR_TIMEOUT
    _context_still_works()
    _hessian_matches_oracle(X[:2048])
