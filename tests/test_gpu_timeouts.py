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
