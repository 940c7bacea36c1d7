"""The multi-GPU layer path (sharded.py) as gloo ranks on CPU.

Calibration tokens are split unevenly over two or three ranks (some cases give a
rank no tokens) and the rows of W are split by row_range.  The library's three steps are
replaced on CPU by stand-ins: the running-mean Hessian of the rank's tokens in
torch (started, like the library's, at the other ranks' token count on a zero H),
and the oracle's factorization and sweep.  What is checked is the sharding itself:
  * the combined H equals the Hessian of all tokens and is bitwise the same on
    both ranks (each rank factors its own copy);
  * the token count is the total over ranks;
  * each rank's codes, scales and zeros are exactly its rows of the oracle's
    full-layer result on that H, and the summed losses are the full layer's.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from post_weight_quantization_20_b200 import sharded as SH


def test_row_range_partitions_rows():
    for rows in (0, 1, 7, 64, 1001):
        for world in (1, 2, 3, 8):
            spans = [SH.row_range(rows, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == rows
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        SH.row_range(5, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _cpu_steps(G, o):
    """CPU stand-ins for the library's Hessian, factorization and sweep."""
    def hessian(X, C, dev, status, chunk_tokens, stream, n_start=0):
        # the library's running mean, started at n_start tokens of a zero Hessian
        X = X.double()
        m = X.shape[0]
        if n_start > 0:
            H = torch.zeros((C, C), dtype=torch.float64)
        else:
            H = torch.full((C, C), float("nan"), dtype=torch.float64)   # like torch.empty
        if m:
            # with no tokens seen, the first chunk overwrites H (the library's rule)
            prev = H * (n_start / (n_start + m)) if n_start > 0 else 0.0
            H = prev + (2.0 / (n_start + m)) * (X.T @ X)
        return H.float(), n_start + m

    def factor(H, cfg, perm, rows, dev, status, stream):
        p, _, U = o.prepare(H.double().numpy(), cfg.damp, cfg.act_order == 1)
        return torch.from_numpy(U.astype(np.float32)), torch.from_numpy(p.astype(np.int32))

    def sweep(W, U, perm, cfg, dev, status, stream):
        p = perm.numpy().astype(np.int64)
        res = o.sweep(W.double().numpy()[:, p], U.double().numpy(), cfg.bits, cfg.group_size,
                      bool(cfg.sym), cfg.block_size)
        out = o.finalize(res, p, cfg.group_size)
        return (torch.from_numpy(out["codes"].astype(np.uint8)),
                torch.from_numpy(out["scales"].astype(np.float32)),
                torch.from_numpy(out["zeros"].astype(np.float32)),
                torch.from_numpy(out["g_idx"].astype(np.int32)),
                torch.from_numpy(out["losses"].astype(np.float64)),
                torch.from_numpy(o.pack(out["codes"], cfg.bits).view(np.int32)))
    return hessian, factor, sweep


def _rank(rank, world, port, split, qcfg, q):
    import datetime

    import torch.distributed as dist

    from oracle import gptq_ref as o
    from post_weight_quantization_20_b200 import gptq as G
    from post_weight_quantization_20_b200 import sharded as SH
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        G._hessian, G._factor, G._sweep = _cpu_steps(G, o)
        rng = np.random.default_rng(5)
        R, C = 7, 48
        X = rng.standard_normal((sum(split), C)) @ rng.standard_normal((C, C)) * 0.3
        X = X.astype(np.float32)
        W = (0.02 * rng.standard_normal((R, C))).astype(np.float32)
        t0 = sum(split[:rank])
        r0, r1 = SH.row_range(R, world, rank)
        bits, group, act = qcfg
        cfg = G.make_config(bits, group, act_order=act)
        res = SH.quantize_layer_sharded(torch.from_numpy(W[r0:r1]),
                                        torch.from_numpy(X[t0:t0 + split[rank]]), cfg,
                                        check=False)
        q.put((rank, r0, r1, res.n_tokens, res.H.numpy(), res.codes.numpy(), res.scales.numpy(),
               res.zeros.numpy(), res.losses.numpy()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
@pytest.mark.parametrize("split,qcfg", [((700, 300), (4, 16, True)), ((1000, 0), (4, 16, True)),
                                        ((500, 0, 300), (3, 0, False))],
                         ids=["2-ranks", "2-ranks-one-empty", "3-ranks-per-row"])
def test_ranks_shard_tokens_and_rows(split, qcfg):
    from oracle import gptq_ref as o
    world, port = len(split), _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, split, qcfg, q))
             for r in range(world)]
    for p in procs:
        p.start()
    out = sorted((q.get(timeout=150) for _ in range(world)), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    rng = np.random.default_rng(5)
    R, C = 7, 48
    X = (rng.standard_normal((sum(split), C)) @ rng.standard_normal((C, C)) * 0.3).astype(np.float32)
    W = (0.02 * rng.standard_normal((R, C))).astype(np.float32)
    H_all, n = o.hessian(X.astype(np.float64))
    H0 = out[0][4]
    assert all(np.array_equal(H0, t[4]) for t in out)   # every rank factors the same bits
    assert np.linalg.norm(H0 - H_all) <= 1e-6 * np.linalg.norm(H_all)
    assert all(t[3] == n for t in out)
    # the full layer on the same H: each rank holds exactly its rows
    # the ranks' config holds damp as a float32 (0.00999999977...), as the C struct does
    bits, group, act = qcfg
    p, _, U = o.prepare(H0.astype(np.float64), float(np.float32(0.01)), act)
    U = U.astype(np.float32).astype(np.float64)
    full = o.finalize(o.sweep(W.astype(np.float64)[:, p], U, bits, group, False, 128), p, group)
    for rank, r0, r1, _, _, codes, scales, zeros, losses in out:
        np.testing.assert_array_equal(codes, full["codes"][r0:r1])
        np.testing.assert_array_equal(scales, full["scales"][r0:r1].astype(np.float32))
        np.testing.assert_array_equal(zeros, full["zeros"][r0:r1].astype(np.float32))
        np.testing.assert_allclose(losses, full["losses"], rtol=1e-12, atol=1e-18)
