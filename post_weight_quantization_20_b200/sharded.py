"""One linear layer over several GPUs, one process per GPU (torch.distributed).

The layer shards two ways (GPTQ量化算法深度解析 §3.1 step 1 and §2.4):

* tokens: H = 2/N sum_t x_t x_t^T is a mean over the calibration tokens.  The
  ranks first add up their token counts (N); rank r then accumulates its share
  (2/N) sum_{t in r} x_t x_t^T with the library, its running mean started at the
  N - n_r tokens of the other ranks, and one all-reduce (a sum) of the shares
  gives the layer's H on every rank;
* rows: given U and the column order, the compensation runs along each row only,
  so every rank sweeps its own rows of W; the per-column losses (sums over rows)
  take one more all-reduce.

Every rank factors the reduced H itself.  The all-reduce leaves the same bits on
every rank and the factorization is deterministic (each output tile is computed
by one CTA in a fixed order; the damping mean is a fixed-order reduction), so U
and the order agree across ranks without a broadcast.

The collectives run on the stream the library's kernels use (torch's current
stream inside `_on(stream)`), so no extra synchronisation is needed.  This is
the plain form of the exchange: the Hessian's last accumulation and its
all-reduce are separate launches.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import gptq as G


def row_range(rows: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous rows [r0, r1) of rank `rank`: the first rows % world ranks take one
    row more than the others."""
    if world < 1 or not 0 <= rank < world or rows < 0:
        raise ValueError("need rows >= 0 and 0 <= rank < world")
    base, extra = divmod(rows, world)
    r0 = rank * base + min(rank, extra)
    return r0, r0 + base + (1 if rank < extra else 0)


def token_count(X_local) -> int:
    """Tokens of a rank's calibration input: a tokens x cols tensor or a sequence of
    such chunks (the count is needed before the first accumulation)."""
    if isinstance(X_local, torch.Tensor):
        return int(X_local.shape[0])
    if isinstance(X_local, (list, tuple)):
        return sum(int(x.shape[0]) for x in X_local)
    raise TypeError("X_local must be a tensor or a list / tuple of chunks")


def total_tokens(n_local: int, device, group=None) -> int:
    """The number of calibration tokens over the ranks of `group`."""
    n = torch.tensor([int(n_local)], dtype=torch.int64, device=device)
    dist.all_reduce(n, group=group)
    total = int(n.item())
    if total <= 0:
        raise ValueError("no calibration tokens on any rank")
    return total


def _any_rank(flag: bool, device, group=None) -> bool:
    t = torch.tensor([1 if flag else 0], dtype=torch.int32, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return bool(t.item())


def quantize_layer_sharded(W_rows: torch.Tensor, X_local, cfg: G.gptq_config, group=None,
                           perm: torch.Tensor | None = None, chunk_tokens: int | None = None,
                           stream=None, check: bool = True) -> G.LayerResult:
    """Quantize this rank's rows W_rows (rows_r x cols) of a layer whose calibration
    tokens are split over the ranks (X_local: this rank's tokens x cols, or a list of
    such chunks; it may hold no tokens).  Returns this rank's rows of
    codes, scales, zeros and packed words, and the layer's g_idx, order, H, U, total
    token count and per-column losses summed over all ranks' rows."""
    dev = W_rows.device
    C = W_rows.shape[1]
    with G._on(stream):
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        n_local = token_count(X_local)
        total = total_tokens(n_local, dev, group)
        H, n = G._hessian(X_local, C, dev, status, chunk_tokens, stream,
                          n_start=total - n_local)
        dist.all_reduce(H, group=group)       # the sum of the shares: the layer's H
        U, perm = G._factor(H, cfg, perm, W_rows.shape[0], dev, status, stream)
        codes, scales, zeros, g_idx, losses, packed = G._sweep(W_rows, U, perm, cfg, dev, status,
                                                               stream)
        dist.all_reduce(losses, group=group)
    if check:
        # every rank raises together, so that none is left waiting in a later collective
        if _any_rank(int(status.item()) != 0, dev, group):
            G.check_status(status, "quantize_layer_sharded")
            raise G.GPTQError(G.GPTQ_ERR_INVALID_ARG, "quantize_layer_sharded: another rank failed")
    return G.LayerResult(codes, scales, zeros, g_idx, losses, perm, packed, H, U, total)
