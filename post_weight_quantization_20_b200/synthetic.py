"""Seeded synthetic inputs for the GPTQ layer solver.

This module holds only random-number generation and storage-format handling
(rounding float32 draws to fp16 / bf16 and back).  It contains none of the
solver's arithmetic, so the float64 oracle and the CUDA path can both be fed
from it without sharing any of the method.

Distributions follow the calibration workloads the GPTQ pages describe for
OPT / LLaMA layers (weights roughly Gaussian with a few large entries;
activations heavy-tailed with a small set of outlier channels).  The datasets
the pages calibrate on (C4, WikiText-2) are not available; these draws stand
in for them.

Every array is generated in fixed-size token (or row) chunks; chunk ``k`` of
stream ``(seed, tag)`` is drawn from ``PCG64(SeedSequence([seed, tag, k]))``,
so the bytes do not depend on how many threads produce them.
"""
from __future__ import annotations

import concurrent.futures as _cf
import os
from dataclasses import dataclass

import numpy as np

CHUNK = 8192

F32 = "f32"
F16 = "f16"
BF16 = "bf16"
DTYPES = (F32, F16, BF16)


# ----------------------------------------------------------------------------
# storage formats
# ----------------------------------------------------------------------------
def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); return raw uint16 bits."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    return r


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of raw bfloat16 bits to float32."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def to_storage(a32: np.ndarray, dtype: str) -> np.ndarray:
    """float32 draws -> the storage array for ``dtype`` (fp16 as float16, bf16 as uint16 bits)."""
    if dtype == F32:
        return np.ascontiguousarray(a32, dtype=np.float32)
    if dtype == F16:
        return a32.astype(np.float16)
    if dtype == BF16:
        return f32_to_bf16_bits(a32)
    raise ValueError(dtype)


def to_f64(a: np.ndarray, dtype: str) -> np.ndarray:
    """Exact widening of a storage array to float64."""
    if dtype == BF16:
        return bf16_bits_to_f32(a).astype(np.float64)
    return np.asarray(a).astype(np.float64)


def to_f32(a: np.ndarray, dtype: str) -> np.ndarray:
    """Exact widening of a storage array to float32."""
    if dtype == BF16:
        return bf16_bits_to_f32(a)
    return np.asarray(a).astype(np.float32)


# ----------------------------------------------------------------------------
# draws
# ----------------------------------------------------------------------------
def _rng(seed: int, tag: int, k: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tag, k])))


def _student_t4(g: np.random.Generator, n: int) -> np.ndarray:
    """Student-t with 4 degrees of freedom: Z / sqrt(V/4), V ~ chi^2_4 = -2 ln(U1 U2)."""
    z = g.standard_normal(n, dtype=np.float32)
    u = g.random(2 * n, dtype=np.float32)
    # (0, 1] keeps the log finite
    u = np.float32(1.0) - u
    v = -2.0 * np.log(u[:n] * u[n:])
    return (z / np.sqrt(v * np.float32(0.25))).astype(np.float32)


def _pool_map(fn, items, threads):
    if threads <= 1 or len(items) <= 1:
        return [fn(i) for i in items]
    with _cf.ThreadPoolExecutor(max_workers=threads) as ex:
        return list(ex.map(fn, items))


def _threads() -> int:
    return max(1, min(16, os.cpu_count() or 1))


@dataclass(frozen=True)
class ActSpec:
    """Calibration activations X (tokens x cols)."""
    dist: str = "t4"              # "t4" Student-t nu=4, or "normal"
    outlier_frac: float = 0.01    # fraction of channels scaled up
    outlier_count: int = 0        # if > 0, exact number of outlier channels (overrides frac)
    outlier_mult: float = 20.0
    mix_rank: int = 0             # > 0 adds a shared low-rank component (correlated channels)
    mix_scale: float = 1.0


@dataclass(frozen=True)
class WeightSpec:
    """Layer weights W (rows x cols)."""
    sigma: float = 0.02
    outlier_frac: float = 0.0     # fraction of entries scaled up
    outlier_mult: float = 8.0


def outlier_channels(cols: int, spec: ActSpec, seed: int, tag: int) -> np.ndarray:
    n = spec.outlier_count if spec.outlier_count > 0 else int(round(spec.outlier_frac * cols))
    n = min(max(n, 0), cols)
    g = _rng(seed, tag, 1_000_003)
    return np.sort(g.choice(cols, size=n, replace=False)) if n else np.zeros(0, dtype=np.int64)


def gen_activations(tokens: int, cols: int, dtype: str, spec: ActSpec, seed: int,
                    tag: int = 0, threads: int | None = None, first_token: int = 0) -> np.ndarray:
    """X (tokens x cols) in storage format ``dtype``, generated in CHUNK-token pieces.
    ``first_token`` (a multiple of CHUNK) starts the block further into the same
    stream, so a large calibration set can be produced piece by piece: the rows
    equal those of one call that covers them all."""
    if first_token < 0 or first_token % CHUNK:
        raise ValueError(f"first_token must be a non-negative multiple of {CHUNK}")
    k0 = first_token // CHUNK
    threads = _threads() if threads is None else threads
    chan = np.ones(cols, dtype=np.float32)
    idx = outlier_channels(cols, spec, seed, tag)
    chan[idx] = np.float32(spec.outlier_mult)
    mix = None
    if spec.mix_rank > 0:
        gm = _rng(seed, tag, 1_000_004)
        mix = (gm.standard_normal((spec.mix_rank, cols), dtype=np.float32)
               * np.float32(spec.mix_scale / np.sqrt(spec.mix_rank)))
    out_dt = {F32: np.float32, F16: np.float16, BF16: np.uint16}[dtype]
    out = np.empty((tokens, cols), dtype=out_dt)
    starts = list(range(0, tokens, CHUNK))

    def work(k):
        t0 = starts[k]
        m = min(CHUNK, tokens - t0)
        g = _rng(seed, tag, k0 + k)
        if spec.dist == "t4":
            a = _student_t4(g, m * cols).reshape(m, cols)
        elif spec.dist == "normal":
            a = g.standard_normal(m * cols, dtype=np.float32).reshape(m, cols)
        else:
            raise ValueError(spec.dist)
        if mix is not None:
            zr = g.standard_normal((m, spec.mix_rank), dtype=np.float32)
            a += zr @ mix
        a *= chan
        out[t0:t0 + m] = to_storage(a, dtype)
        return None

    _pool_map(work, list(range(len(starts))), threads)
    return out


def gen_weight(rows: int, cols: int, dtype: str, spec: WeightSpec, seed: int,
               tag: int = 0, threads: int | None = None) -> np.ndarray:
    """W (rows x cols) in storage format ``dtype``: N(0, sigma^2) with a fraction of entries scaled."""
    threads = _threads() if threads is None else threads
    out_dt = {F32: np.float32, F16: np.float16, BF16: np.uint16}[dtype]
    out = np.empty((rows, cols), dtype=out_dt)
    rchunk = max(1, CHUNK * 64 // max(cols, 1))
    starts = list(range(0, rows, rchunk))

    def work(k):
        r0 = starts[k]
        m = min(rchunk, rows - r0)
        g = _rng(seed, 10_000 + tag, k)
        a = g.standard_normal(m * cols, dtype=np.float32) * np.float32(spec.sigma)
        if spec.outlier_frac > 0:
            sel = g.random(m * cols, dtype=np.float32) < np.float32(spec.outlier_frac)
            a[sel] *= np.float32(spec.outlier_mult)
        out[r0:r0 + m] = to_storage(a.reshape(m, cols), dtype)
        return None

    _pool_map(work, list(range(len(starts))), threads)
    return out


def gen_spd(cols: int, seed: int, cond: float = 100.0, diag_only: bool = False) -> np.ndarray:
    """A float64 symmetric positive definite test matrix Q diag(eig) Q^T with eigenvalues
    log-spaced over [1, cond] (diag_only: a random positive diagonal)."""
    g = _rng(seed, 77, 0)
    if diag_only:
        return np.diag(g.uniform(0.5, 4.0, size=cols))
    q, r = np.linalg.qr(g.standard_normal((cols, cols)))
    q = q * np.sign(np.diag(r))
    eig = np.logspace(0.0, np.log10(cond), cols)
    g.shuffle(eig)
    m = (q * eig) @ q.T
    return 0.5 * (m + m.T)
