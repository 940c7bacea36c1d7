"""Float64 CPU oracle of the GPTQ layer-wise quantization solver.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import or run
this module.  It shares no code with the CUDA library and imports nothing from
the product package; it is plain, slow and written to be checked against the
pages by eye.

Sources (the pages are cited by title and section):

* [Deep-dive] "GPTQ量化算法深度解析：从Hessian曲率到大模型单卡部署" (sheratonhq.com):
  §1.2 round-to-nearest, §2.1 Taylor objective, §2.2 OBS compensation formula,
  §2.4 fixed order / lazy batch updates / Cholesky, §3.1 the four-step
  per-layer flow, §3.3 group size, desc_act, damp_percent.
* [Deploy-guide] the lansai.wang GPTQ deployment guide, table "bits、group_size、
  sym 与 desc_act 分别影响什么" (bits, group size, sym/asym, desc_act, damp).
* [Qwen-Int4] "通义千问1.5-1.8B-Chat-GPTQ-Int4模型压缩技术解析", §2.1 (min-max
  uniform grid over 16 integer levels).
* [gptq-for-llama] the ainews.cool article on gptq-for-llama, "工程细节"
  (four 4-bit codes packed into one 16-bit integer).

Readings taken where the pages are silent or garbled (each is repeated in the
design notes):

* H = 2 X^T X / n with n = number of calibration tokens, accumulated as a
  running mean; the pages write H = 2 X X^T + lambda I with X as cols x tokens
  and an absolute lambda ([Deep-dive §3.1 step 1]).  Damping is relative:
  lambda = damp * mean(diag H) ([Deep-dive §3.3] damp_percent).
* The OBS formula of [Deep-dive §2.2] is printed with the weight w_q in the
  numerator (the pruning form).  For quantization the numerator is the
  quantization error w_q - quant(w_q), and the compensation runs over the
  not-yet-quantized columns F: delta_F = -(w_q - Q_q)/[H_F^-1]_qq * [H_F^-1]_{F,q}.
  With U the upper Cholesky factor of H^-1 (U^T U = H^-1),
  [H_F^-1]_{q,F} / [H_F^-1]_qq = U[q,F] / U[q,q], which is the sweep below.
* Act-order ([Deep-dive §3.3] desc_act) sorts columns by descending diag(H)
  (mean squared activation of the channel), stable (ties keep the lower index).
* Grid ([Qwen-Int4 §2.1], [Deploy-guide] sym row): 2^b levels, min-max range
  widened to contain 0 so the zero-point is an integer code.  Asymmetric:
  lo = min(0, min v), hi = max(0, max v), [-1, 1] if both are 0,
  s = (hi - lo)/maxq, z = rint(-lo/s).  Symmetric: m = max|v| (1 if 0),
  range [-m, m], s = 2m/maxq, z = (maxq + 1)/2.
  code = clamp(rint(x/s) + z, 0, maxq), Q = s (code - z); rint rounds half to even.
* The pages fix no precision for these rounding decisions, so they are taken in
  float32 (the precision the kernels use): x, lo, hi are rounded to float32 and
  the divisions and rint are IEEE float32 operations.  All other state is float64.
* Per-row grids come from the row before any compensation; group grids are
  computed when the sweep reaches the group's first column, from the current
  (compensated) values of its g columns ([Deep-dive §3.1 step 3]).  Groups are
  consecutive in sweep order; g_idx maps each original column to its group.
* Lazy batching needs every group to see all earlier compensation: supported
  when g divides B or B divides g.
* Packing: each row's codes form a little-endian, LSB-first bitstream of b-bit
  fields stored in uint32 words (the same bytes as "four 4-bit codes in one
  16-bit integer" for b = 4, [gptq-for-llama]); rows are padded with zero bits
  to ceil(cols*b/32) words.

Parity pins: every function here is checked against closed forms, hand-worked
fixtures, brute force and independent solves in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import numpy as np
import scipy.linalg as sla


class NotPositiveDefinite(ArithmeticError):
    """The damped (permuted) Hessian has a non-positive pivot."""


# -----------------------------------------------------------------------------
# step 1: Hessian  [Deep-dive §3.1 step 1], [Deep-dive §2.1]
# -----------------------------------------------------------------------------
def _xtx(Xd: np.ndarray) -> np.ndarray:
    """X^T X by general matrix products over blocks of at most 8192 columns (the
    symmetric rank-k routine behind a plain X.T @ X fails in OpenBLAS once the
    result has 2^31 or more entries, e.g. 49152 x 49152)."""
    C = Xd.shape[1]
    if C <= 8192:
        return Xd.T @ Xd
    G = np.empty((C, C))
    for j0 in range(0, C, 8192):
        G[:, j0:j0 + 8192] = Xd.T @ Xd[:, j0:j0 + 8192]
    return G


def hessian_accumulate(H: np.ndarray, n: int, X: np.ndarray):
    """Running-mean update H <- H n/(n+m) + 2/(n+m) X^T X for a chunk X (m x cols).

    Returns (H, n + m).  X is upcast exactly to float64.
    """
    m = int(X.shape[0])
    if m == 0:
        return H, n
    Xd = np.asarray(X, dtype=np.float64)
    H = H * (n / (n + m)) + (2.0 / (n + m)) * _xtx(Xd)
    return H, n + m


def hessian(X: np.ndarray, chunk: int | None = None):
    """H = 2/n X^T X over all tokens of X, accumulated chunk by chunk with the same
    running-mean update as hessian_accumulate (each entry rounded the same way; the
    update is done in place on H so that a wide layer needs no C x C temporaries
    beyond the chunk's X^T X)."""
    cols = X.shape[1]
    H = np.zeros((cols, cols))
    n = 0
    step = chunk or max(1, X.shape[0])
    for t in range(0, X.shape[0], step):
        Xd = np.asarray(X[t:t + step], dtype=np.float64)
        m = int(Xd.shape[0])
        G = _xtx(Xd)
        G *= 2.0 / (n + m)
        H *= n / (n + m)
        H += G
        del G
        n += m
    return H, n


# -----------------------------------------------------------------------------
# step 2: damping, act-order, inverse Cholesky factor
#         [Deep-dive §3.1 step 2], [Deep-dive §2.4], [Deep-dive §3.3]
# -----------------------------------------------------------------------------
def damp(H: np.ndarray, rel: float) -> np.ndarray:
    """H + lambda I with lambda = rel * mean(diag H) (a new array; lambda is added to
    the diagonal entries only, which is H + lambda I entry for entry)."""
    lam = rel * float(np.mean(np.diag(H))) if H.shape[0] else 0.0
    Hd = np.array(H, dtype=np.float64, copy=True)
    Hd[np.diag_indices(H.shape[0])] += lam
    return Hd


def act_order_perm(H: np.ndarray) -> np.ndarray:
    """Columns by descending diag(H); equal keys keep ascending original index."""
    return np.argsort(-np.diag(H), kind="stable").astype(np.int64)


# SciPy's LAPACK here takes 32-bit indices: above this order an n x n matrix has
# 2^31 or more entries and its routines fail; NumPy's own (64-bit) LAPACK and
# symmetric products crash on matrices that large (49152^2).  Above it the
# factorizations run as the textbook block algorithms over WIDE_BLOCK columns, each
# block step a LAPACK call of order WIDE_BLOCK or a general matrix product.
LAPACK32_MAX_ORDER = 46340
WIDE_BLOCK = 8192


def _cholesky_lower_blocked(A: np.ndarray, nb: int = WIDE_BLOCK, overwrite: bool = False):
    """Lower L with L L^T = A (its lower triangle is read) by the right-looking block
    Cholesky algorithm: for each diagonal block k, L_kk = chol(A_kk); the blocks
    below it L_ik = A_ik L_kk^-T; then A_ij -= L_ik L_jk^T on the trailing lower
    blocks.  With overwrite, A's storage becomes L."""
    n = A.shape[0]
    L = A if overwrite else np.array(A, dtype=np.float64, copy=True)
    for k0 in range(0, n, nb):
        k1 = min(k0 + nb, n)
        try:
            Lkk = sla.cholesky(L[k0:k1, k0:k1], lower=True, check_finite=True)
        except (np.linalg.LinAlgError, ValueError) as e:
            raise NotPositiveDefinite(str(e)) from e
        L[k0:k1, k0:k1] = Lkk
        L[k0:k1, k1:] = 0.0
        if k1 == n:
            break
        P = sla.solve_triangular(Lkk, L[k1:, k0:k1].T, lower=True, check_finite=False).T
        L[k1:, k0:k1] = P
        for j0 in range(k1, n, nb):
            j1 = min(j0 + nb, n)
            L[j0:, j0:j1] -= P[j0 - k1:] @ P[j0 - k1:j1 - k1].T
    return L


def _tri_inverse_lower_blocked(L: np.ndarray, nb: int = WIDE_BLOCK) -> np.ndarray:
    """L^-1 for lower triangular L by block forward substitution on the identity:
    X_jj = L_jj^-1 and, below it, X_ij = -L_ii^-1 sum_{j <= k < i} L_ik X_kj."""
    n = L.shape[0]
    X = np.zeros((n, n))
    for j0 in range(0, n, nb):
        j1 = min(j0 + nb, n)
        for i0 in range(j0, n, nb):
            i1 = min(i0 + nb, n)
            if i0 == j0:
                rhs = np.eye(j1 - j0)
            else:
                rhs = -(L[i0:i1, j0:i0] @ X[j0:i0, j0:j1])
            X[i0:i1, j0:j1] = sla.solve_triangular(L[i0:i1, i0:i1], rhs, lower=True,
                                                    check_finite=False)
    return X


def _lower_gram_of_lower(X: np.ndarray, nb: int = WIDE_BLOCK) -> np.ndarray:
    """The lower triangle (by block columns; zeros above them) of X^T X for lower
    triangular X: entry (i, j) sums X[k, i] X[k, j] over k >= j, since X[k, j] = 0
    for k < j, so block column j0 .. j1-1 takes only rows k >= j0."""
    n = X.shape[0]
    G = np.zeros((n, n))
    for j0 in range(0, n, nb):
        j1 = min(j0 + nb, n)
        G[j0:, j0:j1] = X[j0:, j0:].T @ X[j0:, j0:j1]
    return G


def _inverse_cholesky_upper_wide(Hp: np.ndarray, nb: int = WIDE_BLOCK) -> np.ndarray:
    """The same route for orders above LAPACK32_MAX_ORDER, on the block algorithms:
    Hp = L L^T, L^-1, Hp^-1 = L^-T L^-1 (its lower triangle, all the factorization
    reads), U = the upper Cholesky factor of Hp^-1."""
    L = _cholesky_lower_blocked(Hp, nb)
    Linv = _tri_inverse_lower_blocked(L, nb)
    del L
    Hinv = _lower_gram_of_lower(Linv, nb)
    del Linv
    Lu = _cholesky_lower_blocked(Hinv, nb, overwrite=True)
    U = np.ascontiguousarray(Lu.T)
    del Lu, Hinv
    return U


def inverse_cholesky_upper(Hp: np.ndarray) -> np.ndarray:
    """U upper triangular with positive diagonal and U^T U = Hp^-1.

    Textbook route: invert Hp through its Cholesky factorization Hp = L L^T
    (LAPACK potri forms the lower triangle of Hp^-1 = L^-T L^-1 from L), then take
    the upper Cholesky factor of the inverse (its lower triangle is all the
    factorization reads).
    """
    C = Hp.shape[0]
    if C == 0:
        return np.zeros((0, 0))
    if C > LAPACK32_MAX_ORDER:
        return _inverse_cholesky_upper_wide(Hp)
    try:
        cf = sla.cho_factor(Hp, lower=True, check_finite=True)
    except (np.linalg.LinAlgError, ValueError) as e:
        raise NotPositiveDefinite(str(e)) from e
    Hinv, info = sla.lapack.dpotri(cf[0], lower=1, overwrite_c=1)
    del cf
    if info != 0:
        raise NotPositiveDefinite(f"potri info {info}")
    try:
        L = np.linalg.cholesky(Hinv)
    except np.linalg.LinAlgError as e:
        raise NotPositiveDefinite(str(e)) from e
    del Hinv
    return L.T.copy()


def prepare(H: np.ndarray, rel_damp: float, act_order: bool, perm=None):
    """Damp, permute and factor: returns (perm, Hp, U)."""
    C = H.shape[0]
    Hd = damp(H, rel_damp)
    if perm is None:
        perm = act_order_perm(H) if act_order else np.arange(C, dtype=np.int64)
    perm = np.asarray(perm, dtype=np.int64)
    Hp = Hd[np.ix_(perm, perm)]
    del Hd
    U = inverse_cholesky_upper(Hp)
    return perm, Hp, U


# -----------------------------------------------------------------------------
# the quantization grid  [Qwen-Int4 §2.1], [Deploy-guide] bits / sym rows
# -----------------------------------------------------------------------------
def grid(v: np.ndarray, bits: int, sym: bool):
    """Per-row (scale, zero) of the values v (rows x k), in float32.

    Returns float32 arrays s, z and the float32 pre-rounding value of z
    (-lo/s, asymmetric only; None for symmetric) for tie diagnostics.
    """
    maxq = np.float32(2 ** bits - 1)
    v32 = np.asarray(v, dtype=np.float32)
    if v32.ndim == 1:
        v32 = v32[:, None]
    zero = np.float32(0.0)
    if v32.shape[1] == 0:
        lo = np.zeros(v32.shape[0], np.float32)
        hi = np.zeros(v32.shape[0], np.float32)
    else:
        lo = np.minimum(zero, v32.min(axis=1))
        hi = np.maximum(zero, v32.max(axis=1))
    if sym:
        m = np.maximum(-lo, hi)
        m = np.where(m == zero, np.float32(1.0), m).astype(np.float32)
        lo, hi = -m, m
        s = ((hi - lo) / maxq).astype(np.float32)
        z = np.full_like(s, np.float32((2 ** bits) // 2))
        return s, z, None
    both0 = (lo == zero) & (hi == zero)
    lo = np.where(both0, np.float32(-1.0), lo).astype(np.float32)
    hi = np.where(both0, np.float32(1.0), hi).astype(np.float32)
    s = ((hi - lo) / maxq).astype(np.float32)
    tz = ((-lo) / s).astype(np.float32)
    z = np.rint(tz).astype(np.float32)
    return s, z, tz


def quantize(x: np.ndarray, s: np.ndarray, z: np.ndarray, bits: int):
    """code = clamp(rint(x/s) + z, 0, maxq) with the division and rint in float32.

    Returns (code as int64, Q = s (code - z) in float64, pre-rounding x/s in float32).
    """
    maxq = np.float32(2 ** bits - 1)
    x32 = np.asarray(x, dtype=np.float32)
    t = (x32 / s).astype(np.float32)
    c = np.clip(np.rint(t) + z, np.float32(0.0), maxq).astype(np.float32)
    Q = s.astype(np.float64) * (c.astype(np.float64) - z.astype(np.float64))
    return c.astype(np.int64), Q, t


def _tie_distance(t: np.ndarray) -> np.ndarray:
    """Distance (in grid steps) of t from the nearest half-integer."""
    t = np.asarray(t, dtype=np.float64)
    return np.abs(t - np.floor(t) - 0.5)


# -----------------------------------------------------------------------------
# step 3: the column sweep  [Deep-dive §2.2], [Deep-dive §2.4], [Deep-dive §3.1 step 3]
# -----------------------------------------------------------------------------
def supported(group_size: int, block_size: int) -> bool:
    g, B = group_size, block_size
    return B >= 1 and (g <= 0 or g % B == 0 or B % g == 0)


def sweep(Wp: np.ndarray, U: np.ndarray, bits: int, group_size: int, sym: bool,
          block_size: int = 128, hints: dict | None = None, tau: float = 0.0,
          stop_after: int | None = None):
    """Quantize the columns of Wp (rows x cols, already in sweep order) left to right.

    Within a block of B columns each column is quantized, its error divided by
    U[q,q] and fed into the block's remaining columns; after the block the
    trailing columns receive Err @ U[block, end:].

    hints / tau: where a rounding decision (a code, or an asymmetric group's zero)
    is within tau grid steps of a tie, the decision in ``hints`` ("codes": rows x
    cols in sweep order, "zeros": rows x groups) is taken instead, provided it is
    one of the two nearest integers.  Every such entry is listed in ``forced``.
    stop_after: process only the first k columns (flushing the lazy update) and
    return the working weights, for the one-step checks.
    """
    if not supported(group_size, block_size):
        raise ValueError("group size must divide the block size or be a multiple of it")
    W = np.array(Wp, dtype=np.float64, copy=True)
    R, C = W.shape
    g = group_size if group_size > 0 else 0
    G = (C + g - 1) // g if g else 1
    B = block_size
    codes = np.zeros((R, C), dtype=np.int64)
    Q = np.zeros((R, C))
    losses = np.zeros(C)
    scales = np.zeros((R, G), dtype=np.float32)
    zeros = np.zeros((R, G), dtype=np.float32)
    forced = {"codes": [], "zeros": [], "bad_hint": []}
    hc = None if hints is None else hints.get("codes")
    hz = None if hints is None else hints.get("zeros")

    def take_zero(col_group, z, tz):
        if hz is None or tz is None or tau <= 0:
            return z
        near = _tie_distance(tz) <= tau
        for r in np.nonzero(near)[0]:
            cand = (np.floor(tz[r]), np.floor(tz[r]) + 1)
            h = float(hz[r, col_group])
            if h != z[r]:
                if h in cand:
                    z[r] = np.float32(h)
                    forced["zeros"].append((int(r), int(col_group), float(_tie_distance(tz[r]))))
                else:
                    forced["bad_hint"].append(("zero", int(r), int(col_group)))
        return z

    if g == 0 and R and C:
        s_row, z_row, tz_row = grid(W, bits, sym)
        z_row = take_zero(0, z_row, tz_row)
        scales[:, 0], zeros[:, 0] = s_row, z_row
    ncols = C if stop_after is None else min(C, stop_after)
    maxq = 2 ** bits - 1
    for i in range(0, ncols, B):
        e = min(i + B, C)
        E = np.zeros((R, e - i))
        for q in range(i, min(e, ncols)):
            if g and q % g == 0:
                s_g, z_g, tz_g = grid(W[:, q:min(q + g, C)], bits, sym)
                z_g = take_zero(q // g, z_g, tz_g)
                scales[:, q // g], zeros[:, q // g] = s_g, z_g
            s = scales[:, q // g] if g else scales[:, 0]
            z = zeros[:, q // g] if g else zeros[:, 0]
            x = W[:, q]
            c, Qq, t = quantize(x, s, z, bits)
            if hc is not None and tau > 0:
                near = _tie_distance(t) <= tau
                for r in np.nonzero(near)[0]:
                    h = int(hc[r, q])
                    if h != c[r]:
                        cand = {int(np.clip(np.floor(t[r]) + z[r], 0, maxq)),
                                int(np.clip(np.floor(t[r]) + 1 + z[r], 0, maxq))}
                        if h in cand:
                            c[r] = h
                            Qq[r] = float(s[r]) * (h - float(z[r]))
                            forced["codes"].append((int(r), int(q), float(_tie_distance(t[r]))))
                        else:
                            forced["bad_hint"].append(("code", int(r), int(q)))
            d = U[q, q]
            codes[:, q] = c
            Q[:, q] = Qq
            err = (x - Qq) / d
            E[:, q - i] = err
            losses[q] = float(np.sum((x - Qq) ** 2)) / (2.0 * d * d)
            # OBS compensation of the block's remaining columns
            W[:, q + 1:e] -= np.outer(err, U[q, q + 1:e])
        # lazy batch update of everything right of the block
        if e < C:
            W[:, e:] -= E @ U[i:e, e:]
    return {"codes": codes, "Q": Q, "losses": losses, "scales": scales,
            "zeros": zeros, "forced": forced, "W": W}


# -----------------------------------------------------------------------------
# step 4: outputs in the original column order, packing  [Deep-dive §3.1 step 4]
# -----------------------------------------------------------------------------
def finalize(res: dict, perm: np.ndarray, group_size: int) -> dict:
    C = len(perm)
    inv = np.empty(C, dtype=np.int64)
    inv[perm] = np.arange(C)
    codes = np.empty_like(res["codes"])
    codes[:, perm] = res["codes"]
    Q = np.empty_like(res["Q"])
    Q[:, perm] = res["Q"]
    losses = np.empty_like(res["losses"])
    losses[perm] = res["losses"]
    g_idx = (inv // group_size) if group_size > 0 else np.zeros(C, dtype=np.int64)
    return {"codes": codes, "Q": Q, "losses": losses, "scales": res["scales"],
            "zeros": res["zeros"], "g_idx": g_idx.astype(np.int64), "perm": perm,
            "inv_perm": inv, "forced": res["forced"]}


def gptq_quantize(W: np.ndarray, H: np.ndarray, bits: int = 4, group_size: int = 128,
                  sym: bool = False, act_order: bool = False, damp_rel: float = 0.01,
                  block_size: int = 128, perm=None, hints: dict | None = None,
                  tau: float = 0.0) -> dict:
    """The whole layer: damp, (act-order) permute, factor, sweep, restore column order."""
    W = np.asarray(W, dtype=np.float64)
    perm, Hp, U = prepare(H, damp_rel, act_order, perm)
    res = sweep(W[:, perm], U, bits, group_size, sym, block_size, hints=hints, tau=tau)
    out = finalize(res, perm, group_size)
    out["U"] = U
    out["Hp"] = Hp
    out["Wp"] = W[:, perm]
    out["Qp"] = res["Q"]
    out["losses_p"] = res["losses"]
    return out


def pack(codes: np.ndarray, bits: int) -> np.ndarray:
    """Row-wise LSB-first bitstream of b-bit codes in little-endian uint32 words."""
    codes = np.asarray(codes, dtype=np.uint64)
    R, C = codes.shape
    nw = (C * bits + 31) // 32
    acc = np.zeros((R, nw + 1), dtype=np.uint64)
    for c in range(C):
        p = c * bits
        w, o = p // 32, p % 32
        acc[:, w] |= (codes[:, c] << np.uint64(o)) & np.uint64(0xFFFFFFFF)
        if o + bits > 32:
            acc[:, w + 1] |= codes[:, c] >> np.uint64(32 - o)
    return acc[:, :nw].astype(np.uint32)


def unpack(packed: np.ndarray, bits: int, cols: int) -> np.ndarray:
    packed = np.asarray(packed, dtype=np.uint64)
    R = packed.shape[0]
    ext = np.concatenate([packed, np.zeros((R, 1), dtype=np.uint64)], axis=1)
    out = np.zeros((R, cols), dtype=np.int64)
    mask = np.uint64((1 << bits) - 1)
    for c in range(cols):
        p = c * bits
        w, o = p // 32, p % 32
        v = ext[:, w] >> np.uint64(o)
        if o + bits > 32:
            v |= ext[:, w + 1] << np.uint64(32 - o)
        out[:, c] = (v & mask).astype(np.int64)
    return out


# -----------------------------------------------------------------------------
# inference side: the layer's product from the stored form
# [Deep-dive §3.3] (desc_act needs a gather at inference), [gptq-for-llama]
# "工程细节" (matrix products straight from the packed 4-bit codes)
# -----------------------------------------------------------------------------
def dequantize(packed: np.ndarray, scales: np.ndarray, zeros: np.ndarray, g_idx: np.ndarray,
               bits: int, cols: int) -> np.ndarray:
    """Q[r, c] = s[r, g] (code[r, c] - z[r, g]) with g = g_idx[c], from the packed codes
    and the float32 scales / zeros (rows x groups); float64 out, rows x cols."""
    codes = unpack(packed, bits, cols).astype(np.float64)
    g = np.asarray(g_idx, dtype=np.int64)
    s = np.asarray(scales, dtype=np.float32).astype(np.float64)[:, g]
    z = np.asarray(zeros, dtype=np.float32).astype(np.float64)[:, g]
    return s * (codes - z)


def dequant_matmul(X: np.ndarray, packed: np.ndarray, scales: np.ndarray, zeros: np.ndarray,
                   g_idx: np.ndarray, bits: int) -> np.ndarray:
    """Y = X Q^T for activations X (tokens x cols, widened exactly to float64) and the
    stored layer; Y is tokens x rows, float64."""
    X = np.asarray(X, dtype=np.float64)
    Q = dequantize(packed, scales, zeros, g_idx, bits, X.shape[1])
    return X @ Q.T


# -----------------------------------------------------------------------------
# quality measures  [Deep-dive §2.1]
# -----------------------------------------------------------------------------
def half_trace_loss(Wp: np.ndarray, Qp: np.ndarray, Hp: np.ndarray) -> float:
    """1/2 tr((Wp - Qp) Hp (Wp - Qp)^T), the quadratic term of the Taylor objective."""
    D = np.asarray(Wp, np.float64) - np.asarray(Qp, np.float64)
    return 0.5 * float(np.sum((D @ Hp) * D))


def reconstruction_error(W: np.ndarray, Q: np.ndarray, H: np.ndarray, n: int) -> float:
    """||(W - Q) X^T||_F^2 = (n/2) tr((W - Q) H (W - Q)^T) with the undamped H = 2 X^T X / n."""
    D = np.asarray(W, np.float64) - np.asarray(Q, np.float64)
    return 0.5 * n * float(np.sum((D @ H) * D))
