"""Comparison of the CUDA path with the float64 oracle on the same seeded inputs.

Rounding decisions (codes, asymmetric zero-points) are unique except where the
pre-rounding value sits at a tie.  The GPU state is fp32 and the oracle's is
fp64, so where the oracle's value lies within ``tau`` grid steps of a tie the
other neighbour is also a valid decision.  The comparison therefore replays the
oracle with the GPU's decision taken at those entries only (it must be one of
the two neighbours; anything else is recorded as a bad hint) and then requires
every code to match.  The forced entries are counted and bounded separately.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from oracle import gptq_ref as o


@dataclass
class Parity:
    R: int
    C: int
    code_mismatch: int           # after the replay; must be 0
    forced_codes: int            # near-tie entries where the GPU's neighbour was taken
    forced_zeros: int
    bad_hints: int               # GPU decisions that are not a neighbour of the oracle's value
    scale_rel: float             # max relative difference of scales
    zero_diff: float             # max abs difference of zeros
    loss_rel: float              # relative L1 difference of per-column losses
    recon_rel: float             # relative difference of ||(W - Q) X^T||^2
    recon_gpu: float
    recon_oracle: float
    max_forced_dist: float       # largest tie distance among forced entries (grid steps)

    @property
    def forced_frac(self) -> float:
        return (self.forced_codes) / max(1, self.R * self.C)

    def summary(self) -> str:
        return (f"R={self.R} C={self.C} mismatch={self.code_mismatch} forced={self.forced_codes}"
                f" ({self.forced_frac:.2e}) zeros_forced={self.forced_zeros} bad={self.bad_hints}"
                f" scale_rel={self.scale_rel:.2e} zero_diff={self.zero_diff} loss_rel={self.loss_rel:.2e}"
                f" recon_rel={self.recon_rel:.2e} max_forced_offset={self.max_forced_dist:.2e}")


def compare_layer(W64, H64, n, perm, gpu, bits, group, sym, tau, damp=0.01, block_size=128):
    """gpu: dict of numpy arrays codes, scales, zeros, losses, g_idx (original order)."""
    R, C = W64.shape
    perm = np.asarray(perm, dtype=np.int64)
    hints = {"codes": gpu["codes"][:, perm].astype(np.int64), "zeros": gpu["zeros"]}
    ref = o.gptq_quantize(W64, H64, bits, group, sym, False, damp, block_size, perm=perm,
                          hints=hints, tau=tau)
    mism = int(np.count_nonzero(ref["codes"] != gpu["codes"]))
    s_o, s_g = ref["scales"].astype(np.float64), gpu["scales"].astype(np.float64)
    scale_rel = float(np.max(np.abs(s_o - s_g) / np.maximum(np.abs(s_o), 1e-30))) if s_o.size else 0.0
    zero_diff = float(np.max(np.abs(ref["zeros"] - gpu["zeros"]))) if s_o.size else 0.0
    lo, lg = ref["losses"], gpu["losses"].astype(np.float64)
    # floor: a millionth of the loss of quantizing every weight to zero, so that
    # layers whose weights sit on the grid (losses at rounding level) compare sanely
    U = ref["U"]
    zero_loss = float(np.sum(np.sum(ref["Wp"] ** 2, axis=0) / (2.0 * np.diag(U) ** 2))) if R else 0.0
    loss_rel = float(np.sum(np.abs(lo - lg)) / max(np.sum(np.abs(lo)), 1e-6 * zero_loss, 1e-300))
    Qg = gpu["scales"][:, gpu["g_idx"]].astype(np.float64) * \
        (gpu["codes"].astype(np.float64) - gpu["zeros"][:, gpu["g_idx"]].astype(np.float64))
    rg = o.reconstruction_error(W64, Qg, H64, n)
    ro = o.reconstruction_error(W64, ref["Q"], H64, n)
    return Parity(R, C, mism, len(ref["forced"]["codes"]), len(ref["forced"]["zeros"]),
                  len(ref["forced"]["bad_hint"]), scale_rel, zero_diff, loss_rel,
                  abs(rg - ro) / max(ro, 1e-300), rg, ro,
                  max([f[2] for f in ref["forced"]["codes"]] + [0.0])), ref
