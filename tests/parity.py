"""Comparison of the CUDA path with the float64 oracle on the same seeded inputs.

Rounding decisions (codes, asymmetric zero-points) are unique except where the
pre-rounding value sits at a tie.  Both sides take each decision in IEEE float32
(the quotient x/s and rint), but the GPU's working weights are float32 and the
oracle's are float64, so where the oracle's pre-rounding value lies within
``TIE_TAU`` grid steps of a half-integer the other neighbour is also a valid
decision.  The comparison replays the oracle with the GPU's decision taken at
those entries only (it must be one of the two neighbours; anything else is
recorded as a bad hint) and then requires every code to match.  The forced
entries are counted and bounded separately.

The bars are the stated parity tolerances of the layer solver: mismatching codes
only at ties within 1e-6 grid steps of a midpoint and on at most 0.1% of entries,
scales and zeros within 1e-5 relative, reconstruction error within 0.5%.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from oracle import gptq_ref as o

TIE_TAU = 1e-6          # grid steps from a midpoint within which either neighbour is valid
MAX_FORCED_FRAC = 1e-3  # forced (near-tie) decisions, fraction of all codes
SCALE_REL = 1e-5        # scales (and zeros) relative
RECON_REL = 5e-3        # ||(W - Q) X^T||^2 relative
LOSS_REL = 1e-3         # per-column losses, L1 relative

# one line per compared layer, printed at the end of the session (tests/conftest.py)
REPORT: list = []


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
    loss_abs: float              # L1 difference of per-column losses / loss of zeroing W
    recon_rel: float             # relative difference of ||(W - Q) X^T||^2
    recon_gpu: float
    recon_oracle: float
    max_forced_dist: float       # largest tie distance among forced entries (grid steps)
    raw_mismatch: int = 0        # codes differing before the replay

    @property
    def forced_frac(self) -> float:
        return (self.forced_codes) / max(1, self.R * self.C)

    def summary(self) -> str:
        return (f"R={self.R} C={self.C} raw_mismatch={self.raw_mismatch} "
                f"mismatch={self.code_mismatch} forced={self.forced_codes}"
                f" ({self.forced_frac:.2e}) zeros_forced={self.forced_zeros} bad={self.bad_hints}"
                f" scale_rel={self.scale_rel:.2e} zero_diff={self.zero_diff} loss_rel={self.loss_rel:.2e}"
                f" recon_rel={self.recon_rel:.2e} max_forced_offset={self.max_forced_dist:.2e}")

    def assert_bars(self, name: str, check_losses: bool = True) -> None:
        """The stated tolerances; the summary goes to the session report first."""
        REPORT.append(f"{name}: {self.summary()}")
        print(f"{name}: {self.summary()}", flush=True)
        assert self.bad_hints == 0, name
        assert self.code_mismatch == 0, name
        assert self.max_forced_dist <= TIE_TAU, name
        assert self.forced_frac <= MAX_FORCED_FRAC, name
        assert self.zero_diff == 0.0, name
        assert self.scale_rel <= SCALE_REL, name
        assert self.recon_rel <= RECON_REL, name
        if check_losses:
            assert self.loss_rel <= LOSS_REL, name


def compare_layer(W64, H64, n, perm, gpu, bits, group, sym, tau=TIE_TAU, damp=0.01,
                  block_size=128, prepared=None):
    """gpu: dict of numpy arrays codes, scales, zeros, losses, g_idx (original order).
    prepared: the oracle's (perm, Hp, U) for H64 and perm, if already formed."""
    R, C = W64.shape
    perm = np.asarray(perm, dtype=np.int64)
    if prepared is None:
        prepared = o.prepare(H64, damp, False, perm)
    perm_o, Hp, U = prepared
    assert np.array_equal(perm_o, perm)
    Wp = np.asarray(W64, dtype=np.float64)[:, perm]
    hints = {"codes": gpu["codes"][:, perm].astype(np.int64), "zeros": gpu["zeros"]}
    ref = o.finalize(o.sweep(Wp, U, bits, group, sym, block_size, hints=hints, tau=tau), perm,
                     group)
    # codes as the plain oracle decides them, before any near-tie entry is replayed
    raw = o.finalize(o.sweep(Wp, U, bits, group, sym, block_size), perm, group)
    raw_mismatch = int(np.count_nonzero(raw["codes"] != gpu["codes"]))
    mism = int(np.count_nonzero(ref["codes"] != gpu["codes"]))
    s_o, s_g = ref["scales"].astype(np.float64), gpu["scales"].astype(np.float64)
    scale_rel = float(np.max(np.abs(s_o - s_g) / np.maximum(np.abs(s_o), 1e-30))) if s_o.size else 0.0
    zero_diff = float(np.max(np.abs(ref["zeros"] - gpu["zeros"]))) if s_o.size else 0.0
    lo, lg = ref["losses"], gpu["losses"].astype(np.float64)
    zero_loss = float(np.sum(np.sum(Wp ** 2, axis=0) / (2.0 * np.diag(U) ** 2))) if R else 0.0
    l1 = float(np.sum(np.abs(lo - lg)))
    loss_rel = l1 / max(float(np.sum(np.abs(lo))), 1e-300)
    loss_abs = l1 / max(zero_loss, 1e-300)
    Qg = gpu["scales"][:, gpu["g_idx"]].astype(np.float64) * \
        (gpu["codes"].astype(np.float64) - gpu["zeros"][:, gpu["g_idx"]].astype(np.float64))
    rg = o.reconstruction_error(W64, Qg, H64, n)
    ro = o.reconstruction_error(W64, ref["Q"], H64, n)
    ref["U"], ref["Hp"], ref["Wp"] = U, Hp, Wp
    return Parity(R, C, mism, len(ref["forced"]["codes"]), len(ref["forced"]["zeros"]),
                  len(ref["forced"]["bad_hint"]), scale_rel, zero_diff, loss_rel, loss_abs,
                  abs(rg - ro) / max(ro, 1e-300), rg, ro,
                  max([f[2] for f in ref["forced"]["codes"]] +
                      [f[2] for f in ref["forced"]["zeros"]] + [0.0]),
                  raw_mismatch), ref
