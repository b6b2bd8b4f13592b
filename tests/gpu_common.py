"""Shared helpers of the GPU parity tests: device transfer of the seeded
inputs, and the comparison rules.

Comparison rules (fixed by the method's arithmetic and the stated bar):
  * quantise outputs and permutation results: bit-exact;
  * expert ids: exact, except that two ids may trade places where the oracle's
    fp64 logits of the two differ by less than 1e-6 (near-ties that an fp32
    computation may order either way);
  * routing weights: relative error <= 1e-5 (fp32 arithmetic against fp64);
  * forward output y (bf16): relative L2 error <= 2e-3 and max-abs error
    <= 2e-2 * rms(y) against the unrounded fp64 oracle; where the ids of a
    token legitimately differ (near-tie), the oracle is evaluated with the
    GPU's ids.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import formats as F

ID_TIE = 1e-6
W_RTOL = 1e-5
Y_REL_L2 = 2e-3
Y_MAX_ABS_OVER_RMS = 2e-2


def bf16_to_dev(bits: np.ndarray, dev) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)


def bf16_from_dev(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def check_ids(ids_gpu: np.ndarray, ids_ref: np.ndarray, logits_ref: np.ndarray) -> np.ndarray:
    """Assert the id rule; return a bool mask of tokens whose ids differ
    (legitimately) from the oracle's."""
    ids_gpu = np.asarray(ids_gpu)
    differ = np.any(ids_gpu != ids_ref, axis=1)
    for t in np.flatnonzero(differ):
        g, r = ids_gpu[t], ids_ref[t]
        assert len(set(g.tolist())) == len(g), f"token {t}: repeated ids {g}"
        # every position that differs must hold an expert whose logit is within
        # ID_TIE of the oracle's expert at that position
        for j in np.flatnonzero(g != r):
            lg, lr = logits_ref[t, g[j]], logits_ref[t, r[j]]
            assert abs(lg - lr) < ID_TIE, (
                f"token {t} position {j}: gpu id {g[j]} (logit {lg!r}) vs oracle id {r[j]} (logit {lr!r})")
    return differ


def check_weights(w_gpu: np.ndarray, w_ref: np.ndarray, differ: np.ndarray) -> None:
    ok = ~differ
    err = np.abs(w_gpu[ok] - w_ref[ok]) / np.abs(w_ref[ok])
    assert err.size == 0 or err.max() <= W_RTOL, f"max weight rel err {err.max():.3e}"


def forward_errors(y_bits: np.ndarray, y64: np.ndarray) -> tuple[float, float]:
    y = F.bf16_to_f64(y_bits)
    rms = np.sqrt(np.mean(y64 ** 2))
    rel = np.linalg.norm(y - y64) / np.linalg.norm(y64)
    mx = np.abs(y - y64).max() / rms
    return float(rel), float(mx)


def check_forward(y_bits: np.ndarray, y64: np.ndarray) -> tuple[float, float]:
    assert np.all(np.isfinite(F.bf16_to_f64(y_bits)))
    rel, mx = forward_errors(y_bits, y64)
    assert rel <= Y_REL_L2, f"relative L2 error {rel:.3e} > {Y_REL_L2}"
    assert mx <= Y_MAX_ABS_OVER_RMS, f"max-abs / rms {mx:.3e} > {Y_MAX_ABS_OVER_RMS}"
    return rel, mx
