"""Shared test helpers: tolerance checks against the oracle."""
import numpy as np
import torch

import oracle

# Floating-point bar for bf16 / FP8 outputs: relative L2 error <= 5e-3 and
# |delta| <= 3e-2 * max(1, |ref|) per element; plus an internal guard
# max|delta| <= 1e-2 * max|ref| (outputs of these layers are small, so the
# per-element bound alone would be loose).
REL_L2 = 5e-3
ABS_REL = 3e-2
MAX_GUARD = 1e-2


def to_f64(out_bf16: torch.Tensor) -> np.ndarray:
    return out_bf16.detach().float().cpu().double().numpy()


def assert_matches_oracle(out_bf16: torch.Tensor, ref_bits: np.ndarray, what=""):
    o = to_f64(out_bf16)
    r = oracle.bf16_to_f64(ref_bits)
    assert o.shape == r.shape, (o.shape, r.shape)
    assert np.all(np.isfinite(o)), "%s: non-finite output" % what
    d = np.abs(o - r)
    nr = np.linalg.norm(r)
    rel = np.linalg.norm(o - r) / max(nr, 1e-30)
    if nr == 0:
        assert d.max() == 0, "%s: expected zeros" % what
        return
    assert rel <= REL_L2, "%s: rel L2 %.3e" % (what, rel)
    assert np.all(d <= ABS_REL * np.maximum(1.0, np.abs(r))), "%s: elementwise bound" % what
    assert d.max() <= MAX_GUARD * np.abs(r).max(), "%s: max|d| %.3e vs max|ref| %.3e" % (
        what, d.max(), np.abs(r).max())
    return rel
