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


# ---------------------------------------------------------------- sampling --
# Full-size parity checks compare the outputs of a sample of tokens (tokens
# are independent, so each sampled row is checked exactly as in a full
# comparison).  The sample always holds the rows where tiling mistakes would
# show: the hottest expert's last row tile of every tile height the grouped
# GEMMs use for the call, and every token routed to the rarest expert that
# has any rows.

def row_tiles(n_rows, bn):
    """(first row, rows) of each routed-row tile of an expert with n_rows
    rows when tiles hold at most bn rows: ceil(n/bn) near-equal tiles whose
    height is a multiple of 16 (the grouped GEMMs' split)."""
    if n_rows <= 0:
        return []
    nt = -(-n_rows // bn)
    rpt = min(bn, ((-(-n_rows // nt)) + 15) // 16 * 16)
    return [(i * rpt, min(rpt, n_rows - i * rpt)) for i in range(nt) if i * rpt < n_rows]


def parity_sample(idx, E, tile_heights, n_min=16, seed=0):
    """Token indices (sorted) for a sampled full-size check: every token in
    the hottest expert's last row tile for each height in tile_heights, every
    token routed to the rarest non-empty expert, the first and last token,
    then random tokens up to n_min."""
    idx = np.asarray(idx)
    T, K = idx.shape
    flat = idx.reshape(-1)
    valid = (flat >= 0) & (flat < E)
    counts = np.bincount(flat[valid], minlength=E)
    chosen = {0, T - 1}
    if counts.max() > 0:
        hot = int(counts.argmax())
        slots = np.nonzero(flat == hot)[0]              # ascending slot order
        for bn in tile_heights:
            r0, n = row_tiles(len(slots), bn)[-1]
            chosen |= {int(s) // K for s in slots[r0:r0 + n]}
        nz = np.nonzero(counts)[0]
        rare = int(nz[np.argmin(counts[nz])])
        chosen |= {int(s) // K for s in np.nonzero(flat == rare)[0]}
    rng = np.random.default_rng(seed)
    rest = np.setdiff1d(np.arange(T), np.fromiter(chosen, dtype=np.int64))
    need = max(0, n_min - len(chosen))
    if need and len(rest):
        chosen |= {int(t) for t in rng.choice(rest, min(need, len(rest)), replace=False)}
    return sorted(chosen)


def grouped_tile_heights(T, K, E, wtype):
    """Routed-row tile heights of the grouped GEMMs for a call: bf16 gate_up
    128 and down 256; E4M3 16 for few rows per expert (T*K <= 64 or
    <= 6 rows per expert) else 64; MXFP4 as E4M3, or 112 at >= 48 rows per
    expert."""
    n = T * K
    if wtype == "bf16":
        return [128, 256]
    bn = 16 if (n <= 64 or n <= 6 * E) else 64
    if wtype == "mxfp4" and n >= 48 * E:
        bn = 112
    return [bn]
