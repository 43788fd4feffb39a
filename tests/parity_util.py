"""Helpers shared by the GPU parity tests: tensor conversion, the output
tolerance, and id comparison that allows only logged near-ties."""

import numpy as np

# Layer outputs: max|gpu - oracle| / max|oracle| <= REL_TOL (bf16/int4 weights,
# fp32 accumulation on the GPU, fp64 in the oracle).
REL_TOL = 1e-2
# Expert ids may differ only at positions whose fp64 logit lies within
# TIE_TOL of a neighbouring expert's logit.
TIE_TOL = 1e-5


def f64(t):
    """torch tensor (any device, bf16/fp32/int) -> numpy fp64 (exact)."""
    t = t.detach().cpu()
    if t.dtype.is_floating_point:
        t = t.float()
    return t.double().numpy()


def rel_err(got, want):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    den = np.abs(want).max()
    if den == 0:
        return float(np.abs(got).max())
    return float(np.abs(got - want).max() / den)


def check_ids(got, want, logits, log, tag=""):
    """Compare one token's ordered id list; near-ties are logged, not failed.
    Returns the number of tolerated tie positions that differed."""
    from oracle import moe_oracle as O
    got = [int(v) for v in got]
    want = [int(v) for v in want]
    ties = O.tie_positions(logits, np.array(want), TIE_TOL)
    n_tie = 0
    for i, (g, w) in enumerate(zip(got, want)):
        if g != w:
            assert i in ties, f"{tag}: id mismatch at position {i}: gpu {got} oracle {want}"
            n_tie += 1
            log.append((tag, i, g, w))
    return n_tie
