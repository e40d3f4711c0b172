"""Error metric and tolerances shared by the GPU parity tests.

The bound of the target ("max relative error 1e-4 for fp32 inputs and 2e-2
for bf16 inputs with fp32 accumulation; final states within the same bounds")
leaves "relative error" undefined; element-wise relative error is meaningless
near sign changes of outputs of mixed sign.  The reading used here: for every
(sequence, head) slice, max|x - ref| / max|ref| over the slice; the reported
error is the maximum over slices, taken separately for `out` and for the
final state.
"""
import numpy as np
import torch

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


def slice_rel_err(x, ref, seq_slices, scale=None):
    """x, ref: [B, T, H, D] arrays; seq_slices: list of (b, start, end).

    scale (optional, ref's shape): where ref is a difference of terms that cancel,
    the size of one of those terms; a slice's denominator is then the larger of
    max|ref| and max|scale| over it."""
    worst = 0.0
    H = ref.shape[2]
    for b, s, e in seq_slices:
        if e <= s:
            continue
        for h in range(H):
            r = ref[b, s:e, h]
            d = np.max(np.abs(r))
            if scale is not None:
                d = max(d, np.max(np.abs(scale[b, s:e, h])))
            err = np.max(np.abs(x[b, s:e, h] - r))
            worst = max(worst, float(err / d) if d > 0 else float(err))
    return worst


def state_rel_err(x, ref):
    """x, ref: [N, H, d_k, d_v]; max over (n, h) of max|x - ref| / max|ref|."""
    worst = 0.0
    for n in range(ref.shape[0]):
        for h in range(ref.shape[1]):
            d = np.max(np.abs(ref[n, h]))
            err = np.max(np.abs(x[n, h] - ref[n, h]))
            worst = max(worst, float(err / d) if d > 0 else float(err))
    return worst


def seq_slices(B, T, cu=None):
    if cu is None:
        return [(b, 0, T) for b in range(B)]
    cu = [int(x) for x in cu]
    return [(0, cu[i], cu[i + 1]) for i in range(len(cu) - 1)]


def to_np(x):
    return x.detach().float().cpu().numpy().astype(np.float64)
