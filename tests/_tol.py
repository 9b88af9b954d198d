"""The parity bound shared by every GPU test, and a record of how it was used.

Stated target: max |GPU - oracle| <= 1e-2 and mean |GPU - oracle| <= 1e-3 per
call, the oracle being unrounded fp64.

Where the target cannot bind.  The outputs are bf16 (the pages' code returns
the input dtype); bf16 numbers in [2^e, 2^(e+1)) are 2^(e-7) apart, so
rounding the output alone costs up to half that, 2^(e-8).  Below |O| = 4 this
is at most 2^-7 = 0.0078 and the 1e-2 target is held strictly.  From |O| = 4
up, half a step is 2^-6 = 0.0156 > 1e-2: no bf16 result can meet 1e-2 there,
and such an element is held to the error the arithmetic itself allows:

    |err| <= 0.5 step(O) + eps_P + eps_acc

  eps_P   the kernels round each softmax weight p_j to the precision of the
          tensor-core operand (bf16, unit roundoff u = 2^-9; f16 for the
          8-bit caches, u = 2^-11) and divide by the sum of the ROUNDED
          weights.  With w_j = p_j / sum p and w~_j the rounded normalised
          weights, w~_j - w_j = w_j (d_j - d) / (1 + d), |d_j| <= u, d the
          w-weighted mean of the d_j; since both weight sets sum to 1,
          O~ - O = sum_j (w~_j - w_j) v_j, so
              |O~ - O| <= 2u / (1 - u) * max_j |v_j|.
  eps_acc fp32 accumulation of n products and of the n-term weight sum
          (the textbook bound for recursive summation with unit roundoff
          2^-23, allowing truncating accumulators):
              n 2^-23 (max_j |v_j| + |O|).

max_j |v_j| is taken over the call's whole value tensor (an upper bound of
each row's visible keys) and n is the most keys any row of the call sees.
The mean bound is unchanged.  Every call counts the elements whose error is
above 1e-2 (all of them necessarily at |O| >= 4); the counts are printed in
the pytest summary (tests/conftest.py), so no relaxation is silent.
"""
import os

import numpy as np
import torch

MAX_ABS = 1e-2
MEAN_ABS = 1e-3
STRICT_BELOW = 4.0           # |O| below which 1e-2 is held strictly (half a bf16 step <= 2^-7)
U_BF16 = 2.0 ** -9           # unit roundoff of a bf16 softmax weight
U_F16 = 2.0 ** -11           # unit roundoff of an f16 softmax weight (8-bit caches)
U_ACC = 2.0 ** -23           # fp32 accumulation, truncating or rounding

# one entry per check() call: (what, elements, max err, mean err, elements above 1e-2, failed)
RECORD = []
# GQA_PARITY_AUDIT=1: record failures instead of raising (a diagnosis run; never the default)
AUDIT = os.environ.get("GQA_PARITY_AUDIT", "") == "1"


def bf16_step(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers around |x| (normal range)."""
    a = np.maximum(np.abs(x), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def value_absmax(v, v_scale=None) -> float:
    """max |value| of a value tensor: bf16 values, or 8-bit E4M3 codes times the
    per-KV-head scale (the scales may be passed as a tensor; the largest is
    used).  Non-finite entries (unused paged slots) are ignored."""
    t = v if isinstance(v, torch.Tensor) else torch.as_tensor(v)
    if t.dtype in (torch.uint8, torch.float8_e4m3fn):
        x = t.view(torch.float8_e4m3fn).float()
        s = float(torch.as_tensor(v_scale).float().abs().max()) if v_scale is not None else 1.0
    else:
        x, s = t.float(), 1.0
    x = x[torch.isfinite(x)]
    return (float(x.abs().max()) if x.numel() else 0.0) * s


def bound(ref: np.ndarray, vmax: float, n_keys: int, u_p: float = U_BF16) -> np.ndarray:
    """Per-element bound: 1e-2 below |ref| = 4, the derived arithmetic bound above."""
    a = np.abs(ref)
    derived = 0.5 * bf16_step(ref) + 2 * u_p / (1 - u_p) * vmax + n_keys * U_ACC * (vmax + a)
    return np.where(a < STRICT_BELOW, MAX_ABS, np.maximum(MAX_ABS, derived))


def check(got: torch.Tensor, ref: np.ndarray, what: str, *, v, n_keys: int, v_scale=None):
    """Compare a GPU result with the fp64 oracle under the bound above.

    v        the value tensor the outputs average (bf16, or E4M3 codes with
             v_scale; the 8-bit path rounds its weights to f16)
    n_keys   the most keys any output row of the call attends to
    """
    g = got.detach().float().cpu().double().numpy()
    assert g.shape == ref.shape, (g.shape, ref.shape)
    fp8 = isinstance(v, torch.Tensor) and v.dtype in (torch.uint8, torch.float8_e4m3fn)
    vmax = value_absmax(v, v_scale)
    finite = np.all(np.isfinite(g))
    err = np.abs(g - ref)
    lim = bound(ref, vmax, max(int(n_keys), 1), U_F16 if fp8 else U_BF16)
    over = err > lim
    mx = float(err.max()) if err.size else 0.0
    mean = float(err.mean()) if err.size else 0.0
    above = int((err > MAX_ABS).sum())
    ok = finite and not over.any() and mean <= MEAN_ABS
    RECORD.append((what, int(err.size), mx, mean, above, not ok))
    msg = (f"{what}: max abs {mx:.3e}, mean abs {mean:.3e}, {int(over.sum())} element(s) beyond the bound "
           f"(1e-2 below |O| = 4; half a bf16 step + weight rounding + fp32 sums above), "
           f"{above} above 1e-2, finite={finite}")
    if not ok and not AUDIT:
        raise AssertionError(msg)
    return mx, mean
