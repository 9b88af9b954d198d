"""The parity bound shared by every GPU test.

Stated bound: max |GPU - oracle| <= 1e-2 and mean |GPU - oracle| <= 1e-3, the
oracle being unrounded fp64.  The outputs are bf16 (the pages' code returns the
input dtype), whose spacing is 2^(e - 7) for |x| in [2^e, 2^(e+1)): at |x| >= 2
one step is 2^-6 = 0.0156 and rounding alone can cost 0.0078, so no bf16
result can meet 1e-2 there with the softmax weights' own rounding on top.  So
an element passes when its error is within 1e-2 OR within one bf16 step of the
oracle value; below |x| = 2 that is exactly the stated 1e-2.  The mean bound is
unchanged.
"""
import numpy as np
import torch

MAX_ABS = 1e-2
MEAN_ABS = 1e-3


def bf16_step(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers around |x| (normal range)."""
    a = np.maximum(np.abs(x), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def check(got: torch.Tensor, ref: np.ndarray, what: str):
    g = got.detach().float().cpu().double().numpy()
    assert g.shape == ref.shape, (g.shape, ref.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    err = np.abs(g - ref)
    bound = np.maximum(MAX_ABS, bf16_step(ref))
    over = err > bound
    mx, mean = float(err.max()), float(err.mean())
    assert not over.any() and mean <= MEAN_ABS, (
        f"{what}: max abs {mx:.3e}, mean abs {mean:.3e}, {int(over.sum())} element(s) beyond "
        f"max(1e-2, one bf16 step)")
    return mx, mean
