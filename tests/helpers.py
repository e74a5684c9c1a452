"""Shared test utilities: bf16 <-> numpy bit views and the parity tolerances.

Tolerances (fp64 oracle as reference):
  o   : |o_gpu - o_ref| <= 1e-2 + 2^-8 |o_ref|.  The 1e-2 absolute budget
        covers the fp32/bf16 arithmetic; 2^-8 |o_ref| is the bf16 rounding of
        the output itself (half an ulp: relative 2^-8), which alone exceeds
        1e-2 once |o| >= 2.56 and cannot be avoided by any bf16 output.
  lse : |lse_gpu - lse_ref| <= 1e-3 * max(1, |lse_ref|)  (relative 1e-3, with
        an absolute floor near lse = 0 where a relative bound is undefined).
  RoPE outputs and cache writes: bit-exact.
"""
import os

import numpy as np
import torch

O_ABS = 1e-2
O_REL = 2.0 ** -8
LSE_REL = 1e-3
# below this magnitude the bf16 rounding of o alone (at most 2^-8 |o|) stays
# under the literal 1e-2 bound, so there the literal bound is the meaningful one
O_LITERAL_BELOW = 2.56

# per check_o call: (test, what, max |o - o_ref|, elements with |o_ref| < 2.56 and
# |o - o_ref| > 1e-2, elements with |o_ref| < 2.56); printed at the end of the run
MARGINS = []


def bits(x: torch.Tensor) -> np.ndarray:
    """bf16 tensor (any device) -> numpy uint16 bit patterns."""
    return x.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


def f64(x: torch.Tensor) -> np.ndarray:
    return x.detach().to("cpu").to(torch.float64).numpy()


def check_o(got: np.ndarray, ref: np.ndarray, what: str = "o") -> float:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(ref).all(), f"{what}: oracle produced non-finite values"
    err = np.abs(got - ref)
    small = np.abs(ref) < O_LITERAL_BELOW
    MARGINS.append((os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0], what,
                    float(np.nanmax(err)) if err.size else 0.0, int(np.sum(small & ~(err <= O_ABS))),
                    int(np.sum(small))))
    bound = O_ABS + O_REL * np.abs(ref)
    bad = ~(err <= bound)
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; first at "
                             f"{idx.tolist()}: got {got[tuple(idx[0])]} ref {ref[tuple(idx[0])]}")
    return float(err.max()) if err.size else 0.0


def check_lse(got: np.ndarray, ref: np.ndarray, what: str = "lse") -> float:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    inf_ref = np.isinf(ref)
    assert np.array_equal(np.isinf(got), inf_ref), f"{what}: -inf pattern differs"
    if inf_ref.any():
        assert np.array_equal(got[inf_ref], ref[inf_ref])
    g, r = got[~inf_ref], ref[~inf_ref]
    err = np.abs(g - r)
    bound = LSE_REL * np.maximum(1.0, np.abs(r))
    bad = ~(err <= bound)
    if bad.any():
        i = int(np.argmax(bad))
        raise AssertionError(f"{what}: {int(bad.sum())} outside tolerance; e.g. got {g[i]} ref {r[i]}")
    return float(err.max()) if err.size else 0.0
