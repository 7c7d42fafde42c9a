"""Shared parity helpers for the GPU tests (test infrastructure).

Tolerances (max-abs against the fp64 oracle):
  * fp32 path: O within 1e-5, LSE within 1e-5 (LSE is computed in fp32).
  * bf16 / f16 path: O within 1e-2 for the arithmetic.  The output is stored
    in the 16-bit format, so its final rounding (half an ulp of the format,
    0.0156 for bf16 values in [4, 8)) comes on top: elements whose exact
    value has magnitude below 4 must meet 1e-2 outright, larger ones 1e-2
    plus half an ulp.  LSE within 1e-3.
"""
import math

import torch

import oracle

TOL_O = {torch.float32: 1e-5, torch.bfloat16: 1e-2, torch.float16: 1e-2}
TOL_LSE = {torch.float32: 1e-5, torch.bfloat16: 1e-3, torch.float16: 1e-3}
MANT = {torch.bfloat16: 8, torch.float16: 11}


def half_ulp(x: torch.Tensor, dtype) -> torch.Tensor:
    if dtype == torch.float32:
        return torch.zeros_like(x)
    e = torch.floor(torch.log2(x.abs().clamp_min(2.0 ** -14)))
    return 0.5 * torch.pow(2.0, e - (MANT[dtype] - 1))


# Figures of the last compare() call: the max-abs error against the oracle,
# against the oracle rounded to the output format (what a correctly rounded
# kernel would store), and the number of elements whose exact value has
# magnitude >= 4 (where the output rounding alone can exceed 1e-2).
LAST: dict = {}


def compare(o_gpu, lse_gpu, o_ref, lse_ref, dtype, what="", lse_tol=None):
    """o_gpu / lse_gpu: device or host tensors shaped like o_ref / lse_ref (fp64).
    lse_tol overrides the LSE bound (a float, or a tensor per row).  Every
    failure message carries the figures of ``LAST``."""
    o = o_gpu.detach().double().cpu()
    assert torch.isfinite(o).all(), f"{what}: non-finite output"
    err = (o - o_ref).abs()
    tol = TOL_O[dtype]
    small = o_ref.abs() < 4.0
    LAST.clear()
    LAST.update(max_abs=err.max().item() if err.numel() else 0.0,
                max_abs_vs_rounded=(o - o_ref.to(dtype).double()).abs().max().item() if err.numel() else 0.0,
                n_big=int((~small).sum()))
    figs = (f"max|dO| {LAST['max_abs']:.3e}, vs oracle rounded to {dtype}: {LAST['max_abs_vs_rounded']:.3e}, "
            f"{LAST['n_big']} elements with |O| >= 4")
    assert err[small].numel() == 0 or err[small].max().item() <= tol, \
        f"{what}: max |dO| = {err[small].max().item():.3e} > {tol} ({figs})"
    big_tol = tol + half_ulp(o_ref, dtype)
    assert bool((err <= big_tol).all()), f"{what}: |dO| beyond tolerance + output rounding ({figs})"
    if lse_gpu is not None:
        l = lse_gpu.detach().double().cpu()
        fin = torch.isfinite(lse_ref)
        assert torch.equal(torch.isfinite(l), fin), f"{what}: LSE finiteness differs"
        if fin.any():
            tol_l = TOL_LSE[dtype] if lse_tol is None else lse_tol
            if isinstance(tol_l, torch.Tensor):
                tol_l = tol_l.double()[fin]
            lerr = (l[fin] - lse_ref[fin]).abs()
            assert bool((lerr <= tol_l).all()), f"{what}: max |dLSE| = {lerr.max().item():.3e}"
    return err.max().item()


def oracle_pairs(p, pairs):
    return oracle.problem(p, pairs=pairs)
